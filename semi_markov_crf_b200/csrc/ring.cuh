// ring.cuh -- device machinery shared by the ring recursions (forward,
// backward, posterior recompute, Viterbi): shared-memory carve, the TMA
// prefix-sum tile stream, per-lane constant operands and the two fan-ins.
//
// Ring layout.  Each label owns RL = K + KBT float2 entries (value, exact
// integer part); boundary x lives in slot x mod K, and slots below KBT are
// mirrored at slot + K.  A lane owns KBT consecutive durations, so at every
// step it reads KBT consecutive entries starting at a base index that moves by
// one per step: no per-term index arithmetic, no wrap test.  Entries of
// boundaries that do not exist (before 0, after L) hold -inf, and durations
// above K carry dur2 = -inf, so no per-term validity test is needed either.
#pragma once

#include <climits>

#include "kernels.cuh"

namespace semicrf {
namespace ring {

// Per-step buffers are double-buffered by step parity (pcur, Acur) or
// triple-buffered (maxslot): with one CTA barrier per step, a fast warp may
// write the next step's copy while a slow one still reads this step's.
struct Smem {
  uint64_t* mbar;   // [2] tile barriers
  int* maxslot;     // [3] per-step max (order-preserving ints)
  int32_t* tint;    // [2][TS][C]
  float* tfrac;     // [2][TS][C]
  float2* ring;     // [C][RL]
  float* pcur;      // [2][PC] exp-domain label vector (zero padded)
  float* Acur;      // [2][C]
  float* tmp;       // [C]
  int* Sbase;       // [C]
  float* store;     // [delta][store_w] (posterior kernel, when in shared memory)
};

__device__ __forceinline__ Smem carve(unsigned char* raw, const Dims& d, bool with_store) {
  Smem s;
  const int C = d.C;
  unsigned char* p = raw;
  s.mbar = reinterpret_cast<uint64_t*>(p);
  s.maxslot = reinterpret_cast<int*>(p + 16);
  p += 64;
  s.tint = reinterpret_cast<int32_t*>(p);
  p += 2ull * TS * C * sizeof(int32_t);
  s.tfrac = reinterpret_cast<float*>(p);
  p += 2ull * TS * C * sizeof(float);
  s.ring = reinterpret_cast<float2*>(p);
  p += (size_t)d.RL * C * sizeof(float2);
  p = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 15) & ~uintptr_t(15));
  float* f = reinterpret_cast<float*>(p);  // 16-byte aligned: vector loads of pcur
  s.pcur = f;                              // PC is a multiple of 4
  f += 2 * d.PC;
  s.Acur = f;
  s.tmp = f + 2 * C;
  s.Sbase = reinterpret_cast<int*>(f + 3 * C);
  p = reinterpret_cast<unsigned char*>(f + 4 * C);
  p = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 15) & ~uintptr_t(15));
  s.store = with_store ? reinterpret_cast<float*>(p) : nullptr;
  return s;
}

// Fills the ring with (-inf, 0), zeroes the padded label vector and resets
// the barriers' and the max slots' state.  Call before the first __syncthreads.
__device__ __forceinline__ void init_smem(const Smem& sm, const Dims& d) {
  for (int i = threadIdx.x; i < d.RL * d.C; i += blockDim.x) sm.ring[i] = make_float2(NEG_INF, 0.f);
  for (int i = threadIdx.x; i < 2 * d.PC; i += blockDim.x) sm.pcur[i] = 0.f;
  if (threadIdx.x == 0) {
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    fence_mbar_init();
    for (int i = 0; i < 3; ++i) sm.maxslot[i] = f2ord(NEG_INF);
  }
}

// Writes ring slot `slot` of label c (and its mirror).
template <int KBT>
__device__ __forceinline__ void ring_put(const Smem& sm, const Dims& d, int c, int slot, float2 v) {
  float2* r = sm.ring + (size_t)c * d.RL;
  r[slot] = v;
  if (slot < KBT) r[slot + d.K] = v;
}

// Ring entry of boundary `bnd` (0 <= bnd) for label c.
__device__ __forceinline__ float2& ring_at(const Smem& sm, const Dims& d, int c, int bnd) {
  return sm.ring[(size_t)c * d.RL + (bnd % d.K)];
}

// ----------------------------------------------------------------------------- tile stream
// Double-buffered TMA stream of prefix-sum tiles (TS rows) for one sequence,
// moving up (dir = +1) or down (dir = -1).  Entering a tile issues the next.
struct TileStream {
  int cur, lo, hi, dir;
  uint32_t ph[2];
};

__device__ __forceinline__ void tile_issue(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                           const TileStream& ts, int i) {
  if (i < ts.lo || i > ts.hi || threadIdx.x != 0) return;
  const int buf = i & 1;
  const uint32_t bytes = (uint32_t)(TS * d.C * 4);
  const size_t row0 = (size_t)b * d.Tstride + (size_t)i * TS;
  fence_proxy_async();
  mbar_expect_tx(&sm.mbar[buf], 2 * bytes);
  bulk_g2s(sm.tint + (size_t)buf * TS * d.C, ws.sint + row0 * d.C, bytes, &sm.mbar[buf]);
  bulk_g2s(sm.tfrac + (size_t)buf * TS * d.C, ws.sfrac + row0 * d.C, bytes, &sm.mbar[buf]);
}

__device__ __forceinline__ void tile_start(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                           TileStream& ts, int first_row, int lo_row, int hi_row,
                                           int dir) {
  ts.lo = lo_row / TS;
  ts.hi = hi_row / TS;
  ts.dir = dir;
  ts.cur = -1;
  tile_issue(sm, d, ws, b, ts, first_row / TS);
}

// Makes row r readable (ri, rf); returns false (uniformly) if a wait gave up.
__device__ __forceinline__ bool tile_row(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                         TileStream& ts, int r, const int32_t*& ri,
                                         const float*& rf) {
  const int i = r / TS;
  bool ok = true;
  if (i != ts.cur) {
    const int buf = i & 1;
    ok = mbar_wait(&sm.mbar[buf], ts.ph[buf], WAIT_SPIN_LIMIT);
    ts.ph[buf] ^= 1u;
    ts.cur = i;
    // every thread is done with the previous tile before its buffer is refilled
    ok = !__syncthreads_or(!ok);
    tile_issue(sm, d, ws, b, ts, i + ts.dir);
  }
  const size_t o = ((size_t)(i & 1) * TS + (r - i * TS)) * d.C;
  ri = sm.tint + o;
  rf = sm.tfrac + o;
  return ok;
}

// After a timeout: bounded wait for copies still in flight, then the CTA may exit.
__device__ __forceinline__ void tile_drain(const Smem& sm, TileStream& ts) {
  if (threadIdx.x == 0)
    for (int buf = 0; buf < 2; ++buf) mbar_wait(&sm.mbar[buf], ts.ph[buf], WAIT_SPIN_LIMIT);
}

// ----------------------------------------------------------------------------- lanes
__device__ __forceinline__ float l2e() { return (float)LOG2E_D; }

// k fan-in role: label cB, lane jB of GB; durations of lane term i:
//   up   (forward, terms at t - k):  k_i = (jB + 1) * KBT - i
//   down (backward, terms at s + k): k_i = jB * KBT + 1 + i
template <int KBT>
struct KLane {
  int c, j;
  bool act;
  float d[KBT];
  __device__ __forceinline__ int k_of(int i, bool up) const {
    return up ? (j + 1) * KBT - i : j * KBT + 1 + i;
  }
  __device__ __forceinline__ void init(const Dims& dm, const float* dur, bool up) {
    c = threadIdx.x / dm.GB;
    j = threadIdx.x % dm.GB;
    act = c < dm.C;
    const int cc = act ? c : 0;
#pragma unroll
    for (int i = 0; i < KBT; ++i) {
      const int k = k_of(i, up);
      d[i] = (act && k <= dm.K) ? __ldg(dur + (size_t)(k - 1) * dm.C + cc) * l2e() : NEG_INF;
    }
  }
  // first ring index of this lane's window
  __device__ __forceinline__ int base_up(int t, int K) const {
    int x = (t - (j + 1) * KBT) % K;
    return x < 0 ? x + K : x;
  }
  __device__ __forceinline__ int base_down(int s, int K) const { return (s + j * KBT + 1) % K; }
};

// label fan-in role: output label c of GA lanes; lane j owns labels
// j*CAT .. j*CAT+CAT-1 of the other side.  e[i] = 2^(trans2 - max) with the
// forward (column, rows=false) or backward (row, rows=true) normalisation.
template <int CAT>
struct ALane {
  int c, j;
  bool act;
  float tmax;
  float e[CAT];
  __device__ __forceinline__ void init(const Dims& dm, const float* trans, bool rows) {
    c = threadIdx.x / dm.GB;  // same lane groups as the k fan-in
    j = threadIdx.x % dm.GB;
    act = c < dm.C;
    const int C = dm.C;
    const int o = act ? c : 0;
    float mx = NEG_INF;
    for (int x = 0; x < C; ++x)
      mx = fmaxf(mx, __ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * l2e());
    if (mx == NEG_INF) mx = 0.f;
    tmax = mx;
#pragma unroll
    for (int i = 0; i < CAT; ++i) {
      const int x = j * CAT + i;
      e[i] = (act && x < C)
                 ? ex2(__ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * l2e() - mx)
                 : 0.f;
    }
  }
};

// Loads v[0..CAT) = p[j*CAT ..] with the widest aligned vector loads.
template <int CAT>
__device__ __forceinline__ void load_block(const float* p, float (&v)[CAT]) {
  if constexpr (CAT % 4 == 0) {
#pragma unroll
    for (int i = 0; i < CAT; i += 4) {
      const float4 q = *reinterpret_cast<const float4*>(p + i);
      v[i] = q.x;
      v[i + 1] = q.y;
      v[i + 2] = q.z;
      v[i + 3] = q.w;
    }
  } else if constexpr (CAT % 2 == 0) {
#pragma unroll
    for (int i = 0; i < CAT; i += 2) {
      const float2 q = *reinterpret_cast<const float2*>(p + i);
      v[i] = q.x;
      v[i + 1] = q.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < CAT; ++i) v[i] = p[i];
  }
}

// k fan-in over this lane's window: y_i = (P + Q) + v + dur2[k_i - 1];
// group LSE (lse, m, sum valid in every lane of the group); e[i] = 2^(y_i - m).
struct KFan {
  float lse, m, sum;
};

template <int KBT>
__device__ __forceinline__ KFan k_fanin(const Smem& sm, const Dims& d, const KLane<KBT>& L, int base,
                                        float Q, float (&e)[KBT]) {
  const float2* r = sm.ring + (size_t)(L.act ? L.c : 0) * d.RL + base;
  float y[KBT];
  float m = NEG_INF;
#pragma unroll
  for (int i = 0; i < KBT; ++i) {
    const float2 v = r[i];
    y[i] = ((v.y + Q) + v.x) + L.d[i];
    m = fmaxf(m, y[i]);
  }
  m = group_max(m, d.GB);
  float s = 0.f;
  const float mm = (m == NEG_INF) ? 0.f : m;
#pragma unroll
  for (int i = 0; i < KBT; ++i) {
    e[i] = ex2(y[i] - mm);
    s += e[i];
  }
  s = group_sum(s, d.GB);
  KFan out;
  out.m = m;
  out.sum = s;
  out.lse = (m == NEG_INF) ? NEG_INF : m + lg2(s);
  return out;
}

// Label fan-in in the exponential domain: sum_x pcur[x] * e[x], group-summed.
// prod[i] keeps the per-term products.
template <int CAT>
__device__ __forceinline__ float label_fanin(const float* pcur, const Dims& d, const ALane<CAT>& A,
                                             float (&prod)[CAT]) {
  float p[CAT];
  load_block<CAT>(pcur + A.j * CAT, p);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < CAT; ++i) {
    prod[i] = p[i] * A.e[i];
    acc += prod[i];
  }
  return group_sum(acc, d.GB);
}

constexpr float EXP_SAFE = 100.f;       // |frame step| beyond which p is recomputed
constexpr float UNDERFLOW = 0x1p-100f;  // label sums below this use the log domain

// Log-domain label fan-in for one output (rare fallback when the
// exponential-domain sum underflows): LSE_x (vals[x] - shift + trans2).
__device__ __forceinline__ float label_lse_slow(const Dims& d, const float* vals, float shift,
                                                const float* trans, int o, bool rows) {
  const int C = d.C;
  float mx = NEG_INF;
  for (int x = 0; x < C; ++x) {
    const float t2 = __ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * l2e();
    mx = fmaxf(mx, vals[x] - shift + t2);
  }
  if (mx == NEG_INF) return NEG_INF;
  float s = 0.f;
  for (int x = 0; x < C; ++x) {
    const float t2 = __ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * l2e();
    s += ex2(vals[x] - shift + t2 - mx);
  }
  return mx + lg2(s);
}

// Reads the max of step `q` (mod 3), resets slot q+2 for the step after next,
// and returns the integer frame step n; `slow` is set when 2^(value) could
// overflow or underflow in the exponential-domain fan-in.
__device__ __forceinline__ float step_frame(const Smem& sm, int q, bool& slow) {
  const float M = ord2f(sm.maxslot[q]);
  if (threadIdx.x == 0) sm.maxslot[q == 0 ? 2 : q - 1] = f2ord(NEG_INF);
  const bool fin = isfinite(M);
  slow = fin && (M > EXP_SAFE || M < -EXP_SAFE);
  return fin ? rintf(M) : 0.f;
}

__device__ __forceinline__ int mod3_next(int q) { return q == 2 ? 0 : q + 1; }

}  // namespace ring
}  // namespace semicrf
