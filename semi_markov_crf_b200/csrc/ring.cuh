// ring.cuh -- device machinery shared by the ring recursions (forward,
// backward, posterior recompute, Viterbi): shared-memory carve, the TMA
// prefix-sum tile stream, per-lane constant operands and the two fan-ins.
//
// Ring layout.  Each label owns RL = K + KBT float2 entries (value, exact
// integer part); boundary x lives in slot x mod K, and slots below KBT are
// mirrored at slot + K (and further multiples of K when K < KBT).  A lane
// owns KBT consecutive durations, so at every step it reads KBT consecutive
// entries starting at a base index that moves by one per step: no per-term
// index arithmetic, no wrap test.  Entries of boundaries that do not exist
// (before 0, after L) hold -inf, and durations above K carry dur2 = -inf, so
// no per-term validity test is needed either.
//
// Lane groups.  A group of G consecutive lanes (G a power of two, a
// compile-time shape parameter) owns one label for both fan-ins; per-step
// work is latency bound (about one warp per scheduler), so the step code keeps
// everything a lane needs in registers and avoids index arithmetic and
// branches on the critical path.
#pragma once

#include <climits>

#include "kernels.cuh"

namespace semicrf {
namespace ring {

// Bounds-check sites (status >> 8 in the debug build), one per guarded access.
enum BoundsSite {
  SITE_TILE_ISSUE = 1,    // TMA prefix-sum tile: source rows inside the sequence
  SITE_TILE_ROW = 2,      // a row pointer into the tile buffers
  SITE_RING_WINDOW = 3,   // a lane's k fan-in window inside its label's ring row
  SITE_RING_SLOT = 4,     // a ring write slot
  SITE_VECTOR = 5,        // label-vector (p or V) store, local or in a cluster peer
  SITE_KEPT_ROW = 6,      // kept per-boundary rows (p, acc, V, durations, frames)
  SITE_STEP_ARRAYS = 7,   // per-label step arrays written by the helpers
  SITE_WALK_STAGE = 8,    // traceback stage: rows copied fit the staging buffer
  SITE_WALK_MARK = 9,     // traceback: a segment-start mark inside the stage
  SITE_POST_TILE = 10,    // posterior pass: tile rows and halo inside the staged tile
  SITE_POST_ITEM = 11,    // posterior pass: a segment end inside the staged rows
  SITE_SEG_STORE = 12,    // checkpoint walk: the per-position store
  SITE_SELFTEST = 13      // semicrf_selftest_bounds: an index past its array on purpose
};

// Per-step buffers are double-buffered by step parity (pcur, Acur) or
// triple-buffered (maxslot): with one CTA barrier per step, a fast warp may
// write the next step's copy while a slow one still reads this step's.
struct Smem {
  uint64_t* mbar;   // [2] tile barriers
  int* maxslot;     // [3] per-step max (order-preserving ints)
  int* aux;         // [1] block-wide max of the transition scores
  int32_t* tint;    // [2][TS][C]
  float* tfrac;     // [2][TS][C]
  float* tpd;       // [2][TS][C] projection start terms (pipelined kernels with
                    // boundary projections; nullptr otherwise)
  float2* ring;     // [C][RL]
  float* pcur;      // [2][PC] exp-domain label vector (zero padded)
  float* Acur;      // [2][C]
  float* tmp;       // [C]
  int* Sbase;       // [C]
  float* store;     // [delta][store_w] (posterior kernel, when in shared memory)
};

__device__ __forceinline__ float l2e() { return (float)LOG2E_D; }

__device__ __forceinline__ Smem carve(unsigned char* raw, const Dims& d, bool with_store) {
  Smem s;
  const int C = d.C;
  unsigned char* p = raw;
  s.mbar = reinterpret_cast<uint64_t*>(p);
  s.maxslot = reinterpret_cast<int*>(p + 16);
  s.aux = reinterpret_cast<int*>(p + 32);
  p += 64;
  s.tint = reinterpret_cast<int32_t*>(p);
  p += 2ull * TS * C * sizeof(int32_t);
  s.tfrac = reinterpret_cast<float*>(p);
  p += 2ull * TS * C * sizeof(float);
  s.tpd = nullptr;
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

// Fills the ring with (-inf, 0), zeroes the padded label vectors and resets
// the barriers and the max slots.  A __syncthreads must follow.
__device__ __forceinline__ void init_smem(const Smem& sm, const Dims& d) {
  for (int i = threadIdx.x; i < d.RL * d.C; i += blockDim.x) sm.ring[i] = make_float2(NEG_INF, 0.f);
  for (int i = threadIdx.x; i < 2 * d.PC; i += blockDim.x) sm.pcur[i] = 0.f;
  if (threadIdx.x == 0) {
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    fence_mbar_init();
    for (int i = 0; i < 3; ++i) sm.maxslot[i] = f2ord(NEG_INF);
    sm.aux[0] = f2ord(NEG_INF);
  }
}

// Largest transition score (base 2) over the whole C x C matrix, by every
// thread of the block (called after init_smem's barrier; holds one barrier).
// Both directions and every kernel scale the exp-domain transition weights
// 2^(trans2 - M) by this same M, so the forward and backward label fan-ins
// use bitwise the same weights: their rounding is one model, not two, and
// the posteriors (ratios of forward, backward and log Z) see no drift
// between the chains.  0 if nothing is finite.
__device__ __forceinline__ float block_trans_max(const Smem& sm, const Dims& d, const float* trans) {
  float mx = NEG_INF;
  for (int i = threadIdx.x; i < d.C * d.C; i += blockDim.x) mx = fmaxf(mx, __ldg(trans + i) * l2e());
  warp_max_to_shared(sm.aux, f2ord(mx));
  __syncthreads();
  const float m = ord2f(sm.aux[0]);
  return isfinite(m) ? m : 0.f;
}

// Writes ring slot `slot` of one label (rl = its first entry) and its mirrors
// (every index slot + mK below RL = K + KBT).
template <int KBT>
__device__ __forceinline__ void ring_put(float2* rl, const Dims& d, int slot, float2 v) {
  rl[slot] = v;
  if (slot < KBT)
    for (int x = slot + d.K; x < d.RL; x += d.K) rl[x] = v;
}

// A lane's ring window base and a ring write slot, after the bounds-check
// build's test (in the release build: the base itself, and true).
__device__ __forceinline__ int checked_base(const WsPtrs& ws, int base, int K) {
  return SEMICRF_INB(ws.status, base >= 0 && base < K, SITE_RING_WINDOW) ? base : 0;
}
__device__ __forceinline__ bool checked_slot(const WsPtrs& ws, int slot, int K) {
  return SEMICRF_INB(ws.status, slot >= 0 && slot < K, SITE_RING_SLOT);
}

// Ring entry of boundary `bnd` (0 <= bnd) for label c.
__device__ __forceinline__ float2& ring_at(const Smem& sm, const Dims& d, int c, int bnd) {
  return sm.ring[(size_t)c * d.RL + (bnd % d.K)];
}

// ----------------------------------------------------------------------------- tile stream
// Double-buffered TMA stream of prefix-sum tiles (TS rows) for one sequence,
// moving up (dir = +1) or down (dir = -1).  Entering a tile issues the next.
struct TileStream {
  int lo, hi, dir;
  uint32_t ph[2];
};

__device__ __forceinline__ void tile_issue(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                           const TileStream& ts, int i) {
  if (i < ts.lo || i > ts.hi || threadIdx.x != 0) return;
  const int buf = i & 1;
  const uint32_t bytes = (uint32_t)(TS * d.C * 4);
  const size_t row0 = (size_t)b * d.Tstride + (size_t)i * TS;
  // bounds-check build: the tile's rows lie in sequence b's rows
  if (!SEMICRF_INB(ws.status, i >= 0 && b >= 0 && b < d.B && (size_t)(i + 1) * TS <= (size_t)d.Tstride,
                   SITE_TILE_ISSUE))
    return;
  fence_proxy_async();
  mbar_expect_tx(&sm.mbar[buf], (sm.tpd ? 3 : 2) * bytes);
  bulk_g2s(sm.tint + (size_t)buf * TS * d.C, ws.sint + row0 * d.C, bytes, &sm.mbar[buf]);
  bulk_g2s(sm.tfrac + (size_t)buf * TS * d.C, ws.sfrac + row0 * d.C, bytes, &sm.mbar[buf]);
  if (sm.tpd) bulk_g2s(sm.tpd + (size_t)buf * TS * d.C, ws.pd + row0 * d.C, bytes, &sm.mbar[buf]);
}

// Rows lo_row..hi_row will be visited starting at first_row.
__device__ __forceinline__ void tile_start(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                           TileStream& ts, int first_row, int lo_row, int hi_row,
                                           int dir) {
  ts.lo = lo_row / TS;
  ts.hi = hi_row / TS;
  ts.dir = dir;
  tile_issue(sm, d, ws, b, ts, first_row / TS);
}

// Waits for tile i, then (after every thread is done with the previous tile)
// issues the next one into the other buffer.  Returns false, uniformly, if
// the bounded wait gave up.
__device__ __forceinline__ bool tile_enter(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                           TileStream& ts, int i) {
  const int buf = i & 1;
  bool ok = mbar_wait(&sm.mbar[buf], ts.ph[buf], WAIT_SPIN_LIMIT);
  ts.ph[buf] ^= 1u;
  ok = !__syncthreads_or(!ok);
  tile_issue(sm, d, ws, b, ts, i + ts.dir);
  return ok;
}

// After a timeout: bounded wait for copies still in flight, then the CTA may exit.
__device__ __forceinline__ void tile_drain(const Smem& sm, TileStream& ts) {
  if (threadIdx.x == 0)
    for (int buf = 0; buf < 2; ++buf) mbar_wait(&sm.mbar[buf], ts.ph[buf], WAIT_SPIN_LIMIT);
}

// Offset of row r in the tile buffers (its tile must be the current one).
__device__ __forceinline__ size_t tile_row_off(int r, int C) {
  const int i = r / TS;
  return ((size_t)(i & 1) * TS + (r - i * TS)) * C;
}

// ----------------------------------------------------------------------------- reductions
template <int G>
__device__ __forceinline__ float gsum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
  return v;
}

template <int G>
__device__ __forceinline__ unsigned gmask() {
  if constexpr (G >= 32) {
    return FULL_MASK;
  } else {
    const int lane = threadIdx.x & 31;
    return ((1u << G) - 1u) << (lane & ~(G - 1));
  }
}

// (value, index) max with ties to the smaller index, over the lane group.
template <int G>
__device__ __forceinline__ void gargmax(float& v, int& i) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(FULL_MASK, v, o);
    const int i2 = __shfl_xor_sync(FULL_MASK, i, o);
    if (v2 > v || (v2 == v && i2 < i)) {
      v = v2;
      i = i2;
    }
  }
}

// ----------------------------------------------------------------------------- projections
// Start-side boundary projection term of boundary t for label c, base-2
// units ("Streaming Structured Inference with Flash-SemiCRF", explainer
// section 2, "Boundary Projections"): a segment [s, t) scores
// P_start[s] + P_end[t-1] on top of its content.  The end side P_end[t-1]
// is part of the stored prefix sum S'[t] = S[t] + P_end[t-1]; the start side
// uses S'[s] - pd[s] with pd[s] = P_end[s-1] + P_start[s], so a ring entry
// (the start role of its boundary) adds pd.  0 when the call has none.
__device__ __forceinline__ bool proj_on(const WsPtrs& ws) { return ws.pon && *ws.pon != 0; }
__device__ __forceinline__ float proj_d(const WsPtrs& ws, const Dims& d, bool on, int b, int t, int c) {
  return on ? ws.pd[((size_t)b * d.Tstride + t) * d.C + c] : 0.f;
}

// ----------------------------------------------------------------------------- lanes

// One lane of a label group: label c, lane j of G.  Durations of window
// element w of the lane (its ring entries r[0..KBT), contiguous):
//   up   (forward, terms at t - k):  k_w = (j + 1) * KBT - w
//   down (backward, terms at s + k): k_w = j * KBT + 1 + w
// The lane visits its window in rotated order, element widx(i) = (i + j) mod
// KBT at term i: lanes of a label start KBT entries apart, so in plain order
// a half warp's 64-bit reads would all fall in the same shared-memory banks
// (16-way for KBT >= 16); rotated, consecutive lanes read consecutive banks.
// The duration scores d[i] are stored in the same rotated order.
// Label-fan-in operands e[i] = 2^(trans2 - max) for the other side's labels
// j*CAT + i: column-normalised for the forward side (sum over c' into c),
// row-normalised for the backward side (sum over c out of c').
template <int KBT, int CAT, int G>
struct Lane {
  int c, cc, j;
  bool act, leader;
  float tmax;
  float d[KBT];
  float e[CAT];
  __device__ __forceinline__ int k_of(int w, bool up) const {
    return up ? (j + 1) * KBT - w : j * KBT + 1 + w;
  }
  // window element visited at term i
  __device__ __forceinline__ int widx(int i) const { return (i + j) & (KBT - 1); }
  __device__ __forceinline__ void init_ids(const Dims& dm) {
    c = threadIdx.x / G;
    j = threadIdx.x % G;
    act = c < dm.C;
    cc = act ? c : 0;
    leader = act && j == 0;
  }
  __device__ __forceinline__ void init_dur(const Dims& dm, const float* dur, bool up) {
#pragma unroll
    for (int i = 0; i < KBT; ++i) {
      const int k = k_of(widx(i), up);
      d[i] = (act && k <= dm.K) ? __ldg(dur + (size_t)(k - 1) * dm.C + cc) * l2e() : NEG_INF;
    }
  }
  // e[i] = 2^(trans2 - mx) for this lane's CAT sources (rows: trans[c][x],
  // else trans[x][c]); mx is block_trans_max, the same in every kernel.
  __device__ __forceinline__ void init_trans(const Dims& dm, const float* trans, bool rows,
                                             float mx) {
    const int C = dm.C;
    tmax = mx;
#pragma unroll
    for (int i = 0; i < CAT; ++i) {
      const int x = j * CAT + i;
      e[i] = (act && x < C)
                 ? ex2(__ldg(trans + (rows ? (size_t)cc * C + x : (size_t)x * C + cc)) * l2e() - mx)
                 : 0.f;
    }
  }
  // first ring index of this lane's window
  __device__ __forceinline__ int base_up(int t, int K) const {
    int x = (t - (j + 1) * KBT) % K;
    return x < 0 ? x + K : x;
  }
  __device__ __forceinline__ int base_down(int s, int K) const { return (s + j * KBT + 1) % K; }
};

// Loads v[0..CAT) = p[0..CAT) with the widest aligned vector loads.
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

// ----------------------------------------------------------------------------- fan-ins
// k fan-in over a lane's window r[0..KBT), visited in the lane's rotated
// order (term i reads r[(i + rot) mod KBT], d[i] is its duration score),
// y_i = ((P + Q) + v) + dur2.
// The exponentials are taken against an exact-integer shift m (a prediction
// of the group LSE: no max pass, no max reduction): e[i] = 2^(y_i - m) and
// s = group sum.  If s leaves [2^-64, 2^64] the group redoes the fan-in
// against ceil(exact max).  Returns the LSE (NEG_INF if nothing is finite);
// on return m and s describe e[] (e[i] / s are the normalised weights).
// `live` is false (uniformly over the group) for the padding groups of labels
// >= C: their sum is 0 by construction and must not take the fallback, which
// would hold up the rest of their warp every step.
template <int KBT, int G>
__device__ __forceinline__ float k_fanin(const float2* r, int rot, float Q, const float (&d)[KBT],
                                         float& m, float& s, float (&e)[KBT], bool live = true) {
  static_assert((KBT & (KBT - 1)) == 0, "KBT must be a power of two");
  {
    const float Qm = Q - m;  // exact: both integers
    float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < KBT; ++i) {
      const float2 v = r[(i + rot) & (KBT - 1)];
      e[i] = ex2(((v.y + Qm) + v.x) + d[i]);
      sp[i & 3] += e[i];
    }
    s = gsum<G>((sp[0] + sp[1]) + (sp[2] + sp[3]));
  }
  if (live && !(s >= 0x1p-64f && s <= 0x1p64f)) {
    // rare: the prediction was far off (or nothing is finite)
    const unsigned gm = gmask<G>();
    float mx = NEG_INF;
#pragma unroll
    for (int i = 0; i < KBT; ++i) {
      const float2 v = r[(i + rot) & (KBT - 1)];
      mx = fmaxf(mx, ((v.y + Q) + v.x) + d[i]);
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(gm, mx, o));
    m = (mx == NEG_INF) ? 0.f : ceilf(mx);
    const float Qm = Q - m;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < KBT; ++i) {
      const float2 v = r[(i + rot) & (KBT - 1)];
      e[i] = ex2(((v.y + Qm) + v.x) + d[i]);
      ss += e[i];
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(gm, ss, o);
    s = ss;
  }
  return (s > 0.f) ? m + lg2(s) : NEG_INF;
}

// k fan-in over a strided window: lane term q reads r[q * H] (the lanes of a
// group interleave over consecutive ring entries, so a group's reads of one q
// are contiguous), y_q = ((P + Q) + v) + dur2.  Same predicted-shift scheme
// and fallback as k_fanin; returns the group LSE, m and s describe the sum.
// With H > 32 (long durations) the lanes of a label span H / 32 warps and
// every sum, max and shift here is per warp: the caller adds the warps'
// partial sums, each in the linear domain of the same frame.
template <int KBH, int H, int N>
__device__ __forceinline__ float k_fanin_strided(const float2* r, float Q, const float (&d)[N],
                                                 float& m, float& s, bool live) {
  static_assert(N >= KBH, "duration array shorter than the lane's terms");
  constexpr int HG = H > 32 ? 32 : H;
  {
    const float Qm = Q - m;  // exact: both integers
    float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < KBH; ++q) {
      const float2 v = r[q * H];
      sp[q & 3] += ex2(((v.y + Qm) + v.x) + d[q]);
    }
    s = gsum<HG>((sp[0] + sp[1]) + (sp[2] + sp[3]));
  }
  if (live && !(s >= 0x1p-64f && s <= 0x1p64f)) {
    const unsigned gm = gmask<HG>();
    float mx = NEG_INF;
#pragma unroll
    for (int q = 0; q < KBH; ++q) {
      const float2 v = r[q * H];
      mx = fmaxf(mx, ((v.y + Q) + v.x) + d[q]);
    }
#pragma unroll
    for (int o = HG / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(gm, mx, o));
    m = (mx == NEG_INF) ? 0.f : ceilf(mx);
    const float Qm = Q - m;
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < KBH; ++q) {
      const float2 v = r[q * H];
      ss += ex2(((v.y + Qm) + v.x) + d[q]);
    }
#pragma unroll
    for (int o = HG / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(gm, ss, o);
    s = ss;
  }
  return (s > 0.f) ? m + lg2(s) : NEG_INF;
}

// Next step's shift: this step's LSE moved into the next frame (step n).
__device__ __forceinline__ float next_shift(float lse, float n, float m) {
  return isfinite(lse) ? rintf(lse) - n : m;
}

// Label fan-in in the exponential domain: sum_x pcur[x] * e[x] over the group;
// p[i] keeps this lane's loaded pcur values.
template <int CAT, int G>
__device__ __forceinline__ float label_fanin(const float* pj, const float (&e)[CAT],
                                             float (&p)[CAT]) {
  load_block<CAT>(pj, p);
  float ap[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < CAT; ++i) ap[i & 3] = fmaf(p[i], e[i], ap[i & 3]);
  return gsum<G>((ap[0] + ap[1]) + (ap[2] + ap[3]));
}

constexpr float EXP_SAFE = 100.f;       // |frame step| beyond which p is recomputed
constexpr float UNDERFLOW = 0x1p-100f;  // label sums below this use the log domain

// Log-domain label fan-in for one output (rare fallback when the
// exponential-domain sum underflows): LSE_x (vals[x] - shift + trans2).
static __device__ __noinline__ float label_lse_slow(int C, const float* vals, float shift,
                                             const float* trans, int o, bool rows) {
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

// log2 of a label sum minus the frame shift, with the log-domain fallback.
__device__ __forceinline__ float label_log(float acc, float tmax, float shift, int C,
                                           const float* vals, float n, const float* trans, int o,
                                           bool rows) {
  if (acc >= UNDERFLOW && acc <= 3.0e38f) return lg2(acc) + tmax - shift;
  return label_lse_slow(C, vals, n, trans, o, rows);
}

// Reads the max of step slot q (mod 3), resets slot q+2 for the step after
// next, and returns the integer frame step n; `slow` is set when 2^(value)
// could overflow or underflow in the exponential-domain fan-in.
__device__ __forceinline__ float step_frame(const Smem& sm, int q, bool& slow) {
  const float M = ord2f(sm.maxslot[q]);
  if (threadIdx.x == 0) sm.maxslot[q == 0 ? 2 : q - 1] = f2ord(NEG_INF);
  const bool fin = isfinite(M);
  slow = fin && (M > EXP_SAFE || M < -EXP_SAFE);
  return fin ? rintf(M) : 0.f;
}

__device__ __forceinline__ int mod3_next(int q) { return q == 2 ? 0 : q + 1; }

// Uniform slow path: the step's frame jump is too large for 2^A in float32.
__device__ __forceinline__ void refresh_p(const Smem& sm, const Dims& d, int par, float n) {
  for (int c = threadIdx.x; c < d.C; c += blockDim.x)
    sm.pcur[par * d.PC + c] = ex2(sm.Acur[par * d.C + c] - n);
  __syncthreads();
}

}  // namespace ring
}  // namespace semicrf
