// recursion.cu -- steps 2 and 3: the streaming forward and backward rings
// and the checkpoint-parallel posterior pass.
//
// "Streaming Structured Inference with Flash-SemiCRF", explainer section 2,
// "Streaming Forward-Backward with Ring Buffers": the forward message at
// boundary t only needs the last K boundaries, so it lives in a K-slot ring;
// the ring and its normaliser are saved every Delta = ceil(sqrt(T K))
// positions and the backward pass restores them and recomputes locally.
//
// Arithmetic (all log values in base-2 units, x2 = x * log2 e):
//   gamma[s, c] = LSE_{c'} alpha[s, c'] + trans[c', c]        (gamma[0, c] = 0)
//   alpha[t, c] = LSE_{k <= min(K,t)} gamma[t-k, c] + S[t,c] - S[t-k,c] + dur[k-1,c]
// which is the pages' recursion with the c' fan-in shared by every k (an exact
// regrouping of the same sum of exponentials).  Backward mirror:
//   btil[s, c]  = LSE_k S[s+k,c] - S[s,c] + dur[k-1,c] + beta[s+k, c]
//   beta[s, c'] = LSE_c trans[c', c] + btil[s, c]                (beta[L, c] = 0)
// and log Z = LSE_c alpha[L, c] = LSE_c btil[0, c].
//
// Numerics.  Every stored value is kept O(1): each boundary carries an exact
// integer frame F (the running normaliser, rounded to an integer so that frame
// differences are exact in float32), the prefix sums enter as an exact int32
// integer part plus a float32 fraction, and the integer parts of a term are
// summed before the O(1) fractional parts are added.  The label fan-in runs in
// the exponential domain (sum_c' 2^alpha[c'] * 2^trans[c',c], one ex2 per
// label) and falls back to the log domain for any label whose sum underflows.
//
// Lane mapping (per CTA = one sequence or one checkpoint segment):
//   k fan-in:     GB lanes per label, lane j handles k = 1 + j + i*GB (i < KB)
//   label fan-in: GA lanes per label, lane j handles c' = j + i*GA (i < CA)
// Group reductions are xor-shuffles inside aligned lane groups.
#include "kernels.cuh"

namespace semicrf {

namespace {

struct Smem {
  uint64_t* mbar;   // [2] tile barriers
  int* maxslot;     // [2] per-step max (order-preserving ints)
  int* flag;        // [4]
  int32_t* tint;    // [2][TS][C]
  float* tfrac;     // [2][TS][C]
  float2* ring;     // [K][C] (value, exact integer part)
  float* Acur;      // [C]
  float* pcur;      // [C]
  float* stS;       // [2][C]
  float* stE;       // [2][C]
  float* tmp;       // [C]
  int* Sbase;       // [C]
  float* store;     // [delta][store_w] (segment kernel, when in shared memory)
};

__device__ Smem carve(unsigned char* raw, const Dims& d, bool with_store) {
  Smem s;
  const int C = d.C;
  unsigned char* p = raw;
  s.mbar = reinterpret_cast<uint64_t*>(p);
  s.maxslot = reinterpret_cast<int*>(p + 16);
  s.flag = reinterpret_cast<int*>(p + 32);
  p += 64;
  s.tint = reinterpret_cast<int32_t*>(p);
  p += 2ull * TS * C * sizeof(int32_t);
  s.tfrac = reinterpret_cast<float*>(p);
  p += 2ull * TS * C * sizeof(float);
  s.ring = reinterpret_cast<float2*>(p);
  p += (size_t)d.K * C * sizeof(float2);
  float* f = reinterpret_cast<float*>(p);
  s.Acur = f;
  s.pcur = f + C;
  s.stS = f + 2 * C;
  s.stE = f + 4 * C;
  s.tmp = f + 6 * C;
  s.Sbase = reinterpret_cast<int*>(f + 7 * C);
  p += 8ull * C * sizeof(float);
  p = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 15) & ~uintptr_t(15));
  s.store = with_store ? reinterpret_cast<float*>(p) : nullptr;
  return s;
}

// Double-buffered TMA stream of prefix-sum tiles (TS rows each) for one
// sequence, moving up (dir = +1) or down (dir = -1).
struct TileStream {
  int cur, lo, hi, dir;
  uint32_t ph[2];
};

__device__ __forceinline__ void tile_issue(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                           const TileStream& ts, int i) {
  if (i < ts.lo || i > ts.hi) return;
  if (threadIdx.x == 0) {
    const int buf = i & 1;
    const uint32_t bytes = (uint32_t)(TS * d.C * 4);
    const size_t row0 = (size_t)b * d.Tstride + (size_t)i * TS;
    fence_proxy_async();
    mbar_expect_tx(&sm.mbar[buf], 2 * bytes);
    bulk_g2s(sm.tint + (size_t)buf * TS * d.C, ws.sint + row0 * d.C, bytes, &sm.mbar[buf]);
    bulk_g2s(sm.tfrac + (size_t)buf * TS * d.C, ws.sfrac + row0 * d.C, bytes, &sm.mbar[buf]);
  }
}

// Makes row r readable; returns false (uniformly) if a tile wait gave up.
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
    tile_issue(sm, d, ws, b, ts, i + ts.dir);
    ok = !__syncthreads_or(!ok);
  }
  const int buf = i & 1;
  const size_t o = ((size_t)buf * TS + (r - i * TS)) * d.C;
  ri = sm.tint + o;
  rf = sm.tfrac + o;
  return ok;
}

__device__ __forceinline__ void tile_start(const Smem& sm, const Dims& d, const WsPtrs& ws, int b,
                                           TileStream& ts, int first_row, int lo_row, int hi_row,
                                           int dir) {
  ts.lo = lo_row / TS;
  ts.hi = hi_row / TS;
  ts.dir = dir;
  ts.cur = -1;
  // only the first tile here: entering a tile (tile_row) issues the next one
  tile_issue(sm, d, ws, b, ts, first_row / TS);
}

// Gives up on outstanding tiles after a timeout (bounded), so the CTA can
// exit without copies in flight.
__device__ void tile_drain(const Smem& sm, TileStream& ts) {
  if (threadIdx.x == 0) {
    for (int buf = 0; buf < 2; ++buf) mbar_wait(&sm.mbar[buf], ts.ph[buf], WAIT_SPIN_LIMIT);
  }
}

// Per-thread constant operands of the two fan-ins.
struct Roles {
  int cB, jB, cA, jA;
  bool warpB, warpA;  // warp has at least one active lane in the phase
};

__device__ __forceinline__ Roles make_roles(const Dims& d) {
  Roles r;
  const int tid = threadIdx.x;
  r.cB = tid / d.GB;
  r.jB = tid % d.GB;
  r.cA = tid / d.GA;
  r.jA = tid % d.GA;
  const int w0 = tid & ~31;
  r.warpB = (w0 / d.GB) < d.C;
  r.warpA = (w0 / d.GA) < d.C;
  return r;
}

__device__ __forceinline__ float LOG2E() { return (float)LOG2E_D; }

// dur2 values for this lane's durations.
__device__ __forceinline__ void load_dur(const Dims& d, const Roles& r, const float* dur,
                                         float (&dreg)[KB_MAX]) {
  const int c = r.cB < d.C ? r.cB : 0;
#pragma unroll
  for (int i = 0; i < KB_MAX; ++i) {
    const int k = 1 + r.jB + i * d.GB;
    dreg[i] = (i < d.KB && k <= d.K) ? __ldg(dur + (size_t)(k - 1) * d.C + c) * LOG2E() : NEG_INF;
  }
}

// Column-normalised 2^(trans2[c', c] - max_c' trans2[c', c]) for output c = cA
// (forward label fan-in), or row-normalised for output row c' = cA (backward).
__device__ __forceinline__ float load_trans_exp(const Dims& d, const Roles& r, const float* trans,
                                                bool rows, float (&ereg)[CA_MAX]) {
  const int C = d.C;
  const int o = r.cA < C ? r.cA : 0;
  float mx = NEG_INF;
  for (int x = 0; x < C; ++x) {
    const float v = __ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * LOG2E();
    mx = fmaxf(mx, v);
  }
  if (mx == NEG_INF) mx = 0.f;
#pragma unroll
  for (int i = 0; i < CA_MAX; ++i) {
    const int x = r.jA + i * d.GA;
    float e = 0.f;
    if (i < d.CA && x < C) {
      const float v = __ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * LOG2E();
      e = ex2(v - mx);
    }
    ereg[i] = e;
  }
  return mx;
}

// Log-domain label fan-in for one output (rare fallback when the
// exponential-domain sum underflows): LSE_x (vals[x] - shift + trans2).
__device__ float label_lse_slow(const Dims& d, const float* vals, float shift, const float* trans,
                                int o, bool rows) {
  const int C = d.C;
  float mx = NEG_INF;
  for (int x = 0; x < C; ++x) {
    const float t2 = __ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * LOG2E();
    mx = fmaxf(mx, vals[x] - shift + t2);
  }
  if (mx == NEG_INF) return NEG_INF;
  float s = 0.f;
  for (int x = 0; x < C; ++x) {
    const float t2 = __ldg(trans + (rows ? (size_t)o * C + x : (size_t)x * C + o)) * LOG2E();
    s += ex2(vals[x] - shift + t2 - mx);
  }
  return mx + lg2(s);
}

// ---------------------------------------------------------------------------
// k fan-in.  Forward (up = true): terms at boundary t from ring slots t-k,
//   y_k = (P[t-k] + Q) + v[t-k] + dur2[k-1],  Q = (Sint[t]-Sbase) - Frel.
// Backward (up = false): terms at boundary s from ring slots s+k,
//   y_k = (P[s+k] + Q) + v[s+k] + dur2[k-1],  Q = -(Sint[s]-Sbase) - Grel.
// Returns the group LSE (valid in every lane of the group) and leaves the
// per-term exponentials e[i] = 2^(y_i - m) and their sum for posterior use.
struct KFan {
  float lse;  // m + lg2(sum), NEG_INF if no valid term
  float m, sum;
};

__device__ __forceinline__ KFan k_fanin(const Smem& sm, const Dims& d, const Roles& r, int tb,
                                        int kmax, float Q, bool up, const float (&dreg)[KB_MAX],
                                        float (&e)[KB_MAX]) {
  const int C = d.C, K = d.K;
  const bool act = r.cB < C;
  const int c = act ? r.cB : 0;
  float y[KB_MAX];
  float m = NEG_INF;
#pragma unroll
  for (int i = 0; i < KB_MAX; ++i) {
    y[i] = NEG_INF;
    const int k = 1 + r.jB + i * d.GB;
    if (i < d.KB && act && k <= kmax) {
      int slot = up ? tb - k : tb + k;
      if (up) {
        if (slot < 0) slot += K;
      } else {
        if (slot >= K) slot -= K;
      }
      const float2 v = sm.ring[slot * C + c];
      y[i] = ((v.y + Q) + v.x) + dreg[i];
      m = fmaxf(m, y[i]);
    }
  }
  m = group_max(m, d.GB);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < KB_MAX; ++i) {
    e[i] = 0.f;
    if (i < d.KB && m != NEG_INF) {
      e[i] = ex2(y[i] - m);
      s += e[i];
    }
  }
  s = group_sum(s, d.GB);
  KFan out;
  out.m = m;
  out.sum = s;
  out.lse = (m == NEG_INF) ? NEG_INF : m + lg2(s);
  return out;
}

// Label fan-in in the exponential domain: sum_x p[x] * ereg[x] over this
// lane's labels, group-reduced.  prod[i] keeps the per-term products.
__device__ __forceinline__ float label_fanin(const Smem& sm, const Dims& d, const Roles& r,
                                             const float (&ereg)[CA_MAX], float (&prod)[CA_MAX]) {
  const bool act = r.cA < d.C;
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < CA_MAX; ++i) {
    prod[i] = 0.f;
    const int x = r.jA + i * d.GA;
    if (i < d.CA && act && x < d.C) {
      prod[i] = sm.pcur[x] * ereg[i];
      acc += prod[i];
    }
  }
  return group_sum(acc, d.GA);
}

constexpr float EXP_SAFE = 100.f;      // |frame jump| beyond which p is recomputed
constexpr float UNDERFLOW = 0x1p-100f;  // label sums below this use the log domain

// Reads the step max, resets the other slot, and returns the integer frame
// step n.  `slow` is set when 2^(value) may overflow/underflow.
__device__ __forceinline__ float step_frame(const Smem& sm, int parity, bool& slow) {
  const float M = ord2f(sm.maxslot[parity]);
  __syncwarp();
  const bool fin = isfinite(M);
  slow = fin && (M > EXP_SAFE || M < -EXP_SAFE);
  return fin ? rintf(M) : 0.f;
}

}  // namespace

// ===========================================================================
// Forward and backward rings over whole sequences.
// ===========================================================================
__global__ void __launch_bounds__(NT_MAX, 1)
    chain_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                 const float* __restrict__ trans, const float* __restrict__ dur,
                 double* __restrict__ logZ_out, int n_alpha) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem sm = carve(smem_raw, d, false);
  const int C = d.C, K = d.K, tid = threadIdx.x;
  const bool is_alpha = (int)blockIdx.x < n_alpha;
  const int b = is_alpha ? blockIdx.x : blockIdx.x - n_alpha;
  const int L = lengths[b];
  if (L < 0 || L > d.T) {
    if (tid == 0) {
      set_status(ws.status, ST_BAD_LENGTH);
      if (is_alpha) {
        logZ_out[b] = __longlong_as_double(0x7ff8000000000000ll);
        ws.logz2[b] = __longlong_as_double(0x7ff8000000000000ll);
      } else {
        ws.logz2b[b] = __longlong_as_double(0x7ff8000000000000ll);
      }
    }
    return;
  }
  if (L == 0) {
    if (tid == 0) {
      if (is_alpha) {
        logZ_out[b] = 0.0;
        ws.logz2[b] = 0.0;
      } else {
        ws.logz2b[b] = 0.0;
      }
    }
    return;
  }
  const Roles r = make_roles(d);
  float dreg[KB_MAX], ereg[CA_MAX], e[KB_MAX], prod[CA_MAX];
  load_dur(d, r, dur, dreg);
  const float tmax2 = load_trans_exp(d, r, trans, !is_alpha, ereg);

  if (tid == 0) {
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    fence_mbar_init();
    sm.maxslot[0] = f2ord(NEG_INF);
    sm.maxslot[1] = f2ord(NEG_INF);
  }
  __syncthreads();
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  const int* Sb = sm.Sbase;
  const int32_t* ri;
  const float* rf;

  if (is_alpha) {
    // ---------------------------------------------------------------- forward
    for (int c = tid; c < C; c += blockDim.x) {
      sm.ring[c] = make_float2(0.f, 0.f);  // boundary 0: gamma = 0, frame 0, S = 0
      sm.Sbase[c] = 0;
    }
    tile_start(sm, d, ws, b, ts, 0, 0, L, +1);
    double F0 = 0.0;
    float Frel = 0.f;
    int tb = 0;
    __syncthreads();
    for (int t = 1; t <= L; ++t) {
      tb = (tb + 1 == K) ? 0 : tb + 1;
      if (!tile_row(sm, d, ws, b, ts, t, ri, rf)) {
        if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
        tile_drain(sm, ts);
        return;
      }
      if (t % d.delta == 0 && t < L) {
        // checkpoint j: rebase frames to (F0 + Frel, S_int[t]) and save the ring
        const int j = t / d.delta;
        const float dF = Frel;
        for (int idx = tid; idx < K * C; idx += blockDim.x) {
          const int i = idx / C, c = idx % C;
          if (t - K + i < 0) continue;
          int slot = tb + i;
          if (slot >= K) slot -= K;
          float2 v = sm.ring[slot * C + c];
          v.y = (v.y - dF) + (float)(ri[c] - Sb[c]);
          sm.ring[slot * C + c] = v;
          ws.ack[(((size_t)b * d.nck + j) * K + i) * C + c] = v;
        }
        __syncthreads();
        for (int c = tid; c < C; c += blockDim.x) sm.Sbase[c] = ri[c];
        F0 += (double)dF;
        Frel = 0.f;
        if (tid == 0) ws.acf[(size_t)b * d.nck + j] = F0;
        __syncthreads();
      }
      const int par = t & 1;
      if (r.warpB) {
        const bool act = r.cB < C;
        const int c = act ? r.cB : 0;
        const float Q = (float)(ri[c] - Sb[c]) - Frel;
        const KFan kf = k_fanin(sm, d, r, tb, min(K, t), Q, true, dreg, e);
        if (act && r.jB == 0) {
          const float A = (kf.lse == NEG_INF) ? NEG_INF : rf[c] + kf.lse;
          sm.Acur[c] = A;
          sm.pcur[c] = ex2(A);
          atomicMax(&sm.maxslot[par], f2ord(A));
        }
      }
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, par, slow);
      if (tid == 0) sm.maxslot[par ^ 1] = f2ord(NEG_INF);
      if (t == L) break;
      float shift = n;
      if (slow) {
        for (int c = tid; c < C; c += blockDim.x) sm.pcur[c] = ex2(sm.Acur[c] - n);
        __syncthreads();
        shift = 0.f;
      }
      if (r.warpA) {
        const float acc = label_fanin(sm, d, r, ereg, prod);
        if (r.cA < C && r.jA == 0) {
          const int c = r.cA;
          float g;
          if (acc >= UNDERFLOW && acc <= 3.0e38f)
            g = lg2(acc) + tmax2 - shift;
          else
            g = label_lse_slow(d, sm.Acur, n, trans, c, false);
          sm.ring[tb * C + c] = make_float2(g - rf[c], (Frel + n) - (float)(ri[c] - Sb[c]));
        }
      }
      Frel += n;
      __syncthreads();
    }
    // log Z = F_{L-1} + LSE_c A_L[c]
    if (tid < 32) {
      float m = NEG_INF;
      for (int c = tid; c < C; c += 32) m = fmaxf(m, sm.Acur[c]);
      m = group_max(m, 32);
      float s = 0.f;
      if (m != NEG_INF)
        for (int c = tid; c < C; c += 32) s += ex2(sm.Acur[c] - m);
      s = group_sum(s, 32);
      if (tid == 0) {
        const double lz = (m == NEG_INF) ? -INFINITY : F0 + (double)Frel + (double)(m + lg2(s));
        ws.logz2[b] = lz;
        logZ_out[b] = lz * LN2_D;
      }
    }
  } else {
    // --------------------------------------------------------------- backward
    tile_start(sm, d, ws, b, ts, L, 0, L, -1);
    if (!tile_row(sm, d, ws, b, ts, L, ri, rf)) {
      if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
      tile_drain(sm, ts);
      return;
    }
    int sb = L % K;
    for (int c = tid; c < C; c += blockDim.x) {
      sm.ring[sb * C + c] = make_float2(rf[c], 0.f);  // beta[L] = 0, frame 0, base S_int[L]
      sm.Sbase[c] = ri[c];
    }
    double G0 = 0.0;
    float Grel = 0.f;
    __syncthreads();
    for (int s = L - 1; s >= 0; --s) {
      sb = (sb == 0) ? K - 1 : sb - 1;
      if (!tile_row(sm, d, ws, b, ts, s, ri, rf)) {
        if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
        tile_drain(sm, ts);
        return;
      }
      const int t1 = s + 1;
      if (t1 % d.delta == 0 && t1 < L) {
        // checkpoint j: the ring holds boundaries t1..t1+K-1; rebase to (G0 + Grel, S_int[t1])
        const int j = t1 / d.delta - 1;
        int s1 = sb + 1;
        if (s1 >= K) s1 -= K;
        for (int c = tid; c < C; c += blockDim.x) sm.tmp[c] = sm.ring[s1 * C + c].y;
        __syncthreads();
        for (int idx = tid; idx < K * C; idx += blockDim.x) {
          const int i = idx / C, c = idx % C;
          if (t1 + i > L) continue;
          int slot = s1 + i;
          if (slot >= K) slot -= K;
          float2 v = sm.ring[slot * C + c];
          v.y = v.y - sm.tmp[c];
          sm.ring[slot * C + c] = v;
          ws.bck[(((size_t)b * d.nck + j) * K + i) * C + c] = v;
        }
        __syncthreads();
        for (int c = tid; c < C; c += blockDim.x)
          sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t1) * C + c];
        G0 += (double)Grel;
        Grel = 0.f;
        if (tid == 0) ws.bcf[(size_t)b * d.nck + j] = G0;
        __syncthreads();
      }
      const int par = s & 1;
      if (r.warpB) {
        const bool act = r.cB < C;
        const int c = act ? r.cB : 0;
        const float Q = -(float)(ri[c] - Sb[c]) - Grel;
        const KFan kf = k_fanin(sm, d, r, sb, min(K, L - s), Q, false, dreg, e);
        if (act && r.jB == 0) {
          const float Bt = (kf.lse == NEG_INF) ? NEG_INF : kf.lse - rf[c];
          sm.Acur[c] = Bt;
          sm.pcur[c] = ex2(Bt);
          atomicMax(&sm.maxslot[par], f2ord(Bt));
        }
      }
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, par, slow);
      if (tid == 0) sm.maxslot[par ^ 1] = f2ord(NEG_INF);
      if (s == 0) break;
      float shift = n;
      if (slow) {
        for (int c = tid; c < C; c += blockDim.x) sm.pcur[c] = ex2(sm.Acur[c] - n);
        __syncthreads();
        shift = 0.f;
      }
      if (r.warpA) {
        const float acc = label_fanin(sm, d, r, ereg, prod);
        if (r.cA < C && r.jA == 0) {
          const int c = r.cA;
          float g;
          if (acc >= UNDERFLOW && acc <= 3.0e38f)
            g = lg2(acc) + tmax2 - shift;
          else
            g = label_lse_slow(d, sm.Acur, n, trans, c, true);
          sm.ring[sb * C + c] = make_float2(g + rf[c], (Grel + n) + (float)(ri[c] - Sb[c]));
        }
      }
      Grel += n;
      __syncthreads();
    }
    if (tid < 32) {
      float m = NEG_INF;
      for (int c = tid; c < C; c += 32) m = fmaxf(m, sm.Acur[c]);
      m = group_max(m, 32);
      float s = 0.f;
      if (m != NEG_INF)
        for (int c = tid; c < C; c += 32) s += ex2(sm.Acur[c] - m);
      s = group_sum(s, 32);
      if (tid == 0)
        ws.logz2b[b] = (m == NEG_INF) ? -INFINITY : G0 + (double)Grel + (double)(m + lg2(s));
    }
  }
}

// ===========================================================================
// Checkpoint-parallel posteriors: one CTA per (segment j, sequence b).
// ===========================================================================
__global__ void __launch_bounds__(NT_MAX, 1)
    segment_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                   const float* __restrict__ trans, const float* __restrict__ dur,
                   const double* __restrict__ grad_logZ, float* __restrict__ grad_em,
                   float* __restrict__ start_marg, float* __restrict__ end_marg) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem sm = carve(smem_raw, d, d.store_smem != 0);
  const int C = d.C, K = d.K, tid = threadIdx.x;
  const int j = blockIdx.x, b = blockIdx.y;
  const int L = lengths[b];
  if (L < 0 || L > d.T) return;  // reported by the forward pass
  const int t0 = j * d.delta;
  if (t0 >= L) return;
  const int t1 = min(t0 + d.delta, L);
  const bool last = (t1 == L);
  const double gb = grad_logZ ? grad_logZ[b] : 1.0;
  const float gbf = (float)gb;
  const double logz2 = ws.logz2[b];
  const int SW = d.store_w;
  float* store = sm.store ? sm.store : ws.store + ((size_t)b * d.nck + j) * d.delta * SW;
  const size_t seg = (size_t)b * d.nck + j;

  const Roles r = make_roles(d);
  float dreg[KB_MAX], ereg[CA_MAX], e[KB_MAX], prod[CA_MAX];
  float accd[KB_MAX], acct[CA_MAX];
  load_dur(d, r, dur, dreg);
#pragma unroll
  for (int i = 0; i < KB_MAX; ++i) accd[i] = 0.f;
#pragma unroll
  for (int i = 0; i < CA_MAX; ++i) acct[i] = 0.f;
  // zero this CTA's float64 partials (each thread its own entries)
  if (r.cB < C) {
    for (int i = 0; i < d.KB; ++i) {
      const int k = 1 + r.jB + i * d.GB;
      if (k <= K) ws.pgd[(seg * K + (k - 1)) * C + r.cB] = 0.0;
    }
  }
  if (r.cA < C) {
    for (int i = 0; i < d.CA; ++i) {
      const int x = r.jA + i * d.GA;
      if (x < C) ws.pgt[(seg * C + r.cA) * C + x] = 0.0;
    }
  }
  if (tid == 0) {
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    fence_mbar_init();
    sm.maxslot[0] = f2ord(NEG_INF);
    sm.maxslot[1] = f2ord(NEG_INF);
  }
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  const int* Sb = sm.Sbase;
  const int32_t* ri;
  const float* rf;

  // ------------------------------------------------------ alpha recompute
  float tmax2 = load_trans_exp(d, r, trans, false, ereg);
  double F0 = 0.0;
  float Frel = 0.f;
  int t_start;
  if (j == 0) {
    for (int c = tid; c < C; c += blockDim.x) {
      sm.ring[c] = make_float2(0.f, 0.f);
      sm.Sbase[c] = 0;
      store[c] = NEG_INF;   // no alpha at boundary 0
      store[C + c] = 0.f;   // gamma[0] = 0 in frame 0
    }
    if (tid == 0) {
      store[2 * C] = 0.f;
      store[2 * C + 1] = 0.f;
    }
    t_start = 1;
  } else {
    const float2* ck = ws.ack + seg * K * C;
    for (int idx = tid; idx < K * C; idx += blockDim.x) {
      const int i = idx / C, c = idx % C;
      const int bnd = t0 - K + i;
      if (bnd < 0) continue;
      sm.ring[(bnd % K) * C + c] = ck[idx];
    }
    for (int c = tid; c < C; c += blockDim.x)
      sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t0) * C + c];
    F0 = ws.acf[seg];
    t_start = t0;
  }
  const int t_end = last ? L : t1 - 1;
  __syncthreads();
  if (t_start <= t_end) {
    tile_start(sm, d, ws, b, ts, t_start, t_start, t_end, +1);
    int tb = t_start % K;
    for (int t = t_start; t <= t_end; ++t) {
      if (t > t_start) tb = (tb + 1 == K) ? 0 : tb + 1;
      if (!tile_row(sm, d, ws, b, ts, t, ri, rf)) {
        if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
        tile_drain(sm, ts);
        return;
      }
      const int par = t & 1;
      if (r.warpB) {
        const bool act = r.cB < C;
        const int c = act ? r.cB : 0;
        const float Q = (float)(ri[c] - Sb[c]) - Frel;
        const KFan kf = k_fanin(sm, d, r, tb, min(K, t), Q, true, dreg, e);
        if (act && r.jB == 0) {
          const float A = (kf.lse == NEG_INF) ? NEG_INF : rf[c] + kf.lse;
          sm.Acur[c] = A;
          sm.pcur[c] = ex2(A);
          atomicMax(&sm.maxslot[par], f2ord(A));
        }
      }
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, par, slow);
      if (tid == 0) sm.maxslot[par ^ 1] = f2ord(NEG_INF);
      if (t == L) break;
      float shift = n;
      if (slow) {
        for (int c = tid; c < C; c += blockDim.x) sm.pcur[c] = ex2(sm.Acur[c] - n);
        __syncthreads();
        shift = 0.f;
      }
      float* row = store + (size_t)(t - t0) * SW;
      if (r.warpA) {
        const float acc = label_fanin(sm, d, r, ereg, prod);
        if (r.cA < C && r.jA == 0) {
          const int c = r.cA;
          float g;
          if (acc >= UNDERFLOW && acc <= 3.0e38f)
            g = lg2(acc) + tmax2 - shift;
          else
            g = label_lse_slow(d, sm.Acur, n, trans, c, false);
          sm.ring[tb * C + c] = make_float2(g - rf[c], (Frel + n) - (float)(ri[c] - Sb[c]));
          row[c] = sm.Acur[c];
          row[C + c] = g;
        }
      }
      if (tid == 0) {
        row[2 * C] = Frel;
        row[2 * C + 1] = Frel + n;
      }
      Frel += n;
      __syncthreads();
    }
  }
  if (last) {
    // end marginal at boundary L (beta[L] = 0); nothing starts at L
    const float XL = (float)(F0 + (double)Frel - logz2);
    for (int c = tid; c < C; c += blockDim.x) {
      const size_t o = ((size_t)b * (d.T + 1) + L) * C + c;
      if (end_marg) end_marg[o] = ex2(sm.Acur[c] + XL);
      if (start_marg) start_marg[o] = 0.f;
    }
  }
  __syncthreads();

  // ------------------------------------------------------ beta recompute + posteriors
  tmax2 = load_trans_exp(d, r, trans, true, ereg);  // row-normalised now
  double G0 = 0.0;
  float Grel = 0.f;
  int sb = t1 % K;
  if (last) {
    for (int c = tid; c < C; c += blockDim.x) {
      const size_t o = ((size_t)b * d.Tstride + L) * C + c;
      sm.ring[sb * C + c] = make_float2(ws.sfrac[o], 0.f);
      sm.Sbase[c] = ws.sint[o];
    }
  } else {
    const float2* ck = ws.bck + seg * K * C;
    for (int idx = tid; idx < K * C; idx += blockDim.x) {
      const int i = idx / C, c = idx % C;
      if (t1 + i > L) continue;
      sm.ring[((t1 + i) % K) * C + c] = ck[idx];
    }
    for (int c = tid; c < C; c += blockDim.x)
      sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t1) * C + c];
    G0 = ws.bcf[seg];
  }
  const double Xc = F0 + G0 - logz2;
  double accmu = 0.0, vsum = 0.0;  // thread c < C: suffix sum of (start - end) marginals
  __syncthreads();
  tile_start(sm, d, ws, b, ts, t1 - 1, t0, t1 - 1, -1);
  int nflush = 0;
  for (int s = t1 - 1; s >= t0; --s) {
    sb = (sb == 0) ? K - 1 : sb - 1;
    if (!tile_row(sm, d, ws, b, ts, s, ri, rf)) {
      if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
      tile_drain(sm, ts);
      return;
    }
    const int par = s & 1;
    if (s < t1 - 1 && tid < C) {
      // position s+1: v = sum of (start - end) marginals strictly after it
      const int u = s + 1;
      const float v = (float)accmu;
      grad_em[((size_t)b * d.T + u) * C + tid] = v;
      vsum += (double)v;
      accmu += (double)sm.stS[(par ^ 1) * C + tid] - (double)sm.stE[(par ^ 1) * C + tid];
    }
    const float* row = store + (size_t)(s - t0) * SW;
    if (r.warpB) {
      const bool act = r.cB < C;
      const int c = act ? r.cB : 0;
      const float Q = -(float)(ri[c] - Sb[c]) - Grel;
      const KFan kf = k_fanin(sm, d, r, sb, min(K, L - s), Q, false, dreg, e);
      const float Bt = (kf.lse == NEG_INF) ? NEG_INF : kf.lse - rf[c];
      // start marginal St[s, c] = 2^(gamma[s,c] + btil[s,c] - log2 Z)
      float St = 0.f;
      if (act && r.jB == 0) {
        const float Xs = (float)(Xc + (double)row[2 * C + 1] + (double)Grel);
        St = (Bt == NEG_INF) ? 0.f : ex2(row[C + c] + Bt + Xs);
        sm.Acur[c] = Bt;
        sm.pcur[c] = ex2(Bt);
        atomicMax(&sm.maxslot[par], f2ord(Bt));
        sm.stS[par * C + c] = St;
        if (start_marg) start_marg[((size_t)b * (d.T + 1) + s) * C + c] = St;
      }
      St = __shfl_sync(FULL_MASK, St, (threadIdx.x & 31) & ~(d.GB - 1));
      if (act && kf.sum > 0.f) {
        const float coef = gbf * St / kf.sum;
#pragma unroll
        for (int i = 0; i < KB_MAX; ++i)
          if (i < d.KB) accd[i] += coef * e[i];
      }
    }
    __syncthreads();
    bool slow;
    const float n = step_frame(sm, par, slow);
    if (tid == 0) sm.maxslot[par ^ 1] = f2ord(NEG_INF);
    if (s >= 1) {
      float shift = n;
      if (slow) {
        for (int c = tid; c < C; c += blockDim.x) sm.pcur[c] = ex2(sm.Acur[c] - n);
        __syncthreads();
        shift = 0.f;
      }
      if (r.warpA) {
        const bool act = r.cA < C;
        const int c = act ? r.cA : 0;
        const float acc = label_fanin(sm, d, r, ereg, prod);
        float E = 0.f;
        if (act && r.jA == 0) {
          float g;
          if (acc >= UNDERFLOW && acc <= 3.0e38f)
            g = lg2(acc) + tmax2 - shift;
          else
            g = label_lse_slow(d, sm.Acur, n, trans, c, true);
          sm.ring[sb * C + c] = make_float2(g + rf[c], (Grel + n) + (float)(ri[c] - Sb[c]));
          // end marginal E[s, c] = 2^(alpha[s,c] + beta[s,c] - log2 Z)
          const float Ys = (float)(Xc + (double)row[2 * C] + (double)(Grel + n));
          E = (g == NEG_INF || row[c] == NEG_INF) ? 0.f : ex2(row[c] + g + Ys);
          sm.stE[par * C + c] = E;
          if (end_marg) end_marg[((size_t)b * (d.T + 1) + s) * C + c] = E;
        }
        E = __shfl_sync(FULL_MASK, E, (threadIdx.x & 31) & ~(d.GA - 1));
        if (act && acc > 0.f) {
          const float coef = gbf * E / acc;
#pragma unroll
          for (int i = 0; i < CA_MAX; ++i)
            if (i < d.CA) acct[i] += coef * prod[i];
        }
      }
    } else {
      for (int c = tid; c < C; c += blockDim.x) {
        sm.stE[par * C + c] = 0.f;
        if (end_marg) end_marg[((size_t)b * (d.T + 1)) * C + c] = 0.f;
      }
    }
    Grel += n;
    if (++nflush == FLUSH_EVERY || s == t0) {
      nflush = 0;
      if (r.cB < C) {
#pragma unroll
        for (int i = 0; i < KB_MAX; ++i) {
          const int k = 1 + r.jB + i * d.GB;
          if (i < d.KB && k <= K) {
            ws.pgd[(seg * K + (k - 1)) * C + r.cB] += (double)accd[i];
            accd[i] = 0.f;
          }
        }
      }
      if (r.cA < C) {
#pragma unroll
        for (int i = 0; i < CA_MAX; ++i) {
          const int x = r.jA + i * d.GA;
          if (i < d.CA && x < C) {
            ws.pgt[(seg * C + r.cA) * C + x] += (double)acct[i];
            acct[i] = 0.f;
          }
        }
      }
    }
    __syncthreads();
  }
  if (tid < C) {
    const int par = t0 & 1;
    const float v = (float)accmu;
    grad_em[((size_t)b * d.T + t0) * C + tid] = v;
    vsum += (double)v;
    accmu += (double)sm.stS[par * C + tid] - (double)sm.stE[par * C + tid];
    ws.segT[seg * C + tid] = accmu;
    ws.segV[seg * C + tid] = vsum;
  }
}

__global__ void selftest_wait_kernel(int* status, int spins) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must give up.
  const bool ok = mbar_wait(&bar, 0, spins);
  if (!__syncthreads_or(!ok)) return;
  if (threadIdx.x == 0) set_status(status, ST_DEVICE_TIMEOUT);
}

}  // namespace semicrf
