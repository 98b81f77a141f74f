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
// Schedule.  One lane group owns one label for both fan-ins, so the k fan-in
// of label c only reads label c's own ring, written by the same warp: a step
// needs a single CTA barrier (between the k fan-in, which produces alpha[t, :],
// and the label fan-in, which reads all of it).
//
// Ring entries are float2 (value v, exact integer part P); a term of the k
// fan-in is ((P + Q) + v) + dur2 with Q the per-step integer offset.
#include "ring.cuh"

namespace semicrf {

using namespace ring;

namespace {

// Forward k fan-in at boundary t: A = alpha[t,c] - F_{t-1}; the leader writes
// Acur/pcur (buffer `par`) and every warp adds to the step max (slot q).
template <int KBT>
__device__ __forceinline__ float fwd_kphase(const Smem& sm, const Dims& d, const KLane<KBT>& kl,
                                            int base, const int32_t* ri, const float* rf,
                                            float Frel, int par, int q, float (&e)[KBT]) {
  const int c = kl.act ? kl.c : 0;
  const float Q = (float)(ri[c] - sm.Sbase[c]) - Frel;
  const KFan kf = k_fanin<KBT>(sm, d, kl, base, Q, e);
  const float A = (kf.lse == NEG_INF) ? NEG_INF : rf[c] + kf.lse;
  int key = INT_MIN;
  if (kl.act && kl.j == 0) {
    sm.Acur[par * d.C + c] = A;
    sm.pcur[par * d.PC + c] = ex2(A);
    key = f2ord(A);
  }
  warp_max_to_shared(&sm.maxslot[q], key);
  return A;
}

// Label fan-in for output label al.c; returns the log2 sum minus the shift
// (gamma - F_t for the forward side, beta - G_s for the backward side) in
// the leader lane, with the log-domain fallback when the sum underflows.
template <int CAT>
__device__ __forceinline__ float aphase(const Smem& sm, const Dims& d, const ALane<CAT>& al, int par,
                                        float n, float shift, const float* trans, bool rows,
                                        float& acc, float (&prod)[CAT]) {
  acc = label_fanin<CAT>(sm.pcur + par * d.PC, d, al, prod);
  float g = 0.f;
  if (al.act && al.j == 0) {
    if (acc >= UNDERFLOW && acc <= 3.0e38f)
      g = lg2(acc) + al.tmax - shift;
    else
      g = label_lse_slow(d, sm.Acur + par * d.C, n, trans, al.c, rows);
  }
  return g;
}

// Uniform slow path: the step's frame jump is too large for 2^A in float32.
__device__ __forceinline__ void refresh_p(const Smem& sm, const Dims& d, int par, float n) {
  for (int c = threadIdx.x; c < d.C; c += blockDim.x)
    sm.pcur[par * d.PC + c] = ex2(sm.Acur[par * d.C + c] - n);
  __syncthreads();
}

__device__ __forceinline__ void final_lse(const float* A, int C, double base, double* out2,
                                          double* out_nat) {
  if (threadIdx.x >= 32) return;
  float m = NEG_INF;
  for (int c = threadIdx.x; c < C; c += 32) m = fmaxf(m, A[c]);
  m = group_max(m, 32);
  float s = 0.f;
  if (m != NEG_INF)
    for (int c = threadIdx.x; c < C; c += 32) s += ex2(A[c] - m);
  s = group_sum(s, 32);
  if (threadIdx.x == 0) {
    const double lz = (m == NEG_INF) ? -INFINITY : base + (double)(m + lg2(s));
    *out2 = lz;
    if (out_nat) *out_nat = lz * LN2_D;
  }
}

}  // namespace

// ===========================================================================
// Forward and backward rings over whole sequences.
// ===========================================================================
template <int KBT, int CAT>
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
  if (L < 0 || L > d.T || L == 0) {
    if (tid == 0) {
      const double v = (L == 0) ? 0.0 : __longlong_as_double(0x7ff8000000000000ll);
      if (L != 0) set_status(ws.status, ST_BAD_LENGTH);
      if (is_alpha) {
        logZ_out[b] = v;
        ws.logz2[b] = v;
      } else {
        ws.logz2b[b] = v;
      }
    }
    return;
  }
  const bool warp_on = ((tid & ~31) / d.GB) < C;
  KLane<KBT> kl;
  kl.init(d, dur, is_alpha);
  ALane<CAT> al;
  al.init(d, trans, !is_alpha);
  float e[KBT], prod[CAT], acc;
  init_smem(sm, d);
  __syncthreads();
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  const int32_t* ri;
  const float* rf;
  int par = 0, q = 0;

  if (is_alpha) {
    // ---------------------------------------------------------------- forward
    for (int c = tid; c < C; c += blockDim.x) {
      ring_put<KBT>(sm, d, c, 0, make_float2(0.f, 0.f));  // boundary 0: gamma 0, frame 0, S 0
      sm.Sbase[c] = 0;
    }
    tile_start(sm, d, ws, b, ts, 1, 0, L, +1);
    double F0 = 0.0;
    float Frel = 0.f;
    int slot = 0;                 // t mod K
    int base = kl.base_up(1, K);  // window base at t = 1
    int to_ck = d.delta;          // steps to the next checkpoint boundary
    __syncthreads();
    for (int t = 1; t <= L; ++t) {
      if (t > 1) base = (base + 1 == K) ? 0 : base + 1;
      slot = (slot + 1 == K) ? 0 : slot + 1;
      par = t & 1;
      q = mod3_next(q);
      if (!tile_row(sm, d, ws, b, ts, t, ri, rf)) {
        if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
        tile_drain(sm, ts);
        return;
      }
      if (--to_ck == 0) {
        to_ck = d.delta;
        if (t < L) {
          // checkpoint j: rebase to (F0 + Frel, S_int[t]), save the ring in boundary order
          __syncthreads();
          const int j = t / d.delta;
          const float dF = Frel;
          for (int idx = tid; idx < C * d.RL; idx += blockDim.x) {
            const int c = idx / d.RL;
            float2 v = sm.ring[idx];
            v.y = (v.y - dF) + (float)(ri[c] - sm.Sbase[c]);
            sm.ring[idx] = v;
          }
          __syncthreads();
          for (int idx = tid; idx < K * C; idx += blockDim.x) {
            const int i = idx / C, c = idx % C;
            if (t - K + i >= 0)
              ws.ack[(((size_t)b * d.nck + j) * K + i) * C + c] = ring_at(sm, d, c, t - K + i);
          }
          for (int c = tid; c < C; c += blockDim.x) sm.Sbase[c] = ri[c];
          F0 += (double)dF;
          Frel = 0.f;
          if (tid == 0) ws.acf[(size_t)b * d.nck + j] = F0;
          __syncthreads();
        }
      }
      if (warp_on) fwd_kphase<KBT>(sm, d, kl, base, ri, rf, Frel, par, q, e);
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, q, slow);
      if (t == L) break;
      float shift = n;
      if (slow) {
        refresh_p(sm, d, par, n);
        shift = 0.f;
      }
      if (warp_on) {
        const float g = aphase<CAT>(sm, d, al, par, n, shift, trans, false, acc, prod);
        if (al.act && al.j == 0) {
          const int c = al.c;
          ring_put<KBT>(sm, d, c, slot,
                        make_float2(g - rf[c], (Frel + n) - (float)(ri[c] - sm.Sbase[c])));
        }
        __syncwarp();
      }
      Frel += n;
    }
    final_lse(sm.Acur + par * C, C, F0 + (double)Frel, &ws.logz2[b], &logZ_out[b]);
  } else {
    // --------------------------------------------------------------- backward
    tile_start(sm, d, ws, b, ts, L, 0, L, -1);
    if (!tile_row(sm, d, ws, b, ts, L, ri, rf)) {
      if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
      tile_drain(sm, ts);
      return;
    }
    int slot = L % K;
    for (int c = tid; c < C; c += blockDim.x) {
      ring_put<KBT>(sm, d, c, slot, make_float2(rf[c], 0.f));  // beta[L] = 0, frame 0, base S_int[L]
      sm.Sbase[c] = ri[c];
    }
    double G0 = 0.0;
    float Grel = 0.f;
    int base = kl.base_down(L - 1, K);
    int to_ck = L % d.delta;  // (s + 1) mod delta
    __syncthreads();
    for (int s = L - 1; s >= 0; --s) {
      if (s < L - 1) base = (base == 0) ? K - 1 : base - 1;
      slot = (slot == 0) ? K - 1 : slot - 1;
      par = s & 1;
      q = mod3_next(q);
      if (!tile_row(sm, d, ws, b, ts, s, ri, rf)) {
        if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
        tile_drain(sm, ts);
        return;
      }
      if (to_ck == 0 && s + 1 < L) {
        // checkpoint j: the ring holds boundaries t1..t1+K-1; rebase to (G0 + Grel, S_int[t1])
        __syncthreads();
        const int t1 = s + 1;
        const int j = t1 / d.delta - 1;
        for (int c = tid; c < C; c += blockDim.x) sm.tmp[c] = ring_at(sm, d, c, t1).y;
        __syncthreads();
        for (int idx = tid; idx < C * d.RL; idx += blockDim.x) sm.ring[idx].y -= sm.tmp[idx / d.RL];
        __syncthreads();
        for (int idx = tid; idx < K * C; idx += blockDim.x) {
          const int i = idx / C, c = idx % C;
          if (t1 + i <= L)
            ws.bck[(((size_t)b * d.nck + j) * K + i) * C + c] = ring_at(sm, d, c, t1 + i);
        }
        for (int c = tid; c < C; c += blockDim.x)
          sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t1) * C + c];
        G0 += (double)Grel;
        Grel = 0.f;
        if (tid == 0) ws.bcf[(size_t)b * d.nck + j] = G0;
        __syncthreads();
      }
      to_ck = (to_ck == 0) ? d.delta - 1 : to_ck - 1;
      if (warp_on) {
        const int c = kl.act ? kl.c : 0;
        const float Q = -(float)(ri[c] - sm.Sbase[c]) - Grel;
        const KFan kf = k_fanin<KBT>(sm, d, kl, base, Q, e);
        const float Bt = (kf.lse == NEG_INF) ? NEG_INF : kf.lse - rf[c];
        int key = INT_MIN;
        if (kl.act && kl.j == 0) {
          sm.Acur[par * C + c] = Bt;
          sm.pcur[par * d.PC + c] = ex2(Bt);
          key = f2ord(Bt);
        }
        warp_max_to_shared(&sm.maxslot[q], key);
      }
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, q, slow);
      if (s == 0) break;
      float shift = n;
      if (slow) {
        refresh_p(sm, d, par, n);
        shift = 0.f;
      }
      if (warp_on) {
        const float g = aphase<CAT>(sm, d, al, par, n, shift, trans, true, acc, prod);
        if (al.act && al.j == 0) {
          const int c = al.c;
          ring_put<KBT>(sm, d, c, slot,
                        make_float2(g + rf[c], (Grel + n) + (float)(ri[c] - sm.Sbase[c])));
        }
        __syncwarp();
      }
      Grel += n;
    }
    final_lse(sm.Acur + par * C, C, G0 + (double)Grel, &ws.logz2b[b], nullptr);
  }
}

// ===========================================================================
// Checkpoint-parallel posteriors: one CTA per (segment j, sequence b).
// Restores the forward ring at t0 = j*Delta and recomputes alpha over
// [t0, t1) into a per-position store, then restores the backward ring at t1
// and walks down to t0 accumulating the exact posteriors:
//   start_marg[s,c] = 2^(gamma[s,c] + btil[s,c] - log2 Z)
//   end_marg[s,c]   = 2^(alpha[s,c] + beta[s,c] - log2 Z)
//   P(segment [s, s+k), c) = start_marg[s,c] * (normalised k term of btil)
//   P(c' -> c at s)        = end_marg[s,c'] * (normalised c term of beta)
// The leader lane of label c's group keeps c's running sums.
// ===========================================================================
template <int KBT, int CAT>
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
  const float gbf = (float)(grad_logZ ? grad_logZ[b] : 1.0);
  const double logz2 = ws.logz2[b];
  const int SW = d.store_w;
  float* store = sm.store ? sm.store : ws.store + ((size_t)b * d.nck + j) * d.delta * SW;
  const size_t seg = (size_t)b * d.nck + j;
  const bool warp_on = ((tid & ~31) / d.GB) < C;
  float e[KBT], prod[CAT], acc;
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  const int32_t* ri;
  const float* rf;
  double F0 = 0.0;
  float Frel = 0.f;
  int par = 0, q = 0;

  // ------------------------------------------------------ alpha recompute
  {
    KLane<KBT> kl;
    kl.init(d, dur, true);
    ALane<CAT> al;
    al.init(d, trans, false);
    init_smem(sm, d);
    __syncthreads();
    int t_start;
    if (j == 0) {
      for (int c = tid; c < C; c += blockDim.x) {
        ring_put<KBT>(sm, d, c, 0, make_float2(0.f, 0.f));
        sm.Sbase[c] = 0;
        store[c] = NEG_INF;  // no alpha at boundary 0
        store[C + c] = 0.f;  // gamma[0] = 0 in frame 0
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
        if (bnd >= 0) ring_put<KBT>(sm, d, c, bnd % K, ck[idx]);
      }
      for (int c = tid; c < C; c += blockDim.x)
        sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t0) * C + c];
      F0 = ws.acf[seg];
      t_start = t0;
    }
    const int t_end = last ? L : t1 - 1;
    __syncthreads();
    tile_start(sm, d, ws, b, ts, t_start, t_start, t_end, +1);
    int slot = t_start % K;
    int base = kl.base_up(t_start, K);
    for (int t = t_start; t <= t_end; ++t) {
      if (t > t_start) {
        base = (base + 1 == K) ? 0 : base + 1;
        slot = (slot + 1 == K) ? 0 : slot + 1;
      }
      par = t & 1;
      q = mod3_next(q);
      if (!tile_row(sm, d, ws, b, ts, t, ri, rf)) {
        if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
        tile_drain(sm, ts);
        return;
      }
      float A = 0.f;
      if (warp_on) A = fwd_kphase<KBT>(sm, d, kl, base, ri, rf, Frel, par, q, e);
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, q, slow);
      if (t == L) break;
      float shift = n;
      if (slow) {
        refresh_p(sm, d, par, n);
        shift = 0.f;
      }
      float* row = store + (size_t)(t - t0) * SW;
      if (warp_on) {
        const float g = aphase<CAT>(sm, d, al, par, n, shift, trans, false, acc, prod);
        if (al.act && al.j == 0) {
          const int c = al.c;
          ring_put<KBT>(sm, d, c, slot,
                        make_float2(g - rf[c], (Frel + n) - (float)(ri[c] - sm.Sbase[c])));
          row[c] = A;
          row[C + c] = g;
        }
        __syncwarp();
      }
      if (tid == 0) {
        row[2 * C] = Frel;
        row[2 * C + 1] = Frel + n;
      }
      Frel += n;
    }
  }
  __syncthreads();
  if (last) {
    // end marginal at boundary L (beta[L] = 0); nothing starts at L
    const float XL = (float)(F0 + (double)Frel - logz2);
    for (int c = tid; c < C; c += blockDim.x) {
      const size_t o = ((size_t)b * (d.T + 1) + L) * C + c;
      if (end_marg) end_marg[o] = ex2(sm.Acur[par * C + c] + XL);
      if (start_marg) start_marg[o] = 0.f;
    }
  }

  // ------------------------------------------------------ beta recompute + posteriors
  KLane<KBT> kb;
  kb.init(d, dur, false);
  ALane<CAT> ab;
  ab.init(d, trans, true);
  __syncthreads();
  for (int i = tid; i < d.RL * C; i += blockDim.x) sm.ring[i] = make_float2(NEG_INF, 0.f);
  __syncthreads();
  double G0 = 0.0;
  float Grel = 0.f;
  if (last) {
    for (int c = tid; c < C; c += blockDim.x) {
      const size_t o = ((size_t)b * d.Tstride + L) * C + c;
      ring_put<KBT>(sm, d, c, L % K, make_float2(ws.sfrac[o], 0.f));
      sm.Sbase[c] = ws.sint[o];
    }
  } else {
    const float2* ck = ws.bck + seg * K * C;
    for (int idx = tid; idx < K * C; idx += blockDim.x) {
      const int i = idx / C, c = idx % C;
      if (t1 + i <= L) ring_put<KBT>(sm, d, c, (t1 + i) % K, ck[idx]);
    }
    for (int c = tid; c < C; c += blockDim.x)
      sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t1) * C + c];
    G0 = ws.bcf[seg];
  }
  // this CTA's float64 partials start at zero (each thread its own entries)
  float accd[KBT];
  float acct[CAT];
#pragma unroll
  for (int i = 0; i < KBT; ++i) {
    accd[i] = 0.f;
    const int k = kb.k_of(i, false);
    if (kb.act && k <= K) ws.pgd[(seg * K + (k - 1)) * C + kb.c] = 0.0;
  }
#pragma unroll
  for (int i = 0; i < CAT; ++i) {
    acct[i] = 0.f;
    const int x = ab.j * CAT + i;
    if (ab.act && x < C) ws.pgt[(seg * C + ab.c) * C + x] = 0.0;
  }
  const double Xc = F0 + G0 - logz2;
  double accmu = 0.0, vsum = 0.0;  // leader of label c: suffix sum of (start - end) marginals
  const bool leader = kb.act && kb.j == 0;
  __syncthreads();
  tile_start(sm, d, ws, b, ts, t1 - 1, t0, t1 - 1, -1);
  int nflush = 0;
  int slot = t1 % K;
  int base = kb.base_down(t1 - 1, K);
  for (int s = t1 - 1; s >= t0; --s) {
    if (s < t1 - 1) base = (base == 0) ? K - 1 : base - 1;
    slot = (slot == 0) ? K - 1 : slot - 1;
    par = s & 1;
    q = mod3_next(q);
    if (!tile_row(sm, d, ws, b, ts, s, ri, rf)) {
      if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
      tile_drain(sm, ts);
      return;
    }
    const float* row = store + (size_t)(s - t0) * SW;
    float St = 0.f;
    if (warp_on) {
      const int c = kb.act ? kb.c : 0;
      const float Q = -(float)(ri[c] - sm.Sbase[c]) - Grel;
      const KFan kf = k_fanin<KBT>(sm, d, kb, base, Q, e);
      const float Bt = (kf.lse == NEG_INF) ? NEG_INF : kf.lse - rf[c];
      int key = INT_MIN;
      if (leader) {
        const float Xs = (float)(Xc + (double)row[2 * C + 1] + (double)Grel);
        St = (Bt == NEG_INF) ? 0.f : ex2(row[C + c] + Bt + Xs);
        sm.Acur[par * C + c] = Bt;
        sm.pcur[par * d.PC + c] = ex2(Bt);
        key = f2ord(Bt);
        if (start_marg) start_marg[((size_t)b * (d.T + 1) + s) * C + c] = St;
      }
      warp_max_to_shared(&sm.maxslot[q], key);
      const float Stg = __shfl_sync(FULL_MASK, St, (tid & 31) & ~(d.GB - 1));
      if (kb.act && kf.sum > 0.f) {
        const float coef = gbf * Stg / kf.sum;
#pragma unroll
        for (int i = 0; i < KBT; ++i) accd[i] += coef * e[i];
      }
    }
    __syncthreads();
    bool slow;
    const float n = step_frame(sm, q, slow);
    float E = 0.f;
    if (s >= 1) {
      float shift = n;
      if (slow) {
        refresh_p(sm, d, par, n);
        shift = 0.f;
      }
      if (warp_on) {
        const float g = aphase<CAT>(sm, d, ab, par, n, shift, trans, true, acc, prod);
        if (leader) {
          const int c = ab.c;
          ring_put<KBT>(sm, d, c, slot,
                        make_float2(g + rf[c], (Grel + n) + (float)(ri[c] - sm.Sbase[c])));
          const float Ys = (float)(Xc + (double)row[2 * C] + (double)(Grel + n));
          E = (g == NEG_INF || row[c] == NEG_INF) ? 0.f : ex2(row[c] + g + Ys);
          if (end_marg) end_marg[((size_t)b * (d.T + 1) + s) * C + c] = E;
        }
        const float Eg = __shfl_sync(FULL_MASK, E, (tid & 31) & ~(d.GB - 1));
        if (ab.act && acc > 0.f) {
          const float coef = gbf * Eg / acc;
#pragma unroll
          for (int i = 0; i < CAT; ++i) acct[i] += coef * prod[i];
        }
        __syncwarp();
      }
    } else if (leader && end_marg) {
      end_marg[((size_t)b * (d.T + 1)) * C + kb.c] = 0.f;
    }
    if (leader) {
      // position s: v = sum of (start - end) marginals strictly after it in the segment
      const float v = (float)accmu;
      grad_em[((size_t)b * d.T + s) * C + kb.c] = v;
      vsum += (double)v;
      accmu += (double)St - (double)E;
    }
    Grel += n;
    if (++nflush == FLUSH_EVERY || s == t0) {
      nflush = 0;
      if (kb.act) {
#pragma unroll
        for (int i = 0; i < KBT; ++i) {
          const int k = kb.k_of(i, false);
          if (k <= K) ws.pgd[(seg * K + (k - 1)) * C + kb.c] += (double)accd[i];
          accd[i] = 0.f;
        }
      }
      if (ab.act) {
#pragma unroll
        for (int i = 0; i < CAT; ++i) {
          const int x = ab.j * CAT + i;
          if (x < C) ws.pgt[(seg * C + ab.c) * C + x] += (double)acct[i];
          acct[i] = 0.f;
        }
      }
    }
  }
  if (leader) {
    ws.segT[seg * C + kb.c] = accmu;
    ws.segV[seg * C + kb.c] = vsum;
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

// ----------------------------------------------------------------------------- launchers
bool shape_supported(int KBT, int CAT) {
#define SEMICRF_SHAPE_OK(a, b) \
  if (KBT == a && CAT == b) return true;
  SEMICRF_FOR_EACH_SHAPE(SEMICRF_SHAPE_OK)
#undef SEMICRF_SHAPE_OK
  return false;
}

namespace {
template <typename F>
cudaError_t allow_smem(F fn, size_t sm) {
  if (sm <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
}
}  // namespace

cudaError_t launch_chain(const Dims& d, const WsPtrs& ws, const int32_t* lengths, const float* trans,
                         const float* dur, double* logZ_out, int n_alpha, int n_beta,
                         cudaStream_t st) {
  const size_t sm = recursion_smem_bytes(d, false);
#define SEMICRF_LAUNCH_CHAIN(a, b)                                                          \
  if (d.KBT == a && d.CAT == b) {                                                           \
    const cudaError_t e = allow_smem(chain_kernel<a, b>, sm);                               \
    if (e != cudaSuccess) return e;                                                         \
    chain_kernel<a, b><<<n_alpha + n_beta, d.NT, sm, st>>>(d, ws, lengths, trans, dur, logZ_out, \
                                                           n_alpha);                        \
    return cudaGetLastError();                                                              \
  }
  SEMICRF_FOR_EACH_SHAPE(SEMICRF_LAUNCH_CHAIN)
#undef SEMICRF_LAUNCH_CHAIN
  return cudaErrorInvalidConfiguration;
}

cudaError_t launch_segment(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                           const float* trans, const float* dur, const double* grad_logZ,
                           float* grad_em, float* start_marg, float* end_marg, cudaStream_t st) {
  const size_t sm = recursion_smem_bytes(d, d.store_smem != 0);
#define SEMICRF_LAUNCH_SEG(a, b)                                                         \
  if (d.KBT == a && d.CAT == b) {                                                        \
    const cudaError_t e = allow_smem(segment_kernel<a, b>, sm);                          \
    if (e != cudaSuccess) return e;                                                      \
    segment_kernel<a, b><<<dim3(d.nck, d.B), d.NT, sm, st>>>(d, ws, lengths, trans, dur,   \
                                                             grad_logZ, grad_em, start_marg, \
                                                             end_marg);                    \
    return cudaGetLastError();                                                           \
  }
  SEMICRF_FOR_EACH_SHAPE(SEMICRF_LAUNCH_SEG)
#undef SEMICRF_LAUNCH_SEG
  return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
