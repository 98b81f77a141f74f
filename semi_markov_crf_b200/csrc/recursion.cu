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

// Forward checkpoint at boundary t (start of step t): rebase every ring entry
// to the frame (F0 + Frel, S_int[t]) and save the K boundaries before t.
__device__ __forceinline__ void fwd_checkpoint(const Smem& sm, const Dims& d, const WsPtrs& ws,
                                               int b, int t, const int32_t* ri, float Frel) {
  const int C = d.C, K = d.K;
  const int j = t / d.delta;
  __syncthreads();
  for (int idx = threadIdx.x; idx < C * d.RL; idx += blockDim.x) {
    const int c = idx / d.RL;
    float2 v = sm.ring[idx];
    v.y = (v.y - Frel) + (float)(ri[c] - sm.Sbase[c]);
    sm.ring[idx] = v;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < K * C; idx += blockDim.x) {
    const int i = idx / C, c = idx % C;
    if (t - K + i >= 0)
      ws.ack[(((size_t)b * d.nck + j) * K + i) * C + c] = ring_at(sm, d, c, t - K + i);
  }
  for (int c = threadIdx.x; c < C; c += blockDim.x) sm.Sbase[c] = ri[c];
  __syncthreads();
}

// Backward checkpoint at boundary t1 (start of step t1 - 1): rebase to
// (G0 + Grel, S_int[t1]) and save boundaries t1..t1+K-1.
__device__ __forceinline__ void bwd_checkpoint(const Smem& sm, const Dims& d, const WsPtrs& ws,
                                               int b, int t1, int L) {
  const int C = d.C, K = d.K;
  const int j = t1 / d.delta - 1;
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) sm.tmp[c] = ring_at(sm, d, c, t1).y;
  __syncthreads();
  for (int idx = threadIdx.x; idx < C * d.RL; idx += blockDim.x) sm.ring[idx].y -= sm.tmp[idx / d.RL];
  __syncthreads();
  for (int idx = threadIdx.x; idx < K * C; idx += blockDim.x) {
    const int i = idx / C, c = idx % C;
    if (t1 + i <= L) ws.bck[(((size_t)b * d.nck + j) * K + i) * C + c] = ring_at(sm, d, c, t1 + i);
  }
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t1) * C + c];
  __syncthreads();
}

// Normaliser of checkpoint segment j >= 1, from the cut at position
// u = t0 - 1 (t0 = j Delta): every segmentation has exactly one segment
// [s, t) with s <= u < t, so
//   Z = sum_{c, s < t0 <= t, t - s <= K} 2^(gamma[s,c] - S[s,c]) 2^(dur2[t-s-1,c]) 2^(S[t,c] + beta[t,c])
// and the share of label c in that sum is mu[u, c].  The forward factors come
// from the ring the forward chain saved at t0 (boundaries t0-K..t0-1, entry
// (x, y) encoding gamma - S = x + y + F0 - S_int[t0]), which is also where
// the segment's alpha recompute starts; the backward factors from the
// segment's own backward ring once its walk has reached t0 (boundaries
// t0..t0+K-1, beta + S = x + y + G0 + Sbase[c]).  Dividing the segment's
// posteriors by this Z makes them ratios of the very values they were built
// from, whatever rounding separates those from the chains' values over the
// positions before t0 and after t1 -- and whatever arithmetic the chains used.
// Returns log2 Z (float64) to every thread and leaves mu[u, c] in sm.tmp[c].
// Uses sm.Acur as scratch; starts and ends with a barrier.
__device__ double segment_cut(const Smem& sm, const Dims& d, const WsPtrs& ws, int b, int j, int L,
                              double G0, const float* __restrict__ dur, double* lz_out) {
  const int C = d.C, K = d.K, t0 = j * d.delta;
  const size_t seg = (size_t)b * d.nck + j;
  const float2* fa = ws.ack + seg * K * C;  // boundary t0 - K + i
  const int32_t* s0 = ws.sint + ((size_t)b * d.Tstride + t0) * C;
  __syncthreads();
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int kb_max = min(K - 1, L - t0);  // t - t0 <= K - 1 and t <= L
  for (int c = threadIdx.x >> 5; c < C; c += nw) {
    const float2* bc = sm.ring + (size_t)c * d.RL;
    const float sh = (float)(sm.Sbase[c] - __ldg(s0 + c));  // exact integer
    float zmax = NEG_INF;
    for (int ia = lane; ia < K; ia += 32) {
      if (t0 - K + ia < 0) continue;
      const float2 a = fa[(size_t)ia * C + c];
      const int kbe = min(ia, kb_max);  // t = t0 + kb <= s + K = t0 + ia
      for (int kb = 0; kb <= kbe; ++kb) {
        const float2 v = bc[(t0 + kb) % K];
        const float dk = __ldg(dur + (size_t)(kb + K - ia - 1) * C + c) * l2e();
        zmax = fmaxf(zmax, (((a.y + v.y) + sh) + (a.x + v.x)) + dk);
      }
    }
    zmax = group_max(zmax, 32);
    const float M = (zmax == NEG_INF) ? 0.f : ceilf(zmax);
    float sum = 0.f;
    for (int ia = lane; ia < K; ia += 32) {
      if (t0 - K + ia < 0) continue;
      const float2 a = fa[(size_t)ia * C + c];
      const int kbe = min(ia, kb_max);
      for (int kb = 0; kb <= kbe; ++kb) {
        const float2 v = bc[(t0 + kb) % K];
        const float dk = __ldg(dur + (size_t)(kb + K - ia - 1) * C + c) * l2e();
        sum += ex2(((((a.y + v.y) + sh) - M) + (a.x + v.x)) + dk);
      }
    }
    sum = group_sum(sum, 32);
    if (lane == 0) {
      sm.Acur[c] = M;                                 // exact integer shift
      sm.tmp[c] = (sum > 0.f) ? lg2(sum) : NEG_INF;  // log2 of the label's share
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    float Mz = NEG_INF;
    for (int c = lane; c < C; c += 32)
      if (sm.tmp[c] != NEG_INF) Mz = fmaxf(Mz, sm.Acur[c]);
    Mz = group_max(Mz, 32);
    if (Mz == NEG_INF) Mz = 0.f;
    float tot = 0.f;
    for (int c = lane; c < C; c += 32) tot += ex2((sm.Acur[c] - Mz) + sm.tmp[c]);
    tot = group_sum(tot, 32);
    const float lt = (tot > 0.f) ? lg2(tot) : NEG_INF;
    __syncwarp();
    for (int c = lane; c < C; c += 32) sm.tmp[c] = ex2(((sm.Acur[c] - Mz) + sm.tmp[c]) - lt);
    if (lane == 0) *lz_out = (ws.acf[seg] + G0) + ((double)Mz + (double)lt);
  }
  __syncthreads();
  return *lz_out;
}

}  // namespace

// ===========================================================================
// Forward and backward rings over whole sequences.
// ===========================================================================
template <int KBT, int CAT, int G, int LB>
__global__ void __launch_bounds__(LB, 1)
    chain_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                 const float* __restrict__ trans, const float* __restrict__ dur,
                 double* __restrict__ logZ_out, int n_alpha) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem sm = carve(smem_raw, d, false);
  const int C = d.C, K = d.K, PC = d.PC, tid = threadIdx.x;
  const bool is_alpha = (int)blockIdx.x < n_alpha;
  const int b = is_alpha ? blockIdx.x : blockIdx.x - n_alpha;
  // already run by the exponential-domain kernel (chain_exp.cu)
  if (ws.mode && ws.mode[(is_alpha ? 0 : d.B) + b] == 1) return;
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
  Lane<KBT, CAT, G> ln;
  ln.init_ids(d);
  ln.init_dur(d, dur, is_alpha);
  float2* const rl = sm.ring + (size_t)ln.cc * d.RL;  // this lane's label ring
  float e[KBT], p[CAT];
  const bool pj = proj_on(ws);  // boundary projections
  init_smem(sm, d);
  __syncthreads();
  ln.init_trans(d, trans, !is_alpha, block_trans_max(sm, d, trans));
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  int par = 0, q = 0;
  float mk = 0.f;  // shift of the k fan-in (predicted LSE)

  if (is_alpha) {
    // ---------------------------------------------------------------- forward
    for (int c = tid; c < C; c += blockDim.x) {
      ring_put<KBT>(sm.ring + (size_t)c * d.RL, d, 0,
                    make_float2(proj_d(ws, d, pj, b, 0, c), 0.f));  // boundary 0
      sm.Sbase[c] = 0;
    }
    tile_start(sm, d, ws, b, ts, 1, 1, L, +1);
    double F0 = 0.0;
    float Frel = 0.f;
    int Sb = 0;                   // Sbase of this lane's label
    int wslot = 0;                // t mod K
    int base = ln.base_up(1, K);  // window base at t = 1
    int to_ck = d.delta;          // steps to the next checkpoint boundary
    int cur = -1, t = 1;
    __syncthreads();
    for (;;) {
      const int ti = t / TS;
      if (ti != cur) {
        if (!tile_enter(sm, d, ws, b, ts, ti)) {
          if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
          tile_drain(sm, ts);
          return;
        }
        cur = ti;
      }
      const int t_stop = min(L, ti * TS + TS - 1);
      const size_t off = tile_row_off(t, C);
      const int32_t* ri = sm.tint + off;
      const float* rf = sm.tfrac + off;
      bool done = false;
      for (; t <= t_stop; ++t, ri += C, rf += C) {
        if (t > 1) base = (base + 1 == K) ? 0 : base + 1;
        wslot = (wslot + 1 == K) ? 0 : wslot + 1;
        par = t & 1;
        q = mod3_next(q);
        if (--to_ck == 0) {
          to_ck = d.delta;
          if (t < L) {
            fwd_checkpoint(sm, d, ws, b, t, ri, Frel);
            F0 += (double)Frel;
            Frel = 0.f;
            if (tid == 0) ws.acf[(size_t)b * d.nck + t / d.delta] = F0;
            Sb = ri[ln.cc];
          }
        }
        const int si = ri[ln.cc];
        const float sf = rf[ln.cc];
        float s;
        const float lse =
            k_fanin<KBT, G>(rl + checked_base(ws, base, K),
                            ln.j, (float)(si - Sb) - Frel, ln.d, mk, s, e, ln.act);
        const float A = (lse == NEG_INF) ? NEG_INF : sf + lse;
        if (ln.leader) {
          sm.Acur[par * C + ln.c] = A;
          sm.pcur[par * PC + ln.c] = ex2(A);
        }
        warp_max_to_shared(&sm.maxslot[q], ln.leader ? f2ord(A) : INT_MIN);
        __syncthreads();
        bool slow;
        const float n = step_frame(sm, q, slow);
        if (t == L) {
          done = true;
          break;
        }
        mk = next_shift(lse, n, mk);
        float shift = n;
        if (slow) {
          refresh_p(sm, d, par, n);
          shift = 0.f;
        }
        const float acc = label_fanin<CAT, G>(sm.pcur + par * PC + ln.j * CAT, ln.e, p);
        if (ln.leader) {
          const float g = label_log(acc, ln.tmax, shift, C, sm.Acur + par * C, n, trans, ln.c, false);
          if (checked_slot(ws, wslot, K))
            ring_put<KBT>(rl, d, wslot, make_float2((g - sf) + proj_d(ws, d, pj, b, t, ln.c),
                                                    (Frel + n) - (float)(si - Sb)));
        }
        __syncwarp();
        Frel += n;
      }
      if (done) break;
    }
    final_lse(sm.Acur + par * C, C, F0 + (double)Frel, &ws.logz2[b], &logZ_out[b]);
  } else {
    // --------------------------------------------------------------- backward
    tile_start(sm, d, ws, b, ts, L, 0, L, -1);
    int cur = L / TS;
    if (!tile_enter(sm, d, ws, b, ts, cur)) {
      if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
      tile_drain(sm, ts);
      return;
    }
    {
      const size_t off = tile_row_off(L, C);
      for (int c = tid; c < C; c += blockDim.x) {
        // beta[L] = 0 in frame 0 with base S_int[L]
        ring_put<KBT>(sm.ring + (size_t)c * d.RL, d, L % K, make_float2(sm.tfrac[off + c], 0.f));
        sm.Sbase[c] = sm.tint[off + c];
      }
    }
    __syncthreads();
    int Sb = sm.Sbase[ln.cc];
    double G0 = 0.0;
    float Grel = 0.f;
    int wslot = L % K;
    int base = ln.base_down(L - 1, K);
    int to_ck = L % d.delta;  // (s + 1) mod delta
    int s = L - 1;
    for (;;) {
      const int ti = s / TS;
      if (ti != cur) {
        if (!tile_enter(sm, d, ws, b, ts, ti)) {
          if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
          tile_drain(sm, ts);
          return;
        }
        cur = ti;
      }
      const int s_stop = ti * TS;
      const size_t off = tile_row_off(s, C);
      const int32_t* ri = sm.tint + off;
      const float* rf = sm.tfrac + off;
      bool done = false;
      for (; s >= s_stop; --s, ri -= C, rf -= C) {
        if (s < L - 1) base = (base == 0) ? K - 1 : base - 1;
        wslot = (wslot == 0) ? K - 1 : wslot - 1;
        par = s & 1;
        q = mod3_next(q);
        if (to_ck == 0 && s + 1 < L) {
          bwd_checkpoint(sm, d, ws, b, s + 1, L);
          G0 += (double)Grel;
          Grel = 0.f;
          if (tid == 0) ws.bcf[(size_t)b * d.nck + (s + 1) / d.delta - 1] = G0;
          Sb = sm.Sbase[ln.cc];
        }
        to_ck = (to_ck == 0) ? d.delta - 1 : to_ck - 1;
        const int si = ri[ln.cc];
        const float sf = rf[ln.cc];
        float ssum;
        const float lse =
            k_fanin<KBT, G>(rl + checked_base(ws, base, K),
                            ln.j, -(float)(si - Sb) - Grel, ln.d, mk, ssum, e, ln.act);
        const float Bt = (lse == NEG_INF) ? NEG_INF : (lse - sf) + proj_d(ws, d, pj, b, s, ln.cc);
        if (ln.leader) {
          sm.Acur[par * C + ln.c] = Bt;
          sm.pcur[par * PC + ln.c] = ex2(Bt);
        }
        warp_max_to_shared(&sm.maxslot[q], ln.leader ? f2ord(Bt) : INT_MIN);
        __syncthreads();
        bool slow;
        const float n = step_frame(sm, q, slow);
        if (s == 0) {
          done = true;
          break;
        }
        mk = next_shift(lse, n, mk);
        float shift = n;
        if (slow) {
          refresh_p(sm, d, par, n);
          shift = 0.f;
        }
        const float acc = label_fanin<CAT, G>(sm.pcur + par * PC + ln.j * CAT, ln.e, p);
        if (ln.leader) {
          const float g = label_log(acc, ln.tmax, shift, C, sm.Acur + par * C, n, trans, ln.c, true);
          if (checked_slot(ws, wslot, K))
            ring_put<KBT>(rl, d, wslot, make_float2(g + sf, (Grel + n) + (float)(si - Sb)));
        }
        __syncwarp();
        Grel += n;
      }
      if (done) break;
    }
    final_lse(sm.Acur + par * C, C, G0 + (double)Grel, &ws.logz2b[b], nullptr);
  }
}

// ===========================================================================
// Checkpoint-parallel posteriors: one CTA per (segment j, sequence b).
// Restores the forward ring at t0 = j*Delta and recomputes alpha over
// [t0, t1) into a per-position store, then restores the backward ring at t1
// and walks down to t0 accumulating the exact posteriors:
//   start_marg[s,c] = 2^(gamma[s,c] + btil[s,c] - log2 Z_j)
//   end_marg[s,c]   = 2^(alpha[s,c] + beta[s,c] - log2 Z_j)
//   P(segment [s, s+k), c) = start_marg[s,c] * (normalised k term of btil)
//   P(c' -> c at s)        = end_marg[s,c'] * (normalised c term of beta)
// Z_j is the segment's own cut normaliser (segment_cut; sum_c start_marg[0, c]
// for j = 0), found when the walk reaches t0 -- equal to Z in exact
// arithmetic and made of the same forward and backward values as the
// segment's posteriors -- which rescales the walk's provisional results.
// The leader lane of label c's group keeps c's running sums.
// ===========================================================================
template <int KBT, int CAT, int G, int LB>
__global__ void __launch_bounds__(LB, 1)
    segment_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                   const float* __restrict__ trans, const float* __restrict__ dur,
                   const double* __restrict__ grad_logZ, float* __restrict__ grad_em,
                   float* __restrict__ start_marg, float* __restrict__ end_marg,
                   float* __restrict__ seg_marg) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem sm = carve(smem_raw, d, d.store_smem != 0);
  const int C = d.C, K = d.K, PC = d.PC, tid = threadIdx.x;
  const int j = blockIdx.x, b = blockIdx.y;
  const int L = lengths[b];
  if (L < 0 || L > d.T) return;  // reported by the forward pass
  if (posterior_from_kept(ws, d, b)) return;  // posterior_kernel runs it
  const int t0 = j * d.delta;
  if (t0 >= L) return;
  const int t1 = min(t0 + d.delta, L);
  const bool last = (t1 == L);
  const float gbf = (float)(grad_logZ ? grad_logZ[b] : 1.0);
  const int SW = d.store_w;
  float* store = sm.store ? sm.store : ws.store + ((size_t)b * d.nck + j) * d.delta * SW;
  const size_t seg = (size_t)b * d.nck + j;
  Lane<KBT, CAT, G> ln;
  ln.init_ids(d);
  float2* const rl = sm.ring + (size_t)ln.cc * d.RL;
  float e[KBT], p[CAT];
  const bool pj = proj_on(ws);  // boundary projections
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  double F0 = 0.0;
  float Frel = 0.f;
  float tmax2 = 0.f;
  int par = 0, q = 0;

  // Provisional normaliser for the walk (the forward chain's log Z: close
  // enough to keep every posterior O(1)); the segment's own normaliser is
  // computed once its backward walk has reached t0, and the outputs are
  // rescaled by the ratio.
  __shared__ double s_lz;
  __shared__ float s_r;
  const double logz2 = ws.logz2[b];

  // ------------------------------------------------------ alpha recompute
  {
    ln.init_dur(d, dur, true);
    init_smem(sm, d);
    __syncthreads();
    tmax2 = block_trans_max(sm, d, trans);
    ln.init_trans(d, trans, false, tmax2);
    int t_start, Sb;
    if (j == 0) {
      for (int c = tid; c < C; c += blockDim.x) {
        ring_put<KBT>(sm.ring + (size_t)c * d.RL, d, 0, make_float2(proj_d(ws, d, pj, b, 0, c), 0.f));
        store[c] = NEG_INF;  // no alpha at boundary 0
        store[C + c] = 0.f;  // gamma[0] = 0 in frame 0
      }
      if (tid == 0) {
        store[2 * C] = 0.f;
        store[2 * C + 1] = 0.f;
      }
      Sb = 0;
      t_start = 1;
    } else {
      const float2* ck = ws.ack + seg * K * C;
      for (int idx = tid; idx < K * C; idx += blockDim.x) {
        const int i = idx / C, c = idx % C;
        const int bnd = t0 - K + i;
        if (bnd >= 0) ring_put<KBT>(sm.ring + (size_t)c * d.RL, d, bnd % K, ck[idx]);
      }
      Sb = ws.sint[((size_t)b * d.Tstride + t0) * C + ln.cc];
      F0 = ws.acf[seg];
      t_start = t0;
    }
    const int t_end = last ? L : t1 - 1;
    __syncthreads();
    tile_start(sm, d, ws, b, ts, t_start, t_start, t_end, +1);
    int wslot = t_start % K;
    int base = ln.base_up(t_start, K);
    float mk = 0.f;
    int cur = -1, t = t_start;
    bool done = false;
    while (!done) {
      const int ti = t / TS;
      if (ti != cur) {
        if (!tile_enter(sm, d, ws, b, ts, ti)) {
          if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
          tile_drain(sm, ts);
          return;
        }
        cur = ti;
      }
      const int t_stop = min(t_end, ti * TS + TS - 1);
      const size_t off = tile_row_off(t, C);
      const int32_t* ri = sm.tint + off;
      const float* rf = sm.tfrac + off;
      for (; t <= t_stop; ++t, ri += C, rf += C) {
        if (t > t_start) {
          base = (base + 1 == K) ? 0 : base + 1;
          wslot = (wslot + 1 == K) ? 0 : wslot + 1;
        }
        par = t & 1;
        q = mod3_next(q);
        const int si = ri[ln.cc];
        const float sf = rf[ln.cc];
        float s;
        const float lse = k_fanin<KBT, G>(rl + checked_base(ws, base, K),
                                          ln.j, (float)(si - Sb) - Frel, ln.d, mk, s, e, ln.act);
        const float A = (lse == NEG_INF) ? NEG_INF : sf + lse;
        if (ln.leader) {
          sm.Acur[par * C + ln.c] = A;
          sm.pcur[par * PC + ln.c] = ex2(A);
        }
        warp_max_to_shared(&sm.maxslot[q], ln.leader ? f2ord(A) : INT_MIN);
        __syncthreads();
        bool slow;
        const float n = step_frame(sm, q, slow);
        if (t == L) {
          done = true;
          break;
        }
        mk = next_shift(lse, n, mk);
        float shift = n;
        if (slow) {
          refresh_p(sm, d, par, n);
          shift = 0.f;
        }
        const float acc = label_fanin<CAT, G>(sm.pcur + par * PC + ln.j * CAT, ln.e, p);
        float* row = store + (size_t)(t - t0) * SW;
        if (ln.leader) {
          const float g = label_log(acc, ln.tmax, shift, C, sm.Acur + par * C, n, trans, ln.c, false);
          if (checked_slot(ws, wslot, K))
            ring_put<KBT>(rl, d, wslot, make_float2((g - sf) + proj_d(ws, d, pj, b, t, ln.c),
                                                    (Frel + n) - (float)(si - Sb)));
          row[ln.c] = A;
          row[C + ln.c] = g;
        }
        if (tid == 0) {
          row[2 * C] = Frel;
          row[2 * C + 1] = Frel + n;
        }
        __syncwarp();
        Frel += n;
      }
      if (t > t_end) done = true;
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
  ln.init_dur(d, dur, false);
  ln.init_trans(d, trans, true, tmax2);
  __syncthreads();
  for (int i = tid; i < d.RL * C; i += blockDim.x) sm.ring[i] = make_float2(NEG_INF, 0.f);
  __syncthreads();
  double G0 = 0.0;
  float Grel = 0.f;
  int Sb;
  if (last) {
    for (int c = tid; c < C; c += blockDim.x) {
      const size_t o = ((size_t)b * d.Tstride + L) * C + c;
      ring_put<KBT>(sm.ring + (size_t)c * d.RL, d, L % K, make_float2(ws.sfrac[o], 0.f));
    }
    Sb = ws.sint[((size_t)b * d.Tstride + L) * C + ln.cc];
    for (int c = tid; c < C; c += blockDim.x) sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + L) * C + c];
  } else {
    const float2* ck = ws.bck + seg * K * C;
    for (int idx = tid; idx < K * C; idx += blockDim.x) {
      const int i = idx / C, c = idx % C;
      if (t1 + i <= L) ring_put<KBT>(sm.ring + (size_t)c * d.RL, d, (t1 + i) % K, ck[idx]);
    }
    Sb = ws.sint[((size_t)b * d.Tstride + t1) * C + ln.cc];
    for (int c = tid; c < C; c += blockDim.x) sm.Sbase[c] = ws.sint[((size_t)b * d.Tstride + t1) * C + c];
    G0 = ws.bcf[seg];
  }
  // this CTA's float64 partials start at zero (each thread its own entries)
  float accd[KBT];
  float acct[CAT];
#pragma unroll
  for (int i = 0; i < KBT; ++i) {
    accd[i] = 0.f;
    const int k = ln.k_of(ln.widx(i), false);
    if (ln.act && k <= K) ws.pgd[(seg * K + (k - 1)) * C + ln.c] = 0.0;
  }
#pragma unroll
  for (int i = 0; i < CAT; ++i) {
    acct[i] = 0.f;
    const int x = ln.j * CAT + i;
    if (ln.act && x < C) ws.pgt[(seg * C + ln.c) * C + x] = 0.0;
  }
  const double Xc = F0 + G0 - logz2;
  double accmu = 0.0, vsum = 0.0;  // leader of label c: suffix sum of (start - end) marginals
  __syncthreads();
  tile_start(sm, d, ws, b, ts, t1 - 1, t0, t1 - 1, -1);
  int nflush = 0;
  int wslot = t1 % K;
  int base = ln.base_down(t1 - 1, K);
  float mk = 0.f;
  int cur = -1, s = t1 - 1;
  while (s >= t0) {
    const int ti = s / TS;
    if (ti != cur) {
      if (!tile_enter(sm, d, ws, b, ts, ti)) {
        if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
        tile_drain(sm, ts);
        return;
      }
      cur = ti;
    }
    const int s_stop = max(t0, ti * TS);
    const size_t off = tile_row_off(s, C);
    const int32_t* ri = sm.tint + off;
    const float* rf = sm.tfrac + off;
    for (; s >= s_stop; --s, ri -= C, rf -= C) {
      if (s < t1 - 1) base = (base == 0) ? K - 1 : base - 1;
      wslot = (wslot == 0) ? K - 1 : wslot - 1;
      par = s & 1;
      q = mod3_next(q);
      const float* row = store + (size_t)(s - t0) * SW;
      const int si = ri[ln.cc];
      const float sf = rf[ln.cc];
      float ksum;
      const float lse = k_fanin<KBT, G>(rl + checked_base(ws, base, K),
                                        ln.j, -(float)(si - Sb) - Grel, ln.d, mk, ksum, e, ln.act);
      const float Bt = (lse == NEG_INF) ? NEG_INF : (lse - sf) + proj_d(ws, d, pj, b, s, ln.cc);
      float St = 0.f;
      if (ln.leader) {
        const float Xs = (float)(Xc + (double)row[2 * C + 1] + (double)Grel);
        St = (Bt == NEG_INF) ? 0.f : ex2(row[C + ln.c] + Bt + Xs);
        sm.Acur[par * C + ln.c] = Bt;
        sm.pcur[par * PC + ln.c] = ex2(Bt);
        if (start_marg) start_marg[((size_t)b * (d.T + 1) + s) * C + ln.c] = St;
        if (s == 0) sm.tmp[ln.c] = St;  // segment 0's normaliser: sum_c St[0, c]
      }
      warp_max_to_shared(&sm.maxslot[q], ln.leader ? f2ord(Bt) : INT_MIN);
      {
        const float Stg = __shfl_sync(FULL_MASK, St, (tid & 31) & ~(G - 1));
        const float coef = (ksum > 0.f) ? gbf * Stg / ksum : 0.f;
#pragma unroll
        for (int i = 0; i < KBT; ++i) accd[i] = fmaf(coef, e[i], accd[i]);
        if (seg_marg && ln.act) {
          // P([s, s+k), c) = start marginal x normalised k term (not scaled
          // by g: a marginal); rescaled with the rest below
          const float cs = (ksum > 0.f) ? Stg / ksum : 0.f;
          float* const row = seg_marg + ((size_t)b * d.T + s) * K * C + ln.c;
#pragma unroll
          for (int i = 0; i < KBT; ++i) {
            const int k = ln.k_of(ln.widx(i), false);
            if (k <= K && s + k <= L) row[(size_t)(k - 1) * C] = cs * e[i];
          }
        }
      }
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, q, slow);
      mk = next_shift(lse, n, mk);
      float E = 0.f;
      if (s >= 1) {
        float shift = n;
        if (slow) {
          refresh_p(sm, d, par, n);
          shift = 0.f;
        }
        const float acc = label_fanin<CAT, G>(sm.pcur + par * PC + ln.j * CAT, ln.e, p);
        if (ln.leader) {
          const float g = label_log(acc, ln.tmax, shift, C, sm.Acur + par * C, n, trans, ln.c, true);
          if (checked_slot(ws, wslot, K))
            ring_put<KBT>(rl, d, wslot, make_float2(g + sf, (Grel + n) + (float)(si - Sb)));
          const float Ys = (float)(Xc + (double)row[2 * C] + (double)(Grel + n));
          E = (g == NEG_INF || row[ln.c] == NEG_INF) ? 0.f : ex2(row[ln.c] + g + Ys);
          if (end_marg) end_marg[((size_t)b * (d.T + 1) + s) * C + ln.c] = E;
        }
        // transition posterior = coef * p * e; the constant e is applied at flush
        const float Eg = __shfl_sync(FULL_MASK, E, (tid & 31) & ~(G - 1));
        const float coef = (acc > 0.f) ? gbf * Eg / acc : 0.f;
#pragma unroll
        for (int i = 0; i < CAT; ++i) acct[i] = fmaf(coef, p[i], acct[i]);
        __syncwarp();
      } else if (ln.leader && end_marg) {
        end_marg[((size_t)b * (d.T + 1)) * C + ln.c] = 0.f;
      }
      if (ln.leader) {
        // position s: v = sum of (start - end) marginals strictly after it in the segment
        const float v = (float)accmu;
        grad_em[((size_t)b * d.T + s) * C + ln.c] = v;
        vsum += (double)v;
        accmu += (double)St - (double)E;
      }
      Grel += n;
      if (++nflush == FLUSH_EVERY || s == t0) {
        nflush = 0;
        if (ln.act) {
#pragma unroll
          for (int i = 0; i < KBT; ++i) {
            const int k = ln.k_of(ln.widx(i), false);
            if (k <= K) ws.pgd[(seg * K + (k - 1)) * C + ln.c] += (double)accd[i];
            accd[i] = 0.f;
          }
#pragma unroll
          for (int i = 0; i < CAT; ++i) {
            const int x = ln.j * CAT + i;
            if (x < C) ws.pgt[(seg * C + ln.c) * C + x] += (double)(acct[i] * ln.e[i]);
            acct[i] = 0.f;
          }
        }
      }
    }
  }
  // ---- the segment's own normaliser: r = Z_provisional / Z_j
  __syncthreads();
  if (j == 0) {
    // position 0 is covered by the segments starting at 0: Z_0 / Z_prov = sum_c St[0, c]
    if (tid < 32) {
      float tot = 0.f;
      for (int c = tid; c < C; c += 32) tot += sm.tmp[c];
      tot = group_sum(tot, 32);
      __syncwarp();
      for (int c = tid; c < C; c += 32) sm.tmp[c] = 0.f;  // nothing before position 0
      if (tid == 0) s_r = (tot > 0.f) ? 1.f / tot : 1.f;
    }
  } else {
    const double lzj = segment_cut(sm, d, ws, b, j, L, G0, dur, &s_lz);
    if (tid == 0) s_r = ex2((float)(logz2 - lzj));
  }
  __syncthreads();
  const float rs = s_r;
  // rescale what the walk wrote: boundary rows [t0, t1) (and the end
  // marginal at L), the suffix sums v, the count partials
  for (int idx = tid; idx < (t1 - t0) * C; idx += blockDim.x) {
    const int u = t0 + idx / C, c = idx % C;
    const size_t ob = ((size_t)b * (d.T + 1) + u) * C + c;
    if (start_marg) start_marg[ob] *= rs;
    if (end_marg) end_marg[ob] *= rs;
    grad_em[((size_t)b * d.T + u) * C + c] *= rs;
  }
  if (last && end_marg)
    for (int c = tid; c < C; c += blockDim.x) end_marg[((size_t)b * (d.T + 1) + L) * C + c] *= rs;
  for (int idx = tid; idx < K * C; idx += blockDim.x) ws.pgd[seg * K * C + idx] *= (double)rs;
  if (seg_marg)
    for (size_t idx = tid; idx < (size_t)(t1 - t0) * K * C; idx += blockDim.x)
      seg_marg[((size_t)b * d.T + t0) * K * C + idx] *= rs;
  for (int idx = tid; idx < C * C; idx += blockDim.x) ws.pgt[seg * C * C + idx] *= (double)rs;
  if (ln.leader) {
    ws.segT[seg * C + ln.c] = (double)sm.tmp[ln.c] + (double)rs * accmu;  // mu[t0 - 1] + total
    ws.segV[seg * C + ln.c] = (double)rs * vsum;
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

#ifdef SEMICRF_BOUNDS_CHECK
// One guarded store whose index is one past a 32-entry shared array: the
// check records SITE_SELFTEST and skips the store (debug build only).
__global__ void selftest_bounds_kernel(int* status, int idx) {
  __shared__ int buf[32];
  buf[threadIdx.x & 31] = 0;
  __syncthreads();
  if (threadIdx.x == 0 && SEMICRF_INB(status, idx >= 0 && idx < 32, ring::SITE_SELFTEST))
    buf[idx] = 1;
  __syncthreads();
  if (threadIdx.x == 0 && buf[0] == 12345) set_status(status, 0x7fffffff);  // keeps buf live
}
#endif

// ----------------------------------------------------------------------------- launchers
bool shape_supported(int KBT, int CAT, int G, int LB) {
#define SEMICRF_SHAPE_OK(a, b, g, lb) \
  if (KBT == a && CAT == b && G == g && LB == lb) return true;
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

namespace {

// Long durations have no log-domain kernel: a ring the exponential-domain
// kernel declined (mode 2: a score outside its exponent range) is reported
// as SEMICRF_ERR_UNSUPPORTED in the status word and its log Z is NaN.
__global__ void declined_chain_kernel(Dims d, WsPtrs ws, double* __restrict__ logZ_out,
                                      int n_alpha) {
  const bool up = (int)blockIdx.x < n_alpha;
  const int b = up ? blockIdx.x : blockIdx.x - n_alpha;
  if (threadIdx.x != 0 || !ws.mode || ws.mode[(up ? 0 : d.B) + b] != 2) return;
  set_status(ws.status, 2);  // SEMICRF_ERR_UNSUPPORTED
  const double nan = __longlong_as_double(0x7ff8000000000000ll);
  if (up) {
    if (logZ_out) logZ_out[b] = nan;
    ws.logz2[b] = nan;
  } else {
    ws.logz2b[b] = nan;
  }
}

// ... and its posteriors are zero: the per-segment partials, the emission
// gradient's suffix sums and the boundary marginals of the declined
// sequences (every other sequence took the posterior pass).
__global__ void declined_segment_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                                        float* __restrict__ grad_em, float* __restrict__ start_marg,
                                        float* __restrict__ end_marg, float* __restrict__ seg_marg) {
  const int j = blockIdx.x, b = blockIdx.y, C = d.C, K = d.K;
  const int L = lengths[b];
  if (L <= 0 || L > d.T || posterior_from_kept(ws, d, b)) return;
  const int t0 = j * d.delta;
  if (t0 >= L) return;
  const int t1 = min(t0 + d.delta, L);
  const size_t seg = (size_t)b * d.nck + j;
  for (int i = threadIdx.x; i < K * C; i += blockDim.x) ws.pgd[seg * K * C + i] = 0.0;
  for (int i = threadIdx.x; i < C * C; i += blockDim.x) ws.pgt[seg * C * C + i] = 0.0;
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    ws.segT[seg * C + i] = 0.0;
    ws.segV[seg * C + i] = 0.0;
  }
  const int t_end = (t1 == L) ? L + 1 : t1;  // the last segment also clears boundary L
  for (int i = threadIdx.x; i < (t1 - t0) * C; i += blockDim.x)
    grad_em[((size_t)b * d.T + t0) * C + i] = 0.f;
  for (int i = threadIdx.x; i < (t_end - t0) * C; i += blockDim.x) {
    const size_t ob = ((size_t)b * (d.T + 1) + t0) * C + i;
    if (start_marg) start_marg[ob] = 0.f;
    if (end_marg) end_marg[ob] = 0.f;
  }
  if (seg_marg)
    for (size_t i = threadIdx.x; i < (size_t)(t1 - t0) * K * C; i += blockDim.x)
      seg_marg[((size_t)b * d.T + t0) * K * C + i] = 0.f;
}

}  // namespace

cudaError_t launch_chain(const Dims& d, const WsPtrs& ws, const int32_t* lengths, const float* trans,
                         const float* dur, double* logZ_out, int n_alpha, int n_beta,
                         cudaStream_t st) {
  if (d.KBT == 0) {  // long durations: no log-domain kernel
    if (n_alpha + n_beta > 0)
      declined_chain_kernel<<<n_alpha + n_beta, 32, 0, st>>>(d, ws, logZ_out, n_alpha);
    return cudaGetLastError();
  }
  const size_t sm = recursion_smem_bytes(d, false);
#define SEMICRF_LAUNCH_CHAIN(a, b, g, lb)                                                    \
  if (d.KBT == a && d.CAT == b && d.GB == g && d.LB == lb) {                                 \
    const cudaError_t e = allow_smem(chain_kernel<a, b, g, lb>, sm);                         \
    if (e != cudaSuccess) return e;                                                          \
    chain_kernel<a, b, g, lb><<<n_alpha + n_beta, d.NT, sm, st>>>(d, ws, lengths, trans, dur, \
                                                                  logZ_out, n_alpha);        \
    return cudaGetLastError();                                                               \
  }
  SEMICRF_FOR_EACH_SHAPE(SEMICRF_LAUNCH_CHAIN)
#undef SEMICRF_LAUNCH_CHAIN
  return cudaErrorInvalidConfiguration;
}

cudaError_t launch_segment(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                           const float* trans, const float* dur, const double* grad_logZ,
                           float* grad_em, float* start_marg, float* end_marg, cudaStream_t st,
                           float* seg_marg) {
  if (d.KBT == 0) {  // long durations: zero the declined sequences' posteriors
    declined_segment_kernel<<<dim3(d.nck, d.B), 256, 0, st>>>(d, ws, lengths, grad_em, start_marg,
                                                               end_marg, seg_marg);
    return cudaGetLastError();
  }
  const size_t sm = recursion_smem_bytes(d, d.store_smem != 0);
#define SEMICRF_LAUNCH_SEG(a, b, g, lb)                                                      \
  if (d.KBT == a && d.CAT == b && d.GB == g && d.LB == lb) {                                 \
    const cudaError_t e = allow_smem(segment_kernel<a, b, g, lb>, sm);                       \
    if (e != cudaSuccess) return e;                                                          \
    segment_kernel<a, b, g, lb><<<dim3(d.nck, d.B), d.NT, sm, st>>>(                         \
        d, ws, lengths, trans, dur, grad_logZ, grad_em, start_marg, end_marg, seg_marg);     \
    return cudaGetLastError();                                                               \
  }
  SEMICRF_FOR_EACH_SHAPE(SEMICRF_LAUNCH_SEG)
#undef SEMICRF_LAUNCH_SEG
  return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
