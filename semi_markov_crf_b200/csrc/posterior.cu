// posterior.cu -- step 3's posteriors from the values the exponential-domain
// rings kept, with no serial walk.
//
// "Streaming Structured Inference with Flash-SemiCRF", explainer section 2
// (marginals and gradients of the streaming forward-backward).  When both
// rings of a sequence ran in the exponential domain (chain_exp.cu) they kept,
// for every boundary t and label c, relative to a per-boundary frame:
//   forward  pf[t] = 2^(alpha[t] - Pf_t),  af[t] = 2^(gamma[t] - Pf_t - M)
//   backward pb[t] = 2^(btil[t]  - Pb_t),  ab[t] = 2^(beta[t]  - Pb_t - M)
// (M = max trans2).  Every posterior is then a product of kept values:
//   start_marg[s, c] = 2^(gamma[s] + btil[s] - log2 Z)
//   end_marg[t, c]   = 2^(alpha[t] + beta[t] - log2 Z)
//   P([s, s+k), c)   = 2^(gamma[s] - S[s] + dur2[k-1] + S[s+k] + beta[s+k] - log2 Z)
//   P(c' -> c at s)  = 2^(alpha[s, c'] + trans2[c', c] + btil[s, c] - log2 Z)
// and they are computed in parallel over (boundary, label, duration or
// label pair).
//
// Normaliser.  The two rings' rounding drifts apart slowly (about 1e-7 per
// position), so the posteriors are not divided by either ring's log Z but by
// a local one: the cut identity (every segmentation has exactly one segment
// covering a position) evaluated from the kept values every GS positions --
// cut_grid_kernel -- and interpolated linearly in between.  At position 0
// the cut is the backward ring's log Z, at L - 1 the forward ring's.
#include "ring.cuh"

namespace semicrf {

using namespace ring;

namespace {

// kept values of direction dir (0 forward, 1 backward) of sequence b
__device__ __forceinline__ const float* kv_row(const WsPtrs& ws, const Dims& d, int b, int dir,
                                               int t) {
  return ws.kv + ((((size_t)b * 2 + dir) * (d.T + 1)) + t) * 2 * d.C;
}
__device__ __forceinline__ double kf_at(const WsPtrs& ws, const Dims& d, int b, int dir, int t) {
  return ws.kf[((size_t)b * 2 + dir) * (d.T + 1) + t];
}

// Grid position g of a sequence of length L (g <= G1 = (L-1)/GS: g*GS; the
// last one L - 1).  Returns -1 past the last.
__device__ __forceinline__ int grid_pos(const Dims& d, int L, int g) {
  const int G1 = (L - 1) / d.GS;
  if (g <= G1) return g * d.GS;
  return g == G1 + 1 ? L - 1 : -1;
}

// log2 Z at position u, interpolated between the grid values.
__device__ __forceinline__ double local_logz(const Dims& d, const double* nc, int L, int u) {
  const int G1 = (L - 1) / d.GS;
  const int g = min(u / d.GS, G1);
  const int u0 = g * d.GS, u1 = (g < G1) ? u0 + d.GS : L - 1;
  const double n0 = nc[g], n1 = nc[g + 1];
  return u1 > u0 ? n0 + (n1 - n0) * (double)(u - u0) / (double)(u1 - u0) : n0;
}

}  // namespace

// One CTA per (grid position, sequence): log2 of the cut at position u,
//   Z(u) = sum over segments [s, t) with s <= u < t, t - s <= K, and labels c of
//          2^(gamma[s, c] - S[s, c] + dur2[t-s-1, c] + S[t, c] + beta[t, c]),
// from the kept values; every large quantity (frames, prefix sums) enters as
// a difference from the reference R = Pf_u + Pb_{u+1} before float32 sees it.
__global__ void __launch_bounds__(256)
    cut_grid_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                    const float* __restrict__ trans, const float* __restrict__ dur) {
  __shared__ int aux[2];
  __shared__ float lab_M[128], lab_f[128];  // per label: shift, log2 share
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int C = d.C, K = d.K;
  const int L = lengths[b];
  if (L <= 0 || L > d.T) return;
  if (!posterior_from_kept(ws, d, b)) return;  // segment_kernel runs it
  const int u = grid_pos(d, L, g);
  if (u < 0) return;
  double* out = ws.ncut + (size_t)b * d.ngrid + g;
  if (u == 0) {
    if (tid == 0) *out = ws.logz2b[b];
    return;
  }
  if (u == L - 1) {
    if (tid == 0) *out = ws.logz2[b];
    return;
  }
  if (tid == 0) aux[0] = f2ord(NEG_INF);
  __syncthreads();
  float M;
  {
    float m = NEG_INF;
    for (int i = tid; i < C * C; i += blockDim.x) m = fmaxf(m, __ldg(trans + i) * l2e());
    warp_max_to_shared(&aux[0], f2ord(m));
    __syncthreads();
    M = ord2f(aux[0]);
  }
  const double Fu = kf_at(ws, d, b, 0, u), Gu = kf_at(ws, d, b, 1, u + 1);
  const int32_t* si = ws.sint + (size_t)b * d.Tstride * C;
  const float* sf = ws.sfrac + (size_t)b * d.Tstride * C;
  const int lane = tid & 31, nw = blockDim.x >> 5;
  for (int c = tid >> 5; c < C; c += nw) {
    // lanes over the start s = u - ia (ia < K), inner loop over the end t
    float zmax = NEG_INF, sum = 0.f;
    for (int pass = 0; pass < 2; ++pass) {
      const float Mz = (pass == 0) ? 0.f : ((zmax == NEG_INF) ? 0.f : ceilf(zmax));
      for (int ia = lane; ia < K; ia += 32) {
        const int s = u - ia;
        if (s < 0) break;
        const float a = kv_row(ws, d, b, 0, s)[C + c];
        if (!(a > 0.f)) continue;
        const float la = lg2(a) + (float)(kf_at(ws, d, b, 0, s) - Fu);
        const int sis = si[(size_t)s * C + c];
        const float sfs = sf[(size_t)s * C + c];
        const int tmax = min(s + K, L);
        for (int t = u + 1; t <= tmax; ++t) {
          const float bt = kv_row(ws, d, b, 1, t)[C + c];
          if (!(bt > 0.f)) continue;
          const float z = ((float)(si[(size_t)t * C + c] - sis) +
                           (la + (lg2(bt) + (float)(kf_at(ws, d, b, 1, t) - Gu)))) +
                          ((2.f * M + __ldg(dur + (size_t)(t - s - 1) * C + c) * l2e()) +
                           (sf[(size_t)t * C + c] - sfs));
          if (pass == 0) {
            zmax = fmaxf(zmax, z);
          } else {
            sum += ex2(z - Mz);
          }
        }
      }
      if (pass == 0) {
        zmax = group_max(zmax, 32);
      } else {
        sum = group_sum(sum, 32);
        if (lane == 0) {
          lab_M[c] = Mz;
          lab_f[c] = (sum > 0.f) ? lg2(sum) : NEG_INF;
        }
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    float Mz = NEG_INF;
    for (int c = lane; c < C; c += 32)
      if (lab_f[c] != NEG_INF) Mz = fmaxf(Mz, lab_M[c]);
    Mz = group_max(Mz, 32);
    if (Mz == NEG_INF) Mz = 0.f;
    float tot = 0.f;
    for (int c = lane; c < C; c += 32) tot += ex2((lab_M[c] - Mz) + lab_f[c]);
    tot = group_sum(tot, 32);
    if (lane == 0) *out = (Fu + Gu) + ((double)Mz + (double)(tot > 0.f ? lg2(tot) : NEG_INF));
  }
}


// One CTA per (checkpoint segment j, sequence b): every posterior whose start
// boundary lies in [t0, t1), written in the same per-segment layout as
// segment_kernel (suffix sums v in grad_em, per-segment totals, float64
// count partials), so finalize and the partial reduction are shared; here
// the per-segment total is the plain sum over the segment (finalize takes the
// running sum over segments), because the normaliser is continuous.
__global__ void __launch_bounds__(512)
    posterior_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                     const float* __restrict__ trans, const float* __restrict__ dur,
                     const double* __restrict__ grad_logZ, float* __restrict__ grad_em,
                     float* __restrict__ start_marg, float* __restrict__ end_marg) {
  extern __shared__ float fsh[];  // [delta + 1] per-boundary factor f_s
  __shared__ int aux[1];
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int C = d.C, K = d.K;
  const int L = lengths[b];
  if (L <= 0 || L > d.T) return;
  if (!posterior_from_kept(ws, d, b)) return;  // segment_kernel runs it
  const int t0 = j * d.delta;
  if (t0 >= L) return;
  const int t1 = min(t0 + d.delta, L);
  const bool last = (t1 == L);
  const size_t seg = (size_t)b * d.nck + j;
  const float gb = (float)(grad_logZ ? grad_logZ[b] : 1.0);
  if (tid == 0) aux[0] = f2ord(NEG_INF);
  __syncthreads();
  float M;
  {
    float m = NEG_INF;
    for (int i = tid; i < C * C; i += blockDim.x) m = fmaxf(m, __ldg(trans + i) * l2e());
    warp_max_to_shared(&aux[0], f2ord(m));
    __syncthreads();
    M = ord2f(aux[0]);
  }
  const float* pfr = kv_row(ws, d, b, 0, 0);  // row t: pfr + t*2C (p), + C (acc)
  const float* pbr = kv_row(ws, d, b, 1, 0);
  const double* kff = ws.kf + ((size_t)b * 2 + 0) * (d.T + 1);
  const double* kfb = ws.kf + ((size_t)b * 2 + 1) * (d.T + 1);
  const double* nc = ws.ncut + (size_t)b * d.ngrid;
  const int32_t* si = ws.sint + (size_t)b * d.Tstride * C;
  const float* sf = ws.sfrac + (size_t)b * d.Tstride * C;
  // f_s = 2^(Pf_s + Pb_s + M - log2 Z(s)), s in [t0, t1] (t1 = L: the end
  // marginal at L, normalised at position L - 1)
  const int n = t1 - t0;
  for (int s = t0 + tid; s <= t1; s += blockDim.x)
    fsh[s - t0] = ex2((float)(((kff[s] + kfb[s]) + (double)M) - local_logz(d, nc, L, min(s, L - 1))));
  __syncthreads();

  // start / end marginals, suffix sums v and the segment's totals (one
  // thread per label, walking the segment downwards)
  for (int c = tid; c < C; c += blockDim.x) {
    double acc = 0.0, vsum = 0.0;
    for (int s = t1 - 1; s >= t0; --s) {
      const float f = fsh[s - t0];
      const float St = pfr[(size_t)s * 2 * C + C + c] * pbr[(size_t)s * 2 * C + c] * f;
      const float E = pbr[(size_t)s * 2 * C + C + c] * pfr[(size_t)s * 2 * C + c] * f;
      const size_t ob = ((size_t)b * (d.T + 1) + s) * C + c;
      if (start_marg) start_marg[ob] = St;
      if (end_marg) end_marg[ob] = E;
      grad_em[((size_t)b * d.T + s) * C + c] = (float)acc;  // v[s]: after s
      vsum += (double)(float)acc;
      acc += (double)St - (double)E;
    }
    ws.segT[seg * C + c] = acc;
    ws.segV[seg * C + c] = vsum;
    if (last) {
      const size_t ob = ((size_t)b * (d.T + 1) + L) * C + c;
      if (end_marg)
        end_marg[ob] = pfr[(size_t)L * 2 * C + c] * pbr[(size_t)L * 2 * C + C + c] * fsh[n];
      if (start_marg) start_marg[ob] = 0.f;
    }
  }

  // duration counts: thread (k, c) sums P([s, s+k), c) over the segment's s
  for (int idx = tid; idx < K * C; idx += blockDim.x) {
    const int k = idx / C + 1, c = idx % C;
    const float dk = M + __ldg(dur + (size_t)(k - 1) * C + c) * l2e();
    float accd = 0.f;
    const int s_end = min(t1, L - k + 1);  // s + k <= L
    for (int s = t0; s < s_end; ++s) {
      const float a = pfr[(size_t)s * 2 * C + C + c];
      const float bt = pbr[(size_t)(s + k) * 2 * C + C + c];
      const float z = (float)(kfb[s + k] - kfb[s]) + (float)(si[(size_t)(s + k) * C + c] - si[(size_t)s * C + c]) +
                      (dk + (sf[(size_t)(s + k) * C + c] - sf[(size_t)s * C + c]));
      accd = fmaf(a * bt, fsh[s - t0] * ex2(z), accd);
    }
    ws.pgd[(seg * K + (k - 1)) * C + c] = (double)(gb * accd);
  }

  // transition counts: thread (c', c) sums P(c' -> c at s) over the
  // segment's boundaries s >= 1 (pf[0] = 0 takes care of s = 0)
  for (int idx = tid; idx < C * C; idx += blockDim.x) {
    const int c1 = idx / C, c = idx % C;
    float acct = 0.f;
    for (int s = t0; s < t1; ++s)
      acct = fmaf(pfr[(size_t)s * 2 * C + c1] * fsh[s - t0], pbr[(size_t)s * 2 * C + c], acct);
    const float w = ex2(__ldg(trans + (size_t)c1 * C + c) * l2e() - M);
    ws.pgt[(seg * C + c1) * C + c] = (double)(gb * acct * w);
  }
}

// Shared memory of posterior_kernel.
size_t posterior_smem_bytes(const Dims& d) { return ((size_t)d.delta + 1) * sizeof(float); }

}  // namespace semicrf
