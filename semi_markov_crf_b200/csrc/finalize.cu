// finalize.cu -- step 3 epilogue: position marginals, the emission gradient
// through centering, and the fixed-order reduction of per-segment partials.
//
// The checkpoint segments leave, for every position u of segment j, the
// suffix sum v[u, c] = sum_{u < s < t1_j} (start_marg[s,c] - end_marg[s,c]) in
// the grad_em buffer, plus per segment P_j[c] = mu[t0_j - 1, c] + the total
// of (start - end) over the segment (mu[t0_j - 1] from the segment's cut
// normaliser, 0 for j = 0) and V_j[c] = sum_u v[u, c].  Then
//   pos_marg[u, c] = sum_{s <= u} (start_marg[s,c] - end_marg[s,c])
//                  = P_j[c] - v[u, c]
// (a position lies in a label-c segment iff one started at or before it and
// none of those ended at or before it); taking the carry from the cut rather
// than summing earlier segments' totals keeps every segment independent of
// the others' rounding.  With centering the emission
// gradient is g_b * (pos_marg[u,c] - mean_v pos_marg[v,c]) (the Jacobian of
// subtracting the per-label mean; "Emission Baseline Centering", explainer
// section 2).
#include <algorithm>

#include "kernels.cuh"

namespace semicrf {

constexpr int FIN_ROWS = 64;

__global__ void __launch_bounds__(256)
    finalize_positions_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                              const double* __restrict__ grad_logZ, unsigned center,
                              float* __restrict__ grad_em, float* __restrict__ pos_marg,
                              float* __restrict__ start_marg, float* __restrict__ end_marg) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* mean = reinterpret_cast<double*>(smem_raw);  // [C]
  double* pinc = mean + d.C;                            // [nj][C]
  const int C = d.C, T = d.T;
  const int b = blockIdx.y;
  const int u0 = blockIdx.x * FIN_ROWS;
  const int u1 = min(u0 + FIN_ROWS, T);
  int L = lengths[b];
  const bool bad = (L < 0 || L > T);
  if (bad) L = 0;
  const double gb = grad_logZ ? grad_logZ[b] : 1.0;
  const int delta = d.delta;
  const int j_lo = u0 / delta;
  const int j_hi = (max(u0, min(u1, L) - 1)) / delta;
  if (threadIdx.x < C && L > 0) {
    const int c = threadIdx.x;
    const int nseg = (L + delta - 1) / delta;
    // segT: mu[t0 - 1] + segment total (segment_kernel, its own carry from
    // the cut) or the plain segment total (posterior_kernel: running sum)
    const bool cum = posterior_from_kept(ws, d, b);
    double run = 0.0, msum = 0.0;
    for (int j = 0; j < nseg; ++j) {
      const size_t o = ((size_t)b * d.nck + j) * C + c;
      run = cum ? run + ws.segT[o] : ws.segT[o];
      const int len = min((j + 1) * delta, L) - j * delta;
      msum += (double)len * run - ws.segV[o];
      if (j >= j_lo && j <= j_hi) pinc[(j - j_lo) * C + c] = run;
    }
    mean[c] = center ? msum / (double)L : 0.0;
  }
  __syncthreads();
  // FU entries per thread at a time, their loads issued before the stores
  // (grad_em is read and written here: otherwise each load would wait for
  // the store before it)
  constexpr int FU = 4;
  const int n = (u1 - u0) * C;
  const size_t ob = ((size_t)b * T + u0) * C;
  for (int i0 = threadIdx.x; i0 < n; i0 += FU * blockDim.x) {
    float v[FU];
#pragma unroll
    for (int q = 0; q < FU; ++q) {
      const int idx = i0 + q * blockDim.x;
      v[q] = (idx < n && u0 + idx / C < L) ? grad_em[ob + idx] : 0.f;
    }
#pragma unroll
    for (int q = 0; q < FU; ++q) {
      const int idx = i0 + q * blockDim.x;
      if (idx >= n) break;
      const int u = u0 + idx / C, c = idx % C;
      if (u < L) {
        const int j = u / delta;
        const double mu = pinc[(j - j_lo) * C + c] - (double)v[q];
        grad_em[ob + idx] = (float)(gb * (mu - mean[c]));
        if (pos_marg) pos_marg[ob + idx] = (float)mu;
      } else {
        grad_em[ob + idx] = 0.f;
        if (pos_marg) pos_marg[ob + idx] = 0.f;
      }
    }
  }
  // boundary rows t in [u0, u1) (and t = T for the last block) past the length
  const int tb1 = (u1 == T) ? T + 1 : u1;
  for (int idx = threadIdx.x; idx < (tb1 - u0) * C; idx += blockDim.x) {
    const int t = u0 + idx / C, c = idx % C;
    if (t > L || L == 0) {
      const size_t o = ((size_t)b * (T + 1) + t) * C + c;
      if (start_marg) start_marg[o] = 0.f;
      if (end_marg) end_marg[o] = 0.f;
    }
  }
}

// grad_trans (entries 0..C*C-1) and grad_dur (entries C*C..C*C+K*C-1):
// float64 sums of the per-segment partials.  A block takes RP_E consecutive
// entries; its RP_S thread rows split the (sequence, segment) list, strided,
// and the rows' sums are added in row order: a fixed order, so the result
// does not depend on scheduling.
__global__ void __launch_bounds__(RP_E * RP_S)
    reduce_partials_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                           float* __restrict__ grad_trans, float* __restrict__ grad_dur) {
  __shared__ double part[RP_S][RP_E];
  const int C = d.C, K = d.K;
  const int ex = threadIdx.x % RP_E, sy = threadIdx.x / RP_E;
  const int e = blockIdx.x * RP_E + ex;
  const int nt = C * C, ne = nt + K * C;
  double acc = 0.0;
  if (e < ne) {
    const double* src = (e < nt) ? ws.pgt + e : ws.pgd + (e - nt);
    const size_t stride = (e < nt) ? (size_t)nt : (size_t)K * C;
    const int nrow = d.B * d.nck;
    for (int r = sy; r < nrow; r += RP_S) {
      const int b = r / d.nck, j = r - b * d.nck;
      const int L = lengths[b];
      if (L <= 0 || L > d.T || j * d.delta >= L) continue;
      acc += src[(size_t)r * stride];
    }
  }
  part[sy][ex] = acc;
  __syncthreads();
  if (sy == 0 && e < ne) {
    double t = 0.0;
    for (int q = 0; q < RP_S; ++q) t += part[q][ex];
    if (e < nt)
      grad_trans[e] = (float)t;
    else
      grad_dur[e - nt] = (float)t;
  }
}

// Gradients of g_b * log Z_b with respect to the boundary projections
// ("Streaming Structured Inference with Flash-SemiCRF", explainer section 2,
// "Boundary Projections"): log Z depends on P_start[b, u, c] through the
// segments that start at u with label c, and on P_end[b, u, c] through those
// that end after position u, so
//   grad_p_start[b, u, c] = g_b * start_marg[b, u, c]
//   grad_p_end[b, u, c]   = g_b * end_marg[b, u + 1, c]      (u < L_b; else 0).
__global__ void __launch_bounds__(256) proj_grad_kernel(Dims d, const int32_t* __restrict__ lengths,
                                                        const double* __restrict__ grad_logZ,
                                                        const float* __restrict__ start_marg,
                                                        const float* __restrict__ end_marg,
                                                        float* __restrict__ grad_p_start,
                                                        float* __restrict__ grad_p_end) {
  const int b = blockIdx.y, C = d.C, T = d.T;
  int L = lengths[b];
  if (L < 0 || L > T) L = 0;
  const float g = (float)(grad_logZ ? grad_logZ[b] : 1.0);
  const size_t n = (size_t)T * C;
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256) {
    const int u = (int)(i / C);
    const bool in = u < L;
    const size_t o = (size_t)b * n + i;
    const size_t m = (size_t)b * (T + 1) * C + i;  // row u of the [T+1] marginals
    if (grad_p_start) grad_p_start[o] = in ? g * start_marg[m] : 0.f;
    if (grad_p_end) grad_p_end[o] = in ? g * end_marg[m + C] : 0.f;
  }
}

cudaError_t launch_proj_grad(const Dims& d, const int32_t* lengths, const double* grad_logZ,
                             const float* start_marg, const float* end_marg, float* grad_p_start,
                             float* grad_p_end, cudaStream_t st) {
  if (d.T == 0 || d.B == 0) return cudaSuccess;
  const size_t n = (size_t)d.T * d.C;
  const int gx = (int)std::min<size_t>((n + 255) / 256, 1024);
  proj_grad_kernel<<<dim3(gx, d.B), 256, 0, st>>>(d, lengths, grad_logZ, start_marg, end_marg,
                                                 grad_p_start, grad_p_end);
  return cudaGetLastError();
}

}  // namespace semicrf
