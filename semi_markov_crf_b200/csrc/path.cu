// path.cu -- score of a given segmentation and its gradient, for the
// training loss.
//
// "Streaming Structured Inference with Flash-SemiCRF": the model of explainer
// section 1 ("Problem Statement") scores a segmentation as the sum over its
// segments [s, t) with label c of content(s, t, c) + dur[t-s-1, c], plus
// trans[c', c] between consecutive segments, with the centred emissions of
// section 2 ("Emission Baseline Centering").  Section 4 ("Results and
// Benchmarks", Correctness) trains the model to the usual CRF loss, the
// negative log-likelihood of the gold segmentation, log Z - score(gold).  Its
// gradient is the gradient of log Z (the backward pass) minus the gradient of
// the gold score, which is a count:
//   d score / d em[u, c]     = [y_u = c] - n_c / L   (n_c positions labelled c;
//                                                    the second term through
//                                                    the centring mean)
//   d score / d trans[c', c] = number of c' -> c transitions on the path
//   d score / d dur[k-1, c]  = number of label-c segments of length k
//
// The path comes as two per-position arrays, the form the decoder writes:
// labels[b, u] (int32) and seg_start[b, u] (1 where a segment starts).
//
// Three passes, each coalesced over positions:
//   path_terms_kernel  one CTA per (chunk of PATH_ROWS positions, sequence):
//                      the chunk's emission column sums (for nu), its gold
//                      emission, duration and transition terms, its label
//                      counts, and the gold duration / transition counts,
//                      added to per-sequence int32 tables by integer atomics
//                      (exact, so their order does not matter);
//   path_final_kernel  one CTA per sequence: nu, the centred score, n_c / L;
//   path_grad_*        grad += w_b * d score_b / d x for the emissions and
//                      for the transition / duration tables (summed over b in
//                      a fixed order).
// Every floating-point sum runs in float64 in a fixed order.
#include "kernels.cuh"

namespace semicrf {

namespace {

constexpr int PT_THREADS = 256;

// Malformed-path bits (any of them makes the score NaN).
constexpr int PB_START = 1;   // no segment starts at position 0
constexpr int PB_LABEL = 2;   // a label outside [0, C)
constexpr int PB_CHANGE = 4;  // a label that changes inside a segment
constexpr int PB_LONG = 8;    // a segment longer than K
constexpr int PB_LEN = 16;    // the sequence length is outside [0, T]

__device__ __forceinline__ double block_sum_fixed(double v, double* red) {
  // Fixed-order block reduction (PT_THREADS threads): warp tree, then warp 0.
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < PT_THREADS / 32; ++i) s += red[i];
  return s;  // valid in thread 0
}

}  // namespace

__global__ void __launch_bounds__(PT_THREADS) path_terms_kernel(
    const float* __restrict__ em, const int32_t* __restrict__ lengths,
    const float* __restrict__ trans, const float* __restrict__ dur,
    const int32_t* __restrict__ labels, const uint8_t* __restrict__ seg_start, Dims d,
    WsPtrs ws, unsigned center) {
  const int b = blockIdx.y, j = blockIdx.x;
  const int C = d.C, K = d.K, T = d.T;
  int L = lengths[b];
  if (L < 0 || L > T) {
    if (j == 0 && threadIdx.x == 0) {
      set_status(ws.status, ST_BAD_LENGTH);
      atomicOr(ws.pbad + b, PB_LEN);
    }
    return;
  }
  const int u0 = j * PATH_ROWS;
  if (u0 >= L) return;
  const int u1 = min(u0 + PATH_ROWS, L);

  __shared__ double part[PT_THREADS];
  __shared__ double red[PT_THREADS / 32];
  __shared__ int cnt[C_MAX];
  for (int c = threadIdx.x; c < C; c += PT_THREADS) cnt[c] = 0;

  const float* eb = em + (size_t)b * T * C;
  const int32_t* yb = labels + (size_t)b * T;
  const uint8_t* sb = seg_start + (size_t)b * T;

  // Emission column sums of the chunk: thread (g, c) sums rows u0+g, u0+g+G, ...
  if (center) {
    const int G = PT_THREADS / C;
    const int g = threadIdx.x / C, c = threadIdx.x % C;
    double acc = 0.0;
    if (g < G)
      for (int u = u0 + g; u < u1; u += G) acc += (double)eb[(size_t)u * C + c];
    part[threadIdx.x] = acc;
  }
  __syncthreads();  // part[] ready, cnt[] zeroed
  if (center && threadIdx.x < C) {
    const int G = PT_THREADS / C;
    double s = 0.0;
    for (int g = 0; g < G; ++g) s += part[g * C + threadIdx.x];
    ws.psum[((size_t)b * d.npch + j) * C + threadIdx.x] = s;
  }

  // Gold terms, one position per thread and pass.
  int* cnt_t = ws.pcnt + (size_t)b * (C * C + K * C);
  int* cnt_d = cnt_t + C * C;
  double acc = 0.0;
  int bad = 0;
  for (int u = u0 + threadIdx.x; u < u1; u += PT_THREADS) {
    const int y = yb[u];
    const bool st = sb[u] != 0;
    if (y < 0 || y >= C) {
      bad |= PB_LABEL;
      continue;
    }
    if (u == 0 && !st) bad |= PB_START;
    if (u > 0 && !st && yb[u - 1] != y) bad |= PB_CHANGE;
    acc += (double)eb[(size_t)u * C + y];
    atomicAdd(&cnt[y], 1);
    if (st) {
      // Duration: distance to the next start, or to the end of the sequence.
      int k = 0;
      for (int q = 1; q <= K; ++q) {
        if (u + q >= L || sb[u + q]) {
          k = q;
          break;
        }
      }
      if (k == 0) {
        bad |= PB_LONG;
        continue;
      }
      acc += (double)dur[(k - 1) * C + y];
      atomicAdd(cnt_d + (k - 1) * C + y, 1);
      if (u > 0) {
        const int yp = yb[u - 1];
        if (yp >= 0 && yp < C) {
          acc += (double)trans[yp * C + y];
          atomicAdd(cnt_t + yp * C + y, 1);
        }
      }
    }
  }
  if (bad) atomicOr(ws.pbad + b, bad);
  const double tot = block_sum_fixed(acc, red);
  __syncthreads();  // cnt[] complete
  if (threadIdx.x == 0) ws.pscr[(size_t)b * d.npch + j] = tot;
  for (int c = threadIdx.x; c < C; c += PT_THREADS)
    ws.plab[((size_t)b * d.npch + j) * C + c] = cnt[c];
}

// One CTA per sequence: nu[c] = (sum of the chunk column sums) / L, the score
// sum_chunks(partial) - sum_c n_c nu[c], the fractions n_c / L for the
// emission gradient and the weight w_b = +-grad_score[b] (0 for a malformed
// path).
__global__ void __launch_bounds__(C_MAX) path_final_kernel(const int32_t* __restrict__ lengths,
                                                           Dims d, WsPtrs ws, unsigned center,
                                                           const double* __restrict__ grad_score,
                                                           int negate, double* __restrict__ score) {
  const int b = blockIdx.x, C = d.C;
  __shared__ double corr[C_MAX];
  const int bad = ws.pbad[b];
  int L = lengths[b];
  if (L < 0 || L > d.T) L = 0;
  const int nch = (L + PATH_ROWS - 1) / PATH_ROWS;
  const int c = threadIdx.x;
  double cr = 0.0;
  if (c < C) {
    double es = 0.0;
    long long n = 0;
    for (int j = 0; j < nch; ++j) {
      const size_t o = ((size_t)b * d.npch + j) * C + c;
      if (center) es += ws.psum[o];
      n += ws.plab[o];
    }
    const double nu = (center && L > 0) ? es / (double)L : 0.0;
    cr = (double)n * nu;
    ws.pfr[(size_t)b * C + c] = (center && L > 0) ? (double)n / (double)L : 0.0;
  }
  corr[c] = cr;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int j = 0; j < nch; ++j) s += ws.pscr[(size_t)b * d.npch + j];
    for (int cc = 0; cc < C; ++cc) s -= corr[cc];
    double g = grad_score ? grad_score[b] : 1.0;
    if (negate) g = -g;
    if (bad) {
      if (score) score[b] = __longlong_as_double(0x7ff8000000000000ll);  // NaN
      ws.pw[b] = 0.0;
    } else {
      if (score) score[b] = s;
      ws.pw[b] = g;
    }
  }
}

// grad_em[b, u, c] += w_b * ([y_u = c] - n_c / L) for u < L_b.
__global__ void __launch_bounds__(PT_THREADS) path_grad_em_kernel(
    const int32_t* __restrict__ lengths, const int32_t* __restrict__ labels, Dims d, WsPtrs ws,
    float* __restrict__ grad_em) {
  const int b = blockIdx.y, C = d.C;
  const double w = ws.pw[b];
  if (w == 0.0) return;
  int L = lengths[b];
  if (L < 0 || L > d.T) return;
  const size_t n = (size_t)L * C;
  const int32_t* yb = labels + (size_t)b * d.T;
  const double* fr = ws.pfr + (size_t)b * C;
  float* gb = grad_em + (size_t)b * d.T * C;
  for (size_t i = (size_t)blockIdx.x * PT_THREADS + threadIdx.x; i < n;
       i += (size_t)gridDim.x * PT_THREADS) {
    const int u = (int)(i / C), c = (int)(i - (size_t)u * C);
    const double v = ((yb[u] == c) ? 1.0 : 0.0) - fr[c];
    gb[i] += (float)(w * v);
  }
}

// grad_trans[c', c] += sum_b w_b * (#c' -> c transitions of path b) and
// grad_dur[k-1, c] += sum_b w_b * (#label-c segments of length k), b in order.
__global__ void __launch_bounds__(PT_THREADS) path_grad_param_kernel(Dims d, WsPtrs ws,
                                                                     float* __restrict__ grad_trans,
                                                                     float* __restrict__ grad_dur) {
  const int C = d.C, K = d.K;
  const int nt = C * C, nall = C * C + K * C;
  const int i = blockIdx.x * PT_THREADS + threadIdx.x;
  if (i >= nall) return;
  float* out = (i < nt) ? grad_trans : grad_dur;
  if (!out) return;
  double s = 0.0;
  for (int b = 0; b < d.B; ++b) {
    const int v = ws.pcnt[(size_t)b * nall + i];
    if (v) s += ws.pw[b] * (double)v;
  }
  out[i < nt ? i : i - nt] += (float)s;
}

cudaError_t launch_path_terms(const Dims& d, const WsPtrs& ws, const float* em,
                              const int32_t* lengths, const float* trans, const float* dur,
                              const int32_t* labels, const uint8_t* seg_start, unsigned center,
                              cudaStream_t st) {
  path_terms_kernel<<<dim3(d.npch, d.B), PT_THREADS, 0, st>>>(em, lengths, trans, dur, labels,
                                                               seg_start, d, ws, center);
  return cudaGetLastError();
}

cudaError_t launch_path_final(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                              unsigned center, const double* grad_score, int negate,
                              double* score, cudaStream_t st) {
  path_final_kernel<<<d.B, C_MAX, 0, st>>>(lengths, d, ws, center, grad_score, negate, score);
  return cudaGetLastError();
}

cudaError_t launch_path_grad_em(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                const int32_t* labels, float* grad_em, int sms, cudaStream_t st) {
  // At most about four waves of 2048 threads per SM over the whole batch.
  const size_t per_seq_full = ((size_t)d.T * d.C + PT_THREADS - 1) / PT_THREADS;
  const size_t cap = (size_t)std::max(1, 4 * 8 * sms / std::max(d.B, 1));
  const int per_seq = (int)std::max<size_t>(1, std::min(per_seq_full, cap));
  path_grad_em_kernel<<<dim3(per_seq, d.B), PT_THREADS, 0, st>>>(lengths, labels, d, ws, grad_em);
  return cudaGetLastError();
}

cudaError_t launch_path_grad_param(const Dims& d, const WsPtrs& ws, float* grad_trans,
                                   float* grad_dur, cudaStream_t st) {
  const int nall = d.C * d.C + d.K * d.C;
  path_grad_param_kernel<<<(nall + PT_THREADS - 1) / PT_THREADS, PT_THREADS, 0, st>>>(
      d, ws, grad_trans, grad_dur);
  return cudaGetLastError();
}

}  // namespace semicrf
