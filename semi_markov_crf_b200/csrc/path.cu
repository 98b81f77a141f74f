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
// Two launches, each coalesced over positions:
//   path_terms_kernel  one CTA per (chunk of PATH_ROWS positions, sequence),
//                      one position per thread: the chunk's emission column
//                      sums (for nu), its gold emission, duration and
//                      transition terms and its label counts; the gold
//                      duration / transition counts go to per-sequence int32
//                      tables by integer atomics (exact, so their order does
//                      not matter).  The last CTA of a sequence to finish
//                      (a per-sequence counter) reduces the chunks in order:
//                      nu, the centred score, n_c / L and the weight w_b.
//   path_grad_kernel   grad += w_b * d score_b / d x: the emission gradient
//                      element by element, the transition / duration tables
//                      summed over b in a fixed order (the last CTAs).
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
    WsPtrs ws, unsigned center, const double* __restrict__ grad_score, int negate,
    double* __restrict__ score, const float* __restrict__ p_start,
    const float* __restrict__ p_end) {
  const int b = blockIdx.y, j = blockIdx.x, tid = threadIdx.x;
  const int C = d.C, K = d.K, T = d.T;
  const int L = lengths[b];
  const double g = (grad_score ? grad_score[b] : 1.0) * (negate ? -1.0 : 1.0);
  if (L <= 0 || L > T) {
    // Nothing to sum: chunk 0 alone reports the sequence.
    if (j == 0 && tid == 0) {
      const bool bad = L != 0;
      if (bad) set_status(ws.status, ST_BAD_LENGTH);
      if (score) score[b] = bad ? __longlong_as_double(0x7ff8000000000000ll) : 0.0;
      ws.pw[b] = bad ? 0.0 : g;
    }
    return;
  }
  const int u0 = j * PATH_ROWS;
  if (u0 >= L) return;
  const int u1 = min(u0 + PATH_ROWS, L);
  const int nchb = (L + PATH_ROWS - 1) / PATH_ROWS;

  __shared__ double part[PT_THREADS];
  __shared__ double red[PT_THREADS / 32];
  __shared__ int cnt[C_MAX];
  __shared__ unsigned char fl[PATH_ROWS + K_MAX];  // start flags of [u0, u0 + PATH_ROWS + K)
  __shared__ int last;

  const float* eb = em + (size_t)b * T * C;
  const int32_t* yb = labels + (size_t)b * T;
  const uint8_t* sb = seg_start + (size_t)b * T;

  for (int c = tid; c < C; c += PT_THREADS) cnt[c] = 0;
  const int nfl = min(PATH_ROWS + K, L - u0);
  for (int q = tid; q < nfl; q += PT_THREADS) fl[q] = sb[u0 + q];

  // Emission column sums of the chunk: thread (g, c) sums rows u0+g, u0+g+G, ...
  double es = 0.0;
  if (center) {
    const int G = PT_THREADS / C;
    const int gi = tid / C, c = tid - (tid / C) * C;
    if (gi < G) {
      const float* col = eb + c;
      // independent loads, many in flight: the chain is one add per row
#pragma unroll 16
      for (int u = u0 + gi; u < u1; u += G) es += (double)col[(size_t)u * C];
    }
  }
  part[tid] = es;

  // The gold terms of position u = u0 + tid.
  int* cnt_t = ws.pcnt + (size_t)b * (C * C + K * C);
  int* cnt_d = cnt_t + C * C;
  const int u = u0 + tid;
  double acc = 0.0;
  int bad = 0;
  int y = -1, yp = -1;
  if (u < u1) {
    y = yb[u];
    if (u > 0) yp = yb[u - 1];
  }
  __syncthreads();  // fl[], cnt[] and part[] ready
  if (u < u1) {
    const bool st = fl[tid] != 0;
    if (y < 0 || y >= C) {
      bad |= PB_LABEL;
    } else {
      if (u == 0 && !st) bad |= PB_START;
      if (u > 0 && !st && yp != y) bad |= PB_CHANGE;
      acc = (double)eb[(size_t)u * C + y];
      atomicAdd(&cnt[y], 1);
      // boundary projections: a segment's first and last positions
      if (p_start && st) acc += (double)p_start[((size_t)b * T + u) * C + y];
      if (p_end && (u + 1 >= L || fl[tid + 1])) acc += (double)p_end[((size_t)b * T + u) * C + y];
      if (st) {
        // Duration: distance to the next start, or to the end of the sequence.
        int k = 0;
        for (int q = 1; q <= K; ++q) {
          if (u + q >= L || fl[tid + q]) {
            k = q;
            break;
          }
        }
        if (k == 0) {
          bad |= PB_LONG;
        } else {
          acc += (double)dur[(k - 1) * C + y];
          atomicAdd(cnt_d + (k - 1) * C + y, 1);
          if (u > 0 && yp >= 0 && yp < C) {
            acc += (double)trans[yp * C + y];
            atomicAdd(cnt_t + yp * C + y, 1);
          }
        }
      }
    }
  }
  if (bad) atomicOr(ws.pbad + b, bad);
  if (center && tid < C) {
    const int G = PT_THREADS / C;
    double s = 0.0;
    for (int gi = 0; gi < G; ++gi) s += part[gi * C + tid];
    ws.psum[((size_t)b * d.npch + j) * C + tid] = s;
  }
  const double tot = block_sum_fixed(acc, red);
  __syncthreads();  // cnt[] complete
  if (tid == 0) ws.pscr[(size_t)b * d.npch + j] = tot;
  for (int c = tid; c < C; c += PT_THREADS) ws.plab[((size_t)b * d.npch + j) * C + c] = cnt[c];

  // The last chunk of the sequence to finish reduces all of them.
  __threadfence();
  __syncthreads();
  if (tid == 0) last = (atomicAdd(ws.pdone + b, 1) == nchb - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  double cr = 0.0;
  if (tid < C) {
    double e = 0.0;
    long long n = 0;
    for (int jj = 0; jj < nchb; ++jj) {
      const size_t o = ((size_t)b * d.npch + jj) * C + tid;
      if (center) e += __ldcg(ws.psum + o);
      n += __ldcg(ws.plab + o);
    }
    cr = center ? (double)n * (e / (double)L) : 0.0;
    ws.pfr[(size_t)b * C + tid] = center ? (double)n / (double)L : 0.0;
  }
  part[tid] = cr;
  __syncthreads();
  if (tid == 0) {
    double sc = 0.0;
    for (int jj = 0; jj < nchb; ++jj) sc += __ldcg(ws.pscr + (size_t)b * d.npch + jj);
    for (int c = 0; c < C; ++c) sc -= part[c];
    const int anybad = __ldcg(ws.pbad + b);
    if (score) score[b] = anybad ? __longlong_as_double(0x7ff8000000000000ll) : sc;
    ws.pw[b] = anybad ? 0.0 : g;
  }
}

// grad_em[b, u, c] += w_b * ([y_u = c] - n_c / L) for u < L_b (and, with
// boundary projections, grad_p_start / grad_p_end += w_b at each segment's
// first / last position and label), four elements
// per thread (blocks [0, nbe)); then grad_trans[c', c] += sum_b w_b *
// (#c' -> c transitions of path b) and grad_dur[k-1, c] += sum_b w_b *
// (#label-c segments of length k) in a fixed order (blocks [nbe, gridDim.x)).
__global__ void __launch_bounds__(PT_THREADS) path_grad_kernel(
    const int32_t* __restrict__ lengths, const int32_t* __restrict__ labels,
    const uint8_t* __restrict__ seg_start, Dims d, WsPtrs ws, float* __restrict__ grad_em,
    float* __restrict__ grad_trans, float* __restrict__ grad_dur, float* __restrict__ grad_p_start,
    float* __restrict__ grad_p_end, int nbe) {
  const int C = d.C, K = d.K, T = d.T;
  if ((int)blockIdx.x < nbe) {
    const size_t per_seq = (size_t)T * C;
    const size_t base = (size_t)blockIdx.x * (4 * PT_THREADS) + threadIdx.x;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const size_t i = base + (size_t)q * PT_THREADS;
      if (i >= (size_t)d.B * per_seq) break;
      const int b = (int)(i / per_seq);
      const size_t r = i - (size_t)b * per_seq;
      const int u = (int)(r / C), c = (int)(r - (size_t)u * C);
      const int L = __ldg(lengths + b);
      const double w = ws.pw[b];
      if (u >= L || w == 0.0) continue;
      const bool is_y = labels[(size_t)b * T + u] == c;
      if (grad_em) grad_em[i] += (float)(w * ((is_y ? 1.0 : 0.0) - ws.pfr[(size_t)b * C + c]));
      if (is_y && grad_p_start && seg_start[(size_t)b * T + u]) grad_p_start[i] += (float)w;
      if (is_y && grad_p_end && (u + 1 >= L || seg_start[(size_t)b * T + u + 1]))
        grad_p_end[i] += (float)w;
    }
    return;
  }
  // Count tables: 32 entries per block, the 8 warps take every 8th sequence
  // and their sums are added in warp order.
  __shared__ double ps[PT_THREADS / 32][32];
  const int nt = C * C, nall = C * C + K * C;
  const int lane = threadIdx.x & 31, wg = threadIdx.x >> 5;
  const int i = (blockIdx.x - nbe) * 32 + lane;
  double s = 0.0;
  if (i < nall)
#pragma unroll 4
    for (int b = wg; b < d.B; b += PT_THREADS / 32)
      s += ws.pw[b] * (double)ws.pcnt[(size_t)b * nall + i];
  ps[wg][lane] = s;
  __syncthreads();
  if (wg == 0 && i < nall) {
    double t = 0.0;
    for (int w = 0; w < PT_THREADS / 32; ++w) t += ps[w][lane];
    float* out = (i < nt) ? grad_trans : grad_dur;
    if (out) out[i < nt ? i : i - nt] += (float)t;
  }
}

cudaError_t launch_path_terms(const Dims& d, const WsPtrs& ws, const float* em,
                              const int32_t* lengths, const float* trans, const float* dur,
                              const int32_t* labels, const uint8_t* seg_start, unsigned center,
                              const double* grad_score, int negate, double* score,
                              const float* p_start, const float* p_end, cudaStream_t st) {
  path_terms_kernel<<<dim3(d.npch, d.B), PT_THREADS, 0, st>>>(
      em, lengths, trans, dur, labels, seg_start, d, ws, center, grad_score, negate, score, p_start,
      p_end);
  return cudaGetLastError();
}

cudaError_t launch_path_grad(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                             const int32_t* labels, const uint8_t* seg_start, float* grad_em,
                             float* grad_trans, float* grad_dur, float* grad_p_start,
                             float* grad_p_end, cudaStream_t st) {
  const size_t nem = (size_t)d.B * d.T * d.C;
  const bool per_pos = grad_em || grad_p_start || grad_p_end;
  const int nbe = per_pos ? (int)((nem + 4 * PT_THREADS - 1) / (4 * PT_THREADS)) : 0;
  const int nall = d.C * d.C + d.K * d.C;
  const int nbp = (grad_trans || grad_dur) ? (nall + 31) / 32 : 0;
  if (nbe + nbp == 0) return cudaSuccess;
  path_grad_kernel<<<nbe + nbp, PT_THREADS, 0, st>>>(lengths, labels, seg_start, d, ws, grad_em,
                                                     grad_trans, grad_dur, grad_p_start,
                                                     grad_p_end, nbe);
  return cudaGetLastError();
}

}  // namespace semicrf
