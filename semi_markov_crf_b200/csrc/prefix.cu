// prefix.cu -- step 1: emission centering and prefix sums.
//
// "Streaming Structured Inference with Flash-SemiCRF", explainer section 2,
// "On-the-Fly Edge Computation via Prefix Sums" and "Emission Baseline
// Centering": nu[b, c] is the mean emission of label c over the valid
// positions of sequence b, and S[b, t, c] = sum_{u < t} (em[b, u, c] - nu[b, c]).
//
// Two passes over the emissions, both coalesced: pass 1 sums fixed-size row
// chunks (float64), pass 2 re-reads each chunk into shared memory with 16-byte
// vector loads, scans it in float64 from the chunk's exclusive offset and
// writes either the float64 prefix sums (public entry point) or the split
// base-2 form the recursions consume: S2 = S * log2(e) as an int32 integer
// part plus a float32 fraction in [-0.5, 0.5].
#include "kernels.cuh"

namespace semicrf {

// Pass 1: chunk[b][j][c] = sum of em[b, u, c] over the chunk's valid rows.
__global__ void __launch_bounds__(256) prefix_reduce_kernel(const float* __restrict__ em,
                                                            const int32_t* __restrict__ lengths,
                                                            Dims d, WsPtrs ws) {
  const int b = blockIdx.y, j = blockIdx.x;
  const int C = d.C, R = d.prefR;
  int L = lengths[b];
  if (L < 0 || L > d.T) L = 0;  // reported by the scan pass
  const int r0 = j * R;
  const int r1 = min(r0 + R, L);
  if (j == 0 && threadIdx.x == 0 && ws.emax) ws.emax[b] = 0.f;  // maxed by the scan pass
  __shared__ double part[256];
  const int G = 256 / C;  // row groups
  const int g = threadIdx.x / C, c = threadIdx.x % C;
  double acc = 0.0;
  if (g < G) {
    const float* base = em + ((size_t)b * d.T) * C;
    for (int r = r0 + g; r < r1; r += G) acc += (double)base[(size_t)r * C + c];
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < C) {
    double s = 0.0;
    for (int gg = 0; gg < G; ++gg) s += part[gg * C + threadIdx.x];
    ws.chunk[((size_t)b * d.nchunk + j) * C + threadIdx.x] = s;
  }
}

// Pass 2.  mode 0: write S64 [B][T+1][C] (float64) and nu [B][C] (float32).
//          mode 1: write the split base-2 arrays into the workspace.
__global__ void __launch_bounds__(256) prefix_scan_kernel(const float* __restrict__ em,
                                                          const int32_t* __restrict__ lengths,
                                                          Dims d, WsPtrs ws, unsigned center,
                                                          int mode, double* __restrict__ S64,
                                                          float* __restrict__ nu_out,
                                                          const float* __restrict__ p_start,
                                                          const float* __restrict__ p_end) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int b = blockIdx.y, j = blockIdx.x;
  const int C = d.C, R = d.prefR, T = d.T;
  int L = lengths[b];
  const bool bad = (L < 0 || L > T);
  if (bad) {
    if (j == 0 && threadIdx.x == 0) set_status(ws.status, ST_BAD_LENGTH);
    L = 0;
  }
  float* tile = reinterpret_cast<float*>(smem_raw);              // [R][C]
  double* nu = reinterpret_cast<double*>(tile + R * C + 4);      // [C] (8-byte aligned below)
  nu = reinterpret_cast<double*>((reinterpret_cast<uintptr_t>(nu) + 7) & ~uintptr_t(7));
  double* off = nu + C;          // [C] exclusive chunk offset
  double* grp = off + C;         // [G][C] per-group partial sums

  // nu and this chunk's offset from the pass-1 chunk sums (fixed order).
  if (threadIdx.x < C) {
    const int c = threadIdx.x;
    const double* cs = ws.chunk + (size_t)b * d.nchunk * C + c;
    double tot = 0.0, before = 0.0;
    const int nch_valid = (L + R - 1) / R;
    for (int jj = 0; jj < nch_valid; ++jj) {
      double v = cs[(size_t)jj * C];
      if (jj < j) before += v;
      tot += v;
    }
    const double nuc = (center && L > 0) ? tot / (double)L : 0.0;
    nu[c] = nuc;
    off[c] = before - (double)min(j * R, L) * nuc;
    if (mode == 0 && j == 0 && nu_out) nu_out[(size_t)b * C + c] = (float)nuc;
  }

  // Stage the chunk's rows into shared memory (16-byte loads when aligned).
  const int r0 = j * R;
  const int nrows = max(0, min(R, L - r0));
  const size_t gbase = ((size_t)b * T + r0) * C;
  const int nel = nrows * C;
  const float* src = em + gbase;
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    const int n4 = nel >> 2;
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float4* t4 = reinterpret_cast<float4*>(tile);
    for (int i = threadIdx.x; i < n4; i += blockDim.x) t4[i] = __ldg(s4 + i);
    for (int i = (n4 << 2) + threadIdx.x; i < nel; i += blockDim.x) tile[i] = __ldg(src + i);
  } else {
    for (int i = threadIdx.x; i < nel; i += blockDim.x) tile[i] = __ldg(src + i);
  }
  __syncthreads();

  // Thread (g, c) scans rows [g*RB, (g+1)*RB) of column c.
  const int G = blockDim.x / C;
  const int RB = (R + G - 1) / G;
  const int g = threadIdx.x / C, c = threadIdx.x % C;
  double local = 0.0;
  if (g < G) {
    const double nuc = nu[c];
    for (int r = g * RB; r < min((g + 1) * RB, nrows); ++r) local += (double)tile[r * C + c] - nuc;
    grp[g * C + c] = local;
  }
  __syncthreads();
  float emx = 0.f;  // largest |centred emission| of this thread's rows
  if (g < G) {
    const double nuc = nu[c];
    double run = off[c];
    for (int gg = 0; gg < g; ++gg) run += grp[gg * C + c];
    // rows of S written by this thread: t = r0 + r + 1 for r in its block
    for (int r = g * RB; r < min((g + 1) * RB, R); ++r) {
      const int t = r0 + r + 1;
      if (t > T) break;
      double val = 0.0, xa = 0.0;
      if (r < nrows) {
        const double x = (double)tile[r * C + c] - nuc;
        run += x;
        val = run;
        xa = fabs(x);
        emx = fmaxf(emx, (float)xa);
      }
      const bool valid = (t <= L);
      if (mode == 0) {
        S64[((size_t)b * (T + 1) + t) * C + c] = valid ? val : 0.0;
      } else {
        const size_t o = ((size_t)b * d.Tstride + t) * C + c;
        double pe = 0.0;
        if (p_start || p_end) {
          // boundary projections: P_end[t-1] joins S[t]; pd[t] is the start side
          const size_t q = ((size_t)b * T + (t - 1)) * C + c;
          pe = (valid && p_end) ? (double)__ldg(p_end + q) : 0.0;
          const double ps = (t < L && p_start) ? (double)__ldg(p_start + q + C) : 0.0;
          ws.pd[o] = (float)((pe + ps) * LOG2E_D);
          // the exponential-domain test bounds a step's swing: with
          // projections a position's terms include both of them
          if (valid) emx = fmaxf(emx, (float)(xa + fabs(pe) + fabs(ps)));
        }
        const double s2 = valid ? (val + pe) * LOG2E_D : 0.0;
        const double ip = rint(s2);
        ws.sint[o] = (int32_t)ip;
        ws.sfrac[o] = (float)(s2 - ip);
      }
    }
    if (j == 0 && g == 0) {  // row t = 0
      if (mode == 0) {
        S64[((size_t)b * (T + 1)) * C + c] = 0.0;
      } else {
        const size_t o = ((size_t)b * d.Tstride) * C + c;
        ws.sint[o] = 0;
        ws.sfrac[o] = 0.f;
        if (p_start || p_end) {
          const double ps0 = (p_start && L > 0) ? (double)__ldg(p_start + (size_t)b * T * C + c) : 0.0;
          ws.pd[o] = (float)(ps0 * LOG2E_D);
          emx = fmaxf(emx, (float)fabs(ps0));
        }
      }
    }
  }
  // per-sequence bound for the choice of the ring arithmetic (non-negative
  // floats order like their bit patterns); NaN never compares larger
  if (mode == 1 && ws.emax) {
    float m = emx * (float)LOG2E_D;
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL_MASK, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0.f)
      atomicMax(reinterpret_cast<int*>(ws.emax + b), __float_as_int(m));
  }
}

}  // namespace semicrf
