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
#include <algorithm>

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
//          2^(gamma[s, c] - S[s, c] + dur2[t-s-1, c] + S[t, c] + beta[t, c]).
// The start side (s = u - ia) and the end side (t = u + 1 + jb) are staged
// once per label as logs relative to R = Pf_u + Pb_{u+1} and S[u, c]:
//   la[ia, c] = log2 af[s] + (Pf_s - Pf_u) - (S[s, c] - S[u, c])
//   lb[jb, c] = log2 ab[t] + (Pb_t - Pb_{u+1}) + (S[t, c] - S[u, c])
// (every large quantity enters as a difference before float32 sees it), and
// the segment term is la + lb + (2M + dur2[ia + jb, c]), ia + jb < K.  A warp
// per label sums them (its max first, so the sum cannot overflow).
__global__ void __launch_bounds__(256)
    cut_grid_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                    const float* __restrict__ trans, const float* __restrict__ dur, int pj,
                    int per_label) {
  // la, lb, dd: [C][K + 1] each; per_label (long durations): [K + 1] each,
  // one label at a time, every thread of the block on that label
  extern __shared__ float csh[];
  __shared__ float lab_M[128], lab_f[128];  // per label: shift, log2 share
  __shared__ float red[32];
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
  const float M = *ws.tmax;  // max trans2, written by the rings
  // label-major rows of KP = K + 1 floats (the odd stride keeps both the
  // staging stores, consecutive labels, and the sums' reads, consecutive
  // offsets of one label, free of bank conflicts)
  const int KP = K + 1;
  const int CB = per_label ? 1 : C;  // labels staged at once
  float* const la = csh;
  float* const lb = csh + (size_t)KP * CB;
  float* const dd = csh + 2 * (size_t)KP * CB;
  const double Fu = kf_at(ws, d, b, 0, u), Gu = kf_at(ws, d, b, 1, u + 1);
  const int32_t* si = ws.sint + (size_t)b * d.Tstride * C;
  const float* sf = ws.sfrac + (size_t)b * d.Tstride * C;
  const float* kf0 = kv_row(ws, d, b, 0, 0);
  const float* kf1 = kv_row(ws, d, b, 1, 0);
  // the start side (s = u - q) and end side (t = u + 1 + q) of label c
  auto stage = [&](int i, int q, int c, int slot) {
    const int su = si[(size_t)u * C + c];
    const float fu = sf[(size_t)u * C + c];
    float va = NEG_INF, vb = NEG_INF;
    const int s = u - q, t = u + 1 + q;
    if (s >= 0) {
      const float a = kf0[(size_t)s * 2 * C + C + c];
      if (a > 0.f)
        va = (lg2(a) + (float)(kf_at(ws, d, b, 0, s) - Fu)) -
             ((float)(si[(size_t)s * C + c] - su) + (sf[(size_t)s * C + c] - fu)) +
             (pj ? ws.pd[((size_t)b * d.Tstride + s) * C + c] : 0.f);  // start-side projection
    }
    if (t <= L) {
      const float bt = kf1[(size_t)t * 2 * C + C + c];
      if (bt > 0.f)
        vb = (lg2(bt) + (float)(kf_at(ws, d, b, 1, t) - Gu)) +
             ((float)(si[(size_t)t * C + c] - su) + (sf[(size_t)t * C + c] - fu));
    }
    la[slot * KP + q] = va;
    lb[slot * KP + q] = vb;
    dd[slot * KP + q] = 2.f * M + __ldg(dur + i) * l2e();
  };
  const int lane = tid & 31;
  if (per_label) {
    // long durations: label by label, all threads over the start offset ia
    const int nw = blockDim.x >> 5, wid = tid >> 5;
    for (int c = 0; c < C; ++c) {
      for (int q = tid; q < K; q += blockDim.x) stage(q * C + c, q, c, 0);
      __syncthreads();
      float zmax = NEG_INF;
      for (int ia = tid; ia < K; ia += blockDim.x) {
        const float a = la[ia];
        if (a == NEG_INF) continue;
        for (int jb = 0; jb < K - ia; ++jb) zmax = fmaxf(zmax, (a + lb[jb]) + dd[ia + jb]);
      }
      zmax = group_max(zmax, 32);
      if (lane == 0) red[wid] = zmax;
      __syncthreads();
      float mz = NEG_INF;
      for (int w2 = 0; w2 < nw; ++w2) mz = fmaxf(mz, red[w2]);
      const float Mz = (mz == NEG_INF) ? 0.f : ceilf(mz);
      __syncthreads();
      float sum = 0.f;
      for (int ia = tid; ia < K; ia += blockDim.x) {
        const float a = la[ia] - Mz;
        if (a == NEG_INF) continue;
        for (int jb = 0; jb < K - ia; ++jb) sum += ex2((a + lb[jb]) + dd[ia + jb]);
      }
      sum = group_sum(sum, 32);
      if (lane == 0) red[wid] = sum;
      __syncthreads();
      if (tid == 0) {
        float tot = 0.f;
        for (int w2 = 0; w2 < nw; ++w2) tot += red[w2];  // fixed order: deterministic
        lab_M[c] = Mz;
        lab_f[c] = (tot > 0.f) ? lg2(tot) : NEG_INF;
      }
      __syncthreads();
    }
  } else {
  #pragma unroll 4
  for (int i = tid; i < K * C; i += blockDim.x) {
    const int q = i / C, c = i - q * C;
    stage(i, q, c, c);
  }
  __syncthreads();
  const int nw = blockDim.x >> 5;
  for (int c = tid >> 5; c < C; c += nw) {
    // a warp per label: lanes over pairs of start offsets (ia, K-1-ia), so
    // every lane sums about K + 1 terms, the inner loop over the end offset
    const float* const lac = la + c * KP;
    const float* const lbc = lb + c * KP;
    const float* const ddc = dd + c * KP;
    auto pair_sum = [&](float Mz) {
      float sum = 0.f;
      for (int p = lane; p < (K + 1) / 2; p += 32) {
        for (int h = 0; h < 2; ++h) {
          const int ia = h ? K - 1 - p : p;
          if (h && ia == p) break;
          const float a = lac[ia] - Mz;
          if (a == NEG_INF) continue;
          for (int jb = 0; jb < K - ia; ++jb) sum += ex2((a + lbc[jb]) + ddc[ia + jb]);
        }
      }
      return group_sum(sum, 32);
    };
    // the shift: a bound on every term, max la + max lb + max dd; only when
    // the sum then falls below 2^-60 (the bound far above the largest term)
    // is the exact largest term found and the sum taken again
    float ma = NEG_INF, mb = NEG_INF, md = NEG_INF;
    for (int q = lane; q < K; q += 32) {
      ma = fmaxf(ma, lac[q]);
      mb = fmaxf(mb, lbc[q]);
      md = fmaxf(md, ddc[q]);
    }
    ma = group_max(ma, 32);
    mb = group_max(mb, 32);
    md = group_max(md, 32);
    const bool any = ma != NEG_INF && mb != NEG_INF && md != NEG_INF;
    float Mz = any ? ceilf((ma + mb) + md) : 0.f;
    float sum = any ? pair_sum(Mz) : 0.f;
    if (any && !(sum >= 0x1p-60f)) {
      float zmax = NEG_INF;
      for (int p = lane; p < (K + 1) / 2; p += 32) {
        for (int h = 0; h < 2; ++h) {
          const int ia = h ? K - 1 - p : p;
          if (h && ia == p) break;
          const float a = lac[ia];
          if (a == NEG_INF) continue;
          for (int jb = 0; jb < K - ia; ++jb) zmax = fmaxf(zmax, (a + lbc[jb]) + ddc[ia + jb]);
        }
      }
      zmax = group_max(zmax, 32);
      Mz = (zmax == NEG_INF) ? 0.f : ceilf(zmax);
      sum = pair_sum(Mz);
    }
    if (lane == 0) {
      lab_M[c] = Mz;
      lab_f[c] = (sum > 0.f) ? lg2(sum) : NEG_INF;
    }
  }
  __syncthreads();
  }
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

// Shared memory of cut_grid_kernel: every label's rows when they fit the
// budget, else one label's (cut_grid_per_label).
bool cut_grid_per_label(const Dims& d, size_t budget) {
  return 3ull * (d.K + 1) * d.C * sizeof(float) > budget;
}
size_t cut_grid_smem_bytes(const Dims& d, size_t budget) {
  return 3ull * (d.K + 1) * (cut_grid_per_label(d, budget) ? 1 : d.C) * sizeof(float);
}

namespace {

// Shared memory of posterior_kernel for a tile of RT boundaries (Cp = C
// rounded up to a multiple of 4, R = RT + KH staged segment-end rows).
//
// Every duration term is one power of two,
//   P([s, s+k), c) = 2^(Y[s+k, c] - X[s, c] + dur2'[k-1, c])        (dur2' = M + dur2)
//   Y[t, c] = I[t, c] + S_frac[t, c] + log2 ab[t, c]                 (end side)
//   X[s, c] = I[s, c] + S_frac[s, c] - pd[s, c] - log2 af[s, c] - log2 f_s   (start side)
// with I[t, c] = (Pb_t - Pb_t0) + S_int[t, c] the exact integer part of the
// prefix sum.  Both sides are stored split into an integer (held exactly in a
// float: the integers are taken relative to the segment's first row t0, so
// they stay far below 2^24) and a fraction in [-1/2, 1/2], so the large
// values only ever meet as an exact integer difference.  A side whose kept value is
// zero is stored as an infinite integer part (its terms are 0).
struct PTile {
  float* pa;    // [RT][Cp]  forward p of the tile rows times f_s (transition items)
  float* pbt;   // [RT][Cp]  backward p of the tile rows (transition items)
  double* dif;  // [RT][C]   St - E of each boundary and label
  float* xi;    // [RT][C]   start side X: integer part
  float* xf;    // [RT][C]   start side X: fraction
  float* yi;    // [R][C]    end side Y of the staged rows: integer part
  float* yf;    // [R][C]    end side Y: fraction
  int* li;      // [2][RT]   log2 f_s: integer part (this tile's and the next's)
  float* lf;    // [2][RT]   log2 f_s: remainder
  float* fs;    // [2][RT]   f_s
};
__host__ __device__ __forceinline__ int pad4(int C) { return (C + 3) & ~3; }
__host__ __device__ __forceinline__ size_t ptile_bytes(int RT, int KH, int C) {
  const size_t R = (size_t)RT + KH;
  return 8ull * RT * pad4(C) + 16ull * RT * C + 8ull * R * C + 24ull * RT;
}
__device__ __forceinline__ PTile ptile_carve(unsigned char* raw, int RT, int KH, int C) {
  PTile t;
  const size_t R = (size_t)RT + KH, Cp = pad4(C);
  t.pa = reinterpret_cast<float*>(raw);  // 16-byte aligned: read as float4
  t.pbt = t.pa + RT * Cp;
  t.dif = reinterpret_cast<double*>(t.pbt + RT * Cp);
  t.xi = reinterpret_cast<float*>(t.dif + (size_t)RT * C);
  t.xf = t.xi + (size_t)RT * C;
  t.yi = t.xf + (size_t)RT * C;
  t.yf = t.yi + R * C;
  t.li = reinterpret_cast<int*>(t.yf + R * C);
  t.lf = reinterpret_cast<float*>(t.li + 2 * RT);
  t.fs = t.lf + 2 * RT;
  return t;
}

// log2 that keeps subnormal inputs (the ftz form would send them to -inf)
__device__ __forceinline__ float lg2_sub(float x) {
  float y;
  asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Split v into an integer (added to the exact integer base ib) and a
// fraction in [-1/2, 1/2] and store both; a value too large to split (an
// infinite side: a kept value of 0) is stored whole as the integer part.
__device__ __forceinline__ void split_store(float v, int ib, float* pi, float* pf) {
  if (fabsf(v) < 1e7f) {
    const float n = rintf(v);
    *pi = (float)(ib + (int)n);
    *pf = v - n;
  } else {
    *pi = v;
    *pf = 0.f;
  }
}

// The kernel variant: two CTAs per SM (one quad and one transition block per
// thread) when the items fit that, else one.
inline bool posterior_pair(const Dims& d) {
  const long long nq = (long long)((d.K + 3) / 4) * d.C, nbk = pad4(d.C) / 4;
  return nq <= 512 && nbk * nbk <= 512;
}

// One CTA per (checkpoint segment j, sequence b): every posterior whose start
// boundary lies in [t0, t1), written in the same per-segment layout as
// segment_kernel (suffix sums v in grad_em, per-segment totals, float64
// count partials), so finalize and the partial reduction are shared; here
// the per-segment total is the plain sum over the segment (finalize takes the
// running sum over segments), because the normaliser is continuous.
//
// The segment is cut into tiles of d.pRT boundaries, taken downwards (the
// suffix sums run that way).  A tile stages, with coalesced loads, its start
// sides X and its transition operands, and the end sides Y of the rows its
// segments end on (KH rows at a time: all K at once, or chunks of the
// duration range for long durations).  Then:
//   duration counts -- a thread owns quads (4 consecutive durations, one
//     label) and slides a 4-row window of Y down the tile's starts: per term
//     one exponential and four adds, one new Y row per start;
//   transition counts -- sum over s of pa[s, c'] pb[s, c], a rank-RT update
//     of a C x C matrix, in 4 x 4 register blocks;
//   suffix sums -- one thread per label, running up the tile.
// Each thread keeps its first NQ quads and NB blocks in registers across
// tiles (512 threads: K C <= 8192, C <= 128); the quads beyond (long
// durations) add per-tile sums to the float64 partials.
template <int NQ, int NB>
__global__ void __launch_bounds__(512, NQ > 1 ? 1 : 2)
    posterior_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                     const float* __restrict__ trans, const float* __restrict__ dur,
                     const double* __restrict__ grad_logZ, float* __restrict__ grad_em,
                     float* __restrict__ start_marg, float* __restrict__ end_marg,
                     float* __restrict__ seg_marg, int pj) {
  extern __shared__ __align__(16) unsigned char psh[];
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, nthr = blockDim.x;
  const int C = d.C, K = d.K, RT = d.pRT, KH = d.pKH, Cp = pad4(C);
  const int R = RT + KH;  // staged segment-end rows
  const int L = lengths[b];
  if (L <= 0 || L > d.T) return;
  if (!posterior_from_kept(ws, d, b)) return;  // segment_kernel runs it
  const int t0 = j * d.delta;
  if (t0 >= L) return;
  const int t1 = min(t0 + d.delta, L);
  const size_t seg = (size_t)b * d.nck + j;
  const float gb = (float)(grad_logZ ? grad_logZ[b] : 1.0);
  const float M = *ws.tmax;  // max trans2, written by the rings
  const PTile tl = ptile_carve(psh, RT, KH, C);
  const float* pfr = kv_row(ws, d, b, 0, 0);  // row t: pfr + t*2C (p), + C (acc)
  const float* pbr = kv_row(ws, d, b, 1, 0);
  const double* kff = ws.kf + ((size_t)b * 2 + 0) * (d.T + 1);
  const double* kfb = ws.kf + ((size_t)b * 2 + 1) * (d.T + 1);
  const double* nc = ws.ncut + (size_t)b * d.ngrid;
  const int32_t* si = ws.sint + (size_t)b * d.Tstride * C;
  const float* sfp = ws.sfrac + (size_t)b * d.Tstride * C;
  const int nd = K * C, ntr = C * C;
  const int nq = ((K + 3) >> 2) * C;  // quads
  const int nbk = Cp >> 2, nblk = nbk * nbk;
  float accq[NQ][4], acct[NB][16];
#pragma unroll
  for (int m = 0; m < NQ; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u) accq[m][u] = 0.f;
#pragma unroll
  for (int m = 0; m < NB; ++m)
#pragma unroll
    for (int u = 0; u < 16; ++u) acct[m][u] = 0.f;
  double lacc = 0.0, lvs = 0.0;  // thread c < C: running suffix sum, sum of v
  // integer bases of the segment: every staged integer is relative to row t0
  const double kbase = kfb[t0];
  const int32_t* sib = si + (size_t)t0 * C;
  // f_s = 2^(Pf_s + Pb_s + M - log2 Z(s)) of a tile's rows, also split for
  // the start sides, into buffer slot fb (the next tile's are taken while
  // this one computes)
  auto stage_f = [&](int lo, int n, int fb) {
    for (int r = tid; r < n; r += nthr) {
      const int s = lo + r;
      const double l = ((kff[s] + kfb[s]) + (double)M) - local_logz(d, nc, L, min(s, L - 1));
      const double nn = fabs(l) < 1e9 ? rint(l) : 0.0;
      tl.li[fb * RT + r] = (int)nn;
      tl.lf[fb * RT + r] = (float)(l - nn);
      tl.fs[fb * RT + r] = ex2((float)l);
    }
  };
  // All segment ends staged at once (KH = K): the staged rows roll.  Row t
  // sits in slot (t - t0) mod R; a tile needs rows [s_lo, s_lo + nr + K), so
  // the next tile down (s_lo - RT) stages only its RT new rows, whose slots
  // held rows at least RT + K above them, past what it reads.
  const bool roll = KH == K;
  int fb = 0;
  stage_f(max(t0, t1 - RT), t1 - max(t0, t1 - RT), 0);
  __syncthreads();

  for (int s_hi = t1; s_hi > t0; s_hi -= RT) {
    const int s_lo = max(t0, s_hi - RT);
    const int nr = s_hi - s_lo;
    const int Lr = L - s_lo;                         // a segment [s_lo + r, s_lo + r + k) needs r + k <= Lr
    const int nh = min(s_hi - 1 + K, L) - s_lo + 1;  // rows a segment of the tile ends on
    const bool first = (s_hi == t1);
    // bounds-check build: the tile fits its rows
    if (!SEMICRF_INB(ws.status, nr >= 1 && nr <= RT && nh <= RT + K, SITE_POST_TILE)) break;
    const float* const fsb = tl.fs + fb * RT;
    const int* const lib = tl.li + fb * RT;
    const float* const lfb = tl.lf + fb * RT;
    // staged slot of segment-end row s_lo + h (h < R)
    const int off = roll ? (s_lo - t0) % R : 0;
    auto slot = [&](int h) {
      const int q = off + h;
      return q >= R ? q - R : q;
    };
    // ------------------------------------------------------------ stage the tile rows
    // start / end marginals and St - E; transition operands; start sides X.
    // SU items per thread at a time, every load of a batch issued before its
    // first store (the marginal stores could alias the kept rows as far as
    // the compiler can tell, which would hold each load behind them)
    constexpr int SU = NQ > 1 ? 4 : 2;  // (the two-CTA variant has half the registers)
    for (int i0 = tid; i0 < nr * Cp; i0 += SU * nthr) {
      float tp[SU], ta[SU], bp[SU], ba[SU], pdv[SU], sfv[SU];
      int siv[SU];
      double kfv[SU];
#pragma unroll
      for (int u = 0; u < SU; ++u) {
        const int i = i0 + u * nthr;
        const int r = i / Cp, c = i - r * Cp;
        const bool ok = i < nr * Cp && c < C;
        const size_t row = (size_t)(s_lo + (ok ? r : 0));
        const int cc = ok ? c : 0;
        tp[u] = ok ? pfr[row * 2 * C + cc] : 0.f;
        ta[u] = ok ? pfr[row * 2 * C + C + cc] : 0.f;
        bp[u] = ok ? pbr[row * 2 * C + cc] : 0.f;
        ba[u] = ok ? pbr[row * 2 * C + C + cc] : 0.f;
        pdv[u] = (ok && pj) ? ws.pd[((size_t)b * d.Tstride + row) * C + cc] : 0.f;
        sfv[u] = ok ? sfp[row * C + cc] : 0.f;
        siv[u] = ok ? si[row * C + cc] - sib[cc] : 0;
        kfv[u] = ok ? kfb[row] : kbase;
      }
#pragma unroll
      for (int u = 0; u < SU; ++u) {
        const int i = i0 + u * nthr;
        if (i >= nr * Cp) break;
        const int r = i / Cp, c = i - r * Cp;
        if (c >= C) {
          tl.pa[i] = 0.f;
          tl.pbt[i] = 0.f;
          continue;
        }
        const size_t row = (size_t)(s_lo + r);
        const float f = fsb[r];
        const float St = ta[u] * bp[u] * f, E = ba[u] * tp[u] * f;
        const size_t ob = ((size_t)b * (d.T + 1) + row) * C + c;
        if (start_marg) start_marg[ob] = St;
        if (end_marg) end_marg[ob] = E;
        const int o = r * C + c;
        tl.dif[o] = (double)St - (double)E;
        tl.pa[i] = tp[u] * f;
        tl.pbt[i] = bp[u];
        const int ib = (int)(kfv[u] - kbase) + siv[u];
        split_store((sfv[u] - pdv[u]) - (lg2_sub(ta[u]) + lfb[r]), ib - lib[r], tl.xi + o,
                    tl.xf + o);
      }
    }
    // ------------------------------------------------------------ segment ends, by chunk
    // chunk kc: durations [kc, kc + KH), staged rows at offsets [kc - 1, kc - 1 + nr + KH)
    // from s_lo (the first chunk includes the tile rows themselves)
    for (int kc = 1; kc <= K; kc += KH) {
      const int base = kc - 1;
      const int nst = max(0, min(base + nr + KH, nh) - base);
      if (kc > 1) __syncthreads();  // the previous chunk's reads are done
      // rolling: the first tile stages all its rows, later ones the RT below
      // the previous tile; chunks: all of the chunk's rows, slot = offset
      const int nnew = roll ? (first ? nst : min(nst, nr)) : nst;
      for (int i0 = tid; i0 < nnew * C; i0 += SU * nthr) {
        float sv[SU], bv[SU];
        int iv[SU];
#pragma unroll
        for (int u = 0; u < SU; ++u) {  // loads first (as above)
          const int i = i0 + u * nthr;
          const bool ok = i < nnew * C;
          const int h = ok ? i / C : 0, c = ok ? i - h * C : 0;
          const size_t row = (size_t)(s_lo + base + h);
          iv[u] = (int)(kfb[row] - kbase) + (si[row * C + c] - sib[c]);
          sv[u] = sfp[row * C + c];
          bv[u] = pbr[row * 2 * C + C + c];
        }
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int i = i0 + u * nthr;
          if (i >= nnew * C) break;
          const int h = i / C, c = i - h * C;
          const int p = slot(h);
          split_store(sv[u] + lg2_sub(bv[u]), iv[u], tl.yi + (size_t)p * C + c,
                      tl.yf + (size_t)p * C + c);
        }
      }
      __syncthreads();
      // -------------------------------------------------------- segment marginals
      // (optional output) P([s, s+k), c) for every start of the tile and
      // every duration of the chunk, not scaled by g (a marginal)
      if (seg_marg) {
        const int lo_i = base * C, nci = min(nd, (base + KH) * C) - lo_i;
        for (int i = tid; i < nr * nci; i += nthr) {
          const int r = i / nci, idx = lo_i + (i - r * nci);
          const int k = idx / C + 1, c = idx - (k - 1) * C;
          if (r + k > Lr) continue;
          if (!SEMICRF_INB(ws.status, r + k - base < nst, SITE_POST_ITEM)) continue;
          const int o = r * C + c, ok = slot(r + k - base) * C + c;
          const float z = (tl.yi[ok] - tl.xi[o]) +
                          ((tl.yf[ok] - tl.xf[o]) + (M + __ldg(dur + idx) * l2e()));
          seg_marg[((size_t)b * d.T + s_lo + r) * nd + idx] = ex2(z);
        }
      }
      // -------------------------------------------------------- duration counts
      // quad q = (kq, c): durations k0 .. k0 + 3 (k0 = 4 kq + 1) of label c, each
      // summed over the tile's starts r with r + k <= Lr
      const int q_lo = (base >> 2) * C, q_hi = min(nq, ((base + KH + 3) >> 2) * C);
      auto quad = [&](int q, float (&a)[4]) {
        const int kq = q / C, c = q - kq * C, k0 = 4 * kq + 1;
        float dk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dk[u] = (k0 + u <= K) ? M + __ldg(dur + (k0 + u - 1) * C + c) * l2e() : -INFINITY;
        const int h0 = k0 - base;  // staged row of (r = 0, u = 0)
        const int r_all = max(0, min(nr, Lr - (k0 + 3) + 1));  // every k0 + u valid
        const int r_any = max(0, min(nr, Lr - k0 + 1));        // k0 valid
        // bounds-check build: the window stays in the staged rows
        if (!SEMICRF_INB(ws.status, h0 >= 1 && h0 + nr + 2 < R &&
                                        (r_any == 0 || r_any - 1 + k0 - base < nst),
                         SITE_POST_ITEM))
          return;
        const float* yi = tl.yi + c;
        const float* yf = tl.yf + c;
        float w0i = yi[slot(h0) * C], w0f = yf[slot(h0) * C];
        float w1i = yi[slot(h0 + 1) * C], w1f = yf[slot(h0 + 1) * C];
        float w2i = yi[slot(h0 + 2) * C], w2f = yf[slot(h0 + 2) * C];
        int r = 0;
#pragma unroll 4
        for (; r < r_all; ++r) {
          const int h3 = slot(h0 + r + 3) * C;
          const float w3i = yi[h3], w3f = yf[h3];
          const float oi = tl.xi[r * C + c], of = tl.xf[r * C + c];
          a[0] += ex2((w0i - oi) + ((w0f - of) + dk[0]));
          a[1] += ex2((w1i - oi) + ((w1f - of) + dk[1]));
          a[2] += ex2((w2i - oi) + ((w2f - of) + dk[2]));
          a[3] += ex2((w3i - oi) + ((w3f - of) + dk[3]));
          w0i = w1i; w0f = w1f;
          w1i = w2i; w1f = w2f;
          w2i = w3i; w2f = w3f;
        }
        // the last starts of a sequence: the longer durations run past L
        for (; r < r_any; ++r) {
          const float oi = tl.xi[r * C + c], of = tl.xf[r * C + c];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (r + k0 + u > Lr) break;
            const int h = slot(h0 + r + u) * C;
            a[u] += ex2((yi[h] - oi) + ((yf[h] - of) + dk[u]));
          }
        }
      };
#pragma unroll
      for (int m = 0; m < NQ; ++m) {
        const int q = tid + m * nthr;
        if (q >= q_lo && q < q_hi) quad(q, accq[m]);
      }
      for (int q = tid + NQ * nthr; q < q_hi; q += nthr) {
        if (q < q_lo) continue;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        quad(q, a);
        const int kq = q / C, c = q - kq * C;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = 4 * kq + 1 + u;
          if (k > K) break;
          double* pd = ws.pgd + seg * nd + (size_t)(k - 1) * C + c;
          const double v = (double)(gb * a[u]);
          *pd = first ? v : *pd + v;
        }
      }
    }
    // ------------------------------------------------------------ transition counts
    // block (bi, bj): labels c' in 4 bi .. 4 bi + 3, c in 4 bj .. 4 bj + 3
    auto tblock = [&](int q, float (&a)[16]) {
      const int bi = q / nbk, bj = q - bi * nbk;
      const float4* pa4 = reinterpret_cast<const float4*>(tl.pa) + bi;
      const float4* pb4 = reinterpret_cast<const float4*>(tl.pbt) + bj;
#pragma unroll 2
      for (int r = 0; r < nr; ++r) {
        const float4 x = pa4[r * nbk], y = pb4[r * nbk];
        const float xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) a[u * 4 + v] = fmaf(xs[u], ys[v], a[u * 4 + v]);
      }
    };
    auto tblock_out = [&](int q, const float (&a)[16], bool to_partials) {
      const int bi = q / nbk, bj = q - bi * nbk;
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int c1 = 4 * bi + u, c = 4 * bj + v;
          if (c1 >= C || c >= C) continue;
          const int idx = c1 * C + c;
          const double val = (double)(gb * a[u * 4 + v] * ex2(__ldg(trans + idx) * l2e() - M));
          double* pt = ws.pgt + seg * ntr + idx;
          *pt = (to_partials && !first) ? *pt + val : val;
        }
    };
#pragma unroll
    for (int m = 0; m < NB; ++m)
      if (tid + m * nthr < nblk) tblock(tid + m * nthr, acct[m]);
    for (int q = tid + NB * nthr; q < nblk; q += nthr) {
      float a[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) a[u] = 0.f;
      tblock(q, a);
      tblock_out(q, a, true);
    }
    // ------------------------------------------------------------ suffix sums
    // v[s] = sum of (St - E) over the segment's boundaries after s
    if (tid < C) {
      for (int r = nr - 1; r >= 0; --r) {
        grad_em[((size_t)b * d.T + s_lo + r) * C + tid] = (float)lacc;
        lvs += (double)(float)lacc;
        lacc += tl.dif[r * C + tid];
      }
    }
    // the next tile's f_s into the other slot (nobody reads it now)
    if (s_hi - RT > t0) {
      const int nlo = max(t0, s_hi - 2 * RT);
      stage_f(nlo, s_lo - nlo, fb ^ 1);
    }
    fb ^= 1;
    __syncthreads();  // the next tile overwrites the staged rows
  }
  // register items: the segment's partials
#pragma unroll
  for (int m = 0; m < NQ; ++m) {
    const int q = tid + m * nthr;
    if (q >= nq) continue;
    const int kq = q / C, c = q - kq * C;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = 4 * kq + 1 + u;
      if (k <= K) ws.pgd[seg * nd + (size_t)(k - 1) * C + c] = (double)(gb * accq[m][u]);
    }
  }
#pragma unroll
  for (int m = 0; m < NB; ++m) {
    const int q = tid + m * nthr;
    if (q >= nblk) continue;
    const int bi = q / nbk, bj = q - bi * nbk;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int c1 = 4 * bi + u, c = 4 * bj + v;
        if (c1 < C && c < C)
          ws.pgt[seg * ntr + c1 * C + c] =
              (double)(gb * acct[m][u * 4 + v] * ex2(__ldg(trans + c1 * C + c) * l2e() - M));
      }
  }
  if (tid < C) {
    ws.segT[seg * C + tid] = lacc;
    ws.segV[seg * C + tid] = lvs;
  }
  if (t1 == L) {
    // boundary L: its end marginal (normalised at position L - 1), no start
    const float fL = ex2((float)(((kff[L] + kfb[L]) + (double)M) - local_logz(d, nc, L, L - 1)));
    for (int c = tid; c < C; c += nthr) {
      const size_t ob = ((size_t)b * (d.T + 1) + L) * C + c;
      if (end_marg) end_marg[ob] = pfr[(size_t)L * 2 * C + c] * pbr[(size_t)L * 2 * C + C + c] * fL;
      if (start_marg) start_marg[ob] = 0.f;
    }
  }
}

}  // namespace

// Tile rows of the posterior pass: the largest power of two up to 64 (and
// not past the segment) whose tile, with all K segment-end rows, fits
// `budget` bytes; with `pair` (the kernel that runs two CTAs per SM) a tile
// that fits half the SM first, unless that halves the rows.  Long
// durations: the segment ends are staged in chunks of KH rows (a multiple of
// 64), the tile as tall as fits.  Sets d.pKH; 0 if nothing fits.
int posterior_tile_rows(Dims& d, size_t budget) {
  int cap = 64;
  while (cap > 8 && cap / 2 >= d.delta) cap /= 2;
  d.pKH = d.K;
  int best = 0;
  for (int rt = cap; rt >= 8 && !best; rt /= 2)
    if (ptile_bytes(rt, d.K, d.C) <= budget) best = rt;
  if (best && posterior_pair(d))
    for (int rt = best; rt >= 8 && rt * 2 > best; rt /= 2)
      if (ptile_bytes(rt, d.K, d.C) <= std::min<size_t>(budget, 112u * 1024u)) return rt;
  if (best) return best;
  for (int rt = cap; rt >= 8; rt /= 2) {
    const size_t fixed = ptile_bytes(rt, 0, d.C);
    if (fixed >= budget) continue;
    const long long kh = ((long long)((budget - fixed) / (8ull * d.C)) - rt) / 64 * 64;
    if (kh >= 64) {
      d.pKH = (int)std::min<long long>(kh, d.K);
      return rt;
    }
  }
  return 0;
}

size_t posterior_smem_bytes(const Dims& d) { return ptile_bytes(d.pRT, d.pKH, d.C); }

cudaError_t launch_posterior(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                             const float* trans, const float* dur, const double* grad_logZ,
                             float* grad_em, float* start_marg, float* end_marg, cudaStream_t st,
                             float* seg_marg, int pj) {
  const size_t sm = posterior_smem_bytes(d);
  const bool pair = posterior_pair(d);
  const void* fn = pair ? (const void*)posterior_kernel<1, 1> : (const void*)posterior_kernel<4, 2>;
  if (sm > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
  }
  if (pair)
    posterior_kernel<1, 1><<<dim3(d.nck, d.B), 512, sm, st>>>(d, ws, lengths, trans, dur, grad_logZ,
                                                              grad_em, start_marg, end_marg,
                                                              seg_marg, pj);
  else
    posterior_kernel<4, 2><<<dim3(d.nck, d.B), 512, sm, st>>>(d, ws, lengths, trans, dur, grad_logZ,
                                                              grad_em, start_marg, end_marg,
                                                              seg_marg, pj);
  return cudaGetLastError();
}

}  // namespace semicrf
