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
    // lanes over the start offset ia, inner loop over the end offset jb
    float zmax = NEG_INF, sum = 0.f;
    const float* const lac = la + c * KP;
    const float* const lbc = lb + c * KP;
    const float* const ddc = dd + c * KP;
    for (int ia = lane; ia < K; ia += 32) {
      const float a = lac[ia];
      if (a == NEG_INF) continue;
      for (int jb = 0; jb < K - ia; ++jb) zmax = fmaxf(zmax, (a + lbc[jb]) + ddc[ia + jb]);
    }
    zmax = group_max(zmax, 32);
    const float Mz = (zmax == NEG_INF) ? 0.f : ceilf(zmax);
    for (int ia = lane; ia < K; ia += 32) {
      const float a = lac[ia] - Mz;
      if (a == NEG_INF) continue;
      for (int jb = 0; jb < K - ia; ++jb) sum += ex2((a + lbc[jb]) + ddc[ia + jb]);
    }
    sum = group_sum(sum, 32);
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

// Shared memory of cut_grid_kernel.
// Shared memory of cut_grid_kernel: every label's rows when they fit the
// budget, else one label's (cut_grid_per_label).
bool cut_grid_per_label(const Dims& d, size_t budget) {
  return 3ull * (d.K + 1) * d.C * sizeof(float) > budget;
}
size_t cut_grid_smem_bytes(const Dims& d, size_t budget) {
  return 3ull * (d.K + 1) * (cut_grid_per_label(d, budget) ? 1 : d.C) * sizeof(float);
}

namespace {

// Shared memory carve of posterior_kernel for a tile of RT boundaries.
// (With boundary projections pd holds the start terms of the tile's rows.)
// Segment ends: a tile's segments end on up to RT + K rows.  Those rows are
// staged KH at a time (KH = K: all at once; long durations: chunks of the
// duration range, each staging RT + KH rows), so the halo arrays hold
// R = RT + KH rows and, when chunked, the tile rows' own integer and
// fractional prefix sums have arrays of their own (tii, tsf).
struct PTile {
  double* dif;  // [RT][C]   St - E of each boundary and label
  float* tf;    // [RT][2C]  forward kept rows: p, acc
  float* pb;    // [RT][C]   backward p
  float* ab;    // [R][C]    backward acc of the staged segment-end rows
  int* ii;      // [R][C]    (Pb_r - Pb_lo) + S_int[r, c], exact integers
  float* sf;    // [R][C]    S_frac[r, c]
  float* vv;    // [RT][C]   suffix sums v of the tile
  float* fs;    // [RT]      f_s
  float* pd;    // [RT][C]   projection start terms of the tile's rows (0 without)
  int* tii;     // [RT][C]   ii of the tile rows (aliases ii when not chunked)
  float* tsf;   // [RT][C]   sf of the tile rows (aliases sf when not chunked)
};
__host__ __device__ __forceinline__ size_t ptile_bytes(int RT, int KH, int C, bool chunked) {
  const size_t R = (size_t)RT + KH;
  return (size_t)C * (28ull * RT + 12ull * R + (chunked ? 8ull * RT : 0)) + 4ull * RT;
}
__device__ __forceinline__ PTile ptile_carve(unsigned char* raw, int RT, int KH, int C,
                                             bool chunked) {
  PTile t;
  const size_t R = (size_t)RT + KH;
  t.dif = reinterpret_cast<double*>(raw);
  t.tf = reinterpret_cast<float*>(t.dif + (size_t)RT * C);
  t.pb = t.tf + (size_t)RT * 2 * C;
  t.ab = t.pb + (size_t)RT * C;
  t.ii = reinterpret_cast<int*>(t.ab + R * C);
  t.sf = reinterpret_cast<float*>(t.ii + R * C);
  t.vv = t.sf + R * C;
  t.fs = t.vv + (size_t)RT * C;
  t.pd = t.fs + RT;
  t.tii = t.ii;
  t.tsf = t.sf;
  if (chunked) {
    t.tii = reinterpret_cast<int*>(t.pd + (size_t)RT * C);
    t.tsf = reinterpret_cast<float*>(t.tii + (size_t)RT * C);
  }
  return t;
}

// One CTA per (checkpoint segment j, sequence b): every posterior whose start
// boundary lies in [t0, t1), written in the same per-segment layout as
// segment_kernel (suffix sums v in grad_em, per-segment totals, float64
// count partials), so finalize and the partial reduction are shared; here
// the per-segment total is the plain sum over the segment (finalize takes the
// running sum over segments), because the normaliser is continuous.
//
// The segment is cut into tiles of d.pRT boundaries, taken downwards (the
// suffix sums run that way).  A tile stages its kept rows, and the K rows
// after it that its segments end on, in shared memory with coalesced loads;
// then every (boundary, label), (duration, label) and (label, label) item is
// computed from shared memory.  Each thread keeps the duration and transition
// sums of its first NID / NIT items in registers across tiles (with 512
// threads that covers K C <= 8192 and C <= 128); the items beyond (long
// durations: K C up to 16384) add their per-tile sums to the float64
// partials.
template <int NID, int NIT>
__global__ void __launch_bounds__(512, NID > 4 ? 1 : 2)
    posterior_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                     const float* __restrict__ trans, const float* __restrict__ dur,
                     const double* __restrict__ grad_logZ, float* __restrict__ grad_em,
                     float* __restrict__ start_marg, float* __restrict__ end_marg,
                     float* __restrict__ seg_marg, int pj) {
  extern __shared__ __align__(16) unsigned char psh[];
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, nthr = blockDim.x;
  const int C = d.C, K = d.K, RT = d.pRT, KH = d.pKH;
  const bool chunked = KH < K;  // long durations: the segment ends come KH rows at a time
  const int L = lengths[b];
  if (L <= 0 || L > d.T) return;
  if (!posterior_from_kept(ws, d, b)) return;  // segment_kernel runs it
  const int t0 = j * d.delta;
  if (t0 >= L) return;
  const int t1 = min(t0 + d.delta, L);
  const size_t seg = (size_t)b * d.nck + j;
  const float gb = (float)(grad_logZ ? grad_logZ[b] : 1.0);
  const float M = *ws.tmax;  // max trans2, written by the rings
  const PTile tl = ptile_carve(psh, RT, KH, C, chunked);
  const float* pfr = kv_row(ws, d, b, 0, 0);  // row t: pfr + t*2C (p), + C (acc)
  const float* pbr = kv_row(ws, d, b, 1, 0);
  const double* kff = ws.kf + ((size_t)b * 2 + 0) * (d.T + 1);
  const double* kfb = ws.kf + ((size_t)b * 2 + 1) * (d.T + 1);
  const double* nc = ws.ncut + (size_t)b * d.ngrid;
  const int32_t* si = ws.sint + (size_t)b * d.Tstride * C;
  const float* sfp = ws.sfrac + (size_t)b * d.Tstride * C;
  const int nd = K * C, ntr = C * C;
  float accd[NID], acct[NIT];
#pragma unroll
  for (int m = 0; m < NID; ++m) accd[m] = 0.f;
#pragma unroll
  for (int m = 0; m < NIT; ++m) acct[m] = 0.f;
  double lacc = 0.0, lvs = 0.0;  // thread c < C: running suffix sum, sum of v

  for (int s_hi = t1; s_hi > t0; s_hi -= RT) {
    const int s_lo = max(t0, s_hi - RT);
    const int nr = s_hi - s_lo;
    const int nh = min(s_hi - 1 + K, L) - s_lo + 1;  // rows a segment of the tile ends on
    const bool first = (s_hi == t1);
    // bounds-check build: the tile fits its rows
    if (!SEMICRF_INB(ws.status, nr >= 1 && nr <= RT && nh <= RT + K, SITE_POST_TILE)) break;
    // ------------------------------------------------------------ stage the tile rows
    const double kb0 = kfb[s_lo];
    #pragma unroll 4
    for (int i = tid; i < nr * 2 * C; i += nthr) tl.tf[i] = pfr[(size_t)s_lo * 2 * C + i];
    #pragma unroll 4
    for (int i = tid; i < nr * C; i += nthr) {
      const int r = i / C, c = i - r * C;
      const size_t row = (size_t)(s_lo + r);
      tl.pb[i] = pbr[row * 2 * C + c];
      tl.pd[i] = pj ? ws.pd[((size_t)b * d.Tstride + row) * C + c] : 0.f;
      if (chunked) {
        tl.tii[i] = (int)(kfb[row] - kb0) + si[row * C + c];
        tl.tsf[i] = sfp[row * C + c];
      }
    }
    // f_s = 2^(Pf_s + Pb_s + M - log2 Z(s))
    for (int s = s_lo + tid; s < s_hi; s += nthr)
      tl.fs[s - s_lo] = ex2((float)(((kff[s] + kfb[s]) + (double)M) - local_logz(d, nc, L, min(s, L - 1))));
    // ------------------------------------------------------------ segment ends, by chunk
    // chunk kc: durations [kc, kc + KH), staged rows at offsets [kc - 1, kc - 1 + nr + KH)
    // from s_lo (the first chunk includes the tile rows themselves)
    for (int kc = 1; kc <= K; kc += KH) {
      const int base = kc - 1;
      const int nst = max(0, min(base + nr + KH, nh) - base);
      if (kc > 1) __syncthreads();  // the previous chunk's reads are done
      #pragma unroll 4
      for (int i = tid; i < nst * C; i += nthr) {
        const int r = i / C, c = i - r * C;
        const size_t row = (size_t)(s_lo + base + r);
        tl.ab[i] = pbr[row * 2 * C + C + c];
        tl.ii[i] = (int)(kfb[row] - kb0) + si[row * C + c];
        tl.sf[i] = sfp[row * C + c];
      }
      __syncthreads();
      if (kc == 1) {
        // ---------------------------------------------------------- start / end marginals
        for (int i = tid; i < nr * C; i += nthr) {
          const int r = i / C, c = i - r * C;
          const float f = tl.fs[r];
          const float St = tl.tf[r * 2 * C + C + c] * tl.pb[i] * f;
          const float E = tl.ab[i] * tl.tf[r * 2 * C + c] * f;
          const size_t ob = ((size_t)b * (d.T + 1) + s_lo + r) * C + c;
          if (start_marg) start_marg[ob] = St;
          if (end_marg) end_marg[ob] = E;
          tl.dif[i] = (double)St - (double)E;
        }
      }
      const int lo_i = base * C, hi_i = min(nd, (base + KH) * C);  // this chunk's (k, c) items
      // -------------------------------------------------------- segment marginals
      // (optional output) P([s, s+k), c) for every start of the tile, the same
      // product as the duration counts below, not scaled by g (a marginal)
      if (seg_marg) {
        const int nci = hi_i - lo_i;
        for (int i = tid; i < nr * nci; i += nthr) {
          const int r = i / nci, idx = lo_i + (i - r * nci);
          const int k = idx / C + 1, c = idx - (k - 1) * C;
          if (s_lo + r + k > L) continue;
          if (!SEMICRF_INB(ws.status, r + k - base < nst, SITE_POST_ITEM)) continue;
          const int o = r * C + c, ok = (r + k - base) * C + c;
          const float z = (float)(tl.ii[ok] - tl.tii[o]) +
                          ((M + __ldg(dur + idx) * l2e()) + ((tl.sf[ok] - tl.tsf[o]) + tl.pd[o]));
          seg_marg[((size_t)b * d.T + s_lo + r) * nd + idx] =
              tl.tf[r * 2 * C + C + c] * tl.ab[ok] * (tl.fs[r] * ex2(z));
        }
      }
      // -------------------------------------------------------- duration counts
      // item (k, c): sum over the tile's s of P([s, s+k), c), s + k <= L
      auto dur_item = [&](int idx) {
        const int k = idx / C + 1, c = idx - (k - 1) * C;
        const float dk = M + __ldg(dur + idx) * l2e();
        int r_end = min(s_hi, L - k + 1) - s_lo;
        if (!SEMICRF_INB(ws.status, r_end <= 0 || r_end - 1 + k - base < nst, SITE_POST_ITEM))
          r_end = 0;
        // two accumulators and an unrolled loop: independent terms overlap
        // their shared-memory loads and exponentials
        float a0 = 0.f, a1 = 0.f;
        int r = 0;
#pragma unroll 2
        for (; r + 1 < r_end; r += 2) {
          const int o = r * C + c, ok = (r + k - base) * C + c;
          const float z0 = (float)(tl.ii[ok] - tl.tii[o]) + (dk + ((tl.sf[ok] - tl.tsf[o]) + tl.pd[o]));
          const float z1 = (float)(tl.ii[ok + C] - tl.tii[o + C]) +
                           (dk + ((tl.sf[ok + C] - tl.tsf[o + C]) + tl.pd[o + C]));
          a0 = fmaf(tl.tf[r * 2 * C + C + c] * tl.ab[ok], tl.fs[r] * ex2(z0), a0);
          a1 = fmaf(tl.tf[(r + 1) * 2 * C + C + c] * tl.ab[ok + C], tl.fs[r + 1] * ex2(z1), a1);
        }
        if (r < r_end) {
          const int o = r * C + c, ok = (r + k - base) * C + c;
          const float z = (float)(tl.ii[ok] - tl.tii[o]) + (dk + ((tl.sf[ok] - tl.tsf[o]) + tl.pd[o]));
          a0 = fmaf(tl.tf[r * 2 * C + C + c] * tl.ab[ok], tl.fs[r] * ex2(z), a0);
        }
        return a0 + a1;
      };
#pragma unroll
      for (int m = 0; m < NID; ++m) {
        const int idx = tid + m * nthr;
        if (idx >= lo_i && idx < hi_i) accd[m] += dur_item(idx);
      }
      for (int idx = tid + NID * nthr; idx < hi_i; idx += nthr) {
        if (idx < lo_i) continue;
        double* pd = ws.pgd + seg * nd + idx;
        const double v = (double)(gb * dur_item(idx));
        *pd = first ? v : *pd + v;
      }
    }
    // item (c', c): sum over the tile's s of P(c' -> c at s) / w[c', c]
    auto tr_item = [&](int idx) {
      const int c1 = idx / C, c = idx - c1 * C;
      float a0 = 0.f, a1 = 0.f;
      int r = 0;
#pragma unroll 4
      for (; r + 1 < nr; r += 2) {
        a0 = fmaf(tl.tf[r * 2 * C + c1] * tl.fs[r], tl.pb[r * C + c], a0);
        a1 = fmaf(tl.tf[(r + 1) * 2 * C + c1] * tl.fs[r + 1], tl.pb[(r + 1) * C + c], a1);
      }
      if (r < nr) a0 = fmaf(tl.tf[r * 2 * C + c1] * tl.fs[r], tl.pb[r * C + c], a0);
      return a0 + a1;
    };
#pragma unroll
    for (int m = 0; m < NIT; ++m)
      if (tid + m * nthr < ntr) acct[m] += tr_item(tid + m * nthr);
    for (int idx = tid + NIT * nthr; idx < ntr; idx += nthr) {
      double* pt = ws.pgt + seg * ntr + idx;
      const double v = (double)(gb * tr_item(idx) * ex2(__ldg(trans + idx) * l2e() - M));
      *pt = first ? v : *pt + v;
    }
    __syncthreads();
    // ------------------------------------------------------------ suffix sums
    // v[s] = sum of (St - E) over the segment's boundaries after s
    if (tid < C) {
      for (int r = nr - 1; r >= 0; --r) {
        tl.vv[r * C + tid] = (float)lacc;
        lvs += (double)(float)lacc;
        lacc += tl.dif[r * C + tid];
      }
    }
    __syncthreads();
    for (int i = tid; i < nr * C; i += nthr) grad_em[((size_t)b * d.T + s_lo) * C + i] = tl.vv[i];
  }
  // register items: the segment's partials
#pragma unroll
  for (int m = 0; m < NID; ++m)
    if (tid + m * nthr < nd) ws.pgd[seg * nd + tid + m * nthr] = (double)(gb * accd[m]);
#pragma unroll
  for (int m = 0; m < NIT; ++m) {
    const int idx = tid + m * nthr;
    if (idx < ntr) ws.pgt[seg * ntr + idx] = (double)(gb * acct[m] * ex2(__ldg(trans + idx) * l2e() - M));
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
// `budget` bytes, preferring tiles that leave room for two CTAs per SM.
// Long durations: the segment ends are staged in chunks of KH rows (a
// multiple of 64), the tile as tall as fits.  Sets d.pKH; 0 if nothing fits.
int posterior_tile_rows(Dims& d, size_t budget) {
  int cap = 64;
  while (cap > 8 && cap / 2 >= d.delta) cap /= 2;
  d.pKH = d.K;
  for (const size_t lim : {std::min<size_t>(budget, 112u * 1024u), budget})
    for (int rt = cap; rt >= 8; rt /= 2)
      if (ptile_bytes(rt, d.K, d.C, false) <= lim) return rt;
  for (int rt = cap; rt >= 8; rt /= 2) {
    const size_t fixed = ptile_bytes(rt, 0, d.C, true);
    if (fixed >= budget) continue;
    const long long kh = ((long long)((budget - fixed) / (12ull * d.C)) - rt) / 64 * 64;
    if (kh >= 64) {
      d.pKH = (int)std::min<long long>(kh, d.K);
      return rt;
    }
  }
  return 0;
}

size_t posterior_smem_bytes(const Dims& d) {
  return ptile_bytes(d.pRT, d.pKH, d.C, d.pKH < d.K);
}

cudaError_t launch_posterior(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                             const float* trans, const float* dur, const double* grad_logZ,
                             float* grad_em, float* start_marg, float* end_marg, cudaStream_t st,
                             float* seg_marg, int pj) {
  const size_t sm = posterior_smem_bytes(d);
  const bool small = (size_t)d.K * d.C <= 4u * 512u && (size_t)d.C * d.C <= 4u * 512u;
  const void* fn = small ? (const void*)posterior_kernel<4, 4> : (const void*)posterior_kernel<16, 32>;
  if (sm > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
  }
  if (small)
    posterior_kernel<4, 4><<<dim3(d.nck, d.B), 512, sm, st>>>(d, ws, lengths, trans, dur, grad_logZ,
                                                              grad_em, start_marg, end_marg,
                                                              seg_marg, pj);
  else
    posterior_kernel<16, 32><<<dim3(d.nck, d.B), 512, sm, st>>>(d, ws, lengths, trans, dur, grad_logZ,
                                                                grad_em, start_marg, end_marg,
                                                                seg_marg, pj);
  return cudaGetLastError();
}

}  // namespace semicrf
