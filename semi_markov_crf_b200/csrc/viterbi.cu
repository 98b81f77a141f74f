// viterbi.cu -- step 4: max-semiring decoding.
//
// The forward recursion of recursion.cu with max in place of log-sum-exp:
//   G[s, c] = max_{c'} V[s, c'] + trans[c', c]             (G[0, c] = 0)
//   V[t, c] = max_{k <= min(K,t)} G[t-k, c] + S[t,c] - S[t-k,c] + dur[k-1,c]
// on the same mirrored K-slot ring, exact integer frames, base-2 units and
// one-barrier-per-step schedule.  Ties go to the smallest k and then the
// smallest c' (first maximum in ascending order within a lane, then the
// smaller index across lanes), and at the end to the smallest final label.
// Backpointers are packed per (boundary, label): bits 0-15 the best duration
// of a segment ending there, bits 16-31 the best previous label of a segment
// starting there.  One warp then walks them back from the best final label.
#include "ring.cuh"

namespace semicrf {

using namespace ring;

namespace {

// (value, index) max with ties to the smaller index, over aligned groups.
__device__ __forceinline__ void group_argmax(float& v, int& i, int G) {
  for (int o = G >> 1; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(FULL_MASK, v, o);
    const int i2 = __shfl_xor_sync(FULL_MASK, i, o);
    if (v2 > v || (v2 == v && i2 < i)) {
      v = v2;
      i = i2;
    }
  }
}

}  // namespace

template <int KBT, int CAT>
__global__ void __launch_bounds__(NT_MAX, 1)
    viterbi_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                   const float* __restrict__ trans, const float* __restrict__ dur,
                   double* __restrict__ score, int32_t* __restrict__ labels,
                   uint8_t* __restrict__ seg_start) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem sm = carve(smem_raw, d, false);
  const int C = d.C, K = d.K, T = d.T, tid = threadIdx.x;
  const int b = blockIdx.x;
  const int L = lengths[b];
  const bool bad = (L < 0 || L > T);
  // positions past the length (all of them for a bad length)
  for (int u = (bad ? 0 : L) + tid; u < T; u += blockDim.x) {
    labels[(size_t)b * T + u] = -1;
    seg_start[(size_t)b * T + u] = 0;
  }
  if (bad || L == 0) {
    if (tid == 0) {
      if (bad) set_status(ws.status, ST_BAD_LENGTH);
      score[b] = bad ? __longlong_as_double(0x7ff8000000000000ll) : 0.0;
    }
    return;
  }
  const bool warp_on = ((tid & ~31) / d.GB) < C;
  KLane<KBT> kl;
  kl.init(d, dur, true);
  // raw trans2 column values for this lane's previous labels (no exponentials)
  float tr[CAT];
#pragma unroll
  for (int i = 0; i < CAT; ++i) {
    const int x = kl.j * CAT + i;
    tr[i] = (kl.act && x < C) ? __ldg(trans + (size_t)x * C + kl.c) * l2e() : NEG_INF;
  }
  init_smem(sm, d);
  __syncthreads();
  for (int c = tid; c < C; c += blockDim.x) {
    ring_put<KBT>(sm, d, c, 0, make_float2(0.f, 0.f));
    sm.Sbase[c] = 0;
  }
  __syncthreads();
  int32_t* bp = ws.bp + (size_t)b * (T + 1) * C;
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  const int32_t* ri;
  const float* rf;
  tile_start(sm, d, ws, b, ts, 1, 0, L, +1);
  double F0 = 0.0;
  float Frel = 0.f;
  int slot = 0, par = 0, q = 0;
  int base = kl.base_up(1, K);
  int to_ck = d.delta;
  int bk = 0;
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
      // rebase the integer frames (keeps every stored integer small)
      to_ck = d.delta;
      __syncthreads();
      const float dF = Frel;
      for (int idx = tid; idx < C * d.RL; idx += blockDim.x) {
        const int c = idx / d.RL;
        float2 v = sm.ring[idx];
        v.y = (v.y - dF) + (float)(ri[c] - sm.Sbase[c]);
        sm.ring[idx] = v;
      }
      __syncthreads();
      for (int c = tid; c < C; c += blockDim.x) sm.Sbase[c] = ri[c];
      F0 += (double)dF;
      Frel = 0.f;
      __syncthreads();
    }
    if (warp_on) {
      const int c = kl.act ? kl.c : 0;
      const float Q = (float)(ri[c] - sm.Sbase[c]) - Frel;
      const float2* r = sm.ring + (size_t)c * d.RL + base;
      // lane term i has k = (j+1)*KBT - i: walk i downwards for ascending k
      float best = NEG_INF;
      bk = 0x7fffffff;
#pragma unroll
      for (int i = KBT - 1; i >= 0; --i) {
        const float2 v = r[i];
        const float y = ((v.y + Q) + v.x) + kl.d[i];
        if (y > best || bk == 0x7fffffff) {
          best = y;
          bk = kl.k_of(i, true);
        }
      }
      group_argmax(best, bk, d.GB);
      int key = INT_MIN;
      if (kl.act && kl.j == 0) {
        const float V = rf[c] + best;
        sm.Acur[par * C + c] = V;
        key = f2ord(V);
      }
      warp_max_to_shared(&sm.maxslot[q], key);
    }
    __syncthreads();
    bool slow;
    const float n = step_frame(sm, q, slow);
    if (t == L) break;
    if (warp_on) {
      const float* V = sm.Acur + par * C;
      float best = NEG_INF;
      int bc = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < CAT; ++i) {
        const int x = kl.j * CAT + i;
        const float vx = (x < C) ? V[x] + tr[i] : NEG_INF;
        if (vx > best || bc == 0x7fffffff) {
          best = vx;
          bc = x;
        }
      }
      group_argmax(best, bc, d.GB);
      if (kl.act && kl.j == 0) {
        const int c = kl.c;
        const float g = best - n;
        ring_put<KBT>(sm, d, c, slot,
                      make_float2(g - rf[c], (Frel + n) - (float)(ri[c] - sm.Sbase[c])));
        bp[(size_t)t * C + c] = (bk & 0xffff) | (bc << 16);
      }
      __syncwarp();
    }
    Frel += n;
  }
  // the last step's best durations, then the best final label (smallest on ties)
  if (kl.act && kl.j == 0) bp[(size_t)L * C + kl.c] = bk & 0xffff;
  __syncthreads();
  if (tid < 32) {
    const float* V = sm.Acur + par * C;
    float best = NEG_INF;
    int bc = 0x7fffffff;
    for (int c = tid; c < C; c += 32) {
      const float v = V[c];
      if (v > best || bc == 0x7fffffff) {
        best = v;
        bc = c;
      }
    }
    group_argmax(best, bc, 32);
    if (tid == 0) score[b] = (F0 + (double)Frel + (double)best) * LN2_D;
    int t = L, c = bc;
    while (t > 0) {
      const int k = bp[(size_t)t * C + c] & 0xffff;
      const int s = t - k;
      for (int u = s + tid; u < t; u += 32) {
        labels[(size_t)b * T + u] = c;
        seg_start[(size_t)b * T + u] = (u == s) ? 1 : 0;
      }
      if (s > 0) c = (bp[(size_t)s * C + c] >> 16) & 0xffff;
      t = s;
    }
  }
}

cudaError_t launch_viterbi(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                           const float* trans, const float* dur, double* score, int32_t* labels,
                           uint8_t* seg_start, cudaStream_t st) {
  const size_t sm = recursion_smem_bytes(d, false);
#define SEMICRF_LAUNCH_VIT(a, b)                                                               \
  if (d.KBT == a && d.CAT == b) {                                                              \
    if (sm > 48 * 1024) {                                                                      \
      const cudaError_t e = cudaFuncSetAttribute(viterbi_kernel<a, b>,                         \
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                                 (int)sm);                                     \
      if (e != cudaSuccess) return e;                                                          \
    }                                                                                          \
    viterbi_kernel<a, b><<<d.B, d.NT, sm, st>>>(d, ws, lengths, trans, dur, score, labels,     \
                                                seg_start);                                    \
    return cudaGetLastError();                                                                 \
  }
  SEMICRF_FOR_EACH_SHAPE(SEMICRF_LAUNCH_VIT)
#undef SEMICRF_LAUNCH_VIT
  return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
