// viterbi.cu -- step 4: max-semiring decoding.
//
// The forward recursion of recursion.cu with max in place of log-sum-exp:
//   G[s, c] = max_{c'} V[s, c'] + trans[c', c]             (G[0, c] = 0)
//   V[t, c] = max_{k <= min(K,t)} G[t-k, c] + S[t,c] - S[t-k,c] + dur[k-1,c]
// with the same exact integer frames, base-2 units and K-slot ring.  Ties go
// to the smallest k and then the smallest c' (first maximum in ascending
// order within a lane, then the smaller index across lanes), and at the end to
// the smallest final label.  Backpointers are packed per (boundary, label):
// bits 0-15 the best duration of a segment ending there, bits 16-31 the best
// previous label of a segment starting there.  One warp then walks them back
// from the best final label.
#include "kernels.cuh"

namespace semicrf {

namespace {

struct VSmem {
  uint64_t* mbar;
  int* maxslot;
  int32_t* tint;
  float* tfrac;
  float2* ring;
  float* Vcur;
  int* kbest;
  int* Sbase;
};

__device__ VSmem vcarve(unsigned char* raw, const Dims& d) {
  VSmem s;
  const int C = d.C;
  unsigned char* p = raw;
  s.mbar = reinterpret_cast<uint64_t*>(p);
  s.maxslot = reinterpret_cast<int*>(p + 16);
  p += 64;
  s.tint = reinterpret_cast<int32_t*>(p);
  p += 2ull * TS * C * sizeof(int32_t);
  s.tfrac = reinterpret_cast<float*>(p);
  p += 2ull * TS * C * sizeof(float);
  s.ring = reinterpret_cast<float2*>(p);
  p += (size_t)d.K * C * sizeof(float2);
  s.Vcur = reinterpret_cast<float*>(p);
  s.kbest = reinterpret_cast<int*>(s.Vcur + C);
  s.Sbase = s.kbest + C;
  return s;
}

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

__global__ void __launch_bounds__(NT_MAX, 1)
    viterbi_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                   const float* __restrict__ trans, const float* __restrict__ dur,
                   double* __restrict__ score, int32_t* __restrict__ labels,
                   uint8_t* __restrict__ seg_start) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const VSmem sm = vcarve(smem_raw, d);
  const int C = d.C, K = d.K, T = d.T, tid = threadIdx.x;
  const int b = blockIdx.x;
  int L = lengths[b];
  const bool bad = (L < 0 || L > T);
  // positions past the length (all of them for a bad length)
  for (int u = (bad ? 0 : L) + tid; u < T; u += blockDim.x) {
    labels[(size_t)b * T + u] = -1;
    seg_start[(size_t)b * T + u] = 0;
  }
  if (bad) {
    if (tid == 0) {
      set_status(ws.status, ST_BAD_LENGTH);
      score[b] = __longlong_as_double(0x7ff8000000000000ll);
    }
    return;
  }
  if (L == 0) {
    if (tid == 0) score[b] = 0.0;
    return;
  }
  const int GB = d.GB, GA = d.GA;
  const int cB = tid / GB, jB = tid % GB, cA = tid / GA, jA = tid % GA;
  const bool warpB = ((tid & ~31) / GB) < C, warpA = ((tid & ~31) / GA) < C;
  const float l2e = (float)LOG2E_D;
  float dreg[KB_MAX], treg[CA_MAX];
  {
    const int c = cB < C ? cB : 0;
#pragma unroll
    for (int i = 0; i < KB_MAX; ++i) {
      const int k = 1 + jB + i * GB;
      dreg[i] = (i < d.KB && k <= K) ? __ldg(dur + (size_t)(k - 1) * C + c) * l2e : NEG_INF;
    }
    const int o = cA < C ? cA : 0;
#pragma unroll
    for (int i = 0; i < CA_MAX; ++i) {
      const int x = jA + i * GA;
      treg[i] = (i < d.CA && x < C) ? __ldg(trans + (size_t)x * C + o) * l2e : NEG_INF;
    }
  }
  if (tid == 0) {
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    fence_mbar_init();
    sm.maxslot[0] = f2ord(NEG_INF);
    sm.maxslot[1] = f2ord(NEG_INF);
  }
  for (int c = tid; c < C; c += blockDim.x) {
    sm.ring[c] = make_float2(0.f, 0.f);
    sm.Sbase[c] = 0;
  }
  __syncthreads();
  int32_t* bp = ws.bp + (size_t)b * (T + 1) * C;
  // tile stream (same protocol as the recursion kernels)
  const int lo = 0, hi = L / TS;
  uint32_t ph[2] = {0u, 0u};
  int cur = -1;
  auto issue = [&](int i) {
    if (i < lo || i > hi || tid != 0) return;
    const int buf = i & 1;
    const uint32_t bytes = (uint32_t)(TS * C * 4);
    const size_t row0 = (size_t)b * d.Tstride + (size_t)i * TS;
    fence_proxy_async();
    mbar_expect_tx(&sm.mbar[buf], 2 * bytes);
    bulk_g2s(sm.tint + (size_t)buf * TS * C, ws.sint + row0 * C, bytes, &sm.mbar[buf]);
    bulk_g2s(sm.tfrac + (size_t)buf * TS * C, ws.sfrac + row0 * C, bytes, &sm.mbar[buf]);
  };
  issue(0);  // entering a tile issues the next one
  double F0 = 0.0;
  float Frel = 0.f;
  int tb = 0;
  for (int t = 1; t <= L; ++t) {
    tb = (tb + 1 == K) ? 0 : tb + 1;
    const int ti = t / TS;
    if (ti != cur) {
      const int buf = ti & 1;
      bool ok = mbar_wait(&sm.mbar[buf], ph[buf], WAIT_SPIN_LIMIT);
      ph[buf] ^= 1u;
      cur = ti;
      issue(ti + 1);
      if (__syncthreads_or(!ok)) {
        if (tid == 0) {
          set_status(ws.status, ST_DEVICE_TIMEOUT);
          for (int q = 0; q < 2; ++q) mbar_wait(&sm.mbar[q], ph[q], WAIT_SPIN_LIMIT);
        }
        return;
      }
    }
    const size_t ro = ((size_t)(ti & 1) * TS + (t - ti * TS)) * C;
    const int32_t* ri = sm.tint + ro;
    const float* rf = sm.tfrac + ro;
    if (t % d.delta == 0) {
      // rebase the integer frames (keeps every stored integer small)
      const float dF = Frel;
      for (int idx = tid; idx < K * C; idx += blockDim.x) {
        const int i = idx / C, c = idx % C;
        if (t - K + i < 0) continue;
        int slot = tb + i;
        if (slot >= K) slot -= K;
        float2 v = sm.ring[slot * C + c];
        v.y = (v.y - dF) + (float)(ri[c] - sm.Sbase[c]);
        sm.ring[slot * C + c] = v;
      }
      __syncthreads();
      for (int c = tid; c < C; c += blockDim.x) sm.Sbase[c] = ri[c];
      F0 += (double)dF;
      Frel = 0.f;
      __syncthreads();
    }
    const int par = t & 1;
    if (warpB) {
      const bool act = cB < C;
      const int c = act ? cB : 0;
      const float Q = (float)(ri[c] - sm.Sbase[c]) - Frel;
      const int kmax = min(K, t);
      float best = NEG_INF;
      int bk = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < KB_MAX; ++i) {
        const int k = 1 + jB + i * GB;
        if (i < d.KB && act && k <= kmax) {
          int slot = tb - k;
          if (slot < 0) slot += K;
          const float2 v = sm.ring[slot * C + c];
          const float y = ((v.y + Q) + v.x) + dreg[i];
          if (y > best || bk == 0x7fffffff) {
            best = y;
            bk = k;
          }
        }
      }
      group_argmax(best, bk, GB);
      if (act && jB == 0) {
        const float V = rf[c] + best;
        sm.Vcur[c] = V;
        sm.kbest[c] = bk;
        atomicMax(&sm.maxslot[par], f2ord(V));
      }
    }
    __syncthreads();
    const float M = ord2f(sm.maxslot[par]);
    const float n = isfinite(M) ? rintf(M) : 0.f;
    if (tid == 0) sm.maxslot[par ^ 1] = f2ord(NEG_INF);
    if (t == L) break;
    if (warpA) {
      const bool act = cA < C;
      float best = NEG_INF;
      int bc = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < CA_MAX; ++i) {
        const int x = jA + i * GA;
        if (i < d.CA && act && x < C) {
          const float v = sm.Vcur[x] + treg[i];
          if (v > best || bc == 0x7fffffff) {
            best = v;
            bc = x;
          }
        }
      }
      group_argmax(best, bc, GA);
      if (act && jA == 0) {
        const int c = cA;
        const float g = best - n;
        sm.ring[tb * C + c] = make_float2(g - rf[c], (Frel + n) - (float)(ri[c] - sm.Sbase[c]));
        bp[(size_t)t * C + c] = (sm.kbest[c] & 0xffff) | (bc << 16);
      }
    }
    Frel += n;
    __syncthreads();
  }
  // best final label (smallest on ties), score, then the traceback
  if (tid < 32) {
    float best = NEG_INF;
    int bc = 0x7fffffff;
    for (int c = tid; c < C; c += 32) {
      const float v = sm.Vcur[c];
      if (v > best || bc == 0x7fffffff) {
        best = v;
        bc = c;
      }
    }
    group_argmax(best, bc, 32);
    if (tid == 0) score[b] = (F0 + (double)Frel + (double)best) * LN2_D;
    int t = L, c = bc;
    int kL = sm.kbest[bc];
    while (t > 0) {
      const int k = (t == L) ? kL : (bp[(size_t)t * C + c] & 0xffff);
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

}  // namespace semicrf
