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

template <int KBT, int CAT, int G, int LB>
__global__ void __launch_bounds__(LB, 1)
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
  Lane<KBT, CAT, G> ln;
  ln.init_ids(d);
  ln.init_dur(d, dur, true);
  // raw trans2 column values for this lane's previous labels (no exponentials)
  float tr[CAT];
#pragma unroll
  for (int i = 0; i < CAT; ++i) {
    const int x = ln.j * CAT + i;
    tr[i] = (ln.act && x < C) ? __ldg(trans + (size_t)x * C + ln.cc) * l2e() : NEG_INF;
  }
  float2* const rl = sm.ring + (size_t)ln.cc * d.RL;
  const bool pj = proj_on(ws);  // boundary projections
  init_smem(sm, d);
  __syncthreads();
  for (int c = tid; c < C; c += blockDim.x) {
    ring_put<KBT>(sm.ring + (size_t)c * d.RL, d, 0, make_float2(proj_d(ws, d, pj, b, 0, c), 0.f));
    sm.Sbase[c] = 0;
  }
  __syncthreads();
  int32_t* bp = ws.bp + (size_t)b * (T + 1) * C;
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  tile_start(sm, d, ws, b, ts, 1, 1, L, +1);
  double F0 = 0.0;
  float Frel = 0.f;
  int Sb = 0;
  int wslot = 0, par = 0, q = 0;
  int base = ln.base_up(1, K);
  int to_ck = d.delta;
  int bk = 0;
  int cur = -1, t = 1;
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
    const int t_stop = min(L, ti * TS + TS - 1);
    const size_t off = tile_row_off(t, C);
    const int32_t* ri = sm.tint + off;
    const float* rf = sm.tfrac + off;
    for (; t <= t_stop; ++t, ri += C, rf += C) {
      if (t > 1) base = (base + 1 == K) ? 0 : base + 1;
      wslot = (wslot + 1 == K) ? 0 : wslot + 1;
      par = t & 1;
      q = mod3_next(q);
      if (--to_ck == 0) {
        // rebase the integer frames (keeps every stored integer small)
        to_ck = d.delta;
        __syncthreads();
        for (int idx = tid; idx < C * d.RL; idx += blockDim.x) {
          const int c = idx / d.RL;
          float2 v = sm.ring[idx];
          v.y = (v.y - Frel) + (float)(ri[c] - sm.Sbase[c]);
          sm.ring[idx] = v;
        }
        __syncthreads();
        for (int c = tid; c < C; c += blockDim.x) sm.Sbase[c] = ri[c];
        F0 += (double)Frel;
        Frel = 0.f;
        Sb = ri[ln.cc];
        __syncthreads();
      }
      const int si = ri[ln.cc];
      const float sf = rf[ln.cc];
      {
        const float Q = (float)(si - Sb) - Frel;
        const float2* r = rl + base;
        // the lane's window in its rotated order (Lane::widx); ties go to
        // the smallest k
        float best = NEG_INF;
        bk = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < KBT; ++i) {
          const int w = ln.widx(i);
          const float2 v = r[w];
          const float y = ((v.y + Q) + v.x) + ln.d[i];
          const int k = ln.k_of(w, true);
          if (y > best || (y == best && k < bk) || bk == 0x7fffffff) {
            best = y;
            bk = k;
          }
        }
        gargmax<G>(best, bk);
        const float V = sf + best;
        if (ln.leader) sm.Acur[par * C + ln.c] = V;
        warp_max_to_shared(&sm.maxslot[q], ln.leader ? f2ord(V) : INT_MIN);
      }
      __syncthreads();
      bool slow;
      const float n = step_frame(sm, q, slow);
      if (t == L) {
        done = true;
        break;
      }
      {
        const float* V = sm.Acur + par * C;
        float best = NEG_INF;
        int bc = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < CAT; ++i) {
          const int x = ln.j * CAT + i;
          const float vx = (x < C) ? V[x] + tr[i] : NEG_INF;
          if (vx > best || bc == 0x7fffffff) {
            best = vx;
            bc = x;
          }
        }
        gargmax<G>(best, bc);
        if (ln.leader) {
          ring_put<KBT>(rl, d, wslot, make_float2(((best - n) - sf) + proj_d(ws, d, pj, b, t, ln.c),
                                                  (Frel + n) - (float)(si - Sb)));
          bp[(size_t)t * C + ln.c] = (bk & 0xffff) | (bc << 16);
        }
      }
      __syncwarp();
      Frel += n;
    }
  }
  // the last step's best durations, then the best final label (smallest on ties)
  if (ln.leader) bp[(size_t)L * C + ln.c] = bk & 0xffff;
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
    gargmax<32>(best, bc);
    if (tid == 0) score[b] = (F0 + (double)Frel + (double)best) * LN2_D;
    int tt = L, c = bc;
    while (tt > 0) {
      const int k = bp[(size_t)tt * C + c] & 0xffff;
      if (k < 1 || k > tt) {  // impossible for backpointers this kernel wrote
        for (int u = tid; u < tt; u += 32) labels[(size_t)b * T + u] = -1;
        break;
      }
      const int s = tt - k;
      for (int u = s + tid; u < tt; u += 32) {
        labels[(size_t)b * T + u] = c;
        seg_start[(size_t)b * T + u] = (u == s) ? 1 : 0;
      }
      if (s > 0) {
        const int nc = (bp[(size_t)s * C + c] >> 16) & 0xffff;
        if (nc >= C) {  // impossible for backpointers this kernel wrote
          for (int u = tid; u < s; u += 32) labels[(size_t)b * T + u] = -1;
          break;
        }
        c = nc;
      }
      tt = s;
    }
  }
}

cudaError_t launch_viterbi(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                           const float* trans, const float* dur, double* score, int32_t* labels,
                           uint8_t* seg_start, cudaStream_t st) {
  const size_t sm = recursion_smem_bytes(d, false);
#define SEMICRF_LAUNCH_VIT(a, b, g, lb)                                                      \
  if (d.KBT == a && d.CAT == b && d.GB == g && d.LB == lb) {                                 \
    if (sm > 48 * 1024) {                                                                    \
      const cudaError_t e = cudaFuncSetAttribute(viterbi_kernel<a, b, g, lb>,                \
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                                 (int)sm);                                   \
      if (e != cudaSuccess) return e;                                                        \
    }                                                                                        \
    viterbi_kernel<a, b, g, lb><<<d.B, d.NT, sm, st>>>(d, ws, lengths, trans, dur, score,    \
                                                       labels, seg_start);                   \
    return cudaGetLastError();                                                               \
  }
  SEMICRF_FOR_EACH_SHAPE(SEMICRF_LAUNCH_VIT)
#undef SEMICRF_LAUNCH_VIT
  return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
