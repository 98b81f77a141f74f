// viterbi_pipe.cu -- step 4: max-semiring decoding, pipelined.
//
// The recursion of viterbi.cu (base-2 units, exact integer frames):
//   G[s, c] = max_{c'} V[s, c'] + trans2[c', c]                 (G[0, c] = 0)
//   V[t, c] = S[t,c] + max_{k <= min(K,t)} G[t-k, c] - S[t-k, c] + dur2[k-1, c]
// organised around its real dependency: only the k = 1 term of V[t] needs
// G[t-1], which needs all of V[t-1, :]; the k = 2 term needs G[t-2] (known a
// step earlier) and the k >= 3 terms only ring entries written two or more
// steps before.
//
// Roles (one CTA per sequence).  Combine warps (G lanes per label, CAT
// source labels per lane) run only the critical path of step t: read
// V[t-1, :], take max_{c'} V + trans2 for their label, compare it with the
// step's precomputed candidates, store V[t] and the chosen duration, write
// G[t-1] into the label's ring.  Helper warps (H lanes per label, KBH
// durations per lane, strided over the window so that a label's lanes read
// consecutive ring entries) compute during step t everything else: the best
// k >= 3 term of step t+1 and its k and the additive constants of its k = 1
// and k = 2 terms; they never read the row V[t-1], so in a cluster they
// finish before the exchange brings it.  One barrier per step.
//
// Frames: V[t, :] is stored relative to Phi_t with Phi_t = rint(max V[t-2])
// (absolute): n_t = rint(m_{t-2}) - n_{t-1}, m the max every combine group
// takes of the row it reads for the label fan-in (one step before it is
// used), so the reduction runs beside the fan-in's and the frame follows the
// maximum two steps late without oscillating.
//
// Ties: k = 1 before k = 2 before the helpers' best k (itself the smallest
// k among equal terms), the smallest c' among equal label terms, and the
// smallest final label.
//
// Decoding: no argmax label is computed during the recursion.  The combine
// leaders write out, at the end of each step, the boundary's row of V
// (relative to its frame) and of chosen durations.  The traceback needs the
// best previous label only
// where a decoded segment starts, and recomputes it there from the kept row:
// argmax_{c'} V[s, c'] + trans2[c', c] is the same float sum the combine
// compared (the frame shifts every term alike), so the result, ties
// included, is the recursion's own.
#include <algorithm>

#include "ring.cuh"

namespace semicrf {

using namespace ring;

namespace {

constexpr int VREBASE = 4096;  // steps between integer rebases (keeps y exact)

// Per-label arrays cover the CTA's own labels (Cr = xCr of them, local
// index); V holds the whole row in every CTA of a cluster.
struct VSmem {
  Smem s;      // mbar, tint, tfrac (every label), ring (own labels)
  float* V;    // [2][xPC]  V of the step of that parity (-inf padded, all labels)
  float* Om;   // [HW][2][Cr] helpers' best k >= 3 candidate, frame Phi_{t-2}, one per
               // helper warp of a label (HW = ceil(xH / 32))
  int* Ok;     // [HW][2][Cr] its duration
  float* A1;   // [2][Cr]   dur2[0] + S[t] - S[t-1]
  float* A2;   // [2][Cr]   dur2[1] + S[t] - S[t-2]
  float* nsl;  // [2]       frame step published by the combine warps
  int* Sb;     // [Cr]      label integer bases
  uint64_t* vbar;  // [2]   cluster: arrival of the step's V row, by step parity
};

__device__ __forceinline__ VSmem vcarve(unsigned char* raw, const Dims& d, bool pj) {
  VSmem x;
  const int C = d.C, Cr = d.xCr;
  unsigned char* p = raw;
  x.s.mbar = reinterpret_cast<uint64_t*>(p);
  x.s.maxslot = reinterpret_cast<int*>(p + 16);
  x.s.aux = reinterpret_cast<int*>(p + 32);
  x.nsl = reinterpret_cast<float*>(p + 48);
  x.vbar = reinterpret_cast<uint64_t*>(p + 64);
  p += 96;
  x.s.tint = reinterpret_cast<int32_t*>(p);
  p += 2ull * TS * C * sizeof(int32_t);
  x.s.tfrac = reinterpret_cast<float*>(p);
  p += 2ull * TS * C * sizeof(float);
  x.s.tpd = nullptr;
  if (pj) {  // boundary projections: start terms stream with the prefix sums
    x.s.tpd = reinterpret_cast<float*>(p);
    p += 2ull * TS * C * sizeof(float);
  }
  x.s.ring = reinterpret_cast<float2*>(p);
  p += (size_t)d.xRLP * Cr * sizeof(float2);
  p = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 15) & ~uintptr_t(15));
  float* f = reinterpret_cast<float*>(p);
  x.V = f;
  f += 2 * d.xPC;
  const int hw = (d.xH + 31) / 32;
  x.Om = f;
  f += 2 * Cr * hw;
  x.Ok = reinterpret_cast<int*>(f);
  f += 2 * Cr * hw;
  x.A1 = f;
  f += 2 * Cr;
  x.A2 = f;
  f += 2 * Cr;
  x.Sb = reinterpret_cast<int*>(f);
  x.s.pcur = nullptr;
  x.s.Acur = nullptr;
  x.s.tmp = nullptr;
  x.s.Sbase = x.Sb;
  x.s.store = nullptr;
  return x;
}

// Dynamic shared memory of the kernel (carve order of vcarve).
__host__ __device__ __forceinline__ size_t vsmem_bytes(const Dims& d, bool pj) {
  const size_t hw = (d.xH + 31) / 32;  // helper warps per label (long durations: > 1)
  return 96 + 2ull * TS * d.C * (pj ? 12 : 8) + (size_t)d.xRLP * d.xCr * 8 + 16 +
         (2ull * d.xPC + (5ull + 4 * hw) * d.xCr) * 4;
}

// Bounded wait for prefix-sum tile `ti`; false (uniformly) if it gave up.
__device__ __forceinline__ bool vtile_wait(const Smem& sm, TileStream& ts, int ti) {
  const int buf = ti & 1;
  bool ok = mbar_wait(&sm.mbar[buf], ts.ph[buf], WAIT_SPIN_LIMIT);
  ts.ph[buf] ^= 1u;
  return !__syncthreads_or(!ok);
}

// Smallest i' > i with i' % TS == rem.
__device__ __forceinline__ int next_with_rem(int i, int rem) {
  int x = (i / TS) * TS + rem;
  return x > i ? x : x + TS;
}

//
// With a cluster of N > 1 CTAs per sequence, CTA `rank` owns labels
// [rank*Cr, rank*Cr + Cr) (ring, k fan-in, label fan-in outputs); each
// combine group sends its V[t] into the V buffer of every CTA of the cluster
// with asynchronous distributed-shared-memory stores counted by the
// destination's arrival barrier vbar[t & 1] (4 C bytes per step); a combine
// lane waits on it before reading V[t-1] and a thread off the combine path
// re-arms it at the top of step t+1 (the same exchange as the
// exponential-domain rings), so every CTA holds the whole row and takes the
// same frame.  Every CTA takes the same early exits
// (they depend only on the inputs).
template <int N, int G, int CAT, int H, int KBH, int LB>
__global__ void __launch_bounds__(LB, 1)
    viterbi_pipe_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                        const float* __restrict__ trans, const float* __restrict__ dur,
                        double* __restrict__ score, int32_t* __restrict__ labels,
                        uint8_t* __restrict__ seg_start, int pj) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const VSmem vs = vcarve(smem_raw, d, pj != 0);
  const Smem& sm = vs.s;
  const int C = d.C, K = d.K, T = d.T, Cr = d.xCr, tid = threadIdx.x;
  const int rank = N > 1 ? (int)cluster_ctarank() : 0;
  const int b = (int)blockIdx.x / N;
  const int L = lengths[b];
  const bool bad = (L < 0 || L > T);
  // positions past the length (all of them for a bad length)
  if (rank == 0)
    for (int u = (bad ? 0 : L) + tid; u < T; u += blockDim.x) {
      labels[(size_t)b * T + u] = -1;
      seg_start[(size_t)b * T + u] = 0;
    }
  if (bad || L == 0) {
    if (tid == 0 && rank == 0) {
      if (bad) set_status(ws.status, ST_BAD_LENGTH);
      score[b] = bad ? __longlong_as_double(0x7ff8000000000000ll) : 0.0;
    }
    return;
  }

  // ---------------------------------------------------------------- roles
  // Long durations: H > 32 lanes per label spread over HW = H / 32 helper
  // warps; each warp finds the best k >= 3 candidate of its share of the
  // window and the combine takes the best of the warps' candidates.
  constexpr int HG = H > 32 ? 32 : H;       // lanes per reduction group
  constexpr int HW = H > 32 ? H / 32 : 1;   // helper warps per label
  constexpr int LPWC = 32 / G, LPWH = 32 / HG, WL = H * KBH;
  constexpr int NR = CAT > KBH ? CAT : KBH;
  const int warp = tid >> 5, lane = tid & 31;
  const int nwc = (Cr + LPWC - 1) / LPWC;
  const bool comb = warp < nwc;
  const int c0 = rank * Cr;  // first label of this CTA
  const int hwi = warp - nwc;  // helper warp index
  const int cl = comb ? warp * LPWC + lane / G
                      : (HW > 1 ? hwi / HW : hwi * LPWH + lane / H);  // local label
  const int hwarp = HW > 1 && !comb ? hwi % HW : 0;  // this lane's warp among its label's
  const int c = c0 + cl;     // global label
  const int jl = comb ? lane % G : (HW > 1 ? hwarp * 32 + lane : lane % H);
  const bool act = cl < Cr && c < C;
  const int cc = act ? c : 0;     // global label (tile rows, parameters, outputs)
  const int ccl = act ? cl : 0;   // local label (ring, per-label arrays)
  const bool leader = act && jl == 0;
  const int RL = K + WL, RLP = d.xRLP;
  float2* const rl = sm.ring + (size_t)ccl * RLP;
  const uint32_t vbytes = 4u * (uint32_t)C;  // V-row bytes arriving per step (clusters)
  // clusters: the destinations of this combine lane's sends (CTAs jl,
  // jl + G, ...), their buffer and barrier mapped once
  constexpr int ND = (N + G - 1) / G;
  uint32_t rbuf[ND], rbar[ND];
#pragma unroll
  for (int u = 0; u < ND; ++u) {
    rbuf[u] = rbar[u] = 0u;
    if constexpr (N > 1) {
      const int q = jl + u * G;
      if (comb && q < N) {
        rbuf[u] = cluster_addr(vs.V, (uint32_t)q);
        rbar[u] = cluster_addr(vs.vbar, (uint32_t)q);
      }
    }
  }
  // bounds-check build: a row pointer lies inside the two tile buffers
  auto row_ok = [&](const int32_t* row) {
    const ptrdiff_t o = row - sm.tint;
    return o >= 0 && o + C <= 2 * TS * C;
  };

  // combine lanes: trans2[x][c] of their sources x = jl*CAT + q (-inf past C);
  // helper lanes: dur2 of window index q*H + jl, k = 2 + WL - (q*H + jl)
  float w[NR];
  float d1 = NEG_INF, d2 = NEG_INF;
  if (comb) {
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      // interleaved 16-byte chunks: chunk q/4 of lane jl is label block
      // (q/4) * G + jl, so a group's lanes read consecutive chunks (no shared
      // memory bank conflicts on the critical path's vector loads)
      const int x = 4 * ((q >> 2) * G + jl) + (q & 3);
      w[q] = (q < CAT && act && x < C) ? __ldg(trans + (size_t)x * C + cc) * l2e() : NEG_INF;
    }
  } else {
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      const int k = 2 + WL - (q * H + jl);
      w[q] = (q < KBH && act && k >= 3 && k <= K) ? __ldg(dur + (size_t)(k - 1) * C + cc) * l2e()
                                                 : NEG_INF;
    }
    d1 = __ldg(dur + cc) * l2e();
    if (K >= 2) d2 = __ldg(dur + C + cc) * l2e();
  }

  // ---------------------------------------------------------------- shared state
  for (int i = tid; i < RLP * Cr; i += blockDim.x) sm.ring[i] = make_float2(NEG_INF, 0.f);
  for (int i = tid; i < 2 * d.xPC; i += blockDim.x) vs.V[i] = NEG_INF;
  for (int i = tid; i < 2 * Cr * HW; i += blockDim.x) {
    vs.Om[i] = NEG_INF;
    vs.Ok[i] = 3;
  }
  for (int i = tid; i < 2 * Cr; i += blockDim.x) {
    vs.A1[i] = NEG_INF;
    vs.A2[i] = NEG_INF;
  }
  if (tid == 0) {
    vs.nsl[0] = vs.nsl[1] = 0.f;
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    if constexpr (N > 1) {
      mbar_init(&vs.vbar[0], 1);
      mbar_init(&vs.vbar[1], 1);
    }
    fence_mbar_init();
    if constexpr (N > 1) {
      mbar_expect_tx(&vs.vbar[1], vbytes);  // step 1's row
      mbar_expect_tx(&vs.vbar[0], vbytes);  // step 2's row
    }
  }
  __syncthreads();
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  ts.lo = 0;
  ts.hi = L / TS;
  ts.dir = 1;
  tile_issue(sm, d, ws, b, ts, 0);
  tile_issue(sm, d, ws, b, ts, 1);
  // A wait that gives up records the timeout and drains the copies in
  // flight.  One CTA returns at once; in a cluster the CTA instead stops
  // waiting and issuing copies (`dead`) and keeps taking part in the
  // cluster barriers until the last step (its results are then meaningless;
  // the status word says so).
  bool dead = false;
  if (!vtile_wait(sm, ts, 0)) {
    if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
    tile_drain(sm, ts);
    if constexpr (N == 1) return;
    dead = true;
  }
  // boundary 0: G = 0 at S = 0, base 0 (with boundary projections: the
  // start term of boundary 0); helpers set step 1's k = 1 constant
  for (int x = tid; x < Cr; x += blockDim.x) {
    float2* r = sm.ring + (size_t)x * RLP;
    const float v0 = (sm.tpd && c0 + x < C) ? sm.tpd[c0 + x] : 0.f;
    for (int y = 0; y < RL; y += K) r[y] = make_float2(v0, 0.f);
    vs.Sb[x] = 0;
  }
  // helper state: rows i (cur) and i-1 (prev) of S, frame Phi_{i-1} - F0;
  // with boundary projections the start terms pd of those rows (the k = 1
  // and k = 2 factors' start boundaries)
  int hs_c = 0, hs_p = 0;
  float hf_c = 0.f, hf_p = 0.f, Fph = 0.f, hd_c = 0.f, hd_p = 0.f;
  const int32_t* hrow_i = sm.tint;  // row i+1 of the current step (set below)
  const float* hrow_f = sm.tfrac;
  const float* hrow_d = nullptr;
  if (!comb) {
    hs_c = sm.tint[C + cc];  // row 1
    hf_c = sm.tfrac[C + cc];
    if (sm.tpd) {
      hd_p = sm.tpd[cc];      // row 0
      hd_c = sm.tpd[C + cc];  // row 1
      hrow_d = sm.tpd + 2 * C;
    }
    if (leader) vs.A1[1 * Cr + cl] = (d1 + hd_p) + ((float)hs_c + hf_c);  // S[1] - S[0]
    hrow_i = sm.tint + 2 * C;  // row 2 for step 1
    hrow_f = sm.tfrac + 2 * C;
  }
  int hbase = (((-WL) % K) + K) % K;  // window start b_lo = i - 1 - WL, at i = 1
  // kept rows of boundaries 1..L: V (frame-relative) and the chosen duration
  float* const vrw = ws.vrow + (size_t)b * (T + 1) * C;
  int32_t* const kdw = ws.bp + (size_t)b * (T + 1) * C;
  // combine state: S at row i - 1, ring slot of boundary i - 1
  float g2 = NEG_INF, nprev = 0.f, Fp = 0.f, mp = NEG_INF;
  int si_p = 0;
  float sf_p = 0.f, pd_p = sm.tpd ? sm.tpd[cc] : 0.f;  // row i - 1 (pd: start term)
  const int32_t* crow_i = sm.tint + C;  // row i of the current step
  const float* crow_f = sm.tfrac + C;
  const float* crow_d = sm.tpd ? sm.tpd + C : nullptr;
  int wslot = 0;
  double F0 = 0.0;
  // every CTA of a cluster has initialised its V buffer and arrival barriers
  // before any other CTA stores into them
  if constexpr (N > 1) {
    cluster_sync();
  } else {
    __syncthreads();
  }
  bool xdead = false;  // cluster: an arrival wait gave up (results are then meaningless)
  int Sbc = 0;
  int next_rb = VREBASE + 1;
  // next step with an event: a tile to wait for (row i+1 opens a tile), a
  // tile to issue (row i opens a tile), a rebase, or the last step
  auto next_event = [&](int i) {
    int e = min(next_with_rem(i, TS - 1), next_with_rem(i, 0));
    e = min(e, next_rb);
    return min(e, L);
  };
  int next_ev = next_event(0);

  for (int i = 1; i <= L; ++i) {
    // clusters: re-arm the arrival barrier of step i's vector (its previous
    // phase, step i-2's, completed before step i-1's label fan-in) for this
    // step's arrivals, by a thread off the combine path (bytes arriving
    // before the arm only take the count below zero)
    if constexpr (N > 1)
      if (tid == (int)blockDim.x - 32 && i >= 3) mbar_expect_tx(&vs.vbar[i & 1], vbytes);
    if (!comb && i >= 2) Fph += vs.nsl[(i - 1) & 1];
    if (i == next_ev) {
      if (i < L && (i + 1) % TS == 0) {
        if (!dead && !vtile_wait(sm, ts, (i + 1) / TS)) {
          if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
          tile_drain(sm, ts);
          if constexpr (N == 1) return;
          dead = true;
        }
        const size_t o = tile_row_off(i + 1, C);
        hrow_i = sm.tint + o;
        hrow_f = sm.tfrac + o;
        if (sm.tpd) hrow_d = sm.tpd + o;
      }
      if (i % TS == 0) {
        if (!dead) tile_issue(sm, d, ws, b, ts, i / TS + 1);
        const size_t o = tile_row_off(i, C);
        crow_i = sm.tint + o;
        crow_f = sm.tfrac + o;
        if (sm.tpd) crow_d = sm.tpd + o;
      }
      if (i == next_rb) {
        // rebase the integer frames to (F0 + Phi_{i-1}, S_int[i-1])
        const float D = comb ? Fp : Fph;
        if (!comb && act) {
          const float adj = (float)(hs_p - Sbc) - D;
          for (int x = jl; x < RL; x += H) rl[x].y += adj;
          if (leader) vs.Sb[cl] = hs_p;
        }
        __syncthreads();
        F0 += (double)D;
        if (comb) {
          Fp -= D;
        } else {
          Fph -= D;
        }
        Sbc = vs.Sb[ccl];
        next_rb += VREBASE;
      }
      next_ev = next_event(i);
    }
    // Each role issues all of its shared-memory reads first and its stores
    // last: a store the compiler cannot separate from later reads keeps
    // those reads from being issued early, and every access of the step must
    // complete before the barrier releases.
    if (comb) {
      // ---------------------------------------------------------- combine
      if constexpr (N > 1) {
        if (i >= 2) {
          // V[i-1] from every CTA of the cluster
          const int pb = (i - 1) & 1;
          if (!xdead && !mbar_wait_cluster(&vs.vbar[pb], ((i - 2) >> 1) & 1, WAIT_SPIN_LIMIT)) {
            set_status(ws.status, ST_DEVICE_TIMEOUT);
            xdead = true;
          }
        }
      }
      const float a1 = vs.A1[(i & 1) * Cr + ccl];
      const float a2 = vs.A2[(i & 1) * Cr + ccl];
      float om = vs.Om[(i & 1) * Cr + ccl];
      int okd = vs.Ok[(i & 1) * Cr + ccl];
#pragma unroll
      for (int hw = 1; hw < HW; ++hw) {  // long durations: the warps' best, smallest k on ties
        const float o2 = vs.Om[hw * 2 * Cr + (i & 1) * Cr + ccl];
        const int k2 = vs.Ok[hw * 2 * Cr + (i & 1) * Cr + ccl];
        if (o2 > om || (o2 == om && k2 < okd)) {
          om = o2;
          okd = k2;
        }
      }
      const bool rok = SEMICRF_INB(ws.status, row_ok(crow_i), SITE_TILE_ROW);
      const int si_n = rok ? crow_i[cc] : 0;  // row i: the next step's ring entry
      const float pd_n = (crow_d && rok) ? crow_d[cc] : 0.f;
      const float sf_n = rok ? crow_f[cc] : 0.f;
      const float* pv = vs.V + ((i - 1) & 1) * d.xPC + 4 * jl;
      // the label fan-in and, beside it, max V[i-1] (a group's lanes read
      // the whole row; padding entries hold -inf): the frame of step i+1
      float b0 = NEG_INF, b1 = NEG_INF, b2 = NEG_INF, b3 = NEG_INF, m0 = NEG_INF, m1 = NEG_INF;
#pragma unroll
      for (int q = 0; q < CAT; q += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pv + q * G);
        b0 = fmaxf(b0, v.x + w[q]);
        b1 = fmaxf(b1, v.y + w[q + 1]);
        b2 = fmaxf(b2, v.z + w[q + 2]);
        b3 = fmaxf(b3, v.w + w[q + 3]);
        m0 = fmaxf(m0, fmaxf(v.x, v.y));
        m1 = fmaxf(m1, fmaxf(v.z, v.w));
      }
      float gv = fmaxf(fmaxf(b0, b1), fmaxf(b2, b3));
      float mcur = fmaxf(m0, m1);
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) {
        gv = fmaxf(gv, __shfl_xor_sync(FULL_MASK, gv, o));
        mcur = fmaxf(mcur, __shfl_xor_sync(FULL_MASK, mcur, o));
      }
      if (i == 1) gv = 0.f;  // G[0] = 0 in frame 0 (V[0] is all -inf)
      // frame: Phi_i = Phi_{i-2} + rint(max V[i-2]), the max this lane took
      // a step ago
      const float n = ((mp == NEG_INF) ? 0.f : rintf(mp)) - nprev;
      mp = mcur;
      // candidates relative to Phi_{i-1}; ties to the smaller k
      const float c1 = gv + a1;
      const float c2 = (g2 + a2) - nprev;
      const float c3 = om - nprev;
      const float v = fmaxf(c1, fmaxf(c2, c3));
      const int kdec = (c1 >= c2 && c1 >= c3) ? 1 : (c2 >= c3 ? 2 : okd);
      const bool pok = SEMICRF_INB(ws.status, !act || c < d.xPC, SITE_VECTOR);
      if constexpr (N > 1) {
        // into every CTA of the cluster (this one included)
        if (act && pok) {
          const uint32_t po = 4u * (uint32_t)((i & 1) * d.xPC + c), bo = 8u * (uint32_t)(i & 1);
#pragma unroll
          for (int u = 0; u < ND; ++u)
            if (jl + u * G < N) st_async_mapped(rbuf[u] + po, rbar[u] + bo, v - n);
        }
      } else {
        if (leader && pok) vs.V[(i & 1) * d.xPC + c] = v - n;
      }
      if (tid == 0) vs.nsl[i & 1] = n;
      // off the path: boundary i's kept rows (V relative to Phi_i, the chosen
      // duration; global stores after the critical store cost the path
      // least), then G[i-1]'s ring entry (frame Phi_{i-1})
      if (leader && SEMICRF_INB(ws.status, i <= T, SITE_KEPT_ROW)) {
        vrw[(size_t)i * C + c] = v - n;
        kdw[(size_t)i * C + c] = kdec;
      }
      if (leader && i >= 2 && SEMICRF_INB(ws.status, wslot >= 0 && wslot < K, SITE_RING_SLOT)) {
        const float2 e = make_float2((gv - sf_p) + pd_p, Fp - (float)(si_p - Sbc));
        for (int x = wslot; x < RL; x += K) rl[x] = e;
      }
      wslot = (wslot + 1 == K) ? 0 : wslot + 1;
      g2 = gv;
      nprev = n;
      Fp += n;
      si_p = si_n;
      sf_p = sf_n;
      pd_p = pd_n;
      if (crow_d) crow_d += C;
      crow_i += C;
      crow_f += C;
    } else {
      // ---------------------------------------------------------- helpers
      // reads: the window of the k >= 3 terms of step i + 1 (boundaries
      // i - 1 - WL .. i - 2) and its prefix-sum row (not the row V[i-1]: in a
      // cluster the helpers never wait for the exchange)
      const bool hok = i < L && SEMICRF_INB(ws.status, row_ok(hrow_i), SITE_TILE_ROW);
      const int sn = hok ? hrow_i[cc] : 0;
      const float fn = hok ? hrow_f[cc] : 0.f;
      const float Qh = (float)(sn - Sbc) - Fph;
      const int hb = SEMICRF_INB(ws.status, hbase >= 0 && hbase + jl + (KBH - 1) * H < RLP,
                                 SITE_RING_WINDOW) ? hbase : 0;
      float best = NEG_INF;
      float tv[KBH];
#pragma unroll
      for (int q = 0; q < KBH; ++q) {
        const float2 e = rl[hb + q * H + jl];
        tv[q] = ((e.y + Qh) + e.x) + w[q];
        best = fmaxf(best, tv[q]);
      }
#pragma unroll
      for (int o = HG / 2; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(FULL_MASK, best, o));
      // smallest k among equal terms: k falls as the window index grows
      int kb = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < KBH; ++q)
        if (tv[q] == best) kb = 2 + WL - (q * H + jl);
#pragma unroll
      for (int o = HG / 2; o > 0; o >>= 1) kb = min(kb, __shfl_xor_sync(FULL_MASK, kb, o));
      // stores
      if (act && lane % HG == 0 && i < L) {  // each helper warp's candidate
        const int o2 = ((i + 1) & 1) * Cr + cl;
        vs.Om[hwarp * 2 * Cr + o2] = best + fn;
        vs.Ok[hwarp * 2 * Cr + o2] = kb;
      }
      if (leader && i < L) {
        const int o2 = ((i + 1) & 1) * Cr + cl;
        vs.A1[o2] = (d1 + hd_c) + ((float)(sn - hs_c) + (fn - hf_c));
        vs.A2[o2] = (d2 + hd_p) + ((float)(sn - hs_p) + (fn - hf_p));
      }
      if (i < L) {
        hs_p = hs_c;
        hf_p = hf_c;
        hs_c = sn;
        hf_c = fn;
        hd_p = hd_c;
        if (hrow_d) {
          hd_c = hok ? hrow_d[cc] : 0.f;
          hrow_d += C;
        }
        hrow_i += C;
        hrow_f += C;
        hbase = (hbase + 1 == K) ? 0 : hbase + 1;
      }
    }
    __syncthreads();
  }
  if constexpr (N > 1) {
    // the last row has arrived here (the score reads it; no store into this
    // CTA is left in flight), then no CTA leaves before every CTA is done
    if (comb && !xdead &&
        !mbar_wait_cluster(&vs.vbar[L & 1], ((L - 1) >> 1) & 1, WAIT_SPIN_LIMIT))
      set_status(ws.status, ST_DEVICE_TIMEOUT);
    cluster_sync();
  }
  // the optimum: max over the final labels of V[L] in frame Phi_L
  if (tid < 32 && rank == 0) {
    const float* V = vs.V + (L & 1) * d.xPC;
    float best = NEG_INF;
    for (int x = tid; x < C; x += 32) best = fmaxf(best, V[x]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(FULL_MASK, best, o));
    if (tid == 0) score[b] = (F0 + (double)Fp + (double)best) * LN2_D;
  }
}

// Label argmax rows, in parallel over (boundary, label): for boundary s in
// [1, L - 1] and label c,
//   A[s, c] = argmax_{c'} (V[s, c'] + trans2[c', c])   (smallest c' on ties),
// the label before a segment of label c that starts at s.  It depends on s
// and c only, not on where the segment ends, so it is computed once per
// boundary.  One CTA per block of VA_ROWS boundaries of a sequence stages
// those rows of V (rows of VS = C rounded up to 4 floats, -inf padded);
// thread (label c, row phase) keeps trans2[., c] in registers and reads each
// row as float4 broadcasts (the lanes of one row phase read the same row).
// The argmax runs four independent compare chains (c' mod 4) and merges
// them by value, then index, so it is the smallest c' among equal maxima, as
// the recursion's own comparisons would give.
constexpr int VA_ROWS = 64;
template <int NW>
__global__ void __launch_bounds__(256)
    viterbi_argmax_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                          const float* __restrict__ trans) {
  __shared__ __align__(16) float vsh[VA_ROWS * NW];
  const int C = d.C, tid = threadIdx.x, b = blockIdx.y;
  const int L = lengths[b];
  if (L < 1 || L > d.T) return;
  const int s0 = blockIdx.x * VA_ROWS + 1;
  if (s0 >= L) return;  // boundaries [1, L - 1] start a segment with a predecessor
  const int s1 = min(s0 + VA_ROWS - 1, L - 1);
  const int VS = (C + 3) & ~3;
  const float* vrw = ws.vrow + (size_t)b * (d.T + 1) * C;
  int32_t* arg = ws.varg + (size_t)b * (d.T + 1) * VS;
  const int nv = (s1 - s0 + 1) * VS;
#pragma unroll 4
  for (int i = tid; i < nv; i += blockDim.x) {
    const int r = i / VS, x = i - r * VS;
    vsh[i] = (x < C) ? vrw[(size_t)(s0 + r) * C + x] : NEG_INF;
  }
  const int pc = tid % C, pg = tid / C, png = blockDim.x / C;
  float w2[NW];
#pragma unroll
  for (int q = 0; q < NW; ++q)
    w2[q] = (q < C && pg < png) ? __ldg(trans + (size_t)q * C + pc) * l2e() : NEG_INF;
  __syncthreads();
  if (pg >= png) return;
  // VR rows at a time (4 VR independent chains); per element an add, a
  // compare-select of the index and a max of the value, so a chain's value
  // update does not wait on its compare
  constexpr int VR = 4;
  for (int s = s0 + pg; s <= s1; s += VR * png) {
    const float4* vr[VR];
#pragma unroll
    for (int w = 0; w < VR; ++w)  // rows past s1 repeat s1 (not stored)
      vr[w] = reinterpret_cast<const float4*>(vsh + (size_t)(min(s + w * png, s1) - s0) * VS);
    float bv[VR][4];
    int qv[VR][4];
#pragma unroll
    for (int w = 0; w < VR; ++w)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        bv[w][u] = NEG_INF;
        qv[w][u] = u;
      }
#pragma unroll
    for (int q4 = 0; q4 < NW / 4; ++q4) {
      if (4 * q4 < VS) {
#pragma unroll
        for (int w = 0; w < VR; ++w) {
          const float4 x = vr[w][q4];
          const float ex[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float e = ex[u] + w2[4 * q4 + u];
            qv[w][u] = (e > bv[w][u]) ? 4 * q4 + u : qv[w][u];
            bv[w][u] = fmaxf(bv[w][u], e);
          }
        }
      }
    }
    // merge the chains by value, then index: the smallest c' among equal
    // maxima (a chain that never improved on -inf keeps its first index, so
    // an all -inf row yields label 0)
#pragma unroll
    for (int w = 0; w < VR; ++w) {
      float* b = bv[w];
      int* q = qv[w];
      if (b[1] > b[0] || (b[1] == b[0] && q[1] < q[0])) { b[0] = b[1]; q[0] = q[1]; }
      if (b[3] > b[2] || (b[3] == b[2] && q[3] < q[2])) { b[2] = b[3]; q[2] = q[3]; }
      if (b[2] > b[0] || (b[2] == b[0] && q[2] < q[0])) { b[0] = b[2]; q[0] = q[2]; }
      if (s + w * png <= s1) arg[(size_t)(s + w * png) * VS + pc] = q[0];
    }
  }
}

// Backpointer words, in parallel over (boundary, label): for boundary t in
// [1, L] and label c with k = kd[t, c] in [1, K] and s = t - k >= 1, the word
// is k | A[s, c] << 16; otherwise (s = 0, or a duration the recursion never
// set) it is k.  Rows of CP = C rounded up to 4 words (16-byte rows, copied
// to shared memory in bulk by the walk).
__global__ void __launch_bounds__(256)
    viterbi_words_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths) {
  const int C = d.C, CP = (C + 3) & ~3, b = blockIdx.y;
  const int L = lengths[b];
  if (L < 1 || L > d.T) return;
  const int32_t* kdw = ws.bp + (size_t)b * (d.T + 1) * C;
  const int32_t* arg = ws.varg + (size_t)b * (d.T + 1) * CP;
  int32_t* wrd = ws.wrd + (size_t)b * (d.T + 1) * CP;
  const size_t n = (size_t)L * C;  // boundaries [1, L]
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / C) + 1, c = (int)(i - (size_t)(t - 1) * C);
    const int k = kdw[(size_t)t * C + c];
    const int s = t - k;
    int word = k;
    if (k >= 1 && k <= d.K && s >= 1) word = k | (arg[(size_t)s * CP + c] << 16);
    wrd[(size_t)t * CP + c] = word;
  }
}

// The traceback, one CTA per sequence.  Start: the best final label
// (argmax of the kept row V[L], smallest on ties).  The word rows are cut
// into fixed windows of WR rows, [1 + w WR, (w + 1) WR], taken downwards
// through two buffers: while the walk reads window w, a bulk copy (TMA,
// completion on that buffer's mbarrier, bounded waits) brings window w - 1
// into the other.  Thread 0 follows the words through the window -- one
// shared-memory read per decoded segment -- and marks each segment's start
// position with its label; then warp 0 fills every position from where the
// walk left the window up to where it entered it with the label of the last
// mark at or below it (a running "last mark" scan, 32 positions per shuffle
// round) and writes labels and start flags out coalesced.  A segment that
// jumps past the prefetched window has its window copied in before the walk
// goes on.  A word with a duration outside [1, min(t, K)] or a previous
// label >= C ends the walk with the positions not reached labelled -1.
__global__ void __launch_bounds__(256)
    viterbi_walk_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                        int32_t* __restrict__ labels, uint8_t* __restrict__ seg_start, int WR) {
  extern __shared__ __align__(16) int wsh[];  // words [2][WR][CP], marks [WR + K]
  __shared__ int s_tb[2];
  __shared__ __align__(8) uint64_t wbar[2];
  const int C = d.C, K = d.K, T = d.T, tid = threadIdx.x, lane = tid & 31, b = blockIdx.x;
  const int CP = (C + 3) & ~3;
  const int L = lengths[b];
  if (L < 1 || L > T) return;
  const int32_t* wrd = ws.wrd + (size_t)b * (T + 1) * CP;
  const float* vrw = ws.vrow + (size_t)b * (T + 1) * C;
  int* const lbuf = wsh + 2 * (size_t)WR * CP;
  if (tid == 0) {
    mbar_init(&wbar[0], 1);
    mbar_init(&wbar[1], 1);
    fence_mbar_init();
  }
  if (tid < 32) {
    float best = NEG_INF;
    int bc = 0x7fffffff;
    for (int x = tid; x < C; x += 32) {
      const float v = vrw[(size_t)L * C + x];
      if (v > best || bc == 0x7fffffff) {
        best = v;
        bc = x;
      }
    }
    gargmax<32>(best, bc);
    if (tid == 0) {
      s_tb[0] = L;
      s_tb[1] = bc;
    }
  }
  __syncthreads();
  // copy window w (its rows up to L) into buffer p; thread 0
  auto issue = [&](int w, int p) {
    const int lo = 1 + w * WR, hi = min(L, lo + WR - 1);
    const uint32_t bytes = (uint32_t)((hi - lo + 1) * CP * 4);
    fence_proxy_async();  // earlier reads of the buffer come before the copy's writes
    mbar_expect_tx(&wbar[p], bytes);
    bulk_g2s(wsh + (size_t)p * WR * CP, wrd + (size_t)lo * CP, bytes, &wbar[p]);
  };
  uint32_t ph[2] = {0u, 0u};    // every thread tracks both barriers' phases
  bool busy[2] = {true, false};  // a copy into the buffer is in flight
  // a bounded wait for buffer p's copy, by every thread together; false: a
  // thread gave up (the state is left as it was, the same in every thread)
  bool timed_out = false;
  auto land = [&](int p) {
    const bool ok = mbar_wait(&wbar[p], ph[p], WAIT_SPIN_LIMIT);
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      return false;
    }
    ph[p] ^= 1u;
    busy[p] = false;
    return true;
  };
  int w = (L - 1) / WR, p = 0;
  if (tid == 0) issue(w, 0);
  for (;;) {
    const int tt0 = s_tb[0];  // 1 <= tt0, inside window w
    const int lo = 1 + w * WR;
    const int pb = lo - K;  // mark of position u at lbuf[u - pb]
    // bounds-check build: the walk starts inside the window
    if (!SEMICRF_INB(ws.status, tt0 >= lo && tt0 - lo < WR && tt0 <= L, SITE_WALK_STAGE)) break;
    if (!land(p)) break;
    const bool pre = w > 0;
    if (pre) {
      if (tid == 0) issue(w - 1, p ^ 1);
      busy[p ^ 1] = true;
    }
    for (int i = tid; i < WR + K; i += blockDim.x) lbuf[i] = -1;
    __syncthreads();
    if (tid == 0) {
      const int* kb = wsh + (size_t)p * WR * CP;
      int tt = tt0, cl = s_tb[1];
      bool broken = false;
      while (tt >= lo) {
        const int wd = kb[(tt - lo) * CP + cl];
        const int k = wd & 0xffff, pred = (wd >> 16) & 0xffff;
        if (k < 1 || k > tt || k > K || (tt - k > 0 && pred >= C)) {
          broken = true;
          break;
        }
        tt -= k;
        if (SEMICRF_INB(ws.status, tt - pb >= 0 && tt - pb < WR + K, SITE_WALK_MARK))
          lbuf[tt - pb] = cl;
        cl = pred;
      }
      s_tb[0] = broken ? -tt : tt;  // -tt: stop, positions below tt get -1
      s_tb[1] = cl;
    }
    __syncthreads();
    const int te = s_tb[0];
    const int end = te < 0 ? -te : te;
    if (tid < 32) {
      int carry = -1;
      for (int u0 = end; u0 < tt0; u0 += 32) {
        const int u = u0 + lane;
        const int m = (u < tt0) ? lbuf[u - pb] : -1;
        int v = m;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int up = __shfl_up_sync(FULL_MASK, v, o);
          if (lane >= o && v < 0) v = up;
        }
        if (v < 0) v = carry;
        carry = __shfl_sync(FULL_MASK, v, 31);
        if (u < tt0) {
          labels[(size_t)b * T + u] = v;
          seg_start[(size_t)b * T + u] = (m >= 0) ? 1 : 0;
        }
      }
    }
    if (te < 0)
      for (int u = tid; u < end; u += blockDim.x) labels[(size_t)b * T + u] = -1;
    __syncthreads();  // every thread has read s_tb and the marks before the next window
    if (te <= 0) break;
    // the next window: the one holding te (the prefetched one unless a
    // segment jumped past it)
    const int wn = (te - 1) / WR;
    if (wn != w - 1) {
      if (!land(p ^ 1)) break;
      if (tid == 0) issue(wn, p ^ 1);
      busy[p ^ 1] = true;
    }
    w = wn;
    p ^= 1;
  }
  // leave no copy in flight into this CTA's shared memory
  for (int q = 0; q < 2; ++q)
    if (busy[q]) land(q);
  if (timed_out && tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
}

}  // namespace

size_t viterbi_pipe_smem_bytes(const Dims& d, bool pj) { return vsmem_bytes(d, pj); }

#define SEMICRF_VA_WIDTHS(X) X(8) X(16) X(32) X(48) X(64) X(96) X(128)

cudaError_t launch_viterbi_argmax(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                  const float* trans, cudaStream_t st) {
  if (d.T == 0 || d.B == 0) return cudaSuccess;
  const dim3 grid((d.T + VA_ROWS - 1) / VA_ROWS, d.B);
#define SEMICRF_VA_LAUNCH(nw)                                                 \
  if (d.C <= nw) {                                                            \
    viterbi_argmax_kernel<nw><<<grid, 256, 0, st>>>(d, ws, lengths, trans);   \
    return cudaGetLastError();                                                \
  }
  SEMICRF_VA_WIDTHS(SEMICRF_VA_LAUNCH)
#undef SEMICRF_VA_LAUNCH
  return cudaErrorInvalidConfiguration;
}

cudaError_t launch_viterbi_words(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                 cudaStream_t st) {
  if (d.T == 0 || d.B == 0) return cudaSuccess;
  const size_t items = (size_t)d.T * d.C;
  const dim3 grid((unsigned)std::min<size_t>((items + 255) / 256, 1184), d.B);
  viterbi_words_kernel<<<grid, 256, 0, st>>>(d, ws, lengths);
  return cudaGetLastError();
}

// Shared memory of the walk: up to 200 KB (long windows: fewer of them), at
// least the K marks and one row of words per buffer.
size_t viterbi_walk_smem_bytes(const Dims& d, size_t budget) {
  const size_t CP = (d.C + 3) & ~3;
  const size_t want = std::min<size_t>(budget, 200u * 1024u);
  const size_t need = ((size_t)d.K + 1 + 2 * CP) * sizeof(int);
  return std::max(want, need);
}

cudaError_t launch_viterbi_walk(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                int32_t* labels, uint8_t* seg_start, size_t sm, cudaStream_t st) {
  const size_t CP = (d.C + 3) & ~3;
  const int WR = (int)((sm / sizeof(int) - (size_t)d.K) / (2 * CP + 1));
  if (sm > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(viterbi_walk_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
  }
  viterbi_walk_kernel<<<d.B, 256, sm, st>>>(d, ws, lengths, labels, seg_start, WR);
  return cudaGetLastError();
}

}  // namespace semicrf

namespace semicrf {

cudaError_t launch_viterbi_pipe(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                const float* trans, const float* dur, double* score,
                                int32_t* labels, uint8_t* seg_start, cudaStream_t st, int pj) {
  const size_t sm = viterbi_pipe_smem_bytes(d, pj != 0);
#define SEMICRF_LAUNCH_VPIPE(n, g, cat, h, kbh, lb)                                            \
  if (d.xN == n && d.xG == g && d.xCAT == cat && d.xH == h && d.xKBH == kbh && d.xLB == lb)    \
    return launch_clustered(viterbi_pipe_kernel<n, g, cat, h, kbh, lb>, n, d.B * n, d.xNT, sm,  \
                            st, d, ws, lengths, trans, dur, score, labels, seg_start, pj);
  SEMICRF_FOR_EACH_XSHAPE(SEMICRF_LAUNCH_VPIPE)
#undef SEMICRF_LAUNCH_VPIPE
  return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
