// chain_exp.cu -- steps 2 and 3: the forward and backward rings with the
// label fan-in in the exponential domain on the critical path and the rest of
// each step computed one step ahead.
//
// "Streaming Structured Inference with Flash-SemiCRF", explainer section 2,
// "Streaming Forward-Backward with Ring Buffers".  The recursion is the one of
// chain_kernel (recursion.cu), in base-2 log units:
//   gamma[s, c] = LSE_{c'} alpha[s, c'] + trans[c', c]             (gamma[0] = 0)
//   alpha[t, c] = S[t,c] + LSE_{k <= min(K,t)} gamma[t-k, c] - S[t-k, c] + dur[k-1, c]
// with the backward mirror (btil after the k fan-in, beta after the label
// fan-in).  What one step really waits for is small: only the k = 1 term of
// alpha[t] needs gamma[t-1], which needs the whole vector alpha[t-1, :].
// The kernel is organised around that dependency.
//
// Representation.  Step t keeps the label vector in the exponential domain,
//   p_t[c] = 2^(alpha[t, c] - Phi_t),   Phi_t = Phi_{t-1} + n_t  (integers),
// with n_t the binary exponent of max_c p_{t-1}[c]: Phi_t follows max alpha[t-1]
// one step late, so no reduction sits on the critical path.  With
//   acc_s[c] = sum_{c'} p_s[c'] * 2^(trans2[c', c] - M)          (M = max trans2)
// we have gamma[s, c] = Phi_s + M + log2 acc_s[c] (acc_0 = 2^-M, Phi_0 = 0), and
//   p_t = 2^-n_t * ( acc_{t-1} A1_t + 2^-n_{t-1} (acc_{t-2} A2_t + O_t) )
//   A1_t = 2^(M + dur2[0] + S[t] - S[t-1]),  A2_t = 2^(M + dur2[1] + S[t] - S[t-2]),
// where O_t is the k >= 3 part of the duration sum relative to Phi_{t-2}.
// Everything but acc_{t-1} and n_t is known when step t begins, so the
// critical path of a step is: read p_{t-1} -> dot product with the transition
// weights -> two multiplies and a multiply-add -> store p_t -> barrier.
//
// Roles.  Combine warps (xG lanes per label, xCAT weights per lane) run that
// path, keep acc_{t-2} and the previous prefix-sum row in registers, publish
// n_t, and write gamma[t-1] into the label's ring in the log domain (off the
// critical path; exactly the entry format of chain_kernel, so checkpoints and
// the posterior kernel are shared).  Helper warps (xH lanes per label, xKBH
// durations each, interleaved over the window so that a label's lanes read
// consecutive ring entries) compute during step t everything step t+1 needs
// besides acc_t: O_{t+1} -- the same predicted-shift k fan-in as chain_kernel,
// from ring entries of boundaries <= t-2 -- and A1_{t+1}, A2_{t+1}.  One CTA
// barrier per step orders everything.  The two directions are separate
// instantiations (no per-step direction tests).
//
// Exactness.  The exponential domain is exact up to float32 rounding while
// every label's alpha stays within fp32's exponent range of the frame.  Per
// step, alpha[t, c] - max alpha[t-1] lies in
//   [tmin + dmin - e, log2(K C) + max(tmax + dmax, dmax - dmin) + e]
// (tmin/tmax, dmin/dmax: ranges of the finite transition and duration scores,
// e: the largest |centred emission|), and O_t spans two steps, so the kernel
// takes a sequence only when all scores are finite and that span is below
// FAST_BOUND (half the exponent range); otherwise it records mode 2 and
// chain_kernel (log domain, any input) runs the sequence.
#include "ring.cuh"

namespace semicrf {

using namespace ring;

namespace {

constexpr float FAST_BOUND = 60.f;  // log2 units; two steps stay inside fp32's 126

// Per-label arrays cover the CTA's own labels (Cr = xCr of them, local
// index); P holds the whole label vector in every CTA of a cluster.
struct XSmem {
  Smem s;      // mbar, tint, tfrac (every label), ring (own labels)
  float* P;    // [2][xPC] exp-domain label vector, by step parity (all labels)
  float* Oh;   // [HW][2][Cr] k >= 3 sums for the step of that parity (frame Phi_{t-2}),
               // one partial per helper warp of a label (HW = ceil(xH / 32))
  float* A1;   // [2][Cr]  k = 1 factors
  float* A2;   // [2][Cr]  k = 2 factors
  float* nsl;  // [2]      frame step n published by the combine warps
  int* aux;    // [4]      block reductions
  int* Sb;     // [Cr]     label integer bases of the prefix sums
  uint64_t* pbar;  // [2]  cluster: arrival of the step's label vector, by step parity
};

__device__ __forceinline__ XSmem xcarve(unsigned char* raw, const Dims& d, bool pj) {
  XSmem x;
  const int C = d.C, Cr = d.xCr;  // tile rows hold every label, the rest this CTA's
  unsigned char* p = raw;
  x.s.mbar = reinterpret_cast<uint64_t*>(p);
  x.s.maxslot = reinterpret_cast<int*>(p + 16);
  x.aux = reinterpret_cast<int*>(p + 32);
  x.s.aux = x.aux;
  x.nsl = reinterpret_cast<float*>(p + 48);
  x.pbar = reinterpret_cast<uint64_t*>(p + 64);
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
  x.P = f;
  f += 2 * d.xPC;
  x.Oh = f;
  f += 2 * Cr * ((d.xH + 31) / 32);
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

// 2^-n for an integer-valued n in [-126, 127] (exact, no rounding).
__device__ __forceinline__ float pow2_neg(float n) {
  return __int_as_float((127 - (int)n) << 23);
}

// Binary exponent of a positive normal float (0 for 0).
__device__ __forceinline__ float exponent_of(float x) {
  return x > 0.f ? (float)(((__float_as_int(x) >> 23) & 0xff) - 127) : 0.f;
}

// Bounded wait for prefix-sum tile `ti`; false (uniformly) if it gave up.
__device__ __forceinline__ bool xtile_wait(const Smem& sm, TileStream& ts, int ti) {
  const int buf = ti & 1;
  bool ok = mbar_wait(&sm.mbar[buf], ts.ph[buf], WAIT_SPIN_LIMIT);
  ts.ph[buf] ^= 1u;
  return !__syncthreads_or(!ok);
}

// Smallest i' > i with i' = rem (mod TS), rem in [0, TS).
__device__ __forceinline__ int next_mod(int i, int rem) {
  const int x = (i / TS) * TS + rem;
  return x > i ? x : x + TS;
}

// One ring (direction UP: forward over rows 1..L; else backward over rows
// L-1..0) of sequence b, after the fast-path test has passed.
//
// With a cluster of N > 1 CTAs per ring, CTA `rank` owns labels
// [rank*Cr, rank*Cr + Cr): its ring, its k fan-in and its label fan-in
// outputs.  The label fan-in of every label needs the whole vector p_{t-1},
// so each combine group sends its p_t into the P buffer of every CTA of the
// cluster with asynchronous distributed-shared-memory stores (the group's
// lanes taking different destination CTAs) that count against the
// destination's arrival barrier pbar[t & 1] (4 C bytes per step).  A combine
// lane waits on its own CTA's barrier before reading p_{t-1}; a thread off
// the combine path re-arms it at the top of step t+1 (for step t+1's
// vector); steps still end with the CTA barrier only.  The send addresses
// in the other CTAs are mapped once, before the walk.  No release fence sits in the step (a cluster barrier's release
// would also wait for the kept rows' global stores).  Every CTA holds the
// same full vector and computes the same frame step n from it.  A barrier
// phase is reused two steps later, by which time every CTA has read the
// vector it held (the senders of step t+1 have received step t from all).
template <bool UP, int N, int G, int CAT, int H, int KBH>
__device__ __forceinline__ void xring(const XSmem& xs, const Dims& d, const WsPtrs& ws, int b,
                                      int L, const float* __restrict__ trans,
                                      const float* __restrict__ dur, float M,
                                      double* __restrict__ logZ_out, int rank) {
  const Smem& sm = xs.s;
  const int C = d.C, K = d.K, Cr = d.xCr, tid = threadIdx.x;
  // Long durations: H > 32 lanes per label spread over HW = H / 32 helper
  // warps; each warp sums its share of the window (its own predicted shift)
  // and publishes a partial k >= 3 sum, which the combine adds up.
  constexpr int HG = H > 32 ? 32 : H;       // lanes per reduction group
  constexpr int HW = H > 32 ? H / 32 : 1;   // helper warps per label
  constexpr int LPWC = 32 / G, LPWH = 32 / HG, WL = H * KBH;
  constexpr int NR = CAT > KBH ? CAT : KBH;
  constexpr int SG = UP ? 1 : -1;  // walk direction over rows
  const float sg = UP ? 1.f : -1.f;
  const int warp = tid >> 5, lane = tid & 31;
  const int nwc = (Cr + LPWC - 1) / LPWC;
  const bool comb = warp < nwc;
  const int c0 = rank * Cr;  // first label of this CTA
  const int hwi = warp - nwc;  // helper warp index
  const int cl = comb ? warp * LPWC + lane / G
                      : (HW > 1 ? hwi / HW : hwi * LPWH + lane / H);  // local label
  const int hwarp = HW > 1 && !comb ? hwi % HW : 0;  // this lane's warp among its label's
  const int c = c0 + cl;     // global label
  const bool act = cl < Cr && c < C;
  const int cc = act ? c : 0;     // global label (tile rows, parameters, outputs)
  const int ccl = act ? cl : 0;   // local label (ring, per-label arrays)
  const int jl = comb ? lane % G : (HW > 1 ? hwarp * 32 + lane : lane % H);
  const bool leader = act && jl == 0;
  const int RL = K + WL, RLP = d.xRLP;
  float2* const rl = sm.ring + (size_t)ccl * RLP;
  const uint32_t vbytes = 4u * (uint32_t)C;  // label-vector bytes arriving per step (clusters)
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
        rbuf[u] = cluster_addr(xs.P, (uint32_t)q);
        rbar[u] = cluster_addr(xs.pbar, (uint32_t)q);
      }
    }
  }
  auto put = [&](int slot, float2 v) {  // slot and its mirrors slot + mK < RL
    for (int x = slot; x < RL; x += K) rl[x] = v;
  };
  // bounds-check build: a row pointer lies inside the two tile buffers
  auto row_ok = [&](const int32_t* row) {
    const ptrdiff_t o = row - sm.tint;
    return o >= 0 && o + C <= 2 * TS * C;
  };

  // One register array serves both roles: combine lanes keep the transition
  // weights 2^(trans2 - M) of their CAT source labels (forward trans[x][c],
  // backward trans[c][x]); helper lanes the durations of window index
  // q*H + jl: k = 2 + WL - (q*H + jl) forward, 3 + q*H + jl backward.
  float w[NR];
  float d1 = NEG_INF, d2 = NEG_INF;
  if (comb) {
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      // interleaved 16-byte chunks: chunk q/4 of lane jl is label block
      // (q/4) * G + jl, so a group's lanes read consecutive chunks (no shared
      // memory bank conflicts on the critical path's vector loads)
      const int x = 4 * ((q >> 2) * G + jl) + (q & 3);
      w[q] = (q < CAT && act && x < C)
                 ? ex2(__ldg(trans + (UP ? (size_t)x * C + cc : (size_t)cc * C + x)) * l2e() - M)
                 : 0.f;
    }
  } else {
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      const int k = UP ? 2 + WL - (q * H + jl) : 3 + q * H + jl;
      w[q] = (q < KBH && act && k <= K) ? __ldg(dur + (size_t)(k - 1) * C + cc) * l2e() : NEG_INF;
    }
    d1 = __ldg(dur + cc) * l2e();
    if (K >= 2) d2 = __ldg(dur + C + cc) * l2e();
  }

  // ---------------------------------------------------------------- shared state
  for (int i = tid; i < RLP * Cr; i += blockDim.x) sm.ring[i] = make_float2(NEG_INF, 0.f);
  for (int i = tid; i < 2 * d.xPC; i += blockDim.x) xs.P[i] = 0.f;
  for (int i = tid; i < 2 * Cr * HW; i += blockDim.x) xs.Oh[i] = 0.f;
  for (int i = tid; i < 2 * Cr; i += blockDim.x) {
    xs.A1[i] = 0.f;
    xs.A2[i] = 0.f;
  }
  if (tid == 0) {
    xs.nsl[0] = xs.nsl[1] = 0.f;
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    if constexpr (N > 1) {
      mbar_init(&xs.pbar[0], 1);
      mbar_init(&xs.pbar[1], 1);
    }
    fence_mbar_init();
    if constexpr (N > 1) {
      mbar_expect_tx(&xs.pbar[1], vbytes);  // step 1's vector
      mbar_expect_tx(&xs.pbar[0], vbytes);  // step 2's vector
    }
  }
  __syncthreads();
  const int r0 = UP ? 0 : L;  // the walk's start boundary
  const int r1 = r0 + SG;
  TileStream ts;
  ts.ph[0] = ts.ph[1] = 0;
  ts.lo = 0;
  ts.hi = L / TS;
  ts.dir = SG;
  tile_issue(sm, d, ws, b, ts, r0 / TS);
  tile_issue(sm, d, ws, b, ts, r0 / TS + SG);
  // A wait that gives up records the timeout and drains the copies in
  // flight.  One CTA returns at once; in a cluster the CTA instead stops
  // waiting and issuing copies (`dead`) and keeps taking part in the
  // cluster barriers until the last step, so that no CTA waits for one that
  // left (its results are then meaningless; the status word says so).
  bool dead = false;
  bool ok = xtile_wait(sm, ts, r0 / TS);
  if (ok && r1 / TS != r0 / TS) ok = xtile_wait(sm, ts, r1 / TS);
  if (!ok) {
    if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
    tile_drain(sm, ts);
    if constexpr (N == 1) return;
    dead = true;
  }
  const size_t o0 = tile_row_off(r0, C), o1 = tile_row_off(r1, C);
  for (int x = tid; x < Cr && c0 + x < C; x += blockDim.x) {
    // gamma[0] = 0 at S = 0 (forward; with projections the start term of
    // boundary 0); beta[L] = 0 at S[L] (backward)
    const float2 v = make_float2(UP ? (sm.tpd ? sm.tpd[o0 + c0 + x] : 0.f) : sm.tfrac[o0 + c0 + x],
                                 0.f);
    float2* r = sm.ring + (size_t)x * RLP;
    for (int y = r0 % K; y < RL; y += K) r[y] = v;
    xs.Sb[x] = UP ? 0 : sm.tint[o0 + c0 + x];
  }
  // combine state: rows r-1 and r-2 (walk order) of S_int, row r-1 of S_frac,
  // acc and n of the last step, the frame of p_{i-1} relative to F0
  int si_p = UP ? 0 : sm.tint[o0 + cc], si_pp = si_p;
  float sf_p = UP ? 0.f : sm.tfrac[o0 + cc];
  // boundary projections (sm.tpd set): the start term pd of a row, added
  // wherever its boundary takes the start role -- forward ring entries and
  // the k = 1, 2 factors (rows r-1, r-2 of the step); backward every term
  // of the step's own row
  float pd_p = sm.tpd ? sm.tpd[o0 + cc] : 0.f;
  float acc2 = 0.f, snprev = 1.f, Fp = 0.f;
  int wslot = r0 % K;
  const int32_t* crow_i = sm.tint + o1;
  const float* crow_f = sm.tfrac + o1;
  const float* crow_d = sm.tpd ? sm.tpd + o1 : nullptr;
  // helper state: rows r (cur) and r-1 (prev) of S, frame Phi_{i-1} - F0,
  // predicted shift relative to Q, window base
  int hs_c = sm.tint[o1 + cc], hs_p = si_p;
  float hf_c = sm.tfrac[o1 + cc], hf_p = sf_p;
  float hd_c = sm.tpd ? sm.tpd[o1 + cc] : 0.f, hd_p = pd_p;
  float Fph = 0.f, rel = 0.f;
  const int32_t* hrow_i = sm.tint + o1 + SG * C;  // row r + SG of step 1
  const float* hrow_f = sm.tfrac + o1 + SG * C;
  const float* hrow_d = sm.tpd ? sm.tpd + o1 + SG * C : nullptr;
  int hbase = UP ? -WL : L + 1;  // window start boundary at step 1
  hbase = ((hbase % K) + K) % K;
  if (!comb && leader)  // step 1's k = 1 factor (no k = 2 term, no k >= 3 terms)
    xs.A1[Cr + cl] = ex2(((M + d1) + (UP ? hd_p : hd_c)) +
                         sg * ((float)(hs_c - hs_p) + (hf_c - hf_p)));
  double F0 = 0.0;
  // kept values for the posterior pass: per boundary (row) the vector p and
  // the label fan-in acc, relative to the boundary's frame kf, stored by the
  // combine leaders at the end of their step
  const int dir = UP ? 0 : 1;
  float* const kv = ws.kv ? ws.kv + (((size_t)b * 2 + dir) * (d.T + 1)) * 2 * C : nullptr;
  double* const kf = ws.kf ? ws.kf + ((size_t)b * 2 + dir) * (d.T + 1) : nullptr;
  if (kv) {
    const int rL = UP ? L : 0;  // the walk's last row: no label fan-in there
    for (int x = c0 + tid; x < c0 + Cr && x < C; x += blockDim.x) {
      kv[(size_t)r0 * 2 * C + x] = 0.f;  // no forward vector at 0, no btil at L
      kv[(size_t)rL * 2 * C + C + x] = 0.f;
    }
    if (tid == 0 && rank == 0) kf[r0] = 0.0;
  }
  // every CTA of a cluster has initialised its P buffer and arrival
  // barriers before any other CTA stores into them
  if constexpr (N > 1) {
    cluster_sync();
  } else {
    __syncthreads();
  }
  bool xdead = false;  // cluster: an arrival wait gave up (results are then meaningless)
  int Sbc = xs.Sb[ccl];
  // checkpoint steps: forward boundary t = i - 1 at step i; backward
  // boundary t1 = r + 2 at step i
  const int delta = d.delta;
  int next_ck;
  if (UP) {
    next_ck = delta + 1;
  } else {
    const int t1 = ((L - 1) / delta) * delta;
    next_ck = (t1 >= delta && t1 >= 2) ? L + 2 - t1 : INT_MAX;
  }
  // events: a tile to wait for (the helpers' row opens a tile), a tile to
  // issue (the combine's row opens a tile), a checkpoint, the last step
  const int rem_w = UP ? TS - 1 : L % TS, rem_i = UP ? 0 : (L + 1) % TS;
  auto next_event = [&](int i) {
    return min(min(next_mod(i, rem_w), next_mod(i, rem_i)), min(next_ck, L));
  };
  int next_ev = next_event(0);

  const float acc_start = ex2(-M);
  for (int i = 1; i <= L; ++i) {
    const int r = UP ? i : L - i;
    // clusters: re-arm the arrival barrier of step i's vector (its previous
    // phase, step i-2's, completed before step i-1's label fan-in) for this
    // step's arrivals, by a thread off the combine path (bytes arriving
    // before the arm only take the count below zero)
    if constexpr (N > 1)
      if (tid == (int)blockDim.x - 32 && i >= 3) mbar_expect_tx(&xs.pbar[i & 1], vbytes);
    if (!comb && i >= 2) Fph += xs.nsl[(i - 1) & 1];
    if (i == next_ev) {
      if (i < L && i % TS == rem_w) {
        if (!dead && !xtile_wait(sm, ts, (r + SG) / TS)) {
          if (tid == 0) set_status(ws.status, ST_DEVICE_TIMEOUT);
          tile_drain(sm, ts);
          if constexpr (N == 1) return;
          dead = true;
        }
        const size_t o = tile_row_off(r + SG, C);
        hrow_i = sm.tint + o;
        hrow_f = sm.tfrac + o;
        if (sm.tpd) hrow_d = sm.tpd + o;
      }
      if (i % TS == rem_i) {
        if (!dead) tile_issue(sm, d, ws, b, ts, r / TS + SG);
        const size_t o = tile_row_off(r, C);
        crow_i = sm.tint + o;
        crow_f = sm.tfrac + o;
        if (sm.tpd) crow_d = sm.tpd + o;
      }
      if (i == next_ck) {
        // rebase the ring to (F0 + D, S_int at the boundary): keeps the
        // integer parts small over long walks.  (No checkpoint is saved: both
        // rings of a sequence take the same domain, so the posteriors of this
        // kernel's sequences come from the kept rows, never from a walk.)
        const float D = comb ? Fp : Fph;  // both are Phi_{i-1} - F0
        if (comb) {
          const int sit = UP ? si_p : si_pp;
          if (act) {
            const float adj = sg * (float)(sit - Sbc) - D;
            for (int x = jl; x < RL; x += G) rl[x].y += adj;
            if (leader) xs.Sb[cl] = sit;
          }
        }
        __syncthreads();
        F0 += (double)D;
        if (comb) {
          Fp -= D;
        } else {
          Fph -= D;
        }
        Sbc = xs.Sb[ccl];
        next_ck += delta;
        if (UP ? next_ck - 1 >= L : L + 2 - next_ck < delta) next_ck = INT_MAX;
      }
      next_ev = next_event(i);
    }
    // the frame of the row the combine kept last step (Phi_{i-1})
    if (kv && rank == 0 && tid == nwc * 32 && i >= 2) kf[r - SG] = F0 + (double)Fph;
    // Each role issues its shared-memory reads first and its stores last: a
    // store the compiler cannot separate from later reads keeps those reads
    // from being issued early, and every access of the step must complete
    // before the barrier releases.
    if (comb) {
      // ---------------------------------------------------------- combine
      if constexpr (N > 1) {
        if (i >= 2) {
          // p_{i-1} from every CTA of the cluster
          const int pb = (i - 1) & 1;
          if (!xdead && !mbar_wait_cluster(&xs.pbar[pb], ((i - 2) >> 1) & 1, WAIT_SPIN_LIMIT)) {
            set_status(ws.status, ST_DEVICE_TIMEOUT);
            xdead = true;
          }
        }
      }
      const int po = (i & 1) * Cr + ccl;
      const float a1v = xs.A1[po], a2v = xs.A2[po];
      float ohv = xs.Oh[po];
#pragma unroll
      for (int hw = 1; hw < HW; ++hw) ohv += xs.Oh[hw * 2 * Cr + po];  // long durations
      const bool rok = SEMICRF_INB(ws.status, row_ok(crow_i), SITE_TILE_ROW);
      const int si_n = rok ? crow_i[cc] : 0;  // the walk's row r: the next step's ring entry
      const float sf_n = rok ? crow_f[cc] : 0.f;
      const float pd_n = (UP && crow_d && rok) ? crow_d[cc] : 0.f;
      const float* pv = xs.P + ((i - 1) & 1) * d.xPC + 4 * jl;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, m0 = 0.f, m1 = 0.f, m2 = 0.f, m3 = 0.f;
#pragma unroll
      for (int q = 0; q < CAT; q += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pv + q * G);
        a0 = fmaf(v.x, w[q], a0);
        a1 = fmaf(v.y, w[q + 1], a1);
        a2 = fmaf(v.z, w[q + 2], a2);
        a3 = fmaf(v.w, w[q + 3], a3);
        m0 = fmaxf(m0, v.x);
        m1 = fmaxf(m1, v.y);
        m2 = fmaxf(m2, v.z);
        m3 = fmaxf(m3, v.w);
      }
      float acc = gsum<G>((a0 + a1) + (a2 + a3));
      float mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL_MASK, mx, o));
      if (i == 1) {
        acc = acc_start;  // the start boundary: gamma = 0 in frame 0
        mx = 0.f;
      }
      // gamma (beta) of the previous row's boundary, frame Phi_{i-1}: its
      // logarithm is issued first so that its latency hides under the path
      const float gprev = (acc > 0.f) ? M + lg2(acc) : NEG_INF;
      const float n = exponent_of(mx);
      const float sn = pow2_neg(n);
      const float R = fmaf(acc2, a2v, ohv) * snprev;  // frame Phi_{i-1}
      const float pn = fmaf(acc * sn, a1v, R * sn);
      const bool pok = SEMICRF_INB(ws.status, !act || c < d.xPC, SITE_VECTOR);
      if constexpr (N > 1) {
        // into every CTA of the cluster (this one included)
        if (act && pok) {
          const uint32_t po = 4u * (uint32_t)((i & 1) * d.xPC + c), bo = 8u * (uint32_t)(i & 1);
#pragma unroll
          for (int u = 0; u < ND; ++u)
            if (jl + u * G < N) st_async_mapped(rbuf[u] + po, rbar[u] + bo, pn);
        }
      } else {
        if (leader && pok) xs.P[(i & 1) * d.xPC + c] = pn;
      }
      if (tid == 0) xs.nsl[i & 1] = n;
      // the kept row of this boundary, then the ring entry: global stores
      // after the critical store cost the path least (measured against the
      // helpers copying the row, and against storing after the ring entry)
      if (kv && leader &&
          SEMICRF_INB(ws.status, r >= 0 && r <= d.T && r - SG >= 0 && r - SG <= d.T, SITE_KEPT_ROW)) {
        kv[(size_t)r * 2 * C + c] = pn;                // row r, frame Phi_i
        kv[(size_t)(r - SG) * 2 * C + C + c] = acc;    // row r - SG, frame Phi_{i-1}
      }
      if (i >= 2 && leader && SEMICRF_INB(ws.status, wslot >= 0 && wslot < K, SITE_RING_SLOT))
        put(wslot, make_float2((gprev - sg * sf_p) + pd_p, Fp - sg * (float)(si_p - Sbc)));
      wslot = UP ? (wslot + 1 == K ? 0 : wslot + 1) : (wslot == 0 ? K - 1 : wslot - 1);
      acc2 = acc;
      snprev = sn;
      Fp += n;
      si_pp = si_p;
      si_p = si_n;
      sf_p = sf_n;
      pd_p = pd_n;
      crow_i += SG * C;
      crow_f += SG * C;
      if (crow_d) crow_d += SG * C;
    } else if (i < L) {
      // ---------------------------------------------------------- helpers
      const bool hok = SEMICRF_INB(ws.status, row_ok(hrow_i), SITE_TILE_ROW);
      const int sn = hok ? hrow_i[cc] : 0;
      const float fn = hok ? hrow_f[cc] : 0.f;
      const float dn = (hrow_d && hok) ? hrow_d[cc] : 0.f;
      const bool wok = SEMICRF_INB(ws.status, hbase >= 0 && hbase + jl + (KBH - 1) * H < RLP,
                                   SITE_RING_WINDOW);
      const float Qh = sg * (float)(sn - Sbc) - Fph;
      float m = Qh + rel;
      float s;
      const float lse = k_fanin_strided<KBH, H>(rl + (wok ? hbase : 0) + jl, Qh, w, m, s, act);
      if (isfinite(lse)) rel = rintf(lse - Qh);
      // the three values step i+1 reads: lanes 0, 1, 2 of the group take one
      // exponential each (no divergent branches); narrower groups take all
      const float aO = (m + (UP ? 0.f : dn)) + sg * fn;
      const float aA1 = ((M + d1) + (UP ? hd_c : dn)) + sg * ((float)(sn - hs_c) + (fn - hf_c));
      const float aA2 = ((M + d2) + (UP ? hd_p : dn)) + sg * ((float)(sn - hs_p) + (fn - hf_p));
      const int o2 = ((i + 1) & 1) * Cr + ccl;
      if constexpr (H >= 3) {
        // (several helper warps per label: each warp's lane 0 its partial
        // k >= 3 sum, the label's first warp the k = 1, 2 factors)
        const int ln = jl % HG;
        const float e = ex2(ln == 0 ? aO : (jl == 1 ? aA1 : aA2));
        if (act && ln == 0) xs.Oh[hwarp * 2 * Cr + o2] = (s > 0.f) ? s * e : 0.f;
        if (act && jl == 1) xs.A1[o2] = e;
        if (act && jl == 2) xs.A2[o2] = e;
      } else {
        const float eO = ex2(aO), e1 = ex2(aA1), e2 = ex2(aA2);
        if (leader) {
          xs.Oh[o2] = (s > 0.f) ? s * eO : 0.f;
          xs.A1[o2] = e1;
          xs.A2[o2] = e2;
        }
      }
      hs_p = hs_c;
      hf_p = hf_c;
      hd_p = hd_c;
      hs_c = sn;
      hf_c = fn;
      hd_c = dn;
      hrow_i += SG * C;
      hrow_f += SG * C;
      if (hrow_d) hrow_d += SG * C;
      hbase = UP ? (hbase + 1 == K ? 0 : hbase + 1) : (hbase == 0 ? K - 1 : hbase - 1);
    }
    __syncthreads();
  }
  if constexpr (N > 1) {
    // the last vector has arrived here (log Z reads it; no store into this
    // CTA is left in flight), then no CTA leaves before every CTA is done
    if (comb && !xdead &&
        !mbar_wait_cluster(&xs.pbar[L & 1], ((L - 1) >> 1) & 1, WAIT_SPIN_LIMIT))
      set_status(ws.status, ST_DEVICE_TIMEOUT);
    cluster_sync();
  }
  if (kv && rank == 0 && tid == nwc * 32)  // the last row's frame (its vector was kept at step L)
    kf[UP ? L : 0] = F0 + (double)(Fph + xs.nsl[L & 1]);

  // log2 Z = F0 + Phi_L + log2 sum_c p_L[c]
  if (warp == 0 && rank == 0) {
    float s = 0.f;
    for (int x = lane; x < C; x += 32) s += xs.P[(L & 1) * d.xPC + x];
    s = group_sum(s, 32);
    if (lane == 0) {
      const double lz = (s > 0.f) ? F0 + (double)Fp + (double)lg2(s) : -INFINITY;
      if (UP) {
        ws.logz2[b] = lz;
        logZ_out[b] = lz * LN2_D;
      } else {
        ws.logz2b[b] = lz;
      }
    }
  }
}

}  // namespace

size_t chain_exp_smem_bytes(const Dims& d, bool pj) {
  const size_t hw = (d.xH + 31) / 32;  // helper warps per label (long durations: > 1)
  return 96 + 2ull * TS * d.C * (pj ? 12 : 8) + (size_t)d.xRLP * d.xCr * 8 + 16 +
         (2ull * d.xPC + (5ull + 2 * hw) * d.xCr) * 4;
}

}  // namespace semicrf

namespace semicrf {
namespace {

// ===========================================================================
// One CTA, or one cluster of N CTAs, per (direction, sequence): ring q =
// blockIdx.x / N < n_alpha runs the forward ring of sequence q, the others
// the backward ring of sequence q - n_alpha.  Writes mode[direction][b];
// returns at once (mode 2) when the sequence needs the log-domain kernel.
// Every CTA of a cluster takes the same early exits (they depend only on the
// inputs), before any of them touches another's shared memory.
// ===========================================================================
template <int N, int G, int CAT, int H, int KBH, int LB>
__global__ void __launch_bounds__(LB, 1)
    chain_exp_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                     const float* __restrict__ trans, const float* __restrict__ dur,
                     double* __restrict__ logZ_out, int n_alpha, int pj) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const XSmem xs = xcarve(smem_raw, d, pj != 0);
  const int C = d.C, K = d.K, tid = threadIdx.x;
  const int rank = N > 1 ? (int)cluster_ctarank() : 0;
  const int q = (int)blockIdx.x / N;
  const bool up = q < n_alpha;
  const int b = up ? q : q - n_alpha;
  const int L = lengths[b];
  int* const mode = ws.mode + (up ? 0 : d.B) + b;
  if (L < 0 || L > d.T || L == 0) {
    if (tid == 0 && rank == 0) {
      const double v = (L == 0) ? 0.0 : __longlong_as_double(0x7ff8000000000000ll);
      if (L != 0) set_status(ws.status, ST_BAD_LENGTH);
      if (up) {
        logZ_out[b] = v;
        ws.logz2[b] = v;
      } else {
        ws.logz2b[b] = v;
      }
      *mode = 1;
    }
    return;
  }
  // ---- the fast-path test (identical in every CTA of the sequence): one
  // pass over trans and one over dur for finiteness and both extremes
  if (tid < 4) xs.aux[tid] = f2ord(NEG_INF);
  __syncthreads();
  bool bad = false;
  float tmx = NEG_INF, tmn = INFINITY, dmx = NEG_INF, dmn = INFINITY;
  for (int i = tid; i < C * C; i += blockDim.x) {
    const float raw = __ldg(trans + i);
    bad |= !isfinite(raw);
    tmx = fmaxf(tmx, raw * l2e());
    tmn = fminf(tmn, raw * l2e());
  }
  for (int i = tid; i < K * C; i += blockDim.x) {
    const float raw = __ldg(dur + i);
    bad |= !isfinite(raw);
    dmx = fmaxf(dmx, raw * l2e());
    dmn = fminf(dmn, raw * l2e());
  }
  warp_max_to_shared(&xs.aux[0], f2ord(tmx));
  warp_max_to_shared(&xs.aux[1], f2ord(-tmn));
  warp_max_to_shared(&xs.aux[2], f2ord(dmx));
  warp_max_to_shared(&xs.aux[3], f2ord(-dmn));
  bad = __syncthreads_or(bad);  // also completes the four reductions
  const float M = ord2f(xs.aux[0]);
  if (ws.tmax && threadIdx.x == 0 && blockIdx.x == 0) *ws.tmax = M;  // for the posterior pass
  const float tmin = -ord2f(xs.aux[1]);
  const float dmax = ord2f(xs.aux[2]);
  const float dmin = -ord2f(xs.aux[3]);
  const float span = fabsf(M) + (M - tmin) + fabsf(dmax) + fabsf(dmin) + 2.f * ws.emax[b] +
                     lg2((float)(K * C));
  if (bad || !(span < FAST_BOUND)) {
    if (tid == 0 && rank == 0) *mode = 2;
    return;
  }
  if (tid == 0 && rank == 0) *mode = 1;
  if (up)
    xring<true, N, G, CAT, H, KBH>(xs, d, ws, b, L, trans, dur, M, logZ_out, rank);
  else
    xring<false, N, G, CAT, H, KBH>(xs, d, ws, b, L, trans, dur, M, logZ_out, rank);
}

}  // namespace

bool xshape_supported(int N, int G, int CAT, int H, int KBH, int LB) {
#define SEMICRF_XSHAPE_OK(n, g, cat, h, kbh, lb) \
  if (N == n && G == g && CAT == cat && H == h && KBH == kbh && LB == lb) return true;
  SEMICRF_FOR_EACH_XSHAPE(SEMICRF_XSHAPE_OK)
#undef SEMICRF_XSHAPE_OK
  return false;
}

cudaError_t launch_chain_exp(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                             const float* trans, const float* dur, double* logZ_out, int n_alpha,
                             int n_beta, cudaStream_t st, int pj) {
  const size_t sm = chain_exp_smem_bytes(d, pj != 0);
#define SEMICRF_LAUNCH_XCHAIN(n, g, cat, h, kbh, lb)                                           \
  if (d.xN == n && d.xG == g && d.xCAT == cat && d.xH == h && d.xKBH == kbh && d.xLB == lb)    \
    return launch_clustered(chain_exp_kernel<n, g, cat, h, kbh, lb>, n, (n_alpha + n_beta) * n, \
                            d.xNT, sm, st, d, ws, lengths, trans, dur, logZ_out, n_alpha, pj);
  SEMICRF_FOR_EACH_XSHAPE(SEMICRF_LAUNCH_XCHAIN)
#undef SEMICRF_LAUNCH_XCHAIN
  return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
