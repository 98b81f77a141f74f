// api.cu -- the C ABI declared in include/semicrf.h: argument validation,
// launch geometry, workspace layout and kernel launches.  Host code only.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "semicrf.h"
#include "kernels.cuh"

namespace semicrf {

namespace {

constexpr int FIN_ROWS_HOST = 64;  // must match FIN_ROWS in finalize.cu

int pow2floor(int x) {
  int p = 1;
  while (p * 2 <= x) p *= 2;
  return p;
}


size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int isqrt_ceil(long long v) {
  long long r = (long long)std::sqrt((double)v);
  while (r * r > v) --r;
  while (r * r < v) ++r;
  return (int)r;
}

int sm_count() {
  static int cached = -1;
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (cached < 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1) {
      cudaGetLastError();
      v = 148;  // B200
    }
    cached = v;
  }
  return cached;
}

int max_smem_optin() {
  static int cached = -1;
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (cached < 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
      cudaGetLastError();
      v = 227 * 1024;  // sm_100 opt-in limit
    }
    cached = v;
  }
  return cached;
}

}  // namespace

// Shape of the pipelined exponential-domain rings (xG = 0: none fits, every
// sequence takes the log-domain kernel).  The step's latency is the longer of
// the combine path (CAT multiply-adds, log2 G shuffle levels) and the helper
// path (KBH exponentials, log2 H shuffle levels), plus issue time for the
// warps that share a scheduler.  One CTA per ring serves narrow label sets
// best; from C >= CLUSTER_MIN_C labels a ring is split over a thread-block
// cluster (N CTAs, C / N labels each): the per-step work of one SM shrinks
// N-fold and each step pays the label vector's exchange through distributed
// shared memory (about 400 cycles measured on B200, beside about 200 for a
// CTA barrier), which pays when one SM's step is several thousand cycles.
// At C = 128, K = 64 a step measured about 4300 cycles on one CTA; 1270 on
// a cluster of 4 and 1240 on 8 (forward-backward), 1280 and 1020 (the
// decoder, whose helpers are lighter).  Forward-backward prefers clusters of
// 4 and the decoder 8 where its clusters fit the GPU at once: at B = 8 the
// two rings (64 SMs) and the decoder (64) then run side by side.
// SEMICRF_XSHAPE=i forces the i-th fitting shape of the menu and
// SEMICRF_XCLUSTER=n restricts the choice to clusters of n CTAs (tuning).
constexpr int CLUSTER_MIN_C = 96;
constexpr int LONG_K = 2050;  // above: helper lanes of a label span several warps
// Fills the derived fields of a pipelined shape (ring rows, label-vector
// length, bank padding).
void xshape_derive(Dims& d) {
  d.xRL = d.K + d.xKBH;
  // label vector row: the combine lanes' blocks (xG x xCAT) and the helper
  // lanes' strided sources (xH x ceil(xG xCAT / xH)), whichever is longer
  d.xPC = std::max(d.xG * d.xCAT, d.xH * ((d.xG * d.xCAT + d.xH - 1) / d.xH));
  d.xRLP = d.K + d.xH * d.xKBH;
  if (d.xH < 16) d.xRLP += (((d.xH - d.xRLP) % 16) + 16) % 16;
}

void choose_xshape(Dims& d, size_t budget, int prefer_n) {
  const int C = d.C, K = d.K;
  int forced = -1, forced_n = 0;
  if (const char* env = std::getenv("SEMICRF_XSHAPE")) forced = std::atoi(env);
  if (const char* env = std::getenv("SEMICRF_XCLUSTER")) forced_n = std::atoi(env);
  d.xG = 0;
  d.xN = 1;
  d.xCr = C;
  d.pRT = 0;
  double best = 1e30;
  int idx = 0;
  auto lg = [](int v) {
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
  };
  const int want_n = forced_n > 0 ? forced_n : 0;
  // wide label sets, and long durations (a label's ring and window then fill
  // one SM's shared memory: one label per CTA)
  const bool needs_cluster = C >= CLUSTER_MIN_C || (K > LONG_K && C > 1);
  Dims pick = d;
#define SEMICRF_XCONSIDER(n, g, cat, h, kbh, lb)                                          \
  {                                                                                       \
    const int cr = (C + n - 1) / n;                                                       \
    const int nwc = (cr + 32 / g - 1) / (32 / g);                                         \
    const int nwh = h > 32 ? cr * (h / 32) : (cr + 32 / h - 1) / (32 / h);                \
    const int nt = 32 * (nwc + nwh);                                                      \
    const bool cl_ok = want_n ? (n == want_n) : ((n > 1) == needs_cluster);              \
    if (C <= g * cat && K <= h * kbh + 2 && nt <= lb && cl_ok && (n == 1 || cr * n - C < cr)) { \
      Dims t = d;                                                                         \
      t.xN = n;                                                                           \
      t.xCr = cr;                                                                         \
      t.xG = g;                                                                           \
      t.xCAT = cat;                                                                       \
      t.xH = h;                                                                           \
      t.xKBH = kbh;                                                                       \
      t.xLB = lb;                                                                         \
      t.xNT = nt;                                                                         \
      xshape_derive(t);                                                                   \
      if (chain_exp_smem_bytes(t) <= budget && viterbi_pipe_smem_bytes(t) <= budget) {   \
        const double cost = std::max(cat + 25.0 * lg(g), 2.0 * kbh + 25.0 * lg(h)) +      \
                            10.0 * ((nwc + nwh + 3) / 4) + (lb > 512 ? 1000.0 : 0.0) +    \
                            (n > 1 ? 100.0 + 25.0 * std::abs(n - prefer_n) : 0.0);        \
        if ((forced < 0 && cost < best) || forced == idx) {                               \
          best = cost;                                                                    \
          pick = t;                                                                       \
        }                                                                                 \
        ++idx;                                                                            \
      }                                                                                   \
    }                                                                                     \
  }
  SEMICRF_FOR_EACH_XSHAPE(SEMICRF_XCONSIDER)
#undef SEMICRF_XCONSIDER
  if (pick.xG == 0) return;
  d = pick;
  // the posterior pass from the kept values and the cut normaliser must fit too
  d.pRT = posterior_tile_rows(d, budget);
  if (d.pRT == 0 || cut_grid_smem_bytes(d, budget) > budget || d.C > 128) {
    d.xG = 0;
    d.xN = 1;
    d.xCr = C;
  }
}

// Sizes, lane mapping and limits.  Returns a semicrf_status.
int make_dims(int B, int T, int C, int K, Dims& d) {
  if (B < 0 || T < 0 || C < 1 || K < 1) return SEMICRF_ERR_INVALID_ARG;
  if (C > C_MAX || K > K_MAX || (long long)K * C > KC_MAX || T > (1 << 26) || B > (1 << 20))
    return SEMICRF_ERR_UNSUPPORTED;
  d = Dims{};
  d.B = B;
  d.T = T;
  d.C = C;
  d.K = K;
  // Checkpoint spacing: ceil(sqrt(T K)) balances checkpoint memory against
  // recompute, but memory is not what binds here -- the posterior pass runs
  // one CTA per (segment, sequence).  So Delta is also capped at what gives
  // the batch at most two segment CTAs per SM in all (one wave), each
  // sequence an equal share, though never below 2K.  Any spacing gives the
  // same results in exact arithmetic.
  d.delta = T > 0 ? isqrt_ceil((long long)T * K) : 1;
  if (T > 0) {
    const long long per_seq = std::max<long long>(1, 2LL * sm_count() / std::max(B, 1));
    const long long par = (T + per_seq - 1) / per_seq;
    d.delta = (int)std::min<long long>(d.delta, std::max<long long>(2LL * K, par));
  }
  if (d.delta < 1) d.delta = 1;
  d.nck = T > 0 ? (T + d.delta - 1) / d.delta : 1;
  d.Tstride = ((T + 1 + TS - 1) / TS) * TS;
  // Cut-normaliser grid: every 256 positions, sparser for long durations (a
  // grid point costs K(K+1)/2 C terms; the two rings' rounding drifts by about
  // 1e-7 per position, so linear interpolation over 2048 positions still
  // keeps the marginals' error far below 1e-4)
  d.GS = 256;
  while (d.GS < 2048 && d.GS * 4 < K) d.GS *= 2;
  d.ngrid = T > 0 ? (T - 1) / d.GS + 2 : 1;  // positions 0, GS, 2GS, ... and L - 1
  d.npch = std::max(1, (T + PATH_ROWS - 1) / PATH_ROWS);
  // Kernel shape: G lanes per label (a power of two), each with KBT durations
  // and CAT labels, picked from the instantiated menu by a latency model.
  // Per step about one warp runs per scheduler and the step is latency
  // bound: the model charges the warps sharing a scheduler, the sequential
  // k fan-in terms of a lane, its shuffle levels and its label terms (weights
  // fitted to measured step times on B200).
  // SEMICRF_LANES=G restricts the choice to that G (tuning; ignored if no
  // shape with that G fits).
  int forced = 0;
  if (const char* env = std::getenv("SEMICRF_LANES")) forced = std::atoi(env);
  d.KBT = 0;
  double best = 1e30;
  for (int pass = 0; pass < 2 && d.KBT == 0; ++pass) {
#define SEMICRF_CONSIDER(a, b, g, lb)                                                   \
  {                                                                                     \
    const int nt = std::max(32, ((C * g + 31) / 32) * 32);                              \
    const bool fits = (K <= a * g) && (C <= b * g) && (nt <= lb) && (lb == 512 || nt <= 256); \
    if (fits && (pass == 1 || forced <= 0 || forced == g)) {                            \
      int lg = 0;                                                                       \
      while ((1 << lg) < g) ++lg;                                                       \
      const int warps = nt / 32;                                                        \
      const double cost = ((warps + 3) / 4) * 60.0 + 12.0 * a + 6.0 * lg + 1.25 * b;   \
      if (cost < best) {                                                                \
        best = cost;                                                                    \
        d.KBT = a;                                                                      \
        d.CAT = b;                                                                      \
        d.GB = g;                                                                       \
        d.LB = lb;                                                                      \
        d.NT = nt;                                                                      \
      }                                                                                 \
    }                                                                                   \
  }
    SEMICRF_FOR_EACH_SHAPE(SEMICRF_CONSIDER)
#undef SEMICRF_CONSIDER
  }
  d.prefR = std::max(16, pow2floor(8192 / C));
  d.nchunk = T > 0 ? (T + d.prefR - 1) / d.prefR : 1;
  d.store_w = 2 * C + 2;
  // the per-block limit covers static shared memory too (a few bytes here)
  const size_t budget = (size_t)max_smem_optin() - 256;
  if (d.KBT) {
    d.GA = d.GB;
    d.RL = K + d.KBT;
    d.PC = ((std::max(C, d.GB * d.CAT) + 3) / 4) * 4;
    d.store_smem = recursion_smem_bytes(d, true) <= budget ? 1 : 0;
    if (recursion_smem_bytes(d, false) > budget) d.KBT = 0;
  }
  // sizes without a log-domain shape are served only in the long-duration
  // regime (K > LOG_K_MAX, C <= 8: the pipelined kernels alone)
  if (!d.KBT && K <= LOG_K_MAX) return SEMICRF_ERR_UNSUPPORTED;
  if (!d.KBT) {  // no log-domain kernels for these sizes (long durations)
    d.KBT = d.GB = d.CAT = d.GA = d.RL = d.NT = d.LB = 0;
    d.PC = ((C + 3) / 4) * 4;
    d.store_smem = 1;  // nothing to store
  }
  choose_xshape(d, budget, 4);
  // a size needs the pipelined kernels or the log-domain ones
  if (!d.KBT && !d.xG) return SEMICRF_ERR_UNSUPPORTED;
  return SEMICRF_OK;
}

namespace {

// Workspace layout; fills `p` when base != nullptr.  Returns total bytes.
size_t layout(const Dims& d, void* base, WsPtrs* p, size_t* groups = nullptr) {
  size_t off = 0;
  int group = 0;  // SEMICRF_WS_* group of the regions taken next
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    if (groups) groups[group] += off - o;
    return o;
  };
  const size_t B = d.B, C = d.C, K = d.K, nck = d.nck;
  group = SEMICRF_WS_OTHER;
  const size_t o_status = take(256);
  group = SEMICRF_WS_PREFIX;
  const size_t o_sint = take(B * d.Tstride * C * 4);
  const size_t o_sfrac = take(B * d.Tstride * C * 4);
  const size_t o_chunk = take(B * d.nchunk * C * 8);
  group = SEMICRF_WS_OTHER;
  const size_t o_lz = take(B * 8);
  const size_t o_lzb = take(B * 8);
  group = SEMICRF_WS_CHECKPOINTS;
  const size_t o_ack = take(B * nck * K * C * 8);
  const size_t o_acf = take(B * nck * 8);
  const size_t o_bck = take(B * nck * K * C * 8);
  const size_t o_bcf = take(B * nck * 8);
  group = SEMICRF_WS_RECOMPUTE;
  const size_t o_store = take(d.store_smem ? 0 : B * nck * (size_t)d.delta * d.store_w * 4);
  const size_t o_pgt = take(B * nck * C * C * 8);
  const size_t o_pgd = take(B * nck * K * C * 8);
  const size_t o_segT = take(B * nck * C * 8);
  const size_t o_segV = take(B * nck * C * 8);
  group = SEMICRF_WS_VITERBI;
  const size_t o_bp = take(B * (size_t)(d.T + 1) * C * 4);
  const size_t o_vrow = take(d.xG ? B * (size_t)(d.T + 1) * C * 4 : 0);
  const size_t CP = (C + 3) / 4 * 4;
  const size_t o_wrd = take(d.xG ? B * (size_t)(d.T + 1) * CP * 4 : 0);
  const size_t o_varg = take(d.xG ? B * (size_t)(d.T + 1) * CP * 4 : 0);
  group = SEMICRF_WS_KEPT_ROWS;
  const size_t o_kv = take(B * 2ull * (d.T + 1) * 2 * C * 4);
  const size_t o_kf = take(B * 2ull * (d.T + 1) * 8);
  const size_t o_ncut = take(B * (size_t)d.ngrid * 8);
  group = SEMICRF_WS_OTHER;
  const size_t o_emax = take(B * 4);
  const size_t o_mode = take(2 * B * 4);
  const size_t o_tmax = take(4);
  const size_t pz = (B * (C * C + K * C) + 2 * B) * 4;  // pcnt | pbad | pdone
  group = SEMICRF_WS_PATH;
  const size_t o_pcnt = take(pz);
  group = SEMICRF_WS_PROJ;
  const size_t o_pd = take(B * d.Tstride * C * 4);
  group = SEMICRF_WS_PATH;
  const size_t o_psum = take(B * (size_t)d.npch * C * 8);
  const size_t o_plab = take(B * (size_t)d.npch * C * 4);
  const size_t o_pscr = take(B * (size_t)d.npch * 8);
  const size_t o_pfr = take(B * C * 8);
  const size_t o_pw = take(B * 8);
  if (base && p) {
    char* c = static_cast<char*>(base);
    p->status = reinterpret_cast<int*>(c + o_status);
    p->sint = reinterpret_cast<int32_t*>(c + o_sint);
    p->sfrac = reinterpret_cast<float*>(c + o_sfrac);
    p->chunk = reinterpret_cast<double*>(c + o_chunk);
    p->logz2 = reinterpret_cast<double*>(c + o_lz);
    p->logz2b = reinterpret_cast<double*>(c + o_lzb);
    p->ack = reinterpret_cast<float2*>(c + o_ack);
    p->acf = reinterpret_cast<double*>(c + o_acf);
    p->bck = reinterpret_cast<float2*>(c + o_bck);
    p->bcf = reinterpret_cast<double*>(c + o_bcf);
    p->store = reinterpret_cast<float*>(c + o_store);
    p->pgt = reinterpret_cast<double*>(c + o_pgt);
    p->pgd = reinterpret_cast<double*>(c + o_pgd);
    p->segT = reinterpret_cast<double*>(c + o_segT);
    p->segV = reinterpret_cast<double*>(c + o_segV);
    p->bp = reinterpret_cast<int32_t*>(c + o_bp);
    p->vrow = reinterpret_cast<float*>(c + o_vrow);
    p->wrd = reinterpret_cast<int32_t*>(c + o_wrd);
    p->varg = reinterpret_cast<int32_t*>(c + o_varg);
    p->kv = reinterpret_cast<float*>(c + o_kv);
    p->kf = reinterpret_cast<double*>(c + o_kf);
    p->ncut = reinterpret_cast<double*>(c + o_ncut);
    p->emax = reinterpret_cast<float*>(c + o_emax);
    p->mode = reinterpret_cast<int*>(c + o_mode);
    p->tmax = reinterpret_cast<float*>(c + o_tmax);
    p->pcnt = reinterpret_cast<int32_t*>(c + o_pcnt);
    p->psum = reinterpret_cast<double*>(c + o_psum);
    p->plab = reinterpret_cast<int32_t*>(c + o_plab);
    p->pscr = reinterpret_cast<double*>(c + o_pscr);
    p->pfr = reinterpret_cast<double*>(c + o_pfr);
    p->pw = reinterpret_cast<double*>(c + o_pw);
    p->pbad = p->pcnt + B * (C * C + K * C);
    p->pdone = p->pbad + B;
    p->pzero_bytes = pz;
    p->pon = p->status + 1;
    p->pd = reinterpret_cast<float*>(c + o_pd);
  }
  return off;
}

constexpr unsigned KNOWN_FLAGS = SEMICRF_FLAG_NO_CENTER | SEMICRF_FLAG_FORWARD_ONLY |
                                  SEMICRF_FLAG_LOG_DOMAIN | SEMICRF_FLAG_NEGATE_GRAD;

int prepare(int B, int T, int C, int K, unsigned flags, void* ws, size_t ws_bytes, Dims& d,
            WsPtrs& p) {
  if (flags & ~KNOWN_FLAGS) return SEMICRF_ERR_INVALID_ARG;
  const int rc = make_dims(B, T, C, K, d);
  if (rc != SEMICRF_OK) return rc;
  if (!ws) return SEMICRF_ERR_INVALID_ARG;
  const size_t need = layout(d, nullptr, nullptr);
  if (ws_bytes < need) return SEMICRF_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(ws) & 255) return SEMICRF_ERR_INVALID_ARG;
  layout(d, ws, &p);
  return SEMICRF_OK;
}

int set_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return SEMICRF_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return SEMICRF_ERR_CUDA;
  }
  return SEMICRF_OK;
}

int launched() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SEMICRF_OK : SEMICRF_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Optional per-kernel device timing: when enabled, every kernel launch is
// bracketed by two CUDA events recorded on its own stream; reading the
// profile synchronises on them and sums the elapsed times per kernel name.
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex prof_mu;
bool prof_on = false;
std::vector<ProfRec> prof_recs;

// A second stream, per host thread and device, for the kernels of the
// backward pass that do not depend on each other; forked from and joined
// back into the caller's stream with events (which stream capture also
// records), so the call stays ordered on the caller's stream.  nullptr if
// it cannot be created: the caller's stream then runs everything.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
SideStream* side_stream() {
  thread_local std::vector<SideStream> per_dev;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return nullptr;
  }
  if ((int)per_dev.size() <= dev) per_dev.resize(dev + 1);
  SideStream& ss = per_dev[dev];
  if (!ss.s) {
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      ss = SideStream{};
      return nullptr;
    }
  }
  return &ss;
}
// The side stream waits for everything queued on st so far.
bool side_fork(SideStream* ss, cudaStream_t st) {
  return !ss || (cudaEventRecord(ss->fork, st) == cudaSuccess &&
                 cudaStreamWaitEvent(ss->s, ss->fork, 0) == cudaSuccess);
}
// st waits for everything queued on the side stream so far.
bool side_join(SideStream* ss, cudaStream_t st) {
  return !ss || (cudaEventRecord(ss->join, ss->s) == cudaSuccess &&
                 cudaStreamWaitEvent(st, ss->join, 0) == cudaSuccess);
}

struct ProfScope {
  cudaStream_t st;
  ProfRec rec{nullptr, nullptr, nullptr};
  ProfScope(const char* name, cudaStream_t s) : st(s) {
    std::lock_guard<std::mutex> g(prof_mu);
    if (!prof_on) return;
    rec.name = name;
    if (cudaEventCreate(&rec.a) != cudaSuccess || cudaEventCreate(&rec.b) != cudaSuccess) {
      cudaGetLastError();
      rec.name = nullptr;
      return;
    }
    cudaEventRecord(rec.a, st);
  }
  ~ProfScope() {
    if (!rec.name) return;
    cudaEventRecord(rec.b, st);
    std::lock_guard<std::mutex> g(prof_mu);
    prof_recs.push_back(rec);
  }
};

// Both rings (forward of n_alpha sequences, backward of n_beta): the
// exponential-domain kernel takes every sequence whose scores fit it and
// marks the rest, which the log-domain kernel then runs.
// Whether the pipelined exponential-domain kernels serve this call: their
// shape exists, the log domain is not forced, and with boundary projections
// their larger tile stream still fits shared memory.
bool pipelined(const Dims& d, unsigned flags, bool proj) {
  if (!d.xG || (flags & SEMICRF_FLAG_LOG_DOMAIN)) return false;
  if (!proj) return true;
  const size_t budget = (size_t)max_smem_optin() - 256;
  return chain_exp_smem_bytes(d, true) <= budget && viterbi_pipe_smem_bytes(d, true) <= budget &&
         posterior_smem_bytes(d) <= budget;
}

int run_chains(const Dims& d, WsPtrs p, const int32_t* lengths, const float* trans,
               const float* dur, double* logZ, int n_alpha, int n_beta, unsigned flags,
               cudaStream_t st, bool proj = false) {
  cudaError_t e = cudaSuccess;
  // long durations have only the pipelined kernels
  if (!d.KBT && !pipelined(d, flags, proj)) return SEMICRF_ERR_UNSUPPORTED;
  if (pipelined(d, flags, proj)) {
    ProfScope ps("chain_exp_kernel", st);
    e = launch_chain_exp(d, p, lengths, trans, dur, logZ, n_alpha, n_beta, st, proj ? 1 : 0);
  } else {
    // no ring kept anything: the posterior pass must not trust a record left
    // in the workspace by an earlier call
    if (cudaMemsetAsync(p.mode, 0, 2ull * d.B * sizeof(int), st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
    p.mode = nullptr;  // the log-domain kernel runs every sequence
  }
  if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
  {
    ProfScope ps("chain_kernel", st);
    e = launch_chain(d, p, lengths, trans, dur, logZ, n_alpha, n_beta, st);
  }
  return e == cudaSuccess ? SEMICRF_OK : SEMICRF_ERR_CUDA;
}

int run_prefix(const float* em, const int32_t* lengths, const Dims& d, const WsPtrs& p,
               unsigned flags, int mode, double* S64, float* nu, cudaStream_t st,
               const float* p_start = nullptr, const float* p_end = nullptr) {
  if (d.B == 0 || d.T == 0) return SEMICRF_OK;
  const dim3 grid(d.nchunk, d.B);
  {
    ProfScope ps("prefix_reduce_kernel", st);
    prefix_reduce_kernel<<<grid, 256, 0, st>>>(em, lengths, d, p);
  }
  const size_t sm = prefix_scan_smem_bytes(d);
  int rc = set_smem((const void*)prefix_scan_kernel, sm);
  if (rc) return rc;
  {
    ProfScope ps("prefix_scan_kernel", st);
    prefix_scan_kernel<<<grid, 256, sm, st>>>(em, lengths, d, p,
                                              (flags & SEMICRF_FLAG_NO_CENTER) ? 0u : 1u, mode,
                                              S64, nu, p_start, p_end);
  }
  return launched();
}

}  // namespace
}  // namespace semicrf

using namespace semicrf;

extern "C" int semicrf_workspace_bytes(int B, int T, int C, int K, unsigned flags, size_t* bytes) {
  if (!bytes || (flags & ~KNOWN_FLAGS)) return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  const int rc = make_dims(B, T, C, K, d);
  if (rc != SEMICRF_OK) return rc;
  *bytes = layout(d, nullptr, nullptr);
  return SEMICRF_OK;
}

extern "C" int semicrf_launch_shape(int B, int T, int C, int K, int32_t* shape, int n) {
  if (!shape || n < 0) return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  const int rc = make_dims(B, T, C, K, d);
  if (rc != SEMICRF_OK) return rc;
  const int32_t v[SEMICRF_SHAPE_FIELDS] = {d.xG ? d.xN : 0, d.xCr, d.xG, d.xCAT, d.xH, d.xKBH,
                                           d.xNT, d.delta, d.nck, d.pRT, d.KBT, d.GB, d.CAT, d.NT,
                                           d.pKH, d.GS};
  for (int i = 0; i < n; ++i) shape[i] = i < SEMICRF_SHAPE_FIELDS ? v[i] : 0;
  return SEMICRF_OK;
}

extern "C" int semicrf_workspace_itemize(int B, int T, int C, int K, unsigned flags,
                                         size_t* bytes, int n) {
  if (!bytes || n < 0 || (flags & ~KNOWN_FLAGS)) return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  const int rc = make_dims(B, T, C, K, d);
  if (rc != SEMICRF_OK) return rc;
  size_t g[SEMICRF_WS_GROUPS] = {};
  layout(d, nullptr, nullptr, g);
  for (int i = 0; i < n; ++i) bytes[i] = i < SEMICRF_WS_GROUPS ? g[i] : 0;
  return SEMICRF_OK;
}

extern "C" int semicrf_prefix_center(const float* em, const int32_t* lengths, int B, int T, int C,
                                     unsigned flags, void* ws, size_t ws_bytes, double* S,
                                     float* nu, semicrf_stream_t stream) {
  if (!lengths || !S || !nu || (B > 0 && T > 0 && !em)) return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  const int rc = prepare(B, T, C, 1, flags & ~SEMICRF_FLAG_FORWARD_ONLY, ws, ws_bytes, d, p);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(p.status, 0, sizeof(int), st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  if (B == 0) return SEMICRF_OK;
  if (T == 0) {
    if (cudaMemsetAsync(S, 0, (size_t)B * C * sizeof(double), st) != cudaSuccess ||
        cudaMemsetAsync(nu, 0, (size_t)B * C * sizeof(float), st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
    return SEMICRF_OK;
  }
  return run_prefix(em, lengths, d, p, flags, 0, S, nu, st);
}

namespace {

// Status word and projection switch: every forward / decode starts with both
// cleared; a call with boundary projections then sets the switch, which the
// kernels of this call and of the backward that consumes it read.
int reset_status(const WsPtrs& p, bool proj, cudaStream_t st) {
  if (cudaMemsetAsync(p.status, 0, 2 * sizeof(int), st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  if (proj && cudaMemsetAsync(p.pon, 1, 1, st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  return SEMICRF_OK;
}

int forward_impl(const float* em, const int32_t* lengths, const float* trans, const float* dur,
                 const float* p_start, const float* p_end, int B, int T, int C, int K,
                 unsigned flags, void* ws, size_t ws_bytes, double* logZ, cudaStream_t st) {
  if (!lengths || !trans || !dur || !logZ || (B > 0 && T > 0 && !em)) return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  int rc = prepare(B, T, C, K, flags, ws, ws_bytes, d, p);
  if (rc) return rc;
  const bool proj = p_start || p_end;
  if ((rc = reset_status(p, proj, st))) return rc;
  if (B == 0) return SEMICRF_OK;
  rc = run_prefix(em, lengths, d, p, flags, 1, nullptr, nullptr, st, p_start, p_end);
  if (rc) return rc;
  const int nbeta = (flags & SEMICRF_FLAG_FORWARD_ONLY) ? 0 : B;
  return run_chains(d, p, lengths, trans, dur, logZ, B, nbeta, flags, st, proj);
}

}  // namespace

extern "C" int semicrf_forward(const float* em, const int32_t* lengths, const float* trans,
                               const float* dur, int B, int T, int C, int K, unsigned flags,
                               void* ws, size_t ws_bytes, double* logZ, semicrf_stream_t stream) {
  return forward_impl(em, lengths, trans, dur, nullptr, nullptr, B, T, C, K, flags, ws, ws_bytes,
                      logZ, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int semicrf_forward_proj(const float* em, const int32_t* lengths, const float* trans,
                                    const float* dur, const float* p_start, const float* p_end,
                                    int B, int T, int C, int K, unsigned flags, void* ws,
                                    size_t ws_bytes, double* logZ, semicrf_stream_t stream) {
  return forward_impl(em, lengths, trans, dur, p_start, p_end, B, T, C, K, flags, ws, ws_bytes,
                      logZ, reinterpret_cast<cudaStream_t>(stream));
}

namespace {

int backward_impl(const int32_t* lengths, const float* trans, const float* dur, int B, int T,
                  int C, int K, unsigned flags, void* ws, size_t ws_bytes,
                  const double* grad_logZ, float* grad_em, float* grad_trans, float* grad_dur,
                  float* grad_p_start, float* grad_p_end, float* pos_marg, float* start_marg,
                  float* end_marg, bool proj, cudaStream_t st, float* seg_marg = nullptr) {
  if (!lengths || !trans || !dur || !grad_trans || !grad_dur || (B > 0 && T > 0 && !grad_em))
    return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  int rc = prepare(B, T, C, K, flags, ws, ws_bytes, d, p);
  if (rc) return rc;
  if (proj && !pipelined(d, flags, true)) flags |= SEMICRF_FLAG_LOG_DOMAIN;  // as the forward ran
  const bool want_pg = (grad_p_start || grad_p_end) && T > 0;
  if (want_pg) {
    // the projection gradients are g times the boundary marginals; without
    // caller buffers those go to the decoder's rows of the workspace
    // ([B][T+1][C] four-byte entries each, unused between a forward and its
    // backward), or, without a pipelined shape, to the exponential-domain
    // rows (then unused too)
    if (d.xG) {
      if (!start_marg) start_marg = p.vrow;
      if (!end_marg) end_marg = reinterpret_cast<float*>(p.bp);
    } else {
      if (!start_marg) start_marg = p.kv;
      if (!end_marg) end_marg = p.kv + (size_t)B * (T + 1) * C;
    }
  }
  if (B == 0) {
    if (cudaMemsetAsync(grad_trans, 0, (size_t)C * C * 4, st) != cudaSuccess ||
        cudaMemsetAsync(grad_dur, 0, (size_t)K * C * 4, st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
    return SEMICRF_OK;
  }
  if (flags & SEMICRF_FLAG_FORWARD_ONLY) {
    rc = run_chains(d, p, lengths, trans, dur, nullptr, 0, B, flags, st, proj);
    if (rc) return rc;
  }
  // segment marginals: every entry the posterior kernels do not write (past
  // a length, segments running past the end) is zero
  if (seg_marg && T > 0 &&
      cudaMemsetAsync(seg_marg, 0, (size_t)B * T * K * C * sizeof(float), st) != cudaSuccess)
    return SEMICRF_ERR_CUDA;
  if (T > 0) {
    // sequences whose rings both ran in the exponential domain: posteriors
    // from the kept values (cut normalisers, then one parallel pass); the
    // others: the checkpoint walk.  Each kernel skips the other's sequences.
    cudaError_t e = cudaSuccess, e_seg;
    // the checkpoint walk (side stream) and the posterior pass take
    // different sequences
    SideStream* ss = side_stream();
    const cudaStream_t s2 = ss ? ss->s : st;
    if (!side_fork(ss, st)) return SEMICRF_ERR_CUDA;
    {
      ProfScope ps("segment_kernel", s2);
      e_seg = launch_segment(d, p, lengths, trans, dur, grad_logZ, grad_em, start_marg, end_marg, s2,
                             seg_marg);
    }
    if (d.xG) {
      const size_t budget = (size_t)max_smem_optin() - 256;
      const size_t csm = cut_grid_smem_bytes(d, budget);
      if ((rc = set_smem((const void*)cut_grid_kernel, csm))) return rc;
      {
        ProfScope ps("cut_grid_kernel", st);
        cut_grid_kernel<<<dim3(d.ngrid, B), 256, csm, st>>>(d, p, lengths, trans, dur,
                                                            proj ? 1 : 0,
                                                            cut_grid_per_label(d, budget) ? 1 : 0);
      }
      if ((rc = launched())) return rc;
      {
        ProfScope ps("posterior_kernel", st);
        e = launch_posterior(d, p, lengths, trans, dur, grad_logZ, grad_em, start_marg, end_marg, st,
                             seg_marg, proj ? 1 : 0);
      }
    }
    if (!side_join(ss, st)) return SEMICRF_ERR_CUDA;
    if (e != cudaSuccess || e_seg != cudaSuccess) return SEMICRF_ERR_CUDA;
    const int nj = FIN_ROWS_HOST / d.delta + 2;
    const size_t fsm = ((size_t)C + (size_t)nj * C) * sizeof(double);
    rc = set_smem((const void*)finalize_positions_kernel, fsm);
    if (rc) return rc;
    // the parameter-gradient sums (side stream) and the per-position outputs
    // read different partials
    if (!side_fork(ss, st)) return SEMICRF_ERR_CUDA;
    {
      ProfScope ps("reduce_partials_kernel", s2);
      reduce_partials_kernel<<<(C * C + K * C + RP_E - 1) / RP_E, RP_E * RP_S, 0, s2>>>(
          d, p, lengths, grad_trans, grad_dur);
    }
    const int rc_red = launched();
    {
      ProfScope ps("finalize_positions_kernel", st);
      finalize_positions_kernel<<<dim3((T + FIN_ROWS_HOST - 1) / FIN_ROWS_HOST, B), 256, fsm,
                                  st>>>(d, p, lengths, grad_logZ,
                                        (flags & SEMICRF_FLAG_NO_CENTER) ? 0u : 1u, grad_em,
                                        pos_marg, start_marg, end_marg);
    }
    rc = launched();
    if (!side_join(ss, st)) return SEMICRF_ERR_CUDA;
    if (rc_red || rc) return rc_red ? rc_red : rc;
    if (want_pg) {
      ProfScope ps("proj_grad_kernel", st);
      if (launch_proj_grad(d, lengths, grad_logZ, start_marg, end_marg, grad_p_start, grad_p_end,
                           st) != cudaSuccess)
        return SEMICRF_ERR_CUDA;
    }
    return SEMICRF_OK;
  } else {
    // T == 0: only boundary row 0 exists, and nothing starts or ends there
    if (start_marg && cudaMemsetAsync(start_marg, 0, (size_t)B * C * 4, st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
    if (end_marg && cudaMemsetAsync(end_marg, 0, (size_t)B * C * 4, st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
  }
  const int ne = C * C + K * C;
  {
    ProfScope ps("reduce_partials_kernel", st);
    reduce_partials_kernel<<<(ne + RP_E - 1) / RP_E, RP_E * RP_S, 0, st>>>(d, p, lengths, grad_trans,
                                                                      grad_dur);
  }
  return launched();
}

}  // namespace

extern "C" int semicrf_backward(const int32_t* lengths, const float* trans, const float* dur,
                                int B, int T, int C, int K, unsigned flags, void* ws,
                                size_t ws_bytes, const double* grad_logZ, float* grad_em,
                                float* grad_trans, float* grad_dur, float* pos_marg,
                                float* start_marg, float* end_marg, semicrf_stream_t stream) {
  return backward_impl(lengths, trans, dur, B, T, C, K, flags, ws, ws_bytes, grad_logZ, grad_em,
                       grad_trans, grad_dur, nullptr, nullptr, pos_marg, start_marg, end_marg,
                       false, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int semicrf_backward_segments(const int32_t* lengths, const float* trans,
                                         const float* dur, int B, int T, int C, int K,
                                         unsigned flags, void* ws, size_t ws_bytes,
                                         const double* grad_logZ, float* grad_em,
                                         float* grad_trans, float* grad_dur, float* pos_marg,
                                         float* start_marg, float* end_marg, float* seg_marg,
                                         semicrf_stream_t stream) {
  if (!seg_marg && B > 0 && T > 0) return SEMICRF_ERR_INVALID_ARG;
  return backward_impl(lengths, trans, dur, B, T, C, K, flags, ws, ws_bytes, grad_logZ, grad_em,
                       grad_trans, grad_dur, nullptr, nullptr, pos_marg, start_marg, end_marg,
                       false, reinterpret_cast<cudaStream_t>(stream), seg_marg);
}

extern "C" int semicrf_backward_proj(const int32_t* lengths, const float* trans, const float* dur,
                                     int B, int T, int C, int K, unsigned flags, void* ws,
                                     size_t ws_bytes, const double* grad_logZ, float* grad_em,
                                     float* grad_trans, float* grad_dur, float* grad_p_start,
                                     float* grad_p_end, float* pos_marg, float* start_marg,
                                     float* end_marg, semicrf_stream_t stream) {
  return backward_impl(lengths, trans, dur, B, T, C, K, flags, ws, ws_bytes, grad_logZ, grad_em,
                       grad_trans, grad_dur, grad_p_start, grad_p_end, pos_marg, start_marg,
                       end_marg, true, reinterpret_cast<cudaStream_t>(stream));
}

namespace {

int viterbi_impl(const float* em, const int32_t* lengths, const float* trans, const float* dur,
                 const float* p_start, const float* p_end, int B, int T, int C, int K,
                 unsigned flags, void* ws, size_t ws_bytes, double* score, int32_t* labels,
                 uint8_t* seg_start, cudaStream_t st) {
  if (!lengths || !trans || !dur || !score || (B > 0 && T > 0 && (!em || !labels || !seg_start)))
    return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  int rc = prepare(B, T, C, K, flags, ws, ws_bytes, d, p);
  if (rc) return rc;
  // The decoder's ring prefers clusters of 8 where all 8 B CTAs fit the GPU
  // at once: its helpers are light, so splitting the labels finer shortens
  // the step (the workspace layout does not depend on the cluster shape).
  if (d.xG && d.xN > 1 && 8LL * B <= sm_count()) {
    Dims e = d;
    choose_xshape(e, (size_t)max_smem_optin() - 256, 8);
    if (e.xG) d = e;
  }
  const bool proj = p_start || p_end;
  if ((rc = reset_status(p, proj, st))) return rc;
  if (B == 0) return SEMICRF_OK;
  rc = run_prefix(em, lengths, d, p, flags, 1, nullptr, nullptr, st, p_start, p_end);
  if (rc) return rc;
  cudaError_t e;
  // the pipelined decoder, unless no shape fits (then the one-role kernel)
  if (!d.KBT && !pipelined(d, 0, proj)) return SEMICRF_ERR_UNSUPPORTED;
  if (pipelined(d, 0, proj)) {
    {
      ProfScope ps("viterbi_pipe_kernel", st);
      e = launch_viterbi_pipe(d, p, lengths, trans, dur, score, labels, seg_start, st,
                              proj ? 1 : 0);
    }
    if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
    {
      ProfScope ps("viterbi_argmax_kernel", st);
      e = launch_viterbi_argmax(d, p, lengths, trans, st);
    }
    if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
    {
      ProfScope ps("viterbi_words_kernel", st);
      e = launch_viterbi_words(d, p, lengths, st);
    }
    if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
    ProfScope ps("viterbi_walk_kernel", st);
    e = launch_viterbi_walk(d, p, lengths, labels, seg_start,
                            viterbi_walk_smem_bytes(d, (size_t)max_smem_optin() - 256), st);
  } else {
    ProfScope ps("viterbi_kernel", st);
    e = launch_viterbi(d, p, lengths, trans, dur, score, labels, seg_start, st);
  }
  return e == cudaSuccess ? SEMICRF_OK : SEMICRF_ERR_CUDA;
}

}  // namespace

extern "C" int semicrf_viterbi(const float* em, const int32_t* lengths, const float* trans,
                               const float* dur, int B, int T, int C, int K, unsigned flags,
                               void* ws, size_t ws_bytes, double* score, int32_t* labels,
                               uint8_t* seg_start, semicrf_stream_t stream) {
  return viterbi_impl(em, lengths, trans, dur, nullptr, nullptr, B, T, C, K, flags, ws, ws_bytes,
                      score, labels, seg_start, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int semicrf_viterbi_proj(const float* em, const int32_t* lengths, const float* trans,
                                    const float* dur, const float* p_start, const float* p_end,
                                    int B, int T, int C, int K, unsigned flags, void* ws,
                                    size_t ws_bytes, double* score, int32_t* labels,
                                    uint8_t* seg_start, semicrf_stream_t stream) {
  return viterbi_impl(em, lengths, trans, dur, p_start, p_end, B, T, C, K, flags, ws, ws_bytes,
                      score, labels, seg_start, reinterpret_cast<cudaStream_t>(stream));
}

namespace {

int path_score_impl(const float* em, const int32_t* lengths, const float* trans, const float* dur,
                    const float* p_start, const float* p_end, const int32_t* labels,
                    const uint8_t* seg_start, int B, int T, int C, int K, unsigned flags, void* ws,
                    size_t ws_bytes, const double* grad_score, double* score, float* grad_em,
                    float* grad_trans, float* grad_dur, float* grad_p_start, float* grad_p_end,
                    cudaStream_t st) {
  if (!lengths || !trans || !dur || (B > 0 && T > 0 && (!em || !labels || !seg_start)))
    return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  int rc = prepare(B, T, C, K, flags, ws, ws_bytes, d, p);
  if (rc) return rc;
  if (B == 0) return SEMICRF_OK;
  const unsigned center = (flags & SEMICRF_FLAG_NO_CENTER) ? 0u : 1u;
  if (cudaMemsetAsync(p.pcnt, 0, p.pzero_bytes, st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  cudaError_t e;
  {
    ProfScope ps("path_terms_kernel", st);
    e = launch_path_terms(d, p, em, lengths, trans, dur, labels, seg_start, center, grad_score,
                          (flags & SEMICRF_FLAG_NEGATE_GRAD) ? 1 : 0, score, p_start, p_end, st);
  }
  if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
  if (grad_em || grad_trans || grad_dur || grad_p_start || grad_p_end) {
    ProfScope ps("path_grad_kernel", st);
    e = launch_path_grad(d, p, lengths, labels, seg_start, grad_em, grad_trans, grad_dur,
                         grad_p_start, grad_p_end, st);
  }
  return e == cudaSuccess ? SEMICRF_OK : SEMICRF_ERR_CUDA;
}

}  // namespace

extern "C" int semicrf_path_score(const float* em, const int32_t* lengths, const float* trans,
                                  const float* dur, const int32_t* labels,
                                  const uint8_t* seg_start, int B, int T, int C, int K,
                                  unsigned flags, void* ws, size_t ws_bytes,
                                  const double* grad_score, double* score, float* grad_em,
                                  float* grad_trans, float* grad_dur, semicrf_stream_t stream) {
  return path_score_impl(em, lengths, trans, dur, nullptr, nullptr, labels, seg_start, B, T, C, K,
                         flags, ws, ws_bytes, grad_score, score, grad_em, grad_trans, grad_dur,
                         nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int semicrf_path_score_proj(const float* em, const int32_t* lengths, const float* trans,
                                       const float* dur, const float* p_start, const float* p_end,
                                       const int32_t* labels, const uint8_t* seg_start, int B,
                                       int T, int C, int K, unsigned flags, void* ws,
                                       size_t ws_bytes, const double* grad_score, double* score,
                                       float* grad_em, float* grad_trans, float* grad_dur,
                                       float* grad_p_start, float* grad_p_end,
                                       semicrf_stream_t stream) {
  return path_score_impl(em, lengths, trans, dur, p_start, p_end, labels, seg_start, B, T, C, K,
                         flags, ws, ws_bytes, grad_score, score, grad_em, grad_trans, grad_dur,
                         grad_p_start, grad_p_end, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int semicrf_get_status(const void* ws, semicrf_stream_t stream, int* status) {
  if (!ws || !status) return SEMICRF_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SEMICRF_ERR_CUDA;
  *status = v;
  return SEMICRF_OK;
}

extern "C" int semicrf_ring_domains(const void* ws, size_t ws_bytes, int B, int T, int C, int K,
                                    unsigned flags, semicrf_stream_t stream, int32_t* domains) {
  if (!domains) return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  const int rc = prepare(B, T, C, K, flags, const_cast<void*>(ws), ws_bytes, d, p);
  if (rc) return rc;
  if (B == 0) return SEMICRF_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(domains, p.mode, 2ull * B * sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SEMICRF_ERR_CUDA;
  // a run without the exponential-domain kernel leaves the array untouched:
  // report those rings as log domain
  if (!d.xG || (flags & SEMICRF_FLAG_LOG_DOMAIN))
    for (int i = 0; i < 2 * B; ++i) domains[i] = 2;
  return SEMICRF_OK;
}

#ifndef SEMICRF_SOURCE_DIGEST
#define SEMICRF_SOURCE_DIGEST "unknown"
#endif
extern "C" const char* semicrf_source_digest(void) { return SEMICRF_SOURCE_DIGEST; }

extern "C" const char* semicrf_strerror(int code) {
  switch (code) {
    case SEMICRF_OK: return "ok";
    case SEMICRF_ERR_INVALID_ARG: return "invalid argument";
    case SEMICRF_ERR_UNSUPPORTED: return "unsupported size (above the library's limits)";
    case SEMICRF_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case SEMICRF_ERR_CUDA: return "CUDA launch or copy failed";
    case SEMICRF_ERR_DEVICE_TIMEOUT: return "a bounded device wait gave up";
    case SEMICRF_ERR_BAD_LENGTH: return "a sequence length is outside [0, T]";
    default:
      if ((code & 0xff) == SEMICRF_ERR_BOUNDS)
        return "an index check failed (bounds-checking build; status >> 8 is the site)";
      return "unknown status";
  }
}

extern "C" int semicrf_selftest_bounded_wait(void* ws, size_t ws_bytes, int spins,
                                             semicrf_stream_t stream) {
  if (!ws || ws_bytes < 256 || spins < 0) return SEMICRF_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, st>>>(status, spins);
  return launched();
}

extern "C" int semicrf_selftest_bounds(void* ws, size_t ws_bytes, semicrf_stream_t stream) {
#ifdef SEMICRF_BOUNDS_CHECK
  if (!ws || ws_bytes < 256) return SEMICRF_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  selftest_bounds_kernel<<<1, 32, 0, st>>>(status, 32);
  return launched();
#else
  (void)ws;
  (void)ws_bytes;
  (void)stream;
  return SEMICRF_ERR_UNSUPPORTED;  // the release build has no index checks to exercise
#endif
}

extern "C" int semicrf_profile_enable(int on) {
  std::lock_guard<std::mutex> g(prof_mu);
  prof_on = on != 0;
  if (on) {
    for (auto& r : prof_recs) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
    prof_recs.clear();
  }
  return SEMICRF_OK;
}

extern "C" int semicrf_profile_read(const char* kernel, double* total_ms, int* launches) {
  if (!kernel || !total_ms || !launches) return SEMICRF_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(prof_mu);
  double tot = 0.0;
  int n = 0;
  for (auto& r : prof_recs) {
    if (std::strcmp(r.name, kernel) != 0) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return SEMICRF_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return SEMICRF_ERR_CUDA;
    tot += ms;
    ++n;
  }
  *total_ms = tot;
  *launches = n;
  return SEMICRF_OK;
}
