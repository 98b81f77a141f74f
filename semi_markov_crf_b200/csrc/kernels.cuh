// kernels.cuh -- declarations of the semi-CRF kernels, their shared-memory
// budgets and the host-side launchers that pick a compile-time lane shape.
// Definitions live in prefix.cu, recursion.cu, finalize.cu and viterbi.cu.
#pragma once

#include "device.cuh"
#include "layout.cuh"

namespace semicrf {

// Shared-memory bytes of the recursion kernels (carve order in ring.cuh).
__host__ __device__ inline size_t recursion_smem_bytes(const Dims& d, bool with_store) {
  size_t b = 64;                                  // mbarriers + max slots + flags
  b += 2ull * TS * d.C * sizeof(int32_t);         // prefix-sum integer tiles
  b += 2ull * TS * d.C * sizeof(float);           // prefix-sum fraction tiles
  b += (size_t)d.RL * d.C * sizeof(float2);       // mirrored ring
  b += (2ull * d.PC + 4ull * d.C) * sizeof(float);  // pcur[2], Acur[2], tmp, Sbase
  b += 32;
  if (with_store) b += (size_t)d.delta * d.store_w * sizeof(float);
  return b;
}

__host__ __device__ inline size_t prefix_scan_smem_bytes(const Dims& d) {
  const int G = 256 / d.C;
  return (size_t)d.prefR * d.C * sizeof(float) + 32 + (2ull * d.C + (size_t)G * d.C) * sizeof(double);
}

__global__ void prefix_reduce_kernel(const float* __restrict__ em, const int32_t* __restrict__ lengths,
                                     Dims d, WsPtrs ws);
__global__ void prefix_scan_kernel(const float* __restrict__ em, const int32_t* __restrict__ lengths,
                                   Dims d, WsPtrs ws, unsigned center, int mode,
                                   double* __restrict__ S64, float* __restrict__ nu_out,
                                   const float* __restrict__ p_start, const float* __restrict__ p_end);

__global__ void finalize_positions_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                                          const double* __restrict__ grad_logZ, unsigned center,
                                          float* __restrict__ grad_em, float* __restrict__ pos_marg,
                                          float* __restrict__ start_marg,
                                          float* __restrict__ end_marg);

// reduce_partials_kernel: entries per block, thread rows per entry.
constexpr int RP_E = 32, RP_S = 8;
__global__ void reduce_partials_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                                       float* __restrict__ grad_trans, float* __restrict__ grad_dur);

__global__ void selftest_wait_kernel(int* status, int spins);
#ifdef SEMICRF_BOUNDS_CHECK
__global__ void selftest_bounds_kernel(int* status, int idx);
#endif

// Posteriors of sequence b come from the values both exponential-domain
// rings kept (posterior.cu) rather than from the checkpoint walk
// (segment_kernel).  The same test in every kernel that depends on it.
__device__ __forceinline__ bool posterior_from_kept(const WsPtrs& ws, const Dims& d, int b) {
  return ws.kv != nullptr && ws.mode != nullptr && ws.mode[b] == 1 && ws.mode[d.B + b] == 1;
}

__global__ void cut_grid_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                                const float* __restrict__ trans, const float* __restrict__ dur,
                                int pj, int per_label);
// The posterior pass (one CTA per checkpoint segment and sequence).
// seg_marg (nullable) [B][T][K][C]: the segment marginals of the sequences
// the kernel takes (the caller zeroes the array first).
cudaError_t launch_posterior(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                             const float* trans, const float* dur, const double* grad_logZ,
                             float* grad_em, float* start_marg, float* end_marg, cudaStream_t st,
                             float* seg_marg = nullptr, int pj = 0);
size_t posterior_smem_bytes(const Dims& d);
// Tile rows for the posterior pass under `budget` bytes of shared memory (0:
// none fits).
int posterior_tile_rows(Dims& d, size_t budget);
bool cut_grid_per_label(const Dims& d, size_t budget);
size_t cut_grid_smem_bytes(const Dims& d, size_t budget);

// Sizes, launch geometry and limits for (B, T, C, K); returns a semicrf_status.
int make_dims(int B, int T, int C, int K, Dims& d);

// Lane shapes with a compiled instantiation (KBT durations, CAT labels per lane).
bool shape_supported(int KBT, int CAT, int G, int LB);

// Host launchers for the shape in `d` (return the cudaError_t of the launch).
// Forward ring of sequences [0, n_alpha) and backward ring of the rest:
// grid = n_alpha + n_beta CTAs.
cudaError_t launch_chain(const Dims& d, const WsPtrs& ws, const int32_t* lengths, const float* trans,
                         const float* dur, double* logZ_out, int n_alpha, int n_beta,
                         cudaStream_t st);
// One CTA per (checkpoint segment, sequence).
cudaError_t launch_segment(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                           const float* trans, const float* dur, const double* grad_logZ,
                           float* grad_em, float* start_marg, float* end_marg, cudaStream_t st,
                           float* seg_marg = nullptr);
cudaError_t launch_viterbi(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                           const float* trans, const float* dur, double* score, int32_t* labels,
                           uint8_t* seg_start, cudaStream_t st);

// Every kernel shape the library instantiates: (durations per lane KBT,
// labels per lane CAT, lanes per label G, launch bound LB).  The (16, 32, G,
// 512) family alone covers every size with K <= 512; the others are tuned for
// smaller problems (fewer wasted terms, fewer registers), and (64, 1, 32, 256)
// takes long durations, K <= 2048 with C <= 8.
#define SEMICRF_FOR_EACH_SHAPE(X)                                                        \
  X(4, 4, 1, 256) X(8, 4, 1, 256) X(4, 8, 1, 256) X(8, 8, 1, 256) X(16, 8, 1, 256)       \
  X(16, 32, 1, 256) X(4, 4, 2, 256) X(8, 8, 2, 256) X(16, 32, 2, 256) X(4, 8, 4, 256)    \
  X(8, 16, 4, 256) X(16, 32, 4, 512) X(4, 8, 8, 512) X(8, 4, 8, 256) X(8, 8, 8, 512)     \
  X(16, 8, 8, 512) X(16, 32, 8, 512) X(8, 1, 16, 256) X(16, 1, 16, 256) X(16, 4, 16, 512) \
  X(16, 32, 16, 512) X(8, 1, 32, 256) X(16, 1, 32, 512) X(16, 32, 32, 512)              \
  X(64, 1, 32, 256)

// Pipelined exponential-domain rings (chain_exp.cu) and decoder
// (viterbi_pipe.cu): shapes (CTAs per ring N, combine lanes per label G,
// weights per combine lane CAT, helper lanes per label H, durations per
// helper lane KBH, launch bound LB).  Each CTA owns Cr = ceil(C / N) labels;
// a shape serves C <= G*CAT and K <= H*KBH + 2 with
// 32*(ceil(Cr*G/32) + ceil(Cr*H/32)) <= LB threads (labels never straddle a
// warp).  N > 1 runs each ring on a thread-block cluster of N CTAs.  H = 128
// (long durations, K up to 8194): a label's helper lanes span four warps,
// one label per CTA (its ring of K + 8192 entries fills the CTA's shared
// memory).
#define SEMICRF_FOR_EACH_XSHAPE(X)                                                     \
  X(1, 1, 8, 1, 8, 64) X(1, 1, 8, 4, 8, 64) X(1, 1, 8, 8, 16, 96) X(1, 1, 8, 16, 16, 160)          \
  X(1, 1, 8, 32, 16, 288) X(1, 1, 16, 1, 8, 64) X(1, 1, 16, 4, 8, 96) X(1, 1, 16, 8, 16, 160)      \
  X(1, 1, 16, 16, 16, 288) X(1, 1, 16, 32, 16, 544) X(1, 1, 32, 4, 8, 160) X(1, 1, 32, 8, 16, 288) \
  X(1, 1, 32, 16, 16, 544) X(1, 2, 24, 4, 8, 288) X(1, 2, 24, 4, 16, 288) X(1, 2, 24, 8, 16, 480) \
  X(1, 2, 32, 4, 8, 384) X(1, 2, 32, 4, 16, 384) X(1, 2, 32, 8, 16, 640) X(1, 4, 24, 4, 8, 768)   \
  X(1, 4, 12, 4, 8, 384) X(1, 4, 12, 4, 16, 384) X(1, 2, 48, 2, 32, 384) X(1, 2, 64, 2, 32, 512)  \
  X(1, 4, 24, 2, 32, 576) X(1, 4, 32, 4, 8, 1024) X(1, 4, 32, 2, 32, 768) X(1, 1, 8, 32, 64, 224) \
  X(1, 1, 8, 32, 64, 288) \
  X(2, 2, 24, 4, 8, 160) X(2, 4, 32, 4, 16, 512) X(4, 4, 32, 4, 16, 256) X(8, 4, 32, 4, 16, 128) \
  X(4, 8, 16, 4, 16, 384) X(4, 4, 32, 8, 8, 384) X(8, 8, 16, 8, 8, 256) X(8, 4, 32, 8, 8, 192) \
  X(1, 1, 8, 128, 64, 160) X(2, 1, 8, 128, 64, 160) X(3, 1, 8, 128, 64, 160)                 \
  X(4, 1, 8, 128, 64, 160) X(5, 1, 8, 128, 64, 160) X(6, 1, 8, 128, 64, 160)                 \
  X(7, 1, 8, 128, 64, 160) X(8, 1, 8, 128, 64, 160)

// Launches `kern` on `grid` CTAs of `threads` threads grouped in clusters of
// n_cluster CTAs (grid a multiple of n_cluster; n_cluster = 1: a plain
// launch), with `smem` bytes of dynamic shared memory each.
template <typename... KArgs, typename... Args>
cudaError_t launch_clustered(void (*kern)(KArgs...), int n_cluster, int grid, int threads,
                             size_t smem, cudaStream_t st, Args... args) {
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (n_cluster <= 1) {
    kern<<<grid, threads, smem, st>>>(args...);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = n_cluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// pj: the call has boundary projections (the tile stream carries their
// start terms; the kernels add them where a boundary takes the start role).
size_t chain_exp_smem_bytes(const Dims& d, bool pj = false);
size_t viterbi_pipe_smem_bytes(const Dims& d, bool pj = false);
// After viterbi_pipe: the label argmax of every segment start and the
// backpointer words from the kept rows (grid-wide), then the traceback (one
// CTA per sequence, `sm` bytes of shared memory).
cudaError_t launch_viterbi_argmax(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                  const float* trans, cudaStream_t st);
cudaError_t launch_viterbi_words(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                 cudaStream_t st);
size_t viterbi_walk_smem_bytes(const Dims& d, size_t budget);
cudaError_t launch_viterbi_walk(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                int32_t* labels, uint8_t* seg_start, size_t sm, cudaStream_t st);
// Viterbi with the pipelined schedule (shapes of SEMICRF_FOR_EACH_XSHAPE).
cudaError_t launch_viterbi_pipe(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                                const float* trans, const float* dur, double* score,
                                int32_t* labels, uint8_t* seg_start, cudaStream_t st, int pj = 0);
bool xshape_supported(int N, int G, int CAT, int H, int KBH, int LB);
// Same grid and outputs as launch_chain for the sequences whose scores fit
// the exponential domain; writes ws.mode for every (direction, sequence).
cudaError_t launch_chain_exp(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                             const float* trans, const float* dur, double* logZ_out, int n_alpha,
                             int n_beta, cudaStream_t st, int pj = 0);

// g_b times the boundary marginals as the boundary-projection gradients
// (finalize.cu); start_marg / end_marg are [B][T+1][C].
cudaError_t launch_proj_grad(const Dims& d, const int32_t* lengths, const double* grad_logZ,
                             const float* start_marg, const float* end_marg, float* grad_p_start,
                             float* grad_p_end, cudaStream_t st);

// Score of given segmentations and its gradient (path.cu).  The caller zeroes
// the ws.pzero_bytes region at ws.pcnt first.  The terms pass writes score[b]
// (nullable) and the weights; the gradient pass adds into the non-null outputs.
cudaError_t launch_path_terms(const Dims& d, const WsPtrs& ws, const float* em,
                              const int32_t* lengths, const float* trans, const float* dur,
                              const int32_t* labels, const uint8_t* seg_start, unsigned center,
                              const double* grad_score, int negate, double* score,
                              const float* p_start, const float* p_end, cudaStream_t st);
cudaError_t launch_path_grad(const Dims& d, const WsPtrs& ws, const int32_t* lengths,
                             const int32_t* labels, const uint8_t* seg_start, float* grad_em,
                             float* grad_trans, float* grad_dur, float* grad_p_start,
                             float* grad_p_end, cudaStream_t st);

}  // namespace semicrf
