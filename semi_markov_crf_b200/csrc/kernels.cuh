// kernels.cuh -- declarations of the semi-CRF kernels and their shared-memory
// budgets.  Definitions live in prefix.cu, recursion.cu, finalize.cu and
// viterbi.cu; the host layer in api.cu launches them.
#pragma once

#include "device.cuh"
#include "layout.cuh"

namespace semicrf {

// Shared-memory bytes of the recursion kernels (carve order in recursion.cu).
__host__ __device__ inline size_t recursion_smem_bytes(const Dims& d, bool with_store) {
  size_t b = 64;                                  // mbarriers + max slots + flags
  b += 2ull * TS * d.C * sizeof(int32_t);         // prefix-sum integer tiles
  b += 2ull * TS * d.C * sizeof(float);           // prefix-sum fraction tiles
  b += (size_t)d.K * d.C * sizeof(float2);        // ring
  b += 8ull * d.C * sizeof(float);                // Acur, pcur, stS[2], stE[2], tmp, Sbase
  b += 16;
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
                                   double* __restrict__ S64, float* __restrict__ nu_out);

// grid.x = n_alpha + n_beta CTAs: the first n_alpha run the forward ring of
// sequence blockIdx.x, the rest the backward ring of sequence
// blockIdx.x - n_alpha (n_alpha is 0 or B; so is n_beta).
__global__ void chain_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                             const float* __restrict__ trans, const float* __restrict__ dur,
                             double* __restrict__ logZ_out, int n_alpha);

// grid = (nck, B): one CTA per checkpoint segment.
__global__ void segment_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                               const float* __restrict__ trans, const float* __restrict__ dur,
                               const double* __restrict__ grad_logZ, float* __restrict__ grad_em,
                               float* __restrict__ start_marg, float* __restrict__ end_marg);

__global__ void finalize_positions_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                                          const double* __restrict__ grad_logZ, unsigned center,
                                          float* __restrict__ grad_em, float* __restrict__ pos_marg,
                                          float* __restrict__ start_marg,
                                          float* __restrict__ end_marg);

__global__ void reduce_partials_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                                       float* __restrict__ grad_trans, float* __restrict__ grad_dur);

__global__ void viterbi_kernel(Dims d, WsPtrs ws, const int32_t* __restrict__ lengths,
                               const float* __restrict__ trans, const float* __restrict__ dur,
                               double* __restrict__ score, int32_t* __restrict__ labels,
                               uint8_t* __restrict__ seg_start);

__global__ void selftest_wait_kernel(int* status, int spins);

}  // namespace semicrf
