// noalloc.cu -- a log Z entry point that needs no caller-provided workspace
// and allocates nothing.
//
// Some callers cannot allocate device memory when they run: a plugin whose
// execution hook is forbidden to allocate (its memory was planned ahead),
// code that runs where a cudaMalloc would stall or synchronise the device, or
// a host integration with no allocator to hand.  For them this file keeps
// the scratch memory of the forward pass in one fixed array that lives in the
// library's device image: every GPU that loads the library holds
// NOALLOC_SCRATCH_BYTES for it until the process exits.
//
// The array is shared by every call on a device and keeps the last call's
// contents; calls that overlap on the GPU (two streams, two host threads)
// race on it and must be serialised by the caller.
#include <mutex>

#include "semicrf.h"
#include "kernels.cuh"

namespace semicrf {
namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = SEMICRF_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex scratch_mu;
void* scratch_ptr[MAX_DEVICES] = {};

// Device address of the array on the current device.  Looked up once per
// device (host code cannot use the array's name as an address) and kept for
// the life of the process; a device reset unloads the module the address
// belongs to, so a process that resets a device must restart before calling
// the entry point again.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
    cudaGetLastError();
    return SEMICRF_ERR_CUDA;
  }
  std::lock_guard<std::mutex> g(scratch_mu);
  if (!scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SEMICRF_ERR_CUDA;
    }
    scratch_ptr[dev] = p;
  }
  *out = scratch_ptr[dev];
  return SEMICRF_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Carves the forward-only working set (status word, split prefix sums,
// per-chunk sums, log Z, forward checkpoints) out of `base`; returns bytes.
size_t forward_layout(const Dims& d, void* base, WsPtrs* p) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t B = d.B, C = d.C, K = d.K, nck = d.nck;
  const size_t o_status = take(256);
  const size_t o_sint = take(B * d.Tstride * C * 4);
  const size_t o_sfrac = take(B * d.Tstride * C * 4);
  const size_t o_chunk = take(B * d.nchunk * C * 8);
  const size_t o_lz = take(B * 8);
  const size_t o_ack = take(B * nck * K * C * 8);
  const size_t o_acf = take(B * nck * 8);
  const size_t o_emax = take(B * 4);
  const size_t o_mode = take(2 * B * 4);
  if (base && p) {
    char* c = static_cast<char*>(base);
    *p = WsPtrs{};
    p->status = reinterpret_cast<int*>(c + o_status);
    p->sint = reinterpret_cast<int32_t*>(c + o_sint);
    p->sfrac = reinterpret_cast<float*>(c + o_sfrac);
    p->chunk = reinterpret_cast<double*>(c + o_chunk);
    p->logz2 = reinterpret_cast<double*>(c + o_lz);
    p->ack = reinterpret_cast<float2*>(c + o_ack);
    p->acf = reinterpret_cast<double*>(c + o_acf);
    p->emax = reinterpret_cast<float*>(c + o_emax);
    p->mode = reinterpret_cast<int*>(c + o_mode);
  }
  return off;
}

}  // namespace
}  // namespace semicrf

using namespace semicrf;

extern "C" int semicrf_forward_noalloc(const float* em, const int32_t* lengths, const float* trans,
                                       const float* dur, int B, int T, int C, int K,
                                       unsigned flags, double* logZ, semicrf_stream_t stream) {
  if (!lengths || !trans || !dur || !logZ || (B > 0 && T > 0 && !em)) return SEMICRF_ERR_INVALID_ARG;
  if (flags & ~(SEMICRF_FLAG_NO_CENTER | SEMICRF_FLAG_FORWARD_ONLY | SEMICRF_FLAG_LOG_DOMAIN))
    return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  int rc = make_dims(B, T, C, K, d);
  if (rc != SEMICRF_OK) return rc;
  if (forward_layout(d, nullptr, nullptr) > NOALLOC_SCRATCH_BYTES) return SEMICRF_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch)) != SEMICRF_OK) return rc;
  WsPtrs p;
  forward_layout(d, scratch, &p);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the only state that must start at zero is the status word
  if (cudaMemsetAsync(p.status, 0, sizeof(int), st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  if (B == 0) return SEMICRF_OK;
  if (T > 0) {
    const dim3 grid(d.nchunk, d.B);
    prefix_reduce_kernel<<<grid, 256, 0, st>>>(em, lengths, d, p);
    const size_t sm = prefix_scan_smem_bytes(d);
    if (sm > 48 * 1024 &&
        cudaFuncSetAttribute(prefix_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
    prefix_scan_kernel<<<grid, 256, sm, st>>>(em, lengths, d, p,
                                              (flags & SEMICRF_FLAG_NO_CENTER) ? 0u : 1u, 1,
                                              nullptr, nullptr, nullptr, nullptr);
    if (cudaGetLastError() != cudaSuccess) return SEMICRF_ERR_CUDA;
  }
  // exponential-domain ring where the scores allow it, log domain for the rest
  // (long durations have no log-domain kernel: declined rings are reported)
  if (!d.KBT && (!d.xG || (flags & SEMICRF_FLAG_LOG_DOMAIN))) return SEMICRF_ERR_UNSUPPORTED;
  if (d.xG && !(flags & SEMICRF_FLAG_LOG_DOMAIN)) {
    if (launch_chain_exp(d, p, lengths, trans, dur, logZ, B, 0, st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
  } else {
    p.mode = nullptr;
  }
  return launch_chain(d, p, lengths, trans, dur, logZ, B, 0, st) == cudaSuccess ? SEMICRF_OK
                                                                                : SEMICRF_ERR_CUDA;
}
