// api.cu -- the C ABI declared in include/semicrf.h: argument validation,
// launch geometry, workspace layout and kernel launches.  Host code only.
#include <cmath>
#include <cstring>
#include <mutex>

#include "semicrf.h"
#include "kernels.cuh"

namespace semicrf {

namespace {

constexpr int FIN_ROWS_HOST = 32;  // must match FIN_ROWS in finalize.cu

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

// Sizes, lane mapping and limits.  Returns a semicrf_status.
int make_dims(int B, int T, int C, int K, Dims& d) {
  if (B < 0 || T < 0 || C < 1 || K < 1) return SEMICRF_ERR_INVALID_ARG;
  if (C > C_MAX || K > K_MAX || (long long)K * C > KC_MAX || T > (1 << 26) || B > (1 << 20))
    return SEMICRF_ERR_UNSUPPORTED;
  d.B = B;
  d.T = T;
  d.C = C;
  d.K = K;
  d.delta = T > 0 ? isqrt_ceil((long long)T * K) : 1;
  if (d.delta < 1) d.delta = 1;
  d.nck = T > 0 ? (T + d.delta - 1) / d.delta : 1;
  d.Tstride = ((T + 1 + TS - 1) / TS) * TS;
  d.GB = std::min(32, pow2floor(NT_MAX / C));
  d.KB = (K + d.GB - 1) / d.GB;
  d.GA = std::min(std::min(32, pow2floor(NT_MAX / C)), pow2floor(C));
  d.CA = (C + d.GA - 1) / d.GA;
  if (d.KB > KB_MAX || d.CA > CA_MAX) return SEMICRF_ERR_UNSUPPORTED;
  int nt = std::max(C * d.GB, C * d.GA);
  nt = ((nt + 31) / 32) * 32;
  d.NT = std::max(nt, 32);
  d.prefR = std::max(16, pow2floor(8192 / C));
  d.nchunk = T > 0 ? (T + d.prefR - 1) / d.prefR : 1;
  d.store_w = 2 * C + 2;
  const size_t budget = (size_t)max_smem_optin();
  d.store_smem = recursion_smem_bytes(d, true) <= budget ? 1 : 0;
  if (recursion_smem_bytes(d, false) > budget) return SEMICRF_ERR_UNSUPPORTED;
  return SEMICRF_OK;
}

// Workspace layout; fills `p` when base != nullptr.  Returns total bytes.
size_t layout(const Dims& d, void* base, WsPtrs* p) {
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
  const size_t o_lzb = take(B * 8);
  const size_t o_ack = take(B * nck * K * C * 8);
  const size_t o_acf = take(B * nck * 8);
  const size_t o_bck = take(B * nck * K * C * 8);
  const size_t o_bcf = take(B * nck * 8);
  const size_t o_store = take(d.store_smem ? 0 : B * nck * (size_t)d.delta * d.store_w * 4);
  const size_t o_pgt = take(B * nck * C * C * 8);
  const size_t o_pgd = take(B * nck * K * C * 8);
  const size_t o_segT = take(B * nck * C * 8);
  const size_t o_segV = take(B * nck * C * 8);
  const size_t o_bp = take(B * (size_t)(d.T + 1) * C * 4);
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
  }
  return off;
}

constexpr unsigned KNOWN_FLAGS = SEMICRF_FLAG_NO_CENTER | SEMICRF_FLAG_FORWARD_ONLY;

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

int run_prefix(const float* em, const int32_t* lengths, const Dims& d, const WsPtrs& p,
               unsigned flags, int mode, double* S64, float* nu, cudaStream_t st) {
  if (d.B == 0 || d.T == 0) return SEMICRF_OK;
  const dim3 grid(d.nchunk, d.B);
  prefix_reduce_kernel<<<grid, 256, 0, st>>>(em, lengths, d, p);
  const size_t sm = prefix_scan_smem_bytes(d);
  int rc = set_smem((const void*)prefix_scan_kernel, sm);
  if (rc) return rc;
  prefix_scan_kernel<<<grid, 256, sm, st>>>(em, lengths, d, p,
                                            (flags & SEMICRF_FLAG_NO_CENTER) ? 0u : 1u, mode, S64,
                                            nu);
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

extern "C" int semicrf_forward(const float* em, const int32_t* lengths, const float* trans,
                               const float* dur, int B, int T, int C, int K, unsigned flags,
                               void* ws, size_t ws_bytes, double* logZ, semicrf_stream_t stream) {
  if (!lengths || !trans || !dur || !logZ || (B > 0 && T > 0 && !em)) return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  int rc = prepare(B, T, C, K, flags, ws, ws_bytes, d, p);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(p.status, 0, sizeof(int), st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  if (B == 0) return SEMICRF_OK;
  rc = run_prefix(em, lengths, d, p, flags, 1, nullptr, nullptr, st);
  if (rc) return rc;
  const size_t sm = recursion_smem_bytes(d, false);
  rc = set_smem((const void*)chain_kernel, sm);
  if (rc) return rc;
  const int nb = (flags & SEMICRF_FLAG_FORWARD_ONLY) ? B : 2 * B;
  chain_kernel<<<nb, d.NT, sm, st>>>(d, p, lengths, trans, dur, logZ, B);
  return launched();
}

extern "C" int semicrf_backward(const int32_t* lengths, const float* trans, const float* dur,
                                int B, int T, int C, int K, unsigned flags, void* ws,
                                size_t ws_bytes, const double* grad_logZ, float* grad_em,
                                float* grad_trans, float* grad_dur, float* pos_marg,
                                float* start_marg, float* end_marg, semicrf_stream_t stream) {
  if (!lengths || !trans || !dur || !grad_trans || !grad_dur || (B > 0 && T > 0 && !grad_em))
    return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  int rc = prepare(B, T, C, K, flags, ws, ws_bytes, d, p);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0) {
    if (cudaMemsetAsync(grad_trans, 0, (size_t)C * C * 4, st) != cudaSuccess ||
        cudaMemsetAsync(grad_dur, 0, (size_t)K * C * 4, st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
    return SEMICRF_OK;
  }
  if (flags & SEMICRF_FLAG_FORWARD_ONLY) {
    const size_t sm = recursion_smem_bytes(d, false);
    rc = set_smem((const void*)chain_kernel, sm);
    if (rc) return rc;
    chain_kernel<<<B, d.NT, sm, st>>>(d, p, lengths, trans, dur, nullptr, 0);
    if ((rc = launched())) return rc;
  }
  if (T > 0) {
    const size_t sm = recursion_smem_bytes(d, d.store_smem != 0);
    rc = set_smem((const void*)segment_kernel, sm);
    if (rc) return rc;
    segment_kernel<<<dim3(d.nck, B), d.NT, sm, st>>>(d, p, lengths, trans, dur, grad_logZ, grad_em,
                                                     start_marg, end_marg);
    if ((rc = launched())) return rc;
    const int nj = FIN_ROWS_HOST / d.delta + 2;
    const size_t fsm = ((size_t)C + (size_t)nj * C) * sizeof(double);
    rc = set_smem((const void*)finalize_positions_kernel, fsm);
    if (rc) return rc;
    finalize_positions_kernel<<<dim3((T + FIN_ROWS_HOST - 1) / FIN_ROWS_HOST, B), 256, fsm, st>>>(
        d, p, lengths, grad_logZ, (flags & SEMICRF_FLAG_NO_CENTER) ? 0u : 1u, grad_em, pos_marg,
        start_marg, end_marg);
    if ((rc = launched())) return rc;
  } else {
    // T == 0: only boundary row 0 exists, and nothing starts or ends there
    if (start_marg && cudaMemsetAsync(start_marg, 0, (size_t)B * C * 4, st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
    if (end_marg && cudaMemsetAsync(end_marg, 0, (size_t)B * C * 4, st) != cudaSuccess)
      return SEMICRF_ERR_CUDA;
  }
  const int ne = C * C + K * C;
  reduce_partials_kernel<<<(ne + 255) / 256, 256, 0, st>>>(d, p, lengths, grad_trans, grad_dur);
  return launched();
}

extern "C" int semicrf_viterbi(const float* em, const int32_t* lengths, const float* trans,
                               const float* dur, int B, int T, int C, int K, unsigned flags,
                               void* ws, size_t ws_bytes, double* score, int32_t* labels,
                               uint8_t* seg_start, semicrf_stream_t stream) {
  if (!lengths || !trans || !dur || !score || (B > 0 && T > 0 && (!em || !labels || !seg_start)))
    return SEMICRF_ERR_INVALID_ARG;
  Dims d;
  WsPtrs p;
  int rc = prepare(B, T, C, K, flags, ws, ws_bytes, d, p);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(p.status, 0, sizeof(int), st) != cudaSuccess) return SEMICRF_ERR_CUDA;
  if (B == 0) return SEMICRF_OK;
  rc = run_prefix(em, lengths, d, p, flags, 1, nullptr, nullptr, st);
  if (rc) return rc;
  const size_t sm = recursion_smem_bytes(d, false);
  rc = set_smem((const void*)viterbi_kernel, sm);
  if (rc) return rc;
  viterbi_kernel<<<B, d.NT, sm, st>>>(d, p, lengths, trans, dur, score, labels, seg_start);
  return launched();
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

extern "C" const char* semicrf_strerror(int code) {
  switch (code) {
    case SEMICRF_OK: return "ok";
    case SEMICRF_ERR_INVALID_ARG: return "invalid argument";
    case SEMICRF_ERR_UNSUPPORTED: return "unsupported size (above this build's limits)";
    case SEMICRF_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case SEMICRF_ERR_CUDA: return "CUDA launch or copy failed";
    case SEMICRF_ERR_DEVICE_TIMEOUT: return "a bounded device wait gave up";
    case SEMICRF_ERR_BAD_LENGTH: return "a sequence length is outside [0, T]";
    default: return "unknown status";
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
