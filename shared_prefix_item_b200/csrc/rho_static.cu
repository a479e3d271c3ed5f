// duolm_embedding_rho_static: the embedding's reference scale rho computed
// with a scratch array built into the library instead of allocated memory,
// for callers that cannot allocate device memory (see include/duolm.h).  The
// arithmetic is the context's own (duolm::embed_rho: per-row RMS in fp64,
// then their mean); only where the per-row values live differs.
#include <cstdio>
#include <mutex>
#include <string>

#include "common.cuh"
#include "duolm.h"
#include "kernels.cuh"

// reason of the calling thread's last failed context-free call (runtime.cu)
extern thread_local std::string g_noctx_err;

namespace {

constexpr int64_t kMaxRows = DUOLM_RHO_STATIC_MAX_ROWS;
constexpr int kMaxDevices = 64;

// Per-row RMS of the last call.  One copy per GPU, alive until the process
// exits; shared by every call on that GPU.
static __device__ __align__(256) double g_rho_rows[kMaxRows];

std::mutex g_mu;
double* g_rows_addr[kMaxDevices] = {};  // last looked-up address of g_rho_rows, per device

int fail_cuda(const char* what, cudaError_t e) {
  char buf[256];
  std::snprintf(buf, sizeof buf, "embedding_rho_static: %s: %s", what, cudaGetErrorString(e));
  g_noctx_err = buf;
  return DUOLM_E_CUDA;
}

// Device address of the scratch array on the current device.  Host code
// cannot use the array's name as a device pointer, so the address is looked
// up with the device current.  Outside stream capture it is looked up on
// every call (a reset device or another context may have moved the module);
// while the stream is being captured the address of the last call outside
// capture on this device is used, so one such call must come first.
int rows_address(cudaStream_t s, double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) return fail_cuda("device index", cudaErrorInvalidDevice);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if ((e = cudaStreamIsCapturing(s, &cap)) != cudaSuccess) return fail_cuda("cudaStreamIsCapturing", e);
  std::lock_guard<std::mutex> lock(g_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_rho_rows)) != cudaSuccess) return fail_cuda("cudaGetSymbolAddress", e);
    g_rows_addr[dev] = static_cast<double*>(p);
  } else if (!g_rows_addr[dev]) {
    g_noctx_err = "embedding_rho_static: first call on this device made during stream capture";
    return DUOLM_E_STATE;
  }
  *out = g_rows_addr[dev];
  return 0;
}

}  // namespace

extern "C" int duolm_embedding_rho_static(const void* embed, int dtype, int64_t vocab, int d, double* rho_out,
                                          void* cuda_stream) {
  g_noctx_err.clear();
  if (!embed || !rho_out || d < 1 || (dtype != DUOLM_DTYPE_BF16 && dtype != DUOLM_DTYPE_FP32)) {
    g_noctx_err = "embedding_rho_static: null pointer, d < 1 or unknown dtype";
    return DUOLM_E_ARG;
  }
  if (vocab < 1 || vocab > kMaxRows) {
    g_noctx_err = "embedding_rho_static: vocab outside [1, DUOLM_RHO_STATIC_MAX_ROWS]";
    return DUOLM_E_CAPACITY;
  }
  // an error left by earlier work is reported now, before anything is
  // enqueued, so that a failed call has launched nothing
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail_cuda("error pending before the call", e);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  double* rows = nullptr;
  if (const int rc = rows_address(s, &rows)) return rc;
  if ((e = duolm::embed_rho(embed, dtype == DUOLM_DTYPE_BF16, vocab, d, rows, rho_out, s)) != cudaSuccess)
    return fail_cuda("launch", e);
  return 0;
}
