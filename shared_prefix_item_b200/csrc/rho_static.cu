// duolm_embedding_rho_static: the embedding's reference scale rho computed
// with a scratch array built into the library instead of allocated memory,
// for callers that cannot allocate device memory (see include/duolm.h).
#include <mutex>

#include "common.cuh"
#include "duolm.h"

namespace {

constexpr int64_t kMaxRows = DUOLM_RHO_STATIC_MAX_ROWS;
constexpr int kMaxDevices = 64;

// Per-row RMS of the last call.  One copy per GPU, alive until the process
// exits; shared by every call on that GPU.
static __device__ __align__(256) double g_rho_rows[kMaxRows];

std::mutex g_mu;
double* g_rows_addr[kMaxDevices] = {};  // device address of g_rho_rows, per device

// RMS of each embedding row in fp64, one block per row (fixed-order reduction).
__global__ void rho_rows_kernel(const void* __restrict__ embed, bool bf16, int64_t vocab, int d,
                                double* __restrict__ rows) {
  __shared__ double red[256];
  for (int64_t r = blockIdx.x; r < vocab; r += gridDim.x) {
    double ss = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      double v;
      if (bf16) {
        const uint16_t u = reinterpret_cast<const uint16_t*>(embed)[r * d + i];
        v = (double)__uint_as_float((uint32_t)u << 16);
      } else {
        v = (double)reinterpret_cast<const float*>(embed)[r * d + i];
      }
      ss += v * v;
    }
    red[threadIdx.x] = ss;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
      __syncthreads();
    }
    if (threadIdx.x == 0) rows[r] = sqrt(red[0] / (double)d);
    __syncthreads();
  }
}

// Mean of the per-row values, one block, fixed-order reduction.
__global__ void rho_mean_kernel(const double* __restrict__ rows, int64_t vocab, double* __restrict__ out) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < vocab; i += blockDim.x) s += rows[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = red[0] / (double)vocab;
}

// Device address of the scratch array on the current device, looked up once
// per device (host code cannot use the array's name as a device pointer).
cudaError_t rows_address(double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_rows_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rho_rows);
    if (e != cudaSuccess) return e;
    g_rows_addr[dev] = static_cast<double*>(p);
  }
  *out = g_rows_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int duolm_embedding_rho_static(const void* embed, int dtype, int64_t vocab, int d, double* rho_out,
                                          void* cuda_stream) {
  if (!embed || !rho_out || d < 1 || (dtype != DUOLM_DTYPE_BF16 && dtype != DUOLM_DTYPE_FP32))
    return DUOLM_E_ARG;
  if (vocab < 1 || vocab > kMaxRows) return DUOLM_E_CAPACITY;
  double* rows = nullptr;
  if (rows_address(&rows) != cudaSuccess) return DUOLM_E_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int grid = (int)(vocab < 148 * 16 ? vocab : 148 * 16);
  rho_rows_kernel<<<grid, 256, 0, s>>>(embed, dtype == DUOLM_DTYPE_BF16, vocab, d, rows);
  if (cudaGetLastError() != cudaSuccess) return DUOLM_E_CUDA;
  rho_mean_kernel<<<1, 1024, 0, s>>>(rows, vocab, rho_out);
  if (cudaGetLastError() != cudaSuccess) return DUOLM_E_CUDA;
  return 0;
}
