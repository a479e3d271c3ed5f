// fp32 projection GEMM of the fp32 path (CUDA cores; tensor cores have no
// fp32 operand kind): C[M, N] (+)= A[M, K] * B[N, K]^T, M = batch tokens.
// 64x64 tiles, 256 threads, 4x4 outputs per thread, k summed in order.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

__global__ void __launch_bounds__(256)
    gemm_simt_kernel(const float* __restrict__ A, const float* __restrict__ B, float* __restrict__ C, int K, int N,
                     int ldc, bool accumulate, const PlanHdr* __restrict__ plan) {
  const int M = plan->n_tokens;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (m0 >= M) return;
  __shared__ float As[16][65];
  __shared__ float Bs[16][65];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float c[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) c[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 1024; i += 256) {
      const int r = i >> 4, kk = i & 15, gk = k0 + kk;
      const int gm = m0 + r, gn = n0 + r;
      As[kk][r] = (gm < M && gk < K) ? A[(int64_t)gm * K + gk] : 0.f;
      Bs[kk][r] = (gn < N && gk < K) ? B[(int64_t)gn * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) c[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      float* p = C + (int64_t)gm * ldc + gn;
      *p = accumulate ? *p + c[i][j] : c[i][j];
    }
  }
}

cudaError_t gemm_simt(const float* A, const float* B, float* C, int K, int N, int ldc, bool accumulate,
                      const PlanHdr* plan, int max_rows, cudaStream_t s) {
  dim3 grid((N + 63) / 64, std::max(1, (max_rows + 63) / 64));
  gemm_simt_kernel<<<grid, 256, 0, s>>>(A, B, C, K, N, ldc, accumulate, plan);
  return cudaGetLastError();
}

}  // namespace duolm
