// Row-wise kernels of the ranker: virtual-id gather + RMSNorm, RMSNorm,
// score head, the fp32 path's QK-norm/RoPE and SwiGLU steps, the continuous
// interface that builds the item table, and the mask dump used by the tests.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

constexpr int kRowThreads = 256;  // 8 warps, one row per warp
constexpr int kMaxRowBlocks = 148 * 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

template <typename T>
__device__ __forceinline__ void store8(T* dst, const float (&v)[8], DevStatus* st);
template <>
__device__ __forceinline__ void store8<__half>(__half* dst, const float (&v)[8], DevStatus* st) {
  uint32_t p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h = __halves2half2(to_half_checked(v[2 * i], st, 30), to_half_checked(v[2 * i + 1], st, 30));
    p[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(p[0], p[1], p[2], p[3]);
}
template <>
__device__ __forceinline__ void store8<float>(float* dst, const float (&v)[8], DevStatus*) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Load 8 consecutive elements of a row as fp32 (16- or 32-byte vector loads).
__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8_f16(const __half* p, float (&v)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8_f32(const float* p, float (&v)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ---------------------------------------------------------------------------
// Virtual-id gather + RMSNorm (first layer's attention norm).  Ranker id
// id < vocab reads the embedding, id = vocab + i reads row i of the FP16 item
// table (DuoLM summary page, 方法步骤详情 step 3).  One warp per token; each
// lane moves 8-element (16-byte) chunks, chunks lane, lane+32, ... of the row.
// Writes the fp32 residual x and the normed operand xn.
// ---------------------------------------------------------------------------
template <typename OutT, int CH>  // CH = chunks of 8 per lane = d / 256
__global__ void __launch_bounds__(kRowThreads)
    embed_norm_kernel(const PlanHdr* __restrict__ plan, const void* __restrict__ embed, bool embed_bf16,
                      const __half* __restrict__ table, int64_t n_table, int vocab, int d,
                      const float* __restrict__ gain, float eps, float* __restrict__ x, OutT* __restrict__ xn,
                      DevStatus* st) {
  const int T = plan->n_tokens;
  const int* ids = plan_array<int32_t>(plan, plan->off_ids);
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nw) {
    const int id = ids[t];
    float v[CH][8];
    const bool vid = id >= vocab;
    const bool ok = id >= 0 && (int64_t)id < (int64_t)vocab + n_table;
    if (!ok) {
      if (lane == 0) raise_error(st, ERR_BAD_INDEX, 31);
#pragma unroll
      for (int c = 0; c < CH; ++c)
#pragma unroll
        for (int i = 0; i < 8; ++i) v[c][i] = 0.f;
    } else {
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int col = (lane + 32 * c) * 8;
        if (col >= d) {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[c][i] = 0.f;
        } else if (vid) {
          load8_f16(table + (int64_t)(id - vocab) * d + col, v[c]);
        } else if (embed_bf16) {
          load8_bf16(reinterpret_cast<const __nv_bfloat16*>(embed) + (int64_t)id * d + col, v[c]);
        } else {
          load8_f32(reinterpret_cast<const float*>(embed) + (int64_t)id * d + col, v[c]);
        }
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c)
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += v[c][i] * v[c][i];
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)d + eps);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col >= d) continue;
      store8<float>(x + (int64_t)t * d + col, v[c], st);
      float nv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) nv[i] = (v[c][i] * r) * gain[col + i];
      store8<OutT>(xn + (int64_t)t * d + col, nv, st);
    }
  }
}

// fp16 path: the same gather, but the layer-0 norm is left to the QKV
// epilogue: writes x, fp16(x * gain) and the row's sum of x^2 (slot 0; the
// other n_slots - 1 partial-sum slots of the row are zeroed).
template <int CH>
__global__ void __launch_bounds__(kRowThreads)
    embed_gain_kernel(const PlanHdr* __restrict__ plan, const void* __restrict__ embed,
                      const __half* __restrict__ table, int64_t n_table, int vocab, int d,
                      const float* __restrict__ gain, float* __restrict__ x, __half* __restrict__ xg,
                      float* __restrict__ ssp, int n_slots, DevStatus* st) {
  pdl_launch_dependents();
  pdl_wait();
  const int T = plan->n_tokens;
  const int* ids = plan_array<int32_t>(plan, plan->off_ids);
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nw) {
    const int id = ids[t];
    float v[CH][8];
    const bool ok = id >= 0 && (int64_t)id < (int64_t)vocab + n_table;
    if (!ok && lane == 0) raise_error(st, ERR_BAD_INDEX, 33);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (!ok || col >= d) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[c][i] = 0.f;
      } else if (id >= vocab) {
        load8_f16(table + (int64_t)(id - vocab) * d + col, v[c]);
      } else {
        load8_bf16(reinterpret_cast<const __nv_bfloat16*>(embed) + (int64_t)id * d + col, v[c]);
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col >= d) continue;
      float gv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ss += v[c][i] * v[c][i];
        gv[i] = v[c][i] * gain[col + i];
      }
      store8<float>(x + (int64_t)t * d + col, v[c], st);
      store8<__half>(xg + (int64_t)t * d + col, gv, st);
    }
    ss = warp_sum(ss);
    if (lane < n_slots) ssp[(int64_t)t * n_slots + lane] = lane == 0 ? ss : 0.f;
  }
}

cudaError_t embed_gain(const PlanHdr* plan, const void* embed, const __half* table, int64_t n_table, int vocab, int d,
                       const float* gain, float* x, __half* xg, float* ssp, int n_slots, DevStatus* st, int max_rows,
                       cudaStream_t s, bool pdl) {
  const int g = std::max(1, std::min((max_rows + 7) / 8, kMaxRowBlocks));
  if (d % 8 || n_slots > 32 || n_slots % 4) return cudaErrorInvalidValue;
  switch ((d + 255) / 256) {
#define DUOLM_EG_CASE(n)                                                                                            \
  case n:                                                                                                           \
    if (cudaError_t e_ = launch_ex(embed_gain_kernel<n>, dim3(g), dim3(kRowThreads), 0, s, pdl, plan, embed, table,   \
                                   n_table, vocab, d, gain, x, xg, ssp, n_slots, st))                                 \
      return e_;                                                                                                    \
    break;
    DUOLM_EG_CASE(1) DUOLM_EG_CASE(2) DUOLM_EG_CASE(3) DUOLM_EG_CASE(4) DUOLM_EG_CASE(8)
#undef DUOLM_EG_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename OutT, int CH>
__global__ void __launch_bounds__(kRowThreads)
    rmsnorm_kernel(const PlanHdr* __restrict__ plan, const float* __restrict__ x, int d,
                   const float* __restrict__ gain, float eps, OutT* __restrict__ xn, DevStatus* st) {
  const int T = plan->n_tokens;
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nw) {
    float v[CH][8];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col < d) {
        load8_f32(x + (int64_t)t * d + col, v[c]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[c][i] = 0.f;
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c)
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += v[c][i] * v[c][i];
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)d + eps);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int col = (lane + 32 * c) * 8;
      if (col >= d) continue;
      float nv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) nv[i] = (v[c][i] * r) * gain[col + i];
      store8<OutT>(xn + (int64_t)t * d + col, nv, st);
    }
  }
}

static int row_blocks(int max_rows) {
  return std::max(1, std::min((max_rows + 7) / 8, kMaxRowBlocks));
}

template <typename OutT>
cudaError_t embed_norm(const PlanHdr* plan, const void* embed, bool embed_bf16, const __half* table,
                       int64_t n_table, int vocab, int d, const float* gain, float eps, float* x, OutT* xn,
                       DevStatus* st, int max_rows, cudaStream_t s) {
  const int g = row_blocks(max_rows);
  if (d % 8) return cudaErrorInvalidValue;
  switch ((d + 255) / 256) {
#define DUOLM_EMB_CASE(n)                                                                                   \
  case n:                                                                                                   \
    embed_norm_kernel<OutT, n><<<g, kRowThreads, 0, s>>>(plan, embed, embed_bf16, table, n_table, vocab, d, \
                                                         gain, eps, x, xn, st);                             \
    break;
    DUOLM_EMB_CASE(1) DUOLM_EMB_CASE(2) DUOLM_EMB_CASE(3) DUOLM_EMB_CASE(4) DUOLM_EMB_CASE(8)
#undef DUOLM_EMB_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename OutT>
cudaError_t rmsnorm_rows(const PlanHdr* plan, const float* x, int d, const float* gain, float eps, OutT* xn,
                         DevStatus* st, int max_rows, cudaStream_t s) {
  const int g = row_blocks(max_rows);
  if (d % 8) return cudaErrorInvalidValue;
  switch ((d + 255) / 256) {
#define DUOLM_RMS_CASE(n)                                                                         \
  case n:                                                                                         \
    rmsnorm_kernel<OutT, n><<<g, kRowThreads, 0, s>>>(plan, x, d, gain, eps, xn, st);             \
    break;
    DUOLM_RMS_CASE(1) DUOLM_RMS_CASE(2) DUOLM_RMS_CASE(3) DUOLM_RMS_CASE(4) DUOLM_RMS_CASE(8)
#undef DUOLM_RMS_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template cudaError_t embed_norm<float>(const PlanHdr*, const void*, bool, const __half*, int64_t, int, int,
                                       const float*, float, float*, float*, DevStatus*, int, cudaStream_t);
template cudaError_t rmsnorm_rows<float>(const PlanHdr*, const float*, int, const float*, float, float*,
                                         DevStatus*, int, cudaStream_t);

// ---------------------------------------------------------------------------
// Score head: s = w . (RMSNorm(x) * g_final) at the last token of every
// candidate branch, in input order (DuoLM summary page, 核心方法).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kRowThreads)
    score_head_kernel(const PlanHdr* __restrict__ plan, const float* __restrict__ x, int d,
                      const float* __restrict__ gain, const float* __restrict__ w, float eps,
                      float* __restrict__ scores) {
  pdl_wait();
  const int n = plan->n_cand;
  const int* rows = plan_array<int32_t>(plan, plan->off_cand);
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; c < n; c += nw) {
    const float* xr = x + (int64_t)rows[c] * d;
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) ss += xr[i] * xr[i];
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)d + eps);
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) acc += w[i] * ((xr[i] * r) * gain[i]);
    acc = warp_sum(acc);
    if (lane == 0) scores[c] = acc;
  }
}

cudaError_t score_head(const PlanHdr* plan, const float* x, int d, const float* gain, const float* w, float eps,
                       float* scores, int max_cand, cudaStream_t s, bool pdl) {
  return launch_ex(score_head_kernel, dim3(row_blocks(max_cand)), dim3(kRowThreads), 0, s, pdl, plan, x, d, gain, w,
                   eps, scores);
}

// ---------------------------------------------------------------------------
// fp32 path: per (token, head) QK-norm + RoPE for q and k, copy for v.
// qkv rows are [q heads | k heads | v heads].
// ---------------------------------------------------------------------------
__global__ void qkv_post_f32_kernel(const PlanHdr* __restrict__ plan, const float* __restrict__ qkv, int nq,
                                    int nkv, int hd, const float* __restrict__ gq, const float* __restrict__ gk,
                                    float eps, const float2* __restrict__ rope, int max_pos, float* __restrict__ q,
                                    float* __restrict__ kc, float* __restrict__ vc, int64_t kv_rows,
                                    DevStatus* st) {
  const int T = plan->n_tokens;
  const int* pos = plan_array<int32_t>(plan, plan->off_pos);
  const int heads = nq + 2 * nkv;
  const int width = heads * hd;
  const int half = hd / 2;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < (int64_t)T * heads;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(w / heads), h = (int)(w % heads);
    const float* src = qkv + (int64_t)t * width + h * hd;
    if (h >= nq + nkv) {
      float* dst = vc + ((int64_t)(h - nq - nkv) * kv_rows + t) * hd;
      for (int i = 0; i < hd; ++i) dst[i] = src[i];
      continue;
    }
    const bool is_q = h < nq;
    const float* g = is_q ? gq : gk;
    float* dst = is_q ? q + ((int64_t)t * nq + h) * hd : kc + ((int64_t)(h - nq) * kv_rows + t) * hd;
    float ss = 0.f;
    for (int i = 0; i < hd; ++i) ss += src[i] * src[i];
    const float r = 1.0f / sqrtf(ss / (float)hd + eps);
    int p = pos[t];
    if (p < 0 || p >= max_pos) {
      raise_error(st, ERR_BAD_INDEX, 32);
      p = 0;
    }
    const float2* cs = rope + p;  // entry (i, p) at cs[i * max_pos]
    for (int i = 0; i < half; ++i) {
      const float a = (src[i] * r) * g[i];
      const float bb = (src[i + half] * r) * g[i + half];
      const float2 t = cs[(int64_t)i * max_pos];
      dst[i] = a * t.x - bb * t.y;
      dst[i + half] = bb * t.x + a * t.y;
    }
  }
}

cudaError_t qkv_post_f32(const PlanHdr* plan, const float* qkv, int n_q_heads, int n_kv_heads, int hd,
                         const float* gq, const float* gk, float eps, const float2* rope, int max_pos, float* q,
                         float* kc, float* vc, int64_t kv_rows, DevStatus* st, int max_rows, cudaStream_t s) {
  const int64_t work = (int64_t)max_rows * (n_q_heads + 2 * n_kv_heads);
  const int g = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, 148 * 8));
  qkv_post_f32_kernel<<<g, 256, 0, s>>>(plan, qkv, n_q_heads, n_kv_heads, hd, gq, gk, eps, rope, max_pos, q, kc,
                                        vc, kv_rows, st);
  return cudaGetLastError();
}

__global__ void swiglu_f32_kernel(const PlanHdr* __restrict__ plan, const float* __restrict__ gu, int F,
                                  float* __restrict__ h) {
  const int T = plan->n_tokens;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)T * F;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / F, f = i % F;
    const float g = gu[t * 2 * F + f];
    const float u = gu[t * 2 * F + F + f];
    h[i] = g / (1.0f + expf(-g)) * u;
  }
}

cudaError_t swiglu_f32(const PlanHdr* plan, const float* gu, int F, float* h, int max_rows, cudaStream_t s) {
  const int64_t work = (int64_t)max_rows * F;
  const int g = (int)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, 148 * 8));
  swiglu_f32_kernel<<<g, 256, 0, s>>>(plan, gu, F, h);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Continuous interface: z = (e^gamma * rho) * a / RMS(a) per row, RMS without
// epsilon, in fp64, stored as FP16 rounded to nearest even (DuoLM summary page,
// 前置知识 连续输入接口 and 核心方法).  One block per row; the sum of squares
// is reduced in a fixed order.
// ---------------------------------------------------------------------------
__global__ void table_build_kernel(const float* __restrict__ a, int64_t n, int d, double scale_num,
                                   __half* __restrict__ out) {
  __shared__ double red[256];
  for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
    const float* row = a + r * d;
    double ss = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) ss += (double)row[i] * (double)row[i];
    red[threadIdx.x] = ss;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
      __syncthreads();
    }
    const double rms = sqrt(red[0] / (double)d);
    __syncthreads();
    for (int i = threadIdx.x; i < d; i += blockDim.x) out[r * d + i] = __double2half(scale_num * (double)row[i] / rms);
  }
}

cudaError_t table_build(const float* a, int64_t n, int d, double scale_num, __half* out, cudaStream_t s) {
  const int g = (int)std::min<int64_t>(n, 148 * 16);
  if (g <= 0) return cudaSuccess;
  table_build_kernel<<<g, 256, 0, s>>>(a, n, d, scale_num, out);
  return cudaGetLastError();
}

__global__ void row_rms_kernel(const void* __restrict__ embed, bool bf16, int64_t vocab, int d,
                               double* __restrict__ out) {
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
    if (threadIdx.x == 0) out[r] = sqrt(red[0] / (double)d);
    __syncthreads();
  }
}

__global__ void mean_kernel(const double* __restrict__ v, int64_t n, double* __restrict__ out) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += v[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = red[0] / (double)n;
}

cudaError_t embed_rho(const void* embed, bool embed_bf16, int64_t vocab, int d, double* row_rms, double* out,
                      cudaStream_t s) {
  row_rms_kernel<<<(int)std::min<int64_t>(vocab, 148 * 16), 256, 0, s>>>(embed, embed_bf16, vocab, d, row_rms);
  mean_kernel<<<1, 1024, 0, s>>>(row_rms, vocab, out);
  return cudaGetLastError();
}

// A wait that nothing completes: exercises the bounded-wait error path.
__global__ void wait_timeout_kernel(DevStatus* st) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t a = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(a, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(a, 0, st, 90);
  __syncthreads();
}

cudaError_t debug_wait_timeout(DevStatus* st, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(st);
  return cudaGetLastError();
}

// The attention kernels' visibility rule evaluated for every pair of one request.
__global__ void debug_mask_kernel(const PlanHdr* __restrict__ plan, int request, uint8_t* __restrict__ out,
                                  int64_t tq_n) {
  const int4 rq = plan_array<int4>(plan, plan->off_req)[request];
  const int b = plan->branch_len;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < tq_n * tq_n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = tree_visible((int)(i / tq_n), (int)(i % tq_n), rq.y, b) ? 1 : 0;
}

cudaError_t debug_mask(const PlanHdr* plan, int request, uint8_t* out, int64_t tq, cudaStream_t s) {
  const int g = (int)std::max<int64_t>(1, std::min<int64_t>((tq * tq + 255) / 256, 1024));
  debug_mask_kernel<<<g, 256, 0, s>>>(plan, request, out, tq);
  return cudaGetLastError();
}

}  // namespace duolm
