// Shared-prefix, tree-masked attention of the multi-item layout.
//
// DuoLM summary page (paper.rainbus.top), 方法步骤详情 step 4 and 研究动机:
// the prefix of a request is computed once and its K/V are shared by all K
// candidate branches; candidate j attends to the prefix and to its own branch
// only.  Work is cut into items of 64 query slots of one request and one KV
// head (a slot is a (token, query head of the KV head's group) pair):
//   kind 0  prefix rows  [row0, row0 + R): causal over the prefix;
//   kind 1  branch rows  [row0, row0 + R') of the request's branch region:
//           every prefix key, then one extra 64-key tile with the branch
//           rows the item's candidates can see (tree rule).
// Each item streams its KV head's prefix tiles through shared memory once and
// serves all 64 slots from them.  QK^T and PV run on fp16 mma.sync
// (m16n8k16, fp32 accumulate); softmax is online in fp32 with the row max and
// sum reduced across the four threads of a quad by warp shuffles.
#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

constexpr int kHD = 128;       // head dim of the fp16 path
constexpr int kSlots = 64;     // query slots per item
constexpr int kKT = 64;        // keys per tile
constexpr int kAttnThreads = 128;
constexpr int kTileBytes = kKT * kHD * 2;  // 16 KB

int attention_rows_per_item(int group) { return kSlots / group; }

// fp16 tile of 64 rows x 128 columns, rows of 256 bytes; 16-byte chunk c of
// row r is stored at chunk c ^ (r & 7) (keeps ldmatrix free of bank conflicts).
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int chunk) {
  return base + r * 256 + ((chunk ^ (r & 7)) << 4);
}

__device__ __forceinline__ void load_tile_async(uint32_t sbase, const __half* g, int tid) {
  // 64 rows x 16 chunks = 1024 chunks, 8 per thread; rows contiguous in global.
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = tid + i * kAttnThreads;
    const int r = idx >> 4, c = idx & 15;
    cp_async16(swz(sbase, r, c), g + (int64_t)r * kHD + c * 8);
  }
}

template <int G>
__global__ void __launch_bounds__(kAttnThreads, 2)
    attention_f16_kernel(const PlanHdr* __restrict__ plan, const __half* __restrict__ q,
                         const __half* __restrict__ kc, const __half* __restrict__ vc, int64_t kv_rows,
                         int n_q_heads, float scale_log2, __half* __restrict__ o, DevStatus* st) {
  extern __shared__ __align__(1024) uint8_t smem[];
  // layout: Q | K buffer 0 | K buffer 1 | V buffer 0 | V buffer 1  (5 x 16 KB)
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK0 = sQ + kTileBytes;
  const uint32_t sV0 = sK0 + 2 * kTileBytes;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = plan->n_items;
  const int b = plan->branch_len;
  const int4* items = plan_array<int4>(plan, plan->off_items);
  const int4* reqs = plan_array<int4>(plan, plan->off_req);
  constexpr int R = kSlots / G;  // token rows per item

  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
    const int4 item = items[it];
    const int4 rq = reqs[item.x];
    const int tok0 = rq.x, L = rq.y, K = rq.z;
    const int kvh = item.y;
    const bool branch = item.z != 0;
    const int row0 = item.w;
    // request-local index of the item's first query token and its row count
    const int q0 = branch ? L + row0 : row0;
    int nrows;
    if (branch) {
      const int per = (R / b) * b;
      nrows = min(per, K * b - row0);
    } else {
      nrows = min(R, L - row0);
    }

    // ---- Q: slot s = (token q0 + s / G, query head kvh * G + s % G)
    __syncthreads();  // previous item's readers of sQ/sK/sV are done
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = tid + i * kAttnThreads;
      const int s = idx >> 4, c = idx & 15;
      const int rl = s / G;
      if (rl < nrows) {
        const int64_t tok = tok0 + q0 + rl;
        cp_async16(swz(sQ, s, c), q + (tok * n_q_heads + kvh * G + (s % G)) * kHD + c * 8);
      } else {
        asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(swz(sQ, s, c)), "r"(0u) : "memory");
      }
    }
    cp_async_commit();

    // key tiles: prefix tiles [0, kend) then, for branch items, one branch tile
    const int kend = branch ? L : min(row0 + R, L);
    const int n_prefix_tiles = (kend + kKT - 1) / kKT;
    const int n_tiles = n_prefix_tiles + (branch ? 1 : 0);
    const __half* kbase = kc + ((int64_t)kvh * kv_rows + tok0) * kHD;
    const __half* vbase = vc + ((int64_t)kvh * kv_rows + tok0) * kHD;
    auto tile_start = [&](int t) { return t < n_prefix_tiles ? t * kKT : q0; };

    load_tile_async(sK0, kbase + (int64_t)tile_start(0) * kHD, tid);
    load_tile_async(sV0, vbase + (int64_t)tile_start(0) * kHD, tid);
    cp_async_commit();

    // per-thread state: rows g = lane/4 and g + 8 of this warp's 16 slots
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float acc[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    const int slot_a = warp * 16 + (lane >> 2);
    const KeyRange kr_a = tree_keys(q0 + slot_a / G, L, b);
    const KeyRange kr_b = tree_keys(q0 + (slot_a + 8) / G, L, b);

    uint32_t qf[8][4];
    for (int t = 0; t < n_tiles; ++t) {
      const int cur = t & 1;
      if (t + 1 < n_tiles) {
        const int nx = (t + 1) & 1;
        load_tile_async(sK0 + nx * kTileBytes, kbase + (int64_t)tile_start(t + 1) * kHD, tid);
        load_tile_async(sV0 + nx * kTileBytes, vbase + (int64_t)tile_start(t + 1) * kHD, tid);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      if (t == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int r = warp * 16 + (lane & 15);
          ldmatrix_x4(swz(sQ, r, 2 * kk + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
      }
      const uint32_t sK = sK0 + cur * kTileBytes;
      const uint32_t sV = sV0 + cur * kTileBytes;
      const int k0 = tile_start(t);

      // S = Q K^T for 16 slots x 64 keys
      float s[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          uint32_t b0, b1, b2, b3;
          const int kr = j * 8 + (lane & 7) + ((lane >> 4) << 3);
          ldmatrix_x4(swz(sK, kr, 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
          mma_16816(s[j], qf[kk], b0, b1);
          mma_16816(s[j + 1], qf[kk], b2, b3);
        }
      }

      // tree mask on the tiles that can reach keys a row may not see: the
      // causal diagonal of prefix items, the prefix end and the branch tile
      // of branch items
      // The visible keys of a row are [0, pre_hi] in the prefix and
      // [br_lo, br_hi] in its own branch; prefix tiles take the first part,
      // the branch tile the second (the two never overlap: br_lo >= L).
      const bool is_branch_tile = branch && t == n_prefix_tiles;
      const bool need_mask = is_branch_tile || (!branch && k0 + kKT > row0) || (branch && k0 + kKT > L);
      float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = s[j][e] * scale_log2;
          if (need_mask) {
            const KeyRange& kr = e < 2 ? kr_a : kr_b;
            const int tk = k0 + j * 8 + 2 * (lane & 3) + (e & 1);
            const bool vis = is_branch_tile ? (tk >= kr.br_lo && tk <= kr.br_hi) : (tk <= kr.pre_hi);
            if (!vis) v = -INFINITY;
          }
          s[j][e] = v;
          tmax[e >> 1] = fmaxf(tmax[e >> 1], v);
        }
      }
      float corr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 1));
        tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 2));
        const float m_new = fmaxf(m_run[h], tmax[h]);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        corr[h] = fast_exp2(m_run[h] - m_use);
        m_run[h] = m_new;
        tmax[h] = m_use;
        l_run[h] *= corr[h];
      }
      float psum[2] = {0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = fast_exp2(s[j][e] - tmax[e >> 1]);
          s[j][e] = p;
          psum[e >> 1] += p;
        }
      }
      l_run[0] += psum[0];
      l_run[1] += psum[1];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        acc[j][0] *= corr[0];
        acc[j][1] *= corr[0];
        acc[j][2] *= corr[1];
        acc[j][3] *= corr[1];
      }
      // O += P V
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_half2(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack_half2(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack_half2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack_half2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) {
          uint32_t b0, b1, b2, b3;
          const int vr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          ldmatrix_x4_trans(swz(sV, vr, 2 * jn + (lane >> 4)), b0, b1, b2, b3);
          mma_16816(acc[2 * jn], pa, b0, b1);
          mma_16816(acc[2 * jn + 1], pa, b2, b3);
        }
      }
      __syncthreads();  // tile buffer `cur` is refilled two iterations later
    }

    // ---- finish: O / l, staged through sQ for 16-byte stores
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
      l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
    }
    const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
    const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int col = j * 8 + 2 * (lane & 3);
      const uint32_t v0 = pack_half2(acc[j][0] * inv0, acc[j][1] * inv0);
      const uint32_t v1 = pack_half2(acc[j][2] * inv1, acc[j][3] * inv1);
      const int r0 = warp * 16 + (lane >> 2);
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(swz(sQ, r0, col >> 3) + (col & 7) * 2), "r"(v0) : "memory");
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(swz(sQ, r0 + 8, col >> 3) + (col & 7) * 2), "r"(v1) : "memory");
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = tid + i * kAttnThreads;
      const int sl = idx >> 4, c = idx & 15;
      const int rl = sl / G;
      if (rl < nrows) {
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(swz(sQ, sl, c)));
        const int64_t tok = tok0 + q0 + rl;
        *reinterpret_cast<uint4*>(o + (tok * n_q_heads + kvh * G + (sl % G)) * kHD + c * 8) = v;
      }
    }
  }
  (void)st;
}

cudaError_t attention_setup() {
  const int smem = 5 * kTileBytes;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(attention_f16_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
    return e;
  if ((e = cudaFuncSetAttribute(attention_f16_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
    return e;
  return cudaFuncSetAttribute(attention_f16_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

cudaError_t attention_f16(const PlanHdr* plan, const __half* q, const __half* kc, const __half* vc, int64_t kv_rows,
                          int n_q_heads, int n_kv_heads, float scale, __half* o, DevStatus* st, int grid,
                          cudaStream_t s) {
  const int G = n_q_heads / n_kv_heads;
  const int smem = 5 * kTileBytes;
  const float sl2 = scale * 1.4426950408889634f;  // softmax in base 2
  switch (G) {
    case 1:
      attention_f16_kernel<1><<<grid, kAttnThreads, smem, s>>>(plan, q, kc, vc, kv_rows, n_q_heads, sl2, o, st);
      break;
    case 2:
      attention_f16_kernel<2><<<grid, kAttnThreads, smem, s>>>(plan, q, kc, vc, kv_rows, n_q_heads, sl2, o, st);
      break;
    case 4:
      attention_f16_kernel<4><<<grid, kAttnThreads, smem, s>>>(plan, q, kc, vc, kv_rows, n_q_heads, sl2, o, st);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// fp32 path: one warp per (token, query head), keys visited in order with an
// online softmax; head_dim a multiple of 32.
// ---------------------------------------------------------------------------
__global__ void attention_f32_kernel(const PlanHdr* __restrict__ plan, const float* __restrict__ q,
                                     const float* __restrict__ kc, const float* __restrict__ vc, int64_t kv_rows,
                                     int n_q_heads, int n_kv_heads, int hd, float scale, float* __restrict__ o) {
  const int T = plan->n_tokens;
  const int b = plan->branch_len;
  const int* treq = plan_array<int32_t>(plan, plan->off_treq);
  const int4* reqs = plan_array<int4>(plan, plan->off_req);
  const int lane = threadIdx.x & 31;
  const int warps_total = (gridDim.x * blockDim.x) >> 5;
  const int group = n_q_heads / n_kv_heads;
  const int per_lane = hd >> 5;  // <= 8
  for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < T * n_q_heads; w += warps_total) {
    const int t = w / n_q_heads, h = w % n_q_heads, kvh = h / group;
    const int4 rq = reqs[treq[t]];
    const int tok0 = rq.x, L = rq.y;
    const int tq = t - tok0;
    float qv[8], accv[8];
    for (int i = 0; i < per_lane; ++i) {
      qv[i] = q[((int64_t)t * n_q_heads + h) * hd + lane + 32 * i];
      accv[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int tk = 0; tk <= tq; ++tk) {
      if (!tree_visible(tq, tk, L, b)) continue;
      const float* kr = kc + ((int64_t)kvh * kv_rows + tok0 + tk) * hd;
      const float* vr = vc + ((int64_t)kvh * kv_rows + tok0 + tk) * hd;
      float d = 0.f;
      for (int i = 0; i < per_lane; ++i) d += qv[i] * kr[lane + 32 * i];
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      const float sc = d * scale;
      const float mn = fmaxf(m, sc);
      const float corr = expf(m - mn);
      const float p = expf(sc - mn);
      l = l * corr + p;
      for (int i = 0; i < per_lane; ++i) accv[i] = accv[i] * corr + p * vr[lane + 32 * i];
      m = mn;
    }
    for (int i = 0; i < per_lane; ++i) o[((int64_t)t * n_q_heads + h) * hd + lane + 32 * i] = accv[i] / l;
  }
}

cudaError_t attention_f32(const PlanHdr* plan, const float* q, const float* kc, const float* vc, int64_t kv_rows,
                          int n_q_heads, int n_kv_heads, int hd, float scale, float* o, int max_rows,
                          cudaStream_t s) {
  const int64_t warps = (int64_t)max_rows * n_q_heads;
  const int blocks = (int)std::min<int64_t>((warps + 7) / 8, 148 * 16);
  attention_f32_kernel<<<blocks, 256, 0, s>>>(plan, q, kc, vc, kv_rows, n_q_heads, n_kv_heads, hd, scale, o);
  return cudaGetLastError();
}

}  // namespace duolm
