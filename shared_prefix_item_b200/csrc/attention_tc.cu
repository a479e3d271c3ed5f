// Shared-prefix, tree-masked attention on 5th-generation tensor cores.
//
// DuoLM summary page (paper.rainbus.top), 方法步骤详情 step 4 and 研究动机:
// the prefix of a request is computed once and its K/V are shared by all K
// candidate branches; candidate j attends to the prefix and to its own branch
// only.  Work is cut into items of 128 query slots of one request and one KV
// head (a slot is a (token, query head of the KV head's group) pair; 64
// tokens x 2 heads for Qwen3's grouping):
//   kind 0  prefix tokens [row0, row0 + R): causal over the prefix;
//   kind 1  branch tokens [row0, row0 + R') (whole candidates): every prefix
//           key, then one extra 128-key tile of branch rows under the tree rule.
// Per item each KV head's prefix tiles stream through shared memory once for
// all 128 slots.  One CTA per SM, 192 threads:
//   warp 0   TMA: Q (3-D map, 2 x 16 KB), then K and V tiles of 128 keys
//            (2 x 32 KB each, double buffered); 128-byte swizzle, no multicast;
//   warp 1   one lane issues tcgen05.mma: S = Q K^T (M 128, N 128 keys,
//            K-major operands) into one of two TMEM S buffers, then
//            O += P V (P from shared memory K-major, V MN-major) into TMEM;
//            S of tile t + 1 is issued before P V of tile t;
//   warps 2-5 softmax, one thread per slot row (TMEM lane): load S, mask,
//            row max, P = 2^(s - m) in fp16 to shared memory, row sum; O in
//            TMEM is rescaled only when the running max grows by more than
//            2^8 (P stays below 256, exact after the final division);
//            finally O / l to global memory.
// Every mbarrier wait is bounded; after a timeout the kernel raises the
// status flag and returns.
#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

namespace {

constexpr int kSlots = 128;   // query slots per item (MMA M)
constexpr int kKeys = 128;    // keys per tile (MMA N of Q K^T)
constexpr int kHD = 128;
constexpr int kThreads = 192;
constexpr int kHalf = 16384;  // one 128-row x 64-element fp16 box
constexpr int kQOff = 0;                  // Q: 2 boxes
constexpr int kKOff = 2 * kHalf;          // K: 2 slots x 2 boxes
constexpr int kVOff = kKOff + 4 * kHalf;  // V: 2 slots x 2 boxes
constexpr int kPOff = kVOff + 4 * kHalf;  // P: 2 boxes
constexpr int kBarOff = kPOff + 2 * kHalf;
constexpr int kSmem = kBarOff + 256 + 1024;
constexpr uint32_t kIdescS = idesc_f16_f32(128, kKeys);
constexpr uint32_t kIdescPV = idesc_f16_f32_bmn(128, kHD);
constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O [256,384)
constexpr float kRescaleLog2 = 8.0f;

enum { B_QFULL, B_KVFULL0, B_KVFULL1, B_KVEMPTY0, B_KVEMPTY1, B_SFULL0, B_SFULL1, B_SEMPTY0, B_SEMPTY1,
       B_PFULL, B_PEMPTY, B_OFULL, B_COUNT };

struct Item {
  int tok0, L, K, kvh, branch, row0, q0, nrows, n_prefix_tiles, n_tiles;
  __device__ int tile_start(int t) const { return t < n_prefix_tiles ? t * kKeys : q0; }
};

template <int G>
__device__ __forceinline__ Item load_item(const PlanHdr* plan, int it, int b) {
  constexpr int R = kSlots / G;
  const int4 item = plan_array<int4>(plan, plan->off_items)[it];
  const int4 rq = plan_array<int4>(plan, plan->off_req)[item.x];
  Item m;
  m.tok0 = rq.x;
  m.L = rq.y;
  m.K = rq.z;
  m.kvh = item.y;
  m.branch = item.z;
  m.row0 = item.w;
  m.q0 = m.branch ? m.L + m.row0 : m.row0;
  m.nrows = m.branch ? min((R / b) * b, m.K * b - m.row0) : min(R, m.L - m.row0);
  const int kend = m.branch ? m.L : min(m.row0 + R, m.L);
  m.n_prefix_tiles = (kend + kKeys - 1) / kKeys;
  m.n_tiles = m.n_prefix_tiles + (m.branch ? 1 : 0);
  return m;
}

}  // namespace

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PlanHdr* __restrict__ plan, int64_t kv_rows,
                        int n_q_heads, float scale_log2, __half* __restrict__ o, DevStatus* st) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);

  if (*reinterpret_cast<volatile const uint32_t*>(&st->flags) & ERR_WAIT_TIMEOUT) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = plan->n_items;
  const int b = plan->branch_len;
  constexpr int R = kSlots / G;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    for (int i = 0; i < B_COUNT; ++i) {
      const uint32_t cnt = (i == B_SEMPTY0 || i == B_SEMPTY1 || i == B_PFULL) ? 128u : 1u;
      mbar_init(bar(i), cnt);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmemO = tmem + 256;

  // running counts, identical in every role (same items, same tiles)
  uint32_t n_item = 0, n_kv = 0, n_s = 0, n_p = 0;
  bool ok = true;

  for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++n_item) {
    const Item m = load_item<G>(plan, it, b);
    if (warp == 0) {
      if (lane == 0 && ok) {
        mbar_arrive_expect_tx(bar(B_QFULL), 2 * kHalf);
        for (int h = 0; h < 2; ++h)
          tma_load_3d(&tmQ, sbase + kQOff + h * kHalf, bar(B_QFULL), h * 64, m.kvh * G, m.tok0 + m.q0);
        for (int t = 0; t < m.n_tiles && ok; ++t) {
          const uint32_t slot = (n_kv + t) & 1, use = (n_kv + t) >> 1;
          if (!mbar_wait(bar(B_KVEMPTY0 + slot), (use & 1u) ^ 1u, st, 40)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(B_KVFULL0 + slot), 4 * kHalf);
          const int y = (int)((int64_t)m.kvh * kv_rows + m.tok0 + m.tile_start(t));
          for (int h = 0; h < 2; ++h) {
            tma_load_2d(&tmK, sbase + kKOff + (2 * slot + h) * kHalf, bar(B_KVFULL0 + slot), h * 64, y);
            tma_load_2d(&tmV, sbase + kVOff + (2 * slot + h) * kHalf, bar(B_KVFULL0 + slot), h * 64, y);
          }
        }
      }
    } else if (warp == 1) {
      if (lane == 0 && ok) {
        auto pv = [&](int t) -> bool {
          if (!mbar_wait(bar(B_PFULL), (n_p + t) & 1u, st, 41)) return false;
          tc_fence_after();
          const uint32_t slot = (n_kv + t) & 1;
#pragma unroll
          for (int k = 0; k < kKeys / 16; ++k) {
            const uint64_t da = smem_desc_sw128(sbase + kPOff + (k >> 2) * kHalf + (k & 3) * 32);
            const uint64_t db = smem_desc_sw128_mn(sbase + kVOff + 2 * slot * kHalf + k * 2048, kHalf);
            tc_mma_f16(tmemO, da, db, kIdescPV, (t > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(bar(B_KVEMPTY0 + slot));
          tc_commit(bar(B_PEMPTY));
          return true;
        };
        if (!mbar_wait(bar(B_QFULL), n_item & 1u, st, 42)) ok = false;
        tc_fence_after();
        for (int t = 0; t < m.n_tiles && ok; ++t) {
          const uint32_t slot = (n_kv + t) & 1, kuse = (n_kv + t) >> 1;
          const uint32_t sb = (n_s + t) & 1, suse = (n_s + t) >> 1;
          if (!mbar_wait(bar(B_KVFULL0 + slot), kuse & 1u, st, 43) ||
              !mbar_wait(bar(B_SEMPTY0 + sb), (suse & 1u) ^ 1u, st, 44)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kHD / 16; ++k) {
            const uint64_t da = smem_desc_sw128(sbase + kQOff + (k >> 2) * kHalf + (k & 3) * 32);
            const uint64_t db = smem_desc_sw128(sbase + kKOff + (2 * slot + (k >> 2)) * kHalf + (k & 3) * 32);
            tc_mma_f16(tmem + sb * kKeys, da, db, kIdescS, k > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_SFULL0 + sb));
          if (t > 0 && !pv(t - 1)) ok = false;
        }
        if (ok && !pv(m.n_tiles - 1)) ok = false;
        if (ok) tc_commit(bar(B_OFULL));
      }
    } else {
      // ---- softmax: thread = slot row r = TMEM lane
      const int q4 = warp & 3;
      const int r = q4 * 32 + lane;
      const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
      const KeyRange kr = tree_keys(m.q0 + r / G, m.L, b);
      float m_used = -INFINITY, l = 0.f;
      for (int t = 0; t < m.n_tiles && ok; ++t) {
        const uint32_t sb = (n_s + t) & 1, suse = (n_s + t) >> 1;
        if (!mbar_wait_warp(bar(B_SFULL0 + sb), suse & 1u, st, 45)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int k0 = m.tile_start(t);
        const bool is_branch_tile = m.branch && t == m.n_prefix_tiles;
        const bool need_mask = is_branch_tile || (!m.branch && k0 + kKeys > m.row0) || (m.branch && k0 + kKeys > m.L);
        const uint32_t s_addr = tmem + lane_off + sb * kKeys;
        // the whole S row in registers: four loads, one wait
        uint32_t sr[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32_async(s_addr + 32 * q, sr[q]);
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            tmem_ld_fence(sr[q][j]);
            float x = __uint_as_float(sr[q][j]) * scale_log2;
            if (need_mask) {
              const int tk = k0 + 32 * q + j;
              const bool vis = is_branch_tile ? (tk >= kr.br_lo && tk <= kr.br_hi) : (tk <= kr.pre_hi);
              if (!vis) x = -INFINITY;
            }
            sr[q][j] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
        // P buffer free and O complete for the previous tile
        if (!mbar_wait_warp(bar(B_PEMPTY), ((n_p + t) & 1u) ^ 1u, st, 46)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float m_new = fmaxf(m_used, mx);
        // the O rescale uses warp-collective TMEM loads and stores: decide it
        // for the whole warp (a row that did not need it is rescaled to its
        // new max as well, which is just as exact)
        if (t == 0) {
          m_used = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m_used + kRescaleLog2)) {
          const float corr = m_new == m_used ? 1.f : fast_exp2(m_used - m_new);  // 0 while nothing was visible
#pragma unroll 1
          for (int c = 0; c < kHD; c += 32) {
            float v[32];
            tmem_ld32(tmemO + lane_off + c, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= corr;
            tmem_st32(tmemO + lane_off + c, v);
          }
          l *= corr;
          m_used = m_new;
        }
        const float mu = m_used == -INFINITY ? 0.f : m_used;
        // P = 2^(s - mu) in fp16, K-major 128-byte-swizzled rows
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const __half2 h = __floats2half2_rn(fast_exp2(__uint_as_float(sr[q][j]) - mu),
                                                fast_exp2(__uint_as_float(sr[q][j + 1]) - mu));
            const float2 hf = __half22float2(h);  // sum what the tensor core will see
            sum += hf.x + hf.y;
            pk[j / 2] = *reinterpret_cast<const uint32_t*>(&h);
          }
          const uint32_t pbox = sbase + kPOff + (q >> 1) * kHalf + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int chunk = (q & 1) * 4 + u;
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(pbox + ((chunk ^ (r & 7)) << 4)),
                         "r"(pk[4 * u]), "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]), "r"(pk[4 * u + 3])
                         : "memory");
          }
        }
        l += sum;
        tc_fence_before();
        mbar_arrive(bar(B_SEMPTY0 + sb));
        fence_proxy_async_smem();
        mbar_arrive(bar(B_PFULL));
      }
      // ---- epilogue: O / l -> fp16
      if (ok && mbar_wait_warp(bar(B_OFULL), n_item & 1u, st, 47)) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const int rl = r / G;
        const bool valid = rl < m.nrows;
        __half* dst = o + (((int64_t)m.tok0 + m.q0 + rl) * n_q_heads + m.kvh * G + (r % G)) * kHD;
#pragma unroll 1
        for (int c = 0; c < kHD; c += 32) {
          float v[32];
          tmem_ld32(tmemO + lane_off + c, v);
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const __half2 h = __floats2half2_rn(v[2 * j] * inv, v[2 * j + 1] * inv);
              pk[j] = *reinterpret_cast<const uint32_t*>(&h);
            }
            uint4* p = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int q = 0; q < 4; ++q) p[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        tc_fence_before();
      } else {
        ok = false;
      }
    }
    n_kv += m.n_tiles;
    n_s += m.n_tiles;
    n_p += m.n_tiles;
    // every async operation of this item is complete (the epilogue saw O):
    // Q, the KV slots and O can be reused by the next item; a failed wait in
    // any thread stops the whole CTA
    if (__syncthreads_or(ok ? 0 : 1)) break;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

int attention_tc_rows_per_item(int group) { return kSlots / group; }
int attention_tc_smem_bytes() { return kSmem; }

cudaError_t attention_tc_setup() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(attention_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem)))
    return e;
  if ((e = cudaFuncSetAttribute(attention_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem)))
    return e;
  return cudaFuncSetAttribute(attention_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
}

cudaError_t attention_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const PlanHdr* plan,
                         int64_t kv_rows, int n_q_heads, int n_kv_heads, float scale, __half* o, DevStatus* st,
                         int grid, cudaStream_t s) {
  const int G = n_q_heads / n_kv_heads;
  const float sl2 = scale * 1.4426950408889634f;  // softmax in base 2
  switch (G) {
    case 1:
      attention_tc_kernel<1><<<grid, kThreads, kSmem, s>>>(tq, tk, tv, plan, kv_rows, n_q_heads, sl2, o, st);
      break;
    case 2:
      attention_tc_kernel<2><<<grid, kThreads, kSmem, s>>>(tq, tk, tv, plan, kv_rows, n_q_heads, sl2, o, st);
      break;
    case 4:
      attention_tc_kernel<4><<<grid, kThreads, kSmem, s>>>(tq, tk, tv, plan, kv_rows, n_q_heads, sl2, o, st);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace duolm
