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
// all 128 slots.  One CTA per SM, 320 threads:
//   warp 0   TMA: Q (3-D map, 2 x 16 KB, double buffered so the next item's
//            Q arrives early), then K and V tiles of 128 keys (2 x 32 KB
//            each, double buffered); 128-byte swizzle, no multicast;
//   warp 1   one lane issues tcgen05.mma: S = Q K^T (M 128, N 128 keys,
//            K-major operands) into one of two TMEM S buffers, then
//            O += P V (P from shared memory K-major, V MN-major) into TMEM;
//            S of tile t + 1 is issued before P V of tile t;
//   warps 2-9 softmax, two threads per slot row (TMEM lane), each on half of
//            the keys: load S, mask, row max (halves combined through shared
//            memory), P = 2^(s - m) in fp16 to shared memory, row sum; O in
//            TMEM is rescaled only when the running max grows by more than
//            2^8 (P stays below 256, exact after the final division);
//            finally O / l to global memory.
// The three roles run ahead of each other across item boundaries; every
// mbarrier wait is bounded, and after a timeout the kernel raises the status
// flag and returns.
#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

namespace {

constexpr int kSlots = 128;   // query slots per item (MMA M)
constexpr int kKeys = 128;    // keys per tile (MMA N of Q K^T)
constexpr int kHD = 128;
constexpr int kSoftmax = 256;             // 8 softmax warps: two per TMEM lane quadrant
constexpr int kThreads = 64 + kSoftmax;
constexpr int kHalf = 16384;  // one 128-row x 64-element fp16 box
constexpr int kQOff = 0;                  // Q: 2 slots x 2 boxes (next item's Q loads early)
constexpr int kKOff = 4 * kHalf;          // K: 2 slots x 2 boxes
constexpr int kVOff = kKOff + 4 * kHalf;  // V: 2 slots x 2 boxes
constexpr int kPOff = kVOff + 4 * kHalf;  // P: 2 boxes
constexpr int kBarOff = kPOff + 2 * kHalf;
constexpr int kRedOff = kBarOff + 256;     // per-row partial maxima / sums of the two column halves
constexpr int kSmem = kRedOff + 2 * 128 * 4 + 1024;
constexpr uint32_t kIdescS = idesc_f16_f32(128, kKeys);
constexpr uint32_t kIdescPV = idesc_f16_f32_bmn(128, kHD);
constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O [256,384)
constexpr float kRescaleLog2 = 8.0f;

enum { B_QFULL0, B_QFULL1, B_QEMPTY0, B_QEMPTY1, B_KVFULL0, B_KVFULL1, B_KVEMPTY0, B_KVEMPTY1, B_SFULL0,
       B_SFULL1, B_SEMPTY0, B_SEMPTY1, B_PFULL, B_PEMPTY, B_OFULL, B_DRAIN, B_COUNT };

struct Item {
  int tok0, L, K, kvh, branch, row0, q0, nrows, n_prefix_tiles, n_tiles;
  __device__ int tile_start(int t) const { return t < n_prefix_tiles ? t * kKeys : q0; }
};

template <int G>
__device__ __forceinline__ Item make_item(int4 item, int4 rq, int b) {
  constexpr int R = kSlots / G;
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

// Work-list reader that keeps the descriptors of the next two items in
// flight, so a role never waits on global memory at an item boundary.
template <int G>
struct ItemStream {
  const int4* items;
  const int4* reqs;
  int n, step, b;
  int it;
  int4 d1, d2, r1;  // descriptor of it + step, it + 2 step; request of it + step
  __device__ ItemStream(const PlanHdr* plan, int first, int step_, int b_)
      : items(plan_array<int4>(plan, plan->off_items)), reqs(plan_array<int4>(plan, plan->off_req)),
        n(plan->n_items), step(step_), b(b_), it(first) {
    const int4 z = make_int4(0, 0, 0, 0);
    d1 = it < n ? items[it] : z;
    d2 = it + step < n ? items[it + step] : z;
    r1 = reqs[d1.x];
  }
  __device__ bool valid() const { return it < n; }
  // the current item; advances the prefetch window
  __device__ Item next() {
    const Item m = make_item<G>(d1, r1, b);
    const int4 z = make_int4(0, 0, 0, 0);
    it += step;
    d1 = d2;
    r1 = reqs[d1.x];
    d2 = it + step < n ? items[it + step] : z;
    return m;
  }
};

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
  const int b = plan->branch_len;
  constexpr int R = kSlots / G;

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    for (int i = 0; i < B_COUNT; ++i) {
      const uint32_t cnt = (i == B_SEMPTY0 || i == B_SEMPTY1 || i == B_PFULL) ? (uint32_t)kSoftmax : 1u;
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

  // Every role walks the same items and tiles, so the running counts below
  // (items, KV tiles, S buffers, P buffers) agree across roles and give each
  // barrier's phase.  Roles run ahead of each other across item boundaries.
  if (warp == 0) {
    // ---- TMA producer
    if (lane == 0) {
      uint32_t n_kv = 0, n_item = 0;
      for (ItemStream<G> is(plan, blockIdx.x, gridDim.x, b); is.valid(); ++n_item) {
        const Item m = is.next();
        const uint32_t qs = n_item & 1, quse = n_item >> 1;
        if (!mbar_wait(bar(B_QEMPTY0 + qs), (quse & 1u) ^ 1u, st, 40)) break;
        mbar_arrive_expect_tx(bar(B_QFULL0 + qs), 2 * kHalf);
        for (int h = 0; h < 2; ++h)
          tma_load_3d(&tmQ, sbase + kQOff + (2 * qs + h) * kHalf, bar(B_QFULL0 + qs), h * 64, m.kvh * G,
                      m.tok0 + m.q0);
        bool ok = true;
        for (int t = 0; t < m.n_tiles; ++t, ++n_kv) {
          const uint32_t slot = n_kv & 1, use = n_kv >> 1;
          if (!mbar_wait(bar(B_KVEMPTY0 + slot), (use & 1u) ^ 1u, st, 41)) {
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
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      uint32_t n_kv = 0, n_s = 0, n_p = 0, n_item = 0;
      bool ok = true;
      for (ItemStream<G> is(plan, blockIdx.x, gridDim.x, b); is.valid() && ok; ++n_item) {
        const Item m = is.next();
        const uint32_t qs = n_item & 1, quse = n_item >> 1;
        if (!mbar_wait(bar(B_QFULL0 + qs), quse & 1u, st, 43)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Issue S = QK^T of tile s_next and P V of tile pv_next in whatever
        // order their inputs become ready (K/V tile landed and an S buffer
        // free, or the softmax's P written), so neither waits on the other.
        auto issue_s = [&](int t) {
          const uint32_t slot = (n_kv + t) & 1;
          const uint32_t sb = (n_s + t) & 1;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kHD / 16; ++k) {
            const uint64_t da = smem_desc_sw128(sbase + kQOff + (2 * qs + (k >> 2)) * kHalf + (k & 3) * 32);
            const uint64_t db = smem_desc_sw128(sbase + kKOff + (2 * slot + (k >> 2)) * kHalf + (k & 3) * 32);
            tc_mma_f16(tmem + sb * kKeys, da, db, kIdescS, k > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_SFULL0 + sb));
          if (t == m.n_tiles - 1) tc_commit(bar(B_QEMPTY0 + qs));  // Q slot free once these S are done
        };
        auto issue_pv = [&](int t) {
          const uint32_t slot = (n_kv + t) & 1;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kKeys / 16; ++k) {
            const uint64_t da = smem_desc_sw128(sbase + kPOff + (k >> 2) * kHalf + (k & 3) * 32);
            const uint64_t db = smem_desc_sw128_mn(sbase + kVOff + 2 * slot * kHalf + k * 2048, kHalf);
            tc_mma_f16(tmemO, da, db, kIdescPV, (t > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(bar(B_KVEMPTY0 + slot));
          tc_commit(bar(B_PEMPTY));
        };
        int s_next = 0, pv_next = 0;
        const uint64_t t0 = global_ns();
        uint32_t spins = 0;
        while (pv_next < m.n_tiles) {
          bool progressed = false;
          // S of the next tile: its K/V landed and its S buffer is free (the
          // softmax is done with the tile two back); never more than one S
          // ahead of the oldest P V not yet issued
          if (s_next < m.n_tiles && s_next <= pv_next + 1) {
            const uint32_t kuse = (n_kv + s_next) >> 1, suse = (n_s + s_next) >> 1;
            if (mbar_try_wait(bar(B_KVFULL0 + ((n_kv + s_next) & 1)), kuse & 1u) &&
                mbar_try_wait(bar(B_SEMPTY0 + ((n_s + s_next) & 1)), (suse & 1u) ^ 1u)) {
              issue_s(s_next++);
              progressed = true;
            }
          }
          if (pv_next < s_next && mbar_try_wait(bar(B_PFULL), (n_p + pv_next) & 1u)) {
            issue_pv(pv_next++);
            progressed = true;
          }
          if (!progressed && (++spins & 255u) == 0 && global_ns() - t0 > kWaitLimitNs) {
            raise_error(st, ERR_WAIT_TIMEOUT, 44);
            ok = false;
            break;
          }
        }
        if (ok) tc_commit(bar(B_OFULL));
        n_kv += m.n_tiles;
        n_s += m.n_tiles;
        n_p += m.n_tiles;
      }
      // no tensor-core operation of this CTA may outlive its TMEM
      tc_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, st, 46);
    }
  } else {
    // ---- softmax: thread = (slot row r = TMEM lane, column half ch); the two
    // threads of a row exchange partial maxima (and at the end the sums)
    // through shared memory
    const int q4 = warp & 3;
    const int ch = (warp - 2) >> 2;  // 0: keys / dims [0, 64), 1: [64, 128)
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + kRedOff);  // [2][128]
    // Barrier over the softmax threads that also ANDs a flag across them, so
    // that a failed (timed-out) wait stops all eight warps together and none
    // is left at a named barrier.
    auto softmax_all = [](bool v) -> bool {
      uint32_t res;
      asm volatile(
          "{ .reg .pred pin, pout; setp.ne.u32 pin, %1, 0; bar.red.and.pred pout, 1, %2, pin; "
          "selp.u32 %0, 1, 0, pout; }"
          : "=r"(res)
          : "r"(v ? 1u : 0u), "n"(kSoftmax)
          : "memory");
      return res != 0;
    };
    uint32_t n_s = 0, n_p = 0, n_item = 0;
    bool ok = true;
    for (ItemStream<G> is(plan, blockIdx.x, gridDim.x, b); is.valid() && ok; ++n_item) {
      const Item m = is.next();
      const KeyRange kr = tree_keys(m.q0 + r / G, m.L, b);
      float m_used = -INFINITY, l = 0.f;
      for (int t = 0; t < m.n_tiles && ok; ++t) {
        const uint32_t sb = (n_s + t) & 1, suse = (n_s + t) >> 1;
        if (!softmax_all(mbar_wait_warp(bar(B_SFULL0 + sb), suse & 1u, st, 47))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int k0 = m.tile_start(t) + 64 * ch;
        const bool is_branch_tile = m.branch && t == m.n_prefix_tiles;
        const bool need_mask = is_branch_tile || (!m.branch && m.tile_start(t) + kKeys > m.row0) ||
                               (m.branch && m.tile_start(t) + kKeys > m.L);
        const uint32_t s_addr = tmem + lane_off + sb * kKeys + 64 * ch;
        // this thread's 64 S values: two loads, one wait
        uint32_t sr[2][32];
#pragma unroll
        for (int q = 0; q < 2; ++q) tmem_ld32_async(s_addr + 32 * q, sr[q]);
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < 2; ++q)
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
        // S buffer consumed: the MMA may refill it
        tc_fence_before();
        mbar_arrive(bar(B_SEMPTY0 + sb));
        // row max over both halves; the barrier that publishes the partial
        // maxima also confirms the P buffer is free and O complete for the
        // previous tile (the next tile's writes of red[] come after its first
        // barrier, which every thread reaches only after reading red[] here)
        red[ch * 128 + r] = mx;
        if (!softmax_all(mbar_wait_warp(bar(B_PEMPTY), ((n_p + t) & 1u) ^ 1u, st, 48))) {
          ok = false;
          break;
        }
        mx = fmaxf(mx, red[(ch ^ 1) * 128 + r]);
        tc_fence_after();
        const float m_new = fmaxf(m_used, mx);
        // the O rescale uses warp-collective TMEM loads and stores: decide it
        // for the whole warp (both warps of a row group see the same maxima,
        // so they decide alike; a row that did not need it is rescaled to its
        // new max as well, which is just as exact)
        if (t == 0) {
          m_used = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m_used + kRescaleLog2)) {
          const float corr = m_new == m_used ? 1.f : fast_exp2(m_used - m_new);  // 0 while nothing was visible
#pragma unroll 1
          for (int c = 64 * ch; c < 64 * ch + 64; c += 32) {
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
        // P = 2^(s - mu) in fp16 into this half's K-major 128-byte-swizzled box
        float sum = 0.f;
        const uint32_t pbox = sbase + kPOff + ch * kHalf + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float p0 = fast_exp2(__uint_as_float(sr[q][j]) - mu);
            const float p1 = fast_exp2(__uint_as_float(sr[q][j + 1]) - mu);
            sum += p0 + p1;
            const __half2 h = __floats2half2_rn(p0, p1);
            pk[j / 2] = *reinterpret_cast<const uint32_t*>(&h);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int chunk = q * 4 + u;
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(pbox + ((chunk ^ (r & 7)) << 4)),
                         "r"(pk[4 * u]), "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]), "r"(pk[4 * u + 3])
                         : "memory");
          }
        }
        l += sum;
        tc_fence_before();
        fence_proxy_async_smem();
        mbar_arrive(bar(B_PFULL));
      }
      // ---- epilogue: O / l -> fp16, this thread's 64 dims (O is
      // overwritten only after the next item's first P, which these warps
      // release after this read)
      if (!ok) break;
      // (this barrier also orders the partner's read of the last partial
      // max before the sum overwrites it)
      if (!softmax_all(mbar_wait_warp(bar(B_OFULL), n_item & 1u, st, 49))) {
        ok = false;
        break;
      }
      tc_fence_after();
      red[ch * 128 + r] = l;
      asm volatile("bar.sync 1, %0;" ::"n"(kSoftmax) : "memory");
      l += red[(ch ^ 1) * 128 + r];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int rl = r / G;
      const bool valid = rl < m.nrows;
      __half* dst = o + (((int64_t)m.tok0 + m.q0 + rl) * n_q_heads + m.kvh * G + (r % G)) * kHD;
#pragma unroll 1
      for (int c = 64 * ch; c < 64 * ch + 64; c += 32) {
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
      n_s += m.n_tiles;
      n_p += m.n_tiles;
    }
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
