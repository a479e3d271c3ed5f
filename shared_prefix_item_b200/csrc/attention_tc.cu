// Shared-prefix, tree-masked attention on 5th-generation tensor cores.
//
// DuoLM summary page (paper.rainbus.top), 方法步骤详情 step 4 and 研究动机:
// the prefix of a request is computed once and its K/V are shared by all K
// candidate branches; candidate j attends to the prefix and to its own branch
// only.  Work is cut into items of one request and one KV head.  An item holds
// two sub-tiles A and B of 128 query slots each (a slot is a (token, query
// head of the KV head's group) pair: 64 tokens x 2 heads per sub-tile for
// Qwen3's grouping), and every K/V tile the item loads serves both:
//   kind 0  prefix tokens [row0, row0 + 2R): causal over the prefix;
//   kind 1  branch tokens (whole candidates): every prefix key tile, then the
//           tiles of the item's own branch rows under the tree rule.
// B is left out when the item's rows all fit in A; a batch too small to
// give half the CTAs an item (one or two requests) is planned with items of
// one sub-tile (the plan's att_rows), so that twice as many CTAs take part.
// A request may continue a cached prefix (incremental history append): its
// first c prefix tokens were computed by an earlier call and their K/V sit
// in a slot of the per-layer KV store; the batch holds only the tokens after
// them.  Request-local indices still count from the first cached token, so
// masks and positions are those of the whole sequence: key tiles
// [0, ceil(c / 128)) come from the store (keys >= c masked), the remaining
// prefix tiles start at c and come from this batch's K/V, and query rows
// start at c.  With c = 0 the item is exactly the uncached one.
// One CTA per SM, 384
// threads in three warpgroups:
//   warps 0-3 softmax of A, warps 4-7 softmax of B: one thread per slot row
//             (TMEM lane) and 128 keys: load S, mask, row max, P = 2^(s - m)
//             as fp16 written back over S in tensor memory, row sum; O_X is
//             rescaled only when the running max grows by more than 2^8 (P
//             stays below 256, exact after the final division); at the end of
//             an item O_X / l to global memory;
//   warp 8    TMA: Q of A and B (3-D map, 32 KB each), K and V tiles of 128
//             keys (32 KB each, two slots each, separate barriers so a K tile
//             can land while the previous V is still in use); 128-byte
//             swizzle, no multicast;
//   warp 9    one lane issues tcgen05.mma, per key tile and per sub-tile X:
//             O_X (+)= P_X V of the previous tile (P read from tensor
//             memory), then S_X = Q_X K^T of this tile into the same columns;
//   warps 10-11 idle.
// The softmax warpgroups hold a whole 128-key row of S in registers: they
// take registers from the third warpgroup (setmaxnreg; 2 x 128 x kRegSoftmax
// + 128 x kRegOther is exactly the launch's 384 x 168).
// Tensor memory: S/P of A in columns [0, 128), of B in [128, 256), O of A in
// [256, 384), O of B in [384, 512).  tcgen05.mma operations issued by one
// thread run in issue order, so S_X of a tile may be issued right after the
// P V that reads the same columns, and the commit that reports S_X complete
// also reports the preceding P V complete (O_X current for a rescale).
// Every mbarrier wait is bounded; after a timeout the kernel raises the status
// flag and returns.
#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

namespace {

constexpr int kSub = 128;   // query slots per sub-tile (MMA M)
constexpr int kKeys = 128;  // keys per tile (MMA N of Q K^T)
constexpr int kHD = 128;
constexpr int kSoftmaxWG = 128;  // threads of one softmax warpgroup
constexpr int kThreads = 3 * kSoftmaxWG;
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr int kRegLaunch = 168;  // 65536 / 384 rounded down to a multiple of 8
constexpr int kRegSoftmax = 200, kRegOther = 104;
static_assert(2 * kSoftmaxWG * kRegSoftmax + kSoftmaxWG * kRegOther <= kThreads * kRegLaunch,
              "register split above the launch's registers");
constexpr int kHalf = 16384;         // one 128-row x 64-element fp16 box
constexpr int kQOff = 0;             // Q: 2 sub-tiles x 2 boxes
constexpr int kKOff = 4 * kHalf;     // K: 2 slots x 2 boxes
constexpr int kVOff = 8 * kHalf;     // V: 2 slots x 2 boxes
constexpr int kBarOff = 12 * kHalf;
constexpr int kSmem = kBarOff + 256 + 1024;
constexpr uint32_t kIdescS = idesc_f16_f32(kSub, kKeys);
constexpr uint32_t kIdescPV = idesc_f16_f32_bmn(kSub, kHD);
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

enum { B_QFULL0, B_QFULL1, B_QEMPTY0, B_QEMPTY1, B_KFULL0, B_KFULL1, B_VFULL0, B_VFULL1, B_KEMPTY0, B_KEMPTY1,
       B_VEMPTY0, B_VEMPTY1, B_SFULL0, B_SFULL1, B_PFULL0, B_PFULL1, B_OFULL0, B_OFULL1, B_DRAIN, B_COUNT };

struct Item {
  // qbase: batch row of request-local index 0 (the first cached token's
  // index; batch rows hold only indices >= c); slot0: the request's first
  // store row; tiles [0, n_cached_tiles) are store tiles
  int qbase, c, slot0, L, K, kvh, branch, row0, q0, nrows, n_cached_tiles, n_prefix_tiles, n_tiles, has_b;
  __device__ int tile_start(int t) const {
    return t < n_cached_tiles ? t * kKeys
                              : (t < n_prefix_tiles ? c + (t - n_cached_tiles) * kKeys
                                                    : q0 + (t - n_prefix_tiles) * kKeys);
  }
};

// R2: tokens per item, 2R (two sub-tiles) or R (one, for small batches)
template <int G>
__device__ __forceinline__ Item make_item(int4 item, int4 rq, int2 rx, int b, int R2) {
  constexpr int R = kSub / G;  // tokens per sub-tile
  Item m;
  m.c = rx.x;
  m.slot0 = rx.y;
  m.qbase = rq.x - rx.x;
  m.L = rq.y;
  m.K = rq.z;
  m.kvh = item.y;
  m.branch = item.z;
  m.row0 = item.w;
  m.q0 = m.branch ? m.L + m.row0 : m.row0;
  m.nrows = m.branch ? min((R2 / b) * b, m.K * b - m.row0) : min(R2, m.L - m.row0);
  const int kend = m.branch ? m.L : min(m.row0 + R2, m.L);
  m.n_cached_tiles = (m.c + kKeys - 1) / kKeys;
  m.n_prefix_tiles = m.n_cached_tiles + (kend - m.c + kKeys - 1) / kKeys;
  m.n_tiles = m.n_prefix_tiles + (m.branch ? (m.nrows + kKeys - 1) / kKeys : 0);
  m.has_b = m.nrows > R;
  return m;
}

// Work-list reader that keeps the descriptors of the next two items in
// flight, so a role never waits on global memory at an item boundary.  A
// CTA runs the contiguous range of the work list the plan gives it (the
// host's load-balanced schedule), or, for a plan divided among a different
// number of CTAs, every gridDim.x-th item.
template <int G>
struct ItemStream {
  const int4* items;
  const int4* reqs;
  const int2* reqx;
  int n, step, b;
  int rows;  // tokens per item
  int it;
  int4 d1, d2, r1;  // descriptor of it + step, it + 2 step; request of it + step
  int2 x1;          // cached prefix of that request
  __device__ ItemStream(const PlanHdr* plan, const int2* reqx_, int cta, int n_ctas, int b_)
      : items(plan_array<int4>(plan, plan->off_items)), reqs(plan_array<int4>(plan, plan->off_req)), reqx(reqx_),
        b(b_), rows(plan->att_rows == kSub / G ? kSub / G : 2 * kSub / G) {
    if (plan->att_ctas == n_ctas) {
      const int32_t* off = plan_array<int32_t>(plan, plan->off_cta);
      it = off[cta];
      n = off[cta + 1];
      step = 1;
    } else {
      it = cta;
      n = plan->n_items;
      step = n_ctas;
    }
    const int4 z = make_int4(0, 0, 0, 0);
    d1 = it < n ? items[it] : z;
    d2 = it + step < n ? items[it + step] : z;
    r1 = reqs[d1.x];
    x1 = reqx[d1.x];
  }
  __device__ bool valid() const { return it < n; }
  // the current item; advances the prefetch window
  __device__ Item next() {
    const Item m = make_item<G>(d1, r1, x1, b, rows);
    const int4 z = make_int4(0, 0, 0, 0);
    it += step;
    d1 = d2;
    r1 = reqs[d1.x];
    x1 = reqx[d1.x];
    d2 = it + step < n ? items[it + step] : z;
    return m;
  }
};

// Packed fp32 pairs (Blackwell's f32x2 forms: one instruction does the work
// of two) and the three-input maximum, for the softmax's per-element work.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

}  // namespace

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKs,
                        const __grid_constant__ CUtensorMap tmVs, const PlanHdr* __restrict__ plan,
                        const int2* __restrict__ reqx, int64_t kv_rows, int64_t store_rows, int n_q_heads,
                        float scale_log2, __half* __restrict__ o, DevStatus* st) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + B_COUNT);

  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = plan->branch_len;
  constexpr int R = kSub / G;

  if (warp == kWarpTma && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    prefetch_tensormap(&tmKs);
    prefetch_tensormap(&tmVs);
    for (int i = 0; i < B_COUNT; ++i)
      mbar_init(bar(i), (i == B_PFULL0 || i == B_PFULL1) ? (uint32_t)kSoftmaxWG : 1u);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // everything below reads what the previous kernels wrote; a bounded wait
  // that already gave up in an earlier launch makes the CTA skip its work
  pdl_wait();
  const bool skip = (*reinterpret_cast<volatile const uint32_t*>(&st->flags) & ERR_WAIT_TIMEOUT) != 0;

  // Every role walks the same items and tiles, so the running counts below
  // (K/V tiles, and per sub-tile its items and tiles) agree across roles and
  // give each barrier's phase.
  if (skip) {
    // nothing to do: straight to the teardown
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
    // ---- softmax of sub-tile X: thread = slot row r = TMEM lane
    const int X = warp >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128 * X, tO = tmem + lane_off + 256 + 128 * X;
    uint32_t n_xt = 0, n_xi = 0;
    bool ok = true;
    for (ItemStream<G> is(plan, reqx, blockIdx.x, gridDim.x, b); is.valid() && ok;) {
      const Item m = is.next();
      if (X == 1 && !m.has_b) continue;
      const int rl = X * R + r / G;  // row of the item (token offset from q0)
      const KeyRange kr = tree_keys(m.q0 + rl, m.L, b);
      float m_used = -INFINITY, l = 0.f;
      for (int t = 0; t < m.n_tiles; ++t, ++n_xt) {
        if (!mbar_wait_warp(bar(B_SFULL0 + X), n_xt & 1u, st, 48)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32_async(tS + 32 * c, sr[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) tmem_ld_fence(sr[c][j]);
        const int k0 = m.tile_start(t);
        const bool is_branch_tile = t >= m.n_prefix_tiles;
        const bool is_cached_tile = t < m.n_cached_tiles;
        const bool need_mask = is_branch_tile || (is_cached_tile && k0 + kKeys > m.c) ||
                               (!is_cached_tile && ((!m.branch && k0 + kKeys > m.row0) || (m.branch && k0 + kKeys > m.L)));
        if (need_mask) {
          // this row's visible keys in the tile are one window [lo0, lo0 + n)
          // of tile-local indices: its own branch keys in a branch tile, the
          // cached keys (all below every query row) in a store tile, the
          // prefix keys up to pre_hi otherwise
          const int lo = is_branch_tile ? kr.br_lo - k0 : 0;
          const int hi = (is_branch_tile ? kr.br_hi : (is_cached_tile ? m.c - 1 : kr.pre_hi)) - k0;  // inclusive
          const uint32_t lo0 = (uint32_t)max(lo, 0);
          const uint32_t n = (uint32_t)max(0, min(hi, kKeys - 1) - max(lo, 0) + 1);
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if ((uint32_t)(32 * c + j) - lo0 >= n) sr[c][j] = __float_as_uint(-INFINITY);
        }
        // row max of the raw scores (the scale is positive: applied after)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; j += 2)
            mx[(j >> 1) & 3] = fmax3f(mx[(j >> 1) & 3], __uint_as_float(sr[c][j]), __uint_as_float(sr[c][j + 1]));
        const float m_new = fmaxf(m_used, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale_log2);
        // the O rescale uses warp-collective TMEM loads and stores: decide it
        // for the whole warp (a row that did not need it is rescaled to its
        // new max as well, which is just as exact)
        if (t == 0) {
          m_used = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m_used + kRescaleLog2)) {
          const float corr = m_new == m_used ? 1.f : fast_exp2(m_used - m_new);  // 0 while nothing was visible
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tmem_ld32(tO + 32 * c, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= corr;
            tmem_st32(tO + 32 * c, v);
          }
          l *= corr;
          m_used = m_new;
        }
        const float nmu = m_used == -INFINITY ? 0.f : -m_used;
        // P = 2^(s scale - m) in fp16 over the first 64 columns of S (the
        // scaling and the row sum on packed pairs)
        const float2 sv = make_float2(scale_log2, scale_log2), nv = make_float2(nmu, nmu);
        float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const float2 x =
                ffma2(make_float2(__uint_as_float(sr[c][2 * jj]), __uint_as_float(sr[c][2 * jj + 1])), sv, nv);
            const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            ls2[jj & 1] = fadd2(ls2[jj & 1], p);
            pk[jj] = pack_half2(p.x, p.y);
          }
          tmem_st16_async(tS + 16 * c, pk);
        }
        l += (ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL0 + X));
      }
      if (!ok) break;
      // ---- end of the item: O_X / l -> fp16, this thread's row (O_X is
      // overwritten only by the P V of the next item's first P, which this
      // thread releases after this read)
      if (!mbar_wait_warp(bar(B_OFULL0 + X), n_xi & 1u, st, 49)) {
        ok = false;
        break;
      }
      tc_fence_after();
      ++n_xi;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool valid = rl < m.nrows;
      __half* dst = o + (((int64_t)m.qbase + m.q0 + rl) * n_q_heads + m.kvh * G + (r % G)) * kHD;
      {
        // all 128 columns in one batch of TMEM loads (the S registers are
        // free by now), then the row out in 32-byte stores (one full sector
        // each)
        uint32_t ov[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32_async(tO + 32 * c, ov[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) tmem_ld_fence(ov[c][j]);
        if (valid) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                w[j] = pack_half2(__uint_as_float(ov[c][16 * h + 2 * j]) * inv,
                                  __uint_as_float(ov[c][16 * h + 2 * j + 1]) * inv);
              st_global_v8(dst + 32 * c + 16 * h, w);
            }
        }
      }
      tc_fence_before();
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegOther));
    if (warp == kWarpTma) {
      // ---- TMA producer
      if (lane == 0) {
        uint32_t n_kv = 0, n_xi[2] = {0, 0};
        bool ok = true;
        for (ItemStream<G> is(plan, reqx, blockIdx.x, gridDim.x, b); is.valid() && ok;) {
          const Item m = is.next();
#pragma unroll
          for (int X = 0; X < 2; ++X) {
            if (X > m.has_b) break;
            if (!mbar_wait(bar(B_QEMPTY0 + X), (n_xi[X] & 1u) ^ 1u, st, 40)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(B_QFULL0 + X), 2 * kHalf);
            for (int h = 0; h < 2; ++h)
              tma_load_3d(&tmQ, sbase + kQOff + (2 * X + h) * kHalf, bar(B_QFULL0 + X), h * 64, m.kvh * G,
                          m.qbase + m.q0 + X * R);
            ++n_xi[X];
          }
          for (int t = 0; t < m.n_tiles && ok; ++t, ++n_kv) {
            const uint32_t slot = n_kv & 1, use = n_kv >> 1;
            // a store tile reads the request's slot, every other tile this batch's K/V
            const bool cached = t < m.n_cached_tiles;
            const CUtensorMap* mk = cached ? &tmKs : &tmK;
            const CUtensorMap* mv = cached ? &tmVs : &tmV;
            const int y = cached ? (int)((int64_t)m.kvh * store_rows + m.slot0 + m.tile_start(t))
                                 : (int)((int64_t)m.kvh * kv_rows + m.qbase + m.tile_start(t));
            if (!mbar_wait(bar(B_KEMPTY0 + slot), (use & 1u) ^ 1u, st, 41)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(B_KFULL0 + slot), 2 * kHalf);
            for (int h = 0; h < 2; ++h)
              tma_load_2d(mk, sbase + kKOff + (2 * slot + h) * kHalf, bar(B_KFULL0 + slot), h * 64, y);
            if (!mbar_wait(bar(B_VEMPTY0 + slot), (use & 1u) ^ 1u, st, 42)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(B_VFULL0 + slot), 2 * kHalf);
            for (int h = 0; h < 2; ++h)
              tma_load_2d(mv, sbase + kVOff + (2 * slot + h) * kHalf, bar(B_VFULL0 + slot), h * 64, y);
          }
        }
        if (!ok) {
          // leave no copy in flight into shared memory this CTA is giving up:
          // wait (bounded) for the last phase armed on every full barrier
#pragma unroll
          for (int X = 0; X < 2; ++X)
            if (n_xi[X] > 0) mbar_wait(bar(B_QFULL0 + X), (n_xi[X] - 1) & 1u, st, 50);
          for (uint32_t k = n_kv > 2 ? n_kv - 2 : 0; k < n_kv; ++k) {
            mbar_wait(bar(B_KFULL0 + (k & 1)), (k >> 1) & 1u, st, 50);
            mbar_wait(bar(B_VFULL0 + (k & 1)), (k >> 1) & 1u, st, 50);
          }
        }
      }
    } else if (warp == kWarpMma) {
      // ---- MMA issuer
      if (lane == 0) {
        // (all state in named registers: runtime-indexed arrays would sit in
        // local memory, and this thread's instruction path bounds the step)
        struct Pending {  // P V of a sub-tile's tile, issued at the next tile
          int valid, first, last, release_v;
          uint32_t slot, use, xt;
        };
        Pending pa{}, pb{};
        uint32_t n_kv = 0, xt_a = 0, xt_b = 0, xi_a = 0, xi_b = 0;
        bool ok = true;
        auto issue_pv = [&](int X, Pending& p) -> bool {
          if (!mbar_wait(bar(B_PFULL0 + X), p.xt & 1u, st, 43)) return false;
          if (!mbar_wait(bar(B_VFULL0 + p.slot), p.use & 1u, st, 44)) return false;
          tc_fence_after();
          const uint32_t tS = tmem + 128 * X, tO = tmem + 256 + 128 * X;
          const uint32_t vbase = sbase + kVOff + 2 * p.slot * kHalf;
#pragma unroll
          for (int k = 0; k < kKeys / 16; ++k)
            tc_mma_f16_ts(tO, tS + 8 * k, smem_desc_sw128_mn(vbase + k * 2048, kHalf), kIdescPV,
                          (p.first && k == 0) ? 0u : 1u);
          if (p.last) tc_commit(bar(B_OFULL0 + X));
          if (p.release_v) tc_commit(bar(B_VEMPTY0 + p.slot));
          p.valid = 0;
          return true;
        };
        for (ItemStream<G> is(plan, reqx, blockIdx.x, gridDim.x, b); is.valid() && ok;) {
          const Item m = is.next();
          const int nx = 1 + m.has_b;
          for (int t = 0; t < m.n_tiles && ok; ++t, ++n_kv) {
            const uint32_t slot = n_kv & 1, use = n_kv >> 1;
            const bool last = t == m.n_tiles - 1;
            const uint32_t kbase = sbase + kKOff + 2 * slot * kHalf;
#pragma unroll
            for (int X = 0; X < 2; ++X) {
              Pending& p = X == 0 ? pa : pb;
              // P V of this sub-tile's previous tile first: S of this tile
              // overwrites the P it reads
              if (p.valid && !issue_pv(X, p)) {
                ok = false;
                break;
              }
              if (X >= nx) continue;
              uint32_t& xi = X == 0 ? xi_a : xi_b;
              uint32_t& xt = X == 0 ? xt_a : xt_b;
              if (t == 0 && !mbar_wait(bar(B_QFULL0 + X), xi & 1u, st, 45)) {
                ok = false;
                break;
              }
              if (X == 0 && !mbar_wait(bar(B_KFULL0 + slot), use & 1u, st, 46)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t qbase = sbase + kQOff + 2 * X * kHalf;
#pragma unroll
              for (int k = 0; k < kHD / 16; ++k)
                tc_mma_f16(tmem + 128 * X, smem_desc_sw128(qbase + (k >> 2) * kHalf + (k & 3) * 32),
                           smem_desc_sw128(kbase + (k >> 2) * kHalf + (k & 3) * 32), kIdescS, k > 0 ? 1u : 0u);
              tc_commit(bar(B_SFULL0 + X));
              if (last) {
                tc_commit(bar(B_QEMPTY0 + X));  // Q_X free once these S are done
                ++xi;
              }
              p = Pending{1, t == 0, last, X == nx - 1, slot, use, xt};
              ++xt;
            }
            if (ok) tc_commit(bar(B_KEMPTY0 + slot));  // both S of this tile issued
          }
        }
        if (ok && pa.valid && !issue_pv(0, pa)) ok = false;
        if (ok && pb.valid && !issue_pv(1, pb)) ok = false;
        // no tensor-core operation of this CTA may outlive its TMEM
        tc_commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0, st, 47);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

int attention_tc_rows_per_item(int group) { return 2 * kSub / group; }

cudaError_t attention_tc_setup() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(attention_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem)))
    return e;
  if ((e = cudaFuncSetAttribute(attention_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem)))
    return e;
  return cudaFuncSetAttribute(attention_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
}

cudaError_t attention_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tks,
                         const CUtensorMap& tvs, const PlanHdr* plan, const int2* reqx, int64_t kv_rows,
                         int64_t store_rows, int n_q_heads, int n_kv_heads, float scale, __half* o, DevStatus* st,
                         int grid, cudaStream_t s, bool pdl) {
  const int G = n_q_heads / n_kv_heads;
  const float sl2 = scale * 1.4426950408889634f;  // softmax in base 2
  auto run = [&](auto kernel) {
    return launch_ex(kernel, dim3(grid), dim3(kThreads), kSmem, s, pdl, tq, tk, tv, tks, tvs, plan, reqx, kv_rows,
                     store_rows, n_q_heads, sl2, o, st);
  };
  switch (G) {
    case 1:
      return run(attention_tc_kernel<1>);
    case 2:
      return run(attention_tc_kernel<2>);
    case 4:
      return run(attention_tc_kernel<4>);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace duolm
