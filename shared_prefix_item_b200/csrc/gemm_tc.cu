// Projection GEMMs of the ranker on 5th-generation tensor cores (sm_100a).
//
// C[M, N] = A[M, K] * B[N, K]^T with fp16 operands and fp32 accumulation in
// tensor memory.  Persistent clusters of two CTAs (one per SM), each pair
// computing 256 x BN tiles, warp-specialised per CTA:
//   warp 0      TMA producer: streams this CTA's 128x64 A block and its
//               (BN/2)x64 half of the B block per k-block (128-byte swizzle,
//               no multicast) into a STAGES-deep shared-memory ring, the
//               completions landing on the leader CTA's barriers;
//   warp 1      allocates 2*BN TMEM columns in both CTAs; on the leader,
//               lane 0 issues tcgen05.mma.cta_group::2 (256 x BN x 16 per
//               instruction) and commits to both CTAs' barriers;
//   warps 2..   epilogue, in groups of four warps (one per TMEM lane
//               quadrant): each thread owns one accumulator row and its
//               group's share of the columns, reads them with tcgen05.ld and
//               applies a fused epilogue; most epilogues turn their rows
//               around in a per-warp shared-memory scratch so that global
//               memory is written (and the residual read) in full lines.
// Two accumulator buffers let the epilogue of tile i overlap the mainloop of
// tile i+1.  Every mbarrier wait is bounded (see common.cuh).
#include <cstdio>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

constexpr int kBM = 128;
constexpr int kBK = 64;  // one 128-byte swizzle row of fp16

// A CTA pair (cluster of 2) computes a 256 x BN tile: each CTA loads its 128
// rows of A and its BN/2 rows of B per k-block (32 KB), the leader issues
// the pair MMAs (M = 256), each CTA's TMEM receives its 128 accumulator rows.
// Tiles are visited N-fastest, so the pairs running at the same time share
// an A row block and it is read from DRAM once.
// An epilogue may ask for shared-memory scratch per epilogue warp (then the
// ring is shallower, so the CTA stays near 197 KB of shared memory).
// Narrower QKV tiles (BN 128, one epilogue group) serve small batches,
// where 256-wide tiles leave most CTA pairs without work; their smaller
// stages let the ring hold more k-blocks in the same shared memory.
template <int BN, class Epi>
struct TcCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;        // this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * kBK * 2;   // this CTA's half of the B tile
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT = Epi::STAGES * (kBM * kBK * 2 + 128 * kBK * 2) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFF = EPI_OFF + 4 * Epi::EG * Epi::SCRATCH_PER_WARP;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;    // barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = 2 * BN;        // two accumulator buffers
  static constexpr uint32_t IDESC = idesc_f16_f32(2 * kBM, BN);
};

// ---------------------------------------------------------------------------
// fused epilogues.  EG groups of four warps share each tile: group g handles
// columns [g * BN / EG, (g + 1) * BN / EG) (for QKV, head g of the tile).
// `taddr` addresses this thread's row, column 0 of the tile's accumulator;
// all lanes of a warp execute the TMEM loads.  `scratch` is this warp's
// shared-memory scratch (SCRATCH_PER_WARP bytes).  prefetch() runs before the
// wait for the accumulator and loads what does not depend on it (the input
// row's norm factor, positions, tables); its result is passed to run().
// ---------------------------------------------------------------------------
__device__ __forceinline__ float silu_fast(float g) {
  return __fdividef(g, 1.0f + fast_exp2(-1.4426950408889634f * g));
}

// r = 1 / sqrt(mean(x^2) + eps) of one input row from its partial sums
__device__ __forceinline__ float row_rnorm(const float* ssp, int n_slots, int row, float inv_d, float eps) {
  const float4* p = reinterpret_cast<const float4*>(ssp + (int64_t)row * n_slots);
  float ss = 0.f;
  for (int i = 0; i < n_slots / 4; ++i) {
    const float4 v = p[i];
    ss += v.x;
    ss += v.y;
    ss += v.z;
    ss += v.w;
  }
  return 1.0f / sqrtf(ss * inv_d + eps);
}

// x += scale * acc (the residual stream, fp32) and, for the next norm,
// xg = fp16(x * g_next) with per-64-column partial sums of x^2.  The
// accumulator arrives one row per thread; each warp turns its 32 x 32 block
// around in shared memory so that the residual is read and written a row
// segment of 128 bytes per 8 threads (four full lines per warp access)
// instead of 32 rows per access.
// Warp store of 32 rows x 128 bytes: thread `lane` holds row `lane` as 32
// words; the rows go out through a padded shared-memory scratch (36 words a
// row: 16-byte accesses without bank conflicts) so that eight threads store
// one row's 128 bytes, four full lines per warp access.  dst(r) is the
// 16-byte-aligned destination of row r of the warp, or null to skip it.
constexpr int kScratchPad = 36;
constexpr int kScratchPerWarp = 32 * kScratchPad * 4;
// The second half of that: the scratch already holds the warp's 32 rows.
template <class Dst>
__device__ __forceinline__ void warp_flush_rows_128B(const uint32_t* buf, Dst dst) {
  const int lane = threadIdx.x & 31;
  __syncwarp();  // every lane's writes to the scratch are done
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + (lane >> 3);
    const uint4 w = *reinterpret_cast<const uint4*>(buf + r * kScratchPad + (lane & 7) * 4);
    uint4* p = dst(r);
    if (p) p[lane & 7] = w;
  }
}
template <class Dst>
__device__ __forceinline__ void warp_store_rows_128B(uint32_t* buf, const uint32_t (&v)[32], Dst dst) {
  const int lane = threadIdx.x & 31;
  __syncwarp();  // earlier reads of the scratch are done
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4*>(buf + lane * kScratchPad + 4 * q) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  warp_flush_rows_128B(buf, dst);
}

template <int EG_>
struct EpiResidT {
  EpiResidArgs a;
  static constexpr int EG = EG_;
  static constexpr int STAGES = 5;
  static constexpr int kPad = kScratchPad;
  static constexpr int SCRATCH_PER_WARP = kScratchPerWarp;
  struct Pre {};
  template <int BN>
  __device__ __forceinline__ Pre prefetch(int, int, int, bool, const PlanHdr*, DevStatus*) const {
    return Pre{};
  }
  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int row, int n0, int g, bool, const PlanHdr*, DevStatus* st,
                                      uint8_t* scratch, int M, const Pre&, int) const {
    constexpr int W = BN / EG;
    static_assert(W % 64 == 0, "a group covers whole 64-column norm slots");
    const int lane = threadIdx.x & 31;
    const int row0 = row - lane;      // the warp's first row
    const int cq = (lane & 7) * 4;    // this thread's 4 columns of a 32-column chunk
    const int rsub = lane >> 3;       // and its rows row0 + 4 i + rsub, i = 0..7
    float* buf = reinterpret_cast<float*>(scratch);
    float ss[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) ss[i] = 0.f;
#pragma unroll 1
    for (int c = g * W; c < (g + 1) * W; c += 32) {
      // residual block: rows row0 + 4 i + rsub, columns c + cq .. + 3 (the
      // loads do not depend on the accumulator: issue them first)
      float4 xr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = row0 + 4 * i + rsub;
        xr[i] = rr < M ? *reinterpret_cast<const float4*>(a.x + (int64_t)rr * a.ldx + n0 + c + cq)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      uint32_t vr[32];
      tmem_ld32_async(taddr + c, vr);
      tmem_wait_ld();
      __syncwarp();  // the previous chunk's reads of the scratch are done
#pragma unroll
      for (int q = 0; q < 8; ++q) {
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld_fence(vr[4 * q + j]);
        *reinterpret_cast<float4*>(buf + lane * kPad + 4 * q) =
            make_float4(__uint_as_float(vr[4 * q]), __uint_as_float(vr[4 * q + 1]), __uint_as_float(vr[4 * q + 2]),
                        __uint_as_float(vr[4 * q + 3]));
      }
      __syncwarp();
      float4 gn = make_float4(0.f, 0.f, 0.f, 0.f);
      if (a.xg) gn = *reinterpret_cast<const float4*>(a.g_next + n0 + c + cq);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rl = 4 * i + rsub;
        const int rr = row0 + rl;
        const float4 acc = *reinterpret_cast<const float4*>(buf + rl * kPad + cq);
        float4 t = xr[i];
        t.x += acc.x * a.scale;
        t.y += acc.y * a.scale;
        t.z += acc.z * a.scale;
        t.w += acc.w * a.scale;
        if (rr < M) {
          *reinterpret_cast<float4*>(a.x + (int64_t)rr * a.ldx + n0 + c + cq) = t;
          if (a.xg) {
            ss[i] += t.x * t.x + t.y * t.y + t.z * t.z + t.w * t.w;
            const __half2 h0 = __halves2half2(to_half_checked(t.x * gn.x, st, 23), to_half_checked(t.y * gn.y, st, 23));
            const __half2 h1 = __halves2half2(to_half_checked(t.z * gn.z, st, 23), to_half_checked(t.w * gn.w, st, 23));
            *reinterpret_cast<uint2*>(a.xg + (int64_t)rr * a.ldx + n0 + c + cq) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
          }
        }
      }
      if (a.xg && (c & 63) == 32) {
        // a 64-column slot is complete: sum each row over its 8 threads
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v = ss[i];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          const int rr = row0 + 4 * i + rsub;
          if ((lane & 7) == 0 && rr < M) a.ssp[(int64_t)rr * a.n_slots + (n0 + c) / 64] = v;
          ss[i] = 0.f;
        }
      }
    }
  }
};

struct EpiSwiglu {
  EpiSwigluArgs a;
  static constexpr int EG = 2;
  static constexpr int STAGES = 5;
  static constexpr int SCRATCH_PER_WARP = kScratchPerWarp;
  struct Pre {
    float sc;  // weight scale times the input row's RMSNorm factor
  };
  template <int BN>
  __device__ __forceinline__ Pre prefetch(int row, int, int, bool row_ok, const PlanHdr*, DevStatus*) const {
    return Pre{row_ok ? a.scale * row_rnorm(a.ssp, a.n_slots, row, a.inv_d, a.eps) : 0.f};
  }
  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int row, int n0, int g, bool row_ok, const PlanHdr*,
                                      DevStatus* st, uint8_t* scratch, int M, const Pre& pre, int) const {
    constexpr int H = BN / 2;   // gate columns [0, H), up columns [H, BN)
    constexpr int W = H / EG;   // outputs of this group: one 128-byte fp16 row segment
    static_assert(W == 64, "one warp store per group");
    const int out0 = n0 / 2 + g * W;
    const float sc = pre.sc;
    uint32_t packed[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int c = g * W + 32 * half;
      uint32_t gr[32], ur[32];
      tmem_ld32_async(taddr + c, gr);
      tmem_ld32_async(taddr + H + c, ur);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        tmem_ld_fence(gr[2 * j]);
        tmem_ld_fence(gr[2 * j + 1]);
        tmem_ld_fence(ur[2 * j]);
        tmem_ld_fence(ur[2 * j + 1]);
        const float h0 = silu_fast(__uint_as_float(gr[2 * j]) * sc) * (__uint_as_float(ur[2 * j]) * sc);
        const float h1 = silu_fast(__uint_as_float(gr[2 * j + 1]) * sc) * (__uint_as_float(ur[2 * j + 1]) * sc);
        __half2 hh = row_ok ? __halves2half2(to_half_checked(h0, st, 20), to_half_checked(h1, st, 20))
                            : __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f));
        packed[16 * half + j] = *reinterpret_cast<uint32_t*>(&hh);
      }
    }
    const int row0 = row - (int)(threadIdx.x & 31);
    warp_store_rows_128B(reinterpret_cast<uint32_t*>(scratch), packed, [&](int r) -> uint4* {
      const int rr = row0 + r;
      return rr < M ? reinterpret_cast<uint4*>(a.h + (int64_t)rr * a.ldh + out0) : nullptr;
    });
  }
};

// Per 128-column head of the fused Q|K|V output: q and k get RMSNorm over the
// head (QK-norm) and rotate-half RoPE at the token's logical position; v is
// copied.  q goes to [T][Hq][128], k and v to the per-head KV buffers.
template <int EG_>
struct EpiQkvT {
  EpiQkvArgs a;
  static constexpr int EG = EG_;  // one head of the tile (256 or 128 columns) per group
  // rows leave through two per-warp scratches (the head's two 64-column
  // halves), four full lines per warp store; a 4-stage ring keeps the CTA
  // near 200 KB
  static constexpr int STAGES = 4;
  static constexpr int SCRATCH_PER_WARP = 2 * kScratchPerWarp;
  struct Pre {};
  template <int BN>
  __device__ __forceinline__ Pre prefetch(int, int, int, bool, const PlanHdr*, DevStatus*) const {
    return Pre{};
  }
  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int row, int n0, int g, bool row_ok, const PlanHdr* plan,
                                      DevStatus* st, uint8_t* scratch, int M, const Pre&, int) const {
    static_assert(BN == 128 * EG, "one 128-column head per epilogue group");
    const int gc = n0 + 128 * g;
    const uint32_t base = taddr + 128 * g;
    const int lane = threadIdx.x & 31;
    const int row0 = row - lane;
    uint32_t* buf1 = reinterpret_cast<uint32_t*>(scratch);
    uint32_t* buf2 = buf1 + 32 * kScratchPad;
    // weight scale times the input row's RMSNorm factor
    const float sc = row_ok ? a.scale * row_rnorm(a.ssp, a.n_slots, row, a.inv_d, a.norm_eps) : 0.f;
    // the store row this thread's token goes to (-1: none), shared with the
    // warp's other lanes by shuffles when the rows are written out
    int srow = -1;
    if (a.ks && gc >= a.qd && row_ok) {
      const int r = plan_array<int32_t>(plan, plan->off_treq)[row];
      const int i = row - plan_array<int4>(plan, plan->off_req)[r].x;
      const int2 ap = a.append[r];
      if (i >= 0 && i < ap.x) srow = ap.y + i;
    }
    auto store_dst = [&](__half* base_, int head_, int r, int col) -> uint4* {
      const int sr = __shfl_sync(0xffffffffu, srow, r);
      return sr >= 0 ? reinterpret_cast<uint4*>(base_ + ((int64_t)head_ * a.store_rows + sr) * 128 + col) : nullptr;
    };
    if (gc >= a.qd + a.kd) {  // value head
      const int head = (gc - a.qd - a.kd) >> 7;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float v[32];
          tmem_ld32(base + 64 * half + 32 * q, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            __half2 hh = row_ok ? __halves2half2(to_half_checked(v[2 * j] * sc, st, 21),
                                                 to_half_checked(v[2 * j + 1] * sc, st, 21))
                                : __halves2half2(__float2half_rn(0.f), __float2half_rn(0.f));
            pk[16 * q + j] = *reinterpret_cast<uint32_t*>(&hh);
          }
        }
        warp_store_rows_128B(buf1, pk, [&](int r) -> uint4* {
          const int rr = row0 + r;
          return rr < M ? reinterpret_cast<uint4*>(a.vc + ((int64_t)head * a.kv_rows + rr) * 128 + 64 * half)
                        : nullptr;
        });
        if (a.ks) warp_flush_rows_128B(buf1, [&](int r) -> uint4* { return store_dst(a.vs, head, r, 64 * half); });
      }
      return;
    }
    const bool is_q = gc < a.qd;
    const int head = is_q ? (gc >> 7) : ((gc - a.qd) >> 7);
    const float* gain = is_q ? a.gq : a.gk;
    auto dst = [&](int rr) -> __half* {
      return is_q ? a.q + ((int64_t)rr * a.n_q_heads + head) * 128 : a.kc + ((int64_t)head * a.kv_rows + rr) * 128;
    };
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < 128; c += 16) {
      float v[16];
      tmem_ld16(base + c, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float t = v[j] * sc;
        ss += t * t;
      }
    }
    const float r = rsqrtf(ss * (1.0f / 128.0f) + a.eps);
    int p = 0;
    if (row_ok) {
      p = plan_array<int32_t>(plan, plan->off_pos)[row];
      if (p < 0 || p >= a.max_pos) {
        raise_error(st, ERR_BAD_INDEX, 22);
        p = 0;
      }
    }
    const float2* cs = a.rope + p;  // entry (i, p) at cs[i * max_pos]
    __syncwarp();  // the previous tile's reads of the scratches are done
#pragma unroll 1
    for (int c = 0; c < 64; c += 16) {
      float x1[16], x2[16];
      tmem_ld16(base + c, x1);
      tmem_ld16(base + 64 + c, x2);
      if (row_ok) {
        // this chunk's 16 + 16 norm gains as four 16-byte loads each (the
        // same addresses in every lane: broadcasts)
        float g1[16], g2[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 u = reinterpret_cast<const float4*>(gain + c)[q];
          const float4 w = reinterpret_cast<const float4*>(gain + 64 + c)[q];
          g1[4 * q] = u.x, g1[4 * q + 1] = u.y, g1[4 * q + 2] = u.z, g1[4 * q + 3] = u.w;
          g2[4 * q] = w.x, g2[4 * q + 1] = w.y, g2[4 * q + 2] = w.z, g2[4 * q + 3] = w.w;
        }
        const float scr = sc * r;
        uint32_t o1[8], o2[8];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          float r1[2], r2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int i = c + j + e;
            const float a1 = (x1[j + e] * scr) * g1[j + e];
            const float a2 = (x2[j + e] * scr) * g2[j + e];
            const float2 t = cs[(int64_t)i * a.max_pos];
            r1[e] = a1 * t.x - a2 * t.y;
            r2[e] = a2 * t.x + a1 * t.y;
          }
          __half2 h1 = __floats2half2_rn(r1[0], r1[1]);
          __half2 h2 = __floats2half2_rn(r2[0], r2[1]);
          o1[j / 2] = *reinterpret_cast<uint32_t*>(&h1);
          o2[j / 2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        // this chunk's 16 + 16 outputs into the row's slots of the scratches
        uint32_t* s1 = buf1 + lane * kScratchPad + c / 2;
        uint32_t* s2 = buf2 + lane * kScratchPad + c / 2;
        reinterpret_cast<uint4*>(s1)[0] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
        reinterpret_cast<uint4*>(s1)[1] = make_uint4(o1[4], o1[5], o1[6], o1[7]);
        reinterpret_cast<uint4*>(s2)[0] = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        reinterpret_cast<uint4*>(s2)[1] = make_uint4(o2[4], o2[5], o2[6], o2[7]);
      }
    }
    warp_flush_rows_128B(buf1, [&](int r) -> uint4* {
      const int rr = row0 + r;
      return rr < M ? reinterpret_cast<uint4*>(dst(rr)) : nullptr;
    });
    warp_flush_rows_128B(buf2, [&](int r) -> uint4* {
      const int rr = row0 + r;
      return rr < M ? reinterpret_cast<uint4*>(dst(rr) + 64) : nullptr;
    });
    if (a.ks && !is_q) {
      warp_flush_rows_128B(buf1, [&](int r) -> uint4* { return store_dst(a.ks, head, r, 0); });
      warp_flush_rows_128B(buf2, [&](int r) -> uint4* { return store_dst(a.ks, head, r, 64); });
    }
  }
};

// Split-K slice: the fp32 accumulator rows to the workspace, 32-byte stores.
struct EpiPartial {
  EpiPartialArgs a;
  static constexpr int EG = 2;
  static constexpr int STAGES = 6;
  static constexpr int SCRATCH_PER_WARP = 0;
  struct Pre {};
  template <int BN>
  __device__ __forceinline__ Pre prefetch(int, int, int, bool, const PlanHdr*, DevStatus*) const {
    return Pre{};
  }
  template <int BN>
  __device__ __forceinline__ void run(uint32_t taddr, int row, int n0, int g, bool row_ok, const PlanHdr*,
                                      DevStatus*, uint8_t*, int, const Pre&, int split) const {
    constexpr int W = BN / EG;
    float* dst = a.ws + ((int64_t)split * a.ws_rows + row) * a.ldw + n0 + g * W;
#pragma unroll 1
    for (int c = 0; c < W; c += 32) {
      uint32_t v[32];
      tmem_ld32_async(taddr + g * W + c, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) tmem_ld_fence(v[j]);
      if (row_ok) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint32_t w[8] = {v[8 * h], v[8 * h + 1], v[8 * h + 2], v[8 * h + 3],
                                 v[8 * h + 4], v[8 * h + 5], v[8 * h + 6], v[8 * h + 7]};
          st_global_v8(dst + c + 8 * h, w);
        }
      }
    }
  }
};

using EpiResid = EpiResidT<2>;
using EpiQkv = EpiQkvT<2>;
using EpiQkvNarrow = EpiQkvT<1>;      // 128-column tiles

// ---------------------------------------------------------------------------
// the kernel, per CTA of a pair: warp 0 TMA producer, warp 1 TMEM allocation
// and (leader only) the MMA issuer, warps 2 .. 2 + 4*EG - 1 epilogue (group
// g = (warp - 2) / 4; each group spans the four TMEM lane quadrants, warp w
// accessing lanes 32 * (w % 4) .. + 31)
// ---------------------------------------------------------------------------
template <int BN, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(64 + 128 * Epi::EG, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int Kdim,
                   int N, const PlanHdr* __restrict__ plan, const Epi epi, DevStatus* st, int splits) {
  using C = TcCfg<BN, Epi>;
  constexpr int EG = Epi::EG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + C::STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * C::STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * C::STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * C::STAGES + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5);
  uint32_t* skip_flag = tmem_holder + 1;

  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = plan->n_tokens;
  const int m_tiles = (M + 2 * kBM - 1) / (2 * kBM);
  const int n_tiles = N / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int kblocks = Kdim / kBK;
  // work units: (tile, k-slice) pairs; with splits > 1 each unit sums a
  // slice of K and the epilogue stores that partial (split-K for batches too
  // small to give every CTA pair a tile of its own)
  const int num_units = num_tiles * splits;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  pdl_launch_dependents();
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 2 * 128 * EG);  // the epilogue threads of both CTAs
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    // the weight blocks of this CTA's first stages into L2 while the previous
    // kernel finishes (weights are never written during a pass, so this may
    // run before the wait for the predecessor)
    if (pair < num_units) {
      const int split = pair % splits, n_blk = (pair / splits) % n_tiles;
      const int kb0 = split * kblocks / splits, kb1 = min((split + 1) * kblocks / splits, kb0 + C::STAGES);
      for (int kb = kb0; kb < kb1; ++kb) tma_prefetch_2d(&tmB, kb * kBK, n_blk * BN + (int)rank * (BN / 2));
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // everything below reads what the previous kernels wrote
  pdl_wait();
  // a bounded wait already gave up in an earlier launch: the pair skips its
  // work, on the leader's reading of the flag so both CTAs agree
  if (threadIdx.x == 0 && leader)
    *skip_flag = (*reinterpret_cast<volatile const uint32_t*>(&st->flags) & ERR_WAIT_TIMEOUT) ? 1u : 0u;
  cluster_sync();
  const bool skip = ld_shared_cluster_u32(map_to_rank(smem_u32(skip_flag), 0)) != 0;

  if (!skip) {
    if (warp == 0) {
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = pair; u < num_units && ok; u += n_pairs) {
          const int tile = u / splits, split = u % splits;
          const int m_blk = tile / n_tiles, n_blk = tile % n_tiles;
          for (int kb = split * kblocks / splits; kb < (split + 1) * kblocks / splits; ++kb) {
            if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, st, 1)) {
              ok = false;
              break;
            }
            const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
            const uint32_t sb = sa + C::A_BYTES;
            // both CTAs' bytes complete on the leader's full barrier
            const uint32_t full_leader = map_to_rank(full0 + 8 * stage, 0);
            if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, 2 * C::STAGE_BYTES);
            tma_load_2d_pair(&tmA, sa, full_leader, kb * kBK, m_blk * 2 * kBM + (int)rank * kBM);
            tma_load_2d_pair(&tmB, sb, full_leader, kb * kBK, n_blk * BN + (int)rank * (BN / 2));
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    } else if (warp == 1) {
      if (lane == 0 && leader) {
        int stage = 0;
        uint32_t phase = 0;
        int local = 0;
        bool ok = true;
        for (int u = pair; u < num_units && ok; u += n_pairs, ++local) {
          const int split = u % splits;
          const int kb0 = split * kblocks / splits, kb1 = (split + 1) * kblocks / splits;
          const int acc = local & 1;
          const uint32_t use = (uint32_t)(local >> 1);
          if (!mbar_wait(tempty0 + 8 * acc, (use & 1u) ^ 1u, st, 2)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * BN;
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(full0 + 8 * stage, phase, st, 3)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
            const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              tc_mma_f16_pair(d_tmem, smem_desc_sw128(sa + 32 * k), smem_desc_sw128(sb + 32 * k), C::IDESC,
                              (kb != kb0 || k != 0) ? 1u : 0u);
            }
            tc_commit_pair_both(empty0 + 8 * stage);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) tc_commit_pair_both(tfull0 + 8 * acc);
        }
        // one more commit, observed by both CTAs before they leave: every
        // earlier arrival of this pair's MMAs has landed by then
        tc_commit_pair_both(drain);
      }
    } else {
      const int q4 = warp & 3;            // TMEM lane quadrant this warp may access
      const int group = (warp - 2) >> 2;  // column group of the tile
      int local = 0;
      for (int u = pair; u < num_units; u += n_pairs, ++local) {
        const int tile = u / splits, split = u % splits;
        const int acc = local & 1;
        const uint32_t use = (uint32_t)(local >> 1);
        const int m_blk = tile / n_tiles, n_blk = tile % n_tiles;
        const int row = m_blk * 2 * kBM + (int)rank * kBM + q4 * 32 + lane;
        const typename Epi::Pre pre = epi.template prefetch<BN>(row, n_blk * BN, group, row < M, plan, st);
        if (!mbar_wait_warp(tfull0 + 8 * acc, use & 1u, st, 4)) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q4 * 32) << 16);
        epi.template run<BN>(taddr, row, n_blk * BN, group, row < M, plan, st,
                             smem + C::EPI_OFF + (warp - 2) * Epi::SCRATCH_PER_WARP, M, pre, split);
        // the accumulator may be overwritten once every epilogue thread of
        // the pair has read it; the reads are ordered by the tcgen05 fence,
        // the global stores need no ordering with the MMA
        tc_fence_before();
        mbar_arrive_cluster_relaxed(map_to_rank(tempty0 + 8 * acc, 0));
      }
    }
    if (threadIdx.x == 0) mbar_wait(drain, 0, st, 5);
  }

  // no CTA leaves while its peer may still signal it or read its memory
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

bool make_tmap_f16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                      uint32_t box_outer, char* err, size_t errlen) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled unavailable");
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (%d): inner %llu outer %llu box %u x %u", (int)r,
             (unsigned long long)inner, (unsigned long long)outer, box_inner, box_outer);
    return false;
  }
  return true;
}

bool make_tmap_f16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides_bytes[2],
                      const uint32_t box[3], char* err, size_t errlen) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled unavailable");
    return false;
  }
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t s[2] = {strides_bytes[0], strides_bytes[1]};
  cuuint32_t bx[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), d, s, bx, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
    return false;
  }
  return true;
}

template <int BN, class Epi>
static cudaError_t set_smem() {
  return cudaFuncSetAttribute(gemm_tc_kernel<BN, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TcCfg<BN, Epi>::SMEM);
}

template <int BN, class Epi>
static cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                          const Epi& e, DevStatus* st, int grid, cudaStream_t s, bool pdl, int splits = 1) {
  return launch_ex(gemm_tc_kernel<BN, Epi>, dim3(grid), dim3(64 + 128 * Epi::EG), TcCfg<BN, Epi>::SMEM, s, pdl, a, b,
                   K, N, plan, e, st, splits);
}

cudaError_t gemm_tc_setup() {
  cudaError_t e;
  if ((e = set_smem<256, EpiResid>()) != cudaSuccess ||
      (e = set_smem<256, EpiSwiglu>()) != cudaSuccess || (e = set_smem<256, EpiQkv>()) != cudaSuccess ||
      (e = set_smem<kNarrowQkv, EpiQkvNarrow>()) != cudaSuccess || (e = set_smem<256, EpiPartial>()) != cudaSuccess)
    return e;
  return cudaSuccess;
}

cudaError_t gemm_tc_resid(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                          EpiResidArgs e, DevStatus* st, int grid, cudaStream_t s, bool pdl) {
  return launch<256>(a, b, K, N, plan, EpiResid{e}, st, grid, s, pdl);
}
cudaError_t gemm_tc_partial(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                            EpiPartialArgs e, DevStatus* st, int grid, cudaStream_t s, int splits, bool pdl) {
  if (splits < 1 || splits > K / kBK) return cudaErrorInvalidValue;
  return launch<256>(a, b, K, N, plan, EpiPartial{e}, st, grid, s, pdl, splits);
}

// One CTA per row: x += scale * (sum of the split slices, in slice order),
// then fp16(x * g_next) and the per-64-column sums of x^2 (one writer per
// slot), the same outputs as the residual epilogue.  N a multiple of 128.
__global__ void __launch_bounds__(256) resid_reduce_kernel(const PlanHdr* __restrict__ plan,
                                                           const float* __restrict__ ws, int64_t ws_rows, int splits,
                                                           EpiResidArgs e, int N, DevStatus* st) {
  pdl_launch_dependents();
  pdl_wait();
  const int M = plan->n_tokens;
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    for (int c = 4 * threadIdx.x; c < N; c += 4 * blockDim.x) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < splits; ++sp) {
        const float4 v = *reinterpret_cast<const float4*>(ws + ((int64_t)sp * ws_rows + r) * N + c);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      float4* xp = reinterpret_cast<float4*>(e.x + (int64_t)r * e.ldx + c);
      float4 t = *xp;
      t.x += acc.x * e.scale;
      t.y += acc.y * e.scale;
      t.z += acc.z * e.scale;
      t.w += acc.w * e.scale;
      *xp = t;
      if (e.xg) {
        const float4 gn = *reinterpret_cast<const float4*>(e.g_next + c);
        const __half2 h0 = __halves2half2(to_half_checked(t.x * gn.x, st, 24), to_half_checked(t.y * gn.y, st, 24));
        const __half2 h1 = __halves2half2(to_half_checked(t.z * gn.z, st, 24), to_half_checked(t.w * gn.w, st, 24));
        *reinterpret_cast<uint2*>(e.xg + (int64_t)r * e.ldx + c) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
        // the 16 threads of a 64-column slot sum their squares
        float ss = t.x * t.x + t.y * t.y + t.z * t.z + t.w * t.w;
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        ss += __shfl_xor_sync(0xffffffffu, ss, 4);
        ss += __shfl_xor_sync(0xffffffffu, ss, 8);
        if ((threadIdx.x & 15) == 0) e.ssp[(int64_t)r * e.n_slots + c / 64] = ss;
      }
    }
  }
}

cudaError_t resid_reduce(const PlanHdr* plan, const float* ws, int64_t ws_rows, int splits, EpiResidArgs e, int N,
                         DevStatus* st, int max_rows, cudaStream_t s, bool pdl) {
  if (N % 128) return cudaErrorInvalidValue;
  return launch_ex(resid_reduce_kernel, dim3(std::max(1, max_rows)), dim3(256), 0, s, pdl, plan, ws, ws_rows, splits, e,
                   N, st);
}

cudaError_t gemm_tc_swiglu(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                           EpiSwigluArgs e, DevStatus* st, int grid, cudaStream_t s, bool pdl) {
  return launch<256>(a, b, K, N, plan, EpiSwiglu{e}, st, grid, s, pdl);
}
cudaError_t gemm_tc_qkv(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                        EpiQkvArgs e, DevStatus* st, int grid, cudaStream_t s, bool narrow, bool pdl) {
  return narrow ? launch<kNarrowQkv>(a, b, K, N, plan, EpiQkvNarrow{e}, st, grid, s, pdl)
                : launch<256>(a, b, K, N, plan, EpiQkv{e}, st, grid, s, pdl);
}

}  // namespace duolm
