// Launch interfaces of the ranker's kernels (host side).
#pragma once

#include "common.cuh"

namespace duolm {

// ---- tcgen05 GEMM:  C[M, N] = A[M, K] * B[N, K]^T, fp16 operands, fp32 accumulate.
// M is the batch's token count, read on the device from the plan.

// The normed operand of the QKV and gate/up projections is carried as
// xg = fp16(x * g) (g: the norm's gain) plus per-row partial sums of x^2 in
// `ssp` ([rows][n_slots], one writer per slot); the consuming epilogue scales
// its accumulator row by r = 1 / sqrt(sum(ssp) / d + eps), since
// RMSNorm(x) * g * W = r * ((x * g) * W).
struct EpiResidArgs {   // x[row][col] += scale * acc  (fp32 residual stream)
  float* x;
  int ldx;
  float scale;
  __half* xg;           // optional: fp16(x * g_next) for the next projection
  const float* g_next;  // gain of the next RMSNorm
  float* ssp;           // partial sums of x^2: slot n_blk * 4 + group of the tile's columns
  int n_slots;
};
struct EpiPartialArgs {  // split-K: the unit's fp32 partial to ws[split][row][col]
  float* ws;
  int64_t ws_rows;      // rows per split slice
  int ldw;              // columns (N)
};
struct EpiSwigluArgs {  // tile columns [0, BN/2) gate, [BN/2, BN) up -> h = silu(g) * u, fp16
  __half* h;
  int ldh;
  float scale;
  const float* ssp;     // partial sums of x^2 of the input rows
  int n_slots;
  float inv_d, eps;
};
struct EpiQkvArgs {     // per 128-wide head: q/k RMSNorm + RoPE, v copy; fp16 out
  __half* q;            // [T][n_q_heads][128]
  __half* kc;           // [n_kv_heads][kv_rows][128]
  __half* vc;           // [n_kv_heads][kv_rows][128]
  const float2* rope;   // [64][max_pos] (cos, sin), frequency-major
  int64_t kv_rows;
  int max_pos;
  const float* gq;      // q_norm gains [128]
  const float* gk;      // k_norm gains [128]
  float scale;
  float eps;
  int qd, kd, n_q_heads;
  const float* ssp;     // partial sums of x^2 of the input rows
  int n_slots;
  float inv_d, norm_eps;
  // prefix KV store of this layer (null: none): a request r with
  // append[r] = {n, dst} keeps its first n new prefix rows, whose K and V
  // also go to store rows [dst, dst + n) ([n_kv_heads][store_rows][128])
  __half* ks;
  __half* vs;
  int64_t store_rows;
  const int2* append;
};

bool make_tmap_f16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                      uint32_t box_outer, char* err, size_t errlen);
bool make_tmap_f16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides_bytes[2],
                      const uint32_t box[3], char* err, size_t errlen);
cudaError_t gemm_tc_setup();
// Tile widths: 256 columns, or 128 for QKV in small batches (the weight's
// tensor map then has boxes of 64 rows).
constexpr int kNarrowQkv = 128;
// pdl: launched with programmatic dependent launch (the kernel waits for its
// predecessor itself; see pdl_wait)
cudaError_t gemm_tc_resid(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                          EpiResidArgs e, DevStatus* st, int grid, cudaStream_t s, bool pdl = false);
// Split-K projection for small batches: each of `splits` K-slices of every
// 256 x 256 tile stores its fp32 partial (EpiPartialArgs); resid_reduce then
// sums the slices in slice order (deterministic) and applies the residual
// epilogue (x += scale * sum, fp16(x * g_next), x^2 slot sums).
cudaError_t gemm_tc_partial(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                            EpiPartialArgs e, DevStatus* st, int grid, cudaStream_t s, int splits, bool pdl = false);
cudaError_t resid_reduce(const PlanHdr* plan, const float* ws, int64_t ws_rows, int splits, EpiResidArgs e, int N,
                         DevStatus* st, int max_rows, cudaStream_t s, bool pdl = false);
cudaError_t gemm_tc_swiglu(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                           EpiSwigluArgs e, DevStatus* st, int grid, cudaStream_t s, bool pdl = false);
cudaError_t gemm_tc_qkv(const CUtensorMap& a, const CUtensorMap& b, int K, int N, const PlanHdr* plan,
                        EpiQkvArgs e, DevStatus* st, int grid, cudaStream_t s, bool narrow = false, bool pdl = false);

// ---- fp32 SIMT GEMM (the fp32 path): C = A * B^T, store or residual add.
cudaError_t gemm_simt(const float* A, const float* B, float* C, int K, int N, int ldc, bool accumulate,
                      const PlanHdr* plan, int max_rows, cudaStream_t s);

// ---- elementwise and small kernels
template <typename OutT>
cudaError_t embed_norm(const PlanHdr* plan, const void* embed, bool embed_bf16, const __half* table,
                       int64_t n_table, int vocab, int d, const float* gain, float eps, float* x, OutT* xn,
                       DevStatus* st, int max_rows, cudaStream_t s);
// fp16 path: gather into x, write fp16(x * gain) and the row's sum of x^2
cudaError_t embed_gain(const PlanHdr* plan, const void* embed, const __half* table, int64_t n_table, int vocab, int d,
                       const float* gain, float* x, __half* xg, float* ssp, int n_slots, DevStatus* st, int max_rows,
                       cudaStream_t s, bool pdl = false);
template <typename OutT>
cudaError_t rmsnorm_rows(const PlanHdr* plan, const float* x, int d, const float* gain, float eps, OutT* xn,
                         DevStatus* st, int max_rows, cudaStream_t s);
cudaError_t score_head(const PlanHdr* plan, const float* x, int d, const float* gain, const float* w, float eps,
                       float* scores, int max_cand, cudaStream_t s, bool pdl = false);
cudaError_t qkv_post_f32(const PlanHdr* plan, const float* qkv, int n_q_heads, int n_kv_heads, int hd,
                         const float* gq, const float* gk, float eps, const float2* rope, int max_pos, float* q,
                         float* kc, float* vc, int64_t kv_rows, DevStatus* st, int max_rows, cudaStream_t s);
cudaError_t swiglu_f32(const PlanHdr* plan, const float* gu, int F, float* h, int max_rows, cudaStream_t s);
cudaError_t table_build(const float* a, int64_t n, int d, double scale_num, __half* out, cudaStream_t s);
cudaError_t embed_rho(const void* embed, bool embed_bf16, int64_t vocab, int d, double* row_rms, double* out,
                      cudaStream_t s);
cudaError_t debug_wait_timeout(DevStatus* st, cudaStream_t s);
cudaError_t debug_mask(const PlanHdr* plan, int request, uint8_t* out, int64_t tq, cudaStream_t s);

// ---- attention
// reqx[r] = {c, s}: request r continues a cached prefix of c tokens whose K/V
// are rows [s, s + c) (of every KV head) of the layer's KV store; {0, 0}
// for a request computed from its first token.
cudaError_t attention_f32(const PlanHdr* plan, const int2* reqx, const float* q, const float* kc, const float* vc,
                          int64_t kv_rows, const float* ks, const float* vs, int64_t store_rows, int n_q_heads,
                          int n_kv_heads, int hd, float scale, float* o, int max_rows, cudaStream_t s);
// tcgen05 attention (fp16 path): items of two 128-slot query sub-tiles, KV
// tiles of 128 keys; tks / tvs map the layer's KV store
cudaError_t attention_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tks,
                         const CUtensorMap& tvs, const PlanHdr* plan, const int2* reqx, int64_t kv_rows,
                         int64_t store_rows, int n_q_heads, int n_kv_heads, float scale, __half* o, DevStatus* st,
                         int grid, cudaStream_t s, bool pdl = false);
// KV store append: for every request r with append[r] = {n, dst} (n > 0),
// rows [tok0_r, tok0_r + n) of this batch's K/V (every KV head) are copied
// to store rows [dst, dst + n); row_bytes a multiple of 16
cudaError_t kv_append(const PlanHdr* plan, const int2* append, const void* kc, const void* vc, int64_t kv_rows,
                      void* ks, void* vs, int64_t store_rows, int n_kv_heads, int row_bytes, int max_req,
                      int grid, cudaStream_t s, bool pdl = false);
cudaError_t attention_tc_setup();
// Host: the batch's attention work list {request, KV head, kind (1 branch,
// 0 prefix), first query row} (req: {tok0, whole prefix L, K, -}; reqx: as
// above) and the CTA ranges of its greedy list schedule (cta_off[n_ctas + 1]).
// Returns the item count, or -1 above cap_items.
int64_t plan_attention(const int4* req, const int2* reqx, int64_t R, int n_kv_heads, int rows_per_item,
                       int branch_len, int n_ctas, int64_t cap_items, int4* items, int32_t* cta_off);
int attention_tc_rows_per_item(int group);

}  // namespace duolm
