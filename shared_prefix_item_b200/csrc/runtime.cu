// C ABI of the DuoLM multi-item-scoring ranker: context, weights, item table,
// per-batch plan, launch sequence and CUDA graph.  Declarations and the
// contract of every entry point are in include/duolm.h.
//
// The launch sequence is fixed for a given workspace capacity: every kernel
// reads the batch's sizes from the device plan, so one captured CUDA graph
// replays any batch that fits (DuoLM summary page, 方法步骤详情 step 5: the
// captured segments are replayed with new inputs and position ids only).
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

#include "common.cuh"
#include "duolm.h"
#include "kernels.cuh"

using namespace duolm;

// reason of the calling thread's last failed call that has no context
// (duolm_model_load, duolm_compile); read by duolm_last_error(NULL)
thread_local std::string g_noctx_err;

namespace {

constexpr int kMaxPos = 32768;   // position ids must stay below this
constexpr int kKvPad = 256;      // spare KV rows so the branch key tiles of an item never leave the buffer
constexpr int kPerLayer = 11;
constexpr int kMaxSplits = 8;    // K-slices of a split-K projection

// Split-K plan of the O and down projections for a token capacity: 1 when
// 256 x 256 tiles already give at least half of the CTA pairs a tile, else
// as many K-slices (at most kMaxSplits, at least 4 k-blocks each) as keep
// the work units within the pairs.
int splitk_factor(int64_t cap_T, int d, int K, int gemm_grid) {
  const int64_t tiles = ((cap_T + 255) / 256) * (d / 256);
  const int pairs = gemm_grid / 2;
  if (tiles >= pairs / 2) return 1;
  const int64_t by_pairs = pairs / std::max<int64_t>(tiles, 1);
  return (int)std::max<int64_t>(1, std::min<int64_t>({(int64_t)kMaxSplits, by_pairs, (int64_t)(K / 64 / 4)}));
}

struct LayerW {
  void* wqkv = nullptr;  // [qd + 2 kd][d]
  void* wo = nullptr;    // [d][qd]
  void* wgu = nullptr;   // fp16 path: [2F][d], 128-row blocks gate/up interleaved; fp32: [gate; up]
  void* wd = nullptr;    // [d][F]
  float s_qkv = 1.f, s_o = 1.f, s_gu = 1.f, s_d = 1.f;  // 2^-shift of the fp16 copies
  CUtensorMap tm_qkv, tm_o, tm_gu, tm_d;
  // the QKV weights in boxes of 64 rows for the 128-column tiles of small batches
  CUtensorMap tm_qkv_n64;
  int64_t g_attn = 0, g_q = 0, g_k = 0, g_mlp = 0;  // offsets into the gain buffer
};

inline int64_t align16(int64_t v) { return (v + 15) & ~int64_t(15); }
inline float bf16_bits_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

}  // namespace

struct duolm_ctx {
  duolm_model_desc desc{};
  int device = 0;
  cudaStream_t stream = nullptr;
  bool own_stream = false;
  bool f16 = false;
  int num_sms = 148;
  int gemm_grid = 148;  // whole CTA pairs
  bool use_pdl = true;  // programmatic dependent launch between the pass's kernels
  int qd = 0, kd = 0, group = 1, rows_per_item = 64;

  void* embed = nullptr;
  float* gains = nullptr;
  float* head = nullptr;
  int64_t g_final = 0;
  std::vector<LayerW> layers;
  __half* table = nullptr;
  int64_t n_items = 0;
  float2* rope = nullptr;
  DevStatus* status = nullptr;
  double* rho_buf = nullptr;
  PlanHdr* gather_hdr = nullptr;  // header through which duolm_gather hands the caller's ids to the gather

  int64_t cap_T = 0, cap_R = 0, cap_C = 0, cap_I = 0, plan_cap = 0;
  float* x = nullptr;
  void* xn = nullptr;
  void* q = nullptr;
  void* kc = nullptr;
  void* vc = nullptr;
  void* o = nullptr;
  void* h = nullptr;
  float* qkv32 = nullptr;
  float* gu32 = nullptr;
  float* ssp = nullptr;  // fp16 path: per-row partial sums of x^2 [T][d / 64]
  float* splitk_ws = nullptr;  // split-K slices of the O / down projections [kMaxSplits][T][d] (small batches)
  float* scores = nullptr;
  char* plan_dev = nullptr;
  char* plan_host = nullptr;
  cudaEvent_t plan_ev = nullptr;
  CUtensorMap tm_xn, tm_oact, tm_h;
  CUtensorMap tm_q3, tm_kc, tm_vc;  // attention operands

  // prefix KV store: per layer [n_kv_heads][n_slots * slot_tokens][head_dim]
  // for K and for V; slot s of a head starts at row s * slot_tokens
  void* ks = nullptr;
  void* vs = nullptr;
  int n_slots = 0, slot_tokens = 0;
  int64_t layer_store_elems = 0;  // elements of one layer's K (or V) store
  std::vector<CUtensorMap> tm_ks, tm_vs;  // per layer (fp16 path)
  std::vector<int> slot_len;     // valid rows of every slot
  std::vector<std::pair<int, int>> slot_update;  // (slot, length) once the prepared batch has run
  int2* reqx = nullptr;          // [cap_R] {cached tokens, first store row}
  int2* append = nullptr;        // [cap_R] {rows kept, first store row they go to}
  int2* reqx_host = nullptr;     // pinned staging of both (2 cap_R)

  bool prepared = false;
  int64_t n_tokens = 0, n_cand = 0;
  int n_req = 0, branch_len = 1;
  PlanHdr hdr{};
  std::vector<int4> req_host;  // {tok0, L, K, cand0} of the prepared batch

  bool use_graph = true;
  cudaGraphExec_t gexec = nullptr;
  bool graph_valid = false;
  int64_t launches = 0;
  std::string err;
};

namespace {


int fail(duolm_ctx* c, int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (c) c->err = buf;
  return code;
}

#define CK(expr)                                                                                          \
  do {                                                                                                    \
    cudaError_t e_ = (expr);                                                                              \
    if (e_ != cudaSuccess)                                                                                \
      return fail(ctx, DUOLM_E_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_), __FILE__, \
                  __LINE__);                                                                              \
  } while (0)

template <typename T>
int dalloc(duolm_ctx* ctx, T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) bytes = 16;
  CK(cudaMalloc(reinterpret_cast<void**>(p), bytes));
  return 0;
}
template <typename T>
void dfree(T*& p) {
  if (p) cudaFree(reinterpret_cast<void*>(p));
  p = nullptr;
}

// Convert bfloat16 values times 2^shift to fp16; returns the number of values
// that do not convert exactly.
int64_t convert_scaled(const uint16_t* src, int64_t n, int shift, uint16_t* dst) {
  const float mul = ldexpf(1.0f, shift);
  const int nth = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
  std::vector<int64_t> bad(nth, 0);
  std::vector<std::thread> th;
  for (int t = 0; t < nth; ++t) {
    th.emplace_back([&, t]() {
      const int64_t b0 = n * t / nth, b1 = n * (t + 1) / nth;
      for (int64_t i = b0; i < b1; ++i) {
        const float f = bf16_bits_to_float(src[i]) * mul;
        const __half hv = __float2half_rn(f);
        if (__half2float(hv) != f) ++bad[t];
        dst[i] = *reinterpret_cast<const uint16_t*>(&hv);
      }
    });
  }
  for (auto& x : th) x.join();
  int64_t tot = 0;
  for (int64_t v : bad) tot += v;
  return tot;
}

float max_abs_bf16(const uint16_t* src, int64_t n) {
  float m = 0.f;
  for (int64_t i = 0; i < n; ++i) m = std::max(m, std::fabs(bf16_bits_to_float(src[i])));
  return m;
}

// Largest shift with max|w| * 2^shift below 2^15 (keeps the fp16 copy far
// from overflow while moving small weights out of the subnormal range).
int choose_shift(float maxabs) {
  if (!(maxabs > 0.f)) return 0;
  int s = 0;
  while (s > -24 && maxabs * ldexpf(1.f, s) >= 32768.f) --s;
  while (s < 24 && maxabs * ldexpf(1.f, s + 1) < 32768.f) ++s;
  return s;
}

struct Part {
  const uint16_t* src;
  int64_t rows;
};

// Upload a matrix made of row blocks of bf16 sources as fp16 x 2^shift.
int upload_f16(duolm_ctx* ctx, const std::vector<Part>& parts, int64_t cols, void** dst, float* scale,
               const char* name) {
  int64_t rows = 0;
  float m = 0.f;
  for (auto& p : parts) {
    rows += p.rows;
    m = std::max(m, max_abs_bf16(p.src, p.rows * cols));
  }
  const int shift = choose_shift(m);
  std::vector<uint16_t> host((size_t)(rows * cols));
  int64_t off = 0, bad = 0;
  for (auto& p : parts) {
    bad += convert_scaled(p.src, p.rows * cols, shift, host.data() + off);
    off += p.rows * cols;
  }
  if (bad)
    return fail(ctx, DUOLM_E_ARG, "%s: %lld bfloat16 values have no exact fp16 form at scale 2^%d", name,
                (long long)bad, shift);
  if (int rc = dalloc(ctx, dst, host.size() * 2)) return rc;
  CK(cudaMemcpy(*dst, host.data(), host.size() * 2, cudaMemcpyHostToDevice));
  *scale = ldexpf(1.f, -shift);
  return 0;
}

int upload_f32(duolm_ctx* ctx, const std::vector<std::pair<const float*, int64_t>>& parts, void** dst) {
  int64_t n = 0;
  for (auto& p : parts) n += p.second;
  if (int rc = dalloc(ctx, reinterpret_cast<float**>(dst), n * 4)) return rc;
  int64_t off = 0;
  for (auto& p : parts) {
    CK(cudaMemcpy(reinterpret_cast<float*>(*dst) + off, p.first, p.second * 4, cudaMemcpyHostToDevice));
    off += p.second;
  }
  return 0;
}

void free_workspace(duolm_ctx* c) {
  dfree(c->x);
  dfree(c->xn);
  dfree(c->q);
  dfree(c->kc);
  dfree(c->vc);
  dfree(c->o);
  dfree(c->h);
  dfree(c->qkv32);
  dfree(c->gu32);
  dfree(c->ssp);
  dfree(c->splitk_ws);
  dfree(c->scores);
  dfree(c->plan_dev);
  dfree(c->reqx);
  dfree(c->append);
  if (c->plan_host) cudaFreeHost(c->plan_host);
  c->plan_host = nullptr;
  if (c->reqx_host) cudaFreeHost(c->reqx_host);
  c->reqx_host = nullptr;
  c->cap_T = c->cap_R = c->cap_C = c->cap_I = c->plan_cap = 0;
}

void invalidate_graph(duolm_ctx* c) {
  if (c->gexec) cudaGraphExecDestroy(c->gexec);
  c->gexec = nullptr;
  c->graph_valid = false;
}

int64_t items_bound(const duolm_ctx* c, int64_t T, int64_t R) {
  const int64_t r = c->rows_per_item;
  return (int64_t)c->desc.n_kv_heads * (2 * T / r + 2 * R + 2);
}

int64_t plan_bytes_for(int64_t T, int64_t R, int64_t C, int64_t I, int64_t G) {
  return (int64_t)sizeof(PlanHdr) + 3 * align16(T * 4) + align16(R * 16) + align16(C * 4) + align16(I * 16) +
         align16((G + 1) * 4);
}

int reserve_impl(duolm_ctx* ctx, int64_t T, int64_t R, int64_t C) {
  T = std::max<int64_t>(T, 128);
  R = std::max<int64_t>(R, 1);
  C = std::max<int64_t>(C, 1);
  if (T <= ctx->cap_T && R <= ctx->cap_R && C <= ctx->cap_C) return 0;
  T = std::max(T, ctx->cap_T);
  R = std::max(R, ctx->cap_R);
  C = std::max(C, ctx->cap_C);
  if (T > INT32_MAX / 2) return fail(ctx, DUOLM_E_CAPACITY, "token capacity %lld too large", (long long)T);
  CK(cudaStreamSynchronize(ctx->stream));
  if (ctx->plan_ev) CK(cudaEventSynchronize(ctx->plan_ev));
  invalidate_graph(ctx);
  free_workspace(ctx);
  const auto& d = ctx->desc;
  const int64_t es = ctx->f16 ? 2 : 4;
  const int64_t kv_rows = T + kKvPad;
  int rc;
  if ((rc = dalloc(ctx, &ctx->x, T * d.d * 4))) return rc;
  if ((rc = dalloc(ctx, &ctx->xn, T * d.d * es))) return rc;
  if ((rc = dalloc(ctx, &ctx->q, T * ctx->qd * es))) return rc;
  if ((rc = dalloc(ctx, &ctx->kc, d.n_kv_heads * kv_rows * d.head_dim * es))) return rc;
  if ((rc = dalloc(ctx, &ctx->vc, d.n_kv_heads * kv_rows * d.head_dim * es))) return rc;
  CK(cudaMemset(ctx->kc, 0, d.n_kv_heads * kv_rows * d.head_dim * es));
  CK(cudaMemset(ctx->vc, 0, d.n_kv_heads * kv_rows * d.head_dim * es));
  if ((rc = dalloc(ctx, &ctx->o, T * ctx->qd * es))) return rc;
  if ((rc = dalloc(ctx, &ctx->h, T * d.ffn * es))) return rc;
  if (ctx->f16) {
    if ((rc = dalloc(ctx, &ctx->ssp, T * (d.d / 64) * 4))) return rc;
    if (splitk_factor(T, d.d, std::max(ctx->qd, d.ffn), ctx->gemm_grid) > 1)
      if ((rc = dalloc(ctx, &ctx->splitk_ws, kMaxSplits * T * d.d * 4))) return rc;
  } else {
    if ((rc = dalloc(ctx, &ctx->qkv32, T * (ctx->qd + 2 * ctx->kd) * 4))) return rc;
    if ((rc = dalloc(ctx, &ctx->gu32, T * 2 * d.ffn * 4))) return rc;
  }
  if ((rc = dalloc(ctx, &ctx->scores, C * 4))) return rc;
  const int64_t I = items_bound(ctx, T, R);
  const int64_t pb = plan_bytes_for(T, R, C, I, ctx->num_sms);
  if ((rc = dalloc(ctx, &ctx->plan_dev, pb))) return rc;
  CK(cudaMallocHost(reinterpret_cast<void**>(&ctx->plan_host), pb));
  if ((rc = dalloc(ctx, &ctx->reqx, R * sizeof(int2)))) return rc;
  if ((rc = dalloc(ctx, &ctx->append, R * sizeof(int2)))) return rc;
  CK(cudaMemset(ctx->reqx, 0, R * sizeof(int2)));
  CK(cudaMemset(ctx->append, 0, R * sizeof(int2)));
  CK(cudaMallocHost(reinterpret_cast<void**>(&ctx->reqx_host), 2 * R * sizeof(int2)));
  ctx->cap_T = T;
  ctx->cap_R = R;
  ctx->cap_C = C;
  ctx->cap_I = I;
  ctx->plan_cap = pb;
  if (ctx->f16) {
    char e[256];
    if (!make_tmap_f16_2d(&ctx->tm_xn, ctx->xn, d.d, T, 64, 128, e, sizeof e) ||
        !make_tmap_f16_2d(&ctx->tm_oact, ctx->o, ctx->qd, T, 64, 128, e, sizeof e) ||
        !make_tmap_f16_2d(&ctx->tm_h, ctx->h, d.ffn, T, 64, 128, e, sizeof e))
      return fail(ctx, DUOLM_E_CUDA, "%s", e);
    // q as [token][head][128]: boxes of 64 dims x (the G heads of one KV head) x (128 / G) tokens
    const uint64_t qdims[3] = {128, (uint64_t)d.n_q_heads, (uint64_t)T};
    const uint64_t qstr[2] = {256, (uint64_t)d.n_q_heads * 256};
    const uint32_t qbox[3] = {64, (uint32_t)ctx->group, (uint32_t)(128 / ctx->group)};
    if (!make_tmap_f16_3d(&ctx->tm_q3, ctx->q, qdims, qstr, qbox, e, sizeof e) ||
        !make_tmap_f16_2d(&ctx->tm_kc, ctx->kc, 128, (uint64_t)d.n_kv_heads * kv_rows, 64, 128, e, sizeof e) ||
        !make_tmap_f16_2d(&ctx->tm_vc, ctx->vc, 128, (uint64_t)d.n_kv_heads * kv_rows, 64, 128, e, sizeof e))
      return fail(ctx, DUOLM_E_CUDA, "%s", e);
  }
  ctx->prepared = false;
  return 0;
}

// Optional per-launch event recorder used by duolm_profile.
struct Prof {
  std::vector<cudaEvent_t> ev;
  std::vector<int> cls;
  size_t used = 0;
};

#define LCK(cls_, expr)                                                 \
  do {                                                                  \
    cudaError_t e_ = (expr);                                            \
    if (e_ != cudaSuccess) return e_;                                   \
    ++launches;                                                         \
    if (prof) {                                                         \
      if (prof->used == prof->ev.size()) {                              \
        cudaEvent_t ev_;                                                \
        if ((e_ = cudaEventCreate(&ev_)) != cudaSuccess) return e_;     \
        prof->ev.push_back(ev_);                                        \
        prof->cls.push_back(0);                                         \
      }                                                                 \
      prof->cls[prof->used] = (cls_);                                   \
      if ((e_ = cudaEventRecord(prof->ev[prof->used++], s)) != cudaSuccess) return e_; \
    }                                                                   \
  } while (0)

// Enqueue the forward pass: embedding, n_layers decoder layers, and (if
// with_head) the score head.  Grid sizes depend only on the capacity.
cudaError_t launch_forward(duolm_ctx* c, int n_layers, bool with_head, int64_t* n_launch, Prof* prof = nullptr) {
  const auto& d = c->desc;
  const PlanHdr* plan = reinterpret_cast<const PlanHdr*>(c->plan_dev);
  cudaStream_t s = c->stream;
  const int maxT = (int)c->cap_T;
  const int64_t kv_rows = c->cap_T + kKvPad;
  const int64_t store_rows = (int64_t)c->n_slots * c->slot_tokens;
  const float attn_scale = 1.0f / sqrtf((float)d.head_dim);
  int64_t launches = 0;
  if (c->f16) {
    // RMSNorm is folded into the projections: x's producer writes
    // fp16(x * g) and per-row partial sums of x^2, the consuming epilogue
    // scales its rows by 1 / sqrt(mean(x^2) + eps)
    __half* xg = static_cast<__half*>(c->xn);
    const int n_slots = d.d / 64;
    const float inv_d = 1.0f / (float)d.d;
    // small batches: narrower tiles wherever 256-wide tiles would leave more
    // than half of the CTA pairs without a tile
    const int64_t m_tiles = (c->cap_T + 255) / 256, half_pairs = c->gemm_grid / 4;
    const bool narrow_qkv = m_tiles * ((c->qd + 2 * c->kd) / 256) < half_pairs;
    // the O and down projections of small batches: split-K (narrow tiles
    // would re-stream the whole activation block per 64 output columns)
    const int split_o = c->splitk_ws ? splitk_factor(c->cap_T, d.d, c->qd, c->gemm_grid) : 1;
    const int split_d = c->splitk_ws ? splitk_factor(c->cap_T, d.d, d.ffn, c->gemm_grid) : 1;
    // every kernel after the first may start its prologue while its
    // predecessor finishes (it waits for the predecessor's data itself)
    const bool pdl = c->use_pdl;
    LCK(DUOLM_PROF_EMBED, embed_gain(plan, c->embed, c->table, c->n_items, d.vocab, d.d, c->gains + c->layers[0].g_attn,
                                     c->x, xg, c->ssp, n_slots, c->status, maxT, s));
    for (int l = 0; l < n_layers; ++l) {
      const LayerW& L = c->layers[l];
      // with a prefix KV store, the kept new prefix rows' K and V also go
      // straight to their store slot from the QKV epilogue
      EpiQkvArgs qa{static_cast<__half*>(c->q), static_cast<__half*>(c->kc), static_cast<__half*>(c->vc), c->rope,
                    kv_rows, kMaxPos, c->gains + L.g_q, c->gains + L.g_k, L.s_qkv, d.rms_eps, c->qd, c->kd,
                    d.n_q_heads, c->ssp, n_slots, inv_d, d.rms_eps,
                    c->ks ? static_cast<__half*>(c->ks) + l * c->layer_store_elems : nullptr,
                    c->ks ? static_cast<__half*>(c->vs) + l * c->layer_store_elems : nullptr, store_rows, c->append};
      LCK(DUOLM_PROF_GEMM_QKV, gemm_tc_qkv(c->tm_xn, narrow_qkv ? L.tm_qkv_n64 : L.tm_qkv, d.d, c->qd + 2 * c->kd,
                                           plan, qa, c->status, c->gemm_grid, s, narrow_qkv, pdl));
      // without a store, the batch's own maps stand in for the store maps
      // (no request has cached tokens then, so no tile reads them)
      LCK(DUOLM_PROF_ATTENTION,
          attention_tc(c->tm_q3, c->tm_kc, c->tm_vc, c->ks ? c->tm_ks[l] : c->tm_kc, c->ks ? c->tm_vs[l] : c->tm_vc,
                       plan, c->reqx, kv_rows, store_rows, d.n_q_heads, d.n_kv_heads, attn_scale,
                       static_cast<__half*>(c->o), c->status, c->num_sms, s, pdl));
      const EpiResidArgs o_args{c->x, d.d, L.s_o, xg, c->gains + L.g_mlp, c->ssp, n_slots};
      if (split_o > 1) {
        LCK(DUOLM_PROF_GEMM_O, gemm_tc_partial(c->tm_oact, L.tm_o, c->qd, d.d, plan,
                                               EpiPartialArgs{c->splitk_ws, c->cap_T, d.d}, c->status, c->gemm_grid,
                                               s, split_o, pdl));
        LCK(DUOLM_PROF_GEMM_O, resid_reduce(plan, c->splitk_ws, c->cap_T, split_o, o_args, d.d, c->status, maxT, s,
                                            pdl));
      } else {
        LCK(DUOLM_PROF_GEMM_O, gemm_tc_resid(c->tm_oact, L.tm_o, c->qd, d.d, plan, o_args, c->status, c->gemm_grid, s,
                                             pdl));
      }
      LCK(DUOLM_PROF_GEMM_GATE_UP,
          gemm_tc_swiglu(c->tm_xn, L.tm_gu, d.d, 2 * d.ffn, plan,
                         EpiSwigluArgs{static_cast<__half*>(c->h), d.ffn, L.s_gu, c->ssp, n_slots, inv_d, d.rms_eps},
                         c->status, c->gemm_grid, s, pdl));
      const bool last = l + 1 == n_layers;
      const EpiResidArgs d_args{c->x, d.d, L.s_d, last ? nullptr : xg,
                                last ? nullptr : c->gains + c->layers[l + 1].g_attn, c->ssp, n_slots};
      if (split_d > 1) {
        LCK(DUOLM_PROF_GEMM_DOWN, gemm_tc_partial(c->tm_h, L.tm_d, d.ffn, d.d, plan,
                                                  EpiPartialArgs{c->splitk_ws, c->cap_T, d.d}, c->status,
                                                  c->gemm_grid, s, split_d, pdl));
        LCK(DUOLM_PROF_GEMM_DOWN, resid_reduce(plan, c->splitk_ws, c->cap_T, split_d, d_args, d.d, c->status, maxT, s,
                                               pdl));
      } else {
        LCK(DUOLM_PROF_GEMM_DOWN, gemm_tc_resid(c->tm_h, L.tm_d, d.ffn, d.d, plan, d_args, c->status, c->gemm_grid, s,
                                                pdl));
      }
    }
  } else {
    float* xn = static_cast<float*>(c->xn);
    LCK(DUOLM_PROF_EMBED, embed_norm<float>(plan, c->embed, false, c->table, c->n_items, d.vocab, d.d, c->gains + c->layers[0].g_attn,
                          d.rms_eps, c->x, xn, c->status, maxT, s));
    const int nqkv = c->qd + 2 * c->kd;
    for (int l = 0; l < n_layers; ++l) {
      const LayerW& L = c->layers[l];
      LCK(DUOLM_PROF_GEMM_QKV, gemm_simt(xn, static_cast<const float*>(L.wqkv), c->qkv32, d.d, nqkv, nqkv, false, plan, maxT, s));
      LCK(DUOLM_PROF_GEMM_QKV, qkv_post_f32(plan, c->qkv32, d.n_q_heads, d.n_kv_heads, d.head_dim, c->gains + L.g_q, c->gains + L.g_k,
                       d.rms_eps, c->rope, kMaxPos, static_cast<float*>(c->q), static_cast<float*>(c->kc),
                       static_cast<float*>(c->vc), kv_rows, c->status, maxT, s));
      const float* ks = c->ks ? static_cast<const float*>(c->ks) + l * c->layer_store_elems : nullptr;
      const float* vs = c->vs ? static_cast<const float*>(c->vs) + l * c->layer_store_elems : nullptr;
      LCK(DUOLM_PROF_ATTENTION, attention_f32(plan, c->reqx, static_cast<float*>(c->q), static_cast<float*>(c->kc),
                                              static_cast<float*>(c->vc), kv_rows, ks, vs, store_rows, d.n_q_heads,
                                              d.n_kv_heads, d.head_dim, attn_scale, static_cast<float*>(c->o), maxT,
                                              s));
      if (c->ks)
        LCK(DUOLM_PROF_KV_APPEND, kv_append(plan, c->append, c->kc, c->vc, kv_rows, const_cast<float*>(ks),
                                            const_cast<float*>(vs), store_rows, d.n_kv_heads, d.head_dim * 4,
                                            (int)c->cap_R, 2 * c->num_sms, s));
      LCK(DUOLM_PROF_GEMM_O, gemm_simt(static_cast<float*>(c->o), static_cast<const float*>(L.wo), c->x, c->qd, d.d, d.d, true, plan,
                    maxT, s));
      LCK(DUOLM_PROF_RMSNORM, rmsnorm_rows<float>(plan, c->x, d.d, c->gains + L.g_mlp, d.rms_eps, xn, c->status, maxT, s));
      LCK(DUOLM_PROF_GEMM_GATE_UP, gemm_simt(xn, static_cast<const float*>(L.wgu), c->gu32, d.d, 2 * d.ffn, 2 * d.ffn, false, plan, maxT,
                    s));
      LCK(DUOLM_PROF_GEMM_GATE_UP, swiglu_f32(plan, c->gu32, d.ffn, static_cast<float*>(c->h), maxT, s));
      LCK(DUOLM_PROF_GEMM_DOWN, gemm_simt(static_cast<float*>(c->h), static_cast<const float*>(L.wd), c->x, d.ffn, d.d, d.d, true, plan,
                    maxT, s));
      if (l + 1 < n_layers)
        LCK(DUOLM_PROF_RMSNORM, rmsnorm_rows<float>(plan, c->x, d.d, c->gains + c->layers[l + 1].g_attn, d.rms_eps, xn, c->status, maxT,
                                s));
    }
  }
  if (with_head)
    LCK(DUOLM_PROF_HEAD, score_head(plan, c->x, d.d, c->gains + c->g_final, c->head, d.rms_eps, c->scores, (int)c->cap_C,
                                    s, c->f16 && c->use_pdl));
  if (n_launch) *n_launch = launches;
  return cudaSuccess;
}

int check_status(duolm_ctx* ctx) {
  DevStatus hs;
  CK(cudaMemcpyAsync(&hs, ctx->status, sizeof(hs), cudaMemcpyDeviceToHost, ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  if (hs.flags) {
    CK(cudaMemsetAsync(ctx->status, 0, sizeof(DevStatus), ctx->stream));
    CK(cudaStreamSynchronize(ctx->stream));
    return fail(ctx, DUOLM_E_DEVICE, "device error flags 0x%x (first at site %u)%s%s%s", hs.flags, hs.where,
                (hs.flags & ERR_WAIT_TIMEOUT) ? " wait-timeout" : "",
                (hs.flags & ERR_FP16_RANGE) ? " fp16-out-of-range" : "",
                (hs.flags & ERR_BAD_INDEX) ? " bad-index" : "");
  }
  return 0;
}

struct ReqView {
  const int32_t* prefix;  // the new prefix tokens (after the cached ones)
  int64_t L;
  const int32_t* branch;  // K * b ids
  int64_t K;
  int cached;             // prefix tokens already in the slot
  int slot;               // KV store slot, -1: none
  int keep;               // new prefix tokens appended to the slot
};

}  // namespace

extern "C" {

int duolm_weight_count(const duolm_model_desc* desc) {
  if (!desc || desc->n_layers < 1) return DUOLM_E_ARG;
  return 1 + kPerLayer * desc->n_layers + 2;
}

int duolm_model_load(const duolm_model_desc* desc, const void* const* host_weights, int device, void* cuda_stream,
                     duolm_ctx** out) {
  if (!out) return DUOLM_E_ARG;
  *out = nullptr;
  if (!desc || !host_weights) return DUOLM_E_ARG;
  const duolm_model_desc d = *desc;
  if (d.n_layers < 1 || d.d < 8 || d.d % 8 || d.d > 2048 || d.n_q_heads < 1 || d.n_kv_heads < 1 ||
      d.n_q_heads % d.n_kv_heads || d.head_dim < 2 || d.head_dim % 2 || d.ffn < 1 || d.vocab < 1 ||
      !(d.rms_eps >= 0.f) || !(d.rope_theta > 0.f) || (d.dtype != DUOLM_DTYPE_FP32 && d.dtype != DUOLM_DTYPE_BF16))
    return DUOLM_E_ARG;
  const int G = d.n_q_heads / d.n_kv_heads;
  if (d.dtype == DUOLM_DTYPE_BF16) {
    if (d.head_dim != 128 || d.d % 256 || d.ffn % 128 || (d.n_q_heads + 2 * d.n_kv_heads) % 2 ||
        (G != 1 && G != 2 && G != 4))
      return DUOLM_E_ARG;
  } else {
    if (d.head_dim % 32 || d.head_dim > 256) return DUOLM_E_ARG;
  }
  for (int i = 0; i < 1 + kPerLayer * d.n_layers + 2; ++i)
    if (!host_weights[i]) return DUOLM_E_ARG;

  duolm_ctx* ctx = new duolm_ctx();
  ctx->desc = d;
  ctx->device = device;
  ctx->f16 = d.dtype == DUOLM_DTYPE_BF16;
  ctx->qd = d.n_q_heads * d.head_dim;
  ctx->kd = d.n_kv_heads * d.head_dim;
  ctx->group = G;
  ctx->rows_per_item = ctx->f16 ? attention_tc_rows_per_item(G) : 64;
  auto bail = [&](int rc) {
    g_noctx_err = ctx->err.empty() ? "model_load failed (code " + std::to_string(rc) + ")" : ctx->err;
    duolm_destroy(ctx);
    return rc;
  };
  if (cudaSetDevice(device) != cudaSuccess) return bail(DUOLM_E_CUDA);
  if (cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return bail(DUOLM_E_CUDA);
  ctx->gemm_grid = ctx->num_sms & ~1;
  if (cuda_stream) {
    ctx->stream = static_cast<cudaStream_t>(cuda_stream);
  } else {
    if (cudaStreamCreateWithFlags(&ctx->stream, cudaStreamNonBlocking) != cudaSuccess) return bail(DUOLM_E_CUDA);
    ctx->own_stream = true;
  }
  if (cudaEventCreateWithFlags(&ctx->plan_ev, cudaEventDisableTiming) != cudaSuccess) return bail(DUOLM_E_CUDA);
  int rc;
  const int64_t D = d.d, hd = d.head_dim, F = d.ffn;
  auto W = [&](int i) { return host_weights[i]; };

  // norm gains (fp32 on the device): per layer attn, q, k, mlp; then final
  {
    std::vector<float> g;
    auto push = [&](const void* p, int64_t n) {
      for (int64_t i = 0; i < n; ++i)
        g.push_back(ctx->f16 ? bf16_bits_to_float(static_cast<const uint16_t*>(p)[i]) : static_cast<const float*>(p)[i]);
    };
    ctx->layers.resize(d.n_layers);
    for (int l = 0; l < d.n_layers; ++l) {
      const int b = 1 + kPerLayer * l;
      LayerW& L = ctx->layers[l];
      L.g_attn = (int64_t)g.size(); push(W(b + 0), D);
      L.g_q = (int64_t)g.size(); push(W(b + 4), hd);
      L.g_k = (int64_t)g.size(); push(W(b + 5), hd);
      L.g_mlp = (int64_t)g.size(); push(W(b + 7), D);
    }
    ctx->g_final = (int64_t)g.size();
    push(W(1 + kPerLayer * d.n_layers), D);
    if ((rc = dalloc(ctx, &ctx->gains, g.size() * 4))) return bail(rc);
    if (cudaMemcpy(ctx->gains, g.data(), g.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) return bail(DUOLM_E_CUDA);
    std::vector<float> hw(D);
    for (int64_t i = 0; i < D; ++i)
      hw[i] = ctx->f16 ? bf16_bits_to_float(static_cast<const uint16_t*>(W(2 + kPerLayer * d.n_layers))[i])
                       : static_cast<const float*>(W(2 + kPerLayer * d.n_layers))[i];
    if ((rc = dalloc(ctx, &ctx->head, D * 4))) return bail(rc);
    if (cudaMemcpy(ctx->head, hw.data(), D * 4, cudaMemcpyHostToDevice) != cudaSuccess) return bail(DUOLM_E_CUDA);
  }
  // embedding: kept in its storage type, read only by the gather
  {
    const int64_t bytes = (int64_t)d.vocab * D * (ctx->f16 ? 2 : 4);
    if ((rc = dalloc(ctx, &ctx->embed, bytes))) return bail(rc);
    if (cudaMemcpy(ctx->embed, W(0), bytes, cudaMemcpyHostToDevice) != cudaSuccess) return bail(DUOLM_E_CUDA);
  }
  // projection matrices
  for (int l = 0; l < d.n_layers; ++l) {
    const int b = 1 + kPerLayer * l;
    LayerW& L = ctx->layers[l];
    if (ctx->f16) {
      auto P = [&](int i, int64_t rows) { return Part{static_cast<const uint16_t*>(W(i)), rows}; };
      if ((rc = upload_f16(ctx, {P(b + 1, ctx->qd), P(b + 2, ctx->kd), P(b + 3, ctx->kd)}, D, &L.wqkv, &L.s_qkv, "wqkv")))
        return bail(rc);
      if ((rc = upload_f16(ctx, {P(b + 6, D)}, ctx->qd, &L.wo, &L.s_o, "wo"))) return bail(rc);
      std::vector<Part> gu;
      for (int64_t blk = 0; blk < F / 128; ++blk) {
        gu.push_back(Part{static_cast<const uint16_t*>(W(b + 8)) + blk * 128 * D, 128});
        gu.push_back(Part{static_cast<const uint16_t*>(W(b + 9)) + blk * 128 * D, 128});
      }
      if ((rc = upload_f16(ctx, gu, D, &L.wgu, &L.s_gu, "w_gate/w_up"))) return bail(rc);
      if ((rc = upload_f16(ctx, {P(b + 10, D)}, F, &L.wd, &L.s_d, "w_down"))) return bail(rc);
      char e[256];
      // B tiles are loaded in halves of 128 rows, one per CTA of a pair
      if (!make_tmap_f16_2d(&L.tm_qkv, L.wqkv, D, ctx->qd + 2 * ctx->kd, 64, 128, e, sizeof e) ||
          !make_tmap_f16_2d(&L.tm_o, L.wo, ctx->qd, D, 64, 128, e, sizeof e) ||
          !make_tmap_f16_2d(&L.tm_gu, L.wgu, D, 2 * F, 64, 128, e, sizeof e) ||
          !make_tmap_f16_2d(&L.tm_d, L.wd, F, D, 64, 128, e, sizeof e) ||
          !make_tmap_f16_2d(&L.tm_qkv_n64, L.wqkv, D, ctx->qd + 2 * ctx->kd, 64, kNarrowQkv / 2, e, sizeof e)) {
        fail(ctx, DUOLM_E_CUDA, "%s", e);
        return bail(DUOLM_E_CUDA);
      }
    } else {
      auto P = [&](int i, int64_t n) { return std::make_pair(static_cast<const float*>(W(i)), n); };
      if ((rc = upload_f32(ctx, {P(b + 1, ctx->qd * D), P(b + 2, ctx->kd * D), P(b + 3, ctx->kd * D)}, &L.wqkv)))
        return bail(rc);
      if ((rc = upload_f32(ctx, {P(b + 6, D * ctx->qd)}, &L.wo))) return bail(rc);
      if ((rc = upload_f32(ctx, {P(b + 8, F * D), P(b + 9, F * D)}, &L.wgu))) return bail(rc);
      if ((rc = upload_f32(ctx, {P(b + 10, D * F)}, &L.wd))) return bail(rc);
    }
  }
  // RoPE table: (cos, sin) of pos * theta^(-2i/hd), computed in double,
  // frequency-major [hd/2][kMaxPos] so that neighbouring tokens read
  // neighbouring entries
  {
    const int64_t half = hd / 2;
    std::vector<float2> t((size_t)(kMaxPos * half));
    for (int64_t i = 0; i < half; ++i) {
      const double inv = std::pow((double)d.rope_theta, -2.0 * (double)i / (double)hd);
      for (int64_t p = 0; p < kMaxPos; ++p) {
        const double a = (double)p * inv;
        t[i * kMaxPos + p] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
    if ((rc = dalloc(ctx, &ctx->rope, t.size() * sizeof(float2)))) return bail(rc);
    if (cudaMemcpy(ctx->rope, t.data(), t.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(DUOLM_E_CUDA);
  }
  if ((rc = dalloc(ctx, &ctx->status, sizeof(DevStatus)))) return bail(rc);
  if (cudaMemset(ctx->status, 0, sizeof(DevStatus)) != cudaSuccess) return bail(DUOLM_E_CUDA);
  if (ctx->f16 && (gemm_tc_setup() != cudaSuccess || attention_tc_setup() != cudaSuccess)) return bail(DUOLM_E_CUDA);
  *out = ctx;
  return 0;
}

int duolm_vid_table_load(duolm_ctx* ctx, const uint16_t* rows, int64_t n_items) {
  if (!ctx || (!rows && n_items > 0) || n_items < 0 || n_items > INT32_MAX - ctx->desc.vocab)
    return fail(ctx, DUOLM_E_ARG, "vid_table_load: bad arguments");
  CK(cudaSetDevice(ctx->device));
  CK(cudaStreamSynchronize(ctx->stream));
  invalidate_graph(ctx);
  dfree(ctx->table);
  ctx->n_items = 0;
  if (int rc = dalloc(ctx, &ctx->table, n_items * ctx->desc.d * 2)) return rc;
  CK(cudaMemcpy(ctx->table, rows, n_items * ctx->desc.d * 2, cudaMemcpyHostToDevice));
  ctx->n_items = n_items;
  return 0;
}

int duolm_vid_table_build(duolm_ctx* ctx, const float* a_rows, int64_t n_items, double gamma, double rho) {
  if (!ctx || (!a_rows && n_items > 0) || n_items < 0 || n_items > INT32_MAX - ctx->desc.vocab ||
      !std::isfinite(gamma) || !std::isfinite(rho))
    return fail(ctx, DUOLM_E_ARG, "vid_table_build: bad arguments");
  CK(cudaSetDevice(ctx->device));
  CK(cudaStreamSynchronize(ctx->stream));
  invalidate_graph(ctx);
  dfree(ctx->table);
  ctx->n_items = 0;
  const int64_t D = ctx->desc.d;
  if (int rc = dalloc(ctx, &ctx->table, n_items * D * 2)) return rc;
  const int64_t chunk = std::max<int64_t>(1, (int64_t(256) << 20) / (D * 4));
  float* tmp = nullptr;
  if (int rc = dalloc(ctx, &tmp, std::min(chunk, std::max<int64_t>(n_items, 1)) * D * 4)) return rc;
  const double scale_num = std::exp(gamma) * rho;
  for (int64_t r0 = 0; r0 < n_items; r0 += chunk) {
    const int64_t n = std::min(chunk, n_items - r0);
    cudaError_t e = cudaMemcpyAsync(tmp, a_rows + r0 * D, n * D * 4, cudaMemcpyHostToDevice, ctx->stream);
    if (e == cudaSuccess) e = table_build(tmp, n, (int)D, scale_num, ctx->table + r0 * D, ctx->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
    if (e != cudaSuccess) {
      cudaFree(tmp);
      return fail(ctx, DUOLM_E_CUDA, "vid_table_build: %s", cudaGetErrorString(e));
    }
  }
  cudaFree(tmp);
  ctx->n_items = n_items;
  return 0;
}

int duolm_embedding_rho(duolm_ctx* ctx, double* rho_out) {
  if (!ctx || !rho_out) return fail(ctx, DUOLM_E_ARG, "embedding_rho: bad arguments");
  CK(cudaSetDevice(ctx->device));
  if (!ctx->rho_buf)
    if (int rc = dalloc(ctx, &ctx->rho_buf, ((int64_t)ctx->desc.vocab + 1) * 8)) return rc;
  CK(embed_rho(ctx->embed, ctx->f16, ctx->desc.vocab, ctx->desc.d, ctx->rho_buf + 1, ctx->rho_buf, ctx->stream));
  CK(cudaMemcpyAsync(rho_out, ctx->rho_buf, 8, cudaMemcpyDeviceToHost, ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  return 0;
}

int duolm_reserve(duolm_ctx* ctx, int64_t max_tokens, int64_t max_requests, int64_t max_candidates) {
  if (!ctx || max_tokens < 0 || max_requests < 0 || max_candidates < 0)
    return fail(ctx, DUOLM_E_ARG, "reserve: bad arguments");
  CK(cudaSetDevice(ctx->device));
  return reserve_impl(ctx, max_tokens, max_requests, max_candidates);
}

}  // extern "C"

namespace {

// duolm_prepare and duolm_prepare_cached.  slot == nullptr: no request
// continues a cached prefix.
int prepare_impl(duolm_ctx* ctx, int n_requests, const int32_t* prefix_ids, const int64_t* prefix_offsets,
                 const int32_t* branch_ids, const int64_t* cand_offsets, int branch_len, int mode,
                 const int32_t* slot, const int32_t* cached, const int32_t* keep) {
  if (!ctx) return DUOLM_E_ARG;
  ctx->prepared = false;
  if (n_requests < 1 || !prefix_ids || !prefix_offsets || !branch_ids || !cand_offsets)
    return fail(ctx, DUOLM_E_ARG, "prepare: null pointer or no requests");
  if (mode != DUOLM_MODE_MIS && mode != DUOLM_MODE_INDEPENDENT) return fail(ctx, DUOLM_E_ARG, "prepare: bad mode");
  if (branch_len < 1) return fail(ctx, DUOLM_E_EMPTY, "prepare: branch_len must be >= 1");
  if (ctx->f16 && branch_len > ctx->rows_per_item)
    return fail(ctx, DUOLM_E_ARG, "prepare: branch_len %d above %d", branch_len, ctx->rows_per_item);
  if (prefix_offsets[0] != 0 || cand_offsets[0] != 0)
    return fail(ctx, DUOLM_E_OFFSETS, "prepare: offsets must start at 0");
  if (slot && (!cached || !keep)) return fail(ctx, DUOLM_E_ARG, "prepare: null cached or keep array");
  const int64_t vocab = ctx->desc.vocab, id_end = vocab + ctx->n_items;
  std::vector<ReqView> reqs;
  std::vector<int> slot_uses(slot ? ctx->n_slots : 0, 0), slot_writers(slot ? ctx->n_slots : 0, 0);
  int64_t n_cand = 0;
  for (int q = 0; q < n_requests; ++q) {
    const int64_t L = prefix_offsets[q + 1] - prefix_offsets[q];
    const int64_t K = cand_offsets[q + 1] - cand_offsets[q];
    if (L < 0 || K < 0) return fail(ctx, DUOLM_E_OFFSETS, "prepare: offsets decrease at request %d", q);
    const int sl = slot ? slot[q] : -1;
    int64_t c = 0, kp = 0;
    if (sl >= 0) {
      if (ctx->n_slots == 0) return fail(ctx, DUOLM_E_STATE, "prepare: request %d names slot %d but no KV store is reserved", q, sl);
      if (sl >= ctx->n_slots) return fail(ctx, DUOLM_E_ARG, "prepare: request %d slot %d (store has %d)", q, sl, ctx->n_slots);
      if (mode != DUOLM_MODE_MIS) return fail(ctx, DUOLM_E_ARG, "prepare: cached prefixes need the multi-item mode");
      c = cached[q];
      kp = keep[q];
      if (c < 0 || kp < 0 || kp > L)
        return fail(ctx, DUOLM_E_ARG, "prepare: request %d cached %lld keep %lld of %lld new tokens", q, (long long)c,
                    (long long)kp, (long long)L);
      if (c > ctx->slot_len[sl])
        return fail(ctx, DUOLM_E_STATE, "prepare: request %d reuses %lld tokens of slot %d, which holds %d", q,
                    (long long)c, sl, ctx->slot_len[sl]);
      if (c + kp > ctx->slot_tokens)
        return fail(ctx, DUOLM_E_CAPACITY, "prepare: request %d keeps slot %d rows up to %lld (slot size %d)", q, sl,
                    (long long)(c + kp), ctx->slot_tokens);
      ++slot_uses[sl];
      if (kp > 0) ++slot_writers[sl];
      if (slot_writers[sl] > 0 && slot_uses[sl] > 1)
        return fail(ctx, DUOLM_E_ARG, "prepare: slot %d is written by one request of the batch and used by another", sl);
    } else if (slot && (cached[q] != 0 || keep[q] != 0)) {
      return fail(ctx, DUOLM_E_ARG, "prepare: request %d has no slot but cached or keep set", q);
    }
    if ((L == 0 && c == 0) || K == 0)
      return fail(ctx, DUOLM_E_EMPTY, "prepare: request %d has L=%lld K=%lld", q, (long long)(c + L), (long long)K);
    if (c + L + branch_len > kMaxPos)
      return fail(ctx, DUOLM_E_CAPACITY, "prepare: request %d needs positions up to %lld (limit %d)", q,
                  (long long)(c + L + branch_len), kMaxPos);
    const int32_t* pre = prefix_ids + prefix_offsets[q];
    const int32_t* br = branch_ids + cand_offsets[q] * branch_len;
    for (int64_t i = 0; i < L; ++i)
      if (pre[i] < 0 || pre[i] >= id_end)
        return fail(ctx, DUOLM_E_ID, "prepare: request %d prefix token %lld has id %d (valid: 0..%lld)", q,
                    (long long)i, pre[i], (long long)id_end - 1);
    for (int64_t i = 0; i < K * branch_len; ++i)
      if (br[i] < 0 || br[i] >= id_end)
        return fail(ctx, DUOLM_E_ID, "prepare: request %d branch token %lld has id %d (valid: 0..%lld)", q,
                    (long long)i, br[i], (long long)id_end - 1);
    if (mode == DUOLM_MODE_MIS) {
      reqs.push_back(ReqView{pre, L, br, K, (int)c, sl, (int)kp});
    } else {
      for (int64_t j = 0; j < K; ++j) reqs.push_back(ReqView{pre, L, br + j * branch_len, 1, 0, -1, 0});
    }
    n_cand += K;
  }
  int64_t T = 0;
  for (auto& r : reqs) T += r.L + r.K * branch_len;
  if (T > INT32_MAX / 2) return fail(ctx, DUOLM_E_CAPACITY, "prepare: %lld tokens", (long long)T);
  CK(cudaSetDevice(ctx->device));
  if (int rc = reserve_impl(ctx, std::max(T, ctx->cap_T), std::max<int64_t>((int64_t)reqs.size(), ctx->cap_R),
                            std::max(n_cand, ctx->cap_C)))
    return rc;

  // ---- fill the host plan
  CK(cudaEventSynchronize(ctx->plan_ev));  // the previous copy out of plan_host is done
  const int64_t R = (int64_t)reqs.size();
  PlanHdr hdr{};
  hdr.n_tokens = (int32_t)T;
  hdr.n_req = (int32_t)R;
  hdr.n_cand = (int32_t)n_cand;
  hdr.branch_len = branch_len;
  int64_t off = sizeof(PlanHdr);
  hdr.off_ids = off; off += align16(T * 4);
  hdr.off_pos = off; off += align16(T * 4);
  hdr.off_treq = off; off += align16(T * 4);
  hdr.off_req = off; off += align16(R * 16);
  hdr.off_cand = off; off += align16(n_cand * 4);
  hdr.off_items = off;
  char* base = ctx->plan_host;
  int32_t* ids = reinterpret_cast<int32_t*>(base + hdr.off_ids);
  int32_t* pos = reinterpret_cast<int32_t*>(base + hdr.off_pos);
  int32_t* treq = reinterpret_cast<int32_t*>(base + hdr.off_treq);
  int4* rq = reinterpret_cast<int4*>(base + hdr.off_req);
  int32_t* cand = reinterpret_cast<int32_t*>(base + hdr.off_cand);
  int2* rx = ctx->reqx_host;               // {cached, first store row}
  int2* ap = ctx->reqx_host + ctx->cap_R;  // {rows kept, store row of the first}
  ctx->req_host.assign(R, int4{0, 0, 0, 0});
  ctx->slot_update.clear();
  int64_t t = 0, c = 0;
  for (int64_t r = 0; r < R; ++r) {
    const ReqView& v = reqs[r];
    // request-local indices count from the first cached token: the prefix
    // is c + L tokens long, the batch holds indices c .. c + L - 1
    const int64_t Lt = v.cached + v.L;
    rq[r] = int4{(int)t, (int)Lt, (int)v.K, (int)c};
    ctx->req_host[r] = rq[r];
    const int row0 = v.slot >= 0 ? v.slot * ctx->slot_tokens : 0;
    rx[r] = int2{v.cached, row0};
    ap[r] = int2{v.keep, row0 + v.cached};
    if (v.slot >= 0 && v.keep > 0) ctx->slot_update.push_back({v.slot, v.cached + v.keep});
    for (int64_t i = 0; i < v.L; ++i, ++t) {
      ids[t] = v.prefix[i];
      pos[t] = (int32_t)(v.cached + i);  // prefix token i at its position in the whole prefix
      treq[t] = (int32_t)r;
    }
    for (int64_t j = 0; j < v.K; ++j) {
      for (int64_t i = 0; i < branch_len; ++i, ++t) {
        ids[t] = v.branch[j * branch_len + i];
        pos[t] = (int32_t)(Lt + i);  // every branch at logical position L (+ i inside the branch)
        treq[t] = (int32_t)r;
      }
      cand[c++] = (int32_t)(t - 1);  // the branch's last token is scored
    }
  }
  // attention work list and its CTA ranges (fp16 path)
  int64_t n_items = 0;
  if (ctx->f16) {
    const int G = ctx->num_sms;
    const int H = ctx->desc.n_kv_heads;
    std::vector<int32_t> cta_range((size_t)G + 1);
    // A batch whose items would fill at most half the CTAs (one or two
    // requests) gets items of one query sub-tile instead of two: twice as
    // many CTAs share the work, and each runs one softmax chain.
    int rows = ctx->rows_per_item;
    if (2 * branch_len <= rows) {
      const int per = (rows / branch_len) * branch_len;
      int64_t n_full = 0;
      for (int64_t r = 0; r < R; ++r)
        n_full += ((int64_t)rq[r].z * branch_len + per - 1) / per + (rq[r].y - rx[r].x + rows - 1) / rows;
      if (2 * n_full * H <= G) rows /= 2;
    }
    n_items = plan_attention(rq, rx, R, H, rows, branch_len, G, ctx->cap_I,
                             reinterpret_cast<int4*>(base + hdr.off_items), cta_range.data());
    if (n_items < 0 && rows != ctx->rows_per_item) {
      rows = ctx->rows_per_item;
      n_items = plan_attention(rq, rx, R, H, rows, branch_len, G, ctx->cap_I,
                               reinterpret_cast<int4*>(base + hdr.off_items), cta_range.data());
    }
    if (n_items < 0) return fail(ctx, DUOLM_E_CAPACITY, "prepare: work list overflow");
    hdr.att_rows = rows;
    hdr.att_ctas = G;
    hdr.off_cta = hdr.off_items + align16(n_items * 16);
    memcpy(base + hdr.off_cta, cta_range.data(), (size_t)(G + 1) * 4);
  }
  hdr.n_items = (int32_t)n_items;
  const int64_t bytes = hdr.att_ctas ? hdr.off_cta + align16((int64_t)(hdr.att_ctas + 1) * 4)
                                     : hdr.off_items + align16(n_items * 16);
  memcpy(base, &hdr, sizeof hdr);
  CK(cudaMemcpyAsync(ctx->plan_dev, base, bytes, cudaMemcpyHostToDevice, ctx->stream));
  CK(cudaMemcpyAsync(ctx->reqx, rx, R * sizeof(int2), cudaMemcpyHostToDevice, ctx->stream));
  CK(cudaMemcpyAsync(ctx->append, ap, R * sizeof(int2), cudaMemcpyHostToDevice, ctx->stream));
  CK(cudaEventRecord(ctx->plan_ev, ctx->stream));
  ctx->hdr = hdr;
  ctx->n_tokens = T;
  ctx->n_cand = n_cand;
  ctx->n_req = (int)R;
  ctx->branch_len = branch_len;
  ctx->prepared = true;
  return 0;
}

}  // namespace

extern "C" {

int duolm_prepare(duolm_ctx* ctx, int n_requests, const int32_t* prefix_ids, const int64_t* prefix_offsets,
                  const int32_t* branch_ids, const int64_t* cand_offsets, int branch_len, int mode) {
  return prepare_impl(ctx, n_requests, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len, mode,
                      nullptr, nullptr, nullptr);
}

int duolm_prepare_cached(duolm_ctx* ctx, int n_requests, const int32_t* prefix_ids, const int64_t* prefix_offsets,
                         const int32_t* branch_ids, const int64_t* cand_offsets, int branch_len, const int32_t* slot,
                         const int32_t* cached, const int32_t* keep) {
  if (!ctx) return DUOLM_E_ARG;
  if (!slot) {
    ctx->prepared = false;
    return fail(ctx, DUOLM_E_ARG, "prepare_cached: null slot array");
  }
  return prepare_impl(ctx, n_requests, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len,
                      DUOLM_MODE_MIS, slot, cached, keep);
}

int duolm_kv_store_reserve(duolm_ctx* ctx, int n_slots, int slot_tokens) {
  if (!ctx) return DUOLM_E_ARG;
  if (n_slots < 0 || slot_tokens < 0 || (n_slots > 0 && slot_tokens < 1) || slot_tokens > kMaxPos)
    return fail(ctx, DUOLM_E_ARG, "kv_store_reserve: %d slots of %d tokens", n_slots, slot_tokens);
  const auto& d = ctx->desc;
  const int64_t rows = (int64_t)n_slots * slot_tokens;
  if (rows * d.n_kv_heads + 256 > INT32_MAX)  // TMA row coordinates are int32
    return fail(ctx, DUOLM_E_CAPACITY, "kv_store_reserve: %lld rows per layer", (long long)(rows * d.n_kv_heads));
  CK(cudaSetDevice(ctx->device));
  CK(cudaStreamSynchronize(ctx->stream));
  invalidate_graph(ctx);
  ctx->prepared = false;
  dfree(ctx->ks);
  dfree(ctx->vs);
  ctx->tm_ks.clear();
  ctx->tm_vs.clear();
  ctx->slot_len.clear();
  ctx->slot_update.clear();
  ctx->n_slots = ctx->slot_tokens = 0;
  ctx->layer_store_elems = 0;
  if (n_slots == 0) return 0;
  const int64_t es = ctx->f16 ? 2 : 4;
  const int64_t elems = rows * d.n_kv_heads * d.head_dim;
  const int64_t bytes = elems * d.n_layers * es;
  int rc;
  if ((rc = dalloc(ctx, &ctx->ks, bytes)) || (rc = dalloc(ctx, &ctx->vs, bytes))) {
    dfree(ctx->ks);
    dfree(ctx->vs);
    return rc;
  }
  // zero rows are finite: a store tile's masked rows never hold NaN
  CK(cudaMemset(ctx->ks, 0, bytes));
  CK(cudaMemset(ctx->vs, 0, bytes));
  if (ctx->f16) {
    ctx->tm_ks.resize(d.n_layers);
    ctx->tm_vs.resize(d.n_layers);
    char e[256];
    for (int l = 0; l < d.n_layers; ++l)
      if (!make_tmap_f16_2d(&ctx->tm_ks[l], static_cast<__half*>(ctx->ks) + l * elems, 128,
                            (uint64_t)d.n_kv_heads * rows, 64, 128, e, sizeof e) ||
          !make_tmap_f16_2d(&ctx->tm_vs[l], static_cast<__half*>(ctx->vs) + l * elems, 128,
                            (uint64_t)d.n_kv_heads * rows, 64, 128, e, sizeof e)) {
        dfree(ctx->ks);
        dfree(ctx->vs);
        return fail(ctx, DUOLM_E_CUDA, "%s", e);
      }
  }
  ctx->n_slots = n_slots;
  ctx->slot_tokens = slot_tokens;
  ctx->layer_store_elems = elems;
  ctx->slot_len.assign(n_slots, 0);
  return 0;
}

int duolm_kv_slot_length(const duolm_ctx* ctx, int slot) {
  if (!ctx || slot < 0 || slot >= ctx->n_slots) return DUOLM_E_ARG;
  return ctx->slot_len[slot];
}

int duolm_execute(duolm_ctx* ctx) {
  if (!ctx) return DUOLM_E_ARG;
  if (!ctx->prepared) return fail(ctx, DUOLM_E_STATE, "execute: nothing prepared");
  CK(cudaSetDevice(ctx->device));
  // the slots this batch appends to hold its rows once the launches below
  // have run (work on the same stream sees them); the lengths change only
  // after the whole pass was enqueued, so a failed call leaves them as they were
  auto commit_slots = [ctx]() {
    for (const auto& u : ctx->slot_update) ctx->slot_len[u.first] = u.second;
  };
  if (!ctx->use_graph) {
    CK(launch_forward(ctx, ctx->desc.n_layers, true, &ctx->launches));
    commit_slots();
    return 0;
  }
  if (!ctx->graph_valid) {
    cudaGraph_t g = nullptr;
    CK(cudaStreamBeginCapture(ctx->stream, cudaStreamCaptureModeThreadLocal));
    int64_t n = 0;
    cudaError_t le = launch_forward(ctx, ctx->desc.n_layers, true, &n);
    cudaError_t ce = cudaStreamEndCapture(ctx->stream, &g);
    if (le != cudaSuccess || ce != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      return fail(ctx, DUOLM_E_CUDA, "execute: graph capture failed: %s",
                  cudaGetErrorString(le != cudaSuccess ? le : ce));
    }
    cudaError_t ie = cudaGraphInstantiate(&ctx->gexec, g, 0);
    cudaGraphDestroy(g);
    if (ie != cudaSuccess) return fail(ctx, DUOLM_E_CUDA, "execute: graph instantiate: %s", cudaGetErrorString(ie));
    ctx->graph_valid = true;
    ctx->launches = n;
  }
  CK(cudaGraphLaunch(ctx->gexec, ctx->stream));
  commit_slots();
  return 0;
}

const float* duolm_scores_device(const duolm_ctx* ctx) { return ctx ? ctx->scores : nullptr; }

int duolm_sync(duolm_ctx* ctx) {
  if (!ctx) return DUOLM_E_ARG;
  CK(cudaSetDevice(ctx->device));
  CK(cudaStreamSynchronize(ctx->stream));
  return check_status(ctx);
}

int duolm_score(duolm_ctx* ctx, int n_requests, const int32_t* prefix_ids, const int64_t* prefix_offsets,
                const int32_t* branch_ids, const int64_t* cand_offsets, int branch_len, int mode, float* scores_out) {
  if (!ctx) return DUOLM_E_ARG;
  if (!scores_out) return fail(ctx, DUOLM_E_ARG, "score: null scores_out");
  if (mode == DUOLM_MODE_INDEPENDENT && n_requests >= 1 && prefix_offsets && cand_offsets && branch_len >= 1) {
    // Expanded independent batches can be ~100x the packed size: run them in
    // chunks of at most max(capacity, 2^18) tokens.
    const int64_t limit = std::max<int64_t>(ctx->cap_T, int64_t(1) << 18);
    int64_t total = 0;
    for (int q = 0; q < n_requests; ++q)
      total += (cand_offsets[q + 1] - cand_offsets[q]) * (prefix_offsets[q + 1] - prefix_offsets[q] + branch_len);
    if (total > limit && prefix_ids && branch_ids) {
      std::vector<int32_t> pids, bids;
      std::vector<int64_t> poff{0}, coff{0};
      int64_t tok = 0, out0 = 0, nout = 0;
      auto flush = [&]() -> int {
        if (coff.size() < 2) return 0;
        const int nr = (int)coff.size() - 1;
        int rc = duolm_prepare(ctx, nr, pids.data(), poff.data(), bids.data(), coff.data(), branch_len, mode);
        if (!rc) rc = duolm_execute(ctx);
        if (rc) return rc;
        CK(cudaMemcpyAsync(scores_out + out0, ctx->scores, nout * 4, cudaMemcpyDeviceToHost, ctx->stream));
        if ((rc = duolm_sync(ctx))) return rc;
        out0 += nout;
        nout = 0;
        tok = 0;
        pids.clear();
        bids.clear();
        poff.assign(1, 0);
        coff.assign(1, 0);
        return 0;
      };
      for (int q = 0; q < n_requests; ++q) {
        const int64_t L = prefix_offsets[q + 1] - prefix_offsets[q];
        for (int64_t c = cand_offsets[q]; c < cand_offsets[q + 1]; ++c) {
          if (tok + L + branch_len > limit && nout > 0)
            if (int rc = flush()) return rc;
          // one request per candidate: the prefix again, then its branch
          pids.insert(pids.end(), prefix_ids + prefix_offsets[q], prefix_ids + prefix_offsets[q + 1]);
          poff.push_back((int64_t)pids.size());
          bids.insert(bids.end(), branch_ids + c * branch_len, branch_ids + (c + 1) * branch_len);
          coff.push_back(coff.back() + 1);
          tok += L + branch_len;
          ++nout;
        }
      }
      return flush();
    }
  }
  int rc = duolm_prepare(ctx, n_requests, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len, mode);
  if (!rc) rc = duolm_execute(ctx);
  if (rc) return rc;
  CK(cudaMemcpyAsync(scores_out, ctx->scores, ctx->n_cand * 4, cudaMemcpyDeviceToHost, ctx->stream));
  return duolm_sync(ctx);
}

int duolm_score_cached(duolm_ctx* ctx, int n_requests, const int32_t* prefix_ids, const int64_t* prefix_offsets,
                       const int32_t* branch_ids, const int64_t* cand_offsets, int branch_len, const int32_t* slot,
                       const int32_t* cached, const int32_t* keep, float* scores_out) {
  if (!ctx) return DUOLM_E_ARG;
  if (!scores_out) return fail(ctx, DUOLM_E_ARG, "score_cached: null scores_out");
  int rc = duolm_prepare_cached(ctx, n_requests, prefix_ids, prefix_offsets, branch_ids, cand_offsets, branch_len,
                                slot, cached, keep);
  if (!rc) rc = duolm_execute(ctx);
  if (rc) return rc;
  CK(cudaMemcpyAsync(scores_out, ctx->scores, ctx->n_cand * 4, cudaMemcpyDeviceToHost, ctx->stream));
  return duolm_sync(ctx);
}

int duolm_set_pdl(duolm_ctx* ctx, int enabled) {
  if (!ctx) return DUOLM_E_ARG;
  if (ctx->use_pdl != (enabled != 0)) invalidate_graph(ctx);
  ctx->use_pdl = enabled != 0;
  return 0;
}

int duolm_set_graph(duolm_ctx* ctx, int enabled) {
  if (!ctx) return DUOLM_E_ARG;
  ctx->use_graph = enabled != 0;
  return 0;
}

int64_t duolm_launches_per_execute(const duolm_ctx* ctx) { return ctx ? ctx->launches : 0; }

const char* duolm_last_error(const duolm_ctx* ctx) { return ctx ? ctx->err.c_str() : g_noctx_err.c_str(); }

void duolm_destroy(duolm_ctx* ctx) {
  if (!ctx) return;
  cudaSetDevice(ctx->device);
  if (ctx->stream) cudaStreamSynchronize(ctx->stream);
  invalidate_graph(ctx);
  free_workspace(ctx);
  dfree(ctx->ks);
  dfree(ctx->vs);
  for (auto& L : ctx->layers) {
    dfree(L.wqkv);
    dfree(L.wo);
    dfree(L.wgu);
    dfree(L.wd);
  }
  dfree(ctx->embed);
  dfree(ctx->gains);
  dfree(ctx->head);
  dfree(ctx->table);
  dfree(ctx->rope);
  dfree(ctx->status);
  dfree(ctx->rho_buf);
  dfree(ctx->gather_hdr);
  if (ctx->plan_ev) cudaEventDestroy(ctx->plan_ev);
  if (ctx->own_stream && ctx->stream) cudaStreamDestroy(ctx->stream);
  delete ctx;
}

int duolm_debug_layout(duolm_ctx* ctx, int64_t* n_tokens, int32_t* ids_out, int32_t* pos_out) {
  if (!ctx) return DUOLM_E_ARG;
  if (!ctx->prepared) return fail(ctx, DUOLM_E_STATE, "debug_layout: nothing prepared");
  CK(cudaSetDevice(ctx->device));
  if (n_tokens) *n_tokens = ctx->n_tokens;
  if (ids_out)
    CK(cudaMemcpyAsync(ids_out, ctx->plan_dev + ctx->hdr.off_ids, ctx->n_tokens * 4, cudaMemcpyDeviceToHost, ctx->stream));
  if (pos_out)
    CK(cudaMemcpyAsync(pos_out, ctx->plan_dev + ctx->hdr.off_pos, ctx->n_tokens * 4, cudaMemcpyDeviceToHost, ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  return 0;
}

int duolm_debug_mask(duolm_ctx* ctx, int request, uint8_t* out) {
  if (!ctx || !out) return fail(ctx, DUOLM_E_ARG, "debug_mask: bad arguments");
  if (!ctx->prepared) return fail(ctx, DUOLM_E_STATE, "debug_mask: nothing prepared");
  if (request < 0 || request >= ctx->n_req) return fail(ctx, DUOLM_E_ARG, "debug_mask: request out of range");
  CK(cudaSetDevice(ctx->device));
  const int4 r = ctx->req_host[request];
  const int64_t tq = r.y + (int64_t)r.z * ctx->branch_len;
  uint8_t* dbuf = nullptr;
  if (int rc = dalloc(ctx, &dbuf, tq * tq)) return rc;
  cudaError_t e = debug_mask(reinterpret_cast<const PlanHdr*>(ctx->plan_dev), request, dbuf, tq, ctx->stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, dbuf, tq * tq, cudaMemcpyDeviceToHost, ctx->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
  cudaFree(dbuf);
  if (e != cudaSuccess) return fail(ctx, DUOLM_E_CUDA, "debug_mask: %s", cudaGetErrorString(e));
  return 0;
}

int duolm_debug_residual(duolm_ctx* ctx, int n_layers, float* x_out) {
  if (!ctx || !x_out || n_layers < 0 || n_layers > ctx->desc.n_layers)
    return fail(ctx, DUOLM_E_ARG, "debug_residual: bad arguments");
  if (!ctx->prepared) return fail(ctx, DUOLM_E_STATE, "debug_residual: nothing prepared");
  CK(cudaSetDevice(ctx->device));
  int64_t n = 0;
  CK(launch_forward(ctx, n_layers, false, &n));
  CK(cudaMemcpyAsync(x_out, ctx->x, ctx->n_tokens * ctx->desc.d * 4, cudaMemcpyDeviceToHost, ctx->stream));
  return duolm_sync(ctx);
}

int64_t duolm_plan_bytes(const duolm_ctx* ctx) {
  if (!ctx || !ctx->prepared) return 0;
  const int64_t plan = ctx->hdr.att_ctas ? ctx->hdr.off_cta + align16((int64_t)(ctx->hdr.att_ctas + 1) * 4)
                                         : ctx->hdr.off_items + align16((int64_t)ctx->hdr.n_items * 16);
  return plan + 2 * (int64_t)ctx->n_req * (int64_t)sizeof(int2);  // + the cached-prefix and append records
}

int duolm_debug_gemm(duolm_ctx* ctx, int layer, int which, const uint16_t* a, float* out) {
  if (!ctx || !a || !out || layer < 0 || layer >= ctx->desc.n_layers || which < 0 || which > 7 || !ctx->f16)
    return fail(ctx, DUOLM_E_ARG, "debug_gemm: bad arguments");
  const bool split = which >= 4;  // split-K: four K-slices summed by the reduction kernel
  which &= 3;
  if (!ctx->prepared) return fail(ctx, DUOLM_E_STATE, "debug_gemm: nothing prepared");
  CK(cudaSetDevice(ctx->device));
  const auto& d = ctx->desc;
  const LayerW& L = ctx->layers[layer];
  const int K = which == 1 ? ctx->qd : which == 3 ? d.ffn : d.d;
  const int N = which == 0 ? ctx->qd + 2 * ctx->kd : which == 2 ? 2 * d.ffn : d.d;
  const CUtensorMap& ta = which == 1 ? ctx->tm_oact : which == 3 ? ctx->tm_h : ctx->tm_xn;
  void* abuf = which == 1 ? ctx->o : which == 3 ? ctx->h : ctx->xn;
  const CUtensorMap& tb = which == 0 ? L.tm_qkv : which == 1 ? L.tm_o : which == 2 ? L.tm_gu : L.tm_d;
  const float sc = which == 0 ? L.s_qkv : which == 1 ? L.s_o : which == 2 ? L.s_gu : L.s_d;
  const int64_t T = ctx->n_tokens;
  constexpr int kSlices = 4;
  float* tmp = nullptr;
  float* ws = nullptr;
  if (int rc = dalloc(ctx, &tmp, T * N * 4)) return rc;
  if (split)
    if (int rc = dalloc(ctx, &ws, kSlices * T * N * 4)) {
      cudaFree(tmp);
      return rc;
    }
  const PlanHdr* plan = reinterpret_cast<const PlanHdr*>(ctx->plan_dev);
  const EpiResidArgs args{tmp, N, sc, nullptr, nullptr, nullptr, 0};
  cudaError_t e = cudaMemsetAsync(tmp, 0, T * N * 4, ctx->stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(abuf, a, T * K * 2, cudaMemcpyHostToDevice, ctx->stream);
  if (e == cudaSuccess && split) {
    e = gemm_tc_partial(ta, tb, K, N, plan, EpiPartialArgs{ws, T, N}, ctx->status, ctx->gemm_grid, ctx->stream,
                        kSlices);
    if (e == cudaSuccess) e = resid_reduce(plan, ws, T, kSlices, args, N, ctx->status, (int)T, ctx->stream);
  } else if (e == cudaSuccess) {
    e = gemm_tc_resid(ta, tb, K, N, plan, args, ctx->status, ctx->gemm_grid, ctx->stream);
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, tmp, T * N * 4, cudaMemcpyDeviceToHost, ctx->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
  cudaFree(tmp);
  if (ws) cudaFree(ws);
  if (e != cudaSuccess) return fail(ctx, DUOLM_E_CUDA, "debug_gemm: %s", cudaGetErrorString(e));
  return check_status(ctx);
}

int duolm_gather(duolm_ctx* ctx, const int32_t* ids, int64_t n, float* x, uint16_t* xg, float* ssp) {
  if (!ctx || n < 0 || n > INT32_MAX || (n > 0 && (!ids || !x || !xg || !ssp)))
    return fail(ctx, DUOLM_E_ARG, "gather: bad arguments");
  if (!ctx->f16) return fail(ctx, DUOLM_E_STATE, "gather: only bf16 models run the fp16 gather");
  if (n == 0) return 0;
  CK(cudaSetDevice(ctx->device));
  if (!ctx->gather_hdr)
    if (int rc = dalloc(ctx, &ctx->gather_hdr, sizeof(PlanHdr))) return rc;
  // the kernel finds its ids at a byte offset from the header: point it at
  // the caller's array (the header is staged from host memory before the
  // copy call returns, so a stack copy is fine)
  PlanHdr h{};
  h.n_tokens = (int32_t)n;
  h.off_ids = (int64_t)(reinterpret_cast<const char*>(ids) - reinterpret_cast<const char*>(ctx->gather_hdr));
  CK(cudaMemcpyAsync(ctx->gather_hdr, &h, sizeof h, cudaMemcpyHostToDevice, ctx->stream));
  const duolm_model_desc& d = ctx->desc;
  CK(embed_gain(ctx->gather_hdr, ctx->embed, ctx->table, ctx->n_items, d.vocab, d.d,
                ctx->gains + ctx->layers[0].g_attn, x, reinterpret_cast<__half*>(xg), ssp, d.d / 64, ctx->status,
                (int)std::min<int64_t>(n, INT32_MAX), ctx->stream));
  return 0;
}

int duolm_debug_wait_timeout(duolm_ctx* ctx) {
  if (!ctx) return DUOLM_E_ARG;
  CK(cudaSetDevice(ctx->device));
  CK(debug_wait_timeout(ctx->status, ctx->stream));
  return duolm_sync(ctx);
}

int duolm_profile(duolm_ctx* ctx, int n_steps, double* ms_out, int64_t* count_out) {
  if (!ctx || !ms_out || !count_out || n_steps < 1) return fail(ctx, DUOLM_E_ARG, "profile: bad arguments");
  if (!ctx->prepared) return fail(ctx, DUOLM_E_STATE, "profile: nothing prepared");
  CK(cudaSetDevice(ctx->device));
  for (int i = 0; i < DUOLM_PROF_N; ++i) {
    ms_out[i] = 0.0;
    count_out[i] = 0;
  }
  Prof prof;
  cudaEvent_t start;
  CK(cudaEventCreate(&start));
  int rc = 0;
  for (int step = 0; step < n_steps && !rc; ++step) {
    prof.used = 0;
    cudaError_t e = cudaEventRecord(start, ctx->stream);
    int64_t n = 0;
    if (e == cudaSuccess) e = launch_forward(ctx, ctx->desc.n_layers, true, &n, &prof);
    if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
    if (e != cudaSuccess) {
      rc = fail(ctx, DUOLM_E_CUDA, "profile: %s", cudaGetErrorString(e));
      break;
    }
    for (size_t i = 0; i < prof.used; ++i) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, i == 0 ? start : prof.ev[i - 1], prof.ev[i]);
      ms_out[prof.cls[i]] += ms;
      count_out[prof.cls[i]] += 1;
    }
  }
  cudaEventDestroy(start);
  for (auto ev : prof.ev) cudaEventDestroy(ev);
  if (rc) return rc;
  return check_status(ctx);
}

int duolm_debug_table(duolm_ctx* ctx, uint16_t* out, int64_t n_items) {
  if (!ctx || !out || n_items < 0 || n_items > ctx->n_items) return fail(ctx, DUOLM_E_ARG, "debug_table: bad arguments");
  CK(cudaSetDevice(ctx->device));
  CK(cudaMemcpy(out, ctx->table, n_items * ctx->desc.d * 2, cudaMemcpyDeviceToHost));
  return 0;
}

}  // extern "C"
