// Shared-prefix, tree-masked attention of the fp32 path (the fp16 path runs
// on the tensor cores, attention_tc.cu).  Same visibility rule (tree_visible,
// common.cuh): DuoLM summary page (paper.rainbus.top), 方法步骤详情 step 4.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

// ---------------------------------------------------------------------------
// fp32 path: one warp per (token, query head), keys visited in order with an
// online softmax; head_dim a multiple of 32.  A request that continues a
// cached prefix of c tokens reads keys [0, c) from its slot of the layer's
// KV store (ks, vs: [n_kv_heads][store_rows][hd]) and the rest from this
// batch; request-local indices count from the first cached token.
// ---------------------------------------------------------------------------
__global__ void attention_f32_kernel(const PlanHdr* __restrict__ plan, const int2* __restrict__ reqx,
                                     const float* __restrict__ q, const float* __restrict__ kc,
                                     const float* __restrict__ vc, int64_t kv_rows, const float* __restrict__ ks,
                                     const float* __restrict__ vs, int64_t store_rows, int n_q_heads, int n_kv_heads,
                                     int hd, float scale, float* __restrict__ o) {
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
    const int2 rx = reqx[treq[t]];
    const int tok0 = rq.x, L = rq.y, c = rx.x;
    const int tq = t - tok0 + c;
    float qv[8], accv[8];
    for (int i = 0; i < per_lane; ++i) {
      qv[i] = q[((int64_t)t * n_q_heads + h) * hd + lane + 32 * i];
      accv[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int tk = 0; tk <= tq; ++tk) {
      if (!tree_visible(tq, tk, L, b)) continue;
      const int64_t row = tk < c ? (int64_t)kvh * store_rows + rx.y + tk : (int64_t)kvh * kv_rows + tok0 + tk - c;
      const float* kr = (tk < c ? ks : kc) + row * hd;
      const float* vr = (tk < c ? vs : vc) + row * hd;
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

cudaError_t attention_f32(const PlanHdr* plan, const int2* reqx, const float* q, const float* kc, const float* vc,
                          int64_t kv_rows, const float* ks, const float* vs, int64_t store_rows, int n_q_heads,
                          int n_kv_heads, int hd, float scale, float* o, int max_rows, cudaStream_t s) {
  const int64_t warps = (int64_t)max_rows * n_q_heads;
  const int blocks = (int)std::min<int64_t>((warps + 7) / 8, 148 * 16);
  attention_f32_kernel<<<blocks, 256, 0, s>>>(plan, reqx, q, kc, vc, kv_rows, ks, vs, store_rows, n_q_heads,
                                              n_kv_heads, hd, scale, o);
  return cudaGetLastError();
}

}  // namespace duolm
