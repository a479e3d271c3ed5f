// Append step of the prefix KV store (incremental history append).
//
// DuoLM summary page (paper.rainbus.top), 未来方向 (3): when new history
// items arrive within a session, only their vectors and K/V are added; the
// K/V of the earlier prefix is reused instead of recomputed.  A request that
// keeps n of its new prefix tokens has their K/V (rows tok0 .. tok0 + n - 1
// of this batch, at the positions that continue its cached prefix) copied
// into its slot of the layer's store right after the layer's attention, so a
// later call can start from them.  One CTA per (request, KV head, K or V):
// the rows of one head are contiguous in both buffers, so the copy is one
// run of 16-byte words.
#include "common.cuh"
#include "kernels.cuh"

namespace duolm {

namespace {

__global__ void kv_append_kernel(const PlanHdr* __restrict__ plan, const int2* __restrict__ append,
                                 const uint4* __restrict__ kc, const uint4* __restrict__ vc, int64_t kv_rows,
                                 uint4* __restrict__ ks, uint4* __restrict__ vs, int64_t store_rows, int n_kv_heads,
                                 int row_words) {
  pdl_launch_dependents();
  pdl_wait();
  const int n_req = plan->n_req;
  const int4* reqs = plan_array<int4>(plan, plan->off_req);
  const int64_t units = (int64_t)n_req * n_kv_heads * 2;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int r = (int)(u / (2 * n_kv_heads));
    const int h = (int)(u % (2 * n_kv_heads)) >> 1;
    const bool is_v = u & 1;
    const int2 ap = append[r];  // {rows, first store row}
    if (ap.x <= 0) continue;
    const uint4* src = (is_v ? vc : kc) + ((int64_t)h * kv_rows + reqs[r].x) * row_words;
    uint4* dst = (is_v ? vs : ks) + ((int64_t)h * store_rows + ap.y) * row_words;
    const int64_t n = (int64_t)ap.x * row_words;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[i];
  }
}

}  // namespace

cudaError_t kv_append(const PlanHdr* plan, const int2* append, const void* kc, const void* vc, int64_t kv_rows,
                      void* ks, void* vs, int64_t store_rows, int n_kv_heads, int row_bytes, int max_req, int grid,
                      cudaStream_t s, bool pdl) {
  if (row_bytes % 16) return cudaErrorInvalidValue;
  const int64_t units = (int64_t)max_req * n_kv_heads * 2;
  const int g = (int)std::max<int64_t>(1, std::min<int64_t>(units, grid));
  return launch_ex(kv_append_kernel, dim3(g), dim3(256), 0, s, pdl, plan, append, static_cast<const uint4*>(kc),
                   static_cast<const uint4*>(vc), kv_rows, static_cast<uint4*>(ks), static_cast<uint4*>(vs),
                   store_rows, n_kv_heads, row_bytes / 16);
}

}  // namespace duolm
