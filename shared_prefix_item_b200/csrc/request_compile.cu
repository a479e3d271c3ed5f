// Request compiler (host only): turns request records -- history items with
// their feedback tokens, candidate items -- into the packed layout that
// duolm_prepare / duolm_score take.
//
// DuoLM summary page (paper.rainbus.top), 方法步骤详情 step 3 and 核心方法; the
// onedev.kr page, 어떻게 쓰나: a request carries item ids and feedback, not
// vectors; each history item is a marker token followed by the item's VID(s)
// and its feedback text, after an instruction; each candidate branch is the
// candidate's VID(s), scored at the last one.  The pages name this host-side
// input compilation as the serving bottleneck at high request rates, so the
// requests are compiled by several threads at once: offsets first (a
// sequential prefix sum over lengths), then every request's slice in
// parallel.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <string>
#include <thread>
#include <vector>

#include "duolm.h"

extern thread_local std::string g_noctx_err;

namespace {

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_noctx_err = buf;
  return code;
}

bool offsets_ok(const int64_t* off, int64_t n) {
  if (off[0] != 0) return false;
  for (int64_t i = 0; i < n; ++i)
    if (off[i + 1] < off[i]) return false;
  return true;
}

}  // namespace

// hist_cached == nullptr: whole prefixes.  Otherwise request r's slot of the
// prefix KV store holds its instruction and first hist_cached[r] history
// items (hist_cached[r] < 0: the request does not use the store): only the
// rest is compiled, and cached_out / keep_out receive the arguments of
// duolm_prepare_cached.
static int compile_impl(const duolm_template* tpl, int n_requests, const int64_t* hist_items,
                        const int64_t* hist_offsets, const int32_t* feedback, const int64_t* feedback_offsets,
                        const int64_t* cand_items, const int64_t* cand_offsets, int64_t n_items, int n_threads,
                        const int32_t* hist_cached, int32_t* prefix_ids, int64_t prefix_capacity,
                        int64_t* prefix_offsets, int32_t* branch_ids, int64_t branch_capacity, int32_t* cached_out,
                        int32_t* keep_out) {
  g_noctx_err.clear();
  if (!tpl || n_requests < 1 || !hist_offsets || !feedback_offsets || !cand_offsets || !prefix_offsets ||
      n_items < 1 || tpl->vocab < 1 || tpl->m < 1 || tpl->n_instr < 0 || tpl->n_header < 0 ||
      tpl->n_branch_header < 0 || (tpl->n_instr && !tpl->instr) || (tpl->n_header && !tpl->header) ||
      (tpl->n_branch_header && !tpl->branch_header))
    return fail(DUOLM_E_ARG, "compile: bad arguments");
  const int64_t V = tpl->vocab, m = tpl->m;
  if (V + n_items * m > INT32_MAX) return fail(DUOLM_E_ID, "compile: vocab + items x m exceeds int32");
  const int R = n_requests;
  if (!offsets_ok(hist_offsets, R) || !offsets_ok(cand_offsets, R))
    return fail(DUOLM_E_OFFSETS, "compile: history or candidate offsets do not start at 0 or decrease");
  const int64_t H = hist_offsets[R], C = cand_offsets[R];
  if (!offsets_ok(feedback_offsets, H))
    return fail(DUOLM_E_OFFSETS, "compile: feedback offsets do not start at 0 or decrease");
  if ((H && !hist_items) || (feedback_offsets[H] && !feedback) || !cand_items)
    return fail(DUOLM_E_ARG, "compile: null item or feedback array");
  for (int r = 0; r < R; ++r)
    if (cand_offsets[r + 1] == cand_offsets[r]) return fail(DUOLM_E_EMPTY, "compile: request %d has no candidates", r);
  for (const auto& t : {std::pair<const int32_t*, int>{tpl->instr, tpl->n_instr},
                        std::pair<const int32_t*, int>{tpl->header, tpl->n_header},
                        std::pair<const int32_t*, int>{tpl->branch_header, tpl->n_branch_header}})
    for (int i = 0; i < t.second; ++i)
      if (t.first[i] < 0 || t.first[i] >= V) return fail(DUOLM_E_ID, "compile: template token %d out of range", t.first[i]);
  if (tpl->marker < 0 || tpl->marker >= V) return fail(DUOLM_E_ID, "compile: marker out of range");
  if (hist_cached) {
    if (!cached_out || !keep_out) return fail(DUOLM_E_ARG, "compile: null cached or keep output");
    for (int r = 0; r < R; ++r)
      if (hist_cached[r] < -1 || hist_cached[r] > hist_offsets[r + 1] - hist_offsets[r])
        return fail(DUOLM_E_ARG, "compile: request %d has %lld history items, %d of them cached", r,
                    (long long)(hist_offsets[r + 1] - hist_offsets[r]), hist_cached[r]);
  }
  // first history item each request compiles (the ones before it are in the store)
  auto first_item = [&](int r) -> int64_t {
    return hist_offsets[r] + (hist_cached && hist_cached[r] > 0 ? hist_cached[r] : 0);
  };
  auto item_len = [&](int64_t h) -> int64_t { return 1 + m + (feedback_offsets[h + 1] - feedback_offsets[h]); };

  // lengths and offsets
  const int64_t b = tpl->n_branch_header + m;
  // cached / keep are written only once the capacities are known to hold
  std::vector<int32_t> cached_v(hist_cached ? R : 0), keep_v(hist_cached ? R : 0);
  prefix_offsets[0] = 0;
  for (int r = 0; r < R; ++r) {
    const int hc = hist_cached ? hist_cached[r] : -1;
    int64_t stored = hc > 0 ? tpl->n_instr : 0;  // tokens already in the slot
    for (int64_t h = hist_offsets[r]; h < first_item(r); ++h) stored += item_len(h);
    int64_t L = (hc > 0 ? 0 : tpl->n_instr) + tpl->n_header;
    for (int64_t h = first_item(r); h < hist_offsets[r + 1]; ++h) L += item_len(h);
    prefix_offsets[r + 1] = prefix_offsets[r] + L;
    if (hist_cached) {
      if (stored > INT32_MAX || L > INT32_MAX) return fail(DUOLM_E_CAPACITY, "compile: request %d too long", r);
      cached_v[r] = (int32_t)stored;
      keep_v[r] = hc < 0 ? 0 : (int32_t)(L - tpl->n_header);  // all new history, not the header
    }
  }
  if (prefix_offsets[R] > prefix_capacity)
    return fail(DUOLM_E_CAPACITY, "compile: %lld prefix tokens, capacity %lld", (long long)prefix_offsets[R],
                (long long)prefix_capacity);
  if (C * b > branch_capacity)
    return fail(DUOLM_E_CAPACITY, "compile: %lld branch tokens, capacity %lld", (long long)(C * b),
                (long long)branch_capacity);
  if ((prefix_offsets[R] && !prefix_ids) || !branch_ids) return fail(DUOLM_E_ARG, "compile: null output array");
  if (hist_cached) {
    std::copy(cached_v.begin(), cached_v.end(), cached_out);
    std::copy(keep_v.begin(), keep_v.end(), keep_out);
  }

  // every request's slice; a worker records the first bad id of its range
  // Starting a thread costs tens of microseconds, about what one thread
  // needs to write 64K tokens: by default one worker per 256K tokens.
  const int64_t tokens = prefix_offsets[R] + C * b;
  const int hw = (int)std::max(1u, std::thread::hardware_concurrency());
  int T = n_threads > 0 ? std::min(n_threads, hw) : (int)std::min<int64_t>(hw, 1 + tokens / (1 << 18));
  T = std::min(T, R);
  std::vector<int64_t> bad(T, -1);  // request index of a bad id, per worker
  auto work = [&](int w) {
    for (int r = w; r < R; r += T) {
      int32_t* p = prefix_ids + prefix_offsets[r];
      if (!(hist_cached && hist_cached[r] > 0)) p = std::copy(tpl->instr, tpl->instr + tpl->n_instr, p);
      for (int64_t h = first_item(r); h < hist_offsets[r + 1]; ++h) {
        const int64_t it = hist_items[h];
        if ((it < 0 || it >= n_items) && bad[w] < 0) bad[w] = r;
        const int64_t row = std::min<int64_t>(std::max<int64_t>(it, 0), n_items - 1) * m;
        *p++ = tpl->marker;
        for (int64_t k = 0; k < m; ++k) *p++ = (int32_t)(V + row + k);
        for (int64_t f = feedback_offsets[h]; f < feedback_offsets[h + 1]; ++f) {
          const int32_t tok = feedback[f];
          if ((tok < 0 || tok >= V) && bad[w] < 0) bad[w] = r;
          *p++ = tok;
        }
      }
      std::copy(tpl->header, tpl->header + tpl->n_header, p);
      for (int64_t c = cand_offsets[r]; c < cand_offsets[r + 1]; ++c) {
        const int64_t it = cand_items[c];
        if ((it < 0 || it >= n_items) && bad[w] < 0) bad[w] = r;
        const int64_t row = std::min<int64_t>(std::max<int64_t>(it, 0), n_items - 1) * m;
        int32_t* q = std::copy(tpl->branch_header, tpl->branch_header + tpl->n_branch_header, branch_ids + c * b);
        for (int64_t k = 0; k < m; ++k) *q++ = (int32_t)(V + row + k);
      }
    }
  };
  if (T == 1) {
    work(0);
  } else {
    std::vector<std::thread> pool;
    pool.reserve(T);
    for (int w = 0; w < T; ++w) pool.emplace_back(work, w);
    for (auto& t : pool) t.join();
  }
  int64_t first_bad = -1;
  for (int64_t v : bad)
    if (v >= 0 && (first_bad < 0 || v < first_bad)) first_bad = v;
  if (first_bad >= 0)
    return fail(DUOLM_E_ID, "compile: request %lld has an item id outside [0, %lld) or a feedback token outside "
                "the vocabulary", (long long)first_bad, (long long)n_items);
  return DUOLM_OK;
}

extern "C" int duolm_compile(const duolm_template* tpl, int n_requests, const int64_t* hist_items,
                             const int64_t* hist_offsets, const int32_t* feedback, const int64_t* feedback_offsets,
                             const int64_t* cand_items, const int64_t* cand_offsets, int64_t n_items, int n_threads,
                             int32_t* prefix_ids, int64_t prefix_capacity, int64_t* prefix_offsets,
                             int32_t* branch_ids, int64_t branch_capacity) {
  return compile_impl(tpl, n_requests, hist_items, hist_offsets, feedback, feedback_offsets, cand_items, cand_offsets,
                      n_items, n_threads, nullptr, prefix_ids, prefix_capacity, prefix_offsets, branch_ids,
                      branch_capacity, nullptr, nullptr);
}

extern "C" int duolm_compile_append(const duolm_template* tpl, int n_requests, const int64_t* hist_items,
                                    const int64_t* hist_offsets, const int32_t* feedback,
                                    const int64_t* feedback_offsets, const int64_t* cand_items,
                                    const int64_t* cand_offsets, int64_t n_items, int n_threads,
                                    const int32_t* hist_cached, int32_t* prefix_ids, int64_t prefix_capacity,
                                    int64_t* prefix_offsets, int32_t* branch_ids, int64_t branch_capacity,
                                    int32_t* cached_out, int32_t* keep_out) {
  if (!hist_cached) {
    g_noctx_err = "compile_append: null hist_cached";
    return DUOLM_E_ARG;
  }
  return compile_impl(tpl, n_requests, hist_items, hist_offsets, feedback, feedback_offsets, cand_items, cand_offsets,
                      n_items, n_threads, hist_cached, prefix_ids, prefix_capacity, prefix_offsets, branch_ids,
                      branch_capacity, cached_out, keep_out);
}
