// mqa_plan.cuh -- attended-row list and split-KV workspace layout shared by the
// MQA kernels.
#pragma once

#include "csa_internal.cuh"
#include "indexer_plan.cuh"
#include "sm100.cuh"

namespace csa {

// How a query's rows are split over CTAs and how the splits are combined.
enum MqaMode {
  kMqaWhole = 0,  // one CTA per (query, head group): normalised output directly
  kMqaSplit = 1,  // split rows; partials combined by a separate kernel
};

struct MqaPlan {
  int heads_per_cta;
  int n_splits;
  int64_t rows_per_split;  // SIMT kernel only
  int mode;                // MqaMode
  int64_t ws_head;         // bytes of the workspace before the partials
};



// Rows attended by one query ("DeepSeek-V4 内部机制" 1.2 Step 2 and 1.4): the
// selected entries (CSA: k slots, -1 unused; HCA: every visible entry), then
// the window tokens max(0, t-window+1) .. t.
struct RowList {
  int64_t vis, n_sel, win_lo, n_win, n_rows;
  const int32_t* sel;  // nullptr for HCA
};

__device__ __forceinline__ RowList make_row_list(const MqaArgs& a, int64_t bt, int64_t t) {
  RowList r;
  r.vis = visible_entries(t, a.m, a.n_entries);
  r.sel = a.idx ? a.idx + bt * a.k : nullptr;
  r.n_sel = a.idx ? a.k : r.vis;
  r.win_lo = t - a.window + 1 < 0 ? 0 : t - a.window + 1;
  r.n_win = a.window > 0 ? t - r.win_lo + 1 : 0;
  r.n_rows = r.n_sel + r.n_win;
  return r;
}

// Address of entry e of request b (contiguous or through the block table);
// nullptr, with the bad-page status bit set, when its page is outside the pool.
__device__ __forceinline__ const uint8_t* entry_row(const MqaArgs& a, int b, int64_t e, int64_t rb) {
  const uint8_t* base = static_cast<const uint8_t*>(a.entries);
  if (a.pages.table == nullptr) return base + ((int64_t)b * a.n_entries + e) * rb;
  const int64_t pr = pool_row(a.pages, b, e);
  if (pr < 0) {
    flag_status(kStatusBadPage);
    return nullptr;
  }
  return base + pr * rb;
}

// Address of attended row r, or nullptr when the slot is unused / invalid.
__device__ __forceinline__ const uint8_t* row_ptr(const MqaArgs& a, const RowList& rl, int b, int64_t r,
                                                  int64_t rb) {
  if (r < rl.n_sel) {
    const int64_t e = rl.sel ? (int64_t)rl.sel[r] : r;
    if (e < 0 || e >= rl.vis) return nullptr;
    return entry_row(a, b, e, rb);
  }
  const int64_t w = rl.win_lo + (r - rl.n_sel) - a.win_start[b];
  if (w < 0 || w >= a.win_len) return nullptr;
  return static_cast<const uint8_t*>(a.win) + ((int64_t)b * a.win_len + w) * rb;
}

__device__ __forceinline__ bool row_valid(const MqaArgs& a, const RowList& rl, int b, int64_t r) {
  return row_ptr(a, rl, b, r, 1) != nullptr;
}

inline int64_t max_rows_per_query(const MqaArgs& a) {
  return (a.idx ? (int64_t)a.k : a.n_entries) + a.window;
}

__host__ __device__ __forceinline__ float* plan_partials(const MqaPlan& p, const MqaArgs& a) {
  return reinterpret_cast<float*>(static_cast<char*>(a.ws) + p.ws_head);
}
__host__ __device__ __forceinline__ float* plan_partial_o(const MqaPlan& p, const MqaArgs& a, int64_t bt,
                                                         int s, int h) {
  return plan_partials(p, a) + (((bt * p.n_splits + s) * a.n_heads) + h) * (int64_t)a.dim;
}
__host__ __device__ __forceinline__ float* plan_partial_ml(const MqaPlan& p, const MqaArgs& a, int64_t bt,
                                                          int s, int h) {
  const int64_t n_bt = (int64_t)a.batch * a.n_q;
  return plan_partials(p, a) + n_bt * p.n_splits * a.n_heads * (int64_t)a.dim +
         ((bt * p.n_splits + s) * a.n_heads + h) * 2;
}

inline size_t plan_mqa_workspace_bytes(const MqaPlan& p, const MqaArgs& a) {
  if (p.n_splits <= 1) return 0;
  const size_t n_bt = (size_t)a.batch * a.n_q;
  return (size_t)p.ws_head + n_bt * p.n_splits * a.n_heads * ((size_t)a.dim + 2) * 4;
}

}  // namespace csa
