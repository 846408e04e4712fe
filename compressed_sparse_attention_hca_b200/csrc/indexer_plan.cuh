// indexer_plan.cuh -- slicing plan and candidate workspace layout shared by the
// indexer producers (SIMT and tcgen05) and the merge kernel.
#pragma once

#include <stdint.h>

namespace csa {

constexpr int kMergeNT = 1024;
constexpr int kMergeSmemKeys = 40960;  // candidate keys the merge stages in shared memory (160 KB)

// Entries visible to a query at absolute position t: an entry becomes visible
// once its whole group of m tokens is at or before t, i.e. s < floor((t+1)/m)
// ("DeepSeek-V4 内部机制" 1.4: a query cannot see its own unfinished block).
__host__ __device__ __forceinline__ int64_t visible_entries(int64_t t, int m, int64_t n_entries) {
  int64_t v = (t + 1) / m;
  if (v > n_entries) v = n_entries;
  return v < 0 ? 0 : v;
}

struct IndexPlan {
  int slice_len;      // entries per slice (multiple of 128)
  int n_slices;       // slices per query row
  int64_t cand_cap;   // candidate slots per query row (n_slices * k), 0 when n_slices == 1
  int64_t n_rows;     // batch * n_q
  int coop;           // 1: the slices of a row select together (cooperative launch), no merge
};

// Cooperative selection workspace per query row: 12-bit key-prefix histogram
// [4096], counters (+pad) [8], per-slice slots [17 * n_slices] (keys above
// the k-th key's prefix, suffix histogram of keys inside it).  It must be zero
// before the first call; every call leaves it at zero.
__host__ __device__ __forceinline__ int64_t plan_coop_stride(const IndexPlan& p) {
  return (4096 + 8 + 17 * (int64_t)p.n_slices + 7) / 8 * 8;
}
__host__ __device__ __forceinline__ uint32_t* plan_coop_row(const IndexPlan& p, void* ws, int64_t row) {
  return static_cast<uint32_t*>(ws) + row * plan_coop_stride(p);
}

__host__ __device__ __forceinline__ int64_t slice_valid(const IndexPlan& p, int sl, int64_t vis,
                                                        int64_t n_entries) {
  const int64_t s0 = (int64_t)sl * p.slice_len;
  int64_t len = n_entries - s0;
  if (len > p.slice_len) len = p.slice_len;
  int64_t v = vis - s0;
  if (v > len) v = len;
  return v < 0 ? 0 : v;
}

// Candidate slots used by slices [0, sl): slice j contributes min(k, valid_j).
__host__ __device__ __forceinline__ int64_t slice_cand_offset(const IndexPlan& p, int sl, int64_t vis,
                                                              int64_t n_entries, int k) {
  int64_t off = 0;
  for (int j = 0; j < sl; ++j) {
    const int64_t v = slice_valid(p, j, vis, n_entries);
    off += v < k ? v : k;
  }
  return off;
}

__host__ __device__ __forceinline__ uint32_t* plan_cand_keys(const IndexPlan& p, void* ws, int64_t row) {
  return static_cast<uint32_t*>(ws) + row * p.cand_cap;
}
__host__ __device__ __forceinline__ int32_t* plan_cand_idx(const IndexPlan& p, void* ws, int64_t row) {
  return reinterpret_cast<int32_t*>(static_cast<uint32_t*>(ws) + p.n_rows * p.cand_cap) + row * p.cand_cap;
}

// Per-slice k-th largest key (0 when the slice kept all its entries): the
// final k-th key is at least the largest of them, so the merge ignores every
// candidate below that floor.
__host__ __device__ __forceinline__ uint32_t* plan_cand_thr(const IndexPlan& p, void* ws, int64_t row) {
  return static_cast<uint32_t*>(ws) + 2 * p.n_rows * p.cand_cap + row * p.n_slices;
}

inline size_t plan_workspace_bytes(const IndexPlan& p) {
  if (p.coop) return (size_t)p.n_rows * (size_t)plan_coop_stride(p) * 4;
  if (p.cand_cap == 0) return 0;
  return (size_t)p.n_rows * (size_t)p.cand_cap * 8 + (size_t)p.n_rows * (size_t)p.n_slices * 4;
}

// Tensor-core producer (indexer_tc.cu): BF16 q / K with 64 heads of dim 128.
struct IndexArgs;
bool index_tc_eligible(const IndexArgs& a);
IndexPlan make_tc_plan(int batch, int n_q, int64_t n_entries, int k, int dt);
cudaError_t launch_index_tc(const IndexArgs& a, const IndexPlan& p, cudaStream_t s);
// Key-stage ring of the tensor-core producer for this query count and dtype:
// stages in the ring and 128-entry tiles per stage.
void index_tc_ring(int n_q, int dt, int* stages, int* tiles_per_stage);

}  // namespace csa
