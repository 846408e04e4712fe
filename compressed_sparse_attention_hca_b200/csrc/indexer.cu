// indexer.cu -- Lightning Indexer score fused with the top-k selector
// ("DeepSeek-V4 内部机制" 1.2 Step 2: I[t,s] = sum_h w[t,h] ReLU(q[t,h].K[s]),
// top-k over I[t,:]; section 6.2: fp32 score rounded to BF16 before top-k).
//
// Work split: the visible entries of a query are cut into slices; one CTA
// scores one slice of one query into shared memory and selects the slice's
// top k there (a radix select on the score keys, so the score row never goes
// to HBM).  A query whose entries need several slices gets a second, small
// merge kernel that selects the final k among the per-slice candidates.
//
// This file holds the SIMT score producer (fp32 FMA), used for F32 inputs
// (exact-fp32 mode) and for shapes the tensor-core producer does not take;
// indexer_tc.cu holds the tcgen05 producer for BF16 / NVFP4 inputs.
#include "csa_internal.cuh"
#include "sm100.cuh"
#include "topk_select.cuh"
#include "indexer_plan.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_indexer)

namespace {

constexpr int kNT = 512;

__global__ void __launch_bounds__(kNT) index_slice_simt_kernel(IndexArgs a, IndexPlan plan) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int sl = blockIdx.x, t = blockIdx.y, b = blockIdx.z;
  const int64_t bt = (int64_t)b * a.n_q + t;
  float* q = reinterpret_cast<float*>(smem_raw);                 // [n_heads][dim]
  float* w = q + a.n_heads * a.dim;                               // [n_heads]
  uint32_t* keys = reinterpret_cast<uint32_t*>(w + a.n_heads);    // [slice_len]
  SelectSmem<kNT>& sm = *reinterpret_cast<SelectSmem<kNT>*>(keys + plan.slice_len);

  const int64_t vis = visible_entries(a.q_pos[bt], a.m, a.n_entries);
  const int64_t s0 = (int64_t)sl * plan.slice_len;
  const int len = (int)min64(plan.slice_len, a.n_entries - s0);
  const int n_valid = (int)max64(0, min64(len, vis - s0));

  // decode the query heads and the head weights
  const int qrb = (int)row_bytes(a.dt, a.dim);
  const uint8_t* qbase = static_cast<const uint8_t*>(a.qI) + bt * a.n_heads * qrb;
  const uint8_t* qsf = a.dt == CSA_IDX_NVFP4
                           ? static_cast<const uint8_t*>(a.qI_sf) + bt * a.n_heads * (a.dim / 16)
                           : nullptr;
  for (int c = threadIdx.x; c < a.n_heads * (a.dim / 8); c += kNT) {
    const int h = c / (a.dim / 8), d0 = (c % (a.dim / 8)) * 8;
    decode_row_chunk8(qbase + (int64_t)h * qrb, qsf ? qsf + h * (a.dim / 16) : nullptr, a.dt, a.dim,
                      d0, q + h * a.dim + d0);
  }
  for (int h = threadIdx.x; h < a.n_heads; h += kNT) w[h] = a.wI[bt * a.n_heads + h];
  __syncthreads();

  const bool f32mode = a.dt == CSA_F32;
  const uint8_t* kbase = static_cast<const uint8_t*>(a.KI) + (int64_t)b * a.n_entries * qrb;
  const uint8_t* ksf = a.dt == CSA_IDX_NVFP4
                           ? static_cast<const uint8_t*>(a.KI_sf) + (int64_t)b * nvfp4_blocked_sf_bytes(a.n_entries, a.dim)
                           : nullptr;
  for (int p = threadIdx.x; p < len; p += kNT) {
    const int64_t e = s0 + p;
    uint32_t key = 0;
    float score = -INFINITY;
    if (p < n_valid) {
      const uint8_t* krow = kbase + e * qrb;
      const uint8_t* ksrow = ksf ? ksf + nvfp4_blocked_sf_offset(e, a.dim) : nullptr;
      if (a.pages.table != nullptr) {
        // through the block table: the pool row, and the scale block of the
        // pool page holding row 128 * (e / 128)
        const int64_t pr = pool_row(a.pages, b, e);
        const int64_t pg = ksf ? pool_sf_page(a.pages, b, e) : 0;
        if (pr < 0 || pg < 0) flag_status(kStatusBadPage);
        krow = static_cast<const uint8_t*>(a.KI) + (pr < 0 ? 0 : pr) * qrb;
        if (ksf)
          ksrow = static_cast<const uint8_t*>(a.KI_sf) + (pg < 0 ? 0 : pg) * nvfp4_blocked_sf_bytes(128, a.dim) +
                  nvfp4_blocked_sf_offset(e % 128, a.dim);
      }
      float I = 0.f;
      for (int h = 0; h < a.n_heads; ++h) {
        float dot = 0.f;
        for (int d0 = 0; d0 < a.dim; d0 += 8) {
          float kv[8];
          decode_row_chunk8(krow, ksrow, a.dt, a.dim, d0, kv, true);
          const float* qh = q + h * a.dim + d0;
#pragma unroll
          for (int j = 0; j < 8; ++j) dot = fmaf(qh[j], kv[j], dot);
        }
        I = fmaf(w[h], fmaxf(dot, 0.f), I);
      }
      if (f32mode) {
        score = I;
        key = f32_key(I);
      } else {
        key = bf16_key(I);
        score = key_to_f32(key);
      }
    }
    if (p < n_valid) keys[p] = key;
    if (a.scores_out) {
      if (f32mode) static_cast<float*>(a.scores_out)[bt * a.n_entries + e] = score;
      else static_cast<__nv_bfloat16*>(a.scores_out)[bt * a.n_entries + e] = __float2bfloat16_rn(score);
    }
  }
  __syncthreads();

  const int kk = min(a.k, n_valid);
  const int passes = f32mode ? 4 : 2;
  auto key_at = [&](int i) { return keys[i]; };
  if (plan.n_slices == 1) {
    int32_t* out = a.idx_out + bt * a.k;
    block_select<kNT>(key_at, n_valid, kk, passes, sm,
                      [&](int slot, int pos) { out[slot] = (int32_t)(s0 + pos); });
    for (int j = kk + threadIdx.x; j < a.k; j += kNT) out[j] = -1;
  } else {
    const int64_t off = slice_cand_offset(plan, sl, vis, a.n_entries, a.k);
    uint32_t* ck = plan_cand_keys(plan, a.ws, bt) + off;
    int32_t* ci = plan_cand_idx(plan, a.ws, bt) + off;
    uint32_t T = 0;
    block_select<kNT>(
        key_at, n_valid, kk, passes, sm,
        [&](int slot, int pos) {
          ck[slot] = keys[pos];
          ci[slot] = (int32_t)(s0 + pos);
        },
        0u, &T);
    if (threadIdx.x == 0) plan_cand_thr(plan, a.ws, bt)[sl] = T;
  }
}

}  // namespace

// Final selection of one query row among the per-slice candidates.  The
// candidate keys are first copied into shared memory with batches of
// independent, coalesced loads (up to kMergeSmemKeys of them), so the
// range-adaptive radix select runs on shared memory; the final k-th key is at
// least every slice's own k-th key, which serves as the floor.
__global__ void __launch_bounds__(kMergeNT) index_merge_kernel(IndexArgs a, IndexPlan plan) {
  extern __shared__ __align__(16) uint32_t merge_keys[];
  __shared__ SelectSmem<kMergeNT> sm;
  __shared__ uint32_t floor_s;
  const int t = blockIdx.x, b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t bt = (int64_t)b * a.n_q + t;
  const int64_t vis = visible_entries(a.q_pos[bt], a.m, a.n_entries);
  const int n = (int)slice_cand_offset(plan, plan.n_slices, vis, a.n_entries, a.k);
  const uint32_t* ck = plan_cand_keys(plan, a.ws, bt);
  const int32_t* ci = plan_cand_idx(plan, a.ws, bt);
  const int kk = (int)min64(min64(a.k, vis), n);
  int32_t* out = a.idx_out + bt * a.k;
  if (warp == 0) {
    const uint32_t* thr = plan_cand_thr(plan, a.ws, bt);
    uint32_t f = 0;
    for (int j = lane; j < plan.n_slices; j += 32) f = max(f, thr[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) f = max(f, __shfl_xor_sync(0xffffffffu, f, o));
    if (lane == 0) floor_s = f;
  }
  const bool staged = n <= kMergeSmemKeys;
  if (staged) {
    constexpr int kBatch = 8;
    for (int base = 0; base < n; base += kMergeNT * kBatch) {
      uint32_t kv[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = base + u * kMergeNT + threadIdx.x;
        kv[u] = i < n ? ck[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = base + u * kMergeNT + threadIdx.x;
        if (i < n) merge_keys[i] = kv[u];
      }
    }
  }
  __syncthreads();
  const uint32_t floor = floor_s;
  auto emit = [&](int slot, int pos) { out[slot] = ci[pos]; };
  if (staged)
    block_select<kMergeNT>([&](int i) { return merge_keys[i]; }, n, kk, 0, sm, emit, floor);
  else
    block_select<kMergeNT>([&](int i) { return ck[i]; }, n, kk, 0, sm, emit, floor);
  for (int j = kk + threadIdx.x; j < a.k; j += kMergeNT) out[j] = -1;
  // The row's candidates are consumed: zero them (and the per-slice floors),
  // so that the workspace is all zero again when the call ends, as the
  // cooperative selection of a later call on the same workspace requires.
  __syncthreads();
  uint32_t* ckw = plan_cand_keys(plan, a.ws, bt);
  int32_t* ciw = plan_cand_idx(plan, a.ws, bt);
  for (int i = threadIdx.x; i < n; i += kMergeNT) {
    ckw[i] = 0u;
    ciw[i] = 0;
  }
  for (int j = threadIdx.x; j < plan.n_slices; j += kMergeNT) plan_cand_thr(plan, a.ws, bt)[j] = 0u;
}

size_t index_merge_smem(const IndexPlan& plan) {
  const int64_t cap = plan.cand_cap < kMergeSmemKeys ? plan.cand_cap : kMergeSmemKeys;
  return (size_t)cap * 4;
}

cudaError_t launch_index_merge(const IndexArgs& a, const IndexPlan& plan, cudaStream_t s) {
  const size_t smem = index_merge_smem(plan);
  cudaError_t e = cudaFuncSetAttribute(index_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  index_merge_kernel<<<dim3(a.n_q, a.batch), kMergeNT, smem, s>>>(a, plan);
  ++launch_counter();
  return cudaGetLastError();
}

// Slices: enough CTAs to cover the GPU about twice, each slice at most
// kMaxSlice entries (its keys live in shared memory).
IndexPlan make_simt_plan(int batch, int n_q, int64_t n_entries, int k) {
  constexpr int kMaxSlice = 16384;
  IndexPlan p{};
  p.n_rows = (int64_t)batch * n_q;
  const int64_t rows = p.n_rows > 0 ? p.n_rows : 1;
  const int64_t per_row = (296 + rows - 1) / rows;
  int64_t len = (n_entries + per_row - 1) / per_row;
  len = (len + 127) / 128 * 128;
  const int64_t lo = ((n_entries < 1024 ? n_entries : 1024) + 127) / 128 * 128;
  if (len < lo) len = lo;
  if (len < 128) len = 128;
  if (len > kMaxSlice) len = kMaxSlice;
  p.slice_len = (int)len;
  p.n_slices = (int)((n_entries + len - 1) / len);
  if (p.n_slices < 1) p.n_slices = 1;
  p.cand_cap = p.n_slices > 1 ? (int64_t)p.n_slices * k : 0;
  return p;
}

size_t index_simt_smem(const IndexArgs& a, const IndexPlan& plan) {
  return (size_t)a.n_heads * a.dim * 4 + (size_t)a.n_heads * 4 + (size_t)plan.slice_len * 4 +
         sizeof(SelectSmem<kNT>) + 16;
}

cudaError_t launch_index_simt(const IndexArgs& a, const IndexPlan& plan, cudaStream_t s) {
  const size_t smem = index_simt_smem(a, plan);
  cudaError_t e = cudaFuncSetAttribute(index_slice_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(plan.n_slices, a.n_q, a.batch);
  index_slice_simt_kernel<<<grid, kNT, smem, s>>>(a, plan);
  ++launch_counter();
  e = cudaGetLastError();
  if (e != cudaSuccess || plan.n_slices == 1) return e;
  return launch_index_merge(a, plan, s);
}

void index_topk_plan_info(int batch, int n_q, int64_t n_entries, int k, int n_heads, int dim, int dt,
                          int32_t* out) {
  IndexArgs probe{};
  probe.batch = batch; probe.n_q = n_q; probe.n_entries = n_entries; probe.k = k;
  probe.n_heads = n_heads; probe.dim = dim; probe.dt = dt;
  const bool tc = index_tc_eligible(probe);
  const IndexPlan p = tc ? make_tc_plan(batch, n_q, n_entries, k, dt) : make_simt_plan(batch, n_q, n_entries, k);
  out[0] = p.slice_len;
  out[1] = p.n_slices;
  out[2] = p.coop;
  out[3] = tc ? 1 : 0;
  int stages = 0, tiles_per_stage = 1;
  if (tc) index_tc_ring(n_q, dt, &stages, &tiles_per_stage);
  out[4] = stages;
  out[5] = tiles_per_stage;
}

size_t index_topk_workspace(int batch, int n_q, int64_t n_entries, int k, int n_heads, int dim,
                            int dt) {
  IndexArgs probe{};
  probe.batch = batch; probe.n_q = n_q; probe.n_entries = n_entries; probe.k = k;
  probe.n_heads = n_heads; probe.dim = dim; probe.dt = dt;
  if (index_tc_eligible(probe)) return plan_workspace_bytes(make_tc_plan(batch, n_q, n_entries, k, dt));
  return plan_workspace_bytes(make_simt_plan(batch, n_q, n_entries, k));
}

cudaError_t launch_index_topk(const IndexArgs& a, cudaStream_t s) {
  if ((int64_t)a.batch * a.n_q == 0) return cudaSuccess;
  if (index_tc_eligible(a)) {
    const IndexPlan plan = make_tc_plan(a.batch, a.n_q, a.n_entries, a.k, a.dt);
    cudaError_t e = launch_index_tc(a, plan, s);
    if (e != cudaSuccess || plan.n_slices == 1 || plan.coop) return e;
    return launch_index_merge(a, plan, s);
  }
  const IndexPlan plan = make_simt_plan(a.batch, a.n_q, a.n_entries, a.k);
  return launch_index_simt(a, plan, s);
}

}  // namespace csa
