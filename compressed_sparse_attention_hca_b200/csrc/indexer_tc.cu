// indexer_tc.cu -- tensor-core producer of the Lightning Indexer score
// ("DeepSeek-V4 内部机制" 1.2 Step 2: I[t,s] = sum_h w[t,h] ReLU(q[t,h].K[s]);
// 6.2: fp32 score rounded to BF16 before top-k), fused with the per-slice
// top-k selection.
//
// One CTA owns a group of NQ queries of one request and a slice of that
// request's entries.  The score tile is a dense contraction
//     D[128 entries, 64*NQ heads] = K_tile[128 x 128] . Q_group[64*NQ x 128]^T
// issued as tcgen05.mma (bf16 in, fp32 accumulate in TMEM), with both
// operands staged by TMA in the 128-byte-swizzled K-major layout.  Warp roles:
//   warp 0     TMA producer (query tile once, then a ring of K tiles),
//   warp 1     TMEM owner and MMA issuer (8 MMAs of K = 16 per tile),
//   warps 4-7  epilogue: each thread owns one entry row of the tile (one TMEM
//              lane), reads its 64 head scores per query, forms
//              sum_h w_h relu(score_h), rounds to bf16 and stores the 16-bit
//              order key in shared memory.
// The TMEM accumulator is double buffered so the epilogue of tile i overlaps
// the MMAs of tile i+1 and the loads of the following tiles.  After the last
// tile the whole CTA runs the radix select on the slice's keys (the score row
// never reaches HBM).
#include <cudaTypedefs.h>

#include "csa_internal.cuh"
#include "indexer_plan.cuh"
#include "sm100.cuh"
#include "topk_select.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_indexer_tc)

namespace {

constexpr int kTcThreads = 256;
constexpr int kBM = 128;                 // entries per tile (MMA M)
constexpr int kDI = 128;                 // indexer dim handled here
constexpr int kHI = 64;                  // indexer heads handled here
constexpr int kAtom = kBM * 128;         // bytes of one 128-byte-wide K atom of a K tile

template <int NQ>
struct TcCfg {
  static constexpr int N = kHI * NQ;                 // MMA N
  static constexpr int STAGES = NQ == 1 ? 4 : 3;
  static constexpr int Q_BYTES = N * 2 * kDI;        // two atoms of N rows x 128 B
  static constexpr int K_STAGE = kBM * 2 * kDI;      // two atoms of 128 rows x 128 B
  static constexpr int TMEM_COLS = 2 * N;            // double-buffered accumulator (128 or 256)
  static constexpr int FIXED_SMEM = 1024 /*align slack*/ + STAGES * K_STAGE + Q_BYTES + NQ * kHI * 4 +
                                    256 /*barriers*/ + (int)sizeof(SelectSmem<kTcThreads>);
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

template <int NQ>
__global__ void __launch_bounds__(kTcThreads, 1)
    index_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                    IndexArgs a, IndexPlan plan) {
  using C = TcCfg<NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ks = align1024(smem_raw);                        // K ring
  uint8_t* qs = ks + C::STAGES * C::K_STAGE;                // query tile
  uint16_t* keys = reinterpret_cast<uint16_t*>(qs + C::Q_BYTES);  // [NQ][slice_len]
  float* wsm = reinterpret_cast<float*>(keys + NQ * plan.slice_len);
  uint64_t* full = reinterpret_cast<uint64_t*>(wsm + NQ * kHI);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* qbar = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 1);
  SelectSmem<kTcThreads>& sel = *reinterpret_cast<SelectSmem<kTcThreads>*>(tmem_slot + 4);

  const int sl = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
  const int t0 = grp * NQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t s0 = (int64_t)sl * plan.slice_len;
  const int len = (int)min64(plan.slice_len, a.n_entries - s0);

  int n_valid[NQ];
  int64_t vis[NQ];
  int max_valid = 0;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int t = t0 + q;
    vis[q] = t < a.n_q ? visible_entries(a.q_pos[(int64_t)b * a.n_q + t], a.m, a.n_entries) : 0;
    n_valid[q] = (int)max64(0, min64(len, vis[q] - s0));
    max_valid = max(max_valid, n_valid[q]);
  }
  const int n_tiles = (max_valid + kBM - 1) / kBM;

  for (int i = threadIdx.x; i < NQ * kHI; i += kTcThreads) {
    const int t = t0 + i / kHI;
    wsm[i] = t < a.n_q ? a.wI[((int64_t)b * a.n_q + t) * kHI + (i % kHI)] : 0.f;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 4); }
    mbar_init(qbar, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      const int qrow = (b * a.n_q + t0) * kHI;
      mbar_arrive_expect_tx(qbar, C::Q_BYTES);
      tma_load_2d(qs, &tmQ, qbar, 0, qrow);
      tma_load_2d(qs + C::N * 128, &tmQ, qbar, 64, qrow);
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % C::STAGES, j = i / C::STAGES;
        if (j > 0 && !mbar_wait(&empty[s], (j - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[s], C::K_STAGE);
        const int row = (int)((int64_t)b * a.n_entries + s0 + (int64_t)i * kBM);
        uint8_t* dst = ks + s * C::K_STAGE;
        tma_load_2d(dst, &tmK, &full[s], 0, row);
        tma_load_2d(dst + kAtom, &tmK, &full[s], 64, row);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, C::N);
      bool ok = mbar_wait(qbar, 0);
      const uint32_t qa = smem_u32(qs);
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int s = i % C::STAGES, j = i / C::STAGES, buf = i & 1, u = i >> 1;
        if (!mbar_wait(&full[s], j & 1)) break;
        if (u > 0 && !mbar_wait(&acce[buf], (u - 1) & 1)) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(ks + s * C::K_STAGE);
        const uint32_t d = tmem + (uint32_t)(buf * C::N);
#pragma unroll
        for (int kk = 0; kk < kDI / 16; ++kk) {
          const uint32_t within = (uint32_t)(kk & 3) * 32u;  // 16 bf16 = 32 bytes
          const uint32_t a_addr = ka + (uint32_t)(kk >> 2) * kAtom + within;
          const uint32_t b_addr = qa + (uint32_t)(kk >> 2) * (C::N * 128) + within;
          tc_mma_f16(d, umma_desc_sw128(a_addr), umma_desc_sw128(b_addr), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
        tc_commit(&accf[buf]);
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    for (int i = 0; i < n_tiles; ++i) {
      const int buf = i & 1, u = i >> 1;
      if (!mbar_wait(&accf[buf], u & 1)) break;
      tc_fence_after();
      float acc[NQ][kHI];
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * C::N);
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        tmem_ld_32x32b_x32(taddr + q * kHI, &acc[q][0]);
        tmem_ld_32x32b_x32(taddr + q * kHI + 32, &acc[q][32]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
      const int pos = i * kBM + r;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        float I = 0.f;
#pragma unroll
        for (int h = 0; h < kHI; ++h) I = fmaf(wsm[q * kHI + h], fmaxf(acc[q][h], 0.f), I);
        const uint32_t key = bf16_key(I);
        const bool valid = pos < n_valid[q];
        keys[q * plan.slice_len + pos] = valid ? (uint16_t)(key >> 16) : (uint16_t)0;
        if (a.scores_out != nullptr && pos < len && t0 + q < a.n_q) {
          const float sc = valid ? key_to_f32(key) : -INFINITY;
          static_cast<__nv_bfloat16*>(a.scores_out)[((int64_t)b * a.n_q + t0 + q) * a.n_entries + s0 + pos] =
              __float2bfloat16_rn(sc);
        }
      }
    }
  }
  // debug scores of positions past the last computed tile
  if (a.scores_out != nullptr) {
    for (int q = 0; q < NQ; ++q) {
      if (t0 + q >= a.n_q) continue;
      for (int pos = n_tiles * kBM + threadIdx.x; pos < len; pos += kTcThreads)
        static_cast<__nv_bfloat16*>(a.scores_out)[((int64_t)b * a.n_q + t0 + q) * a.n_entries + s0 + pos] =
            __float2bfloat16_rn(-INFINITY);
    }
  }
  tc_fence_before();
  __syncthreads();

  // per-query top-k over this slice's keys
  for (int q = 0; q < NQ; ++q) {
    const int t = t0 + q;
    if (t >= a.n_q) break;
    const int64_t bt = (int64_t)b * a.n_q + t;
    const int nv = n_valid[q];
    const int kk = min(a.k, nv);
    const uint16_t* kq = keys + q * plan.slice_len;
    auto key_at = [&](int i) { return ((uint32_t)kq[i]) << 16; };
    if (plan.n_slices == 1) {
      int32_t* out = a.idx_out + bt * a.k;
      block_select<kTcThreads>(key_at, nv, kk, 2, sel, [&](int slot, int pos) { out[slot] = (int32_t)(s0 + pos); });
      for (int j = kk + threadIdx.x; j < a.k; j += kTcThreads) out[j] = -1;
    } else {
      const int64_t off = slice_cand_offset(plan, sl, vis[q], a.n_entries, a.k);
      uint32_t* ck = plan_cand_keys(plan, a.ws, bt) + off;
      int32_t* ci = plan_cand_idx(plan, a.ws, bt) + off;
      block_select<kTcThreads>(key_at, nv, kk, 2, sel, [&](int slot, int pos) {
        ck[slot] = key_at(pos);
        ci[slot] = (int32_t)(s0 + pos);
      });
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 tensor [rows][128] with 128-byte swizzled boxes of 64 x box_rows.
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDI * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NQ>
size_t tc_smem(const IndexPlan& p) {
  return (size_t)TcCfg<NQ>::FIXED_SMEM + (size_t)NQ * p.slice_len * 2;
}

template <int NQ>
cudaError_t launch_tc(const IndexArgs& a, const IndexPlan& p, cudaStream_t s) {
  CUtensorMap tmK, tmQ;
  if (!make_map_bf16(&tmK, a.KI, (uint64_t)a.batch * a.n_entries, kBM)) return cudaErrorInvalidValue;
  if (!make_map_bf16(&tmQ, a.qI, (uint64_t)a.batch * a.n_q * kHI, TcCfg<NQ>::N)) return cudaErrorInvalidValue;
  const size_t smem = tc_smem<NQ>(p);
  cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_slices, (a.n_q + NQ - 1) / NQ, a.batch);
  index_tc_kernel<NQ><<<grid, kTcThreads, smem, s>>>(tmK, tmQ, a, p);
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace

bool index_tc_eligible(const IndexArgs& a) {
  return a.dt == CSA_BF16 && a.n_heads == kHI && a.dim == kDI && a.n_entries > 0 &&
         (int64_t)a.batch * a.n_entries < ((int64_t)1 << 31) &&
         (int64_t)a.batch * a.n_q * kHI < ((int64_t)1 << 31);
}

int index_tc_nq(int n_q) { return n_q >= 2 ? 2 : 1; }

IndexPlan make_tc_plan(int batch, int n_q, int64_t n_entries, int k) {
  const int NQ = index_tc_nq(n_q);
  const int fixed = NQ == 1 ? TcCfg<1>::FIXED_SMEM : TcCfg<2>::FIXED_SMEM;
  constexpr int kSmemCap = 227 * 1024;
  int64_t max_slice = ((kSmemCap - fixed) / (2 * NQ)) / kBM * kBM;
  const int64_t groups = (n_q + NQ - 1) / NQ;
  const int64_t units = (int64_t)batch * groups;
  const int64_t want = units >= 148 ? 1 : (148 + units - 1) / units;
  int64_t len = (n_entries + want - 1) / want;
  len = (len + kBM - 1) / kBM * kBM;
  if (len < kBM) len = kBM;
  if (len > max_slice) len = max_slice;
  IndexPlan p{};
  p.slice_len = (int)len;
  p.n_slices = (int)((n_entries + len - 1) / len);
  if (p.n_slices < 1) p.n_slices = 1;
  p.n_rows = (int64_t)batch * n_q;
  p.cand_cap = p.n_slices > 1 ? (int64_t)p.n_slices * k : 0;
  return p;
}

cudaError_t launch_index_tc(const IndexArgs& a, const IndexPlan& p, cudaStream_t s) {
  return index_tc_nq(a.n_q) == 1 ? launch_tc<1>(a, p, s) : launch_tc<2>(a, p, s);
}

}  // namespace csa
