// indexer_tc.cu -- tensor-core producer of the Lightning Indexer score
// ("DeepSeek-V4 内部机制" 1.2 Step 2: I[t,s] = sum_h w[t,h] ReLU(q[t,h].K[s]);
// 6.2: FP4 q/K, fp32 score rounded to BF16 before top-k), fused with the
// per-slice top-k selection.
//
// One CTA owns a group of NQ queries of one request and a slice of that
// request's entries.  The score tile is a dense contraction
//     D[128 entries, 64*NQ heads] = K_tile[128 x 128] . Q_group[64*NQ x 128]^T
// issued as tcgen05.mma (16-bit inputs, fp32 accumulate in TMEM) over operands
// in the 128-byte-swizzled K-major shared-memory layout.
//
// BF16 inputs: TMA writes the K tiles straight into the operand ring.
// NVFP4 inputs: TMA brings the packed E2M1 codes and E4M3 block scales (72
//   bytes per entry, the HBM traffic) into a raw ring; converter warps expand
//   them to fp16 in the swizzled layout.  Every e2m1 x e4m3 product is exact
//   in fp16 (at most 6 significant bits, magnitudes 2^-10 .. 2688), so the
//   fp16 MMA with fp32 accumulation sees exactly the decoded values.
//
// Warp roles: warp 0 TMA producer; warp 1 TMEM owner and MMA issuer (8 MMAs of
// K = 16 per tile); warps 4-7 epilogue (each thread owns one entry row = one
// TMEM lane, reads its 64 head scores per query, forms sum_h w_h relu(s_h),
// rounds to bf16, stores the 16-bit order key in shared memory); NVFP4 only:
// warps 2, 3, 8-11 convert.  The TMEM accumulator is double buffered.  After
// the last tile the whole CTA runs the radix select on the slice's keys (the
// score row never reaches HBM).
#include <cudaTypedefs.h>

#include "csa_internal.cuh"
#include "indexer_plan.cuh"
#include "sm100.cuh"
#include "topk_select.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_indexer_tc)

namespace {

constexpr int kBM = 128;          // entries per tile (MMA M)
constexpr int kDI = 128;          // indexer dim handled here
constexpr int kHI = 64;           // indexer heads handled here
constexpr int kAtom = kBM * 128;  // bytes of one 128-byte-wide K atom of a K tile
constexpr int kConvWarps = 6;     // NVFP4 converter warps: 2, 3, 8, 9, 10, 11

template <int NQ, bool FP4>
struct TcCfg {
  static constexpr int N = kHI * NQ;                        // MMA N
  static constexpr int THREADS = FP4 ? 384 : 256;
  static constexpr int STAGES = FP4 ? 3 : (NQ == 1 ? 4 : 3);  // 16-bit operand ring
  static constexpr int RSTAGES = FP4 ? 6 : 0;               // raw NVFP4 ring
  static constexpr int Q_BYTES = N * 2 * kDI;               // two atoms of N rows x 128 B
  static constexpr int K_STAGE = kBM * 2 * kDI;             // two atoms of 128 rows x 128 B
  static constexpr int R_CODES = kBM * kDI / 2;             // 8 KB of E2M1 codes per tile
  static constexpr int R_STAGE = R_CODES + kBM * kDI / 16;  // + 1 KB of scales
  static constexpr int QRAW = FP4 ? (N * kDI / 2 + N * kDI / 16 + 1023) / 1024 * 1024 : 0;
  static constexpr int TMEM_COLS = 2 * N;                   // double-buffered accumulator
  static constexpr int FIXED_SMEM = 1024 /*align slack*/ + STAGES * K_STAGE + Q_BYTES + RSTAGES * R_STAGE +
                                    QRAW + NQ * kHI * 4 + 512 /*barriers*/ +
                                    (int)sizeof(SelectSmem<THREADS>);
  static constexpr uint32_t IDESC = FP4 ? idesc_f16_f32(kBM, N) : idesc_bf16_f32(kBM, N);
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// 8 E2M1 values (4 bytes, element 2j in the low nibble of byte j) times their
// E4M3 block scale -> 8 fp16 values (exact).
__device__ __forceinline__ uint4 fp4x8_to_f16x8(uint32_t codes, uint8_t sf) {
  const __half2_raw sr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(sf | (sf << 8)), __NV_E4M3);
  __half2 s;
  memcpy(&s, &sr, 4);
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __half2_raw vr = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((codes >> (8 * j)) & 0xFFu), __NV_E2M1);
    __half2 v;
    memcpy(&v, &vr, 4);
    const __half2 p = __hmul2(v, s);
    memcpy(&w[j], &p, 4);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Offset of 16-byte chunk c (elements 8c..8c+7) of row r inside a K-major
// operand of `rows` rows stored as two 128-byte-swizzled atoms.
__device__ __forceinline__ uint32_t sw128_chunk_offset(int r, int c, int rows) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int NQ, bool FP4>
__global__ void __launch_bounds__(TcCfg<NQ, FP4>::THREADS, 1)
    index_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmQs,
                    IndexArgs a, IndexPlan plan) {
  using C = TcCfg<NQ, FP4>;
  constexpr int NT = C::THREADS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ks = align1024(smem_raw);                          // 16-bit operand ring
  uint8_t* qs = ks + C::STAGES * C::K_STAGE;                  // 16-bit query tile
  uint8_t* rs = qs + C::Q_BYTES;                              // raw NVFP4 ring
  uint8_t* qraw = rs + C::RSTAGES * C::R_STAGE;               // raw NVFP4 query tile
  uint16_t* keys = reinterpret_cast<uint16_t*>(qraw + C::QRAW);  // [NQ][slice_len]
  float* wsm = reinterpret_cast<float*>(keys + NQ * plan.slice_len);
  uint64_t* ofull = reinterpret_cast<uint64_t*>(wsm + NQ * kHI);
  uint64_t* oempty = ofull + C::STAGES;
  uint64_t* rfull = oempty + C::STAGES;
  uint64_t* rempty = rfull + 8;
  uint64_t* accf = rempty + 8;
  uint64_t* acce = accf + 2;
  uint64_t* qbar = acce + 2;
  uint64_t* qconv = qbar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qconv + 1);
  SelectSmem<NT>& sel = *reinterpret_cast<SelectSmem<NT>*>(tmem_slot + 4);

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

  for (int i = threadIdx.x; i < NQ * kHI; i += NT) {
    const int t = t0 + i / kHI;
    wsm[i] = t < a.n_q ? a.wI[((int64_t)b * a.n_q + t) * kHI + (i % kHI)] : 0.f;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&ofull[s], FP4 ? kConvWarps : 1);
      mbar_init(&oempty[s], 1);
    }
    for (int s = 0; s < C::RSTAGES; ++s) {
      mbar_init(&rfull[s], 1);
      mbar_init(&rempty[s], kConvWarps);
    }
    for (int i = 0; i < 2; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 4); }
    mbar_init(qbar, 1);
    mbar_init(qconv, kConvWarps);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool conv_warp = FP4 && (warp == 2 || warp == 3 || warp >= 8);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int qrow = (b * a.n_q + t0) * kHI;
      if (FP4) {
        mbar_arrive_expect_tx(qbar, C::N * kDI / 2 + C::N * kDI / 16);
        tma_load_2d(qraw, &tmQ, qbar, 0, qrow);
        tma_load_2d(qraw + C::N * kDI / 2, &tmQs, qbar, 0, qrow / 2);
      } else {
        mbar_arrive_expect_tx(qbar, C::Q_BYTES);
        tma_load_2d(qs, &tmQ, qbar, 0, qrow);
        tma_load_2d(qs + C::N * 128, &tmQ, qbar, 64, qrow);
      }
      for (int i = 0; i < n_tiles; ++i) {
        const int row = (int)((int64_t)b * a.n_entries + s0 + (int64_t)i * kBM);
        if (FP4) {
          const int s = i % C::RSTAGES, j = i / C::RSTAGES;
          if (j > 0 && !mbar_wait(&rempty[s], (j - 1) & 1)) break;
          mbar_arrive_expect_tx(&rfull[s], C::R_STAGE);
          uint8_t* dst = rs + s * C::R_STAGE;
          tma_load_2d(dst, &tmK, &rfull[s], 0, row);
          tma_load_2d(dst + C::R_CODES, &tmKs, &rfull[s], 0, row / 2);
        } else {
          const int s = i % C::STAGES, j = i / C::STAGES;
          if (j > 0 && !mbar_wait(&oempty[s], (j - 1) & 1)) break;
          mbar_arrive_expect_tx(&ofull[s], C::K_STAGE);
          uint8_t* dst = ks + s * C::K_STAGE;
          tma_load_2d(dst, &tmK, &ofull[s], 0, row);
          tma_load_2d(dst + kAtom, &tmK, &ofull[s], 64, row);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(FP4 ? qconv : qbar, 0);
      const uint32_t qa = smem_u32(qs);
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int s = i % C::STAGES, j = i / C::STAGES, buf = i & 1, u = i >> 1;
        if (!mbar_wait(&ofull[s], j & 1)) break;
        if (u > 0 && !mbar_wait(&acce[buf], (u - 1) & 1)) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(ks + s * C::K_STAGE);
        const uint32_t d = tmem + (uint32_t)(buf * C::N);
#pragma unroll
        for (int kk = 0; kk < kDI / 16; ++kk) {
          const uint32_t within = (uint32_t)(kk & 3) * 32u;  // 16 elements of 2 bytes
          const uint32_t a_addr = ka + (uint32_t)(kk >> 2) * kAtom + within;
          const uint32_t b_addr = qa + (uint32_t)(kk >> 2) * (C::N * 128) + within;
          tc_mma_f16(d, umma_desc_sw128(a_addr), umma_desc_sw128(b_addr), C::IDESC, kk > 0 ? 1u : 0u);
        }
        tc_commit(&oempty[s]);
        tc_commit(&accf[buf]);
      }
    }
  } else if (conv_warp) {
    // ------------------------------------------------- NVFP4 -> fp16 converters
    const int ct = (warp < 4 ? warp - 2 : warp - 6) * 32 + lane;
    constexpr int CT = kConvWarps * 32;
    bool ok = mbar_wait(qbar, 0);
    if (ok) {
      for (int ch = ct; ch < C::N * 16; ch += CT) {
        const int r = ch >> 4, c = ch & 15;
        const uint32_t codes = *reinterpret_cast<const uint32_t*>(qraw + r * 64 + c * 4);
        const uint8_t sf = qraw[C::N * kDI / 2 + r * 8 + (c >> 1)];
        *reinterpret_cast<uint4*>(qs + sw128_chunk_offset(r, c, C::N)) = fp4x8_to_f16x8(codes, sf);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(qconv);
    for (int i = 0; ok && i < n_tiles; ++i) {
      const int rsi = i % C::RSTAGES, rj = i / C::RSTAGES;
      const int osi = i % C::STAGES, oj = i / C::STAGES;
      if (!mbar_wait(&rfull[rsi], rj & 1)) break;
      if (oj > 0 && !mbar_wait(&oempty[osi], (oj - 1) & 1)) break;
      const uint8_t* src = rs + rsi * C::R_STAGE;
      uint8_t* dst = ks + osi * C::K_STAGE;
      for (int ch = ct; ch < kBM * 16; ch += CT) {
        const int r = ch >> 4, c = ch & 15;
        const uint32_t codes = *reinterpret_cast<const uint32_t*>(src + r * 64 + c * 4);
        const uint8_t sf = src[C::R_CODES + r * 8 + (c >> 1)];
        *reinterpret_cast<uint4*>(dst + sw128_chunk_offset(r, c, kBM)) = fp4x8_to_f16x8(codes, sf);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&rempty[rsi]);
        mbar_arrive(&ofull[osi]);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // --------------------------------------------------------------- epilogue
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
      for (int pos = n_tiles * kBM + threadIdx.x; pos < len; pos += NT)
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
      block_select<NT>(key_at, nv, kk, 2, sel, [&](int slot, int pos) { out[slot] = (int32_t)(s0 + pos); });
      for (int j = kk + threadIdx.x; j < a.k; j += NT) out[j] = -1;
    } else {
      const int64_t off = slice_cand_offset(plan, sl, vis[q], a.n_entries, a.k);
      uint32_t* ck = plan_cand_keys(plan, a.ws, bt) + off;
      int32_t* ci = plan_cand_idx(plan, a.ws, bt) + off;
      block_select<NT>(key_at, nv, kk, 2, sel, [&](int slot, int pos) {
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

// 2D tensor [rows][cols] of `dtype` elements (row stride cols * esize bytes)
// with boxes of box_cols x box_rows.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int esize, const void* base, uint64_t rows,
                 uint64_t cols, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NQ, bool FP4>
size_t tc_smem(const IndexPlan& p) {
  return (size_t)TcCfg<NQ, FP4>::FIXED_SMEM + (size_t)NQ * p.slice_len * 2;
}

template <int NQ, bool FP4>
cudaError_t launch_tc(const IndexArgs& a, const IndexPlan& p, cudaStream_t s) {
  using C = TcCfg<NQ, FP4>;
  CUtensorMap tmK, tmQ, tmKs, tmQs;
  const uint64_t krows = (uint64_t)a.batch * a.n_entries, qrows = (uint64_t)a.batch * a.n_q * kHI;
  bool ok;
  if (FP4) {
    // codes [rows][64 B]; scales viewed as [rows/2][16 B] (two entries per line)
    ok = make_map_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.KI, krows, kDI / 2, kDI / 2, kBM,
                     CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map_2d(&tmKs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.KI_sf, krows / 2, 16, 16, kBM / 2,
                     CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.qI, qrows, kDI / 2, kDI / 2, C::N,
                     CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_map_2d(&tmQs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.qI_sf, qrows / 2, 16, 16, C::N / 2,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    ok = make_map_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.KI, krows, kDI, 64, kBM,
                     CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.qI, qrows, kDI, 64, C::N,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    tmKs = tmK;
    tmQs = tmQ;
  }
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = tc_smem<NQ, FP4>(p);
  cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<NQ, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_slices, (a.n_q + NQ - 1) / NQ, a.batch);
  index_tc_kernel<NQ, FP4><<<grid, C::THREADS, smem, s>>>(tmK, tmQ, tmKs, tmQs, a, p);
  ++launch_counter();
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool index_tc_eligible(const IndexArgs& a) {
  if (a.n_heads != kHI || a.dim != kDI || a.n_entries <= 0) return false;
  if ((int64_t)a.batch * a.n_entries >= ((int64_t)1 << 31) || (int64_t)a.batch * a.n_q * kHI >= ((int64_t)1 << 31))
    return false;
  if (a.dt == CSA_BF16) return true;
  // NVFP4: the scale arrays are streamed as 16-byte lines of two entries, so
  // the entry count must be even and the scale arrays 16-byte aligned.
  return a.dt == CSA_IDX_NVFP4 && a.n_entries % 2 == 0 && aligned16(a.KI_sf) && aligned16(a.qI_sf);
}

int index_tc_nq(int n_q) { return n_q >= 2 ? 2 : 1; }

IndexPlan make_tc_plan(int batch, int n_q, int64_t n_entries, int k, int dt) {
  const int NQ = index_tc_nq(n_q);
  const bool fp4 = dt == CSA_IDX_NVFP4;
  const int fixed = NQ == 1 ? (fp4 ? TcCfg<1, true>::FIXED_SMEM : TcCfg<1, false>::FIXED_SMEM)
                            : (fp4 ? TcCfg<2, true>::FIXED_SMEM : TcCfg<2, false>::FIXED_SMEM);
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
  const bool fp4 = a.dt == CSA_IDX_NVFP4;
  if (index_tc_nq(a.n_q) == 1) return fp4 ? launch_tc<1, true>(a, p, s) : launch_tc<1, false>(a, p, s);
  return fp4 ? launch_tc<2, true>(a, p, s) : launch_tc<2, false>(a, p, s);
}

}  // namespace csa
