// mqa_umma.cu -- shared-KV multi-query attention on the 5th-generation tensor
// cores (tcgen05.mma, bf16 in, fp32 accumulate in TMEM) for c = 512 and head
// counts that are a multiple of 64 ("DeepSeek-V4 内部机制" 1.2 Step 2
// shared-KV MQA, 1.3 HCA, 1.4 window branch and sink equation; yunpan.plus
// eq. 9).
//
// A CTA owns one query, a group of 64 heads and a range of that query's
// attended rows, taken 128 at a time.  Each row is both key and value, so one
// gathered tile serves both products:
//   S^T[128 rows, 64 heads]  = K[128, 512] . Q[64, 512]^T
//       A = the row tile, K-major (128-byte swizzle, 8 atoms of 64 dims),
//       B = the query tile, K-major; D in TMEM (lane = row, column = head);
//   O^T[512 dims, 64 heads] += V^T[512, 128] . P^T[128, 64]
//       A = the same row tile read MN-major (a line = 64 dims of one row),
//       B = P written by the softmax threads MN-major (a line = the 64 heads
//       of one row); D = four 128-dim slabs in TMEM (lane = dim).
// The softmax runs on the 128 threads that own the TMEM lanes: thread r holds
// row r's 64 scores; per-head maxima across rows are warp max-reductions
// (redux.sync) and per-head sums warp reduce-scatters (each lane ends with
// two heads), both combined over four warps.
// The running maximum is only raised when a chunk exceeds it by more than
// 2^8, so O^T is rescaled in TMEM rarely (never within one chunk).
// FP8MIX rows are expanded to bf16 (value = e4m3 * block scale; RoPE dims
// copied) on their way into the row tile.
//
// With few queries (decode) a query's row chunks are split over several CTAs
// so that the grid fills the GPU; each writes its unnormalised partial
// (max, sum, o) to the workspace, and a combine kernel adds them in split
// order with the sink.
#include "csa_internal.cuh"
#include "mqa_plan.cuh"
#include "sm100.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_mqa_umma)

cudaError_t launch_mqa_combine(const MqaArgs& a, const MqaPlan& p, cudaStream_t s);

namespace {

constexpr int kDim = 512;
constexpr int kHG = 64;          // heads per CTA (N of both products)
constexpr int kRows = 128;       // rows per chunk (M of S^T)
constexpr int kThreads = 256;
constexpr int kMaxSel = 2048;    // selected entries per query (the top-k limit)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.f;     // log2 headroom before the running max is raised

// Shared memory (offsets from a 1024-byte aligned base).  The buffers are
// contiguous so that any descriptor stride stays inside them; the upper half
// of the row tile and P together stage a chunk of raw FP8MIX rows.
constexpr int kOffKV = 0;                        // 8 x [128 rows][128 B]    128 KB
constexpr int kOffP = kOffKV + 8 * kRows * 128;  // [128 rows][128 B]        16 KB
constexpr int kOffQ = kOffP + kRows * 128;       // 8 x [64 heads][128 B]    64 KB
constexpr int kOffMisc = kOffQ + 8 * kHG * 128;
constexpr int kRawRow = 608;                     // FP8MIX row at c = 512
constexpr int kOffRaw = kOffKV + 4 * kRows * 128;  // atoms 4..7 and P
static_assert(kOffRaw + kRows * kRawRow <= kOffQ, "raw staging fits in atoms 4..7 and P");
struct Misc {
  float m_use[kHG];    // running max per head (log2 domain)
  float l_run[kHG];    // running sum per head (relative to m_use)
  float corr[kHG];     // this chunk's rescale factor per head
  float fac[kHG];      // epilogue scale per head
  float red[4][kHG];   // per-warp partial max / sum
  const uint8_t* rowp[kRows];
  int32_t sel[kMaxSel];
  uint64_t bar_qk, bar_pv;
  uint32_t tmem_slot;
  int rescale;
};
constexpr int kSmemBytes = 1024 + kOffMisc + (int)sizeof(Misc);
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// TMEM columns: S^T (64), then O^T slabs s = 0..3 (64 each).
constexpr int kColS = 0;
constexpr int kColO = 64;
constexpr int kTmemCols = 512;

constexpr uint32_t kIdescQK = idesc_bf16_f32(kRows, kHG);
constexpr uint32_t kIdescPV = idesc_bf16_f32_major(128, kHG, 1, 1);

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}
// Row tile: byte offset of 16-byte chunk g (dims 8g .. 8g+7) of row r.
__device__ __forceinline__ uint32_t kv_off(int r, int g) {
  return (uint32_t)((g >> 3) * (kRows * 128) + r * 128 + ((((g & 7) ^ (r & 7))) << 4));
}
// Query tile: byte offset of 16-byte chunk g of head h.
__device__ __forceinline__ uint32_t q_off(int h, int g) {
  return (uint32_t)((g >> 3) * (kHG * 128) + h * 128 + ((((g & 7) ^ (h & 7))) << 4));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 bytes read -> 16 zero bytes written
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// Maximum over the warp's 32 lanes, returned to every lane (sm_100a).
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
// Barrier of the 128 softmax threads (warps 0-3).
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Producer / consumer halves of a named barrier over n threads.
__device__ __forceinline__ void named_barrier_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_barrier_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Warp reduce-scatter of 64 per-lane values (one per head): afterwards lane l
// holds the sum (or max) over the warp's 32 lanes for heads 2l and 2l+1.
template <bool MAX>
__device__ __forceinline__ void reduce_scatter64(float* v, int lane, float& r0, float& r1) {
#pragma unroll
  for (int k = 16, n = 32; k >= 1; k >>= 1, n >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float send = upper ? v[j] : v[j + n];
      const float keep = upper ? v[j + n] : v[j];
      const float recv = __shfl_xor_sync(0xffffffffu, send, k);
      v[j] = MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  r0 = v[0];
  r1 = v[1];
}

// How a CTA finishes: the whole query (normalised output) or one split of
// several (unnormalised partial for the combine kernel).
enum { kWhole = 0, kSplit = 1 };

template <bool FP8, int MODE>
__global__ void __launch_bounds__(kThreads, 1) mqa_umma_kernel(MqaArgs a, MqaPlan plan) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* Ps = base + kOffP;
  uint8_t* KV = base + kOffKV;
  uint8_t* Qs = base + kOffQ;
  Misc& ms = *reinterpret_cast<Misc*>(base + kOffMisc);

  const int split = blockIdx.x, hg = blockIdx.y;
  const int64_t bt = blockIdx.z;
  const int b = (int)(bt / a.n_q);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // query tile (64 heads x 512 dims) -> K-major swizzled atoms, issued first
  // (it depends on nothing)
  {
    const uint8_t* qg = static_cast<const uint8_t*>(a.Q) + ((bt * a.n_heads + (int64_t)hg * kHG) * kDim) * 2;
    for (int i = tid; i < kHG * 64; i += kThreads) {
      const int h = i >> 6, g = i & 63;
      cp_async16(smem_u32(Qs + q_off(h, g)), qg + (int64_t)h * (kDim * 2) + g * 16, true);
    }
    cp_async_commit();
  }
  const int64_t tq = a.q_pos[bt];
  const RowList rl = make_row_list(a, bt, tq);
  // split s of NS takes chunks [s * nch / NS, (s + 1) * nch / NS) of the rows
  const int NS = plan.n_splits;
  const int64_t nch = (rl.n_rows + kRows - 1) / kRows;
  const int64_t r_begin = (int64_t)split * nch / NS * kRows;
  const int64_t r_end = min64(rl.n_rows, ((int64_t)split + 1) * nch / NS * kRows);
  const int n_chunks = r_end > r_begin ? (int)((r_end - r_begin + kRows - 1) / kRows) : 0;
  const int64_t rb = row_bytes(a.kv_dt, kDim);

  if (tid == 0) {
    mbar_init(&ms.bar_qk, 1);
    mbar_init(&ms.bar_pv, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(&ms.tmem_slot, kTmemCols);
  if (tid < kHG) {
    ms.m_use[tid] = -INFINITY;
    ms.l_run[tid] = 0.f;
  }
  // the selected entry indices of this CTA's rows, fetched once
  const int64_t sel_end = rl.sel ? min64(r_end, rl.n_sel) : r_begin;
  for (int64_t r = r_begin + tid; r < sel_end; r += kThreads) ms.sel[r - r_begin] = rl.sel[r];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_slot;
  const float sl2 = a.scale * kLog2e;

  for (int ci = 0; ci < n_chunks; ++ci) {
    // ---- row pointers and validity
    if (tid < kRows) {
      const int64_t r = r_begin + (int64_t)ci * kRows + tid;
      const uint8_t* p = nullptr;
      if (r < r_end) {
        if (r < rl.n_sel) {
          const int64_t e = rl.sel ? (int64_t)ms.sel[r - r_begin] : r;
          if (e >= 0 && e < rl.vis) p = static_cast<const uint8_t*>(a.entries) + ((int64_t)b * a.n_entries + e) * rb;
        } else {
          p = row_ptr(a, rl, b, r, rb);
        }
      }
      ms.rowp[tid] = p;
    }
    __syncthreads();
    // ---- gather the rows into the row tile (zeros for absent rows)
    if (!FP8) {
      for (int u = tid; u < kRows * 64; u += kThreads) {
        const int r = u >> 6, g = u & 63;
        const uint8_t* src = ms.rowp[r];
        cp_async16(smem_u32(KV + kv_off(r, g)), src ? src + g * 16 : static_cast<const uint8_t*>(a.Q), src != nullptr);
      }
      cp_async_commit();
      cp_async_wait_all();
    } else {
      // FP8MIX: the raw rows land in atoms 4..7 + P in one cp.async round
      // trip, then expand (codes x block scale -> bf16, RoPE dims copied):
      // dims 0..255 straight into atoms 0..3, dims 256..511 through registers
      // (their destination overlaps the staging area)
      uint8_t* raw = base + kOffRaw;
      for (int u = tid; u < kRows * (kRawRow / 16); u += kThreads) {
        const int r = u / (kRawRow / 16), c = u % (kRawRow / 16);
        const uint8_t* src = ms.rowp[r];
        cp_async16(smem_u32(raw + r * kRawRow + c * 16), src ? src + c * 16 : static_cast<const uint8_t*>(a.Q),
                   src != nullptr);
      }
      cp_async_commit();
      cp_async_wait_all();
      __syncthreads();
      auto expand = [&](int r, int g) -> uint4 {
        const uint8_t* row = raw + r * kRawRow;
        if (g >= 56) return *reinterpret_cast<const uint4*>(row + 448 + (g - 56) * 16);
        const uint2 v = *reinterpret_cast<const uint2*>(row + g * 8);
        const float sc = *reinterpret_cast<const float*>(row + 576 + 4 * (g >> 3));
        uint32_t w[4];
        const uint32_t src[2] = {v.x, v.y};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float2 lo = e4m3x2_to_float2((uint16_t)(src[q] & 0xFFFF));
          const float2 hi = e4m3x2_to_float2((uint16_t)(src[q] >> 16));
          const __nv_bfloat162 x0 = __floats2bfloat162_rn(lo.x * sc, lo.y * sc);
          const __nv_bfloat162 x1 = __floats2bfloat162_rn(hi.x * sc, hi.y * sc);
          memcpy(&w[2 * q], &x0, 4);
          memcpy(&w[2 * q + 1], &x1, 4);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
      };
      // absent rows were zero-filled: zero codes and scales expand to zeros
      for (int u = tid; u < kRows * 32; u += kThreads) {
        const int r = u >> 5, g = u & 31;
        *reinterpret_cast<uint4*>(KV + kv_off(r, g)) = expand(r, g);
      }
      constexpr int kHi = kRows * 32 / kThreads;  // 16 chunks per thread
      uint4 hi[kHi];
#pragma unroll
      for (int j = 0; j < kHi; ++j) {
        const int u = tid + j * kThreads;
        hi[j] = expand(u >> 5, 32 + (u & 31));
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kHi; ++j) {
        const int u = tid + j * kThreads;
        *reinterpret_cast<uint4*>(KV + kv_off(u >> 5, 32 + (u & 31))) = hi[j];
      }
    }
    fence_proxy_async_smem();  // generic-proxy tile writes -> tensor core reads
    __syncthreads();

    // ---- S^T = K Q^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kva = smem_u32(KV), qa = smem_u32(Qs);
#pragma unroll
      for (int at = 0; at < 8; ++at)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_f16(tmem + kColS, umma_desc_sw128(kva + at * (kRows * 128) + kk * 32),
                     umma_desc_sw128(qa + at * (kHG * 128) + kk * 32), kIdescQK, (at | kk) ? 1u : 0u);
      tc_commit(&ms.bar_qk);
    }

    // ---- softmax on the 128 threads that own the TMEM lanes (row = tid)
    if (warp < 4) {
      mbar_wait(&ms.bar_qk, (uint32_t)(ci & 1));
      tc_fence_after();
      float s[kHG];
      const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
      tmem_ld_32x32b_x32(tmem + lane_base + kColS, s);
      tmem_ld_32x32b_x32(tmem + lane_base + kColS + 32, s + 32);
      tmem_ld_wait();
      const bool ok = ms.rowp[tid] != nullptr;
#pragma unroll
      for (int h = 0; h < kHG; ++h) s[h] = ok ? s[h] * sl2 : -INFINITY;
      // per-head maximum over the warp's 32 rows (one redux per head)
#pragma unroll
      for (int h = 0; h < kHG; ++h) {
        const float wm = warp_max_f32(s[h]);
        if (lane == (h >> 1)) ms.red[warp][h] = wm;
      }
      softmax_sync();
      if (warp == 0) {
        bool raised = false;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int h = 2 * lane + j;
          const float cm = fmaxf(fmaxf(ms.red[0][h], ms.red[1][h]), fmaxf(ms.red[2][h], ms.red[3][h]));
          const float mold = ms.m_use[h];
          float use = mold;
          if (mold == -INFINITY || cm > mold + kLazy) use = fmaxf(mold, cm);
          ms.corr[h] = (mold == -INFINITY || use == mold) ? 1.f : exp2f(mold - use);
          raised |= mold != -INFINITY && use != mold;
          ms.m_use[h] = use;
        }
        const unsigned any = __ballot_sync(0xffffffffu, raised);
        if (lane == 0) ms.rescale = any != 0u;
      }
      softmax_sync();
      // P = 2^(s - m) as bf16, written MN-major (a 128-byte line per row)
#pragma unroll
      for (int h = 0; h < kHG; ++h) {
        const float m = ms.m_use[h];
        s[h] = (s[h] == -INFINITY || m == -INFINITY) ? 0.f : exp2f(s[h] - m);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 x = __floats2bfloat162_rn(s[8 * c + 2 * q], s[8 * c + 2 * q + 1]);
          memcpy(&w[q], &x, 4);
        }
        *reinterpret_cast<uint4*>(Ps + tid * 128 + ((c ^ (tid & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      // row sums per head of the bf16 probabilities the product will use
      float v[kHG], c0, c1;
#pragma unroll
      for (int h = 0; h < kHG; ++h) v[h] = __bfloat162float(__float2bfloat16_rn(s[h]));
      reduce_scatter64<false>(v, lane, c0, c1);
      ms.red[warp][2 * lane] = c0;
      ms.red[warp][2 * lane + 1] = c1;
      softmax_sync();
      if (warp == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int h = 2 * lane + j;
          const float cs = (ms.red[0][h] + ms.red[1][h]) + (ms.red[2][h] + ms.red[3][h]);
          ms.l_run[h] = ms.l_run[h] * ms.corr[h] + cs;
        }
      }
      // a raised max rescales the output accumulated so far (lane = dim)
      if (ci > 0 && ms.rescale) {
#pragma unroll 1
        for (int sl = 0; sl < 4; ++sl) {
          float o[kHG];
          const uint32_t ta = tmem + lane_base + kColO + sl * kHG;
          tmem_ld_32x32b_x32(ta, o);
          tmem_ld_32x32b_x32(ta + 32, o + 32);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < kHG; ++h) o[h] *= ms.corr[h];
          tmem_st_32x32b_x32(ta, o);
          tmem_st_32x32b_x32(ta + 32, o + 32);
        }
        tmem_st_wait();
      }
      tc_fence_before();
    }
    fence_proxy_async_smem();  // P (generic stores) -> tensor core reads
    __syncthreads();

    // ---- O^T += V^T P^T, four 128-dim slabs
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kva = smem_u32(KV), pa = smem_u32(Ps);
#pragma unroll
      for (int sl = 0; sl < 4; ++sl)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_f16(tmem + kColO + sl * kHG,
                     umma_desc_sw128_mn(kva + (2 * sl) * (kRows * 128) + kk * 2048, kRows * 128, 1024),
                     umma_desc_sw128_mn(pa + kk * 2048, kRows * 128, 1024), kIdescPV,
                     (ci > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&ms.bar_pv);
    }
    // the next chunk overwrites the row tile and P: wait for the product
    mbar_wait(&ms.bar_pv, (uint32_t)(ci & 1));
    tc_fence_after();
  }
  cp_async_wait_all();
  __syncthreads();
  // ---- epilogue: O[h][d] = O^T[d][h] * fac[h]
  const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
  auto load_slab = [&](int sl, float* o) {  // warps 0-3: lane = dim sl * 128 + tid
    if (n_chunks > 0) {
      tmem_ld_32x32b_x32(tmem + lb + kColO + sl * kHG, o);
      tmem_ld_32x32b_x32(tmem + lb + kColO + sl * kHG + 32, o + 32);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int h = 0; h < kHG; ++h) o[h] = 0.f;
    }
  };
  if constexpr (MODE != kWhole) {
    // one split of many: the unnormalised partial (m, l, o).  Warps 0-3 stage
    // the O^T slabs in the idle row tile as [slab][head][128 dims] while warps
    // 4-7 write the slabs already staged in 16-byte pieces (each warp store
    // covers 512 contiguous bytes of one head); named barrier 2 + s marks
    // slab s staged.
    float* stg = reinterpret_cast<float*>(KV);
    if (tid < kHG) {
      float* ml = plan_partial_ml(plan, a, bt, split, hg * kHG + tid);
      const float m = ms.m_use[tid];
      ml[0] = m == -INFINITY ? -INFINITY : m / kLog2e;  // natural-log domain
      ml[1] = ms.l_run[tid];
    }
    if (warp < 4) {
#pragma unroll 1
      for (int sl = 0; sl < 4; ++sl) {
        float o[kHG];
        load_slab(sl, o);
#pragma unroll
        for (int h = 0; h < kHG; ++h) stg[(sl * kHG + h) * 128 + tid] = o[h];
        named_barrier_arrive(2 + sl, kThreads);
      }
    } else {
      const int t = tid - 128;
#pragma unroll 1
      for (int sl = 0; sl < 4; ++sl) {
        named_barrier_sync(2 + sl, kThreads);
        for (int q = t; q < kHG * 32; q += 128) {
          const int h = q >> 5, c = q & 31;
          const float4 v = *reinterpret_cast<const float4*>(stg + (sl * kHG + h) * 128 + 4 * c);
          *reinterpret_cast<float4*>(plan_partial_o(plan, a, bt, split, hg * kHG + h) + sl * 128 + 4 * c) = v;
        }
      }
    }
  } else {
    if (tid < kHG) {
      const float sink = a.sink[hg * kHG + tid] * kLog2e;  // log2 domain
      const float m = ms.m_use[tid];
      const float M = fmaxf(m, sink);
      float f = 0.f;
      if (!(sink == INFINITY) && M != -INFINITY) {
        const float em = m == -INFINITY ? 0.f : exp2f(m - M);
        f = em / (ms.l_run[tid] * em + exp2f(sink - M));
      }
      ms.fac[tid] = f;
    }
    __syncthreads();
    if (warp < 4) {
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(a.O) + (bt * a.n_heads + (int64_t)hg * kHG) * kDim;
#pragma unroll 1
      for (int sl = 0; sl < 4; ++sl) {
        float o[kHG];
        load_slab(sl, o);
#pragma unroll
        for (int h = 0; h < kHG; ++h) ob[(int64_t)h * kDim + sl * 128 + tid] = __float2bfloat16_rn(o[h] * ms.fac[h]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

bool mqa_umma_eligible(const MqaArgs& a) {
  return a.q_dt == CSA_BF16 && (a.kv_dt == CSA_BF16 || a.kv_dt == CSA_KV_FP8MIX) && a.dim == kDim &&
         a.n_heads % kHG == 0 && (int64_t)a.batch * a.n_q <= 65535 && (a.idx == nullptr || a.k <= kMaxSel);
}

MqaPlan make_umma_mqa_plan(const MqaArgs& a) {
  MqaPlan p{};
  p.heads_per_cta = kHG;
  p.rows_per_split = 0;
  // few queries (decode): a query's row chunks are split over CTAs until the
  // grid fills one wave; the partials are combined by mqa_combine_kernel
  const int64_t units = (int64_t)a.batch * a.n_q * (a.n_heads / kHG);
  const int64_t nch = (max_rows_per_query(a) + kRows - 1) / kRows;
  int64_t ns = 148 / units;
  if (ns > nch) ns = nch;
  if (ns < 1) ns = 1;
  p.n_splits = (int)ns;
  return p;
}

template <bool FP8, int MODE>
cudaError_t launch_umma(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  auto kern = mqa_umma_kernel<FP8, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)p.n_splits, a.n_heads / kHG, (unsigned)((int64_t)a.batch * a.n_q));
  kern<<<grid, kThreads, kSmemBytes, s>>>(a, p);
  ++launch_counter();
  e = cudaGetLastError();
  if (e != cudaSuccess || MODE != kSplit) return e;
  return launch_mqa_combine(a, p, s);
}

template <bool FP8>
cudaError_t launch_umma_fmt(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  return p.n_splits > 1 ? launch_umma<FP8, kSplit>(a, p, s) : launch_umma<FP8, kWhole>(a, p, s);
}

}  // namespace

bool mqa_umma_path(const MqaArgs& a) { return mqa_umma_eligible(a); }
MqaPlan mqa_umma_plan(const MqaArgs& a) { return make_umma_mqa_plan(a); }
cudaError_t launch_mqa_umma(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  return a.kv_dt == CSA_KV_FP8MIX ? launch_umma_fmt<true>(a, p, s) : launch_umma_fmt<false>(a, p, s);
}

}  // namespace csa
