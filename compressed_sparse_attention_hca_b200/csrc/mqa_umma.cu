// mqa_umma.cu -- shared-KV multi-query attention on the 5th-generation tensor
// cores (tcgen05.mma, bf16 in, fp32 accumulate in TMEM) for c = 512 and head
// counts that are a multiple of 64 ("DeepSeek-V4 内部机制" 1.2 Step 2
// shared-KV MQA, 1.3 HCA, 1.4 window branch, sink equation, and the RMSNorm /
// partial-RoPE rows of its table; yunpan.plus eq. 9).
//
// A CTA owns one query, a group of 64 heads and a range of that query's
// attended rows, taken 128 at a time (a chunk).  Each row is both key and
// value, so one gathered tile serves both products:
//   S^T[128 rows, 64 heads]  = K[128, 512] . Q[64, 512]^T
//       A = the row tile, K-major (128-byte swizzle, 8 atoms of 64 dims),
//       B = the query tile, K-major; D in TMEM (lane = row, column = head);
//   O^T[512 dims, 64 heads] += V^T[512, 128] . P^T[128, 64]
//       A = the same row tile read MN-major (a line = 64 dims of one row),
//       B = P written by the softmax threads MN-major (a line = the 64 heads
//       of one row); D = four 128-dim slabs in TMEM (lane = dim);
//   L[., 64 heads]          += 1[128, 128] . P^T[128, 64]
//       the per-head sums of P on the tensor core (A = ones kept in TMEM):
//       every lane of L holds the running denominators.
// Per chunk: the rows are gathered (FP8MIX rows by one bulk copy each, then
// expanded to bf16 -- value = e4m3 * block scale, RoPE dims copied -- half
// the tile at a time, the S^T MMAs of a half issued as soon as it is ready;
// BF16 rows by cp.async, the S^T MMAs of each 128-dim pair of atoms issued as
// it lands); eight warps then take the softmax (per-head maxima over the rows
// by warp max-reductions, P = 2^(s - m) in bf16); the running maximum is only
// raised when a chunk exceeds it by more than 2^8, so O^T and L are rescaled
// in TMEM rarely.  A CTA with several BF16 chunks gathers the next chunk's
// atoms as soon as the products of the current chunk have read them.
//
// The query tile arrives by TMA; the first chunk's entry indices are fetched
// together with the query position.
//
// Rows split over several CTAs (decode: few queries) give partials
// (max, sum, o) per split, o stored as bf16 from the registers that load it
// from TMEM; a combine kernel (a CTA per query and four heads, all of a
// thread's split operands loaded at once) adds them in split order with the
// sink.  With a
// fixed split count (an option) the split boundaries depend only on the
// query's rows: a request's output then does not depend on the batch it runs
// in.  (Measured alternatives, removed: the splits meeting on a global
// counter in one cooperative launch, and a thread block cluster exchanging
// the partials through distributed shared memory; both spent longer in the
// exchange than the partial write and the combine launch cost.)
//
// Options: RMSNorm of the query and RoPE of its last dims at the query
// position (prologue, the same arithmetic as csa_rmsnorm_rope), and RoPE of
// the output's last dims at minus the query position (output write).
#include "csa_internal.cuh"
#include "mqa_plan.cuh"
#include "rope_dev.cuh"
#include "sm100.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_mqa_umma)

namespace {

constexpr int kDim = 512;
constexpr int kHG = 64;          // heads per CTA (N of the products)
constexpr int kRows = 128;       // rows per chunk (M of S^T)
constexpr int kThreads = 256;
constexpr int kItems = kHG * kDim / 8;  // output items of a head group: (head, 8 dims)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.f;     // log2 headroom before the running max is raised
constexpr int kMaxRope = 64;     // RoPE dims the fused options support
constexpr int kMaxSplits = 256;        // splits of a query (the combine's shared memory)

// Shared memory (offsets from a 1024-byte aligned base).  The upper half of
// the row tile and P together stage a chunk of raw FP8MIX rows.
constexpr int kAtom = kRows * 128;               // one 64-dim atom of the row tile
constexpr int kOffKV = 0;                        // 8 x [128 rows][128 B]    128 KB
constexpr int kOffP = kOffKV + 8 * kAtom;        // [128 rows][128 B]        16 KB
constexpr int kOffQ = kOffP + kRows * 128;       // 8 x [64 heads][128 B]    64 KB
constexpr int kOffMisc = kOffQ + 8 * kHG * 128;
constexpr int kRawRow = 608;                     // FP8MIX row at c = 512
constexpr int kOffRaw = kOffKV + 4 * kAtom;      // atoms 4..7 and P
static_assert(kOffRaw + kRows * kRawRow <= kOffQ, "raw staging fits in atoms 4..7 and P");
static_assert(kHG * kDim * 4 <= 8 * kAtom, "the fp32 output staging fits in the row tile");
struct Misc {
  float m_use[kHG];    // running max per head (log2 domain)
  float corr[kHG];     // this chunk's rescale factor per head
  float fac[kHG];      // epilogue scale per head
  float lsum[kHG];     // final sums per head
  float red[4][kHG];   // per-quadrant maxima
  float qcs[kMaxRope / 2], qsn[kMaxRope / 2];  // RoPE at +t (query)
  float ocs[kMaxRope / 2], osn[kMaxRope / 2];  // RoPE at -t (output)
  const uint8_t* rowp[2][kRows];               // rows of the current / next chunk
  uint64_t bar_q, bar_raw, bar_half[2], bar_pair[4], bar_qk, bar_slab[4], bar_pv;
  uint32_t tmem_slot;
};
constexpr int kSmemBytes = 1024 + kOffMisc + (int)sizeof(Misc);
static_assert(kOffMisc % 16 == 0, "bulk-copy sources are 16-byte aligned");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// TMEM columns: S^T over the first and the second half of the dims (64
// each: two threads issue the two halves at once), O^T slabs 0..3 (64 each),
// L (64), ones (32).
constexpr int kColS = 0;
constexpr int kColS2 = 416;
constexpr int kColO = 64;
constexpr int kColL = 320;
constexpr int kColOnes = 384;
constexpr int kTmemCols = 512;

constexpr uint32_t kIdescQK = idesc_bf16_f32(kRows, kHG);
constexpr uint32_t kIdescPV = idesc_bf16_f32_major(128, kHG, 1, 1);
constexpr uint32_t kIdescL = idesc_bf16_f32_major(128, kHG, 0, 1);

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}
// Row tile: byte offset of 16-byte chunk g (dims 8g .. 8g+7) of row r.
__device__ __forceinline__ uint32_t kv_off(int r, int g) {
  return (uint32_t)((g >> 3) * kAtom + r * 128 + ((((g & 7) ^ (r & 7))) << 4));
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
// Waits until at most n of this thread's most recent cp.async groups are pending.
__device__ __forceinline__ void cp_async_wait_pending(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
  }
}
// Maximum over the warp's 32 lanes, returned to every lane (sm_100a).
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Address of row r of the query's attended rows when it lies in [.., r_end),
// else nullptr (absent rows are zero-filled and masked).
__device__ __forceinline__ const uint8_t* chunk_row(const MqaArgs& a, const RowList& rl, int b, int64_t r,
                                                    int64_t r_end, int64_t rb) {
  return r < r_end ? row_ptr(a, rl, b, r, rb) : nullptr;
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
    memcpy(&w[q], &h, 4);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// BF16 rows: one cp.async commit group per pair of atoms (128 dims).
__device__ __forceinline__ void gather_bf16(uint8_t* KV, const uint8_t* const* rowp, const void* dummy) {
  for (int p = 0; p < 4; ++p) {
    for (int u = threadIdx.x; u < kRows * 16; u += kThreads) {
      const int r = u >> 4, g = 16 * p + (u & 15);
      const uint8_t* src = rowp[r];
      cp_async16(smem_u32(KV + kv_off(r, g)), src ? src + g * 16 : dummy, src != nullptr);
    }
    cp_async_commit();
  }
}

// FP8MIX rows: one bulk copy per row into the raw staging area (absent rows
// zero-filled); threads 0..127 each arrive once on bar_raw.
__device__ __forceinline__ void gather_fp8(uint8_t* raw, const uint8_t* const* rowp, uint64_t* bar_raw) {
  const int r = threadIdx.x;
  if (r >= kRows) return;
  const uint8_t* src = rowp[r];
  uint8_t* dst = raw + r * kRawRow;
  if (src != nullptr) {
    mbar_arrive_expect_tx(bar_raw, kRawRow);
    bulk_load(dst, src, kRawRow, bar_raw);
  } else {
#pragma unroll 1
    for (int c = 0; c < kRawRow / 16; ++c) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0u, 0u, 0u, 0u);
    mbar_arrive(bar_raw);
  }
}

// 16-byte chunk g (dims 8g .. 8g+7) of raw FP8MIX row r as bf16: each value
// is code * scale (the code decoded exactly by the hardware conversion,
// the product rounded once to fp32), then rounded to bf16.
__device__ __forceinline__ uint4 expand_fp8(const uint8_t* raw, int r, int g) {
  const uint8_t* row = raw + r * kRawRow;
  if (g >= 56) return *reinterpret_cast<const uint4*>(row + 448 + (g - 56) * 16);
  const uint2 v = *reinterpret_cast<const uint2*>(row + g * 8);
  const float sc = *reinterpret_cast<const float*>(row + 576 + 4 * (g >> 3));
  float f[8];
  const uint32_t src[2] = {v.x, v.y};
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float2 lo = e4m3x2_to_float2((uint16_t)(src[q] & 0xFFFF));
    const float2 hi = e4m3x2_to_float2((uint16_t)(src[q] >> 16));
    f[4 * q + 0] = lo.x * sc; f[4 * q + 1] = lo.y * sc;
    f[4 * q + 2] = hi.x * sc; f[4 * q + 3] = hi.y * sc;
  }
  return pack_bf16x8(f);
}

// Partial S^T += K Q^T over atoms [at0, at1) into TMEM column `col` (atom
// `first` overwrites).  One thread issues atoms 0..3 into kColS, another
// atoms 4..7 into kColS2: a tcgen05.mma costs its issuing thread ~0.1 us, so
// the 32 products of a chunk are issued by two threads at once.
__device__ __forceinline__ void issue_qk(uint32_t tmem, uint32_t col, uint32_t kva, uint32_t qa, int at0, int at1,
                                         int first) {
  for (int at = at0; at < at1; ++at)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      tc_mma_f16(tmem + col, umma_desc_sw128(kva + at * kAtom + kk * 32),
                 umma_desc_sw128(qa + at * (kHG * 128) + kk * 32), kIdescQK, (at != first || kk) ? 1u : 0u);
}

// The combine of a head group's splits ("DeepSeek-V4 内部机制" sink equation):
//   M = max(sink, m_j),  w_j = e^{m_j - M},
//   O = sum_j w_j o_j / (sum_j w_j l_j + e^{sink - M}),
// with the splits added in split order.  The in-kernel combine (operands in
// shared memory) and the combine kernel (operands in global memory) run these
// two functions, so both give the same bytes.
//
// Weights of one head: W[j] = w_j / den (0 for an empty split, all 0 when the
// sink is +inf or nothing is attended).  ml(j) returns (m_j, l_j); callers
// fetch every split's statistics before calling, so no loads wait here.
// MAXS > 0: S <= MAXS and the loops are unrolled (ml may index a register
// array); MAXS = 0: plain loops.  The operations and their order are the
// same either way.
template <int MAXS, class ML>
__device__ __forceinline__ void combine_weights(int S, float sink, const ML& ml, float* W, int stride) {
  constexpr int kN = MAXS > 0 ? MAXS : 1 << 30;
  float M = sink;
#pragma unroll
  for (int j = 0; j < (MAXS > 0 ? MAXS : S); ++j) {
    if (j >= S || j >= kN) break;
    M = fmaxf(M, ml(j).x);
  }
  const bool zero = (sink == INFINITY) || (M == -INFINITY);
  float den = 0.f;
#pragma unroll
  for (int j = 0; j < (MAXS > 0 ? MAXS : S); ++j) {
    if (j >= S) break;
    const float2 v = ml(j);
    const float w = (zero || v.x == -INFINITY) ? 0.f : expf(v.x - M);
    W[j * stride] = w;
    den += w > 0.f ? v.y * w : 0.f;
  }
  if (!zero) den += expf(sink - M);
  for (int j = 0; j < S; ++j) W[j * stride] = zero ? 0.f : W[j * stride] / den;
}

// RoPE tables of the query at +t and of the output at -t (threads < 32).
__device__ __forceinline__ void rope_tables(const MqaArgs& a, int64_t t, float* qcs, float* qsn, float* ocs,
                                            float* osn) {
  const int k = threadIdx.x;
  if (k < a.q_rope_dims / 2) rope_sincos((double)t, rope_theta(a.rope_base, k, a.q_rope_dims), &qsn[k], &qcs[k]);
  if (k < a.out_rope_dims / 2)
    rope_sincos((double)t * -1.0, rope_theta(a.rope_base, k, a.out_rope_dims), &osn[k], &ocs[k]);
}

// Split partials of this kernel: o of (query bt, split s) as [head quad][512
// dims][4 heads] bf16 (unnormalised, rounded once from the fp32 TMEM
// accumulator; four heads of a dim side by side so a thread stores them at
// once), then (m, l) per head in fp32.  The o region is sized for fp32 rows
// (the split-KV workspace layout shared with the SIMT kernel); this kernel
// uses its first half.
__host__ __device__ __forceinline__ __nv_bfloat16* quad_partial_o(const MqaPlan& p, const MqaArgs& a, int64_t bt,
                                                                  int s, int hq) {
  return reinterpret_cast<__nv_bfloat16*>(plan_partials(p, a)) +
         (((bt * p.n_splits + s) * (a.n_heads / 4)) + hq) * (int64_t)a.dim * 4;
}

template <bool FP8, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    mqa_umma_kernel(const __grid_constant__ CUtensorMap tmQ, MqaArgs a, MqaPlan plan) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* KV = base + kOffKV;
  uint8_t* Ps = base + kOffP;
  uint8_t* Qs = base + kOffQ;
  uint8_t* raw = base + kOffRaw;
  Misc& ms = *reinterpret_cast<Misc*>(base + kOffMisc);

  const int split = blockIdx.x, hg = blockIdx.y;
  const int64_t bt = blockIdx.z;
  const int b = (int)(bt / a.n_q);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;

  if (tid == 0) {
    mbar_init(&ms.bar_q, 1);
    mbar_init(&ms.bar_raw, kRows);
    for (int i = 0; i < 2; ++i) mbar_init(&ms.bar_half[i], kThreads);
    for (int i = 0; i < 4; ++i) mbar_init(&ms.bar_pair[i], kThreads);
    mbar_init(&ms.bar_qk, 2);  // the two half-S^T issuers
    for (int i = 0; i < 4; ++i) mbar_init(&ms.bar_slab[i], 1);
    mbar_init(&ms.bar_pv, 5);  // the four slab issuers and the L issuer
    fence_barrier_init();
    // query tile (64 heads x 512 dims): eight TMA boxes of 64 heads x 64 dims
    // in the 128-byte swizzle, the K-major operand layout (depends on nothing)
    mbar_arrive_expect_tx(&ms.bar_q, kHG * kDim * 2);
    const int qrow = (int)(bt * a.n_heads + (int64_t)hg * kHG);
    for (int at = 0; at < 8; ++at) tma_load_2d(Qs + at * (kHG * 128), &tmQ, &ms.bar_q, 64 * at, qrow);
  }
  // The first chunk's entry indices are fetched together with the query
  // position, assuming the query's window is full (decode); a query whose
  // window is cut by the start of the sequence has fewer rows and fetches its
  // own range again below.
  const int NS = plan.n_splits;
  const int64_t full_rows = a.idx ? (int64_t)a.k + a.window : 0;
  const int64_t full_nch = (full_rows + kRows - 1) / kRows;
  const int64_t guess_begin = (int64_t)split * full_nch / NS * kRows;
  int32_t e_guess = -1;
  if (a.idx != nullptr && tid < kRows && guess_begin + tid < a.k) e_guess = a.idx[bt * a.k + guess_begin + tid];
  const int64_t tq = a.q_pos[bt];
  const RowList rl = make_row_list(a, bt, tq);
  // split s of NS takes chunks [s * nch / NS, (s + 1) * nch / NS) of the rows
  const int64_t nch = (rl.n_rows + kRows - 1) / kRows;
  const int64_t r_begin = (int64_t)split * nch / NS * kRows;
  const int64_t r_end = min64(rl.n_rows, ((int64_t)split + 1) * nch / NS * kRows);
  const int n_chunks = r_end > r_begin ? (int)((r_end - r_begin + kRows - 1) / kRows) : 0;
  const int64_t rb = row_bytes(a.kv_dt, kDim);

  if (warp == 0) tmem_alloc(&ms.tmem_slot, kTmemCols);
  if (tid < kHG) ms.m_use[tid] = -INFINITY;
  if (tid < 32) rope_tables(a, tq, ms.qcs, ms.qsn, ms.ocs, ms.osn);
  if (tid < kRows) {
    const int64_t r = r_begin + tid;
    const uint8_t* p = nullptr;
    if (n_chunks > 0 && r < r_end) {
      if (r < rl.n_sel && a.idx != nullptr && r_begin == guess_begin) {
        const int64_t e = e_guess;
        if (e >= 0 && e < rl.vis) p = entry_row(a, b, e, rb);
      } else {
        p = row_ptr(a, rl, b, r, rb);
      }
    }
    ms.rowp[0][tid] = p;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_slot;
  // the first chunk's rows are on their way while the rest is set up
  if (n_chunks > 0) {
    if (FP8) gather_fp8(raw, ms.rowp[0], &ms.bar_raw);
    else gather_bf16(KV, ms.rowp[0], a.Q);
  }
  if (warp < 4) {  // the all-ones A operand of the row-sum product
    float ones[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) ones[i] = __uint_as_float(0x3F803F80u);
    tmem_st_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + kColOnes, ones);
    tmem_st_wait();
  }
  tc_fence_before();
  if (a.q_norm_g != nullptr || a.q_rope_dims > 0) mbar_wait(&ms.bar_q, 0);
  if (a.q_norm_g != nullptr || a.q_rope_dims > 0) {
    // RMSNorm and RoPE of the query rows in place: warp w takes heads w, w+8,
    // ...; lane l owns dims 8l..8l+7 and 256+8l..+7 (the order of
    // csa_rmsnorm_rope, so the bytes agree)
    const int d_rope = kDim - a.q_rope_dims;
    for (int h = warp; h < kHG; h += kThreads / 32) {
      float v[2][8];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint4 u = *reinterpret_cast<const uint4*>(Qs + q_off(h, lane + 32 * k));
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[k][2 * j] = __uint_as_float(w4[j] << 16);
          v[k][2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
        }
      }
      if (a.q_norm_g != nullptr) {
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int q = 0; q < 8; ++q) ss = fmaf(v[k][q], v[k][q], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = rms_inv(ss, kDim, a.q_norm_eps);
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int q = 0; q < 8; ++q) v[k][q] = __fmul_rn(__fmul_rn(v[k][q], inv), a.q_norm_g[8 * (lane + 32 * k) + q]);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int d0 = 8 * (lane + 32 * k);
        if (a.q_rope_dims > 0 && d0 >= d_rope) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int kp = (d0 - d_rope) / 2 + j;
            rope_turn(v[k][2 * j], v[k][2 * j + 1], ms.qcs[kp], ms.qsn[kp]);
          }
        }
        *reinterpret_cast<uint4*>(Qs + q_off(h, lane + 32 * k)) = pack_bf16x8(v[k]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
  }
  if (tid == 0) mbar_wait(&ms.bar_q, 0);  // the query tile, before the first product
  const float sl2 = a.scale * kLog2e;
  const uint32_t kva = smem_u32(KV), qa = smem_u32(Qs), pa = smem_u32(Ps);
  constexpr int kHalf = kRows * 32 / kThreads;  // 16-byte chunks per thread in half a tile

  for (int ci = 0; ci < n_chunks; ++ci) {
    const uint32_t par = (uint32_t)(ci & 1);
    const uint8_t* const* rowp = ms.rowp[ci & 1];
    // ---- rows -> row tile, S^T = K Q^T issued part by part
    if (FP8) {
      mbar_wait(&ms.bar_raw, par);
      // dims 0..255 into atoms 0..3 (no overlap with the staging); every
      // chunk is decoded before any is stored, so the loads are all in flight
#pragma unroll 1
      for (int j0 = 0; j0 < kHalf; j0 += 4) {
        uint4 lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int u = tid + (j0 + j) * kThreads;
          lo[j] = expand_fp8(raw, u >> 5, u & 31);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int u = tid + (j0 + j) * kThreads;
          *reinterpret_cast<uint4*>(KV + kv_off(u >> 5, u & 31)) = lo[j];
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&ms.bar_half[0]);
      if (tid == 0) {
        mbar_wait(&ms.bar_half[0], par);
        tc_fence_after();
        issue_qk(tmem, kColS, kva, qa, 0, 4, 0);
        tc_commit(&ms.bar_qk);
      }
      // dims 256..511 through registers (their destination overlaps the staging)
      uint4 hi[kHalf];
#pragma unroll
      for (int j = 0; j < kHalf; ++j) {
        const int u = tid + j * kThreads;
        hi[j] = expand_fp8(raw, u >> 5, 32 + (u & 31));
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kHalf; ++j) {
        const int u = tid + j * kThreads;
        *reinterpret_cast<uint4*>(KV + kv_off(u >> 5, 32 + (u & 31))) = hi[j];
      }
      fence_proxy_async_smem();
      mbar_arrive(&ms.bar_half[1]);
      if (tid == 32) {
        mbar_wait(&ms.bar_half[1], par);
        tc_fence_after();
        issue_qk(tmem, kColS2, kva, qa, 4, 8, 4);
        tc_commit(&ms.bar_qk);
      }
    } else {
      for (int p = 0; p < 4; ++p) {
        cp_async_wait_pending(3 - p);
        fence_proxy_async_smem();
        mbar_arrive(&ms.bar_pair[p]);
        if (tid == (p < 2 ? 0 : 32)) {
          mbar_wait(&ms.bar_pair[p], par);
          tc_fence_after();
          issue_qk(tmem, p < 2 ? kColS : kColS2, kva, qa, 2 * p, 2 * p + 2, p < 2 ? 0 : 4);
          if (p == 1 || p == 3) tc_commit(&ms.bar_qk);
        }
      }
    }

    // ---- softmax: warp (quad, half) owns rows 32 quad.. and heads 32 half..
    mbar_wait(&ms.bar_qk, par);
    // P and the O^T / L columns are rewritten below: every product of the
    // previous chunk must have finished (its five issuers each commit to
    // bar_pv; the FP8 path already waited for them before its gather)
    if (!FP8 && ci > 0) mbar_wait(&ms.bar_pv, par ^ 1u);
    tc_fence_after();
    const int r = 32 * quad + lane;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    float s[32], s2[32];
    tmem_ld_32x32b_x32(tmem + lane_base + kColS + 32 * half, s);
    tmem_ld_32x32b_x32(tmem + lane_base + kColS2 + 32 * half, s2);
    tmem_ld_wait();
#pragma unroll
    for (int h = 0; h < 32; ++h) s[h] += s2[h];
    const bool ok = rowp[r] != nullptr;
#pragma unroll
    for (int h = 0; h < 32; ++h) s[h] = ok ? s[h] * sl2 : -INFINITY;
#pragma unroll
    for (int h = 0; h < 32; ++h) {
      const float wm = warp_max_f32(s[h]);
      if (lane == h) ms.red[quad][32 * half + h] = wm;
    }
    __syncthreads();
    bool raised = false;
    if (tid < kHG) {
      const float cm = fmaxf(fmaxf(ms.red[0][tid], ms.red[1][tid]), fmaxf(ms.red[2][tid], ms.red[3][tid]));
      const float mold = ms.m_use[tid];
      float use = mold;
      if (mold == -INFINITY || cm > mold + kLazy) use = fmaxf(mold, cm);
      ms.corr[tid] = (mold == -INFINITY || use == mold) ? 1.f : exp2f(mold - use);
      raised = mold != -INFINITY && use != mold;
      ms.m_use[tid] = use;
    }
    const int rescale = __syncthreads_or(raised ? 1 : 0);
    // P = 2^(s - m) as bf16, MN-major: row r's 128-byte line, heads 32 half..
#pragma unroll
    for (int h = 0; h < 32; ++h) {
      const float m = ms.m_use[32 * half + h];
      s[h] = (s[h] == -INFINITY || m == -INFINITY) ? 0.f : exp2f(s[h] - m);
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      *reinterpret_cast<uint4*>(Ps + r * 128 + (((4 * half + c4) ^ (r & 7)) << 4)) = pack_bf16x8(s + 8 * c4);
    // a raised max rescales what O^T and L accumulated so far (lane = dim)
    if (ci > 0 && rescale) {
#pragma unroll 1
      for (int sl = 2 * half; sl < 2 * half + 2 + (half == 0 ? 1 : 0); ++sl) {
        const uint32_t col = sl < 2 * half + 2 ? kColO + sl * kHG : kColL;
        float o[kHG];
        tmem_ld_32x32b_x32(tmem + lane_base + col, o);
        tmem_ld_32x32b_x32(tmem + lane_base + col + 32, o + 32);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < kHG; ++h) o[h] *= ms.corr[h];
        tmem_st_32x32b_x32(tmem + lane_base + col, o);
        tmem_st_32x32b_x32(tmem + lane_base + col + 32, o + 32);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    fence_proxy_async_smem();  // P (generic stores) -> tensor core reads
    __syncthreads();

    // ---- O^T += V^T P^T (slab sl issued by warp sl) and L += 1 P^T (warp 4):
    // five threads issue at once (each product costs its issuer ~0.1 us)
    if (lane == 0 && warp < 5) {
      tc_fence_after();
      if (warp < 4) {
        const int sl = warp;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_f16(tmem + kColO + sl * kHG, umma_desc_sw128_mn(kva + (2 * sl) * kAtom + kk * 2048, kAtom, 1024),
                     umma_desc_sw128_mn(pa + kk * 2048, kAtom, 1024), kIdescPV, (ci > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&ms.bar_slab[sl]);
      } else {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_f16_ta(tmem + kColL, tmem + kColOnes, umma_desc_sw128_mn(pa + kk * 2048, kAtom, 1024), kIdescL,
                        (ci > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(&ms.bar_pv);
    }

    // ---- the next chunk's rows
    if (ci + 1 < n_chunks) {
      if (tid < kRows)
        ms.rowp[(ci + 1) & 1][tid] = chunk_row(a, rl, b, r_begin + (int64_t)(ci + 1) * kRows + tid, r_end, rb);
      if (FP8) {
        // the staging overlaps atoms 4..7 and P: wait for every product
        mbar_wait(&ms.bar_pv, par);
        tc_fence_after();
        __syncthreads();
        gather_fp8(raw, ms.rowp[(ci + 1) & 1], &ms.bar_raw);
      } else {
        __syncthreads();
        // atoms 2p, 2p+1 are free once the slab-p products have read them
        for (int p = 0; p < 4; ++p) {
          mbar_wait(&ms.bar_slab[p], par);
          const uint8_t* const* nrow = ms.rowp[(ci + 1) & 1];
          for (int u = tid; u < kRows * 16; u += kThreads) {
            const int rr = u >> 4, g = 16 * p + (u & 15);
            const uint8_t* src = nrow[rr];
            cp_async16(smem_u32(KV + kv_off(rr, g)), src ? src + g * 16 : a.Q, src != nullptr);
          }
          cp_async_commit();
        }
      }
    }
  }
  if (n_chunks > 0) mbar_wait(&ms.bar_pv, (uint32_t)((n_chunks - 1) & 1));
  tc_fence_after();

  // ---- epilogue: sums, then O^T staged as fp32 [head][512 dims] in the row tile
  if (warp == 0) {
    float l[kHG];
    if (n_chunks > 0) {
      tmem_ld_32x32b_x32(tmem + kColL, l);
      tmem_ld_32x32b_x32(tmem + kColL + 32, l + 32);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int h = 0; h < kHG; ++h) l[h] = 0.f;
    }
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < kHG; ++h) ms.lsum[h] = l[h];
  }
  float* stg = reinterpret_cast<float*>(KV);
#pragma unroll 1
  for (int sl = 2 * half; sl < 2 * half + 2; ++sl) {
    float o[kHG];
    if (n_chunks > 0) {
      const uint32_t ta = tmem + ((uint32_t)(32 * quad) << 16) + kColO + sl * kHG;
      tmem_ld_32x32b_x32(ta, o);
      tmem_ld_32x32b_x32(ta + 32, o + 32);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int h = 0; h < kHG; ++h) o[h] = 0.f;
    }
    const int d = sl * 128 + 32 * quad + lane;
    if constexpr (MODE == kMqaWhole) {
#pragma unroll
      for (int h = 0; h < kHG; ++h) stg[h * kDim + d] = o[h];
    } else {
      // a split's partial o goes straight from the registers to global
      // memory as bf16, four heads interleaved per dim (lane = dim: a warp
      // stores 256 contiguous bytes per head quad; the combine reads it from
      // L2)
      __nv_bfloat16* po = quad_partial_o(plan, a, bt, split, hg * (kHG / 4)) + 4 * d;
#pragma unroll
      for (int q = 0; q < kHG / 4; ++q) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(o[4 * q], o[4 * q + 1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(o[4 * q + 2], o[4 * q + 3]);
        uint2 pk;
        memcpy(&pk.x, &lo, 4);
        memcpy(&pk.y, &hi, 4);
        *reinterpret_cast<uint2*>(po + (int64_t)q * kDim * 4) = pk;
      }
    }
  }
  fence_proxy_async_smem();  // the staging is read by bulk copies
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }

  if constexpr (MODE == kMqaWhole) {
    if (tid < kHG) {
      const float sink = a.sink[hg * kHG + tid] * kLog2e;  // log2 domain
      const float m = ms.m_use[tid];
      const float M = fmaxf(m, sink);
      float f = 0.f;
      if (!(sink == INFINITY) && M != -INFINITY) {
        const float em = m == -INFINITY ? 0.f : exp2f(m - M);
        f = em / (ms.lsum[tid] * em + exp2f(sink - M));
      }
      ms.fac[tid] = f;
    }
    __syncthreads();
    // normalised (and optionally turned) bf16 rows [head][512] in the query
    // region, then one bulk copy per 16 KB to the output
    const int d_rope = kDim - a.out_rope_dims;
    for (int it = tid; it < kItems; it += kThreads) {
      const int h = it >> 6, d0 = 8 * (it & 63);
      const float4 x0 = *reinterpret_cast<const float4*>(stg + h * kDim + d0);
      const float4 x1 = *reinterpret_cast<const float4*>(stg + h * kDim + d0 + 4);
      const float f = ms.fac[h];
      float v[8] = {x0.x * f, x0.y * f, x0.z * f, x0.w * f, x1.x * f, x1.y * f, x1.z * f, x1.w * f};
      if (a.out_rope_dims > 0 && d0 >= d_rope) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = (d0 - d_rope) / 2 + q;
          rope_turn(v[2 * q], v[2 * q + 1], ms.ocs[k], ms.osn[k]);
        }
      }
      *reinterpret_cast<uint4*>(Qs + it * 16) = pack_bf16x8(v);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid < 4) {
      constexpr uint32_t kPiece = kHG * kDim * 2 / 4;
      bulk_store(static_cast<uint8_t*>(a.O) + (bt * a.n_heads + (int64_t)hg * kHG) * kDim * 2 + tid * kPiece,
                 Qs + tid * kPiece, kPiece);
      bulk_commit();
      bulk_wait_read();  // the shared memory may go once the copy has read it
    }
  } else {
    // one split of several: the unnormalised partial's statistics (m, l)
    // for the combine kernel (o was stored above)
    if (tid < kHG) {
      float* ml = plan_partial_ml(plan, a, bt, split, hg * kHG + tid);
      const float m = ms.m_use[tid];
      ml[0] = m == -INFINITY ? -INFINITY : m / kLog2e;  // natural-log domain
      ml[1] = ms.lsum[tid];
    }
  }
}

// The combine of kMqaSplit mode: one CTA per (head quad, query), a thread
// per 2 dims of the four heads; the splits' statistics go through shared
// memory once, and each thread's partials (16 bytes per split) are loaded 16
// splits at a time, all in flight together.
constexpr int kCombineThreads = 256;
constexpr int kLoadSplits = 16;
__global__ void __launch_bounds__(kCombineThreads) mqa_umma_combine_kernel(MqaArgs a, MqaPlan plan) {
  __shared__ float2 mls[4][kMaxSplits];
  __shared__ float W[4][kMaxSplits];
  __shared__ float ocs[kMaxRope / 2], osn[kMaxRope / 2], qcs[kMaxRope / 2], qsn[kMaxRope / 2];
  const int hq = blockIdx.x;
  const int64_t bt = blockIdx.y;
  const int S = plan.n_splits, tid = threadIdx.x;
  if (tid < 32) rope_tables(a, a.q_pos[bt], qcs, qsn, ocs, osn);
  for (int u = tid; u < 4 * S; u += kCombineThreads)
    mls[u & 3][u >> 2] = __ldcg(reinterpret_cast<const float2*>(plan_partial_ml(plan, a, bt, u >> 2, 4 * hq + (u & 3))));
  // this thread's dims d0, d0 + 1 (four heads each, 16 bytes) of the first
  // (up to) 16 splits, loaded while the weights are formed
  const int d0 = 2 * tid;
  uint4 x[kLoadSplits];
#pragma unroll
  for (int u = 0; u < kLoadSplits; ++u)
    if (u < S) x[u] = __ldcg(reinterpret_cast<const uint4*>(quad_partial_o(plan, a, bt, u, hq) + 4 * d0));
  __syncthreads();
  if (tid < 4) combine_weights<0>(S, a.sink[4 * hq + tid], [&](int j) { return mls[tid][j]; }, W[tid], 1);
  __syncthreads();
  float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
  for (int j0 = 0; j0 < S; j0 += kLoadSplits) {
    if (j0 > 0) {
#pragma unroll
      for (int u = 0; u < kLoadSplits; ++u)
        if (j0 + u < S) x[u] = __ldcg(reinterpret_cast<const uint4*>(quad_partial_o(plan, a, bt, j0 + u, hq) + 4 * d0));
    }
#pragma unroll
    for (int u = 0; u < kLoadSplits; ++u) {
      if (j0 + u >= S) break;
      // x[u]: (d0, heads 0 1), (d0, heads 2 3), (d0 + 1, heads 0 1), (d0 + 1, heads 2 3)
      const uint32_t wv[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t w = wv[2 * e + (i >> 1)];
          const float v = __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
          acc[i][e] = fmaf(W[i][j0 + u], v, acc[i][e]);
        }
    }
  }
  const int d_rope = kDim - a.out_rope_dims;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (a.out_rope_dims > 0 && d0 >= d_rope)
      rope_turn(acc[i][0], acc[i][1], ocs[(d0 - d_rope) / 2], osn[(d0 - d_rope) / 2]);
    const __nv_bfloat162 v = __floats2bfloat162_rn(acc[i][0], acc[i][1]);
    *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.O) + (bt * a.n_heads + 4 * hq + i) * kDim + d0) =
        v;
  }
}

int sm_count_mqa() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        v <= 0) {
      cudaGetLastError();
      return 148;
    }
    n = v;
  }
  return n;
}

bool mqa_umma_eligible(const MqaArgs& a) {
  return a.q_dt == CSA_BF16 && (a.kv_dt == CSA_BF16 || a.kv_dt == CSA_KV_FP8MIX) && a.dim == kDim &&
         a.n_heads % kHG == 0 && (int64_t)a.batch * a.n_q <= 65535 && (a.idx == nullptr || a.k <= 2048) &&
         a.q_rope_dims <= kMaxRope && a.out_rope_dims <= kMaxRope;
}

MqaPlan make_umma_mqa_plan(const MqaArgs& a) {
  MqaPlan p{};
  p.heads_per_cta = kHG;
  p.rows_per_split = 0;
  p.ws_head = 0;
  // automatic: a query's row chunks are split over CTAs until the grid fills
  // one wave; a fixed count (a.splits) depends on the row count only
  const int sms = sm_count_mqa();
  const int64_t units = (int64_t)a.batch * a.n_q * (a.n_heads / kHG);
  const int64_t nch = (max_rows_per_query(a) + kRows - 1) / kRows;
  int64_t ns = a.splits > 0 ? a.splits : (units >= sms ? 1 : sms / units);
  if (ns > nch) ns = nch;
  if (ns > kMaxSplits) ns = kMaxSplits;
  if (ns < 1) ns = 1;
  p.n_splits = (int)ns;
  p.mode = ns == 1 ? kMqaWhole : kMqaSplit;
  return p;
}

template <bool FP8, int MODE>
cudaError_t launch_umma(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  auto kern = mqa_umma_kernel<FP8, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  // the queries as [B * T * n_heads rows][512] bf16, boxes of 64 heads x 64 dims
  CUtensorMap tmQ;
  if (!make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.Q, (uint64_t)a.batch * a.n_q * a.n_heads, kDim, 64,
                   kHG, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const dim3 grid((unsigned)p.n_splits, a.n_heads / kHG, (unsigned)((int64_t)a.batch * a.n_q));
  kern<<<grid, kThreads, kSmemBytes, s>>>(tmQ, a, p);
  ++launch_counter();
  e = cudaGetLastError();
  if (e != cudaSuccess || MODE != kMqaSplit) return e;
  mqa_umma_combine_kernel<<<dim3(a.n_heads / 4, (unsigned)((int64_t)a.batch * a.n_q)), kCombineThreads, 0, s>>>(a, p);
  ++launch_counter();
  return cudaGetLastError();
}

template <bool FP8>
cudaError_t launch_umma_fmt(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  if (p.mode == kMqaSplit) return launch_umma<FP8, kMqaSplit>(a, p, s);
  return launch_umma<FP8, kMqaWhole>(a, p, s);
}

}  // namespace

bool mqa_umma_path(const MqaArgs& a) { return mqa_umma_eligible(a); }
MqaPlan mqa_umma_plan(const MqaArgs& a) { return make_umma_mqa_plan(a); }
cudaError_t launch_mqa_umma(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  return a.kv_dt == CSA_KV_FP8MIX ? launch_umma_fmt<true>(a, p, s) : launch_umma_fmt<false>(a, p, s);
}

}  // namespace csa
