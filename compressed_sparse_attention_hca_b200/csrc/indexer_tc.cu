// indexer_tc.cu -- tensor-core producers of the Lightning Indexer score
// ("DeepSeek-V4 内部机制" 1.2 Step 2: I[t,s] = sum_h w[t,h] ReLU(q[t,h].K[s]);
// 6.2: FP4 q/K, fp32 score rounded to BF16 before top-k), fused with the
// top-k selection.
//
// One CTA owns a group of NQ queries of one request and a slice of that
// request's entries.  The score tile is a dense contraction
//     D[128 entries, 64*NQ heads] = K_tile[128 x 128] . Q_group[64*NQ x 128]^T
// issued as tcgen05.mma with fp32 accumulation in TMEM:
//   BF16 inputs:  kind::f16, K tiles TMA-staged in the 128-byte swizzle;
//   NVFP4 inputs: kind::mxf4nvf4 block16 on the packed E2M1 tiles (64-byte
//     swizzle), their E4M3 scales moved to TMEM by tcgen05.cp from 512-byte
//     atoms (byte m0*16 + m1*4 + kk = scale of tile row m0 + 32*m1, K-block
//     kk).  Key scales are stored in HBM in exactly that layout, so each
//     tile's two atoms arrive by one 1 KB bulk copy; the query's row-major
//     scales are permuted once per CTA.
// Warp roles: 0 TMA producer; 1 TMEM owner and MMA issuer with further
// issuers taking every other (BF16: warp 2) or every fourth (NVFP4 decode:
// warps 3, 12, 13) tile, since a tcgen05.mma costs its issuing thread about as
// long as a tile's data takes to stream; 2 query scale atoms (NVFP4); 4-7 and
// 8-11 two epilogue groups.  The accumulator has NBUF TMEM buffers so that the MMAs
// run several tiles ahead of the epilogue; epilogue group g drains the tiles
// i with i % 2 == g: each thread owns one entry row
// (one TMEM lane), reads its 64 head scores per query, forms
// sum_h w_h relu(s_h), rounds to bf16 and stores the 16-bit order key in
// shared memory.  After the last tile the CTA selects on those keys (the score
// row never reaches HBM): alone when it holds the whole row, cooperatively
// with the other slices of the row (decode), or by writing candidates for the
// merge kernel.  A whole row of several queries (prefill) selects from
// per-query 12-bit prefix histograms the epilogue builds during the stream.
#include <cudaTypedefs.h>

#include "compress_dev.cuh"
#include "csa_internal.cuh"
#include "indexer_plan.cuh"
#include "rope_dev.cuh"
#include "sm100.cuh"
#include "topk_select.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_indexer_tc)

namespace {

constexpr int kBM = 128;          // entries per tile (MMA M)
constexpr int kDI = 128;          // indexer dim handled here
constexpr int kHI = 64;           // indexer heads handled here
constexpr int kAtom = kBM * 128;  // bytes of one 128-byte-wide K atom of a bf16 K tile
constexpr int kThreads = 384;
constexpr int kPrefixBins = 4096;  // 12-bit key prefixes (cooperative select)

__host__ __device__ constexpr int pow2_cols(int c) {
  return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512;
}

template <int NQ>
struct Bf16Cfg {
  static constexpr int N = kHI * NQ;
  static constexpr int STAGES = NQ == 1 ? 4 : 3;
  static constexpr int Q_BYTES = N * 2 * kDI;             // two atoms of N rows x 128 B
  static constexpr int K_STAGE = kBM * 2 * kDI;           // two atoms of 128 rows x 128 B
  static constexpr int NBUF = 512 / N;                    // 8 (NQ 1) or 4 (NQ 2)
  static_assert(NBUF % 2 == 0, "one epilogue group and one MMA issuer per buffer");
  static constexpr int TMEM_COLS = 512;
  static constexpr int NT = kThreads;
  // prefix histogram: the cooperative select's (NQ 1), or one per query with
  // two 16-bit counts per word for the one-slice select (NQ 2)
  static constexpr int HIST = NQ == 1 ? kPrefixBins * 4 : NQ * kPrefixBins * 2;
  static constexpr int FIXED_SMEM = 1024 + STAGES * K_STAGE + Q_BYTES + NQ * kHI * 4 + 1024 /*barriers*/ +
                                    (int)sizeof(SelectSmem<NT>) + HIST;
  // shared memory per slice entry: NQ keys (the cooperative select's
  // candidate list reuses the K ring, idle by then)
  static constexpr int PER_ENTRY = 2 * NQ;
  static constexpr uint32_t IDESC = idesc_bf16_f32(kBM, N);
};

template <int NQ>
struct Nvf4Cfg {
  static constexpr int N = kHI * NQ;
  static constexpr int TPS = 2;                         // tiles per stage: one 16 KB code copy
  static constexpr int STAGES = NQ == 1 ? 9 : 8;
  static constexpr int CODES = kBM * kDI / 2;           // 8 KB of E2M1 per tile
  static constexpr int ATOMS = 2 * 512;                 // the tile's two scale atoms
  static constexpr int STAGE = TPS * (CODES + ATOMS);   // 18 KB: codes of both tiles, then their atoms
  static constexpr int QCODES = N * kDI / 2;
  static constexpr int QRAWSF = N * kDI / 16;
  static constexpr int QREG = (QCODES + QRAWSF + ATOMS + 1023) / 1024 * 1024;
  // MMA issue costs a thread more time per tile than the tile's data takes to
  // arrive, so tiles are spread over NI issuer warps (tile i -> issuer i % NI).
  static constexpr int NI = NQ == 1 ? 4 : 2;
  static constexpr int NT = NQ == 1 ? 448 : 384;        // + issuer warps 12, 13
  // NBUF a multiple of NI: buffer i % NBUF then always belongs to the same
  // issuer (i % NI) and epilogue group (i % 2), so each side waits on every
  // phase of its barriers in order (otherwise a waiter could skip a phase and
  // take the parity of an older one for the one it wants).
  static constexpr int NBUF = NQ == 1 ? 4 : 2;
  static_assert(NBUF % NI == 0 && NBUF % 2 == 0, "one issuer and one epilogue group per buffer");
  static constexpr int ACC_COLS = NBUF * N;             // 256
  static constexpr int SFA_COL = ACC_COLS;              // NI x 8 columns (one set per issuer)
  static constexpr int SFB_COL = ACC_COLS + 32;         // NI x 8 columns
  static constexpr int TMEM_COLS = pow2_cols(ACC_COLS + 64);
  static constexpr int HIST = NQ == 1 ? kPrefixBins * 4 : 0;  // prefix histogram (cooperative select)
  static constexpr int FIXED_SMEM = 1024 + STAGES * STAGE + QREG + NQ * kHI * 4 + 1024 +
                                    (int)sizeof(SelectSmem<NT>) + HIST;
  // shared memory per slice entry: NQ keys (the cooperative select's
  // candidate list reuses the stage ring, idle by then)
  static constexpr int PER_ENTRY = 2 * NQ;
  static constexpr uint32_t IDESC = idesc_nvf4(kBM, N);
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// Per-CTA description of the slice and its queries.
template <int NQ>
struct SliceCtx {
  int sl, t0, b, len, n_tiles;
  int64_t s0;
  int n_valid[NQ];
  int64_t vis[NQ];
};

template <int NQ>
__device__ __forceinline__ SliceCtx<NQ> slice_ctx(const IndexArgs& a, const IndexPlan& plan) {
  SliceCtx<NQ> c;
  c.sl = blockIdx.x;
  c.t0 = blockIdx.y * NQ;
  c.b = blockIdx.z;
  c.s0 = (int64_t)c.sl * plan.slice_len;
  c.len = (int)min64(plan.slice_len, a.n_entries - c.s0);
  int max_valid = 0;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int t = c.t0 + q;
    c.vis[q] = t < a.n_q ? visible_entries(a.q_pos[(int64_t)c.b * a.n_q + t], a.m, a.n_entries) : 0;
    c.n_valid[q] = (int)max64(0, min64(c.len, c.vis[q] - c.s0));
    max_valid = max(max_valid, c.n_valid[q]);
  }
  c.n_tiles = (max_valid + kBM - 1) / kBM;
  return c;
}

// Epilogue group `g` (warps 4-7: g = 0, warps 8-11: g = 1) drains the tiles
// i with i % 2 == g from TMEM buffer i % NBUF.
template <int NQ, int N, int NBUF>
__device__ __forceinline__ void epilogue_group(const SliceCtx<NQ>& c, const IndexArgs& a, const IndexPlan& plan,
                                               uint32_t tmem, uint64_t* accf, uint64_t* acce, const float* wsm,
                                               uint16_t* keys, bool coop, uint32_t* hist, bool hist2 = false) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3, g = (warp - 4) >> 2;
  const int r = quarter * 32 + lane;
  for (int i = g; i < c.n_tiles; i += 2) {
    const int buf = i % NBUF, u = i / NBUF;
    if (!mbar_wait(&accf[buf], u & 1)) break;
    tc_fence_after();
    float acc[NQ][kHI];
    const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * N);
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
      // four independent partial sums (heads h = 4i + j) keep the FMA pipe
      // busy; the weights are warp-uniform shared-memory broadcasts
      float part[4] = {0.f, 0.f, 0.f, 0.f};
      const float4* w4 = reinterpret_cast<const float4*>(wsm + q * kHI);
#pragma unroll
      for (int h4 = 0; h4 < kHI / 4; ++h4) {
        const float4 w = w4[h4];
        part[0] = fmaf(w.x, fmaxf(acc[q][4 * h4 + 0], 0.f), part[0]);
        part[1] = fmaf(w.y, fmaxf(acc[q][4 * h4 + 1], 0.f), part[1]);
        part[2] = fmaf(w.z, fmaxf(acc[q][4 * h4 + 2], 0.f), part[2]);
        part[3] = fmaf(w.w, fmaxf(acc[q][4 * h4 + 3], 0.f), part[3]);
      }
      const float I = (part[0] + part[1]) + (part[2] + part[3]);
      const uint32_t key = bf16_key(I);
      const bool valid = pos < c.n_valid[q];
      keys[q * plan.slice_len + pos] = valid ? (uint16_t)(key >> 16) : (uint16_t)0;
      if (coop && valid) atomicAdd(&hist[key >> 20], 1u);
      if (hist2 && valid) atomicAdd(&hist[q * (kPrefixBins / 2) + (key >> 21)], ((key >> 20) & 1u) ? 0x10000u : 1u);
      if (a.scores_out != nullptr && pos < c.len && c.t0 + q < a.n_q) {
        const float sc = valid ? key_to_f32(key) : -INFINITY;
        static_cast<__nv_bfloat16*>(a.scores_out)[((int64_t)c.b * a.n_q + c.t0 + q) * a.n_entries + c.s0 + pos] =
            __float2bfloat16_rn(sc);
      }
    }
  }
}

// Debug score output (-inf) for the positions past the last computed tile.
template <int NQ, int NT>
__device__ __forceinline__ void scores_tail(const SliceCtx<NQ>& c, const IndexArgs& a) {
  if (a.scores_out == nullptr) return;
  for (int q = 0; q < NQ; ++q) {
    if (c.t0 + q >= a.n_q) continue;
    for (int pos = c.n_tiles * kBM + threadIdx.x; pos < c.len; pos += NT)
      static_cast<__nv_bfloat16*>(a.scores_out)[((int64_t)c.b * a.n_q + c.t0 + q) * a.n_entries + c.s0 + pos] =
          __float2bfloat16_rn(-INFINITY);
  }
}

// Selection by one CTA over its own slice: final indices when it holds the
// whole row, else the slice's top k as candidates (and its k-th key) for the
// merge kernel.
template <int NT>
__device__ void hist_select(const uint16_t* kq, const uint32_t* h2, uint16_t* cand, int nv, int kk, int64_t s0,
                            int32_t* out, SelectSmem<NT>& sm);

template <int NQ, int NT>
__device__ void slice_select(const SliceCtx<NQ>& c, const IndexArgs& a, const IndexPlan& plan, const uint16_t* keys,
                             SelectSmem<NT>& sel, const uint32_t* hist2 = nullptr, uint16_t* cand = nullptr) {
  for (int q = 0; q < NQ; ++q) {
    const int t = c.t0 + q;
    if (t >= a.n_q) break;
    const int64_t bt = (int64_t)c.b * a.n_q + t;
    const int nv = c.n_valid[q];
    const int kk = min(a.k, nv);
    const uint16_t* kq = keys + q * plan.slice_len;
    auto key_at = [&](int i) { return ((uint32_t)kq[i]) << 16; };
    if (plan.n_slices == 1) {
      int32_t* out = a.idx_out + bt * a.k;
      if (hist2 != nullptr && kk < nv)
        hist_select<NT>(kq, hist2 + q * (kPrefixBins / 2), cand, nv, kk, c.s0, out, sel);
      else
        block_select<NT>(key_at, nv, kk, 0, sel, [&](int slot, int pos) { out[slot] = (int32_t)(c.s0 + pos); });
      for (int j = kk + threadIdx.x; j < a.k; j += NT) out[j] = -1;
    } else {
      const int64_t off = slice_cand_offset(plan, c.sl, c.vis[q], a.n_entries, a.k);
      uint32_t* ck = plan_cand_keys(plan, a.ws, bt) + off;
      int32_t* ci = plan_cand_idx(plan, a.ws, bt) + off;
      uint32_t T = 0;
      block_select<NT>(
          key_at, nv, kk, 0, sel,
          [&](int slot, int pos) {
            ck[slot] = key_at(pos);
            ci[slot] = (int32_t)(c.s0 + pos);
          },
          0u, &T);
      if (threadIdx.x == 0) plan_cand_thr(plan, a.ws, bt)[c.sl] = T;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Cooperative selection: the slice CTAs of one query row (all resident at once,
// cooperative launch) pick the row's top k together, with no candidate lists
// and no merge kernel.  Keys are 16-bit (bf16 score images), split into a
// 12-bit prefix (sign, exponent, 3 mantissa bits) and a 4-bit suffix:
//   1. each CTA adds its prefix histogram (built by the epilogue) into the
//      row's global histogram H; barrier; every CTA finds the prefix d1 of the
//      k-th key and how many keys (rem1) it still needs inside that prefix;
//   2. each CTA publishes, in its own slot, its count of keys with prefix > d1
//      and its 16-bin suffix histogram of keys with prefix d1 (each word
//      stored as value + 1, so readers poll the slots instead of a barrier);
//   3. every CTA reads all slots and derives the k-th key T, the ties at T to
//      take (lowest entry indices first, i.e. lowest slices first), its output
//      offset and its share of the ties, and writes its winners in index order
//      straight into the output row.
// The barrier is a global counter and the slots are polled, both with a
// bounded wait (the status word records a timeout).
constexpr int kSlotWords = 17;  // keys with prefix > d1, then suffix counts 0..15

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// The row's barrier in two halves, so that work needing no other slice runs
// between them.  Arrive: after a CTA barrier, thread 0 adds 1 with release
// semantics (this CTA's global writes and atomics, ordered before by the CTA
// barrier, are visible to every CTA that acquires the counter).  Wait:
// thread 0 polls the counter with acquire semantics (bounded), then a CTA
// barrier.
__device__ __forceinline__ void coop_arrive(uint32_t* ctr) {
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}
__device__ __forceinline__ void coop_wait(uint32_t* ctr, uint32_t target) {
  if (threadIdx.x == 0) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1; ld_acquire_gpu(ctr) < target; ++it) {
      if ((it & 255u) == 0 && globaltimer_ns() - t0 > kWaitTimeoutNs) {
        atomicOr(&g_device_status, 1u);
        break;
      }
    }
  }
  __syncthreads();
}

// Exclusive prefix sum of v over the block's NT threads (thread order);
// *total receives the block sum.  Ends with a block barrier.
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot, uint32_t* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    before += w < warp ? warp_tot[w] : 0u;
    all += warp_tot[w];
  }
  *total = all;
  __syncthreads();
  return before + inc - v;
}

// kq: the slice's 16-bit keys in position order; cand: scratch for up to nv
// positions.  Warp w scans positions [w * span, (w + 1) * span).
template <int NT>
__device__ void coop_select(const uint16_t* kq, uint16_t* cand, int nv, int64_t vis, int64_t s0, int sl,
                            const IndexPlan& plan, const IndexArgs& a, int64_t bt, const uint32_t* hist_local,
                            SelectSmem<NT>& sm) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const unsigned lt = (1u << lane) - 1u;
  const int S = plan.n_slices;
  int32_t* out = a.idx_out + bt * a.k;
  const int kk = (int)min64(a.k, vis);
  if (sl == 0)
    for (int j = kk + tid; j < a.k; j += NT) out[j] = -1;
  if (vis <= a.k) {  // every visible entry is selected: offsets in closed form
    const int64_t off = slice_cand_offset(plan, sl, vis, a.n_entries, a.k);
    for (int p = tid; p < nv; p += NT) out[off + p] = (int32_t)(s0 + p);
    return;
  }
  uint32_t* row = plan_coop_row(plan, a.ws, bt);
  uint32_t* H = row;
  uint32_t* ctr = row + kPrefixBins;       // [0] barrier, [1] highest prefix, [2] completions
  uint32_t* Hmax = row + kPrefixBins + 1;
  uint32_t* slots = row + kPrefixBins + 8;
  uint32_t total;

  // Warp 0 walks a prefix histogram down from bin `hi`, 32 bins at a time,
  // to the bin holding the want-th largest key; returns that bin and how many
  // keys of it are still needed (only the few bins above it are read).
  auto kth_prefix = [&](const uint32_t* hist, int hi, uint32_t want, bool global, uint32_t* d_out,
                        uint32_t* rem_out) {
    uint32_t above = 0;
    for (int base = hi; base >= 0; base -= 32) {
      const int d = base - lane;
      const uint32_t c = d >= 0 ? (global ? __ldcg(hist + d) : hist[d]) : 0u;
      uint32_t inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, above + inc >= want);
      if (hit) {
        const int l = __ffs(hit) - 1;
        if (lane == l) {
          *d_out = (uint32_t)d;
          *rem_out = want - (above + inc - c);
        }
        return;
      }
      above += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {  // fewer than `want` keys: every bin
      *d_out = 0u;
      *rem_out = 0u;
    }
  };

  // 1. this slice's prefix histogram into the row's histogram H (and its
  //    highest prefix into the row's), then arrive on the row's barrier
  if (tid == 0) sm.hist[64] = 0u;
  __syncthreads();
  uint32_t top = 0;
  for (int d = tid; d < kPrefixBins; d += NT)
    if (hist_local[d]) {
      atomicAdd(&H[d], hist_local[d]);
      top = (uint32_t)d;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = max(top, __shfl_xor_sync(0xffffffffu, top, o));
  if (lane == 0 && top) {
    atomicMax(Hmax, top);
    atomicMax(&sm.hist[64], top);
  }
  coop_arrive(ctr);

  // 1b. while the other slices arrive: this slice alone has min(k, nv) keys
  //     at or above its own k-th key, so the row's k-th key is not below it
  //     and no key with a smaller prefix L can win; compact the positions of
  //     the keys with prefix >= L into the warp's part of cand, in order.  A
  //     lane reads 8 consecutive keys (16 bytes) per step.
  if (warp == 0) kth_prefix(hist_local, (int)sm.hist[64], (uint32_t)min(a.k, nv), false, &sm.bcast[2], &sm.bcast[3]);
  __syncthreads();
  const uint32_t L = sm.bcast[2];
  const int span = ((nv + NW - 1) / NW + 255) / 256 * 256;
  const int w0 = min(nv, warp * span), w1 = min(nv, w0 + span);
  uint32_t n_cand = 0;
  for (int base = w0; base < w1; base += 256) {
    const int p0 = base + 8 * lane;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (p0 < w1) v = *reinterpret_cast<const uint4*>(kq + p0);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t cmask = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t k16 = (wv[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
      cmask |= (p0 + j < w1 && (k16 >> 4) >= L) ? (1u << j) : 0u;
    }
    const uint32_t cnt = __popc(cmask);
    uint32_t inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    uint32_t at = (uint32_t)w0 + n_cand + inc - cnt;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (cmask & (1u << j)) cand[at++] = (uint16_t)(p0 + j);
    n_cand += __shfl_sync(0xffffffffu, inc, 31);
  }

  // 1c. every slice has arrived: prefix d1 of the row's k-th key (d1 >= L)
  coop_wait(ctr, (uint32_t)S);
  if (warp == 0) kth_prefix(H, (int)__ldcg(Hmax), (uint32_t)kk, true, &sm.bcast[0], &sm.bcast[1]);
  if (tid < 32) sm.hist[tid] = 0;
  __syncthreads();
  const uint32_t d1 = sm.bcast[0], rem1 = sm.bcast[1];

  // 2. the warp's candidates: count those above prefix d1, histogram the
  //    suffixes of those inside it, and keep both (the only possible
  //    winners), in order, dropping the others
  uint16_t* cw0 = cand + w0;
  uint32_t kept = 0, gt1 = 0;
  for (int base = 0; base < (int)n_cand; base += 32) {
    const int j = base + lane;
    const bool in = j < (int)n_cand;
    const uint16_t p = in ? cw0[j] : (uint16_t)0;
    const uint32_t k16 = in ? kq[p] : 0u;
    const uint32_t pre = k16 >> 4;
    const bool hi = in && pre > d1, mid = in && pre == d1;
    if (mid) atomicAdd(&sm.hist[k16 & 15u], 1u);
    gt1 += hi ? 1u : 0u;
    const unsigned keep = __ballot_sync(0xffffffffu, hi || mid);
    __syncwarp();  // every lane has read its entry before any is overwritten
    if (hi || mid) cw0[kept + __popc(keep & lt)] = p;
    kept += __popc(keep);
  }
  n_cand = kept;
  __syncthreads();  // the suffix histogram is complete
  block_exclusive_scan<NT>(gt1, sm.warp_tot, &total);
  // slot words are stored as value + 1 into a zeroed workspace, so a reader
  // knows a word has arrived when it is nonzero: the exchange needs no
  // barrier, only each reader's bounded poll of the slots it reads
  if (tid == 0) st_relaxed_gpu(slots + sl * kSlotWords, total + 1u);
  if (tid < 16) st_relaxed_gpu(slots + sl * kSlotWords + 1 + tid, sm.hist[tid] + 1u);

  // 3. every slot -> k-th key T, ties to take, this slice's offset and ties
  uint32_t h4[16], g1 = 0;
#pragma unroll
  for (int n = 0; n < 16; ++n) h4[n] = 0;
  if (tid < S) {
    const uint32_t* sj = slots + tid * kSlotWords;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      bool all = true;
      g1 = ld_relaxed_gpu(sj);
      all = all && g1 != 0u;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        h4[n] = ld_relaxed_gpu(sj + 1 + n);
        all = all && h4[n] != 0u;
      }
      if (all) break;
      if ((it & 15u) == 0 && globaltimer_ns() - t0 > kWaitTimeoutNs) {
        atomicOr(&g_device_status, 1u);
        break;
      }
    }
    g1 = g1 - 1u;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      h4[n] = h4[n] - 1u;
      if (h4[n]) atomicAdd(&sm.hist[16 + n], h4[n]);
    }
  }
  __syncthreads();
  // Every slot has arrived, so every CTA of the row is past step 1 and the
  // workspace can go back to zeros (after the write below).  The ticket that
  // finds the last CTA is taken now and read at the end, so its round trip
  // overlaps the write.
  uint32_t ticket = 0;
  if (tid == 0) ticket = atomicAdd(ctr + 2, 1u);
  if (tid == 0) {
    uint32_t above = 0;
    for (int n = 15; n >= 0; --n) {
      if (above + sm.hist[16 + n] >= rem1) {
        sm.bcast[2] = (uint32_t)n;
        sm.bcast[3] = rem1 - above;
        break;
      }
      above += sm.hist[16 + n];
    }
  }
  __syncthreads();
  const uint32_t d2 = sm.bcast[2], need_eq = sm.bcast[3];
  const uint32_t T = (d1 << 4) | d2;
  uint32_t gt_j = g1, eq_j = 0;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    gt_j += (uint32_t)n > d2 ? h4[n] : 0u;
    eq_j += (uint32_t)n == d2 ? h4[n] : 0u;
  }
  if (tid >= S) gt_j = eq_j = 0;
  const uint32_t eq_prev = block_exclusive_scan<NT>(eq_j, sm.warp_tot, &total);
  const uint32_t take_j = need_eq > eq_prev ? min(need_eq - eq_prev, eq_j) : 0u;
  const uint32_t off_j = block_exclusive_scan<NT>(gt_j + take_j, sm.warp_tot, &total);
  if (tid == sl) {
    sm.bcast[0] = off_j;
    sm.bcast[1] = take_j;
  }
  __syncthreads();
  const uint32_t off = sm.bcast[0];
  const int eq_take_cta = (int)sm.bcast[1];

  // 4. per-warp counts over the compacted candidates, offsets, ordered write
  const uint16_t* cw = cand + w0;
  uint32_t c_gt = 0, c_eq = 0;
  for (int base = 0; base < (int)n_cand; base += 32) {
    const int j = base + lane;
    const uint32_t k16 = j < (int)n_cand ? kq[cw[j]] : 0u;
    c_gt += __popc(__ballot_sync(0xffffffffu, j < (int)n_cand && k16 > T));
    c_eq += __popc(__ballot_sync(0xffffffffu, j < (int)n_cand && k16 == T));
  }
  const uint32_t eq_before_w =
      __shfl_sync(0xffffffffu, block_exclusive_scan<NT>(lane == 0 ? c_eq : 0u, sm.warp_tot, &total), 0);
  int eq_take_w = eq_take_cta - (int)eq_before_w;
  eq_take_w = eq_take_w < 0 ? 0 : (eq_take_w > (int)c_eq ? (int)c_eq : eq_take_w);
  uint32_t o = off + block_exclusive_scan<NT>(lane == 0 ? c_gt + (uint32_t)eq_take_w : 0u, sm.warp_tot, &total);
  o = __shfl_sync(0xffffffffu, o, 0);
  int eq_seen = 0;
  for (int base = 0; base < (int)n_cand; base += 32) {
    const int j = base + lane;
    const bool in = j < (int)n_cand;
    const int p = in ? cw[j] : 0;
    const uint32_t k16 = in ? kq[p] : 0u;
    const unsigned eqm = __ballot_sync(0xffffffffu, in && k16 == T);
    const bool take = in && (k16 > T || (k16 == T && eq_seen + __popc(eqm & lt) < eq_take_w));
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) out[o + __popc(tm & lt)] = (int32_t)(s0 + p);
    o += __popc(tm);
    eq_seen += __popc(eqm);
  }

  // 5. the workspace back to zeros: this CTA's share of the prefix
  //    histogram; the last CTA to take a ticket (every other has read every
  //    slot by then) clears the slots and the counters
  for (int d = sl * kPrefixBins / S + tid; d < (sl + 1) * kPrefixBins / S; d += NT) H[d] = 0u;
  if (tid == 0) sm.hist[65] = ticket == (uint32_t)S - 1 ? 1u : 0u;
  __syncthreads();
  if (sm.hist[65]) {
    for (int i = tid; i < S * kSlotWords; i += NT) slots[i] = 0u;
    if (tid == 0) {
      ctr[0] = 0u;
      ctr[1] = 0u;  // the row's highest prefix
      ctr[2] = 0u;
    }
  }
}

// ------------------------------------------------------- fused decode form
// With a.fused set (one query per CTA, so one CTA per slice of a request):
// every CTA whose slice holds new key rows a.comp.e0 .. +n_out compresses
// them into the key cache before its producer loads the stage holding them,
// and the CTA holding row a.comp.e0 (the lead) also runs the extra job
// a.comp2 for its request.  The CTA starts the key stages before the first
// new row, then compresses while they land, in ring stages it has not used.
// One query's top k from its whole row in one CTA, with the 12-bit prefix
// histogram the epilogue built while the keys streamed (two 16-bit counts per
// word: bin d in half d & 1 of word d >> 1): the prefix d1 of the k-th key
// from the histogram, one pass over the keys that counts those above d1,
// histograms the 4-bit suffixes of those at d1 and keeps both as candidates,
// then the k-th key T and the ordered write over the candidates.  The same
// order as block_select: (key desc, position asc).  kk < nv.
template <int NT>
__device__ void hist_select(const uint16_t* kq, const uint32_t* h2, uint16_t* cand, int nv, int kk, int64_t s0,
                            int32_t* out, SelectSmem<NT>& sm) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t total;
  // 1. prefix d1 of the kk-th key and the keys still needed inside it (warp 0
  //    walks the bins down, 32 at a time)
  if (warp == 0) {
    uint32_t above = 0;
    bool found = false;
    for (int base = kPrefixBins - 1; base >= 0 && !found; base -= 32) {
      const int d = base - lane;
      const uint32_t c = d >= 0 ? (h2[d >> 1] >> (16 * (d & 1))) & 0xFFFFu : 0u;
      uint32_t inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, above + inc >= (uint32_t)kk);
      if (hit) {
        const int l = __ffs(hit) - 1;
        if (lane == l) {
          sm.bcast[0] = (uint32_t)d;
          sm.bcast[1] = (uint32_t)kk - (above + inc - c);
        }
        found = true;
      } else {
        above += __shfl_sync(0xffffffffu, inc, 31);
      }
    }
  }
  if (tid < 16) sm.hist[tid] = 0;
  __syncthreads();
  const uint32_t d1 = sm.bcast[0], rem1 = sm.bcast[1];
  // 2. candidates (prefix >= d1) of the warp's span, in order; keys above d1
  //    counted, suffixes at d1 histogrammed.  A lane reads 8 keys per step.
  const int span = ((nv + NW - 1) / NW + 255) / 256 * 256;
  const int w0 = min(nv, warp * span), w1 = min(nv, w0 + span);
  uint32_t n_cand = 0;
  for (int base = w0; base < w1; base += 256) {
    const int p0 = base + 8 * lane;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (p0 < w1) v = *reinterpret_cast<const uint4*>(kq + p0);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t cmask = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t k16 = (wv[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
      const bool in = p0 + j < w1 && (k16 >> 4) >= d1;
      cmask |= in ? (1u << j) : 0u;
      if (in && (k16 >> 4) == d1) atomicAdd(&sm.hist[k16 & 15u], 1u);
    }
    const uint32_t cnt = __popc(cmask);
    uint32_t inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    uint32_t at = (uint32_t)w0 + n_cand + inc - cnt;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (cmask & (1u << j)) cand[at++] = (uint16_t)(p0 + j);
    n_cand += __shfl_sync(0xffffffffu, inc, 31);
  }
  __syncthreads();  // the suffix histogram is complete
  // 3. the kk-th key T = (d1 << 4) | d2 and how many keys equal to T to take
  if (tid == 0) {
    uint32_t above = 0;
    for (int n = 15; n >= 0; --n) {
      if (above + sm.hist[n] >= rem1) {
        sm.bcast[2] = (uint32_t)n;
        sm.bcast[3] = rem1 - above;
        break;
      }
      above += sm.hist[n];
    }
  }
  __syncthreads();
  const uint32_t T = (d1 << 4) | sm.bcast[2];
  const int need_eq = (int)sm.bcast[3];
  // 4. per-warp counts over the candidates, offsets, ordered write
  const uint16_t* cw = cand + w0;
  uint32_t c_gt = 0, c_eq = 0;
  for (int base = 0; base < (int)n_cand; base += 32) {
    const int j = base + lane;
    const uint32_t k16 = j < (int)n_cand ? kq[cw[j]] : 0u;
    c_gt += __popc(__ballot_sync(0xffffffffu, j < (int)n_cand && k16 > T));
    c_eq += __popc(__ballot_sync(0xffffffffu, j < (int)n_cand && k16 == T));
  }
  const uint32_t eq_before_w =
      __shfl_sync(0xffffffffu, block_exclusive_scan<NT>(lane == 0 ? c_eq : 0u, sm.warp_tot, &total), 0);
  int eq_take_w = need_eq - (int)eq_before_w;
  eq_take_w = eq_take_w < 0 ? 0 : (eq_take_w > (int)c_eq ? (int)c_eq : eq_take_w);
  uint32_t o = block_exclusive_scan<NT>(lane == 0 ? c_gt + (uint32_t)eq_take_w : 0u, sm.warp_tot, &total);
  o = __shfl_sync(0xffffffffu, o, 0);
  int eq_seen = 0;
  for (int base = 0; base < (int)n_cand; base += 32) {
    const int j = base + lane;
    const bool in = j < (int)n_cand;
    const int p = in ? cw[j] : 0;
    const uint32_t k16 = in ? kq[p] : 0u;
    const unsigned eqm = __ballot_sync(0xffffffffu, in && k16 == T);
    const bool take = in && (k16 > T || (k16 == T && eq_seen + __popc(eqm & lt) < eq_take_w));
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) out[o + __popc(tm & lt)] = (int32_t)(s0 + p);
    o += __popc(tm);
    eq_seen += __popc(eqm);
  }
  __syncthreads();  // cand and the histogram are reused by the next query
}

// TMA row of logical key row lr of request b: the contiguous cache, or the
// pool row through the block table (rows at or past n_entries, never visible,
// read pool row 0; a page outside the pool is flagged and read as row 0).
__device__ __forceinline__ int key_tma_row(const IndexArgs& a, int b, int64_t lr) {
  if (a.pages.table == nullptr) return (int)((int64_t)b * a.n_entries + lr);
  if (lr >= a.n_entries) return 0;
  const int64_t r = pool_row(a.pages, b, lr);
  if (r < 0) {
    flag_status(kStatusBadPage);
    return 0;
  }
  return (int)r;
}

// Loads `rows` key rows of request b from logical row lr0 (a multiple of 128)
// into dst with the map's boxes: one box of `rows` rows when contiguous, one
// box per page (page_entries rows, which divides 128) when paged.  Boxes land
// row_bytes * rows apart, so the smem tile is the one a single box gives.
// half_bytes > 0: a second box column (x = 64) lands half_bytes after dst.
__device__ __forceinline__ void load_key_rows(const IndexArgs& a, const CUtensorMap* tm, uint8_t* dst,
                                              uint64_t* bar, int b, int64_t lr0, int rows, int row_bytes,
                                              int half_bytes) {
  const int step = a.pages.table == nullptr ? rows : a.pages.page_entries;
  for (int q = 0; q < rows; q += step) {
    const int row = key_tma_row(a, b, lr0 + q);
    tma_load_2d(dst + q * row_bytes, tm, bar, 0, row);
    if (half_bytes > 0) tma_load_2d(dst + half_bytes + q * row_bytes, tm, bar, 64, row);
  }
}

template <int NQ>
__device__ __forceinline__ bool fused_keys(const IndexArgs& a, int64_t s0, int len) {
  return NQ == 1 && a.fused && s0 < a.comp.e0 + a.comp.n_out && a.comp.e0 < s0 + len;
}
template <int NQ>
__device__ __forceinline__ bool fused_lead(const IndexArgs& a, int64_t s0, int len) {
  return NQ == 1 && a.fused && s0 <= a.comp.e0 && a.comp.e0 < s0 + len;
}
// Shared memory the fused jobs stage (all rows of both jobs at once), and
// whether the staged form applies (at most 32 token positions per entry).
__host__ __device__ __forceinline__ int fused_scratch_bytes(const IndexArgs& a) {
  int need = (int)a.comp.n_out * staged_entry_bytes(a.comp);
  if (a.comp2.n_out > 0) need += (int)a.comp2.n_out * staged_entry_bytes(a.comp2);
  return need;
}
__host__ __device__ __forceinline__ int fused_scratch_stages(const IndexArgs& a, int stage_bytes) {
  return (fused_scratch_bytes(a) + stage_bytes - 1) / stage_bytes;
}
__host__ __device__ __forceinline__ bool fused_jobs_staged(const IndexArgs& a) {
  return (a.comp.Cb != nullptr ? 2 : 1) * a.comp.m <= 32 &&
         (a.comp2.n_out == 0 || (a.comp2.Cb != nullptr ? 2 : 1) * a.comp2.m <= 32);
}
template <int NT>
__device__ void run_fused_jobs(const IndexArgs& a, int b, int64_t s0, int len, uint8_t* scratch, bool keys,
                               bool lead) {
  const int64_t lo = keys ? max64(a.comp.e0, s0) : 0, hi = keys ? min64(a.comp.e0 + a.comp.n_out, s0 + len) : 0;
  const int nk = (int)(hi - lo), nx = lead ? (int)a.comp2.n_out : 0;
  const int kb = staged_entry_bytes(a.comp), xb = nx > 0 ? staged_entry_bytes(a.comp2) : 0;
  const int64_t ik = lo - a.comp.e0;  // first key entry of this CTA, relative to e0
  uint8_t* const xbuf = scratch + (size_t)nk * kb;
  for (int e = 0; e < nk; ++e) stage_entry<NT>(a.comp, b, ik + e, scratch + (size_t)e * kb);
  for (int e = 0; e < nx; ++e) stage_entry<NT>(a.comp2, b, e, xbuf + (size_t)e * xb);
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // one channel per thread: the key entries' channels, then the extra job's
  const int dk = a.comp.dim, dx = a.comp2.dim, ck = nk * dk, cx = nx * dx;
  for (int g = threadIdx.x; g < ck + cx; g += NT) {
    if (g < ck) {
      staged_channel(a.comp, ik + g / dk, scratch + (size_t)(g / dk) * kb, g % dk);
    } else {
      const int h = g - ck;
      staged_channel(a.comp2, h / dx, xbuf + (size_t)(h / dx) * xb, h % dx);
    }
  }
  __syncthreads();
  // normalisation / RoPE epilogue of the pooled rows: a warp per entry
  const bool nk_row = compress_row_epilogue(a.comp), nx_row = nx > 0 && compress_row_epilogue(a.comp2);
  if (nk_row || nx_row) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = warp; e < nk + nx; e += NT / 32) {
      const bool key = e < nk;
      const CompressArgs& c = key ? a.comp : a.comp2;
      if (key ? !nk_row : !nx_row) continue;
      const int64_t ie = key ? ik + e : e - nk;
      uint8_t* buf = key ? scratch + (size_t)e * kb : xbuf + (size_t)(e - nk) * xb;
      const int esz = c.in_dt == CSA_F32 ? 4 : 2;
      float* xr = reinterpret_cast<float*>(buf + (size_t)staged_positions(c) * c.dim * (2 * esz + 4));
      warp_norm_rope_row(xr, c.dim, c.norm_g, c.norm_eps, c.rope_dims, c.rope_base,
                         (double)(c.pos_stride * (c.e0 + ie) + c.pos_offset), lane);
    }
    __syncthreads();
  }
  // quantise and write, 8 channels per thread (whole warps: the scale blocks
  // of a row are consecutive lanes)
  const int qk = nk * (dk / 8), qx = nx * (dx / 8);
  for (int c0 = 0; c0 < qk; c0 += NT) {
    const int q = c0 + threadIdx.x;
    const bool v = q < qk;
    const int e = v ? q / (dk / 8) : 0;
    staged_store(a.comp, b, ik + e, scratch + (size_t)e * kb, v ? q % (dk / 8) : 0, v);
  }
  for (int c0 = 0; c0 < qx; c0 += NT) {
    const int q = c0 + threadIdx.x;
    const bool v = q < qx;
    const int e = v ? q / (dx / 8) : 0;
    staged_store(a.comp2, b, e, xbuf + (size_t)e * xb, v ? q % (dx / 8) : 0, v);
  }
  fence_proxy_async_global();  // the new key rows are read back by this CTA's TMA
  __syncthreads();
}

// ----------------------------------------------------------------- BF16 kernel
template <int NQ>
__global__ void __launch_bounds__(kThreads, 1)
    index_bf16_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, IndexArgs a,
                      IndexPlan plan) {
  using C = Bf16Cfg<NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ks = align1024(smem_raw);                        // K ring
  uint8_t* qs = ks + C::STAGES * C::K_STAGE;                // query tile
  uint16_t* keys = reinterpret_cast<uint16_t*>(qs + C::Q_BYTES);
  uint16_t* cand = reinterpret_cast<uint16_t*>(ks);          // [slice_len] candidates, on the idle ring
  float* wsm = reinterpret_cast<float*>(keys + NQ * plan.slice_len);
  uint64_t* full = reinterpret_cast<uint64_t*>(wsm + NQ * kHI);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + C::NBUF;
  uint64_t* qbar = acce + C::NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 1);
  SelectSmem<kThreads>& sel = *reinterpret_cast<SelectSmem<kThreads>*>(tmem_slot + 4);
  uint32_t* hist = reinterpret_cast<uint32_t*>(&sel + 1);  // prefix histogram(s) (HIST bytes)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool coop = NQ == 1 && plan.coop;
  const bool h2 = NQ == 2 && plan.n_slices == 1;  // one-slice rows select from the epilogue's histograms
  // The queries and the first key tiles do not depend on the query
  // positions: the producer thread starts them before anything is loaded.
  const int64_t s0 = (int64_t)blockIdx.x * plan.slice_len;
  const int len0 = (int)min64(plan.slice_len, a.n_entries - s0);
  const bool fkeys = fused_keys<NQ>(a, s0, len0), flead = fused_lead<NQ>(a, s0, len0);
  const int nscr = (fkeys || flead) ? fused_scratch_stages(a, C::K_STAGE) : 0;
  int pre = min(C::STAGES - nscr, (len0 + kBM - 1) / kBM);
  if (fkeys) pre = min(pre, (int)(max64(0, a.comp.e0 - s0) / kBM));
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int i = 0; i < C::NBUF; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 4); }
    mbar_init(qbar, 1);
    fence_barrier_init();
    const int qrow = (blockIdx.z * a.n_q + blockIdx.y * NQ) * kHI;
    mbar_arrive_expect_tx(qbar, C::Q_BYTES);
    tma_load_2d(qs, &tmQ, qbar, 0, qrow);
    tma_load_2d(qs + C::N * 128, &tmQ, qbar, 64, qrow);
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&full[i], C::K_STAGE);
      load_key_rows(a, &tmK, ks + i * C::K_STAGE, &full[i], blockIdx.z, s0 + (int64_t)i * kBM, kBM, 128, kAtom);
    }
  }
  if (fkeys || flead)
    run_fused_jobs<kThreads>(a, blockIdx.z, s0, len0, ks + (C::STAGES - nscr) * C::K_STAGE, fkeys, flead);
  const SliceCtx<NQ> c = slice_ctx<NQ>(a, plan);
  for (int i = threadIdx.x; i < NQ * kHI; i += kThreads) {
    const int t = c.t0 + i / kHI;
    wsm[i] = t < a.n_q ? a.wI[((int64_t)c.b * a.n_q + t) * kHI + (i % kHI)] : 0.f;
  }
  if (coop)
    for (int i = threadIdx.x; i < kPrefixBins; i += kThreads) hist[i] = 0;
  if (h2)
    for (int i = threadIdx.x; i < NQ * kPrefixBins / 2; i += kThreads) hist[i] = 0;
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = pre; i < c.n_tiles; ++i) {
        const int s = i % C::STAGES, j = i / C::STAGES;
        if (j > 0 && !mbar_wait(&empty[s], (j - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[s], C::K_STAGE);
        load_key_rows(a, &tmK, ks + s * C::K_STAGE, &full[s], c.b, c.s0 + (int64_t)i * kBM, kBM, 128, kAtom);
      }
      // tiles started early but beyond the visible entries: wait for their
      // bytes before the CTA moves on
      for (int i = c.n_tiles; i < pre; ++i) mbar_wait(&full[i], 0);
    }
  } else if (warp == 1 || warp == 2) {
    // MMA issuers: warp 1 issues the even tiles, warp 2 the odd ones (eight
    // tcgen05.mma per tile cost one issuing thread about as long as the
    // tile's data takes to stream).  NBUF is even, so a buffer always belongs
    // to the same issuer and each issuer waits on every phase of its
    // barriers in order; a stage's uses alternate issuers, but a stage is
    // refilled only after its previous use committed, so no phase is missed.
    if (lane == 0) {
      const int w = warp - 1;
      bool ok = mbar_wait(qbar, 0);
      const uint32_t qa = smem_u32(qs);
      for (int i = w; ok && i < c.n_tiles; i += 2) {
        const int s = i % C::STAGES, j = i / C::STAGES, buf = i % C::NBUF, u = i / C::NBUF;
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
          tc_mma_f16(d, umma_desc_sw128(a_addr), umma_desc_sw128(b_addr), C::IDESC, kk > 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
        tc_commit(&accf[buf]);
      }
    }
  } else if (warp >= 4) {
    epilogue_group<NQ, C::N, C::NBUF>(c, a, plan, tmem, accf, acce, wsm, keys, coop, hist, h2);
  }
  scores_tail<NQ, kThreads>(c, a);
  tc_fence_before();
  __syncthreads();
  if (coop) {
    coop_select<kThreads>(keys, cand, c.n_valid[0], c.vis[0], c.s0, c.sl, plan, a, (int64_t)c.b * a.n_q + c.t0, hist,
                          sel);
    __syncthreads();
  } else {
    slice_select<NQ, kThreads>(c, a, plan, keys, sel, h2 ? hist : nullptr, cand);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- NVFP4 kernel
// rows [0, rows) of a row-major [rows][8] scale block -> two 512-byte atoms
// (rows >= `rows` are zero).  One warp.
__device__ __forceinline__ void permute_scales(const uint8_t* raw, uint8_t* atoms, int rows, int lane) {
  const uint32_t* src = reinterpret_cast<const uint32_t*>(raw);
  uint32_t* dst = reinterpret_cast<uint32_t*>(atoms);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int w = lane + 32 * j;                 // output word: kb * 128 + m0 * 4 + m1
    const int kb = w >> 7, m0 = (w & 127) >> 2, m1 = w & 3;
    const int m = m0 + 32 * m1;
    dst[w] = m < rows ? src[m * 2 + kb] : 0u;
  }
}

template <int NQ>
__global__ void __launch_bounds__(Nvf4Cfg<NQ>::NT, 1)
    index_nvf4_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmQs, IndexArgs a, IndexPlan plan) {
  using C = Nvf4Cfg<NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* st = align1024(smem_raw);                          // stages: codes x2 | scale atoms x2
  uint8_t* qreg = st + C::STAGES * C::STAGE;                  // q codes | q raw scales | q atoms
  uint16_t* keys = reinterpret_cast<uint16_t*>(qreg + C::QREG);
  uint16_t* cand = reinterpret_cast<uint16_t*>(st);          // [slice_len] candidates, on the idle ring
  float* wsm = reinterpret_cast<float*>(keys + NQ * plan.slice_len);
  uint64_t* full = reinterpret_cast<uint64_t*>(wsm + NQ * kHI);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* acce = accf + C::NBUF;
  uint64_t* qbar = acce + C::NBUF;
  uint64_t* qsf = qbar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qsf + 1);
  SelectSmem<C::NT>& sel = *reinterpret_cast<SelectSmem<C::NT>*>(tmem_slot + 4);
  uint32_t* hist = reinterpret_cast<uint32_t*>(&sel + 1);  // prefix histogram(s) (HIST bytes)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool coop = NQ == 1 && plan.coop;
  // The queries and the first stages of key codes do not depend on the query
  // positions: the producer thread starts them before anything is loaded.
  const int64_t s0 = (int64_t)blockIdx.x * plan.slice_len;
  const int len0 = (int)min64(plan.slice_len, a.n_entries - s0);
  const int b0 = blockIdx.z, t00 = blockIdx.y * NQ;
  const bool fkeys = fused_keys<NQ>(a, s0, len0), flead = fused_lead<NQ>(a, s0, len0);
  const int nscr = (fkeys || flead) ? fused_scratch_stages(a, C::STAGE) : 0;
  int pre = min(C::STAGES - nscr, ((len0 + kBM - 1) / kBM + C::TPS - 1) / C::TPS);
  if (fkeys) pre = min(pre, (int)(max64(0, a.comp.e0 - s0) / (C::TPS * kBM)));
  if (threadIdx.x == 0) {
    // full: one arrival from each producer (codes, scales); empty: one
    // commit from each issuer (the stage's two tiles)
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 2); mbar_init(&empty[s], C::TPS); }
    for (int i = 0; i < C::NBUF; ++i) { mbar_init(&accf[i], 1); mbar_init(&acce[i], 4); }
    mbar_init(qbar, 1);
    mbar_init(qsf, 1);
    fence_barrier_init();
    const int qrow = (b0 * a.n_q + t00) * kHI;
    mbar_arrive_expect_tx(qbar, C::QCODES + C::QRAWSF);
    tma_load_2d(qreg, &tmQ, qbar, 0, qrow);
    tma_load_2d(qreg + C::QCODES, &tmQs, qbar, 0, qrow / 2);
    for (int g = 0; g < pre; ++g) {
      // a 256-row box: rows past the tensor read as zero, rows of the next
      // request are never valid positions here
      mbar_arrive_expect_tx(&full[g], C::TPS * C::CODES);
      load_key_rows(a, &tmK, st + g * C::STAGE, &full[g], b0, s0 + (int64_t)g * C::TPS * kBM, C::TPS * kBM, 64, 0);
    }
  }
  if (fkeys || flead)
    run_fused_jobs<C::NT>(a, b0, s0, len0, st + (C::STAGES - nscr) * C::STAGE, fkeys, flead);
  const SliceCtx<NQ> c = slice_ctx<NQ>(a, plan);
  const int n_stages = (c.n_tiles + C::TPS - 1) / C::TPS;
  for (int i = threadIdx.x; i < NQ * kHI; i += C::NT) {
    const int t = c.t0 + i / kHI;
    wsm[i] = t < a.n_q ? a.wI[((int64_t)c.b * a.n_q + t) * kHI + (i % kHI)] : 0.f;
  }
  if (coop)
    for (int i = threadIdx.x; i < kPrefixBins; i += C::NT) hist[i] = 0;
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------- producer: codes, 2 tiles per copy
    if (lane == 0) {
      for (int g = pre; g < n_stages; ++g) {
        const int s = g % C::STAGES, j = g / C::STAGES;
        if (j > 0 && !mbar_wait(&empty[s], (j - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[s], C::TPS * C::CODES);
        load_key_rows(a, &tmK, st + s * C::STAGE, &full[s], c.b, c.s0 + (int64_t)g * C::TPS * kBM, C::TPS * kBM, 64,
                      0);
      }
      // stages started early but beyond the visible entries: add the missing
      // scale-side arrival and wait for their bytes before the CTA moves on
      for (int g = n_stages; g < pre; ++g) {
        mbar_arrive(&full[g]);
        mbar_wait(&full[g], 0);
      }
    }
  } else if (warp == 2) {
    // ------------- query scales into their atoms, then producer: key scale atoms
    if (mbar_wait(qbar, 0)) permute_scales(qreg + C::QCODES, qreg + C::QCODES + C::QRAWSF, C::N, lane);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(qsf);
      // request b's blocked key scales: 1 KB (two atoms) per 128-entry block;
      // slices start on block boundaries, so tile i is block s0/128 + i
      // (paged: the block of the pool page holding the tile's first row)
      const uint8_t* ksf = static_cast<const uint8_t*>(a.KI_sf) +
                           (int64_t)c.b * nvfp4_blocked_sf_bytes(a.n_entries, kDI) + (c.s0 / kBM) * C::ATOMS;
      for (int g = 0; g < n_stages; ++g) {
        const int s = g % C::STAGES, j = g / C::STAGES;
        if (j > 0 && !mbar_wait(&empty[s], (j - 1) & 1)) break;
        const int nt = min(C::TPS, c.n_tiles - g * C::TPS);  // blocks that exist
        mbar_arrive_expect_tx(&full[s], nt * C::ATOMS);
        uint8_t* dst = st + s * C::STAGE + C::TPS * C::CODES;
        if (a.pages.table == nullptr) {
          bulk_load(dst, ksf + (int64_t)g * C::TPS * C::ATOMS, nt * C::ATOMS, &full[s]);
        } else {
          for (int h = 0; h < nt; ++h) {
            int64_t pg = pool_sf_page(a.pages, c.b, c.s0 + (int64_t)(g * C::TPS + h) * kBM);
            if (pg < 0) {
              flag_status(kStatusBadPage);
              pg = 0;
            }
            bulk_load(dst + h * C::ATOMS, static_cast<const uint8_t*>(a.KI_sf) + pg * C::ATOMS, C::ATOMS, &full[s]);
          }
        }
      }
    }
  } else if (warp == 1 || warp == 3 || warp >= 12) {
    // ------------------------------------------------------------ MMA issuers
    // issuer w (warps 1, 3, 12, 13) issues the tiles i with i % NI == w, with
    // its own TMEM scale columns; tcgen05.commit tracks the issuing thread's
    // work only, so each stage's empty barrier takes one commit per tile.
    if (lane == 0) {
      const int w = warp == 1 ? 0 : warp == 3 ? 1 : warp - 10;
      const bool ok = mbar_wait(qsf, 0);
      const uint32_t qa = smem_u32(qreg);
      const uint32_t sfa = tmem + C::SFA_COL + 8 * w, sfb = tmem + C::SFB_COL + 8 * w;
      if (ok) {
        tc_fence_after();
        for (int kb = 0; kb < 2; ++kb)
          tc_cp_32x128b_warpx4(sfb + kb * 4, umma_desc_rows16(qa + C::QCODES + C::QRAWSF + kb * 512));
      }
      for (int i = w; ok && i < c.n_tiles; i += C::NI) {
        const int g = i / C::TPS, s = g % C::STAGES, j = g / C::STAGES, buf = i % C::NBUF, u = i / C::NBUF;
        if (!mbar_wait(&full[s], j & 1)) break;
        if (u > 0 && !mbar_wait(&acce[buf], (u - 1) & 1)) break;
        tc_fence_after();
        const int h = i % C::TPS;  // tile within the stage
        const uint32_t codes = smem_u32(st + s * C::STAGE) + (uint32_t)(h * C::CODES);
        const uint32_t atoms = smem_u32(st + s * C::STAGE) + (uint32_t)(C::TPS * C::CODES + h * C::ATOMS);
        for (int kb = 0; kb < 2; ++kb) tc_cp_32x128b_warpx4(sfa + kb * 4, umma_desc_rows16(atoms + kb * 512));
        const uint32_t d = tmem + (uint32_t)(buf * C::N);
        for (int kb = 0; kb < 2; ++kb)
          tc_mma_nvf4(d, umma_desc_sw64(codes + kb * 32), umma_desc_sw64(qa + kb * 32), C::IDESC, sfa + kb * 4,
                      sfb + kb * 4, kb > 0 ? 1u : 0u);
        tc_commit(&empty[s]);
        tc_commit(&accf[buf]);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    epilogue_group<NQ, C::N, C::NBUF>(c, a, plan, tmem, accf, acce, wsm, keys, coop, hist);
  }
  scores_tail<NQ, C::NT>(c, a);
  tc_fence_before();
  __syncthreads();
  if (coop) {
    coop_select<C::NT>(keys, cand, c.n_valid[0], c.vis[0], c.s0, c.sl, plan, a, (int64_t)c.b * a.n_q + c.t0, hist,
                       sel);
    __syncthreads();
  } else {
    slice_select<NQ, C::NT>(c, a, plan, keys, sel);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

// Rows of the key tensor map: every request's cache, or the pool.
uint64_t key_map_rows(const IndexArgs& a) {
  return a.pages.table == nullptr ? (uint64_t)a.batch * a.n_entries
                                  : (uint64_t)a.pages.n_pages * a.pages.page_entries;
}
// Box height of the key map: `rows` (a stage's tiles), or one page.
uint32_t key_box_rows(const IndexArgs& a, int rows) {
  return a.pages.table == nullptr ? (uint32_t)rows : (uint32_t)a.pages.page_entries;
}

template <int NQ>
cudaError_t launch_bf16(const IndexArgs& a, const IndexPlan& p, cudaStream_t s) {
  using C = Bf16Cfg<NQ>;
  CUtensorMap tmK, tmQ;
  const uint64_t krows = key_map_rows(a), qrows = (uint64_t)a.batch * a.n_q * kHI;
  if (!make_map_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.KI, krows, kDI, 64, key_box_rows(a, kBM),
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.qI, qrows, kDI, 64, C::N, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = (size_t)C::FIXED_SMEM + (size_t)C::PER_ENTRY * p.slice_len;
  cudaError_t e = cudaFuncSetAttribute(index_bf16_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_slices, (a.n_q + NQ - 1) / NQ, a.batch);
  if (p.coop) {
    // the slices of a row wait on one another: launch cooperatively so that
    // every CTA is resident (their counters and histograms start at zero and
    // the kernel leaves them at zero)
    IndexArgs aa = a;
    IndexPlan pp = p;
    CUtensorMap m0 = tmK, m1 = tmQ;
    void* args[] = {&m0, &m1, &aa, &pp};
    e = cudaLaunchCooperativeKernel((const void*)index_bf16_kernel<NQ>, grid, dim3(kThreads), args, smem, s);
    ++launch_counter();
    return e;
  }
  index_bf16_kernel<NQ><<<grid, kThreads, smem, s>>>(tmK, tmQ, a, p);
  ++launch_counter();
  return cudaGetLastError();
}

template <int NQ>
cudaError_t launch_nvf4(const IndexArgs& a, const IndexPlan& p, cudaStream_t s) {
  using C = Nvf4Cfg<NQ>;
  CUtensorMap tmK, tmQ, tmQs;
  const uint64_t krows = key_map_rows(a), qrows = (uint64_t)a.batch * a.n_q * kHI;
  // packed E2M1 rows of 64 bytes in the 64-byte swizzle; query scales as
  // 16-byte lines holding two head rows each (key scales are bulk-copied)
  const bool ok =
      make_map_2d(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.KI, krows, kDI / 2, kDI / 2,
                  key_box_rows(a, C::TPS * kBM), CU_TENSOR_MAP_SWIZZLE_64B) &&
      make_map_2d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.qI, qrows, kDI / 2, kDI / 2, C::N,
                  CU_TENSOR_MAP_SWIZZLE_64B) &&
      make_map_2d(&tmQs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.qI_sf, qrows / 2, 16, 16, C::N / 2,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = (size_t)C::FIXED_SMEM + (size_t)C::PER_ENTRY * p.slice_len;
  cudaError_t e = cudaFuncSetAttribute(index_nvf4_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_slices, (a.n_q + NQ - 1) / NQ, a.batch);
  if (p.coop) {
    // the slices of a row wait on one another: launch cooperatively so that
    // every CTA is resident (their counters and histograms start at zero and
    // the kernel leaves them at zero)
    IndexArgs aa = a;
    IndexPlan pp = p;
    CUtensorMap m0 = tmK, m1 = tmQ, m2 = tmQs;
    void* args[] = {&m0, &m1, &m2, &aa, &pp};
    e = cudaLaunchCooperativeKernel((const void*)index_nvf4_kernel<NQ>, grid, dim3(C::NT), args, smem, s);
    ++launch_counter();
    return e;
  }
  index_nvf4_kernel<NQ><<<grid, C::NT, smem, s>>>(tmK, tmQ, tmQs, a, p);
  ++launch_counter();
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SMs of the current device (148 when it cannot be queried, e.g. no GPU).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn() {
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

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int esize, const void* base, uint64_t rows,
                 uint64_t cols, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  auto fn = tma_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool index_tc_eligible(const IndexArgs& a) {
  if (a.n_heads != kHI || a.dim != kDI || a.n_entries <= 0) return false;
  if ((int64_t)a.batch * a.n_entries >= ((int64_t)1 << 31) || (int64_t)a.batch * a.n_q * kHI >= ((int64_t)1 << 31))
    return false;
  // the key tensor must be at least one TMA box high (128 rows BF16, 256 NVFP4)
  const int64_t krows = (int64_t)a.batch * a.n_entries;
  if (a.dt == CSA_BF16) return krows >= kBM;
  // NVFP4: key scale atoms are bulk-copied and query scales streamed as
  // 16-byte lines, so both arrays must be 16-byte aligned.
  return a.dt == CSA_IDX_NVFP4 && krows >= 2 * kBM && aligned16(a.KI_sf) && aligned16(a.qI_sf);
}

int index_tc_nq(int n_q) { return n_q >= 2 ? 2 : 1; }

bool index_fusable(const IndexArgs& a) {
  if (!index_tc_eligible(a) || index_tc_nq(a.n_q) != 1 || a.n_entries < 1 || !fused_jobs_staged(a)) return false;
  // a decode step closes a few groups; larger jobs run as separate launches
  // (which also keeps the kernel's int scratch arithmetic far from overflow)
  if (a.comp.n_out > 64 || a.comp2.n_out > 64 || a.comp.dim > 8192 || a.comp2.dim > 8192) return false;
  // the compress scratch must leave the ring at least one stage
  if (a.dt == CSA_IDX_NVFP4) return fused_scratch_stages(a, Nvf4Cfg<1>::STAGE) < Nvf4Cfg<1>::STAGES;
  return fused_scratch_stages(a, Bf16Cfg<1>::K_STAGE) < Bf16Cfg<1>::STAGES;
}

IndexPlan make_tc_plan(int batch, int n_q, int64_t n_entries, int k, int dt) {
  const int NQ = index_tc_nq(n_q);
  const bool fp4 = dt == CSA_IDX_NVFP4;
  const int fixed = NQ == 1 ? (fp4 ? Nvf4Cfg<1>::FIXED_SMEM : Bf16Cfg<1>::FIXED_SMEM)
                            : (fp4 ? Nvf4Cfg<2>::FIXED_SMEM : Bf16Cfg<2>::FIXED_SMEM);
  const int per_entry = NQ == 1 ? (fp4 ? Nvf4Cfg<1>::PER_ENTRY : Bf16Cfg<1>::PER_ENTRY)
                                : (fp4 ? Nvf4Cfg<2>::PER_ENTRY : Bf16Cfg<2>::PER_ENTRY);
  constexpr int kSmemCap = 227 * 1024;
  int64_t max_slice = ((kSmemCap - fixed) / per_entry) / kBM * kBM;
  // the cooperative select keeps a 16-bit candidate per entry on the stage ring
  const int64_t ring = NQ == 1 ? (fp4 ? Nvf4Cfg<1>::STAGES * Nvf4Cfg<1>::STAGE : Bf16Cfg<1>::STAGES * Bf16Cfg<1>::K_STAGE)
                               : (int64_t)1 << 40;
  if (max_slice > ring / 2 / kBM * kBM) max_slice = ring / 2 / kBM * kBM;
  const int64_t groups = (n_q + NQ - 1) / NQ;
  const int64_t units = (int64_t)batch * groups;
  const int sms = sm_count();
  // one wave: at most one CTA per SM (the kernels' shared memory allows one)
  const int64_t want = units >= sms ? 1 : sms / units;
  int64_t len = (n_entries + want - 1) / want;
  len = (len + kBM - 1) / kBM * kBM;
  if (len < kBM) len = kBM;
  if (len > max_slice) len = max_slice;
  IndexPlan p{};
  p.slice_len = (int)len;
  p.n_slices = (int)((n_entries + len - 1) / len);
  if (p.n_slices < 1) p.n_slices = 1;
  p.n_rows = (int64_t)batch * n_q;
  // decode rows split over several slices select cooperatively when the
  // whole grid fits on the GPU at once
  p.coop = (NQ == 1 && p.n_slices > 1 && units * p.n_slices <= sms) ? 1 : 0;
  p.cand_cap = (p.n_slices > 1 && !p.coop) ? (int64_t)p.n_slices * k : 0;
  return p;
}

void index_tc_ring(int n_q, int dt, int* stages, int* tiles_per_stage) {
  const bool one = index_tc_nq(n_q) == 1;
  if (dt == CSA_IDX_NVFP4) {
    *stages = one ? Nvf4Cfg<1>::STAGES : Nvf4Cfg<2>::STAGES;
    *tiles_per_stage = Nvf4Cfg<1>::TPS;
  } else {
    *stages = one ? Bf16Cfg<1>::STAGES : Bf16Cfg<2>::STAGES;
    *tiles_per_stage = 1;
  }
}

cudaError_t launch_index_tc(const IndexArgs& a, const IndexPlan& p, cudaStream_t s) {
  const bool fp4 = a.dt == CSA_IDX_NVFP4;
  if (index_tc_nq(a.n_q) == 1) return fp4 ? launch_nvf4<1>(a, p, s) : launch_bf16<1>(a, p, s);
  return fp4 ? launch_nvf4<2>(a, p, s) : launch_bf16<2>(a, p, s);
}

}  // namespace csa
