// out_proj.cu -- grouped output projection after the core attention
// ("DeepSeek-V4 内部机制" 1.2 Step 3: the n_h head outputs of a token are cut
// into g groups of n_h/g heads; each group is projected to d_g, the g results
// are concatenated and projected to the model dimension d).
//
//   Z[t, i d_g + e] = sum_j O[t, i n_h/g c + j] Wg[i][j][e]     (per group i)
//   Y[t, o]         = sum_j Z[t, j] Wo[j][o]
//
// Both steps are one tcgen05 GEMM kernel in the transposed form
//   out^T[n, t] = sum_k W[k][n] X[t][k]
// so that the weight columns fill the 128 rows of the MMA (M) and the tokens,
// few in decode, are its N: A = a 128 x 64 tile of W read MN-major (two TMA
// boxes of 64 columns x 64 rows, 128-byte swizzle), B = an N x 64 tile of X
// read K-major (one TMA box), fp32 accumulation in TMEM.  A CTA owns 128
// weight columns of one group, up to 256 tokens and one slice of K; warp 0
// issues the TMA loads of a 4-stage ring, warp 1 the MMAs, warps 2-5 drain
// TMEM (lane = weight column).
//
// In decode the weights (128 MB + 235 MB for V4-Pro's g = 16, d_g = 1024,
// d = 7168) are the whole traffic, so K is split until every SM holds CTAs:
// each slice writes its fp32 partial sums, and the last slice of a tile to
// finish (a counter per tile, left zero again) adds the slices in slice order
// and writes the bf16 result, so the sum is the same whatever order the CTAs
// ran in.  Z is kept in bf16 between the steps (the precision of the
// activations around it).
#include "csa_internal.cuh"
#include "sm100.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_out_proj)

namespace {

constexpr int kBN = 128;               // weight columns per CTA (MMA M)
constexpr int kBK = 64;                // K per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 4;
constexpr int kThreads = 192;          // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kATile = kBN * kBK * 2;  // 16 KB: two boxes of 64 columns x 64 rows
constexpr int kMaxNT = 256;            // tokens per CTA (MMA N)
constexpr int kSMs = 148;              // B200; fixed so that the plan (and the sum order) is device-independent
constexpr int kMaxSplits = 16;
constexpr int kMaxResident = 16;
// K is split only while the tiles are fewer than the CTA slots, so at most
// kSMs * kMaxResident tiles ever use a counter; the counters sit at the start
// of the workspace in a region of that fixed size, where no other data of any
// shape's call lands.
constexpr int kMaxTickets = kSMs * kMaxResident;
constexpr size_t kTicketBytes = (kMaxTickets * sizeof(int) + 255) / 256 * 256;

struct ProjArgs {
  int T;               // tokens
  int K;               // reduction length per group
  int Nw;              // weight columns per group (multiple of 128)
  int nt;              // tokens per CTA (multiple of 16, <= 256)
  int splits;          // K slices per tile
  __nv_bfloat16* Y;    // [T][ldy], group i's columns at i * Nw
  int64_t ldy;
  float* part;         // [splits][T][groups * Nw] fp32 partial sums (splits > 1)
  int* tickets;        // one per tile, zero on entry and on exit (splits > 1)
};

__host__ __device__ constexpr int tmem_cols_for(int n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : 256; }

struct ProjPlan {
  int nt, splits, tiles;
  size_t smem;
};

ProjPlan plan_projection(int T, int K, int Nw, int groups) {
  ProjPlan p{};
  p.nt = T >= kMaxNT ? kMaxNT : (T + 15) / 16 * 16;
  p.smem = 1024 + (size_t)kStages * (kATile + p.nt * 128) + 256;
  const int by_smem = (int)(233472 / (p.smem + 1024));
  const int by_tmem = 512 / tmem_cols_for(p.nt);
  int resident = by_smem < by_tmem ? by_smem : by_tmem;
  if (resident > kMaxResident) resident = kMaxResident;
  const int64_t tiles = (int64_t)(Nw / kBN) * ((T + p.nt - 1) / p.nt) * groups;
  p.tiles = (int)tiles;
  const int64_t slots = (int64_t)kSMs * (resident > 0 ? resident : 1);
  int s = tiles >= slots ? 1 : (int)(slots / tiles);  // splits > 1 implies tiles < slots <= kMaxTickets
  const int by_k = (K / kBK) / 4;  // at least 4 K steps per slice
  if (s > by_k) s = by_k;
  if (s > kMaxSplits) s = kMaxSplits;
  p.splits = s < 1 ? 1 : s;
  return p;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    out_proj_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = align1024(smem_raw);
  const int stage_bytes = kATile + a.nt * 128;  // A tile, then the N x 64 tile of X
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * stage_bytes);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  int* last_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // token tiles vary fastest, so the CTAs that read one weight strip run
  // together and the strip comes from HBM once (the token tiles, shared by
  // every strip of a group, stay in L2)
  const int tiles_n = a.Nw / kBN, tiles_t = (a.T + a.nt - 1) / a.nt;
  const int t_tile = (int)(blockIdx.x % tiles_t);
  const int n_tile = (int)((blockIdx.x / tiles_t) % tiles_n), split = (int)(blockIdx.x / tiles_t / tiles_n);
  const int n0 = n_tile * kBN, t0 = t_tile * a.nt, grp = blockIdx.y;
  const int n_k = a.K / kBK;
  const int ks0 = (int)((int64_t)split * n_k / a.splits), ks1 = (int)((int64_t)(split + 1) * n_k / a.splits);
  const uint32_t tcols = (uint32_t)tmem_cols_for(a.nt);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, tcols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmW);
      tma_prefetch_desc(&tmX);
      int issued = 0;
      for (int ks = ks0; ks < ks1; ++ks, ++issued) {
        const int s = issued % kStages, j = issued / kStages;
        if (j > 0 && !mbar_wait(&empty[s], (j - 1) & 1)) break;
        uint8_t* st = ring + s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
        const int kg = grp * a.K + ks * kBK;
        tma_load_2d(st, &tmW, &full[s], n0, kg);
        tma_load_2d(st + kATile / 2, &tmW, &full[s], n0 + 64, kg);
        tma_load_2d(st + kATile, &tmX, &full[s], kg, t0);
      }
      // the last loads of every stage have landed before the CTA may end
      // (they normally have: the MMAs consumed them)
      for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32_major(kBN, a.nt, 1, 0);
      for (int ks = ks0, i = 0; ks < ks1; ++ks, ++i) {
        const int s = i % kStages, j = i / kStages;
        if (!mbar_wait(&full[s], j & 1)) break;
        tc_fence_after();
        const uint32_t st = smem_u32(ring + s * stage_bytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          tc_mma_f16(tmem, umma_desc_sw128_mn(st + kk * 2048, kATile / 2, 1024),
                     umma_desc_sw128(st + kATile + kk * 32), idesc, (i | kk) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accf);
    }
  } else {
    // epilogue: lane = weight column n0 + 32 q + lane, TMEM columns = tokens
    const int q = warp & 3;
    const int col = grp * a.Nw + n0 + 32 * q + lane;
    const int t_end = a.T - t0 < a.nt ? a.T - t0 : a.nt;
    mbar_wait(accf, 0);
    tc_fence_after();
    const int64_t cols = (int64_t)gridDim.y * a.Nw;
    float* part = a.part + (int64_t)split * a.T * cols + col;
    __nv_bfloat16* y = a.Y + col;
    for (int c0 = 0; c0 < t_end; c0 += 32) {
      float v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int t = c0 + j;
        if (t < t_end) {
          if (a.splits == 1)
            y[(int64_t)(t0 + t) * a.ldy] = __float2bfloat16_rn(v[j]);
          else
            part[(int64_t)(t0 + t) * cols] = v[j];
        }
      }
    }
    if (a.splits > 1) {
      __threadfence();
      epilogue_bar();
      int* ticket = a.tickets + ((int64_t)grp * tiles_t + t_tile) * tiles_n + n_tile;
      if (threadIdx.x == 64) *last_flag = atomicAdd(ticket, 1) == a.splits - 1;
      epilogue_bar();
      if (*last_flag) {
        __threadfence();
        const float* p0 = a.part + col;
        for (int t = t0; t < t0 + t_end; ++t) {
          float acc = 0.f;
          for (int s = 0; s < a.splits; ++s) acc += __ldcg(p0 + ((int64_t)s * a.T + t) * cols);
          y[(int64_t)t * a.ldy] = __float2bfloat16_rn(acc);
        }
        if (threadIdx.x == 64) atomicExch(ticket, 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// One projection out[t, grp * Nw + n] = sum_k W[grp * K + k][n] X[t][grp * K + k]
// for every group: W is [groups * K][Nw] and X is [T][groups * K] (bf16,
// row-major); Y is [T][groups * Nw].
cudaError_t launch_projection(const void* W, const void* X, __nv_bfloat16* Y, int T, int K, int Nw, int groups,
                              float* part, int* tickets, cudaStream_t s) {
  const ProjPlan p = plan_projection(T, K, Nw, groups);
  CUtensorMap tmW, tmX;
  if (!make_map_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, (uint64_t)groups * K, (uint64_t)Nw, 64, kBK,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, (uint64_t)T, (uint64_t)groups * K, kBK,
                   (uint32_t)p.nt, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  ProjArgs a{T, K, Nw, p.nt, p.splits, Y, (int64_t)groups * Nw, part, tickets};
  cudaError_t e = cudaFuncSetAttribute(out_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((int64_t)(Nw / kBN) * p.splits * ((T + p.nt - 1) / p.nt)), (unsigned)groups);
  out_proj_kernel<<<grid, kThreads, p.smem, s>>>(tmW, tmX, a);
  ++launch_counter();
  return cudaGetLastError();
}

struct OutProjLayout {
  size_t z, tickets, part, total;
};

OutProjLayout out_proj_layout(int T, int n_h, int c, int g, int d_g, int d) {
  const ProjPlan p1 = plan_projection(T, n_h / g * c, d_g, g), p2 = plan_projection(T, g * d_g, d, 1);
  OutProjLayout l{};
  l.tickets = 0;
  l.z = kTicketBytes;
  l.part = l.z + align256((size_t)T * g * d_g * 2);
  const size_t b1 = p1.splits > 1 ? (size_t)p1.splits * T * g * d_g * 4 : 0;
  const size_t b2 = p2.splits > 1 ? (size_t)p2.splits * T * d * 4 : 0;
  l.total = l.part + align256(b1 > b2 ? b1 : b2);
  return l;
}

}  // namespace

size_t out_proj_workspace(int T, int n_h, int c, int g, int d_g, int d) {
  return out_proj_layout(T, n_h, c, g, d_g, d).total;
}

void out_proj_plan_info(int T, int n_h, int c, int g, int d_g, int d, int32_t* out) {
  const ProjPlan p1 = plan_projection(T, n_h / g * c, d_g, g), p2 = plan_projection(T, g * d_g, d, 1);
  out[0] = p1.nt;
  out[1] = p1.splits;
  out[2] = p1.tiles * p1.splits;
  out[3] = p2.nt;
  out[4] = p2.splits;
  out[5] = p2.tiles * p2.splits;
}

cudaError_t launch_out_proj(const OutProjArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const OutProjLayout l = out_proj_layout(a.T, a.n_h, a.c, a.g, a.d_g, a.d);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  __nv_bfloat16* Z = reinterpret_cast<__nv_bfloat16*>(ws + l.z);
  int* tickets = reinterpret_cast<int*>(ws + l.tickets);
  float* part = reinterpret_cast<float*>(ws + l.part);
  cudaError_t e = launch_projection(a.Wg, a.O, Z, a.T, a.n_h / a.g * a.c, a.d_g, a.g, part, tickets, s);
  if (e != cudaSuccess) return e;
  return launch_projection(a.Wo, Z, static_cast<__nv_bfloat16*>(a.Y), a.T, a.g * a.d_g, a.d, 1, part, tickets, s);
}

}  // namespace csa
