// mqa_tc.cu -- shared-KV multi-query attention on tensor cores (mma.sync
// m16n8k16, bf16 in, fp32 accumulate) for c = 512 and head counts that are a
// multiple of 64 ("DeepSeek-V4 内部机制" 1.2 Step 2 shared-KV MQA, 1.3 HCA,
// 1.4 window branch and sink equation; yunpan.plus eq. 9).
//
// A CTA owns one query, a group of 64 heads and a contiguous range of that
// query's attended rows (split-KV).  The 64 x 512 query tile stays in shared
// memory; the rows are gathered 64 at a time (selected entries by index, HCA
// entries in order, then the window) with 16-byte cp.async into a double
// buffer.  FP8MIX rows are staged raw and expanded to bf16 in shared memory
// (value = e4m3 * block scale; RoPE dims copied).  Per chunk:
//   S = Q K^T (warp = 16 heads x 32 rows), online softmax per head across the
//   two warps that share a head block, P (bf16) through shared memory,
//   O += P V (warp = 16 heads x 256 dims, 128 fp32 accumulators per thread).
// Every row is both key and value.  Shared-memory tiles use a 16-byte-chunk
// XOR swizzle (chunk ^ row % 8) so ldmatrix row gathers are conflict free.
// With one split the CTA adds the sink and writes O.  A query whose rows are
// split over CL CTAs (decode: few queries, many rows) runs them as one thread
// block cluster: the CTAs exchange their per-head (max, sum) through
// distributed shared memory, each scales its partial o to its share of the
// final output and pushes it to the CTA that owns those heads, and the owner
// adds the CL partials in rank order and writes O.  No partial result goes
// through global memory and no second kernel runs.
#include "csa_internal.cuh"
#include "mqa_plan.cuh"

namespace csa {
namespace {

constexpr int kDim = 512;
constexpr int kHG = 64;        // heads per CTA
constexpr int kRC = 64;        // rows per chunk
constexpr int kThreads = 256;
constexpr int kRowBytes = kDim * 2;  // bf16 row in shared memory
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_u32_generic(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t swz(int row, int chunk) {  // byte offset in a [rows][1024 B] tile
  return (uint32_t)(row * kRowBytes + (((chunk & ~7) | ((chunk & 7) ^ (row & 7))) << 4));
}
__device__ __forceinline__ uint32_t swz_p(int row, int chunk) {  // [64][128 B] tile
  return (uint32_t)(row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 bytes read -> 16 zero bytes written
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ------------------------------------------------- thread block cluster (DSMEM)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address in CTA `rank`'s shared memory of the variable at local address `addr`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_dsmem(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_dsmem_v2(uint32_t addr, float x, float y) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}
// All threads of all CTAs of the cluster; orders shared-memory accesses
// (local and remote) before the barrier with those after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <bool FP8>
struct MqaTcSmem {
  static constexpr int Q = kHG * kRowBytes;                 // 64 KB
  static constexpr int KV = kRC * kRowBytes;                // 64 KB per buffer
  static constexpr int NKV = FP8 ? 1 : 2;
  static constexpr int RAW_ROW = 608;                       // FP8MIX row at c = 512
  static constexpr int RAW = FP8 ? kRC * RAW_ROW : 0;       // per raw buffer
  static constexpr int P = kHG * 128;                       // 8 KB
  static constexpr int RED = 4 * kHG * 4;
  static constexpr int STATS = 2 * kHG * 4;                 // cluster: per-head max and sum
  static constexpr int TOTAL = Q + NKV * KV + 2 * RAW + P + RED + kRC * 8 + STATS + 128;
  // cluster: the receive buffer [CL sources][64 / CL heads][512] fp32 reuses
  // the query, chunk and raw buffers once every CTA of the cluster is done
  static_assert(Q + NKV * KV + 2 * RAW >= kHG * kDim * 4, "receive buffer fits");
};

template <bool FP8, int CL>
__global__ void __launch_bounds__(kThreads, 1) mqa_tc_kernel(MqaArgs a, MqaPlan plan) {
  using S = MqaTcSmem<FP8>;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* qs = sm;
  uint8_t* kvs = qs + S::Q;                       // NKV bf16 chunk buffers
  uint8_t* raws = kvs + S::NKV * S::KV;           // FP8: two raw chunk buffers
  uint8_t* ps = raws + 2 * S::RAW;
  float* red = reinterpret_cast<float*>(ps + S::P);          // [2][64] max, [2][64] l
  const uint8_t** rowp = reinterpret_cast<const uint8_t**>(red + 4 * kHG);  // [64] row pointers
  float* st_m = reinterpret_cast<float*>(rowp + kRC);        // cluster: [64] max (log2 domain)
  float* st_l = st_m + kHG;                                   // cluster: [64] sum

  const int split = blockIdx.x, hg = blockIdx.y;
  const int64_t bt = blockIdx.z;
  const int b = (int)(bt / a.n_q);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hb = warp & 3, half = warp >> 2;
  const int g = lane >> 2, t4 = lane & 3;

  const int64_t tq = a.q_pos[bt];
  const RowList rl = make_row_list(a, bt, tq);
  // split s of CL takes chunks [s * nch / CL, (s + 1) * nch / CL) of the rows
  const int64_t nch = (rl.n_rows + kRC - 1) / kRC;
  const int64_t r_begin = (int64_t)split * nch / CL * kRC;
  const int64_t r_end = min64(rl.n_rows, ((int64_t)split + 1) * nch / CL * kRC);
  const int n_chunks = r_end > r_begin ? (int)((r_end - r_begin + kRC - 1) / kRC) : 0;
  const int64_t rb = row_bytes(a.kv_dt, kDim);

  // query tile (64 heads x 512 dims) -> swizzled shared memory
  {
    const uint8_t* qg = static_cast<const uint8_t*>(a.Q) + ((bt * a.n_heads + (int64_t)hg * kHG) * kDim) * 2;
    for (int i = threadIdx.x; i < kHG * 64; i += kThreads) {
      const int h = i >> 6, c = i & 63;
      cp_async16(smem_u32_generic(qs + swz(h, c)), qg + (int64_t)h * kRowBytes + c * 16, true);
    }
  }

  // issue the gather of chunk `ci` (row pointers resolved first)
  auto resolve_rows = [&](int ci) {
    __syncthreads();
    if (threadIdx.x < kRC) {
      const int64_t r = r_begin + (int64_t)ci * kRC + threadIdx.x;
      rowp[threadIdx.x] = r < r_end ? row_ptr(a, rl, b, r, rb) : nullptr;
    }
    __syncthreads();
  };
  auto issue_chunk = [&](int ci) {
    if (FP8) {
      uint8_t* dst = raws + (ci & 1) * S::RAW;
      for (int i = threadIdx.x; i < kRC * (S::RAW_ROW / 16); i += kThreads) {
        const int r = i / (S::RAW_ROW / 16), c = i % (S::RAW_ROW / 16);
        const uint8_t* src = rowp[r];
        cp_async16(smem_u32_generic(dst + r * S::RAW_ROW + c * 16), src ? src + c * 16 : a.Q, src != nullptr);
      }
    } else {
      uint8_t* dst = kvs + (ci & 1) * S::KV;
      for (int i = threadIdx.x; i < kRC * 64; i += kThreads) {
        const int r = i >> 6, c = i & 63;
        const uint8_t* src = rowp[r];
        cp_async16(smem_u32_generic(dst + swz(r, c)), src ? src + c * 16 : a.Q, src != nullptr);
      }
    }
    cp_async_commit();
  };

  float o[32][4];
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};  // heads g, g+8 of this warp's block (log2 domain)
  float l_run[2] = {0.f, 0.f};              // partial sums over this warp's S rows
  const float sl2 = a.scale * kLog2e;
  bool valid_row[8];                        // rows of this thread's S columns in the chunk

  if (n_chunks > 0) {
    resolve_rows(0);
    issue_chunk(0);
  } else {
    cp_async_commit();
  }

  for (int ci = 0; ci < n_chunks; ++ci) {
    cp_async_wait_all();
    __syncthreads();
    // row validity of this chunk (before the pointers are overwritten)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r0 = half * 32 + j * 8 + 2 * t4;
      valid_row[2 * j] = rowp[r0] != nullptr;
      valid_row[2 * j + 1] = rowp[r0 + 1] != nullptr;
    }
    const uint8_t* kv;
    if (FP8) {
      // expand the raw chunk to bf16 (value = e4m3 * scale; RoPE dims copied)
      const uint8_t* raw = raws + (ci & 1) * S::RAW;
      for (int i = threadIdx.x; i < kRC * 64; i += kThreads) {
        const int r = i >> 6, c = i & 63;
        const uint8_t* row = raw + r * S::RAW_ROW;
        uint4 out;
        if (c < 56) {
          const uint2 v = *reinterpret_cast<const uint2*>(row + c * 8);
          const float s = *reinterpret_cast<const float*>(row + 576 + 4 * (c >> 3));
          uint32_t w[4];
          const uint32_t src[2] = {v.x, v.y};
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float2 lo = e4m3x2_to_float2((uint16_t)(src[q] & 0xFFFF));
            const float2 hi = e4m3x2_to_float2((uint16_t)(src[q] >> 16));
            const __nv_bfloat162 x0 = __floats2bfloat162_rn(lo.x * s, lo.y * s);
            const __nv_bfloat162 x1 = __floats2bfloat162_rn(hi.x * s, hi.y * s);
            memcpy(&w[2 * q], &x0, 4);
            memcpy(&w[2 * q + 1], &x1, 4);
          }
          out = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
          out = *reinterpret_cast<const uint4*>(row + 448 + (c - 56) * 16);
        }
        *reinterpret_cast<uint4*>(kvs + swz(r, c)) = out;
      }
      kv = kvs;
    } else {
      kv = kvs + (ci & 1) * S::KV;
    }
    // prefetch the next chunk
    if (ci + 1 < n_chunks) {
      resolve_rows(ci + 1);
      issue_chunk(ci + 1);
    } else {
      __syncthreads();
    }

    // ---- S = Q K^T : 16 heads (hb) x 32 rows (half) ----
    float s[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    const uint32_t q_base = smem_u32_generic(qs), kv_base = smem_u32_generic(kv);
#pragma unroll 4
    for (int ks = 0; ks < 32; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(q_base + swz(hb * 16 + (lane & 15), 2 * ks + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
      for (int jp = 0; jp < 2; ++jp) {
        uint32_t b0, b1, b2, b3;
        const int row = half * 32 + (2 * jp + (lane >> 4)) * 8 + (lane & 7);
        ldsm_x4(kv_base + swz(row, 2 * ks + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma_bf16(s[2 * jp], a0, a1, a2, a3, b0, b1);
        mma_bf16(s[2 * jp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // ---- online softmax (log2 domain) ----
    float cmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = valid_row[2 * j + (e & 1)];
        s[j][e] = ok ? s[j][e] * sl2 : -INFINITY;
        cmax[e >> 1] = fmaxf(cmax[e >> 1], s[j][e]);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cmax[h] = fmaxf(cmax[h], __shfl_xor_sync(0xffffffffu, cmax[h], 1));
      cmax[h] = fmaxf(cmax[h], __shfl_xor_sync(0xffffffffu, cmax[h], 2));
    }
    if (t4 == 0) {
      red[half * kHG + hb * 16 + g] = cmax[0];
      red[half * kHG + hb * 16 + g + 8] = cmax[1];
    }
    __syncthreads();
    float corr[2], mnew[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int head = hb * 16 + g + 8 * h;
      const float cm = fmaxf(red[head], red[kHG + head]);
      mnew[h] = fmaxf(m_run[h], cm);
      corr[h] = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - mnew[h]);
      m_run[h] = mnew[h];
    }
    float psum[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = mnew[e >> 1];
        p[e] = (s[j][e] == -INFINITY || m == -INFINITY) ? 0.f : exp2f(s[j][e] - m);
        psum[e >> 1] += p[e];
      }
      const int col = half * 32 + j * 8 + 2 * t4;
      const __nv_bfloat162 p01 = __floats2bfloat162_rn(p[0], p[1]);
      const __nv_bfloat162 p23 = __floats2bfloat162_rn(p[2], p[3]);
      const int h0 = hb * 16 + g, h1 = h0 + 8;
      *reinterpret_cast<__nv_bfloat162*>(ps + swz_p(h0, col >> 3) + (col & 7) * 2) = p01;
      *reinterpret_cast<__nv_bfloat162*>(ps + swz_p(h1, col >> 3) + (col & 7) * 2) = p23;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 1);
      psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 2);
      l_run[h] = l_run[h] * corr[h] + psum[h];
    }
    __syncthreads();
    // ---- O = O * corr + P V : 16 heads (hb) x 256 dims (half) ----
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      o[j][0] *= corr[0]; o[j][1] *= corr[0];
      o[j][2] *= corr[1]; o[j][3] *= corr[1];
    }
    const uint32_t p_base = smem_u32_generic(ps);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(p_base + swz_p(hb * 16 + (lane & 15), 2 * kk + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < 16; ++np) {
        uint32_t b0, b1, b2, b3;
        const int row = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = half * 32 + 2 * np + (lane >> 4);
        ldsm_x4_t(kv_base + swz(row, chunk), b0, b1, b2, b3);
        mma_bf16(o[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }

  // ---- combine the two warps' row sums of each head block ----
  cp_async_wait_all();
  __syncthreads();
  if (t4 == 0) {
    red[2 * kHG + half * kHG + hb * 16 + g] = l_run[0];
    red[2 * kHG + half * kHG + hb * 16 + g + 8] = l_run[1];
  }
  __syncthreads();
  float l_tot[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int head = hb * 16 + g + 8 * h;
    l_tot[h] = red[2 * kHG + head] + red[3 * kHG + head];
  }
  const int hbase = hg * kHG + hb * 16 + g;
  if constexpr (CL == 1) {
    float f[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float sink = a.sink[hbase + 8 * h] * kLog2e;  // log2 domain
      const float M = fmaxf(m_run[h], sink);
      f[h] = 0.f;
      if (!(sink == INFINITY) && M != -INFINITY) {
        const float em = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - M);
        f[h] = em / (l_tot[h] * em + exp2f(sink - M));
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.O) + ((bt * a.n_heads + hbase + 8 * h) * kDim);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int d = half * 256 + j * 8 + 2 * t4;
        *reinterpret_cast<__nv_bfloat162*>(orow + d) =
            __floats2bfloat162_rn(o[j][2 * h] * f[h], o[j][2 * h + 1] * f[h]);
      }
    }
  } else {
    // 1. per-head (max, sum) of every CTA of the cluster
    if (half == 0 && t4 == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        st_m[hb * 16 + g + 8 * h] = m_run[h];
        st_l[hb * 16 + g + 8 * h] = l_tot[h];
      }
    }
    cluster_sync();
    // 2. the factor that turns this CTA's partial into its share of O:
    //    O = sum_s o_s 2^(m_s - M) / (sum_s l_s 2^(m_s - M) + 2^(sink - M))
    float f[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int head = hb * 16 + g + 8 * h;
      const uint32_t am = smem_u32_generic(st_m + head), al = smem_u32_generic(st_l + head);
      float ms[CL];
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < CL; ++r) {
        ms[r] = ld_dsmem(mapa_shared(am, (uint32_t)r));
        M = fmaxf(M, ms[r]);
      }
      const float sink = a.sink[hbase + 8 * h] * kLog2e;
      const float Mt = fmaxf(M, sink);
      f[h] = 0.f;
      if (!(sink == INFINITY) && Mt != -INFINITY) {
        float L = exp2f(sink - Mt);
#pragma unroll
        for (int r = 0; r < CL; ++r)
          if (ms[r] != -INFINITY) L += ld_dsmem(mapa_shared(al, (uint32_t)r)) * exp2f(ms[r] - Mt);
        f[h] = m_run[h] == -INFINITY ? 0.f : exp2f(m_run[h] - Mt) / L;
      }
    }
    // 3. push the scaled partial to the owner of its heads: CTA r owns heads
    //    [r * HPC, (r + 1) * HPC) and receives [CL sources][HPC heads][512]
    constexpr int HPC = kHG / CL;
    float* recv = reinterpret_cast<float*>(sm);
    const uint32_t rank = cluster_ctarank();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int head = hb * 16 + g + 8 * h;
      const uint32_t owner = (uint32_t)(head / HPC);
      const uint32_t dst =
          mapa_shared(smem_u32_generic(recv + ((int)rank * HPC + head % HPC) * kDim), owner);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int d = half * 256 + j * 8 + 2 * t4;
        st_dsmem_v2(dst + 4u * (uint32_t)d, o[j][2 * h] * f[h], o[j][2 * h + 1] * f[h]);
      }
    }
    cluster_sync();
    // 4. add the CL partials of the owned heads in rank order and write O
    for (int i = threadIdx.x; i < HPC * kDim / 2; i += kThreads) {
      const int hl = i / (kDim / 2), d = 2 * (i % (kDim / 2));
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int r = 0; r < CL; ++r) {
        const float2 v = *reinterpret_cast<const float2*>(recv + (r * HPC + hl) * kDim + d);
        x += v.x;
        y += v.y;
      }
      __nv_bfloat16* orow =
          static_cast<__nv_bfloat16*>(a.O) + ((bt * a.n_heads + hg * kHG + (int)rank * HPC + hl) * kDim);
      *reinterpret_cast<__nv_bfloat162*>(orow + d) = __floats2bfloat162_rn(x, y);
    }
  }
}

}  // namespace

bool mqa_tc_eligible(const MqaArgs& a) {
  return a.q_dt == CSA_BF16 && (a.kv_dt == CSA_BF16 || a.kv_dt == CSA_KV_FP8MIX) && a.dim == kDim &&
         a.n_heads % kHG == 0 && (int64_t)a.batch * a.n_q <= 65535;
}

MqaPlan make_tc_mqa_plan(const MqaArgs& a) {
  MqaPlan p{};
  p.heads_per_cta = kHG;
  // rows of one query are split over a cluster of CL CTAs (a power of two up
  // to the portable cluster size 8) while the grid stays within one wave
  const int64_t units = (int64_t)a.batch * a.n_q * (a.n_heads / kHG);
  const int64_t nch = (max_rows_per_query(a) + kRC - 1) / kRC;
  int cl = 1;
  while (cl < 8 && units * cl * 2 <= 148 && cl * 2 <= nch) cl *= 2;
  p.n_splits = cl;
  p.cluster = 1;
  p.rows_per_split = 0;
  return p;
}

template <bool FP8, int CL>
cudaError_t launch_tc(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  const size_t smem = MqaTcSmem<FP8>::TOTAL;
  cudaError_t e = cudaFuncSetAttribute(mqa_tc_kernel<FP8, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, a.n_heads / kHG, (unsigned)((int64_t)a.batch * a.n_q));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = CL > 1 ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, mqa_tc_kernel<FP8, CL>, a, p);
  ++launch_counter();
  return e;
}

template <bool FP8>
cudaError_t launch_tc_fmt(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  switch (p.n_splits) {
    case 1: return launch_tc<FP8, 1>(a, p, s);
    case 2: return launch_tc<FP8, 2>(a, p, s);
    case 4: return launch_tc<FP8, 4>(a, p, s);
    case 8: return launch_tc<FP8, 8>(a, p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_mqa_tc(const MqaArgs& a, const MqaPlan& p, cudaStream_t s) {
  return a.kv_dt == CSA_KV_FP8MIX ? launch_tc_fmt<true>(a, p, s) : launch_tc_fmt<false>(a, p, s);
}

}  // namespace csa
