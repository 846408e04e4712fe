// norm_rope.cu -- Q / KV-entry RMSNorm and partial RoPE ("DeepSeek-V4 内部机制"
// 1.4 table; admirer.cn article, RoPE paragraph): a warp per row at a time,
// two passes over the row (sum of squares, then normalise, turn the last
// rope_dims dims and store), 16-byte loads and stores; the second read of a
// row comes from L1/L2.  Angles are formed and reduced to [-pi, pi] in fp64
// (a position of 10^6 times a frequency near 1 leaves fp32 no fractional
// bits); the sine and cosine of the reduced angle are taken in fp32.
#include "csa_internal.cuh"
#include "rope_dev.cuh"

namespace csa {
namespace {

__device__ __forceinline__ void nr_load8(const void* base, int dt, int64_t elem, float* v) {
  if (dt == CSA_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void nr_store8(void* base, int dt, int64_t elem, const float* v) {
  if (dt == CSA_F32) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + elem);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
      memcpy(&w[q], &h, 4);
    }
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(base) + elem) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Grid-stride over rows, one warp per row at a time.  A lane owns chunks
// lane, lane + 32, ... of every row, so the frequencies of its (at most
// kMaxOwn) rotated chunks are computed once, in fp64, before the row loop.
// Per pair and row: angle = p * theta in fp64, reduced to [-pi, pi] by two-
// constant Cody-Waite subtraction of the nearest multiple of 2 pi, then
// sincosf on the fp32 residual.
constexpr int kMaxOwn = 2;

__global__ void __launch_bounds__(256) norm_rope_kernel(NormRopeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int nch = a.dim / 8, d_rope = a.dim - a.rope_dims;
  double theta[kMaxOwn][4];
  int own = 0;
  for (int c = lane; c < nch && own < kMaxOwn; c += 32) {
    if (8 * c < d_rope) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) theta[own][j] = rope_theta(a.base, (8 * c - d_rope) / 2 + j, a.rope_dims);
    ++own;
  }
  const bool table = (nch - d_rope / 8 + 31) / 32 <= kMaxOwn;  // every lane's rotated chunks fit
  for (int64_t r = warp0; r < a.n_rows; r += n_warps) {
    const int64_t row = r * a.dim;
    float inv = 1.f;
    if (a.g != nullptr) {
      float ss = 0.f;
      for (int c = lane; c < nch; c += 32) {
        float v[8];
        nr_load8(a.x, a.in_dt, row + 8 * c, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) ss = fmaf(v[q], v[q], ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      inv = rms_inv(ss, a.dim, a.eps);
    }
    const double p = a.rope_dims > 0 ? (double)a.pos[r / a.rows_per_pos] * (double)a.pos_sign : 0.0;
    int slot = 0;
    for (int c = lane; c < nch; c += 32) {
      float v[8];
      nr_load8(a.x, a.in_dt, row + 8 * c, v);
      if (a.g != nullptr) {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = __fmul_rn(__fmul_rn(v[q], inv), a.g[8 * c + q]);
      }
      if (8 * c >= d_rope) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const double th = table ? theta[slot][j] : rope_theta(a.base, (8 * c - d_rope) / 2 + j, a.rope_dims);
          float sn, cs;
          rope_sincos(p, th, &sn, &cs);
          rope_turn(v[2 * j], v[2 * j + 1], cs, sn);
        }
        if (table) ++slot;
      }
      nr_store8(a.y, a.out_dt, row + 8 * c, v);
    }
  }
}

}  // namespace

cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s) {
  if (a.n_rows == 0) return cudaSuccess;
  // one wave of 8-warp blocks (rows beyond it loop), at most one block per 8 rows
  int64_t blocks = (a.n_rows + 7) / 8;
  if (blocks > 148 * 8) blocks = 148 * 8;
  norm_rope_kernel<<<(unsigned)blocks, 256, 0, s>>>(a);
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace csa
