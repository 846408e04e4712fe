// norm_rope.cu -- Q / KV-entry RMSNorm and partial RoPE ("DeepSeek-V4 内部机制"
// 1.4 table; admirer.cn article, RoPE paragraph): one warp per row, two passes
// over the row (sum of squares, then normalise, turn the last rope_dims dims
// and store), 16-byte loads and stores.  The row is read twice; the second
// read comes from L1/L2.  Angles are formed and reduced in fp64 (a position
// of 10^6 times a frequency near 1 leaves fp32 no fractional bits).
#include "csa_internal.cuh"

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

__global__ void __launch_bounds__(256) norm_rope_kernel(NormRopeArgs a) {
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= a.n_rows) return;  // a whole warp per row: the warp leaves together
  const int nch = a.dim / 8;
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
    inv = 1.f / sqrtf(ss / (float)a.dim + a.eps);
  }
  const int d_rope = a.dim - a.rope_dims;
  const double p = a.rope_dims > 0 ? (double)a.pos[r / a.rows_per_pos] * (double)a.pos_sign : 0.0;
  for (int c = lane; c < nch; c += 32) {
    float v[8];
    nr_load8(a.x, a.in_dt, row + 8 * c, v);
    if (a.g != nullptr) {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = v[q] * inv * a.g[8 * c + q];
    }
    if (8 * c >= d_rope) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = (8 * c - d_rope) / 2 + j;
        double sd, cd;
        sincos(p * pow(a.base, -2.0 * k / a.rope_dims), &sd, &cd);
        const float cs = (float)cd, sn = (float)sd, x0 = v[2 * j], x1 = v[2 * j + 1];
        v[2 * j] = x0 * cs - x1 * sn;
        v[2 * j + 1] = x0 * sn + x1 * cs;
      }
    }
    nr_store8(a.y, a.out_dt, row + 8 * c, v);
  }
}

}  // namespace

cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s) {
  if (a.n_rows == 0) return cudaSuccess;
  const int64_t blocks = (a.n_rows * 32 + 255) / 256;
  norm_rope_kernel<<<(unsigned)blocks, 256, 0, s>>>(a);
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace csa
