// rope_dev.cuh -- partial RoPE arithmetic shared by the standalone
// normalisation kernel and the attention kernel's query prologue / output
// epilogue ("DeepSeek-V4 内部机制" 1.4 table: RoPE on the last 64 dims of q,
// of the KV rows and of the output, the output at position -i).  Both callers
// take the same steps, so a query rotated inside the attention kernel has the
// bytes csa_rmsnorm_rope would give it.
#pragma once

#include <stdint.h>

namespace csa {

// Frequency of pair k of a RoPE block of rope_dims dims: base^(-2k/rope_dims).
__device__ __forceinline__ double rope_theta(double base, int k, int rope_dims) {
  return pow(base, -2.0 * k / rope_dims);
}

// sin and cos of the angle p * theta: the angle is formed in fp64 and reduced
// to [-pi, pi] by subtracting the nearest multiple of 2 pi in two parts
// (Cody-Waite: 2 pi = hi + lo, hi exact in fp64), so positions near 10^6 keep
// their fractional turns; the sine and cosine of the fp32 residual are taken
// in fp32.
__device__ __forceinline__ void rope_sincos(double p, double theta, float* sn, float* cs) {
  constexpr double kTwoPiHi = 6.283185307179586232, kTwoPiLo = 2.4492935982947064e-16,
                   kInvTwoPi = 0.15915494309189535;
  const double ang = p * theta;
  const double n = rint(ang * kInvTwoPi);
  const float red = (float)fma(-n, kTwoPiLo, fma(-n, kTwoPiHi, ang));
  sincosf(red, sn, cs);
}

// RMSNorm factor 1 / sqrt(ss / dim + eps) of a row whose squares sum to ss,
// every step rounded once in fp32.
__device__ __forceinline__ float rms_inv(float ss, int dim, float eps) {
  return __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)dim), eps)));
}

// (x0 + i x1) * (cs + i sn), each product and sum rounded once in fp32.
__device__ __forceinline__ void rope_turn(float& x0, float& x1, float cs, float sn) {
  const float a = x0, b = x1;
  x0 = __fsub_rn(__fmul_rn(a, cs), __fmul_rn(b, sn));
  x1 = __fadd_rn(__fmul_rn(a, sn), __fmul_rn(b, cs));
}

// One warp normalises (g != nullptr) and turns the last rope_dims dims of an
// fp32 row x[dim] in shared memory, in place, at position p, with the
// standalone kernel's arithmetic: lane L sums the squares of chunks L, L+32,
// ... (8 values each, fused multiply-adds in order), the xor-shuffle tree adds
// the lanes, every value is multiplied by inv and then by g, and the pairs are
// turned as rope_turn does.  The row is then the fp32 row csa_rmsnorm_rope
// would write for the same input.  dim is a multiple of 8.
__device__ __forceinline__ void warp_norm_rope_row(float* x, int dim, const float* g, float eps, int rope_dims,
                                                   double base, double p, int lane) {
  const int nch = dim / 8, d_rope = dim - rope_dims;
  float inv = 1.f;
  if (g != nullptr) {
    float ss = 0.f;
    for (int c = lane; c < nch; c += 32)
#pragma unroll
      for (int q = 0; q < 8; ++q) ss = fmaf(x[8 * c + q], x[8 * c + q], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    inv = rms_inv(ss, dim, eps);
  }
  for (int c = lane; c < nch; c += 32) {
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = x[8 * c + q];
    if (g != nullptr) {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = __fmul_rn(__fmul_rn(v[q], inv), g[8 * c + q]);
    }
    if (8 * c >= d_rope) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float sn, cs;
        rope_sincos(p, rope_theta(base, (8 * c - d_rope) / 2 + j, rope_dims), &sn, &cs);
        rope_turn(v[2 * j], v[2 * j + 1], cs, sn);
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) x[8 * c + q] = v[q];
  }
  __syncwarp();
}

}  // namespace csa
