// compress.cu -- Token-Level Compressor ("DeepSeek-V4 内部机制" 1.2 Step 1 and
// 1.3; yunpan.plus write-up eq. 6-7 and 10-11).
//
// One thread owns one (request, entry, 8-channel chunk).  It streams the 2m
// (CSA) or m' (HCA) token rows of its chunk once with 16-byte loads and keeps
// an online softmax per channel in fp32, so every input byte is read exactly
// once: the kernel is bound by HBM reads of C and Z.  Lanes that share an FP8
// scale block (8 lanes = 64 dims) or an FP4 block (2 lanes = 16 dims) reduce
// their amax with warp shuffles and quantise in the epilogue.
#include "csa_internal.cuh"

namespace csa {
namespace {

__device__ __forceinline__ void load8(const void* base, int dt, int64_t elem, float* v) {
  if (dt == CSA_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem));
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}

struct OnlineSoftmax8 {
  float mx[8], den[8], acc[8];
  __device__ void init() {
#pragma unroll
    for (int j = 0; j < 8; ++j) { mx[j] = -INFINITY; den[j] = 0.f; acc[j] = 0.f; }
  }
  __device__ void add(const float* logit, const float* val) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (logit[j] > mx[j]) {
        float r = expf(mx[j] - logit[j]);  // 0 on the first token
        den[j] = den[j] * r + 1.f;
        acc[j] = acc[j] * r + val[j];
        mx[j] = logit[j];
      } else {
        float e = expf(logit[j] - mx[j]);
        den[j] += e;
        acc[j] = fmaf(e, val[j], acc[j]);
      }
    }
  }
};

// Writes channels d0 .. d0+7 of entry e0 + ie of request b in the output
// format.  Called by whole warps: the 8 lanes of a 64-dim FP8 scale block (2
// lanes of a 16-dim FP4 block) are consecutive and reduce their amax with
// shuffles; lanes with valid == false take part in the shuffles only.
__device__ __forceinline__ void store_entry(const CompressArgs& a, int b, int64_t ie, int d0, const float* x,
                                            bool valid) {
  const int64_t orow = (int64_t)b * a.out_batch_stride + a.out_row0 + ie;
  const int64_t rb = row_bytes(a.out_dt, a.dim);
  uint8_t* row = static_cast<uint8_t*>(a.out) + orow * rb;

  if (a.out_dt == CSA_F32) {
    if (valid) {
      float4* p = reinterpret_cast<float4*>(row + 4 * d0);
      p[0] = make_float4(x[0], x[1], x[2], x[3]);
      p[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
  } else if (a.out_dt == CSA_BF16) {
    if (valid) {
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
        memcpy(&w[q], &h, 4);
      }
      *reinterpret_cast<uint4*>(row + 2 * d0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else if (a.out_dt == CSA_KV_FP8MIX) {
    const int n8 = a.dim - kRopeDims;
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(x[q]));
    // 8 consecutive lanes hold one 64-dim scale block
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    if (valid) {
      if (d0 < n8) {
        const float scale = amax > 0.f ? amax / 448.f : 1.f;
        uint32_t w[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
              make_float2(x[4 * q] / scale, x[4 * q + 1] / scale), __NV_SATFINITE, __NV_E4M3);
          __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
              make_float2(x[4 * q + 2] / scale, x[4 * q + 3] / scale), __NV_SATFINITE, __NV_E4M3);
          w[q] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
        *reinterpret_cast<uint2*>(row + d0) = make_uint2(w[0], w[1]);
        if ((d0 % kFp8Block) == 0)
          *reinterpret_cast<float*>(row + n8 + 2 * kRopeDims + 4 * (d0 / kFp8Block)) = scale;
      } else {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
          memcpy(&w[q], &h, 4);
        }
        *reinterpret_cast<uint4*>(row + n8 + 2 * (d0 - n8)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (d0 == 0) {
        for (int64_t p = n8 + 2 * kRopeDims + 4 * (n8 / kFp8Block); p < rb; ++p) row[p] = 0;
      }
    }
  } else {  // CSA_IDX_NVFP4
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(x[q]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // 2 lanes = 16 values
    if (valid) {
      const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(amax / 6.f, __NV_SATFINITE, __NV_E4M3);
      const float s = e4m3_to_float((uint8_t)s8);
      uint32_t packed = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_fp4x2_storage_t p2 = 0;
        if (s > 0.f)
          p2 = __nv_cvt_float2_to_fp4x2(make_float2(x[2 * q] / s, x[2 * q + 1] / s), __NV_E2M1,
                                        cudaRoundNearest);
        packed |= ((uint32_t)p2) << (8 * q);
      }
      *reinterpret_cast<uint32_t*>(row + d0 / 2) = packed;
      if ((d0 % kFp4Block) == 0) {
        // key-cache scales live in the blocked scale-factor atom layout
        const int j = d0 / kFp4Block;
        const int64_t off = (int64_t)b * nvfp4_blocked_sf_bytes(a.out_batch_stride, a.dim) +
                            nvfp4_blocked_sf_offset(a.out_row0 + ie, a.dim) + (j / 4) * 512 + (j % 4);
        static_cast<uint8_t*>(a.out_sf)[off] = (uint8_t)s8;
      }
    }
  }
}

__global__ void __launch_bounds__(256) compress_kernel(CompressArgs a) {
  const int chunks = a.dim / 8;
  const int64_t total = (int64_t)a.batch * a.n_out * chunks;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const bool valid = gid < total;
  const int64_t g = valid ? gid : 0;
  const int ch = (int)(g % chunks);
  const int64_t ie = (g / chunks) % a.n_out;
  const int b = (int)(g / chunks / a.n_out);
  const int64_t i = a.e0 + ie;
  const int d0 = ch * 8;

  OnlineSoftmax8 sm;
  sm.init();
  const int64_t in_base = (int64_t)b * a.in_batch_stride;
  // One branch: tokens tok_first .. tok_first+m-1 with biases B[0..m).  Tokens
  // are taken kTB at a time and all their loads are issued before any is used,
  // so a thread waits one memory latency per batch rather than per token.
  auto branch = [&](const void* C, const void* Z, const float* Bias, int64_t tok_first) {
    constexpr int kTB = 4;
    for (int j0 = 0; j0 < a.m; j0 += kTB) {
      float z[kTB][8], c[kTB][8], bias[kTB][8];
#pragma unroll
      for (int u = 0; u < kTB; ++u) {
        if (j0 + u < a.m) {
          const int64_t off = (in_base + tok_first + j0 + u - a.tok0) * a.dim + d0;
          load8(Z, a.in_dt, off, z[u]);
          load8(C, a.in_dt, off, c[u]);
          const float4* bp = reinterpret_cast<const float4*>(Bias + (int64_t)(j0 + u) * a.dim + d0);
          const float4 b0 = __ldg(bp), b1 = __ldg(bp + 1);
          bias[u][0] = b0.x; bias[u][1] = b0.y; bias[u][2] = b0.z; bias[u][3] = b0.w;
          bias[u][4] = b1.x; bias[u][5] = b1.y; bias[u][6] = b1.z; bias[u][7] = b1.w;
        }
      }
#pragma unroll
      for (int u = 0; u < kTB; ++u) {
        if (j0 + u < a.m) {
          float logit[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) logit[q] = z[u][q] + bias[u][q];
          sm.add(logit, c[u]);
        }
      }
    }
  };
  if (valid) {
    branch(a.Ca, a.Za, a.Ba, a.m * i);                                       // current group
    if (a.Cb != nullptr && i >= 1) branch(a.Cb, a.Zb, a.Bb, a.m * (i - 1));  // previous group (CSA)
  }
  float x[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) x[q] = valid ? sm.acc[q] / sm.den[q] : 0.f;

  store_entry(a, b, ie, d0, x, valid);
}

// Merges the softmax state `o` (another set of token positions) into `s`.
__device__ __forceinline__ void merge_state(float& mx, float& den, float& acc, float mx2, float den2, float acc2) {
  if (mx2 == -INFINITY) return;
  if (mx == -INFINITY) {
    mx = mx2;
    den = den2;
    acc = acc2;
    return;
  }
  const float M = fmaxf(mx, mx2);
  const float r1 = expf(mx - M), r2 = expf(mx2 - M);
  den = den * r1 + den2 * r2;
  acc = acc * r1 + acc2 * r2;
  mx = M;
}

// Token-parallel form for few entries with many tokens each (decode; HCA's
// m' = 128): a CTA owns one entry and 64 channels; thread t takes channels
// 8 * (t % 8) .. +7 of the group and every 32nd token position of the entry
// starting at t / 8, so one warp reads 4 token rows x 128 contiguous bytes.
// The 32 partial softmax states of each channel are merged in token-lane
// order (deterministic), and warp 0 writes the entry.
constexpr int kTokLanes = 32;

__global__ void __launch_bounds__(256) compress_tokpar_kernel(CompressArgs a) {
  __shared__ float st[3][kTokLanes][64];
  __shared__ float xs[64];
  const int n_cg = (a.dim + 63) / 64;
  const int cg = (int)(blockIdx.x % n_cg), b = blockIdx.y;
  const int64_t ie = blockIdx.x / n_cg, i = a.e0 + ie;
  const int cl = threadIdx.x & 7, tl = threadIdx.x >> 3;
  const int d0 = cg * 64 + cl * 8;
  const bool ch_ok = d0 < a.dim;
  const bool two = a.Cb != nullptr && i >= 1;
  const int U = two ? 2 * a.m : a.m;  // token positions: current group, then previous group
  const int64_t in_base = (int64_t)b * a.in_batch_stride;

  OnlineSoftmax8 sm;
  sm.init();
  constexpr int kTB = 4;
  for (int u0 = tl; u0 < U; u0 += kTB * kTokLanes) {
    float z[kTB][8], c[kTB][8], bias[kTB][8];
#pragma unroll
    for (int r = 0; r < kTB; ++r) {
      const int u = u0 + r * kTokLanes;
      if (ch_ok && u < U) {
        const bool cur = u < a.m;
        const int j = cur ? u : u - a.m;
        const int64_t tok = cur ? (int64_t)a.m * i + j : (int64_t)a.m * (i - 1) + j;
        const int64_t off = (in_base + tok - a.tok0) * a.dim + d0;
        load8(cur ? a.Za : a.Zb, a.in_dt, off, z[r]);
        load8(cur ? a.Ca : a.Cb, a.in_dt, off, c[r]);
        const float4* bp = reinterpret_cast<const float4*>((cur ? a.Ba : a.Bb) + (int64_t)j * a.dim + d0);
        const float4 b0 = __ldg(bp), b1 = __ldg(bp + 1);
        bias[r][0] = b0.x; bias[r][1] = b0.y; bias[r][2] = b0.z; bias[r][3] = b0.w;
        bias[r][4] = b1.x; bias[r][5] = b1.y; bias[r][6] = b1.z; bias[r][7] = b1.w;
      }
    }
#pragma unroll
    for (int r = 0; r < kTB; ++r) {
      if (ch_ok && u0 + r * kTokLanes < U) {
        float logit[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) logit[q] = z[r][q] + bias[r][q];
        sm.add(logit, c[r]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    st[0][tl][cl * 8 + q] = sm.mx[q];
    st[1][tl][cl * 8 + q] = sm.den[q];
    st[2][tl][cl * 8 + q] = sm.acc[q];
  }
  __syncthreads();
  if (threadIdx.x < 64) {
    const int ch = threadIdx.x;
    float mx = st[0][0][ch], den = st[1][0][ch], acc = st[2][0][ch];
    const int used = U < kTokLanes ? U : kTokLanes;  // lanes that saw a token
    for (int l = 1; l < used; ++l) merge_state(mx, den, acc, st[0][l][ch], st[1][l][ch], st[2][l][ch]);
    xs[ch] = den > 0.f ? acc / den : 0.f;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int dl = cg * 64 + (lane & 7) * 8;
    const bool valid = lane < 8 && dl < a.dim;
    float x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = valid ? xs[(lane & 7) * 8 + q] : 0.f;
    store_entry(a, b, ie, dl, x, valid);
  }
}

}  // namespace

cudaError_t launch_compress(const CompressArgs& a, cudaStream_t s) {
  const int64_t total = (int64_t)a.batch * a.n_out * (a.dim / 8);
  if (total == 0) return cudaSuccess;
  // thread per (entry, 8 channels) when the entries alone fill the GPU and
  // each has few tokens; otherwise the token-parallel form
  const int64_t tokpar_blocks = (int64_t)((a.dim + 63) / 64) * a.n_out;
  if ((total >= 148 * 512 && a.m <= 8) || a.batch > 65535 || tokpar_blocks >= ((int64_t)1 << 31)) {
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    compress_kernel<<<(unsigned)blocks, threads, 0, s>>>(a);
  } else {
    dim3 grid((unsigned)tokpar_blocks, (unsigned)a.batch);
    compress_tokpar_kernel<<<grid, 256, 0, s>>>(a);
  }
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace csa
