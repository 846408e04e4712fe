// compress.cu -- Token-Level Compressor ("DeepSeek-V4 内部机制" 1.2 Step 1 and
// 1.3; yunpan.plus write-up eq. 6-7 and 10-11).
//
// Prefill form: one thread owns one (request, entry, 8-channel chunk) and
// streams the entry's 2m (CSA) or m' (HCA) token rows of its chunk with
// 16-byte loads: a pass over Z and the biases for the max logit, then a pass
// over Z, C and the biases for the weighted sums (the second read of Z and
// the biases normally comes from L1/L2).  Lanes that share an FP8
// scale block (8 lanes = 64 dims) or an FP4 block (2 lanes = 16 dims) reduce
// their amax with warp shuffles and quantise in the epilogue.
#include "compress_dev.cuh"
#include "rope_dev.cuh"
#include "sm100.cuh"

namespace csa {

CSA_DEFINE_STATUS_READER(take_status_compress)

namespace {

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
  const int U = (a.Cb != nullptr && i >= 1) ? 2 * a.m : a.m;
  const int64_t in_base = (int64_t)b * a.in_batch_stride;
  // Positions are taken kTB at a time and all their loads are issued before
  // any is used, so a thread waits one memory latency per batch rather than
  // per position.  The second pass reads Z and the biases again (from L1/L2).
  constexpr int kTB = 4;
  auto load_pos = [&](int u, bool with_c, float* z, float* c, float* bias) {
    const bool cur = u < a.m;
    const int64_t tok = cur ? (int64_t)a.m * i + u : (int64_t)a.m * (i - 1) + (u - a.m);
    const int64_t off = (in_base + tok - a.tok0) * a.dim + d0;
    load8(cur ? a.Za : a.Zb, a.in_dt, off, z);
    if (with_c) load8(cur ? a.Ca : a.Cb, a.in_dt, off, c);
    const float4* bp = reinterpret_cast<const float4*>(
        (cur ? a.Ba + (int64_t)u * a.dim : a.Bb + (int64_t)(u - a.m) * a.dim) + d0);
    const float4 b0 = __ldg(bp), b1 = __ldg(bp + 1);
    bias[0] = b0.x; bias[1] = b0.y; bias[2] = b0.z; bias[3] = b0.w;
    bias[4] = b1.x; bias[5] = b1.y; bias[6] = b1.z; bias[7] = b1.w;
  };
  float M[8], D[8], S[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) { M[q] = -INFINITY; D[q] = 0.f; S[q] = 0.f; }
  if (valid) {
    for (int u0 = 0; u0 < U; u0 += kTB) {  // pass 1: the max logit
      float z[kTB][8], c[kTB][8], bias[kTB][8];
#pragma unroll
      for (int r = 0; r < kTB; ++r)
        if (u0 + r < U) load_pos(u0 + r, false, z[r], c[r], bias[r]);
#pragma unroll
      for (int r = 0; r < kTB; ++r)
        if (u0 + r < U) {
#pragma unroll
          for (int q = 0; q < 8; ++q) M[q] = fmaxf(M[q], z[r][q] + bias[r][q]);
        }
    }
    for (int blk = 0; blk < U; blk += kPosBlock) {  // pass 2: block sums in order
      const int end = min(U, blk + kPosBlock);
      float d[8], s[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) { d[q] = 0.f; s[q] = 0.f; }
      for (int u0 = blk; u0 < end; u0 += kTB) {
        float z[kTB][8], c[kTB][8], bias[kTB][8];
#pragma unroll
        for (int r = 0; r < kTB; ++r)
          if (u0 + r < end) load_pos(u0 + r, true, z[r], c[r], bias[r]);
#pragma unroll
        for (int r = 0; r < kTB; ++r)
          if (u0 + r < end) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float e = expf((z[r][q] + bias[r][q]) - M[q]);
              d[q] += e;
              s[q] = fmaf(e, c[r][q], s[q]);
            }
          }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) { D[q] += d[q]; S[q] += s[q]; }
    }
  }
  float x[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) x[q] = valid ? pooled_value(D[q], S[q]) : 0.f;

  store_entry(a, b, ie, d0, x, valid);
}

__global__ void __launch_bounds__(256) compress_tokpar_kernel(CompressArgs a) {
  extern __shared__ __align__(16) uint8_t tsm[];
  const int n_cg = (a.dim + kTpW - 1) / kTpW;
  const bool rowm = compress_row_epilogue(a);
  const int64_t ie = rowm ? (int64_t)blockIdx.x : (int64_t)(blockIdx.x / n_cg);
  const int cg_lo = rowm ? 0 : (int)(blockIdx.x % n_cg), cg_hi = rowm ? n_cg : cg_lo + 1;
  tokpar_entry(a, (int)blockIdx.y, ie, cg_lo, cg_hi, tsm);
}

}  // namespace

cudaError_t launch_compress(const CompressArgs& a, cudaStream_t s) {
  const int64_t total = (int64_t)a.batch * a.n_out * (a.dim / 8);
  if (total == 0) return cudaSuccess;
  // thread per (entry, 8 channels) when the entries alone fill the GPU and
  // each has few tokens; otherwise the token-parallel form
  const bool rowm = compress_row_epilogue(a);  // normalisation / RoPE: a CTA per entry
  const int64_t tokpar_blocks = rowm ? a.n_out : (int64_t)((a.dim + 63) / 64) * a.n_out;
  if (!rowm && ((total >= 148 * 512 && a.m <= 8) || a.batch > 65535 || tokpar_blocks >= ((int64_t)1 << 31))) {
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    compress_kernel<<<(unsigned)blocks, threads, 0, s>>>(a);
  } else {
    dim3 grid((unsigned)tokpar_blocks, (unsigned)a.batch);
    const int smem = tokpar_smem_bytes(a);
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(compress_tokpar_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
    }
    compress_tokpar_kernel<<<grid, 256, smem, s>>>(a);
  }
  ++launch_counter();
  return cudaGetLastError();
}

}  // namespace csa
