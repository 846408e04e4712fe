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

// Token-parallel form for few entries with many positions each (decode; HCA's
// m' = 128): a CTA owns one entry and 64 channels.  Its 256 threads stage the
// entry's rows of those channels (up to kTpChunk positions at a time) into
// shared memory with cp.async; thread (w, k) then takes channel w and the
// position blocks k, k+4, ... of each chunk.  The block sums are added in
// block order by the k = 0 thread, and warp 0 writes the entry.
constexpr int kTpW = 64;
constexpr int kTpChunk = 128;

__host__ __device__ __forceinline__ int tokpar_smem_bytes(const CompressArgs& a) {
  const int esz = a.in_dt == CSA_F32 ? 4 : 2;
  const int U = staged_positions(a);
  const int P = U < kTpChunk ? U : kTpChunk;
  const int xs = compress_row_epilogue(a) ? a.dim : kTpW;
  return P * kTpW * (2 * esz + 4) + 3 * 4 * kTpW * 4 + xs * 4;
}

__global__ void __launch_bounds__(256) compress_tokpar_kernel(CompressArgs a) {
  extern __shared__ __align__(16) uint8_t tsm[];
  const int esz = a.in_dt == CSA_F32 ? 4 : 2;
  const int n_cg = (a.dim + kTpW - 1) / kTpW;
  // row mode (normalisation / RoPE epilogue): the CTA owns every channel
  // group of its entry, so the whole pooled row is in shared memory at the end
  const bool rowm = compress_row_epilogue(a);
  const int b = blockIdx.y;
  const int64_t ie = rowm ? (int64_t)blockIdx.x : (int64_t)(blockIdx.x / n_cg), i = a.e0 + ie;
  const int cg_lo = rowm ? 0 : (int)(blockIdx.x % n_cg), cg_hi = rowm ? n_cg : cg_lo + 1;
  const int U = (a.Cb != nullptr && i >= 1) ? 2 * a.m : a.m;
  const int Pmax = min(staged_positions(a), kTpChunk);
  const int P = min(U, kTpChunk);
  const int n_chunks = (U + P - 1) / P;
  uint8_t* zs = tsm;
  uint8_t* cs = zs + (size_t)Pmax * kTpW * esz;
  float* bs = reinterpret_cast<float*>(cs + (size_t)Pmax * kTpW * esz);
  float* rmax = bs + (size_t)Pmax * kTpW;  // [4][64]
  float* rd = rmax + 4 * kTpW;             // [4][64]
  float* rs = rd + 4 * kTpW;               // [4][64]
  float* xs = rs + 4 * kTpW;               // [64], or [dim] in row mode
  const int w = threadIdx.x % kTpW, k = threadIdx.x / kTpW;
  const int64_t in_base = (int64_t)b * a.in_batch_stride;

  for (int cg = cg_lo; cg < cg_hi; ++cg) {
    const int c0 = cg * kTpW, W = min(kTpW, a.dim - c0);
    const bool ch_ok = w < W;
    if (cg > cg_lo) __syncthreads();  // the previous group's staged rows are no longer read

    // positions [u0, u0 + n) of the CTA's channels into shared memory
    auto stage = [&](int u0, int n, bool with_c) {
      const int p16 = W * esz / 16;
      for (int q = threadIdx.x; q < n * p16; q += blockDim.x) {
        const int r = q / p16, p = q % p16, u = u0 + r;
        const bool cur = u < a.m;
        const int64_t tok = cur ? (int64_t)a.m * i + u : (int64_t)a.m * (i - 1) + (u - a.m);
        const int64_t off = ((in_base + tok - a.tok0) * a.dim + c0) * esz + (int64_t)p * 16;
        stage_cp16(zs + (size_t)r * kTpW * esz + p * 16, static_cast<const uint8_t*>(cur ? a.Za : a.Zb) + off);
        if (with_c)
          stage_cp16(cs + (size_t)r * kTpW * esz + p * 16, static_cast<const uint8_t*>(cur ? a.Ca : a.Cb) + off);
      }
      const int b16 = W * 4 / 16;
      for (int q = threadIdx.x; q < n * b16; q += blockDim.x) {
        const int r = q / b16, p = q % b16, u = u0 + r;
        const float* src = (u < a.m ? a.Ba + (int64_t)u * a.dim : a.Bb + (int64_t)(u - a.m) * a.dim) + c0;
        stage_cp16(reinterpret_cast<uint8_t*>(bs + (size_t)r * kTpW) + p * 16,
                   reinterpret_cast<const uint8_t*>(src) + p * 16);
      }
      asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
      __syncthreads();
    };

    float M = -INFINITY;  // pass 1: the max logit
    for (int u0 = 0; u0 < U; u0 += P) {
      const int n = min(P, U - u0);
      if (u0 > 0) __syncthreads();
      stage(u0, n, n_chunks == 1);
      if (ch_ok)
        for (int blk = k; blk * kPosBlock < n; blk += 4)
          M = chan_max(zs + ((size_t)blk * kPosBlock * kTpW + w) * esz, bs + (size_t)blk * kPosBlock * kTpW + w,
                       a.in_dt, kTpW, min(kPosBlock, n - blk * kPosBlock), M);
    }
    rmax[k * kTpW + w] = M;
    __syncthreads();
    M = fmaxf(fmaxf(rmax[w], rmax[kTpW + w]), fmaxf(rmax[2 * kTpW + w], rmax[3 * kTpW + w]));

    float D = 0.f, S = 0.f;  // pass 2: block sums, added in block order
    for (int u0 = 0; u0 < U; u0 += P) {
      const int n = min(P, U - u0);
      if (n_chunks > 1) {
        __syncthreads();
        stage(u0, n, true);
      }
      const int nb = (n + kPosBlock - 1) / kPosBlock;  // <= 4
      float d = 0.f, s = 0.f;
      if (ch_ok && k < nb)
        chan_block(zs + ((size_t)k * kPosBlock * kTpW + w) * esz, cs + ((size_t)k * kPosBlock * kTpW + w) * esz,
                   bs + (size_t)k * kPosBlock * kTpW + w, a.in_dt, kTpW, min(kPosBlock, n - k * kPosBlock), M, d,
                   s);
      rd[k * kTpW + w] = d;
      rs[k * kTpW + w] = s;
      __syncthreads();
      if (k == 0)
        for (int q = 0; q < nb; ++q) {
          D += rd[q * kTpW + w];
          S += rs[q * kTpW + w];
        }
    }
    if (k == 0 && ch_ok) xs[(rowm ? c0 : 0) + w] = pooled_value(D, S);
  }
  __syncthreads();
  if (rowm) {
    // normalise and turn the pooled row, then 8 warps store it
    if (threadIdx.x < 32)
      warp_norm_rope_row(xs, a.dim, a.norm_g, a.norm_eps, a.rope_dims, a.rope_base,
                         (double)(a.pos_stride * i + a.pos_offset), threadIdx.x);
    __syncthreads();
    const int nch = a.dim / 8;
    for (int q0 = 0; q0 < nch; q0 += blockDim.x) {
      const int ch = q0 + threadIdx.x;
      const bool valid = ch < nch;
      float x[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) x[q] = valid ? xs[ch * 8 + q] : 0.f;
      store_entry(a, b, ie, valid ? ch * 8 : 0, x, valid);
    }
    return;
  }
  if (threadIdx.x < 32) {
    const int c0 = cg_lo * kTpW;
    const int lane = threadIdx.x;
    const int dl = c0 + (lane & 7) * 8;
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
