// compress_dev.cuh -- device pieces of the Token-Level Compressor
// ("DeepSeek-V4 内部机制" 1.2 Step 1 and 1.3; yunpan.plus write-up eq. 6-7 and
// 10-11) shared by the compressor kernels and by the indexer kernels that
// compress a decode step's new index key before streaming the cache.
#pragma once

#include "csa_internal.cuh"
#include "sm100.cuh"
#include "rope_dev.cuh"

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

// Writes channels d0 .. d0+7 of entry e0 + ie of request b in the output
// format.  Called by whole warps: the 8 lanes of a 64-dim FP8 scale block (2
// lanes of a 16-dim FP4 block) are consecutive and reduce their amax with
// shuffles; lanes with valid == false take part in the shuffles only.
__device__ __forceinline__ void store_entry(const CompressArgs& a, int b, int64_t ie, int d0, const float* x,
                                            bool valid) {
  const bool paged = a.out_pages.table != nullptr;
  const int64_t lr = a.out_row0 + ie;  // logical row of the entry in request b's cache
  int64_t orow = (int64_t)b * a.out_batch_stride + lr;
  if (paged) {
    orow = pool_row(a.out_pages, b, lr);
    if (orow < 0) {
      if (valid) flag_status(kStatusBadPage);
      valid = false;  // the lanes still take part in the scale shuffles
      orow = 0;
    }
  }
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
        int64_t off = (int64_t)b * nvfp4_blocked_sf_bytes(a.out_batch_stride, a.dim) +
                      nvfp4_blocked_sf_offset(lr, a.dim);
        if (paged) {
          // the page's block (one 128-row block per pool page); the page
          // holding the codes was in the pool, so is this one unless the
          // table is inconsistent
          const int64_t pg = pool_sf_page(a.out_pages, b, lr);
          off = pg < 0 ? -1 : pg * nvfp4_blocked_sf_bytes(128, a.dim) + nvfp4_blocked_sf_offset(lr % 128, a.dim);
          if (pg < 0) flag_status(kStatusBadPage);
        }
        if (off >= 0) static_cast<uint8_t*>(a.out_sf)[off + (j / 4) * 512 + (j % 4)] = (uint8_t)s8;
      }
    }
  }
}

// ---- the softmax over token positions, in one fixed order ------------------
// Entry i of a request pools U token positions per channel: u = 0 .. m-1 are
// tokens m*i + u of the current group (biases B^a[u]); with overlap (CSA,
// i >= 1) u = m .. 2m-1 are tokens m*(i-1) + u - m of the previous group
// (biases B^b[u - m]).  Every kernel form computes, per channel,
//   M   = max_u (z_u + b_u)
//   e_u = exp((z_u + b_u) - M)
//   D   = sum over blocks of 32 positions, in order, of (e_u summed in order)
//   S   = the same with e_u * c_u (fused multiply-add)
//   out = S / D
// two passes, so the exponentials of one pass are independent of each other.
// The form that owns a channel (a thread over 8 channels, a thread per
// channel, several threads per channel) only changes who computes which
// block; the operations and their order stay the same, so every form writes
// the same bytes for the same entry.
constexpr int kPosBlock = 32;

__device__ __forceinline__ float pos_elem(const uint8_t* base, int dt, int64_t idx) {
  return dt == CSA_F32 ? reinterpret_cast<const float*>(base)[idx]
                       : __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(base)[idx] << 16);
}
// Running max of channel-relative logits over n rows `stride` elements apart.
__device__ __forceinline__ float chan_max(const uint8_t* z, const float* bias, int dt, int stride, int n, float M) {
  for (int u = 0; u < n; ++u) M = fmaxf(M, pos_elem(z, dt, (int64_t)u * stride) + bias[(int64_t)u * stride]);
  return M;
}
// Sums of one block of n <= kPosBlock rows.
__device__ __forceinline__ void chan_block(const uint8_t* z, const uint8_t* c, const float* bias, int dt, int stride,
                                           int n, float M, float& d, float& s) {
  d = 0.f;
  s = 0.f;
#pragma unroll 4
  for (int u = 0; u < n; ++u) {
    const int64_t k = (int64_t)u * stride;
    const float e = expf((pos_elem(z, dt, k) + bias[k]) - M);
    d += e;
    s = fmaf(e, pos_elem(c, dt, k), s);
  }
}
__device__ __forceinline__ float pooled_value(float D, float S) { return D > 0.f ? S / D : 0.f; }

// ---- staged form (at most kPosBlock positions per entry) --------------------
// All of an entry's inputs are brought into shared memory with one round of
// cp.async, so a block that compresses while the rest of the GPU streams pays
// one memory round trip per call.  Layout of one staged entry (U = 2m with
// overlap, else m; rows of dim elements):
//   Z [U][dim] (in_dt) | C [U][dim] (in_dt) | bias [U][dim] f32 | x [dim] f32
__host__ __device__ __forceinline__ int staged_positions(const CompressArgs& a) {
  return a.Cb != nullptr ? 2 * a.m : a.m;
}
__host__ __device__ __forceinline__ int staged_entry_bytes(const CompressArgs& a) {
  const int esz = a.in_dt == CSA_F32 ? 4 : 2;
  const int U = staged_positions(a);
  return U * a.dim * (2 * esz + 4) + a.dim * 4;
}
__device__ __forceinline__ void stage_cp16(uint8_t* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
// Issues (without waiting) the cp.async copies of entry e0 + ie of request b.
template <int NT>
__device__ void stage_entry(const CompressArgs& a, int b, int64_t ie, uint8_t* buf) {
  const int esz = a.in_dt == CSA_F32 ? 4 : 2;
  const int64_t i = a.e0 + ie;
  const bool two = a.Cb != nullptr && i >= 1;
  const int U = two ? 2 * a.m : a.m, Umax = staged_positions(a);
  const int row16 = a.dim * esz / 16;  // 16-byte pieces per input row
  const int64_t in_base = (int64_t)b * a.in_batch_stride;
  uint8_t* zb = buf;
  uint8_t* cb = buf + (size_t)Umax * a.dim * esz;
  for (int q = threadIdx.x; q < U * row16; q += NT) {
    const int u = q / row16, p = q % row16;
    const bool cur = u < a.m;
    const int64_t tok = cur ? (int64_t)a.m * i + u : (int64_t)a.m * (i - 1) + (u - a.m);
    const int64_t off = ((in_base + tok - a.tok0) * a.dim) * esz + (int64_t)p * 16;
    stage_cp16(zb + (size_t)u * a.dim * esz + p * 16, static_cast<const uint8_t*>(cur ? a.Za : a.Zb) + off);
    stage_cp16(cb + (size_t)u * a.dim * esz + p * 16, static_cast<const uint8_t*>(cur ? a.Ca : a.Cb) + off);
  }
  // bias rows in position order: B^a[0..m), then B^b[0..m)
  uint8_t* bias = buf + (size_t)Umax * a.dim * esz * 2;
  const int brow16 = a.dim * 4 / 16;
  for (int q = threadIdx.x; q < U * brow16; q += NT) {
    const int u = q / brow16, p = q % brow16;
    const float* src = u < a.m ? a.Ba + (int64_t)u * a.dim : a.Bb + (int64_t)(u - a.m) * a.dim;
    stage_cp16(bias + ((size_t)u * a.dim) * 4 + p * 16, reinterpret_cast<const uint8_t*>(src) + p * 16);
  }
}
// Channel w of a staged entry (after the copies landed and a block barrier):
// writes the pooled value into the entry's x row.
__device__ __forceinline__ void staged_channel(const CompressArgs& a, int64_t ie, uint8_t* buf, int w) {
  const int esz = a.in_dt == CSA_F32 ? 4 : 2;
  const int64_t i = a.e0 + ie;
  const int U = (a.Cb != nullptr && i >= 1) ? 2 * a.m : a.m, Umax = staged_positions(a);
  const uint8_t* zb = buf + (size_t)w * esz;
  const uint8_t* cb = buf + (size_t)Umax * a.dim * esz + (size_t)w * esz;
  const float* bias = reinterpret_cast<const float*>(buf + (size_t)Umax * a.dim * esz * 2) + w;
  const float M = chan_max(zb, bias, a.in_dt, a.dim, U, -INFINITY);
  float d, s;
  chan_block(zb, cb, bias, a.in_dt, a.dim, U, M, d, s);
  float D = 0.f, S = 0.f;
  D += d;
  S += s;
  reinterpret_cast<float*>(buf + (size_t)Umax * a.dim * (2 * esz + 4))[w] = pooled_value(D, S);
}
// Writes the 8-channel chunk ch of a staged entry whose x row is complete.
// Called by whole warps (valid == false lanes join the shuffles only).
__device__ __forceinline__ void staged_store(const CompressArgs& a, int b, int64_t ie, const uint8_t* buf, int ch,
                                             bool valid) {
  const int esz = a.in_dt == CSA_F32 ? 4 : 2;
  const float* xr = reinterpret_cast<const float*>(buf + (size_t)staged_positions(a) * a.dim * (2 * esz + 4));
  float x[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) x[q] = valid ? xr[ch * 8 + q] : 0.f;
  store_entry(a, b, ie, valid ? ch * 8 : 0, x, valid);
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

// Entry e0 + ie of request b, channel groups [cg_lo, cg_hi) of 64 channels,
// by a CTA of 256 threads with tokpar_smem_bytes(a) bytes of shared memory at
// tsm (16-byte aligned).  Row mode (normalisation / RoPE epilogue) needs
// every group of the entry in one call, so the whole pooled row is in shared
// memory at the end.
__device__ __forceinline__ void tokpar_entry(const CompressArgs& a, int b, int64_t ie, int cg_lo, int cg_hi,
                                          uint8_t* tsm) {
  const int esz = a.in_dt == CSA_F32 ? 4 : 2;
  const bool rowm = compress_row_epilogue(a);
  const int64_t i = a.e0 + ie;
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
}  // namespace csa
