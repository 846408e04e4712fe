// csa_internal.cuh -- device helpers and internal launcher declarations shared
// by the CUDA translation units of libcsa_b200.  Nothing here is visible
// through the C ABI (include/csa.h is the public surface).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

// ---------------------------------------------------------------------------
// Storage formats (byte layouts documented in include/csa.h).
// ---------------------------------------------------------------------------
constexpr int kRopeDims = 64;        // trailing RoPE dims kept in bf16 (FP8MIX)
constexpr int kFp8Block = 64;        // FP8 dims sharing one fp32 scale
constexpr int kFp4Block = 16;        // FP4 values sharing one E4M3 scale

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

__host__ __device__ inline int64_t row_bytes(int dt, int dim) {
  switch (dt) {
    case CSA_F32: return 4LL * dim;
    case CSA_BF16: return 2LL * dim;
    case CSA_KV_FP8MIX: {
      int64_t n8 = dim - kRopeDims;
      return (n8 + 2 * kRopeDims + 4 * (n8 / kFp8Block) + 15) / 16 * 16;
    }
    case CSA_IDX_NVFP4: return dim / 2;
    default: return -1;
  }
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

// Two E4M3 codes (low byte = first element) -> two floats (hardware convert).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t codes) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)codes, __NV_E4M3);
  __half2 hh;
  memcpy(&hh, &h, sizeof(hh));
  return __half22float2(hh);
}

__device__ __forceinline__ float e4m3_to_float(uint8_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  __half hh;
  memcpy(&hh, &h, sizeof(hh));
  return __half2float(hh);
}

// Two E2M1 codes packed in one byte (low nibble = first element) -> floats.
__device__ __forceinline__ float2 e2m1x2_to_float2(uint8_t byte) {
  __half2_raw h = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)byte, __NV_E2M1);
  __half2 hh;
  memcpy(&hh, &h, sizeof(hh));
  return __half22float2(hh);
}

// Decode `n` consecutive values [d0, d0+n) of one row of format dt into f32.
// n and d0 are multiples of 8 (FP8MIX/BF16/F32) or 16 (NVFP4).
// NVFP4 scales come either row-major (sf_row[j] for values 16j..16j+15) or,
// for key-cache rows, in the blocked atom layout (sf_blocked: sf_row from
// nvfp4_blocked_sf_row, scale j at sf_row[(j / 4) * 512 + j % 4]).
__device__ __forceinline__ void decode_row_chunk8(const uint8_t* row, const uint8_t* sf_row, int dt,
                                                  int dim, int d0, float* out8,
                                                  bool sf_blocked = false) {
  if (dt == CSA_F32) {
    const float4* p = reinterpret_cast<const float4*>(row + 4 * d0);
    float4 a = p[0], b = p[1];
    out8[0] = a.x; out8[1] = a.y; out8[2] = a.z; out8[3] = a.w;
    out8[4] = b.x; out8[5] = b.y; out8[6] = b.z; out8[7] = b.w;
  } else if (dt == CSA_BF16) {
    uint4 v = *reinterpret_cast<const uint4*>(row + 2 * d0);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      out8[2 * j] = __uint_as_float(w[j] << 16);
      out8[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else if (dt == CSA_KV_FP8MIX) {
    const int n8 = dim - kRopeDims;
    if (d0 < n8) {
      uint2 v = *reinterpret_cast<const uint2*>(row + d0);
      const float s = *reinterpret_cast<const float*>(row + n8 + 2 * kRopeDims + 4 * (d0 / kFp8Block));
      uint32_t w[2] = {v.x, v.y};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float2 lo = e4m3x2_to_float2((uint16_t)(w[j] & 0xFFFF));
        float2 hi = e4m3x2_to_float2((uint16_t)(w[j] >> 16));
        out8[4 * j + 0] = lo.x * s; out8[4 * j + 1] = lo.y * s;
        out8[4 * j + 2] = hi.x * s; out8[4 * j + 3] = hi.y * s;
      }
    } else {
      uint4 v = *reinterpret_cast<const uint4*>(row + n8 + 2 * (d0 - n8));
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        out8[2 * j] = __uint_as_float(w[j] << 16);
        out8[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
  } else {  // NVFP4: 8 values = 4 bytes, one scale per 16 values
    uint32_t v = *reinterpret_cast<const uint32_t*>(row + d0 / 2);
    const int j = d0 / kFp4Block;
    const float s = e4m3_to_float(sf_row[sf_blocked ? (j >> 2) * 512 + (j & 3) : j]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = e2m1x2_to_float2((uint8_t)(v >> (8 * j)));
      out8[2 * j] = f.x * s;
      out8[2 * j + 1] = f.y * s;
    }
  }
}

// Start of row r's scales in a blocked NVFP4 key-scale array of dimension
// dim: 128-row blocks of dim/64 atoms of 512 bytes; inside an atom, row r
// owns bytes (r % 32) * 16 + (r % 128 / 32) * 4 .. +3.
__host__ __device__ __forceinline__ int64_t nvfp4_blocked_sf_offset(int64_t r, int dim) {
  return (r / 128) * (dim / 64) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4;
}
// Bytes of the blocked scale array of one request with n_rows rows.
__host__ __device__ __forceinline__ int64_t nvfp4_blocked_sf_bytes(int64_t n_rows, int dim) {
  return (n_rows + 127) / 128 * (dim / 64) * 512;
}

// A paged cache ("CSA / HCA" cache layout: fixed pages of 128 tokens taken
// from a shared pool through a per-request block table): logical row lr of
// request b lives in pool row table[b][lr / page_entries] * page_entries +
// lr % page_entries.  table == nullptr: the contiguous layout, request b's
// rows at b * (rows per request).
struct PageTable {
  const int32_t* table;  // [batch][max_pages]
  int max_pages;
  int page_entries;
  int64_t n_pages;       // pages in the pool
};
// Pool page of logical page j of request b, or -1 when the table names a page
// outside the pool.
__device__ __forceinline__ int64_t pool_page(const PageTable& pt, int b, int64_t j) {
  const int32_t pg = __ldg(pt.table + (int64_t)b * pt.max_pages + j);
  return (pg < 0 || pg >= pt.n_pages) ? -1 : (int64_t)pg;
}
// Pool row of logical row lr of request b, or -1 (page outside the pool).
__device__ __forceinline__ int64_t pool_row(const PageTable& pt, int b, int64_t lr) {
  const int64_t j = lr / pt.page_entries;
  const int64_t pg = pool_page(pt, b, j);
  return pg < 0 ? -1 : pg * pt.page_entries + (lr - j * pt.page_entries);
}
// Paged NVFP4 key scales: one blocked 128-row block (dim/64 atoms) per pool
// page; the 128 logical rows 128 u .. 128 u + 127 (page_entries divides 128)
// keep theirs in the block of the pool page holding logical row 128 u, at the
// offset the contiguous layout gives row lr % 128.  Pool page of that block,
// or -1.
__device__ __forceinline__ int64_t pool_sf_page(const PageTable& pt, int b, int64_t lr) {
  return pool_page(pt, b, (lr / 128) * (128 / pt.page_entries));
}

// Order-preserving key of a float score (larger score -> larger key).
__device__ __forceinline__ uint32_t f32_key(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// bf16 score -> key in the upper 16 bits (lower 16 bits zero).
__device__ __forceinline__ uint32_t bf16_key(float s) {
  __nv_bfloat16 b = __float2bfloat16_rn(s);
  uint16_t h;
  memcpy(&h, &b, 2);
  uint32_t u = ((uint32_t)h) << 16;
  return (u & 0x80000000u) ? (~u & 0xFFFF0000u) : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_f32(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// ---------------------------------------------------------------------------
// Internal launchers (one per translation unit); all return cudaError_t of the
// launch (cudaGetLastError) and never allocate.  Each kernel launch bumps the
// calling thread's launch counter (reported by csa_last_launch_count).
// ---------------------------------------------------------------------------
int& launch_counter();
// Status words of the kernels with bounded waits (read and cleared; nonzero
// means a wait gave up, 2 means the word could not be read).
unsigned int take_status_indexer_tc();
unsigned int take_status_mqa_umma();
unsigned int take_status_out_proj();
unsigned int take_status_mqa();
unsigned int take_status_indexer();
unsigned int take_status_compress();
// Zeroes the current device's built-in indexer scratch (csa_index_topk_noalloc)
// after a timed-out wait; a no-op when the scratch was never used.
void reset_static_scratch();
// Records `msg` as the calling thread's last error and returns `st`.
csa_status_t set_error(csa_status_t st, const char* msg);
struct CompressArgs {
  const void *Ca, *Cb, *Za, *Zb;
  const float *Ba, *Bb;
  int batch;
  int64_t n_tok, tok0, in_batch_stride, e0, n_out;
  int dim, m, in_dt, out_dt;
  void *out, *out_sf;
  int64_t out_batch_stride, out_row0;
  // output rows through a block table (out_pages.table != nullptr): row
  // out_row0 + j of request b is logical row out_row0 + j of its pages
  PageTable out_pages;
  // entry normalisation and partial RoPE before the entry is stored: RMSNorm
  // weights [dim] (nullptr: none) and eps; the last rope_dims dims (0: none)
  // turned at position pos_stride * i + pos_offset for entry i, base rope_base
  const float* norm_g;
  float norm_eps;
  int rope_dims;
  double rope_base;
  int64_t pos_stride, pos_offset;
};
__host__ __device__ __forceinline__ bool compress_row_epilogue(const CompressArgs& a) {
  return a.norm_g != nullptr || a.rope_dims > 0;
}
cudaError_t launch_compress(const CompressArgs& a, cudaStream_t s);

struct NormRopeArgs {
  const void* x;
  void* y;
  int64_t n_rows;
  int dim, rows_per_pos, pos_sign, rope_dims;
  const float* g;
  float eps;
  const int64_t* pos;
  double base;
  int in_dt, out_dt;
};
cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s);

struct IndexArgs {
  const void *qI, *qI_sf;
  const float* wI;
  const void *KI, *KI_sf;
  const int64_t* q_pos;
  int batch, n_q;
  int64_t n_entries;
  int m, n_heads, dim, k, dt;
  int32_t* idx_out;
  void* scores_out;
  void* ws;
  size_t ws_bytes;
  // fused decode form: the CTA whose slice holds the new key rows
  // comp.e0 .. +n_out compresses them into the key cache (comp.out = KI)
  // before streaming them, and runs the extra job comp2 (any other cache;
  // n_out = 0 when absent) for its request
  int fused;
  CompressArgs comp, comp2;
  // keys through a block table (pages.table != nullptr): KI / KI_sf are the
  // pool, n_entries the logical entries per request
  PageTable pages;
};
size_t index_topk_workspace(int batch, int n_q, int64_t n_entries, int k, int n_heads, int dim, int dt);
// out[0..5]: entries per slice, slices per query row, cooperative selection,
// tensor-core producer, key stages in the ring, 128-entry tiles per stage.
void index_topk_plan_info(int batch, int n_q, int64_t n_entries, int k, int n_heads, int dim, int dt,
                          int32_t* out);
// Whether the indexer runs the fused decode form (compress the new keys in
// the indexer launch) for these arguments.
bool index_fusable(const IndexArgs& a);
cudaError_t launch_index_topk(const IndexArgs& a, cudaStream_t s);

struct MqaArgs {
  const void* Q;
  int q_dt;
  const void* entries;
  int64_t n_entries;
  const int32_t* idx;  // nullptr: dense (HCA) over every visible entry
  int k;
  const void* win;
  int64_t win_len;
  const int64_t* win_start;
  const int64_t* q_pos;
  int window, m;
  const float* sink;
  float scale;
  int batch, n_q, n_heads, dim, kv_dt;
  void* O;
  void* ws;
  size_t ws_bytes;
  // options (csa_mqa_options_t): a fixed split count per query (0: chosen
  // from the batch), the query's RMSNorm weights (nullptr: none) and eps, the
  // RoPE dims turned on the query at q_pos and on the output at -q_pos, and
  // the RoPE base
  int splits;
  const float* q_norm_g;
  float q_norm_eps;
  int q_rope_dims, out_rope_dims;
  double rope_base;
  // entries through a block table (pages.table != nullptr): `entries` is the
  // pool, n_entries the logical entries per request
  PageTable pages;
  // the step's entry compression (has_comp), launched before the attention
  int has_comp;
  CompressArgs comp;
};
size_t mqa_workspace(const MqaArgs& a);
// Whether the tensor-core attention kernel takes these arguments (the query
// normalisation and RoPE options exist only there).
bool mqa_tc_path(const MqaArgs& a);
cudaError_t launch_mqa(const MqaArgs& a, cudaStream_t s);

struct OutProjArgs {
  const void *O, *Wg, *Wo;  // bf16: O [T][n_h][c], Wg [g][n_h/g * c][d_g], Wo [g * d_g][d]
  void* Y;                  // bf16 [T][d]
  int T, n_h, c, g, d_g, d;
  void* ws;
};
size_t out_proj_workspace(int T, int n_h, int c, int g, int d_g, int d);
// out[0..5]: tokens per CTA, K slices and CTAs of the group projection, then
// the same three for the output projection.
void out_proj_plan_info(int T, int n_h, int c, int g, int d_g, int d, int32_t* out);
cudaError_t launch_out_proj(const OutProjArgs& a, cudaStream_t s);

}  // namespace csa
