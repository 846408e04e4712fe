// api.cu -- the C ABI of libcsa_b200 (declared and documented in include/csa.h):
// host-side argument validation, workspace sizing and dispatch to the
// kernels.  Nothing here allocates device memory, prints or aborts.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "csa_internal.cuh"

namespace {

thread_local char g_err[512] = "";
thread_local int g_launches = 0;

csa_status_t fail(csa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

csa_status_t ok() {
  g_err[0] = 0;
  return CSA_OK;
}

csa_status_t cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, ...)                                  \
  do {                                                      \
    if (!(cond)) return fail(CSA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define REQUIRE_PTR(p)                                                        \
  do {                                                                        \
    if ((p) == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s is NULL", #p);   \
    if (!aligned16(p)) return fail(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
  } while (0)

#define REQUIRE_ALIGNED_OR_NULL(p)                                            \
  do {                                                                        \
    if ((p) != nullptr && !aligned16(p))                                      \
      return fail(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);     \
  } while (0)

// A block table covering `rows` logical rows per request.
csa_status_t check_pages(const csa_pages_t* p, int64_t rows, const char* what) {
  REQUIRE(p->table != nullptr, "%s: table is NULL", what);
  REQUIRE(aligned16(p->table), "%s: table is not 16-byte aligned", what);
  REQUIRE(p->max_pages >= 1 && p->page_entries >= 1 && p->n_pages >= 1,
          "%s: max_pages, page_entries and n_pages must be >= 1", what);
  REQUIRE(p->n_pages <= ((int64_t)1 << 31) && p->n_pages * p->page_entries <= ((int64_t)1 << 40),
          "%s: pool too large", what);
  REQUIRE(rows <= (int64_t)p->max_pages * p->page_entries,
          "%s: %lld rows per request exceed max_pages * page_entries = %lld", what, (long long)rows,
          (long long)p->max_pages * p->page_entries);
  return CSA_OK;
}

csa::PageTable to_pages(const csa_pages_t* p) {
  return csa::PageTable{p->table, p->max_pages, p->page_entries, p->n_pages};
}

}  // namespace

int& csa::launch_counter() { return g_launches; }

csa_status_t csa::set_error(csa_status_t st, const char* msg) { return fail(st, "%s", msg); }

// Validates a compressor call on the host; fills *args, or sets *empty when
// there is nothing to do.
static csa_status_t check_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                                   const float* Ba, const float* Bb, int batch, int64_t n_tok, int64_t tok0,
                                   int64_t in_batch_stride, int64_t e0, int64_t n_out, int dim, int m,
                                   csa_dtype_t in_dt, void* out, void* out_sf, int64_t out_batch_stride,
                                   int64_t out_row0, csa_dtype_t out_dt, const csa_pages_t* out_pages,
                                   csa::CompressArgs* args, bool* empty, const csa_compress_job_t* epi = nullptr) {
  *empty = false;
  REQUIRE(batch >= 0 && n_tok >= 0 && tok0 >= 0 && e0 >= 0 && n_out >= 0 && out_row0 >= 0,
          "negative size (batch=%d n_tok=%lld tok0=%lld e0=%lld n_out=%lld out_row0=%lld)", batch,
          (long long)n_tok, (long long)tok0, (long long)e0, (long long)n_out, (long long)out_row0);
  REQUIRE(m >= 1 && m <= 4096, "m=%d out of range [1, 4096]", m);
  REQUIRE(dim >= 8 && dim % 8 == 0, "dim=%d must be a positive multiple of 8", dim);
  REQUIRE(in_dt == CSA_F32 || in_dt == CSA_BF16, "in_dt must be CSA_F32 or CSA_BF16");
  REQUIRE(out_dt >= CSA_F32 && out_dt <= CSA_IDX_NVFP4, "unknown out_dt %d", (int)out_dt);
  if (out_dt == CSA_KV_FP8MIX)
    REQUIRE(dim >= 128 && (dim - 64) % 64 == 0, "KV_FP8MIX needs dim = 64 + 64*j (j >= 1), got %d", dim);
  if (out_dt == CSA_IDX_NVFP4) REQUIRE(dim % 64 == 0, "NVFP4 output needs dim %% 64 == 0, got %d", dim);
  REQUIRE(in_batch_stride >= n_tok, "in_batch_stride %lld < n_tok %lld", (long long)in_batch_stride,
          (long long)n_tok);
  if (out_pages == nullptr) {
    REQUIRE(out_batch_stride >= out_row0 + n_out, "out_batch_stride %lld < out_row0 %lld + n_out %lld",
            (long long)out_batch_stride, (long long)out_row0, (long long)n_out);
  } else {
    const csa_status_t st = check_pages(out_pages, out_row0 + n_out, "out_pages");
    if (st != CSA_OK) return st;
    if (out_dt == CSA_IDX_NVFP4)
      REQUIRE(128 % out_pages->page_entries == 0, "paged NVFP4 keys need page_entries dividing 128, got %d",
              out_pages->page_entries);
  }
  if ((int64_t)batch * n_out == 0) {
    *empty = true;
    return ok();
  }
  REQUIRE_PTR(Ca);
  REQUIRE_PTR(Za);
  REQUIRE_PTR(Ba);
  REQUIRE_PTR(out);
  const bool overlap = Cb != nullptr;
  if (overlap) {
    REQUIRE_PTR(Zb);
    REQUIRE_PTR(Bb);
    REQUIRE_ALIGNED_OR_NULL(Cb);
  }
  if (out_dt == CSA_IDX_NVFP4) {
    REQUIRE(out_sf != nullptr, "out_sf is NULL for NVFP4 output");
    REQUIRE_ALIGNED_OR_NULL(out_sf);
  }
  const int64_t first = (overlap && e0 >= 1) ? (int64_t)m * (e0 - 1) : (int64_t)m * e0;
  const int64_t last = (int64_t)m * (e0 + n_out) - 1;
  REQUIRE(first >= tok0 && last < tok0 + n_tok,
          "entries [%lld, %lld) need tokens [%lld, %lld] but rows hold [%lld, %lld)",
          (long long)e0, (long long)(e0 + n_out), (long long)first, (long long)last,
          (long long)tok0, (long long)(tok0 + n_tok));
  *args = csa::CompressArgs{Ca, Cb, Za, Zb, Ba, Bb, batch, n_tok, tok0, in_batch_stride, e0, n_out,
                            dim, m, (int)in_dt, (int)out_dt, out, out_sf, out_batch_stride, out_row0,
                            out_pages ? to_pages(out_pages) : csa::PageTable{nullptr, 0, 0, 0}};
  args->norm_g = nullptr;
  args->norm_eps = 0.f;
  args->rope_dims = 0;
  args->rope_base = 10000.0;
  args->pos_stride = m;
  args->pos_offset = m - 1;
  if (epi != nullptr && (epi->norm_g != nullptr || epi->rope_dims != 0)) {
    REQUIRE(epi->rope_dims >= 0 && epi->rope_dims % 8 == 0 && epi->rope_dims <= dim,
            "rope_dims=%d must be a multiple of 8 in [0, dim=%d]", epi->rope_dims, dim);
    REQUIRE(epi->norm_g == nullptr || epi->norm_eps >= 0.f, "norm_eps must be >= 0");
    REQUIRE(epi->rope_dims == 0 || epi->rope_base > 0.0, "rope_base must be > 0");
    REQUIRE(batch <= 65535, "batch=%d too large for the normalising compressor (<= 65535)", batch);
    REQUIRE(dim <= 16384, "dim=%d too large for the normalising compressor (<= 16384)", dim);
    REQUIRE_ALIGNED_OR_NULL(epi->norm_g);
    args->norm_g = epi->norm_g;
    args->norm_eps = epi->norm_eps;
    args->rope_dims = epi->rope_dims;
    args->rope_base = epi->rope_base;
    args->pos_stride = epi->pos_stride;
    args->pos_offset = epi->pos_offset;
  }
  return ok();
}


// Validates an indexer call on the host; fills *args, or sets *empty when
// there is nothing to do.
static csa_status_t check_index(const void* qI, const void* qI_sf, const float* wI, const void* KI,
                                const void* KI_sf, const int64_t* q_pos, int batch, int n_q, int64_t n_entries,
                                int m, int n_heads, int dim, int k, csa_dtype_t dt, int32_t* idx_out,
                                void* scores_out, void* ws, size_t ws_bytes, const csa_pages_t* key_pages,
                                csa::IndexArgs* args, bool* empty) {
  *empty = false;
  REQUIRE(batch >= 0 && n_q >= 0 && n_entries >= 0, "negative size");
  REQUIRE(n_entries <= (int64_t)1 << 30, "n_entries=%lld too large", (long long)n_entries);
  REQUIRE(m >= 1, "m=%d must be >= 1", m);
  REQUIRE(k >= 1 && k <= 2048, "k=%d out of range [1, 2048]", k);
  REQUIRE(n_heads >= 1 && n_heads <= 128, "n_heads=%d out of range [1, 128]", n_heads);
  REQUIRE(dim >= 32 && dim <= 256 && dim % 32 == 0, "dim=%d must be a multiple of 32 in [32, 256]", dim);
  REQUIRE(dt == CSA_F32 || dt == CSA_BF16 || dt == CSA_IDX_NVFP4, "dt must be F32, BF16 or IDX_NVFP4");
  if ((int64_t)batch * n_q == 0) {
    *empty = true;
    return ok();
  }
  REQUIRE_PTR(qI);
  REQUIRE_PTR(wI);
  REQUIRE_PTR(q_pos);
  REQUIRE_PTR(idx_out);
  REQUIRE_ALIGNED_OR_NULL(scores_out);
  if (n_entries > 0) REQUIRE_PTR(KI);
  if (dt == CSA_IDX_NVFP4) {
    REQUIRE(qI_sf != nullptr && (KI_sf != nullptr || n_entries == 0), "NVFP4 needs qI_sf and KI_sf");
    REQUIRE(dim % 64 == 0, "NVFP4 needs dim %% 64 == 0 (blocked key scales), got %d", dim);
    REQUIRE_ALIGNED_OR_NULL(KI_sf);
  }
  if (key_pages != nullptr) {
    const csa_status_t st = check_pages(key_pages, n_entries, "key_pages");
    if (st != CSA_OK) return st;
    const int pe = key_pages->page_entries;
    REQUIRE(pe >= 8 && 128 % pe == 0, "paged keys need page_entries in {8, 16, 32, 64, 128}, got %d", pe);
    REQUIRE(key_pages->n_pages * pe < ((int64_t)1 << 31), "key pool of %lld rows too large",
            (long long)(key_pages->n_pages * pe));
  }
  const size_t need = csa_index_topk_workspace_size(batch, n_q, n_entries, k, n_heads, dim, dt);
  REQUIRE(ws_bytes >= need, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  REQUIRE_PTR(ws);
  *args = csa::IndexArgs{qI, qI_sf, wI, KI, KI_sf, q_pos, batch, n_q, n_entries, m, n_heads, dim, k,
                         (int)dt, idx_out, scores_out, ws, ws_bytes, 0, csa::CompressArgs{}, csa::CompressArgs{},
                         key_pages ? to_pages(key_pages) : csa::PageTable{nullptr, 0, 0, 0}};
  return ok();
}


extern "C" {

const char* csa_last_error(void) { return g_err; }

int csa_last_launch_count(void) { return g_launches; }

csa_status_t csa_check_device_status(void) {
  const cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "csa_check_device_status");
  const unsigned int st = csa::take_status_indexer_tc() | csa::take_status_mqa_umma() | csa::take_status_out_proj() |
                          csa::take_status_mqa() | csa::take_status_indexer() | csa::take_status_compress();
  if (st & 2u) return fail(CSA_ERR_CUDA, "csa_check_device_status: status word unreadable");
  if (st & 1u) {
    // a selection that gave up may have left counters set in the built-in
    // scratch of csa_index_topk_noalloc: zero it (caller workspaces are the
    // caller's to zero)
    csa::reset_static_scratch();
    return fail(CSA_ERR_TIMEOUT, "a kernel pipeline wait timed out; its results are invalid");
  }
  if (st & 4u) return fail(CSA_ERR_INVALID_ARG, "a page table named a page outside the pool; rows were dropped");
  return ok();
}

int csa_version(void) { return 201; }

int64_t csa_row_bytes(csa_dtype_t dt, int dim) {
  if (dim <= 0) return -1;
  if (dt == CSA_KV_FP8MIX && (dim < 64 || (dim - 64) % 64 != 0)) return -1;
  if (dt == CSA_IDX_NVFP4 && dim % 16 != 0) return -1;
  return csa::row_bytes(dt, dim);
}

int64_t csa_nvfp4_key_scale_bytes(int64_t n_rows, int dim) {
  if (n_rows < 0 || dim <= 0 || dim % 64 != 0) return -1;
  return csa::nvfp4_blocked_sf_bytes(n_rows, dim);
}

csa_status_t csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                          const float* Ba, const float* Bb, int batch, int64_t n_tok,
                          int64_t tok0, int64_t in_batch_stride, int64_t e0, int64_t n_out,
                          int dim, int m, csa_dtype_t in_dt, void* out, void* out_sf,
                          int64_t out_batch_stride, int64_t out_row0, csa_dtype_t out_dt,
                          void* stream) {
  g_launches = 0;
  csa::CompressArgs a{};
  bool empty = false;
  const csa_status_t st = check_compress(Ca, Cb, Za, Zb, Ba, Bb, batch, n_tok, tok0, in_batch_stride, e0, n_out,
                                         dim, m, in_dt, out, out_sf, out_batch_stride, out_row0, out_dt, nullptr, &a,
                                         &empty);
  if (st != CSA_OK || empty) return st;
  return cuda_status(csa::launch_compress(a, static_cast<cudaStream_t>(stream)), "csa_compress");
}

csa_status_t csa_compress_ex(const csa_compress_job_t* job, int batch, void* stream) {
  g_launches = 0;
  REQUIRE(job != nullptr, "job is NULL");
  csa::CompressArgs a{};
  bool empty = false;
  const csa_status_t st = check_compress(job->Ca, job->Cb, job->Za, job->Zb, job->Ba, job->Bb, batch, job->n_tok,
                                         job->tok0, job->in_batch_stride, job->e0, job->n_out, job->dim, job->m,
                                         job->in_dt, job->out, job->out_sf, job->out_batch_stride, job->out_row0,
                                         job->out_dt, job->out_pages, &a, &empty, job);
  if (st != CSA_OK || empty) return st;
  return cuda_status(csa::launch_compress(a, static_cast<cudaStream_t>(stream)), "csa_compress_ex");
}

csa_status_t csa_rmsnorm_rope(const void* x, void* y, int64_t n_rows, int dim, const float* g, float eps,
                              const int64_t* pos, int rows_per_pos, int pos_sign, int rope_dims, double base,
                              csa_dtype_t in_dt, csa_dtype_t out_dt, void* stream) {
  g_launches = 0;
  REQUIRE(n_rows >= 0, "n_rows=%lld is negative", (long long)n_rows);
  REQUIRE(dim >= 8 && dim % 8 == 0, "dim=%d must be a positive multiple of 8", dim);
  REQUIRE(rope_dims >= 0 && rope_dims % 8 == 0 && rope_dims <= dim,
          "rope_dims=%d must be a multiple of 8 in [0, dim=%d]", rope_dims, dim);
  REQUIRE(rows_per_pos >= 1, "rows_per_pos=%d must be >= 1", rows_per_pos);
  REQUIRE(pos_sign == 1 || pos_sign == -1, "pos_sign=%d must be +1 or -1", pos_sign);
  REQUIRE(eps >= 0.f, "eps must be >= 0");
  REQUIRE(base > 0.0, "base must be > 0");
  REQUIRE(in_dt == CSA_F32 || in_dt == CSA_BF16, "in_dt must be CSA_F32 or CSA_BF16");
  REQUIRE(out_dt == CSA_F32 || out_dt == CSA_BF16, "out_dt must be CSA_F32 or CSA_BF16");
  REQUIRE(x != y || in_dt == out_dt, "in place (y == x) needs in_dt == out_dt");
  if (n_rows == 0) return ok();
  REQUIRE_PTR(x);
  REQUIRE_PTR(y);
  if (rope_dims > 0) REQUIRE(pos != nullptr, "pos is NULL with rope_dims > 0");
  REQUIRE(n_rows <= ((int64_t)1 << 40), "n_rows=%lld too large", (long long)n_rows);
  csa::NormRopeArgs a{x, y, n_rows, dim, rows_per_pos, pos_sign, rope_dims, g, eps, pos, base, (int)in_dt,
                      (int)out_dt};
  return cuda_status(csa::launch_norm_rope(a, static_cast<cudaStream_t>(stream)), "csa_rmsnorm_rope");
}

size_t csa_index_topk_workspace_size(int batch, int n_q, int64_t n_entries, int k, int n_heads,
                                     int dim, csa_dtype_t dt) {
  if (batch <= 0 || n_q <= 0 || n_entries <= 0 || k <= 0) return 256;
  size_t s = csa::index_topk_workspace(batch, n_q, n_entries, k, n_heads, dim, (int)dt);
  return s < 256 ? 256 : s;
}

csa_status_t csa_index_topk_plan(int batch, int n_q, int64_t n_entries, int k, int n_heads, int dim,
                                 csa_dtype_t dt, int32_t* out) {
  REQUIRE(out != nullptr, "out is NULL");
  REQUIRE(batch >= 1 && n_q >= 1 && n_entries >= 1, "batch, n_q and n_entries must be >= 1");
  REQUIRE(n_entries <= (int64_t)1 << 30, "n_entries=%lld too large", (long long)n_entries);
  REQUIRE(k >= 1 && k <= 2048, "k=%d out of range [1, 2048]", k);
  REQUIRE(n_heads >= 1 && n_heads <= 128, "n_heads=%d out of range [1, 128]", n_heads);
  REQUIRE(dim >= 32 && dim <= 256 && dim % 32 == 0, "dim=%d must be a multiple of 32 in [32, 256]", dim);
  REQUIRE(dt == CSA_F32 || dt == CSA_BF16 || dt == CSA_IDX_NVFP4, "dt must be F32, BF16 or IDX_NVFP4");
  csa::index_topk_plan_info(batch, n_q, n_entries, k, n_heads, dim, (int)dt, out);
  return ok();
}

csa_status_t csa_index_topk(const void* qI, const void* qI_sf, const float* wI, const void* KI,
                            const void* KI_sf, const int64_t* q_pos, int batch, int n_q,
                            int64_t n_entries, int m, int n_heads, int dim, int k, csa_dtype_t dt,
                            int32_t* idx_out, void* scores_out, void* ws, size_t ws_bytes,
                            void* stream) {
  return csa_index_topk_paged(qI, qI_sf, wI, KI, KI_sf, nullptr, q_pos, batch, n_q, n_entries, m, n_heads, dim, k,
                              dt, idx_out, scores_out, ws, ws_bytes, stream);
}

csa_status_t csa_index_topk_paged(const void* qI, const void* qI_sf, const float* wI, const void* KI,
                                  const void* KI_sf, const csa_pages_t* key_pages, const int64_t* q_pos, int batch,
                                  int n_q, int64_t n_entries, int m, int n_heads, int dim, int k, csa_dtype_t dt,
                                  int32_t* idx_out, void* scores_out, void* ws, size_t ws_bytes, void* stream) {
  g_launches = 0;
  csa::IndexArgs a{};
  bool empty = false;
  const csa_status_t st = check_index(qI, qI_sf, wI, KI, KI_sf, q_pos, batch, n_q, n_entries, m, n_heads, dim, k,
                                      dt, idx_out, scores_out, ws, ws_bytes, key_pages, &a, &empty);
  if (st != CSA_OK || empty) return st;
  return cuda_status(csa::launch_index_topk(a, static_cast<cudaStream_t>(stream)), "csa_index_topk");
}

csa_status_t csa_compress_index_topk(const csa_compress_job_t* keys, const csa_compress_job_t* extra,
                                     const void* qI, const void* qI_sf, const float* wI, void* KI, void* KI_sf,
                                     const int64_t* q_pos, int batch, int n_q, int64_t n_entries, int m,
                                     int n_heads, int dim, int k, csa_dtype_t dt, int32_t* idx_out,
                                     void* scores_out, void* ws, size_t ws_bytes, void* stream) {
  g_launches = 0;
  REQUIRE(keys != nullptr, "keys is NULL");
  REQUIRE(keys->out == KI && keys->out_sf == KI_sf && keys->out_dt == dt && keys->dim == dim &&
              (keys->out_pages != nullptr || keys->out_batch_stride == n_entries) && keys->out_row0 == keys->e0,
          "keys must write entry i into row i of the indexer's cache (out == KI, out_sf == KI_sf, out_dt == dt, "
          "dim == dim, out_batch_stride == n_entries unless paged, out_row0 == e0)");
  csa::CompressArgs c{}, c2{};
  bool c_empty = false, c2_empty = true;
  csa_status_t st = check_compress(keys->Ca, keys->Cb, keys->Za, keys->Zb, keys->Ba, keys->Bb, batch, keys->n_tok,
                                   keys->tok0, keys->in_batch_stride, keys->e0, keys->n_out, keys->dim, keys->m,
                                   keys->in_dt, keys->out, keys->out_sf, keys->out_batch_stride, keys->out_row0,
                                   keys->out_dt, keys->out_pages, &c, &c_empty, keys);
  if (st != CSA_OK) return st;
  if (extra != nullptr) {
    REQUIRE(extra->out != KI && (extra->out_sf == nullptr || extra->out_sf != KI_sf),
            "extra must not write the indexer's cache");
    st = check_compress(extra->Ca, extra->Cb, extra->Za, extra->Zb, extra->Ba, extra->Bb, batch, extra->n_tok,
                        extra->tok0, extra->in_batch_stride, extra->e0, extra->n_out, extra->dim, extra->m,
                        extra->in_dt, extra->out, extra->out_sf, extra->out_batch_stride, extra->out_row0,
                        extra->out_dt, extra->out_pages, &c2, &c2_empty, extra);
    if (st != CSA_OK) return st;
  }
  csa::IndexArgs a{};
  bool i_empty = false;
  st = check_index(qI, qI_sf, wI, KI, KI_sf, q_pos, batch, n_q, n_entries, m, n_heads, dim, k, dt, idx_out,
                   scores_out, ws, ws_bytes, keys->out_pages, &a, &i_empty);
  if (st != CSA_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  a.comp = c;
  a.comp2 = c2;
  if (c2_empty) a.comp2.n_out = 0;
  if (!c_empty && !i_empty && csa::index_fusable(a)) {
    a.fused = 1;
    return cuda_status(csa::launch_index_topk(a, s), "csa_compress_index_topk");
  }
  int launches = 0;
  const csa::CompressArgs* jobs[2] = {c_empty ? nullptr : &c, c2_empty ? nullptr : &c2};
  for (const csa::CompressArgs* j : jobs) {
    if (j == nullptr) continue;
    g_launches = 0;
    const cudaError_t e = csa::launch_compress(*j, s);
    launches += g_launches;
    if (e != cudaSuccess) {
      g_launches = launches;
      return cuda_status(e, "csa_compress_index_topk (compress)");
    }
  }
  if (!i_empty) {
    g_launches = 0;
    const cudaError_t e = csa::launch_index_topk(a, s);
    launches += g_launches;
    if (e != cudaSuccess) {
      g_launches = launches;
      return cuda_status(e, "csa_compress_index_topk (index)");
    }
  }
  g_launches = launches;
  return ok();
}

}  // extern "C"

namespace {

// Copies the attention options into the argument struct (NULL = none).
csa_status_t apply_mqa_options(csa::MqaArgs& a, const csa_mqa_options_t* opt) {
  a.splits = 0;
  a.q_norm_g = nullptr;
  a.q_norm_eps = 0.f;
  a.q_rope_dims = a.out_rope_dims = 0;
  a.rope_base = 10000.0;
  a.pages = csa::PageTable{nullptr, 0, 0, 0};
  a.has_comp = 0;
  if (opt == nullptr) return CSA_OK;
  REQUIRE(opt->splits >= 0 && opt->splits <= 256, "splits=%d out of range [0, 256]", opt->splits);
  REQUIRE(opt->q_rope_dims >= 0 && opt->q_rope_dims <= 64 && opt->q_rope_dims % 8 == 0,
          "q_rope_dims=%d must be a multiple of 8 in [0, 64]", opt->q_rope_dims);
  REQUIRE(opt->out_rope_dims >= 0 && opt->out_rope_dims <= 64 && opt->out_rope_dims % 8 == 0,
          "out_rope_dims=%d must be a multiple of 8 in [0, 64]", opt->out_rope_dims);
  REQUIRE(opt->q_norm_g == nullptr || opt->q_norm_eps >= 0.f, "q_norm_eps must be >= 0");
  REQUIRE(opt->q_rope_dims + opt->out_rope_dims == 0 || opt->rope_base > 0.0, "rope_base must be > 0");
  a.splits = opt->splits;
  a.q_norm_g = opt->q_norm_g;
  a.q_norm_eps = opt->q_norm_eps;
  a.q_rope_dims = opt->q_rope_dims;
  a.out_rope_dims = opt->out_rope_dims;
  a.rope_base = opt->rope_base;
  if (opt->entry_pages != nullptr) {
    const csa_status_t st = check_pages(opt->entry_pages, a.n_entries, "entry_pages");
    if (st != CSA_OK) return st;
    a.pages = to_pages(opt->entry_pages);
  }
  if (opt->compress != nullptr) {
    const csa_compress_job_t* j = opt->compress;
    bool empty = false;
    const csa_status_t st = check_compress(j->Ca, j->Cb, j->Za, j->Zb, j->Ba, j->Bb, a.batch, j->n_tok, j->tok0,
                                           j->in_batch_stride, j->e0, j->n_out, j->dim, j->m, j->in_dt, j->out,
                                           j->out_sf, j->out_batch_stride, j->out_row0, j->out_dt, j->out_pages,
                                           &a.comp, &empty, j);
    if (st != CSA_OK) return st;
    a.has_comp = empty ? 0 : 1;
  }
  return CSA_OK;
}

csa_status_t check_mqa(const csa::MqaArgs& a) {
  REQUIRE(a.batch >= 0 && a.n_q >= 0 && a.n_entries >= 0 && a.win_len >= 0, "negative size");
  REQUIRE(a.m >= 1, "m=%d must be >= 1", a.m);
  REQUIRE(a.window >= 0 && a.window <= 4096, "window=%d out of range [0, 4096]", a.window);
  REQUIRE(a.n_heads >= 1 && a.n_heads <= 128, "n_heads=%d out of range [1, 128]", a.n_heads);
  REQUIRE(a.dim >= 64 && a.dim <= 512 && a.dim % 64 == 0, "dim=%d must be a multiple of 64 in [64, 512]",
          a.dim);
  REQUIRE(a.q_dt == CSA_F32 || a.q_dt == CSA_BF16, "q_dt must be F32 or BF16");
  REQUIRE(a.kv_dt == CSA_F32 || a.kv_dt == CSA_BF16 || a.kv_dt == CSA_KV_FP8MIX,
          "kv_dt must be F32, BF16 or KV_FP8MIX");
  REQUIRE(a.idx == nullptr || (a.k >= 1 && a.k <= 2048), "k=%d out of range [1, 2048]", a.k);
  return CSA_OK;
}

csa_status_t run_mqa(csa::MqaArgs& a, void* stream, const char* name) {
  g_launches = 0;
  csa_status_t st = check_mqa(a);
  if (st != CSA_OK) return st;
  if ((int64_t)a.batch * a.n_q == 0) return ok();
  REQUIRE_PTR(a.Q);
  REQUIRE_PTR(a.O);
  REQUIRE_PTR(a.q_pos);
  REQUIRE_PTR(a.sink);
  if (a.n_entries > 0) REQUIRE_PTR(a.entries);
  if (a.window > 0) {
    REQUIRE_PTR(a.win);
    REQUIRE_PTR(a.win_start);
  }
  if (a.q_norm_g != nullptr || a.q_rope_dims > 0 || a.out_rope_dims > 0) {
    if (!csa::mqa_tc_path(a))
      return fail(CSA_ERR_UNSUPPORTED,
                  "query normalisation / RoPE options need the tensor-core path (bf16 Q, BF16 or KV_FP8MIX rows, "
                  "dim 512, n_heads a multiple of 64)");
    if (a.q_norm_g != nullptr) REQUIRE_PTR(a.q_norm_g);
  }
  const size_t need = csa::mqa_workspace(a);
  REQUIRE(a.ws_bytes >= need, "workspace too small: %zu < %zu bytes", a.ws_bytes, need);
  if (need > 0) REQUIRE_PTR(a.ws);
  return cuda_status(csa::launch_mqa(a, static_cast<cudaStream_t>(stream)), name);
}

csa::MqaArgs mqa_args(const void* Q, csa_dtype_t q_dt, const void* entries, int64_t n_entries,
                      const int32_t* idx, int k, const void* win, int64_t win_len,
                      const int64_t* win_start, const int64_t* q_pos, int window, int m,
                      const float* sink, float scale, int batch, int n_q, int n_heads, int dim,
                      csa_dtype_t kv_dt, void* O, void* ws, size_t ws_bytes) {
  csa::MqaArgs a{};
  a.Q = Q; a.q_dt = (int)q_dt; a.entries = entries; a.n_entries = n_entries; a.idx = idx; a.k = k;
  a.win = win; a.win_len = win_len; a.win_start = win_start; a.q_pos = q_pos; a.window = window;
  a.m = m; a.sink = sink; a.scale = scale; a.batch = batch; a.n_q = n_q; a.n_heads = n_heads;
  a.dim = dim; a.kv_dt = (int)kv_dt; a.O = O; a.ws = ws; a.ws_bytes = ws_bytes;
  apply_mqa_options(a, nullptr);
  return a;
}

}  // namespace

extern "C" {

size_t csa_sparse_mqa_workspace_size(int batch, int n_q, int n_heads, int dim, int k, int window,
                                     csa_dtype_t q_dt, csa_dtype_t kv_dt) {
  csa::MqaArgs a = mqa_args(nullptr, q_dt, nullptr, 0, reinterpret_cast<const int32_t*>(16), k,
                            nullptr, 0, nullptr, nullptr, window, 1, nullptr, 1.f, batch, n_q,
                            n_heads, dim, kv_dt, nullptr, nullptr, 0);
  if (check_mqa(a) != CSA_OK || batch <= 0 || n_q <= 0) return 256;
  const size_t s = csa::mqa_workspace(a);
  return s < 256 ? 256 : s;
}

size_t csa_mqa_workspace_size(int batch, int n_q, int n_heads, int dim, int64_t rows_per_query,
                              csa_dtype_t q_dt, csa_dtype_t kv_dt, const csa_mqa_options_t* opt) {
  // a dense call whose row count per query is rows_per_query (window 0)
  csa::MqaArgs a = mqa_args(nullptr, q_dt, nullptr, rows_per_query < 0 ? 0 : rows_per_query, nullptr, 0, nullptr,
                            0, nullptr, nullptr, 0, 1, nullptr, 1.f, batch, n_q, n_heads, dim, kv_dt, nullptr,
                            nullptr, 0);
  // the block table does not change the workspace (rows_per_query is not an
  // entry count, so the table is not checked against it here)
  csa_mqa_options_t o{};
  if (opt != nullptr) {
    o = *opt;
    o.entry_pages = nullptr;
  }
  if (apply_mqa_options(a, opt ? &o : nullptr) != CSA_OK || check_mqa(a) != CSA_OK || batch <= 0 || n_q <= 0)
    return 256;
  const size_t s = csa::mqa_workspace(a);
  return s < 256 ? 256 : s;
}

csa_status_t csa_sparse_mqa_ex(const void* Q, csa_dtype_t q_dt, const void* entries,
                               int64_t n_entries, const int32_t* idx, int k, const void* win,
                               int64_t win_len, const int64_t* win_start, const int64_t* q_pos,
                               int window, int m, const float* sink, float softmax_scale, int batch,
                               int n_q, int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                               size_t ws_bytes, const csa_mqa_options_t* opt, void* stream) {
  g_launches = 0;
  if (idx == nullptr && (int64_t)batch * n_q > 0) return fail(CSA_ERR_INVALID_ARG, "idx is NULL");
  REQUIRE_ALIGNED_OR_NULL(idx);
  csa::MqaArgs a = mqa_args(Q, q_dt, entries, n_entries, idx, k, win, win_len, win_start, q_pos,
                            window, m, sink, softmax_scale, batch, n_q, n_heads, dim, kv_dt, O, ws,
                            ws_bytes);
  const csa_status_t st = apply_mqa_options(a, opt);
  if (st != CSA_OK) return st;
  return run_mqa(a, stream, "csa_sparse_mqa");
}

csa_status_t csa_sparse_mqa(const void* Q, csa_dtype_t q_dt, const void* entries,
                            int64_t n_entries, const int32_t* idx, int k, const void* win,
                            int64_t win_len, const int64_t* win_start, const int64_t* q_pos,
                            int window, int m, const float* sink, float softmax_scale, int batch,
                            int n_q, int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                            size_t ws_bytes, void* stream) {
  return csa_sparse_mqa_ex(Q, q_dt, entries, n_entries, idx, k, win, win_len, win_start, q_pos, window, m, sink,
                           softmax_scale, batch, n_q, n_heads, dim, kv_dt, O, ws, ws_bytes, nullptr, stream);
}

size_t hca_dense_mqa_workspace_size(int batch, int n_q, int n_heads, int dim, int64_t n_entries,
                                    int window, csa_dtype_t q_dt, csa_dtype_t kv_dt) {
  csa::MqaArgs a = mqa_args(nullptr, q_dt, nullptr, n_entries, nullptr, 0, nullptr, 0, nullptr,
                            nullptr, window, 1, nullptr, 1.f, batch, n_q, n_heads, dim, kv_dt,
                            nullptr, nullptr, 0);
  if (check_mqa(a) != CSA_OK || batch <= 0 || n_q <= 0) return 256;
  const size_t s = csa::mqa_workspace(a);
  return s < 256 ? 256 : s;
}

csa_status_t hca_dense_mqa_ex(const void* Q, csa_dtype_t q_dt, const void* entries,
                              int64_t n_entries, const void* win, int64_t win_len,
                              const int64_t* win_start, const int64_t* q_pos, int window, int m,
                              const float* sink, float softmax_scale, int batch, int n_q,
                              int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                              size_t ws_bytes, const csa_mqa_options_t* opt, void* stream) {
  g_launches = 0;
  csa::MqaArgs a = mqa_args(Q, q_dt, entries, n_entries, nullptr, 0, win, win_len, win_start, q_pos,
                            window, m, sink, softmax_scale, batch, n_q, n_heads, dim, kv_dt, O, ws,
                            ws_bytes);
  const csa_status_t st = apply_mqa_options(a, opt);
  if (st != CSA_OK) return st;
  return run_mqa(a, stream, "hca_dense_mqa");
}

csa_status_t hca_dense_mqa(const void* Q, csa_dtype_t q_dt, const void* entries,
                           int64_t n_entries, const void* win, int64_t win_len,
                           const int64_t* win_start, const int64_t* q_pos, int window, int m,
                           const float* sink, float softmax_scale, int batch, int n_q,
                           int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                           size_t ws_bytes, void* stream) {
  return hca_dense_mqa_ex(Q, q_dt, entries, n_entries, win, win_len, win_start, q_pos, window, m, sink,
                          softmax_scale, batch, n_q, n_heads, dim, kv_dt, O, ws, ws_bytes, nullptr, stream);
}

static csa_status_t check_out_proj(int T, int n_h, int c, int g, int d_g, int d) {
  REQUIRE(T >= 0 && T <= (1 << 24), "T=%d out of range [0, 2^24]", T);
  REQUIRE(n_h >= 1 && c >= 1 && g >= 1 && n_h % g == 0, "n_h=%d must be a positive multiple of g=%d", n_h, g);
  REQUIRE(g <= 65535, "g=%d too large (<= 65535)", g);
  REQUIRE((int64_t)(n_h / g) * c % 64 == 0 && (int64_t)n_h * c <= (1 << 20),
          "n_h/g * c = %lld must be a multiple of 64 (n_h * c <= 2^20)", (long long)(n_h / g) * c);
  REQUIRE(d_g >= 128 && d_g % 128 == 0 && (int64_t)g * d_g <= (1 << 20),
          "d_g=%d must be a multiple of 128 (g * d_g <= 2^20)", d_g);
  REQUIRE(d >= 128 && d % 128 == 0 && d <= (1 << 20), "d=%d must be a multiple of 128 (<= 2^20)", d);
  return CSA_OK;
}

size_t csa_grouped_out_proj_workspace_size(int T, int n_h, int c, int g, int d_g, int d) {
  if (check_out_proj(T, n_h, c, g, d_g, d) != CSA_OK || T == 0) return 256;
  const size_t s = csa::out_proj_workspace(T, n_h, c, g, d_g, d);
  return s < 256 ? 256 : s;
}

csa_status_t csa_grouped_out_proj_plan(int T, int n_h, int c, int g, int d_g, int d, int32_t* out) {
  REQUIRE(out != nullptr, "out is NULL");
  const csa_status_t st = check_out_proj(T, n_h, c, g, d_g, d);
  if (st != CSA_OK) return st;
  REQUIRE(T >= 1, "T must be >= 1");
  csa::out_proj_plan_info(T, n_h, c, g, d_g, d, out);
  return ok();
}

csa_status_t csa_grouped_out_proj(const void* O, const void* Wg, const void* Wo, void* Y, int T, int n_h, int c,
                                  int g, int d_g, int d, void* ws, size_t ws_bytes, void* stream) {
  g_launches = 0;
  const csa_status_t st = check_out_proj(T, n_h, c, g, d_g, d);
  if (st != CSA_OK) return st;
  if (T == 0) return ok();
  REQUIRE_PTR(O);
  REQUIRE_PTR(Wg);
  REQUIRE_PTR(Wo);
  REQUIRE_PTR(Y);
  REQUIRE_PTR(ws);
  const size_t need = csa_grouped_out_proj_workspace_size(T, n_h, c, g, d_g, d);
  REQUIRE(ws_bytes >= need, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  REQUIRE(Y != O && Y != ws && O != ws, "Y, O and ws must be distinct buffers");
  csa::OutProjArgs a{O, Wg, Wo, Y, T, n_h, c, g, d_g, d, ws};
  return cuda_status(csa::launch_out_proj(a, static_cast<cudaStream_t>(stream)), "csa_grouped_out_proj");
}

}  // extern "C"
