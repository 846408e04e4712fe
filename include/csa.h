/*
 * csa.h -- C ABI of libcsa_b200: the hybrid compressed attention forward pass
 * of DeepSeek-V4 (CSA: Compressed Sparse Attention, HCA: Heavily Compressed
 * Attention) on NVIDIA B200 (sm_100a).
 *
 * Passages defining the operations (page title, section, equation):
 *   [P5] "DeepSeek-V4 内部机制" (LLM-101-CN deep dive):
 *        1.2 Step 1 (compressor equations for S and C^Comp),
 *        1.2 Step 2 (index score I[t,s], top-k, shared-KV MQA),
 *        1.2 Step 3 (grouped output projection: g groups, d_g each),
 *        1.3 (HCA: m' tokens per entry, no overlap, no top-k),
 *        1.4 table and sink equation (window branch of n_win = 128 raw
 *        tokens, per-head sink logit in the softmax denominator),
 *        1.5 (RoPE dims BF16, other dims FP8; FP4 indexer),
 *        6.2 (FP4 indexer QK, scores quantised FP32 -> BF16 before top-k).
 *   [P1] yunpan.plus write-up "CSA / HCA: 混合稀疏注意力机制", eq. (6)-(11).
 *   [P2] admirer.cn article, CSA and HCA sections (top-k 512 / 1024,
 *        window 128, sink, mixed FP8/BF16 KV).
 *
 * Conventions shared by every call
 *   - All tensor arguments are DEVICE pointers owned by the caller; the
 *     library allocates no memory.  Scratch space is passed explicitly as
 *     (ws, ws_bytes); the matching *_workspace_size() call returns the
 *     minimum size.  Scratch must not be shared by calls that may overlap.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Host-side validation happens before any launch.
 *   - Tensors are dense, row-major, batch-major, with the shapes given below.
 *     Every device pointer must be 16-byte aligned.
 *   - Errors: a call returns CSA_ERR_INVALID_ARG (bad shape, NULL or
 *     misaligned pointer, workspace too small), CSA_ERR_UNSUPPORTED (a valid
 *     combination this build does not implement), or CSA_ERR_CUDA (a launch
 *     failed; the CUDA error string is in csa_last_error()).  Nothing aborts,
 *     prints or exits.  csa_last_error() is per host thread.
 *
 * Row formats (csa_dtype_t)
 *   CSA_F32        dim float32 values.
 *   CSA_BF16       dim bfloat16 values.
 *   CSA_KV_FP8MIX  KV entry / window row, dim = 64 * j + 64 (512 in the
 *                  workloads): bytes [0, dim-64) E4M3 codes of dims
 *                  0..dim-65; then 64 bf16 (128 bytes) for the RoPE dims
 *                  dim-64..dim-1; then (dim-64)/64 fp32 scales, one per 64
 *                  E4M3 dims; zero padding to a multiple of 16 bytes
 *                  (608 bytes per row at dim 512).  value = code * scale.
 *                  Writers use scale = amax/448 (1 when the block is zero)
 *                  and round to nearest even, saturating at +-448.
 *   CSA_IDX_NVFP4  indexer query/key rows as two arrays: codes
 *                  [rows][dim/2] bytes (element 2j in the low nibble of byte
 *                  j) and E4M3 scales, one per 16 values (dim a multiple of
 *                  64).  value = e2m1 * scale.  Writers use
 *                  scale = E4M3(amax/6) and codes = E2M1(x / scale), both
 *                  rounded to nearest even with saturation.
 *                  Query scales are row-major: [rows][dim/16].
 *                  Key-cache scales are BLOCKED, in the tensor core's
 *                  scale-factor atom layout, per request of n rows:
 *                  ceil(n/128) blocks of dim/64 atoms of 512 bytes
 *                  (csa_nvfp4_key_scale_bytes(n, dim) bytes); scale j of row
 *                  r sits at byte
 *                    (r/128)*(dim/64)*512 + (j/4)*512
 *                      + (r%32)*16 + ((r%128)/32)*4 + j%4.
 *                  Bytes of rows past n in the last block are never read
 *                  into a result.
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,
  CSA_ERR_UNSUPPORTED = 2,
  CSA_ERR_CUDA = 3,
  CSA_ERR_TIMEOUT = 4
} csa_status_t;

typedef enum {
  CSA_F32 = 0,
  CSA_BF16 = 1,
  CSA_KV_FP8MIX = 2,
  CSA_IDX_NVFP4 = 3
} csa_dtype_t;

/* Last error message of the calling host thread ("" after success). */
const char* csa_last_error(void);

/* Library ABI version (major * 100 + minor). */
int csa_version(void);

/* Number of kernels the calling thread's last compute call launched (0 when
 * it returned before launching). */
int csa_last_launch_count(void);

/* Synchronises the current device and reports whether any tensor-core kernel
 * gave up a bounded pipeline wait since the last check (CSA_ERR_TIMEOUT: the
 * results of the affected calls are invalid; the flag is cleared, and the
 * built-in scratch of csa_index_topk_noalloc on this device is zeroed again).
 * Kernels never spin without a limit, so a broken pipeline ends instead of
 * hanging. */
csa_status_t csa_check_device_status(void);

/* Bytes per row of format dt at dimension dim (codes only for NVFP4), or -1
 * when dim is not valid for the format. */
int64_t csa_row_bytes(csa_dtype_t dt, int dim);

/* Bytes of one request's blocked NVFP4 key-scale array of n_rows rows, or -1
 * when n_rows < 0 or dim is not a positive multiple of 64. */
int64_t csa_nvfp4_key_scale_bytes(int64_t n_rows, int dim);

/*
 * csa_pages_t -- a paged compressed cache ([P2] cache paragraph: the
 * compressed cache is kept in fixed pages of 128 tokens, lcm(m, m') for
 * m = 4, m' = 128, so a page holds 32 CSA entries or 1 HCA entry; [P5] 7).
 * The rows of every request live in pages of `page_entries` rows taken from
 * one pool shared by all requests; logical row r of request b is pool row
 *   table[b * max_pages + r / page_entries] * page_entries + r % page_entries.
 *   table         [batch][max_pages] int32 (device): pool page of each of the
 *                 request's pages.  Every slot j < ceil(rows / page_entries),
 *                 rows the call's logical rows per request, must hold a page
 *                 in [0, n_pages).  A kernel that meets a page outside the
 *                 pool touches no memory outside it (it drops the row, or
 *                 reads pool page 0 in its place), the call's results are
 *                 invalid, and csa_check_device_status reports
 *                 CSA_ERR_INVALID_ARG.
 *   max_pages     table row length (>= 1).
 *   page_entries  rows per page (>= 1).
 *   n_pages       pages in the pool (>= 1).
 * A paged call takes the POOL in place of the contiguous cache argument
 * (rows of the same format, n_pages * page_entries of them) and keeps its
 * logical row count argument (n_entries: rows the table maps per request,
 * <= max_pages * page_entries).  NVFP4 key scales of a paged key cache: one
 * blocked 128-row block (dim/64 atoms of 512 bytes) per pool page, so the
 * scale pool is n_pages * (dim/64) * 512 bytes; the scales of logical rows
 * 128u .. 128u+127 are kept in the block of the pool page that holds row
 * 128u, at the offset the contiguous layout gives row r % 128 (page_entries
 * must divide 128).
 */
typedef struct {
  const int32_t* table;
  int max_pages;
  int page_entries;
  int64_t n_pages;
} csa_pages_t;

/*
 * csa_compress -- Token-Level Compressor ([P5] 1.2 Step 1; [P1] eq. 6-7;
 * HCA form [P5] 1.3, [P1] eq. 10-11).
 *
 * For entry i and channel d, the logits of the current group
 * Z^a[m i + j, d] + B^a[j, d] (j < m) and, for CSA with i >= 1, of the
 * previous group Z^b[m (i-1) + j, d] + B^b[j, d] are soft-maxed together over
 * the token positions (per channel), and
 *   C^Comp[i, d] = sum_j S^a_j C^a[m i + j, d] + sum_j S^b_j C^b[m (i-1) + j, d].
 * Entry 0 has no previous group (its b-branch is absent).  Cb == NULL (and
 * Zb, Bb ignored) selects the HCA form: one branch, no overlap.
 * Arithmetic is fp32: per channel the largest logit M is found first, then
 * exp(logit - M) and exp(logit - M) * C are summed over the positions (the
 * current group's, then the previous group's) in blocks of 32, in order, and
 * their ratio is converted once to out_dt.  Every call shape takes these
 * steps in this order, so an entry's bytes do not depend on how many entries
 * a call produces or on which call (csa_compress_index_topk too) writes it.
 *
 *   Ca, Cb, Za, Zb  [batch][in_batch_stride rows][dim] of in_dt (F32/BF16);
 *                   row r of request b holds absolute token tok0 + r, and
 *                   rows 0..n_tok-1 are valid.
 *   Ba, Bb          [m][dim] fp32, indexed by position inside the group.
 *   e0, n_out       entries e0 .. e0+n_out-1 are produced; every token they
 *                   need, m*(e0-1) (or m*e0 without overlap / at e0 = 0) up
 *                   to m*(e0+n_out)-1, must lie in [tok0, tok0+n_tok).
 *   out             [batch][out_batch_stride rows] of out_dt (F32, BF16,
 *                   KV_FP8MIX, IDX_NVFP4): a cache of out_batch_stride rows
 *                   per request; entry i of request b is written to row
 *                   out_row0 + (i - e0) of request b (row
 *                   b*out_batch_stride + out_row0 + i - e0); other rows are
 *                   left untouched.  out_row0 + n_out <= out_batch_stride.
 *   out_sf          NVFP4 only (dim a multiple of 64): the cache's blocked
 *                   key scales, request b's array of
 *                   csa_nvfp4_key_scale_bytes(out_batch_stride, dim) bytes
 *                   starting at b times that size; only the written rows'
 *                   scale bytes change.
 */
csa_status_t csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                          const float* Ba, const float* Bb, int batch, int64_t n_tok,
                          int64_t tok0, int64_t in_batch_stride, int64_t e0, int64_t n_out,
                          int dim, int m, csa_dtype_t in_dt, void* out, void* out_sf,
                          int64_t out_batch_stride, int64_t out_row0, csa_dtype_t out_dt,
                          void* stream);

/*
 * csa_rmsnorm_rope -- Q / KV-entry normalisation and partial RoPE ([P5] 1.4
 * table: RMSNorm on every query head and on the one compressed KV head
 * before the core attention, RoPE on the last 64 dims of q, of the KV rows
 * and of the output, the output at position -i; [P2] RoPE paragraph), in one
 * pass over rows of dim values:
 *   g != NULL:  y = rope(g * x / sqrt(mean_d x_d^2 + eps))
 *   g == NULL:  y = rope(x)            (rotation only: e.g. an output at -t)
 * rope turns the last rope_dims dims of a row: pair k < rope_dims/2, the
 * adjacent dims (dim - rope_dims + 2k, dim - rope_dims + 2k + 1), by the
 * angle pos_sign * p * base^(-2k/rope_dims) (as the complex number
 * x_{2k} + i x_{2k+1} times e^{i angle}); p = pos[r / rows_per_pos] for row r.
 * The first dim - rope_dims dims are only normalised.  Normalisation runs in
 * fp32; angles are reduced in fp64, so large positions keep their accuracy.
 *
 *   x, y          [n_rows][dim] of in_dt / out_dt (CSA_F32 or CSA_BF16),
 *                 16-byte aligned.  y == x (in place) needs in_dt == out_dt;
 *                 otherwise y must not overlap x.
 *   g             [dim] fp32 per-channel weight, or NULL (no normalisation).
 *   pos           [ceil(n_rows / rows_per_pos)] int64 positions (e.g. the
 *                 query positions with rows_per_pos = n_heads, or the
 *                 position of each cache row); may be NULL when rope_dims = 0.
 *   pos_sign      +1, or -1 to turn rows back (the output of the query at t).
 * Limits: dim a positive multiple of 8; rope_dims a multiple of 8 in
 * [0, dim]; rows_per_pos >= 1; eps >= 0; base > 0.  Errors:
 * CSA_ERR_INVALID_ARG before any launch.
 */
csa_status_t csa_rmsnorm_rope(const void* x, void* y, int64_t n_rows, int dim, const float* g, float eps,
                              const int64_t* pos, int rows_per_pos, int pos_sign, int rope_dims, double base,
                              csa_dtype_t in_dt, csa_dtype_t out_dt, void* stream);

/*
 * csa_index_topk -- Lightning Indexer fused with the top-k selector ([P5] 1.2
 * Step 2; [P1] eq. 8; BF16 scores [P5] 6.2).
 *
 *   I[t, s] = sum_h wI[t, h] * ReLU(qI[t, h] . KI[s])
 * over the entries visible to query t: s < floor((q_pos[t] + 1) / m) (an
 * entry is visible once its whole group of m tokens is at or before t), and
 * s < n_entries.  The score is accumulated in fp32 and, for BF16 / NVFP4
 * inputs, rounded once to bf16 (nearest even) before selection; F32 inputs
 * keep fp32 scores.  The k entries first in the order (score desc, index asc)
 * are returned; with fewer than k visible entries the rest is -1.  The k
 * indices of a query are written in ascending index order.
 *
 *   qI        [batch][n_q][n_heads][dim] of dt; NVFP4: codes, with qI_sf
 *             [batch][n_q][n_heads][dim/16] scales.
 *   wI        [batch][n_q][n_heads] fp32 head weights.
 *   KI        [batch][n_entries][dim] of dt; NVFP4: codes, with KI_sf the
 *             blocked key scales, request b's array of
 *             csa_nvfp4_key_scale_bytes(n_entries, dim) bytes at b times
 *             that size.
 *   q_pos     [batch][n_q] int64 absolute position of each query.
 *   idx_out   [batch][n_q][k] int32 entry indices (per request).
 *   scores_out  optional (NULL in production): [batch][n_q][n_entries] of
 *             the selection scores (bf16, or fp32 for F32 inputs), -inf for
 *             entries not visible.  Used by tests to check selection.
 *   dt        CSA_F32, CSA_BF16 or CSA_IDX_NVFP4 (qI and KI share it).
 * Limits: 1 <= k <= 2048, dim a multiple of 32 (<= 256; NVFP4: of 64),
 * n_heads <= 128.
 * Workspace: ws must be zero-filled before its first use with this call
 * (e.g. one cudaMemset after allocation), because decode rows split over
 * several CTAs select together through counters and histograms kept there.
 * Every call that completes leaves the whole workspace zero-filled again
 * (the cooperative selection clears its counters, the merge of per-slice
 * candidates clears the candidate lists), so one workspace, large enough for
 * each shape, may serve calls of different shapes in turn.  After
 * CSA_ERR_TIMEOUT from csa_check_device_status, zero it again.
 */
size_t csa_index_topk_workspace_size(int batch, int n_q, int64_t n_entries, int k, int n_heads,
                                     int dim, csa_dtype_t dt);
csa_status_t csa_index_topk(const void* qI, const void* qI_sf, const float* wI, const void* KI,
                            const void* KI_sf, const int64_t* q_pos, int batch, int n_q,
                            int64_t n_entries, int m, int n_heads, int dim, int k, csa_dtype_t dt,
                            int32_t* idx_out, void* scores_out, void* ws, size_t ws_bytes,
                            void* stream);

/*
 * csa_index_topk_paged -- csa_index_topk over a paged key cache: KI (and
 * NVFP4 KI_sf) are the pool of key_pages (csa_pages_t), n_entries the logical
 * keys per request.  page_entries must be 8, 16, 32, 64 or 128 (a 128-token
 * page holds 32 keys at m = 4) and the pool below 2^31 rows.  Results are
 * those of csa_index_topk on the gathered contiguous cache; the workspace is
 * the same.  key_pages == NULL is csa_index_topk.
 */
csa_status_t csa_index_topk_paged(const void* qI, const void* qI_sf, const float* wI, const void* KI,
                                  const void* KI_sf, const csa_pages_t* key_pages, const int64_t* q_pos,
                                  int batch, int n_q, int64_t n_entries, int m, int n_heads, int dim, int k,
                                  csa_dtype_t dt, int32_t* idx_out, void* scores_out, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * csa_index_topk_plan -- how csa_index_topk divides the work of a call of
 * this shape on the current device (nothing is launched; for tests and
 * tuning).  out[6] receives: entries per slice, slices per query row, 1 when
 * the slices of a row select together (cooperative launch, no merge kernel),
 * 1 when the tensor-core producer runs (0: the SIMT producer), key stages in
 * the producer's shared-memory ring, and 128-entry tiles per stage.  A slice
 * of n entries streams ceil(n / (128 * tiles per stage)) stages through that
 * ring.  Errors: CSA_ERR_INVALID_ARG for the shapes csa_index_topk rejects.
 */
csa_status_t csa_index_topk_plan(int batch, int n_q, int64_t n_entries, int k, int n_heads, int dim,
                                 csa_dtype_t dt, int32_t* out);

/*
 * csa_compress_job_t -- the arguments of one csa_compress call, for calls
 * that run compressions inside another operation's launch.  Field meanings
 * are those of csa_compress; the request count comes from the enclosing call.
 */
typedef struct {
  const void *Ca, *Cb, *Za, *Zb;
  const float *Ba, *Bb;
  int64_t n_tok, tok0, in_batch_stride, e0, n_out;
  int dim, m;
  csa_dtype_t in_dt;
  void *out, *out_sf;
  int64_t out_batch_stride, out_row0;
  csa_dtype_t out_dt;
  /* NULL, or the block table of a paged output cache: `out` (and NVFP4
   * `out_sf`) are then the pool, out_batch_stride is ignored, and entry e0 + j
   * goes to logical row out_row0 + j of request b's pages (csa_pages_t;
   * NVFP4 needs page_entries dividing 128). */
  const csa_pages_t* out_pages;
  /* Entry normalisation and partial RoPE before the entry is stored ([P5]
   * 1.4 table: RMSNorm on the compressed KV entries, RoPE on their last 64
   * dims).  norm_g: NULL or [dim] fp32 RMSNorm weights (x <- g * x /
   * sqrt(mean(x^2) + norm_eps)); rope_dims: 0 or a multiple of 8 <= dim, the
   * last rope_dims dims turned at position pos_stride * i + pos_offset for
   * entry i (pos_stride = m, pos_offset = m - 1 puts an entry at its last
   * token), base rope_base.  The pooled fp32 row is normalised and turned
   * with the arithmetic of csa_rmsnorm_rope, then quantised once into out_dt,
   * so a BF16 entry equals csa_rmsnorm_rope applied to the F32 entry and
   * rounded.  A zero-filled tail (norm_g NULL, rope_dims 0) stores the
   * pooled row as csa_compress does. */
  const float* norm_g;
  float norm_eps;
  int rope_dims;
  double rope_base;
  int64_t pos_stride, pos_offset;
} csa_compress_job_t;

/* csa_compress with the arguments of one job (csa_compress_job_t), which may
 * write a paged cache through out_pages. */
csa_status_t csa_compress_ex(const csa_compress_job_t* job, int batch, void* stream);

/*
 * csa_compress_index_topk -- a decode step's compressions and indexer in one
 * call ([P5] 1.2 Step 1 and Step 2: the newly closed groups are compressed
 * into the KV cache and into the index-key cache K^I that the Lightning
 * Indexer then scores).
 *
 * Same results as csa_compress(*keys); csa_compress(*extra) (when extra is not
 * NULL); csa_index_topk(qI, ..., stream) -- every argument means what it
 * means there.  `keys` must write into the indexer's cache: keys->out == KI,
 * keys->out_sf == KI_sf, keys->out_dt == dt, keys->dim == dim,
 * keys->out_batch_stride == n_entries and keys->out_row0 == keys->e0 (entry i
 * is cache row i); `extra` (e.g. the KV cache's compression) must not write
 * what the indexer reads.  When keys->out_pages is not NULL the key cache is
 * paged: KI / KI_sf are its pool and the indexer reads it through that table
 * (as csa_index_topk_paged; out_batch_stride is then ignored); extra may write
 * a paged cache of its own.  With one query per request on the tensor-core
 * indexer this is one launch: the CTA whose slice of the cache holds the new
 * key rows starts its first key copies, runs both compressions of its request
 * while they land, and then streams the rest, so the compressions add no
 * dependent launch to the step.  Other shapes run the calls in order.  Errors
 * and workspace rules are those of the underlying calls.
 */
csa_status_t csa_compress_index_topk(const csa_compress_job_t* keys, const csa_compress_job_t* extra,
                                     const void* qI, const void* qI_sf, const float* wI, void* KI, void* KI_sf,
                                     const int64_t* q_pos, int batch, int n_q, int64_t n_entries, int m,
                                     int n_heads, int dim, int k, csa_dtype_t dt, int32_t* idx_out,
                                     void* scores_out, void* ws, size_t ws_bytes, void* stream);

/*
 * csa_index_topk_noalloc -- csa_index_topk for callers that cannot allocate
 * device memory.  The paper has no counterpart: this is a library service.
 *
 * Some callers have no allocator to draw a workspace from (a plugin inside a
 * host that owns all device memory, or a serving loop that forbids
 * cudaMalloc after start-up because it can synchronise the device).  This
 * call takes the same inputs and outputs as csa_index_topk, minus the
 * workspace, and runs the same kernels; its scratch is a 4 MiB array built
 * into the library, resident on every GPU that loads the library until the
 * process exits.  It calls no cudaMalloc, cudaFree or allocating routine.
 *   - Shapes whose csa_index_topk_workspace_size exceeds 4 MiB (4194304
 *     bytes) are rejected with CSA_ERR_INVALID_ARG before any launch.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address and caches it with the device's CUDA context
 *     (a new context, e.g. after cudaDeviceReset, is looked up again); make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents; calls that may overlap on the GPU (other streams or
 *     host threads) race on it, so serialise them.  It starts at zero (static
 *     initialisation) and every call that completes leaves it at zero, as
 *     csa_index_topk requires of its workspace.  A call whose selection timed
 *     out (CSA_ERR_TIMEOUT from csa_check_device_status) may leave counters
 *     set: csa_check_device_status zeroes the array of the current device
 *     when it reports the timeout, with a memset (nothing is allocated).
 */
csa_status_t csa_index_topk_noalloc(const void* qI, const void* qI_sf, const float* wI,
                                    const void* KI, const void* KI_sf, const int64_t* q_pos,
                                    int batch, int n_q, int64_t n_entries, int m, int n_heads,
                                    int dim, int k, csa_dtype_t dt, int32_t* idx_out,
                                    void* scores_out, void* stream);

/*
 * csa_sparse_mqa -- CSA core attention: shared-KV multi-query attention over
 * the selected compressed entries plus the sliding window, with a per-head
 * attention sink ([P5] 1.2 Step 2, 1.4 table rows "Sliding-Window" and
 * "Attention Sink" and the sink equation; [P1] eq. 9; [P2] CSA section).
 *
 * For query t and head h, the attended rows J are the entries idx[t, :]
 * (slots with -1 are unused) followed by the window tokens
 * max(0, t-window+1) .. t (the query's own token included).  Each row is both
 * key and value:
 *   z_j = softmax_scale * <Q[t, h], row_j>,
 *   O[t, h] = sum_j exp(z_j) row_j / (sum_j exp(z_j) + exp(sink[h])).
 *
 *   Q         [batch][n_q][n_heads][dim] of q_dt (F32 or BF16); O has the
 *             same shape and dtype.
 *   entries   [batch][n_entries] rows of kv_dt (F32, BF16, KV_FP8MIX).
 *   idx       [batch][n_q][k] int32; an index outside
 *             [0, min(n_entries, floor((q_pos+1)/m))) is ignored.
 *   win       [batch][win_len] rows of kv_dt; row r holds absolute token
 *             win_start[b] + r.  win_start [batch] int64 (device).  Every
 *             window token of every query must be present.
 *   q_pos     [batch][n_q] int64 (device); sink [n_heads] fp32 (device).
 * Limits: dim a multiple of 64 (<= 512), n_heads <= 128, k <= 2048.
 * Workspace: scratch for the split partials; no initialisation needed.
 */
size_t csa_sparse_mqa_workspace_size(int batch, int n_q, int n_heads, int dim, int k, int window,
                                     csa_dtype_t q_dt, csa_dtype_t kv_dt);
csa_status_t csa_sparse_mqa(const void* Q, csa_dtype_t q_dt, const void* entries,
                            int64_t n_entries, const int32_t* idx, int k, const void* win,
                            int64_t win_len, const int64_t* win_start, const int64_t* q_pos,
                            int window, int m, const float* sink, float softmax_scale, int batch,
                            int n_q, int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * csa_mqa_options_t -- options of the attention calls (the *_ex variants; a
 * NULL options pointer, or a zero-filled struct, gives the plain calls).
 *
 *   splits      0: the rows of a query are split over as many CTAs as fill
 *               the GPU for this batch (decode) -- the split count then
 *               depends on the batch, and so do the last bits of the output.
 *               n >= 1: batch-invariant decode ([P1] infrastructure section:
 *               batch-invariant kernels; [P5] 6.3): each query's rows are cut
 *               into min(n, ceil(rows / 128)) splits of whole 128-row chunks,
 *               where rows = k + window (sparse) or n_entries + window
 *               (dense), and the splits are added in split order -- the
 *               accumulation order of a query depends on its own rows only,
 *               so a request gives the same bytes in any batch.  n = 1 runs
 *               each query (per 64 heads) on one SM.  At most 256.
 *   q_norm_g    NULL, or [dim] fp32 RMSNorm weights applied to every query
 *               head before attention ([P5] 1.4 table: RMSNorm on the query
 *               heads): q <- g * q / sqrt(mean(q^2) + q_norm_eps), the
 *               arithmetic of csa_rmsnorm_rope (so the query the products use
 *               has exactly the bytes csa_rmsnorm_rope would give it).
 *   q_rope_dims RoPE dims turned on the query at its position q_pos (after
 *               the normalisation; 0 = none), as csa_rmsnorm_rope with
 *               rows_per_pos = n_heads and pos_sign = +1.
 *   out_rope_dims  RoPE dims of the output turned at -q_pos before the
 *               output is rounded ([P5] 1.4 table: the output at position
 *               -i); 0 = none.
 *   rope_base   RoPE base for both (e.g. 10000).
 *   entry_pages NULL, or the block table of a paged entry cache (csa_pages_t):
 *               `entries` is then the pool of n_pages * page_entries rows and
 *               n_entries the logical entries per request.  The window rows
 *               (the per-request state cache) stay contiguous.
 *   compress    NULL, or the step's entry compression ([P5] 1.3: the closed
 *               block of m' tokens becomes the newest HCA entry), launched on
 *               the same stream before the attention: one call for an HCA
 *               decode step, the same results as csa_compress_ex(job)
 *               followed by the attention call.
 * The normalisation and RoPE options need the tensor-core path (bf16 Q and
 * O, BF16 or KV_FP8MIX rows, dim 512, n_heads a multiple of 64) and
 * q_rope_dims, out_rope_dims multiples of 8 in [0, 64]; otherwise
 * CSA_ERR_UNSUPPORTED / CSA_ERR_INVALID_ARG before any launch.
 */
typedef struct {
  int splits;
  const float* q_norm_g;
  float q_norm_eps;
  int q_rope_dims;
  int out_rope_dims;
  double rope_base;
  const csa_pages_t* entry_pages;
  const csa_compress_job_t* compress;
} csa_mqa_options_t;

/*
 * csa_mqa_workspace_size -- workspace bytes of an attention call with these
 * options (rows_per_query = k + window for csa_sparse_mqa_ex, n_entries +
 * window for hca_dense_mqa_ex); scratch, no initialisation needed.
 */
size_t csa_mqa_workspace_size(int batch, int n_q, int n_heads, int dim, int64_t rows_per_query,
                              csa_dtype_t q_dt, csa_dtype_t kv_dt, const csa_mqa_options_t* opt);

/* csa_sparse_mqa with options (see csa_mqa_options_t). */
csa_status_t csa_sparse_mqa_ex(const void* Q, csa_dtype_t q_dt, const void* entries,
                               int64_t n_entries, const int32_t* idx, int k, const void* win,
                               int64_t win_len, const int64_t* win_start, const int64_t* q_pos,
                               int window, int m, const float* sink, float softmax_scale, int batch,
                               int n_q, int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                               size_t ws_bytes, const csa_mqa_options_t* opt, void* stream);

/*
 * hca_dense_mqa -- HCA core attention ([P5] 1.3: no top-k; every compressed
 * entry is attended) over all visible entries s < floor((q_pos+1)/m) plus
 * the window, with the sink, exactly as csa_sparse_mqa otherwise.
 */
size_t hca_dense_mqa_workspace_size(int batch, int n_q, int n_heads, int dim,
                                    int64_t n_entries, int window, csa_dtype_t q_dt,
                                    csa_dtype_t kv_dt);
csa_status_t hca_dense_mqa(const void* Q, csa_dtype_t q_dt, const void* entries,
                           int64_t n_entries, const void* win, int64_t win_len,
                           const int64_t* win_start, const int64_t* q_pos, int window, int m,
                           const float* sink, float softmax_scale, int batch, int n_q,
                           int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                           size_t ws_bytes, void* stream);

/* hca_dense_mqa with options (see csa_mqa_options_t). */
csa_status_t hca_dense_mqa_ex(const void* Q, csa_dtype_t q_dt, const void* entries,
                              int64_t n_entries, const void* win, int64_t win_len,
                              const int64_t* win_start, const int64_t* q_pos, int window, int m,
                              const float* sink, float softmax_scale, int batch, int n_q,
                              int n_heads, int dim, csa_dtype_t kv_dt, void* O, void* ws,
                              size_t ws_bytes, const csa_mqa_options_t* opt, void* stream);

/*
 * csa_grouped_out_proj -- grouped output projection after the core attention
 * ([P5] 1.2 Step 3: the n_h head outputs of a token, c values each, are cut
 * into g groups of n_h/g consecutive heads; each group is projected to d_g
 * values, the g results are concatenated and projected to d; V4-Pro: g = 16,
 * d_g = 1024, d = 7168).
 *
 *   Z[t, i*d_g + e] = sum_j O[t, i*(n_h/g)*c + j] * Wg[i][j][e]
 *   Y[t, o]         = sum_j Z[t, j] * Wo[j][o]
 *
 *   O    [T][n_h][c] bf16 (the attention output, heads in index order).
 *   Wg   [g][(n_h/g) * c][d_g] bf16, group i's weights at i.
 *   Wo   [g * d_g][d] bf16.
 *   Y    [T][d] bf16 output; distinct from O and ws.
 * Products accumulate in fp32; Z is rounded once to bf16 (round to nearest
 * even) before the second projection, Y once to bf16.  A sum split over
 * several CTAs adds its slices in a fixed order, so results depend only on
 * the shape (never on scheduling or on the device).
 * Limits: (n_h/g) * c a multiple of 64, d_g and d multiples of 128, T <= 2^24.
 * Workspace: csa_grouped_out_proj_workspace_size() bytes holding Z, fp32
 * partial sums and one counter per output tile.  The counters must be zero
 * before the first use (one cudaMemset after allocation); every call that
 * completes leaves them zero, so the workspace may serve calls of other
 * shapes in turn.  After CSA_ERR_TIMEOUT from csa_check_device_status, zero
 * it again.  T = 0 launches nothing.
 */
size_t csa_grouped_out_proj_workspace_size(int T, int n_h, int c, int g, int d_g, int d);
csa_status_t csa_grouped_out_proj(const void* O, const void* Wg, const void* Wo, void* Y, int T, int n_h, int c,
                                  int g, int d_g, int d, void* ws, size_t ws_bytes, void* stream);
/*
 * csa_grouped_out_proj_plan -- how csa_grouped_out_proj divides a call of
 * this shape (nothing is launched).  out[6] receives, for the group
 * projection then for the output projection: tokens per CTA, K slices per
 * output tile, CTAs launched.  Errors: as csa_grouped_out_proj, and T >= 1.
 */
csa_status_t csa_grouped_out_proj_plan(int T, int n_h, int c, int g, int d_g, int d, int32_t* out);

#ifdef __cplusplus
}
#endif
#endif /* CSA_B200_H */
