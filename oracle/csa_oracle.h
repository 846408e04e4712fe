/*
 * csa_oracle.h -- declarations of the float64 CPU oracle (test infrastructure
 * only; see csa_oracle.c for the definitions and the passages they follow).
 * This header belongs to the oracle alone: the CUDA library neither includes
 * it nor shares any of its constants.
 */
#ifndef CSA_ORACLE_H
#define CSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8MIX = 2, ORC_NVFP4 = 3 };
enum { ORC_OK = 0, ORC_EINVAL = -1 };

double orc_bf16_decode(uint16_t h);
uint16_t orc_bf16_encode(double x);
double orc_round_bf16(double x);
double orc_e4m3_decode(uint8_t c);
uint8_t orc_e4m3_encode(double x);
double orc_e2m1_decode(uint8_t c);
uint8_t orc_e2m1_encode(double x);

int64_t orc_row_bytes(int dt, int dim);
int orc_decode_rows(const void* base, const void* sf, int dt, int dim, int64_t n_rows, double* out);
int orc_encode_rows(const double* x, int dt, int dim, int64_t n_rows, void* out, void* sf);
int64_t orc_nvfp4_blocked_bytes(int64_t n_rows, int dim);
int orc_nvfp4_unblock_scales(const uint8_t* blocked, int64_t n_rows, int dim, uint8_t* rowmajor);
int orc_nvfp4_block_scales(const uint8_t* rowmajor, int64_t n_rows, int dim, uint8_t* blocked);

int orc_compress(const double* Ca, const double* Cb, const double* Za, const double* Zb,
                 const double* Ba, const double* Bb, int64_t tok0, int64_t n_tok,
                 int64_t e0, int64_t n_out, int dim, int m, double* out);

void orc_index_scores(const double* q, const double* w, const double* K, int n_h, int dim,
                      int64_t n_vis, double* out);
int orc_topk(const double* score, int64_t n, int k, int32_t* idx);
int64_t orc_visible_entries(int64_t t, int m, int64_t n_entries);
int orc_index_topk(const double* qI, const double* wI, const double* KI, const int64_t* q_pos,
                   int batch, int n_q, int n_hI, int dI, int64_t n_entries, int m, int k,
                   int round_bf16, double* scores_out, int32_t* idx_out);

int orc_rmsnorm(const double* x, int64_t n_rows, int dim, const double* g, double eps, double* y);
int orc_rope_tail(const double* x, int64_t n_rows, int dim, int rope_dims, const double* pos, double base,
                  double* y);

int orc_grouped_out_proj(const double* O, int T, int n_h, int c, int g, int d_g, const double* Wg,
                         const double* Wo, int d, double* Y);

int orc_gather_paged(const uint8_t* pool, int64_t n_pages, int64_t row_bytes, int per_page,
                     const int32_t* table, int max_pages, int batch, int64_t n_entries, uint8_t* out);

void orc_attend(const double* q, int n_h, int dim, const double* KV, int64_t n_rows,
                const double* sink, double scale, double* out);
int orc_sparse_mqa(const double* Q, const void* entries, int kv_dt, int64_t n_entries,
                   const int32_t* idx, int k, const void* win, int64_t win_len,
                   const int64_t* win_start, const int64_t* q_pos, int window, int m,
                   const double* sink, double scale, int batch, int n_q, int n_h, int dim, double* O);
int orc_hca_dense_mqa(const double* Q, const void* entries, int kv_dt, int64_t n_entries,
                      const void* win, int64_t win_len, const int64_t* win_start,
                      const int64_t* q_pos, int window, int m, const double* sink, double scale,
                      int batch, int n_q, int n_h, int dim, double* O);

#ifdef __cplusplus
}
#endif
#endif
