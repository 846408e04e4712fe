/*
 * csa_oracle.c -- float64 CPU oracle for the hybrid compressed attention
 * forward pass (CSA and HCA) of DeepSeek-V4.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
 * definition that the CUDA library is checked against.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg may load it.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * Sources (page titles and sections):
 *   [P5]  "DeepSeek-V4 内部机制" (LLM-101-CN deep dive), section 1.2 "CSA"
 *         (Step 1 compressor equations, Step 2 indexer score equation),
 *         section 1.3 "HCA", section 1.4 table (Q/KV normalisation, partial
 *         RoPE, sliding-window branch, attention sink with its softmax
 *         equation), section 1.5 (FP8/BF16 mixed KV storage, FP4 indexer),
 *         section 6.2 (FP4 indexer QK, BF16 index score), section 7 (state
 *         cache holds the uncompressed tail).
 *   [P1]  yunpan.plus write-up "CSA / HCA: 混合稀疏注意力机制", equations
 *         (6)-(11): Hadamard (per-channel) weighting, overlap of two groups,
 *         HCA without overlap.
 *   [P2]  admirer.cn article, "CSA——壓縮稀疏注意力" and "HCA——重度壓縮注意力":
 *         top-k 512/1024, 128-token window, sink logit in the denominator,
 *         RoPE dims BF16 / other dims FP8.
 *
 * Every floating-point step runs in double precision on inputs that are
 * already rounded/quantised (the formats are decoded exactly first).
 *
 * Readings where the pages are silent (all stated once more next to the code):
 *   - softmax axis: over the 2m (or m') token positions, separately for each
 *     channel d, which is what makes the Hadamard weights of one channel sum
 *     to 1;
 *   - entry 0 has no previous block: its b-branch is absent;
 *   - entries = floor(n/m); a trailing partial block is not compressed;
 *   - entry i is visible to the query at absolute position t iff
 *     m*(i+1)-1 <= t, i.e. i < floor((t+1)/m);
 *   - the window holds tokens max(0,t-W+1)..t, the query's own token included;
 *   - V = K for every attended row (shared KV), all dims;
 *   - the sink adds exp(z'_h) to the softmax denominator only;
 *   - top-k orders by (score desc, index asc) and pads with -1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "csa_oracle.h"

/* ------------------------------------------------------------------------ */
/* Number formats ([P5] section 1.5 and 6.2, [P2] RoPE/FP8 paragraph).       */
/* ------------------------------------------------------------------------ */

/* bfloat16: the upper half of an IEEE-754 binary32. */
double orc_bf16_decode(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bfloat16, ties to even (one rounding step). */
uint16_t orc_bf16_encode(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    /* bf16: 8 exponent bits (bias 127), 7 mantissa bits; subnormals down to 2^-133. */
    int e;
    frexp(a, &e);           /* a = f * 2^e, f in [0.5,1) */
    int E = e - 1;          /* floor(log2 a) */
    if (E < -126) E = -126; /* subnormal range keeps the quantum 2^-133 */
    double q = ldexp(1.0, E - 7);
    double r = rint(a / q) * q; /* default rounding mode: nearest, ties to even */
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80; /* overflow to infinity */
    float f = (float)r;         /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

double orc_round_bf16(double x) { return orc_bf16_decode(orc_bf16_encode(x)); }

/* OCP FP8 E4M3 ("fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no
 * infinities; S.1111.111 is NaN; largest finite value 448. */
double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, ex = (c >> 3) & 0xF, mt = c & 7;
    double v;
    if (ex == 0xF && mt == 7) return NAN;
    if (ex == 0) v = ldexp((double)mt, -9);              /* subnormal: mt * 2^-6 / 8 */
    else v = ldexp(1.0 + mt / 8.0, ex - 7);
    return s ? -v : v;
}

/* Nearest E4M3 value, ties to even, saturating at +-448. */
uint8_t orc_e4m3_encode(double x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int E = e - 1;
    if (E < -6) E = -6;                 /* below 2^-6 the quantum stays 2^-9 */
    double q = ldexp(1.0, E - 3);
    double r = rint(a / q) * q;
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -6)) return sign | (uint8_t)(r / ldexp(1.0, -9));
    frexp(r, &e);
    E = e - 1;
    int mt = (int)((r / ldexp(1.0, E) - 1.0) * 8.0);
    return sign | (uint8_t)(((E + 7) << 3) | mt);
}

/* FP4 E2M1: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} for codes 0..7, bit 3 = sign. */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_decode(uint8_t c) {
    double v = kE2M1[c & 7];
    return (c & 8) ? -v : v;
}

/* Nearest E2M1 value, ties to the even code, saturating at +-6. */
uint8_t orc_e2m1_encode(double x) {
    if (isnan(x)) return 0x7; /* no NaN in E2M1; not reached for finite data */
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs(x);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - kE2M1[c]);
        if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
    }
    return sign | (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* Row formats.                                                              */
/*   F32, BF16 : dim values.                                                 */
/*   FP8MIX    : KV entry with the last 64 (RoPE) dims in BF16 and the other */
/*               dim-64 dims in E4M3 with one fp32 scale per 64 dims         */
/*               ([P2] RoPE/FP8 paragraph; [P5] section 1.5).  Byte layout:  */
/*               [dim-64 E4M3 codes][64 bf16][(dim-64)/64 fp32 scales][pad]  */
/*               padded to a multiple of 16 bytes (608 bytes at dim 512).    */
/*               value = code * scale; scale = amax/448 (1 when amax = 0).   */
/*   NVFP4     : indexer q/K in E2M1 with one unsigned-E4M3 scale per 16     */
/*               values ([P5] section 6.2: FP4 QK path).  Two arrays:        */
/*               codes [rows][dim/2] (element 2j in the low nibble of byte   */
/*               j) and scales [rows][dim/16].  value = e2m1 * scale;        */
/*               scale = E4M3(amax/6); codes = E2M1(x / decoded scale).      */
/* ------------------------------------------------------------------------ */

int64_t orc_row_bytes(int dt, int dim) {
    switch (dt) {
    case ORC_F32: return 4LL * dim;
    case ORC_BF16: return 2LL * dim;
    case ORC_FP8MIX: {
        if (dim < 64 || (dim - 64) % 64 != 0) return -1;
        int64_t n8 = dim - 64;
        int64_t b = n8 + 128 + 4 * (n8 / 64);
        return (b + 15) / 16 * 16;
    }
    case ORC_NVFP4:
        if (dim % 16 != 0) return -1;
        return dim / 2;
    default: return -1;
    }
}

static void decode_fp8mix_row(const uint8_t* row, int dim, double* out) {
    int n8 = dim - 64;
    const uint8_t* bf = row + n8;
    const uint8_t* sc = row + n8 + 128;
    for (int j = 0; j < n8; ++j) {
        float s;
        memcpy(&s, sc + 4 * (j / 64), 4);
        out[j] = orc_e4m3_decode(row[j]) * (double)s;
    }
    for (int j = 0; j < 64; ++j) {
        uint16_t h;
        memcpy(&h, bf + 2 * j, 2);
        out[n8 + j] = orc_bf16_decode(h);
    }
}

static void encode_fp8mix_row(const double* x, int dim, uint8_t* row) {
    int n8 = dim - 64;
    int64_t rb = orc_row_bytes(ORC_FP8MIX, dim);
    memset(row, 0, (size_t)rb);
    for (int blk = 0; blk < n8 / 64; ++blk) {
        double amax = 0.0;
        for (int j = 0; j < 64; ++j) {
            double a = fabs(x[blk * 64 + j]);
            if (a > amax) amax = a;
        }
        float s = (amax > 0.0) ? (float)(amax / 448.0) : 1.0f;
        memcpy(row + n8 + 128 + 4 * blk, &s, 4);
        for (int j = 0; j < 64; ++j) row[blk * 64 + j] = orc_e4m3_encode(x[blk * 64 + j] / (double)s);
    }
    for (int j = 0; j < 64; ++j) {
        uint16_t h = orc_bf16_encode(x[n8 + j]);
        memcpy(row + n8 + 2 * j, &h, 2);
    }
}

static void decode_nvfp4_row(const uint8_t* codes, const uint8_t* sf, int dim, double* out) {
    for (int j = 0; j < dim; ++j) {
        uint8_t byte = codes[j / 2];
        uint8_t nib = (j & 1) ? (byte >> 4) : (byte & 0xF);
        out[j] = orc_e2m1_decode(nib) * orc_e4m3_decode(sf[j / 16]);
    }
}

static void encode_nvfp4_row(const double* x, int dim, uint8_t* codes, uint8_t* sf) {
    memset(codes, 0, (size_t)(dim / 2));
    for (int blk = 0; blk < dim / 16; ++blk) {
        double amax = 0.0;
        for (int j = 0; j < 16; ++j) {
            double a = fabs(x[blk * 16 + j]);
            if (a > amax) amax = a;
        }
        uint8_t s8 = orc_e4m3_encode(amax / 6.0);
        sf[blk] = s8;
        double s = orc_e4m3_decode(s8);
        for (int j = 0; j < 16; ++j) {
            int e = blk * 16 + j;
            uint8_t nib = (s > 0.0) ? orc_e2m1_encode(x[e] / s) : 0;
            codes[e / 2] |= (e & 1) ? (uint8_t)(nib << 4) : nib;
        }
    }
}

/* NVFP4 key-cache scale layout: rows are taken in blocks of 128; block b
 * holds dim/64 atoms of 512 bytes, and byte m0*16 + m1*4 + kk of atom a is the
 * scale of row 128*b + m0 + 32*m1 for values 64*a + 16*kk .. +15 (the layout
 * in which the tensor cores read block scales).  These two functions convert
 * between it and the row-major [rows][dim/16] layout; dim % 64 == 0. */
static int64_t blocked_scale_offset(int64_t r, int j, int dim) {
    int64_t blk = r / 128;
    int m = (int)(r % 128), m0 = m % 32, m1 = m / 32, atom = j / 4, kk = j % 4;
    return blk * (dim / 64) * 512 + (int64_t)atom * 512 + m0 * 16 + m1 * 4 + kk;
}

int64_t orc_nvfp4_blocked_bytes(int64_t n_rows, int dim) {
    if (dim % 64 != 0 || n_rows < 0) return -1;
    return (n_rows + 127) / 128 * (dim / 64) * 512;
}

int orc_nvfp4_unblock_scales(const uint8_t* blocked, int64_t n_rows, int dim, uint8_t* rowmajor) {
    if (dim % 64 != 0) return ORC_EINVAL;
    for (int64_t r = 0; r < n_rows; ++r)
        for (int j = 0; j < dim / 16; ++j)
            rowmajor[r * (dim / 16) + j] = blocked[blocked_scale_offset(r, j, dim)];
    return ORC_OK;
}

int orc_nvfp4_block_scales(const uint8_t* rowmajor, int64_t n_rows, int dim, uint8_t* blocked) {
    if (dim % 64 != 0) return ORC_EINVAL;
    memset(blocked, 0, (size_t)orc_nvfp4_blocked_bytes(n_rows, dim));
    for (int64_t r = 0; r < n_rows; ++r)
        for (int j = 0; j < dim / 16; ++j)
            blocked[blocked_scale_offset(r, j, dim)] = rowmajor[r * (dim / 16) + j];
    return ORC_OK;
}

int orc_decode_rows(const void* base, const void* sf, int dt, int dim, int64_t n_rows, double* out) {
    int64_t rb = orc_row_bytes(dt, dim);
    if (rb < 0) return ORC_EINVAL;
    const uint8_t* p = (const uint8_t*)base;
    for (int64_t r = 0; r < n_rows; ++r) {
        double* o = out + r * dim;
        switch (dt) {
        case ORC_F32:
            for (int j = 0; j < dim; ++j) { float f; memcpy(&f, p + r * rb + 4 * j, 4); o[j] = f; }
            break;
        case ORC_BF16:
            for (int j = 0; j < dim; ++j) { uint16_t h; memcpy(&h, p + r * rb + 2 * j, 2); o[j] = orc_bf16_decode(h); }
            break;
        case ORC_FP8MIX: decode_fp8mix_row(p + r * rb, dim, o); break;
        case ORC_NVFP4:
            if (!sf) return ORC_EINVAL;
            decode_nvfp4_row(p + r * rb, (const uint8_t*)sf + r * (dim / 16), dim, o);
            break;
        }
    }
    return ORC_OK;
}

int orc_encode_rows(const double* x, int dt, int dim, int64_t n_rows, void* out, void* sf) {
    int64_t rb = orc_row_bytes(dt, dim);
    if (rb < 0) return ORC_EINVAL;
    uint8_t* p = (uint8_t*)out;
    for (int64_t r = 0; r < n_rows; ++r) {
        const double* xr = x + r * dim;
        switch (dt) {
        case ORC_F32:
            for (int j = 0; j < dim; ++j) { float f = (float)xr[j]; memcpy(p + r * rb + 4 * j, &f, 4); }
            break;
        case ORC_BF16:
            for (int j = 0; j < dim; ++j) { uint16_t h = orc_bf16_encode(xr[j]); memcpy(p + r * rb + 2 * j, &h, 2); }
            break;
        case ORC_FP8MIX: encode_fp8mix_row(xr, dim, p + r * rb); break;
        case ORC_NVFP4:
            if (!sf) return ORC_EINVAL;
            encode_nvfp4_row(xr, dim, p + r * rb, (uint8_t*)sf + r * (dim / 16));
            break;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Token-level compressor ([P5] 1.2 Step 1; [P1] eq. 6-7; HCA: [P5] 1.3,     */
/* [P1] eq. 10-11).                                                          */
/*                                                                           */
/* For entry i and channel d the logits are                                  */
/*   Z^a[m i + j, d] + B^a[j, d]          j = 0..m-1   (current group)       */
/*   Z^b[m (i-1) + j, d] + B^b[j, d]      j = 0..m-1   (previous group,      */
/*                                                      CSA only, i >= 1)    */
/* S = softmax of all present logits of that channel, and                    */
/*   C^Comp[i, d] = sum_j S^a_j C^a[m i + j, d] + sum_j S^b_j C^b[...]       */
/* (Hadamard products: every channel is weighted on its own).                */
/*                                                                           */
/* Token rows hold absolute tokens tok0 .. tok0+n_tok-1.  Entries e0 ..      */
/* e0+n_out-1 are written to out[n_out][dim].  Cb == NULL selects the HCA    */
/* form (one branch, no overlap).  Returns ORC_EINVAL when a needed token    */
/* row is not present.                                                       */
/* ------------------------------------------------------------------------ */
int orc_compress(const double* Ca, const double* Cb, const double* Za, const double* Zb,
                 const double* Ba, const double* Bb, int64_t tok0, int64_t n_tok,
                 int64_t e0, int64_t n_out, int dim, int m, double* out) {
    if (m <= 0 || dim <= 0 || n_out < 0 || e0 < 0) return ORC_EINVAL;
    int overlap = (Cb != NULL);
    if (overlap && (Zb == NULL || Bb == NULL)) return ORC_EINVAL;
    double* lg = (double*)malloc(sizeof(double) * 2 * (size_t)m);
    double* cv = (double*)malloc(sizeof(double) * 2 * (size_t)m);
    for (int64_t ii = 0; ii < n_out; ++ii) {
        int64_t i = e0 + ii;
        int64_t first = (overlap && i >= 1) ? m * (i - 1) : m * i;
        int64_t last = m * (i + 1) - 1;
        if (first < tok0 || last >= tok0 + n_tok) { free(lg); free(cv); return ORC_EINVAL; }
        for (int d = 0; d < dim; ++d) {
            int n = 0;
            for (int j = 0; j < m; ++j) {
                int64_t r = m * i + j - tok0;
                lg[n] = Za[r * dim + d] + Ba[(int64_t)j * dim + d];
                cv[n] = Ca[r * dim + d];
                ++n;
            }
            if (overlap && i >= 1) {
                for (int j = 0; j < m; ++j) {
                    int64_t r = m * (i - 1) + j - tok0;
                    lg[n] = Zb[r * dim + d] + Bb[(int64_t)j * dim + d];
                    cv[n] = Cb[r * dim + d];
                    ++n;
                }
            }
            double mx = -INFINITY;
            for (int j = 0; j < n; ++j) if (lg[j] > mx) mx = lg[j];
            double den = 0.0;
            for (int j = 0; j < n; ++j) den += exp(lg[j] - mx);
            double acc = 0.0;
            for (int j = 0; j < n; ++j) acc += exp(lg[j] - mx) / den * cv[j];
            out[ii * dim + d] = acc;
        }
    }
    free(lg);
    free(cv);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Lightning indexer score ([P5] 1.2 Step 2; [P1] eq. 8):                    */
/*   I[t, s] = sum_h w[t, h] * ReLU(q[t, h] . K[s])                          */
/* q: [n_h][dim] (one query), w: [n_h], K: decoded [n_vis][dim].             */
/* ------------------------------------------------------------------------ */
void orc_index_scores(const double* q, const double* w, const double* K, int n_h, int dim,
                      int64_t n_vis, double* out) {
    for (int64_t s = 0; s < n_vis; ++s) {
        double I = 0.0;
        for (int h = 0; h < n_h; ++h) {
            double dot = 0.0;
            for (int d = 0; d < dim; ++d) dot += q[(int64_t)h * dim + d] * K[s * dim + d];
            I += w[h] * (dot > 0.0 ? dot : 0.0);
        }
        out[s] = I;
    }
}

/* ------------------------------------------------------------------------ */
/* Top-k selector ([P5] 1.2 Step 2; [P2] CSA paragraph: 512 / 1024).         */
/* The k entries that come first in the order (score desc, index asc); the   */
/* result is written in that order and padded with -1 when n < k.            */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int64_t i; } scored_t;

static int cmp_scored(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

int orc_topk(const double* score, int64_t n, int k, int32_t* idx) {
    if (k < 0 || n < 0) return ORC_EINVAL;
    scored_t* v = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) { v[i].s = score[i]; v[i].i = i; }
    qsort(v, (size_t)n, sizeof(scored_t), cmp_scored);
    for (int j = 0; j < k; ++j) idx[j] = (j < n) ? (int32_t)v[j].i : -1;
    free(v);
    return ORC_OK;
}

/* Entries visible to the query at absolute position t ([P5] 1.4 window row: */
/* a query cannot see its own, not yet complete, block): i < floor((t+1)/m). */
int64_t orc_visible_entries(int64_t t, int m, int64_t n_entries) {
    int64_t v = (t + 1) / m;
    if (v > n_entries) v = n_entries;
    if (v < 0) v = 0;
    return v;
}

/* Indexer + top-k for a batch of queries.
 *   qI [batch][n_q][n_hI][dI] decoded, wI [batch][n_q][n_hI],
 *   KI [batch][n_entries][dI] decoded, q_pos [batch][n_q] absolute positions.
 * scores_out (optional) [batch][n_q][n_entries]: the score of every visible
 * entry (rounded to bf16 when round_bf16), -inf for invisible entries.
 * idx_out [batch][n_q][k]. */
int orc_index_topk(const double* qI, const double* wI, const double* KI, const int64_t* q_pos,
                   int batch, int n_q, int n_hI, int dI, int64_t n_entries, int m, int k,
                   int round_bf16, double* scores_out, int32_t* idx_out) {
    double* sc = (double*)malloc(sizeof(double) * (size_t)(n_entries > 0 ? n_entries : 1));
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < n_q; ++t) {
            int64_t bt = (int64_t)b * n_q + t;
            int64_t vis = orc_visible_entries(q_pos[bt], m, n_entries);
            orc_index_scores(qI + bt * n_hI * dI, wI + bt * n_hI, KI + (int64_t)b * n_entries * dI,
                             n_hI, dI, vis, sc);
            if (round_bf16)
                for (int64_t s = 0; s < vis; ++s) sc[s] = orc_round_bf16(sc[s]);
            if (scores_out) {
                for (int64_t s = 0; s < n_entries; ++s)
                    scores_out[bt * n_entries + s] = (s < vis) ? sc[s] : -INFINITY;
            }
            orc_topk(sc, vis, k, idx_out + bt * k);
        }
    }
    free(sc);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Shared-KV attention of one query ([P5] 1.2 Step 2 "Shared-KV MQA", 1.4    */
/* sink equation; [P1] eq. 9):                                               */
/*   z_j = scale * <q_h, KV_j>,                                              */
/*   p_j = exp(z_j) / (sum_l exp(z_l) + exp(sink_h)),  o_h = sum_j p_j KV_j. */
/* The same row serves as key and value.  With no rows and sink = -inf, or   */
/* sink = +inf, the output is 0 (the limit of the expression).              */
/* ------------------------------------------------------------------------ */
void orc_attend(const double* q, int n_h, int dim, const double* KV, int64_t n_rows,
                const double* sink, double scale, double* out) {
    double* z = (double*)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1));
    for (int h = 0; h < n_h; ++h) {
        double* o = out + (int64_t)h * dim;
        for (int d = 0; d < dim; ++d) o[d] = 0.0;
        double sk = sink ? sink[h] : -INFINITY;
        if (isinf(sk) && sk > 0) continue;
        double mx = sk;
        for (int64_t j = 0; j < n_rows; ++j) {
            double dot = 0.0;
            for (int d = 0; d < dim; ++d) dot += q[(int64_t)h * dim + d] * KV[j * dim + d];
            z[j] = scale * dot;
            if (z[j] > mx) mx = z[j];
        }
        if (n_rows == 0 && isinf(sk)) continue;
        double den = exp(sk - mx);
        for (int64_t j = 0; j < n_rows; ++j) den += exp(z[j] - mx);
        for (int64_t j = 0; j < n_rows; ++j) {
            double p = exp(z[j] - mx) / den;
            for (int d = 0; d < dim; ++d) o[d] += p * KV[j * dim + d];
        }
    }
    free(z);
}

/* ------------------------------------------------------------------------ */
/* Q / KV-entry normalisation and partial RoPE ([P5] section 1.4 table:      */
/* RMSNorm on every query head and on the one compressed KV head before the  */
/* core attention; RoPE on the last 64 dims of q, of the KV rows and of the  */
/* output o_{t,i}, the output at position -i; [P2] RoPE paragraph).  The     */
/* pages give the operations, not their constants; the readings:             */
/*   - RMSNorm of a row x of c values: y_d = g_d x_d / sqrt(mean_d x_d^2 +   */
/*     eps), g a per-channel weight (all ones when g is NULL);               */
/*   - RoPE on the last R dims: pair k (k < R/2) is the adjacent pair        */
/*     (x_{c-R+2k}, x_{c-R+2k+1}), turned by the angle p * base^(-2k/R) as   */
/*     the complex number x_{c-R+2k} + i x_{c-R+2k+1} times e^{i angle};     */
/*     the first c-R dims are left as they are;                              */
/*   - the output of the query at position t is turned at position -t, so   */
/*     its RoPE dims carry positions relative to the query.                  */
/* ------------------------------------------------------------------------ */
int orc_rmsnorm(const double* x, int64_t n_rows, int dim, const double* g, double eps, double* y) {
    if (n_rows < 0 || dim < 1 || !(eps >= 0.0)) return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const double* xr = x + r * dim;
        double ss = 0.0;
        for (int d = 0; d < dim; ++d) ss += xr[d] * xr[d];
        double inv = 1.0 / sqrt(ss / dim + eps);
        for (int d = 0; d < dim; ++d) y[r * dim + d] = xr[d] * inv * (g ? g[d] : 1.0);
    }
    return 0;
}

int orc_rope_tail(const double* x, int64_t n_rows, int dim, int rope_dims, const double* pos, double base,
                  double* y) {
    if (n_rows < 0 || rope_dims < 0 || rope_dims % 2 || rope_dims > dim || !(base > 0.0)) return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const double* xr = x + r * dim;
        double* yr = y + r * dim;
        for (int d = 0; d < dim; ++d) yr[d] = xr[d];
        for (int k = 0; k < rope_dims / 2; ++k) {
            int i0 = dim - rope_dims + 2 * k;
            double angle = pos[r] * pow(base, -2.0 * k / rope_dims);
            double c = cos(angle), s = sin(angle);
            yr[i0] = xr[i0] * c - xr[i0 + 1] * s;
            yr[i0 + 1] = xr[i0] * s + xr[i0 + 1] * c;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Grouped output projection ([P5] section 1.2 Step 3): the n_h head outputs */
/* of a query are split into g groups of n_h/g consecutive heads; group j's  */
/* concatenated outputs (n_h/g * c values) are projected to d_g values by    */
/* its own matrix W_j, and the g results, concatenated, are projected to d   */
/* values by W_O.  Readings: plain linear maps, no bias, no activation      */
/* between the two projections, heads grouped in index order.               */
/*   O [T][n_h][c], Wg [g][n_h/g * c][d_g], Wo [g * d_g][d], Y [T][d].       */
/* ------------------------------------------------------------------------ */
int orc_grouped_out_proj(const double* O, int T, int n_h, int c, int g, int d_g, const double* Wg,
                         const double* Wo, int d, double* Y) {
    if (T < 0 || n_h < 1 || c < 1 || g < 1 || n_h % g || d_g < 1 || d < 1) return -1;
    const int64_t in_g = (int64_t)(n_h / g) * c;
    double* z = (double*)malloc(sizeof(double) * (size_t)g * d_g);
    if (!z) return -2;
    for (int t = 0; t < T; ++t) {
        const double* ot = O + (int64_t)t * n_h * c;
        for (int j = 0; j < g; ++j) {
            const double* x = ot + (int64_t)j * in_g;       /* heads j*n_h/g .. of query t */
            const double* w = Wg + (int64_t)j * in_g * d_g;
            for (int e = 0; e < d_g; ++e) {
                double acc = 0.0;
                for (int64_t i = 0; i < in_g; ++i) acc += x[i] * w[i * d_g + e];
                z[(int64_t)j * d_g + e] = acc;
            }
        }
        for (int o = 0; o < d; ++o) {
            double acc = 0.0;
            for (int64_t i = 0; i < (int64_t)g * d_g; ++i) acc += z[i] * Wo[i * d + o];
            Y[(int64_t)t * d + o] = acc;
        }
    }
    free(z);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Paged compressed cache ([P2] cache paragraph; [P5] section 7): the cache */
/* of every request is stored in fixed pages of lcm(m, m') = 128 tokens,    */
/* i.e. 32 CSA entries or 1 HCA entry per page, taken from a shared pool    */
/* through a per-request block table.  Reading: entry i of request b lives  */
/* in slot i % per_page of pool page table[b][i / per_page].  This gathers  */
/* the first n_entries entries of every request into a contiguous           */
/* [batch][n_entries] cache (rows of row_bytes bytes); -1 when a table slot */
/* is out of the pool.                                                       */
/* ------------------------------------------------------------------------ */
int orc_gather_paged(const uint8_t* pool, int64_t n_pages, int64_t row_bytes, int per_page,
                     const int32_t* table, int max_pages, int batch, int64_t n_entries, uint8_t* out) {
    if (n_pages < 0 || row_bytes < 1 || per_page < 1 || max_pages < 0 || batch < 0 || n_entries < 0) return -1;
    if (n_entries > (int64_t)max_pages * per_page) return -1;
    for (int b = 0; b < batch; ++b)
        for (int64_t i = 0; i < n_entries; ++i) {
            int32_t pg = table[(int64_t)b * max_pages + i / per_page];
            if (pg < 0 || pg >= n_pages) return -1;
            memcpy(out + ((int64_t)b * n_entries + i) * row_bytes,
                   pool + ((int64_t)pg * per_page + i % per_page) * row_bytes, (size_t)row_bytes);
        }
    return 0;
}

/* Gathers the attended rows of one query: `n_sel` entry rows listed in sel
 * (entries; -1 skipped), then the window tokens max(0,t-W+1)..t.  Returns the
 * row count, or -1 if a listed entry is not visible or a window token is not
 * present in the window buffer. */
static int64_t gather_rows(const uint8_t* entries, int kv_dt, int dim, int64_t n_entries,
                           const int32_t* sel, int64_t n_sel, int64_t vis,
                           const uint8_t* win, int64_t win_len, int64_t win_start, int64_t t,
                           int window, double* rows) {
    int64_t rb = orc_row_bytes(kv_dt, dim);
    int64_t n = 0;
    for (int64_t j = 0; j < n_sel; ++j) {
        int64_t e = sel ? sel[j] : j;
        if (e < 0) continue;
        if (e >= vis || e >= n_entries) return -1;
        orc_decode_rows(entries + e * rb, NULL, kv_dt, dim, 1, rows + n * dim);
        ++n;
    }
    int64_t lo = t - window + 1;
    if (lo < 0) lo = 0;
    for (int64_t u = lo; u <= t && window > 0; ++u) {
        int64_t r = u - win_start;
        if (r < 0 || r >= win_len) return -1;
        orc_decode_rows(win + r * rb, NULL, kv_dt, dim, 1, rows + n * dim);
        ++n;
    }
    return n;
}

/* CSA sparse shared-KV MQA over the selected entries plus the window.
 *   Q [batch][n_q][n_h][dim] decoded; entries [batch][n_entries] rows of
 *   kv_dt; idx [batch][n_q][k]; win [batch][win_len] rows of kv_dt whose row
 *   0 is absolute token win_start[b]; sink [n_h]; O [batch][n_q][n_h][dim]. */
int orc_sparse_mqa(const double* Q, const void* entries, int kv_dt, int64_t n_entries,
                   const int32_t* idx, int k, const void* win, int64_t win_len,
                   const int64_t* win_start, const int64_t* q_pos, int window, int m,
                   const double* sink, double scale, int batch, int n_q, int n_h, int dim, double* O) {
    int64_t rb = orc_row_bytes(kv_dt, dim);
    if (rb < 0 || kv_dt == ORC_NVFP4) return ORC_EINVAL;
    double* rows = (double*)malloc(sizeof(double) * (size_t)(k + window + 1) * dim);
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < n_q; ++t) {
            int64_t bt = (int64_t)b * n_q + t;
            int64_t vis = orc_visible_entries(q_pos[bt], m, n_entries);
            int64_t n = gather_rows((const uint8_t*)entries + (int64_t)b * n_entries * rb, kv_dt, dim,
                                    n_entries, idx + bt * k, k, vis,
                                    (const uint8_t*)win + (int64_t)b * win_len * rb, win_len,
                                    win_start[b], q_pos[bt], window, rows);
            if (n < 0) { free(rows); return ORC_EINVAL; }
            orc_attend(Q + bt * n_h * dim, n_h, dim, rows, n, sink, scale, O + bt * n_h * dim);
        }
    }
    free(rows);
    return ORC_OK;
}

/* HCA dense shared-KV MQA ([P5] 1.3: no top-k, every compressed entry) over
 * all visible entries plus the window.  Arguments as orc_sparse_mqa. */
int orc_hca_dense_mqa(const double* Q, const void* entries, int kv_dt, int64_t n_entries,
                      const void* win, int64_t win_len, const int64_t* win_start,
                      const int64_t* q_pos, int window, int m, const double* sink, double scale,
                      int batch, int n_q, int n_h, int dim, double* O) {
    int64_t rb = orc_row_bytes(kv_dt, dim);
    if (rb < 0 || kv_dt == ORC_NVFP4) return ORC_EINVAL;
    double* rows = (double*)malloc(sizeof(double) * (size_t)(n_entries + window + 1) * dim);
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < n_q; ++t) {
            int64_t bt = (int64_t)b * n_q + t;
            int64_t vis = orc_visible_entries(q_pos[bt], m, n_entries);
            int64_t n = gather_rows((const uint8_t*)entries + (int64_t)b * n_entries * rb, kv_dt, dim,
                                    n_entries, NULL, vis, vis,
                                    (const uint8_t*)win + (int64_t)b * win_len * rb, win_len,
                                    win_start[b], q_pos[bt], window, rows);
            if (n < 0) { free(rows); return ORC_EINVAL; }
            orc_attend(Q + bt * n_h * dim, n_h, dim, rows, n, sink, scale, O + bt * n_h * dim);
        }
    }
    free(rows);
    return ORC_OK;
}
