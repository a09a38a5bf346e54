/*
 * CPU ORACLE for 3D Block Sparse Attention (BSA) -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct restatement of what the method computes, used
 * only by the tests, by the benchmark's CPU-baseline leg and by the package's
 * smoke check. It shares no code, header, table or helper with the CUDA path.
 * Floating point is fp64 unless a function's `fp32` flag asks for the single
 * precision decision mode (selection decided in the GPU kernel's precision).
 *
 * Sources (page titles and sections):
 *   [P1] "LongCat-Video Technical Report" (paper summary page), section
 *        "Block Sparse Attention (BSA)": 3D block partitioning, pooled block
 *        similarity, top-r selection, masked softmax attention; section
 *        "Block Attention with KV-Cache for Efficient Multi-Task Inference":
 *        condition tokens attend only to condition tokens, noisy tokens to all.
 *   [P3] "LongCat-Video Technical Report #" (detail page), section
 *        "3D Block Sparse Attention": default chunk shape [4,4,8], Top-K and
 *        CDF-threshold selection modes.
 *
 * Readings where the pages are loose (each also listed in the design notes):
 *   - chunk shape (T,H,W) = (4,4,8), 128 tokens, for queries and keys alike;
 *   - [P1] counts the blocks per axis with a ceiling division, so a grid whose
 *     T, H or W is not a multiple of 4, 4, 8 has partial edge chunks: their
 *     missing tokens (local slots past the grid edge) do not exist -- pooling
 *     averages the chunk's existing tokens and attention ranges over existing
 *     keys only;
 *   - chunk index is 0-based over the rearranged sequence: chunk c holds the
 *     tokens of block (ct,ch,cw) with c = (ct*NH + ch)*NW + cw and local index
 *     (lt*4 + lh)*8 + lw (block order [N_T,N_H,N_W], intra-block order [t,h,w]);
 *   - masked logits are -inf, i.e. an exact softmax over the selected keys;
 *   - ties in selection go to the lower chunk index;
 *   - CDF: softmax of the pooled scores over the candidate set, descending
 *     order, smallest prefix with mass >= p, capped at max(1, floor(cap*|A|));
 *   - block-causal: a query chunk whose frames all lie below t_cond may only
 *     select condition chunks; other query chunks select among all chunks.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define CT 4
#define CH 4
#define CW 8
#define CN (CT * CH * CW)

static inline double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static int ceil_div(int n, int c) { return (n + c - 1) / c; }

/* [P1] 3D block partitioning with blocks of shape (st, sh, sw): chunks per axis
 * by ceiling division. */
int64_t oracle_num_chunks_shape(int T, int H, int W, int st, int sh, int sw) {
    return (int64_t)ceil_div(T, st) * ceil_div(H, sh) * ceil_div(W, sw);
}

/* Token index (THW order) of local slot l = (lt*sh + lh)*sw + lw of chunk c of
 * shape (st, sh, sw), or -1 when that slot of a partial edge chunk lies past
 * the grid. */
int64_t oracle_token_of_shape(int T, int H, int W, int st, int sh, int sw, int64_t c, int l) {
    const int NH = ceil_div(H, sh), NW = ceil_div(W, sw);
    const int64_t ct = c / ((int64_t)NH * NW);
    const int ch = (int)((c / NW) % NH);
    const int cw = (int)(c % NW);
    const int lt = l / (sh * sw), lh = (l / sw) % sh, lw = l % sw;
    const int64_t t = ct * st + lt, h = (int64_t)ch * sh + lh, w = (int64_t)cw * sw + lw;
    if (t >= T || h >= H || w >= W) return -1;
    return (t * H + h) * W + w;
}

/* The query chunk shape (4,4,8) of [P3]: */
int64_t oracle_num_chunks(int T, int H, int W) {
    return oracle_num_chunks_shape(T, H, W, CT, CH, CW);
}

int64_t oracle_token_of(int T, int H, int W, int64_t c, int l) {
    return oracle_token_of_shape(T, H, W, CT, CH, CW, c, l);
}

static int grid_ok(int T, int H, int W) { return T > 0 && H > 0 && W > 0; }

/* [P1] block-contiguous memory order (the tokens of a block made adjacent, in
 * [t,h,w] order inside the block): out[bh][c][l][:] = x[bh][token_of(c,l)][:]
 * (bf16 bits copied); the slots of missing tokens of partial chunks are zero. */
int oracle_rearrange(const uint16_t* x, int BH, int T, int H, int W, int d, uint16_t* out) {
    if (!x || !out || BH <= 0 || d <= 0 || !grid_ok(T, H, W)) return -1;
    const int64_t N = (int64_t)T * H * W, Nc = oracle_num_chunks(T, H, W);
    for (int bh = 0; bh < BH; ++bh)
        for (int64_t c = 0; c < Nc; ++c)
            for (int l = 0; l < CN; ++l) {
                const int64_t tok = oracle_token_of(T, H, W, c, l);
                uint16_t* o = out + (((int64_t)bh * Nc + c) * CN + l) * d;
                if (tok < 0)
                    memset(o, 0, sizeof(uint16_t) * (size_t)d);
                else
                    memcpy(o, x + ((int64_t)bh * N + tok) * d, sizeof(uint16_t) * (size_t)d);
            }
    return 0;
}

/* [P1] pooled representations: mean of the token vectors of a chunk (its
 * existing tokens: 128, fewer for a partial edge chunk). pooled[bh][c][:].
 * fp32 != 0: accumulate in float in local-token order. */
int oracle_pool_shape(const uint16_t* x, int BH, int T, int H, int W, int st, int sh, int sw,
                      int d, int fp32, double* pooled) {
    if (!x || !pooled || BH <= 0 || d <= 0 || !grid_ok(T, H, W) || st <= 0 || sh <= 0 || sw <= 0)
        return -1;
    const int64_t N = (int64_t)T * H * W, Nc = oracle_num_chunks_shape(T, H, W, st, sh, sw);
    const int n_slots = st * sh * sw;
#pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < BH; ++bh)
        for (int64_t c = 0; c < Nc; ++c) {
            double* o = pooled + ((int64_t)bh * Nc + c) * d;
            for (int e = 0; e < d; ++e) {
                double acc = 0.0;
                float accf = 0.0f;
                int n = 0;
                for (int l = 0; l < n_slots; ++l) {
                    const int64_t tok = oracle_token_of_shape(T, H, W, st, sh, sw, c, l);
                    if (tok < 0) continue;
                    const double v = bf16_to_double(x[((int64_t)bh * N + tok) * d + e]);
                    if (fp32) accf += (float)v; else acc += v;
                    ++n;
                }
                o[e] = fp32 ? (double)(accf * (1.0f / (float)n)) : acc / n;
            }
        }
    return 0;
}

int oracle_pool(const uint16_t* x, int BH, int T, int H, int W, int d, int fp32, double* pooled) {
    return oracle_pool_shape(x, BH, T, H, W, CT, CH, CW, d, fp32, pooled);
}

/* [P1] S_pool = Q_pool K_pool^T / sqrt(d) (scale passed in). S[bh][i][m] for Nq
 * query chunks and Nk key chunks. */
int oracle_scores(const double* qp, const double* kp, int BH, int Nq, int Nk, int d, double scale,
                  int fp32, double* S) {
    if (!qp || !kp || !S || BH <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < BH; ++bh)
        for (int i = 0; i < Nq; ++i) {
            const double* q = qp + ((int64_t)bh * Nq + i) * d;
            for (int m = 0; m < Nk; ++m) {
                const double* k = kp + ((int64_t)bh * Nk + m) * d;
                double s;
                if (fp32) {
                    float a = 0.0f;
                    for (int e = 0; e < d; ++e) a += (float)q[e] * (float)k[e];
                    s = (double)(a * (float)scale);
                } else {
                    double a = 0.0;
                    for (int e = 0; e < d; ++e) a += q[e] * k[e];
                    s = a * scale;
                }
                S[((int64_t)bh * Nq + i) * Nk + m] = s;
            }
        }
    return 0;
}

/* [P1] block-causal attention: a chunk is a condition chunk when every frame of
 * it lies below t_cond. */
static int is_condition_chunk(int H, int W, int st, int sh, int sw, int64_t c, int t_cond) {
    const int64_t ct = c / ((int64_t)ceil_div(H, sh) * ceil_div(W, sw));
    return (ct * st + st - 1) < t_cond;
}

typedef struct {
    double s;
    int idx;
} cand_t;

/* descending score, then ascending index */
static int cand_cmp(const void* a, const void* b) {
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int int_cmp(const void* a, const void* b) {
    const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Block selection over the scores S[bh][i][m] -> CSR in row order (bh, i), for
 * query chunks of shape (qst, qsh, qsw) and key chunks of shape (kst, ksh, ksw)
 * ([P1] block-size robustness: query blocks of 64 or 128 tokens, key blocks of
 * 64 to 1024).
 * mode 0 = top-k ([P1] top-r; [P3] Top-K), mode 1 = CDF ([P3] CDF threshold;
 * [P1] CDF-p: walk the chunks from the highest pooled score down and stop as
 * soon as their softmax mass adds up to p or more), mode 2 = combination ([P3] names a combined mode next to Top-K
 * and the CDF threshold without defining it; read as: a chunk is kept when
 * both rules keep it, i.e. the first min(k, CDF count) chunks of the common
 * descending order). k is clamped to |A(i)|. fp32 != 0 takes the CDF
 * decision in float arithmetic (scores are already float-valued then).
 * Column indices of a row are written in ascending order.
 * Returns nnz >= 0, or -1 on bad arguments, -2 if col_cap is too small.
 */
int64_t oracle_select_qk(const double* S, int BH, int T, int H, int W, int qst, int qsh, int qsw,
                         int kst, int ksh, int ksw, int t_cond, int mode, int topk, double cdf_p,
                         double cap_frac, int fp32, int32_t* row_ptr, int32_t* col_idx,
                         int64_t col_cap) {
    if (!S || !row_ptr || !col_idx || BH <= 0 || !grid_ok(T, H, W) || t_cond < 0 || qst <= 0 ||
        qsh <= 0 || qsw <= 0 || t_cond % qst != 0 || kst <= 0 || ksh <= 0 || ksw <= 0 ||
        t_cond % kst != 0 || mode < 0 || mode > 2 || (mode != 1 && topk <= 0))
        return -1;
    const int Nq = (int)oracle_num_chunks_shape(T, H, W, qst, qsh, qsw);  /* query chunks */
    const int Nk = (int)oracle_num_chunks_shape(T, H, W, kst, ksh, ksw);  /* key chunks */
    cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)Nk);
    int32_t* pick = (int32_t*)malloc(sizeof(int32_t) * (size_t)Nk);
    if (!cand || !pick) {
        free(cand);
        free(pick);
        return -1;
    }
    int64_t nnz = 0;
    row_ptr[0] = 0;
    for (int bh = 0; bh < BH; ++bh) {
        for (int i = 0; i < Nq; ++i) {
            const double* row = S + ((int64_t)bh * Nq + i) * Nk;
            const int q_cond = t_cond > 0 && is_condition_chunk(H, W, qst, qsh, qsw, i, t_cond);
            int na = 0;
            for (int m = 0; m < Nk; ++m) {
                if (q_cond && !is_condition_chunk(H, W, kst, ksh, ksw, m, t_cond)) continue;
                cand[na].s = row[m];
                cand[na].idx = m;
                ++na;
            }
            qsort(cand, (size_t)na, sizeof(cand_t), cand_cmp);
            int count;
            if (mode == 0) {
                count = topk < na ? topk : na;
            } else {
                /* softmax over A(i) of the scores, in the chosen precision */
                int mstar = na;
                if (fp32) {
                    const float mx = (float)cand[0].s;
                    float z = 0.0f;
                    for (int a = 0; a < na; ++a) z += expf((float)cand[a].s - mx);
                    float cum = 0.0f;
                    for (int a = 0; a < na; ++a) {
                        cum += expf((float)cand[a].s - mx) / z;
                        if (cum >= (float)cdf_p) { mstar = a + 1; break; }
                    }
                } else {
                    const double mx = cand[0].s;
                    double z = 0.0;
                    for (int a = 0; a < na; ++a) z += exp(cand[a].s - mx);
                    double cum = 0.0;
                    for (int a = 0; a < na; ++a) {
                        cum += exp(cand[a].s - mx) / z;
                        if (cum >= cdf_p) { mstar = a + 1; break; }
                    }
                }
                int cap = (int)floor(cap_frac * na);
                if (cap < 1) cap = 1;
                count = mstar < cap ? mstar : cap;
                /* combination (the reading taken of [P3]'s combined mode): a chunk is
                   kept when both rules keep it; both are prefixes of the same order */
                if (mode == 2 && topk < count) count = topk;
            }
            if (nnz + count > col_cap) {
                free(cand);
                free(pick);
                return -2;
            }
            for (int a = 0; a < count; ++a) pick[a] = cand[a].idx;
            qsort(pick, (size_t)count, sizeof(int32_t), int_cmp);
            memcpy(col_idx + nnz, pick, sizeof(int32_t) * (size_t)count);
            nnz += count;
            row_ptr[(int64_t)bh * Nq + i + 1] = (int32_t)nnz;
        }
    }
    free(cand);
    free(pick);
    return nnz;
}

/* Query chunks of the [P3] shape (4,4,8), key chunks (kst, ksh, ksw). */
int64_t oracle_select_shape(const double* S, int BH, int T, int H, int W, int kst, int ksh, int ksw,
                            int t_cond, int mode, int topk, double cdf_p, double cap_frac, int fp32,
                            int32_t* row_ptr, int32_t* col_idx, int64_t col_cap) {
    return oracle_select_qk(S, BH, T, H, W, CT, CH, CW, kst, ksh, ksw, t_cond, mode, topk, cdf_p,
                            cap_frac, fp32, row_ptr, col_idx, col_cap);
}

int64_t oracle_select(const double* S, int BH, int T, int H, int W, int t_cond, int mode,
                      int topk, double cdf_p, double cap_frac, int fp32, int32_t* row_ptr,
                      int32_t* col_idx, int64_t col_cap) {
    return oracle_select_shape(S, BH, T, H, W, CT, CH, CW, t_cond, mode, topk, cdf_p, cap_frac,
                               fp32, row_ptr, col_idx, col_cap);
}

/*
 * [P1] sparse attention: O = softmax(Q K^T / sqrt(d) with non-selected logits
 * at -inf) V, evaluated for the query chunks (shape (qst, qsh, qsw), Nc of them
 * per (batch, head)) listed in rows[] (row r = bh*Nc+i) over the tokens of the
 * key chunks (shape (kst, ksh, ksw)) in CSR row r. All arithmetic in fp64.
 * out[n][l][:] (l < qst*qsh*qsw) is the output of local query l of rows[n]; lse[n][l] is the
 * natural-log log-sum-exp of the scaled logits (nullable). A row with no
 * selected chunk yields zeros and lse = -inf. Keys are the existing tokens of
 * the selected chunks; a local query slot past the grid edge (partial chunk)
 * has no output: NaN.
 */
int oracle_attend_qk(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int T,
                     int H, int W, int qst, int qsh, int qsw, int kst, int ksh, int ksw, int d,
                     double scale, const int32_t* row_ptr, const int32_t* col_idx,
                     const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    if (!q || !k || !v || !row_ptr || !col_idx || !rows || !out || BH <= 0 || d <= 0 ||
        !grid_ok(T, H, W) || qst <= 0 || qsh <= 0 || qsw <= 0 || kst <= 0 || ksh <= 0 || ksw <= 0)
        return -1;
    const int kn = kst * ksh * ksw;  /* slots of a key chunk */
    const int qn = qst * qsh * qsw;  /* slots of a query chunk */
    const int64_t N = (int64_t)T * H * W, Nc = oracle_num_chunks_shape(T, H, W, qst, qsh, qsw);
    int bad = 0;
#pragma omp parallel
    {
        double* kd = NULL;
        double* vd = NULL;
        double* s = NULL;
        double* qd = (double*)malloc(sizeof(double) * (size_t)d);
        int64_t cap_keys = 0;
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < n_rows; ++n) {
            const int64_t r = rows[n];
            if (r < 0 || r >= (int64_t)BH * Nc) { bad = 1; continue; }
            const int64_t bh = r / Nc, i = r % Nc;
            const int64_t beg = row_ptr[r], end = row_ptr[r + 1];
            const int64_t slots = (end - beg) * kn;
            if (slots > cap_keys) {
                free(kd); free(vd); free(s);
                kd = (double*)malloc(sizeof(double) * (size_t)(slots * d));
                vd = (double*)malloc(sizeof(double) * (size_t)(slots * d));
                s = (double*)malloc(sizeof(double) * (size_t)slots);
                cap_keys = slots;
            }
            /* keys: every existing token of every selected chunk */
            int64_t nk = 0;
            for (int64_t e = beg; e < end; ++e) {
                const int64_t c = col_idx[e];
                for (int l = 0; l < kn; ++l) {
                    const int64_t tok = oracle_token_of_shape(T, H, W, kst, ksh, ksw, c, l);
                    if (tok < 0) continue;
                    const int64_t j = nk++;
                    for (int x = 0; x < d; ++x) {
                        kd[j * d + x] = bf16_to_double(k[(bh * N + tok) * d + x]);
                        vd[j * d + x] = bf16_to_double(v[(bh * N + tok) * d + x]);
                    }
                }
            }
            for (int lq = 0; lq < qn; ++lq) {
                const int64_t qtok = oracle_token_of_shape(T, H, W, qst, qsh, qsw, i, lq);
                double* o = out + (n * qn + lq) * d;
                if (qtok < 0) {
                    for (int x = 0; x < d; ++x) o[x] = NAN;
                    if (lse) lse[n * qn + lq] = NAN;
                    continue;
                }
                for (int x = 0; x < d; ++x) qd[x] = bf16_to_double(q[(bh * N + qtok) * d + x]);
                if (nk == 0) {
                    for (int x = 0; x < d; ++x) o[x] = 0.0;
                    if (lse) lse[n * qn + lq] = -INFINITY;
                    continue;
                }
                double mx = -INFINITY;
                for (int64_t j = 0; j < nk; ++j) {
                    double a = 0.0;
                    for (int x = 0; x < d; ++x) a += qd[x] * kd[j * d + x];
                    s[j] = a * scale;
                    if (s[j] > mx) mx = s[j];
                }
                double z = 0.0;
                for (int64_t j = 0; j < nk; ++j) {
                    s[j] = exp(s[j] - mx);
                    z += s[j];
                }
                for (int x = 0; x < d; ++x) o[x] = 0.0;
                for (int64_t j = 0; j < nk; ++j) {
                    const double w = s[j] / z;
                    for (int x = 0; x < d; ++x) o[x] += w * vd[j * d + x];
                }
                if (lse) lse[n * qn + lq] = mx + log(z);
            }
        }
        free(kd); free(vd); free(s); free(qd);
    }
    return bad ? -1 : 0;
}

/* Query chunks of the [P3] shape (4,4,8), key chunks (kst, ksh, ksw). */
int oracle_attend_shape(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int T,
                        int H, int W, int kst, int ksh, int ksw, int d, double scale,
                        const int32_t* row_ptr, const int32_t* col_idx, const int64_t* rows,
                        int64_t n_rows, double* out, double* lse) {
    return oracle_attend_qk(q, k, v, BH, T, H, W, CT, CH, CW, kst, ksh, ksw, d, scale, row_ptr,
                            col_idx, rows, n_rows, out, lse);
}

int oracle_attend(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int T, int H,
                  int W, int d, double scale, const int32_t* row_ptr, const int32_t* col_idx,
                  const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    return oracle_attend_shape(q, k, v, BH, T, H, W, CT, CH, CW, d, scale, row_ptr, col_idx, rows,
                               n_rows, out, lse);
}

/*
 * Dense attention over the token sequence in THW order, with the block-causal
 * rule of [P1] ("Block Attention with KV-Cache"): a query in a frame below
 * t_cond attends to the keys of frames below t_cond; every other query attends
 * to all keys (t_cond = 0: plain dense attention). qtok[n] = bh*N + token.
 * out[n][:], lse[n] (nullable). fp64.
 */
int oracle_dense(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int T, int H,
                 int W, int d, double scale, int t_cond, const int64_t* qtok, int64_t n_q,
                 double* out, double* lse) {
    if (!q || !k || !v || !qtok || !out || BH <= 0 || T <= 0 || H <= 0 || W <= 0 || d <= 0 ||
        t_cond < 0)
        return -1;
    const int64_t N = (int64_t)T * H * W, HW = (int64_t)H * W;
    int bad = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* qd = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < n_q; ++n) {
            const int64_t g = qtok[n];
            if (g < 0 || g >= (int64_t)BH * N) { bad = 1; continue; }
            const int64_t bh = g / N, tok = g % N;
            const int64_t t = tok / HW;
            const int64_t nkeys = (t_cond > 0 && t < t_cond) ? (int64_t)t_cond * HW : N;
            for (int x = 0; x < d; ++x) qd[x] = bf16_to_double(q[g * d + x]);
            double mx = -INFINITY;
            for (int64_t j = 0; j < nkeys; ++j) {
                const uint16_t* kr = k + (bh * N + j) * d;
                double a = 0.0;
                for (int x = 0; x < d; ++x) a += qd[x] * bf16_to_double(kr[x]);
                s[j] = a * scale;
                if (s[j] > mx) mx = s[j];
            }
            double z = 0.0;
            for (int64_t j = 0; j < nkeys; ++j) {
                s[j] = exp(s[j] - mx);
                z += s[j];
            }
            double* o = out + n * d;
            for (int x = 0; x < d; ++x) o[x] = 0.0;
            for (int64_t j = 0; j < nkeys; ++j) {
                const uint16_t* vr = v + (bh * N + j) * d;
                const double w = s[j] / z;
                for (int x = 0; x < d; ++x) o[x] += w * bf16_to_double(vr[x]);
            }
            if (lse) lse[n] = mx + log(z);
        }
        free(s);
        free(qd);
    }
    return bad ? -1 : 0;
}

/*
 * Gradients of the block-sparse attention of oracle_attend ([P1] "Block Sparse
 * Attention (BSA)", sparse attention computation: O = softmax(QK^T/sqrt(d) with
 * non-selected logits at -inf) V; [P3] section "开源实现" lists the backward
 * kernels of the trainable BSA) for a scalar loss L whose gradient with
 * respect to O is dout. For a query token q with keys J (every token of the
 * chunks in its CSR row), written out by the chain rule through the softmax:
 *   P[q,j]  = exp(s[q,j] - LSE[q]),   s[q,j] = scale * <q, k_j>
 *   O[q]    = sum_j P[q,j] v_j
 *   dV[j]  += P[q,j] dout[q]
 *   dP[q,j] = <dout[q], v_j>
 *   Dq      = <dout[q], O[q]>          (= sum_j P[q,j] dP[q,j])
 *   dS[q,j] = P[q,j] (dP[q,j] - Dq)
 *   dQ[q]   = scale * sum_j dS[q,j] k_j
 *   dK[j]  += scale * dS[q,j] q
 * Inputs are fp64 [BH][N][d] in THW token order (callers widen bf16 exactly),
 * so the same routine serves finite-difference checks. Query chunks have shape
 * (qst,qsh,qsw) and key chunks (kst,ksh,ksw) ([P1] block-size robustness: query
 * blocks of 64 or 128 tokens); Nc counts the query chunks. The rows listed in
 * rows[] (r = bh*Nc + i) are processed: dq_rows[n][l][:] receives dQ of local
 * query l of rows[n]; dk and dv ([BH][N][d], zeroed by the caller) accumulate
 * the contributions of those rows only (complete for a key chunk when every
 * row that selects it is listed). A row with no selected chunk contributes
 * nothing and has dQ = 0. Keys and queries are the existing tokens of their
 * chunks; a local query slot past the grid edge has no dQ (NaN) and
 * contributes nothing. All arithmetic in fp64.
 */
int oracle_attend_bwd_qk(const double* q, const double* k, const double* v, const double* dout,
                         int BH, int T, int H, int W, int qst, int qsh, int qsw, int kst, int ksh,
                         int ksw, int d, double scale, const int32_t* row_ptr,
                         const int32_t* col_idx, const int64_t* rows, int64_t n_rows,
                         double* dq_rows, double* dk, double* dv) {
    if (!q || !k || !v || !dout || !row_ptr || !col_idx || !rows || !dq_rows || !dk || !dv ||
        BH <= 0 || d <= 0 || !grid_ok(T, H, W) || qst <= 0 || qsh <= 0 || qsw <= 0 || kst <= 0 ||
        ksh <= 0 || ksw <= 0)
        return -1;
    const int kn = kst * ksh * ksw;  /* slots of a key chunk */
    const int CQ = qst * qsh * qsw;  /* slots of a query chunk */
    const int64_t N = (int64_t)T * H * W, Nc = oracle_num_chunks_shape(T, H, W, qst, qsh, qsw);
    for (int64_t n = 0; n < n_rows; ++n)
        if (rows[n] < 0 || rows[n] >= (int64_t)BH * Nc) return -1;
    int64_t cap_keys = 0;
    int64_t* ktok = NULL;  /* token index of each key of the row */
    double* P = NULL;      /* [128][nk] softmax weights */
    double* dS = NULL;     /* [128][nk] */
    for (int64_t n = 0; n < n_rows; ++n) {
        const int64_t r = rows[n];
        const int64_t bh = r / Nc, i = r % Nc;
        const int64_t beg = row_ptr[r], end = row_ptr[r + 1];
        const int64_t slots = (end - beg) * kn;
        double* dqr = dq_rows + n * CQ * d;
        if (slots > cap_keys) {
            free(ktok); free(P); free(dS);
            ktok = (int64_t*)malloc(sizeof(int64_t) * (size_t)slots);
            P = (double*)malloc(sizeof(double) * (size_t)(CQ * slots));
            dS = (double*)malloc(sizeof(double) * (size_t)(CQ * slots));
            cap_keys = slots;
        }
        int64_t nk = 0;  /* existing key tokens of the row */
        for (int64_t e = beg; e < end; ++e)
            for (int l = 0; l < kn; ++l) {
                const int64_t tok = oracle_token_of_shape(T, H, W, kst, ksh, ksw, col_idx[e], l);
                if (tok >= 0) ktok[nk++] = bh * N + tok;
            }
        for (int lq = 0; lq < CQ; ++lq)
            if (oracle_token_of_shape(T, H, W, qst, qsh, qsw, i, lq) < 0)
                for (int x = 0; x < d; ++x) dqr[(int64_t)lq * d + x] = NAN;
        if (nk <= 0) {
            for (int lq = 0; lq < CQ; ++lq)
                if (oracle_token_of_shape(T, H, W, qst, qsh, qsw, i, lq) >= 0)
                    for (int x = 0; x < d; ++x) dqr[(int64_t)lq * d + x] = 0.0;
            continue;
        }
        /* per query: softmax weights, O, D, dS and dQ */
#pragma omp parallel for schedule(static)
        for (int lq = 0; lq < CQ; ++lq) {
            const int64_t qtok = oracle_token_of_shape(T, H, W, qst, qsh, qsw, i, lq);
            double* p = P + (int64_t)lq * nk;
            double* ds = dS + (int64_t)lq * nk;
            if (qtok < 0) {  /* no such query: no weights */
                for (int64_t j = 0; j < nk; ++j) p[j] = ds[j] = 0.0;
                continue;
            }
            const double* qr = q + (bh * N + qtok) * d;
            const double* gr = dout + (bh * N + qtok) * d;
            double mx = -INFINITY;
            for (int64_t j = 0; j < nk; ++j) {
                const double* kr = k + ktok[j] * d;
                double a = 0.0;
                for (int x = 0; x < d; ++x) a += qr[x] * kr[x];
                p[j] = a * scale;
                if (p[j] > mx) mx = p[j];
            }
            double z = 0.0;
            for (int64_t j = 0; j < nk; ++j) {
                p[j] = exp(p[j] - mx);
                z += p[j];
            }
            for (int64_t j = 0; j < nk; ++j) p[j] /= z;
            /* D = <dout, O> with O = sum_j P v_j; dP[j] = <dout, v_j> kept in ds */
            double D = 0.0;
            for (int64_t j = 0; j < nk; ++j) {
                const double* vr = v + ktok[j] * d;
                double a = 0.0;
                for (int x = 0; x < d; ++x) a += gr[x] * vr[x];
                ds[j] = a;
                D += p[j] * a;
            }
            double* dqq = dqr + (int64_t)lq * d;
            for (int x = 0; x < d; ++x) dqq[x] = 0.0;
            for (int64_t j = 0; j < nk; ++j) {
                ds[j] = p[j] * (ds[j] - D);
                const double* kr = k + ktok[j] * d;
                for (int x = 0; x < d; ++x) dqq[x] += ds[j] * kr[x];
            }
            for (int x = 0; x < d; ++x) dqq[x] *= scale;
        }
        /* per key: dV and dK contributions of this row's queries (keys of one
           row are distinct tokens, so the updates do not collide) */
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < nk; ++j) {
            double* dkr = dk + ktok[j] * d;
            double* dvr = dv + ktok[j] * d;
            for (int lq = 0; lq < CQ; ++lq) {
                const int64_t qtok = oracle_token_of_shape(T, H, W, qst, qsh, qsw, i, lq);
                if (qtok < 0) continue;
                const int64_t qt = bh * N + qtok;
                const double pw = P[(int64_t)lq * nk + j];
                const double sw = dS[(int64_t)lq * nk + j] * scale;
                const double* qr = q + qt * d;
                const double* gr = dout + qt * d;
                for (int x = 0; x < d; ++x) {
                    dvr[x] += pw * gr[x];
                    dkr[x] += sw * qr[x];
                }
            }
        }
    }
    free(ktok); free(P); free(dS);
    return 0;
}

int oracle_attend_bwd_shape(const double* q, const double* k, const double* v, const double* dout,
                            int BH, int T, int H, int W, int kst, int ksh, int ksw, int d,
                            double scale, const int32_t* row_ptr, const int32_t* col_idx,
                            const int64_t* rows, int64_t n_rows, double* dq_rows, double* dk,
                            double* dv) {
    return oracle_attend_bwd_qk(q, k, v, dout, BH, T, H, W, CT, CH, CW, kst, ksh, ksw, d, scale,
                                row_ptr, col_idx, rows, n_rows, dq_rows, dk, dv);
}

/*
 * The gradient contributions of one partition of the keys, for context
 * parallelism ([P1] "Block Sparse Attention (BSA)", ring block sparse
 * attention: the keys of a query are split across the ranks of the group; [P3]
 * "开源实现": the trainable BSA's backward kernels and the LSE correction for
 * context parallelism). The softmax of a query runs over ALL its keys, so its
 * weights on the keys of one partition need the whole set's log-sum-exp and
 * the whole output: with lse[q] (natural log) and out[q] of the full
 * attention,
 *   P[q,j]  = exp(s[q,j] - lse[q])          for the keys j of this partition
 *   Dq      = <dout[q], out[q]>
 *   dS[q,j] = P[q,j] (<dout[q], v_j> - Dq)
 *   dQ[q]   = scale * sum_j dS[q,j] k_j,  dK[j] += scale * dS[q,j] q,
 *   dV[j]  += P[q,j] dout[q]
 * and the gradients of the full attention are the sums of these over the
 * partitions (every term of the chain rule above is a sum over keys). The CSR
 * lists the partition's chunks per query row, in the key grid (T,H,W) and key
 * chunk shape (kst,ksh,ksw); q, dout, out, lse live on the query grid, which
 * has the same (T,H,W) (one rank's shard of queries against one shard of
 * keys). Outputs as oracle_attend_bwd_shape: dq_rows for the listed rows
 * (NaN for query slots past the grid edge, 0 for a row with no chunk of the
 * partition), dk/dv accumulated. fp64.
 */
int oracle_attend_bwd_part_shape(const double* q, const double* k, const double* v,
                                 const double* dout, const double* out, const double* lse, int BH,
                                 int T, int H, int W, int kst, int ksh, int ksw, int d,
                                 double scale, const int32_t* row_ptr, const int32_t* col_idx,
                                 const int64_t* rows, int64_t n_rows, double* dq_rows, double* dk,
                                 double* dv) {
    if (!q || !k || !v || !dout || !out || !lse || !row_ptr || !col_idx || !rows || !dq_rows ||
        !dk || !dv || BH <= 0 || d <= 0 || !grid_ok(T, H, W) || kst <= 0 || ksh <= 0 || ksw <= 0)
        return -1;
    const int kn = kst * ksh * ksw;
    const int64_t N = (int64_t)T * H * W, Nc = oracle_num_chunks(T, H, W);
    for (int64_t n = 0; n < n_rows; ++n)
        if (rows[n] < 0 || rows[n] >= (int64_t)BH * Nc) return -1;
    int64_t cap_keys = 0;
    int64_t* ktok = NULL;
    double* P = NULL;
    double* dS = NULL;
    for (int64_t n = 0; n < n_rows; ++n) {
        const int64_t r = rows[n];
        const int64_t bh = r / Nc, i = r % Nc;
        const int64_t beg = row_ptr[r], end = row_ptr[r + 1];
        const int64_t slots = (end - beg) * kn;
        double* dqr = dq_rows + n * CN * d;
        if (slots > cap_keys) {
            free(ktok); free(P); free(dS);
            ktok = (int64_t*)malloc(sizeof(int64_t) * (size_t)slots);
            P = (double*)malloc(sizeof(double) * (size_t)(CN * slots));
            dS = (double*)malloc(sizeof(double) * (size_t)(CN * slots));
            cap_keys = slots;
        }
        int64_t nk = 0;
        for (int64_t e = beg; e < end; ++e)
            for (int l = 0; l < kn; ++l) {
                const int64_t tok = oracle_token_of_shape(T, H, W, kst, ksh, ksw, col_idx[e], l);
                if (tok >= 0) ktok[nk++] = bh * N + tok;
            }
        for (int lq = 0; lq < CN; ++lq) {
            const int exists = oracle_token_of(T, H, W, i, lq) >= 0;
            for (int x = 0; x < d; ++x) dqr[(int64_t)lq * d + x] = exists ? 0.0 : NAN;
        }
        if (nk <= 0) continue;
#pragma omp parallel for schedule(static)
        for (int lq = 0; lq < CN; ++lq) {
            const int64_t qtok = oracle_token_of(T, H, W, i, lq);
            double* p = P + (int64_t)lq * nk;
            double* ds = dS + (int64_t)lq * nk;
            if (qtok < 0) {
                for (int64_t j = 0; j < nk; ++j) p[j] = ds[j] = 0.0;
                continue;
            }
            const int64_t qt = bh * N + qtok;
            const double* qr = q + qt * d;
            const double* gr = dout + qt * d;
            const double* orow = out + qt * d;
            double D = 0.0;
            for (int x = 0; x < d; ++x) D += gr[x] * orow[x];
            double* dqq = dqr + (int64_t)lq * d;
            for (int64_t j = 0; j < nk; ++j) {
                const double* kr = k + ktok[j] * d;
                const double* vr = v + ktok[j] * d;
                double s = 0.0, dp = 0.0;
                for (int x = 0; x < d; ++x) {
                    s += qr[x] * kr[x];
                    dp += gr[x] * vr[x];
                }
                p[j] = exp(s * scale - lse[qt]);
                ds[j] = p[j] * (dp - D);
                for (int x = 0; x < d; ++x) dqq[x] += ds[j] * kr[x];
            }
            for (int x = 0; x < d; ++x) dqq[x] *= scale;
        }
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < nk; ++j) {
            double* dkr = dk + ktok[j] * d;
            double* dvr = dv + ktok[j] * d;
            for (int lq = 0; lq < CN; ++lq) {
                const int64_t qtok = oracle_token_of(T, H, W, i, lq);
                if (qtok < 0) continue;
                const int64_t qt = bh * N + qtok;
                const double pw = P[(int64_t)lq * nk + j];
                const double sw = dS[(int64_t)lq * nk + j] * scale;
                const double* qr = q + qt * d;
                const double* gr = dout + qt * d;
                for (int x = 0; x < d; ++x) {
                    dvr[x] += pw * gr[x];
                    dkr[x] += sw * qr[x];
                }
            }
        }
    }
    free(ktok); free(P); free(dS);
    return 0;
}

int oracle_attend_bwd(const double* q, const double* k, const double* v, const double* dout,
                      int BH, int T, int H, int W, int d, double scale, const int32_t* row_ptr,
                      const int32_t* col_idx, const int64_t* rows, int64_t n_rows,
                      double* dq_rows, double* dk, double* dv) {
    return oracle_attend_bwd_shape(q, k, v, dout, BH, T, H, W, CT, CH, CW, d, scale, row_ptr,
                                   col_idx, rows, n_rows, dq_rows, dk, dv);
}

/*
 * Context-parallel merge of two partial attention results over disjoint key
 * sets ([P1] ring block sparse attention: the output of a query is assembled
 * with an online softmax over key partitions; [P3] "开源实现": LSE and output
 * correction for context parallelism). For each query, with natural-log
 * log-sum-exps l1, l2 of the two partitions:
 *   l = log(exp(l1) + exp(l2)),   o = exp(l1 - l) o1 + exp(l2 - l) o2
 * which is the softmax-weighted output over the union of the key sets. A
 * partition with no keys has l = -inf and weight 0 (both empty: o = 0,
 * l = -inf). o1/l1 are overwritten with the merge. fp64.
 */
int oracle_lse_merge(double* o1, double* l1, const double* o2, const double* l2, int64_t n, int d) {
    if (!o1 || !l1 || !o2 || !l2 || n < 0 || d <= 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        const double a = l1[i], b = l2[i];
        if (b == -INFINITY) continue;
        if (a == -INFINITY) {
            for (int x = 0; x < d; ++x) o1[i * d + x] = o2[i * d + x];
            l1[i] = b;
            continue;
        }
        const double m = a > b ? a : b;
        const double l = m + log(exp(a - m) + exp(b - m));
        const double wa = exp(a - l), wb = exp(b - l);
        for (int x = 0; x < d; ++x) o1[i * d + x] = wa * o1[i * d + x] + wb * o2[i * d + x];
        l1[i] = l;
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
