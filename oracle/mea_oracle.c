/*
 * mea_oracle.c -- plain fp64 CPU oracle for memory-efficient exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this library.  It shares no code, header,
 * table or helper with the CUDA path and must never be reached from it.
 *
 * What it computes is the plain definition, one query row at a time:
 *
 *     s_j   = scale * <q_i, k_j> + b_ij            (b_ij = -inf where masked)
 *     w_j   = exp(s_j - max_j s_j) / sum_j exp(s_j - max_j s_j)
 *     out_i = sum_j w_j v_j
 *     lse_i = ln sum_j exp(s_j)
 *
 * Sources (page title, section):
 *  - "Transformer : comprendre l'entrainement et l'inference", section
 *    "Un cache KV simple": scores are q.k^T divided by sqrt(head_dim), masked
 *    with tril(ones(seq_len, total_len), diagonal=past_len) and -inf fill,
 *    then softmax and a product with v.  That mask is the bottom-right causal
 *    rule used below: query i (of M) sees key j (of N) iff j <= i + (N - M).
 *  - "Come costruire Transformer efficienti in memoria con xFormers ...",
 *    sections "Applicare Attenzione Causale con Maschere Inferiori" (lower
 *    triangular mask), "Utilizzare Sequenze di Lunghezza Variabile"
 *    (block-diagonal masks for packed sequences, plain and causal),
 *    "Dimotrazione di Gruppo Query Attention (GQA)" (several query heads share
 *    one key/value head) and "Utilizzare SwiGLU e ALiBi" (ALiBi bias).
 *  - "FlashAttention (2022)", section "L'idea: non scrivere mai la matrice
 *    intera": the tiled method returns exactly this result, so the oracle is
 *    the definition itself, not the tiled algorithm.
 *  - "Transformerを実装して少し理解した気になる会(その4)", section "KV Cache":
 *    a decode step needs only the last query row against all cached keys.
 *
 * Readings where the pages are silent (each one listed in the design notes):
 *  - ALiBi: b_ij = -slope_h * |pos_i - pos_j| added after scaling, positions
 *    local to the sequence, pos_i = i + (N - M); slope_h = 2^(-8 (h+1) / Hq),
 *    indexed by query head.  The caller passes the slopes (NULL = no ALiBi).
 *  - GQA: query head h reads key/value head floor(h / (Hq / Hkv)).
 *  - A row with no visible key has out = 0 and lse = -inf.
 *  - lse is the natural log.
 *
 * Layouts (all contiguous, fp64):
 *   q, out   [B, M, Hq, D]      k, v   [B, N, Hkv, D]      lse  [B, Hq, M]
 * For block-diagonal masks B must be 1 and seqstart_q / seqstart_k (length
 * num_seqs + 1) split the M query rows and the N key rows into sequences.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BIAS_NONE 0
#define ORACLE_BIAS_CAUSAL 1
#define ORACLE_BIAS_BLOCKDIAG 2
#define ORACLE_BIAS_BLOCKDIAG_CAUSAL 3

/* ALiBi slope of query head h out of Hq heads: 2^(-8 (h + 1) / Hq). */
double oracle_alibi_slope(int h, int Hq) {
    return pow(2.0, -8.0 * (double)(h + 1) / (double)Hq);
}

void oracle_alibi_slopes(int Hq, double* slopes) {
    for (int h = 0; h < Hq; ++h) slopes[h] = oracle_alibi_slope(h, Hq);
}

/* Which sequence of a packed batch holds row r: the s with
 * start[s] <= r < start[s+1], or -1. */
static int find_seq(const int32_t* start, int num_seqs, int64_t r) {
    for (int s = 0; s < num_seqs; ++s)
        if (r >= start[s] && r < start[s + 1]) return s;
    return -1;
}

/*
 * One output row: query row i of batch b, query head h.  Writes D values to
 * out_row and one value to *lse_row.  `score` is caller scratch of N doubles.
 * `keep` (NULL: no block mask) is this row's row of a block mask: key j is
 * visible only if keep[j / block_n] is nonzero.
 */
static void attention_row(const double* q, const double* k, const double* v,
                          int M, int N, int Hq, int Hkv, int D, int bias_kind,
                          const int32_t* seqstart_q, const int32_t* seqstart_k,
                          int num_seqs, const double* slopes, double scale,
                          int64_t b, int64_t i, int h, const uint8_t* keep, int64_t block_n,
                          double* score, double* out_row, double* lse_row) {
    const int group = Hq / Hkv;
    const int kvh = h / group;
    const double* qi = q + ((b * M + i) * Hq + h) * D;

    /* The key range this row may see, and the row's local position. */
    int64_t j_lo = 0, j_hi = N;   /* keys [j_lo, j_hi) belong to this row's sequence */
    int64_t pos_i = i + (N - M);  /* bottom-right alignment */
    int64_t m_len = M, n_len = N, i_loc = i;
    if (bias_kind == ORACLE_BIAS_BLOCKDIAG || bias_kind == ORACLE_BIAS_BLOCKDIAG_CAUSAL) {
        int s = find_seq(seqstart_q, num_seqs, i);
        if (s < 0) { j_lo = 0; j_hi = 0; }
        else {
            j_lo = seqstart_k[s];
            j_hi = seqstart_k[s + 1];
            m_len = seqstart_q[s + 1] - seqstart_q[s];
            n_len = j_hi - j_lo;
            i_loc = i - seqstart_q[s];
        }
        pos_i = i_loc + (n_len - m_len);
    }
    const int causal = (bias_kind == ORACLE_BIAS_CAUSAL || bias_kind == ORACLE_BIAS_BLOCKDIAG_CAUSAL);

    double mx = -INFINITY;
    for (int64_t j = 0; j < N; ++j) {
        int64_t pos_j = j - j_lo;
        int visible = (j >= j_lo && j < j_hi);
        if (causal && pos_j > pos_i) visible = 0;
        if (keep && !keep[j / block_n]) visible = 0;
        if (!visible) { score[j] = -INFINITY; continue; }
        const double* kj = k + ((b * N + j) * Hkv + kvh) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
        double s = scale * dot;
        if (slopes) s -= slopes[h] * fabs((double)(pos_i - pos_j));
        score[j] = s;
        if (s > mx) mx = s;
    }

    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    if (mx == -INFINITY) { *lse_row = -INFINITY; return; }

    double z = 0.0;
    for (int64_t j = 0; j < N; ++j) {
        if (score[j] == -INFINITY) { score[j] = 0.0; continue; }
        score[j] = exp(score[j] - mx);
        z += score[j];
    }
    for (int64_t j = 0; j < N; ++j) {
        if (score[j] == 0.0) continue;
        const double w = score[j] / z;
        const double* vj = v + ((b * N + j) * Hkv + kvh) * D;
        for (int d = 0; d < D; ++d) out_row[d] += w * vj[d];
    }
    *lse_row = mx + log(z);
}

static int check_args(int B, int M, int N, int Hq, int Hkv, int D, int bias_kind,
                      const int32_t* seqstart_q, const int32_t* seqstart_k, int num_seqs) {
    if (B < 0 || M < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (bias_kind < 0 || bias_kind > 3) return -1;
    if (bias_kind >= ORACLE_BIAS_BLOCKDIAG) {
        if (B != 1 || !seqstart_q || !seqstart_k || num_seqs <= 0) return -1;
        if (seqstart_q[0] != 0 || seqstart_k[0] != 0) return -1;
        if (seqstart_q[num_seqs] != M || seqstart_k[num_seqs] != N) return -1;
        for (int s = 0; s < num_seqs; ++s)
            if (seqstart_q[s + 1] < seqstart_q[s] || seqstart_k[s + 1] < seqstart_k[s]) return -1;
    }
    return 0;
}

/*
 * Attention over a list of rows.  rows holds n_rows triples (b, i, h); row r
 * is written to out[r * D ...] and lse[r].  Returns 0, or -1 on bad arguments.
 */
int oracle_attention_rows(const double* q, const double* k, const double* v,
                          int B, int M, int N, int Hq, int Hkv, int D, int bias_kind,
                          const int32_t* seqstart_q, const int32_t* seqstart_k, int num_seqs,
                          const double* slopes, double scale,
                          const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    if (check_args(B, M, N, Hq, Hkv, D, bias_kind, seqstart_q, seqstart_k, num_seqs)) return -1;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
        if (b < 0 || b >= B || i < 0 || i >= M || h < 0 || h >= Hq) return -1;
    }
    int failed = 0;
#pragma omp parallel
    {
        double* score = (double*)malloc(sizeof(double) * (N > 0 ? (size_t)N : 1));
        if (!score) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < n_rows; ++r) {
                attention_row(q, k, v, M, N, Hq, Hkv, D, bias_kind, seqstart_q, seqstart_k,
                              num_seqs, slopes, scale, rows[3 * r], rows[3 * r + 1],
                              (int)rows[3 * r + 2], NULL, 1, score, out + r * D, lse + r);
            }
            free(score);
        }
    }
    return failed ? -1 : 0;
}

/* Every row: out [B, M, Hq, D], lse [B, Hq, M]. */
int oracle_attention(const double* q, const double* k, const double* v,
                     int B, int M, int N, int Hq, int Hkv, int D, int bias_kind,
                     const int32_t* seqstart_q, const int32_t* seqstart_k, int num_seqs,
                     const double* slopes, double scale, double* out, double* lse) {
    if (check_args(B, M, N, Hq, Hkv, D, bias_kind, seqstart_q, seqstart_k, num_seqs)) return -1;
    int failed = 0;
    const int64_t total = (int64_t)B * M * Hq;
#pragma omp parallel
    {
        double* score = (double*)malloc(sizeof(double) * (N > 0 ? (size_t)N : 1));
        if (!score) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < total; ++r) {
                const int64_t b = r / ((int64_t)M * Hq);
                const int64_t i = (r / Hq) % M;
                const int h = (int)(r % Hq);
                double lse_val;
                attention_row(q, k, v, M, N, Hq, Hkv, D, bias_kind, seqstart_q, seqstart_k,
                              num_seqs, slopes, scale, b, i, h, NULL, 1, score,
                              out + ((b * M + i) * Hq + h) * D, &lse_val);
                lse[(b * Hq + h) * M + i] = lse_val;
            }
            free(score);
        }
    }
    return failed ? -1 : 0;
}

/*
 * Block-sparse attention ("FlashAttention (2022)", section "Cosa mostravano i
 * numeri", which names the block-sparse variant of the method): the score
 * matrix of each (batch, query head) is cut into block_m x block_n blocks and
 * a block whose mask entry is zero is left out, i.e. its scores are -inf, on
 * top of the bias kind (none or causal).  The result is the dense definition
 * above with that mask; a row left with no visible key has out = 0, lse = -inf.
 *   block_mask  uint8 [B, Hq, ceil(M / block_m), ceil(N / block_n)], contiguous;
 *               query row i, key j of (b, h) use entry
 *               [b][h][i / block_m][j / block_n].
 * rows (n_rows triples (b, i, h)) selects rows as in oracle_attention_rows,
 * with out [n_rows, D] and lse [n_rows]; rows == NULL computes every row into
 * out [B, M, Hq, D] and lse [B, Hq, M].
 */
int oracle_attention_block_sparse(const double* q, const double* k, const double* v,
                                  int B, int M, int N, int Hq, int Hkv, int D, int bias_kind,
                                  const uint8_t* block_mask, int block_m, int block_n,
                                  const double* slopes, double scale,
                                  const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    if (check_args(B, M, N, Hq, Hkv, D, bias_kind, NULL, NULL, 0)) return -1;
    if (bias_kind != ORACLE_BIAS_NONE && bias_kind != ORACLE_BIAS_CAUSAL) return -1;
    if (!block_mask || block_m <= 0 || block_n <= 0) return -1;
    const int64_t mblocks = (M + block_m - 1) / block_m, nblocks = (N + block_n - 1) / block_n;
    const int64_t total = rows ? n_rows : (int64_t)B * M * Hq;
    for (int64_t r = 0; rows && r < n_rows; ++r) {
        const int64_t b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
        if (b < 0 || b >= B || i < 0 || i >= M || h < 0 || h >= Hq) return -1;
    }
    int failed = 0;
#pragma omp parallel
    {
        double* score = (double*)malloc(sizeof(double) * (N > 0 ? (size_t)N : 1));
        if (!score) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < total; ++r) {
                int64_t b, i;
                int h;
                if (rows) {
                    b = rows[3 * r]; i = rows[3 * r + 1]; h = (int)rows[3 * r + 2];
                } else {
                    b = r / ((int64_t)M * Hq); i = (r / Hq) % M; h = (int)(r % Hq);
                }
                const uint8_t* keep =
                    block_mask + (((b * Hq + h) * mblocks) + i / block_m) * nblocks;
                double* orow = rows ? out + r * D : out + ((b * M + i) * Hq + h) * D;
                double lse_val;
                attention_row(q, k, v, M, N, Hq, Hkv, D, bias_kind, NULL, NULL, 0, slopes,
                              scale, b, i, h, keep, block_n, score, orow, &lse_val);
                if (rows) lse[r] = lse_val;
                else lse[(b * Hq + h) * M + i] = lse_val;
            }
            free(score);
        }
    }
    return failed ? -1 : 0;
}

/*
 * One decode step against a packed, ragged KV cache ("Pre-remplissage et
 * decodage"; "KV Cache"): sequence b holds keys kv_seqstart[b] ..
 * kv_seqstart[b+1]-1 and its single new query sits at the last position, so it
 * sees every cached key of its sequence.  With ALiBi the query position is
 * n_b - 1 and key position j - kv_seqstart[b].
 *   q, out [B, Hq, D]   k_cache, v_cache [T, Hkv, D]   lse [B, Hq]
 */
int oracle_decode(const double* q, const double* k_cache, const double* v_cache,
                  const int32_t* kv_seqstart, int B, int Hq, int Hkv, int D,
                  const double* slopes, double scale, double* out, double* lse) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0 || !kv_seqstart) return -1;
    if (kv_seqstart[0] != 0) return -1;
    for (int b = 0; b < B; ++b)
        if (kv_seqstart[b + 1] < kv_seqstart[b]) return -1;
    const int group = Hq / Hkv;
    int failed = 0;
#pragma omp parallel
    {
        int64_t max_len = 1;
        for (int b = 0; b < B; ++b) {
            int64_t n = kv_seqstart[b + 1] - kv_seqstart[b];
            if (n > max_len) max_len = n;
        }
        double* w = (double*)malloc(sizeof(double) * (size_t)max_len);
        if (!w) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < (int64_t)B * Hq; ++r) {
                const int b = (int)(r / Hq), h = (int)(r % Hq), kvh = h / group;
                const int64_t t0 = kv_seqstart[b], n = kv_seqstart[b + 1] - t0;
                const double* qv = q + r * D;
                double* o = out + r * D;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                if (n == 0) { lse[r] = -INFINITY; continue; }
                double mx = -INFINITY;
                for (int64_t j = 0; j < n; ++j) {
                    const double* kj = k_cache + ((t0 + j) * Hkv + kvh) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += qv[d] * kj[d];
                    double s = scale * dot;
                    if (slopes) s -= slopes[h] * (double)(n - 1 - j);
                    w[j] = s;
                    if (s > mx) mx = s;
                }
                double z = 0.0;
                for (int64_t j = 0; j < n; ++j) { w[j] = exp(w[j] - mx); z += w[j]; }
                for (int64_t j = 0; j < n; ++j) {
                    const double* vj = v_cache + ((t0 + j) * Hkv + kvh) * D;
                    const double c = w[j] / z;
                    for (int d = 0; d < D; ++d) o[d] += c * vj[d];
                }
                lse[r] = mx + log(z);
            }
            free(w);
        }
    }
    return failed ? -1 : 0;
}

/*
 * Gradients of the attention above ("FlashAttention (2022)", section "Il trucco
 * della softmax che non ha bisogno di vedere tutto": the backward pass recomputes
 * the scores instead of storing them).  For one row i of query head h, with
 * p_ij = exp(s_ij - lse_i) its softmax weights over the visible keys:
 *     dV_j += p_ij dO_i                      dP_ij = <dO_i, v_j>
 *     D_i   = sum_j p_ij dP_ij (= <dO_i, out_i>)
 *     dS_ij = p_ij (dP_ij - D_i)
 *     dQ_i  = scale sum_j dS_ij k_j          dK_j += scale dS_ij q_i
 * dK and dV of a key/value head sum over the query heads that read it.  The
 * bias (mask, ALiBi) does not depend on q, k or v.  Same layouts as
 * oracle_attention; dout like out; dq like q; dk, dv like k, v.
 */
int oracle_attention_bwd(const double* q, const double* k, const double* v, const double* dout,
                         int B, int M, int N, int Hq, int Hkv, int D, int bias_kind,
                         const int32_t* seqstart_q, const int32_t* seqstart_k, int num_seqs,
                         const double* slopes, double scale, double* dq, double* dk, double* dv) {
    if (check_args(B, M, N, Hq, Hkv, D, bias_kind, seqstart_q, seqstart_k, num_seqs)) return -1;
    const int group = Hq / Hkv;
    memset(dq, 0, sizeof(double) * (size_t)B * M * Hq * D);
    memset(dk, 0, sizeof(double) * (size_t)B * N * Hkv * D);
    memset(dv, 0, sizeof(double) * (size_t)B * N * Hkv * D);
    int failed = 0;
    /* One (batch, kv head) per task: its dK, dV rows are written by nobody else. */
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (N > 0 ? (size_t)N : 1));
        double* dp = (double*)malloc(sizeof(double) * (N > 0 ? (size_t)N : 1));
        double* o = (double*)malloc(sizeof(double) * (size_t)D);
        if (!p || !dp || !o) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < (int64_t)B * Hkv; ++task) {
                const int64_t b = task / Hkv;
                const int kvh = (int)(task % Hkv);
                for (int h = kvh * group; h < (kvh + 1) * group; ++h) {
                    for (int64_t i = 0; i < M; ++i) {
                        double lse;
                        /* forward row: p holds the scores, then the weights */
                        attention_row(q, k, v, M, N, Hq, Hkv, D, bias_kind, seqstart_q, seqstart_k,
                                      num_seqs, slopes, scale, b, i, h, NULL, 1, p, o, &lse);
                        if (lse == -INFINITY) continue;  /* row sees no key: no gradient */
                        /* attention_row left exp(s - max) (0 where masked) in p */
                        double z = 0.0;
                        for (int64_t j = 0; j < N; ++j) z += p[j];
                        const double* doi = dout + ((b * M + i) * Hq + h) * D;
                        double Di = 0.0;
                        for (int64_t j = 0; j < N; ++j) {
                            p[j] /= z;
                            if (p[j] == 0.0) { dp[j] = 0.0; continue; }
                            const double* vj = v + ((b * N + j) * Hkv + kvh) * D;
                            double s = 0.0;
                            for (int d = 0; d < D; ++d) s += doi[d] * vj[d];
                            dp[j] = s;
                            Di += p[j] * s;
                        }
                        const double* qi = q + ((b * M + i) * Hq + h) * D;
                        double* dqi = dq + ((b * M + i) * Hq + h) * D;
                        for (int64_t j = 0; j < N; ++j) {
                            if (p[j] == 0.0) continue;
                            const double ds = p[j] * (dp[j] - Di);
                            const double* kj = k + ((b * N + j) * Hkv + kvh) * D;
                            double* dkj = dk + ((b * N + j) * Hkv + kvh) * D;
                            double* dvj = dv + ((b * N + j) * Hkv + kvh) * D;
                            for (int d = 0; d < D; ++d) {
                                dvj[d] += p[j] * doi[d];
                                dqi[d] += scale * ds * kj[d];
                                dkj[d] += scale * ds * qi[d];
                            }
                        }
                    }
                }
            }
        }
        free(p);
        free(dp);
        free(o);
    }
    return failed ? -1 : 0;
}

/*
 * One chunk of prefill against a KV cache ("Transformer : comprendre
 * l'entrainement et l'inference", sections "Pre-remplissage et decodage" and
 * "Un cache KV simple": the keys and values of the new tokens are concatenated
 * after the cached ones, and the new queries attend to the whole result under
 * tril(ones(seq_len, total_len), diagonal=past_len)).
 * For sequence b with past = cache_len[b] cached rows and n = q_len[b] new rows
 * (q_len NULL: n = M for every sequence):
 *   1. append: k_cache[b, past + r] = k_new[b, r], v likewise, for r < n;
 *   2. for query row i < n (position past + i) and query head h: attention over
 *      cache rows j < past + n, causal: visible iff j <= past + i; ALiBi bias
 *      -slope_h * |past + i - j|; weights and lse as in oracle_attention.
 * Rows i >= n of out and lse are left as they are.
 *   q, out [B, M, Hq, D]   k_new, v_new [B, M, Hkv, D]   lse [B, Hq, M]
 *   k_cache, v_cache [B, cap, Hkv, D] (updated in place)
 * Returns -1 if past < 0, n outside [0, M] or past + n > cap.
 */
int oracle_prefill_chunk(const double* q, const double* k_new, const double* v_new,
                         double* k_cache, double* v_cache, const int32_t* cache_len,
                         const int32_t* q_len, int B, int M, int cap, int Hq, int Hkv, int D,
                         int causal, const double* slopes, double scale, double* out,
                         double* lse) {
    if (B < 0 || M < 0 || cap < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return -1;
    if (!cache_len) return -1;
    for (int b = 0; b < B; ++b) {
        const int64_t past = cache_len[b], n = q_len ? q_len[b] : M;
        if (past < 0 || n < 0 || n > M || past + n > cap) return -1;
    }
    const int group = Hq / Hkv;
    /* 1. the append */
    for (int b = 0; b < B; ++b) {
        const int64_t past = cache_len[b], n = q_len ? q_len[b] : M;
        for (int64_t r = 0; r < n; ++r)
            for (int kvh = 0; kvh < Hkv; ++kvh)
                for (int d = 0; d < D; ++d) {
                    const int64_t src = ((b * (int64_t)M + r) * Hkv + kvh) * D + d;
                    const int64_t dst = ((b * (int64_t)cap + past + r) * Hkv + kvh) * D + d;
                    k_cache[dst] = k_new[src];
                    v_cache[dst] = v_new[src];
                }
    }
    /* 2. attention of the chunk's queries over the extended cache */
    int failed = 0;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (cap > 0 ? (size_t)cap : 1));
        if (!w) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t task = 0; task < (int64_t)B * Hq * M; ++task) {
                const int b = (int)(task / ((int64_t)Hq * M));
                const int h = (int)((task / M) % Hq);
                const int64_t i = task % M;
                const int64_t past = cache_len[b], n = q_len ? q_len[b] : M;
                if (i >= n) continue;
                const int kvh = h / group;
                const int64_t total = past + n, pos_i = past + i;
                const double* qi = q + ((b * (int64_t)M + i) * Hq + h) * D;
                double* o = out + ((b * (int64_t)M + i) * Hq + h) * D;
                double mx = -INFINITY;
                for (int64_t j = 0; j < total; ++j) {
                    if (causal && j > pos_i) { w[j] = -INFINITY; continue; }
                    const double* kj = k_cache + ((b * (int64_t)cap + j) * Hkv + kvh) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
                    double s = scale * dot;
                    if (slopes) s -= slopes[h] * fabs((double)(pos_i - j));
                    w[j] = s;
                    if (s > mx) mx = s;
                }
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                double* l = lse + ((int64_t)b * Hq + h) * M + i;
                if (mx == -INFINITY) { *l = -INFINITY; continue; }
                double z = 0.0;
                for (int64_t j = 0; j < total; ++j) {
                    w[j] = (w[j] == -INFINITY) ? 0.0 : exp(w[j] - mx);
                    z += w[j];
                }
                for (int64_t j = 0; j < total; ++j) {
                    if (w[j] == 0.0) continue;
                    const double* vj = v_cache + ((b * (int64_t)cap + j) * Hkv + kvh) * D;
                    for (int d = 0; d < D; ++d) o[d] += (w[j] / z) * vj[d];
                }
                *l = mx + log(z);
            }
            free(w);
        }
    }
    return failed ? -1 : 0;
}
