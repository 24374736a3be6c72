/*
 * Attention forward oracle -- plain, slow, fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the test suite, the smoke check and the benchmark's
 * cpu_baseline / reference leg do.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * What it computes (FlashAttention/ops-transformer article on ai6s.net,
 * section "传统注意力的显存陷阱" -- the conventional attention definition:
 * scores = Q K^T / sqrt(d_k), probabilities = softmax over the key axis,
 * output = probabilities . V), generalised to an explicit scale, an optional
 * causal mask and an fp32-style natural-log row LSE:
 *
 *   for every batch b, head h, query i:
 *     allowed(i, j)  <=>  j < Nk  and (not causal or j <= i + (Nk - Nq))
 *     s_ij  = scale * sum_t q[b,i,h,t] * k[b,j,h,t]          (allowed j only)
 *     m_i   = max_j s_ij
 *     p_ij  = exp(s_ij - m_i)
 *     l_i   = sum_j p_ij
 *     O[b,i,h,:] = sum_j p_ij v[b,j,h,:] / l_i
 *     lse[b,h,i] = m_i + ln l_i
 *   A row with no allowed key gives O = 0 and lse = -inf.
 *
 * Readings where the article is silent (each one is listed in the design
 * notes): the scale is an explicit argument (the article divides by sqrt(d_k)
 * and its API example passes none); a causal mask with Nq != Nk is aligned to
 * the bottom-right corner; lse is the natural-log row LSE of the scaled,
 * masked scores.
 *
 * Layouts: q, o are [B, Nq, H, d]; k, v are [B, Nk, H, d]; lse is [B, H, Nq];
 * p (probabilities, tiny cases only) is [B, H, Nq, Nk].  Everything is double.
 *
 * Three orderings of the forward are provided.  oracle_attn_fwd_f64 follows the
 * definition literally and materialises each (b, h) score matrix.  The blocked
 * variant follows the article's "FlashAttention的核心逻辑" section: an outer loop
 * over query blocks, an inner loop over key/value blocks, a running row maximum
 * and row sum updated block by block (the online softmax update, written out in
 * its standard form because the article only names it), and one normalisation
 * after the inner loop.  The split-KV variant keeps one state per key range and
 * merges them at the end, the order of the decode path.  All must agree to
 * rounding.
 *
 * Further down, for the steps next to this one on the pages: the score term of
 * a relative-position embedding, the backward pass, attention over a paged
 * key/value cache with several query tokens per request, and the lightning
 * indexer's rectified head-weighted score with its top-k selection.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX4(b, n, h, t, N, H, D) ((((long)(b) * (N) + (n)) * (H) + (h)) * (D) + (t))

static int is_allowed(long i, long j, long Nq, long Nk, int causal)
{
    if (j >= Nk) return 0;
    if (causal && j > i + (Nk - Nq)) return 0;
    return 1;
}

static double dot_qk(const double* q, const double* k, int b, int h, long i, long j,
                     int H, int Nq, int Nk, int d)
{
    double acc = 0.0;
    const double* qi = q + IDX4(b, i, h, 0, Nq, H, d);
    const double* kj = k + IDX4(b, j, h, 0, Nk, H, d);
    for (int t = 0; t < d; ++t) acc += qi[t] * kj[t];
    return acc;
}

static int check_args(int B, int H, int Nq, int Nk, int d)
{
    return (B > 0 && H > 0 && Nq > 0 && Nk > 0 && d > 0) ? 0 : -1;
}

/* Definition order: materialise S for one (b, h), then softmax, then P.V. */
int oracle_attn_fwd_f64(const double* q, const double* k, const double* v,
                        double* o, double* lse,
                        int B, int H, int Nq, int Nk, int d, int causal, double scale)
{
    if (check_args(B, H, Nq, Nk, d)) return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const int b = (int)(bh / H), h = (int)(bh % H);
        double* S = (double*)malloc(sizeof(double) * (size_t)Nq * (size_t)Nk);
        if (!S) {
#pragma omp atomic write
            err = -2;
            continue;
        }
        /* scores, -inf where not allowed */
        for (long i = 0; i < Nq; ++i)
            for (long j = 0; j < Nk; ++j)
                S[i * Nk + j] = is_allowed(i, j, Nq, Nk, causal)
                                    ? scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d)
                                    : -INFINITY;
        for (long i = 0; i < Nq; ++i) {
            double* Si = S + i * Nk;
            double m = -INFINITY;
            for (long j = 0; j < Nk; ++j) if (Si[j] > m) m = Si[j];
            double* oi = o + IDX4(b, i, h, 0, Nq, H, d);
            if (m == -INFINITY) {          /* no allowed key in this row */
                for (int t = 0; t < d; ++t) oi[t] = 0.0;
                lse[((long)b * H + h) * Nq + i] = -INFINITY;
                continue;
            }
            double l = 0.0;
            for (long j = 0; j < Nk; ++j) {
                Si[j] = (Si[j] == -INFINITY) ? 0.0 : exp(Si[j] - m);   /* Si now holds p_ij */
                l += Si[j];
            }
            for (int t = 0; t < d; ++t) {
                double acc = 0.0;
                for (long j = 0; j < Nk; ++j)
                    if (Si[j] != 0.0) acc += Si[j] * v[IDX4(b, j, h, t, Nk, H, d)];
                oi[t] = acc / l;
            }
            lse[((long)b * H + h) * Nq + i] = m + log(l);
        }
        free(S);
    }
    return err;
}

/* Row-normalised probabilities P[b,h,i,j] (masked entries are exactly 0). */
int oracle_attn_probs_f64(const double* q, const double* k, double* p,
                          int B, int H, int Nq, int Nk, int d, int causal, double scale)
{
    if (check_args(B, H, Nq, Nk, d)) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const int b = (int)(bh / H), h = (int)(bh % H);
        for (long i = 0; i < Nq; ++i) {
            double* Pi = p + (bh * Nq + i) * (long)Nk;
            double m = -INFINITY;
            for (long j = 0; j < Nk; ++j) {
                Pi[j] = is_allowed(i, j, Nq, Nk, causal)
                            ? scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d)
                            : -INFINITY;
                if (Pi[j] > m) m = Pi[j];
            }
            if (m == -INFINITY) { for (long j = 0; j < Nk; ++j) Pi[j] = 0.0; continue; }
            double l = 0.0;
            for (long j = 0; j < Nk; ++j) {
                Pi[j] = (Pi[j] == -INFINITY) ? 0.0 : exp(Pi[j] - m);
                l += Pi[j];
            }
            for (long j = 0; j < Nk; ++j) Pi[j] /= l;
        }
    }
    return 0;
}

/*
 * Blocked online order (the article's core-logic section): query blocks of
 * block_m rows, key/value blocks of block_n rows.  Per query row the running
 * state is (m, l, acc[d]); for each key block:
 *   m' = max(m, max_j s_ij);  alpha = exp(m - m');
 *   l  = alpha * l + sum_j exp(s_ij - m');
 *   acc = alpha * acc + sum_j exp(s_ij - m') v_j;   m = m'
 * and after the last block O = acc / l, lse = m + ln l.
 */
int oracle_attn_fwd_blocked_f64(const double* q, const double* k, const double* v,
                                double* o, double* lse,
                                int B, int H, int Nq, int Nk, int d, int causal, double scale,
                                int block_m, int block_n)
{
    if (check_args(B, H, Nq, Nk, d) || block_m <= 0 || block_n <= 0) return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const int b = (int)(bh / H), h = (int)(bh % H);
        double* m = (double*)malloc(sizeof(double) * (size_t)block_m);
        double* l = (double*)malloc(sizeof(double) * (size_t)block_m);
        double* acc = (double*)malloc(sizeof(double) * (size_t)block_m * (size_t)d);
        double* s = (double*)malloc(sizeof(double) * (size_t)block_n);
        if (!m || !l || !acc || !s) {
#pragma omp atomic write
            err = -2;
            free(m); free(l); free(acc); free(s);
            continue;
        }
        for (long i0 = 0; i0 < Nq; i0 += block_m) {
            const long rows = (Nq - i0 < block_m) ? (Nq - i0) : block_m;
            for (long r = 0; r < rows; ++r) {
                m[r] = -INFINITY;
                l[r] = 0.0;
                for (int t = 0; t < d; ++t) acc[r * d + t] = 0.0;
            }
            for (long j0 = 0; j0 < Nk; j0 += block_n) {
                const long cols = (Nk - j0 < block_n) ? (Nk - j0) : block_n;
                for (long r = 0; r < rows; ++r) {
                    const long i = i0 + r;
                    double bmax = -INFINITY;
                    for (long c = 0; c < cols; ++c) {
                        const long j = j0 + c;
                        s[c] = is_allowed(i, j, Nq, Nk, causal)
                                   ? scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d)
                                   : -INFINITY;
                        if (s[c] > bmax) bmax = s[c];
                    }
                    if (bmax == -INFINITY) continue;       /* nothing allowed in this block */
                    const double mnew = (bmax > m[r]) ? bmax : m[r];
                    const double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - mnew);
                    double bsum = 0.0;
                    for (int t = 0; t < d; ++t) acc[r * d + t] *= alpha;
                    for (long c = 0; c < cols; ++c) {
                        if (s[c] == -INFINITY) continue;
                        const double pc = exp(s[c] - mnew);
                        bsum += pc;
                        const double* vj = v + IDX4(b, j0 + c, h, 0, Nk, H, d);
                        for (int t = 0; t < d; ++t) acc[r * d + t] += pc * vj[t];
                    }
                    l[r] = alpha * l[r] + bsum;
                    m[r] = mnew;
                }
            }
            for (long r = 0; r < rows; ++r) {
                const long i = i0 + r;
                double* oi = o + IDX4(b, i, h, 0, Nq, H, d);
                if (l[r] == 0.0) {
                    for (int t = 0; t < d; ++t) oi[t] = 0.0;
                    lse[((long)b * H + h) * Nq + i] = -INFINITY;
                } else {
                    for (int t = 0; t < d; ++t) oi[t] = acc[r * d + t] / l[r];
                    lse[((long)b * H + h) * Nq + i] = m[r] + log(l[r]);
                }
            }
        }
        free(m); free(l); free(acc); free(s);
    }
    return err;
}

/*
 * The split-KV ordering of the decode path: the keys of each query row are cut
 * into `splits` contiguous ranges of ceil(Nk / splits) keys (the last range holds
 * the rest), each range keeps its own state
 *   m_s = max_j s_ij,   l_s = sum_j exp(s_ij - m_s),   o_s = sum_j exp(s_ij - m_s) v_j
 * and a combine step merges them:
 *   M = max_s m_s,   L = sum_s l_s exp(m_s - M),   O = sum_s o_s exp(m_s - M) / L,
 *   lse = M + ln L.
 * This is the same recurrence as the blocked ordering (the ai6s.net article's
 * online softmax, section "FlashAttention的核心逻辑"), applied to ranges that are
 * processed side by side instead of one after another.  A range with no allowed key
 * (m_s = -inf) drops out.  Must agree with oracle_attn_fwd_f64 to rounding.
 */
int oracle_attn_fwd_splitkv_f64(const double* q, const double* k, const double* v,
                                double* o, double* lse,
                                int B, int H, int Nq, int Nk, int d, int causal, double scale,
                                int splits)
{
    if (check_args(B, H, Nq, Nk, d) || splits <= 0) return -1;
    const long span = ((long)Nk + splits - 1) / splits;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const int b = (int)(bh / H), h = (int)(bh % H);
        double* part_m = (double*)malloc(sizeof(double) * (size_t)splits);
        double* part_l = (double*)malloc(sizeof(double) * (size_t)splits);
        double* part_o = (double*)malloc(sizeof(double) * (size_t)splits * (size_t)d);
        if (!part_m || !part_l || !part_o) {
#pragma omp atomic write
            err = -2;
            free(part_m); free(part_l); free(part_o);
            continue;
        }
        for (long i = 0; i < Nq; ++i) {
            for (int sp = 0; sp < splits; ++sp) {
                const long j_lo = (long)sp * span;
                const long j_hi = (j_lo + span < Nk) ? j_lo + span : Nk;
                double ms = -INFINITY;
                for (long j = j_lo; j < j_hi; ++j) {
                    if (!is_allowed(i, j, Nq, Nk, causal)) continue;
                    const double sc = scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d);
                    ms = sc > ms ? sc : ms;
                }
                part_m[sp] = ms;
                part_l[sp] = 0.0;
                for (int t = 0; t < d; ++t) part_o[(long)sp * d + t] = 0.0;
                if (ms == -INFINITY) continue;
                for (long j = j_lo; j < j_hi; ++j) {
                    if (!is_allowed(i, j, Nq, Nk, causal)) continue;
                    const double e = exp(scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d) - ms);
                    part_l[sp] += e;
                    const double* vrow = v + IDX4(b, j, h, 0, Nk, H, d);
                    for (int t = 0; t < d; ++t) part_o[(long)sp * d + t] += e * vrow[t];
                }
            }
            /* combine */
            double big_m = -INFINITY;
            for (int sp = 0; sp < splits; ++sp) big_m = part_m[sp] > big_m ? part_m[sp] : big_m;
            double* orow = o + IDX4(b, i, h, 0, Nq, H, d);
            double* lse_row = lse + ((long)b * H + h) * Nq + i;
            if (big_m == -INFINITY) {
                for (int t = 0; t < d; ++t) orow[t] = 0.0;
                *lse_row = -INFINITY;
                continue;
            }
            double big_l = 0.0;
            for (int sp = 0; sp < splits; ++sp)
                if (part_m[sp] != -INFINITY) big_l += part_l[sp] * exp(part_m[sp] - big_m);
            for (int t = 0; t < d; ++t) {
                double num = 0.0;
                for (int sp = 0; sp < splits; ++sp)
                    if (part_m[sp] != -INFINITY) num += part_o[(long)sp * d + t] * exp(part_m[sp] - big_m);
                orow[t] = num / big_l;
            }
            *lse_row = big_m + log(big_l);
        }
        free(part_m); free(part_l); free(part_o);
    }
    return err;
}

/*
 * Attention with a relative-position score term (the Granite-Speech conformer
 * attention of the vLLM page "PR #42933", section "关键源码片段": the term
 * einsum("bnhid,ijd->bnhij", q, rel_pos_emb) * scale is added to the scores that
 * masking and SDPA then use).  rel_pos_emb[i, j, :] is the embedding row
 * emb[dist[i, j]] of a relative-distance index, as the page builds it from
 * `dist`; dist is an input here (int32 [Nq, Nk], values in [0, n_emb)), emb is
 * [n_emb, d], both shared by every batch and head:
 *
 *   s_ij = scale * (sum_t q[b,i,h,t] * k[b,j,h,t] + sum_t q[b,i,h,t] * emb[dist[i,j], t])
 *
 * over allowed j, then the same softmax, output and lse as oracle_attn_fwd_f64.
 */
int oracle_attn_fwd_relpos_f64(const double* q, const double* k, const double* v,
                               const double* emb, const int* dist, double* o, double* lse,
                               int B, int H, int Nq, int Nk, int d, int n_emb, int causal,
                               double scale)
{
    if (check_args(B, H, Nq, Nk, d) || n_emb <= 0) return -1;
    for (long ij = 0; ij < (long)Nq * Nk; ++ij)
        if (dist[ij] < 0 || dist[ij] >= n_emb) return -3;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const int b = (int)(bh / H), h = (int)(bh % H);
        double* S = (double*)malloc(sizeof(double) * (size_t)Nq * (size_t)Nk);
        if (!S) {
#pragma omp atomic write
            err = -2;
            continue;
        }
        for (long i = 0; i < Nq; ++i) {
            const double* qi = q + IDX4(b, i, h, 0, Nq, H, d);
            for (long j = 0; j < Nk; ++j) {
                if (!is_allowed(i, j, Nq, Nk, causal)) {
                    S[i * Nk + j] = -INFINITY;
                    continue;
                }
                const double* e = emb + (long)dist[i * Nk + j] * d;
                double rel = 0.0;
                for (int t = 0; t < d; ++t) rel += qi[t] * e[t];
                S[i * Nk + j] = scale * (dot_qk(q, k, b, h, i, j, H, Nq, Nk, d) + rel);
            }
        }
        /* softmax over each row, output and lse, as in oracle_attn_fwd_f64 */
        for (long i = 0; i < Nq; ++i) {
            double* row = S + i * Nk;
            double mx = -INFINITY;
            for (long j = 0; j < Nk; ++j) mx = row[j] > mx ? row[j] : mx;
            double* out_i = o + IDX4(b, i, h, 0, Nq, H, d);
            double* lse_i = lse + ((long)b * H + h) * Nq + i;
            if (mx == -INFINITY) {
                for (int t = 0; t < d; ++t) out_i[t] = 0.0;
                *lse_i = -INFINITY;
                continue;
            }
            double denom = 0.0;
            for (long j = 0; j < Nk; ++j) {
                row[j] = (row[j] == -INFINITY) ? 0.0 : exp(row[j] - mx);
                denom += row[j];
            }
            for (int t = 0; t < d; ++t) {
                double num = 0.0;
                for (long j = 0; j < Nk; ++j)
                    if (row[j] != 0.0) num += row[j] * v[IDX4(b, j, h, t, Nk, H, d)];
                out_i[t] = num / denom;
            }
            *lse_i = mx + log(denom);
        }
        free(S);
    }
    return err;
}

/*
 * Gradients of the forward above (the step after it on the pages: the ai6s.net
 * article notes that eager attention keeps the N x N matrix for the backward
 * pass, section "传统注意力的显存陷阱"), from the definition by the chain rule,
 * for an upstream gradient dO of O:
 *
 *   P = softmax(S) row-wise (S = scale * Q K^T, masked),  O = P V
 *   dV = P^T dO
 *   dP = dO V^T
 *   dS_ij = P_ij * (dP_ij - sum_t dO_it O_it)      (softmax Jacobian; sum_t dO.O = sum_j P_ij dP_ij)
 *   dQ = scale * dS K,   dK = scale * dS^T Q
 *
 * Masked entries have P = 0, hence dS = 0; a row with no allowed key has O = 0 and
 * contributes nothing.  Layouts as the forward; dq [B,Nq,H,d], dk and dv [B,Nk,H,d].
 */
int oracle_attn_bwd_f64(const double* q, const double* k, const double* v, const double* dout,
                        double* dq, double* dk, double* dv,
                        int B, int H, int Nq, int Nk, int d, int causal, double scale)
{
    if (check_args(B, H, Nq, Nk, d)) return -1;
    const size_t n_q = (size_t)B * (size_t)Nq * (size_t)H * (size_t)d;
    const size_t n_kv = (size_t)B * (size_t)Nk * (size_t)H * (size_t)d;
    memset(dq, 0, sizeof(double) * n_q);
    memset(dk, 0, sizeof(double) * n_kv);
    memset(dv, 0, sizeof(double) * n_kv);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const int b = (int)(bh / H), h = (int)(bh % H);
        double* P = (double*)malloc(sizeof(double) * (size_t)Nq * (size_t)Nk);
        double* dP = (double*)malloc(sizeof(double) * (size_t)Nq * (size_t)Nk);
        if (!P || !dP) {
            free(P);
            free(dP);
#pragma omp atomic write
            err = -2;
            continue;
        }
        /* P row by row */
        for (long i = 0; i < Nq; ++i) {
            double* Pi = P + i * Nk;
            double top = -INFINITY;
            for (long j = 0; j < Nk; ++j) {
                Pi[j] = is_allowed(i, j, Nq, Nk, causal) ? scale * dot_qk(q, k, b, h, i, j, H, Nq, Nk, d)
                                                          : -INFINITY;
                if (Pi[j] > top) top = Pi[j];
            }
            if (top == -INFINITY) {
                for (long j = 0; j < Nk; ++j) Pi[j] = 0.0;
                continue;
            }
            double z = 0.0;
            for (long j = 0; j < Nk; ++j) {
                Pi[j] = (Pi[j] == -INFINITY) ? 0.0 : exp(Pi[j] - top);
                z += Pi[j];
            }
            for (long j = 0; j < Nk; ++j) Pi[j] /= z;
        }
        /* dV = P^T dO and dP = dO V^T */
        for (long i = 0; i < Nq; ++i) {
            const double* doi = dout + IDX4(b, i, h, 0, Nq, H, d);
            for (long j = 0; j < Nk; ++j) {
                const double pij = P[i * Nk + j];
                const double* vj = v + IDX4(b, j, h, 0, Nk, H, d);
                double* dvj = dv + IDX4(b, j, h, 0, Nk, H, d);
                double g = 0.0;
                for (int t = 0; t < d; ++t) {
                    dvj[t] += pij * doi[t];
                    g += doi[t] * vj[t];
                }
                dP[i * Nk + j] = g;
            }
        }
        /* dS, then dQ and dK */
        for (long i = 0; i < Nq; ++i) {
            double delta = 0.0;  /* sum_j P_ij dP_ij */
            for (long j = 0; j < Nk; ++j) delta += P[i * Nk + j] * dP[i * Nk + j];
            const double* qi = q + IDX4(b, i, h, 0, Nq, H, d);
            double* dqi = dq + IDX4(b, i, h, 0, Nq, H, d);
            for (long j = 0; j < Nk; ++j) {
                const double ds = P[i * Nk + j] * (dP[i * Nk + j] - delta);
                if (ds == 0.0) continue;
                const double* krow = k + IDX4(b, j, h, 0, Nk, H, d);
                double* dkj = dk + IDX4(b, j, h, 0, Nk, H, d);
                for (int t = 0; t < d; ++t) {
                    dqi[t] += scale * ds * krow[t];
                    dkj[t] += scale * ds * qi[t];
                }
            }
        }
        free(P);
        free(dP);
    }
    return err;
}

/*
 * Attention over a paged key/value cache, for one or more query tokens per
 * request (the vLLM page "PR #45743 完整报告": decode metadata of per-request
 * seq_lens and a block table, section "关键源码片段", and several query tokens of
 * one request scored together, section "功能与动机").  Request b owns the first
 * L = seq_lens[b] rows of its logical sequence; logical row j sits in row
 * j mod page_size of cache page block_table[b][j / page_size].  Its Lq query
 * tokens are the last Lq positions of the sequence, so under the causal flag
 * query i sees logical rows j <= i + L - Lq (the bottom-right alignment of the
 * dense definition); without it every query sees all L rows.  Scores, softmax,
 * output and lse are then those of oracle_attn_fwd_f64 on the gathered rows.
 * Layouts: q, o [B, Lq, H, d]; k_cache, v_cache [num_blocks, page_size, H, d];
 * block_table [B, max_blocks] int; seq_lens [B] int; lse [B, H, Lq].
 * Returns -3 when a seq_len exceeds max_blocks * page_size or a table entry a
 * row below it needs lies outside [0, num_blocks).
 */
int oracle_attn_fwd_paged_f64(const double* q, const double* k_cache, const double* v_cache,
                              const int* block_table, const int* seq_lens, double* o,
                              double* lse, int B, int Lq, int H, int d, int num_blocks,
                              int page_size, int max_blocks, int causal, double scale)
{
    if (B <= 0 || Lq <= 0 || H <= 0 || d <= 0 || num_blocks <= 0 || page_size <= 0 ||
        max_blocks <= 0)
        return -1;
    for (int b = 0; b < B; ++b) {
        const long L = seq_lens[b];
        if (L < 0 || L > (long)max_blocks * page_size) return -3;
        for (long pg = 0; pg * page_size < L; ++pg) {
            const int e = block_table[(long)b * max_blocks + pg];
            if (e < 0 || e >= num_blocks) return -3;
        }
    }
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const int b = (int)(bh / H), h = (int)(bh % H);
        const long L = seq_lens[b];
        double* w = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        if (!w) {
#pragma omp atomic write
            err = -2;
            continue;
        }
        for (long i = 0; i < Lq; ++i) {
            const double* qrow = q + (((long)b * Lq + i) * H + h) * d;
            double* orow = o + (((long)b * Lq + i) * H + h) * d;
            double top = -INFINITY;
            for (long j = 0; j < L; ++j) {
                if (causal && j > i + (L - Lq)) {
                    w[j] = -INFINITY;
                    continue;
                }
                const long page = block_table[(long)b * max_blocks + j / page_size];
                const long slot = page * page_size + j % page_size;
                const double* krow = k_cache + (slot * H + h) * d;
                double dotp = 0.0;
                for (int t = 0; t < d; ++t) dotp += qrow[t] * krow[t];
                w[j] = scale * dotp;
                top = w[j] > top ? w[j] : top;
            }
            double* lse_bhi = lse + ((long)b * H + h) * Lq + i;
            if (top == -INFINITY) {
                for (int t = 0; t < d; ++t) orow[t] = 0.0;
                *lse_bhi = -INFINITY;
                continue;
            }
            double total = 0.0;
            for (long j = 0; j < L; ++j) {
                w[j] = (w[j] == -INFINITY) ? 0.0 : exp(w[j] - top);
                total += w[j];
            }
            for (int t = 0; t < d; ++t) {
                double sum_wv = 0.0;
                for (long j = 0; j < L; ++j) {
                    if (w[j] == 0.0) continue;
                    const long page = block_table[(long)b * max_blocks + j / page_size];
                    const long slot = page * page_size + j % page_size;
                    sum_wv += w[j] * v_cache[(slot * H + h) * d + t];
                }
                orow[t] = sum_wv / total;
            }
            *lse_bhi = top + log(total);
        }
        free(w);
    }
    return err;
}

/*
 * Lightning-indexer score (the aispot.cmou.io report "llama.cpp 最佳化 lightning
 * indexer 視訊記憶體與多後端支援", release b11372, entry "compute the indexer score
 * with the lightning indexer"): every query token scores every pooled key by the
 * rectified dot product of each of its indexer heads with that key, weighted per
 * head and summed over heads; the keys have no head axis (one key row serves all
 * heads).  An additive pool mask (0 or -inf) follows the sum:
 *
 *   score[b,t,p] = sum_h w[b,t,h] * max(0, sum_c q[b,t,h,c] * kp[b,p,c]) + mask[b,t,p]
 *
 * The report's unweighted variant is w = 1/sqrt(d) for every head.  Readings: the
 * weights may differ per token as well as per head (the per-head case has equal
 * rows); the mask is per (token, pool entry) and may be NULL (no mask).
 * Layouts: q [B, T, H, d], kp [B, P, d], w [B, T, H], mask and score [B, T, P].
 */
int oracle_indexer_score_f64(const double* q, const double* kp, const double* w,
                             const double* mask, double* score,
                             int B, int T, int H, int P, int d)
{
    if (B <= 0 || T <= 0 || H <= 0 || P <= 0 || d <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (long bt = 0; bt < (long)B * T; ++bt) {
        const long b = bt / T, t = bt % T;
        for (long p = 0; p < P; ++p) {
            const double* key = kp + (b * P + p) * d;
            double acc = 0.0;
            for (int h = 0; h < H; ++h) {
                const double* qh = q + ((b * T + t) * H + h) * d;
                double dotp = 0.0;
                for (int c = 0; c < d; ++c) dotp += qh[c] * key[c];
                const double relu = dotp > 0.0 ? dotp : 0.0;
                acc += w[(b * T + t) * H + h] * relu;
            }
            if (mask) acc += mask[(b * T + t) * P + p];
            score[(b * T + t) * P + p] = acc;
        }
    }
    return 0;
}

/*
 * Top-k selection over each score row (the prhub.com.cn report "PR #45743 完整报告",
 * section "实现拆解": the decode-side indexer keeps only the order of the scores,
 * which is why its kernel drops the softmax scale).  For each of R rows of P
 * scores, idx receives the positions of the kk largest finite scores, largest
 * first; equal scores go lowest position first (reading: the report fixes no
 * order among ties); -inf and NaN entries are never chosen, and slots left over
 * when a row has fewer than kk finite scores hold -1.  Layouts: score [R, P],
 * idx [R, kk].
 */
int oracle_topk_f64(const double* score, int R, int P, int kk, int* idx)
{
    if (R <= 0 || P <= 0 || kk <= 0) return -1;
    int err = 0;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < R; ++r) {
        const double* srow = score + r * P;
        char* taken = (char*)calloc((size_t)P, 1);
        if (!taken) {
#pragma omp atomic write
            err = -2;
            continue;
        }
        for (int s = 0; s < kk; ++s) {
            long best = -1;
            for (long j = 0; j < P; ++j) {
                if (taken[j] || !(srow[j] > -INFINITY)) continue;  /* skips -inf and NaN */
                if (best < 0 || srow[j] > srow[best]) best = j;
            }
            idx[r * kk + s] = (int)best;
            if (best >= 0) taken[best] = 1;
        }
        free(taken);
    }
    return err;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
