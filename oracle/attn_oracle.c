/*
 * attn_oracle.c -- plain fp64 CPU oracle for the scaled-dot-product attention
 * forward with log-sum-exp output, over varlen batches, grouped-query heads,
 * an optional paged KV cache and causal / patch masks.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg
 * do.  It shares no code with the CUDA library.
 *
 * What it computes (the plain definition, written out without blocking,
 * fusion or reordering):
 *   For sequence b, query head h, query i:
 *     g      = h / (Hq / Hkv)                       grouped-query head sharing
 *     s_ij   = scale * sum_d q[i,h,d] * k[j,g,d]    explicit score row, all j < Lk_b
 *     s_ij   = c * tanh(s_ij / c)                   only with a softcap c > 0
 *     allowed(i,j) by index (none / causal / patch; causal optionally with a
 *                  sliding window of W keys before the diagonal)
 *     M      = max_{allowed j} s_ij
 *     p_ij   = exp(s_ij - M) for allowed j, else 0
 *     O[i,h] = sum_j p_ij v[j,g] / sum_j p_ij
 *     LSE    = M + ln(sum_j p_ij)                   natural log, scale included
 *   A row with no allowed key gives O = 0 and LSE = -inf.
 *
 * Sources (page title, section):
 *   - "[FlexAttention] Enforce Q,K,V memory layouts for fp8 flex attention"
 *     (pytorch commit 7e16cb99), flex_attention docstring: shapes
 *     (B,Hq,L,E)/(B,Hkv,S,E), default scale 1/sqrt(E), enable_gqa; the causal
 *     mask_mod q_idx >= kv_idx in the test's expected graph.
 *   - "Cross Attention does not work on CPU and older GPUs" (BLT issue #6),
 *     FlexAttention lowering arguments: OUTPUT_LOGSUMEXP, ROWS_GUARANTEED_SAFE
 *     False (rows may be fully masked), scale 0.0625 for E = 256.
 *   - "[CUDA] PagedAttention: add SM<80 fp16 fallback via memory-efficient
 *     attention" (onnxruntime PR 28200), Implementation: block_table walk over
 *     the paged cache, packed varlen [total_tokens, num_heads, head_size]
 *     addressed by cumulative sequence lengths, GQA head expansion.
 *   - "Rope dim" (vllm-project/flash-attention PR 172): seqused_k beside the
 *     varlen arguments (number of KV tokens used per sequence).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - causal alignment for Lq != Lk is bottom-right: j <= i + (Lk - Lq); it is
 *     the page's q_idx >= kv_idx when Lq == Lk;
 *   - the patch predicate is start_i <= j < end_i, sequence-local;
 *   - paged layout [num_blocks][block_size][Hkv][D], block_table[b][j / bs];
 *   - "local window on/off" and "softcap 0/50" (the parity matrix of "[CUDA]
 *     PagedAttention: add SM<80 fp16 fallback via memory-efficient
 *     attention", Testing) are read as: a causal row keeps only the keys
 *     i' - W <= j <= i' (i' = i + Lk - Lq, W >= 0; W < 0 means no window),
 *     and a softcap c > 0 maps each scaled score s to c * tanh(s / c)
 *     (c = 0 means none);
 *   - the Qv term of "Rope dim" (overview: Qv GEMM, only_qv) is read as an
 *     extra dot product of a query-side vector qv with the value row,
 *     s_ij = scale * (q.k_j + qv.v_j), with only_qv dropping q.k_j; qv has the
 *     value head dimension, equal to the key one here (attn_oracle_fwd_qv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_MASK_NONE = 0, ORACLE_MASK_CAUSAL = 1, ORACLE_MASK_PATCH = 2 };

/* Row j of head g of sequence b in the K (or V) store. */
static const double *kv_row(const double *base, int b, int j, int g, int Hkv, int D,
                            const int32_t *block_table, int max_blocks_per_seq,
                            int block_size, const int32_t *cu_seqlens_k) {
    long long row;
    if (block_table) {
        int page = block_table[(long long)b * max_blocks_per_seq + j / block_size];
        row = (long long)page * block_size + (j % block_size);
    } else {
        row = (long long)cu_seqlens_k[b] + j;
    }
    return base + (row * Hkv + g) * (long long)D;
}

static int allowed(int mask, int i, int j, int Lq, int Lk, const int32_t *range_i,
                   int window_left) {
    switch (mask) {
    case ORACLE_MASK_NONE: return 1;
    case ORACLE_MASK_CAUSAL:
        if (window_left >= 0 && j < i + (Lk - Lq) - window_left) return 0;
        return j <= i + (Lk - Lq);
    case ORACLE_MASK_PATCH: return range_i[0] <= j && j < range_i[1];
    default: return 0;
    }
}

/*
 * q    [total_q][Hq][D]
 * k, v paged: [num_blocks][block_size][Hkv][D] (block_table != NULL)
 *      else : [total_k][Hkv][D] addressed by cu_seqlens_k
 * Lk_b = seqused_k[b] if seqused_k, else cu_seqlens_k[b+1] - cu_seqlens_k[b]
 * window_left >= 0 only with the causal mask; softcap >= 0 (0: none)
 * o    [total_q][Hq][D];  lse [Hq][total_q]
 * Returns 0, or -1 for arguments it cannot interpret.
 */
int attn_oracle_fwd(const double *q, const double *k, const double *v,
                    const int32_t *block_table, int max_blocks_per_seq, int block_size,
                    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                    const int32_t *seqused_k, int B, int Hq, int Hkv, int D,
                    double scale, int mask, const int32_t *patch_kv_range,
                    int window_left, double softcap,
                    double *o, double *lse, int total_q, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return -1;
    if (window_left >= 0 && mask != ORACLE_MASK_CAUSAL) return -1;
    if (!(softcap >= 0.0)) return -1;
    if (!seqused_k && !cu_seqlens_k) return -1;
    if (!block_table && !cu_seqlens_k) return -1;
    if (mask == ORACLE_MASK_PATCH && !patch_kv_range) return -1;
    const int group = Hq / Hkv;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(|| : bad)
    for (long long task = 0; task < (long long)B * Hq; ++task) {
        const int b = (int)(task / Hq), h = (int)(task % Hq);
        const int g = h / group;
        const int q0 = cu_seqlens_q[b];
        const int Lq = cu_seqlens_q[b + 1] - q0;
        const int Lk = seqused_k ? seqused_k[b] : cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        if (!s) { bad = 1; continue; }
        for (int i = 0; i < Lq; ++i) {
            const double *qi = q + ((long long)(q0 + i) * Hq + h) * D;
            const int32_t *range_i = patch_kv_range ? patch_kv_range + 2LL * (q0 + i) : NULL;
            double *oi = o + ((long long)(q0 + i) * Hq + h) * D;
            double *lse_i = lse + (long long)h * total_q + (q0 + i);
            /* explicit score row */
            for (int j = 0; j < Lk; ++j) {
                const double *kj = kv_row(k, b, j, g, Hkv, D, block_table,
                                          max_blocks_per_seq, block_size, cu_seqlens_k);
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qi[d] * kj[d];
                s[j] = scale * acc;
                if (softcap > 0.0) s[j] = softcap * tanh(s[j] / softcap);
            }
            /* max over the allowed keys */
            double M = -INFINITY;
            int any = 0;
            for (int j = 0; j < Lk; ++j) {
                if (!allowed(mask, i, j, Lq, Lk, range_i, window_left)) continue;
                if (!any || s[j] > M) M = s[j];
                any = 1;
            }
            for (int d = 0; d < D; ++d) oi[d] = 0.0;
            if (!any) { *lse_i = -INFINITY; continue; }
            /* max-subtracted softmax and the weighted sum of V rows */
            double Z = 0.0;
            for (int j = 0; j < Lk; ++j) {
                if (!allowed(mask, i, j, Lq, Lk, range_i, window_left)) continue;
                const double p = exp(s[j] - M);
                const double *vj = kv_row(v, b, j, g, Hkv, D, block_table,
                                          max_blocks_per_seq, block_size, cu_seqlens_k);
                Z += p;
                for (int d = 0; d < D; ++d) oi[d] += p * vj[d];
            }
            for (int d = 0; d < D; ++d) oi[d] /= Z;
            *lse_i = M + log(Z);
        }
        free(s);
    }
    return bad ? -2 : 0;
}

/*
 * Forward with the extra "Qv" score term of "Rope dim" (vllm-project
 * flash-attention PR 172, overview: the Qv GEMM, and an only_qv mode that
 * skips the Q/K loads and the QK GEMM and zero-initialises the score with the
 * Qv GEMM).  Reading: for query i and key j, with qv [total_q][Hq][D] paired
 * with the value rows,
 *   s_ij = scale * (q_i . k_j + qv_i . v_j)        (only_qv: the first term is dropped)
 * then the softcap, masks, softmax, O and LSE exactly as attn_oracle_fwd, over
 * the same packed or paged stores (k is not read with only_qv and may be NULL).
 * Written out plainly (explicit score row, max-subtracted softmax).
 */
int attn_oracle_fwd_qv(const double *q, const double *qv, const double *k, const double *v,
                       const int32_t *block_table, int max_blocks_per_seq, int block_size,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       const int32_t *seqused_k, int B, int Hq, int Hkv, int D, double scale,
                       int mask, const int32_t *patch_kv_range, int window_left, double softcap,
                       int only_qv, double *o, double *lse, int total_q, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return -1;
    if (!qv || !v || (!only_qv && (!q || !k))) return -1;
    if (window_left >= 0 && mask != ORACLE_MASK_CAUSAL) return -1;
    if (!(softcap >= 0.0)) return -1;
    if (!seqused_k && !cu_seqlens_k) return -1;
    if (!block_table && !cu_seqlens_k) return -1;
    if (mask == ORACLE_MASK_PATCH && !patch_kv_range) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(|| : bad)
    for (long long task = 0; task < (long long)B * Hq; ++task) {
        const int b = (int)(task / Hq), h = (int)(task % Hq);
        const int g = h / (Hq / Hkv);   /* the KV head query head h reads */
        const int q0 = cu_seqlens_q[b];
        const int Lq = cu_seqlens_q[b + 1] - q0;
        const int Lk = seqused_k ? seqused_k[b] : cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        double *srow = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        if (!srow) { bad = 1; continue; }
        for (int i = 0; i < Lq; ++i) {
            const double *qi = only_qv ? NULL : q + ((long long)(q0 + i) * Hq + h) * D;
            const double *qvi = qv + ((long long)(q0 + i) * Hq + h) * D;
            const int32_t *range_i = patch_kv_range ? patch_kv_range + 2LL * (q0 + i) : NULL;
            double *oi = o + ((long long)(q0 + i) * Hq + h) * D;
            double *lse_i = lse + (long long)h * total_q + (q0 + i);
            for (int j = 0; j < Lk; ++j) {
                const double *v_j = kv_row(v, b, j, g, Hkv, D, block_table, max_blocks_per_seq,
                                          block_size, cu_seqlens_k);
                double qk = 0.0, qvv = 0.0;
                if (!only_qv) {
                    const double *kj = kv_row(k, b, j, g, Hkv, D, block_table, max_blocks_per_seq,
                                              block_size, cu_seqlens_k);
                    for (int d = 0; d < D; ++d) qk += qi[d] * kj[d];
                }
                for (int d = 0; d < D; ++d) qvv += qvi[d] * v_j[d];
                srow[j] = scale * (qk + qvv);
                if (softcap > 0.0) srow[j] = softcap * tanh(srow[j] / softcap);
            }
            double M = -INFINITY;
            int any = 0;
            for (int j = 0; j < Lk; ++j) {
                if (!allowed(mask, i, j, Lq, Lk, range_i, window_left)) continue;
                if (!any || srow[j] > M) M = srow[j];
                any = 1;
            }
            for (int d = 0; d < D; ++d) oi[d] = 0.0;
            if (!any) { *lse_i = -INFINITY; continue; }
            double Z = 0.0;
            for (int j = 0; j < Lk; ++j) {
                if (!allowed(mask, i, j, Lq, Lk, range_i, window_left)) continue;
                const double pj = exp(srow[j] - M);
                const double *v_j = kv_row(v, b, j, g, Hkv, D, block_table, max_blocks_per_seq,
                                          block_size, cu_seqlens_k);
                Z += pj;
                for (int d = 0; d < D; ++d) oi[d] += pj * v_j[d];
            }
            for (int d = 0; d < D; ++d) oi[d] = oi[d] / Z;
            *lse_i = log(Z) + M;
        }
        free(srow);
    }
    return bad ? -2 : 0;
}

/*
 * Merge of partial results over disjoint key ranges (split-KV):
 *   LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) * O_s
 * o_parts [S][N][D], lse_parts [S][N] -> o [N][D], lse [N].
 * Parts with LSE_s = -inf (no keys) contribute nothing; if every part is
 * empty the result is O = 0, LSE = -inf.
 */
void attn_oracle_combine(const double *o_parts, const double *lse_parts, int S, int N,
                         int D, double *o, double *lse) {
    for (int n = 0; n < N; ++n) {
        double M = -INFINITY;
        for (int s = 0; s < S; ++s)
            if (lse_parts[(long long)s * N + n] > M) M = lse_parts[(long long)s * N + n];
        double *on = o + (long long)n * D;
        for (int d = 0; d < D; ++d) on[d] = 0.0;
        if (M == -INFINITY) { lse[n] = -INFINITY; continue; }
        double W = 0.0;
        for (int s = 0; s < S; ++s) W += exp(lse_parts[(long long)s * N + n] - M);
        lse[n] = M + log(W);
        for (int s = 0; s < S; ++s) {
            const double w = exp(lse_parts[(long long)s * N + n] - lse[n]);
            const double *os = o_parts + ((long long)s * N + n) * D;
            for (int d = 0; d < D; ++d) on[d] += w * os[d];
        }
    }
}

/*
 * Backward of the same forward (the gradients of the attention output, for
 * the training path the BLT page runs through the FlexAttention autograd and
 * the FlashAttnVarlenFunc backward of "Rope dim"), written out as the plain
 * derivative of the definition above.  Packed varlen [total, heads, D]
 * (no paging), masks none / causal (optionally windowed); no softcap.
 *
 * For sequence b, query head h (kv head g), query i and allowed key j:
 *   P_ij     = exp(s_ij - LSE_i)                    the forward's probabilities
 *   dV_j    += P_ij dO_i                            summed over the group's heads
 *   dP_ij    = dO_i . v_j
 *   Delta_i  = sum_j P_ij dP_ij                      (= dO_i . O_i)
 *   dS_ij    = P_ij (dP_ij - Delta_i)
 *   dQ_i     = scale * sum_j dS_ij k_j
 *   dK_j    += scale * dS_ij q_i                    summed over the group's heads
 * O, LSE are recomputed here from q, k, v (exactly, in fp64).  A row with no
 * allowed key contributes nothing and gets dQ = 0.
 *   q, do_ [total_q][Hq][D];  k, v [total_k][Hkv][D];  dq like q; dk, dv like k.
 * Returns 0, or -1 for arguments it cannot interpret.
 */
int attn_oracle_bwd(const double *q, const double *k, const double *v, const double *do_,
                    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int B, int Hq,
                    int Hkv, int D, double scale, int mask, int window_left, double *dq,
                    double *dk, double *dv, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return -1;
    if (!cu_seqlens_q || !cu_seqlens_k) return -1;
    if (mask != ORACLE_MASK_NONE && mask != ORACLE_MASK_CAUSAL) return -1;
    if (window_left >= 0 && mask != ORACLE_MASK_CAUSAL) return -1;
    const int group = Hq / Hkv;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(|| : bad)
    for (long long task = 0; task < (long long)B * Hkv; ++task) {
        const int b = (int)(task / Hkv), g = (int)(task % Hkv);
        const int q0 = cu_seqlens_q[b], k0 = cu_seqlens_k[b];
        const int Lq = cu_seqlens_q[b + 1] - q0, Lk = cu_seqlens_k[b + 1] - k0;
        for (int j = 0; j < Lk; ++j)
            for (int d = 0; d < D; ++d) {
                dk[((long long)(k0 + j) * Hkv + g) * D + d] = 0.0;
                dv[((long long)(k0 + j) * Hkv + g) * D + d] = 0.0;
            }
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        double *p = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        double *dp = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        if (!s || !p || !dp) { bad = 1; free(s); free(p); free(dp); continue; }
        for (int h = g * group; h < (g + 1) * group; ++h) {
            for (int i = 0; i < Lq; ++i) {
                const double *qi = q + ((long long)(q0 + i) * Hq + h) * D;
                const double *doi = do_ + ((long long)(q0 + i) * Hq + h) * D;
                double *dqi = dq + ((long long)(q0 + i) * Hq + h) * D;
                for (int d = 0; d < D; ++d) dqi[d] = 0.0;
                /* scores, max and log-sum-exp of the row (the forward) */
                double M = -INFINITY;
                int any = 0;
                for (int j = 0; j < Lk; ++j) {
                    const double *kj = k + ((long long)(k0 + j) * Hkv + g) * D;
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += qi[d] * kj[d];
                    s[j] = acc * scale;
                    if (!allowed(mask, i, j, Lq, Lk, NULL, window_left)) continue;
                    if (!any || s[j] > M) M = s[j];
                    any = 1;
                }
                if (!any) continue;
                double Z = 0.0;
                for (int j = 0; j < Lk; ++j)
                    if (allowed(mask, i, j, Lq, Lk, NULL, window_left)) Z += exp(s[j] - M);
                const double lse = M + log(Z);
                /* P, dP and Delta */
                double delta = 0.0;
                for (int j = 0; j < Lk; ++j) {
                    if (!allowed(mask, i, j, Lq, Lk, NULL, window_left)) { p[j] = 0.0; dp[j] = 0.0; continue; }
                    p[j] = exp(s[j] - lse);
                    const double *vj = v + ((long long)(k0 + j) * Hkv + g) * D;
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += doi[d] * vj[d];
                    dp[j] = acc;
                    delta += p[j] * dp[j];
                }
                /* gradients */
                for (int j = 0; j < Lk; ++j) {
                    if (p[j] == 0.0) continue;
                    const double ds = p[j] * (dp[j] - delta);
                    const double *kj = k + ((long long)(k0 + j) * Hkv + g) * D;
                    double *dkj = dk + ((long long)(k0 + j) * Hkv + g) * D;
                    double *dvj = dv + ((long long)(k0 + j) * Hkv + g) * D;
                    for (int d = 0; d < D; ++d) {
                        dqi[d] += scale * ds * kj[d];
                        dkj[d] += scale * ds * qi[d];
                        dvj[d] += p[j] * doi[d];
                    }
                }
            }
        }
        free(s);
        free(p);
        free(dp);
    }
    return bad ? -2 : 0;
}
