/*
 * Exact attention backward, fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Like attn_oracle.c, this is the independent
 * checker for the CUDA path: only the test suite and the benchmark's
 * CPU-baseline / reference leg may load or call it, and it shares no code,
 * header or constant with the CUDA library.
 *
 * What it computes (FlashAttention: Fast and Memory-Efficient Exact Attention
 * with IO-Awareness, wiki notes, section "Recomputation": the backward pass
 * rebuilds S and P from Q, K and the softmax statistics instead of storing
 * them).  The pages do not print the gradient formulas; the oracle takes the
 * plain reading -- the exact gradients of O = softmax(scale * Q K^T) V with
 * respect to Q, K and V for an upstream gradient dO -- and writes out the
 * chain rule, materialising every row exactly as the standard backward does:
 *
 *     S_ij  = scale * q_i . k_j                   (visible keys only)
 *     P_ij  = exp(S_ij - max_j S_ij) / sum_j exp(S_ij - max_j S_ij)
 *     dV_j  = sum_i P_ij dO_i                     (O = P V)
 *     dP_ij = dO_i . v_j
 *     dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik)     (the softmax Jacobian)
 *     dQ_i  = scale * sum_j dS_ij k_j              (S = scale Q K^T)
 *     dK_j  = scale * sum_i dS_ij q_i
 *
 * Causal: key j is visible to query i iff j <= i.  Key padding (the forward
 * oracle's convention, from flash-attnの代役がVRAMを18GB溶かしていたので87%削った話,
 * §3 and §6): key_pad NULL or [B, N] bytes, nonzero = padded key, invisible to
 * every row.  A row with no visible key has O = 0 whatever Q, K, V are, so
 * its dQ is 0 and it adds nothing to dK, dV.  Block mask (the forward
 * oracle's convention, FlashAttention wiki notes, section "Block-sparse
 * FlashAttention"): NULL or [ceil(N/br), ceil(N/bc)] bytes; key j is visible
 * to query i only if entry (i / br, j / bc) is nonzero.  bf16 inputs are
 * widened exactly to fp64.
 *
 * Parity status: pinned by the CPU tests (central finite differences, the
 * invariants sum_j dK_j = 0, <Q, dQ> = <K, dK> and <V, dV> = <O, dO>, and a
 * second derivation through torch.autograd in fp64).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double widen(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * One head.  q_sel: NULL (every row) or the query rows whose dQ is wanted;
 * k_sel likewise for dK and dV.  dq: [n_q, d]; dk, dv: [n_k, d].
 */
static int bwd_head(const double* qh, const double* kh, const double* vh, const double* doh, int N,
                    int d, double scale, int causal, const unsigned char* pad,
                    const unsigned char* block_mask, int br, int bc, const int32_t* q_sel, int n_q,
                    const int32_t* k_sel, int n_k, double* dq, double* dk, double* dv, int n_threads) {
    /* position of each row in the selections (-1: not selected) */
    int* q_pos = (int*)malloc(sizeof(int) * (size_t)N);
    int* k_pos = (int*)malloc(sizeof(int) * (size_t)N);
    if (!q_pos || !k_pos) {
        free(q_pos); free(k_pos);
        return -2;
    }
    for (int i = 0; i < N; ++i) q_pos[i] = q_sel ? -1 : i;
    for (int j = 0; j < N; ++j) k_pos[j] = k_sel ? -1 : j;
    if (q_sel) for (int r = 0; r < n_q; ++r) q_pos[q_sel[r]] = r;
    if (k_sel) for (int r = 0; r < n_k; ++r) k_pos[k_sel[r]] = r;
    memset(dk, 0, sizeof(double) * (size_t)n_k * d);
    memset(dv, 0, sizeof(double) * (size_t)n_k * d);
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : omp_get_max_threads())
#endif
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* p = (double*)malloc(sizeof(double) * (size_t)N);
        double* dp = (double*)malloc(sizeof(double) * (size_t)N);
        double* dk_part = (double*)calloc((size_t)n_k * d, sizeof(double));
        double* dv_part = (double*)calloc((size_t)n_k * d, sizeof(double));
        if (!s || !p || !dp || !dk_part || !dv_part) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
            for (int i = 0; i < N; ++i) {
                const int visible = causal ? i + 1 : N;
                const double* qi = qh + (size_t)i * d;
                const int tc = bc > 0 ? (N + bc - 1) / bc : 0;
                const unsigned char* brow = block_mask ? block_mask + (size_t)(i / br) * tc : NULL;
                const double* doi = doh + (size_t)i * d;
                /* scores and the softmax row (padded keys: P = 0) */
                double m = -INFINITY;
                int any = 0;
                for (int j = 0; j < visible; ++j) {
                    if ((pad && pad[j]) || (brow && !brow[j / bc])) continue;
                    double acc = 0.0;
                    for (int t = 0; t < d; ++t) acc += qi[t] * kh[(size_t)j * d + t];
                    s[j] = scale * acc;
                    if (!any || s[j] > m) m = s[j];
                    any = 1;
                }
                double sum = 0.0;
                for (int j = 0; j < visible; ++j) {
                    p[j] = ((pad && pad[j]) || (brow && !brow[j / bc])) ? 0.0 : exp(s[j] - m);
                    sum += p[j];
                }
                for (int j = 0; j < visible; ++j) p[j] = any ? p[j] / sum : 0.0;
                /* dP and the row term sum_k P_ik dP_ik */
                double row = 0.0;
                for (int j = 0; j < visible; ++j) {
                    double acc = 0.0;
                    for (int t = 0; t < d; ++t) acc += doi[t] * vh[(size_t)j * d + t];
                    dp[j] = acc;
                    row += p[j] * dp[j];
                }
                /* dS, kept in dp */
                for (int j = 0; j < visible; ++j) dp[j] = p[j] * (dp[j] - row);
                if (q_pos[i] >= 0) {
                    double* out = dq + (size_t)q_pos[i] * d;
                    for (int t = 0; t < d; ++t) out[t] = 0.0;
                    for (int j = 0; j < visible; ++j)
                        for (int t = 0; t < d; ++t) out[t] += dp[j] * kh[(size_t)j * d + t];
                    for (int t = 0; t < d; ++t) out[t] *= scale;
                }
                for (int j = 0; j < visible; ++j) {
                    const int r = k_pos[j];
                    if (r < 0) continue;
                    for (int t = 0; t < d; ++t) {
                        dk_part[(size_t)r * d + t] += scale * dp[j] * qi[t];
                        dv_part[(size_t)r * d + t] += p[j] * doi[t];
                    }
                }
            }
#ifdef _OPENMP
#pragma omp critical
#endif
            {
                for (size_t e = 0; e < (size_t)n_k * d; ++e) {
                    dk[e] += dk_part[e];
                    dv[e] += dv_part[e];
                }
            }
        }
        free(s); free(p); free(dp); free(dk_part); free(dv_part);
    }
    free(q_pos);
    free(k_pos);
    return failed ? -2 : 0;
}

static int sel_ok(const int32_t* sel, long count, int N) {
    if (!sel) return 1;
    for (long r = 0; r < count; ++r)
        if (sel[r] < 0 || sel[r] >= N) return 0;
    return 1;
}

/*
 * bf16 inputs (raw 16-bit patterns) Q, K, V, dO, layout [B, H, N, d]
 * contiguous.  key_pad: NULL or [B, N] bytes, nonzero = padded key.
 * block_mask: NULL or [ceil(N / br), ceil(N / bc)] bytes, nonzero = computed.
 * q_rows: NULL (all rows, n_q must equal N) or int32
 * [B*H, n_q], distinct rows per head; k_rows likewise for dK / dV.
 * dq: fp64 [B*H, n_q, d]; dk, dv: fp64 [B*H, n_k, d].
 * Returns 0, -1 on bad arguments, -2 when out of memory.
 */
int attn_oracle_bwd_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const uint16_t* dout, int B, int H, int N, int d, double scale,
                         int causal, const unsigned char* key_pad, const unsigned char* block_mask,
                         int br, int bc, const int32_t* q_rows, int n_q, const int32_t* k_rows,
                         int n_k, double* dq, double* dk, double* dv, int n_threads) {
    if (B < 1 || H < 1 || N < 1 || d < 1 || n_q < 0 || n_k < 0) return -1;
    if ((!q_rows && n_q != N) || (!k_rows && n_k != N)) return -1;
    if (!sel_ok(q_rows, (long)B * H * n_q, N) || !sel_ok(k_rows, (long)B * H * n_k, N)) return -1;
    if (block_mask && (br < 1 || bc < 1)) return -1;
    const size_t head = (size_t)N * d;
    double* buf = (double*)malloc(sizeof(double) * head * 4);
    if (!buf) return -2;
    double *qh = buf, *kh = buf + head, *vh = buf + 2 * head, *doh = buf + 3 * head;
    int rc = 0;
    for (long bh = 0; rc == 0 && bh < (long)B * H; ++bh) {
        for (size_t e = 0; e < head; ++e) {
            qh[e] = widen(q[bh * head + e]);
            kh[e] = widen(k[bh * head + e]);
            vh[e] = widen(v[bh * head + e]);
            doh[e] = widen(dout[bh * head + e]);
        }
        const unsigned char* pad = key_pad ? key_pad + (size_t)(bh / H) * N : NULL;
        rc = bwd_head(qh, kh, vh, doh, N, d, scale, causal, pad, block_mask, br, bc,
                      q_rows ? q_rows + bh * n_q : NULL, n_q,
                      k_rows ? k_rows + bh * n_k : NULL, n_k, dq + (size_t)bh * n_q * d,
                      dk + (size_t)bh * n_k * d, dv + (size_t)bh * n_k * d, n_threads);
    }
    free(buf);
    return rc;
}

/* fp64 inputs, otherwise as attn_oracle_bwd_bf16. */
int attn_oracle_bwd_f64(const double* q, const double* k, const double* v, const double* dout,
                        int B, int H, int N, int d, double scale, int causal,
                        const unsigned char* key_pad, const unsigned char* block_mask, int br,
                        int bc, const int32_t* q_rows, int n_q, const int32_t* k_rows, int n_k,
                        double* dq, double* dk, double* dv, int n_threads) {
    if (B < 1 || H < 1 || N < 1 || d < 1 || n_q < 0 || n_k < 0) return -1;
    if ((!q_rows && n_q != N) || (!k_rows && n_k != N)) return -1;
    if (!sel_ok(q_rows, (long)B * H * n_q, N) || !sel_ok(k_rows, (long)B * H * n_k, N)) return -1;
    if (block_mask && (br < 1 || bc < 1)) return -1;
    const size_t head = (size_t)N * d;
    int rc = 0;
    for (long bh = 0; rc == 0 && bh < (long)B * H; ++bh)
        rc = bwd_head(q + bh * head, k + bh * head, v + bh * head, dout + bh * head, N, d, scale,
                      causal, key_pad ? key_pad + (size_t)(bh / H) * N : NULL, block_mask, br, bc,
                      q_rows ? q_rows + bh * n_q : NULL, n_q,
                      k_rows ? k_rows + bh * n_k : NULL, n_k, dq + (size_t)bh * n_q * d,
                      dk + (size_t)bh * n_k * d, dv + (size_t)bh * n_k * d, n_threads);
    return rc;
}
