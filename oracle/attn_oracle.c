/*
 * Exact attention forward, fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker for the
 * CUDA path.  Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline / reference leg may load or call it; the product path never
 * does.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (FlashAttention: Fast and Memory-Efficient Exact Attention
 * with IO-Awareness, wiki notes, section "Problem setting"): for every
 * (batch b, head h) and every selected query row i,
 *
 *     s_j   = scale * sum_t q[i,t] * k[j,t]          for every visible key j
 *     M     = max_j s_j
 *     P_ij  = exp(s_j - M) / sum_j' exp(s_j' - M)      (the softmax row)
 *     O_i   = sum_j P_ij * v_j
 *     LSE_i = M + ln(sum_j exp(s_j - M))
 *
 * The score row and the probability row are materialised in full (this is
 * the "standard attention" the notes contrast with the tiled method, section
 * "IO complexity analysis"); nothing is blocked, fused or reordered.
 *
 * Key padding (flash-attnの代役がVRAMを18GB溶かしていたので87%削った話, §3 and
 * §6): key_pad is NULL or a [B, N] byte mask in which a nonzero byte marks a
 * padded key, excluded from every row of that batch (the key_padding_mask
 * convention: nonzero = ignore, the opposite of a boolean "attend" mask).
 *
 * Block sparsity (FlashAttention: Fast and Memory-Efficient Exact Attention
 * with IO-Awareness, wiki notes, section "Block-sparse FlashAttention"): a
 * predefined block mask M in {0,1}^{Tr x Tc}, Tr = ceil(N / Br) query blocks
 * by Tc = ceil(N / Bc) key blocks, shared by every batch and head; key j is
 * visible to query i only if M[i / Br][j / Bc] != 0.  Padding, causality and
 * the block mask combine (a key must pass all of them).
 *
 * Readings where the pages are silent:
 *   - scale is an explicit argument (the notes' formula omits it);
 *   - LSE is the natural log of sum_j exp(s_j), in scaled-logit units;
 *   - causal is the square top-left mask: key j is visible to query i iff j <= i;
 *   - a row with no visible key (every key it may see is padded) has O = 0 and
 *     LSE = -inf;
 *   - bf16 inputs are widened exactly to fp64 before any arithmetic.
 *
 * Parity status: pinned by the CPU tests (closed forms, invariants, a
 * 40-digit decimal brute force and a NumPy twin).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the top half of an IEEE binary32; widening is exact. */
static double widen_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One query row against one head's keys and values; s and p are scratch rows
 * of length N.  Keys 0..visible-1 are candidates; pad (NULL or [N]) removes
 * the padded ones.  Excluded keys get no score and probability 0. */
static void one_row(const double* qi, const double* kh, const double* vh, int N, int d,
                    double scale, int visible, const unsigned char* pad, const unsigned char* brow,
                    int bc, double* s, double* p, double* oi, double* lse) {
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
    for (int t = 0; t < d; ++t) oi[t] = 0.0;
    if (!any) {
        *lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int j = 0; j < visible; ++j) {
        p[j] = ((pad && pad[j]) || (brow && !brow[j / bc])) ? 0.0 : exp(s[j] - m);
        sum += p[j];
    }
    for (int j = 0; j < visible; ++j) p[j] /= sum;
    for (int j = 0; j < visible; ++j) {
        const double* vj = vh + (size_t)j * d;
        for (int t = 0; t < d; ++t) oi[t] += p[j] * vj[t];
    }
    *lse = m + log(sum);
    (void)N;
}

/* All selected rows of one head.  rows == NULL means every row 0..N-1. */
static void one_head(const double* qh, const double* kh, const double* vh, int N, int d,
                     double scale, int causal, const unsigned char* pad,
                     const unsigned char* block_mask, int br, int bc, const int32_t* rows,
                     int n_rows, double* o, double* lse, int n_threads) {
    const int tc = bc > 0 ? (N + bc - 1) / bc : 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : omp_get_max_threads())
#endif
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* p = (double*)malloc(sizeof(double) * (size_t)N);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (int r = 0; r < n_rows; ++r) {
            int i = rows ? rows[r] : r;
            int visible = causal ? i + 1 : N;
            const unsigned char* brow = block_mask ? block_mask + (size_t)(i / br) * tc : NULL;
            one_row(qh + (size_t)i * d, kh, vh, N, d, scale, visible, pad, brow, bc, s, p,
                    o + (size_t)r * d, lse + r);
        }
        free(s);
        free(p);
    }
    (void)n_threads;
}

static int args_ok(int B, int H, int N, int d, const int32_t* rows, int n_rows) {
    if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
    if (!rows && n_rows != N) return 0;
    if (rows) {
        if (n_rows < 0) return 0;
        for (long r = 0; r < (long)B * H * n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= N) return 0;
    }
    return 1;
}

/*
 * fp64 inputs, layout [B, H, N, d] contiguous.
 * key_pad: NULL or [B, N] bytes, nonzero = padded key.
 * block_mask: NULL or [ceil(N / br), ceil(N / bc)] bytes, nonzero = the
 * (query block, key block) pair is computed; br, bc >= 1 when it is given.
 * rows: NULL (all rows, n_rows must equal N) or int32 [B*H, n_rows], the
 * query rows to evaluate for each head.  o: fp64 [B*H, n_rows, d];
 * lse: fp64 [B*H, n_rows].  Returns 0 on success, -1 on bad arguments.
 */
int attn_oracle_f64(const double* q, const double* k, const double* v, int B, int H, int N,
                    int d, double scale, int causal, const unsigned char* key_pad,
                    const unsigned char* block_mask, int br, int bc, const int32_t* rows,
                    int n_rows, double* o, double* lse, int n_threads) {
    if (!args_ok(B, H, N, d, rows, n_rows)) return -1;
    if (block_mask && (br < 1 || bc < 1)) return -1;
    size_t head = (size_t)N * d;
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const unsigned char* pad = key_pad ? key_pad + (size_t)(bh / H) * N : NULL;
        one_head(q + bh * head, k + bh * head, v + bh * head, N, d, scale, causal, pad, block_mask,
                 br, bc, rows ? rows + bh * n_rows : NULL, n_rows, o + (size_t)bh * n_rows * d,
                 lse + (size_t)bh * n_rows, n_threads);
    }
    return 0;
}

/*
 * bf16 inputs (raw 16-bit patterns), layout [B, H, N, d] contiguous; every
 * value is widened exactly to fp64 first, one head at a time.  Other
 * arguments and outputs as attn_oracle_f64.
 */
int attn_oracle_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H,
                     int N, int d, double scale, int causal, const unsigned char* key_pad,
                     const unsigned char* block_mask, int br, int bc, const int32_t* rows,
                     int n_rows, double* o, double* lse, int n_threads) {
    if (!args_ok(B, H, N, d, rows, n_rows)) return -1;
    if (block_mask && (br < 1 || bc < 1)) return -1;
    size_t head = (size_t)N * d;
    double* qh = (double*)malloc(sizeof(double) * head);
    double* kh = (double*)malloc(sizeof(double) * head);
    double* vh = (double*)malloc(sizeof(double) * head);
    if (!qh || !kh || !vh) {
        free(qh); free(kh); free(vh);
        return -2;
    }
    for (long bh = 0; bh < (long)B * H; ++bh) {
        for (size_t e = 0; e < head; ++e) {
            qh[e] = widen_bf16(q[bh * head + e]);
            kh[e] = widen_bf16(k[bh * head + e]);
            vh[e] = widen_bf16(v[bh * head + e]);
        }
        const unsigned char* pad = key_pad ? key_pad + (size_t)(bh / H) * N : NULL;
        one_head(qh, kh, vh, N, d, scale, causal, pad, block_mask, br, bc,
                 rows ? rows + bh * n_rows : NULL, n_rows,
                 o + (size_t)bh * n_rows * d, lse + (size_t)bh * n_rows, n_threads);
    }
    free(qh); free(kh); free(vh);
    return 0;
}

/* Threads an OpenMP region would use by default (1 without OpenMP). */
int attn_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
