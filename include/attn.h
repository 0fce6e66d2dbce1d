/*
 * attn.h -- C ABI of the exact, IO-aware attention forward library (libattn.so).
 *
 * The operation (FlashAttention: Fast and Memory-Efficient Exact Attention
 * with IO-Awareness, wiki notes, sections "Problem setting", "Tiling",
 * "Recomputation" and "Kernel fusion"): for every batch b and head h,
 *
 *     O[b,h] = softmax(scale * Q[b,h] K[b,h]^T) V[b,h]
 *     LSE[b,h,i] = ln sum_j exp(scale * q_i . k_j)        (natural log)
 *
 * computed tile by tile in one kernel with a running row maximum m and a
 * running row sum l, so the N x N score and probability matrices never reach
 * device memory; the softmax statistics are kept as one fp32 log-sum-exp per
 * query row (per the notes' section "Recomputation", only O and the row
 * statistics outlive the kernel).
 * With causal != 0, key j is visible to query i iff j <= i (square, top-left
 * aligned); tiles entirely above the diagonal are never computed.
 *
 * Every pointer is a DEVICE pointer on the current CUDA device.  The caller
 * owns every buffer; the library allocates no device memory and keeps no
 * pointer after a call returns.  Calls are asynchronous on `stream` and never
 * synchronise the host.
 */
#ifndef EXACT_ATTN_H
#define EXACT_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; 0 is the legacy default stream. */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or scale          */
    ATTN_ERR_UNSUPPORTED = 2,  /* head size other than 64 or 128                  */
    ATTN_ERR_CUDA = 3,         /* a CUDA runtime or driver call failed            */
    ATTN_ERR_TIMEOUT = 4       /* a bounded wait inside a kernel ran out (device) */
} attn_status;

/*
 * attn_fwd -- exact attention forward.
 *
 *   q, k, v : bf16 [B, H, N, d], contiguous, 16-byte aligned, read only.
 *   o       : bf16 [B, H, N, d], contiguous, 16-byte aligned, written.
 *   lse     : fp32 [B, H, N], contiguous, 4-byte aligned, written: natural-log
 *             log-sum-exp of the scaled scores of each query row.
 *   B, H, N : >= 1;  B*H <= 2^31-1;  N <= 2^31-1 - 256.
 *   d       : 64 or 128 (other values return ATTN_ERR_UNSUPPORTED).
 *   scale   : finite and >= 1e-30 (positive); the usual choice is 1/sqrt(d).
 *             Scores scale * q.k must be finite in fp32.
 *   causal  : 0 = every key visible; nonzero = key j visible to query i iff j <= i.
 *   stream  : CUDA stream the kernel is queued on.
 *
 * Each pointer must lie in device memory of the current device, and the
 * allocation that holds it must cover the whole tensor (checked on the host,
 * before anything is launched: violations return ATTN_ERR_INVALID_ARG and
 * nothing is written).  o and lse must not overlap q, k or v.
 * Returns ATTN_OK once the kernel is queued.  A device-side failure (a wait
 * that ran out) is reported later by attn_check_device_status().
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int N, int d, float scale, int causal, attn_stream_t stream);

/*
 * attn_fwd_strided -- attn_fwd on strided tensors, with no copy, and an
 * optional key-padding mask.
 *
 * Element (b, h, n, t) of Q, K and V is at ptr[b*qkv_sb + h*qkv_sh + n*qkv_sn
 * + t]; element (b, h, n, t) of O at o[b*o_sb + h*o_sh + n*o_sn + t] (strides in
 * elements; the head dimension t is contiguous).  This covers, for example,
 * Q, K and V taken as views of one packed projection output [B, N, 3, H, d]
 * (qkv_sb = 3*N*H*d, qkv_sh = d, qkv_sn = 3*H*d) and O written straight into a
 * [B, N, H, d] buffer (o_sb = N*H*d, o_sh = d, o_sn = H*d): the physical
 * layout the pages' patch self-attention module builds before its transpose
 * (flash-attnの代役がVRAMを18GB溶かしていたので87%削った話, §4).  LSE stays
 * contiguous fp32 [B, H, N].
 *
 * key_padding_mask: NULL, or a device byte mask [B, N] (contiguous, read
 * only, any alignment) in which a nonzero byte marks a padded key of that
 * batch: it is excluded from every query row, as the key_padding_mask of the
 * pages' module (same page, §3 and §6: nonzero = ignore, the opposite of a
 * boolean "attend" mask).  A query row with no visible key (all keys it may
 * see padded) gets O = 0 and LSE = -inf.  Reading the mask 16 bytes at a time
 * needs a 16-byte aligned mask and N % 16 == 0; otherwise it is read byte by
 * byte (same result, slower).
 *
 * Every stride must be a positive multiple of 8 (16 bytes, for the tensor
 * memory accelerator and the 16-byte O stores), qkv_sn and o_sn at least d,
 * and each pointer's allocation must cover its strided span.  The d-element
 * rows of O must not alias: taking the dimensions of O with extent > 1 in
 * order of increasing stride, each stride must be at least the span of the
 * rows below it (every contiguous or transposed layout, [B, N, H, d]
 * included, meets this).  Otherwise ATTN_ERR_INVALID_ARG and nothing is
 * launched.  Other arguments, ownership and errors as attn_fwd (which is
 * this call with contiguous strides and no padding).
 */
int attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int N, int d,
                     long long qkv_sb, long long qkv_sh, long long qkv_sn,
                     long long o_sb, long long o_sh, long long o_sn,
                     const unsigned char* key_padding_mask,
                     float scale, int causal, attn_stream_t stream);

/*
 * attn_fwd_block_sparse -- attn_fwd_strided with a block-sparse mask: only the
 * (query block, key block) pairs whose mask entry is nonzero are loaded and
 * multiplied (FlashAttention: Fast and Memory-Efficient Exact Attention with
 * IO-Awareness, wiki notes, section "Block-sparse FlashAttention": a
 * predefined mask M in {0,1}^{N/Br x N/Bc} over the kernel's blocks).
 *
 * block_mask: NULL (then this is exactly attn_fwd_strided), or a device byte
 * matrix [T, T], T = ceil(N / 128), row-major, 16-byte aligned, read only:
 * entry (r, c) nonzero means query rows [128 r, 128 r + 128) may see keys
 * [128 c, 128 c + 128).  Br = Bc = 128 are the kernel's tile sizes.  One mask
 * serves every batch and head.  It combines with causal (a key must also be
 * at or before its query) and with key_padding_mask (and not padded).  A
 * query row left with no visible key gets O = 0 and LSE = -inf.  T must be at
 * most 512 (N <= 65536): the mask is copied to on-chip memory as bits.
 *
 * Work and memory traffic scale with the number of nonzero blocks.  The two
 * 128-row Q tiles of a work unit walk the union of their mask rows, so
 * neighbouring rows with similar patterns cost least.  Other arguments,
 * ownership and errors as attn_fwd_strided; a misaligned or too large mask,
 * or one that overlaps o or lse, gives ATTN_ERR_INVALID_ARG.
 */
int attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d,
                          long long qkv_sb, long long qkv_sh, long long qkv_sn,
                          long long o_sb, long long o_sh, long long o_sn,
                          const unsigned char* key_padding_mask,
                          const unsigned char* block_mask,
                          float scale, int causal, attn_stream_t stream);

/*
 * attn_bwd -- exact attention backward by recomputation (FlashAttention:
 * Fast and Memory-Efficient Exact Attention with IO-Awareness, wiki notes,
 * section "Recomputation": S and P are rebuilt tile by tile from Q, K and the
 * forward's statistics; no N x N matrix is stored).  Given the upstream
 * gradient dO of O = softmax(scale Q K^T) V it writes
 *
 *     dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO,
 *     dS = P o (dO V^T - delta),   delta_i = dO_i . O_i.
 *
 *   q, k, v, o, dout : bf16 [B, H, N, d], contiguous, 16-byte aligned, read
 *                      only; o is the attn_fwd output for these q, k, v.
 *   lse              : fp32 [B, H, N], the attn_fwd LSE, read only.
 *   key_padding_mask : NULL, or the [B, N] byte mask the forward used
 *                      (nonzero = padded key): padded keys get dK = dV = 0
 *                      and no query row attends to them; a row that saw no
 *                      key (LSE = -inf, O = 0) gets dQ = 0.
 *   block_mask       : NULL, or the [T, T] byte block mask the forward used
 *                      (T = ceil(N / 128), see attn_fwd_block_sparse): only
 *                      nonzero (query block, key block) pairs are recomputed;
 *                      a key block no query block meets gets dK = dV = 0.
 *   delta            : fp32 [B, H, N], written (delta_i above; a workspace
 *                      the caller owns, useful to nobody else).
 *   dq               : fp32 [B, H, N, d], written: dQ in fp32 (cleared, then
 *                      accumulated over key blocks by the call itself).
 *   dk, dv           : bf16 [B, H, N, d], written.
 *   d                : 64 or 128 (other values return ATTN_ERR_UNSUPPORTED).
 *   scale, causal, stream, B, H, N : as attn_fwd.
 *
 * Pointers must be device memory of the current device covering their
 * tensors; no output may overlap an input or another output (checked on the
 * host before anything is launched; ATTN_ERR_INVALID_ARG otherwise).  Two
 * kernels are queued on `stream` (delta and the dQ clear, then the backward
 * proper); the library allocates nothing.  Device-side timeouts are reported
 * by attn_check_device_status().
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, const unsigned char* key_padding_mask, const unsigned char* block_mask,
             float* delta, float* dq, void* dk, void* dv,
             int B, int H, int N, int d, float scale, int causal, attn_stream_t stream);

/*
 * attn_bwd_noalloc -- attn_bwd without the delta workspace argument: the
 * call allocates nothing and needs no caller scratch.  The pages have no
 * counterpart; it exists for callers that may not allocate (for example
 * inside a captured CUDA graph).
 *
 * delta is kept in a static device array of the library (1 << 20 fp32 rows,
 * 4 MiB, part of the module image), so B*H*N must be at most 1048576
 * (otherwise ATTN_ERR_INVALID_ARG, checked before anything runs).  Its
 * address is looked up (cudaGetSymbolAddress) on the first call in each CUDA
 * context of a device and cached under that context's id, so a device reset
 * or a new context looks it up again: make the first call in a context
 * outside stream capture.  The
 * array is shared by every call on a device, so calls whose executions may
 * overlap (different streams without ordering between them) race on it:
 * order them on one stream or by events.  Everything else as attn_bwd.
 */
int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, const unsigned char* key_padding_mask, const unsigned char* block_mask,
                     float* dq, void* dk, void* dv,
                     int B, int H, int N, int d, float scale, int causal, attn_stream_t stream);

/* Human-readable name of an attn_status value (static string, never NULL). */
const char* attn_status_string(int status);

/*
 * attn_check_device_status -- synchronise `stream`, then read and clear the
 * library's device status word on the current device.  Returns ATTN_OK,
 * ATTN_ERR_TIMEOUT if any kernel of this library gave up on a bounded wait
 * since the last check (its outputs are then undefined), or ATTN_ERR_CUDA.
 */
int attn_check_device_status(attn_stream_t stream);

/*
 * attn_selftest_wait_timeout -- exercise the bounded-wait path without any
 * fault: queue on `stream` one tiny kernel that waits on a barrier nobody
 * arrives at, with a limit of `limit_ns` nanoseconds (1e3 .. 1e10).  The wait
 * gives up, records ATTN_ERR_TIMEOUT in the device status word and the kernel
 * returns normally; attn_check_device_status() then reports it.
 */
int attn_selftest_wait_timeout(unsigned long long limit_ns, attn_stream_t stream);

/*
 * attn_selftest_ex2 -- evaluate, on the device, the exponential that the
 * forward's softmax runs on the FMA pipe for part of its 2^x evaluations
 * (a degree-3 polynomial for 2^f on [-1/2, 1/2] with 2^round(x) put into the
 * exponent field), so that callers and tests can check it against 2^x.
 *
 *   x : fp32 [n] device buffer of arguments (read only).
 *   y : fp32 [n] device buffer, written: y[i] ~ 2^x[i] for x[i] <= 127,
 *       relative error at most 1.02e-4 for -126 <= x[i] <= 127; exactly +0
 *       for x[i] <= -127 and for x[i] = -inf (a masked score); a subnormal
 *       below 2^-126 for -127 < x[i] < -126.
 *   n : >= 1.  x and y must be 4-byte aligned, must not overlap, and must lie
 *       in device memory of the current device covering n floats
 *       (ATTN_ERR_INVALID_ARG otherwise; nothing is launched).
 *
 * The polynomial is not the page's: the notes compute the softmax with exact
 * exponentials; this is how part of them is evaluated on B200, and the test
 * entry point exists so that its accuracy can be pinned.
 * Asynchronous on `stream`.
 */
int attn_selftest_ex2(const float* x, float* y, int n, attn_stream_t stream);

/* Library version, major*10000 + minor*100 + patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* EXACT_ATTN_H */
