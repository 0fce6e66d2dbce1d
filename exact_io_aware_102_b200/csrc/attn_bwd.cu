// Exact attention backward for B200 (sm_100a), head sizes 64 and 128.
//
// What is computed (FlashAttention: Fast and Memory-Efficient Exact Attention
// with IO-Awareness, wiki notes, section "Recomputation"): the forward kept
// only O and one log-sum-exp per query row; the backward rebuilds the score
// tiles S = scale Q K^T and the probabilities P = exp(S - LSE) tile by tile on
// chip and never stores an N x N matrix.  For an upstream gradient dO:
//
//     dV = P^T dO,  dP = dO V^T,  dS = P o (dP - delta),  delta_i = dO_i . O_i,
//     dQ = scale dS K,  dK = scale dS^T Q
//
// (delta_i = sum_j P_ij dP_ij, written through O = P V).
//
// How it maps to sm_100a:
//   * a small kernel first writes delta = rowsum(dO o O) and clears the fp32
//     dQ accumulator;
//   * the main kernel runs a persistent grid, one CTA per SM; a work unit is
//     one (batch, head, 128-key block).  dK and dV of the block accumulate in
//     TMEM over the query tiles (128 rows each) the block interacts with;
//   (warp numbers for d = 64; the d = 128 kernel below has its own layout)
//   * warp 20 loads K, V once per unit and Q_i, dO_i per query tile (three
//     stages) by TMA, and writes each tile's offset rows (below); warps 21
//     and 22 issue the tcgen05.mma (each runs its loop with the whole warp,
//     one elected lane issuing): warp 21 S^T = K Q_i^T and dP^T = V dO_i^T
//     into TMEM, warp 22 dV += P^T dO_i, dK += dS^T Q_i and the dQ partial
//     dS K_j;
//   * the row terms of P = 2^(log2(e) (scale S - LSE)) and of dP - delta
//     ride on the tensor core: S^T and dP^T take one more K = 16 slice, the
//     product of a block of ones (keys) with a block holding -LSE/scale
//     (resp. -delta) of each query row, split into three bf16 parts
//     (c = h1 + h2 + h3 to 2^-24 |c|), so the accumulators hold S - LSE/scale
//     and dP - delta and the elementwise warps need no per-column values;
//   * warps 0-15 (four threads per key row: warp w takes query columns
//     32 (w / 4) .. 32 (w / 4) + 31, so each SM sub-partition runs four of
//     them, which hide one another's latency) turn the S^T, dP^T rows into
//     P^T (bf16, into TMEM: the A operand of dV) and dS^T
//     (bf16, into one of two shared-memory buffers in the 128-byte-swizzled
//     layout the tensor core reads -- one dS^T tile serves dK (K-major) and,
//     read transposed, dQ (M-major)).  A tile's P^T and dS^T only wait for
//     dV of the previous tile, so the products of tile i overlap the
//     elementwise work of tile i+1;
//   * warps 16-19 (one thread per query row) read the dQ partial from TMEM and
//     add it to the fp32 dQ accumulator in global memory with tensor
//     reductions (cp.reduce.async.bulk.tensor .add), two [32 x 32] boxes per
//     warp through one staging box;
//   * at the end of a unit warps 0-7 write dV and warps 8-15 dK (times
//     scale) in bf16, 32 columns each, each warp passing its [32 x 32] block
//     through its own bytes of a (then free) dS^T buffer so that four lanes
//     store one 64-byte row segment.
//   Every wait is bounded (see sm100_ptx.cuh) and no barrier spans warps
//   other than mbarriers, so a timeout never leaves a thread blocked.
//
// TMEM columns: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384),
// dQ [384,448), P^T [448,512) (bf16 pairs).  Shared memory (230,656 bytes
// with alignment): K, V (16 KB each), three stages of Q and dO (16 KB each),
// two dS^T buffers (32 KB each, two 64-column halves), four 4 KB dQ staging
// boxes, one offset block per stage and the ones (4 KB each), barriers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "attn.h"
#include "sm100_ptx.cuh"

namespace {

constexpr int kD = 64;            // head size handled here
constexpr int kBK = 128;          // keys per unit (= TMEM lanes)
constexpr int kBQ = 128;          // query rows per tile
// Warps: 0-15 P/dS (four per SM sub-partition, 32 query columns each),
// 16-19 dQ, 20 load, 21-22 MMA (S^T / dP^T; dV, dK, dQ), 23 idle.  Register split (setmaxnreg): the
// block launches with 768 x 80 registers; the four P/dS warpgroups take 88,
// the dQ warpgroup keeps 80, the load / MMA warpgroup gives back to 48
// (512 x 88 + 128 x 80 + 128 x 48 = 768 x 80).
constexpr int kThreads = 768;
constexpr int kPdsWarps = 16;
constexpr int kPdsThreads = kPdsWarps * 32;
constexpr int kDqWarp0 = 16;
constexpr int kLoadWarp = 20;
constexpr int kMmaWarp = 21;
constexpr int kPdsRegs = 88, kCtlRegs = 48, kLaunchRegs = 80;
static_assert(kPdsThreads * kPdsRegs + 128 * kLaunchRegs + 128 * kCtlRegs == kThreads * kLaunchRegs,
              "setmaxnreg split must equal the launch budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 320, kColDQ = 384, kColP = 448;
constexpr float kLog2eB = 1.4426950408889634f;
constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s per wait
constexpr unsigned long long kDrainNs = 100000000ull;   // 0.1 s per drain wait

constexpr int kTile = kBQ * kD * 2;   // one bf16 [128 x 64] tile, 128-byte swizzle
constexpr int kHalf = 128 * 64 * 2;   // one 64-column half of a [128 x 128] bf16 tile
// shared-memory map (offsets from the 1 KB aligned base)
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kTile;
constexpr int kStages = 3;                    // Q / dO stages
constexpr int kOffQ = kOffV + kTile;          // [kStages]
constexpr int kOffDO = kOffQ + kStages * kTile;  // [kStages]
constexpr int kOffDS = kOffDO + kStages * kTile;  // [2] dS^T buffers, each two 64-column halves
constexpr int kDsBytes = 2 * kHalf;
constexpr int kOffStage = kOffDS + 2 * kDsBytes;  // dQ staging: per dQ warp one [32 x 32] fp32 box
constexpr int kStageBoxBytes = 32 * 32 * 4;   // 128-byte-swizzled, as the tensor reduction reads it
// Offset blocks ([128 x 16] bf16, 32-byte swizzle, one K = 16 slice): one
// per stage, holding the tile's Q offsets (-LSE / scale, logical columns 0-2)
// and dO offsets (-delta, columns 8-10), then the block of ones (columns 0-2)
constexpr int kAugBytes = 128 * 16 * 2;
constexpr int kOffAug = kOffStage + 4 * kStageBoxBytes;  // [kStages]
constexpr int kOffOnes = kOffAug + kStages * kAugBytes;
constexpr int kOffBar = kOffOnes + kAugBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
static_assert(kOffAug % 1024 == 0 && kSmemBytes <= 227 * 1024, "shared memory map");

// Barriers.  The tensor-core thread waits on two per query tile (Ready,
// PFull) and commits three (SFull, PTFree, TileDone): each wait or commit
// leaves the shallow tensor-instruction queue to drain for tens of cycles.
struct Bars {
    static constexpr int kKVFull = 0, kKVEmpty = 8;
    // [kStages] tile g may start: its Q, dO (bytes) and offset rows (32 load
    // lanes) have landed, and the P/dS warps (256) have read S^T of tile g-1
    static constexpr int kReady = 16;
    // [kStages] the products of tile g retired: its stage, its dS^T buffer
    // and (for the dQ warps) its dQ partial in TMEM
    static constexpr int kTileDone = 40;
    static constexpr int kSFull = 64;
    // P^T (TMEM) and dS^T (SMEM) of tile g written (256 P/dS threads), and
    // the dQ partial of tile g-1 read (128 dQ threads)
    static constexpr int kPFull = 72;
    static constexpr int kPTFree = 80;   // dV of a tile retired: P^T's TMEM columns free
    static constexpr int kDKVFull = 88, kDKVEmpty = 96;
    static constexpr int kDrain = 104;
    static constexpr int kTmemSlot = 112, kAbort = 116;
    static constexpr int kDrain2 = 120;  // the second issuing warp's drain
};
static_assert(Bars::kReady + 8 * kStages <= Bars::kTileDone && Bars::kTileDone + 8 * kStages <= Bars::kSFull,
              "barrier map");

struct BwdParams {
    int BH, H, N, n_kb, n_qt, total_units, causal;
    const uint8_t* key_pad;     // [B, N] (nonzero = padded key) or null
    const uint8_t* block_mask;  // [n_bt, n_bt] (nonzero = block computed) or null
    int n_bt;                   // ceil(N / 128)
    float scale, scale_log2;
    float neg_inv_scale;  // -1 / scale, rounded once
    const float* lse;     // [BH, N]
    const float* delta;   // [BH, N]
    float* dq;            // [BH, N, 64] fp32, accumulated
    uint16_t* dk;         // [BH, N, 64] bf16
    uint16_t* dv;
    unsigned long long wait_ns;
};

struct BwdUnit {
    int bh, kb, i0;  // head, key block, first query tile
};

// Units: (head, key block).  Non-causal: heads-major, so the CTAs running at
// one time stream the same Q / dO tiles (L2 reuse).  Causal: key block kb
// meets query tiles kb .. n_qt-1; the blocks with most tiles go first, and
// since CTA c takes units c, c + grid, ..., odd rounds run that list
// backwards ("snake" order) so that every CTA's total is close to the mean.
__device__ __forceinline__ BwdUnit bwd_unit(int u, const BwdParams& p) {
    BwdUnit w;
    if (p.causal) {
        const int g = static_cast<int>(gridDim.x);
        const int k = u / g, c = u - k * g;
        const int rem = min(g, p.total_units - k * g);  // the last round may be partial
        const int pos = (k & 1) ? k * g + (rem - 1 - c) : u;
        w.kb = pos / p.BH;
        w.bh = pos - w.kb * p.BH;
        w.i0 = w.kb;
    } else {
        w.bh = u / p.n_kb;
        w.kb = u - w.bh * p.n_kb;
        w.i0 = 0;
    }
    return w;
}

// Query tiles a unit visits: from w.i0 on, those whose block-mask entry
// (query block, key block kb) is nonzero -- every one without a mask.  rows:
// query rows per tile (128 at d = 64, 64 at d = 128); mask blocks are 128.
__device__ __forceinline__ int next_tile(const BwdParams& p, const BwdUnit& w, int i, int rows) {
    if (p.block_mask == nullptr) return i;
    for (; i < p.n_qt; ++i)
        if (p.block_mask[static_cast<size_t>(i * rows / 128) * p.n_bt + w.kb] != 0) break;
    return i;
}

struct Ctx {
    uint32_t base, bar, tmem;
    volatile uint32_t* abort_flag;
    uint8_t* gbase;
    BwdParams p;
};

__device__ __forceinline__ bool wait_b(const Ctx& c, uint32_t bar, uint32_t parity) {
    return wait_bounded(bar, parity, c.abort_flag, c.p.wait_ns);
}

// c = h1 + h2 + h3 with bf16 parts rounded to nearest, |c - (h1 + h2 + h3)|
// <= 2^-24 |c| (each difference is exact in fp32): packed (h1 | h2 << 16, h3)
__device__ __forceinline__ uint2 split_bf16x3(float c) {
    const uint32_t h1 = pack_bf16x2(c, 0.f) & 0xFFFFu;
    const float r1 = c - __uint_as_float(h1 << 16);
    const uint32_t h2 = pack_bf16x2(r1, 0.f) & 0xFFFFu;
    const float r2 = r1 - __uint_as_float(h2 << 16);
    const uint32_t h3 = pack_bf16x2(r2, 0.f) & 0xFFFFu;
    return make_uint2(h1 | (h2 << 16), h3);
}

// The lowest bf16 (-0x1.fep127): the score offset of a query row without
// probability mass (past N, or LSE = -inf), so that every scaled score of the
// row is <= -4.8e8 and its P is exactly 0 (scale >= 1e-30).
constexpr float kNoRowOffset = -0x1.fep127f;

// 32-byte swizzle (K-major, 32-byte rows): logical 16-byte chunk c of row j
// sits at chunk c ^ ((j >> 2) & 1) -- address bit 4 takes bit 7's value.
__device__ __forceinline__ uint32_t sw32_off(int j, int c) {
    return static_cast<uint32_t>(j) * 32u + (static_cast<uint32_t>(c ^ ((j >> 2) & 1)) << 4);
}

// Offset rows of query tile i into one [rows x 16] block: row j holds
// split(-LSE_q / scale) in logical columns 0-2 and split(-delta_q) in columns
// 8-10; the other columns stay zero.  S^T reads the block from its start, dP^T
// 16 bytes in, so that columns 8-15 come first (its columns 8-15 are then
// the next row's first ones, finite, and meet the zeros of the ones block).
// Lane `lane` of the load warp writes rows lane, lane + 32, ...
template <int ROWS>
struct OffsetRows {
    float l[ROWS / 32], d[ROWS / 32];
    __device__ __forceinline__ void fetch(const BwdParams& p, const float* lse_h, const float* dl_h, int row0,
                                          int lane) {
#pragma unroll
        for (int t = 0; t < ROWS / 32; ++t) {
            const int q = row0 + lane + 32 * t;
            l[t] = q < p.N ? lse_h[q] : -INFINITY;
            d[t] = q < p.N ? dl_h[q] : 0.f;
        }
    }
    __device__ __forceinline__ void store(const BwdParams& p, uint32_t aug, int lane) const {
#pragma unroll
        for (int t = 0; t < ROWS / 32; ++t) {
            const int j = lane + 32 * t;
            const bool in = l[t] > -INFINITY;
            const uint2 a = split_bf16x3(in ? l[t] * p.neg_inv_scale : kNoRowOffset);
            const uint2 b = split_bf16x3(in ? -d[t] : 0.f);
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(aug + sw32_off(j, 0)), "r"(a.x), "r"(a.y) : "memory");
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(aug + sw32_off(j, 1)), "r"(b.x), "r"(b.y) : "memory");
        }
    }
};

// Zeroes `bytes` of offset blocks from `zero` and fills the ones block (bf16
// 1.0 in logical columns 0-2 of each of `rows` rows, zero elsewhere); all
// threads of the CTA take part, before the barrier that starts the roles.
__device__ __forceinline__ void init_offset_blocks(uint8_t* zero, int bytes, uint8_t* ones, int rows) {
    for (int k = threadIdx.x; k < bytes / 16; k += blockDim.x)
        reinterpret_cast<uint4*>(zero)[k] = make_uint4(0u, 0u, 0u, 0u);
    for (int k = threadIdx.x; k < rows * 2; k += blockDim.x) {
        const int j = k >> 1, c = k & 1;  // logical chunk c of row j
        *reinterpret_cast<uint4*>(ones + sw32_off(j, c)) =
            c == 0 ? make_uint4(0x3F803F80u, 0x3F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async();
}

// ---------------------------------------------------------------- TMA producer
// The whole warp: lane 0 issues the copies (its arrival on the stage's Ready
// barrier carries the expected bytes); every lane writes offset rows and
// arrives on Ready.
__device__ __forceinline__ void role_load(const Ctx& c, const CUtensorMap* tq, const CUtensorMap* tk,
                                          const CUtensorMap* tv, const CUtensorMap* tdo, int lane) {
    const BwdParams& p = c.p;
    const bool leader = lane == 0;
    uint32_t g = 0;      // query tiles issued
    uint32_t units = 0;  // units whose K / V were issued
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = bwd_unit(u, p);
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) continue;  // no query tile meets this key block
        if (!__all_sync(0xffffffffu, wait_b(c, c.bar + Bars::kKVEmpty, (units & 1) ^ 1))) {
            ok = false;
            break;
        }
        if (leader) {
            mbar_expect_tx(c.bar + Bars::kKVFull, 2 * kTile);
            tma_load_4d(c.base + kOffK, tk, c.bar + Bars::kKVFull, 0, w.kb * kBK, w.bh, 0);
            tma_load_4d(c.base + kOffV, tv, c.bar + Bars::kKVFull, 0, w.kb * kBK, w.bh, 0);
        }
        ++units;
        const float* lse_h = p.lse + static_cast<size_t>(w.bh) * p.N;
        const float* dl_h = p.delta + static_cast<size_t>(w.bh) * p.N;
        for (; i < p.n_qt; i = next_tile(p, w, i + 1, kBQ), ++g) {
            const uint32_t s = g % kStages;
            OffsetRows<kBQ> rows;
            rows.fetch(p, lse_h, dl_h, i * kBQ, lane);  // in flight while the stage drains
            // the stage (and its offset block) is free once tile g-3 retired
            if (!__all_sync(0xffffffffu, wait_b(c, c.bar + Bars::kTileDone + 8 * s, ((g / kStages) & 1) ^ 1))) {
                ok = false;
                break;
            }
            rows.store(p, c.base + kOffAug + s * kAugBytes, lane);
            fence_proxy_async();  // the tensor core reads what the generic proxy wrote
            const uint32_t rb = c.bar + Bars::kReady + 8 * s;
            if (leader) {
                mbar_expect_tx(rb, 2 * kTile);
                tma_load_4d(c.base + kOffQ + s * kTile, tq, rb, 0, i * kBQ, w.bh, 0);
                tma_load_4d(c.base + kOffDO + s * kTile, tdo, rb, 0, i * kBQ, w.bh, 0);
            } else {
                mbar_arrive(rb);
            }
        }
    }
    if (!ok && leader) {
        // every issued copy lands before the CTA may exit (the Ready phases
        // also need arrivals that an aborted CTA may never make: these waits
        // then end at their limit, long after the copies landed)
        if (units > 0) wait_bounded(c.bar + Bars::kKVFull, (units - 1) & 1, nullptr, kDrainNs);
        for (uint32_t k = (g > kStages ? g - kStages : 0); k < g; ++k)
            wait_bounded(c.bar + Bars::kReady + 8 * (k % kStages), (k / kStages) & 1, nullptr, kDrainNs);
    }
    __syncwarp();
}

// ---------------------------------------------------------------- MMA issuing
struct BwdMma {
    static constexpr uint32_t kHi = sdesc_hi_sw128(1024);
    // M = 128, N = 128, both operands K-major (S^T, dP^T)
    static constexpr uint32_t kIdescNN = idesc_bf16_f32(128, 128, false);
    // M = 128, N = 64, A K-major, B M/N-major (dV, dK)
    static constexpr uint32_t kIdescKT = idesc_bf16_f32(128, 64, true);
    // M = 128, N = 64, A and B M/N-major (dQ: A = dS read from the dS^T tile)
    static constexpr uint32_t kIdescTT = idesc_bf16_f32(128, 64, true) | (1u << 15);

    static constexpr uint32_t kHiAug = sdesc_hi_sw32(256);

    // D[128 x 128] = A[128 x 64] B[128 x 64]^T + ones[128 x 16] aug[128 x 16]^T,
    // all K-major: the tile product plus each column's offset
    __device__ __forceinline__ static void nt(uint32_t d, uint32_t a, uint32_t b, uint32_t ones, uint32_t aug,
                                              uint32_t issue) {
        const uint32_t a0 = sdesc_lo(a, 16), b0 = sdesc_lo(b, 16);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss_lo_w(d, a0 + ((kk * 32) >> 4), b0 + ((kk * 32) >> 4), kHi, kIdescNN, kk > 0 ? 1u : 0u,
                        issue);
        mma_ss_lo_w(d, sdesc_lo(ones, 16), sdesc_lo(aug, 16), kHiAug, kIdescNN, 1u, issue);
    }
    // D[128 x 64] (+)= A[128 x 128] B[128 x 64]: A K-major in two 64-column
    // halves, B M/N-major (rows = the 128-long K dimension)
    __device__ __forceinline__ static void kt(uint32_t d, uint32_t a, uint32_t b, bool acc, uint32_t issue) {
        const uint32_t a0 = sdesc_lo(a, 16), b0 = sdesc_lo(b, kHalf);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
            mma_ss_lo_w(d, a0 + (((kk / 4) * kHalf + (kk % 4) * 32) >> 4), b0 + ((kk * 16 * 128) >> 4), kHi,
                        kIdescKT, (acc || kk > 0) ? 1u : 0u, issue);
    }
    // D[128 x 64] (+)= A[128 x 128] B[128 x 64]: A bf16 pairs in TMEM (P^T),
    // B M/N-major
    __device__ __forceinline__ static void ts(uint32_t d, uint32_t a_tmem, uint32_t b, bool acc, uint32_t issue) {
        const uint32_t b0 = sdesc_lo(b, kHalf);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
            mma_ts_lo_w(d, a_tmem + kk * 8, b0 + ((kk * 16 * 128) >> 4), kHi, kIdescKT, (acc || kk > 0) ? 1u : 0u,
                        issue);
    }
    // D[128 x 64] = A[128 x 128] B[128 x 64] with A stored transposed (the
    // dS^T tile: rows = K, two 64-wide halves of M), B M/N-major
    __device__ __forceinline__ static void tt(uint32_t d, uint32_t a_t, uint32_t b, uint32_t issue) {
        const uint32_t a0 = sdesc_lo(a_t, kHalf), b0 = sdesc_lo(b, kHalf);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
            mma_ss_lo_w(d, a0 + ((kk * 16 * 128) >> 4), b0 + ((kk * 16 * 128) >> 4), kHi, kIdescTT,
                        kk > 0 ? 1u : 0u, issue);
    }
};

// Two issuing warps, each running its loop with the whole warp (warp-uniform
// control flow keeps descriptors and counters on the uniform datapath) and one
// elected lane issuing: warp 21 the S^T / dP^T products, warp 22 dV, dK, dQ.
// Either warp's waits, commits and loop overhead then overlap the other's
// products in the shallow tensor instruction queue.  They touch disjoint TMEM
// columns; every cross-stream order goes through the P/dS warps (tile g's
// products need P of tile g, which needs S of tile g).

// S^T - LSE/scale and dP^T - delta of each tile into TMEM, once its inputs
// have landed and the P/dS warps have read the previous tile's.
__device__ __forceinline__ void role_mma_s(const Ctx& c) {
    const BwdParams& p = c.p;
    const uint32_t t = c.tmem;
    bool ok = true;
    const uint32_t issue = elect_lane();
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (ok && !__all_sync(0xffffffffu, wait_b(c, bar, parity))) ok = false;
        return ok;
    };
    uint32_t g = 0, units = 0;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = bwd_unit(u, p);
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) continue;  // no query tile meets this key block
        if (!wait(c.bar + Bars::kKVFull, units & 1)) break;
        for (; ok && i < p.n_qt; i = next_tile(p, w, i + 1, kBQ), ++g) {
            const uint32_t s = g % kStages;
            if (!wait(c.bar + Bars::kReady + 8 * s, (g / kStages) & 1)) break;
            tc_fence_after();
            const uint32_t aug = c.base + kOffAug + s * kAugBytes;
            BwdMma::nt(t + kColS, c.base + kOffK, c.base + kOffQ + s * kTile, c.base + kOffOnes, aug, issue);
            BwdMma::nt(t + kColDP, c.base + kOffV, c.base + kOffDO + s * kTile, c.base + kOffOnes, aug + 16,
                       issue);
            tc_commit_w(c.bar + Bars::kSFull, issue);
        }
        ++units;
    }
    if (!ok) {
        tc_commit_w(c.bar + Bars::kDrain, issue);
        wait_bounded(c.bar + Bars::kDrain, 0, nullptr, kDrainNs);
    }
}

// dV += P^T dO, dK += dS^T Q and the dQ partial dS K of each tile once the
// P/dS warps have written P^T and dS^T (and the dQ warps read the previous
// partial).
__device__ __forceinline__ void role_mma_d(const Ctx& c) {
    const BwdParams& p = c.p;
    const uint32_t t = c.tmem;
    bool ok = true;
    const uint32_t issue = elect_lane();
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (ok && !__all_sync(0xffffffffu, wait_b(c, bar, parity))) ok = false;
        return ok;
    };
    uint32_t g = 0, units = 0;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = bwd_unit(u, p);
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) continue;
        for (int it = 0; ok && i < p.n_qt; ++it, ++g) {
            const int inext = next_tile(p, w, i + 1, kBQ);
            // P^T, dS^T of tile g written and the dQ partial of tile g-1 read
            if (!wait(c.bar + Bars::kPFull, g & 1)) break;
            if (it == 0 && !wait(c.bar + Bars::kDKVEmpty, (units & 1) ^ 1)) break;
            tc_fence_after();
            const uint32_t s = g % kStages;
            const uint32_t ds = c.base + kOffDS + (g & 1) * kDsBytes;
            BwdMma::ts(t + kColDV, t + kColP, c.base + kOffDO + s * kTile, it > 0, issue);  // dV += P^T dO
            tc_commit_w(c.bar + Bars::kPTFree, issue);
            BwdMma::kt(t + kColDK, ds, c.base + kOffQ + s * kTile, it > 0, issue);  // dK += dS^T Q
            BwdMma::tt(t + kColDQ, ds, c.base + kOffK, issue);                       // dQ_j = dS K
            // the stage's last reads (S^T, dP^T of tile g retired before its P existed)
            tc_commit_w(c.bar + Bars::kTileDone + 8 * s, issue);
            if (inext >= p.n_qt) {
                tc_commit_w(c.bar + Bars::kDKVFull, issue);
                tc_commit_w(c.bar + Bars::kKVEmpty, issue);
            }
            i = inext;
        }
        ++units;
    }
    if (!ok) {
        tc_commit_w(c.bar + Bars::kDrain2, issue);
        wait_bounded(c.bar + Bars::kDrain2, 0, nullptr, kDrainNs);
    }
}

// Byte offset of element (row r, column col) of a [128 x 128] bf16 tile kept
// as two 128-byte-swizzled 64-column halves (the layout TMA writes and the
// tensor core reads): 16-byte chunk c of row r sits at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t sw128_off(int r, int col) {
    const int h = col >> 6, c16 = (col & 63) >> 3;
    return static_cast<uint32_t>(h * kHalf + r * 128 + ((c16 ^ (r & 7)) << 4) + (col & 7) * 2);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c4, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c4), "r"(d)
                 : "memory");
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// ---------------------------------------------------------- P / dS warps (0-15)
// Thread = key row r of the unit's block (TMEM lane r) and one quarter (32
// columns) of the 128 query columns of a tile.
__device__ __forceinline__ void role_pds(const Ctx& c, int warp, int lane) {
    const BwdParams& p = c.p;
    const int quarter = warp & 3, part = warp >> 2;
    const int r = quarter * 32 + lane;
    const int col0 = part * 32;  // first query column of this thread
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = c.tmem + lane_off + kColS + col0, t_dp = c.tmem + lane_off + kColDP + col0;
    // unit epilogue: 32 columns of dV (parts 0, 1) or dK (parts 2, 3)
    const uint32_t t_acc = c.tmem + lane_off + (part < 2 ? kColDV : kColDK) + (part & 1) * 32;
    uint16_t* const acc_out = part < 2 ? p.dv : p.dk;
    const int acc_col = (part & 1) * 32;
    const uint32_t t_p = c.tmem + lane_off + kColP + col0 / 2;  // bf16 pairs
    const float sl2 = p.scale_log2;
    uint32_t g = 0, units = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = bwd_unit(u, p);
        const int key = w.kb * kBK + r;
        // padded keys (and rows past N) take no part: P = dS = 0 on their rows
        const bool key_ok = key < p.N && (p.key_pad == nullptr || p.key_pad[static_cast<size_t>(w.bh / p.H) * p.N + key] == 0);
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) {
            // no query tile meets this key block: its dK and dV rows are zero
            if (key < p.N) {
                uint4* dst =
                    reinterpret_cast<uint4*>(acc_out + (static_cast<size_t>(w.bh) * p.N + key) * kD + acc_col);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
            }
            continue;
        }
        for (; i < p.n_qt; ++g) {
            const int inext = next_tile(p, w, i + 1, kBQ);
            bool got = wait_b(c, c.bar + Bars::kSFull, g & 1);
            got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool diag = p.causal && i == w.kb;  // causal: query q sees key r iff q >= r
            // a warp-uniform fast path when no element of the warp's rows is masked
            const bool masked = __any_sync(0xffffffffu, !key_ok || diag);
            const uint32_t ds_buf = c.base + kOffDS + (g & 1) * kDsBytes;
            // this thread's 32 columns of S^T - LSE/scale and dP^T - delta,
            // then release them: the next tile's products start now (rows
            // past N, or without any visible key, carry the lowest offset
            // and give P = dS = 0)
            uint32_t sr[32], dr[32];
            tmem_ld32(t_s, sr);
            tmem_ld32(t_dp, dr);
            tmem_wait_ld();
            reg_fence32(sr);
            reg_fence32(dr);
            tc_fence_before();
            mbar_arrive(c.bar + Bars::kReady + 8 * ((g + 1) % kStages));  // S^T / dP^T may be overwritten
            uint32_t pk[16], dk[16];
            const float2 sl2x2 = make_float2(sl2, sl2);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                float2 x = __fmul2_rn(make_float2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), sl2x2);
                x.x = ex2(x.x);
                x.y = ex2(x.y);
                if (masked) {
                    const int q = col0 + e;
                    if (!key_ok || (diag && q < r)) x.x = 0.f;
                    if (!key_ok || (diag && q + 1 < r)) x.y = 0.f;
                }
                const float2 dsv = __fmul2_rn(x, make_float2(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])));
                pk[e >> 1] = pack_bf16x2(x.x, x.y);
                dk[e >> 1] = pack_bf16x2(dsv.x, dsv.y);
            }
            if (g > 0) {
                // P^T's TMEM columns: dV of the previous tile must have retired
                bool free = wait_b(c, c.bar + Bars::kPTFree, (g - 1) & 1);
                free = __all_sync(0xffffffffu, free);
                if (!free) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            if (g > 1) {
                // this dS^T buffer: dK and dQ of tile g-2 must have retired
                bool free = wait_b(c, c.bar + Bars::kTileDone + 8 * ((g - 2) % kStages), ((g - 2) / kStages) & 1);
                free = __all_sync(0xffffffffu, free);
                if (!free) {
                    ok = false;
                    break;
                }
            }
            tmem_st16(t_p, pk);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
                const uint32_t off = sw128_off(r, col0 + q8 * 8);
                st_shared_v4(ds_buf + off, dk[q8 * 4], dk[q8 * 4 + 1], dk[q8 * 4 + 2], dk[q8 * 4 + 3]);
            }
            if (!ok) break;
            tmem_wait_st();
            tc_fence_before();
            fence_proxy_async();  // the tensor core reads what the generic proxy wrote
            mbar_arrive(c.bar + Bars::kPFull);
            i = inext;
        }
        if (!ok) break;
        // unit epilogue: 32 columns of dV (warps 0-7) or dK times scale
        // (warps 8-15) of this key row
        bool got = wait_b(c, c.bar + Bars::kDKVFull, units & 1);
        got = __all_sync(0xffffffffu, got);
        if (!got) {
            ok = false;
            break;
        }
        ++units;
        tc_fence_after();
        uint32_t acc[32];
        tmem_ld32(t_acc, acc);
        tmem_wait_ld();
        reg_fence32(acc);
        tc_fence_before();
        mbar_arrive(c.bar + Bars::kDKVEmpty);
        // The warp's 32 rows x 32 columns go out through its own 2 KB of a
        // dS^T buffer (the same bytes it writes dS^T to; free between units:
        // the unit's products have retired and this warp's next dS^T comes
        // later), so that a store covers 64-byte row segments of 8 rows
        // instead of 32 scattered 16-byte pieces.  Padded keys store their
        // (zero) rows too.
        {
            const float f = part < 2 ? 1.f : p.scale;
            const uint32_t scratch = c.base + kOffDS;
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
                uint32_t x[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int cc = v4 * 8 + e * 2;
                    x[e] = pack_bf16x2(__uint_as_float(acc[cc]) * f, __uint_as_float(acc[cc + 1]) * f);
                }
                st_shared_v4(scratch + sw128_off(r, col0 + v4 * 8), x[0], x[1], x[2], x[3]);
            }
            __syncwarp();
#pragma unroll
            for (int k8 = 0; k8 < 4; ++k8) {
                const int rr = quarter * 32 + 8 * k8 + (lane >> 2), ch = lane & 3;
                const uint4 v = lds_u32x4(scratch + sw128_off(rr, col0 + ch * 8));
                const int key_rr = w.kb * kBK + rr;
                if (key_rr < p.N)
                    *reinterpret_cast<uint4*>(acc_out + (static_cast<size_t>(w.bh) * p.N + key_rr) * kD + acc_col +
                                              ch * 8) = v;
            }
            __syncwarp();
        }
    }
}

// ------------------------------------------------------------ dQ warps (16-19)
// Thread = query row of the tile = TMEM lane.  Each warp reads its 32 rows
// (64 columns) from TMEM, releases the accumulator, and adds them to dQ as
// two [32 x 32] fp32 boxes, one after the other through one 128-byte-
// swizzled staging box, with tensor reductions (cp.reduce.async.bulk.tensor
// .add); the tensor map clips rows past N.
__device__ __forceinline__ void role_dq(const Ctx& c, const CUtensorMap* tm_dq, int warp, int lane) {
    const BwdParams& p = c.p;
    const int quarter = warp & 3;
    const uint32_t t_dq = c.tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kColDQ;
    const uint32_t stage = c.base + kOffStage + quarter * kStageBoxBytes;
    uint32_t g = 0;
    bool pending = false;  // lane 0: this warp's last reduction may still read the staging box
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = bwd_unit(u, p);
        for (int i = next_tile(p, w, w.i0, kBQ); i < p.n_qt; i = next_tile(p, w, i + 1, kBQ), ++g) {
            bool got = wait_b(c, c.bar + Bars::kTileDone + 8 * (g % kStages), (g / kStages) & 1);
            got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t a[2][32];
            tmem_ld32(t_dq, a[0]);
            tmem_ld32(t_dq + 32, a[1]);
            tmem_wait_ld();
            reg_fence32(a[0]);
            reg_fence32(a[1]);
            tc_fence_before();
            mbar_arrive(c.bar + Bars::kPFull);  // counts toward tile g+1
            const int row0 = i * kBQ + quarter * 32;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // the box is free once the previous reduction has read it
                if (lane == 0 && pending) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                pending = false;
                __syncwarp();
                // row `lane` of the box: 16-byte chunk v4 at chunk v4 ^ (lane % 8)
#pragma unroll
                for (int v4 = 0; v4 < 8; ++v4)
                    st_shared_v4(stage + lane * 128 + ((v4 ^ (lane & 7)) << 4),
                                 __float_as_uint(__uint_as_float(a[h][v4 * 4]) * p.scale),
                                 __float_as_uint(__uint_as_float(a[h][v4 * 4 + 1]) * p.scale),
                                 __float_as_uint(__uint_as_float(a[h][v4 * 4 + 2]) * p.scale),
                                 __float_as_uint(__uint_as_float(a[h][v4 * 4 + 3]) * p.scale));
                fence_proxy_async();
                __syncwarp();
                if (lane == 0 && row0 < p.N) {
                    asm volatile(
                        "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3}], [%4];"
                        ::"l"(reinterpret_cast<uint64_t>(tm_dq)), "r"(h * 32), "r"(row0), "r"(w.bh), "r"(stage)
                        : "memory");
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    pending = true;
                }
            }
        }
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
}

// ------------------------------------------------------------------ kernels
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gbase = smem_raw + (base - raw);
    const uint32_t bar = base + kOffBar;
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + kOffBar + Bars::kAbort);
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + Bars::kTmemSlot);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar + Bars::kKVFull, 1);
        mbar_init(bar + Bars::kKVEmpty, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar + Bars::kReady + 8 * s, kPdsThreads + 32);  // P/dS threads, load lanes
            mbar_init(bar + Bars::kTileDone + 8 * s, 1);
        }
        mbar_init(bar + Bars::kSFull, 1);
        mbar_init(bar + Bars::kPFull, kPdsThreads + kBQ);  // P/dS threads, dQ threads
        mbar_init(bar + Bars::kPTFree, 1);
        mbar_init(bar + Bars::kDKVFull, 1);
        mbar_init(bar + Bars::kDKVEmpty, kPdsThreads);
        mbar_init(bar + Bars::kDrain, 1);
        mbar_init(bar + Bars::kDrain2, 1);
        *abort_flag = 0u;
        fence_barrier_init();
        fence_proxy_async();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
        prefetch_tmap(&tm_dq);
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    init_offset_blocks(gbase + kOffAug, kStages * kAugBytes, gbase + kOffOnes, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const Ctx ctx{base, bar, *tmem_slot, abort_flag, gbase, p};
    if (warp < kPdsWarps) {
        regs_increase<kPdsRegs>();
        mbar_arrive(bar + Bars::kReady);  // tile 0 has no earlier S^T to read
        role_pds(ctx, warp, lane);
    } else if (warp < kDqWarp0 + 4) {
        mbar_arrive(bar + Bars::kPFull);  // tile 0 has no earlier dQ partial
        role_dq(ctx, &tm_dq, warp, lane);
    } else {
        regs_decrease<kCtlRegs>();
        if (warp == kLoadWarp) {
            role_load(ctx, &tm_q, &tm_k, &tm_v, &tm_do, lane);
        } else if (warp == kMmaWarp) {
            role_mma_s(ctx);
        } else if (warp == kMmaWarp + 1) {
            role_mma_d(ctx);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(ctx.tmem, kTmemCols);
    }
}

// delta[row] = sum_t dO[row, t] * O[row, t] (fp32), and the dQ accumulator
// cleared; one thread per row of D elements.
template <int D>
__global__ void attn_bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                     float* __restrict__ delta, float* __restrict__ dq, long long rows) {
    for (long long row = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; row < rows;
         row += static_cast<long long>(gridDim.x) * blockDim.x) {
        const uint4* a = reinterpret_cast<const uint4*>(o + row * D);
        const uint4* b = reinterpret_cast<const uint4*>(dout + row * D);
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < D / 8; ++v) {
            const uint4 x = a[v], y = b[v];
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc = fmaf(__uint_as_float(xs[e] << 16), __uint_as_float(ys[e] << 16), acc);
                acc = fmaf(__uint_as_float(xs[e] & 0xFFFF0000u), __uint_as_float(ys[e] & 0xFFFF0000u), acc);
            }
        }
        delta[row] = acc;
        float4* z = reinterpret_cast<float4*>(dq + row * D);
#pragma unroll
        for (int v = 0; v < D / 4; ++v) z[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ============================================================== head size 128
// The same backward at d = 128 with 64-row query tiles, so that TMEM holds
// dV and dK (128 columns each): S^T [0,64), dP^T [64,128), dV [128,256),
// dK [256,384), dQ^T [384,448), P^T [448,480).  dQ is formed transposed,
// dQ^T = K^T dS^T (M = 128 over the head dimension), because a 64-row dQ tile
// would need the M = 64 accumulator shape; warps 8-11 (one thread per head
// column) write it transposed into a [64 x 128] fp32 staging tile, which one
// bulk reduction (32 KB, contiguous in dQ) adds to the accumulator.
namespace b128 {

constexpr int kThreads = 512;     // warps 0-7 P/dS, 8-11 dQ, 12 load, 13-14 MMA, 15 idle
// Register split (setmaxnreg): the block launches with 512 x 128 registers;
// the two P/dS warpgroups take 176 each, the dQ and load/MMA warpgroups keep
// 80 (256 x 176 + 256 x 80 = 512 x 128).
constexpr int kPdsRegs = 176;
constexpr int kOtherRegs = 80;
static_assert(256 * kPdsRegs + 256 * kOtherRegs == kThreads * 128, "setmaxnreg split must equal the launch budget");
constexpr int kPdsWarps = 8;      // two per SM sub-partition: query columns 0-31 and 32-63
constexpr int kPdsThreads = kPdsWarps * 32;
constexpr int kDqWarp0 = 8;
constexpr int kLoadWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kD = 128;
constexpr int kBQ = 64;                     // query rows per tile
constexpr uint32_t kColS = 0, kColDP = 64, kColDV = 128, kColDK = 256, kColDQ = 384, kColP = 448;
constexpr int kKHalf = 128 * 64 * 2;        // a [128 x 64] bf16 half of the K or V tile
constexpr int kQHalf = 64 * 64 * 2;         // a [64 x 64] bf16 half of a Q or dO tile
constexpr int kKTile = 2 * kKHalf;
constexpr int kQTile = 2 * kQHalf;
constexpr int kDsTile = 128 * 64 * 2;       // dS^T [128 keys x 64 queries], one 128-byte-swizzled half
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKTile;
constexpr int kOffQ = kOffV + kKTile;       // [2] stages
constexpr int kOffDO = kOffQ + 2 * kQTile;  // [2] stages
constexpr int kOffDS = kOffDO + 2 * kQTile; // [2] dS^T buffers
constexpr int kOffStage = kOffDS + 2 * kDsTile;  // dQ staging: [64 rows x 128] fp32, row-major
constexpr int kStageBytes = kBQ * kD * 4;
constexpr int kOffRow = kOffStage + kStageBytes;  // per P/dS warp: lse2[32], delta[32]
constexpr int kRowWarpBytes = 2 * 32 * 4;
constexpr int kOffBar = kOffRow + kPdsWarps * kRowWarpBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

struct Bars {
    static constexpr int kKVFull = 0, kKVEmpty = 8;
    static constexpr int kQFull = 16, kQEmpty = 32;  // [2] each
    static constexpr int kSFull = 48, kSFree = 56;
    static constexpr int kPFull = 64, kPTFree = 72;
    static constexpr int kDQFull = 80, kDQEmpty = 88;
    static constexpr int kDKVFull = 96, kDKVEmpty = 104;
    static constexpr int kDrain = 112;
    static constexpr int kDsFree = 120;              // [2]
    static constexpr int kStageFull = 136;           // 128 dQ threads wrote the staging tile
    static constexpr int kStageFree = 144;           // its bulk reduction has read it
    static constexpr int kTmemSlot = 152, kAbort = 156;
    static constexpr int kDrain2 = 160;
};

// Causal: key block kb (keys 128 kb ..) meets 64-row query tiles 2 kb ..
__device__ __forceinline__ BwdUnit unit(int u, const BwdParams& p) {
    BwdUnit w = bwd_unit(u, p);
    if (p.causal) w.i0 = 2 * w.kb;
    return w;
}

__device__ __forceinline__ void role_load(const Ctx& c, const CUtensorMap* tq, const CUtensorMap* tk,
                                          const CUtensorMap* tv, const CUtensorMap* tdo) {
    const BwdParams& p = c.p;
    uint32_t g = 0, units = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = unit(u, p);
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) continue;  // no query tile meets this key block
        if (!wait_b(c, c.bar + Bars::kKVEmpty, (units & 1) ^ 1)) {
            ok = false;
            break;
        }
        mbar_expect_tx(c.bar + Bars::kKVFull, 2 * kKTile);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(c.base + kOffK + x * kKHalf, tk, c.bar + Bars::kKVFull, x * 64, w.kb * 128, w.bh, 0);
            tma_load_4d(c.base + kOffV + x * kKHalf, tv, c.bar + Bars::kKVFull, x * 64, w.kb * 128, w.bh, 0);
        }
        ++units;
        for (; i < p.n_qt; i = next_tile(p, w, i + 1, kBQ), ++g) {
            const uint32_t s = g & 1;
            if (!wait_b(c, c.bar + Bars::kQEmpty + 8 * s, ((g >> 1) & 1) ^ 1)) {
                ok = false;
                break;
            }
            const uint32_t fb = c.bar + Bars::kQFull + 8 * s;
            mbar_expect_tx(fb, 2 * kQTile);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                tma_load_4d(c.base + kOffQ + s * kQTile + x * kQHalf, tq, fb, x * 64, i * kBQ, w.bh, 0);
                tma_load_4d(c.base + kOffDO + s * kQTile + x * kQHalf, tdo, fb, x * 64, i * kBQ, w.bh, 0);
            }
        }
    }
    if (!ok) {
        if (units > 0) wait_bounded(c.bar + Bars::kKVFull, (units - 1) & 1, nullptr, kDrainNs);
        for (uint32_t k = (g > 2 ? g - 2 : 0); k < g; ++k)
            wait_bounded(c.bar + Bars::kQFull + 8 * (k & 1), (k >> 1) & 1, nullptr, kDrainNs);
    }
}

struct Mma {
    static constexpr uint32_t kHi = sdesc_hi_sw128(1024);
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, false);                 // S^T, dP^T
    static constexpr uint32_t kIdescKV = idesc_bf16_f32(128, 128, true);                // dV, dK
    static constexpr uint32_t kIdescQ = idesc_bf16_f32(128, 64, true) | (1u << 15);     // dQ^T
    // D[128 x 64] = A[128 x 128] B[64 x 128]^T: A a K / V tile, B a Q / dO tile,
    // both K-major in two 64-column halves
    __device__ __forceinline__ static void nt(uint32_t d, uint32_t a, uint32_t b, uint32_t issue) {
        const uint32_t a0 = sdesc_lo(a, 16), b0 = sdesc_lo(b, 16);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
            mma_ss_lo_w(d, a0 + (((kk / 4) * kKHalf + (kk % 4) * 32) >> 4),
                      b0 + (((kk / 4) * kQHalf + (kk % 4) * 32) >> 4), kHi, kIdescS, kk > 0 ? 1u : 0u, issue);
    }
    // dV (+)= P^T dO: A = P^T bf16 pairs in TMEM (K = 64 queries), B = the dO
    // tile M/N-major (N = 128 over two 64-column halves)
    __device__ __forceinline__ static void pv(uint32_t d, uint32_t a_tmem, uint32_t b, bool acc, uint32_t issue) {
        const uint32_t b0 = sdesc_lo(b, kQHalf);
#pragma unroll
        for (int kk = 0; kk < kBQ / 16; ++kk)
            mma_ts_lo_w(d, a_tmem + kk * 8, b0 + ((kk * 16 * 128) >> 4), kHi, kIdescKV, (acc || kk > 0) ? 1u : 0u,
                        issue);
    }
    // dK (+)= dS^T Q: A = dS^T K-major (one 64-wide half), B = the Q tile M/N-major
    __device__ __forceinline__ static void dsq(uint32_t d, uint32_t a, uint32_t b, bool acc, uint32_t issue) {
        const uint32_t a0 = sdesc_lo(a, 16), b0 = sdesc_lo(b, kQHalf);
#pragma unroll
        for (int kk = 0; kk < kBQ / 16; ++kk)
            mma_ss_lo_w(d, a0 + ((kk * 32) >> 4), b0 + ((kk * 16 * 128) >> 4), kHi, kIdescKV,
                        (acc || kk > 0) ? 1u : 0u, issue);
    }
    // dQ^T = K^T dS^T: A = the K tile read M-major (M = 128 head columns over two
    // halves, K = 128 keys), B = dS^T M/N-major (N = 64 queries)
    __device__ __forceinline__ static void kds(uint32_t d, uint32_t a, uint32_t b, uint32_t issue) {
        const uint32_t a0 = sdesc_lo(a, kKHalf), b0 = sdesc_lo(b, kDsTile);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
            mma_ss_lo_w(d, a0 + ((kk * 16 * 128) >> 4), b0 + ((kk * 16 * 128) >> 4), kHi, kIdescQ, kk > 0 ? 1u : 0u,
                        issue);
    }
};

// Two issuing warps, as at d = 64: warp 13 S^T / dP^T, warp 14 dV, dK, dQ^T.
__device__ __forceinline__ void role_mma_s(const Ctx& c) {
    const BwdParams& p = c.p;
    const uint32_t t = c.tmem;
    bool ok = true;
    const uint32_t issue = elect_lane();
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (ok && !__all_sync(0xffffffffu, wait_b(c, bar, parity))) ok = false;
        return ok;
    };
    uint32_t g = 0, units = 0;
    auto issue_s = [&](uint32_t gg) {
        const uint32_t s = gg & 1;
        if (!wait(c.bar + Bars::kQFull + 8 * s, (gg >> 1) & 1)) return;
        if (gg > 0 && !wait(c.bar + Bars::kSFree, (gg - 1) & 1)) return;
        tc_fence_after();
        Mma::nt(t + kColS, c.base + kOffK, c.base + kOffQ + s * kQTile, issue);
        Mma::nt(t + kColDP, c.base + kOffV, c.base + kOffDO + s * kQTile, issue);
        tc_commit_w(c.bar + Bars::kSFull, issue);
    };
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = unit(u, p);
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) continue;  // no query tile meets this key block
        if (!wait(c.bar + Bars::kKVFull, units & 1)) break;
        for (; ok && i < p.n_qt; i = next_tile(p, w, i + 1, kBQ), ++g) issue_s(g);
        ++units;
    }
    if (!ok) {
        tc_commit_w(c.bar + Bars::kDrain, issue);
        wait_bounded(c.bar + Bars::kDrain, 0, nullptr, kDrainNs);
    }
}

__device__ __forceinline__ void role_mma_d(const Ctx& c) {
    const BwdParams& p = c.p;
    const uint32_t t = c.tmem;
    bool ok = true;
    const uint32_t issue = elect_lane();
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (ok && !__all_sync(0xffffffffu, wait_b(c, bar, parity))) ok = false;
        return ok;
    };
    uint32_t g = 0, units = 0;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = unit(u, p);
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) continue;  // no query tile meets this key block
        for (int it = 0; ok && i < p.n_qt; ++it, ++g) {
            const int inext = next_tile(p, w, i + 1, kBQ);
            if (!wait(c.bar + Bars::kPFull, g & 1)) break;
            if (it == 0 && !wait(c.bar + Bars::kDKVEmpty, (units & 1) ^ 1)) break;
            tc_fence_after();
            const uint32_t s = g & 1, ds = c.base + kOffDS + s * kDsTile;
            Mma::pv(t + kColDV, t + kColP, c.base + kOffDO + s * kQTile, it > 0, issue);   // dV += P^T dO
            tc_commit_w(c.bar + Bars::kPTFree, issue);
            Mma::dsq(t + kColDK, ds, c.base + kOffQ + s * kQTile, it > 0, issue);         // dK += dS^T Q
            if (!wait(c.bar + Bars::kDQEmpty, (g & 1) ^ 1)) break;
            tc_fence_after();
            Mma::kds(t + kColDQ, c.base + kOffK, ds, issue);                                // dQ^T = K^T dS^T
            tc_commit_w(c.bar + Bars::kDsFree + 8 * s, issue);
            tc_commit_w(c.bar + Bars::kQEmpty + 8 * s, issue);
            tc_commit_w(c.bar + Bars::kDQFull, issue);
            if (inext >= p.n_qt) {
                tc_commit_w(c.bar + Bars::kDKVFull, issue);
                tc_commit_w(c.bar + Bars::kKVEmpty, issue);
            }
            i = inext;
        }
        ++units;
    }
    if (!ok) {
        tc_commit_w(c.bar + Bars::kDrain2, issue);
        wait_bounded(c.bar + Bars::kDrain2, 0, nullptr, kDrainNs);
    }
}

// Thread = key row r (TMEM lane) and 32 of the tile's 64 query columns.
__device__ __forceinline__ void role_pds(const Ctx& c, int warp, int lane) {
    const BwdParams& p = c.p;
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int col0 = half * 32;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = c.tmem + lane_off + kColS + col0, t_dp = c.tmem + lane_off + kColDP + col0;
    const uint32_t t_p = c.tmem + lane_off + kColP + col0 / 2;
    const uint32_t t_acc = c.tmem + lane_off + (half == 0 ? kColDV : kColDK);
    const uint32_t rows_smem = c.base + kOffRow + warp * kRowWarpBytes;  // lse2[32], delta[32]
    const float sl2 = p.scale_log2;
    uint32_t g = 0, units = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = unit(u, p);
        const int key = w.kb * 128 + r;
        const bool key_ok = key < p.N && (p.key_pad == nullptr || p.key_pad[static_cast<size_t>(w.bh / p.H) * p.N + key] == 0);
        const float* lse_h = p.lse + static_cast<size_t>(w.bh) * p.N;
        const float* dl_h = p.delta + static_cast<size_t>(w.bh) * p.N;
        // fetched one tile ahead, converted when staged (as at d = 64)
        float raw_l, raw_d;
        auto fetch = [&](int i) {
            const int q = i * kBQ + col0 + lane;
            raw_l = q < p.N ? lse_h[q] : -INFINITY;
            raw_d = q < p.N ? dl_h[q] : 0.f;
        };
        int i = next_tile(p, w, w.i0, kBQ);
        if (i >= p.n_qt) {
            // no query tile meets this key block: its dK and dV rows are zero
            if (key < p.N) {
                uint4* dst = reinterpret_cast<uint4*>((half == 0 ? p.dv : p.dk) +
                                                      (static_cast<size_t>(w.bh) * p.N + key) * kD);
#pragma unroll
                for (int v4 = 0; v4 < kD / 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
            }
            continue;
        }
        fetch(i);
        for (; i < p.n_qt; ++g) {
            const bool in = raw_l > -INFINITY;
            const float pre_l = in ? raw_l * kLog2eB : INFINITY, pre_d = in ? raw_d : 0.f;
            __syncwarp();
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(rows_smem + lane * 4), "f"(pre_l) : "memory");
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(rows_smem + 128 + lane * 4), "f"(pre_d) : "memory");
            __syncwarp();
            const int inext = next_tile(p, w, i + 1, kBQ);
            if (inext < p.n_qt) fetch(inext);
            bool got = wait_b(c, c.bar + Bars::kSFull, g & 1);
            got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[32], dr[32];
            tmem_ld32(t_s, sr);
            tmem_ld32(t_dp, dr);
            tmem_wait_ld();
            reg_fence32(sr);
            reg_fence32(dr);
            tc_fence_before();
            mbar_arrive(c.bar + Bars::kSFree);
            // causal: query 64 i + col sees key 128 kb + r iff it is not smaller
            const bool diag = p.causal && (i >> 1) == w.kb;
            const bool masked = __any_sync(0xffffffffu, !key_ok || diag);
            const int qbase = i * kBQ + col0 - w.kb * 128;  // query minus key block start
            uint32_t pk[16], dk[16];
            const float2 sl2x2 = make_float2(sl2, sl2);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const float4 l2 = ld_shared_f4(rows_smem + v * 16);
                const float4 dl = ld_shared_f4(rows_smem + 128 + v * 16);
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int e = v * 4 + e2 * 2;
                    const float2 nl = e2 == 0 ? make_float2(-l2.x, -l2.y) : make_float2(-l2.z, -l2.w);
                    const float2 nd = e2 == 0 ? make_float2(-dl.x, -dl.y) : make_float2(-dl.z, -dl.w);
                    float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), sl2x2, nl);
                    x.x = ex2(x.x);
                    x.y = ex2(x.y);
                    if (masked) {
                        if (!key_ok || (diag && qbase + e < r)) x.x = 0.f;
                        if (!key_ok || (diag && qbase + e + 1 < r)) x.y = 0.f;
                    }
                    const float2 dsv =
                        __fmul2_rn(x, __fadd2_rn(make_float2(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), nd));
                    pk[e >> 1] = pack_bf16x2(x.x, x.y);
                    dk[e >> 1] = pack_bf16x2(dsv.x, dsv.y);
                }
            }
            if (g > 0) {
                bool free = wait_b(c, c.bar + Bars::kPTFree, (g - 1) & 1);
                free = __all_sync(0xffffffffu, free);
                if (!free) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            if (g > 1) {
                bool free = wait_b(c, c.bar + Bars::kDsFree + 8 * (g & 1), ((g >> 1) & 1) ^ 1);
                free = __all_sync(0xffffffffu, free);
                if (!free) {
                    ok = false;
                    break;
                }
            }
            tmem_st16(t_p, pk);
            const uint32_t ds_buf = c.base + kOffDS + (g & 1) * kDsTile;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
                const uint32_t off = sw128_off(r, col0 + q8 * 8);
                st_shared_v4(ds_buf + off, dk[q8 * 4], dk[q8 * 4 + 1], dk[q8 * 4 + 2], dk[q8 * 4 + 3]);
            }
            tmem_wait_st();
            tc_fence_before();
            fence_proxy_async();
            mbar_arrive(c.bar + Bars::kPFull);
            i = inext;
        }
        if (!ok) break;
        // unit epilogue: dV (warps 0-3) or dK times scale (warps 4-7), 32 columns at a time
        bool got = wait_b(c, c.bar + Bars::kDKVFull, units & 1);
        got = __all_sync(0xffffffffu, got);
        if (!got) {
            ok = false;
            break;
        }
        ++units;
        tc_fence_after();
        const float f = half == 0 ? 1.f : p.scale;
        uint4* dst = reinterpret_cast<uint4*>((half == 0 ? p.dv : p.dk) + (static_cast<size_t>(w.bh) * p.N + key) * kD);
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t a[32];
            tmem_ld32(t_acc + c4 * 32, a);
            tmem_wait_ld();
            reg_fence32(a);
            if (c4 == 3) {
                tc_fence_before();
                mbar_arrive(c.bar + Bars::kDKVEmpty);
            }
            if (key < p.N) {
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    uint32_t x[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        x[e] = pack_bf16x2(__uint_as_float(a[v4 * 8 + e * 2]) * f, __uint_as_float(a[v4 * 8 + e * 2 + 1]) * f);
                    dst[c4 * 4 + v4] = make_uint4(x[0], x[1], x[2], x[3]);
                }
            }
        }
    }
}

// Thread = head column t (TMEM lane) of dQ^T; writes column t of the [64 x 128]
// staging tile; one thread adds the tile to dQ with one bulk reduction.
__device__ __forceinline__ void role_dq(const Ctx& c, int warp, int lane) {
    const BwdParams& p = c.p;
    const int quarter = warp & 3;
    const int col = quarter * 32 + lane;
    const uint32_t t_dq = c.tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kColDQ;
    const uint32_t stage = c.base + kOffStage;
    const bool issuer = warp == kDqWarp0 && lane == 0;
    uint32_t g = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const BwdUnit w = unit(u, p);
        for (int i = next_tile(p, w, w.i0, kBQ); i < p.n_qt; i = next_tile(p, w, i + 1, kBQ), ++g) {
            bool got = wait_b(c, c.bar + Bars::kDQFull, g & 1);
            got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
            tc_fence_after();
            got = wait_b(c, c.bar + Bars::kStageFree, (g & 1) ^ 1);  // the previous reduction has read it
            got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t a[32];
                tmem_ld32(t_dq + h * 32, a);
                tmem_wait_ld();
                reg_fence32(a);
                if (h == 1) {
                    tc_fence_before();
                    mbar_arrive(c.bar + Bars::kDQEmpty);
                }
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(stage + (h * 32 + q) * (kD * 4) + col * 4),
                                 "f"(__uint_as_float(a[q]) * p.scale)
                                 : "memory");
            }
            fence_proxy_async();
            mbar_arrive(c.bar + Bars::kStageFull);
            if (issuer) {
                if (wait_b(c, c.bar + Bars::kStageFull, g & 1)) {
                    const int rows = min(kBQ, p.N - i * kBQ);
                    float* dst = p.dq + (static_cast<size_t>(w.bh) * p.N + static_cast<size_t>(i) * kBQ) * kD;
                    asm volatile(
                        "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
                        "r"(stage), "r"(static_cast<uint32_t>(rows * kD * 4))
                        : "memory");
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                    mbar_arrive(c.bar + Bars::kStageFree);
                } else {
                    ok = false;
                }
            }
            ok = __all_sync(0xffffffffu, ok);
        }
    }
    if (issuer) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
}

__global__ void __launch_bounds__(kThreads, 1)
kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
       const __grid_constant__ CUtensorMap /*tm_dq: d = 128 adds whole tiles untiled*/, const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gbase = smem_raw + (base - raw);
    const uint32_t bar = base + kOffBar;
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + kOffBar + Bars::kAbort);
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffBar + Bars::kTmemSlot);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar + Bars::kKVFull, 1);
        mbar_init(bar + Bars::kKVEmpty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar + Bars::kQFull + 8 * s, 1);
            mbar_init(bar + Bars::kQEmpty + 8 * s, 1);
            mbar_init(bar + Bars::kDsFree + 8 * s, 1);
        }
        mbar_init(bar + Bars::kSFull, 1);
        mbar_init(bar + Bars::kSFree, kPdsThreads);
        mbar_init(bar + Bars::kPFull, kPdsThreads);
        mbar_init(bar + Bars::kPTFree, 1);
        mbar_init(bar + Bars::kDQFull, 1);
        mbar_init(bar + Bars::kDQEmpty, 128);
        mbar_init(bar + Bars::kDKVFull, 1);
        mbar_init(bar + Bars::kDKVEmpty, kPdsThreads);
        mbar_init(bar + Bars::kDrain, 1);
        mbar_init(bar + Bars::kDrain2, 1);
        mbar_init(bar + Bars::kStageFull, 128);
        mbar_init(bar + Bars::kStageFree, 1);
        *abort_flag = 0u;
        fence_barrier_init();
        fence_proxy_async();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_do);
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const Ctx ctx{base, bar, *tmem_slot, abort_flag, gbase, p};
    if (warp < kPdsWarps) {
        regs_increase<kPdsRegs>();
        b128::role_pds(ctx, warp, lane);
    } else if (warp < kDqWarp0 + 4) {
        regs_decrease<kOtherRegs>();
        b128::role_dq(ctx, warp, lane);
    } else {
        regs_decrease<kOtherRegs>();
        if (warp == kLoadWarp) {
            if (lane == 0) b128::role_load(ctx, &tm_q, &tm_k, &tm_v, &tm_do);
        } else if (warp == kMmaWarp) {
            b128::role_mma_s(ctx);
        } else if (warp == kMmaWarp + 1) {
            b128::role_mma_d(ctx);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(ctx.tmem, kTmemCols);
    }
}

}  // namespace b128

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

struct BwdDriver {
    EncodeTiledFn encode;
    AddressRangeFn range;
    bool ok;
};

// Driver entry points, looked up once (thread-safe static initialisation).
const BwdDriver& bwd_driver() {
    static const BwdDriver fns = [] {
        BwdDriver f{nullptr, nullptr, false};
        cudaDriverEntryPointQueryResult q1, q2;
        void *f1 = nullptr, *f2 = nullptr;
        f.ok = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
               q1 == cudaDriverEntryPointSuccess &&
               cudaGetDriverEntryPoint("cuMemGetAddressRange", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
               q2 == cudaDriverEntryPointSuccess;
        f.encode = reinterpret_cast<EncodeTiledFn>(f1);
        f.range = reinterpret_cast<AddressRangeFn>(f2);
        return f;
    }();
    return fns;
}

// bf16 [BH, N, d] contiguous as a 4-D (d, N, BH, 1) map, box 64 columns x
// box_rows rows, 128-byte swizzle, rows past N read as zeros.
bool encode_map(EncodeTiledFn enc, CUtensorMap* map, const void* ptr, int BH, int N, int d, int box_rows) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                static_cast<cuuint64_t>(BH), 1};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2,
                                   static_cast<cuuint64_t>(BH) * N * d * 2};
    const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 dQ [BH, N, 64] as a 3-D (64, N, BH) map, box 32 x 32, 128-byte swizzle
// (the tensor reductions of the d = 64 kernel; rows past N are clipped).
bool encode_dq_map(EncodeTiledFn enc, CUtensorMap* map, void* ptr, int BH, int N) {
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {64 * 4, static_cast<cuuint64_t>(N) * 64 * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool span_ok(AddressRangeFn range, const void* ptr, size_t bytes, int device) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if ((a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) || a.device != device) return false;
    CUdeviceptr lo = 0;
    size_t size = 0;
    if (range(&lo, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(ptr);
    return x >= lo && bytes <= size && x - lo <= size - bytes;
}

bool disjoint(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x >= y + nb || y >= x + na;
}

}  // namespace

// Status word of this translation unit (read and cleared by attn_check_device_status).
int attn_bwd_take_device_status(int* status) {
    const int zero = 0;
    if (cudaMemcpyFromSymbol(status, g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}

namespace {

// attn_bwd_noalloc's delta rows live here: file-scope static device memory,
// part of the module image, so that entry point allocates nothing.
constexpr long long kNoAllocDeltaRows = 1LL << 20;  // B*H*N at most (4 MiB of fp32)
__device__ __align__(256) float g_noalloc_delta[kNoAllocDeltaRows];
constexpr int kMaxDevices = 64;

// Device address of g_noalloc_delta in the current context.  It is looked up
// with cudaGetSymbolAddress on the first call in each context of a device
// and cached under that context's id, so a device reset or a new context
// (which loads the module afresh, maybe at another address) resolves it
// again instead of reusing a stale address.  nullptr on failure.
float* noalloc_delta() {
    static std::mutex m;
    static unsigned long long ctx_of[kMaxDevices] = {};  // 0 = nothing cached
    static float* addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(m);
    unsigned long long id = current_context_id();
    if (id == 0 || id != ctx_of[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_delta) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        // the runtime has a context current now (the lookup creates the
        // primary context if needed): cache the address under its id
        id = current_context_id();
        if (id == 0) return nullptr;
        ctx_of[dev] = id;
        addr[dev] = static_cast<float*>(ptr);
    }
    return addr[dev];
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
             const unsigned char* key_pad, const unsigned char* block_mask, float* delta, float* dq, void* dk,
             void* dv, int B, int H, int N, int d, float scale, int causal, attn_stream_t stream);

}  // namespace

extern "C" int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, const unsigned char* key_padding_mask, const unsigned char* block_mask,
                        float* delta, float* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                        int causal, attn_stream_t stream) {
    return bwd_impl(q, k, v, o, dout, lse, key_padding_mask, block_mask, delta, dq, dk, dv, B, H, N, d, scale, causal,
                    stream);
}

extern "C" int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                const float* lse, const unsigned char* key_padding_mask,
                                const unsigned char* block_mask, float* dq, void* dk, void* dv, int B, int H, int N,
                                int d, float scale, int causal, attn_stream_t stream) {
    if (B < 1 || H < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
    if (static_cast<long long>(B) * H * N > kNoAllocDeltaRows) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    float* delta = noalloc_delta();
    if (delta == nullptr) return ATTN_ERR_CUDA;
    return bwd_impl(q, k, v, o, dout, lse, key_padding_mask, block_mask, delta, dq, dk, dv, B, H, N, d, scale,
                    causal, stream);
}

namespace {

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
             const unsigned char* key_pad, const unsigned char* block_mask, float* delta, float* dq, void* dk,
             void* dv, int B, int H, int N, int d, float scale, int causal, attn_stream_t stream) {
    if (B < 1 || H < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !o || !dout || !lse || !delta || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
    if (!isfinite(scale) || !(scale >= 1e-30f)) return ATTN_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(B) * H;
    if (BH > 0x7fffffffLL || N > 0x7fffffff - 128 || BH * N > (1LL << 40) / d) return ATTN_ERR_INVALID_ARG;
    auto mis = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0; };
    if (mis(q, 16) || mis(k, 16) || mis(v, 16) || mis(o, 16) || mis(dout, 16) || mis(dk, 16) || mis(dv, 16) ||
        mis(dq, 16) || mis(lse, 4) || mis(delta, 4))
        return ATTN_ERR_INVALID_ARG;
    const size_t rows = static_cast<size_t>(BH) * N;
    const size_t tb = rows * d * 2, qb = rows * d * 4, lb = rows * 4;
    // outputs must not overlap any input or each other
    const void* ins[6] = {q, k, v, o, dout, lse};
    const size_t in_b[6] = {tb, tb, tb, tb, tb, lb};
    const void* outs[4] = {delta, dq, dk, dv};
    const size_t out_b[4] = {lb, qb, tb, tb};
    const size_t pad_b = static_cast<size_t>(B) * N;
    const int n_bt = (N + 127) / 128;
    const size_t bm_b = static_cast<size_t>(n_bt) * n_bt;
    for (int a = 0; a < 4; ++a) {
        for (int b = 0; b < 6; ++b)
            if (!disjoint(outs[a], out_b[a], ins[b], in_b[b])) return ATTN_ERR_INVALID_ARG;
        for (int b = a + 1; b < 4; ++b)
            if (!disjoint(outs[a], out_b[a], outs[b], out_b[b])) return ATTN_ERR_INVALID_ARG;
        if (key_pad && !disjoint(outs[a], out_b[a], key_pad, pad_b)) return ATTN_ERR_INVALID_ARG;
        if (block_mask && !disjoint(outs[a], out_b[a], block_mask, bm_b)) return ATTN_ERR_INVALID_ARG;
    }
    const BwdDriver& drv = bwd_driver();
    if (!drv.ok) return ATTN_ERR_CUDA;
    const EncodeTiledFn enc = drv.encode;
    const AddressRangeFn range = drv.range;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    for (int a = 0; a < 6; ++a)
        if (!span_ok(range, ins[a], in_b[a], dev)) return ATTN_ERR_INVALID_ARG;
    for (int a = 0; a < 4; ++a)
        if (!span_ok(range, outs[a], out_b[a], dev)) return ATTN_ERR_INVALID_ARG;
    if (key_pad && !span_ok(range, key_pad, pad_b, dev)) return ATTN_ERR_INVALID_ARG;
    if (block_mask && !span_ok(range, block_mask, bm_b, dev)) return ATTN_ERR_INVALID_ARG;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return ATTN_ERR_CUDA;
    alignas(64) CUtensorMap mq, mk, mv, mdo, mdq;
    const int bh = static_cast<int>(BH);
    const int q_rows = d == 64 ? kBQ : b128::kBQ;  // query rows per tile (the Q / dO box)
    if (!encode_map(enc, &mq, q, bh, N, d, q_rows) || !encode_map(enc, &mk, k, bh, N, d, kBK) ||
        !encode_map(enc, &mv, v, bh, N, d, kBK) || !encode_map(enc, &mdo, dout, bh, N, d, q_rows))
        return ATTN_ERR_CUDA;
    if (d == 64) {
        if (!encode_dq_map(enc, &mdq, dq, bh, N)) return ATTN_ERR_CUDA;
    } else {
        mdq = mq;  // unused at d = 128
    }

    BwdParams p;
    p.BH = bh;
    p.H = H;
    p.N = N;
    p.key_pad = key_pad;
    p.block_mask = block_mask;
    p.n_bt = n_bt;
    p.n_kb = (N + kBK - 1) / kBK;
    p.n_qt = (N + q_rows - 1) / q_rows;
    const long long units = BH * p.n_kb;
    if (units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    p.total_units = static_cast<int>(units);
    p.causal = causal ? 1 : 0;
    p.scale = scale;
    p.scale_log2 = scale * kLog2eB;
    p.neg_inv_scale = static_cast<float>(-1.0 / static_cast<double>(scale));
    p.lse = lse;
    p.delta = delta;
    p.dq = dq;
    p.dk = static_cast<uint16_t*>(dk);
    p.dv = static_cast<uint16_t*>(dv);
    p.wait_ns = kWaitNs;

    // every fallible host step comes before the first launch: an error return
    // means nothing was queued (dq, delta untouched)
    auto kern = d == 64 ? attn_bwd_kernel : b128::kernel;
    const int smem = d == 64 ? kSmemBytes : b128::kSmemBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return ATTN_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long prep_blocks = (static_cast<long long>(rows) + 255) / 256;
    const int prep_grid = static_cast<int>(prep_blocks < 4 * sms ? prep_blocks : 4 * sms);
    const uint16_t* o16 = static_cast<const uint16_t*>(o);
    const uint16_t* do16 = static_cast<const uint16_t*>(dout);
    if (d == 64)
        attn_bwd_prep_kernel<64><<<prep_grid, 256, 0, s>>>(o16, do16, delta, dq, static_cast<long long>(rows));
    else
        attn_bwd_prep_kernel<128><<<prep_grid, 256, 0, s>>>(o16, do16, delta, dq, static_cast<long long>(rows));
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    const int grid = static_cast<int>(units < sms ? units : sms);
    kern<<<grid, d == 64 ? kThreads : b128::kThreads, smem, s>>>(mq, mk, mv, mdo, mdq, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace
