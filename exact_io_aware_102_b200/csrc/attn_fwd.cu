// Exact, IO-aware multi-head attention forward for B200 (sm_100a).
//
// What is computed (FlashAttention: Fast and Memory-Efficient Exact Attention
// with IO-Awareness, wiki notes): O = softmax(scale * Q K^T) V per (batch,
// head), "Problem setting"; Q, K and V are processed in on-chip tiles with a
// running row maximum m and running row sum l that are updated from tile to
// tile, so the N x N matrices never reach HBM, "Tiling"; scores, scaling,
// masking, softmax and both matrix products run in ONE kernel, "Kernel
// fusion"; only O and the per-row softmax statistics (here as one log-sum-exp)
// are written, "Recomputation"; with a causal mask or a block mask only the
// non-zero (query block, key block) pairs are loaded and multiplied,
// "Block-sparse FlashAttention"; padded keys (the key-padding mask of the
// pages' patch self-attention module) are masked per element.
//
// How it maps to sm_100a (the page's A100 design is prior art, not followed):
//   * persistent grid, one CTA per SM, each CTA walks work units
//     (b, h, 256 query rows = two 128-row Q tiles), 12 warps;
//   * warp 8 (one lane) issues TMA loads: the two Q tiles once per unit and
//     K / V tiles of 128 keys into shared-memory rings guarded by full/empty
//     mbarriers;
//   * tcgen05.mma computes S_t = Q_t K_j^T into TMEM (fp32, 128 x 128) and
//     O_t += P_t V_j with P_t read from TMEM.  At d = 64, P_t has TMEM columns
//     of its own, so the S stream (warp 9) and the P V stream (warp 10) are
//     issued by two threads and neither waits behind the other; at d = 128,
//     P_t overlays S_t and warp 9 issues both in one ordered stream;
//   * warps 0-3 and 4-7 are the softmax warpgroups of Q tiles 0 and 1: one
//     thread per query row reads its S row from TMEM, masks, updates m and l,
//     writes P (bf16), rescales its O row in TMEM when m moves, and at the
//     end normalises O by l and stores O and LSE;
//   * every mbarrier wait is bounded; on timeout a status word is set, the
//     CTA drains its in-flight copies and MMAs, frees TMEM and returns.
//
// Memory layout: Q, K, V, O bf16 [B, H, N, d] with element strides over
// (b, h, n) and a contiguous head dimension ([B, N, H, d] and packed
// projections included), LSE fp32 [B, H, N] contiguous.
// Shared memory tiles use the 128-byte swizzle (TMA writes them, the tensor
// cores read them through matrix descriptors); d = 128 tiles are stored as two
// 64-column halves.  TMEM: S0 cols [0,128), S1 [128,256), O0 [256,256+d),
// O1 [256+d, 256+2d); P0, P1 at [384,448), [448,512) for d = 64, over the
// first 64 columns of S0, S1 for d = 128.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "attn.h"
#include "sm100_ptx.cuh"

namespace {

constexpr int kBlockM = 128;           // query rows per Q tile (= TMEM lanes)
constexpr int kBlockN = 128;           // keys per K / V tile
constexpr int kUnitRows = 2 * kBlockM;  // query rows per work unit
constexpr int kThreads = 384;          // softmax WG 0, softmax WG 1, WG 2 = {load, MMA S, MMA PV, idle}
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;            // S stream (and, at d = 128, the P V stream too)
constexpr int kMmaPvWarp = 10;         // P V stream at d = 64
// Register split (setmaxnreg): the block launches with 384 x 168 registers;
// the two softmax warpgroups take 192 each, warpgroup 2 keeps 120
// (256 x 192 + 128 x 120 = 384 x 168).
constexpr int kSoftmaxRegs = 192;
constexpr int kOtherRegs = 120;
// The reference maximum of a row moves only when the row maximum exceeds it
// by more than this many powers of two; O and l always share the reference.
constexpr float kLazyRescaleLog2 = 8.0f;
// Of every 8 exponential pairs, this many run on the FMA-pipe polynomial and
// the rest on MUFU (ex2.approx).
#ifndef ATTN_POLY_PAIRS_PER_8
#define ATTN_POLY_PAIRS_PER_8 3
#endif
constexpr int kPolyPairsPer8 = ATTN_POLY_PAIRS_PER_8;
// Which pairs of each group of 8 take the polynomial (best measured patterns).
constexpr uint32_t kPolyMask8 = kPolyPairsPer8 <= 0 ? 0x00u
                              : kPolyPairsPer8 == 1 ? 0x80u
                              : kPolyPairsPer8 == 2 ? 0xC0u
                              : kPolyPairsPer8 == 3 ? 0x70u
                              : kPolyPairsPer8 == 4 ? 0xAAu
                              : 0xFFu;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s per wait
constexpr unsigned long long kDrainWaitNs = 100000000ull;     // 0.1 s per drain wait

template <int D>
struct Cfg {
    static constexpr int kHalfBytes = kBlockN * 64 * 2;       // one 128 x 64 bf16 swizzled half
    static constexpr int kTileBytes = kBlockN * D * 2;        // one Q, K or V tile
    // d = 64: P_t has its own 64 TMEM columns after O, so S_t can be refilled
    // as soon as the softmax has loaded it, and the S and P V streams are
    // independent (two issuing threads, a K ring and a V ring).  d = 128: no
    // TMEM room; P_t overlays S_t and one thread issues P_t V before S_t.
    static constexpr bool kSplit = (D == 64);
    static constexpr int kKSlots = kSplit ? 4 : 4;            // split: K ring; else the shared K/V ring
    static constexpr int kVSlots = kSplit ? 4 : 0;            // split: V ring
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = 2 * kTileBytes;
    static constexpr int kVRingOff = kRingOff + kKSlots * kTileBytes;
    static constexpr int kBarOff = kVRingOff + kVSlots * kTileBytes;
    static constexpr int kMaskOff = kBarOff + 512;             // sparse mode: block mask bits
    static constexpr int kSmemBytes = kBarOff + 512 + 1024;   // barriers + 1 KB alignment slack
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
    static constexpr uint32_t kColP0 = kSplit ? 256 + 2 * D : kColS0;
    static constexpr uint32_t kColP1 = kSplit ? 256 + 2 * D + 64 : kColS1;
    static_assert(256 + 2 * D + (kSplit ? 128 : 0) <= (int)kTmemCols, "TMEM budget");
    static_assert(kKSlots <= 8 && kVSlots <= 8, "barrier block holds 8 + 8 ring slots");
};

// Barrier block (offsets in bytes from the barrier area).  No barrier can
// complete twice before its consumer has waited on it.
struct Bars {
    static constexpr int kQFull = 0;       // [2] TMA -> MMA: Q tile t landed
    static constexpr int kQEmpty = 16;     // [1] MMA -> TMA: the unit's last S MMA retired
    static constexpr int kSFull = 24;      // [2] MMA -> softmax t: S_t computed
    static constexpr int kPFull = 40;      // [2] softmax t -> MMA: P_t written (and O_t rescaled)
    static constexpr int kOFull = 56;      // [2] MMA -> softmax t: O_t of the unit complete
    static constexpr int kOEmpty = 72;     // [2] softmax t -> MMA: O_t read out
    static constexpr int kDrain = 88;      // [2] one per MMA-issuing thread
    static constexpr int kSFree = 104;     // [2] softmax t -> MMA: S_t loaded (split layout)
    static constexpr int kPFree = 120;     // [2] MMA -> softmax t: P_t V retired (split layout)
    static constexpr int kTmemSlot = 136;  // u32: TMEM base address
    static constexpr int kAbort = 140;     // u32: abort flag
    static constexpr int kKFull = 144;     // [8] TMA -> MMA: K (or K/V) ring slot landed
    static constexpr int kKEmpty = 208;    // [8] MMA -> TMA: K (or K/V) ring slot free
    static constexpr int kVFull = 272;     // [8] V ring (split layout)
    static constexpr int kVEmpty = 336;    // [8]
    static constexpr int kPadRows = 400;   // int: staged key-padding rows
};

// ------------------------------------------------------------- the scheduler
// Which key tiles a work unit visits.  Full: all of them.  Causal: a Q tile
// stops at the key tile holding its last row (tiles above the diagonal are
// never loaded or multiplied).  Sparse: the non-zero entries of the block mask
// row of each Q tile (with the causal bound as well when causal is set).
enum : int { kModeFull = 0, kModeCausal = 1, kModeSparse = 2 };

struct Params {
    int BH, H, N, n_pairs, n_kv_all, total_units;
    long long o_sb, o_sh, o_sn;  // element strides of O over (batch, head, row)
    const uint8_t* key_pad;      // [B, N] key-padding mask (nonzero = padded) or null
    int pad_vec;                 // key_pad rows may be read 16 bytes at a time
    // key padding staged in shared memory as one bit per key (set = padded,
    // keys >= N included), one row per batch that the CTA's units touch:
    int pad_staged;              // 0: not staged (no tile is skipped; masks read from global memory)
    int pad_row_words;           // 32-bit words per row (4 per key tile)
    int pad_units;               // units per CTA at most (entries of the unit -> row map)
    int pad_map_off, pad_rowb_off, pad_rows_off;  // byte offsets of the map, row batches and rows
    const uint8_t* block_mask;   // [n_kv_all, n_kv_all] block mask (nonzero = computed), sparse mode
    int causal;                  // causal bound on top of the block mask (sparse mode)
    float scale_log2;  // scale * log2(e)
    unsigned long long wait_ns;
};

struct Unit {
    int bh, b, h, q0;  // head (flat, batch, within batch), first query row
    int local;         // index of the unit among this CTA's units
};

// Work units: (head, pair of Q tiles).  Non-causal: heads-major so the CTAs
// running at one time share K/V of few heads (L2 reuse).  Causal: the pairs
// with the most key tiles first.  CTA c takes units c, c + grid, c + 2 grid,
// ...; with units of unequal cost a plain round-robin over a longest-first
// list gives CTA 0 the longest unit of every round, so odd rounds run the
// list backwards ("snake" order): each CTA's total comes out close to the
// mean.
template <int MODE>
__device__ __forceinline__ Unit decode_unit(int u, const Params& p) {
    Unit w;
    int pair;
    const bool longest_first = MODE == kModeCausal || (MODE == kModeSparse && p.causal);
    if (longest_first) {
        // the last round may be partial: reverse it within its own length
        const int g = static_cast<int>(gridDim.x);
        const int k = u / g, c = u - k * g;
        const int rem = min(g, p.total_units - k * g);
        const int pos = (k & 1) ? k * g + (rem - 1 - c) : u;
        pair = p.n_pairs - 1 - pos / p.BH;
        w.bh = pos % p.BH;
    } else {
        pair = u % p.n_pairs;
        w.bh = u / p.n_pairs;
    }
    w.b = w.bh / p.H;
    w.h = w.bh - w.b * p.H;
    w.q0 = pair * kUnitRows;
    w.local = (u - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x);
    return w;
}

constexpr int kNoTile = 0x7fffffff;

// Bit i set iff byte i of x is nonzero (4 bits).
__device__ __forceinline__ uint32_t nonzero_bytes4(uint32_t x) {
    const uint32_t y = __vcmpne4(x, 0u);  // 0xFF per nonzero byte
    return ((y >> 7) & 1u) | ((y >> 14) & 2u) | ((y >> 21) & 4u) | ((y >> 28) & 8u);
}

// A staged key-padding row (shared memory, one per batch that the CTA's units
// touch): 4 words per key tile with one bit per key (set = padded, keys >= N
// included), then two bitmaps with one bit per key tile: "holds an unpadded
// key" (the tile is visited) and "holds a padded key" (the tile needs the
// per-key mask).
struct PadRow {
    static __device__ __forceinline__ uint32_t occ(uint32_t row, int n_tiles) { return row + 16u * n_tiles; }
    static __device__ __forceinline__ uint32_t mix(uint32_t row, int n_tiles) {
        return row + 16u * n_tiles + 4u * ((n_tiles + 31) / 32);
    }
    // last key tile that holds an unpadded key (-1: none), one int
    static __device__ __forceinline__ uint32_t last(uint32_t row, int n_tiles) {
        return row + 16u * n_tiles + 8u * ((n_tiles + 31) / 32);
    }
    static __host__ __device__ constexpr int words(int n_tiles) {
        return (4 * n_tiles + 2 * ((n_tiles + 31) / 32) + 1 + 3) / 4 * 4;  // 16-byte multiple
    }
};

// The 128 padding bits of key tile j in a staged row; row: shared-window address.
__device__ __forceinline__ uint4 pad_tile_bits(uint32_t row, int j) { return lds_u32x4(row + 16 * j); }

// The key tiles one Q tile visits, in increasing order.  In the sparse mode
// (a block mask, a key-padding mask, or both) a tile is visited when its
// block-mask bit is set (no block mask: every tile up to the causal bound)
// and, with key padding, it holds a key that is not padded: tiles made only
// of padded keys are neither loaded nor multiplied.  Every role evaluates the
// same predicate for the same unit, so they all walk the same tiles.
//
// The predicate of 32 consecutive tiles is read from shared memory into one
// word (block-mask bits, "holds an unpadded key" bits and the causal bound
// combined) and kept: tiles are walked in order, so the common step costs no
// shared-memory load (those queue behind the tensor core's operand reads and
// take hundreds of cycles).
template <int MODE>
struct KeyTiles {
    int lim;               // last key tile it may visit (-1: the tile has no rows)
    int off;               // sparse: bit index of its block-mask row, column 0
    uint32_t bits;         // sparse: shared-window address of the block mask bits, row-major (0: none)
    uint32_t pad;          // sparse: shared-window address of this unit's staged padding row (0: none)
    int n_tiles;           // sparse: key tiles per row (block-mask rows and padding bitmaps)
    mutable int wi;        // sparse: window index held in ww (tiles 32 wi .. 32 wi + 31), -1: none
    mutable uint32_t ww;   // sparse: visited tiles of that window

    __device__ __forceinline__ uint32_t load_window(int i) const {
        const int j0 = 32 * i;
        if (j0 > lim) return 0u;
        uint32_t v = ~0u;
        if (bits != 0u) {
            const int f = off + j0;  // first bit; the row ends at off + n_tiles - 1
            const int total_words = (n_tiles * n_tiles + 31) / 32;
            const uint32_t lo = lds_u32(bits + 4u * (f >> 5));
            const uint32_t hi = ((f & 31) != 0 && (f >> 5) + 1 < total_words) ? lds_u32(bits + 4u * ((f >> 5) + 1)) : 0u;
            v = __funnelshift_r(lo, hi, f & 31);
        }
        if (pad != 0u) v &= lds_u32(PadRow::occ(pad, n_tiles) + 4u * i);
        const int last = lim - j0;  // >= 0 here
        if (last < 31) v &= ~0u >> (31 - last);
        return v;
    }
    __device__ __forceinline__ uint32_t window(int i) const {
        if (i != wi) {
            ww = load_window(i);
            wi = i;
        }
        return ww;
    }
    __device__ __forceinline__ bool has(int j) const {
        if constexpr (MODE != kModeSparse) return j <= lim;
        else return j >= 0 && j <= lim && ((window(j >> 5) >> (j & 31)) & 1u);
    }
    // first key tile >= j (kNoTile if none)
    __device__ __forceinline__ int next(int j) const {
        if constexpr (MODE != kModeSparse) {
            return j <= lim ? j : kNoTile;
        } else {
            while (j <= lim) {
                const uint32_t w = window(j >> 5) >> (j & 31);
                if (w != 0u) return j + __ffs(static_cast<int>(w)) - 1;
                j = (j | 31) + 1;
            }
            return kNoTile;
        }
    }
    // number of key tiles
    __device__ __forceinline__ int count() const {
        if constexpr (MODE != kModeSparse) {
            return lim + 1;
        } else {
            int n = 0;
            for (int i = 0; 32 * i <= lim; ++i) n += __popc(window(i));
            return n;
        }
    }
    // last key tile (-1 if none)
    __device__ __forceinline__ int last() const {
        if constexpr (MODE != kModeSparse) {
            return lim;
        } else {
            for (int i = lim >> 5; i >= 0 && lim >= 0; --i) {
                const uint32_t w = window(i);
                if (w != 0u) return 32 * i + 31 - __clz(static_cast<int>(w));
            }
            return -1;
        }
    }
};

// Per-CTA shared-memory copies of the masks (sparse mode).
struct Masks {
    uint32_t bits;             // shared-window address of the block mask bits (0: none)
    uint32_t pad_map;          // shared-window address of the map local unit -> staged row (u32 each)
    uint32_t pad_rows;         // shared-window address of the staged padding rows (0: none)
};

// Shared-window address of the staged padding row of a unit (0: none).
__device__ __forceinline__ uint32_t pad_row_of(const Unit& w, const Params& p, const Masks& mk) {
    return mk.pad_rows != 0u
               ? mk.pad_rows + 4u * lds_u32(mk.pad_map + 4u * w.local) * static_cast<uint32_t>(p.pad_row_words)
               : 0u;
}

template <int MODE>
__device__ __forceinline__ KeyTiles<MODE> key_tiles_row(const Unit& w, const Params& p, const Masks& mk, int t,
                                                        uint32_t pad_row, int wi = -1, uint32_t ww = 0u) {
    const bool causal = MODE == kModeCausal || (MODE == kModeSparse && p.causal);
    const int qt = w.q0 / kBlockM + t;
    KeyTiles<MODE> k;
    // full and causal modes also walk Q tile 1 of the last unit when it has no
    // rows (nothing of it is stored); the sparse mode skips it
    k.lim = (MODE == kModeSparse && w.q0 + t * kBlockM >= p.N) ? -1
            : causal ? min(p.n_kv_all - 1, qt) : p.n_kv_all - 1;
    if (MODE != kModeSparse && pad_row != 0u) {
        // key padding in the dense loops: the tiles after the batch's last
        // tile holding an unpadded key are never visited (a batch without any
        // visits tile 0, fully masked, so that every Q tile has a tile)
        const int last = static_cast<int>(lds_u32(PadRow::last(pad_row, p.n_kv_all)));
        k.lim = min(k.lim, max(last, 0));
    }
    k.off = qt * p.n_kv_all;
    k.bits = mk.bits;
    k.pad = pad_row;
    k.n_tiles = p.n_kv_all;
    k.wi = wi;
    k.ww = ww;
    return k;
}

template <int MODE>
__device__ __forceinline__ KeyTiles<MODE> key_tiles(const Unit& w, const Params& p, const Masks& mk, int t) {
    return key_tiles_row<MODE>(w, p, mk, t, pad_row_of(w, p, mk));
}

// The key tiles of one unit, as the load and MMA roles walk them: the union
// over the two Q tiles in increasing order; Q tile t takes part in tile j iff
// q[t].has(j).  Every role derives the same tiles from the same unit, so
// their barrier counts agree.
template <int MODE>
struct Plan {
    KeyTiles<MODE> q[2];
    __device__ __forceinline__ bool need(int t, int j) const { return q[t].has(j); }
    __device__ __forceinline__ int next(int j) const {
        if constexpr (MODE != kModeSparse) return j <= max(q[0].lim, q[1].lim) ? j : kNoTile;
        else return min(q[0].next(j), q[1].next(j));
    }
};

template <int MODE>
__device__ __forceinline__ Plan<MODE> make_plan(const Unit& w, const Params& p, const Masks& mk) {
    Plan<MODE> pl;
    pl.q[0] = key_tiles<MODE>(w, p, mk, 0);
    pl.q[1] = key_tiles<MODE>(w, p, mk, 1);
    return pl;
}

// What every role of one CTA shares.
struct Ctx {
    uint32_t base;   // shared-memory base (1 KB aligned)
    uint32_t bar;    // barrier block
    uint32_t tmem;   // TMEM base address
    volatile uint32_t* abort_flag;
    Masks masks;                // sparse mode: shared-memory copies of the masks
    Params p;
};

// A ring of shared-memory tiles with full/empty barriers, walked in order.
struct Ring {
    uint32_t smem, full, empty, slots, i;
    __device__ __forceinline__ uint32_t slot() const { return i % slots; }
    __device__ __forceinline__ uint32_t phase() const { return (i / slots) & 1u; }
};

// ------------------------------------------------------------ TMA producer
// Per unit with at least one key tile: Q0, Q1 once; then the key tiles in
// the order the MMA warps use them (split: K_j into the K ring and V_j into
// the V ring; shared ring: K_j then V_j).
template <int D, int MODE>
__device__ __forceinline__ void role_producer(const Ctx& c, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                              const CUtensorMap* tm_v) {
    if constexpr (MODE != kModeSparse) {
        // full / causal: key tiles [0, n1) of every unit
        using C = Cfg<D>;
        Ring rk{c.base + C::kRingOff, c.bar + Bars::kKFull, c.bar + Bars::kKEmpty, (uint32_t)C::kKSlots, 0};
        Ring rv{c.base + C::kVRingOff, c.bar + Bars::kVFull, c.bar + Bars::kVEmpty, (uint32_t)C::kVSlots, 0};
        uint32_t q_issued = 0;
        bool ok = true;
        auto load = [&](Ring& r, const CUtensorMap* map, int key0, const Unit& w) {
            const uint32_t s = r.slot();
            if (!wait_bounded(r.empty + 8 * s, r.phase() ^ 1u, c.abort_flag, c.p.wait_ns)) return false;
            const uint32_t fb = r.full + 8 * s;
            const uint32_t dst = r.smem + s * C::kTileBytes;
            mbar_expect_tx(fb, C::kTileBytes);
#pragma unroll
            for (int x = 0; x < D / 64; ++x) tma_load_4d(dst + x * C::kHalfBytes, map, fb, x * 64, key0, w.h, w.b);
            ++r.i;
            return true;
        };
        int local = 0;
        for (int u = blockIdx.x; ok && u < c.p.total_units; u += gridDim.x, ++local) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const int n1 = make_plan<MODE>(w, c.p, c.masks).q[1].lim + 1;
            if (!wait_bounded(c.bar + Bars::kQEmpty, (local & 1) ^ 1, c.abort_flag, c.p.wait_ns)) {
                ok = false;
                break;
            }
            for (int t = 0; t < 2; ++t) {
                const uint32_t qb = c.bar + Bars::kQFull + 8 * t;
                const uint32_t dst = c.base + C::kQOff + t * C::kTileBytes;
                mbar_expect_tx(qb, C::kTileBytes);
#pragma unroll
                for (int x = 0; x < D / 64; ++x)
                    tma_load_4d(dst + x * C::kHalfBytes, tm_q, qb, x * 64, w.q0 + t * kBlockM, w.h, w.b);
            }
            q_issued = local + 1;
            for (int j = 0; ok && j < n1; ++j) {
                ok = load(rk, tm_k, j * kBlockN, w);
                if (ok) ok = load(C::kSplit ? rv : rk, tm_v, j * kBlockN, w);
            }
        }
        if (!ok) {
            // Drain: every issued copy lands before the CTA may exit.
            for (Ring* r : {&rk, &rv})
                for (uint32_t i = (r->i > r->slots ? r->i - r->slots : 0); i < r->i; ++i)
                    wait_bounded(r->full + 8 * (i % r->slots), (i / r->slots) & 1, nullptr, kDrainWaitNs);
            if (q_issued > 0)
                for (int t = 0; t < 2; ++t)
                    wait_bounded(c.bar + Bars::kQFull + 8 * t, (q_issued - 1) & 1, nullptr, kDrainWaitNs);
        }
    } else {
        // sparse: the union of both Q tiles' key tiles; units without any are skipped
        using C = Cfg<D>;
        Ring rk{c.base + C::kRingOff, c.bar + Bars::kKFull, c.bar + Bars::kKEmpty, (uint32_t)C::kKSlots, 0};
        Ring rv{c.base + C::kVRingOff, c.bar + Bars::kVFull, c.bar + Bars::kVEmpty, (uint32_t)C::kVSlots, 0};
        uint32_t q_issued = 0;  // units whose Q tiles were loaded
        bool ok = true;
        auto load = [&](Ring& r, const CUtensorMap* map, int key0, const Unit& w) {
            const uint32_t s = r.slot();
            if (!wait_bounded(r.empty + 8 * s, r.phase() ^ 1u, c.abort_flag, c.p.wait_ns)) return false;
            const uint32_t fb = r.full + 8 * s;
            const uint32_t dst = r.smem + s * C::kTileBytes;
            mbar_expect_tx(fb, C::kTileBytes);
#pragma unroll
            for (int x = 0; x < D / 64; ++x) tma_load_4d(dst + x * C::kHalfBytes, map, fb, x * 64, key0, w.h, w.b);
            ++r.i;
            return true;
        };
        for (int u = blockIdx.x; ok && u < c.p.total_units; u += gridDim.x) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const Plan<MODE> pl = make_plan<MODE>(w, c.p, c.masks);
            int j = pl.next(0);
            if (j == kNoTile) continue;
            if (!wait_bounded(c.bar + Bars::kQEmpty, (q_issued & 1) ^ 1, c.abort_flag, c.p.wait_ns)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const uint32_t qb = c.bar + Bars::kQFull + 8 * t;
                const uint32_t dst = c.base + C::kQOff + t * C::kTileBytes;
                mbar_expect_tx(qb, C::kTileBytes);
#pragma unroll
                for (int x = 0; x < D / 64; ++x)
                    tma_load_4d(dst + x * C::kHalfBytes, tm_q, qb, x * 64, w.q0 + t * kBlockM, w.h, w.b);
            }
            ++q_issued;
            for (; ok && j != kNoTile; j = pl.next(j + 1)) {
                ok = load(rk, tm_k, j * kBlockN, w);
                if (ok) ok = load(C::kSplit ? rv : rk, tm_v, j * kBlockN, w);
            }
        }
        if (!ok) {
            // Drain: every issued copy lands before the CTA may exit.
            for (Ring* r : {&rk, &rv})
                for (uint32_t i = (r->i > r->slots ? r->i - r->slots : 0); i < r->i; ++i)
                    wait_bounded(r->full + 8 * (i % r->slots), (i / r->slots) & 1, nullptr, kDrainWaitNs);
            if (q_issued > 0)
                for (int t = 0; t < 2; ++t)
                    wait_bounded(c.bar + Bars::kQFull + 8 * t, (q_issued - 1) & 1, nullptr, kDrainWaitNs);
        }
    }
}

// ---------------------------------------------------------- MMA issuing
template <int D>
struct Mma {
    static constexpr uint32_t kIdescS = idesc_bf16_f32(kBlockM, kBlockN, false);
    static constexpr uint32_t kIdescO = idesc_bf16_f32(kBlockM, D, true);
    static constexpr uint32_t kHi = sdesc_hi_sw128(1024);
    using C = Cfg<D>;
    // S_t = Q_t K^T: K-major A (Q tile) and B (K tile), 16 columns of d per instruction
    __device__ __forceinline__ static void qk(const Ctx& c, int t, uint32_t k_smem) {
        const uint32_t a0 = sdesc_lo(c.base + C::kQOff + t * C::kTileBytes, 16);
        const uint32_t b0 = sdesc_lo(k_smem, 16);
        const uint32_t d = c.tmem + (t == 0 ? C::kColS0 : C::kColS1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk / 4) * C::kHalfBytes + (kk % 4) * 32) >> 4;
            mma_ss_lo(d, a0 + off, b0 + off, kHi, kIdescS, kk > 0 ? 1u : 0u);
        }
    }
    // O_t (+)= P_t V: P from TMEM, V tile MN-major (LBO = one 64-column half), 16 keys per instruction
    __device__ __forceinline__ static void pv(const Ctx& c, int t, uint32_t v_smem, bool accumulate) {
        const uint32_t b0 = sdesc_lo(v_smem, C::kHalfBytes);
        const uint32_t d = c.tmem + (t == 0 ? C::kColO0 : C::kColO1);
        const uint32_t a = c.tmem + (t == 0 ? C::kColP0 : C::kColP1);
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
            mma_ts_lo(d, a + kk * 8, b0 + ((kk * 16 * 128) >> 4), kHi, kIdescO, (accumulate || kk > 0) ? 1u : 0u);
    }
};

// Bounded wait for the MMA-issuing threads: false once anything gave up.
struct Waiter {
    const Ctx& c;
    bool ok;
    __device__ __forceinline__ bool operator()(uint32_t b, uint32_t parity) {
        if (ok && !wait_bounded(b, parity, c.abort_flag, c.p.wait_ns)) ok = false;
        return ok;
    }
    __device__ __forceinline__ bool take(Ring& r, uint32_t& slot) {
        slot = r.slot();
        const bool got = (*this)(r.full + 8 * slot, r.phase());
        ++r.i;
        return got;
    }
};

__device__ __forceinline__ void mma_drain(const Ctx& c, int which) {
    tc_commit(c.bar + Bars::kDrain + 8 * which);
    wait_bounded(c.bar + Bars::kDrain + 8 * which, 0, nullptr, kDrainWaitNs);
}

// Split layout, S stream: S_t(j) once the softmax has loaded S_t's previous tile.
template <int D, int MODE>
__device__ __forceinline__ void role_mma_s(const Ctx& c) {
    if constexpr (MODE != kModeSparse) {
        // full / causal: Q tile 0 visits key tiles [0, n0), Q tile 1 [0, n1), n0 <= n1
        using C = Cfg<D>;
        Ring rk{c.base + C::kRingOff, c.bar + Bars::kKFull, c.bar + Bars::kKEmpty, (uint32_t)C::kKSlots, 0};
        Waiter wait{c, true};
        uint32_t s_issued[2] = {0u, 0u};
        int local = 0;
        for (int u = blockIdx.x; wait.ok && u < c.p.total_units; u += gridDim.x, ++local) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const Plan<MODE> pl = make_plan<MODE>(w, c.p, c.masks);
            const int n0 = pl.q[0].lim + 1, n1 = pl.q[1].lim + 1;
            if (!wait(c.bar + Bars::kQFull + 0, local & 1) || !wait(c.bar + Bars::kQFull + 8, local & 1)) break;
            for (int j = 0; j < n1; ++j) {
                uint32_t ks;
                if (!wait.take(rk, ks)) break;
                for (int t = 0; t < 2; ++t) {
                    if (t == 0 && j >= n0) continue;
                    if (s_issued[t] > 0 && !wait(c.bar + Bars::kSFree + 8 * t, (s_issued[t] - 1) & 1)) break;
                    tc_fence_after();
                    Mma<D>::qk(c, t, rk.smem + ks * C::kTileBytes);
                    tc_commit(c.bar + Bars::kSFull + 8 * t);
                    ++s_issued[t];
                }
                if (!wait.ok) break;
                if (j + 1 == n1) tc_commit(c.bar + Bars::kQEmpty);
                tc_commit(rk.empty + 8 * ks);
            }
        }
        if (!wait.ok) mma_drain(c, 0);
    } else {
        // sparse: the union of both Q tiles' key tiles
        using C = Cfg<D>;
        Ring rk{c.base + C::kRingOff, c.bar + Bars::kKFull, c.bar + Bars::kKEmpty, (uint32_t)C::kKSlots, 0};
        Waiter wait{c, true};
        uint32_t s_issued[2] = {0u, 0u};
        uint32_t q_units = 0;
        for (int u = blockIdx.x; wait.ok && u < c.p.total_units; u += gridDim.x) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const Plan<MODE> pl = make_plan<MODE>(w, c.p, c.masks);
            int j = pl.next(0);
            if (j == kNoTile) continue;
            if (!wait(c.bar + Bars::kQFull + 0, q_units & 1) || !wait(c.bar + Bars::kQFull + 8, q_units & 1)) break;
            ++q_units;
            while (j != kNoTile) {
                uint32_t ks;
                if (!wait.take(rk, ks)) break;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!pl.need(t, j)) continue;
                    if (s_issued[t] > 0 && !wait(c.bar + Bars::kSFree + 8 * t, (s_issued[t] - 1) & 1)) break;
                    tc_fence_after();
                    Mma<D>::qk(c, t, rk.smem + ks * C::kTileBytes);
                    tc_commit(c.bar + Bars::kSFull + 8 * t);
                    ++s_issued[t];
                }
                if (!wait.ok) break;
                j = pl.next(j + 1);
                if (j == kNoTile) tc_commit(c.bar + Bars::kQEmpty);
                tc_commit(rk.empty + 8 * ks);
            }
        }
        if (!wait.ok) mma_drain(c, 0);
    }
}

// Split layout, P V stream: O_t (+)= P_t(j) V_j once the softmax has written P_t(j).
template <int D, int MODE>
__device__ __forceinline__ void role_mma_pv(const Ctx& c) {
    if constexpr (MODE != kModeSparse) {
        // full / causal: Q tile 0 visits key tiles [0, n0), Q tile 1 [0, n1), n0 <= n1
        using C = Cfg<D>;
        Ring rv{c.base + C::kVRingOff, c.bar + Bars::kVFull, c.bar + Bars::kVEmpty, (uint32_t)C::kVSlots, 0};
        Waiter wait{c, true};
        uint32_t p_phase[2] = {0u, 0u};
        int local = 0;
        for (int u = blockIdx.x; wait.ok && u < c.p.total_units; u += gridDim.x, ++local) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const Plan<MODE> pl = make_plan<MODE>(w, c.p, c.masks);
            const int n0 = pl.q[0].lim + 1, n1 = pl.q[1].lim + 1;
            for (int j = 0; j < n1; ++j) {
                uint32_t vs;
                if (!wait.take(rv, vs)) break;
                for (int t = 0; t < 2; ++t) {
                    const int n = t == 0 ? n0 : n1;
                    if (j >= n) continue;
                    if (!wait(c.bar + Bars::kPFull + 8 * t, p_phase[t])) break;
                    p_phase[t] ^= 1u;
                    if (j == 0 && !wait(c.bar + Bars::kOEmpty + 8 * t, (local & 1) ^ 1)) break;
                    tc_fence_after();
                    Mma<D>::pv(c, t, rv.smem + vs * C::kTileBytes, j > 0);
                    tc_commit(c.bar + Bars::kPFree + 8 * t);
                    if (j + 1 == n) tc_commit(c.bar + Bars::kOFull + 8 * t);
                }
                if (!wait.ok) break;
                tc_commit(rv.empty + 8 * vs);
            }
        }
        if (!wait.ok) mma_drain(c, 1);
    } else {
        // sparse: the union of both Q tiles' key tiles
        using C = Cfg<D>;
        Ring rv{c.base + C::kVRingOff, c.bar + Bars::kVFull, c.bar + Bars::kVEmpty, (uint32_t)C::kVSlots, 0};
        Waiter wait{c, true};
        uint32_t p_phase[2] = {0u, 0u};
        uint32_t o_units[2] = {0u, 0u};  // units in which Q tile t accumulated an O
        for (int u = blockIdx.x; wait.ok && u < c.p.total_units; u += gridDim.x) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const Plan<MODE> pl = make_plan<MODE>(w, c.p, c.masks);
            const int first[2] = {pl.q[0].next(0), pl.q[1].next(0)};
            const int last[2] = {pl.q[0].last(), pl.q[1].last()};
            for (int j = pl.next(0); j != kNoTile; j = pl.next(j + 1)) {
                uint32_t vs;
                if (!wait.take(rv, vs)) break;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!pl.need(t, j)) continue;
                    if (!wait(c.bar + Bars::kPFull + 8 * t, p_phase[t])) break;
                    p_phase[t] ^= 1u;
                    const bool is_first = j == first[t];
                    if (is_first && !wait(c.bar + Bars::kOEmpty + 8 * t, (o_units[t] & 1) ^ 1)) break;
                    tc_fence_after();
                    Mma<D>::pv(c, t, rv.smem + vs * C::kTileBytes, !is_first);
                    tc_commit(c.bar + Bars::kPFree + 8 * t);
                    if (j == last[t]) {
                        tc_commit(c.bar + Bars::kOFull + 8 * t);
                        ++o_units[t];
                    }
                }
                if (!wait.ok) break;
                tc_commit(rv.empty + 8 * vs);
            }
        }
        if (!wait.ok) mma_drain(c, 1);
    }
}

// Shared layout (P over S): one ordered stream per key tile j of the union,
// with j' the next one: P_0 V_j, S_0(j'), P_1 V_j, S_1(j') (each product only
// where Q tile t takes part in that tile).  S_t(j') overwrites P_t of t's
// previous tile after the product that reads it, by issue order.
template <int D, int MODE>
__device__ __forceinline__ void role_mma_ordered(const Ctx& c) {
    if constexpr (MODE != kModeSparse) {
        // full / causal: Q tile 0 visits key tiles [0, n0), Q tile 1 [0, n1), n0 <= n1
        using C = Cfg<D>;
        Ring r{c.base + C::kRingOff, c.bar + Bars::kKFull, c.bar + Bars::kKEmpty, (uint32_t)C::kKSlots, 0};
        Waiter wait{c, true};
        uint32_t p_phase[2] = {0u, 0u};
        int local = 0;
        auto smem = [&](uint32_t slot) { return r.smem + slot * C::kTileBytes; };
        for (int u = blockIdx.x; wait.ok && u < c.p.total_units; u += gridDim.x, ++local) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const Plan<MODE> pl = make_plan<MODE>(w, c.p, c.masks);
            const int n0 = pl.q[0].lim + 1, n1 = pl.q[1].lim + 1;
            if (!wait(c.bar + Bars::kQFull + 0, local & 1) || !wait(c.bar + Bars::kQFull + 8, local & 1)) break;
            uint32_t ks;
            if (!wait.take(r, ks)) break;
            tc_fence_after();
            Mma<D>::qk(c, 0, smem(ks));
            tc_commit(c.bar + Bars::kSFull + 0);
            Mma<D>::qk(c, 1, smem(ks));
            tc_commit(c.bar + Bars::kSFull + 8);
            if (n1 == 1) tc_commit(c.bar + Bars::kQEmpty);
            tc_commit(r.empty + 8 * ks);
            for (int j = 0; j < n1; ++j) {
                uint32_t vs, ks2 = 0;
                const bool has_next = j + 1 < n1;
                if (!wait.take(r, vs)) break;
                if (has_next && !wait.take(r, ks2)) break;
                if (j < n0) {
                    if (!wait(c.bar + Bars::kPFull + 0, p_phase[0])) break;
                    p_phase[0] ^= 1u;
                    if (j == 0 && !wait(c.bar + Bars::kOEmpty + 0, (local & 1) ^ 1)) break;
                    tc_fence_after();
                    Mma<D>::pv(c, 0, smem(vs), j > 0);
                    if (j + 1 < n0) {
                        Mma<D>::qk(c, 0, smem(ks2));
                        tc_commit(c.bar + Bars::kSFull + 0);
                    } else {
                        tc_commit(c.bar + Bars::kOFull + 0);
                    }
                }
                if (!wait(c.bar + Bars::kPFull + 8, p_phase[1])) break;
                p_phase[1] ^= 1u;
                if (j == 0 && !wait(c.bar + Bars::kOEmpty + 8, (local & 1) ^ 1)) break;
                tc_fence_after();
                Mma<D>::pv(c, 1, smem(vs), j > 0);
                tc_commit(r.empty + 8 * vs);
                if (has_next) {
                    Mma<D>::qk(c, 1, smem(ks2));
                    tc_commit(c.bar + Bars::kSFull + 8);
                    if (j + 2 == n1) tc_commit(c.bar + Bars::kQEmpty);
                    tc_commit(r.empty + 8 * ks2);
                } else {
                    tc_commit(c.bar + Bars::kOFull + 8);
                }
            }
        }
        if (!wait.ok) mma_drain(c, 0);
    } else {
        // sparse: the union of both Q tiles' key tiles
        using C = Cfg<D>;
        Ring r{c.base + C::kRingOff, c.bar + Bars::kKFull, c.bar + Bars::kKEmpty, (uint32_t)C::kKSlots, 0};
        Waiter wait{c, true};
        uint32_t p_phase[2] = {0u, 0u};
        uint32_t o_units[2] = {0u, 0u};
        uint32_t q_units = 0;
        auto smem = [&](uint32_t slot) { return r.smem + slot * C::kTileBytes; };
        for (int u = blockIdx.x; wait.ok && u < c.p.total_units; u += gridDim.x) {
            const Unit w = decode_unit<MODE>(u, c.p);
            const Plan<MODE> pl = make_plan<MODE>(w, c.p, c.masks);
            int j = pl.next(0);
            if (j == kNoTile) continue;
            const int first[2] = {pl.q[0].next(0), pl.q[1].next(0)};
            const int last[2] = {pl.q[0].last(), pl.q[1].last()};
            if (!wait(c.bar + Bars::kQFull + 0, q_units & 1) || !wait(c.bar + Bars::kQFull + 8, q_units & 1)) break;
            ++q_units;
            uint32_t ks;
            if (!wait.take(r, ks)) break;
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (!pl.need(t, j)) continue;
                Mma<D>::qk(c, t, smem(ks));
                tc_commit(c.bar + Bars::kSFull + 8 * t);
            }
            int jn = pl.next(j + 1);
            if (jn == kNoTile) tc_commit(c.bar + Bars::kQEmpty);
            tc_commit(r.empty + 8 * ks);
            while (j != kNoTile) {
                const bool has_next = jn != kNoTile;
                uint32_t vs, ks2 = 0;
                if (!wait.take(r, vs)) break;
                if (has_next && !wait.take(r, ks2)) break;
                const int jnn = has_next ? pl.next(jn + 1) : kNoTile;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (pl.need(t, j)) {
                        if (!wait(c.bar + Bars::kPFull + 8 * t, p_phase[t])) break;
                        p_phase[t] ^= 1u;
                        const bool is_first = j == first[t];
                        if (is_first && !wait(c.bar + Bars::kOEmpty + 8 * t, (o_units[t] & 1) ^ 1)) break;
                        tc_fence_after();
                        Mma<D>::pv(c, t, smem(vs), !is_first);
                        if (j == last[t]) {
                            tc_commit(c.bar + Bars::kOFull + 8 * t);
                            ++o_units[t];
                        }
                    }
                    if (t == 1) tc_commit(r.empty + 8 * vs);
                    if (has_next && pl.need(t, jn)) {
                        tc_fence_after();
                        Mma<D>::qk(c, t, smem(ks2));
                        tc_commit(c.bar + Bars::kSFull + 8 * t);
                    }
                }
                if (!wait.ok) break;
                if (has_next) {
                    if (jnn == kNoTile) tc_commit(c.bar + Bars::kQEmpty);
                    tc_commit(r.empty + 8 * ks2);
                }
                j = jn;
                jn = jnn;
            }
        }
        if (!wait.ok) mma_drain(c, 0);
    }
}

// ------------------------------------------------------- softmax + epilogue
// Columns [32 G, 32 G + 32) of one row: p = 2^(sl2 * s - m) (negm = -m) as
// 16 bf16 pairs in pk, summed into acc; the pairs marked in kPolyMask8 use
// the FMA-pipe exponential and fold their raw scores into pmax, the rest
// use MUFU (ex2.approx).
// Warpgroup t owns Q tile t; thread = one query row = one TMEM lane.
template <int D, int MODE, bool MASK>
__device__ __forceinline__ void role_softmax(const Ctx& c, int warp, int lane, uint16_t* __restrict__ out_o,
                                             float* __restrict__ out_lse) {
    using C = Cfg<D>;
    const Params& p = c.p;
    const int t = warp >> 2;                  // Q tile of this warpgroup
    const int quarter = warp & 3;             // TMEM lane quarter of this warp
    const int r_in_tile = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = c.tmem + lane_off + (t == 0 ? C::kColS0 : C::kColS1);
    const uint32_t t_o = c.tmem + lane_off + (t == 0 ? C::kColO0 : C::kColO1);
    const uint32_t t_p = c.tmem + lane_off + (t == 0 ? C::kColP0 : C::kColP1);
    const uint32_t b_s = c.bar + Bars::kSFull + 8 * t;
    const uint32_t b_p = c.bar + Bars::kPFull + 8 * t;
    const uint32_t b_of = c.bar + Bars::kOFull + 8 * t;
    const uint32_t b_oe = c.bar + Bars::kOEmpty + 8 * t;
    const uint32_t b_sfree = c.bar + Bars::kSFree + 8 * t;
    const uint32_t b_pfree = c.bar + Bars::kPFree + 8 * t;
    const float sl2 = p.scale_log2;
    uint32_t s_phase = 0;
    uint32_t pv_count = 0;  // P_t V products issued before the current step (split layout)
    bool ok = true;
    int local = 0;
    uint32_t o_units = 0;  // sparse: units in which this Q tile has key tiles
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x, ++local) {
        const Unit w = decode_unit<MODE>(u, p);
        const int row = w.q0 + t * kBlockM + r_in_tile;
        // step j visits key tile j (full, causal) or the j-th key tile kj of
        // this Q tile's mask row (sparse)
        // sparse: walk next() until it runs out.  Across a step only the
        // padding row and the current 32-tile window (which tiles are
        // visited, which hold a padded key) stay live; the rest of the tile
        // walker is rebuilt when needed (the softmax thread is at its
        // register limit during the exponentials).
        const uint32_t pad_row = (MODE == kModeSparse || MASK) ? pad_row_of(w, p, c.masks) : 0u;
        int wi = -1;          // window index (tiles 32 wi .. 32 wi + 31)
        uint32_t ww = 0u;     // its visited tiles
        int mix_i = -1;       // staged padding: index of the "holds a padded key" word in mix_w
        uint32_t mix_w = 0u;
        const int n_kv = MODE == kModeSparse ? 0 : key_tiles<MODE>(w, p, c.masks, t).count();
        int kj;
        {
            const KeyTiles<MODE> kt = key_tiles_row<MODE>(w, p, c.masks, t, pad_row);
            kj = kt.next(0);
            wi = kt.wi;
            ww = kt.ww;
        }
        if constexpr (MODE == kModeSparse) {
            if (kj == kNoTile) {
                // no key block at all: O = 0 and LSE = -inf, as for a row
                // whose keys are all masked (no barrier of this unit is used)
                if (row < p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(out_o + w.b * p.o_sb + w.h * p.o_sh + row * p.o_sn);
#pragma unroll
                    for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
                    out_lse[static_cast<size_t>(w.bh) * p.N + row] = -INFINITY;
                }
                continue;
            }
        }
        // last visible key of this row (the row itself when causal)
        const bool causal = MODE == kModeCausal || (MODE == kModeSparse && p.causal);
        const int last_key = causal ? min(row, p.N - 1) : p.N - 1;
        float m = -INFINITY;  // reference max of scale*log2(e)*s (log2 units), shared by O and l
        float l = 0.f;        // sum of exp2(scale*log2(e)*s - m) over the keys seen so far

        for (int j = 0; MODE == kModeSparse ? kj != kNoTile : j < n_kv; ++j) {
            const int key_tile = MODE == kModeSparse ? kj : j;
            if constexpr (MODE == kModeSparse) {
                // the next step's tile; the window moves (one shared load) every 32 tiles
                const KeyTiles<MODE> kt = key_tiles_row<MODE>(w, p, c.masks, t, pad_row, wi, ww);
                kj = kt.next(kj + 1);
                wi = kt.wi;
                ww = kt.ww;
            }
            if (MASK && pad_row != 0u && (key_tile >> 5) != mix_i) {
                // which tiles of this 32-tile window hold a padded key (one shared load)
                mix_i = key_tile >> 5;
                mix_w = lds_u32(PadRow::mix(pad_row, p.n_kv_all) + 4u * mix_i);
            }
            bool got = wait_bounded(b_s, s_phase, c.abort_flag, p.wait_ns);
            got = __all_sync(0xffffffffu, got);
            if (!got) {
                ok = false;
                break;
            }
            s_phase ^= 1u;
            tc_fence_after();

            float s[kBlockN];
            {
                uint32_t r[4][32];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(t_s + c4 * 32, r[c4]);
                tmem_wait_ld();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    reg_fence32(r[c4]);
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) s[c4 * 32 + cc] = __uint_as_float(r[c4][cc]);
                }
            }
            if (C::kSplit) {
                // S_t is in registers: the S stream may refill it with the next key tile
                tc_fence_before();
                mbar_arrive(b_sfree);
            }
            // key padding: padded keys get -inf.  Staged: the tile's "holds a
            // padded key" bit (one shared load per 32 tiles) says whether its
            // 128 per-key bits are needed at all; otherwise the 128 mask bytes
            // are read.  The masking sits behind one warp-wide branch.
            if (MASK) {
                uint32_t pw[4] = {0u, 0u, 0u, 0u};
                if (pad_row != 0u) {
                    if ((mix_w >> (key_tile & 31)) & 1u) {
                        const uint4 pb = pad_tile_bits(pad_row, key_tile);
                        pw[0] = pb.x, pw[1] = pb.y, pw[2] = pb.z, pw[3] = pb.w;
                    }
                } else {
                    // not staged (too large for shared memory): 16 bytes at a time
                    const int key0 = key_tile * kBlockN;
                    const uint8_t* mrow = p.key_pad + static_cast<size_t>(w.b) * p.N + key0;
                    const bool vec = p.pad_vec && key0 + kBlockN <= p.N;
#pragma unroll
                    for (int g = 0; g < kBlockN / 16; ++g) {
                        uint4 x;
                        if (vec) {
                            x = ldg_nc16(mrow + 16 * g);
                        } else {
                            uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (key0 + 16 * g + e < p.N)
                                    wd[e >> 2] |= static_cast<uint32_t>(mrow[16 * g + e] != 0) << (8 * (e & 3));
                            x = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                        }
                        const uint32_t bits16 = nonzero_bytes4(x.x) | (nonzero_bytes4(x.y) << 4) |
                                                (nonzero_bytes4(x.z) << 8) | (nonzero_bytes4(x.w) << 12);
                        if (g & 1) pw[g >> 1] |= bits16 << 16;
                        else pw[g >> 1] = bits16;
                    }
                }
                if (__any_sync(0xffffffffu, (pw[0] | pw[1] | pw[2] | pw[3]) != 0u)) {
#pragma unroll
                    for (int cc = 0; cc < kBlockN; ++cc)
                        if ((pw[cc >> 5] >> (cc & 31)) & 1u) s[cc] = -INFINITY;
                }
            }
            // key-tail and causal mask: keys past last_key get -inf
            const int lim = last_key - key_tile * kBlockN;
            if (lim < kBlockN - 1) {
#pragma unroll
                for (int cc = 0; cc < kBlockN; ++cc)
                    if (cc > lim) s[cc] = -INFINITY;
            }
            // row maximum (scale > 0, so it is taken on the raw scores)
            float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
            for (int cc = 4; cc < kBlockN; cc += 8) {
                mx[0] = fmax3(mx[0], s[cc], s[cc + 1]);
                mx[1] = fmax3(mx[1], s[cc + 2], s[cc + 3]);
                if (cc + 4 < kBlockN) {
                    mx[2] = fmax3(mx[2], s[cc + 4], s[cc + 5]);
                    mx[3] = fmax3(mx[3], s[cc + 6], s[cc + 7]);
                }
            }
            const float row_max = fmax3(fmax3(mx[0], mx[1], mx[2]), mx[3], -INFINITY) * sl2;
            // lazy rescaling: move the reference only when the row maximum
            // exceeds it by more than 2^8 (always on a row's first visible key);
            // O and l always share the reference, so the result stays exact
            const bool move = row_max > m + kLazyRescaleLog2;
            float alpha = 1.f;
            if (move) {
                alpha = ex2(m - row_max);  // 0 when m was -inf
                m = row_max;
            }
            l *= alpha;
            const float m_use = (m == -INFINITY) ? 0.f : m;
            const float2 sl2x2 = make_float2(sl2, sl2);
            const float2 negm = make_float2(-m_use, -m_use);

            // P = exp2(scale*log2(e)*s - m) as bf16 pairs; the pairs marked in
            // kPolyMask8 use the FMA-pipe exponential, the rest MUFU; masked
            // scores (-inf) give exactly +0 on both.
            float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            uint32_t pk[kBlockN / 2];
#pragma unroll
            for (int cc = 0; cc < kBlockN / 2; ++cc) {
                float2 x = __ffma2_rn(make_float2(s[2 * cc], s[2 * cc + 1]), sl2x2, negm);
                if ((kPolyMask8 >> (cc & 7)) & 1u) {
                    x = ex2_poly2(x);
                } else {
                    x.x = ex2(x.x);
                    x.y = ex2(x.y);
                }
                acc[cc & 1] = __fadd2_rn(acc[cc & 1], x);
                pk[cc] = pack_bf16x2(x.x, x.y);
            }
            l += (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
            const bool rescale = move && j > 0;
            if (C::kSplit) {
                // P_t and O_t belong to the previous P V until it retires
                if (pv_count > 0) {
                    bool done = wait_bounded(b_pfree, (pv_count - 1) & 1, c.abort_flag, p.wait_ns);
                    done = __all_sync(0xffffffffu, done);
                    if (!done) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                ++pv_count;
            }
            tmem_st32(t_p, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(t_p + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            // O holds the sum over earlier tiles at the old reference: bring it
            // to the new one before the next P V accumulates into it (the
            // previous P V has retired: waited for above in the split layout,
            // implied by S_t in the shared one)
            if (__any_sync(0xffffffffu, rescale)) {
                const float a = rescale ? alpha : 1.f;
#pragma unroll
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t r[32];
                    tmem_ld32(t_o + c4 * 32, r);
                    tmem_wait_ld();
                    reg_fence32(r);
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) r[cc] = __float_as_uint(__uint_as_float(r[cc]) * a);
                    tmem_st32(t_o + c4 * 32, r);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(b_p);
        }
        if (!ok) break;

        // ---------------------------------------------------------- epilogue
        bool got = wait_bounded(b_of, (MODE == kModeSparse ? o_units++ : local) & 1, c.abort_flag, p.wait_ns);
        got = __all_sync(0xffffffffu, got);
        if (!got) {
            ok = false;
            break;
        }
        tc_fence_after();
        // a row that saw no visible key (every key it may see is padded) keeps
        // m = -inf: its O is 0 and its LSE -inf
        const bool empty = (m == -INFINITY);
        const float inv_l = empty ? 0.f : 1.f / l;
        const bool store = row < p.N;
        uint16_t* orow = out_o + w.b * p.o_sb + w.h * p.o_sh + (store ? row : 0) * p.o_sn;
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t r[32];
            tmem_ld32(t_o + c4 * 32, r);
            tmem_wait_ld();
            reg_fence32(r);
            if (c4 == D / 32 - 1) {
                tc_fence_before();
                mbar_arrive(b_oe);  // O_t may now be overwritten by the next unit
            }
            uint32_t pk[16];
#pragma unroll
            for (int cc = 0; cc < 16; ++cc)
                pk[cc] = pack_bf16x2(__uint_as_float(r[2 * cc]) * inv_l, __uint_as_float(r[2 * cc + 1]) * inv_l);
            if (store) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            }
        }
        if (store) out_lse[static_cast<size_t>(w.bh) * p.N + row] = empty ? -INFINITY : (m + __log2f(l)) * kLn2;
    }
}

// Sparse mode: the [n_kv_all, n_kv_all] block-mask bytes become bits in shared
// memory (bit f = byte f != 0, row-major), every thread taking whole 32-bit
// words; full words read the bytes 16 at a time (the mask is 16-byte aligned).
__device__ __forceinline__ void stage_block_mask(const Params& p, uint32_t* bits) {
    const long long total = static_cast<long long>(p.n_kv_all) * p.n_kv_all;
    const int words = static_cast<int>((total + 31) / 32);
    for (int wi = threadIdx.x; wi < words; wi += kThreads) {
        const long long f0 = static_cast<long long>(wi) * 32;
        uint32_t word = 0u;
        if (f0 + 32 <= total) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 x = ldg_nc16(p.block_mask + f0 + 16 * h);
                word |= (nonzero_bytes4(x.x) | (nonzero_bytes4(x.y) << 4) | (nonzero_bytes4(x.z) << 8) |
                         (nonzero_bytes4(x.w) << 12)) << (16 * h);
            }
        } else {
            for (int e = 0; f0 + e < total; ++e) word |= static_cast<uint32_t>(p.block_mask[f0 + e] != 0) << e;
        }
        bits[wi] = word;
    }
}

// Key padding, staged: thread 0 maps each of this CTA's units to a row (one
// per distinct batch), then every thread fills whole 32-bit words of the rows
// (bit = key padded; keys past N count as padded).  Rows are read 16 bytes
// at a time when the mask allows it.
template <int MODE>
__device__ __forceinline__ void stage_key_padding(const Params& p, uint32_t* map, int* rowb, uint32_t* rows,
                                                  int& n_rows) {
    if (threadIdx.x == 0) {
        int nr = 0;
        int k = 0;
        for (int u = blockIdx.x; u < p.total_units && k < p.pad_units; u += gridDim.x, ++k) {
            const int b = decode_unit<MODE>(u, p).b;
            int r = 0;
            while (r < nr && rowb[r] != b) ++r;
            if (r == nr) rowb[nr++] = b;
            map[k] = static_cast<uint32_t>(r);
        }
        n_rows = nr;
    }
    __syncthreads();
    const int key_words = 4 * p.n_kv_all;  // per row
    for (int i = threadIdx.x; i < n_rows * key_words; i += kThreads) {
        const int r = i / key_words;
        const int key0 = (i - r * key_words) * 32;
        const uint8_t* src = p.key_pad + static_cast<size_t>(rowb[r]) * p.N;
        uint32_t word;
        if (p.pad_vec && key0 + 32 <= p.N) {
            const uint4 a = ldg_nc16(src + key0), b = ldg_nc16(src + key0 + 16);
            word = nonzero_bytes4(a.x) | (nonzero_bytes4(a.y) << 4) | (nonzero_bytes4(a.z) << 8) |
                   (nonzero_bytes4(a.w) << 12) | (nonzero_bytes4(b.x) << 16) | (nonzero_bytes4(b.y) << 20) |
                   (nonzero_bytes4(b.z) << 24) | (nonzero_bytes4(b.w) << 28);
        } else {
            word = 0u;
            for (int e = 0; e < 32; ++e)
                if (key0 + e >= p.N || src[key0 + e] != 0) word |= 1u << e;
        }
        rows[static_cast<size_t>(r) * p.pad_row_words + (i - r * key_words)] = word;
    }
    __syncthreads();
    // the two tile bitmaps of every row: bit t of word i is tile 32 i + t
    const int n_tiles = p.n_kv_all;
    const int bm_words = (n_tiles + 31) / 32;
    for (int i = threadIdx.x; i < 2 * n_rows * bm_words; i += kThreads) {
        const int kind = i / (n_rows * bm_words);  // 0: holds an unpadded key, 1: holds a padded key
        const int rem = i - kind * n_rows * bm_words;
        const int r = rem / bm_words, wd = rem - r * bm_words;
        const uint32_t* row = rows + static_cast<size_t>(r) * p.pad_row_words;
        uint32_t word = 0u;
        for (int t = 0; t < 32 && 32 * wd + t < n_tiles; ++t) {
            const uint4 b = *reinterpret_cast<const uint4*>(row + 4 * (32 * wd + t));
            const bool flag = kind == 0 ? (b.x & b.y & b.z & b.w) != ~0u : (b.x | b.y | b.z | b.w) != 0u;
            word |= static_cast<uint32_t>(flag) << t;
        }
        rows[static_cast<size_t>(r) * p.pad_row_words + 4 * n_tiles + kind * bm_words + wd] = word;
    }
    __syncthreads();
    // the last tile holding an unpadded key, from the first bitmap
    for (int r = threadIdx.x; r < n_rows; r += kThreads) {
        const uint32_t* occ = rows + static_cast<size_t>(r) * p.pad_row_words + 4 * n_tiles;
        int last = -1;
        for (int wd = bm_words - 1; wd >= 0 && last < 0; --wd)
            if (occ[wd] != 0u) last = 32 * wd + 31 - __clz(static_cast<int>(occ[wd]));
        rows[static_cast<size_t>(r) * p.pad_row_words + 4 * n_tiles + 2 * bm_words] = static_cast<uint32_t>(last);
    }
}

// ----------------------------------------------------------------- the kernel
template <int D, int MODE, bool MASK>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out_o,
                float* __restrict__ out_lse, const Params p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128B-swizzled tiles need 1 KB alignment
    uint8_t* const gbase = smem_raw + (base - raw);
    const uint32_t bar = base + C::kBarOff;
    volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + C::kBarOff + Bars::kAbort);
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::kBarOff + Bars::kTmemSlot);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar + Bars::kQFull + 8 * t, 1);
            mbar_init(bar + Bars::kSFull + 8 * t, 1);
            mbar_init(bar + Bars::kPFull + 8 * t, kBlockM);
            mbar_init(bar + Bars::kOFull + 8 * t, 1);
            mbar_init(bar + Bars::kOEmpty + 8 * t, kBlockM);
            mbar_init(bar + Bars::kDrain + 8 * t, 1);
            mbar_init(bar + Bars::kSFree + 8 * t, kBlockM);
            mbar_init(bar + Bars::kPFree + 8 * t, 1);
        }
        mbar_init(bar + Bars::kQEmpty, 1);
        for (int s = 0; s < 8; ++s) {
            mbar_init(bar + Bars::kKFull + 8 * s, 1);
            mbar_init(bar + Bars::kKEmpty + 8 * s, 1);
            mbar_init(bar + Bars::kVFull + 8 * s, 1);
            mbar_init(bar + Bars::kVEmpty + 8 * s, 1);
        }
        *abort_flag = 0u;
        fence_barrier_init();
        fence_proxy_async();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    uint32_t* const mask_bits = reinterpret_cast<uint32_t*>(gbase + C::kMaskOff);
    if (MODE == kModeSparse && p.block_mask != nullptr) stage_block_mask(p, mask_bits);
    Masks masks{MODE == kModeSparse && p.block_mask != nullptr ? smem_addr(mask_bits) : 0u, 0u, 0u};
    if (MASK && p.pad_staged) {
        uint32_t* map = reinterpret_cast<uint32_t*>(gbase + p.pad_map_off);
        int* rowb = reinterpret_cast<int*>(gbase + p.pad_rowb_off);
        uint32_t* rows = reinterpret_cast<uint32_t*>(gbase + p.pad_rows_off);
        stage_key_padding<MODE>(p, map, rowb, rows, *reinterpret_cast<int*>(gbase + C::kBarOff + Bars::kPadRows));
        masks.pad_map = smem_addr(map);
        masks.pad_rows = smem_addr(rows);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const Ctx ctx{base, bar, *tmem_slot, abort_flag, masks, p};

    if (warp >= kLoadWarp) {
        regs_decrease<kOtherRegs>();
        if (lane == 0) {
            if (warp == kLoadWarp) {
                role_producer<D, MODE>(ctx, &tm_q, &tm_k, &tm_v);
            } else if (warp == kMmaWarp) {
                if (C::kSplit) role_mma_s<D, MODE>(ctx);
                else role_mma_ordered<D, MODE>(ctx);
            } else if (warp == kMmaPvWarp && C::kSplit) {
                role_mma_pv<D, MODE>(ctx);
            }
        }
        __syncwarp();
    } else {
        regs_increase<kSoftmaxRegs>();
        role_softmax<D, MODE, MASK>(ctx, warp, lane, out_o, out_lse);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(ctx.tmem, kTmemCols);
    }
}

// A kernel that waits on a barrier nobody arrives at, to exercise the bounded
// wait: it must give up after limit_ns, record the timeout and return.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t b;
    const uint32_t bar = smem_addr(&b);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_bounded(bar, 0, nullptr, limit_ns);
    __syncthreads();
}

// Evaluates the softmax's FMA-pipe exponential on a device buffer, two
// elements per call as the kernel does, so that it can be checked against
// 2^x on the host.  One thread per pair; an odd last element is paired with
// itself.
__global__ void ex2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    const int pairs = (n + 1) / 2;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < pairs; i += gridDim.x * blockDim.x) {
        const int a = 2 * i, b = min(2 * i + 1, n - 1);
        const float2 r = ex2_poly2(make_float2(x[a], x[b]));
        y[a] = r.x;
        if (b != a) y[b] = r.y;
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

struct DriverFns {
    EncodeTiledFn encode = nullptr;
    AddressRangeFn range = nullptr;
    bool ok = false;
};

DriverFns& driver_fns() {
    static DriverFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q1, q2;
        void* f1 = nullptr;
        void* f2 = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuMemGetAddressRange", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            fns.encode = reinterpret_cast<EncodeTiledFn>(f1);
            fns.range = reinterpret_cast<AddressRangeFn>(f2);
            fns.ok = true;
        }
    });
    return fns;
}

// A bf16 tensor indexed [b, h, n, k] with element strides (sb, sh, sn, 1),
// viewed as a 4-D tensor (k, n, h, b); box = 64 columns x 128 rows x 1 x 1,
// 128-byte swizzle.  Rows past N read as zeros.
bool encode_qkv_map(CUtensorMap* map, const void* ptr, int B, int H, int N, int d, long long sb, long long sh,
                    long long sn) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(sn) * 2, static_cast<cuuint64_t>(sh) * 2,
                                   static_cast<cuuint64_t>(sb) * 2};
    const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(kBlockN), 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return driver_fns().encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
                               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of recent calls.  A map is a pure function of (address, sizes,
// strides), so a hit is always the map a fresh encode would give, whatever
// happened to the memory in between; the cache only saves the encode.
struct MapCache {
    struct Entry {
        const void* ptr;
        int B, H, N, d;
        long long sb, sh, sn;
        bool used;
        CUtensorMap map;
    };
    static constexpr int kEntries = 24;
    std::mutex m;
    Entry e[kEntries] = {};
    int next = 0;
};

bool cached_qkv_map(CUtensorMap* map, const void* ptr, int B, int H, int N, int d, long long sb, long long sh,
                    long long sn) {
    static MapCache cache;
    std::lock_guard<std::mutex> lock(cache.m);
    for (const MapCache::Entry& x : cache.e)
        if (x.used && x.ptr == ptr && x.B == B && x.H == H && x.N == N && x.d == d && x.sb == sb && x.sh == sh &&
            x.sn == sn) {
            *map = x.map;
            return true;
        }
    if (!encode_qkv_map(map, ptr, B, H, N, d, sb, sh, sn)) return false;
    MapCache::Entry& x = cache.e[cache.next];
    cache.next = (cache.next + 1) % MapCache::kEntries;
    x = MapCache::Entry{ptr, B, H, N, d, sb, sh, sn, true, *map};
    return true;
}

constexpr int kMaxDevices = 64;

// Multiprocessor count of a device, looked up once per device (0 on failure).
int sm_count(int dev) {
    static std::atomic<int> cached[kMaxDevices] = {};
    if (dev < 0 || dev >= kMaxDevices) return 0;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 0;
    cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Largest element offset + 1 of a [B, H, N, d] tensor with the given strides
// (0 if it would not fit in 2^46 elements).
size_t span_elems(int B, int H, int N, int d, long long sb, long long sh, long long sn) {
    const unsigned __int128 e = static_cast<unsigned __int128>(B - 1) * sb +
                                static_cast<unsigned __int128>(H - 1) * sh +
                                static_cast<unsigned __int128>(N - 1) * sn + d;
    return e > (static_cast<unsigned __int128>(1) << 46) ? 0 : static_cast<size_t>(e);
}

// The pointer must be device memory of `device` and its allocation must hold `bytes` from it.
bool device_span_ok(const void* ptr, size_t bytes, int device) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return false;
    if (a.device != device) return false;
    CUdeviceptr lo = 0;
    size_t size = 0;
    if (driver_fns().range(&lo, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return false;
    const uintptr_t p = reinterpret_cast<uintptr_t>(ptr);
    return p >= lo && bytes <= size && p - lo <= size - bytes;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// True when the d-element rows (b, h, n) of a strided [B, H, N, d] output are
// nested without overlap: taking the dimensions of extent > 1 by increasing
// stride, each stride is at least the span of the rows below it.  Every
// layout in which rows of different (b, h, n) could share an element fails
// (CTAs would write the same bytes in no defined order); so do a few exotic
// interleavings that happen to be disjoint.
bool rows_nested(int B, int H, int N, int d, long long sb, long long sh, long long sn) {
    struct Dim { long long stride, extent; } dims[3] = {{sb, B}, {sh, H}, {sn, N}};
    for (int i = 1; i < 3; ++i)  // insertion sort by stride
        for (int j = i; j > 0 && dims[j].stride < dims[j - 1].stride; --j) {
            const Dim t = dims[j];
            dims[j] = dims[j - 1];
            dims[j - 1] = t;
        }
    long long span = d;  // elements covered by the rows of the smaller-stride dimensions
    for (const Dim& x : dims) {
        if (x.extent <= 1) continue;
        if (x.stride < span) return false;
        span += (x.extent - 1) * x.stride;  // stride <= 2^36 and extent < 2^31: no overflow
    }
    return true;
}

// Largest block-mask side the shared-memory bit copy takes (N <= 65536).
constexpr int kMaxMaskTiles = 512;

// Dynamic shared memory of one CTA: the fixed part, the block-mask bits, and
// (when it fits) the staged key padding, whose offsets are written to p.
constexpr int kMaxSmemPerBlock = 232448;       // 227 KB opt-in limit per block on sm_100
constexpr int kMaxPadStageBytes = 48 * 1024;   // cap on the staged key padding

template <int D>
int smem_layout(Params& p, bool sparse) {
    const long long bits = p.block_mask != nullptr ? static_cast<long long>(p.n_kv_all) * p.n_kv_all : 0;
    int smem = Cfg<D>::kSmemBytes + (sparse ? static_cast<int>((bits + 127) / 128) * 16 : 0);
    p.pad_staged = 0;
    if (p.key_pad != nullptr) {
        auto up16 = [](long long x) { return (x + 15) / 16 * 16; };
        const long long units = p.pad_units;
        const long long rows = units < p.BH / p.H ? units : p.BH / p.H;  // distinct batches at most
        const long long row_bytes = 4LL * p.pad_row_words;
        const long long need = up16(4 * units) + up16(4 * units) + rows * row_bytes;
        if (need <= kMaxPadStageBytes && smem + need <= kMaxSmemPerBlock) {
            // offsets from the 1 KB aligned base: after the block-mask bits
            const long long base_off = Cfg<D>::kMaskOff + (sparse ? (bits + 127) / 128 * 16 : 0);
            p.pad_map_off = static_cast<int>(base_off);
            p.pad_rowb_off = static_cast<int>(base_off + up16(4 * units));
            p.pad_rows_off = static_cast<int>(base_off + up16(4 * units) + up16(4 * units));
            p.pad_staged = 1;
            smem += static_cast<int>(need);
        }
    }
    return smem;
}

template <int D, int MODE, bool MASK>
int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, void* o, float* lse,
           Params p, int grid, int dev, cudaStream_t stream) {
    auto kernel = attn_fwd_kernel<D, MODE, MASK>;
    const int smem = smem_layout<D>(p, MODE == kModeSparse);
    // the dynamic shared-memory limit of this instantiation, raised once per
    // device to the largest size asked for so far
    // device and context (a reset or a new context starts from the default)
    static std::mutex m;
    static int smem_set[kMaxDevices] = {};
    static unsigned long long ctx_of[kMaxDevices] = {};
    {
        std::lock_guard<std::mutex> lock(m);
        const unsigned long long ctx = current_context_id();
        const bool known = dev >= 0 && dev < kMaxDevices && ctx != 0 && ctx_of[dev] == ctx;
        if (!known || smem > smem_set[dev]) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
                return ATTN_ERR_CUDA;
            if (dev >= 0 && dev < kMaxDevices && ctx != 0) {
                smem_set[dev] = smem;
                ctx_of[dev] = ctx;
            }
        }
    }
    kernel<<<grid, kThreads, smem, stream>>>(mq, mk, mv, static_cast<uint16_t*>(o), lse, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

// The backward kernels keep their own status word (attn_bwd.cu).
int attn_bwd_take_device_status(int* status);

extern "C" {

int attn_version(void) { return 100; }

const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported head size (d must be 64 or 128)";
        case ATTN_ERR_CUDA: return "CUDA call failed";
        case ATTN_ERR_TIMEOUT: return "a bounded device wait ran out";
        default: return "unknown status";
    }
}

int attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                          int d, long long qkv_sb, long long qkv_sh, long long qkv_sn, long long o_sb, long long o_sh,
                          long long o_sn, const unsigned char* key_padding_mask, const unsigned char* block_mask,
                          float scale, int causal, attn_stream_t stream) {
    // ---- host-side validation: nothing touches the GPU until all of it passes
    if (B < 1 || H < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
    // scale must be a positive, finite fp32: masked keys are -inf scores and the
    // row maximum is taken before scaling.
    if (!isfinite(scale) || !(scale >= 1e-30f)) return ATTN_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(B) * H;
    if (BH > 0x7fffffffLL || N > 0x7fffffff - 2 * kBlockM) return ATTN_ERR_INVALID_ARG;
    // strides: positive, 16-byte multiples (TMA and the 16-byte O stores), and
    // small enough that every offset fits the 40-bit TMA stride range
    const long long lim = 1LL << 36;
    for (long long st : {qkv_sb, qkv_sh, qkv_sn, o_sb, o_sh, o_sn})
        if (st < 8 || st % 8 != 0 || st > lim) return ATTN_ERR_INVALID_ARG;
    if (qkv_sn < d || o_sn < d) return ATTN_ERR_INVALID_ARG;  // rows must not overlap
    if (!rows_nested(B, H, N, d, o_sb, o_sh, o_sn)) return ATTN_ERR_INVALID_ARG;  // no two O rows may alias
    auto misaligned = [](const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0; };
    if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(o, 16) || misaligned(lse, 4))
        return ATTN_ERR_INVALID_ARG;
    const size_t in_bytes = span_elems(B, H, N, d, qkv_sb, qkv_sh, qkv_sn) * 2;
    const size_t out_bytes = span_elems(B, H, N, d, o_sb, o_sh, o_sn) * 2;
    const size_t lbytes = static_cast<size_t>(BH) * N * 4;
    if (in_bytes == 0 || out_bytes == 0) return ATTN_ERR_INVALID_ARG;
    if (overlaps(o, out_bytes, q, in_bytes) || overlaps(o, out_bytes, k, in_bytes) ||
        overlaps(o, out_bytes, v, in_bytes) || overlaps(lse, lbytes, q, in_bytes) ||
        overlaps(lse, lbytes, k, in_bytes) || overlaps(lse, lbytes, v, in_bytes) || overlaps(lse, lbytes, o, out_bytes))
        return ATTN_ERR_INVALID_ARG;
    const size_t pad_bytes = static_cast<size_t>(B) * N;
    if (key_padding_mask &&
        (overlaps(o, out_bytes, key_padding_mask, pad_bytes) || overlaps(lse, lbytes, key_padding_mask, pad_bytes)))
        return ATTN_ERR_INVALID_ARG;
    const int n_tiles = (N + kBlockN - 1) / kBlockN;
    const size_t bm_bytes = static_cast<size_t>(n_tiles) * n_tiles;
    if (block_mask && (n_tiles > kMaxMaskTiles || misaligned(block_mask, 16) ||
                       overlaps(o, out_bytes, block_mask, bm_bytes) || overlaps(lse, lbytes, block_mask, bm_bytes)))
        return ATTN_ERR_INVALID_ARG;

    if (!driver_fns().ok) return ATTN_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (!device_span_ok(q, in_bytes, dev) || !device_span_ok(k, in_bytes, dev) || !device_span_ok(v, in_bytes, dev) ||
        !device_span_ok(o, out_bytes, dev) || !device_span_ok(lse, lbytes, dev) ||
        (key_padding_mask && !device_span_ok(key_padding_mask, pad_bytes, dev)) ||
        (block_mask && !device_span_ok(block_mask, bm_bytes, dev)))
        return ATTN_ERR_INVALID_ARG;
    const int sms = sm_count(dev);
    if (sms < 1) return ATTN_ERR_CUDA;

    alignas(64) CUtensorMap mq, mk, mv;
    if (!cached_qkv_map(&mq, q, B, H, N, d, qkv_sb, qkv_sh, qkv_sn) ||
        !cached_qkv_map(&mk, k, B, H, N, d, qkv_sb, qkv_sh, qkv_sn) ||
        !cached_qkv_map(&mv, v, B, H, N, d, qkv_sb, qkv_sh, qkv_sn))
        return ATTN_ERR_CUDA;

    Params p;
    p.BH = static_cast<int>(BH);
    p.H = H;
    p.N = N;
    p.o_sb = o_sb;
    p.o_sh = o_sh;
    p.o_sn = o_sn;
    p.key_pad = key_padding_mask;
    p.pad_vec = key_padding_mask && (reinterpret_cast<uintptr_t>(key_padding_mask) & 15) == 0 && N % 16 == 0;
    p.block_mask = block_mask;
    p.causal = causal ? 1 : 0;
    p.n_pairs = (N + kUnitRows - 1) / kUnitRows;
    p.n_kv_all = (N + kBlockN - 1) / kBlockN;
    const long long units = BH * p.n_pairs;
    if (units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    p.total_units = static_cast<int>(units);
    p.scale_log2 = scale * kLog2e;
    p.wait_ns = kDefaultWaitNs;
    p.pad_row_words = PadRow::words(p.n_kv_all);
    p.pad_staged = 0;
    p.pad_map_off = p.pad_rowb_off = p.pad_rows_off = 0;
    const int grid = static_cast<int>(units < sms ? units : sms);
    p.pad_units = static_cast<int>((units + grid - 1) / grid);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool pad = key_padding_mask != nullptr;
    // a block mask selects the tile-list loops (only visited tiles are loaded
    // and multiplied); key padding masks per key and, once staged, ends each
    // Q tile's walk at its batch's last tile holding an unpadded key (with a
    // block mask: skips every tile made only of padded keys)
    const int mode = block_mask ? kModeSparse : causal ? kModeCausal : kModeFull;
#define ATTN_LAUNCH(D_, M_, P_) launch<D_, M_, P_>(mq, mk, mv, o, lse, p, grid, dev, s)
#define ATTN_BY_MODE(D_, P_)                                      \
    (mode == kModeSparse   ? ATTN_LAUNCH(D_, kModeSparse, P_)     \
     : mode == kModeCausal ? ATTN_LAUNCH(D_, kModeCausal, P_)     \
                           : ATTN_LAUNCH(D_, kModeFull, P_))
    if (d == 64) return pad ? ATTN_BY_MODE(64, true) : ATTN_BY_MODE(64, false);
    return pad ? ATTN_BY_MODE(128, true) : ATTN_BY_MODE(128, false);
#undef ATTN_BY_MODE
#undef ATTN_LAUNCH
}

int attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                     long long qkv_sb, long long qkv_sh, long long qkv_sn, long long o_sb, long long o_sh,
                     long long o_sn, const unsigned char* key_padding_mask, float scale, int causal,
                     attn_stream_t stream) {
    return attn_fwd_block_sparse(q, k, v, o, lse, B, H, N, d, qkv_sb, qkv_sh, qkv_sn, o_sb, o_sh, o_sn,
                                 key_padding_mask, nullptr, scale, causal, stream);
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
             float scale, int causal, attn_stream_t stream) {
    // contiguous [B, H, N, d]
    const long long sn = d, sh = static_cast<long long>(N) * d, sb = static_cast<long long>(H) * N * d;
    return attn_fwd_strided(q, k, v, o, lse, B, H, N, d, sb, sh, sn, sb, sh, sn, nullptr, scale, causal, stream);
}

int attn_check_device_status(attn_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
    int status = 0, bwd_status = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&status, g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (attn_bwd_take_device_status(&bwd_status) != ATTN_OK) return ATTN_ERR_CUDA;
    if (status == 0) status = bwd_status;
    return status == 0 ? ATTN_OK : status;
}

int attn_selftest_ex2(const float* x, float* y, int n, attn_stream_t stream) {
    if (n < 1 || !x || !y) return ATTN_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(n) * 4;
    if ((reinterpret_cast<uintptr_t>(x) & 3) || (reinterpret_cast<uintptr_t>(y) & 3) || overlaps(x, bytes, y, bytes))
        return ATTN_ERR_INVALID_ARG;
    if (!driver_fns().ok) return ATTN_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (!device_span_ok(x, bytes, dev) || !device_span_ok(y, bytes, dev)) return ATTN_ERR_INVALID_ARG;
    const int pairs = (n + 1) / 2;
    const int grid = pairs / 256 + 1 < 1024 ? pairs / 256 + 1 : 1024;
    ex2_selftest_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_selftest_wait_timeout(unsigned long long limit_ns, attn_stream_t stream) {
    if (limit_ns < 1000ull || limit_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
    wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"
