// gemm_sk.cu -- persistent stream-K tensor-core matmul Y = X * W^T on sm_100a
// (tcgen05 MMA, TMEM accumulators), in three flavours that issue the same MMA
// sequence on the same schedule, so their outputs are bit-identical:
//   * plain:   W loaded as BF16 (the uncompressed baseline and the twin);
//   * palette: W rebuilt in shared memory from its sign/mantissa plane, its
//              4-bit palette plane and its raw groups (Unweight page §七, the
//              reconstructive matmul; §五, decompressed weights never go back
//              to HBM);
//   * Huffman: the same rebuild, but the 4-bit palette indices are decoded
//              from the Huffman exponent stream inside the kernel (page §六,
//              pipeline 3's transcode moved into the matmul's producer: the
//              bytes read are the Huffman form and X, the only bytes written
//              are Y).
//
// Work decomposition.  A tile is 128 rows of W (the MMA's M) by BN tokens
// (the MMA's N); a unit is one 64-wide K-step of one tile.  Tiles are ordered
// row block major (the token blocks of one row block are neighbours, so a
// compressed W tile read by one CTA is still in L2 for the next).  The grid
// has one CTA per SM (G = min(SMs, units)), and CTA c owns the contiguous unit
// range [c*U/G, (c+1)*U/G), so every SM gets the same number of K-steps
// whatever the shape (no partial last wave).  A tile whose K range is cut
// between CTAs ("split") is summed by a fix-up: every CTA holding a piece
// writes its fp32 partial tile to the workspace and bumps the tile's counter;
// the CTA that brings the counter to the number of pieces adds all pieces in
// CTA order (= K order) and writes Y, then zeroes the counter.  No CTA waits
// for another, and the sum order is fixed by the schedule alone.
//
// Loads.  Measured on this GPU, a TMA copy costs the SM's copy engine about
// the same time whether it moves 2 KB or 16 KB, so small copies cap the
// bandwidth far below HBM.  Compressed W therefore arrives in super-steps of
// four K-steps (one 4-group chunk of every row): two 16 KB sign/mantissa
// boxes and one 16 KB palette box, all 128-byte swizzled.  Small or scattered
// data -- X tiles of up to 64 tokens, the exponents of raw groups, Huffman
// stream words -- go through the load/store path (cp.async, 16 bytes a lane).
//
// Roles (warps):
//   0      TMA producer: per super-step the compressed boxes (plain flavour:
//          one 16 KB W box per K-step).
//   1      MMA issuer and TMEM owner: 4 x tcgen05.mma (K = 16) per K-step into
//          one of two accumulators (double-buffered, so the epilogue of one
//          tile overlaps the MMAs of the next).
//   2      X producer: cp.async into the 128-byte-swizzled K-major layout for
//          up to 64 tokens, a TMA box per K-step for 128 and 256.
//   3-6    epilogue: TMEM -> registers -> Y (or a partial tile + fix-up);
//          it polls its accumulator barrier with sleeps in between, so that
//          a warp waiting a whole tile leaves the issue slots to the rebuild.
//   7-14   rebuild (palette, Huffman): all 8 warps work on the same K-step;
//          lane l of warp w rebuilds half h = (l >> 3) & 1 (32 weights) of
//          tile row 16w + 8(l >> 4) + (l & 7) into the 128-byte-swizzled
//          K-major BF16 W tile.  A quarter warp covers 8 consecutive rows, so
//          under the 128-byte swizzle every 16-byte shared-memory access of
//          it falls on its own bank group.
//   15-18  (palette; 15-16 Huffman) raw groups: per super-step these warps
//          find the raw (row, group) pairs of the 128 rows (each warp its
//          share of the rows), give each a slot in the stage (cp.async of its
//          64 exponents) and write a 128 x 4 table that tells the rebuild
//          where each group's exponents are (palette plane, a slot, or, when
//          the warp's slots run out, the raw plane in global memory).  One
//          warp alone took longer per super-step than the rebuild.
//   17     (Huffman) stream producer: per super-step it reads the 128 chunks'
//          start bits and copies each chunk's stream words (cp.async) into
//          one slot of a shared-memory ring, with a table of where they are
//          (a chunk that does not fit is read from global memory instead).
//   18-25  (Huffman) decoders: two groups of 4 warps take alternate
//          super-steps, one thread per tile row; a thread decodes its row's
//          chunk with the 12-bit multi-symbol table straight into the
//          super-step's palette area, in the stored 4-bit layout.
// Every wait is bounded; on time-out a role raises UW_DEVERR_TIMEOUT and sets
// the CTA's abort flag, which ends every other wait of the CTA; copies and
// MMAs in flight are waited for (bounded) before TMEM is freed.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kModePlain = 0, kModePal = 1, kModeHuff = 2;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kSuper = 4;               // K-steps per super-step (one 4-group stream chunk)
constexpr int kMaxSmem = 232448;        // 227 KB opt-in per CTA
constexpr int kFixedWarps = 7;          // producer, MMA, X producer, 4 epilogue warps
constexpr int kRebuildWarps = 8;
constexpr int kEpiWarp0 = 3;
constexpr int kFirstRebuildWarp = kFixedWarps;
constexpr int kRawWarp = kFixedWarps + kRebuildWarps;      // first raw-group warp (fused flavours)
constexpr int kRawWarpsPal = 4, kRawWarpsHuff = 2;          // raw-group warps per flavour
constexpr int kStreamWarp = kRawWarp + kRawWarpsHuff;      // Huffman flavour
constexpr int kFirstDecWarp = kStreamWarp + 1;
constexpr int kDecWarps = 8;            // two groups of 4
constexpr int kPlainThreads = kFixedWarps * 32;
constexpr int kPalThreads = (kFixedWarps + kRebuildWarps + kRawWarpsPal) * 32;
constexpr int kHuffThreads = (kFixedWarps + kRebuildWarps + kRawWarpsHuff + 1 + kDecWarps) * 32;

constexpr int kTileW = kBM * kBK * 2;   // BF16 W tile of one K-step (128 rows x 128 B)

// compressed super-step stage (fused flavours)
constexpr int kBox = kBM * 128;                  // one 128-row x 128-byte box
constexpr int kOffSmA = 0;                       // sign/mantissa, K-steps 0-1 of the super-step
constexpr int kOffSmB = kBox;                    //                K-steps 2-3
constexpr int kOffNib = 2 * kBox;                // 4-bit palette indices, K-steps 0-3
constexpr int kRawSlots = 64;                    // raw groups staged per super-step (16 per raw warp)
constexpr int kOffRaw = 3 * kBox;                // kRawSlots x 64 exponent bytes
constexpr int kOffTab = kOffRaw + kRawSlots * kGroup;   // uint32 [128 rows][4 K-steps]
constexpr int kCStage = kOffTab + kBM * kSuper * 4;
static_assert(kCStage % 1024 == 0, "stages keep 1024-byte alignment");
// raw table entry: 0 = palette; kTabSlot | slot = staged exponents;
// kTabRank | rank = the raw plane at 64 * rank (no slot left)
constexpr uint32_t kTabSlot = 0x80000000u, kTabRank = 0x40000000u;

// Huffman flavour
constexpr int kSlots = 3;                        // stream slots (super-steps staged ahead)
constexpr int kSlotBytes = 15 * 1024;            // stream bytes per slot: 128 chunks of ~100 B (2.6 bits/weight
                                                 // and the 16-byte granules around each chunk)
constexpr uint32_t kFromGlobal = 0x80000000u;    // chunk table flag: read the words from global memory
constexpr int kHuffLut = kLutEntries * 4;
constexpr int kHuffTable = kSlots * kBM * 16;    // per slot and row: uint4 {where, first word, start, end}
constexpr int kHuffRaw4 = kSlots * kBM;          // per slot and row: the chunk's raw-group bits
constexpr int kHuffBytes = kHuffLut + kSlots * kSlotBytes + kHuffTable + kHuffRaw4;
static_assert(kHuffBytes % 16 == 0, "Huffman area keeps 16-byte alignment");

struct SkArgs {
    int64_t m, n, k;
    int64_t units;            // tiles * S
    int S;                    // K-steps per tile
    int TB;                   // token blocks
    int G;                    // CTAs
    int dc, dw, dx;           // ring depths: compressed super-steps, W tiles, X tiles
    uint32_t debug_flags;
    uint64_t timeout_ns;
    const uint16_t *x;        // [m, k] BF16 (X by cp.async)
    float *y;
    uint32_t *counters;       // [tiles], zero between calls
    float *partial;           // [2G][BN][128]
    const uint32_t *flagbits;
    const uint32_t *rawbase;
    const uint8_t *rawexp;
    int64_t nflag;            // words of flagbits
    Palette16 pal;
    // Huffman flavour
    const uint32_t *stream;
    const uint32_t *chunk_off;
    const uint32_t *dlut;
    uint64_t stream_bits;
    uint64_t stream_words;    // words of the stream section (padded)
    uint64_t code_len;        // code length of palette index s in bits 4s..4s+3
    uint32_t *status;
};

// first unit of CTA c; the CTA holding unit u
__host__ __device__ __forceinline__ int64_t sk_unit0(int64_t c, int64_t units, int G) { return c * units / G; }
__host__ __device__ __forceinline__ int sk_cta_of(int64_t u, int64_t units, int G) {
    return int(((u + 1) * G - 1) / units);
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    // pointer arithmetic, not an integer round trip: the result stays
    // recognisably a shared-memory pointer, so accesses through it compile
    // to shared-memory loads and stores rather than generic ones
    return p + ((1024u - (smem_addr(p) & 1023u)) & 1023u);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v));
}

template <int BN>
struct SkCfg {
    static constexpr int kX = BN * kBK * 2;
    static constexpr bool kXByTma = BN >= 128;   // X boxes of 16 KB and more by TMA, smaller by cp.async
    static constexpr uint32_t kTmemCols = 2 * BN < 32 ? 32u : uint32_t(2 * BN);   // two accumulators
    static_assert(kX % 1024 == 0, "X stage keeps 1024-byte alignment");
    static_assert(2 * BN <= 512, "accumulators exceed TMEM");
};

// shared-memory bytes after the rings (and the Huffman area): barriers,
// TMEM slot, flags
__host__ __device__ constexpr int sk_tail(int dc, int dw, int dx) {
    return (2 * dc + 2 * dw + 2 * dx + 4 + 2 + 2 * kSlots + 1) * 8 + 16;
}

// The CTA's super-steps: for each tile of its unit range and each chunk
// index j (K-steps 4j..4j+3) touched there, the K-steps [lo, hi) the CTA
// owns.  Walked the same way by every role that works per super-step.
struct SuperSteps {
    int64_t u0, u1, t, t_last, rb;   // rb, tb: row block and token block of tile t
    int S, TB, tb, j, j_last, ka, kb;
    __device__ __forceinline__ void start_tile() {
        ka = t == u0 / S ? int(u0 - t * S) : 0;
        kb = t == t_last ? int(u1 - t * S) : S;
        j = ka / kSuper;
        j_last = (kb - 1) / kSuper;
    }
    __device__ __forceinline__ SuperSteps(int64_t u0_, int64_t u1_, int S_, int TB_)
        : u0(u0_), u1(u1_), S(S_), TB(TB_) {
        t = u0 / S;
        t_last = (u1 - 1) / S;
        rb = t / TB;
        tb = int(t - rb * TB);
        start_tile();
    }
    __device__ __forceinline__ bool valid() const { return u1 > u0 && t <= t_last; }
    __device__ __forceinline__ int lo() const { return max(ka, kSuper * j); }
    __device__ __forceinline__ int hi() const { return min(kb, kSuper * j + kSuper); }
    __device__ __forceinline__ void next() {
        if (++j > j_last) {
            ++t;
            if (++tb == TB) {
                tb = 0;
                ++rb;
            }
            if (t <= t_last) start_tile();
        }
    }
};

// Position in a ring of mbarrier-guarded stages: slot s, and the parity ph
// of the pass over the ring (flips each time s wraps).  Advanced without
// divisions; `wrapped` tells whether the slot was used before (its "empty"
// barrier must then be waited for with parity ph ^ 1).
struct Ring {
    int s = 0;
    uint32_t ph = 0;
    bool wrapped = false;
    __device__ __forceinline__ void next(int depth) {
        if (++s == depth) {
            s = 0;
            ph ^= 1u;
            wrapped = true;
        }
    }
};

// The CTA's units in order as (tile, K-step), advanced without divisions.
struct UnitWalk {
    int64_t t, rb;   // tile, its row block and token block
    int ks, S, TB, tb;
    __device__ __forceinline__ UnitWalk(int64_t u0, int S_, int TB_)
        : t(u0 / S_), ks(int(u0 % S_)), S(S_), TB(TB_) {
        rb = t / TB;
        tb = int(t - rb * TB);
    }
    __device__ __forceinline__ void next() {
        if (++ks == S) {
            ks = 0;
            ++t;
            if (++tb == TB) {
                tb = 0;
                ++rb;
            }
        }
    }
};

// Decode one group's 64 palette indices from bit p of a stream (words read
// through `word(i)`), handing each full word of 8 indices (natural order:
// index i in bits 4(i%8)..) to sink(w, word) for w = 0..7.  Never starts a
// step past `end`; false if a window has no valid code or the group does not
// complete.
template <class Src, class Sink>
__device__ __forceinline__ bool decode_group(const Src &word, uint32_t &p, uint32_t end, uint32_t lut,
                                             uint64_t code_len, const Sink &sink) {
    uint32_t lo = 0, na = 0, w = 0, rem4 = 256, err = 0;
    auto push = [&](uint32_t s, uint32_t nbits) {
        lo |= s << na;
        const uint32_t carry = __funnelshift_l(s, 0u, na);
        na += nbits;
        if (na >= 32) {
            sink(w++, lo);
            lo = carry;
            na -= 32;
        }
    };
    auto window = [&](uint32_t q) {
        const uint32_t wi = q >> 5;
        return __funnelshift_l(word(wi + 1), word(wi), q);
    };
    while (rem4 >= 40 && p <= end) {       // two whole table entries per window
        const uint32_t top = window(p);
        const uint32_t e1 = lds32(lut + ((top >> (32 - kLutBits)) << 2));
        const uint32_t b1 = lut_bits(e1);
        const uint32_t e2 = lds32(lut + (((top << b1) >> (32 - kLutBits)) << 2));
        p += b1 + lut_bits(e2);
        err |= e1 | e2;
        const uint32_t n1 = lut_symbits(e1), n2 = lut_symbits(e2);
        push(e1 & 0xFFFFFu, n1);
        push(e2 & 0xFFFFFu, n2);
        rem4 -= n1 + n2;
    }
    while (rem4 >= 20 && p <= end) {       // whole entries while at least 5 indices remain
        const uint32_t e = lds32(lut + ((window(p) >> (32 - kLutBits)) << 2));
        p += lut_bits(e);
        err |= e;
        const uint32_t n = lut_symbits(e);
        push(e & 0xFFFFFu, n);
        rem4 -= n;
    }
    while (rem4 > 0 && p <= end) {         // the last few one code at a time
        const uint32_t e = lds32(lut + ((window(p) >> (32 - kLutBits)) << 2));
        const uint32_t s = e & 15u;
        p += uint32_t(code_len >> (4 * s)) & 15u;
        err |= e;
        push(s, 4);
        rem4 -= 4;
    }
    return rem4 == 0 && !(err & kLutInvalid);
}

template <int MODE, int BN>
__device__ __forceinline__ void sk_body(const CUtensorMap *tmX, const CUtensorMap *tmA, const CUtensorMap *tmB,
                                        const SkArgs &a) {
    using C = SkCfg<BN>;
    constexpr bool FUSED = MODE != kModePlain;
    constexpr bool HUFF = MODE == kModeHuff;
    extern __shared__ uint8_t smem_dyn[];
    const int dc = FUSED ? a.dc : 0, dw = a.dw, dx = a.dx;
    uint8_t *wring = align1024(smem_dyn);
    uint8_t *xring = wring + size_t(dw) * kTileW;
    uint8_t *cring = xring + size_t(dx) * C::kX;
    uint8_t *huff = cring + size_t(dc) * kCStage;                  // Huffman area
    uint32_t *hlut = reinterpret_cast<uint32_t *>(huff);
    uint8_t *hslots = huff + kHuffLut;
    uint4 *htable = reinterpret_cast<uint4 *>(hslots + kSlots * kSlotBytes);   // [slot][128]
    uint8_t *hraw4 = reinterpret_cast<uint8_t *>(htable + kSlots * kBM);       // [slot][128]
    uint64_t *c_full = reinterpret_cast<uint64_t *>(huff + (HUFF ? kHuffBytes : 0));
    uint64_t *c_empty = c_full + dc;
    uint64_t *w_full = c_empty + dc;
    uint64_t *w_empty = w_full + dw;
    uint64_t *x_full = w_empty + dw;
    uint64_t *x_empty = x_full + dx;
    uint64_t *acc_full = x_empty + dx;      // [2]
    uint64_t *acc_empty = acc_full + 2;     // [2]
    uint64_t *never = acc_empty + 2;
    uint64_t *mma_done = never + 1;
    uint64_t *s_full = mma_done + 1;        // [kSlots] (Huffman)
    uint64_t *s_empty = s_full + kSlots;    // [kSlots]
    uint64_t *lut_full = s_empty + kSlots;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(lut_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *last_flag = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t T = a.timeout_ns;
    const int64_t u0 = sk_unit0(blockIdx.x, a.units, a.G), u1 = sk_unit0(int64_t(blockIdx.x) + 1, a.units, a.G);
    const int nu = int(u1 - u0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < dc; s++) {
            // the TMA producer, the 32 raw-group lanes once their table entries
            // are written and 32 once their copies landed, + the 4 decoder
            // warps of a group
            mbar_init(&c_full[s], HUFF ? 1 + 64 * kRawWarpsHuff + 4 : 1 + 64 * kRawWarpsPal);
            mbar_init(&c_empty[s], kRebuildWarps);
        }
        for (int s = 0; s < dw; s++) {
            mbar_init(&w_full[s], FUSED ? kRebuildWarps : 1);
            mbar_init(&w_empty[s], 1);
        }
        for (int s = 0; s < dx; s++) {
            mbar_init(&x_full[s], C::kXByTma ? 1 : 32);
            mbar_init(&x_empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(never, 1);
        mbar_init(mma_done, 1);
        if (HUFF) {
            for (int s = 0; s < kSlots; s++) {
                mbar_init(&s_full[s], 64);           // stream-producer lanes: table written, words landed
                mbar_init(&s_empty[s], 4);           // the 4 decoder warps of the group
            }
            mbar_init(lut_full, 1);
        }
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
        if (C::kXByTma) prefetch_tensormap(tmX);
        prefetch_tensormap(tmA);
        if (MODE == kModePal) prefetch_tensormap(tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto fail = [&](bool timed_out) {
        if (timed_out) flag_error(a.status, UW_DEVERR_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if constexpr (FUSED) {
            if (lane == 0) {
                int sidx = 0;
                Ring rc;
                for (SuperSteps ss(u0, u1, a.S, a.TB); ss.valid(); ss.next(), sidx++, rc.next(dc)) {
                    const int cs = rc.s;
                    if (rc.wrapped && !mbar_wait_or_abort(&c_empty[cs], rc.ph ^ 1u, T, abort_flag)) {
                        fail(!*abort_flag);
                        break;
                    }
                    if (*abort_flag) break;
                    uint8_t *st = cring + size_t(cs) * kCStage;
                    const int32_t n0 = int32_t(ss.rb * kBM);
                    // 4-byte elements: the chunk's sign/mantissa bytes start at element 64 j
                    // (two boxes of 128 bytes), its palette bytes at element 32 j
                    mbar_arrive_expect_tx(&c_full[cs], HUFF ? uint32_t(2 * kBox) : uint32_t(3 * kBox));
                    tma_load_2d(st + kOffSmA, tmA, 64 * ss.j, n0, &c_full[cs]);
                    tma_load_2d(st + kOffSmB, tmA, 64 * ss.j + 32, n0, &c_full[cs]);
                    if (!HUFF) tma_load_2d(st + kOffNib, tmB, 32 * ss.j, n0, &c_full[cs]);
                }
                // no copy may still be landing when the CTA exits (after an abort
                // another role's arrival may be missing: those waits run out, bounded)
                for (int i = max(0, sidx - dc); i < sidx; i++)
                    mbar_wait(&c_full[i % dc], uint32_t(i / dc) & 1u, *abort_flag ? T / 64 + 1 : T);
            }
        } else if (lane == 0) {
            int issued = 0;
            UnitWalk walk(u0, a.S, a.TB);
            Ring rw;
            for (int i = 0; i < nu; i++, walk.next(), rw.next(dw)) {
                const int64_t n0 = walk.rb * kBM;
                const int ks = walk.ks;
                const int s = rw.s;
                if (rw.wrapped && !mbar_wait_or_abort(&w_empty[s], rw.ph ^ 1u, T, abort_flag)) {
                    fail(!*abort_flag);
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(&w_full[s], uint32_t(kTileW));
                tma_load_2d(wring + size_t(s) * kTileW, tmA, ks * kBK, int32_t(n0), &w_full[s]);
                issued = i + 1;
            }
            for (int i = max(0, issued - dw); i < issued; i++)
                mbar_wait(&w_full[i % dw], uint32_t(i / dw) & 1u, T);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
            bool ok = true;
            if (a.debug_flags & UW_DEBUG_NEVER_ARRIVE) ok = mbar_wait_or_abort(never, 0, T, abort_flag);
            int seg = -1;
            int64_t tprev = -1;
            bool first = true;
            UnitWalk walk(u0, a.S, a.TB);
            Ring rx, rw;
            for (int i = 0; i < nu && ok; i++, walk.next(), rx.next(dx), rw.next(dw)) {
                const int64_t t = walk.t;
                if (t != tprev) {   // a new tile: close the previous accumulator, claim the next
                    if (seg >= 0) tc_commit(&acc_full[seg & 1]);
                    seg++;
                    tprev = t;
                    if (seg >= 2)
                        ok = mbar_wait_or_abort(&acc_empty[seg & 1], (uint32_t(seg >> 1) & 1u) ^ 1u, T, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    first = true;
                }
                const int xs = rx.s, ws = rw.s;
                ok = mbar_wait_or_abort(&x_full[xs], rx.ph, T, abort_flag) &&
                     mbar_wait_or_abort(&w_full[ws], rw.ph, T, abort_flag);
                if (!ok) break;
                // X copied through the load/store path: make it visible to the tensor core
                if (!C::kXByTma) fence_proxy_async_smem();
                tc_fence_after();
                const uint32_t sa = smem_addr(wring + size_t(ws) * kTileW);
                const uint32_t sb = smem_addr(xring + size_t(xs) * C::kX);
                const uint32_t d = tmem + uint32_t((seg & 1) * BN);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; kk++)
                    tc_mma_bf16(d, smem_desc_k128(sa + 32 * kk), smem_desc_k128(sb + 32 * kk), idesc,
                                (!first || kk) ? 1u : 0u);
                first = false;
                tc_commit(&w_empty[ws]);
                tc_commit(&x_empty[xs]);
            }
            if (ok) {
                if (seg >= 0) tc_commit(&acc_full[seg & 1]);
            } else {
                fail(!*abort_flag);
                // every MMA issued so far must finish before TMEM is freed
                tc_commit(mma_done);
                mbar_wait(mma_done, 0, T);
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------------------ X producer
        int issued = 0;
        UnitWalk walk(u0, a.S, a.TB);
        Ring rx;
        for (int i = 0; i < nu; i++, walk.next(), rx.next(dx)) {
            const int64_t m0 = int64_t(walk.tb) * BN;
            const int ks = walk.ks;
            const int s = rx.s;
            int stop = 0;
            if (lane == 0) {
                const bool ok = !rx.wrapped || mbar_wait_lazy(&x_empty[s], rx.ph ^ 1u, T, abort_flag, 64u);
                if (!ok) fail(!*abort_flag);
                stop = !ok || *abort_flag;
            }
            if (__shfl_sync(0xFFFFFFFFu, stop, 0)) break;
            uint8_t *xst = xring + size_t(s) * C::kX;
            if constexpr (C::kXByTma) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&x_full[s], uint32_t(C::kX));   // rows past m read the zero fill
                    tma_load_2d(xst, tmX, ks * kBK, int32_t(m0), &x_full[s]);
                }
            } else {
                // the 128-byte-swizzled K-major tile: 16-byte chunk c of token
                // row r at r * 128 + 16 * (c ^ (r & 7)); rows past m are zeros
#pragma unroll
                for (int idx = lane; idx < BN * 8; idx += 32) {
                    const int r = idx >> 3, c = idx & 7;
                    const int64_t tok = m0 + r;
                    const bool live = tok < a.m;
                    const uint16_t *src = a.x + (live ? tok * a.k + int64_t(ks) * kBK + c * 8 : 0);
                    cp_async16_zfill(xst + r * 128 + ((c ^ (r & 7)) << 4), src, live ? 16u : 0u);
                }
                cp_async_mbar_arrive_noinc(&x_full[s]);
            }
            issued = i + 1;
        }
        if constexpr (!C::kXByTma) cp_async_wait_all();
        if (lane == 0)
            for (int i = max(0, issued - dx); i < issued; i++)
                mbar_wait(&x_full[i % dx], uint32_t(i / dx) & 1u, T);
        __syncwarp();
    } else if (warp < kFirstRebuildWarp) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;               // TMEM lane quarter this warp may read
        const int r = q * 32 + lane;          // tile row
        const int64_t t_first = nu > 0 ? u0 / a.S : 0, t_last = nu > 0 ? (u1 - 1) / a.S : -1;
        int seg = -1;
        for (int64_t t = t_first; t <= t_last; t++) {
            seg++;
            const int b = seg & 1;
            const int64_t ka = t == t_first ? u0 - t * a.S : 0;
            const int64_t kb = t == t_last ? u1 - t * a.S : a.S;
            const bool split = ka != 0 || kb != a.S;
            const int slot = t == t_first ? 0 : 1;
            const bool ok = mbar_wait_lazy(&acc_full[b], uint32_t(seg >> 1) & 1u, T, abort_flag);
            // the four epilogue warps decide together, so that all of them
            // meet the same named barriers below
            if (named_bar_any(1, 128, !ok)) {
                if (!ok && lane == 0 && !*abort_flag) fail(true);
                break;
            }
            tc_fence_after();
            const int64_t n0 = (t / a.TB) * kBM, m0 = (t % a.TB) * BN;
            const int64_t row = n0 + r;
            float *pout = a.partial + (int64_t(2 * blockIdx.x + slot) * BN) * kBM + r;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + (uint32_t(q * 32) << 16) + uint32_t(b * BN + c0), v);
                tmem_ld_wait();
                if (split) {
#pragma unroll
                    for (int j = 0; j < 16; j++) pout[(c0 + j) * kBM] = __uint_as_float(v[j]);
                } else if (row < a.n) {
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const int64_t tok = m0 + c0 + j;
                        if (tok < a.m) a.y[tok * a.n + row] = __uint_as_float(v[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
            if (!split) continue;
            // fix-up: the last piece of the tile to arrive sums all pieces in CTA order
            __threadfence();
            named_bar_sync(1, 128);
            const int ca = sk_cta_of(t * a.S, a.units, a.G), cb = sk_cta_of(t * a.S + a.S - 1, a.units, a.G);
            if (warp == kEpiWarp0 && lane == 0) {
                const uint32_t old = atomicAdd(a.counters + t, 1u);
                *last_flag = old == uint32_t(cb - ca) ? 1 : 0;
            }
            named_bar_sync(1, 128);
            if (*last_flag) {
                __threadfence();
                // every row of every piece is read and then zeroed (rows past
                // n too, which the pieces hold as well), so that a completed
                // call leaves its whole scratch zero: a later call whose tile
                // counters lie where this call's partial tiles were finds them
                // at zero
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 8) {
                    float acc[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) acc[j] = 0.f;
                    for (int c = ca; c <= cb; c++) {
                        const int sl = (t == sk_unit0(c, a.units, a.G) / a.S) ? 0 : 1;
                        float *pin = a.partial + (int64_t(2 * c + sl) * BN + c0) * kBM + r;
                        float v[8];
#pragma unroll
                        for (int j = 0; j < 8; j++) v[j] = __ldcg(pin + j * kBM);
#pragma unroll
                        for (int j = 0; j < 8; j++) __stcg(pin + j * kBM, 0.f);
                        if (c == ca) {
#pragma unroll
                            for (int j = 0; j < 8; j++) acc[j] = v[j];
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; j++) acc[j] += v[j];
                        }
                    }
                    if (row < a.n) {
#pragma unroll
                        for (int j = 0; j < 8; j++) {
                            const int64_t tok = m0 + c0 + j;
                            if (tok < a.m) a.y[tok * a.n + row] = acc[j];
                        }
                    }
                }
                if (warp == kEpiWarp0 && lane == 0) a.counters[t] = 0u;
            }
        }
    } else if (warp < kRawWarp) {
        if constexpr (FUSED) {
            // -------------------------------------------------------- rebuild
            const int wi = warp - kFirstRebuildWarp;   // 0..7
            const int R = 16 * wi + 8 * (lane >> 4) + (lane & 7);   // tile row
            const int h = (lane >> 3) & 1;                          // half of the row's 64 weights
            const int sw = R & 7;                                   // 128-byte swizzle phase of the row
            const Palette16 P = a.pal;
            Ring rc, rw;
            bool ok = true;
            for (SuperSteps ss(u0, u1, a.S, a.TB); ss.valid() && ok; ss.next(), rc.next(dc)) {
                const int cs = rc.s;
                ok = mbar_wait_or_abort(&c_full[cs], rc.ph, T, abort_flag);
                if (__any_sync(0xFFFFFFFFu, !ok)) {
                    ok = false;
                    break;
                }
                const uint8_t *st = cring + size_t(cs) * kCStage;
                const uint32_t *tab = reinterpret_cast<const uint32_t *>(st + kOffTab);
                for (int ks = ss.lo(); ks < ss.hi(); ks++, rw.next(dw)) {
                    const int q = ks - kSuper * ss.j;
                    const int ws = rw.s;
                    if (rw.wrapped) ok = mbar_wait_or_abort(&w_empty[ws], rw.ph ^ 1u, T, abort_flag);
                    if (__any_sync(0xFFFFFFFFu, !ok)) {
                        ok = false;
                        break;
                    }
                    const uint8_t *smrow = st + (q >> 1) * kBox + R * 128;
                    const int c0 = (q & 1) * 4 + 2 * h;
                    const uint4 s0 = *reinterpret_cast<const uint4 *>(smrow + ((c0 ^ sw) << 4));
                    const uint4 s1 = *reinterpret_cast<const uint4 *>(smrow + (((c0 + 1) ^ sw) << 4));
                    const uint32_t e = tab[R * kSuper + q];
                    uint32_t rv[8];
                    if (e == 0u) {
                        const uint4 p = *reinterpret_cast<const uint4 *>(st + kOffNib + R * 128 +
                                                                         (((2 * q + h) ^ sw) << 4));
                        pal_rot(p.x, P, rv[0], rv[1]);
                        pal_rot(p.y, P, rv[2], rv[3]);
                        pal_rot(p.z, P, rv[4], rv[5]);
                        pal_rot(p.w, P, rv[6], rv[7]);
                    } else {
                        uint4 e0, e1;
                        if (e & kTabSlot) {
                            const uint8_t *rp = st + kOffRaw + (e & 0xFFFFu) * kGroup + h * 32;
                            e0 = *reinterpret_cast<const uint4 *>(rp);
                            e1 = *reinterpret_cast<const uint4 *>(rp + 16);
                        } else {   // no slot was left: the raw plane itself
                            const uint4 *rp = reinterpret_cast<const uint4 *>(
                                a.rawexp + uint64_t(e & ~kTabRank) * kGroup + h * 32);
                            e0 = __ldg(rp);
                            e1 = __ldg(rp + 1);
                        }
                        rv[0] = rot4(e0.x); rv[1] = rot4(e0.y); rv[2] = rot4(e0.z); rv[3] = rot4(e0.w);
                        rv[4] = rot4(e1.x); rv[5] = rot4(e1.y); rv[6] = rot4(e1.z); rv[7] = rot4(e1.w);
                    }
                    uint8_t *wrow = wring + size_t(ws) * kTileW + R * 128;
                    const int w0 = 4 * h;
                    *reinterpret_cast<uint4 *>(wrow + (((w0 + 0) ^ sw) << 4)) = join8(rv[0], rv[1], s0.x, s0.y);
                    *reinterpret_cast<uint4 *>(wrow + (((w0 + 1) ^ sw) << 4)) = join8(rv[2], rv[3], s0.z, s0.w);
                    *reinterpret_cast<uint4 *>(wrow + (((w0 + 2) ^ sw) << 4)) = join8(rv[4], rv[5], s1.x, s1.y);
                    *reinterpret_cast<uint4 *>(wrow + (((w0 + 3) ^ sw) << 4)) = join8(rv[6], rv[7], s1.z, s1.w);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&w_full[ws]);
                }
                if (!ok) break;
                // every K-step of the stage is rebuilt: hand it back to the producer
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[cs]);
            }
            if (!ok && lane == 0 && !*abort_flag) fail(true);
        }
    } else if (warp < kRawWarp + (HUFF ? kRawWarpsHuff : kRawWarpsPal)) {
        if constexpr (FUSED) {
            // -------------------------------------------------------- raw groups
            // RAWW warps split the tile's rows: lane l of raw warp v handles
            // rows r = 32 (MM v + m) + l, m < MM, and gives its raw groups
            // slots of the warp's own range.  A row's 4 groups of the chunk
            // are 4 consecutive bits of the raw bitmap (one funnel shift of the
            // two words around them), so rows without raw groups cost a few
            // instructions; a raw group's rank is the word's base plus the bits
            // below it.  The entries are computed before the stage is free.
            constexpr int RAWW = HUFF ? kRawWarpsHuff : kRawWarpsPal;
            constexpr int MM = 4 / RAWW;                      // rows per lane
            constexpr uint32_t kWarpSlots = kRawSlots / RAWW;
            const int v = warp - kRawWarp;
            const uint32_t slot_end = kWarpSlots * uint32_t(v + 1);
            const int64_t G64 = a.k / kGroup;     // groups per row
            int64_t wcur[MM];
            uint32_t blo[MM], bhi[MM], rlo[MM], rhi[MM];
#pragma unroll
            for (int mm = 0; mm < MM; mm++) wcur[mm] = -2;
            Ring rc;
            for (SuperSteps ss(u0, u1, a.S, a.TB); ss.valid(); ss.next(), rc.next(dc)) {
                const int cs = rc.s;
                const int64_t n0 = ss.rb * kBM;
                const int q0 = ss.lo() - kSuper * ss.j, q1 = ss.hi() - kSuper * ss.j;
                const uint32_t qmask = ((1u << q1) - 1u) & ~((1u << q0) - 1u);
                uint32_t rawbits = 0u, rank[4 * MM];
#pragma unroll
                for (int mm = 0; mm < MM; mm++) {
#pragma unroll
                    for (int q = 0; q < kSuper; q++) rank[4 * mm + q] = 0u;
                    const int64_t row = n0 + 32 * (MM * v + mm) + lane;
                    if (row >= a.n) continue;
                    const int64_t g0 = row * G64 + kSuper * ss.j;
                    const int64_t w0 = g0 >> 5;
                    if (w0 != wcur[mm]) {
                        if (w0 == wcur[mm] + 1) {
                            blo[mm] = bhi[mm];
                            rlo[mm] = rhi[mm];
                        } else {
                            blo[mm] = __ldg(a.flagbits + w0);
                            rlo[mm] = __ldg(a.rawbase + w0);
                        }
                        const bool more = w0 + 1 < a.nflag;
                        bhi[mm] = more ? __ldg(a.flagbits + w0 + 1) : 0u;
                        rhi[mm] = more ? __ldg(a.rawbase + w0 + 1) : 0u;
                        wcur[mm] = w0;
                    }
                    const uint32_t b0 = uint32_t(g0) & 31u;
                    const uint32_t bits = __funnelshift_r(blo[mm], bhi[mm], b0) & qmask;
                    if (bits) {
#pragma unroll
                        for (int q = 0; q < kSuper; q++) {
                            if (!((bits >> q) & 1u)) continue;
                            const uint32_t b = b0 + uint32_t(q);
                            rank[4 * mm + q] = b < 32u ? rlo[mm] + __popc(blo[mm] & ((1u << b) - 1u))
                                                       : rhi[mm] + __popc(bhi[mm] & ((1u << (b - 32u)) - 1u));
                        }
                        rawbits |= bits << (4 * mm);
                    }
                }
                // slots: an exclusive prefix sum of the lanes' raw counts
                const uint32_t cnt = __popc(rawbits);
                uint32_t scan = cnt;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, scan, d);
                    if (lane >= d) scan += v;
                }
                uint32_t slot = kWarpSlots * uint32_t(v) + scan - cnt;
                int stop = 0;
                if (lane == 0) {
                    bool ok = true;
                    if (rc.wrapped) ok = mbar_wait_or_abort(&c_empty[cs], rc.ph ^ 1u, T, abort_flag);
                    if (!ok) fail(!*abort_flag);
                    stop = !ok || *abort_flag;
                }
                if (__shfl_sync(0xFFFFFFFFu, stop, 0)) break;
                uint8_t *st = cring + size_t(cs) * kCStage;
                uint32_t *tab = reinterpret_cast<uint32_t *>(st + kOffTab);
#pragma unroll
                for (int mm = 0; mm < MM; mm++) {
                    const int r = 32 * (MM * v + mm) + lane;
#pragma unroll
                    for (int q = 0; q < kSuper; q++) {
                        uint32_t e = 0u;
                        if ((rawbits >> (4 * mm + q)) & 1u) {
                            if (slot < slot_end) {
                                const uint8_t *src = a.rawexp + uint64_t(rank[4 * mm + q]) * kGroup;
                                uint8_t *dst = st + kOffRaw + slot * kGroup;
#pragma unroll
                                for (int c = 0; c < 4; c++) cp_async16(dst + 16 * c, src + 16 * c);
                                e = kTabSlot | slot;
                            } else {
                                e = kTabRank | rank[4 * mm + q];
                            }
                            slot++;
                        }
                        tab[r * kSuper + q] = e;
                    }
                }
                mbar_arrive(&c_full[cs]);                 // this lane's table entries are written
                cp_async_mbar_arrive_noinc(&c_full[cs]);  // ... and, once landed, its raw copies
            }
            cp_async_wait_all();
            __syncwarp();
        }
    } else if (warp == kStreamWarp) {
        if constexpr (HUFF) {
            // -------------------------------------------------------- stream producer
            if (lane == 0) {   // the decode table, once
                mbar_arrive_expect_tx(lut_full, uint32_t(kHuffLut));
                bulk_g2s(hlut, a.dlut, kHuffLut, lut_full);
            }
            const int64_t G4 = a.k / (kSuper * kGroup);   // chunks per row
            int sidx = 0;
            Ring rs;
            for (SuperSteps ss(u0, u1, a.S, a.TB); ss.valid(); ss.next(), sidx++, rs.next(kSlots)) {
                const int slot = rs.s;
                int stop = 0;
                if (lane == 0) {
                    const bool ok = !rs.wrapped || mbar_wait_or_abort(&s_empty[slot], rs.ph ^ 1u, T, abort_flag);
                    if (!ok) fail(!*abort_flag);
                    stop = !ok || *abort_flag;
                }
                if (__shfl_sync(0xFFFFFFFFu, stop, 0)) break;
                const int64_t n0 = ss.rb * kBM;
                uint32_t start[4], end[4], wfirst[4], bytes[4], raw4[4];
#pragma unroll
                for (int mm = 0; mm < 4; mm++) {
                    const int64_t row = n0 + lane + 32 * mm;
                    start[mm] = end[mm] = wfirst[mm] = bytes[mm] = raw4[mm] = 0u;
                    if (row < a.n) {
                        const int64_t c = row * G4 + ss.j;
                        start[mm] = __ldg(a.chunk_off + c);
                        end[mm] = __ldg(a.chunk_off + c + 1);
                        const int64_t g = int64_t(kSuper) * c;
                        raw4[mm] = (__ldg(a.flagbits + (g >> 5)) >> (uint32_t(g) & 31u)) & 15u;
                    }
                }
                // words [wfirst, wlast) hold bits [start, end) and the two words a
                // window at `end` reads; whole 16-byte granules
                uint32_t incl = 0;
#pragma unroll
                for (int mm = 0; mm < 4; mm++) {
                    const bool sane = start[mm] <= end[mm] && uint64_t(end[mm]) <= a.stream_bits;
                    if (sane && end[mm] > start[mm]) {
                        wfirst[mm] = (start[mm] >> 5) & ~3u;
                        const uint32_t wlast = (end[mm] >> 5) + 2u;   // a window at bit p <= end reads words p/32, p/32 + 1
                        const uint32_t nw = (wlast - wfirst[mm] + 3u) & ~3u;
                        // words past the stream section are never staged (those chunks read global memory)
                        bytes[mm] = uint64_t(wfirst[mm]) + nw <= a.stream_words ? nw * 4u : 0u;
                    }
                    incl += bytes[mm];
                }
                // offsets: an exclusive prefix sum over the lanes, then the lane's rows in order
                uint32_t scan = incl;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, scan, d);
                    if (lane >= d) scan += v;
                }
                uint32_t off = scan - incl;
                uint4 *tab = htable + slot * kBM;
                uint8_t *sbase = hslots + slot * kSlotBytes;
#pragma unroll
                for (int mm = 0; mm < 4; mm++) {
                    const int r = lane + 32 * mm;
                    const bool fits = bytes[mm] > 0 && off + bytes[mm] <= uint32_t(kSlotBytes);
                    tab[r] = make_uint4(fits ? off : kFromGlobal, wfirst[mm], start[mm], end[mm]);
                    hraw4[slot * kBM + r] = uint8_t(raw4[mm]);
                    if (fits)
                        for (uint32_t b = 0; b < bytes[mm]; b += 16)
                            cp_async16(sbase + off + b, reinterpret_cast<const uint8_t *>(a.stream + wfirst[mm]) + b);
                    off += bytes[mm];
                }
                mbar_arrive(&s_full[slot]);                 // this lane's table entries are written
                cp_async_mbar_arrive_noinc(&s_full[slot]);  // ... and, once landed, its stream words
            }
            cp_async_wait_all();
            // no copy may still be landing when the CTA exits
            if (lane == 0) {
                for (int i = max(0, sidx - kSlots); i < sidx; i++)
                    mbar_wait(&s_full[i % kSlots], uint32_t(i / kSlots) & 1u, T);
                mbar_wait(lut_full, 0, T);
            }
            __syncwarp();
        }
    } else {
        if constexpr (HUFF) {
            // -------------------------------------------------------- decoders
            const int dt = threadIdx.x - 32 * kFirstDecWarp;   // 0..255
            const int grp = dt >> 7, r = dt & 127;
            const uint32_t lut = smem_addr(hlut);
            const int sw = r & 7;
            bool ok = mbar_wait_or_abort(lut_full, 0, T, abort_flag);
            int sidx = 0;
            Ring rs, rc;
            for (SuperSteps ss(u0, u1, a.S, a.TB); ss.valid() && ok;
                 ss.next(), sidx++, rs.next(kSlots), rc.next(dc)) {
                if ((sidx & 1) != grp) continue;
                const int slot = rs.s, cs = rc.s;
                ok = mbar_wait_or_abort(&s_full[slot], rs.ph, T, abort_flag) &&
                     (!rc.wrapped || mbar_wait_or_abort(&c_empty[cs], rc.ph ^ 1u, T, abort_flag));
                if (__any_sync(0xFFFFFFFFu, !ok)) {
                    ok = false;
                    break;
                }
                const uint4 e = htable[slot * kBM + r];
                const uint32_t raw4 = hraw4[slot * kBM + r];
                const int64_t row = ss.rb * kBM + r;
                uint32_t p = e.z;
                const uint32_t end = e.w;
                bool good = e.z <= e.w && uint64_t(e.w) <= a.stream_bits;
                const uint32_t sbase = smem_addr(hslots + slot * kSlotBytes) + (e.x & ~kFromGlobal);
                const uint32_t wfirst = e.y;
                const auto staged = [&](uint32_t wi) { return lds32(sbase + 4u * (wi - wfirst)); };
                const auto global = [&](uint32_t wi) { return __ldg(a.stream + wi); };
                const uint32_t nib = smem_addr(cring + size_t(cs) * kCStage + kOffNib) + uint32_t(r * 128);
                if (row < a.n) {
#pragma unroll 1
                    for (int q = 0; q < kSuper; q++) {
                        if ((raw4 >> q) & 1u) continue;   // no codes in the stream for a raw group
                        // word w of group q: weights 8w..8w+7 of K-step q, in the
                        // stored 4-bit layout at the swizzled palette position
                        const auto sink = [&](uint32_t w, uint32_t v) {
                            sts32(nib + ((((2 * q) + (w >> 2)) ^ sw) << 4) + 4u * (w & 3u), natural_to_pal(v));
                        };
                        if (good)
                            good = (e.x & kFromGlobal) ? decode_group(global, p, end, lut, a.code_len, sink)
                                                       : decode_group(staged, p, end, lut, a.code_len, sink);
                    }
                    // a chunk must decode cleanly and end exactly where the next starts
                    if (!good || p != end) flag_error(a.status, UW_DEVERR_CORRUPT);
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&c_full[cs]);
                    mbar_arrive(&s_empty[slot]);
                }
            }
            if (!ok && lane == 0 && !*abort_flag) fail(true);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BN>
__global__ void __launch_bounds__(kPalThreads, 1)
    k_gemm_sk_fused(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmSM,
                    const __grid_constant__ CUtensorMap tmPL, const SkArgs a) {
    sk_body<kModePal, BN>(&tmX, &tmSM, &tmPL, a);
}

template <int BN>
__global__ void __launch_bounds__(kHuffThreads, 1)
    k_gemm_sk_huff(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmSM,
                   const SkArgs a) {
    sk_body<kModeHuff, BN>(&tmX, &tmSM, &tmSM, a);
}

template <int BN>
__global__ void __launch_bounds__(kPlainThreads, 1)
    k_gemm_sk_plain(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const SkArgs a) {
    sk_body<kModePlain, BN>(&tmX, &tmW, &tmW, a);
}

// ============================================================== host side

bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ring depths: compressed super-steps (2 when it fits), W tiles and X tiles
// per token tile; the plan's `stages` caps the compressed ring (fused) or the
// W ring (plain)
struct Depths {
    int dc, dw, dx;
};
Depths depths(int mode, int bn, int stages) {
    const int kx = bn * kBK * 2;
    Depths d{};
    if (mode == kModePlain) {
        d.dc = 0;
        d.dx = bn <= 64 ? 8 : (bn == 128 ? 4 : 3);
        const int room = kMaxSmem - 1024 - d.dx * kx - sk_tail(0, 8, d.dx);
        d.dw = std::min(8, room / kTileW);
        if (stages > 0) d.dw = std::min(d.dw, std::max(2, stages));
        return d;
    }
    const int huff = mode == kModeHuff ? kHuffBytes : 0;
    d.dc = 2;
    d.dw = bn <= 64 && mode == kModePal ? 3 : 2;
    int room = kMaxSmem - 1024 - d.dc * kCStage - huff - d.dw * kTileW - sk_tail(3, d.dw, 8);
    d.dx = std::min(8, room / kx);
    if (d.dx > 2) {   // a third compressed stage when X keeps at least 2 stages
        room -= kCStage;
        if (room / kx >= 2) {
            d.dc = 3;
            d.dx = std::min(8, room / kx);
        }
    }
    if (stages > 0) d.dc = std::min(d.dc, std::max(2, stages));
    return d;
}

size_t smem_bytes(int mode, int bn, const Depths &d) {
    const bool fused = mode != kModePlain;
    return size_t(d.dw) * kTileW + size_t(d.dx) * bn * kBK * 2 + (fused ? size_t(d.dc) * kCStage : 0) +
           (mode == kModeHuff ? size_t(kHuffBytes) : 0) + 1024 + sk_tail(fused ? d.dc : 0, d.dw, d.dx);
}

int device_sms() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
            cudaGetLastError();
            return 148;
        }
        cache[dev] = sms;
    }
    return cache[dev];
}

// Once per (kernel, device): the shared-memory opt-in, and a check that one
// CTA fits an SM and that co-resident CTAs would fit the 512 TMEM columns
// (tcgen05.alloc would block).  Launches use at least half the SM's shared
// memory, so the occupancy found for that size holds for every launch.
template <class K>
cudaError_t prepare(K kern, int threads, uint32_t tmem_cols, int (&ready)[64]) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (ready[dev]) return cudaSuccess;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, size_t(kMaxSmem / 2 + 1024));
    if (err != cudaSuccess) return err;
    if (per_sm < 1 || per_sm * int(tmem_cols) > 512) return cudaErrorInvalidConfiguration;
    ready[dev] = 1;
    return cudaSuccess;
}

template <int BN>
cudaError_t launch_bn(const TcLaunch &p, cudaStream_t stream) {
    using C = SkCfg<BN>;
    const int mode = p.w_bf16 ? kModePlain : (p.huffman ? kModeHuff : kModePal);
    const SkGeometry g = sk_geometry(p.m, p.n, p.k, BN);
    if (g.G <= 0) return cudaErrorInvalidValue;
    if (!p.sk_counters || !p.partial) return cudaErrorInvalidValue;
    const Depths d = depths(mode, BN, p.stages);
    if ((mode != kModePlain && d.dc < 2) || d.dw < 2 || d.dx < 2) return cudaErrorInvalidValue;
    size_t smem = smem_bytes(mode, BN, d);
    smem = std::max(smem, size_t(kMaxSmem / 2 + 1024));   // one CTA per SM
    if (smem > size_t(kMaxSmem)) return cudaErrorInvalidValue;

    SkArgs a{};
    a.m = p.m;
    a.n = p.n;
    a.k = p.k;
    a.units = g.units;
    a.S = g.S;
    a.TB = g.TB;
    a.G = g.G;
    a.dc = d.dc;
    a.dw = d.dw;
    a.dx = d.dx;
    a.debug_flags = p.debug_flags;
    a.timeout_ns = p.timeout_ns;
    a.x = p.x;
    a.y = p.y;
    a.counters = p.sk_counters;
    a.partial = p.partial;
    a.status = p.dev_status;

    CUtensorMap mx, ma, mb;
    std::memset(&mx, 0, sizeof(mx));
    if (C::kXByTma && !make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, uint64_t(p.k), uint64_t(p.m),
                                uint64_t(p.k) * 2, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    cudaError_t err;
    if (mode != kModePlain) {
        a.flagbits = p.w->flagbits;
        a.rawbase = p.w->rawbase;
        a.rawexp = p.w->rawexp;
        a.nflag = (p.n * (p.k / kGroup) + 31) / 32;
        a.pal = make_palette16(p.w->palette);
        // sign/mantissa boxes of 128 bytes (two K-steps) x 128 rows, as
        // 4-byte elements (the copy engine moves the same bytes in fewer elements)
        if (!make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.w->sm, uint64_t(p.k / 4), uint64_t(p.n), uint64_t(p.k),
                      32, kBM, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    if (mode == kModePal) {
        // palette boxes of 128 bytes (four K-steps) x 128 rows, 4-byte elements
        if (!make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT32, p.pal, uint64_t(p.k / 8), uint64_t(p.n), uint64_t(p.k / 2),
                      32, kBM, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        static int ready[64] = {0};
        err = prepare(k_gemm_sk_fused<BN>, kPalThreads, C::kTmemCols, ready);
        if (err != cudaSuccess) return err;
        k_gemm_sk_fused<BN><<<unsigned(g.G), kPalThreads, smem, stream>>>(mx, ma, mb, a);
    } else if (mode == kModeHuff) {
        // chunks of 4 groups must not straddle rows; the decoders' table
        // needs the Huffman sections
        if (p.k % (kSuper * kGroup) || !p.w->stream || !p.w->chunk_off || !p.w->dlut) return cudaErrorInvalidValue;
        a.stream = p.w->stream;
        a.chunk_off = p.w->chunk_off;
        a.dlut = p.w->dlut;
        a.stream_bits = p.w->stream_bits;
        a.stream_words = p.w->stream_words;
        a.code_len = 0;
        for (int i = 0; i < 16; i++) a.code_len |= uint64_t(p.w->code_len[i] & 15u) << (4 * i);
        static int ready[64] = {0};
        err = prepare(k_gemm_sk_huff<BN>, kHuffThreads, C::kTmemCols, ready);
        if (err != cudaSuccess) return err;
        k_gemm_sk_huff<BN><<<unsigned(g.G), kHuffThreads, smem, stream>>>(mx, ma, a);
    } else {
        if (!make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.w_bf16, uint64_t(p.k), uint64_t(p.n),
                      uint64_t(p.k) * 2, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        static int ready[64] = {0};
        err = prepare(k_gemm_sk_plain<BN>, kPlainThreads, C::kTmemCols, ready);
        if (err != cudaSuccess) return err;
        k_gemm_sk_plain<BN><<<unsigned(g.G), kPlainThreads, smem, stream>>>(mx, ma, a);
    }
    return cudaGetLastError();
}

}  // namespace

int sm_count() { return device_sms(); }

SkGeometry sk_geometry(int64_t m, int64_t n, int64_t k, int bn) {
    SkGeometry g{};
    if (m <= 0 || n <= 0 || k <= 0 || bn <= 0) return g;
    g.S = int(k / kBK);
    g.TB = int((m + bn - 1) / bn);
    g.RB = (n + kBM - 1) / kBM;
    g.tiles = g.RB * g.TB;
    g.units = g.tiles * g.S;
    g.G = int(std::min<int64_t>(device_sms(), g.units));
    g.counter_bytes = align_up(uint64_t(g.tiles) * 4, 256);
    g.partial_bytes = align_up(uint64_t(2 * g.G) * uint64_t(bn) * kBM * 4, 256);
    return g;
}

int sk_huffman_max_bn() {
    // the largest token tile whose Huffman kernel fits shared memory
    for (int bn : {256, 128, 64, 32, 16}) {
        const Depths d = depths(kModeHuff, bn, 0);
        if (d.dc >= 2 && d.dx >= 2 && smem_bytes(kModeHuff, bn, d) <= size_t(kMaxSmem)) return bn;
    }
    return 0;
}

cudaError_t launch_gemm_sk(const TcLaunch &p, cudaStream_t stream) {
    if (p.huffman && p.bn > sk_huffman_max_bn()) return cudaErrorInvalidValue;
    switch (p.bn) {
        case 16: return launch_bn<16>(p, stream);
        case 32: return launch_bn<32>(p, stream);
        case 64: return launch_bn<64>(p, stream);
        case 128: return launch_bn<128>(p, stream);
        case 256: return launch_bn<256>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace uw
