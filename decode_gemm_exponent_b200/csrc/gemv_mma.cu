// gemv_mma.cu -- skinny matmul Y = X * W^T for m <= 16 tokens on the warp-level
// tensor-core MMA, with W rebuilt in registers (Unweight page §七: the
// reconstructive matmul; §五: decompressed weights never go back to HBM).
//
// At m <= 16 the job is an HBM stream of the compressed planes, and what
// decides whether it keeps up with HBM is the instruction count per weight.
// A CUDA-core FMA costs one instruction per weight and token (plus widening
// the BF16 operands), so it stops being memory-bound at a few tokens.  Here
// each lane rebuilds its weights into BF16 pairs that are exactly the A
// fragment of mma.m16n8k16 (W rows are the MMA's M), X pairs straight from
// their 16-byte loads are the B fragment (tokens are the N), so the dot
// products cost 4 MMA instructions per 64-weight chunk of 16 rows per 8
// tokens, and the weights go from the load registers to the tensor core
// without a shared-memory round trip.
//
// Work split: a warp tile is 16 consecutive rows of W; a CTA of S warps owns
// one tile and splits its K into S contiguous slices of steps.  A step covers
// 64*Q weights along K (Q = 1 or 2, the plan's width): lane (g, c) = (lane / 4,
// lane % 4) loads weights [16Qc, 16Qc + 16Q) of the step for rows g and g + 8
// (4 lanes cover a row's 64*Q sign/mantissa bytes).  The step's K positions
// map onto 4*Q MMA K-steps of 16 as: K-step j, thread c, MMA K slots {2c,
// 2c+1, 2c+8, 2c+9} <- weights 16Qc + 4j + {0, 1, 2, 3}; the X fragment uses
// the same map, so every product is formed exactly once.  Lanes whose token
// is >= m load a valid X row anyway: it only feeds output columns that are not
// stored.  Each warp keeps the loads of the next steps in flight in a register
// ring (3 steps for Q = 1, 2 for Q = 2), and prefetches each ring slot's X rows
// into L1 when it issues the slot's loads.  The raw-group bitmap words of the
// tile's rows and their prefix counts are staged in shared memory; each lane
// keeps a 64-group window of its two rows' raw bits in registers, so a raw
// group's exponents are fetched together with the step's other loads.
// The MMA K-steps alternate between two accumulators (independent MMA
// chains), added at the end, and the S slice results are summed in ascending
// slice order through shared memory.  The fused and plain variants share all
// of this but the loader, so their outputs are bit-identical.
// The batched kernel runs the same tile body for many matrices in one launch
// (the routed experts of a mixture-of-experts layer, Unweight page §十一),
// so each matrix's output is the single kernel's, bit for bit.
#include <algorithm>

#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kTileRows = 16;
constexpr int kChunk = 64;
constexpr int kMaxSlices = 8;
constexpr int kMaxSmem = 48 * 1024;    // dynamic shared memory without opt-in

struct MmaArgs {
    const uint16_t *x;         // [m, k] BF16
    const uint16_t *w_bf16;    // plain: [n, k] BF16
    const uint8_t *sm;         // fused: sign/mantissa plane
    const uint32_t *pal;       // fused: 4-bit plane as words (8 weights each)
    const uint32_t *flagbits;
    const uint32_t *rawbase;
    const uint8_t *rawexp;
    Palette16 palette;
    int64_t n, k;
    int m;
    int flag_words;            // fused: bitmap words staged per CTA (16 rows)
    int w_stable;              // fused: planes no kernel writes (read before pdl_wait)
    float *y;                  // [m, n]
};

// One lane's 16*Q weights of one chunk (64*Q weights along K) of one row, as
// loaded.  Plain: the weights, 16*Q BF16 in a[] then b[].  Fused: sign/mantissa
// bytes in a[]; the palette words (2*Q of them) in b[0], or the raw
// exponents (16*Q bytes) in b[].
template <int Q>
struct Half {
    uint4 a[Q];
    uint4 b[Q];
};

__device__ __forceinline__ void prefetch_l1(const void *p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// raw bits of the 64 groups starting at global group `gfirst` (bit i = group
// gfirst + i) from the staged bitmap (word index relative to `wbase`); words
// past the staged ones read as 0, and bits beyond the caller's chunks are
// never used
__device__ __forceinline__ uint64_t raw_window(const uint32_t *sflags, int nwords, int64_t wbase, int64_t gfirst) {
    const int64_t w = (gfirst >> 5) - wbase;
    const uint32_t sh = uint32_t(gfirst) & 31u;
    uint32_t v[3];
#pragma unroll
    for (int q = 0; q < 3; q++) v[q] = (w + q < nwords) ? sflags[w + q] : 0u;
    const uint64_t lo = (uint64_t(v[1]) << 32 | v[0]) >> sh;
    const uint64_t hi = uint64_t(v[2]) << (64 - sh);   // sh = 0: shift by 64 is avoided below
    return sh ? (lo | hi) : (uint64_t(v[1]) << 32 | v[0]);
}

// loads of one lane's weights of one chunk of one row; `g` is the lane's
// group, `goff` the lane's byte offset inside that group's 64 raw exponents
template <bool PAL, int Q>
__device__ __forceinline__ Half<Q> load_half(const MmaArgs &a, const uint8_t *smp, const uint32_t *palp,
                                             const uint16_t *wp, bool raw, int64_t g, int goff,
                                             const uint32_t *sflags, const uint32_t *srb, int64_t wbase) {
    Half<Q> h;
    if (!PAL) {
        const uint4 *u = reinterpret_cast<const uint4 *>(wp);
#pragma unroll
        for (int i = 0; i < Q; i++) {
            h.a[i] = __ldcs(u + i);
            h.b[i] = __ldcs(u + Q + i);
        }
    } else {
#pragma unroll
        for (int i = 0; i < Q; i++) h.a[i] = __ldcs(reinterpret_cast<const uint4 *>(smp) + i);
        if (raw) {
            const int wi = int((g >> 5) - wbase);
            const uint32_t rank = srb[wi] + __popc(sflags[wi] & ((1u << (uint32_t(g) & 31u)) - 1u));
            const uint4 *e = reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(rank) * kGroup + goff);
#pragma unroll
            for (int i = 0; i < Q; i++) h.b[i] = __ldcs(e + i);
        } else if (Q == 1) {
            const uint2 p = __ldcs(reinterpret_cast<const uint2 *>(palp));
            h.b[0] = make_uint4(p.x, p.y, 0u, 0u);
        } else {
            h.b[0] = __ldcs(reinterpret_cast<const uint4 *>(palp));
#pragma unroll
            for (int i = 1; i < Q; i++) h.b[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    return h;
}

__device__ __forceinline__ uint32_t word(const uint4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// Half -> 8*Q BF16 pairs (weights 2i, 2i+1 in pair i)
template <bool PAL, int Q>
__device__ __forceinline__ void rebuild(const Half<Q> &h, bool raw, const Palette16 &P, uint32_t (&w)[8 * Q]) {
    if (!PAL) {
#pragma unroll
        for (int i = 0; i < 4 * Q; i++) w[i] = word(h.a[i / 4], i % 4);
#pragma unroll
        for (int i = 0; i < 4 * Q; i++) w[4 * Q + i] = word(h.b[i / 4], i % 4);
    } else {
        uint32_t r[4 * Q];   // rotated exponent bytes, 4 weights per word
        if (raw) {
#pragma unroll
            for (int i = 0; i < 4 * Q; i++) r[i] = rot4(word(h.b[i / 4], i % 4));
        } else {
#pragma unroll
            for (int i = 0; i < 2 * Q; i++) pal_rot(word(h.b[0], i), P, r[2 * i], r[2 * i + 1]);
        }
#pragma unroll
        for (int i = 0; i < 4 * Q; i++) join4(r[i], word(h.a[i / 4], i % 4), w[2 * i], w[2 * i + 1]);
    }
}

// One CTA's work: the 16-row tile `tile` of the matmul `a`.
template <bool PAL, int NT, int Q>   // NT: 8-token tiles (1: m <= 8, 2: m <= 16); Q: 16*Q weights per lane and row
__device__ __forceinline__ void gemv_mma_tile(const MmaArgs &a, int64_t tile) {
    constexpr int kCh = kChunk * Q;               // weights per chunk along K
    constexpr int kWl = 16 * Q;                   // weights per lane and row in a chunk
    constexpr int kStages = Q == 1 ? 3 : 2;       // chunks of loads in flight per warp
    constexpr int kWin = 64 / Q;                  // chunks per 64-group window of raw bits
    // dynamic shared memory: [bitmap words][prefix counts] (fused), then the
    // slice results [slices][32][8 * NT] (slices > 1)
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *sflags = smem, *srb = smem + a.flag_words;
    float *red = reinterpret_cast<float *>(smem + 2 * a.flag_words);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slices = blockDim.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    // the next kernel on the stream may be scheduled now; with planes no
    // kernel writes, the raw bitmap and the first loads of W are issued
    // before waiting for the previous kernel (X, Y and everything else after)
    pdl_trigger();
    if (!a.w_stable) pdl_wait();
    const int64_t row0 = tile * kTileRows;
    const int64_t ra = row0 + g, rb = ra + 8;       // this lane's two rows
    const int64_t gpr = a.k / kChunk;               // groups per row
    const int64_t cpr = a.k / kCh;                  // chunks per row
    const int64_t wbase = (row0 * gpr) >> 5;        // first bitmap word of the tile's rows
    int nwords = 0;
    if (PAL) {
        const int64_t wlast = ((row0 + kTileRows) * gpr - 1) >> 5;
        nwords = int(wlast - wbase + 1);            // <= flag_words
        for (int i = threadIdx.x; i < nwords; i += blockDim.x) {
            sflags[i] = __ldg(a.flagbits + wbase + i);
            srb[i] = __ldg(a.rawbase + wbase + i);
        }
        __syncthreads();
    }
    const Palette16 P = a.palette;

    // this warp's chunks [ch0, ch0 + nch)
    const int64_t ch0 = cpr * warp / slices;
    const int nch = int(cpr * (warp + 1) / slices - ch0);

    // per-lane streams, advanced one chunk at a time
    const int64_t ea = ra * a.k + ch0 * kCh + c * kWl, eb = ea + 8 * a.k;
    const uint8_t *sma = a.sm + ea, *smb = a.sm + eb;
    const uint32_t *pala = a.pal + ea / 8, *palb = a.pal + eb / 8;
    const uint16_t *wa = a.w_bf16 + ea, *wb = a.w_bf16 + eb;
    const int coff = (c * kWl) / kChunk;                      // group of the lane inside a chunk
    const int goff = (c * kWl) % kChunk;                      // the lane's offset inside its group
    const int64_t ga = ra * gpr + ch0 * Q, gb = ga + 8 * gpr; // first group of the slice, rows g and g + 8
    // X rows of this lane's tokens (clamped: columns >= m are not stored)
    const uint16_t *x0 = a.x + int64_t(min(g, a.m - 1)) * a.k + ch0 * kCh + c * kWl;
    const uint16_t *x1 = a.x + int64_t(min(g + 8, a.m - 1)) * a.k + ch0 * kCh + c * kWl;

    uint64_t rawa = 0, rawb = 0;
    if (PAL) {
        rawa = raw_window(sflags, nwords, wbase, ga);
        rawb = raw_window(sflags, nwords, wbase, gb);
    }

    float d0[NT][4], d1[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int q = 0; q < 4; q++) d0[t][q] = d1[t][q] = 0.f;

    Half<Q> ha[kStages], hb[kStages];
    bool fa[kStages], fb[kStages];
    auto issue = [&](int i, int s, bool x_prefetch = true) {   // loads of chunk i into ring slot s
        const int bit = ((i * Q) & 63) + coff;
        fa[s] = PAL && ((rawa >> bit) & 1u);
        fb[s] = PAL && ((rawb >> bit) & 1u);
        ha[s] = load_half<PAL, Q>(a, sma + int64_t(i) * kCh, pala + i * (kCh / 8), wa + int64_t(i) * kCh, fa[s],
                                  ga + i * Q + coff, goff, sflags, srb, wbase);
        hb[s] = load_half<PAL, Q>(a, smb + int64_t(i) * kCh, palb + i * (kCh / 8), wb + int64_t(i) * kCh, fb[s],
                                  gb + i * Q + coff, goff, sflags, srb, wbase);
        // the chunk's X rows into L1 now, so that the MMA steps do not wait on L2
        if (x_prefetch) {
            prefetch_l1(x0 + int64_t(i) * kCh);
            if (NT == 2) prefetch_l1(x1 + int64_t(i) * kCh);
        }
    };
    auto mma_tile = [&](int t, const uint32_t (&wA)[8 * Q], const uint32_t (&wB)[8 * Q], const uint16_t *xrow) {
        uint32_t xw[8 * Q];
#pragma unroll
        for (int i = 0; i < 2 * Q; i++) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xrow) + i);
            xw[4 * i] = v.x;
            xw[4 * i + 1] = v.y;
            xw[4 * i + 2] = v.z;
            xw[4 * i + 3] = v.w;
        }
        // step j: A = {row g pair 2j, row g+8 pair 2j, row g pair 2j+1, row g+8 pair 2j+1}
#pragma unroll
        for (int j = 0; j < 4 * Q; j++)
            mma_16816((j & 1) ? d1[t] : d0[t], wA[2 * j], wB[2 * j], wA[2 * j + 1], wB[2 * j + 1], xw[2 * j],
                      xw[2 * j + 1]);
    };
    auto consume = [&](int i, int s) {
        uint32_t wA[8 * Q], wB[8 * Q];
        rebuild<PAL, Q>(ha[s], fa[s], P, wA);
        rebuild<PAL, Q>(hb[s], fb[s], P, wB);
        mma_tile(0, wA, wB, x0 + int64_t(i) * kCh);
        if (NT == 2) mma_tile(NT - 1, wA, wB, x1 + int64_t(i) * kCh);
    };

    // the ring's first loads; X only after the previous kernel has ended (a
    // prefetch before that could keep a stale line of X in L1)
#pragma unroll
    for (int s = 0; s < kStages; s++)
        if (s < nch) issue(s, s, !a.w_stable);
    if (a.w_stable) pdl_wait();
    int i0 = 0;
    for (; i0 + kStages <= nch; i0 += kStages) {
#pragma unroll
        for (int s = 0; s < kStages; s++) {
            const int i = i0 + s;
            consume(i, s);
            const int nx = i + kStages;
            if (nx < nch) {
                if (PAL && nx % kWin == 0) {   // next 64-group window of raw bits
                    rawa = raw_window(sflags, nwords, wbase, ga + nx * Q);
                    rawb = raw_window(sflags, nwords, wbase, gb + nx * Q);
                }
                issue(nx, s);
            }
        }
    }
#pragma unroll
    for (int s = 0; s < kStages; s++)
        if (i0 + s < nch) consume(i0 + s, s);

    // d[t][0..1]: row g, tokens 8t + 2c, +1; d[t][2..3]: row g + 8, same tokens
    float v[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int q = 0; q < 4; q++) v[t][q] = d0[t][q] + d1[t][q];
    if (slices > 1) {
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
            for (int q = 0; q < 4; q++) red[(warp * 32 + lane) * 4 * NT + t * 4 + q] = v[t][q];
        __syncthreads();
        if (warp != 0) return;
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
            for (int q = 0; q < 4; q++) {
                float acc = red[lane * 4 * NT + t * 4 + q];
                for (int w = 1; w < slices; w++) acc += red[(w * 32 + lane) * 4 * NT + t * 4 + q];
                v[t][q] = acc;
            }
    }
#pragma unroll
    for (int t = 0; t < NT; t++) {
        const int tok = 8 * t + 2 * c;
        if (tok < a.m) {
            a.y[int64_t(tok) * a.n + ra] = v[t][0];
            a.y[int64_t(tok) * a.n + rb] = v[t][2];
        }
        if (tok + 1 < a.m) {
            a.y[int64_t(tok + 1) * a.n + ra] = v[t][1];
            a.y[int64_t(tok + 1) * a.n + rb] = v[t][3];
        }
    }
}

template <bool PAL, int NT, int Q>
__global__ void __launch_bounds__(kMaxSlices * 32) k_gemv_mma(const MmaArgs a) {
    gemv_mma_tile<PAL, NT, Q>(a, blockIdx.x);
}

// Many fused matmuls in one launch (the experts of a mixture-of-experts
// layer): CTA b runs tile b - tile_end[i-1] of item i, where item i is the
// first with b < tile_end[i].  Items share the kernel's template arguments
// (token tiles, step width) and the CTA size; each item's tiles compute
// exactly what a launch of k_gemv_mma for that item alone computes.
constexpr int kBatchMax = 32;
struct MmaBatch {
    MmaArgs item[kBatchMax];
    int tile_end[kBatchMax];   // inclusive prefix sums of the items' tile counts
    int n_items;
};

template <int NT, int Q>
__global__ void __launch_bounds__(kMaxSlices * 32) k_gemv_mma_batched(const __grid_constant__ MmaBatch b) {
    const int t = int(blockIdx.x);
    int i = 0;
    while (i + 1 < b.n_items && t >= b.tile_end[i]) i++;
    gemv_mma_tile<true, NT, Q>(b.item[i], t - (i ? b.tile_end[i - 1] : 0));
}

}  // namespace

cudaError_t launch_gemv_mma(const uint16_t *x, int m, const uint16_t *w_bf16, const uw_dmat *w,
                            const uint8_t *pal_plane, int64_t n, int64_t k, float *y, int slices, int width,
                            cudaStream_t stream, bool w_stable) {
    if (m < 1 || m > 16 || slices < 1 || slices > kMaxSlices || n % kTileRows || k % kChunk)
        return cudaErrorInvalidValue;
    const int q = width == 1 ? 1 : width == 2 ? 2 : (k % (2 * kChunk) == 0 ? 2 : 1);
    if (k % (q * kChunk)) return cudaErrorInvalidValue;
    MmaArgs a{};
    a.x = x;
    a.w_bf16 = w_bf16;
    a.n = n;
    a.k = k;
    a.m = m;
    a.y = y;
    const bool pal = pal_plane != nullptr;
    if (pal) {
        // bitmap words touched by one tile's rows (an unaligned run of 16 * k / 64 bits)
        a.flag_words = int(((kTileRows * (k / kChunk)) >> 5) + 2);
        a.sm = w->sm;
        a.pal = reinterpret_cast<const uint32_t *>(pal_plane);
        a.flagbits = w->flagbits;
        a.rawbase = w->rawbase;
        a.rawexp = w->rawexp;
        a.palette = make_palette16(w->palette);
        a.w_stable = w_stable ? 1 : 0;
    }
    const int nt = m > 8 ? 2 : 1;
    const unsigned grid = unsigned(n / kTileRows);
    const unsigned block = unsigned(slices * 32);
    const size_t smem = size_t(2 * a.flag_words) * 4 + (slices > 1 ? size_t(slices) * 32 * 4 * nt * 4 : 0);
    if (smem > size_t(kMaxSmem)) return cudaErrorInvalidValue;
    cudaError_t err = cudaSuccess;
#define UW_MMA_LAUNCH(P_, N_, Q_) \
    err = launch_pdl(a.w_stable != 0, k_gemv_mma<P_, N_, Q_>, dim3(grid), dim3(block), smem, stream, a)
    if (pal) {
        if (q == 2) { if (nt == 2) UW_MMA_LAUNCH(true, 2, 2); else UW_MMA_LAUNCH(true, 1, 2); }
        else { if (nt == 2) UW_MMA_LAUNCH(true, 2, 1); else UW_MMA_LAUNCH(true, 1, 1); }
    } else {
        if (q == 2) { if (nt == 2) UW_MMA_LAUNCH(false, 2, 2); else UW_MMA_LAUNCH(false, 1, 2); }
        else { if (nt == 2) UW_MMA_LAUNCH(false, 2, 1); else UW_MMA_LAUNCH(false, 1, 1); }
    }
#undef UW_MMA_LAUNCH
    return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_gemv_mma_batched(const MmaItem *items, int n_items, int slices, int width,
                                    cudaStream_t stream) {
    if (n_items < 0 || slices < 1 || slices > kMaxSlices) return cudaErrorInvalidValue;
    // one step width for all items: 32 weights per lane only if every K allows it
    bool all128 = true;
    for (int i = 0; i < n_items; i++) all128 = all128 && items[i].w->k % (2 * kChunk) == 0;
    if (width == 2 && !all128) return cudaErrorInvalidValue;
    const int q = width == 1 ? 1 : (all128 ? 2 : 1);
    int i = 0;
    while (i < n_items) {
        MmaBatch b{};
        int tiles = 0, max_m = 0, max_fw = 0;
        for (; i < n_items && b.n_items < kBatchMax; i++) {
            const MmaItem &it = items[i];
            const uw_dmat &w = *it.w;
            if (it.m == 0) continue;   // an expert without tokens
            if (it.m < 0 || it.m > 16 || w.n % kTileRows || w.k % (q * kChunk) || !w.pal) return cudaErrorInvalidValue;
            MmaArgs &a = b.item[b.n_items];
            a.x = it.x;
            a.m = it.m;
            a.y = it.y;
            a.n = w.n;
            a.k = w.k;
            a.flag_words = int(((kTileRows * (w.k / kChunk)) >> 5) + 2);
            a.sm = w.sm;
            a.pal = reinterpret_cast<const uint32_t *>(w.pal);
            a.flagbits = w.flagbits;
            a.rawbase = w.rawbase;
            a.rawexp = w.rawexp;
            a.palette = make_palette16(w.palette);
            tiles += int(w.n / kTileRows);
            b.tile_end[b.n_items] = tiles;
            max_m = it.m > max_m ? it.m : max_m;
            max_fw = a.flag_words > max_fw ? a.flag_words : max_fw;
            b.n_items++;
        }
        if (b.n_items == 0) continue;
        const int nt = max_m > 8 ? 2 : 1;
        const size_t smem = size_t(2 * max_fw) * 4 + (slices > 1 ? size_t(slices) * 32 * 4 * nt * 4 : 0);
        if (smem > size_t(kMaxSmem)) return cudaErrorInvalidValue;
        const unsigned grid = unsigned(tiles), block = unsigned(slices * 32);
        if (q == 2) {
            if (nt == 2) k_gemv_mma_batched<2, 2><<<grid, block, smem, stream>>>(b);
            else k_gemv_mma_batched<1, 2><<<grid, block, smem, stream>>>(b);
        } else {
            if (nt == 2) k_gemv_mma_batched<2, 1><<<grid, block, smem, stream>>>(b);
            else k_gemv_mma_batched<1, 1><<<grid, block, smem, stream>>>(b);
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace uw
