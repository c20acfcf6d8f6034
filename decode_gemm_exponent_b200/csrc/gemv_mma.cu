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
// one tile and splits its K into S contiguous slices of 64-weight chunks.
// Lane (g, c) = (lane / 4, lane % 4) loads weights [16c, 16c + 16) of every
// chunk of rows g and g + 8 (4 lanes cover a row's 64 sign/mantissa bytes).
// A chunk's 64 K positions map onto the MMA's four K = 16 steps as: step j,
// thread c, MMA K slots {2c, 2c+1, 2c+8, 2c+9} <- weights 16c + 4j + {0, 1,
// 2, 3}; the X fragment uses the same map, so every product is formed exactly
// once.  Lanes whose token is >= m load a valid X row anyway: it only feeds
// output columns that are not stored.  Each warp keeps kStages chunks of
// loads in flight in a register ring.  The raw-group bitmap words of the
// tile's rows and their prefix counts are staged in shared memory; each lane
// keeps a 64-chunk window of its two rows' raw bits in registers, so a raw
// group's exponents are fetched together with the chunk's other loads.
// The K steps alternate between two accumulators (independent MMA chains),
// added at the end, and the S slice results are summed in ascending slice
// order through shared memory.  The fused and plain variants share all of
// this but the loader, so their outputs are bit-identical.
#include <algorithm>

#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kTileRows = 16;
constexpr int kChunk = 64;
constexpr int kStages = 3;
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
    float *y;                  // [m, n]
};

// one lane's 16 weights of one chunk of one row, as loaded
struct Half {
    uint4 a;       // plain: weights 0..7; fused: sign/mantissa bytes
    uint4 b;       // plain: weights 8..15; fused: palette words (.x, .y) or raw exponents
};

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

template <bool PAL>
__device__ __forceinline__ Half load_half(const MmaArgs &a, const uint8_t *smp, const uint32_t *palp,
                                          const uint16_t *wp, bool raw, int64_t g, const uint32_t *sflags,
                                          const uint32_t *srb, int64_t wbase, int c) {
    Half h;
    if (!PAL) {
        h.a = __ldcs(reinterpret_cast<const uint4 *>(wp));
        h.b = __ldcs(reinterpret_cast<const uint4 *>(wp) + 1);
    } else {
        h.a = __ldcs(reinterpret_cast<const uint4 *>(smp));
        if (raw) {
            const int wi = int((g >> 5) - wbase);
            const uint32_t rank = srb[wi] + __popc(sflags[wi] & ((1u << (uint32_t(g) & 31u)) - 1u));
            h.b = __ldcs(reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(rank) * kGroup + c * 16));
        } else {
            const uint2 p = __ldcs(reinterpret_cast<const uint2 *>(palp));
            h.b = make_uint4(p.x, p.y, 0u, 0u);
        }
    }
    return h;
}

// Half -> 8 BF16 pairs (weights 2i, 2i+1 in pair i)
template <bool PAL>
__device__ __forceinline__ void rebuild(const Half &h, bool raw, const Palette16 &P, uint32_t (&w)[8]) {
    if (!PAL) {
        w[0] = h.a.x; w[1] = h.a.y; w[2] = h.a.z; w[3] = h.a.w;
        w[4] = h.b.x; w[5] = h.b.y; w[6] = h.b.z; w[7] = h.b.w;
    } else {
        uint32_t r0, r1, r2, r3;
        if (raw) {
            r0 = rot4(h.b.x);
            r1 = rot4(h.b.y);
            r2 = rot4(h.b.z);
            r3 = rot4(h.b.w);
        } else {
            pal_rot(h.b.x, P, r0, r1);
            pal_rot(h.b.y, P, r2, r3);
        }
        join4(r0, h.a.x, w[0], w[1]);
        join4(r1, h.a.y, w[2], w[3]);
        join4(r2, h.a.z, w[4], w[5]);
        join4(r3, h.a.w, w[6], w[7]);
    }
}

template <bool PAL, int NT>   // NT: 8-token tiles (1: m <= 8, 2: m <= 16)
__global__ void __launch_bounds__(kMaxSlices * 32) k_gemv_mma(const MmaArgs a) {
    // dynamic shared memory: [bitmap words][prefix counts] (fused), then the
    // slice results [slices][32][8 * NT] (slices > 1)
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *sflags = smem, *srb = smem + a.flag_words;
    float *red = reinterpret_cast<float *>(smem + 2 * a.flag_words);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slices = blockDim.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t row0 = int64_t(blockIdx.x) * kTileRows;
    const int64_t ra = row0 + g, rb = ra + 8;       // this lane's two rows
    const int64_t gpr = a.k / kChunk;               // groups (chunks) per row
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
    const int64_t ch0 = gpr * warp / slices;
    const int nch = int(gpr * (warp + 1) / slices - ch0);

    // per-lane streams, advanced one chunk at a time
    const int64_t ea = ra * a.k + ch0 * kChunk + c * 16, eb = ea + 8 * a.k;
    const uint8_t *sma = a.sm + ea, *smb = a.sm + eb;
    const uint32_t *pala = a.pal + ea / 8, *palb = a.pal + eb / 8;
    const uint16_t *wa = a.w_bf16 + ea, *wb = a.w_bf16 + eb;
    const int64_t ga = ra * gpr + ch0, gb = rb * gpr + ch0;   // group of the slice's first chunk
    // X rows of this lane's tokens (clamped: columns >= m are not stored)
    const uint16_t *x0 = a.x + int64_t(min(g, a.m - 1)) * a.k + ch0 * kChunk + c * 16;
    const uint16_t *x1 = a.x + int64_t(min(g + 8, a.m - 1)) * a.k + ch0 * kChunk + c * 16;

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

    Half ha[kStages], hb[kStages];
    bool fa[kStages], fb[kStages];
    auto issue = [&](int i, int s) {   // loads of chunk i into ring slot s
        const int bit = i & 63;
        fa[s] = PAL && ((rawa >> bit) & 1u);
        fb[s] = PAL && ((rawb >> bit) & 1u);
        ha[s] = load_half<PAL>(a, sma + int64_t(i) * kChunk, pala + i * 8, wa + int64_t(i) * kChunk, fa[s], ga + i,
                               sflags, srb, wbase, c);
        hb[s] = load_half<PAL>(a, smb + int64_t(i) * kChunk, palb + i * 8, wb + int64_t(i) * kChunk, fb[s], gb + i,
                               sflags, srb, wbase, c);
    };
    auto consume = [&](int i, int s) {
        uint32_t wA[8], wB[8];
        rebuild<PAL>(ha[s], fa[s], P, wA);
        rebuild<PAL>(hb[s], fb[s], P, wB);
        const uint4 *xp0 = reinterpret_cast<const uint4 *>(x0 + int64_t(i) * kChunk);
        const uint4 p0 = __ldg(xp0), q0 = __ldg(xp0 + 1);
        const uint32_t xa[8] = {p0.x, p0.y, p0.z, p0.w, q0.x, q0.y, q0.z, q0.w};
        // step j: A = {row g pair 2j, row g+8 pair 2j, row g pair 2j+1, row g+8 pair 2j+1}
        mma_16816(d0[0], wA[0], wB[0], wA[1], wB[1], xa[0], xa[1]);
        mma_16816(d1[0], wA[2], wB[2], wA[3], wB[3], xa[2], xa[3]);
        mma_16816(d0[0], wA[4], wB[4], wA[5], wB[5], xa[4], xa[5]);
        mma_16816(d1[0], wA[6], wB[6], wA[7], wB[7], xa[6], xa[7]);
        if (NT == 2) {
            const uint4 *xp1 = reinterpret_cast<const uint4 *>(x1 + int64_t(i) * kChunk);
            const uint4 p1 = __ldg(xp1), q1 = __ldg(xp1 + 1);
            const uint32_t xb[8] = {p1.x, p1.y, p1.z, p1.w, q1.x, q1.y, q1.z, q1.w};
            mma_16816(d0[NT - 1], wA[0], wB[0], wA[1], wB[1], xb[0], xb[1]);
            mma_16816(d1[NT - 1], wA[2], wB[2], wA[3], wB[3], xb[2], xb[3]);
            mma_16816(d0[NT - 1], wA[4], wB[4], wA[5], wB[5], xb[4], xb[5]);
            mma_16816(d1[NT - 1], wA[6], wB[6], wA[7], wB[7], xb[6], xb[7]);
        }
    };

#pragma unroll
    for (int s = 0; s < kStages; s++)
        if (s < nch) issue(s, s);
    int i0 = 0;
    for (; i0 + kStages <= nch; i0 += kStages) {
#pragma unroll
        for (int s = 0; s < kStages; s++) {
            const int i = i0 + s;
            consume(i, s);
            const int nx = i + kStages;
            if (nx < nch) {
                if (PAL && (nx & 63) == 0) {   // next 64-chunk window of raw bits
                    rawa = raw_window(sflags, nwords, wbase, ga + nx);
                    rawb = raw_window(sflags, nwords, wbase, gb + nx);
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
                float s = red[lane * 4 * NT + t * 4 + q];
                for (int w = 1; w < slices; w++) s += red[(w * 32 + lane) * 4 * NT + t * 4 + q];
                v[t][q] = s;
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

}  // namespace

cudaError_t launch_gemv_mma(const uint16_t *x, int m, const uint16_t *w_bf16, const uw_dmat *w,
                            const uint8_t *pal_plane, int64_t n, int64_t k, float *y, int slices,
                            cudaStream_t stream) {
    if (m < 1 || m > 16 || slices < 1 || slices > kMaxSlices || n % kTileRows || k % kChunk)
        return cudaErrorInvalidValue;
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
    }
    const int nt = m > 8 ? 2 : 1;
    const unsigned grid = unsigned(n / kTileRows);
    const unsigned block = unsigned(slices * 32);
    const size_t smem = size_t(2 * a.flag_words) * 4 + (slices > 1 ? size_t(slices) * 32 * 4 * nt * 4 : 0);
    if (smem > size_t(kMaxSmem)) return cudaErrorInvalidValue;
    if (pal) {
        if (nt == 2) k_gemv_mma<true, 2><<<grid, block, smem, stream>>>(a);
        else k_gemv_mma<true, 1><<<grid, block, smem, stream>>>(a);
    } else {
        if (nt == 2) k_gemv_mma<false, 2><<<grid, block, smem, stream>>>(a);
        else k_gemv_mma<false, 1><<<grid, block, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace uw
