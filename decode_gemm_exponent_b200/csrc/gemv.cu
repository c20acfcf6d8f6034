// gemv.cu -- CUDA-core GEMV for small batches (m <= 8), Y = X * W^T.
//
// The Unweight page (§十) names the fixed cost of the reconstructive matmul at
// small batch as a main overhead, and (§六) notes that at batch 1-64 the
// plain path often wins.  At m <= 4 the job is a pure HBM stream, so this
// kernel reads the compressed planes with coalesced 16-byte loads straight
// into registers and rebuilds BF16 there (§五: the rebuilt weights never go
// back to HBM), with no shared-memory staging.
//
// One warp owns R consecutive rows of W and walks K in steps of 512: lane l
// handles weights [k0 + 16 l, k0 + 16 l + 16); the loads of the next step
// are issued before the current step's arithmetic.  Before the loop the warp
// loads the raw-group bitmap words of its rows and their prefix counts (one
// word per lane) and later broadcasts them with shuffles, so the loop issues
// only independent loads.  Products are accumulated with the mixed-precision
// FMA (BF16 x BF16 + FP32, one rounding) in a fixed order (k ascending) and
// the 32 lane sums are combined by a fixed xor-butterfly, so the fused kernel
// and its plain-BF16 twin (same template, other loader) are bit-identical.
#include <algorithm>

#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kWarps = 8;

struct GemvArgs {
    const uint16_t *x;
    const uint16_t *w_bf16;
    const uint8_t *sm;
    const uint32_t *pal;       // 4-bit palette plane as words
    const uint32_t *flagbits;
    const uint32_t *rawbase;
    const uint8_t *rawexp;
    Palette16 palette;
    int64_t n, k;
    float *y;
    uint32_t *status;
};

// Loads of one 16-weight piece of one row (issued one iteration ahead).
struct Piece {
    uint4 a;          // plain: weights 0..7 (BF16); fused: sign/mantissa bytes
    uint4 b;          // plain: weights 8..15;       fused: .x/.y palette words
    uint32_t rank;    // fused: raw-group rank
    bool raw;
};

template <bool PAL>
__device__ __forceinline__ Piece load_piece(const GemvArgs &a, int64_t row, int64_t k0, bool live,
                                            uint32_t fw, uint32_t rb, int64_t g) {
    Piece p;
    p.a = make_uint4(0u, 0u, 0u, 0u);
    p.b = p.a;
    p.raw = false;
    p.rank = 0;
    const int64_t e0 = row * a.k + k0;
    if (!PAL) {
        if (live) {
            const uint4 *q = reinterpret_cast<const uint4 *>(a.w_bf16 + e0);
            p.a = __ldcs(q);
            p.b = __ldcs(q + 1);
        }
    } else {
        const uint32_t bit = uint32_t(g) & 31u;
        p.raw = live && ((fw >> bit) & 1u);
        p.rank = rb + __popc(fw & ((1u << bit) - 1u));
        if (live) {
            p.a = __ldcs(reinterpret_cast<const uint4 *>(a.sm + e0));
            const uint2 pw = __ldcs(reinterpret_cast<const uint2 *>(a.pal + e0 / 8));
            p.b.x = pw.x;
            p.b.y = pw.y;
        }
    }
    return p;
}

// Piece -> 8 BF16 pairs
template <bool PAL>
__device__ __forceinline__ void rebuild_piece(const GemvArgs &a, const Piece &p, int64_t k0,
                                              uint32_t (&wv)[8]) {
    if (!PAL) {
        wv[0] = p.a.x; wv[1] = p.a.y; wv[2] = p.a.z; wv[3] = p.a.w;
        wv[4] = p.b.x; wv[5] = p.b.y; wv[6] = p.b.z; wv[7] = p.b.w;
    } else {
        uint32_t r0, r1, r2, r3;
        if (p.raw) {
            const uint4 rx = __ldg(reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(p.rank) * kGroup + (k0 & 63)));
            r0 = rot4(rx.x);
            r1 = rot4(rx.y);
            r2 = rot4(rx.z);
            r3 = rot4(rx.w);
        } else {
            pal_rot(p.b.x, a.palette, r0, r1);
            pal_rot(p.b.y, a.palette, r2, r3);
        }
        join4(r0, p.a.x, wv[0], wv[1]);
        join4(r1, p.a.y, wv[2], wv[3]);
        join4(r2, p.a.z, wv[4], wv[5]);
        join4(r3, p.a.w, wv[6], wv[7]);
    }
}

template <int M, int R, bool PAL>
__global__ void __launch_bounds__(kWarps * 32) k_gemv_fma(const GemvArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t(blockIdx.x) * kWarps + warp) * R;
    if (row0 >= a.n) return;
    const int64_t gpr = a.k >> 6;                 // groups per row
    const int nit = int((a.k + 511) >> 9);

    // raw-group bitmap words covering each row, one per lane
    uint32_t fw_l[R], rb_l[R];
    int64_t wfirst[R];
    bool direct = false;
    if (PAL) {
#pragma unroll
        for (int r = 0; r < R; r++) {
            const int64_t row = min(row0 + r, a.n - 1);
            const int64_t g0 = row * gpr;
            wfirst[r] = g0 >> 5;
            const int64_t nw = ((g0 + gpr - 1) >> 5) - wfirst[r] + 1;
            direct |= nw > 32;
            fw_l[r] = lane < nw ? __ldg(a.flagbits + wfirst[r] + lane) : 0u;
            rb_l[r] = lane < nw ? __ldg(a.rawbase + wfirst[r] + lane) : 0u;
        }
    }

    // issue the loads of iteration `it` (all lanes take part: shuffles)
    auto load_it = [&](int it, Piece (&pc)[R], uint4 (&xc)[M][2]) {
        const int64_t k0 = int64_t(it) * 512 + lane * 16;
        const bool act = k0 < a.k;
#pragma unroll
        for (int r = 0; r < R; r++) {
            const int64_t row = row0 + r;
            const bool live = act && row < a.n;
            uint32_t fw = 0u, rb = 0u;
            int64_t g = 0;
            if (PAL) {
                g = min(row, a.n - 1) * gpr + (k0 >> 6);
                if (!direct) {
                    const int idx = int((g >> 5) - wfirst[r]) & 31;
                    fw = __shfl_sync(0xFFFFFFFFu, fw_l[r], idx);
                    rb = __shfl_sync(0xFFFFFFFFu, rb_l[r], idx);
                } else if (live) {
                    fw = __ldg(a.flagbits + (g >> 5));
                    rb = __ldg(a.rawbase + (g >> 5));
                }
            }
            pc[r] = load_piece<PAL>(a, row, k0, live, fw, rb, g);
        }
#pragma unroll
        for (int m = 0; m < M; m++) {
            xc[m][0] = xc[m][1] = make_uint4(0u, 0u, 0u, 0u);
            if (act) {
                const uint4 *xp = reinterpret_cast<const uint4 *>(a.x + int64_t(m) * a.k + k0);
                xc[m][0] = __ldg(xp);
                xc[m][1] = __ldg(xp + 1);
            }
        }
    };

    float acc[M][R];
#pragma unroll
    for (int m = 0; m < M; m++)
#pragma unroll
        for (int r = 0; r < R; r++) acc[m][r] = 0.f;

    Piece pc[R], pn[R];
    uint4 xc[M][2], xn[M][2];
    load_it(0, pc, xc);
    for (int it = 0; it < nit; it++) {
        if (it + 1 < nit) load_it(it + 1, pn, xn);
        const int64_t k0 = int64_t(it) * 512 + lane * 16;
        uint32_t wv[R][8];
#pragma unroll
        for (int r = 0; r < R; r++) rebuild_piece<PAL>(a, pc[r], k0, wv[r]);
#pragma unroll
        for (int m = 0; m < M; m++) {
            const uint32_t xv[8] = {xc[m][0].x, xc[m][0].y, xc[m][0].z, xc[m][0].w,
                                    xc[m][1].x, xc[m][1].y, xc[m][1].z, xc[m][1].w};
#pragma unroll
            for (int j = 0; j < 8; j++)
#pragma unroll
                for (int r = 0; r < R; r++) acc[m][r] = fma2_bf16(xv[j], wv[r][j], acc[m][r]);
        }
#pragma unroll
        for (int r = 0; r < R; r++) pc[r] = pn[r];
#pragma unroll
        for (int m = 0; m < M; m++) {
            xc[m][0] = xn[m][0];
            xc[m][1] = xn[m][1];
        }
    }

#pragma unroll
    for (int m = 0; m < M; m++)
#pragma unroll
        for (int r = 0; r < R; r++) {
            float v = acc[m][r];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
            acc[m][r] = v;
        }
#pragma unroll
    for (int m = 0; m < M; m++)
#pragma unroll
        for (int r = 0; r < R; r++)
            if (lane == ((m * R + r) & 31) && row0 + r < a.n) a.y[int64_t(m) * a.n + row0 + r] = acc[m][r];
}

template <int M, int R>
cudaError_t launch_mr(const GemvArgs &a, bool pal, cudaStream_t stream) {
    const unsigned grid = unsigned((a.n + int64_t(kWarps) * R - 1) / (int64_t(kWarps) * R));
    if (pal) k_gemv_fma<M, R, true><<<grid, kWarps * 32, 0, stream>>>(a);
    else k_gemv_fma<M, R, false><<<grid, kWarps * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int R>
cudaError_t launch_r(const GemvArgs &a, int m, bool pal, cudaStream_t stream) {
    switch (m) {
        case 1: return launch_mr<1, R>(a, pal, stream);
        case 2: return launch_mr<2, R>(a, pal, stream);
        case 3: return launch_mr<3, R>(a, pal, stream);
        case 4: return launch_mr<4, R>(a, pal, stream);
        case 5: return launch_mr<5, R>(a, pal, stream);
        case 6: return launch_mr<6, R>(a, pal, stream);
        case 7: return launch_mr<7, R>(a, pal, stream);
        case 8: return launch_mr<8, R>(a, pal, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_gemv_fma(const uint16_t *x, int m, const uint16_t *w_bf16, const uw_dmat *w,
                            const uint8_t *pal_plane, int64_t n, int64_t k, float *y,
                            int rows_per_warp, uint32_t *status, cudaStream_t stream) {
    GemvArgs a{};
    a.x = x;
    a.w_bf16 = w_bf16;
    a.n = n;
    a.k = k;
    a.y = y;
    a.status = status;
    const bool pal = pal_plane != nullptr;
    if (pal) {
        a.sm = w->sm;
        a.pal = reinterpret_cast<const uint32_t *>(pal_plane);
        a.flagbits = w->flagbits;
        a.rawbase = w->rawbase;
        a.rawexp = w->rawexp;
        a.palette = make_palette16(w->palette);
    }
    if (rows_per_warp == 1) return launch_r<1>(a, m, pal, stream);
    if (rows_per_warp == 2) return launch_r<2>(a, m, pal, stream);
    return cudaErrorInvalidValue;
}

}  // namespace uw
