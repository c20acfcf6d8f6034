// gemv.cu -- CUDA-core FMA GEMV for small batches (m <= 8), Y = X * W^T.
//
// The Unweight page (§十) names the fixed cost of the reconstructive matmul at
// small batch as a main overhead, and (§六) notes that at batch 1-64 the
// plain path often wins.  At m <= 4 the job is a pure HBM stream, so this
// kernel reads the compressed planes with coalesced 16-byte loads straight
// into registers and rebuilds BF16 there (§五: the rebuilt weights never go
// back to HBM), with no shared-memory staging at all.
//
// One warp owns R consecutive rows of W and walks K in steps of 512: lane l
// handles weights [k0 + 16 l, k0 + 16 l + 16).  Per lane the products are
// accumulated in a fixed order (k ascending) and the 32 lane sums are then
// combined by a fixed xor-butterfly, so the fused kernel and its plain-BF16
// twin (same template, other loader) give bit-identical results.
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
};

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// 16 weights of row `row` starting at column k0, as 8 BF16 pairs.
template <bool PAL>
__device__ __forceinline__ void load_weights(const GemvArgs &a, int64_t row, int64_t k0,
                                             uint32_t (&wv)[8]) {
    const int64_t e0 = row * a.k + k0;
    if (!PAL) {
        const uint4 *p = reinterpret_cast<const uint4 *>(a.w_bf16 + e0);
        const uint4 v0 = __ldcs(p), v1 = __ldcs(p + 1);
        wv[0] = v0.x; wv[1] = v0.y; wv[2] = v0.z; wv[3] = v0.w;
        wv[4] = v1.x; wv[5] = v1.y; wv[6] = v1.z; wv[7] = v1.w;
    } else {
        const uint2 pw = __ldcs(reinterpret_cast<const uint2 *>(a.pal + e0 / 8));
        const uint4 s = __ldcs(reinterpret_cast<const uint4 *>(a.sm + e0));
        const int64_t g = e0 / kGroup;
        const uint32_t fw = __ldg(a.flagbits + (g >> 5));
        uint32_t e[4];
        if ((fw >> (g & 31)) & 1u) {
            const uint32_t rank = __ldg(a.rawbase + (g >> 5)) + __popc(fw & ((1u << (g & 31)) - 1u));
            const uint4 r = __ldg(reinterpret_cast<const uint4 *>(a.rawexp + uint64_t(rank) * kGroup +
                                                                 (e0 & (kGroup - 1))));
            e[0] = r.x; e[1] = r.y; e[2] = r.z; e[3] = r.w;
        } else {
            pal_exponents(pw.x, a.palette, e[0], e[1]);
            pal_exponents(pw.y, a.palette, e[2], e[3]);
        }
        join4(e[0], s.x, wv[0], wv[1]);
        join4(e[1], s.y, wv[2], wv[3]);
        join4(e[2], s.z, wv[4], wv[5]);
        join4(e[3], s.w, wv[6], wv[7]);
    }
}

template <int M, int R, bool PAL>
__global__ void __launch_bounds__(kWarps * 32) k_gemv_fma(const GemvArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t(blockIdx.x) * kWarps + warp) * R;
    if (row0 >= a.n) return;

    float acc[M][R];
#pragma unroll
    for (int m = 0; m < M; m++)
#pragma unroll
        for (int r = 0; r < R; r++) acc[m][r] = 0.f;

#pragma unroll 2
    for (int64_t k0 = int64_t(lane) * 16; k0 < a.k; k0 += 512) {
        uint32_t wv[R][8];
#pragma unroll
        for (int r = 0; r < R; r++) {
            if (row0 + r < a.n) load_weights<PAL>(a, row0 + r, k0, wv[r]);
            else {
#pragma unroll
                for (int j = 0; j < 8; j++) wv[r][j] = 0u;
            }
        }
#pragma unroll
        for (int m = 0; m < M; m++) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(a.x + int64_t(m) * a.k + k0);
            const uint4 x0 = __ldg(xp), x1 = __ldg(xp + 1);
            const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const float xl = bf_lo(xv[j]), xh = bf_hi(xv[j]);
#pragma unroll
                for (int r = 0; r < R; r++) {
                    acc[m][r] = fmaf(xl, bf_lo(wv[r][j]), acc[m][r]);
                    acc[m][r] = fmaf(xh, bf_hi(wv[r][j]), acc[m][r]);
                }
            }
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
                            int rows_per_warp, cudaStream_t stream) {
    GemvArgs a{};
    a.x = x;
    a.w_bf16 = w_bf16;
    a.n = n;
    a.k = k;
    a.y = y;
    const bool pal = pal_plane != nullptr;
    if (pal) {
        a.sm = w->sm;
        a.pal = reinterpret_cast<const uint32_t *>(pal_plane);
        a.flagbits = w->flagbits;
        a.rawbase = w->rawbase;
        a.rawexp = w->rawexp;
        auto pack = [&](int i) {
            return uint32_t(w->palette[i]) | uint32_t(w->palette[i + 1]) << 8 |
                   uint32_t(w->palette[i + 2]) << 16 | uint32_t(w->palette[i + 3]) << 24;
        };
        a.palette = Palette16{pack(0), pack(4), pack(8), pack(12)};
    }
    if (rows_per_warp == 1) return launch_r<1>(a, m, pal, stream);
    if (rows_per_warp == 2) return launch_r<2>(a, m, pal, stream);
    return cudaErrorInvalidValue;
}

}  // namespace uw
