// gemm_tc.cu -- tensor-core GEMM Y = X * W^T on sm_100a with tcgen05 MMA and a
// TMEM accumulator, in two flavours sharing one template:
//   * fused: W arrives compressed (4-bit palette plane + sign/mantissa plane +
//     raw groups) and is rebuilt to BF16 in shared memory (Unweight page §七,
//     the reconstructive matmul; §五, decompress on chip, never back to HBM);
//   * plain: W arrives as BF16 through TMA (the uncompressed baseline and the
//     bit-exactness twin of the fused flavour).
// Both issue the identical MMA sequence, so their outputs are bit-identical.
//
// CTA tile: 128 rows of W (the MMA "M") x `BN` tokens (the MMA "N"), K in
// steps of 64 (one group).  Grid = (n/128, ceil(m/BN), split_k).  Warps:
//   warp 0     producer: per K-step TMA of the X tile and either the BF16 W
//              tile or the compressed tiles (sm plane 64 B/row with the
//              64-byte swizzle, palette plane 32 B/row with the 32-byte
//              swizzle); raw rows are fetched by 64-byte bulk copies; the
//              stage's raw-row bitmap is written to shared memory.
//   warp 1     MMA issuer (one thread): 4 x tcgen05.mma (K = 16 each) per
//              K-step into the TMEM accumulator; tcgen05.commit frees the
//              stage; a final commit signals the epilogue.  Also owns TMEM.
//   warps 2-5  fused: each thread rebuilds one W row per K-step into the
//              128-byte-swizzled K-major tile, then fences the async proxy
//              and arrives.  Then all four read the accumulator back
//              (tcgen05.ld, one TMEM lane quarter each) and store Y (fp32).
// Every wait is bounded (globaltimer); on time-out the kernel raises
// UW_DEVERR_TIMEOUT, stops issuing work, lets copies and MMAs in flight
// finish, frees TMEM and returns.
#include <algorithm>
#include <cstring>

#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kThreads = 192;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxSmem = 232448;   // 227 KB opt-in per CTA

template <int BN, bool PAL>
struct Cfg {
    static constexpr int kW = kBM * kBK * 2;             // rebuilt / loaded W tile
    static constexpr int kX = BN * kBK * 2;              // X tile
    static constexpr int kSM = PAL ? kBM * kBK : 0;      // sign/mantissa tile
    static constexpr int kPL = PAL ? kBM * kBK / 2 : 0;  // palette-index tile
    static constexpr int kRAW = PAL ? kBM * kBK : 0;     // raw exponents, one slot per row
    static constexpr int kStage = kW + kX + kSM + kPL + kRAW;
    static constexpr int kOffX = kW, kOffSM = kW + kX, kOffPL = kOffSM + kSM, kOffRAW = kOffPL + kPL;
    static constexpr uint32_t kTmemCols = BN < 32 ? 32u : uint32_t(BN);
    static_assert(kStage % 1024 == 0, "stage tiles must keep 1024-byte alignment");
};

struct TcArgs {
    int64_t m, n, k;
    int split_k, ks_per_split, stages;
    uint32_t debug_flags;
    uint64_t timeout_ns;
    float *y;
    float *partial;
    const uint32_t *flagbits;
    const uint32_t *rawbase;
    const uint8_t *rawexp;
    Palette16 pal;
    uint32_t *status;
};

__host__ __device__ constexpr int tail_bytes(int stages) {
    // barriers (3 per stage + 2), raw bitmaps (4 words per stage), TMEM slot, abort flag
    return (3 * stages + 2) * 8 + stages * 16 + 16;
}

template <int BN, bool PAL>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
              const __grid_constant__ CUtensorMap tmB, const TcArgs a) {
    using C = Cfg<BN, PAL>;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                                 ~uintptr_t(1023));
    const int S = a.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(tiles + size_t(S) * C::kStage);
    uint64_t *wready = full + S;
    uint64_t *empty = wready + S;
    uint64_t *accf = empty + S;
    uint64_t *never = accf + 1;
    uint32_t *rawmap = reinterpret_cast<uint32_t *>(never + 1);   // 4 words per stage
    uint32_t *tmem_slot = rawmap + 4 * S;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = int64_t(blockIdx.x) * kBM;
    const int64_t m0 = int64_t(blockIdx.y) * BN;
    const int split = blockIdx.z;
    const int nks_total = int(a.k / kBK);
    const int ks_begin = split * a.ks_per_split;
    const int nks = max(0, min(nks_total - ks_begin, a.ks_per_split));
    const uint64_t T = a.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&wready[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(never, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmA);
        if (PAL) prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int issued = 0;
        const int64_t gpr = a.k / kGroup;   // groups per row of W
        for (int ks = 0; ks < nks; ks++) {
            const int s = ks % S;
            const uint32_t ph = uint32_t(ks / S) & 1u;
            if (ks >= S) {
                const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], ph ^ 1u, T));
                if (!ok) {
                    if (lane == 0) {
                        flag_error(a.status, UW_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    }
                    break;
                }
            }
            if (*abort_flag) break;
            const int kg = ks_begin + ks;
            uint8_t *st = tiles + size_t(s) * C::kStage;
            if (PAL) {
                uint32_t mk[4];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int64_t row = n0 + lane + 32 * i;
                    bool raw = false;
                    if (row < a.n) {
                        const int64_t g = row * gpr + kg;
                        raw = (__ldg(a.flagbits + (g >> 5)) >> (g & 31)) & 1u;
                    }
                    mk[i] = __ballot_sync(0xFFFFFFFFu, raw);
                }
                if (lane < 4) rawmap[4 * s + lane] = lane == 0 ? mk[0] : lane == 1 ? mk[1] : lane == 2 ? mk[2] : mk[3];
                const int nraw = __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[s], uint32_t(C::kX + C::kSM + C::kPL + 64 * nraw));
                    tma_load_2d(st + C::kOffX, &tmX, kg * kBK, int32_t(m0), &full[s]);
                    tma_load_2d(st + C::kOffSM, &tmA, kg * kBK, int32_t(n0), &full[s]);
                    tma_load_2d(st + C::kOffPL, &tmB, kg * (kBK / 2), int32_t(n0), &full[s]);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    if ((mk[i] >> lane) & 1u) {
                        const int r = lane + 32 * i;
                        const int64_t g = (n0 + r) * gpr + kg;
                        const uint32_t fw = __ldg(a.flagbits + (g >> 5));
                        const uint32_t rank = __ldg(a.rawbase + (g >> 5)) + __popc(fw & ((1u << (g & 31)) - 1u));
                        bulk_g2s(st + C::kOffRAW + r * 64, a.rawexp + uint64_t(rank) * kGroup, 64, &full[s]);
                    }
                }
            } else if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], uint32_t(C::kX + C::kW));
                tma_load_2d(st + C::kOffX, &tmX, kg * kBK, int32_t(m0), &full[s]);
                tma_load_2d(st, &tmA, kg * kBK, int32_t(n0), &full[s]);
            }
            issued = ks + 1;
        }
        // let every copy this warp issued land before the CTA can exit
        for (int ks = max(0, issued - S); ks < issued; ks++)
            mbar_wait(&full[ks % S], uint32_t(ks / S) & 1u, T);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
            bool ok = true;
            if (a.debug_flags & UW_DEBUG_NEVER_ARRIVE) ok = mbar_wait(never, 0, T);
            for (int ks = 0; ks < nks && ok; ks++) {
                const int s = ks % S;
                const uint32_t ph = uint32_t(ks / S) & 1u;
                ok = mbar_wait(&full[s], ph, T);
                if (ok && PAL) ok = mbar_wait(&wready[s], ph, T);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sa = smem_addr(tiles + size_t(s) * C::kStage);
                const uint32_t sb = sa + C::kOffX;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; kk++)
                    tc_mma_bf16(tmem, smem_desc_k128(sa + 32 * kk), smem_desc_k128(sb + 32 * kk), idesc,
                                (ks | kk) != 0);
                tc_commit(&empty[s]);
            }
            if (!ok) {
                flag_error(a.status, UW_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            tc_commit(accf);   // fires once every MMA issued above has completed
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ rebuild + epilogue
        const int q = warp & 3;          // TMEM lane quarter this warp may access
        const int r = q * 32 + lane;     // tile row
        if (PAL) {
            for (int ks = 0; ks < nks; ks++) {
                const int s = ks % S;
                const uint32_t ph = uint32_t(ks / S) & 1u;
                if (!mbar_wait(&full[s], ph, T)) {
                    flag_error(a.status, UW_DEVERR_TIMEOUT);
                    break;
                }
                uint8_t *st = tiles + size_t(s) * C::kStage;
                const uint8_t *smrow = st + C::kOffSM + r * 64;
                const uint8_t *plrow = st + C::kOffPL + r * 32;
                uint8_t *wrow = st + r * 128;
                const int sw64 = (r >> 1) & 3, sw32 = (r >> 2) & 1, sw128 = r & 7;
                uint4 smv[4], ev[4];
#pragma unroll
                for (int c = 0; c < 4; c++)
                    smv[c] = *reinterpret_cast<const uint4 *>(smrow + ((c ^ sw64) << 4));
                if ((rawmap[4 * s + q] >> lane) & 1u) {
#pragma unroll
                    for (int c = 0; c < 4; c++)
                        ev[c] = *reinterpret_cast<const uint4 *>(st + C::kOffRAW + r * 64 + c * 16);
                } else {
                    const uint4 p0 = *reinterpret_cast<const uint4 *>(plrow + ((0 ^ sw32) << 4));
                    const uint4 p1 = *reinterpret_cast<const uint4 *>(plrow + ((1 ^ sw32) << 4));
                    pal_exponents(p0.x, a.pal, ev[0].x, ev[0].y);
                    pal_exponents(p0.y, a.pal, ev[0].z, ev[0].w);
                    pal_exponents(p0.z, a.pal, ev[1].x, ev[1].y);
                    pal_exponents(p0.w, a.pal, ev[1].z, ev[1].w);
                    pal_exponents(p1.x, a.pal, ev[2].x, ev[2].y);
                    pal_exponents(p1.y, a.pal, ev[2].z, ev[2].w);
                    pal_exponents(p1.z, a.pal, ev[3].x, ev[3].y);
                    pal_exponents(p1.w, a.pal, ev[3].z, ev[3].w);
                }
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    *reinterpret_cast<uint4 *>(wrow + (((2 * c) ^ sw128) << 4)) =
                        join8(ev[c].x, ev[c].y, smv[c].x, smv[c].y);
                    *reinterpret_cast<uint4 *>(wrow + (((2 * c + 1) ^ sw128) << 4)) =
                        join8(ev[c].z, ev[c].w, smv[c].z, smv[c].w);
                }
                fence_proxy_async_smem();
                mbar_arrive(&wready[s]);
            }
        }
        const bool ok = mbar_wait(accf, 0, T);
        tc_fence_after();
        const bool skip = __any_sync(0xFFFFFFFFu, !ok || *abort_flag != 0 || nks == 0);
        if (!ok && lane == 0) flag_error(a.status, UW_DEVERR_TIMEOUT);
        if (!skip) {
            const int64_t row = n0 + r;
            float *out = a.split_k > 1 ? a.partial + int64_t(split) * a.m * a.n : a.y;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + (uint32_t(q * 32) << 16) + uint32_t(c0), v);
                tmem_ld_wait();
                if (row < a.n) {
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const int64_t mm = m0 + c0 + j;
                        if (mm < a.m) out[mm * a.n + row] = __uint_as_float(v[j]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

__global__ void k_splitk_reduce(const float *__restrict__ partial, int split_k, int64_t count,
                                float *__restrict__ y) {
    const int64_t i4 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (i4 >= count) return;
    if (i4 + 4 <= count && (count & 3) == 0) {
        float4 acc = *reinterpret_cast<const float4 *>(partial + i4);
        for (int s = 1; s < split_k; s++) {
            const float4 v = *reinterpret_cast<const float4 *>(partial + int64_t(s) * count + i4);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        *reinterpret_cast<float4 *>(y + i4) = acc;
    } else {
        for (int64_t i = i4; i < min(count, i4 + 4); i++) {
            float acc = partial[i];
            for (int s = 1; s < split_k; s++) acc += partial[int64_t(s) * count + i];
            y[i] = acc;
        }
    }
}

// ------------------------------------------------------------------ host side

bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
              uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool PAL>
cudaError_t launch_bn(const TcLaunch &p, cudaStream_t stream) {
    using C = Cfg<BN, PAL>;
    int stages = p.stages;
    const int max_stages = (kMaxSmem - 1024 - tail_bytes(8)) / C::kStage;
    if (stages <= 0 || stages > max_stages) stages = max_stages;
    if (stages > 8) stages = 8;
    if (stages < 2) return cudaErrorInvalidValue;
    const size_t smem = size_t(stages) * C::kStage + 1024 + tail_bytes(stages);

    CUtensorMap mx, ma, mb;
    std::memset(&mb, 0, sizeof(mb));
    if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, uint64_t(p.k), uint64_t(p.m),
                  uint64_t(p.k) * 2, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (PAL) {
        if (!make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.w->sm, uint64_t(p.k), uint64_t(p.n),
                      uint64_t(p.k), kBK, kBM, CU_TENSOR_MAP_SWIZZLE_64B) ||
            !make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.pal, uint64_t(p.k / 2), uint64_t(p.n),
                      uint64_t(p.k / 2), kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_32B))
            return cudaErrorInvalidValue;
    } else {
        if (!make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.w_bf16, uint64_t(p.k), uint64_t(p.n),
                      uint64_t(p.k) * 2, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        mb = ma;
    }

    TcArgs a{};
    a.m = p.m;
    a.n = p.n;
    a.k = p.k;
    const int nks = int(p.k / kBK);
    int split = std::max(1, std::min(p.split_k, nks));
    a.ks_per_split = (nks + split - 1) / split;
    split = (nks + a.ks_per_split - 1) / a.ks_per_split;   // no empty slice
    a.split_k = split;
    a.stages = stages;
    a.debug_flags = p.debug_flags;
    a.timeout_ns = p.timeout_ns;
    a.y = p.y;
    a.partial = p.partial;
    a.status = p.dev_status;
    if (PAL) {
        a.flagbits = p.w->flagbits;
        a.rawbase = p.w->rawbase;
        a.rawexp = p.w->rawexp;
        auto pack = [&](int i) {
            return uint32_t(p.w->palette[i]) | uint32_t(p.w->palette[i + 1]) << 8 |
                   uint32_t(p.w->palette[i + 2]) << 16 | uint32_t(p.w->palette[i + 3]) << 24;
        };
        a.pal = Palette16{pack(0), pack(4), pack(8), pack(12)};
    }
    if (split > 1 && !p.partial) return cudaErrorInvalidValue;

    auto kern = k_gemm_tc<BN, PAL>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    // TMEM: co-resident CTAs must fit in 512 columns, or tcgen05.alloc would block
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm * int(C::kTmemCols) > 512) return cudaErrorInvalidConfiguration;

    dim3 grid(unsigned((p.n + kBM - 1) / kBM), unsigned((p.m + BN - 1) / BN), unsigned(split));
    kern<<<grid, kThreads, smem, stream>>>(mx, ma, mb, a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (split > 1) return launch_splitk_reduce(p.partial, split, p.m * p.n, p.y, stream);
    return cudaSuccess;
}

template <bool PAL>
cudaError_t launch_pal(const TcLaunch &p, cudaStream_t stream) {
    switch (p.bn) {
        case 16: return launch_bn<16, PAL>(p, stream);
        case 32: return launch_bn<32, PAL>(p, stream);
        case 64: return launch_bn<64, PAL>(p, stream);
        case 128: return launch_bn<128, PAL>(p, stream);
        case 256: return launch_bn<256, PAL>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_splitk_reduce(const float *partial, int split_k, int64_t count, float *y,
                                 cudaStream_t stream) {
    const int threads = 256;
    const int64_t blocks = (count / 4 + 1 + threads - 1) / threads;
    k_splitk_reduce<<<unsigned(blocks), threads, 0, stream>>>(partial, split_k, count, y);
    return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const TcLaunch &p, cudaStream_t stream) {
    return p.w_bf16 ? launch_pal<false>(p, stream) : launch_pal<true>(p, stream);
}

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

}  // namespace uw
