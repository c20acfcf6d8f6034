// gemm_tc.cu -- tensor-core GEMM Y = X * W^T on sm_100a with tcgen05 MMA and a
// TMEM accumulator, in two flavours that issue the identical MMA sequence (so
// their outputs are bit-identical):
//   * fused: W arrives compressed (4-bit palette plane + sign/mantissa plane +
//     raw groups) and is rebuilt to BF16 in shared memory (Unweight page §七,
//     the reconstructive matmul; §五, decompress on chip, never back to HBM);
//   * plain: W arrives as BF16 through TMA (the uncompressed baseline and the
//     bit-exactness twin of the fused flavour).
//
// CTA tile: 128 rows of W (the MMA "M") x `BN` tokens (the MMA "N"); K in
// steps of 64 (one group).  Grid = (n/128, ceil(m/BN), split_k); split-K
// slices are summed afterwards in a fixed order.
//
// Plain kernel (6 warps): warp 0 TMA producer (X tile + W tile per K-step,
// 128-byte swizzle) into an S-stage ring; warp 1 allocates TMEM and issues 4
// x tcgen05.mma (K = 16) per K-step, tcgen05.commit freeing the stage; warps
// 2-5 read the accumulator (tcgen05.ld) and store Y.
//
// Fused kernel (15 warps), three rings so that no load waits for the MMA and
// no MMA operand waits for a load issued late:
//   compressed ring (CS stages): sign/mantissa tile (64-byte swizzle),
//     palette tile (32-byte swizzle) and the exponents of the tile's raw rows
//     (one 64-byte slot per row); freed as soon as the rebuild has read it;
//   W ring (4 stages for BN <= 64, else 2): rebuilt BF16 W tiles, freed by
//     the MMA's commit.  With one token tile per CTA the ring lives in tensor
//     memory, 32 columns per K-step after the accumulator: each rebuild
//     thread writes its row's 32 BF16 pairs to its lane (tcgen05.st), and
//     the MMA takes A from there, so W never goes through shared memory;
//     with two token tiles the accumulators fill TMEM and the ring is in
//     shared memory (128-byte swizzle, K-major);
//   X ring (8 / 4 / 2 stages): X tiles, freed by the MMA's commit.  With a
//   256-token tile and more than 256 tokens, a CTA owns two token tiles: an
//   X stage holds both, the MMA thread issues each K-step for both against
//   the same rebuilt W stage (two accumulators filling the 512 TMEM
//   columns), so a W tile is rebuilt once per 512 tokens instead of 256.
//   warp 0     compressed tiles: two TMA loads per K-step.
//   warp 1     MMA issuer and TMEM owner.
//   warp 2     X producer (TMA).
//   warps 3-6  raw producers: lane l of warp j owns row 32j + l and copies the
//              row's raw exponents for each raw K-step with 16-byte cp.async,
//              arriving on the stage barrier when they land.
//   warps 7-14 two rebuild groups of 4 warps; group j rebuilds the K-steps
//              ks = j (mod 2), each thread one row (64 weights).  The ring
//              depths are even, so a group only ever touches its own stages
//              and meets their barrier phases strictly in order (a parity wait
//              issued a phase early would pass on the previous phase).  Then
//              all eight read the accumulator back and store Y.
// The raw-group bitmap of the tile's rows is staged in shared memory at start.
// Every wait is bounded; on time-out the kernel raises UW_DEVERR_TIMEOUT,
// stops issuing, waits (bounded) for its copies and MMAs, frees TMEM, returns.
#include <algorithm>
#include <cstring>

#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxSmem = 232448;          // 227 KB opt-in per CTA
constexpr int kPlainThreads = 192;
constexpr int kFusedThreads = (3 + 4) * 32 + 2 * 128;   // producers, MMA, raw producers, 2 rebuild groups
constexpr int kGroups = 2;                // rebuild groups (K-steps alternate between them)

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
    int w_stable;              // fused: planes no kernel writes (loaded before pdl_wait)
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    // pointer arithmetic, not an integer round trip: the result stays
    // recognisably a shared-memory pointer, so accesses through it compile
    // to shared-memory loads and stores rather than generic ones
    return p + ((1024u - (smem_addr(p) & 1023u)) & 1023u);
}

// 4 x tcgen05.mma (K = 16 each) for one 64-wide K-step; A = W tile, B = X tile
template <int BN>
__device__ __forceinline__ void mma_kstep(uint32_t tmem, uint32_t sa, uint32_t sb, bool first) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
#pragma unroll
    for (int kk = 0; kk < kBK / 16; kk++)
        tc_mma_bf16(tmem, smem_desc_k128(sa + 32 * kk), smem_desc_k128(sb + 32 * kk), idesc,
                    (!first || kk) ? 1u : 0u);
}

// Accumulator -> Y (or this split's slice of the partial sums).  Warp with
// TMEM lane quarter q reads rows q*32..q*32+31; `slot` of `nslots` warps per
// quarter take interleaved 16-column chunks.
template <int BN>
__device__ __forceinline__ void store_accumulator(uint32_t tmem, int q, int slot, int nslots, int lane,
                                                  int64_t n0, int64_t m0, int split, const TcArgs &a) {
    const int64_t row = n0 + q * 32 + lane;
    float *out = a.split_k > 1 ? a.partial + int64_t(split) * a.m * a.n : a.y;
#pragma unroll 1
    for (int c0 = 16 * slot; c0 < BN; c0 += 16 * nslots) {
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

// ============================================================== plain kernel

template <int BN>
struct PlainCfg {
    static constexpr int kW = kBM * kBK * 2;
    static constexpr int kX = BN * kBK * 2;
    static constexpr int kStage = kW + kX;
    static constexpr uint32_t kTmemCols = BN < 32 ? 32u : uint32_t(BN);
    static_assert(kStage % 1024 == 0, "stage tiles must keep 1024-byte alignment");
};

__host__ __device__ constexpr int plain_tail(int stages) { return (2 * stages + 2) * 8 + 16; }

template <int BN>
__global__ void __launch_bounds__(kPlainThreads, 1)
    k_gemm_tc_plain(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const TcArgs a) {
    using C = PlainCfg<BN>;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *tiles = align1024(smem_dyn);
    const int S = a.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(tiles + size_t(S) * C::kStage);
    uint64_t *empty = full + S;
    uint64_t *accf = empty + S;
    uint64_t *never = accf + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(never + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();   // W may be the output of the kernel before (a decode)
    const int64_t n0 = int64_t(blockIdx.x) * kBM;
    const int64_t m0 = int64_t(blockIdx.y) * BN;
    const int split = blockIdx.z;
    const int ks_begin = split * a.ks_per_split;
    const int nks = max(0, min(int(a.k / kBK) - ks_begin, a.ks_per_split));
    const uint64_t T = a.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(never, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmW);
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
        if (lane == 0) {
            int issued = 0;
            for (int ks = 0; ks < nks; ks++) {
                const int s = ks % S;
                if (ks >= S && !mbar_wait(&empty[s], (uint32_t(ks / S) & 1u) ^ 1u, T)) {
                    flag_error(a.status, UW_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int kg = ks_begin + ks;
                uint8_t *st = tiles + size_t(s) * C::kStage;
                mbar_arrive_expect_tx(&full[s], uint32_t(C::kX + C::kW));
                tma_load_2d(st + C::kW, &tmX, kg * kBK, int32_t(m0), &full[s]);
                tma_load_2d(st, &tmW, kg * kBK, int32_t(n0), &full[s]);
                issued = ks + 1;
            }
            for (int ks = max(0, issued - S); ks < issued; ks++)
                mbar_wait(&full[ks % S], uint32_t(ks / S) & 1u, T);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            bool ok = true;
            if (a.debug_flags & UW_DEBUG_NEVER_ARRIVE) ok = mbar_wait(never, 0, T);
            for (int ks = 0; ks < nks && ok; ks++) {
                const int s = ks % S;
                ok = mbar_wait(&full[s], uint32_t(ks / S) & 1u, T);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sa = smem_addr(tiles + size_t(s) * C::kStage);
                mma_kstep<BN>(tmem, sa, sa + C::kW, ks == 0);
                tc_commit(&empty[s]);
            }
            if (!ok) {
                flag_error(a.status, UW_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            tc_commit(accf);
        }
        __syncwarp();
    } else {
        const bool ok = mbar_wait(accf, 0, T);
        tc_fence_after();
        const bool skip = __any_sync(0xFFFFFFFFu, !ok || *abort_flag != 0 || nks == 0);
        if (!ok && lane == 0) flag_error(a.status, UW_DEVERR_TIMEOUT);
        if (!skip) store_accumulator<BN>(tmem, warp & 3, 0, 1, lane, n0, m0, split, a);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ============================================================== fused kernel

template <int BN, int TT>   // TT: token tiles per CTA sharing each rebuilt W tile
struct FusedCfg {
    static constexpr int kWS = BN <= 64 ? 4 : 2;        // rebuilt-W ring (multiple of kGroups)
    static constexpr int kXS = BN <= 64 ? 8 : (BN == 128 ? 4 : 2);   // X ring
    static constexpr int kW = kBM * kBK * 2;            // rebuilt W tile
    static constexpr int kX = BN * kBK * 2;             // X tile
    static constexpr int kXT = TT * kX;                 // X ring stage: TT token tiles
    static constexpr int kSM = kBM * kBK;               // sign/mantissa tile
    static constexpr int kPL = kBM * kBK / 2;           // palette tile
    static constexpr int kRAW = kBM * kGroup;           // raw exponents, one 64-byte slot per row
    static constexpr int kCStage = kSM + kPL + kRAW;    // compressed ring stage
    static constexpr int kOffPL = kSM, kOffRAW = kSM + kPL;
    // one token tile per CTA: the rebuilt W ring lives in tensor memory (32
    // columns per K-step after the accumulator) and the MMA takes A from
    // there; with two token tiles the accumulators fill TMEM and W stays in
    // shared memory
    static constexpr bool kWInTmem = TT == 1;
    static constexpr uint32_t kAccCols = BN < 32 ? 32u : uint32_t(BN);
    static constexpr uint32_t kWCol0 = kAccCols;                      // first W column (TMEM ring)
    static constexpr uint32_t kTmemUsed = kWInTmem ? kAccCols + uint32_t(kWS) * 32u : uint32_t(TT) * kAccCols;
    static constexpr uint32_t kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                        : kTmemUsed <= 256 ? 256 : 512;
    static constexpr int kWSmem = kWInTmem ? 0 : kWS * kW;              // W ring bytes in shared memory
    static_assert(kW % 1024 == 0 && kX % 1024 == 0 && kCStage % 1024 == 0, "1024-byte alignment");
    static_assert(kTmemUsed <= 512, "accumulators and W ring exceed TMEM");
    static_assert(kWCol0 >= uint32_t(BN), "the W ring starts after the accumulator");
};

constexpr int kRawProducers = 4;      // warps; lane l of warp j owns tile row 32 j + l

// after the rings: raw bitmap (128 rows x bw words), first raw rank per row,
// barriers (c_full, c_empty per compressed stage; w_full, w_empty per W stage;
// x_full, x_empty per X stage; accf, never), TMEM slot, abort flag
__host__ __device__ constexpr int fused_tail(int cs, int ws, int xs, int bw) {
    return kBM * bw * 4 + kBM * 4 + (2 * cs + 2 * ws + 2 * xs + 2) * 8 + 16;
}

template <int BN, int TT>
__global__ void __launch_bounds__(kFusedThreads, 1)
    k_gemm_tc_fused(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmSM,
                    const __grid_constant__ CUtensorMap tmPL, const TcArgs a, int bw) {
    using C = FusedCfg<BN, TT>;
    constexpr int WS = C::kWS, XS = C::kXS;
    extern __shared__ uint8_t smem_dyn[];
    uint8_t *wring = align1024(smem_dyn);
    uint8_t *xring = wring + C::kWSmem;
    uint8_t *cring = xring + XS * C::kXT;
    const int CS = a.stages;                      // compressed stages (even)
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(cring + size_t(CS) * C::kCStage);   // [128][bw]
    uint32_t *rank0 = bitmap + kBM * bw;                                                // [128]
    uint64_t *c_full = reinterpret_cast<uint64_t *>(rank0 + kBM);
    uint64_t *c_empty = c_full + CS;
    uint64_t *w_full = c_empty + CS;
    uint64_t *w_empty = w_full + WS;
    uint64_t *x_full = w_empty + WS;
    uint64_t *x_empty = x_full + XS;
    uint64_t *accf = x_empty + XS;
    uint64_t *never = accf + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(never + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the next kernel on the stream may be scheduled now; with planes no
    // kernel writes, the compressed tiles, the raw bitmap and the raw
    // exponents are loaded before waiting for the previous kernel, X (and
    // every write) only after it
    pdl_trigger();
    if (!a.w_stable) pdl_wait();
    const int64_t n0 = int64_t(blockIdx.x) * kBM;
    const int64_t m0 = int64_t(blockIdx.y) * BN * TT;
    const int split = blockIdx.z;
    const int ks_begin = split * a.ks_per_split;
    const int nks = max(0, min(int(a.k / kBK) - ks_begin, a.ks_per_split));
    const uint64_t T = a.timeout_ns;
    constexpr int kFirstRebuildWarp = 3 + kRawProducers;

    if (threadIdx.x == 0) {
        for (int s = 0; s < CS; s++) {
            mbar_init(&c_full[s], 1 + 32 * kRawProducers);   // TMA producer + raw-producer lanes
            mbar_init(&c_empty[s], 128);
        }
        for (int s = 0; s < WS; s++) {
            mbar_init(&w_full[s], 128);
            mbar_init(&w_empty[s], 1);
        }
        for (int s = 0; s < XS; s++) {
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(never, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmSM);
        prefetch_tensormap(&tmPL);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp >= kFirstRebuildWarp) {
        // raw-group bitmap of the tile's rows over this split's K-steps (word j
        // of row r holds K-steps 32j..32j+31) and each row's first raw rank
        const int t = threadIdx.x - 32 * kFirstRebuildWarp, r = t & (kBM - 1), part = t >> 7;   // part 0..1
        const int64_t row = n0 + r;
        const int64_t gpr = a.k / kGroup;
        const int64_t nflag = (a.n * gpr + 31) >> 5;
        const int64_t g0 = row * gpr + ks_begin;
        for (int j = part; j < bw; j += 2) {
            uint32_t bits = 0u;
            const int base = 32 * j;
            if (row < a.n && base < nks) {
                const int64_t gb = g0 + base;
                const int64_t w = gb >> 5;
                const uint32_t lo = __ldg(a.flagbits + w);
                const uint32_t hi = w + 1 < nflag ? __ldg(a.flagbits + w + 1) : 0u;
                bits = __funnelshift_r(lo, hi, uint32_t(gb & 31));
                const int valid = nks - base;
                if (valid < 32) bits &= (1u << valid) - 1u;
            }
            bitmap[r * bw + j] = bits;
        }
        if (part == 0) {
            uint32_t rk = 0u;
            if (row < a.n && nks > 0) {
                const uint32_t fw = __ldg(a.flagbits + (g0 >> 5));
                rk = __ldg(a.rawbase + (g0 >> 5)) + __popc(fw & ((1u << (g0 & 31)) - 1u));
            }
            rank0[r] = rk;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ compressed tiles (TMA)
        if (lane == 0) {
            int issued = 0;
            for (int ks = 0; ks < nks; ks++) {
                const int s = ks % CS;
                if (ks >= CS && !mbar_wait(&c_empty[s], (uint32_t(ks / CS) & 1u) ^ 1u, T)) {
                    flag_error(a.status, UW_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int kg = ks_begin + ks;
                uint8_t *st = cring + size_t(s) * C::kCStage;
                mbar_arrive_expect_tx(&c_full[s], uint32_t(C::kSM + C::kPL));
                tma_load_2d(st, &tmSM, kg * kBK, int32_t(n0), &c_full[s]);
                tma_load_2d(st + C::kOffPL, &tmPL, kg * (kBK / 2), int32_t(n0), &c_full[s]);
                issued = ks + 1;
            }
            for (int ks = max(0, issued - CS); ks < issued; ks++)
                mbar_wait(&c_full[ks % CS], uint32_t(ks / CS) & 1u, T);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            if (a.debug_flags & UW_DEBUG_NEVER_ARRIVE) ok = mbar_wait(never, 0, T);
            for (int ks = 0; ks < nks && ok; ks++) {
                const int ws = ks % WS, xs = ks % XS;
                ok = mbar_wait(&x_full[xs], uint32_t(ks / XS) & 1u, T) &&
                     mbar_wait(&w_full[ws], uint32_t(ks / WS) & 1u, T);
                if (!ok) break;
                tc_fence_after();
                if constexpr (C::kWInTmem) {
                    constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
                    const uint32_t a0 = tmem + C::kWCol0 + uint32_t(ws) * 32u;
                    const uint32_t sb = smem_addr(xring + size_t(xs) * C::kXT);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; kk++)   // 8 columns = 16 K per MMA
                        tc_mma_bf16_ta(tmem, a0 + 8u * kk, smem_desc_k128(sb + 32 * kk), idesc,
                                       (ks != 0 || kk) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int t = 0; t < TT; t++)
                        mma_kstep<BN>(tmem + uint32_t(t * BN), smem_addr(wring + size_t(ws) * C::kW),
                                      smem_addr(xring + size_t(xs) * C::kXT + size_t(t) * C::kX), ks == 0);
                }
                tc_commit(&w_empty[ws]);
                tc_commit(&x_empty[xs]);
            }
            if (!ok) {
                flag_error(a.status, UW_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            tc_commit(accf);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ X producer
        if (lane == 0) {
            pdl_wait();
            int issued = 0;
            for (int ks = 0; ks < nks; ks++) {
                const int s = ks % XS;
                if (ks >= XS && !mbar_wait(&x_empty[s], (uint32_t(ks / XS) & 1u) ^ 1u, T)) {
                    flag_error(a.status, UW_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(&x_full[s], uint32_t(C::kXT));
#pragma unroll
                for (int t = 0; t < TT; t++)   // a tile past the last token reads the zero fill
                    tma_load_2d(xring + size_t(s) * C::kXT + size_t(t) * C::kX, &tmX, (ks_begin + ks) * kBK,
                                int32_t(m0 + t * BN), &x_full[s]);
                issued = ks + 1;
            }
            for (int ks = max(0, issued - XS); ks < issued; ks++)
                mbar_wait(&x_full[ks % XS], uint32_t(ks / XS) & 1u, T);
        }
        __syncwarp();
    } else if (warp < kFirstRebuildWarp) {
        // ------------------------------------------------ raw producers
        // lane owns row r; for every K-step it copies the row's raw exponents
        // (64 B, four 16-byte cp.async) into the stage when the group is raw,
        // and always arrives on c_full once its copies have landed
        const int r = 32 * (warp - 3) + lane;
        const uint32_t *bm = bitmap + r * bw;
        uint32_t rank = rank0[r];
        bool ok = true;
        for (int ks = 0; ks < nks; ks++) {
            const int s = ks % CS;
            if (ks >= CS) ok = mbar_wait(&c_empty[s], (uint32_t(ks / CS) & 1u) ^ 1u, T);
            if (!ok || *abort_flag) break;
            if ((bm[ks >> 5] >> (ks & 31)) & 1u) {
                const uint8_t *src = a.rawexp + uint64_t(rank) * kGroup;
                uint8_t *dst = cring + size_t(s) * C::kCStage + C::kOffRAW + r * kGroup;
#pragma unroll
                for (int c = 0; c < 4; c++) cp_async16(dst + 16 * c, src + 16 * c);
                rank++;
            }
            cp_async_mbar_arrive_noinc(&c_full[s]);
        }
        if (!ok) flag_error(a.status, UW_DEVERR_TIMEOUT);
        cp_async_wait_all();
    } else {
        // ------------------------------------------------ rebuild groups, then epilogue
        const int wi = warp - kFirstRebuildWarp;  // 0..7
        const int q = warp & 3;               // TMEM lane quarter this warp may access
        const int grp = wi >> 2;              // 0 or 1: K-steps ks = grp (mod 2)
        const int r = q * 32 + lane;          // tile row
        const int sw64 = (r >> 1) & 3, sw32 = (r >> 2) & 1, sw128 = r & 7;
        const uint32_t *bm = bitmap + r * bw;
        for (int ks = grp; ks < nks; ks += kGroups) {
            const int cs = ks % CS, ws = ks % WS;
            bool ok = mbar_wait(&c_full[cs], uint32_t(ks / CS) & 1u, T);
            if (ok && ks >= WS) ok = mbar_wait(&w_empty[ws], (uint32_t(ks / WS) & 1u) ^ 1u, T);
            if (!ok) {
                flag_error(a.status, UW_DEVERR_TIMEOUT);
                break;
            }
            const uint8_t *st = cring + size_t(cs) * C::kCStage;
            const uint8_t *smrow = st + r * 64;
            const uint8_t *plrow = st + C::kOffPL + r * 32;
            uint8_t *wrow = wring + size_t(ws) * C::kW + r * 128;
            const bool raw = (bm[ks >> 5] >> (ks & 31)) & 1u;
            uint32_t wv[32];                   // TMEM ring: BF16 pairs of the row in K order
            if constexpr (C::kWInTmem) tc_fence_after();   // the slot's previous MMAs are done
#pragma unroll
            for (int h = 0; h < 2; h++) {      // two halves of the row, 32 weights each
                const uint4 s0 = *reinterpret_cast<const uint4 *>(smrow + (((2 * h) ^ sw64) << 4));
                const uint4 s1 = *reinterpret_cast<const uint4 *>(smrow + (((2 * h + 1) ^ sw64) << 4));
                uint32_t rv[8];
                if (raw) {
                    const uint8_t *rp = st + C::kOffRAW + r * kGroup + h * 32;
                    const uint4 e0 = *reinterpret_cast<const uint4 *>(rp);
                    const uint4 e1 = *reinterpret_cast<const uint4 *>(rp + 16);
                    rv[0] = rot4(e0.x); rv[1] = rot4(e0.y); rv[2] = rot4(e0.z); rv[3] = rot4(e0.w);
                    rv[4] = rot4(e1.x); rv[5] = rot4(e1.y); rv[6] = rot4(e1.z); rv[7] = rot4(e1.w);
                } else {
                    const uint4 p = *reinterpret_cast<const uint4 *>(plrow + ((h ^ sw32) << 4));
                    pal_rot(p.x, a.pal, rv[0], rv[1]);
                    pal_rot(p.y, a.pal, rv[2], rv[3]);
                    pal_rot(p.z, a.pal, rv[4], rv[5]);
                    pal_rot(p.w, a.pal, rv[6], rv[7]);
                }
                const int c0 = 4 * h;
                const uint4 o0 = join8(rv[0], rv[1], s0.x, s0.y), o1 = join8(rv[2], rv[3], s0.z, s0.w);
                const uint4 o2 = join8(rv[4], rv[5], s1.x, s1.y), o3 = join8(rv[6], rv[7], s1.z, s1.w);
                if constexpr (C::kWInTmem) {
                    const uint4 o[4] = {o0, o1, o2, o3};
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        wv[16 * h + 4 * c + 0] = o[c].x;
                        wv[16 * h + 4 * c + 1] = o[c].y;
                        wv[16 * h + 4 * c + 2] = o[c].z;
                        wv[16 * h + 4 * c + 3] = o[c].w;
                    }
                } else {
                    *reinterpret_cast<uint4 *>(wrow + (((c0 + 0) ^ sw128) << 4)) = o0;
                    *reinterpret_cast<uint4 *>(wrow + (((c0 + 1) ^ sw128) << 4)) = o1;
                    *reinterpret_cast<uint4 *>(wrow + (((c0 + 2) ^ sw128) << 4)) = o2;
                    *reinterpret_cast<uint4 *>(wrow + (((c0 + 3) ^ sw128) << 4)) = o3;
                }
            }
            if constexpr (C::kWInTmem) {
                // the warp writes its 32 rows (lanes 32 q ..) of the slot's 32 columns
                __syncwarp();
                tmem_st32(tmem + (uint32_t(q * 32) << 16) + C::kWCol0 + uint32_t(ws) * 32u, wv);
                tmem_st_wait();
                tc_fence_before();
            } else {
                fence_proxy_async_smem();
            }
            mbar_arrive(&c_empty[cs]);
            mbar_arrive(&w_full[ws]);
        }
        const bool ok = mbar_wait(accf, 0, T);
        tc_fence_after();
        const bool skip = __any_sync(0xFFFFFFFFu, !ok || *abort_flag != 0 || nks == 0);
        if (!ok && lane == 0) flag_error(a.status, UW_DEVERR_TIMEOUT);
        pdl_wait();   // (returns at once: X was read after it)
        if (!skip)
#pragma unroll 1
            for (int t = 0; t < TT; t++)
                if (m0 + t * BN < a.m)
                    store_accumulator<BN>(tmem + uint32_t(t * BN), q, grp, kGroups, lane, n0, m0 + t * BN, split, a);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ============================================================== split-K reduce

__global__ void k_splitk_reduce(const float *__restrict__ partial, int split_k, int64_t count,
                                float *__restrict__ y) {
    pdl_trigger();
    pdl_wait();   // the partials are the previous kernel's output
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

// ============================================================== host side

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

// K split into slices of whole K-steps, none empty
void split_k_slices(const TcLaunch &p, TcArgs &a) {
    const int nks = int(p.k / kBK);
    int split = std::max(1, std::min(p.split_k, nks));
    a.ks_per_split = (nks + split - 1) / split;
    a.split_k = (nks + a.ks_per_split - 1) / a.ks_per_split;
}

// one-time per (kernel, device, stage count): shared-memory opt-in and a check
// that co-resident CTAs fit the 512 TMEM columns (tcgen05.alloc would block)
template <class K>
cudaError_t prepare(K kern, int threads, size_t smem, uint32_t tmem_cols, int key, int (&ready)[16]) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (ready[key] == dev) return cudaSuccess;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm * int(tmem_cols) > 512) return cudaErrorInvalidConfiguration;
    ready[key] = dev;
    return cudaSuccess;
}

template <int BN>
cudaError_t launch_plain(const TcLaunch &p, cudaStream_t stream) {
    using C = PlainCfg<BN>;
    const int max_stages = std::min(8, (kMaxSmem - 1024 - plain_tail(8)) / C::kStage);
    // default depth 4: deeper rings measured slower (more outstanding TMA
    // loads per SM than HBM serves efficiently), 2 too shallow
    int stages = p.stages <= 0 ? std::min(4, max_stages) : std::min(p.stages, max_stages);
    if (stages < 2) return cudaErrorInvalidValue;
    const size_t smem = size_t(stages) * C::kStage + 1024 + plain_tail(stages);
    CUtensorMap mx, mw;
    if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, uint64_t(p.k), uint64_t(p.m), uint64_t(p.k) * 2,
                  kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.w_bf16, uint64_t(p.k), uint64_t(p.n),
                  uint64_t(p.k) * 2, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    TcArgs a{};
    a.m = p.m;
    a.n = p.n;
    a.k = p.k;
    split_k_slices(p, a);
    a.stages = stages;
    a.debug_flags = p.debug_flags;
    a.timeout_ns = p.timeout_ns;
    a.y = p.y;
    a.partial = p.partial;
    a.status = p.dev_status;
    if (a.split_k > 1 && !p.partial) return cudaErrorInvalidValue;
    static thread_local int ready[16] = {-1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1};
    cudaError_t err = prepare(k_gemm_tc_plain<BN>, kPlainThreads, smem, C::kTmemCols, stages, ready);
    if (err != cudaSuccess) return err;
    dim3 grid(unsigned((p.n + kBM - 1) / kBM), unsigned((p.m + BN - 1) / BN), unsigned(a.split_k));
    err = launch_pdl(false, k_gemm_tc_plain<BN>, grid, dim3(kPlainThreads), smem, stream, mx, mw, a);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (a.split_k > 1) return launch_splitk_reduce(p.partial, a.split_k, p.m * p.n, p.y, stream);
    return cudaSuccess;
}

template <int BN, int TT>
cudaError_t launch_fused(const TcLaunch &p, cudaStream_t stream) {
    using C = FusedCfg<BN, TT>;
    TcArgs a{};
    a.m = p.m;
    a.n = p.n;
    a.k = p.k;
    split_k_slices(p, a);
    const int bw = (a.ks_per_split + 31) / 32;     // raw bitmap words per row
    const int fixed = C::kWSmem + C::kXS * C::kXT + 1024 + fused_tail(8, C::kWS, C::kXS, bw);
    int max_cs = (kMaxSmem - fixed) / C::kCStage;
    max_cs = std::min(8, max_cs) & ~1;      // even: each rebuild group owns every other stage
    int cs = (p.stages <= 0 || p.stages > max_cs) ? max_cs : (p.stages & ~1);
    if (cs < 2) return cudaErrorInvalidValue;
    const size_t smem = size_t(C::kWSmem) + size_t(C::kXS) * C::kXT + size_t(cs) * C::kCStage + 1024 +
                        fused_tail(cs, C::kWS, C::kXS, bw);
    CUtensorMap mx, msm, mpl;
    if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, uint64_t(p.k), uint64_t(p.m), uint64_t(p.k) * 2,
                  kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&msm, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.w->sm, uint64_t(p.k), uint64_t(p.n), uint64_t(p.k),
                  kBK, kBM, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&mpl, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.pal, uint64_t(p.k / 2), uint64_t(p.n),
                  uint64_t(p.k / 2), kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    a.stages = cs;
    a.debug_flags = p.debug_flags;
    a.timeout_ns = p.timeout_ns;
    a.y = p.y;
    a.partial = p.partial;
    a.status = p.dev_status;
    a.flagbits = p.w->flagbits;
    a.rawbase = p.w->rawbase;
    a.rawexp = p.w->rawexp;
    a.pal = make_palette16(p.w->palette);
    a.w_stable = p.w_stable ? 1 : 0;
    if (a.split_k > 1 && !p.partial) return cudaErrorInvalidValue;
    static thread_local int ready[16] = {-1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1};
    cudaError_t err = prepare(k_gemm_tc_fused<BN, TT>, kFusedThreads, smem, C::kTmemCols, cs, ready);
    if (err != cudaSuccess) return err;
    dim3 grid(unsigned((p.n + kBM - 1) / kBM), unsigned((p.m + BN * TT - 1) / (BN * TT)), unsigned(a.split_k));
    err = launch_pdl(a.w_stable != 0, k_gemm_tc_fused<BN, TT>, grid, dim3(kFusedThreads), smem, stream, mx, msm, mpl,
                     a, bw);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (a.split_k > 1) return launch_splitk_reduce(p.partial, a.split_k, p.m * p.n, p.y, stream);
    return cudaSuccess;
}

template <int BN>
cudaError_t launch_bn(const TcLaunch &p, cudaStream_t stream) {
    if (p.w_bf16) return launch_plain<BN>(p, stream);
    // more than one 256-token tile: two tiles per CTA share each rebuilt W
    // tile (the two accumulators fill TMEM), halving the rebuild work; every
    // accumulator sees the same MMA sequence, so the result bits do not change
    if (BN == 256 && p.m > BN) return launch_fused<BN, 2>(p, stream);
    return launch_fused<BN, 1>(p, stream);
}

}  // namespace

cudaError_t launch_splitk_reduce(const float *partial, int split_k, int64_t count, float *y,
                                 cudaStream_t stream) {
    const int threads = 256;
    const int64_t blocks = (count / 4 + 1 + threads - 1) / threads;
    const cudaError_t err = launch_pdl(false, k_splitk_reduce, dim3(unsigned(blocks)), dim3(threads), 0, stream,
                                       partial, split_k, count, y);
    return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_gemm_tc(const TcLaunch &p, cudaStream_t stream) {
    switch (p.bn) {
        case 16: return launch_bn<16>(p, stream);
        case 32: return launch_bn<32>(p, stream);
        case 64: return launch_bn<64>(p, stream);
        case 128: return launch_bn<128>(p, stream);
        case 256: return launch_bn<256>(p, stream);
        default: return cudaErrorInvalidValue;
    }
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
