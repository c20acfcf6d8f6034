// gemv_sk.cu -- persistent stream-K form of the warp-MMA skinny matmul
// Y = X * W^T for m <= 16 tokens (Unweight page §七, the reconstructive
// matmul, in the small-batch regime of §十 where the job is an HBM stream).
//
// Why a second form of the warp-MMA kernel.  The one-tile-per-CTA form
// (gemv_mma.cu) keeps the next steps' loads in flight in a register ring,
// about 3 KB per warp, so at the occupancy that ring allows an SM has a few
// tens of KB of W requested at any time, which at HBM's loaded latency caps
// the stream well below the HBM peak; and an 8B gate projection's 896 tiles
// make two full waves of CTAs plus a nearly empty third one.  Here:
//  - one lane of the warp loads each unit's compressed W and the chunk's X
//    rows into the warp's shared-memory ring with 2-D TMA boxes (16 rows x
//    128 sign/mantissa bytes, 16 rows x 64 palette bytes, m rows x 128 X
//    values), completing on one mbarrier per ring slot, so a ring of several
//    units per warp costs no registers and next to no instructions, an SM
//    keeps ~100 KB in flight, and the MMAs never wait on X from L2;
//  - one CTA per SM of `S` warps, and every warp of the grid owns an equal
//    contiguous run of units (16-row tile, 128-wide K chunk), in tile-major
//    order, so every warp streams the same number of bytes: no tail wave;
//  - a tile cut between warps is finished by the warp that completes its
//    last piece: each piece's fp32 MMA fragments go to the workspace, an
//    atomic counter per tile counts the pieces, and the warp that brings it
//    to the number of pieces adds them in warp order (= K order), so the
//    result does not depend on timing, and zeroes each piece after reading
//    it, so that a completed call leaves its whole scratch (counters and
//    pieces) zero.  No warp ever waits for another one: a warp waits only
//    on its own ring slots' barriers (for the boxes its own lane issued)
//    and on its lanes' own copies; there are no CTA-wide barriers.
// Per unit, lane (g, c) = (lane / 4, lane % 4) handles rows g and g + 8 of
// the tile and weights [32c, 32c + 32) of the chunk, with the same fragment
// map as the one-tile kernel at 32 weights per lane (MMA K-step j, thread c,
// K slots {2c, 2c+1, 2c+8, 2c+9} <- weights 32c + 4j + {0, 1, 2, 3}; X uses
// the same map, so every product is formed once).  The boxes land densely
// (row-major) in the slot.  A raw group's 32 exponents of a lane's quarter
// are copied by that lane itself with cp.async from the raw plane (raw groups
// are rare and scattered); the warp learns which groups are raw from one
// bitmap lookup per lane and a ballot.  Every wait on a slot's barrier is
// bounded: on time-out the kernel raises UW_DEVERR_TIMEOUT, stops issuing,
// waits (bounded) for the boxes it has issued and returns.  The fused and
// plain kernels differ only in the W boxes and the rebuild, so their outputs
// are bit-identical.
#include <algorithm>
#include <mutex>

#include "device_common.cuh"
#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

using namespace dev;

constexpr int kRows = 16;                      // W rows per tile (the MMA's M)
constexpr int kChunkK = 128;                   // weights along K per unit
constexpr int kMaxWarps = 16;
constexpr int kMaxStages = 8;
constexpr int kMaxSmem = 227 * 1024;

struct SkArgs {
    const uint16_t *x;         // [m, k] BF16
    const uint16_t *w_bf16;    // plain: [n, k] BF16
    const uint8_t *sm;         // fused: sign/mantissa plane
    const uint8_t *pal;        // fused: 4-bit plane
    const uint32_t *flagbits;  // fused: raw-group bitmap
    const uint32_t *rawbase;   // fused: raw groups before each bitmap word
    const uint8_t *rawexp;     // fused: exponents of the raw groups
    Palette16 palette;
    int64_t n, k;
    int64_t cpr;               // chunks per row (k / 128)
    int64_t units;             // tiles * cpr
    int64_t warps;             // warps of the grid that own units (<= units)
    float *y;                  // [m, n]
    float *partial;            // [2 * warps][NT][32 lanes][4] fp32 fragments
    uint32_t *counters;        // [tiles], zero between calls
    int m;
    int stages;                // ring slots per warp (2..8)
    int slot_bytes;            // bytes of one ring slot (W and the chunk's X rows)
    int w_stable;              // fused: planes no kernel writes (read before pdl_wait)
    uint32_t *status;          // device error word (UW_DEVERR_*), may be null
    uint64_t timeout_ns;       // bound of every barrier wait
};

// first unit of warp w
__device__ __forceinline__ int64_t unit0(int64_t w, int64_t units, int64_t warps) { return w * units / warps; }
// the warp whose run holds unit u (every run is non-empty: warps <= units)
__device__ __forceinline__ int64_t owner(int64_t u, int64_t units, int64_t warps) {
    return ((u + 1) * warps - 1) / units;
}

__device__ __forceinline__ void cp16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most n of this thread's copy groups are still in flight
__device__ __forceinline__ void cp_wait(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
        case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    }
}
// 16-byte load from the ring (a plain load through a pointer into shared
// memory: the compiler keeps it after the copy waits and warp barriers,
// which clobber memory, and schedules it freely against the arithmetic and
// MMAs around it)
__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t w4(const uint4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// Byte offsets inside a ring slot (every region 128-byte aligned, the TMA
// boxes dense):
//  - fused: the 16 rows' sign/mantissa bytes at r * 128 (one box), their
//    palette bytes at kPalOff + r * 64 (one box), and the exponents of a
//    lane's raw quarters at kRawOff + r * 128 + 32 c (copied by that lane);
//  - plain: the 16 rows' BF16 weights at r * 256 (one box);
//  - both: the chunk's m X rows at kXOff + r * 256 (one box).
// A ring slot is followed, after all warps' rings, by one mbarrier per slot.
constexpr int kPalOff = 16 * 128;
constexpr int kRawOff = kPalOff + 16 * 64;
constexpr int kXOff = kRawOff + 16 * 128;
__host__ __device__ constexpr int slot_bytes(int xrows) { return kXOff + xrows * 256; }

// One row's 32 weights (quarter c of the chunk) from a ring slot: its
// sign/mantissa words sm[i] (weights 4i .. 4i + 3) and the rotated exponent
// bytes of the same weights e[i].  `sm0`, `sm1`: the row's two sign/mantissa
// pieces of the quarter (the same offsets inside the raw region hold its raw
// exponents); `pal`: its palette piece.
__device__ __forceinline__ void row_words(const uint8_t *slot, uint32_t sm0, uint32_t sm1, uint32_t pal, bool raw,
                                          const Palette16 &P, uint32_t (&sm)[8], uint32_t (&e)[8]) {
    const uint4 s0 = lds128(slot + sm0), s1 = lds128(slot + sm1);
    sm[0] = s0.x; sm[1] = s0.y; sm[2] = s0.z; sm[3] = s0.w;
    sm[4] = s1.x; sm[5] = s1.y; sm[6] = s1.z; sm[7] = s1.w;
    if (raw) {
        const uint4 b0 = lds128(slot + kRawOff + sm0), b1 = lds128(slot + kRawOff + sm1);
#pragma unroll
        for (int i = 0; i < 4; i++) e[i] = rot4(w4(b0, i));
#pragma unroll
        for (int i = 0; i < 4; i++) e[4 + i] = rot4(w4(b1, i));
    } else {
        const uint4 b0 = lds128(slot + pal);
#pragma unroll
        for (int i = 0; i < 4; i++) pal_rot(w4(b0, i), P, e[2 * i], e[2 * i + 1]);
    }
}

template <bool PAL, int NT>   // NT: 8-token tiles (1: m <= 8, 2: m <= 16)
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
    k_gemv_sk(const __grid_constant__ CUtensorMap tmW,   // fused: sign/mantissa plane; plain: BF16 W
              const __grid_constant__ CUtensorMap tmP,   // fused: 4-bit plane (plain: unused)
              const __grid_constant__ CUtensorMap tmX, const SkArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int S = blockDim.x >> 5;
    // the next kernel on the stream may be scheduled now
    pdl_trigger();
    const int64_t gw = int64_t(blockIdx.x) * S + warp;
    if (gw >= a.warps) return;   // the last CTA's spare warps
    const int64_t u_begin = unit0(gw, a.units, a.warps), u_end = unit0(gw + 1, a.units, a.warps);
    const int nu = int(u_end - u_begin);
    // with planes no kernel writes, W is requested before the previous
    // kernel on the stream has ended, X only after it
    const bool defer_x = a.w_stable != 0;
    if (!defer_x) pdl_wait();

    const int stages = a.stages, slot_b = a.slot_bytes, xrows = a.m;
    // the rings start 128-byte aligned (TMA destinations), the barriers follow
    uint8_t *base = smem + ((128u - (smem_addr(smem) & 127u)) & 127u);
    uint8_t *ring = base + warp * stages * slot_b;
    uint64_t *full = reinterpret_cast<uint64_t *>(base + S * stages * slot_b) + warp * stages;
    const uint32_t k = uint32_t(a.k), gpr = k / 64;
    const int cpr = int(a.cpr);
    const Palette16 P = a.palette;
    const uint64_t T = a.timeout_ns;
    if (lane == 0) {
        for (int s = 0; s < stages; s++) mbar_init(&full[s], 1);
        fence_mbar_init();
        prefetch_tensormap(&tmW);
        if (PAL) prefetch_tensormap(&tmP);
        prefetch_tensormap(&tmX);
    }
    __syncwarp();

    // Element offsets below are 32-bit (n * k < 2^32 is checked at launch).
    // Raw flags: lane l looks up row l / 2, group l % 2 of the unit's chunk.
    const uint32_t lc_flag = uint32_t(lane >> 1) * gpr + uint32_t(lane & 1);
    // consumer side (lane constants): rows g and g + 8, quarter c
    const int fbit_a = 2 * g + (c >> 1), fbit_b = 2 * (g + 8) + (c >> 1);
    const uint32_t o_sm0 = uint32_t(g * 128 + c * 32), o_sm1 = o_sm0 + 16;
    const uint32_t o_pal = uint32_t(kPalOff + g * 64 + c * 16);
    const uint32_t o_bfa = uint32_t(g * 256 + c * 64), o_bfb = o_bfa + 8 * 256;
    // X token rows of this lane (clamped: columns >= m are not stored)
    const uint32_t o_xa = uint32_t(kXOff + min(g, xrows - 1) * 256 + c * 64);
    const uint32_t o_xb = uint32_t(kXOff + min(g + 8, xrows - 1) * 256 + c * 64);
    const uint32_t w_bytes = PAL ? 16 * 128 + 16 * 64 : 16 * 256, x_bytes = uint32_t(xrows) * 256;

    // TMA boxes of unit (tile t, chunk i) into slot s, issued by lane 0; the
    // slot's barrier expects the X bytes too, so that it cannot complete
    // before a deferred X box has landed
    auto issue_w = [&](int64_t t, int i, int s, bool with_x) {
        if (lane != 0) return;
        uint8_t *dst = ring + s * slot_b;
        fence_proxy_async_smem();   // earlier reads of the slot come before the boxes that refill it
        mbar_arrive_expect_tx(&full[s], w_bytes + x_bytes);
        tma_load_2d(dst, &tmW, i * kChunkK, int32_t(t * kRows), &full[s]);
        if (PAL) tma_load_2d(dst + kPalOff, &tmP, i * (kChunkK / 2), int32_t(t * kRows), &full[s]);
        if (with_x) tma_load_2d(dst + kXOff, &tmX, i * kChunkK, 0, &full[s]);
    };
    auto issue_x = [&](int i, int s) {
        if (lane == 0) tma_load_2d(ring + s * slot_b + kXOff, &tmX, i * kChunkK, 0, &full[s]);
    };
    // raw flags of the unit whose first weight is element `uoff`, and this
    // lane's raw quarters copied into slot s; returns the lane's flags as a
    // consumer (bit 0: row g, bit 1: row g + 8, of its quarter)
    auto issue_raw = [&](uint32_t uoff, int s) -> uint32_t {
        if (!PAL) return 0u;
        const uint32_t gl = (uoff >> 6) + lc_flag;
        const uint32_t fw = __ldg(a.flagbits + (gl >> 5));
        const uint32_t mask = __ballot_sync(0xFFFFFFFFu, (fw >> (gl & 31u)) & 1u);
        const uint32_t fl = ((mask >> fbit_a) & 1u) | (((mask >> fbit_b) & 1u) << 1);
        if (fl) {
            const uint32_t dst = smem_addr(ring + s * slot_b + kRawOff);
#pragma unroll
            for (int h = 0; h < 2; h++) {
                if (!((fl >> h) & 1u)) continue;
                const int r = g + 8 * h;
                const uint32_t gg = (uoff >> 6) + uint32_t(r) * gpr + uint32_t(c >> 1);
                const uint32_t fwg = __ldg(a.flagbits + (gg >> 5)), bg = gg & 31u;
                const uint32_t rank = __ldg(a.rawbase + (gg >> 5)) + __popc(fwg & ((1u << bg) - 1u));
                const uint8_t *e = a.rawexp + uint64_t(rank) * kGroup + (c & 1) * 32;
                cp16(dst + uint32_t(r * 128 + c * 32), e);
                cp16(dst + uint32_t(r * 128 + c * 32 + 16), e + 16);
            }
        }
        return fl;
    };

    float d0[NT][4], d1[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int q = 0; q < 4; q++) d0[t][q] = d1[t][q] = 0.f;

    // One unit, in four blocks of 8 weights per row: a block's BF16 pairs
    // (4 per row) feed MMA K-steps 2b and 2b + 1 with 16 bytes of X per token
    // tile, so only one block's pairs are live at a time.  Each accumulator
    // receives its MMAs in K-step order, as if the unit's pairs were built
    // first.
    auto consume = [&](int s, uint32_t flags) {
        const uint8_t *slot = ring + s * slot_b;
        uint32_t smA[8], eA[8], smB[8], eB[8];
        if (PAL) {
            row_words(slot, o_sm0, o_sm1, o_pal, flags & 1u, P, smA, eA);
            row_words(slot, o_sm0 + 8 * 128, o_sm1 + 8 * 128, o_pal + 8 * 64, (flags >> 1) & 1u, P, smB, eB);
        }
#pragma unroll
        for (int b = 0; b < 4; b++) {
            uint32_t wa[4], wb[4];   // pairs 4b .. 4b + 3 of rows g and g + 8
            if (PAL) {
                join4(eA[2 * b], smA[2 * b], wa[0], wa[1]);
                join4(eA[2 * b + 1], smA[2 * b + 1], wa[2], wa[3]);
                join4(eB[2 * b], smB[2 * b], wb[0], wb[1]);
                join4(eB[2 * b + 1], smB[2 * b + 1], wb[2], wb[3]);
            } else {
                const uint4 va = lds128(slot + o_bfa + 16 * b), vb = lds128(slot + o_bfb + 16 * b);
                wa[0] = va.x; wa[1] = va.y; wa[2] = va.z; wa[3] = va.w;
                wb[0] = vb.x; wb[1] = vb.y; wb[2] = vb.z; wb[3] = vb.w;
            }
#pragma unroll
            for (int t = 0; t < NT; t++) {
                const uint4 x = lds128(slot + (t == 0 ? o_xa : o_xb) + 16 * b);
                // K-step j: A = {row g pair 2j, row g+8 pair 2j, row g pair 2j+1, row g+8 pair 2j+1}
                mma16816(d0[t], wa[0], wb[0], wa[1], wb[1], x.x, x.y);   // j = 2b
                mma16816(d1[t], wa[2], wb[2], wa[3], wb[3], x.z, x.w);   // j = 2b + 1
            }
        }
    };

    // end of a piece of tile t: write Y, or hand the piece to the fix-up
    const int64_t t_first = u_begin / a.cpr;
    auto finish = [&](int64_t t, bool whole) {
        float v[NT][4];
#pragma unroll
        for (int tt = 0; tt < NT; tt++)
#pragma unroll
            for (int q = 0; q < 4; q++) {
                v[tt][q] = d0[tt][q] + d1[tt][q];
                d0[tt][q] = d1[tt][q] = 0.f;
            }
        if (!whole) {
            // this warp's first piece goes to slot 2 gw, its last to 2 gw + 1
            const int64_t slot = 2 * gw + (t == t_first ? 0 : 1);
#pragma unroll
            for (int tt = 0; tt < NT; tt++)
                *reinterpret_cast<float4 *>(a.partial + ((slot * NT + tt) * 32 + lane) * 4) =
                    make_float4(v[tt][0], v[tt][1], v[tt][2], v[tt][3]);
            __threadfence();
            __syncwarp();
            uint32_t old = 0;
            if (lane == 0) old = atomicAdd(a.counters + t, 1u);
            old = __shfl_sync(0xFFFFFFFFu, old, 0);
            const int64_t wf = owner(t * a.cpr, a.units, a.warps), wl = owner(t * a.cpr + a.cpr - 1, a.units, a.warps);
            if (old != uint32_t(wl - wf)) return;   // another warp adds the pieces
            __threadfence();
            // the pieces in warp order: the first owner's piece is its last
            // one unless its run starts with this tile
            for (int64_t w = wf; w <= wl; w++) {
                const int64_t sl = 2 * w + ((w == wf && unit0(wf, a.units, a.warps) < t * a.cpr) ? 1 : 0);
#pragma unroll
                for (int tt = 0; tt < NT; tt++) {
                    float4 *pp = reinterpret_cast<float4 *>(a.partial + ((sl * NT + tt) * 32 + lane) * 4);
                    const float4 p = __ldcg(pp);
                    // read once, then zeroed: a completed call leaves its whole
                    // scratch zero, so a later call whose tile counters lie
                    // where these fragments were finds them at zero
                    __stcg(pp, make_float4(0.f, 0.f, 0.f, 0.f));
                    if (w == wf) {
                        v[tt][0] = p.x;
                        v[tt][1] = p.y;
                        v[tt][2] = p.z;
                        v[tt][3] = p.w;
                    } else {
                        v[tt][0] += p.x;
                        v[tt][1] += p.y;
                        v[tt][2] += p.z;
                        v[tt][3] += p.w;
                    }
                }
            }
            if (lane == 0) a.counters[t] = 0u;
        }
        // d[t][0..1]: row g, tokens 8t + 2c, +1; d[t][2..3]: row g + 8, same tokens
        const int64_t ra = t * kRows + g, rb = ra + 8;
#pragma unroll
        for (int tt = 0; tt < NT; tt++) {
            const int tok = 8 * tt + 2 * c;
            if (tok < a.m) {
                a.y[int64_t(tok) * a.n + ra] = v[tt][0];
                a.y[int64_t(tok) * a.n + rb] = v[tt][2];
            }
            if (tok + 1 < a.m) {
                a.y[int64_t(tok + 1) * a.n + ra] = v[tt][1];
                a.y[int64_t(tok + 1) * a.n + rb] = v[tt][3];
            }
        }
    };
    // issue side: the unit after the last one issued: tile it, chunk ii,
    // element offset uoff_i of its first weight; ring slot is_
    const int c_first = int(u_begin - t_first * cpr);
    int64_t it = t_first;
    int ii = c_first;
    uint32_t uoff_i = uint32_t(t_first) * 16u * k + uint32_t(ii) * 128u;
    const uint32_t tile_jump = 16u * k - uint32_t(cpr) * 128u;   // past a tile's last chunk -> next tile
    int is_ = 0, ni = 0;    // next slot, units issued
    uint32_t rawbits = 0;   // consumer raw flags, 2 bits per slot
    auto advance = [&]() {
        uoff_i += 128u;
        if (++ii == cpr) {
            ii = 0;
            ++it;
            uoff_i += tile_jump;
        }
        ++is_;
        ++ni;
    };
    // the ring's first units (one copy group each, empty ones included, so
    // that unit j's raw copies are always group j)
    const int npro = min(stages - 1, nu);
    for (int s = 0; s < stages - 1; s++) {
        if (s < npro) {
            issue_w(it, ii, s, !defer_x);
            rawbits |= issue_raw(uoff_i, s) << (2 * s);
            advance();
        }
        cp_commit();
    }
    if (defer_x) {
        // the previous kernel has ended: the prologue units' X boxes
        pdl_wait();
        int cx = c_first;
        for (int s = 0; s < npro; s++) {
            issue_x(cx, s);
            if (++cx == cpr) cx = 0;
        }
    }

    int64_t ct = t_first;
    int ci = c_first, piece0 = ci, cs = 0, j = 0;
    uint32_t phases = 0;   // bit s: parity of slot s's next barrier phase
    bool dead = false;
    for (; j < nu; j++) {
        cp_wait(stages - 2);   // this lane's raw copies of unit j have landed
        // ... and unit j's boxes (all lanes agree on a time-out)
        dead = __any_sync(0xFFFFFFFFu, !mbar_wait(&full[cs], (phases >> cs) & 1u, T));
        if (dead) break;
        phases ^= 1u << cs;
        // every lane has read the slot consumed last iteration, which is
        // refilled now
        __syncwarp();
        const uint32_t fl = (rawbits >> (2 * cs)) & 3u;
        if (j + stages - 1 < nu) {
            if (is_ == stages) is_ = 0;
            issue_w(it, ii, is_, true);
            rawbits = (rawbits & ~(3u << (2 * is_))) | (issue_raw(uoff_i, is_) << (2 * is_));
            advance();
        }
        cp_commit();
        consume(cs, fl);
        if (++cs == stages) cs = 0;
        if (++ci == cpr || j == nu - 1) {
            finish(ct, piece0 == 0 && ci == cpr);
            if (ci == cpr) {
                ci = 0;
                ++ct;
            }
            piece0 = ci;
        }
    }
    if (dead) {
        // time-out: no more work; wait (bounded) for the boxes and copies
        // this warp has issued, so that none lands after the CTA has exited
        if (lane == 0) flag_error(a.status, UW_DEVERR_TIMEOUT);
        for (int u = j; u < ni; u++) mbar_wait(&full[u % stages], uint32_t(u / stages) & 1u, T);
        cp_async_wait_all();
    }
}


std::mutex g_mu;

template <class K>
cudaError_t prepare(K kern, int (&ready)[64]) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (ready[dev]) return cudaSuccess;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (err != cudaSuccess) return err;
    ready[dev] = 1;
    return cudaSuccess;
}

// 2-D tensor map over a row-major [rows, inner] array (no swizzle, dense box)
bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// shared memory of one warp's ring slot and its barrier
size_t slot_cost(int64_t m) { return size_t(slot_bytes(int(m))) + 8; }

}  // namespace

int gemv_sk_stages(int warps, int stages, int64_t m) {
    if (warps < 1 || warps > kMaxWarps || stages < 0 || stages > kMaxStages || m < 1 || m > 16) return 0;
    const size_t slot = slot_cost(m);
    const size_t room = size_t(kMaxSmem) - 128;   // less the alignment slack
    if (stages == 0) {   // the deepest ring that fits, at most kMaxStages
        stages = int(std::min<size_t>(kMaxStages, room / (size_t(warps) * slot)));
        return stages >= 2 ? stages : 0;
    }
    if (stages < 2 || size_t(warps) * stages * slot > room) return 0;
    return stages;
}

GemvSkGeometry gemv_sk_geometry(int64_t m, int64_t n, int64_t k, int warps) {
    GemvSkGeometry g{};
    if (m <= 0 || m > 16 || n <= 0 || k <= 0 || n % kRows || k % kChunkK || warps < 1 || warps > kMaxWarps)
        return g;
    g.S = warps;
    g.NT = m > 8 ? 2 : 1;
    g.tiles = n / kRows;
    g.cpr = k / kChunkK;
    g.units = g.tiles * g.cpr;
    g.warps = std::min<int64_t>(int64_t(sm_count()) * warps, g.units);
    g.G = int((g.warps + warps - 1) / warps);
    g.counter_bytes = align_up(uint64_t(g.tiles) * 4, 256);
    g.partial_bytes = align_up(uint64_t(2 * g.warps) * uint64_t(g.NT) * 32 * 4 * 4, 256);
    return g;
}

cudaError_t launch_gemv_sk(const GemvSkLaunch &p, cudaStream_t stream) {
    const GemvSkGeometry g = gemv_sk_geometry(p.m, p.n, p.k, p.warps);
    const int stages = gemv_sk_stages(p.warps, p.stages, p.m);
    if (g.G <= 0 || stages == 0 || !p.counters || !p.partial || !p.x || !p.y) return cudaErrorInvalidValue;
    // element offsets inside the kernel are 32-bit
    if (uint64_t(p.n) * uint64_t(p.k) > 0xFFFFFFFFull) return cudaErrorInvalidValue;
    SkArgs a{};
    a.x = p.x;
    a.n = p.n;
    a.k = p.k;
    a.m = int(p.m);
    a.cpr = g.cpr;
    a.units = g.units;
    a.warps = g.warps;
    a.y = p.y;
    a.partial = p.partial;
    a.counters = p.counters;
    a.stages = stages;
    a.slot_bytes = slot_bytes(int(p.m));
    a.status = p.status;
    a.timeout_ns = p.timeout_ns;
    const bool pal = p.pal != nullptr;
    CUtensorMap mw, mp, mx;
    if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, uint64_t(p.k), uint64_t(p.m), uint64_t(p.k) * 2,
                  kChunkK, uint32_t(p.m)))
        return cudaErrorInvalidValue;
    if (pal) {
        if (!p.w) return cudaErrorInvalidValue;
        a.sm = p.w->sm;
        a.pal = p.pal;
        a.flagbits = p.w->flagbits;
        a.rawbase = p.w->rawbase;
        a.rawexp = p.w->rawexp;
        a.palette = make_palette16(p.w->palette);
        a.w_stable = p.w_stable ? 1 : 0;
        if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.w->sm, uint64_t(p.k), uint64_t(p.n), uint64_t(p.k),
                      kChunkK, kRows) ||
            !make_map(&mp, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.pal, uint64_t(p.k / 2), uint64_t(p.n), uint64_t(p.k / 2),
                      kChunkK / 2, kRows))
            return cudaErrorInvalidValue;
    } else {
        if (!p.w_bf16) return cudaErrorInvalidValue;
        a.w_bf16 = p.w_bf16;
        if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.w_bf16, uint64_t(p.k), uint64_t(p.n),
                      uint64_t(p.k) * 2, kChunkK, kRows))
            return cudaErrorInvalidValue;
        mp = mw;
    }
    const size_t smem = size_t(p.warps) * stages * slot_cost(p.m) + 128;
    const dim3 grid(unsigned(g.G)), block(unsigned(p.warps * 32));
    cudaError_t err = cudaSuccess;
#define UW_SK_LAUNCH(P_, N_)                                                    \
    do {                                                                        \
        static int ready[64] = {0};                                             \
        err = prepare(k_gemv_sk<P_, N_>, ready);                                \
        if (err == cudaSuccess)                                                 \
            err = launch_pdl(a.w_stable != 0, k_gemv_sk<P_, N_>, grid, block, smem, stream, mw, mp, mx, a); \
    } while (0)
    if (pal) {
        if (g.NT == 2) UW_SK_LAUNCH(true, 2); else UW_SK_LAUNCH(true, 1);
    } else {
        if (g.NT == 2) UW_SK_LAUNCH(false, 2); else UW_SK_LAUNCH(false, 1);
    }
#undef UW_SK_LAUNCH
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace uw
