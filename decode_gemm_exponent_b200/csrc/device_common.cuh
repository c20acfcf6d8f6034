// device_common.cuh -- sm_100a device helpers for libuw kernels:
// bounded mbarrier waits, bulk/tensor TMA copies, tcgen05 (TMEM + MMA)
// wrappers, and the BF16 rebuild arithmetic of the Unweight page (§四: the
// sign/mantissa byte is raw, the exponent byte comes from a 16-entry palette
// or from the raw plane).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/uw.h"

namespace uw {
namespace dev {

// ---------------------------------------------------------------- misc

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void flag_error(uint32_t *status, uint32_t bits) {
    if (status) atomicOr(status, bits);
}

// byte permute (PTX prmt, default mode: selector bit 3 replicates the sign
// bit of the selected byte)
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(
            smem_addr(bar)),
        "r"(bytes)
        : "memory");
}

// Non-blocking test of phase completion (the waiter spins; no suspension).
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed, or give up after
// about `timeout_ns`.  The bound is counted in SM cycles (clock64 is cheap to
// read; 2 cycles per ns keeps the bound at least timeout_ns for clocks up to
// 2 GHz).  Returns false on time-out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long limit = (long long)(timeout_ns * 2);
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > limit) return false;
    return true;
}

// Potentially blocking test: the thread is suspended in hardware until the
// phase completes or about `hint_ns` pass, so a parked warp takes no issue
// slots from the working ones (a spinning test loop of a dozen parked warps
// measurably slows the producer, MMA and rebuild warps of the same SM).
__device__ __forceinline__ bool mbar_try_wait_susp(uint64_t *bar, uint32_t parity, uint32_t hint_ns = 100000u) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// mbar_wait that also gives up as soon as *abort is set by another role of
// the CTA (so one time-out ends every wait of the CTA quickly).  Returns
// false on time-out or abort.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t *bar, uint32_t parity, uint64_t timeout_ns,
                                                   const volatile int *abort) {
    if (mbar_try_wait_susp(bar, parity)) return true;
    const long long limit = (long long)(timeout_ns * 2);
    const long long t0 = clock64();
    while (!mbar_try_wait_susp(bar, parity)) {
        if (*abort || clock64() - t0 > limit) return false;
    }
    return true;
}

// mbar_wait_or_abort for roles that are not on the critical path (a warp
// that waits a whole tile for its accumulator, a producer far ahead of its
// consumer): between polls the warp sleeps, so that it leaves the issue
// slots to the warps that do the work.  The time limit counts clock64 as
// mbar_wait_or_abort does; sleeping only lengthens each poll.
__device__ __forceinline__ bool mbar_wait_lazy(uint64_t *bar, uint32_t parity, uint64_t timeout_ns,
                                               const volatile int *abort, uint32_t sleep_ns = 256u) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long limit = (long long)(timeout_ns * 2);
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort || clock64() - t0 > limit) return false;
        __nanosleep(sleep_ns);
    }
    return true;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel on its stream is still
// running, once every CTA of that kernel has called pdl_trigger (or exited).
// Before it reads anything an earlier kernel may have written, or writes
// anything an earlier kernel may still read, a thread calls pdl_wait, which
// returns when the earlier kernels have completed and their writes are
// visible.  Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Named barrier over `threads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also ORs a predicate over its threads: every thread
// gets the same answer, so the threads can take one branch together.
__device__ __forceinline__ bool named_bar_any(uint32_t id, uint32_t threads, bool pred) {
    uint32_t out;
    asm volatile(
        "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, %2, %3, p; selp.u32 %0, 1, 0, q; }"
        : "=r"(out)
        : "r"(uint32_t(pred)), "r"(id), "r"(threads)
        : "memory");
    return out != 0;
}

// ---------------------------------------------------------------- TMA

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes and
// both addresses must be multiples of 16).
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// 2-D tiled tensor copy global -> shared (x = innermost coordinate).
__device__ __forceinline__ void tma_load_2d(void *dst_smem, const CUtensorMap *map, int32_t x,
                                            int32_t y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 16-byte asynchronous global -> shared copy (not TMA), L1 bypassed
__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst_smem)), "l"(src)
                 : "memory");
}

// 16-byte cp.async that reads `src_bytes` (0 or 16) bytes and fills the rest
// of the 16 with zeros (src must still be a valid address)
__device__ __forceinline__ void cp_async16_zfill(void *dst_smem, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst_smem)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// Raise the transaction count of `bar`'s current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// Make `bar`'s current phase also wait for this thread's earlier cp.async
// copies (the pending count is raised now and lowered when they land).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Same, but the arrival is counted in the barrier's expected count instead
// of raising the pending count (the barrier must be initialised with it).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// generic-proxy shared-memory writes -> visible to the async proxy (MMA, TMA)
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (BF16 in, FP32 accumulate)
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16: A (M rows x 16 K, BF16)
// occupies 128 lanes x 8 columns from `a_tmem`, row i in lane i, K pair p
// (elements 2p, 2p+1) in column p
__device__ __forceinline__ void tc_mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 bit, 32 consecutive columns per thread (the warp's lane
// quarter), then tmem_st_wait before the data may be consumed
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%32], "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31};" ::"r"(v[0]),
        "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]),
        "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]), "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// arrive on `bar` once all previously issued tcgen05.mma of this thread finish
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major tile whose rows are 128 bytes
// (64 BF16), stored with the 128-byte swizzle in 1024-byte atoms of 8 rows.
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t saddr) {
    uint64_t d = 0;
    d |= uint64_t((saddr & 0x3FFFFu) >> 4);        // start address
    d |= uint64_t(1) << 16;                         // leading byte offset (unused here)
    d |= uint64_t(1024 >> 4) << 32;                 // stride byte offset: 8 rows * 128 B
    d |= uint64_t(1) << 46;                         // descriptor version (sm_100)
    d |= uint64_t(2) << 61;                         // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16, A = B = BF16, D = F32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

// ---------------------------------------------------------------- rebuild
//
// A BF16 pattern s<<15 | e<<7 | m has high byte s<<7 | e>>1 and low byte
// (e&1)<<7 | m.  With the palette stored as r = rotr8(e) = (e>>1) | (e&1)<<7
// both bytes come from one looked-up byte r and the sign/mantissa byte
// sm = s<<7 | m:  high = (r & 0x7F) | (sm & 0x80),  low = (r & 0x80) | (sm & 0x7F).

struct Palette16 {
    uint32_t p0, p1, p2, p3;   // rotr8(palette[0..15]) as bytes, 4 per word
};

__host__ __device__ inline uint8_t rotr8(uint8_t e) { return uint8_t((e >> 1) | ((e & 1u) << 7)); }

__host__ inline Palette16 make_palette16(const uint8_t palette[16]) {
    auto word = [&](int i) {
        return uint32_t(rotr8(palette[i])) | uint32_t(rotr8(palette[i + 1])) << 8 |
               uint32_t(rotr8(palette[i + 2])) << 16 | uint32_t(rotr8(palette[i + 3])) << 24;
    };
    return Palette16{word(0), word(4), word(8), word(12)};
}

// rotr8 of four raw exponent bytes
__device__ __forceinline__ uint32_t rot4(uint32_t e) {
    return ((e >> 1) & 0x7F7F7F7Fu) | ((e << 7) & 0x80808080u);
}

// 16-entry byte lookup for four indices: low three bits as prmt selectors
// (bit 3 cleared) into each 8-byte half-palette, then a byte mask picks the
// upper half where the index has bit 3 set.
__device__ __forceinline__ uint32_t lookup4(uint32_t sel, uint32_t mask, const Palette16 &P) {
    const uint32_t lo = prmt(P.p0, P.p1, sel), hi = prmt(P.p2, P.p3, sel);
    return (hi & mask) | (lo & ~mask);
}

// One stored 4-bit-palette word (8 weights) -> rotated exponent bytes:
// r0 = weights 0..3, r1 = weights 4..7.  In the stored layout bit 3 of index
// j sits in the top bit of byte j (j < 4) or of byte j-4 of the word shifted
// left by 4 (j >= 4), so a sign-replicating prmt yields the byte masks.
__device__ __forceinline__ void pal_rot(uint32_t x, const Palette16 &P, uint32_t &r0, uint32_t &r1) {
    r0 = lookup4(x & 0x7777u, prmt(x, 0u, 0xBA98u), P);
    r1 = lookup4((x >> 16) & 0x7777u, prmt(x << 4, 0u, 0xBA98u), P);
}

// Same for 8 indices in natural nibble order (index j in bits 4j..4j+3).
__device__ __forceinline__ void nat_rot(uint32_t x, const Palette16 &P, uint32_t &r0, uint32_t &r1) {
    const uint32_t m_odd = prmt(x, 0u, 0xBA98u);         // bit 3 of indices 1,3,5,7
    const uint32_t m_even = prmt(x << 4, 0u, 0xBA98u);   // bit 3 of indices 0,2,4,6
    r0 = lookup4(x & 0x7777u, prmt(m_even, m_odd, 0x5140u), P);
    r1 = lookup4((x >> 16) & 0x7777u, prmt(m_even, m_odd, 0x7362u), P);
}

// 4 rotated exponents + 4 sign/mantissa bytes -> 4 BF16 (w01 = weights 0,1)
__device__ __forceinline__ void join4(uint32_t r, uint32_t s, uint32_t &w01, uint32_t &w23) {
    const uint32_t hi = (r & 0x7F7F7F7Fu) | (s & 0x80808080u);
    const uint32_t lo = (r & 0x80808080u) | (s & 0x7F7F7F7Fu);
    w01 = prmt(lo, hi, 0x5140u);
    w23 = prmt(lo, hi, 0x7362u);
}

// 8 weights -> uint4 of 8 BF16
__device__ __forceinline__ uint4 join8(uint32_t r0, uint32_t r1, uint32_t s0, uint32_t s1) {
    uint4 o;
    join4(r0, s0, o.x, o.y);
    join4(r1, s1, o.z, o.w);
    return o;
}

// 8 palette indices in natural order -> the stored 4-bit-palette word layout.
// Low three bits stay in place; bit 3 of index j moves to bit 8j+7 (j < 4) or
// 8(j-4)+3 (j >= 4).  Sign-replicating byte permutes turn bit 3 of the even
// indices (top bit of each byte of x << 4) and of the odd indices (top bit of
// each byte of x) into byte masks, and two interleaving permutes place index
// j's mask in byte j (for bit 7) and index j+4's in byte j (for bit 3).
__device__ __forceinline__ uint32_t natural_to_pal(uint32_t x) {
    const uint32_t even = prmt(x << 4, 0u, 0xBA98u);   // byte k: bit 3 of index 2k
    const uint32_t odd = prmt(x, 0u, 0xBA98u);         // byte k: bit 3 of index 2k+1
    const uint32_t hi = prmt(even, odd, 0x5140u);      // byte j: index j        (j < 4)
    const uint32_t lo = prmt(even, odd, 0x7362u);      // byte j: index j + 4
    return (x & 0x77777777u) | (hi & 0x80808080u) | (lo & 0x08080808u);
}

// acc += a * b over the two BF16 halves of each operand (exact products,
// one rounding per FMA: identical to fmaf on the widened values)
__device__ __forceinline__ float fma2_bf16(uint32_t a, uint32_t b, float acc) {
    asm("{ .reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %0; }"
        : "+f"(acc)
        : "r"(a), "r"(b));
    return acc;
}

}  // namespace dev
}  // namespace uw
