// kernels.h -- host-side launch interface of the libuw CUDA kernels (internal).
#pragma once
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/uw.h"

namespace uw {

// Huffman decode of a whole matrix (Unweight page §六, pipelines 1 and 3).
// out_bf16 != nullptr: write BF16 [n*k]; out_pal != nullptr: write the
// 4-bit palette plane [n*k/2].  Exactly one must be non-null.
cudaError_t launch_huff_decode(const uw_dmat &w, uint16_t *out_bf16, uint8_t *out_pal,
                               cudaStream_t stream);

// Exponent-only Huffman decode (Unweight page §六, pipeline 2): every
// weight's exponent byte, uint8 [n*k] in weight order.  When all_raw_flags and
// all_raw_rank are non-null (n*k/2048 words each) the kernel also writes the
// raw-group bitmap and per-word rank bases of a layout in which every group is
// raw: all bits set, word i's base 32*i.  With those, group g's raw rank is g,
// and the raw plane at byte 64*rank is exactly the exponent plane, so the
// fused kernels read it through their raw-group path (exp_plane_view).
cudaError_t launch_exp_decode(const uw_dmat &w, uint8_t *out_exp, uint32_t *all_raw_flags,
                              uint32_t *all_raw_rank, cudaStream_t stream);

// Pipeline 2's workspace: the exponent plane, then the all-raw bitmap and
// rank bases, each 256-byte aligned.
struct ExpPlaneLayout {
    uint64_t flags_off, rank_off, bytes;
};
inline ExpPlaneLayout exp_plane_layout(int64_t n, int64_t k) {
    const auto up = [](uint64_t x) { return (x + 255u) / 256u * 256u; };
    const uint64_t plane = uint64_t(n) * uint64_t(k);
    const uint64_t words = (plane / 64 + 31) / 32;
    ExpPlaneLayout L;
    L.flags_off = up(plane);
    L.rank_off = L.flags_off + up(words * 4);
    L.bytes = L.rank_off + up(words * 4);
    return L;
}

// The matrix as pipeline 2's fused matmul sees it: sign/mantissa plane of
// `w`, every group raw, the exponent plane in `slot` (laid out as above) as
// the raw plane.  The palette plane pointer is set to the exponent plane too:
// kernels that stage the palette plane unconditionally then read n*k/2 valid
// bytes whose values no raw group uses.
inline uw_dmat exp_plane_view(const uw_dmat &w, uint8_t *slot) {
    const ExpPlaneLayout L = exp_plane_layout(w.n, w.k);
    uw_dmat v = w;
    v.rawexp = slot;
    v.flagbits = reinterpret_cast<const uint32_t *>(slot + L.flags_off);
    v.rawbase = reinterpret_cast<const uint32_t *>(slot + L.rank_off);
    v.n_raw = w.n_groups;
    v.pal = slot;
    return v;
}

// Workspace bytes of a pipeline's preprocessing output (0 for pipeline 4).
inline uint64_t prep_workspace_bytes(int64_t n, int64_t k, int32_t pipeline) {
    const uint64_t nk = uint64_t(n) * uint64_t(k);
    if (pipeline == UW_PIPE_DECODE_GEMM) return (nk * 2 + 255u) / 256u * 256u;
    if (pipeline == UW_PIPE_DECODE_EXP_FUSED) return exp_plane_layout(n, k).bytes;
    if (pipeline == UW_PIPE_TRANSCODE_FUSED) return (nk / 2 + 255u) / 256u * 256u;
    return 0;
}

// CUDA-core FMA GEMV, m <= 8 (Unweight page §七, small-batch case).
// pal_plane == nullptr: plain BF16 weights `w_bf16`; otherwise the fused
// palette path using `w` (sm/raw planes) and `pal_plane`.  One warp per
// `rows_per_warp` (1 or 2) rows.
cudaError_t launch_gemv_fma(const uint16_t *x, int m, const uint16_t *w_bf16, const uw_dmat *w,
                            const uint8_t *pal_plane, int64_t n, int64_t k, float *y,
                            int rows_per_warp, uint32_t *status, cudaStream_t stream);

// Warp-level MMA skinny matmul, m <= 16 (Unweight page §七): W rebuilt in
// registers into mma.m16n8k16 fragments, 16 rows per CTA, `slices` (1..8)
// warps per CTA splitting K; `width` 1: 16 weights per lane and row per step,
// 2: 32, 0: 32 when k is a multiple of 128.  pal_plane == nullptr: plain BF16.
cudaError_t launch_gemv_mma(const uint16_t *x, int m, const uint16_t *w_bf16, const uw_dmat *w,
                            const uint8_t *pal_plane, int64_t n, int64_t k, float *y, int slices, int width,
                            cudaStream_t stream, bool w_stable = false);

// The warp-MMA fused kernel over many matrices in as few launches as
// possible (32 matrices per launch; items with m == 0 are skipped): item i
// computes y[m, n] = x[m, k] * W^T on its palette-form matrix, bit-identical
// to launch_gemv_mma for that item alone with the same slices and step
// width.  width 0 picks 32 weights per lane only if every item's k allows it.
struct MmaItem {
    const uint16_t *x;
    int m;
    const uw_dmat *w;
    float *y;
};
cudaError_t launch_gemv_mma_batched(const MmaItem *items, int n_items, int slices, int width,
                                    cudaStream_t stream);

// SMs of the current device (148 when no device answers, so that workspace
// sizes can be computed on a host without a GPU).
int sm_count();

// Persistent stream-K form of the warp-MMA kernel, m <= 16, k a multiple of
// 128 and n * k < 2^32 (gemv_sk.cu): one CTA of `warps` warps per SM, every
// warp an equal contiguous run of (16-row tile, 128-wide K chunk) units, its
// loads (W and the chunk's X rows, 2-D TMA boxes) in a shared-memory ring of
// `stages` slots of 5120 + 256 m bytes plus an 8-byte barrier (0 = the
// deepest that fits); a tile cut between warps is summed in warp order by
// the warp that finishes its last piece.  Workspace: `counters` (one u32 per tile,
// zero before the call and left zero by it) and `partial` (two fragment
// sets of 32 x 4 x NT floats per warp).  pal == nullptr: plain BF16 `w_bf16`.
struct GemvSkGeometry {
    int G = 0, S = 0, NT = 0;
    int64_t tiles = 0, cpr = 0, units = 0, warps = 0;
    uint64_t counter_bytes = 0, partial_bytes = 0;
};
GemvSkGeometry gemv_sk_geometry(int64_t m, int64_t n, int64_t k, int warps);
int gemv_sk_stages(int warps, int stages, int64_t m);   // the ring depth used, 0 if not valid for m tokens
struct GemvSkLaunch {
    const uint16_t *x;
    int64_t m, n, k;
    const uint16_t *w_bf16;    // plain path
    const uw_dmat *w;          // fused path: sm/raw/flag planes
    const uint8_t *pal;        // fused path: palette plane
    float *y;
    uint32_t *counters;
    float *partial;
    int warps, stages;
    bool w_stable;             // fused: the planes are the blob's (read before the previous kernel ends)
    uint32_t *status;          // device error word (time-out), may be null
    uint64_t timeout_ns;       // bound of every wait in the kernel
};
cudaError_t launch_gemv_sk(const GemvSkLaunch &p, cudaStream_t stream);

// tcgen05 GEMM (Unweight page §七, reconstructive matmul), token tile `bn`.
// Launch, with programmatic stream serialization when `early` is set: the
// kernel calls pdl_wait before touching data an earlier kernel on the stream
// may own, so its CTAs can be scheduled, and start on what no kernel writes,
// while that kernel drains.  Measured on a step of 12 matmuls (Llama-3.1-8B
// MLP layer, M = 1, 4, 16, 64), early launches pay only for kernels that have
// such work -- the fused kernels on the blob's own planes: +11% -- while
// kernels that must wait at their first instruction ran slower launched early
// (the BF16 twins: -11%; the split-K reduce: -4% on the step), so those are
// launched as usual.
template <class... KArgs, class... Args>
cudaError_t launch_pdl(bool early, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = early ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct TcLaunch {
    const uint16_t *x;         // [m, k] BF16
    int64_t m, n, k;
    const uint16_t *w_bf16;    // plain path (nullptr for the fused path)
    const uw_dmat *w;          // fused path: sm/raw/flag planes
    const uint8_t *pal;        // fused path: palette plane
    float *y;                  // [m, n]
    float *partial;            // [split_k, m, n] when split_k > 1; stream-K: partial tiles
    uint32_t *sk_counters;     // stream-K: one counter per tile (zero between calls)
    bool huffman;              // stream-K fused: decode the palette indices from the Huffman stream
    bool w_stable;             // fused: the compressed planes are the blob's (no kernel writes them),
                               // so they may be read before the previous kernel on the stream ends
    int bn, split_k, stages;
    uint32_t debug_flags;
    uint64_t timeout_ns;
    uint32_t *dev_status;
};
cudaError_t launch_gemm_tc(const TcLaunch &p, cudaStream_t stream);

// Persistent stream-K tcgen05 GEMM (same TcLaunch; split_k unused): one CTA
// per SM, each a contiguous run of (tile, K-step) units; tiles cut between
// CTAs are summed in CTA order by the last CTA to finish a piece.
// Workspace: `counters` (one u32 per tile, zero before the first call and
// left zero by every call that completes) and `partial` (two 128 x bn fp32
// tiles per CTA).
struct SkGeometry {
    int S = 0, TB = 0, G = 0;
    int64_t RB = 0, tiles = 0, units = 0;
    uint64_t counter_bytes = 0, partial_bytes = 0;
};
SkGeometry sk_geometry(int64_t m, int64_t n, int64_t k, int bn);
cudaError_t launch_gemm_sk(const TcLaunch &p, cudaStream_t stream);

// uw_fused_matmul / uw_matmul_bf16 with the stream-K tile counters kept
// apart from the workspace (sk_counters != nullptr: at least
// sk_counter_bytes, zero at the call; the workspace then holds only the
// preprocessing output and the partial tiles).  For callers that share one
// scratch region between plans of different kernels (layer stacks, the
// autotuner, the no-workspace entry point), where another kernel's partial
// sums would otherwise land on the counters.
uint64_t sk_counter_bytes(int64_t m, int64_t n, int64_t k, const uw_plan *plan);
uw_status fused_matmul_ex(const uint16_t *x_dev, int64_t m, const uw_dmat *w, const uint8_t *pal_dev, float *y_dev,
                          const uw_plan *plan, void *ws, size_t ws_bytes, uint32_t *sk_counters, cudaStream_t s);
uw_status matmul_bf16_ex(const uint16_t *x_dev, int64_t m, const uint16_t *w_dev, int64_t n, int64_t k, float *y_dev,
                         const uw_plan *plan, void *ws, size_t ws_bytes, uint32_t *dev_status, uint32_t *sk_counters,
                         cudaStream_t s);

// Fixed-order sum of split-K partials: y[i] = sum_s partial[s][i], s ascending.
cudaError_t launch_splitk_reduce(const float *partial, int split_k, int64_t count, float *y,
                                 cudaStream_t stream);

// Driver entry point for cuTensorMapEncodeTiled (resolved once through the
// runtime so that the library needs no link-time libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace uw
