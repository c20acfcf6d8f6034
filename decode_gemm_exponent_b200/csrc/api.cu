// api.cu -- the C ABI of libuw (declared in include/uw.h): binding a device
// copy of a blob, kernel status, the preprocessing kernels and the four matmul
// pipelines of the Unweight page (§六).
#include <algorithm>
#include <cstring>
#include <vector>

#include "kernels.h"
#include "uw_format.h"

namespace uw {
uw_status parse_header(const void *host_blob, size_t bytes, int verify_payload, Header &h);

namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline uw_status cuda_status(cudaError_t e) { return e == cudaSuccess ? UW_OK : UW_ERR_CUDA; }

bool valid_bn_tc(int bn) { return bn == 16 || bn == 32 || bn == 64 || bn == 128 || bn == 256; }

uw_status check_plan(const uw_plan *p, int64_t m, int64_t k) {
    if (!p || k <= 0) return UW_ERR_INVALID_ARG;
    if (p->pipeline != UW_PIPE_DECODE_GEMM && p->pipeline != UW_PIPE_DECODE_EXP_FUSED &&
        p->pipeline != UW_PIPE_TRANSCODE_FUSED && p->pipeline != UW_PIPE_DIRECT_PALETTE &&
        p->pipeline != UW_PIPE_HUFFMAN_FUSED)
        return UW_ERR_INVALID_ARG;
    if (p->pipeline == UW_PIPE_HUFFMAN_FUSED && (p->kernel != UW_KERNEL_TC_SK || p->bn > 32 || k % 256))
        return UW_ERR_INVALID_ARG;
    if (p->kernel == UW_KERNEL_FMA) {
        if (m > 8 || (p->bn != 1 && p->bn != 2) || p->split_k != 1) return UW_ERR_INVALID_ARG;
    } else if (p->kernel == UW_KERNEL_MMA) {
        if (m > 16 || p->bn < 1 || p->bn > 8 || p->split_k != 1) return UW_ERR_INVALID_ARG;
        if (p->stages < 0 || p->stages > 2 || (p->stages == 2 && k % 128)) return UW_ERR_INVALID_ARG;
    } else if (p->kernel == UW_KERNEL_TC) {
        if (!valid_bn_tc(p->bn) || p->split_k < 1 || p->split_k > 64 || p->stages < 0 || p->stages > 8)
            return UW_ERR_INVALID_ARG;
    } else if (p->kernel == UW_KERNEL_TC_SK) {
        if (!valid_bn_tc(p->bn) || p->split_k != 1 || p->stages < 0 || p->stages > 8) return UW_ERR_INVALID_ARG;
    } else if (p->kernel == UW_KERNEL_MMA_SK) {
        if (m > 16 || k % 128 || p->split_k != 1 || gemv_sk_stages(p->bn, p->stages, m) == 0) return UW_ERR_INVALID_ARG;
    } else {
        return UW_ERR_INVALID_ARG;
    }
    if (p->timeout_ns < 0) return UW_ERR_INVALID_ARG;
    return UW_OK;
}

// Scratch after the preprocessing output: split-K partial sums, or for the
// stream-K kernel its tile counters (unless the caller keeps them apart,
// `own_counters`) followed by its partial tiles.
uint64_t partial_bytes(int64_t m, int64_t n, int64_t k, const uw_plan *p, bool own_counters = false) {
    if (p->kernel == UW_KERNEL_MMA_SK) {
        const GemvSkGeometry g = gemv_sk_geometry(m, n, k, p->bn);
        return (own_counters ? 0 : g.counter_bytes) + g.partial_bytes;
    }
    if (p->kernel == UW_KERNEL_TC_SK) {
        const SkGeometry g = sk_geometry(m, n, k, p->bn);
        return (own_counters ? 0 : g.counter_bytes) + g.partial_bytes;
    }
    if (p->kernel != UW_KERNEL_TC || p->split_k <= 1) return 0;
    return align_up(uint64_t(p->split_k) * uint64_t(m) * uint64_t(n) * 4, 256);
}

uint64_t prep_bytes(int64_t n, int64_t k, const uw_plan *p) { return prep_workspace_bytes(n, k, p->pipeline); }

// Run one matmul kernel on prepared weights: w_bf16 (plain) or pal (fused).
uw_status run_kernel(const uint16_t *x, int64_t m, const uint16_t *w_bf16, const uw_dmat *w,
                     const uint8_t *pal, int64_t n, int64_t k, float *y, const uw_plan *plan,
                     float *partial, uint32_t *status, uint32_t *sk_counters, cudaStream_t stream,
                     bool huffman = false, bool w_stable = false) {
    if (plan->kernel == UW_KERNEL_FMA)
        return cuda_status(launch_gemv_fma(x, int(m), w_bf16, w, pal, n, k, y, plan->bn, status, stream));
    if (plan->kernel == UW_KERNEL_MMA)
        return cuda_status(
            launch_gemv_mma(x, int(m), w_bf16, w, pal, n, k, y, plan->bn, plan->stages, stream, w_stable));
    if (plan->kernel == UW_KERNEL_MMA_SK) {
        uint8_t *base = reinterpret_cast<uint8_t *>(partial);
        if (!base) return UW_ERR_WORKSPACE;
        GemvSkLaunch g{};
        g.x = x;
        g.m = m;
        g.n = n;
        g.k = k;
        g.w_bf16 = w_bf16;
        g.w = w;
        g.pal = pal;
        g.y = y;
        g.warps = plan->bn;
        g.stages = plan->stages;
        g.w_stable = w_stable;
        g.status = status;
        g.timeout_ns = plan->timeout_ns > 0 ? uint64_t(plan->timeout_ns) : kDefaultTimeoutNs;
        if (sk_counters) {
            g.counters = sk_counters;
            g.partial = partial;
        } else {
            g.counters = reinterpret_cast<uint32_t *>(base);
            g.partial = reinterpret_cast<float *>(base + gemv_sk_geometry(m, n, k, plan->bn).counter_bytes);
        }
        return cuda_status(launch_gemv_sk(g, stream));
    }
    TcLaunch t{};
    t.x = x;
    t.m = m;
    t.n = n;
    t.k = k;
    t.w_bf16 = w_bf16;
    t.w = w;
    t.pal = pal;
    t.y = y;
    t.partial = partial;
    t.bn = plan->bn;
    t.split_k = plan->split_k;
    t.stages = plan->stages;
    t.debug_flags = plan->debug_flags;
    t.timeout_ns = plan->timeout_ns > 0 ? uint64_t(plan->timeout_ns) : kDefaultTimeoutNs;
    t.dev_status = status;
    t.huffman = huffman;
    t.w_stable = w_stable;
    if (plan->kernel == UW_KERNEL_TC_SK) {
        uint8_t *base = reinterpret_cast<uint8_t *>(partial);
        if (!base) return UW_ERR_WORKSPACE;
        if (sk_counters) {
            t.sk_counters = sk_counters;
        } else {
            t.sk_counters = reinterpret_cast<uint32_t *>(base);
            t.partial = reinterpret_cast<float *>(base + sk_geometry(m, n, k, plan->bn).counter_bytes);
        }
        return cuda_status(launch_gemm_sk(t, stream));
    }
    return cuda_status(launch_gemm_tc(t, stream));
}

}  // namespace
}  // namespace uw

using namespace uw;

extern "C" const char *uw_status_str(int s) {
    switch (s) {
        case UW_OK: return "UW_OK";
        case UW_ERR_INVALID_ARG: return "UW_ERR_INVALID_ARG";
        case UW_ERR_UNSUPPORTED_SHAPE: return "UW_ERR_UNSUPPORTED_SHAPE";
        case UW_ERR_CORRUPT: return "UW_ERR_CORRUPT";
        case UW_ERR_CUDA: return "UW_ERR_CUDA";
        case UW_ERR_NOMEM: return "UW_ERR_NOMEM";
        case UW_ERR_TIMEOUT: return "UW_ERR_TIMEOUT";
        case UW_ERR_WORKSPACE: return "UW_ERR_WORKSPACE";
        default: return "UW_ERR_UNKNOWN";
    }
}

extern "C" const char *uw_version(void) { return "uw 1.1 (blob v2, sm_100a)"; }

extern "C" uw_status uw_matrix_bind(const void *host_blob, size_t bytes, const void *dev_blob,
                                    uint32_t *dev_status, int verify_payload, uw_dmat *out) {
    if (!host_blob || !dev_blob || !out) return UW_ERR_INVALID_ARG;
    if (!aligned(dev_blob, 256)) return UW_ERR_INVALID_ARG;
    Header h;
    uw_status st = parse_header(host_blob, bytes, verify_payload, h);
    if (st != UW_OK) return st;
    std::memset(out, 0, sizeof(*out));
    const uint8_t *b = static_cast<const uint8_t *>(dev_blob);
    out->n = h.n;
    out->k = h.k;
    out->flags = h.flags;
    out->palette_size = h.palette_size;
    std::memcpy(out->palette, h.palette, 16);
    std::memcpy(out->code_len, h.code_len, 16);
    out->n_groups = h.n_groups;
    out->n_raw = h.n_raw;
    out->n_chunks = h.n_chunks;
    out->stream_bits = h.stream_bits;
    out->stream_words = h.stream_words;
    out->sm = b + h.sec_off[UW_SEC_SM];
    out->rawexp = b + h.sec_off[UW_SEC_RAWEXP];
    out->flagbits = reinterpret_cast<const uint32_t *>(b + h.sec_off[UW_SEC_FLAGS]);
    out->rawbase = reinterpret_cast<const uint32_t *>(b + h.sec_off[UW_SEC_RAWBASE]);
    if (h.flags & UW_EMIT_HUFFMAN) {
        out->stream = reinterpret_cast<const uint32_t *>(b + h.sec_off[UW_SEC_STREAM]);
        out->chunk_off = reinterpret_cast<const uint32_t *>(b + h.sec_off[UW_SEC_CHUNKOFF]);
        out->dlut = reinterpret_cast<const uint32_t *>(b + h.sec_off[UW_SEC_DLUT]);
    }
    out->pal = (h.flags & UW_EMIT_PALETTE) ? b + h.sec_off[UW_SEC_PAL] : nullptr;
    out->dev_status = dev_status;
    return UW_OK;
}

extern "C" uw_status uw_device_status(const uw_dmat *w, void *stream) {
    if (!w || !w->dev_status) return UW_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return UW_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, w->dev_status, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return UW_ERR_CUDA;
    if (v) {
        if (cudaMemsetAsync(w->dev_status, 0, 4, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
            return UW_ERR_CUDA;
    }
    if (v & UW_DEVERR_CORRUPT) return UW_ERR_CORRUPT;
    if (v & UW_DEVERR_TIMEOUT) return UW_ERR_TIMEOUT;
    return UW_OK;
}

static uw_status check_dmat(const uw_dmat *w) {
    if (!w || !w->sm || !w->flagbits || !w->rawbase) return UW_ERR_INVALID_ARG;
    if (w->n <= 0 || w->k <= 0) return UW_ERR_INVALID_ARG;
    if (w->n % 64 || w->k % 64) return UW_ERR_UNSUPPORTED_SHAPE;
    return UW_OK;
}

extern "C" uw_status uw_decode_to_bf16(const uw_dmat *w, uint16_t *out_dev, void *stream) {
    uw_status st = check_dmat(w);
    if (st != UW_OK) return st;
    if (!out_dev || !aligned(out_dev, 16)) return UW_ERR_INVALID_ARG;
    if (!(w->flags & UW_EMIT_HUFFMAN) || !w->stream) return UW_ERR_INVALID_ARG;
    return cuda_status(launch_huff_decode(*w, out_dev, nullptr, static_cast<cudaStream_t>(stream)));
}

extern "C" uw_status uw_decode_exponents(const uw_dmat *w, uint8_t *exp_dev, void *stream) {
    uw_status st = check_dmat(w);
    if (st != UW_OK) return st;
    if (!exp_dev || !aligned(exp_dev, 16)) return UW_ERR_INVALID_ARG;
    if (!(w->flags & UW_EMIT_HUFFMAN) || !w->stream) return UW_ERR_INVALID_ARG;
    return cuda_status(launch_exp_decode(*w, exp_dev, nullptr, nullptr, static_cast<cudaStream_t>(stream)));
}

extern "C" uw_status uw_transcode_palette(const uw_dmat *w, uint8_t *pal_dev, void *stream) {
    uw_status st = check_dmat(w);
    if (st != UW_OK) return st;
    if (!pal_dev || !aligned(pal_dev, 16)) return UW_ERR_INVALID_ARG;
    if (!(w->flags & UW_EMIT_HUFFMAN) || !w->stream) return UW_ERR_INVALID_ARG;
    return cuda_status(launch_huff_decode(*w, nullptr, pal_dev, static_cast<cudaStream_t>(stream)));
}

extern "C" uw_status uw_plan_default(int64_t m, int64_t n, int64_t k, int32_t pipeline, uw_plan *plan) {
    if (!plan || m <= 0 || n <= 0 || k <= 0) return UW_ERR_INVALID_ARG;
    std::memset(plan, 0, sizeof(*plan));
    plan->pipeline = pipeline ? pipeline : UW_PIPE_DIRECT_PALETTE;
    if (m <= 8) {
        plan->kernel = UW_KERNEL_MMA;
        plan->bn = 4;            // 4 warps per 16-row tile
        plan->split_k = 1;
        plan->stages = 0;        // 32 weights per lane and step when K allows
    } else {
        plan->kernel = UW_KERNEL_TC;
        int bn = 16;
        while (bn < m && bn < 256) bn *= 2;
        plan->bn = bn;
        const int64_t tiles = ((n + 127) / 128) * ((m + bn - 1) / bn);
        int split = 1;
        while (tiles * split * 2 <= 148 * 2 && split * 2 <= int(k / 64) / 4) split *= 2;
        plan->split_k = split;
    }
    return UW_OK;
}

extern "C" uw_status uw_workspace_size(int64_t m, int64_t n, int64_t k, const uw_plan *plan,
                                       size_t *bytes) {
    if (!bytes || m <= 0 || n <= 0 || k <= 0) return UW_ERR_INVALID_ARG;
    uw_status st = check_plan(plan, m, k);
    if (st != UW_OK) return st;
    *bytes = size_t(prep_bytes(n, k, plan) + partial_bytes(m, n, k, plan));
    return UW_OK;
}

namespace uw {

uint64_t sk_counter_bytes(int64_t m, int64_t n, int64_t k, const uw_plan *plan) {
    if (!plan || m <= 0) return 0;
    if (plan->kernel == UW_KERNEL_MMA_SK) return gemv_sk_geometry(m, n, k, plan->bn).counter_bytes;
    if (plan->kernel != UW_KERNEL_TC_SK) return 0;
    return sk_geometry(m, n, k, plan->bn).counter_bytes;
}

uw_status fused_matmul_ex(const uint16_t *x_dev, int64_t m, const uw_dmat *w, const uint8_t *pal_dev, float *y_dev,
                          const uw_plan *plan, void *ws, size_t ws_bytes, uint32_t *sk_counters, cudaStream_t s) {
    uw_status st = check_dmat(w);
    if (st != UW_OK) return st;
    if (!x_dev || !y_dev || m <= 0) return UW_ERR_INVALID_ARG;
    if (!aligned(x_dev, 16) || !aligned(y_dev, 16)) return UW_ERR_INVALID_ARG;
    st = check_plan(plan, m, w->k);
    if (st != UW_OK) return st;
    const uint64_t need_prep = prep_bytes(w->n, w->k, plan),
                   need_part = partial_bytes(m, w->n, w->k, plan, sk_counters != nullptr);
    if (need_prep + need_part > 0 && (!ws || ws_bytes < need_prep + need_part || !aligned(ws, 256)))
        return UW_ERR_WORKSPACE;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    float *partial = need_part ? reinterpret_cast<float *>(wsb + need_prep) : nullptr;

    if (plan->pipeline == UW_PIPE_DECODE_GEMM) {
        if (!(w->flags & UW_EMIT_HUFFMAN)) return UW_ERR_INVALID_ARG;
        uint16_t *wd = reinterpret_cast<uint16_t *>(wsb);
        st = cuda_status(launch_huff_decode(*w, wd, nullptr, s));
        if (st != UW_OK) return st;
        return run_kernel(x_dev, m, wd, nullptr, nullptr, w->n, w->k, y_dev, plan, partial,
                          w->dev_status, sk_counters, s);
    }
    if (plan->pipeline == UW_PIPE_DECODE_EXP_FUSED) {
        if (!(w->flags & UW_EMIT_HUFFMAN)) return UW_ERR_INVALID_ARG;
        const ExpPlaneLayout L = exp_plane_layout(w->n, w->k);
        st = cuda_status(launch_exp_decode(*w, wsb, reinterpret_cast<uint32_t *>(wsb + L.flags_off),
                                           reinterpret_cast<uint32_t *>(wsb + L.rank_off), s));
        if (st != UW_OK) return st;
        const uw_dmat v = exp_plane_view(*w, wsb);
        return run_kernel(x_dev, m, nullptr, &v, v.pal, w->n, w->k, y_dev, plan, partial, w->dev_status,
                          sk_counters, s);
    }
    if (plan->pipeline == UW_PIPE_HUFFMAN_FUSED) {
        if (!(w->flags & UW_EMIT_HUFFMAN) || !w->stream || !w->chunk_off || !w->dlut) return UW_ERR_INVALID_ARG;
        return run_kernel(x_dev, m, nullptr, w, nullptr, w->n, w->k, y_dev, plan, partial, w->dev_status,
                          sk_counters, s, true);
    }
    const uint8_t *pal = nullptr;
    if (plan->pipeline == UW_PIPE_TRANSCODE_FUSED) {
        if (!(w->flags & UW_EMIT_HUFFMAN)) return UW_ERR_INVALID_ARG;
        st = cuda_status(launch_huff_decode(*w, nullptr, wsb, s));
        if (st != UW_OK) return st;
        pal = wsb;
    } else {
        pal = pal_dev ? pal_dev : w->pal;
        if (!pal || !aligned(pal, 16)) return UW_ERR_INVALID_ARG;
    }
    // the blob's own 4-bit plane: no kernel writes it (a transcoded or
    // caller-provided plane may still be being written by an earlier kernel)
    const bool w_stable = plan->pipeline == UW_PIPE_DIRECT_PALETTE && pal == w->pal;
    return run_kernel(x_dev, m, nullptr, w, pal, w->n, w->k, y_dev, plan, partial, w->dev_status, sk_counters, s,
                      false, w_stable);
}

uw_status matmul_bf16_ex(const uint16_t *x_dev, int64_t m, const uint16_t *w_dev, int64_t n, int64_t k, float *y_dev,
                         const uw_plan *plan, void *ws, size_t ws_bytes, uint32_t *dev_status, uint32_t *sk_counters,
                         cudaStream_t s) {
    if (!x_dev || !w_dev || !y_dev || m <= 0 || n <= 0 || k <= 0) return UW_ERR_INVALID_ARG;
    if (n % 64 || k % 64) return UW_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(x_dev, 16) || !aligned(w_dev, 16) || !aligned(y_dev, 16)) return UW_ERR_INVALID_ARG;
    uw_status st = check_plan(plan, m, k);
    if (st != UW_OK) return st;
    const uint64_t need = partial_bytes(m, n, k, plan, sk_counters != nullptr);
    if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 256))) return UW_ERR_WORKSPACE;
    return run_kernel(x_dev, m, w_dev, nullptr, nullptr, n, k, y_dev, plan, need ? static_cast<float *>(ws) : nullptr,
                      dev_status, sk_counters, s);
}

}  // namespace uw

extern "C" uw_status uw_fused_matmul(const uint16_t *x_dev, int64_t m, const uw_dmat *w,
                                     const uint8_t *pal_dev, float *y_dev, const uw_plan *plan,
                                     void *ws, size_t ws_bytes, void *stream) {
    return fused_matmul_ex(x_dev, m, w, pal_dev, y_dev, plan, ws, ws_bytes, nullptr,
                           static_cast<cudaStream_t>(stream));
}

extern "C" uw_status uw_fused_matmul_batched(const uw_batch_item *items, int n_items, const uw_plan *plan,
                                             void *stream) {
    if (!items || n_items <= 0 || !plan) return UW_ERR_INVALID_ARG;
    if (plan->pipeline != UW_PIPE_DIRECT_PALETTE || plan->kernel != UW_KERNEL_MMA) return UW_ERR_INVALID_ARG;
    std::vector<MmaItem> v(static_cast<size_t>(n_items));
    for (int i = 0; i < n_items; i++) {
        const uw_batch_item &it = items[i];
        uw_status st = check_dmat(it.w);
        if (st != UW_OK) return st;
        if (it.m < 0 || it.m > 16) return UW_ERR_INVALID_ARG;
        st = check_plan(plan, it.m > 0 ? it.m : 1, it.w->k);
        if (st != UW_OK) return st;
        if (it.m > 0) {
            if (!it.x_dev || !it.y_dev || !aligned(it.x_dev, 16) || !aligned(it.y_dev, 16)) return UW_ERR_INVALID_ARG;
            if (!it.w->pal || !aligned(it.w->pal, 16)) return UW_ERR_INVALID_ARG;
        }
        v[size_t(i)] = MmaItem{it.x_dev, int(it.m), it.w, it.y_dev};
    }
    return cuda_status(launch_gemv_mma_batched(v.data(), n_items, plan->bn, plan->stages,
                                               static_cast<cudaStream_t>(stream)));
}

extern "C" uw_status uw_matmul_bf16(const uint16_t *x_dev, int64_t m, const uint16_t *w_dev,
                                    int64_t n, int64_t k, float *y_dev, const uw_plan *plan,
                                    void *ws, size_t ws_bytes, uint32_t *dev_status, void *stream) {
    return matmul_bf16_ex(x_dev, m, w_dev, n, k, y_dev, plan, ws, ws_bytes, dev_status, nullptr,
                          static_cast<cudaStream_t>(stream));
}
