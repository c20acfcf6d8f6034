// autotune.cu -- measured plan selection (Unweight page §九: no single
// pipeline wins everywhere, so an autotuner times the candidates on the target
// GPU for every projection and batch size and writes a per-model plan file).
//
// For each matrix and each batch size m the candidates are the pipelines the
// blob supports (decode + plain kernel, exponent decode + fused kernel,
// runtime transcode + fused kernel, direct palette + fused kernel) crossed
// with the kernel variants: the
// warp-MMA kernel (m <= 16, 2-8 K slices per tile, 16 or 32 weights per lane
// and step), the FMA GEMV (m <= 8, 1 or 2 rows per warp) and the tcgen05
// kernel with token tiles around m and split-K factors 1-8 (so that some
// candidate fills the 148 SMs with close to whole waves).  Each candidate is
// run once to warm up (its status is checked) and then `reps` times, each
// call timed on its own between CUDA events after a 192 MB read of scratch
// space has pushed the matrix out of the 126 MB L2 (a read, so the evicted
// lines are clean and no write-back lands in the timed call): the weights
// stream from HBM as they do in a model's layer sequence.  The fastest
// average wins.  The persistent stream-K warp-MMA kernel (UW_KERNEL_MMA_SK)
// is not a candidate: it wins such single calls on some shapes by a few
// percent, but a step of calls run back to back is slower with it, since it
// fills every SM's shared memory and registers and so cannot start while
// the previous call drains, as the one-tile kernels do; it is used by
// explicit plan.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "kernels.h"
#include "uw_format.h"

namespace {

constexpr int kSMs = 148;
constexpr size_t kScrubBytes = size_t(192) << 20;   // > L2 (126 MB)

// Read `n` 16-byte words through L2 (the result only keeps the loads alive).
__global__ void k_l2_scrub(const uint4 *p, size_t n, uint32_t *sink) {
    uint32_t acc = 0;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x) {
        const uint4 v = __ldcg(p + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    if (acc == 0x9E3779B9u && threadIdx.x == 0 && blockIdx.x == 0) *sink = acc;
}

std::vector<uw_plan> candidates(const uw_dmat &w, int64_t m) {
    std::vector<int> pipes;
    if (w.flags & UW_EMIT_HUFFMAN) {
        pipes.push_back(UW_PIPE_DECODE_GEMM);
        pipes.push_back(UW_PIPE_DECODE_EXP_FUSED);
        pipes.push_back(UW_PIPE_TRANSCODE_FUSED);
    }
    if ((w.flags & UW_EMIT_PALETTE) && w.pal) pipes.push_back(UW_PIPE_DIRECT_PALETTE);
    std::vector<uw_plan> out;
    for (int pipe : pipes) {
        if (m <= 16)
            for (int width : {1, 2}) {
                if (width == 2 && w.k % 128) continue;
                for (int slices : {2, 4, 8}) {
                    uw_plan p{};
                    p.pipeline = pipe;
                    p.kernel = UW_KERNEL_MMA;
                    p.bn = slices;
                    p.split_k = 1;
                    p.stages = width;
                    out.push_back(p);
                }
            }
        if (m <= 8)
            for (int rows : {1, 2}) {
                uw_plan p{};
                p.pipeline = pipe;
                p.kernel = UW_KERNEL_FMA;
                p.bn = rows;
                p.split_k = 1;
                out.push_back(p);
            }
        int bn_hi = 16;
        while (bn_hi < m && bn_hi < 256) bn_hi *= 2;
        for (int bn : {bn_hi / 2, bn_hi}) {   // persistent stream-K kernel
            if (bn < 16) continue;
            uw_plan p{};
            p.pipeline = pipe;
            p.kernel = UW_KERNEL_TC_SK;
            p.bn = bn;
            p.split_k = 1;
            out.push_back(p);
            // the same kernel decoding the Huffman stream itself (pipeline 3's
            // transcode moved into the matmul)
            if (pipe == UW_PIPE_TRANSCODE_FUSED && bn <= 32 && w.k % 256 == 0) {
                p.pipeline = UW_PIPE_HUFFMAN_FUSED;
                out.push_back(p);
            }
        }
        for (int bn : {bn_hi / 2, bn_hi}) {
            if (bn < 16) continue;
            const int64_t tiles = ((w.n + 127) / 128) * ((m + bn - 1) / bn);
            const int ksteps = int(w.k / 64);
            for (int split : {1, 2, 3, 4, 5, 6, 8}) {
                if (split > 1 && (tiles * split > 4 * kSMs || ksteps / split < 4)) continue;
                if (split > 1 && tiles >= 2 * kSMs) continue;
                uw_plan p{};
                p.pipeline = pipe;
                p.kernel = UW_KERNEL_TC;
                p.bn = bn;
                p.split_k = split;
                out.push_back(p);
            }
        }
    }
    return out;
}

const char *pipe_name(int p) {
    switch (p) {
        case UW_PIPE_DECODE_GEMM: return "decode_gemm";
        case UW_PIPE_DECODE_EXP_FUSED: return "decode_exp_fused";
        case UW_PIPE_TRANSCODE_FUSED: return "transcode_fused";
        case UW_PIPE_HUFFMAN_FUSED: return "huffman_fused";
        default: return "direct_palette";
    }
}

const char *kernel_name(int k) {
    switch (k) {
        case UW_KERNEL_FMA: return "fma";
        case UW_KERNEL_MMA: return "mma";
        case UW_KERNEL_TC_SK: return "tc_sk";
        case UW_KERNEL_MMA_SK: return "mma_sk";
        default: return "tc";
    }
}

std::string plan_json(const uw_plan &p, double us) {
    char buf[256];
    std::snprintf(buf, sizeof buf,
                  "{\"pipeline\": \"%s\", \"kernel\": \"%s\", \"bn\": %d, \"split_k\": %d, \"stages\": %d, "
                  "\"us\": %.3f}",
                  pipe_name(p.pipeline), kernel_name(p.kernel),
                  p.bn, p.split_k, p.stages, us);
    return buf;
}

}  // namespace

extern "C" uw_status uw_autotune_workspace_size(const uw_dmat *const *mats, int n_mats,
                                                const int64_t *ms, int n_ms, size_t *bytes) {
    if (!mats || !ms || !bytes || n_mats <= 0 || n_ms <= 0) return UW_ERR_INVALID_ARG;
    size_t best = 0;
    for (int i = 0; i < n_mats; i++) {
        if (!mats[i]) return UW_ERR_INVALID_ARG;
        for (int j = 0; j < n_ms; j++) {
            if (ms[j] <= 0) return UW_ERR_INVALID_ARG;
            for (const uw_plan &p : candidates(*mats[i], ms[j])) {
                size_t b = 0;
                uw_status st = uw_workspace_size(ms[j], mats[i]->n, mats[i]->k, &p, &b);
                if (st != UW_OK) return st;
                best = std::max(best, b);
            }
        }
    }
    *bytes = (best + 255) / 256 * 256 + kScrubBytes;
    return UW_OK;
}

extern "C" uw_status uw_plan_autotune(const uw_dmat *const *mats, int n_mats, const int64_t *ms,
                                      int n_ms, const uint16_t *x_dev, float *y_dev, void *ws,
                                      size_t ws_bytes, int reps, uw_plan *plans_out, char *json_out,
                                      size_t json_cap, void *stream) {
    if (!mats || !ms || !x_dev || !y_dev || !plans_out || n_mats <= 0 || n_ms <= 0) return UW_ERR_INVALID_ARG;
    if (reps <= 0) reps = 5;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    size_t need = 0;
    uw_status ws_st = uw_autotune_workspace_size(mats, n_mats, ms, n_ms, &need);
    if (ws_st != UW_OK) return ws_st;
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return UW_ERR_WORKSPACE;
    const size_t cand_bytes = need - kScrubBytes;          // candidates use the front
    void *scrub = static_cast<uint8_t *>(ws) + cand_bytes;
    cudaEvent_t e0, e1;
    if (cudaEventCreate(&e0) != cudaSuccess) return UW_ERR_CUDA;
    if (cudaEventCreate(&e1) != cudaSuccess) {
        cudaEventDestroy(e0);
        return UW_ERR_CUDA;
    }
    std::string json = "{\"plans\": [";
    uw_status result = UW_OK;
    for (int i = 0; i < n_mats && result == UW_OK; i++) {
        const uw_dmat &w = *mats[i];
        for (int j = 0; j < n_ms && result == UW_OK; j++) {
            const int64_t m = ms[j];
            double best_us = 1e30;
            uw_plan best{};
            std::string cand_json;
            for (const uw_plan &p : candidates(w, m)) {
                // other candidates' partial sums share the front of the
                // workspace: a stream-K candidate starts from zeroed counters
                // (each completed call leaves them zero for its repetitions)
                const uint64_t cnt = uw::sk_counter_bytes(m, w.n, w.k, &p);
                if (cnt && cudaMemsetAsync(static_cast<uint8_t *>(ws) + uw::prep_workspace_bytes(w.n, w.k, p.pipeline),
                                           0, cnt, s) != cudaSuccess) {
                    result = UW_ERR_CUDA;
                    break;
                }
                uw_status st = uw_fused_matmul(x_dev, m, &w, nullptr, y_dev, &p, ws, cand_bytes, stream);
                if (st == UW_OK) st = w.dev_status ? uw_device_status(&w, stream)
                                                   : (cudaStreamSynchronize(s) == cudaSuccess ? UW_OK : UW_ERR_CUDA);
                if (st != UW_OK) {
                    if (st == UW_ERR_CUDA) {
                        result = st;
                        break;
                    }
                    continue;   // candidate not runnable here (e.g. workspace too small)
                }
                double total_ms = 0.0;
                for (int r = 0; r < reps && result == UW_OK; r++) {
                    float ms_el = 0.f;
                    k_l2_scrub<<<kSMs * 8, 256, 0, s>>>(static_cast<const uint4 *>(scrub), kScrubBytes / 16,
                                                       static_cast<uint32_t *>(scrub));
                    if (cudaGetLastError() != cudaSuccess || cudaEventRecord(e0, s) != cudaSuccess ||
                        uw_fused_matmul(x_dev, m, &w, nullptr, y_dev, &p, ws, cand_bytes, stream) != UW_OK ||
                        cudaEventRecord(e1, s) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
                        cudaEventElapsedTime(&ms_el, e0, e1) != cudaSuccess)
                        result = UW_ERR_CUDA;
                    total_ms += ms_el;
                }
                if (result != UW_OK) break;
                const double us = 1000.0 * total_ms / reps;
                if (!cand_json.empty()) cand_json += ", ";
                cand_json += plan_json(p, us);
                if (us < best_us) {
                    best_us = us;
                    best = p;
                }
            }
            if (result != UW_OK) break;
            if (best_us >= 1e30) {
                result = UW_ERR_WORKSPACE;
                break;
            }
            plans_out[i * n_ms + j] = best;
            char head[160];
            std::snprintf(head, sizeof head, "%s{\"matrix\": %d, \"n\": %lld, \"k\": %lld, \"m\": %lld, \"best\": ",
                          (i == 0 && j == 0) ? "" : ", ", i, (long long)w.n, (long long)w.k, (long long)m);
            json += head + plan_json(best, best_us) + ", \"candidates\": [" + cand_json + "]}";
        }
    }
    json += "]}";
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (result != UW_OK) return result;
    if (json_out) {
        if (json.size() + 1 > json_cap) return UW_ERR_INVALID_ARG;
        std::memcpy(json_out, json.c_str(), json.size() + 1);
    }
    return UW_OK;
}
