// stack.cu -- uw_stack_run: a sequence of matmuls (the projections of a
// stack of MLP layers) with cross-layer overlap (Unweight page §八: while a
// palette layer runs the fused matmul, the next Huffman layer is decoded on a
// side stream).
//
// Every step's matmul runs on the main stream, in step order, so a step may
// read what an earlier step wrote.  A step whose plan needs preprocessing
// (pipeline 1: full decode to BF16; pipeline 2: exponent-only decode;
// pipeline 3: transcode to the 4-bit plane) has it issued on the side stream
// into one of two workspace slots,
// as soon as the slot's previous user has finished; its matmul then waits for
// that preprocessing.  So the decode of step i+1 (or i+2) runs while the main
// stream is still busy with step i.  Preprocessing reads only the weights,
// which no step writes.
//
// Synchronisation uses five events per call (slot ready and slot free for
// each slot, and a fork/join marker), created here and released when the
// work that uses them completes.  At entry
// the side stream waits for all work already queued on the main stream (an
// earlier call may still use the workspace), and at exit the main stream waits
// for the side stream, so completion of the main stream means completion of
// the whole call.
#include <algorithm>
#include <cstring>

#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

inline bool needs_prep(const uw_plan &p) {
    return p.pipeline == UW_PIPE_DECODE_GEMM || p.pipeline == UW_PIPE_DECODE_EXP_FUSED ||
           p.pipeline == UW_PIPE_TRANSCODE_FUSED;
}

struct StackLayout {
    uint64_t slot_bytes = 0;      // one preprocessing slot (2 slots)
    uint64_t partial_bytes = 0;   // split-K partial sums / stream-K partial tiles, reused by every step
    uint64_t counter_bytes = 0;   // stream-K tile counters, apart from the partial sums
    uint64_t total() const { return 2 * slot_bytes + partial_bytes + counter_bytes; }
};

uw_status layout(const uw_stack_step *steps, int n_steps, StackLayout &L) {
    if (!steps || n_steps <= 0) return UW_ERR_INVALID_ARG;
    L = StackLayout{};
    for (int i = 0; i < n_steps; i++) {
        const uw_stack_step &s = steps[i];
        if (!s.w) return UW_ERR_INVALID_ARG;
        size_t all = 0;
        uw_status st = uw_workspace_size(s.m, s.w->n, s.w->k, &s.plan, &all);
        if (st != UW_OK) return st;
        const uint64_t prep = prep_workspace_bytes(s.w->n, s.w->k, s.plan.pipeline);
        const uint64_t counters = sk_counter_bytes(s.m, s.w->n, s.w->k, &s.plan);
        L.slot_bytes = std::max(L.slot_bytes, prep);
        L.partial_bytes = std::max(L.partial_bytes, uint64_t(all) - prep - counters);
        L.counter_bytes = std::max(L.counter_bytes, counters);
    }
    return UW_OK;
}

struct Events {
    cudaEvent_t ev[5] = {};
    int made = 0;
    cudaError_t make() {
        for (; made < 5; made++) {
            cudaError_t e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    ~Events() {
        for (int i = 0; i < made; i++) cudaEventDestroy(ev[i]);
    }
};

}  // namespace
}  // namespace uw

using namespace uw;

extern "C" uw_status uw_stack_workspace_size(const uw_stack_step *steps, int n_steps, size_t *bytes) {
    if (!bytes) return UW_ERR_INVALID_ARG;
    StackLayout L;
    uw_status st = layout(steps, n_steps, L);
    if (st != UW_OK) return st;
    *bytes = size_t(L.total());
    return UW_OK;
}

extern "C" uw_status uw_stack_run(const uw_stack_step *steps, int n_steps, void *ws, size_t ws_bytes,
                                  void *stream, void *side_stream) {
    StackLayout L;
    uw_status st = layout(steps, n_steps, L);
    if (st != UW_OK) return st;
    if (L.total() > 0 && (!ws || ws_bytes < L.total() || (reinterpret_cast<uintptr_t>(ws) & 255u)))
        return UW_ERR_WORKSPACE;
    // argument checks up front, so that nothing is launched for a bad stack
    for (int i = 0; i < n_steps; i++) {
        const uw_stack_step &s = steps[i];
        if (!s.x_dev || !s.y_dev || s.m <= 0) return UW_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(s.x_dev) | reinterpret_cast<uintptr_t>(s.y_dev)) & 15u) return UW_ERR_INVALID_ARG;
        if (s.w->n <= 0 || s.w->k <= 0) return UW_ERR_INVALID_ARG;
        if (s.w->n % 64 || s.w->k % 64) return UW_ERR_UNSUPPORTED_SHAPE;
        if (needs_prep(s.plan) || s.plan.pipeline == UW_PIPE_HUFFMAN_FUSED) {
            if (!(s.w->flags & UW_EMIT_HUFFMAN) || !s.w->stream) return UW_ERR_INVALID_ARG;
        } else {
            const uint8_t *pal = s.pal_dev ? s.pal_dev : s.w->pal;
            if (!pal || (reinterpret_cast<uintptr_t>(pal) & 15u)) return UW_ERR_INVALID_ARG;
        }
    }
    cudaStream_t main_s = static_cast<cudaStream_t>(stream);
    cudaStream_t side_s = static_cast<cudaStream_t>(side_stream);
    const bool overlap = side_stream != nullptr && side_s != main_s;
    uint8_t *slot[2] = {static_cast<uint8_t *>(ws), static_cast<uint8_t *>(ws) + L.slot_bytes};
    void *partial = L.partial_bytes ? static_cast<uint8_t *>(ws) + 2 * L.slot_bytes : nullptr;
    uint32_t *counters =
        L.counter_bytes ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + 2 * L.slot_bytes + L.partial_bytes)
                        : nullptr;

    // ev[0..1]: slot s holds its step's prepared weights; ev[2..3]: slot s is
    // free again; ev[4]: fork / join marker
    Events E;
    if (overlap) {
        if (E.make() != cudaSuccess) return UW_ERR_CUDA;
        if (cudaEventRecord(E.ev[4], main_s) != cudaSuccess || cudaStreamWaitEvent(side_s, E.ev[4], 0) != cudaSuccess)
            return UW_ERR_CUDA;
    }
    int n_prep = 0;
    for (int i = 0; i < n_steps && st == UW_OK; i++) {
        const uw_stack_step &s = steps[i];
        const uw_dmat *w = s.w;
        if (!needs_prep(s.plan)) {
            st = fused_matmul_ex(s.x_dev, s.m, w, s.pal_dev, s.y_dev, &s.plan, partial, L.partial_bytes, counters,
                                 main_s);
            continue;
        }
        const int b = n_prep & 1;
        cudaStream_t prep_s = overlap ? side_s : main_s;
        if (overlap && n_prep >= 2 && cudaStreamWaitEvent(side_s, E.ev[2 + b], 0) != cudaSuccess) {
            st = UW_ERR_CUDA;
            break;
        }
        if (s.plan.pipeline == UW_PIPE_DECODE_GEMM) {
            st = uw_decode_to_bf16(w, reinterpret_cast<uint16_t *>(slot[b]), prep_s);
        } else if (s.plan.pipeline == UW_PIPE_DECODE_EXP_FUSED) {
            const ExpPlaneLayout EL = exp_plane_layout(w->n, w->k);
            st = launch_exp_decode(*w, slot[b], reinterpret_cast<uint32_t *>(slot[b] + EL.flags_off),
                                   reinterpret_cast<uint32_t *>(slot[b] + EL.rank_off), prep_s) == cudaSuccess
                     ? UW_OK
                     : UW_ERR_CUDA;
        } else {
            st = uw_transcode_palette(w, slot[b], prep_s);
        }
        if (st != UW_OK) break;
        if (overlap && (cudaEventRecord(E.ev[b], side_s) != cudaSuccess ||
                        cudaStreamWaitEvent(main_s, E.ev[b], 0) != cudaSuccess)) {
            st = UW_ERR_CUDA;
            break;
        }
        if (s.plan.pipeline == UW_PIPE_DECODE_GEMM) {
            st = matmul_bf16_ex(s.x_dev, s.m, reinterpret_cast<const uint16_t *>(slot[b]), w->n, w->k, s.y_dev,
                                &s.plan, partial, L.partial_bytes, w->dev_status, counters, main_s);
        } else {
            // pipeline 3: the fused kernel on the transcoded plane; pipeline 2:
            // on the all-raw view whose raw plane is the decoded exponents
            uw_plan p = s.plan;
            p.pipeline = UW_PIPE_DIRECT_PALETTE;
            const uw_dmat v = s.plan.pipeline == UW_PIPE_DECODE_EXP_FUSED ? exp_plane_view(*w, slot[b]) : *w;
            st = fused_matmul_ex(s.x_dev, s.m, &v, slot[b], s.y_dev, &p, partial, L.partial_bytes, counters, main_s);
        }
        if (st == UW_OK && overlap && cudaEventRecord(E.ev[2 + b], main_s) != cudaSuccess) st = UW_ERR_CUDA;
        n_prep++;
    }
    // join: the main stream waits for everything issued on the side stream (also after an error)
    if (overlap && (cudaEventRecord(E.ev[4], side_s) != cudaSuccess || cudaStreamWaitEvent(main_s, E.ev[4], 0) != cudaSuccess))
        st = st == UW_OK ? UW_ERR_CUDA : st;
    return st;
}
