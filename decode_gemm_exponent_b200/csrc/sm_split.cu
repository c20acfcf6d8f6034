// sm_split.cu -- decode/compute SM split (Unweight page §九: besides the
// pipeline and the kernel variant, the autotuner measures how the SMs are
// divided between decoding and compute).
//
// On this GPU the division is a pair of green contexts: the driver splits the
// device's SMs into a preprocessing partition (whole granules of 8 SMs) and
// the remainder, and each partition gets one stream.  Work on a partition's
// stream runs only on that partition's SMs, so a layer stack run with the
// matmuls on the compute stream and the decodes on the preprocessing stream
// (uw_stack_run) keeps the two apart instead of letting the decode take SMs
// from the matmuls as the hardware scheduler sees fit.  Both streams belong to
// the device's primary context, so the library's kernels, events and the
// caller's memory work on them unchanged.
//
// uw_stack_tune_split measures a stack under several splits (and without one)
// and returns the fastest.  The driver entry points are resolved at run time
// through the CUDA runtime, like the tensor-map encoder, so the library still
// loads where there is no driver; every call then returns UW_ERR_CUDA.
#include <cstring>
#include <vector>

#include "kernels.h"

struct uw_sm_split {
    CUgreenCtx ctx[2] = {nullptr, nullptr};   // [0] preprocessing, [1] compute
    CUstream stream[2] = {nullptr, nullptr};
    int sms[2] = {0, 0};
};

namespace uw {
namespace {

struct GreenApi {
    CUresult (*device_get)(CUdevice *, int) = nullptr;
    CUresult (*get_resource)(CUdevice, CUdevResource *, CUdevResourceType) = nullptr;
    CUresult (*split_by_count)(CUdevResource *, unsigned int *, const CUdevResource *, CUdevResource *,
                               unsigned int, unsigned int) = nullptr;
    CUresult (*generate_desc)(CUdevResourceDesc *, CUdevResource *, unsigned int) = nullptr;
    CUresult (*ctx_create)(CUgreenCtx *, CUdevResourceDesc, CUdevice, unsigned int) = nullptr;
    CUresult (*stream_create)(CUstream *, CUgreenCtx, unsigned int, int) = nullptr;
    CUresult (*ctx_destroy)(CUgreenCtx) = nullptr;
    CUresult (*stream_destroy)(CUstream) = nullptr;
    bool ok = false;
};

template <class F>
bool resolve(const char *name, F &fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return false;
    fn = reinterpret_cast<F>(p);
    return true;
}

const GreenApi &green_api() {
    static const GreenApi api = [] {
        GreenApi a;
        a.ok = resolve("cuDeviceGet", a.device_get) && resolve("cuDeviceGetDevResource", a.get_resource) &&
               resolve("cuDevSmResourceSplitByCount", a.split_by_count) &&
               resolve("cuDevResourceGenerateDesc", a.generate_desc) && resolve("cuGreenCtxCreate", a.ctx_create) &&
               resolve("cuGreenCtxStreamCreate", a.stream_create) && resolve("cuGreenCtxDestroy", a.ctx_destroy) &&
               resolve("cuStreamDestroy", a.stream_destroy);
        return a;
    }();
    return api;
}

void release(uw_sm_split *s) {
    const GreenApi &api = green_api();
    for (int i = 0; i < 2; i++) {
        if (s->stream[i]) api.stream_destroy(s->stream[i]);
        if (s->ctx[i]) api.ctx_destroy(s->ctx[i]);
    }
    delete s;
}

// one candidate's streams: a split, or two ordinary streams sharing all SMs
struct Lanes {
    uw_sm_split *split = nullptr;
    cudaStream_t own[2] = {nullptr, nullptr};
    cudaStream_t prep() const { return split ? reinterpret_cast<cudaStream_t>(split->stream[0]) : own[0]; }
    cudaStream_t compute() const { return split ? reinterpret_cast<cudaStream_t>(split->stream[1]) : own[1]; }
    ~Lanes() {
        for (cudaStream_t s : own)
            if (s) cudaStreamDestroy(s);
        if (split) release(split);
    }
};

}  // namespace
}  // namespace uw

using namespace uw;

extern "C" uw_status uw_sm_split_create(int device, int prep_sms, uw_sm_split **out) {
    if (!out || device < 0 || prep_sms <= 0) return UW_ERR_INVALID_ARG;
    *out = nullptr;
    int total = 0;
    if (cudaDeviceGetAttribute(&total, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return UW_ERR_CUDA;
    if (prep_sms >= total) return UW_ERR_INVALID_ARG;
    const GreenApi &api = green_api();
    if (!api.ok) return UW_ERR_CUDA;
    CUdevice dev;
    CUdevResource all, part, rest;
    std::memset(&all, 0, sizeof all);
    std::memset(&part, 0, sizeof part);
    std::memset(&rest, 0, sizeof rest);
    unsigned int groups = 1;
    if (api.device_get(&dev, device) != CUDA_SUCCESS ||
        api.get_resource(dev, &all, CU_DEV_RESOURCE_TYPE_SM) != CUDA_SUCCESS ||
        api.split_by_count(&part, &groups, &all, &rest, 0u, unsigned(prep_sms)) != CUDA_SUCCESS)
        return UW_ERR_CUDA;
    if (groups != 1 || part.sm.smCount == 0 || rest.sm.smCount == 0) return UW_ERR_INVALID_ARG;
    uw_sm_split *s = new uw_sm_split;
    CUdevResource *res[2] = {&part, &rest};
    for (int i = 0; i < 2; i++) {
        CUdevResourceDesc desc;
        if (api.generate_desc(&desc, res[i], 1) != CUDA_SUCCESS ||
            api.ctx_create(&s->ctx[i], desc, dev, CU_GREEN_CTX_DEFAULT_STREAM) != CUDA_SUCCESS ||
            api.stream_create(&s->stream[i], s->ctx[i], CU_STREAM_NON_BLOCKING, 0) != CUDA_SUCCESS) {
            release(s);
            return UW_ERR_CUDA;
        }
        s->sms[i] = int(res[i]->sm.smCount);
    }
    *out = s;
    return UW_OK;
}

extern "C" uw_status uw_sm_split_get(const uw_sm_split *s, void **prep_stream, void **compute_stream,
                                     int *prep_sms, int *compute_sms) {
    if (!s) return UW_ERR_INVALID_ARG;
    if (prep_stream) *prep_stream = s->stream[0];
    if (compute_stream) *compute_stream = s->stream[1];
    if (prep_sms) *prep_sms = s->sms[0];
    if (compute_sms) *compute_sms = s->sms[1];
    return UW_OK;
}

extern "C" void uw_sm_split_destroy(uw_sm_split *s) {
    if (s) release(s);
}

extern "C" uw_status uw_stack_tune_split(const uw_stack_step *steps, int n_steps, void *ws, size_t ws_bytes,
                                         int device, const int *cand, int n_cand, int reps, int *best,
                                         float *us_out, void *stream) {
    if (!steps || n_steps <= 0 || !cand || n_cand <= 0 || !best || device < 0) return UW_ERR_INVALID_ARG;
    for (int c = 0; c < n_cand; c++)
        if (cand[c] < 0) return UW_ERR_INVALID_ARG;
    size_t need = 0;
    uw_status st = uw_stack_workspace_size(steps, n_steps, &need);
    if (st != UW_OK) return st;
    if (need > 0 && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))) return UW_ERR_WORKSPACE;
    if (reps <= 0) reps = 5;
    // the steps' inputs may still be in flight on the caller's stream
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return UW_ERR_CUDA;
    cudaEvent_t e[2] = {nullptr, nullptr};
    if (cudaEventCreate(&e[0]) != cudaSuccess || cudaEventCreate(&e[1]) != cudaSuccess) {
        if (e[0]) cudaEventDestroy(e[0]);
        return UW_ERR_CUDA;
    }
    float best_us = 0.f;
    *best = -1;
    for (int c = 0; c < n_cand && st == UW_OK; c++) {
        Lanes L;
        if (cand[c] == 0) {
            if (cudaStreamCreateWithFlags(&L.own[0], cudaStreamNonBlocking) != cudaSuccess ||
                cudaStreamCreateWithFlags(&L.own[1], cudaStreamNonBlocking) != cudaSuccess)
                st = UW_ERR_CUDA;
        } else {
            st = uw_sm_split_create(device, cand[c], &L.split);
        }
        if (st != UW_OK) break;
        float ms = 0.f;
        st = uw_stack_run(steps, n_steps, ws, ws_bytes, L.compute(), L.prep());   // warm-up
        if (st == UW_OK && cudaEventRecord(e[0], L.compute()) != cudaSuccess) st = UW_ERR_CUDA;
        for (int r = 0; r < reps && st == UW_OK; r++) st = uw_stack_run(steps, n_steps, ws, ws_bytes, L.compute(), L.prep());
        if (st == UW_OK && (cudaEventRecord(e[1], L.compute()) != cudaSuccess || cudaEventSynchronize(e[1]) != cudaSuccess ||
                            cudaEventElapsedTime(&ms, e[0], e[1]) != cudaSuccess))
            st = UW_ERR_CUDA;
        // whatever happened, nothing may still run on the streams destroyed here
        if (cudaStreamSynchronize(L.compute()) != cudaSuccess || cudaStreamSynchronize(L.prep()) != cudaSuccess)
            st = st == UW_OK ? UW_ERR_CUDA : st;
        if (st != UW_OK) break;
        const float us = 1000.f * ms / float(reps);
        if (us_out) us_out[c] = us;
        if (*best < 0 || us < best_us) {
            best_us = us;
            *best = cand[c];
        }
    }
    cudaEventDestroy(e[0]);
    cudaEventDestroy(e[1]);
    return st;
}
