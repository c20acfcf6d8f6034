// noalloc.cu -- uw_fused_matmul_noalloc: the matmul for callers that cannot
// hand the library any device memory as workspace.
//
// Some callers cannot allocate device memory when they call in: an inference
// engine that gives its plug-ins no allocator and forbids cudaMalloc after
// start-up, or a process whose device memory is already fully reserved by
// another allocator.  For them this entry point keeps its scratch (the split-K
// partial sums) in a fixed array in the library's own device memory, which
// every GPU that loads the library holds until the process exits.
//
// The array's name is only a host-side stand-in: the device address is
// obtained once per device, with that device current, through
// cudaGetSymbolAddress, and that address is what the kernels receive.
#include <atomic>
#include <mutex>

#include "kernels.h"
#include "uw_format.h"

namespace uw {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;   // UW_NOALLOC_SCRATCH_BYTES
constexpr size_t kCounterBytes = size_t(64) << 10;   // UW_NOALLOC_COUNTER_BYTES
static_assert(kScratchBytes == UW_NOALLOC_SCRATCH_BYTES, "header and library disagree");
static_assert(kCounterBytes == UW_NOALLOC_COUNTER_BYTES, "header and library disagree");

// Scratch of uw_fused_matmul_noalloc, shared by every call on a device: the
// first kCounterBytes hold the stream-K kernel's tile counters (zero at
// load, and every completed call leaves them zero), the rest the split-K
// partial sums or stream-K partial tiles.  Keeping the counters apart means
// a split-K call's partial sums never land on them.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];
std::mutex g_setup_mutex;

// Device address of g_noalloc_scratch on the current device (looked up once).
uw_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return UW_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return UW_ERR_INVALID_ARG;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        p = g_scratch_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return UW_ERR_CUDA;
            g_scratch_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return UW_OK;
}

}  // namespace
}  // namespace uw

using namespace uw;

extern "C" uw_status uw_fused_matmul_noalloc(const uint16_t *x_dev, int64_t m, const uw_dmat *w,
                                             float *y_dev, const uw_plan *plan, void *stream) {
    if (!x_dev || !w || !y_dev || !plan || m <= 0) return UW_ERR_INVALID_ARG;
    if (plan->pipeline != UW_PIPE_DIRECT_PALETTE) return UW_ERR_INVALID_ARG;
    size_t need = 0;
    uw_status st = uw_workspace_size(m, w->n, w->k, plan, &need);
    if (st != UW_OK) return st;
    const uint64_t counters = sk_counter_bytes(m, w->n, w->k, plan);
    if (counters > kCounterBytes || need - counters > kScratchBytes - kCounterBytes) return UW_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != UW_OK) return st;
    uint8_t *base = static_cast<uint8_t *>(scratch);
    return fused_matmul_ex(x_dev, m, w, nullptr, y_dev, plan, base + kCounterBytes, kScratchBytes - kCounterBytes,
                           reinterpret_cast<uint32_t *>(base), static_cast<cudaStream_t>(stream));
}
