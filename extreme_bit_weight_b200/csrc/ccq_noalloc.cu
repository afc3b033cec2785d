// ccq_w2a16_gemm_noalloc: the W2A16 matmul for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a device workspace: a plugin that a host framework hands
// only its input and output pointers (the framework owns and pre-plans all device memory), or a
// latency-critical loop that must not call cudaMalloc/cudaFree, which can synchronize the whole
// device.  For them this entry point runs the same matmul as ccq_w2a16_gemm, with its scratch
// (the packed activation operand, group sums and split-K partial sums) in a fixed array in the
// library's own device memory instead of a caller workspace.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// kNoAllocScratchBytes of it until the process exits.  In host code its name is only a host-side
// handle, so the device address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and cached; the first call on each device does this lookup.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/ccq.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device).
void *scratch_for_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" size_t ccq_w2a16_gemm_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

extern "C" ccq_status ccq_w2a16_gemm_noalloc(const ccq_weight *w, const void *x_bf16, int32_t m, void *y_bf16,
                                             ccq_stream_t stream) {
    if (!w || m < 0) return CCQ_ERR_INVALID_ARG;
    if (m == 0) return ccq_w2a16_gemm(w, x_bf16, m, y_bf16, nullptr, 0, stream);
    const size_t need = ccq_gemm_workspace_size(w, m);
    if (need == 0) return CCQ_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return CCQ_ERR_UNSUPPORTED;  // shape needs more scratch than the array holds
    void *scratch = scratch_for_current_device();
    if (!scratch) return CCQ_ERR_CUDA;
    return ccq_w2a16_gemm(w, x_bf16, m, y_bf16, scratch, kNoAllocScratchBytes, stream);
}
