// An allocation-free variant of gdn_prefill_chunked for callers that cannot allocate device
// memory themselves: code running where cudaMalloc is unavailable or forbidden (inside a
// host callback or a capture-restricted region, a plugin whose host owns all allocations,
// a real-time loop that must not touch the allocator). Instead of a caller workspace, the
// tensor-core path uses a fixed scratch array that lives in this library's device image.
//
// The array is a file-scope __device__ object: every GPU that loads this part of the
// library holds kStaticScratchBytes of device memory for it until the process exits. Its
// host-side name is only a stand-in; the device address is looked up once per device with
// cudaGetSymbolAddress while that device is current, on the entry point's first call there.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;   // 32 MiB

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
uint8_t *g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (set-up on first use).
cudaError_t scratch_for_current_device(uint8_t **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

gdn_status gdn_prefill_chunked_static_ws(const void *q, const void *k, const void *v, const float *a,
                                         const float *b, const float *A_log, const float *dt_bias,
                                         const int32_t *cu_seqlens, int32_t num_seqs, int32_t T, int32_t Hk,
                                         int32_t Hv, int32_t Dk, int32_t Dv, float scale, int32_t qk_l2norm,
                                         gdn_dtype in_dtype, const float *initial_state, float *final_state,
                                         void *o, gdn_dtype out_dtype, gdn_stream_t stream) {
    const size_t need = gdn_prefill_workspace_bytes(T, num_seqs, Hk, Hv, Dk, Dv);
    if (need > kStaticScratchBytes) return GDN_ERR_WORKSPACE;   // larger than the fixed scratch
    uint8_t *scratch = nullptr;
    if (need > 0 && scratch_for_current_device(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens, num_seqs, T, Hk, Hv, Dk, Dv, scale,
                               qk_l2norm, in_dtype, initial_state, final_state, o, out_dtype, scratch,
                               need > 0 ? kStaticScratchBytes : 0, stream);
}

}  // extern "C"
