// The whole forward with its workspace in a fixed device-side scratch array,
// for callers that cannot allocate device memory when they call: a host
// program or plugin that is handed device tensors and a stream but owns no
// device allocator, or a latency-bound loop where cudaMalloc and cudaFree are
// off limits because they can synchronise the whole device.  This entry point
// allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
//
// The scratch is one file-scope array per device (the CUDA module's own
// global memory), of kStaticScratchBytes.  The first call on a device looks
// up its address with cudaGetSymbolAddress while that device is current and
// caches it; later calls on that device reuse the cached address (after a
// cudaDeviceReset the cached address is stale: reload the library).  Because
// there is one scratch per device, calls on one device must not overlap in
// time (two streams, two host threads): overlapping calls race on it.
//
// Nothing in the scratch needs to start at zero before a call: the
// mask-preparation kernel that every forward runs first clears the status
// word and the global-row arrival counters and writes every other region
// (indices, counts, flags, bitmaps) before the attention kernels read them.
#include <mutex>

#include "../../include/lf_attention.h"
#include "lf_device.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(LF_STATIC_SCRATCH_BYTES);
constexpr int kMaxScratchDevices = 64;

static_assert(kStaticScratchBytes % 256 == 0, "scratch size must keep 256-byte regions");

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxScratchDevices];

// Address of the current device's scratch, looked up once per device.
int current_scratch(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LF_ERR_NO_DEVICE;
    }
    if (dev < 0 || dev >= kMaxScratchDevices) return LF_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return LF_ERR_CUDA;
        }
        if (reinterpret_cast<uintptr_t>(p) % 256 != 0) return LF_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LF_OK;
}

}  // namespace

extern "C" int lf_attention_forward_static(lf_dtype dtype, int B, int H, int n, int d_head,
                                           const void *q, const void *k, const void *v,
                                           const void *qg, const void *kg, const void *vg,
                                           const uint8_t *local_mask, const uint8_t *global_mask,
                                           int max_global, int window, const int32_t *dilation,
                                           int causal, void *out, lf_stream_t stream,
                                           void **scratch)
{
    // Sizes that have no workspace (lf_workspace_size returns 0) and problems
    // whose workspace does not fit are refused before the device is touched:
    // no context is created and no module is loaded for them.
    if (d_head != lf::kDHead) return LF_ERR_UNSUPPORTED;
    const size_t need = lf_workspace_size(B, H, n, d_head, max_global);
    if (need == 0) return LF_ERR_INVALID_ARG;
    if (need > kStaticScratchBytes) return LF_ERR_SCRATCH_LIMIT;
    void *ws = nullptr;
    if (int rc = current_scratch(&ws)) return rc;
    if (scratch) *scratch = ws;
    return lf_attention_forward(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, local_mask,
                                global_mask, max_global, window, dilation, causal, out, ws,
                                kStaticScratchBytes, stream);
}
