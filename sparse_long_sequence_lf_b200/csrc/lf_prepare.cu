// Mask preparation: global-index compaction and per-batch bitmaps.
//
// The FasterTransformer Longformer Encoder guide ("compute flow") extracts,
// once before the layer loop, the positions of the global tokens of each batch
// and their count from the global mask, and turns the local mask into an
// additive -10000 bias.  Here one CTA per batch does a stable ascending
// compaction with warp ballots and a block-wide prefix sum, and the local mask
// becomes a bitmap of valid keys (exclusion, not a bias).  The same pass
// builds a bitmap of global tokens, a has-padding flag, and clears the
// arrival counters of the global-row combine.
#include "lf_device.cuh"

namespace lf {

constexpr int kPrepThreads = 1024;
constexpr int kPrepWarps = kPrepThreads / 32;

// One CTA per batch.  Any output pointer may be NULL (not written).
__global__ void __launch_bounds__(kPrepThreads)
prepare_kernel(const uint8_t *__restrict__ local_mask, const uint8_t *__restrict__ global_mask,
               int B, int n, int max_global, int32_t *gidx, int32_t *counts, int *flags,
               uint32_t *vbits, uint32_t *gbits, int *status, int *counters, int counters_per_batch)
{
    __shared__ int warp_tot[kPrepWarps];
    __shared__ int s_base;
    __shared__ int s_pad;

    const int b = blockIdx.x;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const uint8_t *lm = local_mask ? local_mask + size_t(b) * n : nullptr;
    const uint8_t *gm = global_mask ? global_mask + size_t(b) * n : nullptr;
    const int nwords = (n + 31) / 32;

    if (tid == 0) {
        s_base = 0;
        s_pad = 0;
        if (b == 0 && status) *status = 0;
    }
    if (counters)
        for (int c = tid; c < counters_per_batch; c += kPrepThreads)
            counters[size_t(b) * counters_per_batch + c] = 0;
    __syncthreads();

    int any_pad = 0;
    for (int start = 0; start < n; start += kPrepThreads) {
        const int p = start + tid;
        const bool in = p < n;
        const bool is_g = in && gm && gm[p] != 0;
        const bool valid = in && (lm == nullptr || lm[p] != 0);
        any_pad |= (in && !valid);
        const unsigned gball = __ballot_sync(0xffffffffu, is_g);
        const unsigned vball = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) {
            const int word = p >> 5;
            if (word < nwords) {
                if (vbits) vbits[size_t(b) * nwords + word] = vball;
                if (gbits) gbits[size_t(b) * nwords + word] = gball;
            }
            warp_tot[warp] = __popc(gball);
        }
        __syncthreads();
        // Exclusive prefix over the warps of this chunk (warp totals are small).
        int before = 0, total = 0;
        for (int w = 0; w < kPrepWarps; ++w) {
            const int t = warp_tot[w];
            before += (w < warp) ? t : 0;
            total += t;
        }
        if (is_g && gidx) {
            const int rank = before + __popc(gball & ((1u << lane) - 1u));
            gidx[size_t(b) * n + s_base + rank] = p;
        }
        __syncthreads();
        if (tid == 0) s_base += total;
        __syncthreads();
    }
    const int count = s_base;
    if (gidx)
        for (int p = count + tid; p < n; p += kPrepThreads) gidx[size_t(b) * n + p] = -1;
    any_pad = __syncthreads_or(any_pad);
    if (tid == 0) {
        if (counts) counts[b] = count;
        if (flags)
            flags[b] = (any_pad ? kFlagHasPadding : 0) | (count > max_global ? kFlagOverflow : 0);
    }
}

int launch_prepare(const uint8_t *local_mask, const uint8_t *global_mask, int B, int n,
                   int max_global, int32_t *gidx, int32_t *counts, int *flags, uint32_t *vbits,
                   uint32_t *gbits, int *status, int *counters, int counters_per_batch,
                   cudaStream_t stream)
{
    prepare_kernel<<<B, kPrepThreads, 0, stream>>>(local_mask, global_mask, B, n, max_global, gidx,
                                                   counts, flags, vbits, gbits, status, counters,
                                                   counters_per_batch);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

}  // namespace lf
