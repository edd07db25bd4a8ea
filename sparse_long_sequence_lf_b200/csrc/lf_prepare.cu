// Mask preparation: global-index compaction and per-batch bitmaps.
//
// The FasterTransformer Longformer Encoder guide ("compute flow") extracts,
// once before the layer loop, the positions of the global tokens of each batch
// and their count from the global mask, and turns the local mask into an
// additive -10000 bias.  Here one CTA per batch does a stable ascending
// compaction in a single pass: every thread owns a run of whole 32-position
// words, loads all of its mask bytes at once, counts its global tokens, and one
// block-wide exclusive scan gives each thread its output offset.  The local
// mask becomes a bitmap of valid keys (exclusion, not a bias).  The same pass
// builds a bitmap of global tokens, a has-padding flag, and clears the arrival
// counters of the global-row combine.
#include <algorithm>

#include "lf_device.cuh"

namespace lf {

constexpr int kPrepThreads = 1024;
constexpr int kPrepWarps = kPrepThreads / 32;
constexpr int kPrepMaxWordsPerThread = 8;    // n up to 1024 * 8 * 32 = 262144 in one pass

// Bit i of the result is set when byte p0 + i of the mask is nonzero (bits past
// n are 0).  A NULL mask reads as all default_value.
__device__ __forceinline__ uint32_t word_bits(const uint8_t *m, int p0, int n, bool present,
                                              bool default_value)
{
    const int left = n - p0;
    const uint32_t inrange = left >= 32 ? 0xffffffffu : (left <= 0 ? 0u : ((1u << left) - 1u));
    if (!present) return default_value ? inrange : 0u;
    uint32_t w = 0;
    if (left >= 32 && (reinterpret_cast<uintptr_t>(m + p0) & 15u) == 0) {
        const uint4 *v = reinterpret_cast<const uint4 *>(m + p0);
        const uint4 a = __ldcg(v), b = __ldcg(v + 1);
        const uint32_t x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if ((x[q] >> (8 * k)) & 0xffu) w |= 1u << (4 * q + k);
        return w;
    }
    for (int i = 0; i < 32 && i < left; ++i)
        if (__ldcg(m + p0 + i) != 0) w |= 1u << i;
    return w;
}

// One CTA per batch.  Any output pointer may be NULL (not written).  The
// entries of gidx past the count are set to -1 only with fill_tail (the
// attention kernels read the first count entries alone).
__global__ void __launch_bounds__(kPrepThreads)
prepare_kernel(const uint8_t *__restrict__ local_mask, const uint8_t *__restrict__ global_mask,
               int B, int n, int max_global, int32_t *gidx, int32_t *counts, int *flags,
               uint32_t *vbits, uint32_t *gbits, int *status, int *counters, int counters_per_batch,
               int fill_tail)
{
    // The attention kernel may start its prologue now; it waits for this
    // grid's results before reading them.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    __shared__ int warp_sum[kPrepWarps];

    const int b = blockIdx.x;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const uint8_t *lm = local_mask ? local_mask + size_t(b) * n : nullptr;
    const uint8_t *gm = global_mask ? global_mask + size_t(b) * n : nullptr;
    const int nwords = (n + 31) / 32;
    const int nthreads = int(blockDim.x);                       // a multiple of 32
    const int wpt = (nwords + nthreads - 1) / nthreads;         // words per thread (<= 8)
    const int w0 = tid * wpt;

    // Launched in stream order (see launch_prepare), so the kernel ahead has
    // completed and its writes are visible; the wait below is then a no-op,
    // kept so that a programmatic launch would stay correct.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t gw[kPrepMaxWordsPerThread], vw[kPrepMaxWordsPerThread];
    int mine = 0, pad = 0;
#pragma unroll
    for (int k = 0; k < kPrepMaxWordsPerThread; ++k) {
        gw[k] = 0u;
        vw[k] = 0u;
        const int w = w0 + k;
        if (k < wpt && w < nwords) {
            gw[k] = word_bits(gm, 32 * w, n, gm != nullptr, false);
            vw[k] = word_bits(lm, 32 * w, n, lm != nullptr, true);
            mine += __popc(gw[k]);
            const int left = n - 32 * w;
            const uint32_t inrange = left >= 32 ? 0xffffffffu : ((1u << left) - 1u);
            pad |= (vw[k] != inrange);
        }
    }
    // Block-wide exclusive scan of the per-thread global counts.
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sum[warp] = incl;
    const int any_pad = __syncthreads_or(pad);
    int before = 0, total = 0;
    for (int w = 0; w < (nthreads >> 5); ++w) {
        const int t = warp_sum[w];
        before += (w < warp) ? t : 0;
        total += t;
    }
    int off = before + incl - mine;

    // The status word, and the attention kernel's item counter and finished
    // count (words 16 and 32 of the status region), start at zero.
    if (tid == 0 && b == 0 && status) {
        status[0] = 0;
        status[16] = 0;
        status[32] = 0;
    }
    if (counters)
        for (int c = tid; c < counters_per_batch; c += nthreads)
            counters[size_t(b) * counters_per_batch + c] = 0;
#pragma unroll
    for (int k = 0; k < kPrepMaxWordsPerThread; ++k) {
        const int w = w0 + k;
        if (k < wpt && w < nwords) {
            if (vbits) vbits[size_t(b) * nwords + w] = vw[k];
            if (gbits) gbits[size_t(b) * nwords + w] = gw[k];
        }
    }
    if (gidx) {
#pragma unroll
        for (int k = 0; k < kPrepMaxWordsPerThread; ++k) {
            uint32_t g = gw[k];
            while (g) {
                const int i = __ffs(g) - 1;
                g &= g - 1u;
                gidx[size_t(b) * n + off++] = 32 * (w0 + k) + i;
            }
        }
        if (fill_tail)
            for (int p = total + tid; p < n; p += nthreads) gidx[size_t(b) * n + p] = -1;
    }
    if (tid == 0) {
        if (counts) counts[b] = total;
        if (flags)
            flags[b] = (any_pad ? kFlagHasPadding : 0) | (total > max_global ? kFlagOverflow : 0);
    }
}

int launch_prepare(const uint8_t *local_mask, const uint8_t *global_mask, int B, int n,
                   int max_global, int32_t *gidx, int32_t *counts, int *flags, uint32_t *vbits,
                   uint32_t *gbits, int *status, int *counters, int counters_per_batch,
                   int fill_tail, cudaStream_t stream)
{
    if ((n + 31) / 32 > kPrepThreads * kPrepMaxWordsPerThread) return kErrUnsupported;
    // An ordinary launch: this kernel starts after the kernel ahead in the
    // stream has completed, so the masks (which that kernel may have written)
    // are read at once.  (Launched with programmatic serialization, it would
    // have to wait before reading them, and measured slower: 45.3 against
    // 43.5 us per step at n4096.)  The attention kernel after it is a
    // programmatic dependent of this one.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(B);
    // One word of each mask per thread while that fits a block: the scan
    // then spans as few warps as the masks need.
    const int nwords = (n + 31) / 32;
    cfg.blockDim = dim3(unsigned(std::min(kPrepThreads, std::max(32, (nwords + 31) / 32 * 32))));
    cfg.stream = stream;
    if (cudaLaunchKernelEx(&cfg, prepare_kernel, local_mask, global_mask, B, n, max_global, gidx,
                           counts, flags, vbits, gbits, status, counters, counters_per_batch,
                           fill_tail) != cudaSuccess)
        return kErrCuda;
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

}  // namespace lf
