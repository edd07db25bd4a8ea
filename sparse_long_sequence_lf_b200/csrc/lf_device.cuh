// Shared definitions of the Longformer attention library: workspace layout,
// launch arguments, status codes and small device helpers.
//
// The method: each valid, non-global query i of head h attends to the window
// taps of i (w/2 taps per side spaced by dilation[h], or w taps to the left
// when causal) together with every global token; a valid global query attends
// to every valid token through Qg, Kg, Vg; padded queries output zero.
// ("LongFormer: The Long-Document Transformer" notes, "Sliding Window",
// "Dilated Sliding Window", "Global Attention"; FasterTransformer Longformer
// Encoder guide, "compute flow".)
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace lf {

constexpr int kDHead = 64;          // the only head size (FT guide, "four hard constraints")
constexpr int kMaxHeads = 256;      // heads per call (per-head tables travel as kernel arguments)
constexpr int kChunkKeys = 512;     // keys per partial result of a global row
constexpr int kPartialFloats = 66;  // m (log2 units), l, acc[64]
constexpr int kSlotGroup = 32;      // global rows per arrival counter

enum Status : int {
    kOk = 0,
    kErrInvalidArg = -1,
    kErrUnsupported = -2,
    kErrWorkspace = -3,
    kErrCuda = -4,
    kErrDeviceTimeout = -5,
    kErrGlobalOverflow = -6,
    kErrNoDevice = -7,
};

// Per-batch flag bits written by the mask-preparation kernel.
constexpr int kFlagHasPadding = 1;
constexpr int kFlagOverflow = 2;

// Workspace layout.  Every region starts on a 256-byte boundary.
struct WsLayout {
    int B, H, n, nwords, max_global, nchunks, ngroups;
    size_t off_status, off_flags, off_counts, off_gidx, off_vbits, off_gbits;
    size_t off_counters, off_partials, total;
};

__host__ __device__ inline size_t lf_align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(int B, int H, int n, int max_global)
{
    WsLayout L{};
    L.B = B;
    L.H = H;
    L.n = n;
    L.nwords = (n + 31) / 32;
    L.max_global = max_global;
    L.nchunks = (n + kChunkKeys - 1) / kChunkKeys;
    L.ngroups = (max_global + kSlotGroup - 1) / kSlotGroup;
    size_t off = 0;
    L.off_status = off;   off += 256;
    L.off_flags = off;    off = lf_align256(off + sizeof(int) * size_t(B));
    L.off_counts = off;   off = lf_align256(off + sizeof(int) * size_t(B));
    L.off_gidx = off;     off = lf_align256(off + sizeof(int) * size_t(B) * n);
    L.off_vbits = off;    off = lf_align256(off + sizeof(uint32_t) * size_t(B) * L.nwords);
    L.off_gbits = off;    off = lf_align256(off + sizeof(uint32_t) * size_t(B) * L.nwords);
    L.off_counters = off; off = lf_align256(off + sizeof(int) * size_t(B) * H * (L.ngroups + 1));
    L.off_partials = off;
    off = lf_align256(off + sizeof(float) * size_t(B) * H * L.nchunks * size_t(max_global) *
                                kPartialFloats);
    L.total = off;
    return L;
}

// Typed views of a workspace.
struct WsPtrs {
    int *status;
    int *flags;
    int *counts;
    int *gidx;
    uint32_t *vbits;
    uint32_t *gbits;
    int *counters;
    float *partials;
};

__host__ __device__ inline WsPtrs ws_ptrs(void *ws, const WsLayout &L)
{
    char *base = static_cast<char *>(ws);
    WsPtrs p;
    p.status = reinterpret_cast<int *>(base + L.off_status);
    p.flags = reinterpret_cast<int *>(base + L.off_flags);
    p.counts = reinterpret_cast<int *>(base + L.off_counts);
    p.gidx = reinterpret_cast<int *>(base + L.off_gidx);
    p.vbits = reinterpret_cast<uint32_t *>(base + L.off_vbits);
    p.gbits = reinterpret_cast<uint32_t *>(base + L.off_gbits);
    p.counters = reinterpret_cast<int *>(base + L.off_counters);
    p.partials = reinterpret_cast<float *>(base + L.off_partials);
    return p;
}

// Arguments shared by the attention kernels.
struct AttnArgs {
    const void *q, *k, *v, *qg, *kg, *vg;
    void *out;
    float *lse_out;   // optional [B*H*n]: log-sum-exp (log2 units) of the band rows
    WsPtrs ws;
    WsLayout L;
    int B, H, n;
    int window;      // w
    int half;        // w/2 (non-causal)
    int causal;
    int max_global;
    float scale_log2;   // log2(e) / sqrt(d_head)
    int band_items_per_batch;
    int dil[kMaxHeads];
    int head_prefix[kMaxHeads + 1];   // band items of one batch before head h
};

// ------------------------------------------------------------------ helpers
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x)
{
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x)
{
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ bool bit_at(const uint32_t *bits, int p)
{
    return (bits[p >> 5] >> (p & 31)) & 1u;
}

// Is key j (sequence position) a window tap of query i?
__device__ __forceinline__ bool is_tap(int i, int j, int w, int half, int dil, int causal)
{
    int diff = j - i;
    if (causal) {
        if (diff > 0) return false;
        int back = -diff;
        if (back % dil) return false;
        return back / dil <= w - 1;
    }
    int a = diff < 0 ? -diff : diff;
    if (a % dil) return false;
    return a / dil <= half;
}

// Records the first device-side error of a call.
__device__ __forceinline__ void set_status(int *status, int code)
{
    atomicCAS(status, 0, code);
}

// Maps a band item to (b, h, residue r, tile of 128 rows in residue space).
__device__ __forceinline__ void band_item(const AttnArgs &a, int item, int &b, int &h, int &r,
                                          int &tile)
{
    b = item / a.band_items_per_batch;
    int rem = item - b * a.band_items_per_batch;
    h = 0;
    while (h + 1 < a.H && a.head_prefix[h + 1] <= rem) ++h;
    rem -= a.head_prefix[h];
    int dil = a.dil[h];
    r = 0;
    for (;;) {
        int n_r = (a.n - r + dil - 1) / dil;
        int t = (n_r + 127) / 128;
        if (rem < t || r + 1 >= dil) break;
        rem -= t;
        ++r;
    }
    tile = rem;
}

// Partial results of the global rows, per (bh, chunk): field-major
// [m (log2 units), l, acc[64]] x max_global slots.
__device__ __forceinline__ float *partial_base(const AttnArgs &a, int bh, int chunk)
{
    return a.ws.partials + (size_t(bh) * a.L.nchunks + chunk) * kPartialFloats * size_t(a.max_global);
}

// Merges the chunk partials of one global row and writes its output row;
// lane l of the calling warp handles dimensions 2l and 2l+1.
template <typename T>
__device__ __forceinline__ void combine_row_partials(const AttnArgs &a, int bh, int slot,
                                                     int nchunks_used, int lane, T *orow)
{
    const size_t mg = size_t(a.max_global);
    const float *P = partial_base(a, bh, 0) + slot;
    const size_t cstride = kPartialFloats * mg;
    float M = -INFINITY;
    for (int c = 0; c < nchunks_used; ++c) M = fmaxf(M, P[c * cstride]);
    float Lsum = 0.f, acc0 = 0.f, acc1 = 0.f;
    for (int c = 0; c < nchunks_used; ++c) {
        const float *pc = P + c * cstride;
        const float mc = pc[0];
        const float f = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
        Lsum += f * pc[mg];
        acc0 += f * pc[(2 + 2 * lane) * mg];
        acc1 += f * pc[(3 + 2 * lane) * mg];
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    orow[2 * lane] = from_f32<T>(acc0 * inv);
    orow[2 * lane + 1] = from_f32<T>(acc1 * inv);
}

}  // namespace lf
