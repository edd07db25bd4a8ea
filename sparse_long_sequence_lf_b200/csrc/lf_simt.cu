// CUDA-core kernels of the attention: the fp32 path.
//
// fp32 inputs are computed in fp32 on the FMA pipes end to end (the tensor
// cores' tf32 mode keeps 10 mantissa bits, too few for fp32 parity), with
// one thread per query row:
//
//   band kernel     one CTA per 128 query rows of one (batch, head, residue
//                   class of the dilation); keys stream through shared memory
//                   32 at a time; an online softmax in registers covers the
//                   window taps and then the global-token columns.  Writes
//                   every row except valid global rows (zeros for padding).
//   global kernel   one CTA per (batch*head, chunk of 512 keys, group of 32
//                   global rows); a warp owns 8 global rows, lanes split the
//                   keys for the scores and the head dimension for Vg; writes
//                   fp32 partials (max, sum, acc) and the last CTA of a group
//                   merges the chunks (log-sum-exp) into the output rows.
//
// ("LongFormer: The Long-Document Transformer" notes, "Sliding Window",
// "Dilated Sliding Window", "Global Attention"; FasterTransformer Longformer
// Encoder guide, "compute flow": softmax of local rows over window + global
// tokens, of global rows over the whole sequence, masked rows zeroed.)
#include "lf_device.cuh"

namespace lf {

constexpr int kSimtRows = 128;
constexpr int kSimtKeys = 32;

template <typename T>
__global__ void __launch_bounds__(kSimtRows)
band_simt_kernel(const AttnArgs a)
{
    __shared__ float ks[kSimtKeys][kDHead];
    __shared__ float vs[kSimtKeys][kDHead];
    __shared__ int kpos[kSimtKeys];    // sequence position of each staged key, -1 = not a key

    int b, h, r, tile;
    band_item(a, blockIdx.x, b, h, r, tile);
    const int dil = a.dil[h];
    const int n = a.n;
    const int n_r = (n - r + dil - 1) / dil;
    const int tid = threadIdx.x;
    const int ir = tile * kSimtRows + tid;          // row in residue space
    const bool row_in = ir < n_r;
    const int i = ir * dil + r;                     // sequence position
    const size_t bh = size_t(b) * a.H + h;
    const T *Q = static_cast<const T *>(a.q) + bh * n * kDHead;
    const T *K = static_cast<const T *>(a.k) + bh * n * kDHead;
    const T *V = static_cast<const T *>(a.v) + bh * n * kDHead;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    if (tid == 0 && a.ws.counts[b] > a.max_global) set_status(a.ws.status, kErrGlobalOverflow);

    float q[kDHead], acc[kDHead];
#pragma unroll
    for (int x = 0; x < kDHead; ++x) {
        q[x] = row_in ? to_f32(Q[size_t(i) * kDHead + x]) * a.scale_log2 : 0.f;
        acc[x] = 0.f;
    }
    float m = -INFINITY, l = 0.f;

    // Residue-space key range covered by the rows of this CTA.
    const int r0 = tile * kSimtRows;
    int lo, hi;
    if (a.causal) {
        lo = r0 - (a.window - 1);
        hi = r0 + kSimtRows - 1;
    } else {
        lo = r0 - a.half;
        hi = r0 + kSimtRows - 1 + a.half;
    }
    lo = max(lo, 0);
    hi = min(hi, n_r - 1);

    auto consume = [&](bool band_tile) {
        float s[kSimtKeys];
        float tmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < kSimtKeys; ++c) {
            const int j = kpos[c];
            bool ok = row_in && j >= 0;
            if (ok) {
                if (band_tile) {
                    const int jr = (j - r) / dil;
                    ok = a.causal ? (jr <= ir && ir - jr <= a.window - 1)
                                  : (jr - ir <= a.half && ir - jr <= a.half);
                } else {
                    ok = !is_tap(i, j, a.window, a.half, dil, a.causal);
                }
            }
            float dot = 0.f;
#pragma unroll
            for (int x = 0; x < kDHead; ++x) dot = fmaf(q[x], ks[c][x], dot);
            s[c] = ok ? dot : -INFINITY;
            tmax = fmaxf(tmax, s[c]);
        }
        const float mnew = fmaxf(m, tmax);
        const float base = (mnew == -INFINITY) ? 0.f : mnew;
        const float corr = exp2f(m - base);
        l *= corr;
#pragma unroll
        for (int x = 0; x < kDHead; ++x) acc[x] *= corr;
#pragma unroll
        for (int c = 0; c < kSimtKeys; ++c) {
            const float p = exp2f(s[c] - base);
            l += p;
#pragma unroll
            for (int x = 0; x < kDHead; ++x) acc[x] = fmaf(p, vs[c][x], acc[x]);
        }
        m = mnew;
    };

    // Window taps, 32 residue-space keys at a time.
    for (int k0 = lo; k0 <= hi; k0 += kSimtKeys) {
        __syncthreads();
        for (int e = tid; e < kSimtKeys * kDHead; e += kSimtRows) {
            const int c = e / kDHead, x = e % kDHead;
            const int jr = k0 + c;
            const int j = jr * dil + r;
            const bool in = jr <= hi && j < n;
            ks[c][x] = in ? to_f32(K[size_t(j) * kDHead + x]) : 0.f;
            vs[c][x] = in ? to_f32(V[size_t(j) * kDHead + x]) : 0.f;
            if (x == 0) kpos[c] = (in && bit_at(vb, j)) ? j : -1;
        }
        __syncthreads();
        consume(true);
    }

    // Global-token columns (keys that are not already window taps).
    int g = a.ws.counts[b];
    g = min(g, a.max_global);
    const int *gl = a.ws.gidx + size_t(b) * n;
    for (int s0 = 0; s0 < g; s0 += kSimtKeys) {
        __syncthreads();
        for (int e = tid; e < kSimtKeys * kDHead; e += kSimtRows) {
            const int c = e / kDHead, x = e % kDHead;
            const int slot = s0 + c;
            const int j = slot < g ? gl[slot] : -1;
            ks[c][x] = j >= 0 ? to_f32(K[size_t(j) * kDHead + x]) : 0.f;
            vs[c][x] = j >= 0 ? to_f32(V[size_t(j) * kDHead + x]) : 0.f;
            if (x == 0) kpos[c] = (j >= 0 && bit_at(vb, j)) ? j : -1;
        }
        __syncthreads();
        consume(false);
    }

    if (!row_in) return;
    T *O = static_cast<T *>(a.out) + bh * n * kDHead + size_t(i) * kDHead;
    if (!bit_at(vb, i)) {
#pragma unroll
        for (int x = 0; x < kDHead; ++x) O[x] = from_f32<T>(0.f);
        return;
    }
    if (bit_at(gb, i)) return;     // written by the global-row kernel
    const float inv = 1.f / l;
#pragma unroll
    for (int x = 0; x < kDHead; ++x) O[x] = from_f32<T>(acc[x] * inv);
}

constexpr int kGlobWarps = 4;
constexpr int kGlobSlotsPerWarp = kSlotGroup / kGlobWarps;   // 8
constexpr int kGlobKeys = 64;

template <typename T>
__global__ void __launch_bounds__(kGlobWarps * 32)
global_simt_kernel(const AttnArgs a)
{
    __shared__ float qs[kSlotGroup][kDHead];
    __shared__ float ks[kGlobKeys][kDHead + 1];
    __shared__ float vs[kGlobKeys][kDHead];
    __shared__ int kok[kGlobKeys];
    __shared__ int s_last;

    const int chunk = blockIdx.x;
    const int bh = blockIdx.y;
    const int group = blockIdx.z;
    const int b = bh / a.H;
    const int n = a.n;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int g = min(a.ws.counts[b], a.max_global);
    if (a.ws.counts[b] > a.max_global && tid == 0 && chunk == 0 && group == 0 && (bh % a.H) == 0)
        set_status(a.ws.status, kErrGlobalOverflow);
    const int slot0 = group * kSlotGroup;
    if (slot0 >= g) return;
    const int *gl = a.ws.gidx + size_t(b) * n;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const T *Qg = static_cast<const T *>(a.qg) + size_t(bh) * n * kDHead;
    const T *Kg = static_cast<const T *>(a.kg) + size_t(bh) * n * kDHead;
    const T *Vg = static_cast<const T *>(a.vg) + size_t(bh) * n * kDHead;

    for (int e = tid; e < kSlotGroup * kDHead; e += blockDim.x) {
        const int s = e / kDHead, x = e % kDHead;
        const int slot = slot0 + s;
        qs[s][x] = slot < g ? to_f32(Qg[size_t(gl[slot]) * kDHead + x]) * a.scale_log2 : 0.f;
    }

    float m[kGlobSlotsPerWarp], l[kGlobSlotsPerWarp], acc0[kGlobSlotsPerWarp],
        acc1[kGlobSlotsPerWarp];
#pragma unroll
    for (int t = 0; t < kGlobSlotsPerWarp; ++t) {
        m[t] = -INFINITY;
        l[t] = 0.f;
        acc0[t] = 0.f;
        acc1[t] = 0.f;
    }

    const int key_begin = chunk * kChunkKeys;
    const int key_end = min(n, key_begin + kChunkKeys);
    for (int k0 = key_begin; k0 < key_end; k0 += kGlobKeys) {
        __syncthreads();
        for (int e = tid; e < kGlobKeys * kDHead; e += blockDim.x) {
            const int c = e / kDHead, x = e % kDHead;
            const int j = k0 + c;
            const bool in = j < key_end;
            ks[c][x] = in ? to_f32(Kg[size_t(j) * kDHead + x]) : 0.f;
            vs[c][x] = in ? to_f32(Vg[size_t(j) * kDHead + x]) : 0.f;
            if (x == 0) kok[c] = in && bit_at(vb, j);
        }
        __syncthreads();
#pragma unroll
        for (int t = 0; t < kGlobSlotsPerWarp; ++t) {
            const int s = warp * kGlobSlotsPerWarp + t;
            if (slot0 + s >= g) break;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll 16
            for (int x = 0; x < kDHead; ++x) {
                s0 = fmaf(qs[s][x], ks[lane][x], s0);
                s1 = fmaf(qs[s][x], ks[lane + 32][x], s1);
            }
            s0 = kok[lane] ? s0 : -INFINITY;
            s1 = kok[lane + 32] ? s1 : -INFINITY;
            float tmax = fmaxf(s0, s1);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
            const float mnew = fmaxf(m[t], tmax);
            const float base = (mnew == -INFINITY) ? 0.f : mnew;
            const float corr = exp2f(m[t] - base);
            const float p0 = exp2f(s0 - base), p1 = exp2f(s1 - base);
            float psum = p0 + p1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
            l[t] = l[t] * corr + psum;
            float a0 = acc0[t] * corr, a1 = acc1[t] * corr;
#pragma unroll 8
            for (int c = 0; c < 32; ++c) {
                const float pa = __shfl_sync(0xffffffffu, p0, c);
                const float pb = __shfl_sync(0xffffffffu, p1, c);
                a0 = fmaf(pa, vs[c][2 * lane], a0);
                a1 = fmaf(pa, vs[c][2 * lane + 1], a1);
                a0 = fmaf(pb, vs[c + 32][2 * lane], a0);
                a1 = fmaf(pb, vs[c + 32][2 * lane + 1], a1);
            }
            acc0[t] = a0;
            acc1[t] = a1;
            m[t] = mnew;
        }
    }

    // Partials of this chunk.
#pragma unroll
    for (int t = 0; t < kGlobSlotsPerWarp; ++t) {
        const int slot = slot0 + warp * kGlobSlotsPerWarp + t;
        if (slot >= g) break;
        float *P = partial_base(a, bh, chunk) + slot;
        const size_t mg = size_t(a.max_global);
        if (lane == 0) {
            P[0] = m[t];
            P[mg] = l[t];
        }
        P[(2 + 2 * lane) * mg] = acc0[t];
        P[(3 + 2 * lane) * mg] = acc1[t];
    }

    // The last CTA of this (bh, group) to finish merges every chunk.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        int *ctr = a.ws.counters + size_t(bh) * (a.L.ngroups + 1) + group;
        const int prev = atomicAdd(ctr, 1);
        s_last = (prev == int(gridDim.x) - 1);
        if (s_last) *ctr = 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    T *Out = static_cast<T *>(a.out) + size_t(bh) * n * kDHead;
    for (int s = warp; s < kSlotGroup; s += kGlobWarps) {
        const int slot = slot0 + s;
        if (slot >= g) break;
        const int p = gl[slot];
        if (!bit_at(vb, p)) continue;   // padded global position: the band kernel wrote zeros
        combine_row_partials<T>(a, bh, slot, gridDim.x, lane, Out + size_t(p) * kDHead);
    }
}

template <typename T>
int launch_simt(const AttnArgs &a, cudaStream_t stream)
{
    const int band_items = a.B * a.band_items_per_batch;
    if (band_items > 0) band_simt_kernel<T><<<band_items, kSimtRows, 0, stream>>>(a);
    if (a.max_global > 0) {
        dim3 grid(a.L.nchunks, a.B * a.H, a.L.ngroups);
        global_simt_kernel<T><<<grid, kGlobWarps * 32, 0, stream>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

template int launch_simt<float>(const AttnArgs &, cudaStream_t);
template int launch_simt<__half>(const AttnArgs &, cudaStream_t);
template int launch_simt<__nv_bfloat16>(const AttnArgs &, cudaStream_t);

}  // namespace lf
