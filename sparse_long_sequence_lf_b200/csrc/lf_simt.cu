// CUDA-core kernels of the attention: the fp32 path.
//
// fp32 inputs are computed in fp32 on the FMA pipes end to end (the tensor
// cores' tf32 mode keeps 10 mantissa bits, too few for fp32 parity):
//
//   band kernel     one CTA per 32 query rows of one (batch, head, residue
//                   class of the dilation), four threads per row; keys stream
//                   through shared memory 32 at a time; an online softmax
//                   covers the window taps and then the global-token columns.
//                   Writes every row except valid global rows (zeros for
//                   padding).
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
#include "lf_vec.cuh"

namespace lf {

constexpr int kSimtRows = 32;                     // query rows per band CTA
constexpr int kSimtThreads = 4 * kSimtRows;       // four threads per row
constexpr int kSimtParts = 128 / kSimtRows;       // band CTAs per 128-row band item
constexpr int kSimtKeys = 32;

// One staged tile of 32 keys: each thread holds 4 of the 512 four-element
// pieces of K and of V (key c = tid/16 + 8u, dims 4*(tid%16) .. +3), loaded
// into registers while the previous tile is being consumed.
struct KvStage {
    float4 k[4], v[4];
    int pos[4];
};

// One CTA per 32 query rows (a quarter of a 128-row band item); four threads
// per row, each holding a quarter of the head dimension of q and of the
// accumulator.  Scores are reduced over the four threads with two shuffles.
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
band_simt_kernel(const AttnArgs a)
{
    __shared__ __align__(16) float ks[kSimtKeys][kDHead];
    __shared__ __align__(16) float vs[kSimtKeys][kDHead];
    __shared__ float ss[kSimtKeys][kSimtRows];   // scores, column = row of this CTA
    __shared__ int kpos[kSimtKeys];    // sequence position of each staged key, -1 = not a key

    int b, h, r, tile;
    band_item(a, blockIdx.x / kSimtParts, b, h, r, tile);
    const int dil = a.dil[h];
    const int n = a.n;
    const int n_r = (n - r + dil - 1) / dil;
    const int tid = threadIdx.x;
    const int rl = tid >> 2;                        // row of this CTA
    const int qd = tid & 3;                         // quarter of the head dimension
    const int r0 = tile * 128 + (blockIdx.x % kSimtParts) * kSimtRows;   // first residue-space row
    const int ir = r0 + rl;                         // row in residue space
    const bool row_in = ir < n_r;
    const int i = ir * dil + r;                     // sequence position
    const size_t bh = size_t(b) * a.H + h;
    const T *Q = static_cast<const T *>(a.q) + bh * n * kDHead;
    const T *K = static_cast<const T *>(a.k) + bh * n * kDHead;
    const T *V = static_cast<const T *>(a.v) + bh * n * kDHead;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    if (tid == 0 && blockIdx.x % kSimtParts == 0 && a.ws.counts[b] > a.max_global)
        set_status(a.ws.status, kErrGlobalOverflow);
    if (r0 >= n_r) return;                          // no rows in this quarter

    constexpr int kQ = kDHead / 4;                  // 16 dimensions per thread
    float q[kQ], acc[kQ];
#pragma unroll
    for (int x = 0; x < kQ; x += 4) {
        const float4 t = row_in ? load4(Q + size_t(i) * kDHead + kQ * qd + x)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        q[x] = t.x * a.scale_log2;
        q[x + 1] = t.y * a.scale_log2;
        q[x + 2] = t.z * a.scale_log2;
        q[x + 3] = t.w * a.scale_log2;
        acc[x] = acc[x + 1] = acc[x + 2] = acc[x + 3] = 0.f;
    }
    float m = -INFINITY, l = 0.f;

    // Residue-space key range covered by the rows of this CTA.
    const int rows_hi = min(r0 + kSimtRows - 1, n_r - 1);
    int lo, hi;
    if (a.causal) {
        lo = r0 - (a.window - 1);
        hi = rows_hi;
    } else {
        lo = r0 - a.half;
        hi = rows_hi + a.half;
    }
    lo = max(lo, 0);
    hi = min(hi, n_r - 1);

    // Pass 1 puts the scores of the staged keys in shared memory, pass 2
    // takes the exponentials and accumulates P V.
    auto consume = [&](int k0, bool band_tile) {
        float tmax = -INFINITY;
#pragma unroll 2
        for (int c = 0; c < kSimtKeys; ++c) {
            float d0 = 0.f, d1 = 0.f;
#pragma unroll
            for (int x = 0; x < kQ; x += 4) {
                const float4 kv = *reinterpret_cast<const float4 *>(&ks[c][kQ * qd + x]);
                d0 = fmaf(q[x], kv.x, d0);
                d1 = fmaf(q[x + 1], kv.y, d1);
                d0 = fmaf(q[x + 2], kv.z, d0);
                d1 = fmaf(q[x + 3], kv.w, d1);
            }
            float dot = d0 + d1;
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            const int j = kpos[c];
            bool ok = row_in && j >= 0;
            if (ok) {
                if (band_tile) {
                    const int jr = k0 + c;
                    ok = a.causal ? (jr <= ir && ir - jr <= a.window - 1)
                                  : (jr - ir <= a.half && ir - jr <= a.half);
                } else {
                    ok = !is_tap(i, j, a.window, a.half, dil, a.causal);
                }
            }
            const float sc = ok ? dot : -INFINITY;
            if (qd == 0) ss[c][rl] = sc;
            tmax = fmaxf(tmax, sc);
        }
        __syncwarp();
        const float mnew = fmaxf(m, tmax);
        const float base = (mnew == -INFINITY) ? 0.f : mnew;
        const float corr = exp2f(m - base);
        l *= corr;
#pragma unroll
        for (int x = 0; x < kQ; ++x) acc[x] *= corr;
#pragma unroll 2
        for (int c = 0; c < kSimtKeys; ++c) {
            const float p = exp2f(ss[c][rl] - base);
            l += p;
#pragma unroll
            for (int x = 0; x < kQ; x += 4) {
                const float4 vv = *reinterpret_cast<const float4 *>(&vs[c][kQ * qd + x]);
                acc[x] = fmaf(p, vv.x, acc[x]);
                acc[x + 1] = fmaf(p, vv.y, acc[x + 1]);
                acc[x + 2] = fmaf(p, vv.z, acc[x + 2]);
                acc[x + 3] = fmaf(p, vv.w, acc[x + 3]);
            }
        }
        __syncwarp();
        m = mnew;
    };

    // Key tiles: the window taps, 32 residue-space keys at a time, then the
    // global-token columns (keys that are not already window taps), 32 slots
    // at a time.  The next tile's loads are in flight during each consume.
    int g = a.ws.counts[b];
    g = min(g, a.max_global);
    const int *gl = a.ws.gidx + size_t(b) * n;
    const int nband = hi >= lo ? (hi - lo) / kSimtKeys + 1 : 0;
    const int ntiles = nband + (g + kSimtKeys - 1) / kSimtKeys;
    const int x4 = 4 * (tid & 15);
    auto fetch = [&](int t, KvStage &st) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = (tid >> 4) + 8 * u;
            int j;
            if (t < nband) {
                const int jr = lo + kSimtKeys * t + c;
                j = (jr <= hi && jr * dil + r < n) ? jr * dil + r : -1;
            } else {
                const int slot = kSimtKeys * (t - nband) + c;
                j = slot < g ? gl[slot] : -1;
            }
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            st.k[u] = j >= 0 ? load4(K + size_t(j) * kDHead + x4) : z;
            st.v[u] = j >= 0 ? load4(V + size_t(j) * kDHead + x4) : z;
            st.pos[u] = (j >= 0 && bit_at(vb, j)) ? j : -1;
        }
    };
    KvStage st;
    if (ntiles > 0) fetch(0, st);
    for (int t = 0; t < ntiles; ++t) {
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = (tid >> 4) + 8 * u;
            *reinterpret_cast<float4 *>(&ks[c][x4]) = st.k[u];
            *reinterpret_cast<float4 *>(&vs[c][x4]) = st.v[u];
            if (x4 == 0) kpos[c] = st.pos[u];
        }
        __syncthreads();
        if (t + 1 < ntiles) fetch(t + 1, st);
        consume(lo + kSimtKeys * t, t < nband);
    }

    if (!row_in) return;
    T *O = static_cast<T *>(a.out) + bh * n * kDHead + size_t(i) * kDHead + kQ * qd;
    if (!bit_at(vb, i)) {
#pragma unroll
        for (int x = 0; x < kQ; x += 4) store4(O + x, make_float4(0.f, 0.f, 0.f, 0.f));
        return;
    }
    if (bit_at(gb, i)) return;     // written by the global-row kernel
    const float inv = 1.f / l;
#pragma unroll
    for (int x = 0; x < kQ; x += 4)
        store4(O + x, make_float4(acc[x] * inv, acc[x + 1] * inv, acc[x + 2] * inv, acc[x + 3] * inv));
}

constexpr int kGlobWarps = 4;
constexpr int kGlobSlotsPerWarp = kSlotGroup / kGlobWarps;   // 8
constexpr int kGlobKeys = 64;

template <typename T>
__global__ void __launch_bounds__(kGlobWarps * 32)
global_simt_kernel(const AttnArgs a)
{
    __shared__ __align__(16) float qs[kSlotGroup][kDHead];
    __shared__ float ks[kGlobKeys][kDHead + 1];
    __shared__ __align__(16) float vs[kGlobKeys][kDHead];
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

    const int x4 = 4 * (tid & 15);
#pragma unroll
    for (int u = 0; u < kSlotGroup / 8; ++u) {
        const int s = (tid >> 4) + 8 * u;
        const int slot = slot0 + s;
        const float4 t = slot < g ? load4(Qg + size_t(gl[slot]) * kDHead + x4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(&qs[s][x4]) =
            make_float4(t.x * a.scale_log2, t.y * a.scale_log2, t.z * a.scale_log2,
                        t.w * a.scale_log2);
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

    // Key tiles of 64: each thread holds 8 of the 1024 four-element pieces of
    // Kg and of Vg (key c = tid/16 + 8u), loaded while the previous tile is
    // being consumed.
    const int key_begin = chunk * kChunkKeys;
    const int key_end = min(n, key_begin + kChunkKeys);
    constexpr int kPieces = kGlobKeys / 8;
    float4 kr[kPieces], vr[kPieces];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int u = 0; u < kPieces; ++u) {
            const int j = k0 + (tid >> 4) + 8 * u;
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            kr[u] = j < key_end ? load4(Kg + size_t(j) * kDHead + x4) : z;
            vr[u] = j < key_end ? load4(Vg + size_t(j) * kDHead + x4) : z;
        }
    };
    fetch(key_begin);
    for (int k0 = key_begin; k0 < key_end; k0 += kGlobKeys) {
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kPieces; ++u) {
            const int c = (tid >> 4) + 8 * u;
            ks[c][x4] = kr[u].x;
            ks[c][x4 + 1] = kr[u].y;
            ks[c][x4 + 2] = kr[u].z;
            ks[c][x4 + 3] = kr[u].w;
            *reinterpret_cast<float4 *>(&vs[c][x4]) = vr[u];
        }
        if (tid < kGlobKeys) kok[tid] = k0 + tid < key_end && bit_at(vb, k0 + tid);
        __syncthreads();
        if (k0 + kGlobKeys < key_end) fetch(k0 + kGlobKeys);
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
    if (band_items > 0) band_simt_kernel<T><<<band_items * kSimtParts, kSimtThreads, 0, stream>>>(a);
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
