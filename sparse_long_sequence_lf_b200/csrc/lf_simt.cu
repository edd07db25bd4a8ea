// CUDA-core attention for fp32 inputs.
//
// fp32 inputs are computed in fp32 on the FMA pipes end to end (the tensor
// cores' tf32 mode keeps 10 mantissa bits, too few for fp32 parity).  One
// launch holds two kinds of CTAs, 256 threads (eight warps) each, so that
// every SM sub-partition has two warps to switch between:
//
//   global CTAs   (batch*head, 512-key chunk, group of 32 global rows): each
//                 of the eight warps takes an eighth of the chunk's keys for
//                 every row of the group (lane = key for the scores, lane =
//                 two head dimensions for Vg), the eight parts are merged in
//                 shared memory into the chunk's fp32 partials (max, sum,
//                 unnormalised output), and the last CTA of a group merges
//                 the chunks by log-sum-exp into the output rows.
//   band CTAs     8 query rows of one (batch, head, residue class of the
//                 dilation), one warp per row; each lane takes 2 of the 64
//                 keys of a staged tile with the full 64-wide dot product
//                 (no reduction per score), the row's lanes share the running
//                 maximum, and their partial sums and outputs are added up
//                 once at the end.  Keys stream through shared memory in
//                 64-key tiles (cp.async, three stages): the window taps,
//                 then the global-token columns that are not taps.  Writes
//                 every row except valid global rows (zeros for padding).
//
// Before waiting for the kernel ahead in the stream, each CTA asks L2 for the
// key and value rows it will read (their addresses follow from the kernel
// arguments alone).
// Shared-memory rows of K/V are 68 floats apart, so 16-byte reads of
// different rows at the same column fall in distinct banks.  The launch is
// chained to the mask-preparation kernel by programmatic dependent launch.
//
// ("LongFormer: The Long-Document Transformer" notes, "Sliding Window",
// "Dilated Sliding Window", "Global Attention"; FasterTransformer Longformer
// Encoder guide, "compute flow": softmax of local rows over window + global
// tokens, of global rows over the whole sequence, masked rows zeroed.)
#include "lf_device.cuh"

namespace lf {

constexpr int kF32Threads = 256;
constexpr int kBandRows = 8;                      // query rows per band CTA
constexpr int kTpr = 32;                          // threads per row (one warp)
constexpr int kBandParts = 128 / kBandRows;       // band CTAs per 128-row band item
constexpr int kTileKeysF = 64;                    // keys per staged band tile
constexpr int kKpt = kTileKeysF / kTpr;           // keys per thread and tile
constexpr int kStride = 68;                       // floats between staged rows
constexpr int kBandStages = 3;
constexpr int kGWarps = kF32Threads / 32;
constexpr int kGKeys = 32;                        // keys per warp tile (lane = key)
constexpr int kGQuarter = kChunkKeys / kGWarps;   // 64 keys of a chunk per warp
constexpr float kRescaleF = 8.f;                  // lazy rescale (log2 units)

struct BandSmem {
    float k[kBandStages][kTileKeysF][kStride];
    float v[kBandStages][kTileKeysF][kStride];
    int pos[kBandStages][kTileKeysF];             // sequence position, -1 = not a key
};

struct GlobSmem {
    float q[kSlotGroup][kDHead];                  // Qg rows, scaled by log2(e)/sqrt(d)
    float k[kGWarps][kGKeys][kStride];
    float v[kGWarps][kGKeys][kDHead];
    int ok[kGWarps][kGKeys];
    float st[kGWarps][kSlotGroup][kPartialFloats];   // per warp and row: m, l, acc[64]
};

constexpr size_t kF32Smem = sizeof(BandSmem) > sizeof(GlobSmem) ? sizeof(BandSmem)
                                                                 : sizeof(GlobSmem);

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid)
{
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    const int n = valid ? 16 : 0;                  // 0: the 16 bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float dot64(const float (&q)[kDHead], const float *krow)
{
    float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
    for (int x = 0; x < kDHead; x += 4) {
        const float4 k4 = *reinterpret_cast<const float4 *>(krow + x);
        d0 = fmaf(q[x], k4.x, d0);
        d1 = fmaf(q[x + 1], k4.y, d1);
        d2 = fmaf(q[x + 2], k4.z, d2);
        d3 = fmaf(q[x + 3], k4.w, d3);
    }
    return (d0 + d1) + (d2 + d3);
}

// ------------------------------------------------------------------ band
__device__ __forceinline__ void band_cta(const AttnArgs &a, int cta, uint8_t *smem_raw)
{
    BandSmem &sm = *reinterpret_cast<BandSmem *>(smem_raw);
    int b, h, r, tile;
    band_item(a, cta / kBandParts, b, h, r, tile);
    const int dil = a.dil[h];
    const int n = a.n;
    const int n_r = (n - r + dil - 1) / dil;
    const int r0 = tile * 128 + (cta % kBandParts) * kBandRows;     // first residue-space row
    if (r0 >= n_r) return;
    const int tid = threadIdx.x;
    const int rl = tid / kTpr, tl = tid % kTpr;
    const int ir = r0 + rl;
    const bool row_in = ir < n_r;
    const int i = ir * dil + r;
    const size_t bh = size_t(b) * a.H + h;
    const float *Q = static_cast<const float *>(a.q) + bh * n * kDHead;
    const float *K = static_cast<const float *>(a.k) + bh * n * kDHead;
    const float *V = static_cast<const float *>(a.v) + bh * n * kDHead;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    const int g = min(a.ws.counts[b], a.max_global);
    const int *gl = a.ws.gidx + size_t(b) * n;

    const int rows_hi = min(r0 + kBandRows - 1, n_r - 1);
    const int lo = max(a.causal ? r0 - (a.window - 1) : r0 - a.half, 0);
    const int hi = min(a.causal ? rows_hi : rows_hi + a.half, n_r - 1);
    const int nband = (hi - lo) / kTileKeysF + 1;
    const int ntiles = nband + (g + kTileKeysF - 1) / kTileKeysF;

    // Loads tile t into its stage.  Sixteen consecutive threads copy one
    // 256-byte row (16 bytes each), so a warp's copy covers two whole rows;
    // thread tid takes rows tid/16 + 16u, u < 4.
    auto issue = [&](int t) {
        if (t < ntiles) {
            const int st = t % kBandStages;
            const int part = (tid & 15) * 4;
#pragma unroll
            for (int u = 0; u < kTileKeysF / 16; ++u) {
                const int c = (tid >> 4) + 16 * u;
                int j;
                if (t < nband) {
                    const int jr = lo + kTileKeysF * t + c;
                    j = jr <= hi ? jr * dil + r : -1;
                } else {
                    const int slot = kTileKeysF * (t - nband) + c;
                    j = slot < g ? gl[slot] : -1;
                }
                const size_t row = size_t(j < 0 ? 0 : j) * kDHead + part;
                cp_async16(&sm.k[st][c][part], K + row, j >= 0);
                cp_async16(&sm.v[st][c][part], V + row, j >= 0);
                if (part == 0) sm.pos[st][c] = (j >= 0 && bit_at(vb, j)) ? j : -1;
            }
        }
        cp_async_commit();
    };
    for (int t = 0; t < kBandStages - 1; ++t) issue(t);

    float q[kDHead], acc[kDHead];
#pragma unroll
    for (int x = 0; x < kDHead; x += 4) {
        const float4 t4 = row_in ? __ldg(reinterpret_cast<const float4 *>(Q + size_t(i) * kDHead + x))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        q[x] = t4.x * a.scale_log2;
        q[x + 1] = t4.y * a.scale_log2;
        q[x + 2] = t4.z * a.scale_log2;
        q[x + 3] = t4.w * a.scale_log2;
        acc[x] = acc[x + 1] = acc[x + 2] = acc[x + 3] = 0.f;
    }
    float m = -INFINITY, l = 0.f;

    for (int t = 0; t < ntiles; ++t) {
        issue(t + kBandStages - 1);
        cp_async_wait<kBandStages - 1>();
        __syncthreads();
        const int st = t % kBandStages;
        const bool band_tile = t < nband;
        float s[kKpt];
        float tmax = -INFINITY;
#pragma unroll
        for (int u = 0; u < kKpt; ++u) {
            const int c = tl + kTpr * u;
            const int j = sm.pos[st][c];
            bool ok = row_in && j >= 0;
            if (ok) {
                if (band_tile) {
                    const int jr = lo + kTileKeysF * t + c;
                    ok = a.causal ? (jr <= ir && ir - jr <= a.window - 1)
                                  : (jr - ir <= a.half && ir - jr <= a.half);
                } else {
                    ok = !is_tap(i, j, a.window, a.half, dil, a.causal);
                }
            }
            s[u] = ok ? dot64(q, &sm.k[st][c][0]) : -INFINITY;
            tmax = fmaxf(tmax, s[u]);
        }
#pragma unroll
        for (int o = 1; o < kTpr; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        if (tmax > m + kRescaleF || (m == -INFINITY && tmax != -INFINITY)) {
            const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - tmax);
            m = tmax;
            l *= alpha;
#pragma unroll
            for (int x = 0; x < kDHead; ++x) acc[x] *= alpha;
        }
        const float base = (m == -INFINITY) ? 0.f : m;
#pragma unroll
        for (int u = 0; u < kKpt; ++u) {
            const float p = exp2f(s[u] - base);
            l += p;
            const float *vrow = &sm.v[st][tl + kTpr * u][0];
#pragma unroll
            for (int x = 0; x < kDHead; x += 4) {
                const float4 v4 = *reinterpret_cast<const float4 *>(vrow + x);
                acc[x] = fmaf(p, v4.x, acc[x]);
                acc[x + 1] = fmaf(p, v4.y, acc[x + 1]);
                acc[x + 2] = fmaf(p, v4.z, acc[x + 2]);
                acc[x + 3] = fmaf(p, v4.w, acc[x + 3]);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    // Sum over the row's 32 threads: l by shuffles, acc through shared memory
    // (the K and V staging areas, contiguous, are free now); thread tl then
    // owns dims 2tl and 2tl+1.
#pragma unroll
    for (int o = 1; o < kTpr; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    __syncthreads();
    static_assert(sizeof(float) * kBandRows * kTpr * (kDHead + 4) <=
                      sizeof(BandSmem::k) + sizeof(BandSmem::v),
                  "row-sum buffer exceeds the staging area");
    float *red = &sm.k[0][0][0];                  // [kBandRows][kTpr][kDHead + 4]
    float *mine = red + (rl * kTpr + tl) * (kDHead + 4);
#pragma unroll
    for (int x = 0; x < kDHead; x += 4)
        *reinterpret_cast<float4 *>(mine + x) = make_float4(acc[x], acc[x + 1], acc[x + 2], acc[x + 3]);
    __syncthreads();
    float2 o2 = make_float2(0.f, 0.f);
#pragma unroll 8
    for (int w = 0; w < kTpr; ++w) {
        const float2 p2 = *reinterpret_cast<const float2 *>(red + (rl * kTpr + w) * (kDHead + 4) + 2 * tl);
        o2.x += p2.x;
        o2.y += p2.y;
    }
    if (!row_in) return;
    float *O = static_cast<float *>(a.out) + bh * n * kDHead + size_t(i) * kDHead + 2 * tl;
    if (!bit_at(vb, i)) {
        *reinterpret_cast<float2 *>(O) = make_float2(0.f, 0.f);
        return;
    }
    if (bit_at(gb, i)) return;     // written by the global rows
    const float inv = 1.f / l;
    *reinterpret_cast<float2 *>(O) = make_float2(o2.x * inv, o2.y * inv);
}

// ---------------------------------------------------------------- global
__device__ __forceinline__ void global_cta(const AttnArgs &a, int cta, uint8_t *smem_raw)
{
    GlobSmem &sm = *reinterpret_cast<GlobSmem *>(smem_raw);
    __shared__ int s_last;
    const int nch = a.L.nchunks;
    const int per_bh = nch * a.L.ngroups;
    const int bh = cta / per_bh;
    const int rem = cta - bh * per_bh;
    const int group = rem / nch;
    const int chunk = rem - group * nch;
    const int b = bh / a.H;
    const int n = a.n;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = min(a.ws.counts[b], a.max_global);
    const int slot0 = group * kSlotGroup;
    if (slot0 >= g) return;
    const int rows = min(kSlotGroup, g - slot0);
    const int *gl = a.ws.gidx + size_t(b) * n;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const float *Qg = static_cast<const float *>(a.qg) + size_t(bh) * n * kDHead;
    const float *Kg = static_cast<const float *>(a.kg) + size_t(bh) * n * kDHead;
    const float *Vg = static_cast<const float *>(a.vg) + size_t(bh) * n * kDHead;

    for (int e = tid; e < kSlotGroup * (kDHead / 4); e += kF32Threads) {
        const int s = e / (kDHead / 4), x = 4 * (e % (kDHead / 4));
        float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s < rows) t4 = __ldg(reinterpret_cast<const float4 *>(Qg + size_t(gl[slot0 + s]) * kDHead + x));
        *reinterpret_cast<float4 *>(&sm.q[s][x]) =
            make_float4(t4.x * a.scale_log2, t4.y * a.scale_log2, t4.z * a.scale_log2,
                        t4.w * a.scale_log2);
    }
    // Per-warp running state of every row: m, l, and lane's two dimensions.
    float *stw = &sm.st[warp][0][0];
    for (int s = lane; s < kSlotGroup; s += 32) {
        stw[s * kPartialFloats] = -INFINITY;
        stw[s * kPartialFloats + 1] = 0.f;
    }
    for (int s = 0; s < kSlotGroup; ++s) {
        stw[s * kPartialFloats + 2 + 2 * lane] = 0.f;
        stw[s * kPartialFloats + 3 + 2 * lane] = 0.f;
    }
    __syncthreads();

    const int key_end = min(n, (chunk + 1) * kChunkKeys);
    const int kbeg = chunk * kChunkKeys + warp * kGQuarter;
    const int kend = min(key_end, kbeg + kGQuarter);
    for (int k0 = kbeg; k0 < kend; k0 += kGKeys) {
        // This warp's tile (lane = key in the arithmetic below).  The copy
        // goes by rows: 16 consecutive lanes take one 256-byte row.
        {
            const int part = (lane & 15) * 4;
#pragma unroll
            for (int u = 0; u < kGKeys / 2; ++u) {
                const int c = (lane >> 4) + 2 * u;
                const int jc = k0 + c;
                const bool inc = jc < kend;
                const size_t row = size_t(inc ? jc : 0) * kDHead + part;
                cp_async16(&sm.k[warp][c][part], Kg + row, inc);
                cp_async16(&sm.v[warp][c][part], Vg + row, inc);
            }
        }
        cp_async_commit();
        const int j = k0 + lane;
        const bool in = j < kend;
        sm.ok[warp][lane] = in && bit_at(vb, j);
        cp_async_wait<0>();
        __syncwarp();
        const bool ok = sm.ok[warp][lane];
        for (int s = 0; s < rows; ++s) {
            float qv[kDHead];
#pragma unroll
            for (int x = 0; x < kDHead; x += 4) {
                const float4 t4 = *reinterpret_cast<const float4 *>(&sm.q[s][x]);
                qv[x] = t4.x;
                qv[x + 1] = t4.y;
                qv[x + 2] = t4.z;
                qv[x + 3] = t4.w;
            }
            const float sc = ok ? dot64(qv, &sm.k[warp][lane][0]) : -INFINITY;
            float tmax = sc;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
            float *row = stw + s * kPartialFloats;
            float mr = row[0], lr = row[1];
            float a0 = row[2 + 2 * lane], a1 = row[3 + 2 * lane];
            if (tmax > mr + kRescaleF || (mr == -INFINITY && tmax != -INFINITY)) {
                const float alpha = (mr == -INFINITY) ? 0.f : exp2f(mr - tmax);
                mr = tmax;
                lr *= alpha;
                a0 *= alpha;
                a1 *= alpha;
            }
            const float base = (mr == -INFINITY) ? 0.f : mr;
            const float p = exp2f(sc - base);
            float psum = p;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
            lr += psum;
#pragma unroll 8
            for (int c = 0; c < kGKeys; ++c) {
                const float pc = __shfl_sync(0xffffffffu, p, c);
                const float2 v2 = *reinterpret_cast<const float2 *>(&sm.v[warp][c][2 * lane]);
                a0 = fmaf(pc, v2.x, a0);
                a1 = fmaf(pc, v2.y, a1);
            }
            __syncwarp();
            if (lane == 0) {
                row[0] = mr;
                row[1] = lr;
            }
            row[2 + 2 * lane] = a0;
            row[3 + 2 * lane] = a1;
            __syncwarp();
        }
    }
    __syncthreads();

    // Merge the eight parts of the chunk into its partials: warp w takes
    // rows w, w+8, ...; lane owns two dimensions.
    const size_t mg = size_t(a.max_global);
    for (int s = warp; s < rows; s += kGWarps) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kGWarps; ++w) M = fmaxf(M, sm.st[w][s][0]);
        float L = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int w = 0; w < kGWarps; ++w) {
            const float mw = sm.st[w][s][0];
            const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            L = fmaf(f, sm.st[w][s][1], L);
            a0 = fmaf(f, sm.st[w][s][2 + 2 * lane], a0);
            a1 = fmaf(f, sm.st[w][s][3 + 2 * lane], a1);
        }
        float *P = partial_base(a, bh, chunk) + slot0 + s;
        if (lane == 0) {
            P[0] = M;
            P[mg] = L;
        }
        P[(2 + 2 * lane) * mg] = a0;
        P[(3 + 2 * lane) * mg] = a1;
    }

    // The last CTA of this (bh, group) to finish merges every chunk.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        int *ctr = a.ws.counters + size_t(bh) * (a.L.ngroups + 1) + group;
        const int prev = atomicAdd(ctr, 1);
        s_last = (prev == nch - 1);
        if (s_last) *ctr = 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float *Out = static_cast<float *>(a.out) + size_t(bh) * n * kDHead;
    for (int s = warp; s < rows; s += kGWarps) {
        const int slot = slot0 + s;
        const int p = gl[slot];
        if (!bit_at(vb, p)) continue;   // padded global position: the band CTAs wrote zeros
        combine_row_partials<float>(a, bh, slot, nch, lane, Out + size_t(p) * kDHead);
    }
}

// Brings `bytes` (a multiple of 16) from 16-byte aligned global memory into L2.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes)
{
    if (bytes == 0) return;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// The key and value rows a CTA will read, into L2, from the kernel arguments
// alone (no workspace value): a global CTA's chunk of Kg and Vg, a band CTA's
// query rows and the contiguous span of sequence positions its window taps
// fall in.  Issued before the wait for the kernel ahead in the stream; L2 is
// the point of coherence, so nothing it holds goes stale.
__device__ __forceinline__ void prefetch_inputs(const AttnArgs &a, int cta, int nglob)
{
    const int n = a.n;
    constexpr uint32_t kRow = kDHead * sizeof(float);
    if (cta < nglob) {
        const int per_bh = a.L.nchunks * a.L.ngroups;
        const int bh = cta / per_bh;
        const int chunk = (cta - bh * per_bh) % a.L.nchunks;
        const int k0 = chunk * kChunkKeys, k1 = min(n, k0 + kChunkKeys);
        const size_t off = (size_t(bh) * n + k0) * kDHead;
        prefetch_l2(static_cast<const float *>(a.kg) + off, uint32_t(k1 - k0) * kRow);
        prefetch_l2(static_cast<const float *>(a.vg) + off, uint32_t(k1 - k0) * kRow);
        return;
    }
    cta -= nglob;
    int b, h, r, tile;
    band_item(a, cta / kBandParts, b, h, r, tile);
    const int dil = a.dil[h];
    const int n_r = (n - r + dil - 1) / dil;
    const int r0 = tile * 128 + (cta % kBandParts) * kBandRows;
    if (r0 >= n_r) return;
    const int rows_hi = min(r0 + kBandRows - 1, n_r - 1);
    const int lo = max(a.causal ? r0 - (a.window - 1) : r0 - a.half, 0);
    const int hi = min(a.causal ? rows_hi : rows_hi + a.half, n_r - 1);
    const size_t base = size_t(b * a.H + h) * n * kDHead;
    const size_t q0 = size_t(r0 * dil + r) * kDHead, q1 = size_t(rows_hi * dil + r + 1) * kDHead;
    const size_t j0 = size_t(lo * dil + r) * kDHead, j1 = size_t(hi * dil + r + 1) * kDHead;
    prefetch_l2(static_cast<const float *>(a.q) + base + q0, uint32_t((q1 - q0) * sizeof(float)));
    prefetch_l2(static_cast<const float *>(a.k) + base + j0, uint32_t((j1 - j0) * sizeof(float)));
    prefetch_l2(static_cast<const float *>(a.v) + base + j0, uint32_t((j1 - j0) * sizeof(float)));
}

__global__ void __launch_bounds__(kF32Threads) attn_f32_kernel(const AttnArgs a, int nglob)
{
    extern __shared__ __align__(16) uint8_t f32_smem[];
    if (threadIdx.x == 0) prefetch_inputs(a, blockIdx.x, nglob);
    // The compacted indices, counts and bitmaps come from the kernel before.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (blockIdx.x == 0)
        for (int b = threadIdx.x; b < a.B; b += kF32Threads)
            if (a.ws.counts[b] > a.max_global) set_status(a.ws.status, kErrGlobalOverflow);
    if (int(blockIdx.x) < nglob)
        global_cta(a, blockIdx.x, f32_smem);
    else
        band_cta(a, blockIdx.x - nglob, f32_smem);
}

int launch_f32(const AttnArgs &a, cudaStream_t stream)
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(attn_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(kF32Smem)) != cudaSuccess)
            return kErrCuda;
        attr_set[dev] = true;
    }
    // Global CTAs first: they hold the longest key ranges.
    const int nglob = a.max_global > 0 ? a.B * a.H * a.L.nchunks * a.L.ngroups : 0;
    const int nband = a.B * a.band_items_per_batch * kBandParts;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nglob + nband);
    cfg.blockDim = dim3(kF32Threads);
    cfg.dynamicSmemBytes = kF32Smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attn_f32_kernel, a, nglob) != cudaSuccess) return kErrCuda;
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

}  // namespace lf
