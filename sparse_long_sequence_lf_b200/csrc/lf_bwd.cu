// Backward pass of the attention on the CUDA cores (fp32 arithmetic for
// every input type): the band kernels of the fp32 path (and of bf16 / fp16
// calls whose dilations exceed the tensor-core path's tensor maps), and the
// global-token kernels of every path.
//
// With s_ij = <q_i, k_j> / sqrt(d), p_ij = exp(s_ij - lse_i) over the key set
// of row i (the same sets as the forward: window taps and global tokens for a
// valid non-global row through Q, K, V; every valid token for a valid global
// row through Qg, Kg, Vg) and D_i = <dO_i, O_i>:
//   dP_ij = <dO_i, v_j>,  dS_ij = p_ij (dP_ij - D_i)
//   dq_i = sum_j dS_ij k_j / sqrt(d),  dk_j = sum_i dS_ij q_i / sqrt(d),
//   dv_j = sum_i p_ij dO_i.
// ("LongFormer: The Long-Document Transformer" notes, "Sliding Window",
// "Dilated Sliding Window", "Global Attention": the attention these rows
// differentiate.)
//
// Threads work in quads, each thread a quarter of the head dimension.
//   rows_kernel    32 query rows of one (batch, head, residue class) per CTA:
//                  pass 1 recomputes each row's log-sum-exp, pass 2 sums dq;
//                  writes lse and D per row.
//   keys_kernel    32 keys of one (batch, head, residue class) per CTA: dk, dv
//                  over the window rows that reach them, plus (for a global
//                  token) the sums gcols_kernel left in the scratch.
//   gcols_kernel   a global token as the key of the valid non-global rows that
//                  do not reach it through the window: chunks of 128 rows,
//                  fp32 atomic sums per slot (gcols_small_kernel: the same
//                  for at most 8 tokens, one warp per row, streamed).
//   grows_chunk_kernel  global rows (Qg) against 128-key chunks of Kg, Vg:
//                  pass 1 the chunk's (max, sum), pass 2 the merged
//                  log-sum-exp and the chunk's dqg terms (fp32 atomics);
//                  gfinal_kernel scales and stores dqg.
//   gkeys_kernel   dkg, dvg of every key over the global rows.
// Order (backward_schedule): band rows; global-token columns; band keys on
// the caller's stream, the global rows and gkeys on a side stream.
#include "lf_bwd.cuh"
#include "lf_vec.cuh"

namespace lf {

namespace bwd {

constexpr int kRows = 32;               // rows (or keys) per CTA
constexpr int kThreads = 4 * kRows;     // four threads per row
constexpr int kParts = 128 / kRows;     // CTAs per 128-row band item
constexpr int kTile = 32;               // keys (or rows) staged at a time
constexpr int kQ = kDHead / 4;          // dimensions per thread

__device__ __forceinline__ float quad_sum(float x)
{
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

// 32 rows of 64 values staged in shared memory by 128 threads: thread t loads
// row t/16 + 8u, dims 4*(t%16) .. +3, for u = 0..3.
template <typename T>
__device__ __forceinline__ void stage_rows(float (*dst)[kDHead], const T *base, const int (&pos)[4],
                                           int tid)
{
    const int x4 = 4 * (tid & 15);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int c = (tid >> 4) + 8 * u;
        const float4 v = pos[u] >= 0 ? load4(base + size_t(pos[u]) * kDHead + x4)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(&dst[c][x4]) = v;
    }
}

template <typename T>
__device__ __forceinline__ void load_quarter(float (&r)[kQ], const T *row, int qd, float scale)
{
#pragma unroll
    for (int x = 0; x < kQ; x += 4) {
        const float4 t = load4(row + kQ * qd + x);
        r[x] = t.x * scale;
        r[x + 1] = t.y * scale;
        r[x + 2] = t.z * scale;
        r[x + 3] = t.w * scale;
    }
}

template <typename T>
__device__ __forceinline__ void store_quarter(T *row, const float (&r)[kQ], int qd, float scale)
{
#pragma unroll
    for (int x = 0; x < kQ; x += 4)
        store4(row + kQ * qd + x,
               make_float4(r[x] * scale, r[x + 1] * scale, r[x + 2] * scale, r[x + 3] * scale));
}

__device__ __forceinline__ float dot_quarter(const float (&r)[kQ], const float *s, int qd)
{
    float d0 = 0.f, d1 = 0.f;
#pragma unroll
    for (int x = 0; x < kQ; x += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(s + kQ * qd + x);
        d0 = fmaf(r[x], v.x, d0);
        d1 = fmaf(r[x + 1], v.y, d1);
        d0 = fmaf(r[x + 2], v.z, d0);
        d1 = fmaf(r[x + 3], v.w, d1);
    }
    return quad_sum(d0 + d1);
}

__device__ __forceinline__ void axpy_quarter(float (&r)[kQ], float a, const float *s, int qd)
{
#pragma unroll
    for (int x = 0; x < kQ; x += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(s + kQ * qd + x);
        r[x] = fmaf(a, v.x, r[x]);
        r[x + 1] = fmaf(a, v.y, r[x + 1]);
        r[x + 2] = fmaf(a, v.z, r[x + 2]);
        r[x + 3] = fmaf(a, v.w, r[x + 3]);
    }
}

// ------------------------------------------------------------------ rows
template <typename T>
__global__ void __launch_bounds__(kThreads) rows_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    __shared__ __align__(16) float ks[kTile][kDHead];
    __shared__ __align__(16) float vs[kTile][kDHead];
    __shared__ int kpos[kTile];

    int b, h, r, tile;
    band_item(a, blockIdx.x / kParts, b, h, r, tile);
    const int dil = a.dil[h];
    const int n = a.n;
    const int n_r = (n - r + dil - 1) / dil;
    const int tid = threadIdx.x, rl = tid >> 2, qd = tid & 3;
    const int r0 = tile * 128 + (blockIdx.x % kParts) * kRows;
    if (r0 >= n_r) return;
    const int ir = r0 + rl;
    const bool row_in = ir < n_r;
    const int i = ir * dil + r;
    const size_t bh = size_t(b) * a.H + h;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    const bool active = row_in && bit_at(vb, i) && !bit_at(gb, i);
    const T *K = static_cast<const T *>(a.k) + bh * n * kDHead;
    const T *V = static_cast<const T *>(a.v) + bh * n * kDHead;
    const size_t rowoff = (bh * n + (row_in ? i : 0)) * kDHead;

    float q[kQ], dO[kQ], dq[kQ];
    float D = 0.f;
    {
        float o[kQ];
        if (active) {
            load_quarter(q, static_cast<const T *>(a.q) + rowoff, qd, a.scale_log2);
            load_quarter(dO, static_cast<const T *>(A.dout) + rowoff, qd, 1.f);
            load_quarter(o, static_cast<const T *>(A.out) + rowoff, qd, 1.f);
        } else {
#pragma unroll
            for (int x = 0; x < kQ; ++x) q[x] = dO[x] = o[x] = 0.f;
        }
        float d = 0.f;
#pragma unroll
        for (int x = 0; x < kQ; ++x) d = fmaf(dO[x], o[x], d);
        D = quad_sum(d);
#pragma unroll
        for (int x = 0; x < kQ; ++x) dq[x] = 0.f;
    }

    const int rows_hi = min(r0 + kRows - 1, n_r - 1);
    int lo = max(r0 - (a.causal ? a.window - 1 : a.half), 0);
    int hi = min(rows_hi + (a.causal ? 0 : a.half), n_r - 1);
    const int g = min(a.ws.counts[b], a.max_global);
    const int *gl = a.ws.gidx + size_t(b) * n;
    const int nband = hi >= lo ? (hi - lo) / kTile + 1 : 0;
    const int ntiles = nband + (g + kTile - 1) / kTile;

    // Key position of column c of tile t, or -1.
    auto key_at = [&](int t, int c) -> int {
        if (t < nband) {
            const int jr = lo + kTile * t + c;
            return (jr <= hi && jr * dil + r < n) ? jr * dil + r : -1;
        }
        const int slot = kTile * (t - nband) + c;
        return slot < g ? gl[slot] : -1;
    };
    // Is key column c of tile t a key of this row?
    auto is_key = [&](int t, int c) -> bool {
        const int j = kpos[c];
        if (!active || j < 0) return false;
        if (t < nband) {
            const int jr = lo + kTile * t + c;
            return a.causal ? (jr <= ir && ir - jr <= a.window - 1)
                            : (jr - ir <= a.half && ir - jr <= a.half);
        }
        return !is_tap(i, j, a.window, a.half, dil, a.causal);
    };
    auto stage = [&](int t, bool with_v) {
        __syncthreads();
        int pos[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = (tid >> 4) + 8 * u;
            const int j = key_at(t, c);
            pos[u] = j;
            if ((tid & 15) == 0) kpos[c] = (j >= 0 && bit_at(vb, j)) ? j : -1;
        }
        stage_rows(ks, K, pos, tid);
        if (with_v) stage_rows(vs, V, pos, tid);
        __syncthreads();
    };

    // Pass 1: log-sum-exp (log2 domain) of the row's scores.
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < ntiles; ++t) {
        stage(t, false);
        for (int c = 0; c < kTile; ++c) {
            const float s = dot_quarter(q, ks[c], qd);
            if (!is_key(t, c)) continue;
            const float mn = fmaxf(m, s);
            l = l * exp2f(m - mn) + exp2f(s - mn);
            m = mn;
        }
    }
    const float lse = l > 0.f ? m + log2f(l) : INFINITY;

    // Pass 2: dq.
    for (int t = 0; t < ntiles; ++t) {
        stage(t, true);
        for (int c = 0; c < kTile; ++c) {
            const float s = dot_quarter(q, ks[c], qd);
            const float dp = dot_quarter(dO, vs[c], qd);
            if (!is_key(t, c)) continue;
            const float p = exp2f(s - lse);
            axpy_quarter(dq, p * (dp - D), ks[c], qd);
        }
    }

    if (!row_in) return;
    // dq = sum dS k / sqrt(d); scale_log2 = log2(e) / sqrt(d).
    const float inv_sqrt_d = a.scale_log2 * 0.69314718055994531f;
    store_quarter(static_cast<T *>(A.dq) + rowoff, dq, qd, inv_sqrt_d);
    if (qd == 0) {
        A.lse[bh * n + i] = active ? lse : INFINITY;
        A.dsum[bh * n + i] = D;
    }
}

// Slot of global token j in the batch's ascending global index (binary search).
__device__ __forceinline__ int global_slot(const AttnArgs &a, int b, int j)
{
    const int *gl = a.ws.gidx + size_t(b) * a.n;
    int lo = 0, hi = min(a.ws.counts[b], a.max_global) - 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (gl[mid] < j) lo = mid + 1; else hi = mid;
    }
    return (hi >= 0 && gl[lo] == j) ? lo : -1;
}

// Adds the non-window contributions to global key j (this thread's quarter).
__device__ __forceinline__ void add_global_key_sums(const BwdArgs &A, int b, size_t bh, int j,
                                                    int qd, float (&dk)[kQ], float (&dv)[kQ])
{
    const int slot = global_slot(A.a, b, j);
    if (slot < 0) return;
    const float *src = A.gkv + (bh * A.a.max_global + slot) * (2 * kDHead);
#pragma unroll
    for (int x = 0; x < kQ; ++x) {
        dk[x] += src[kQ * qd + x];
        dv[x] += src[kDHead + kQ * qd + x];
    }
}

// ------------------------------------------------------------------ keys
template <typename T>
__global__ void __launch_bounds__(kThreads) keys_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    __shared__ __align__(16) float qs[kTile][kDHead];
    __shared__ __align__(16) float ds[kTile][kDHead];
    __shared__ float lse_s[kTile], d_s[kTile];
    __shared__ int rpos[kTile];

    int b, h, r, tile;
    band_item(a, blockIdx.x / kParts, b, h, r, tile);
    const int dil = a.dil[h];
    const int n = a.n;
    const int n_r = (n - r + dil - 1) / dil;
    const int tid = threadIdx.x, rl = tid >> 2, qd = tid & 3;
    const int k0 = tile * 128 + (blockIdx.x % kParts) * kRows;
    if (k0 >= n_r) return;
    const int jr = k0 + rl;
    const bool key_in = jr < n_r;
    const int j = jr * dil + r;
    const size_t bh = size_t(b) * a.H + h;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    const bool kvalid = key_in && bit_at(vb, j);
    const bool kglobal = kvalid && bit_at(gb, j);
    const size_t keyoff = (bh * n + (key_in ? j : 0)) * kDHead;
    const T *Q = static_cast<const T *>(a.q) + bh * n * kDHead;
    const T *dO = static_cast<const T *>(A.dout) + bh * n * kDHead;
    const float *lse = A.lse + bh * n;
    const float *dsum = A.dsum + bh * n;

    float k[kQ], v[kQ], dk[kQ], dv[kQ];
    if (kvalid) {
        load_quarter(k, static_cast<const T *>(a.k) + keyoff, qd, a.scale_log2);
        load_quarter(v, static_cast<const T *>(a.v) + keyoff, qd, 1.f);
    } else {
#pragma unroll
        for (int x = 0; x < kQ; ++x) k[x] = v[x] = 0.f;
    }
#pragma unroll
    for (int x = 0; x < kQ; ++x) dk[x] = dv[x] = 0.f;

    // Stage rows at positions pos (band or any), then accumulate.
    auto stage = [&](const int (&pos)[4]) {
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = (tid >> 4) + 8 * u;
            if ((tid & 15) == 0) {
                const int i = pos[u];
                const bool act = i >= 0 && bit_at(vb, i) && !bit_at(gb, i);
                rpos[c] = act ? i : -1;
                lse_s[c] = act ? lse[i] : INFINITY;
                d_s[c] = act ? dsum[i] : 0.f;
            }
        }
        stage_rows(qs, Q, pos, tid);
        stage_rows(ds, dO, pos, tid);
        __syncthreads();
    };
    auto accumulate = [&](int c) {
        const float s = dot_quarter(k, qs[c], qd);
        const float dp = dot_quarter(v, ds[c], qd);
        return make_float2(s, dp);
    };

    // Window rows: residue rows within reach of these keys.
    const int keys_hi = min(k0 + kRows - 1, n_r - 1);
    const int lo = max(a.causal ? k0 : k0 - a.half, 0);
    const int hi = min(a.causal ? keys_hi + a.window - 1 : keys_hi + a.half, n_r - 1);
    for (int t0 = lo; t0 <= hi; t0 += kTile) {
        int pos[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int ir = t0 + (tid >> 4) + 8 * u;
            pos[u] = (ir <= hi && ir * dil + r < n) ? ir * dil + r : -1;
        }
        stage(pos);
        for (int c = 0; c < kTile; ++c) {
            const float2 sd = accumulate(c);
            const int ir = t0 + c;
            const bool tap = a.causal ? (jr <= ir && ir - jr <= a.window - 1)
                                      : (jr - ir <= a.half && ir - jr <= a.half);
            if (!kvalid || rpos[c] < 0 || !tap) continue;
            const float p = exp2f(sd.x - lse_s[c]);
            axpy_quarter(dv, p, ds[c], qd);
            axpy_quarter(dk, p * (sd.y - d_s[c]), qs[c], qd);
        }
    }
    // A global token is also a key of every other valid non-global row of the
    // head: those sums come from gcols_kernel.
    if (kglobal) add_global_key_sums(A, b, bh, j, qd, dk, dv);

    if (!key_in) return;
    const float inv_sqrt_d = a.scale_log2 * 0.69314718055994531f;
    store_quarter(static_cast<T *>(A.dk) + keyoff, dk, qd, inv_sqrt_d);
    store_quarter(static_cast<T *>(A.dv) + keyoff, dv, qd, 1.f);
}

// Few global tokens leave most thread quads of a CTA without a slot: the CTA's
// gv valid slots (1..32) take G2 = the next power of two quads each, and the
// 32 / G2 groups of quads share out the streamed rows or keys of each tile.
struct SlotGroups {
    int G2, R, sl, grp;
};
__device__ __forceinline__ SlotGroups slot_groups(int gv, int rl)
{
    SlotGroups q;
    q.G2 = 1;
    while (q.G2 < gv) q.G2 <<= 1;
    q.R = kRows / q.G2;
    q.sl = rl & (q.G2 - 1);
    q.grp = rl / q.G2;
    return q;
}

// Sums v over the quads of this warp that share its slot (quads whose index
// differs by a multiple of G2); afterwards every such quad holds the warp's
// sum, and only the first of them (lane / 4 < G2) adds it to shared memory,
// so a shared sum takes one atomic add per warp instead of one per quad.
__device__ __forceinline__ float warp_slot_sum(float v, int G2)
{
    for (int off = 4 * G2; off < 32; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// ------------------------------------------------- global tokens as keys
// Contributions of the rows that reach a global token only as a global key
// (valid non-global rows that are not its window taps): one CTA per
// (batch*head, 32 global slots, kGChunk rows), fp32 sums added atomically to
// A.gkv.  Needs the rows' lse and D.
template <typename T>
__global__ void __launch_bounds__(kThreads) gcols_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    __shared__ __align__(16) float qs[kTile][kDHead];
    __shared__ __align__(16) float ds[kTile][kDHead];
    __shared__ float lse_s[kTile], d_s[kTile];
    __shared__ int rpos[kTile];
    __shared__ __align__(16) float red[kRows][2 * kDHead];

    const int n = a.n;
    const int sparts = (a.max_global + kRows - 1) / kRows;
    const int rchunks = (n + kGChunk - 1) / kGChunk;
    const int bh = blockIdx.x / (sparts * rchunks);
    const int rem = blockIdx.x - bh * sparts * rchunks;
    const int s0 = (rem / rchunks) * kRows;
    const int i0 = (rem % rchunks) * kGChunk;
    const int b = bh / a.H, h = bh - b * a.H;
    const int g = min(a.ws.counts[b], a.max_global);
    if (s0 >= g) return;
    const int tid = threadIdx.x, rl = tid >> 2, qd = tid & 3;
    const int gv = min(g - s0, kRows);
    const SlotGroups sg = slot_groups(gv, rl);
    const int slot = s0 + sg.sl;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    const int j = sg.sl < gv ? a.ws.gidx[size_t(b) * n + slot] : -1;
    for (int e = tid; e < kRows * 2 * kDHead; e += kThreads) (&red[0][0])[e] = 0.f;
    const bool kvalid = j >= 0 && bit_at(vb, j);
    const int dil = a.dil[h];
    const size_t keyoff = (size_t(bh) * n + (kvalid ? j : 0)) * kDHead;
    const T *Q = static_cast<const T *>(a.q) + size_t(bh) * n * kDHead;
    const T *dO = static_cast<const T *>(A.dout) + size_t(bh) * n * kDHead;
    const float *lse = A.lse + size_t(bh) * n;
    const float *dsum = A.dsum + size_t(bh) * n;

    float k[kQ], v[kQ], dk[kQ], dv[kQ];
    if (kvalid) {
        load_quarter(k, static_cast<const T *>(a.k) + keyoff, qd, a.scale_log2);
        load_quarter(v, static_cast<const T *>(a.v) + keyoff, qd, 1.f);
    } else {
#pragma unroll
        for (int x = 0; x < kQ; ++x) k[x] = v[x] = 0.f;
    }
#pragma unroll
    for (int x = 0; x < kQ; ++x) dk[x] = dv[x] = 0.f;

    for (int t0 = i0; t0 < min(i0 + kGChunk, n); t0 += kTile) {
        __syncthreads();
        int pos[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = (tid >> 4) + 8 * u;
            const int i = t0 + c;
            const bool act = i < n && bit_at(vb, i) && !bit_at(gb, i);
            pos[u] = act ? i : -1;
            if ((tid & 15) == 0) {
                rpos[c] = act ? i : -1;
                lse_s[c] = act ? lse[i] : INFINITY;
                d_s[c] = act ? dsum[i] : 0.f;
            }
        }
        stage_rows(qs, Q, pos, tid);
        stage_rows(ds, dO, pos, tid);
        __syncthreads();
#pragma unroll 2
        for (int c = sg.grp; c < kTile; c += sg.R) {
            const float sc = dot_quarter(k, qs[c], qd);
            const float dp = dot_quarter(v, ds[c], qd);
            const int i = rpos[c];
            if (!kvalid || i < 0 || is_tap(i, j, a.window, a.half, dil, a.causal)) continue;
            const float pr = exp2f(sc - lse_s[c]);
            axpy_quarter(dv, pr, ds[c], qd);
            axpy_quarter(dk, pr * (dp - d_s[c]), qs[c], qd);
        }
    }
    // Groups of the same slot meet in shared memory; one global add per value.
#pragma unroll
    for (int x = 0; x < kQ; ++x) {
        dk[x] = warp_slot_sum(dk[x], sg.G2);
        dv[x] = warp_slot_sum(dv[x], sg.G2);
    }
    if (kvalid && ((tid & 31) >> 2) < sg.G2) {
#pragma unroll
        for (int x = 0; x < kQ; ++x) {
            atomicAdd(&red[sg.sl][kQ * qd + x], dk[x]);
            atomicAdd(&red[sg.sl][kDHead + kQ * qd + x], dv[x]);
        }
    }
    __syncthreads();
    for (int e = tid; e < gv * 2 * kDHead; e += kThreads) {
        const int s_ = e / (2 * kDHead), x = e - s_ * (2 * kDHead);
        if (!bit_at(vb, a.ws.gidx[size_t(b) * n + s0 + s_])) continue;
        atomicAdd(A.gkv + (size_t(bh) * a.max_global + s0 + s_) * (2 * kDHead) + x, red[s_][x]);
    }
}

// The same sums for at most G global tokens (G = 1, 2, 4 or 8: the loops
// over tokens and rows are unrolled, so the code grows with G), streamed:
// one warp per row at a time, lane l holding dimensions 2l and 2l+1, the
// tokens' K and V rows and their dk, dv sums in registers; a warp takes
// kColRowsPerWarp rows, col_batch(G) at a time with all their loads (which
// do not depend on one another) issued first.  The warps of a CTA add their
// sums in shared memory, then once to A.gkv.
constexpr int kSmallG = 8;
constexpr int kColWarps = 8;
constexpr int kColRowsPerWarp = 16;
__host__ __device__ constexpr int col_batch(int) { return 4; }
constexpr int kColRows = kColWarps * kColRowsPerWarp;   // rows per CTA

template <typename T> __device__ __forceinline__ float2 load2(const T *p);
template <> __device__ __forceinline__ float2 load2<float>(const float *p)
{
    return *reinterpret_cast<const float2 *>(p);
}
template <> __device__ __forceinline__ float2 load2<__half>(const __half *p)
{
    return __half22float2(*reinterpret_cast<const __half2 *>(p));
}
template <> __device__ __forceinline__ float2 load2<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename T> __device__ void global_stats(const BwdArgs &A, size_t w, int lane);

// kStats (the rows' lse from the forward): the same pass also writes every
// row's lse and D = <dO_i, O_i> into A.lse, A.dsum (+inf and 0 for padded
// and global rows), reading the lse from A.lse_in, and the blocks past the
// rows' write the global slots' statistics (global_stats): one pass leaves
// everything the band keys and the global parts need.
template <typename T, int G, bool kStats>
__global__ void __launch_bounds__(32 * kColWarps) gcols_small_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    __shared__ __align__(16) float red[kColWarps][G][2 * kDHead];
    const int n = a.n;
    const int rchunks = (n + kColRows - 1) / kColRows;
    if (kStats && blockIdx.x >= unsigned(a.B * a.H * rchunks)) {
        global_stats<T>(A, size_t(blockIdx.x - a.B * a.H * rchunks) * 8 + (threadIdx.x >> 5),
                        threadIdx.x & 31);
        return;
    }
    const int bh = blockIdx.x / rchunks;
    const int i0 = (blockIdx.x % rchunks) * kColRows;
    const int b = bh / a.H, h = bh - b * a.H;
    const int g = min(a.ws.counts[b], min(a.max_global, G));
    if (!kStats && g == 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    const int dil = a.dil[h];
    const size_t base = size_t(bh) * n * kDHead + 2 * lane;
    const T *Q = static_cast<const T *>(a.q) + base;
    const T *dO = static_cast<const T *>(A.dout) + base;
    const T *O = static_cast<const T *>(A.out) + base;
    const float *lse = (kStats ? A.lse_in : A.lse) + size_t(bh) * n;
    const float *dsum = A.dsum + size_t(bh) * n;

    int js[G];
    float2 kk[G], vv[G], dk[G], dv[G];
#pragma unroll
    for (int s = 0; s < G; ++s) {
        js[s] = -1;
        kk[s] = vv[s] = dk[s] = dv[s] = make_float2(0.f, 0.f);
        if (s < g) {
            const int j = a.ws.gidx[size_t(b) * n + s];
            if (bit_at(vb, j)) {
                js[s] = j;
                const float2 kf = load2(static_cast<const T *>(a.k) + base + size_t(j) * kDHead);
                kk[s] = make_float2(kf.x * a.scale_log2, kf.y * a.scale_log2);
                vv[s] = load2(static_cast<const T *>(a.v) + base + size_t(j) * kDHead);
            }
        }
    }
    constexpr int kB = col_batch(G);
    const int r0 = i0 + warp * kColRowsPerWarp;
#pragma unroll 1
    for (int rb = r0; rb < min(r0 + kColRowsPerWarp, n); rb += kB) {
        float2 qv[kB], ov[kB], oo[kB];
        float lv[kB], dvv[kB];
        uint32_t vw[kB], gw[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int ii = min(rb + u, n - 1);
            vw[u] = vb[ii >> 5];
            gw[u] = gb[ii >> 5];
            qv[u] = load2(Q + size_t(ii) * kDHead);
            ov[u] = load2(dO + size_t(ii) * kDHead);
            if (kStats) oo[u] = load2(O + size_t(ii) * kDHead);
            lv[u] = lse[ii];
            dvv[u] = kStats ? 0.f : dsum[ii];
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int i = rb + u;
            if (i >= n) continue;
            const bool act = ((vw[u] >> (i & 31)) & 1u) && !((gw[u] >> (i & 31)) & 1u);
            if (kStats) {
                const float D = warp_sum(fmaf(ov[u].x, oo[u].x, ov[u].y * oo[u].y));
                dvv[u] = act ? D : 0.f;
                if (lane == 0) {
                    A.lse[size_t(bh) * n + i] = act ? lv[u] : INFINITY;
                    A.dsum[size_t(bh) * n + i] = dvv[u];
                }
            }
            if (!act) continue;
#pragma unroll
            for (int s = 0; s < G; ++s) {
                if (s >= g || js[s] < 0 || is_tap(i, js[s], a.window, a.half, dil, a.causal)) continue;
                const float sc = warp_sum(fmaf(qv[u].x, kk[s].x, qv[u].y * kk[s].y));
                const float dp = warp_sum(fmaf(ov[u].x, vv[s].x, ov[u].y * vv[s].y));
                const float pr = exp2f(sc - lv[u]);
                const float ds = pr * (dp - dvv[u]);
                dv[s].x = fmaf(pr, ov[u].x, dv[s].x);
                dv[s].y = fmaf(pr, ov[u].y, dv[s].y);
                dk[s].x = fmaf(ds, qv[u].x, dk[s].x);
                dk[s].y = fmaf(ds, qv[u].y, dk[s].y);
            }
        }
    }
#pragma unroll
    for (int s = 0; s < G; ++s) {
        if (s >= g) break;
        *reinterpret_cast<float2 *>(&red[warp][s][2 * lane]) = dk[s];
        *reinterpret_cast<float2 *>(&red[warp][s][kDHead + 2 * lane]) = dv[s];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < g * 2 * kDHead; e += 32 * kColWarps) {
        const int s = e / (2 * kDHead), x = e - s * (2 * kDHead);
        if (!bit_at(vb, a.ws.gidx[size_t(b) * n + s])) continue;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kColWarps; ++w) acc += red[w][s][x];
        atomicAdd(A.gkv + (size_t(bh) * a.max_global + s) * (2 * kDHead) + x, acc);
    }
}

// Global rows and Kg / Vg keys together for at most G global tokens, given
// their lse and D (A.lse_g, A.dsum_g from the forward): one pass over the
// keys computes, per key j and global row s, p = 2^(<qg_s, kg_j> log2e/8 -
// lse_s) and dS = p (<dO_s, vg_j> - D_s); it stores dkg_j = sum_s dS q_s / 8
// and dvg_j = sum_s p dO_s, and sums dq_s += dS kg_j into A.dqg_acc (fp32,
// atomically once per CTA and slot).  One warp per key at a time, lane l
// holding dimensions 2l, 2l+1; the global rows in registers.
template <typename T, int G>
__global__ void __launch_bounds__(32 * kColWarps) gglobal_small_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    __shared__ __align__(16) float red[kColWarps][G][kDHead];
    const int n = a.n;
    const size_t mg = size_t(a.max_global);
    const int kchunks = (n + kColRows - 1) / kColRows;
    const int bh = blockIdx.x / kchunks;
    const int j0 = (blockIdx.x % kchunks) * kColRows;
    const int b = bh / a.H;
    const int g = min(a.ws.counts[b], min(a.max_global, G));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const size_t base = size_t(bh) * n * kDHead + 2 * lane;
    bool act[G];
    float2 qv[G], ov[G], dq[G];
    float ls[G], ds[G];
#pragma unroll
    for (int s = 0; s < G; ++s) {
        act[s] = false;
        qv[s] = ov[s] = dq[s] = make_float2(0.f, 0.f);
        ls[s] = INFINITY;
        ds[s] = 0.f;
        if (s < g) {
            const int pos = a.ws.gidx[size_t(b) * n + s];
            if (bit_at(vb, pos)) {
                act[s] = true;
                qv[s] = load2(static_cast<const T *>(a.qg) + base + size_t(pos) * kDHead);
                ov[s] = load2(static_cast<const T *>(A.dout) + base + size_t(pos) * kDHead);
                ls[s] = A.lse_g[size_t(bh) * mg + s];
                ds[s] = A.dsum_g[size_t(bh) * mg + s];
            }
        }
    }
    const float sl2 = a.scale_log2;
    const float inv_sqrt_d = sl2 * 0.69314718055994531f;
    const int r0 = j0 + warp * kColRowsPerWarp;
#pragma unroll 1
    for (int jb = r0; jb < min(r0 + kColRowsPerWarp, n); jb += 4) {
        float2 kv[4], vv[4];
        uint32_t vw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int jj = min(jb + u, n - 1);
            vw[u] = vb[jj >> 5];
            kv[u] = load2(static_cast<const T *>(a.kg) + base + size_t(jj) * kDHead);
            vv[u] = load2(static_cast<const T *>(a.vg) + base + size_t(jj) * kDHead);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = jb + u;
            if (j >= n) continue;
            const bool kvalid = (vw[u] >> (j & 31)) & 1u;
            float2 dk = make_float2(0.f, 0.f), dv = make_float2(0.f, 0.f);
#pragma unroll
            for (int s = 0; s < G; ++s) {
                if (!act[s] || !kvalid) continue;
                const float sc = warp_sum(fmaf(qv[s].x, kv[u].x, qv[s].y * kv[u].y));
                const float dp = warp_sum(fmaf(ov[s].x, vv[u].x, ov[s].y * vv[u].y));
                const float pr = exp2f(fmaf(sc, sl2, -ls[s]));
                const float dsc = pr * (dp - ds[s]);
                dk.x = fmaf(dsc, qv[s].x, dk.x);
                dk.y = fmaf(dsc, qv[s].y, dk.y);
                dv.x = fmaf(pr, ov[s].x, dv.x);
                dv.y = fmaf(pr, ov[s].y, dv.y);
                dq[s].x = fmaf(dsc, kv[u].x, dq[s].x);
                dq[s].y = fmaf(dsc, kv[u].y, dq[s].y);
            }
            T *dkg = static_cast<T *>(A.dkg) + base + size_t(j) * kDHead;
            T *dvg = static_cast<T *>(A.dvg) + base + size_t(j) * kDHead;
            dkg[0] = from_f32<T>(dk.x * inv_sqrt_d);
            dkg[1] = from_f32<T>(dk.y * inv_sqrt_d);
            dvg[0] = from_f32<T>(dv.x);
            dvg[1] = from_f32<T>(dv.y);
        }
    }
#pragma unroll
    for (int s = 0; s < G; ++s)
        *reinterpret_cast<float2 *>(&red[warp][s][2 * lane]) = dq[s];
    __syncthreads();
    for (int e = threadIdx.x; e < G * kDHead; e += 32 * kColWarps) {
        const int s = e / kDHead, x = e - s * kDHead;
        if (s >= g) continue;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kColWarps; ++w) acc += red[w][s][x];
        if (s < g && bit_at(vb, a.ws.gidx[size_t(b) * n + s]))
            atomicAdd(A.dqg_acc + (size_t(bh) * mg + s) * kDHead + x, acc);
    }
}

// ------------------------------------------------------------ row statistics
// lse and D = <dO_i, O_i> of every position i of every (batch, head) as the
// band kernels leave them: the forward's lse and D for a valid non-global
// row, +inf and 0 otherwise.  Eight threads per row, eight dimensions each.
template <typename T> __device__ void global_stats(const BwdArgs &A, size_t w, int lane);

// Blocks past the rows' take the global slots (global_stats), so that one
// launch leaves every statistic.
template <typename T>
__global__ void __launch_bounds__(256) row_stats_kernel(const BwdArgs A, unsigned row_blocks)
{
    const AttnArgs &a = A.a;
    if (blockIdx.x >= row_blocks) {
        global_stats<T>(A, size_t(blockIdx.x - row_blocks) * 8 + (threadIdx.x >> 5),
                        threadIdx.x & 31);
        return;
    }
    const size_t rows = size_t(a.B) * a.H * a.n;
    const size_t r = size_t(blockIdx.x) * 32 + (threadIdx.x >> 3);
    const int part = threadIdx.x & 7;
    if (r >= rows) return;      // whole groups of 8 lanes leave together
    const int i = int(r % size_t(a.n));
    const int b = int(r / (size_t(a.n) * a.H));
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(b) * a.L.nwords;
    const bool active = bit_at(vb, i) && !bit_at(gb, i);
    const float4 o0 = load4(static_cast<const T *>(A.out) + r * kDHead + 8 * part);
    const float4 o1 = load4(static_cast<const T *>(A.out) + r * kDHead + 8 * part + 4);
    const float4 d0 = load4(static_cast<const T *>(A.dout) + r * kDHead + 8 * part);
    const float4 d1 = load4(static_cast<const T *>(A.dout) + r * kDHead + 8 * part + 4);
    float s = d0.x * o0.x;
    s = fmaf(d0.y, o0.y, s);
    s = fmaf(d0.z, o0.z, s);
    s = fmaf(d0.w, o0.w, s);
    s = fmaf(d1.x, o1.x, s);
    s = fmaf(d1.y, o1.y, s);
    s = fmaf(d1.z, o1.z, s);
    s = fmaf(d1.w, o1.w, s);
    const unsigned grp = 0xffu << (threadIdx.x & 24);
    s += __shfl_xor_sync(grp, s, 1);
    s += __shfl_xor_sync(grp, s, 2);
    s += __shfl_xor_sync(grp, s, 4);
    if (part == 0) {
        A.lse[r] = active ? A.lse_in[r] : INFINITY;
        A.dsum[r] = active ? s : 0.f;
    }
}

// The same for the global rows, per (batch*head, global slot) w: the
// forward's lse and D into A.lse_g, A.dsum_g (+inf and 0 past the count or
// padded).  One warp per slot, two dimensions per lane.
template <typename T>
__device__ void global_stats(const BwdArgs &A, size_t w, int lane)
{
    const AttnArgs &a = A.a;
    const size_t mg = size_t(a.max_global);
    if (w >= size_t(a.B) * a.H * mg) return;    // whole warps leave together
    const int bh = int(w / mg), slot = int(w % mg);
    const int b = bh / a.H;
    const int g = min(a.ws.counts[b], a.max_global);
    const int pos = slot < g ? a.ws.gidx[size_t(b) * a.n + slot] : 0;
    const bool active = slot < g && bit_at(a.ws.vbits + size_t(b) * a.L.nwords, pos);
    const size_t off = (size_t(bh) * a.n + pos) * kDHead + 2 * lane;
    const float2 o = load2(static_cast<const T *>(A.out) + off);
    const float2 d = load2(static_cast<const T *>(A.dout) + off);
    const float s = warp_sum(fmaf(d.x, o.x, d.y * o.y));
    if (lane == 0) {
        A.lse_g[w] = active ? A.lse_in[size_t(bh) * a.n + pos] : INFINITY;
        A.dsum_g[w] = active ? s : 0.f;
    }
}

// ------------------------------------------------------------ global rows
// Global rows against every valid key through Qg, Kg, Vg, split into chunks
// of kGChunk keys: gstats_kernel writes each chunk's (max, sum) of the row's
// scores; ggrad_kernel merges them into the row's log-sum-exp, then sums the
// chunk's dqg terms into A.dqg_acc; gfinal_kernel scales and stores dqg.
// One CTA per (batch*head, 32 global slots, chunk).
template <typename T, bool kGrad>
__global__ void __launch_bounds__(kThreads) grows_chunk_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    __shared__ __align__(16) float ks[kTile][kDHead];
    __shared__ __align__(16) float vs[kTile][kDHead];
    __shared__ int kok[kTile];
    __shared__ float2 ml_s[kRows];
    __shared__ __align__(16) float red[kRows][kDHead];

    const int n = a.n;
    const int sparts = (a.max_global + kRows - 1) / kRows;
    const int nch = A.nchg;
    const int bh = blockIdx.x / (sparts * nch);
    const int rem = blockIdx.x - bh * sparts * nch;
    const int s0 = (rem / nch) * kRows;
    const int chunk = rem % nch;
    const int b = bh / a.H;
    const int g = min(a.ws.counts[b], a.max_global);
    if (s0 >= g) return;
    const int tid = threadIdx.x, rl = tid >> 2, qd = tid & 3;
    const int gv = min(g - s0, kRows);
    const SlotGroups sg = slot_groups(gv, rl);
    const int slot = s0 + sg.sl;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const int i = sg.sl < gv ? a.ws.gidx[size_t(b) * n + slot] : -1;
    const bool active = i >= 0 && bit_at(vb, i);
    if (kGrad)
        for (int e = tid; e < kRows * kDHead; e += kThreads) (&red[0][0])[e] = 0.f;
    const size_t rowoff = (size_t(bh) * n + (active ? i : 0)) * kDHead;
    const T *Kg = static_cast<const T *>(a.kg) + size_t(bh) * n * kDHead;
    const T *Vg = static_cast<const T *>(a.vg) + size_t(bh) * n * kDHead;
    const size_t mg = size_t(a.max_global);
    float2 *part = A.gpart + size_t(bh) * nch * mg;

    float q[kQ], dO[kQ], dq[kQ];
    float D = 0.f, lse = INFINITY;
    if (active) {
        load_quarter(q, static_cast<const T *>(a.qg) + rowoff, qd, a.scale_log2);
    } else {
#pragma unroll
        for (int x = 0; x < kQ; ++x) q[x] = 0.f;
    }
    if (kGrad) {
        float o[kQ];
        if (active) {
            load_quarter(dO, static_cast<const T *>(A.dout) + rowoff, qd, 1.f);
            load_quarter(o, static_cast<const T *>(A.out) + rowoff, qd, 1.f);
        } else {
#pragma unroll
            for (int x = 0; x < kQ; ++x) dO[x] = o[x] = 0.f;
        }
        float d = 0.f;
#pragma unroll
        for (int x = 0; x < kQ; ++x) d = fmaf(dO[x], o[x], d);
        D = quad_sum(d);
        if (A.lse_in) {
            // The forward's lse and D, as row_stats_kernel left them.
            if (active) {
                lse = A.lse_g[size_t(bh) * mg + slot];
                D = A.dsum_g[size_t(bh) * mg + slot];
            }
        } else if (active) {
            // Merge the chunks' (max, sum) into the row's log-sum-exp.
            float M = -INFINITY;
            for (int c = 0; c < nch; ++c) M = fmaxf(M, part[c * mg + slot].x);
            float L = 0.f;
            for (int c = 0; c < nch; ++c) {
                const float2 ml = part[c * mg + slot];
                if (ml.x != -INFINITY) L += ml.y * exp2f(ml.x - M);
            }
            lse = L > 0.f ? M + log2f(L) : INFINITY;
        }
#pragma unroll
        for (int x = 0; x < kQ; ++x) dq[x] = 0.f;
    }

    float m = -INFINITY, l = 0.f;
    const int kend = min(n, (chunk + 1) * kGChunk);
    for (int t0 = chunk * kGChunk; t0 < kend; t0 += kTile) {
        __syncthreads();
        int pos[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = (tid >> 4) + 8 * u;
            const int jj = t0 + c;
            pos[u] = jj < kend ? jj : -1;
            if ((tid & 15) == 0) kok[c] = jj < kend && bit_at(vb, jj);
        }
        stage_rows(ks, Kg, pos, tid);
        if (kGrad) stage_rows(vs, Vg, pos, tid);
        __syncthreads();
#pragma unroll 2
        for (int c = sg.grp; c < kTile; c += sg.R) {
            const float sc = dot_quarter(q, ks[c], qd);
            if (kGrad) {
                const float dp = dot_quarter(dO, vs[c], qd);
                if (!active || !kok[c]) continue;
                const float pr = exp2f(sc - lse);
                axpy_quarter(dq, pr * (dp - D), ks[c], qd);
            } else {
                if (!active || !kok[c]) continue;
                const float mn = fmaxf(m, sc);
                l = l * exp2f(m - mn) + exp2f(sc - mn);
                m = mn;
            }
        }
    }
    if (!kGrad) {
        // Merge the groups' (max, sum) of each slot.
        if (qd == 0) ml_s[rl] = make_float2(m, l);
        __syncthreads();
        if (tid < gv) {
            float M = -INFINITY, L = 0.f;
            for (int q2 = 0; q2 < sg.R; ++q2) M = fmaxf(M, ml_s[q2 * sg.G2 + tid].x);
            if (M != -INFINITY)
                for (int q2 = 0; q2 < sg.R; ++q2) {
                    const float2 v = ml_s[q2 * sg.G2 + tid];
                    if (v.x != -INFINITY) L += v.y * exp2f(v.x - M);
                }
            part[size_t(chunk) * mg + s0 + tid] = make_float2(M, L);
        }
        return;
    }
    if (!A.lse_in && chunk == 0 && sg.grp == 0 && qd == 0 && sg.sl < gv) {
        A.lse_g[size_t(bh) * mg + slot] = lse;
        A.dsum_g[size_t(bh) * mg + slot] = D;
    }
#pragma unroll
    for (int x = 0; x < kQ; ++x) dq[x] = warp_slot_sum(dq[x], sg.G2);
    if (active && ((tid & 31) >> 2) < sg.G2) {
#pragma unroll
        for (int x = 0; x < kQ; ++x) atomicAdd(&red[sg.sl][kQ * qd + x], dq[x]);
    }
    __syncthreads();
    for (int e = tid; e < gv * kDHead; e += kThreads) {
        const int s_ = e / kDHead, x = e - s_ * kDHead;
        if (!bit_at(vb, a.ws.gidx[size_t(b) * n + s0 + s_])) continue;
        atomicAdd(A.dqg_acc + (size_t(bh) * mg + s0 + s_) * kDHead + x, red[s_][x]);
    }
}

// dqg of each valid global row: the fp32 sums scaled by 1/sqrt(d), in T.
// One thread per (batch*head, slot, 4 dimensions).
template <typename T>
__global__ void __launch_bounds__(256) gfinal_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    const size_t t = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t mg = size_t(a.max_global);
    if (t >= size_t(a.B) * a.H * mg * (kDHead / 4)) return;
    const int x4 = int(t % (kDHead / 4)) * 4;
    const size_t rs = t / (kDHead / 4);
    const int slot = int(rs % mg);
    const int bh = int(rs / mg);
    const int b = bh / a.H;
    if (slot >= min(a.ws.counts[b], a.max_global)) return;
    const int i = a.ws.gidx[size_t(b) * a.n + slot];
    if (!bit_at(a.ws.vbits + size_t(b) * a.L.nwords, i)) return;
    const float s = a.scale_log2 * 0.69314718055994531f;
    const float4 v = *reinterpret_cast<const float4 *>(A.dqg_acc + rs * kDHead + x4);
    store4(static_cast<T *>(A.dqg) + (size_t(bh) * a.n + i) * kDHead + x4,
           make_float4(v.x * s, v.y * s, v.z * s, v.w * s));
}

// ------------------------------------------------------------ global keys
template <typename T>
__global__ void __launch_bounds__(kThreads) gkeys_kernel(const BwdArgs A)
{
    const AttnArgs &a = A.a;
    __shared__ __align__(16) float qs[kTile][kDHead];
    __shared__ __align__(16) float ds[kTile][kDHead];
    __shared__ float lse_s[kTile], d_s[kTile];
    __shared__ int rok[kTile];

    // One CTA per (batch*head, 32 keys), flattened.
    const int kparts = (a.n + kRows - 1) / kRows;
    const int bh = blockIdx.x / kparts;
    const int b = bh / a.H;
    const int n = a.n;
    const int tid = threadIdx.x, rl = tid >> 2, qd = tid & 3;
    const int j = (blockIdx.x % kparts) * kRows + rl;
    const bool key_in = j < n;
    const uint32_t *vb = a.ws.vbits + size_t(b) * a.L.nwords;
    const bool kvalid = key_in && bit_at(vb, j);
    const size_t keyoff = (size_t(bh) * n + (key_in ? j : 0)) * kDHead;
    const int g = min(a.ws.counts[b], a.max_global);
    const int *gl = a.ws.gidx + size_t(b) * n;
    const T *Qg = static_cast<const T *>(a.qg) + size_t(bh) * n * kDHead;
    const T *dO = static_cast<const T *>(A.dout) + size_t(bh) * n * kDHead;

    float k[kQ], v[kQ], dk[kQ], dv[kQ];
    if (kvalid) {
        load_quarter(k, static_cast<const T *>(a.kg) + keyoff, qd, a.scale_log2);
        load_quarter(v, static_cast<const T *>(a.vg) + keyoff, qd, 1.f);
    } else {
#pragma unroll
        for (int x = 0; x < kQ; ++x) k[x] = v[x] = 0.f;
    }
#pragma unroll
    for (int x = 0; x < kQ; ++x) dk[x] = dv[x] = 0.f;

    for (int s0 = 0; s0 < g; s0 += kTile) {
        __syncthreads();
        int pos[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = (tid >> 4) + 8 * u;
            const int slot = s0 + c;
            const int i = slot < g ? gl[slot] : -1;
            const bool act = i >= 0 && bit_at(vb, i);
            pos[u] = act ? i : -1;
            if ((tid & 15) == 0) {
                rok[c] = act;
                lse_s[c] = act ? A.lse_g[size_t(bh) * a.max_global + slot] : INFINITY;
                d_s[c] = act ? A.dsum_g[size_t(bh) * a.max_global + slot] : 0.f;
            }
        }
        stage_rows(qs, Qg, pos, tid);
        stage_rows(ds, dO, pos, tid);
        __syncthreads();
        const int cn = min(kTile, g - s0);       // real slots of this tile
#pragma unroll 2
        for (int c = 0; c < cn; ++c) {
            const float s = dot_quarter(k, qs[c], qd);
            const float dp = dot_quarter(v, ds[c], qd);
            if (!kvalid || !rok[c]) continue;
            const float p = exp2f(s - lse_s[c]);
            axpy_quarter(dv, p, ds[c], qd);
            axpy_quarter(dk, p * (dp - d_s[c]), qs[c], qd);
        }
    }
    if (!key_in) return;
    const float inv_sqrt_d = a.scale_log2 * 0.69314718055994531f;
    store_quarter(static_cast<T *>(A.dkg) + keyoff, dk, qd, inv_sqrt_d);
    store_quarter(static_cast<T *>(A.dvg) + keyoff, dv, qd, 1.f);
}

}  // namespace bwd

template <typename T>
int launch_row_stats(const BwdArgs &A, cudaStream_t stream)
{
    using namespace bwd;
    const AttnArgs &a = A.a;
    const size_t rows = size_t(a.B) * a.H * a.n;
    if (rows == 0) return kOk;
    const size_t slots = size_t(a.B) * a.H * a.max_global;
    const unsigned slot_blocks = unsigned((slots + 7) / 8);
    if (a.max_global > 0 && a.max_global <= kSmallG) {
        // At most 8 global tokens: the statistics pass also sums the global
        // columns (gcols_small_kernel<..., true>), so no separate pass
        // stands between it and the band keys.
        if (cudaMemsetAsync(A.gkv, 0, sizeof(float) * slots * 2 * kDHead, stream) != cudaSuccess)
            return kErrCuda;
        const unsigned grid = unsigned(a.B * a.H * ((a.n + kColRows - 1) / kColRows)) + slot_blocks;
        if (a.max_global <= 1)
            gcols_small_kernel<T, 1, true><<<grid, 32 * kColWarps, 0, stream>>>(A);
        else if (a.max_global <= 2)
            gcols_small_kernel<T, 2, true><<<grid, 32 * kColWarps, 0, stream>>>(A);
        else if (a.max_global <= 4)
            gcols_small_kernel<T, 4, true><<<grid, 32 * kColWarps, 0, stream>>>(A);
        else
            gcols_small_kernel<T, kSmallG, true><<<grid, 32 * kColWarps, 0, stream>>>(A);
        return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
    }
    const unsigned row_blocks = unsigned((rows + 31) / 32);
    row_stats_kernel<T><<<row_blocks + slot_blocks, 256, 0, stream>>>(A, row_blocks);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

// Global rows (Qg against Kg, Vg): needs only the inputs and the prepared
// workspace, so it runs beside the band rows.
template <typename T>
int launch_global_rows(const BwdArgs &A, cudaStream_t stream)
{
    using namespace bwd;
    const AttnArgs &a = A.a;
    if (a.max_global == 0) return kOk;
    const int bh = a.B * a.H;
    const int sparts = (a.max_global + kRows - 1) / kRows;
    const size_t mg = size_t(a.max_global);
    if (cudaMemsetAsync(A.dqg_acc, 0, sizeof(float) * bh * mg * kDHead, stream) != cudaSuccess)
        return kErrCuda;
    // With the forward's lse (A.lse_in: row_stats_kernel has run) the
    // first pass is not needed.
    if (!A.lse_in) grows_chunk_kernel<T, false><<<bh * sparts * A.nchg, kThreads, 0, stream>>>(A);
    grows_chunk_kernel<T, true><<<bh * sparts * A.nchg, kThreads, 0, stream>>>(A);
    const size_t nfin = size_t(bh) * mg * (kDHead / 4);
    gfinal_kernel<T><<<unsigned((nfin + 255) / 256), 256, 0, stream>>>(A);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

// Global rows and Kg / Vg keys in one streamed pass for at most 8 global
// tokens, given their lse and D (A.lse_in set: global_stats has run), then
// dqg from the sums.
template <typename T>
int launch_global_small(const BwdArgs &A, cudaStream_t stream)
{
    using namespace bwd;
    const AttnArgs &a = A.a;
    const size_t bh = size_t(a.B) * a.H, mg = size_t(a.max_global);
    if (cudaMemsetAsync(A.dqg_acc, 0, sizeof(float) * bh * mg * kDHead, stream) != cudaSuccess)
        return kErrCuda;
    const int grid = int(bh) * ((a.n + kColRows - 1) / kColRows);
    if (a.max_global <= 1)
        gglobal_small_kernel<T, 1><<<grid, 32 * kColWarps, 0, stream>>>(A);
    else if (a.max_global <= 2)
        gglobal_small_kernel<T, 2><<<grid, 32 * kColWarps, 0, stream>>>(A);
    else if (a.max_global <= 4)
        gglobal_small_kernel<T, 4><<<grid, 32 * kColWarps, 0, stream>>>(A);
    else
        gglobal_small_kernel<T, kSmallG><<<grid, 32 * kColWarps, 0, stream>>>(A);
    if (cudaGetLastError() != cudaSuccess) return kErrCuda;
    return launch_global_final<T>(A, stream);
}

// dqg of the valid global rows from the fp32 sums in A.dqg_acc.
template <typename T>
int launch_global_final(const BwdArgs &A, cudaStream_t stream)
{
    using namespace bwd;
    const AttnArgs &a = A.a;
    const size_t nfin = size_t(a.B) * a.H * a.max_global * (kDHead / 4);
    if (nfin > 0) gfinal_kernel<T><<<unsigned((nfin + 255) / 256), 256, 0, stream>>>(A);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

// dkg, dvg of every key over the global rows (after launch_global_rows, which
// leaves the global rows' lse and D); zeros without global tokens.
template <typename T>
int launch_global_keys(const BwdArgs &A, size_t elem, cudaStream_t stream)
{
    using namespace bwd;
    const AttnArgs &a = A.a;
    if (a.max_global == 0) {
        const size_t bytes = size_t(a.B) * a.H * a.n * kDHead * elem;
        if (cudaMemsetAsync(A.dkg, 0, bytes, stream) != cudaSuccess) return kErrCuda;
        if (cudaMemsetAsync(A.dvg, 0, bytes, stream) != cudaSuccess) return kErrCuda;
        return kOk;
    }
    gkeys_kernel<T><<<a.B * a.H * ((a.n + kRows - 1) / kRows), kThreads, 0, stream>>>(A);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

// Global tokens as keys of the rows outside their window: needs the band
// rows' lse and D; the band keys read its sums.
template <typename T>
int launch_global_cols(const BwdArgs &A, cudaStream_t stream)
{
    using namespace bwd;
    const AttnArgs &a = A.a;
    if (a.max_global == 0) return kOk;
    const int bh = a.B * a.H;
    const int sparts = (a.max_global + kRows - 1) / kRows;
    const size_t mg = size_t(a.max_global);
    if (cudaMemsetAsync(A.gkv, 0, sizeof(float) * bh * mg * 2 * kDHead, stream) != cudaSuccess)
        return kErrCuda;
    const int cgrid = bh * ((a.n + kColRows - 1) / kColRows);
    if (a.max_global <= 1)
        gcols_small_kernel<T, 1, false><<<cgrid, 32 * kColWarps, 0, stream>>>(A);
    else if (a.max_global <= 2)
        gcols_small_kernel<T, 2, false><<<cgrid, 32 * kColWarps, 0, stream>>>(A);
    else if (a.max_global <= 4)
        gcols_small_kernel<T, 4, false><<<cgrid, 32 * kColWarps, 0, stream>>>(A);
    else if (a.max_global <= kSmallG)
        gcols_small_kernel<T, kSmallG, false><<<cgrid, 32 * kColWarps, 0, stream>>>(A);
    else
        gcols_kernel<T><<<bh * sparts * ((a.n + kGChunk - 1) / kGChunk), kThreads, 0, stream>>>(A);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

std::unique_lock<std::mutex> side_stream(SideStream *&out)
{
    static std::mutex mu;
    static SideStream side[64];
    static bool made[64] = {};
    std::unique_lock<std::mutex> lock(mu);
    out = nullptr;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return lock;
    if (!made[dev]) {
        SideStream &s = side[dev];
        if (cudaStreamCreateWithFlags(&s.stream, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&s.stream2, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&s.fork2, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&s.join2, cudaEventDisableTiming) != cudaSuccess)
            return lock;
        made[dev] = true;
    }
    out = &side[dev];
    return lock;
}

template <typename T>
int launch_backward_simt(const BwdArgs &A_in, size_t elem, cudaStream_t stream)
{
    using namespace bwd;
    // The CUDA-core path recomputes every log-sum-exp itself.
    BwdArgs A = A_in;
    A.lse_in = nullptr;
    const int band_ctas = A.a.B * A.a.band_items_per_batch * kParts;
    return backward_schedule<T>(
        A, elem, stream,
        [&](cudaStream_t st) {
            if (band_ctas > 0) rows_kernel<T><<<band_ctas, kThreads, 0, st>>>(A);
            return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
        },
        [&](cudaStream_t st) {
            if (band_ctas > 0) keys_kernel<T><<<band_ctas, kThreads, 0, st>>>(A);
            return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
        },
        [&](cudaStream_t st) { return launch_global_rows<T>(A, st); },
        [&](cudaStream_t st) { return launch_global_cols<T>(A, st); },
        [&](cudaStream_t st) { return launch_global_keys<T>(A, elem, st); }, false);
}

template int launch_global_rows<__half>(const BwdArgs &, cudaStream_t);
template int launch_global_rows<__nv_bfloat16>(const BwdArgs &, cudaStream_t);
template int launch_global_rows<float>(const BwdArgs &, cudaStream_t);
template int launch_global_small<__half>(const BwdArgs &, cudaStream_t);
template int launch_global_small<__nv_bfloat16>(const BwdArgs &, cudaStream_t);
template int launch_global_final<__half>(const BwdArgs &, cudaStream_t);
template int launch_global_final<__nv_bfloat16>(const BwdArgs &, cudaStream_t);
template int launch_global_keys<__half>(const BwdArgs &, size_t, cudaStream_t);
template int launch_global_keys<__nv_bfloat16>(const BwdArgs &, size_t, cudaStream_t);
template int launch_global_keys<float>(const BwdArgs &, size_t, cudaStream_t);
template int launch_global_cols<__half>(const BwdArgs &, cudaStream_t);
template int launch_global_cols<__nv_bfloat16>(const BwdArgs &, cudaStream_t);
template int launch_global_cols<float>(const BwdArgs &, cudaStream_t);
template int launch_row_stats<__half>(const BwdArgs &, cudaStream_t);
template int launch_row_stats<__nv_bfloat16>(const BwdArgs &, cudaStream_t);
template int launch_backward_simt<float>(const BwdArgs &, size_t, cudaStream_t);
template int launch_backward_simt<__half>(const BwdArgs &, size_t, cudaStream_t);
template int launch_backward_simt<__nv_bfloat16>(const BwdArgs &, size_t, cudaStream_t);

}  // namespace lf
