// Projection prologue of the attention: Q, K, V, Kg, Vg of every token and
// Qg of the global tokens, as tcgen05 GEMMs with a bias-and-split-heads
// epilogue (FasterTransformer Longformer Encoder guide, "compute flow": five
// products of the hidden states with the weight matrices over all tokens, a
// batched product for the global rows only, then bias add and transpose to
// [B, H, n, d]).
//
//   C[m, o] = sum_k X[m, k] W[o, k] + bias[o]
//   m = b*n + i (token), o = p*H*d + h*d + e (projection p, head h, dim e)
//   out_p[b, h, i, e] = C[m, o] rounded to the input type.
// The global-query product gathers the rows X[b, global_idx[b, s]] for
// s < counts[b] and writes Qg at those positions only.
//
// One CTA per 128 x 128 tile of C (non-persistent, two CTAs per SM):
//   warps 0-3  epilogue: TMEM -> registers, + bias, round, store rows
//   warp 4     TMA producer: 64-wide K slices of X and W through a 3-stage ring
//              (row by row for the gathered global rows)
//   warp 5     MMA issuer (one thread): tcgen05.mma kind::f16, 128x128x16,
//              both operands K-major in shared memory (128-byte swizzle),
//              fp32 accumulator in 128 TMEM columns.
// Every mbarrier wait is bounded; on expiry the kernel records
// LF_ERR_DEVICE_TIMEOUT in the optional status word, drains its copies and
// MMAs, frees its TMEM and returns.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cudaTypedefs.h>

#include "../../include/lf_attention.h"
#include "lf_sm100.cuh"

namespace lf {
namespace proj {

using namespace sm100;

constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kTileK = 64;                      // 128-byte rows of 16-bit elements
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kWarpProducer = 4;
constexpr int kWarpMma = 5;
constexpr uint32_t kTmemCols = 2 * kTileN;        // two accumulators: epilogue of one
                                                  // tile overlaps the MMAs of the next
constexpr int kSliceBytes = kTileM * kTileK * 2;   // 16 KB slice of A
constexpr int kBSliceBytes = kTileN * kTileK * 2;  // 32 KB slice of W

// One product C = A W^T + bias.
//   heads     A = X [M, K] row-major; C split into the [B, H, n, d] outputs
//   gather    A = the gathered global rows of X; C into out[0] at those rows
//   residual  A = the attention output [B, H, n, d] (one head per K slice);
//             sum = C + bias + residual in fp32
//   rows_res  A = [M, K] row-major; sum = C + bias + residual in fp32
//   gelu      A = [M, K] row-major; out[0] [M, N] = GELU(C + bias)
enum JobMode {
    kModeHeads = 0, kModeGather = 1, kModeResidual = 2, kModeRowsResidual = 3, kModeGelu = 4
};
__host__ __device__ constexpr bool rows_a(int mode)
{
    return mode == kModeHeads || mode == kModeRowsResidual || mode == kModeGelu;
}
struct ProjJob {
    CUtensorMap a_map;       // heads: X as {K, M} tiles of 64 x 128; gather: X as
                             // {K, B*n} single rows; residual: the attention output
                             // as {d, n, B*H} tiles of 64 x 128 x 1 (one head per K slice)
    CUtensorMap b_tile;      // W as {K, N} tiles of 64 x 128
    const void *bias;        // [N] in the input type, or NULL
    void *out[5];            // heads / gather: outputs of the column blocks of width H*d
    const void *residual;    // residual: [B, n, N] in the input type
    float *sum;              // residual: [B, n, N] fp32, C + bias + residual
    int M, N, mode;
    int tiles_per_batch;     // residual: M tiles of 128 tokens per batch
};

// Both products in one launch: grid rows [0, mtiles0) take job 0 (Q, K, V,
// Kg, Vg), the rest job 1 (Qg over the gathered global rows).
struct ProjParams {
    ProjJob job[2];
    const int32_t *gidx;     // [B, n] compacted global positions
    const int32_t *counts;   // [B]
    int32_t *status;         // optional device status word
    int K, B, H, n, max_global, mtiles0;
    int ntiles0, ntiles1, tiles0, tiles;   // column tiles per row of tiles; tile counts
};

// Tile t of the persistent schedule: job, first row, first column (column
// tiles fastest, so consecutive tiles share their rows of A).
__device__ __forceinline__ const ProjJob &tile_of(const ProjParams &p, int t, int &m0, int &n0)
{
    if (t < p.tiles0) {
        m0 = (t / p.ntiles0) * kTileM;
        n0 = (t % p.ntiles0) * kTileN;
        return p.job[0];
    }
    t -= p.tiles0;
    m0 = (t / p.ntiles1) * kTileM;
    n0 = (t % p.ntiles1) * kTileN;
    return p.job[1];
}

struct __align__(1024) ProjSmem {
    uint8_t a[kStages][kSliceBytes];
    uint8_t b[kStages][kBSliceBytes];
    uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    int abort_flag;
};

// Bounded wait (1 s); on expiry records the timeout and raises the abort flag.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         int32_t *status)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spins = 1;; ++spins) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((spins & 31u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                if (status) atomicCAS(status, 0, kErrDeviceTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Waits (bounded, ignoring the abort flag) for work this CTA started.
__device__ __forceinline__ void drain_bar(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
}

// Token row of output row m of the tile (gather mode: -1 for a slot past the
// batch's count), and its batch.
__device__ __forceinline__ int token_of(const ProjParams &p, const ProjJob &J, int m, int &b)
{
    if (J.mode == kModeResidual) {          // m = tile row: b * tiles_per_batch * 128 + i
        const int per = J.tiles_per_batch * kTileM;
        b = m / per;
        const int i = m - b * per;
        return i < p.n ? i : -1;
    }
    if (rows_a(J.mode)) {
        b = m / p.n;
        return m < J.M ? m - b * p.n : -1;
    }
    b = m / p.max_global;
    const int s = m - b * p.max_global;
    if (b >= p.B || s >= min(p.counts[b], p.max_global)) return -1;
    return p.gidx[size_t(b) * p.n + s];
}

template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi)
{
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Persistent: CTA c takes tiles c, c + gridDim.x, ...  The producer and the
// MMA thread run through the K slices of consecutive tiles without a break;
// the epilogue drains accumulator buffer t & 1 while the MMAs fill the other.
template <typename T>
__global__ void __launch_bounds__(kThreads, 1) proj_kernel(const __grid_constant__ ProjParams p)
{
    extern __shared__ uint8_t smem_raw[];
    ProjSmem &sm = *reinterpret_cast<ProjSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ktiles = p.K / kTileK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 4);     // one arrival per epilogue warp
        }
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kWarpProducer && lane == 0) {
        for (int j = 0; j < 2; ++j) {
            tma_prefetch_map(&p.job[j].a_map);
            tma_prefetch_map(&p.job[j].b_tile);
        }
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    if (warp == kWarpProducer) {
        int it = 0;          // K slices issued by this CTA
        bool ok = true;
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
            int m0, n0;
            const ProjJob &J = tile_of(p, t, m0, n0);
            // Gathered rows: only the real global tokens are loaded (the other
            // rows of the tile feed output rows that are never stored).
            int arow[kTileM / 32];
            int a_bytes = kSliceBytes;
            if (J.mode == kModeGather) {
                int valid = 0;
#pragma unroll
                for (int q = 0; q < kTileM / 32; ++q) {
                    int b;
                    const int i = token_of(p, J, m0 + 32 * q + lane, b);
                    arow[q] = i >= 0 ? b * p.n + i : -1;
                    valid += __popc(__ballot_sync(0xffffffffu, i >= 0));
                }
                a_bytes = valid * (kTileK * 2);
            }
            for (int kt = 0; kt < ktiles; ++kt, ++it) {
                const int s = it % kStages;
                const uint32_t ph = uint32_t(it / kStages) & 1u;
                bool w = true;
                if (lane == 0) w = wait_bar(&sm.empty[s], ph ^ 1u, abort_flag, p.status);
                ok = __shfl_sync(0xffffffffu, w, 0);
                if (!ok) break;
                if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], a_bytes + kBSliceBytes);
                __syncwarp();
                if (rows_a(J.mode)) {
                    if (lane == 0) tma_load_2d(sm.a[s], &J.a_map, &sm.full[s], kt * kTileK, m0);
                } else if (J.mode == kModeResidual) {
                    // K slice kt is head kt of the attention output: rows i0 ..
                    // i0+127 of batch b (rows past n read as zeros).
                    const int b = m0 / (J.tiles_per_batch * kTileM);
                    const int i0 = m0 - b * J.tiles_per_batch * kTileM;
                    if (lane == 0)
                        tma_load_3d(sm.a[s], &J.a_map, &sm.full[s], 0, i0, b * p.H + kt);
                } else {
#pragma unroll
                    for (int q = 0; q < kTileM / 32; ++q)
                        if (arow[q] >= 0)
                            tma_load_2d(sm.a[s] + (32 * q + lane) * (kTileK * 2), &J.a_map,
                                        &sm.full[s], kt * kTileK, arow[q]);
                }
                if (lane == 0) tma_load_2d(sm.b[s], &J.b_tile, &sm.full[s], kt * kTileK, n0);
                __syncwarp();
            }
        }
        if (*abort_flag && lane == 0) {
            // Copies still in flight land before the CTA exits.
            for (int k = max(0, it - kStages); k < it; ++k)
                drain_bar(&sm.full[k % kStages], uint32_t(k / kStages) & 1u);
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
            const uint32_t idesc = make_idesc(kTileM, kTileN, kBf16, false);
            bool ok = true;
            int it = 0, tc = 0;
            for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tc) {
                const int buf = tc & 1;
                ok = wait_bar(&sm.acc_empty[buf], (uint32_t(tc >> 1) & 1u) ^ 1u, abort_flag,
                              p.status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t acc = tmem + buf * kTileN;
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % kStages;
                    ok = wait_bar(&sm.full[s], uint32_t(it / kStages) & 1u, abort_flag, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t ad = make_sdesc(smem_u32(sm.a[s]), 16, 1024);
                    const uint64_t bd = make_sdesc(smem_u32(sm.b[s]), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < kTileK / 16; ++kk)
                        mma_ss(acc, ad + uint64_t((kk * 32) >> 4), bd + uint64_t((kk * 32) >> 4),
                               idesc, (kt > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&sm.empty[s]);
                }
                if (ok) tc_commit(&sm.acc_full[buf]);
            }
            // Every MMA issued here has completed once this commit lands.
            tc_commit(&sm.drain);
            drain_bar(&sm.drain, 0);
        }
        __syncwarp();
    } else {
        // Epilogue: thread t owns row m0 + t of each tile (TMEM lane t).
        bool ok = true;
        int tc = 0;
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tc) {
            int m0, n0;
            const ProjJob &J = tile_of(p, t, m0, n0);
            const int buf = tc & 1;
            bool w = true;
            if (lane == 0) w = wait_bar(&sm.acc_full[buf], uint32_t(tc >> 1) & 1u, abort_flag,
                                        p.status);
            ok = __shfl_sync(0xffffffffu, w, 0);
            if (!ok) break;
            tc_fence_after();
            int b;
            const int i = token_of(p, J, m0 + threadIdx.x, b);
            const int hid = p.H * kDHead;
            const uint32_t taddr = tmem + buf * kTileN + (uint32_t(warp * 32) << 16);
#pragma unroll
            for (int c = 0; c < kTileN / 32; ++c) {
                float acc[32];
                tmem_ld32(taddr + 32 * c, acc);
                const int o = n0 + 32 * c;                 // 32 columns within one head
                if (i < 0 || o >= J.N) continue;
                float bias[32];
                if (J.bias) {
                    const uint4 *b4 = reinterpret_cast<const uint4 *>(static_cast<const T *>(J.bias) + o);
                    uint4 bv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) bv[q] = __ldg(b4 + q);
                    const T *bt = reinterpret_cast<const T *>(bv);
#pragma unroll
                    for (int x = 0; x < 32; ++x) bias[x] = to_f32(bt[x]);
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) bias[x] = 0.f;
                }
                if (J.mode == kModeGelu) {
                    // GELU(x) = x * Phi(x), Phi written through erf.
                    T *dst = static_cast<T *>(J.out[0]) + (size_t(b) * p.n + i) * J.N + o;
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float g[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            const float v = acc[8 * q + x] + bias[8 * q + x];
                            g[x] = 0.5f * v * (1.f + erff(v * 0.70710678118654752f));
                        }
                        uint4 u;
                        u.x = pack2<T>(g[0], g[1]);
                        u.y = pack2<T>(g[2], g[3]);
                        u.z = pack2<T>(g[4], g[5]);
                        u.w = pack2<T>(g[6], g[7]);
                        d4[q] = u;
                    }
                    continue;
                }
                if (J.mode == kModeResidual || J.mode == kModeRowsResidual) {
                    const size_t row = (size_t(b) * p.n + i) * J.N + o;
                    // 32 residual values as four 16-byte loads.
                    const uint4 *res4 = reinterpret_cast<const uint4 *>(
                        static_cast<const T *>(J.residual) + row);
                    uint4 rv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) rv[q] = __ldg(res4 + q);
                    const T *res = reinterpret_cast<const T *>(rv);
                    float4 *dst = reinterpret_cast<float4 *>(J.sum + row);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 v;
                        v.x = acc[4 * q + 0] + bias[4 * q + 0] + to_f32(res[4 * q + 0]);
                        v.y = acc[4 * q + 1] + bias[4 * q + 1] + to_f32(res[4 * q + 1]);
                        v.z = acc[4 * q + 2] + bias[4 * q + 2] + to_f32(res[4 * q + 2]);
                        v.w = acc[4 * q + 3] + bias[4 * q + 3] + to_f32(res[4 * q + 3]);
                        dst[q] = v;
                    }
                    continue;
                }
                const int blk = o / hid, rem = o - blk * hid;
                const int h = rem / kDHead, e0 = rem - h * kDHead;
                T *dst = static_cast<T *>(J.out[blk]) +
                         ((size_t(b) * p.H + h) * p.n + i) * kDHead + e0;
                uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float *v = acc + 8 * q;
                    const float *bv = bias + 8 * q;
                    uint4 u;
                    u.x = pack2<T>(v[0] + bv[0], v[1] + bv[1]);
                    u.y = pack2<T>(v[2] + bv[2], v[3] + bv[3]);
                    u.z = pack2<T>(v[4] + bv[4], v[5] + bv[5]);
                    u.w = pack2<T>(v[6] + bv[6], v[7] + bv[7]);
                    d4[q] = u;
                }
            }
            // This warp's rows of the accumulator are read: the buffer may be
            // refilled.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// LayerNorm of each row of the fp32 sums: one warp per row.  Rows of up to
// 32 * 4 * kLnRegs features are read once into registers; longer rows are
// read again for each pass.  Mean first, then the mean square deviation, then
// out = (s - mean) / sqrt(var + eps) * gamma + beta in the output type.
constexpr int kLnRegs = 8;      // float4 per lane kept in registers (rows <= 1024)

template <typename T>
__device__ __forceinline__ void ln_store(T *dst, int o, float4 v, float mean, float inv,
                                         const T *__restrict__ gamma, const T *__restrict__ beta)
{
    const float y0 = (v.x - mean) * inv * to_f32(gamma[o]) + to_f32(beta[o]);
    const float y1 = (v.y - mean) * inv * to_f32(gamma[o + 1]) + to_f32(beta[o + 1]);
    const float y2 = (v.z - mean) * inv * to_f32(gamma[o + 2]) + to_f32(beta[o + 2]);
    const float y3 = (v.w - mean) * inv * to_f32(gamma[o + 3]) + to_f32(beta[o + 3]);
    uint2 u;
    u.x = pack2<T>(y0, y1);
    u.y = pack2<T>(y2, y3);
    *reinterpret_cast<uint2 *>(dst + o) = u;
}

template <typename T>
__global__ void __launch_bounds__(256) layernorm_kernel(const float *__restrict__ sum,
                                                        const T *__restrict__ gamma,
                                                        const T *__restrict__ beta, float eps,
                                                        int rows, int N, T *__restrict__ out)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= rows) return;
    const float4 *r4 = reinterpret_cast<const float4 *>(sum + size_t(warp) * N);
    T *dst = out + size_t(warp) * N;
    const int n4 = N / 4;
    if (n4 <= 32 * kLnRegs) {
        float4 v[kLnRegs];
        float s = 0.f;
#pragma unroll
        for (int u = 0; u < kLnRegs; ++u) {
            const int c = lane + 32 * u;
            v[u] = c < n4 ? __ldcs(r4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            s += (v[u].x + v[u].y) + (v[u].z + v[u].w);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mean = s / float(N);
        float q = 0.f;
#pragma unroll
        for (int u = 0; u < kLnRegs; ++u) {
            if (lane + 32 * u < n4) {
                const float a = v[u].x - mean, b = v[u].y - mean, e = v[u].z - mean,
                            f = v[u].w - mean;
                q += (a * a + b * b) + (e * e + f * f);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        const float inv = rsqrtf(q / float(N) + eps);
#pragma unroll
        for (int u = 0; u < kLnRegs; ++u) {
            const int c = lane + 32 * u;
            if (c < n4) ln_store(dst, 4 * c, v[u], mean, inv, gamma, beta);
        }
        return;
    }
    float s = 0.f;
    for (int c = lane; c < n4; c += 32) {
        const float4 v = r4[c];
        s += (v.x + v.y) + (v.z + v.w);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / float(N);
    float q = 0.f;
    for (int c = lane; c < n4; c += 32) {
        const float4 v = r4[c];
        const float a = v.x - mean, b = v.y - mean, e = v.z - mean, f = v.w - mean;
        q += (a * a + b * b) + (e * e + f * f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float inv = rsqrtf(q / float(N) + eps);
    for (int c = lane; c < n4; c += 32) ln_store(dst, 4 * c, r4[c], mean, inv, gamma, beta);
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// A row-major [rows, K] matrix of 16-bit elements as boxes of 64 x box_rows.
bool encode_matrix(CUtensorMap *m, const void *base, CUtensorMapDataType dt, long rows, int K,
                   int box_rows)
{
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(K) * 2};
    cuuint32_t box[2] = {kTileK, cuuint32_t(box_rows)};
    cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// The attention output [B, H, n, d] as {d, n, B*H} tiles of 64 x 128 x 1.
bool encode_heads(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int B, int H, int n)
{
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cuuint64_t(kDHead), cuuint64_t(n), cuuint64_t(B) * H};
    cuuint64_t strides[2] = {cuuint64_t(kDHead) * 2, cuuint64_t(n) * kDHead * 2};
    cuuint32_t box[3] = {kTileK, kTileM, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <typename T>
int launch(const ProjParams &p, cudaStream_t stream)
{
    const size_t smem = sizeof(ProjSmem) + 1024;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(proj_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess)
            return kErrCuda;
        attr_set[dev] = true;
    }
    ProjParams q = p;
    q.ntiles0 = (p.job[0].N + kTileN - 1) / kTileN;
    q.ntiles1 = p.job[1].N > 0 ? (p.job[1].N + kTileN - 1) / kTileN : 1;
    q.tiles0 = p.mtiles0 * q.ntiles0;
    q.tiles = q.tiles0 + ((p.job[1].M + kTileM - 1) / kTileM) * (p.job[1].M > 0 ? q.ntiles1 : 0);
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::max(1, std::min(q.tiles, sms > 0 ? sms : 1));
    proj_kernel<T><<<grid, kThreads, smem, stream>>>(q);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

}  // namespace proj

int launch_projection(lf_dtype dtype, int B, int n, int H, const void *x, const void *w,
                      const void *bias, const void *wqg, const void *bqg, const int32_t *gidx,
                      const int32_t *counts, int max_global, void *const out[6], int32_t *status,
                      cudaStream_t stream)
{
    using namespace proj;
    const CUtensorMapDataType dt =
        dtype == LF_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const int hid = H * kDHead;
    ProjParams p;
    std::memset(&p, 0, sizeof(p));
    p.K = hid;
    p.B = B;
    p.H = H;
    p.n = n;
    p.status = status;
    p.gidx = gidx;
    p.counts = counts;
    p.max_global = max_global;
    // Job 0: Q, K, V, Kg, Vg over every token.
    ProjJob &J0 = p.job[0];
    J0.M = B * n;
    J0.N = 5 * hid;
    J0.bias = bias;
    for (int j = 0; j < 5; ++j) J0.out[j] = out[j];
    if (!encode_matrix(&J0.a_map, x, dt, long(B) * n, hid, kTileM)) return kErrCuda;
    if (!encode_matrix(&J0.b_tile, w, dt, 5L * hid, hid, kTileN)) return kErrCuda;
    p.mtiles0 = (J0.M + kTileM - 1) / kTileM;
    // Job 1: Qg over the gathered global rows (none when max_global is 0).
    ProjJob &J1 = p.job[1];
    J1.mode = kModeGather;
    J1.M = (max_global > 0 && wqg) ? B * max_global : 0;
    J1.N = hid;
    J1.bias = bqg;
    for (int j = 0; j < 5; ++j) J1.out[j] = out[5];
    if (J1.M > 0) {
        if (!encode_matrix(&J1.a_map, x, dt, long(B) * n, hid, 1)) return kErrCuda;
        if (!encode_matrix(&J1.b_tile, wqg, dt, hid, hid, kTileN)) return kErrCuda;
    }
    return dtype == LF_BF16 ? launch<__nv_bfloat16>(p, stream) : launch<__half>(p, stream);
}

int launch_output_layer(lf_dtype dtype, int B, int n, int H, const void *attn, const void *wo,
                        const void *bo, const void *residual, const void *gamma,
                        const void *beta, float eps, void *out, float *sum, int32_t *status,
                        cudaStream_t stream)
{
    using namespace proj;
    const CUtensorMapDataType dt =
        dtype == LF_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const int hid = H * kDHead;
    ProjParams p;
    std::memset(&p, 0, sizeof(p));
    p.K = hid;
    p.B = B;
    p.H = H;
    p.n = n;
    p.status = status;
    ProjJob &J = p.job[0];
    J.mode = kModeResidual;
    J.tiles_per_batch = (n + kTileM - 1) / kTileM;
    J.M = B * J.tiles_per_batch * kTileM;
    J.N = hid;
    J.bias = bo;
    J.residual = residual;
    J.sum = sum;
    if (!encode_heads(&J.a_map, attn, dt, B, H, n)) return kErrCuda;
    if (!encode_matrix(&J.b_tile, wo, dt, hid, hid, kTileN)) return kErrCuda;
    p.mtiles0 = J.M / kTileM;
    p.job[1].M = 0;
    p.job[1].N = 0;
    int rc = dtype == LF_BF16 ? launch<__nv_bfloat16>(p, stream) : launch<__half>(p, stream);
    if (rc != kOk) return rc;
    const int rows = B * n;
    const int blocks = (rows + 7) / 8;
    if (dtype == LF_BF16)
        layernorm_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
            sum, static_cast<const __nv_bfloat16 *>(gamma), static_cast<const __nv_bfloat16 *>(beta),
            eps, rows, hid, static_cast<__nv_bfloat16 *>(out));
    else
        layernorm_kernel<__half><<<blocks, 256, 0, stream>>>(
            sum, static_cast<const __half *>(gamma), static_cast<const __half *>(beta), eps, rows,
            hid, static_cast<__half *>(out));
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

// C = A W^T (+ bias) over row-major A [M, K] in one persistent launch, with
// the GELU-store or the residual-sum epilogue.  M = B * n tokens.
int launch_rows_gemm(lf_dtype dtype, int mode, int B, int n, int K, int N, const void *a,
                     const void *w, const void *bias, void *out, const void *residual,
                     float *sum, int32_t *status, cudaStream_t stream)
{
    using namespace proj;
    const CUtensorMapDataType dt =
        dtype == LF_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    ProjParams p;
    std::memset(&p, 0, sizeof(p));
    p.K = K;
    p.B = B;
    p.H = 1;
    p.n = n;
    p.status = status;
    ProjJob &J = p.job[0];
    J.mode = mode;
    J.M = B * n;
    J.N = N;
    J.bias = bias;
    J.out[0] = out;
    J.residual = residual;
    J.sum = sum;
    if (!encode_matrix(&J.a_map, a, dt, long(B) * n, K, kTileM)) return kErrCuda;
    if (!encode_matrix(&J.b_tile, w, dt, N, K, kTileN)) return kErrCuda;
    p.mtiles0 = (J.M + kTileM - 1) / kTileM;
    return dtype == LF_BF16 ? launch<__nv_bfloat16>(p, stream) : launch<__half>(p, stream);
}

template <typename T>
static int layer_norm(const float *sum, const void *gamma, const void *beta, float eps, int rows,
                      int N, void *out, cudaStream_t stream)
{
    proj::layernorm_kernel<T><<<(rows + 7) / 8, 256, 0, stream>>>(
        sum, static_cast<const T *>(gamma), static_cast<const T *>(beta), eps, rows, N,
        static_cast<T *>(out));
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

// Feed-forward block: act = GELU(h W1^T + b1) [B*n, inter]; sum = act W2^T +
// b2 + h (fp32); out = LayerNorm(sum) with gamma, beta.
int launch_ffn(lf_dtype dtype, int B, int n, int hidden, int inter, const void *h,
               const void *w1, const void *b1, const void *w2, const void *b2,
               const void *gamma, const void *beta, float eps, void *out, void *act, float *sum,
               int32_t *status, cudaStream_t stream)
{
    using namespace proj;
    int rc = launch_rows_gemm(dtype, kModeGelu, B, n, hidden, inter, h, w1, b1, act, nullptr,
                              nullptr, status, stream);
    if (rc != kOk) return rc;
    rc = launch_rows_gemm(dtype, kModeRowsResidual, B, n, inter, hidden, act, w2, b2, nullptr, h,
                          sum, status, stream);
    if (rc != kOk) return rc;
    return dtype == LF_BF16
               ? layer_norm<__nv_bfloat16>(sum, gamma, beta, eps, B * n, hidden, out, stream)
               : layer_norm<__half>(sum, gamma, beta, eps, B * n, hidden, out, stream);
}

}  // namespace lf
