// Tensor-core (tcgen05) backward of the sliding-window band for bf16 / fp16.
//
// The gradients differentiate the attention of "LongFormer: The Long-Document
// Transformer" notes ("Sliding Window", "Dilated Sliding Window", "Global
// Attention"); with s = <q, k>, P = exp2(s * log2(e)/sqrt(d) - lse) and
// D_i = <dO_i, O_i>:
//   dS = P * (dO V^T - D),  dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d),
//   dV = P^T dO.
// Two kernels over the band items of the forward (128 rows of one batch,
// head and residue class of the head's dilation):
//   rows side  the 128 rows are queries (stationary Q, dO); the window's
//              64-key tiles and the global-token columns stream past twice:
//              pass 1 forms each row's log-sum-exp from S = Q K^T, pass 2
//              forms S, dP = dO V^T, dS, and dQ += dS K.  Writes dq, and lse
//              and D of every row for the keys side.
//   keys side  the 128 rows are keys (stationary K, V); the 64-row tiles of
//              queries that reach them through the window stream past once:
//              S^T = K Q^T, dP^T = V dO^T, P^T and dS^T from the rows' lse
//              and D, then dV += P^T dO and dK += dS^T Q.  A global token's
//              sums over the rows that reach it only as a global key (A.gkv)
//              are added at the end.
// Two more kinds of item run the keys side's products:
//   global keys    128 keys of Kg, Vg (every position) stationary; the
//                  global rows (Qg and dO rows at the global positions)
//                  stream past: dkg, dvg.  Needs the global rows' lse and D
//                  (more than 8 tokens; fewer take the CUDA-core kernel).
//   global columns up to 128 global tokens' K, V rows stationary; a chunk of
//                  the sequence's Q / dO rows streams past, masked to the
//                  valid non-global rows that do not reach the token through
//                  the window; the fp32 sums go atomically into A.gkv (more
//                  than 8 tokens; fewer take the CUDA-core kernel).
//   global rows    up to 128 global rows' Qg, dO stationary; a chunk of Kg,
//                  Vg tiles streams past once (the forward's lse): dqg sums
//                  into A.dqg_acc (more than 8 tokens and the forward's lse;
//                  otherwise the CUDA-core kernels of lf_bwd.cu).
//
// Every product is kind::f16 with fp32 accumulation in TMEM and the operand
// forms of the forward kernel: S-type products with both operands K-major in
// shared memory; accumulating products with the 16-bit P or dS in TMEM as A
// and the streamed tile, MN-major, as B.
//
// One CTA per item, 192 threads: warps 0-3 one thread per stationary row
// (TMEM lane), warp 4 TMA producer, warp 5 MMA issuer and TMEM owner.  TMEM
// (256 columns): T1 = S (P in its first 32 columns on the keys side), T2 =
// dP (dS in its first 32 columns), Acc1 = dQ or dK, Acc2 = dV.  Every
// mbarrier wait is bounded; on expiry the kernel records
// LF_ERR_DEVICE_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cudaTypedefs.h>

#include "lf_bwd.cuh"
#include "lf_sm100.cuh"
#include "lf_vec.cuh"

namespace lf {
namespace bwdtc {

using namespace sm100;

constexpr int kM = 128;                        // stationary rows per CTA
constexpr int kN = 64;                         // streamed rows per tile
constexpr int kStages = 3;
constexpr int kRowBytes = kDHead * 2;          // 128 B
constexpr int kTileBytes = kN * kRowBytes;     // 8 KB
constexpr int kStatBytes = kM * kRowBytes;     // 16 KB
constexpr int kThreads = 192;
constexpr int kWarpProducer = 4;
constexpr int kWarpMma = 5;
constexpr uint32_t kTmemCols = 256;
constexpr int kMaxResidues = 24;
enum { kTQ = 0, kTK = 1, kTV = 2, kTdO = 3 };
// Item kinds (template argument of the kernel).
enum Mode { kRowsMode = 0, kKeysMode = 1, kGKeysMode = 2, kGColsMode = 3, kGRowsMode = 4 };
constexpr int kGColRows = 512;           // rows a global-columns item streams
constexpr int kGRowKeys = 512;           // keys a global-rows item streams
// Items whose stationary rows are keys (dK, dV products) ...
__host__ __device__ constexpr bool keys_side(int mode)
{
    return mode == kKeysMode || mode == kGKeysMode || mode == kGColsMode;
}
// ... and items that stream their tiles once (the rows' lse is known).
__device__ __forceinline__ bool single_pass(int mode, const BwdArgs &A)
{
    return mode != kRowsMode || A.lse_in != nullptr;
}

struct Params {
    CUtensorMap res[4][kMaxResidues];   // 64-row tiles of the residue classes of Q, K, V, dO
    CUtensorMap krow, vrow;             // single rows of K and V (global-token columns)
    CUtensorMap kgt, vgt;               // 64-row tiles of Kg, Vg (global keys items)
    CUtensorMap qgrow, dorow;           // single rows of Qg, dO (global keys items)
    CUtensorMap qt, dot;                // 64-row tiles of Q, dO (global columns items)
    BwdArgs A;
    int res_base[kMaxHeads];            // first residue map of head h
    int oob_row;                        // a row past the end of the row maps (reads zeros)
};
static_assert(sizeof(Params) <= 32000, "kernel arguments exceed the parameter space");

struct __align__(1024) Smem {
    uint8_t a1[kStatBytes];             // stationary Q (rows side) or K (keys side)
    uint8_t a2[kStatBytes];             // stationary dO or V
    uint8_t b1[kStages][kTileBytes];    // streamed K or Q
    uint8_t b2[kStages][kTileBytes];    // streamed V or dO
    uint64_t stat_full, full[kStages], empty[kStages], s_full, p_full, acc_full, drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct Item {
    int b, h, bh, dil, r, n_r;
    int s0;       // first stationary row (residue space)
    int lo;       // first streamed row of band tile 0 (residue space)
    int nband;    // streamed band tiles
    int ngc;      // rows side: global-token column tiles
    int ntiles;   // tiles per pass
    int g;        // global tokens of the batch (clamped to max_global)
};

template <int kMode>
__device__ __forceinline__ Item decode(const AttnArgs &a)
{
    constexpr bool kKeys = keys_side(kMode);
    Item it;
    if (kMode == kGKeysMode || kMode == kGColsMode || kMode == kGRowsMode) {
        const int n = a.n;
        int rem;
        if (kMode == kGKeysMode) {
            const int nkb = (n + kM - 1) / kM;
            it.bh = blockIdx.x / nkb;
            rem = blockIdx.x - it.bh * nkb;
            it.s0 = rem * kM;
            it.lo = 0;
        } else {
            // A block of 128 global slots against a chunk of rows (global
            // columns) or of Kg / Vg keys (global rows).
            const int span = kMode == kGColsMode ? kGColRows : kGRowKeys;
            const int sblocks = (a.max_global + kM - 1) / kM;
            const int chunks = (n + span - 1) / span;
            it.bh = blockIdx.x / (sblocks * chunks);
            rem = blockIdx.x - it.bh * sblocks * chunks;
            it.s0 = (rem / chunks) * kM;
            it.lo = (rem % chunks) * span;
        }
        it.b = it.bh / a.H;
        it.h = it.bh - it.b * a.H;
        // Kg / Vg keys are plain positions; the global columns test window
        // taps with the head's dilation.
        it.dil = kMode == kGColsMode ? a.dil[it.h] : 1;
        it.r = 0;
        it.n_r = n;
        it.g = min(a.ws.counts[it.b], a.max_global);
        it.nband = kMode == kGKeysMode   ? (it.g + kN - 1) / kN
                   : kMode == kGColsMode ? (min(kGColRows, n - it.lo) + kN - 1) / kN
                                         : (min(kGRowKeys, n - it.lo) + kN - 1) / kN;
        it.ngc = 0;
        it.ntiles = it.nband;
        return it;
    }
    int tile;
    band_item(a, blockIdx.x, it.b, it.h, it.r, tile);
    it.bh = it.b * a.H + it.h;
    it.dil = a.dil[it.h];
    it.n_r = (a.n - it.r + it.dil - 1) / it.dil;
    it.s0 = tile * kM;
    const int s_hi = min(it.s0 + kM - 1, it.n_r - 1);
    int lo, hi;
    if (!kKeys) {                   // keys of these rows
        lo = it.s0 - (a.causal ? a.window - 1 : a.half);
        hi = s_hi + (a.causal ? 0 : a.half);
    } else {                        // rows that reach these keys
        lo = a.causal ? it.s0 : it.s0 - a.half;
        hi = s_hi + (a.causal ? a.window - 1 : a.half);
    }
    lo = max(lo, 0);
    hi = min(hi, it.n_r - 1);
    it.lo = lo;
    it.nband = (hi - lo) / kN + 1;
    it.g = min(a.ws.counts[it.b], a.max_global);
    it.ngc = kKeys ? 0 : (it.g + kN - 1) / kN;
    it.ntiles = it.nband + it.ngc;
    return it;
}

// Bounded wait taken by a whole warp: every lane goes on or every lane gives up.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int *status)
{
    const bool ok = mbar_wait(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}

// Waits (bounded, ignoring the abort flag) for work this CTA started.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
}

// Bits of the columns [32w, 32w + 32) that lie inside [clo, chi].
__device__ __forceinline__ uint32_t range_bits(int w, int clo, int chi)
{
    const int lo = min(max(clo - 32 * w, 0), 32);
    const int hi = min(max(chi - 32 * w + 1, 0), 32);
    const uint32_t below_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
    const uint32_t below_lo = lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u);
    return below_hi & ~below_lo;
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

template <typename T>
__device__ __forceinline__ float row_dot(const T *x, const T *y)
{
    float d0 = 0.f, d1 = 0.f;
#pragma unroll
    for (int c = 0; c < kDHead; c += 8) {
        const float4 a0 = load4(x + c), b0 = load4(y + c);
        const float4 a1 = load4(x + c + 4), b1 = load4(y + c + 4);
        d0 = fmaf(a0.x, b0.x, fmaf(a0.y, b0.y, fmaf(a0.z, b0.z, fmaf(a0.w, b0.w, d0))));
        d1 = fmaf(a1.x, b1.x, fmaf(a1.y, b1.y, fmaf(a1.z, b1.z, fmaf(a1.w, b1.w, d1))));
    }
    return d0 + d1;
}

template <typename T>
__device__ __forceinline__ void store_half_row(T *dst, const float (&v)[32], float scale)
{
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 u;
        u.x = pack2<T>(v[8 * q + 0] * scale, v[8 * q + 1] * scale);
        u.y = pack2<T>(v[8 * q + 2] * scale, v[8 * q + 3] * scale);
        u.z = pack2<T>(v[8 * q + 4] * scale, v[8 * q + 5] * scale);
        u.w = pack2<T>(v[8 * q + 6] * scale, v[8 * q + 7] * scale);
        d4[q] = u;
    }
}

// ---------------------------------------------------------------- producer
// Row of the flattened [B*H*n, 64] tensors holding global slot `slot` of
// the item's (batch, head), or a row past the end (reads zeros).
__device__ __forceinline__ int global_row(const Params &p, const Item &it, int slot)
{
    const AttnArgs &a = p.A.a;
    return slot < it.g ? it.bh * a.n + a.ws.gidx[size_t(it.b) * a.n + slot] : p.oob_row;
}

template <int kMode>
__device__ __forceinline__ void producer_role(const Params &p, Smem &sm, const Item &it, int lane)
{
    constexpr bool kKeys = keys_side(kMode);
    const AttnArgs &a = p.A.a;
    const int rb = kMode == kRowsMode || kMode == kKeysMode ? p.res_base[it.h] + it.r : 0;
    const int ta1 = kKeys ? kTK : kTQ, ta2 = kKeys ? kTV : kTdO;
    const int tb1 = kKeys ? kTQ : kTK, tb2 = kKeys ? kTdO : kTV;
    if (kMode == kGColsMode || kMode == kGRowsMode) {
        // The global tokens' K and V rows, or the global rows' Qg and dO
        // rows, gathered.
        const CUtensorMap *m1 = kMode == kGColsMode ? &p.krow : &p.qgrow;
        const CUtensorMap *m2 = kMode == kGColsMode ? &p.vrow : &p.dorow;
        if (lane == 0) mbar_arrive_expect_tx(&sm.stat_full, 2 * kStatBytes);
        __syncwarp();
        for (int rr = lane; rr < kM; rr += 32) {
            const int y = global_row(p, it, it.s0 + rr);
            tma_load_2d(sm.a1 + rr * kRowBytes, m1, &sm.stat_full, 0, y);
            tma_load_2d(sm.a2 + rr * kRowBytes, m2, &sm.stat_full, 0, y);
        }
        __syncwarp();
    } else if (lane == 0) {
        const CUtensorMap *m1 = kMode == kGKeysMode ? &p.kgt : &p.res[ta1][rb];
        const CUtensorMap *m2 = kMode == kGKeysMode ? &p.vgt : &p.res[ta2][rb];
        mbar_arrive_expect_tx(&sm.stat_full, 2 * kStatBytes);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(sm.a1 + hf * kTileBytes, m1, &sm.stat_full, 0, it.s0 + hf * kN, it.bh);
            tma_load_3d(sm.a2 + hf * kTileBytes, m2, &sm.stat_full, 0, it.s0 + hf * kN, it.bh);
        }
    }
    // The rows side streams the tiles twice unless the forward's log-sum-exp
    // of the rows is given (pass 1 only).
    const bool one_pass = single_pass(kMode, p.A);
    const int total = (one_pass ? 1 : 2) * it.ntiles;
    bool armed[kStages] = {};
    uint32_t armed_ph[kStages] = {};
    bool ok = true;
    for (int u = 0; u < total; ++u) {
        const int st = u % kStages;
        const uint32_t ph = uint32_t(u / kStages) & 1u;
        if (!warp_wait(&sm.empty[st], ph ^ 1u, &sm.abort_flag, a.ws.status)) {
            ok = false;
            break;
        }
        const int pass = one_pass ? 1 : u / it.ntiles, t = one_pass ? u : u - it.ntiles * pass;
        const bool need_b2 = kKeys || pass == 1;
        const uint32_t bytes = kTileBytes * (need_b2 ? 2u : 1u);
        if (kMode == kGKeysMode) {
            // The global rows: Qg and dO rows at the global positions.
            if (lane == 0) mbar_arrive_expect_tx(&sm.full[st], bytes);
            __syncwarp();
            for (int rr = lane; rr < kN; rr += 32) {
                const int y = global_row(p, it, t * kN + rr);
                tma_load_2d(sm.b1[st] + rr * kRowBytes, &p.qgrow, &sm.full[st], 0, y);
                tma_load_2d(sm.b2[st] + rr * kRowBytes, &p.dorow, &sm.full[st], 0, y);
            }
        } else if (kMode == kGColsMode || kMode == kGRowsMode) {
            // Q / dO tiles of the sequence, or Kg / Vg tiles.
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.full[st], bytes);
                tma_load_3d(sm.b1[st], kMode == kGColsMode ? &p.qt : &p.kgt, &sm.full[st], 0,
                            it.lo + t * kN, it.bh);
                tma_load_3d(sm.b2[st], kMode == kGColsMode ? &p.dot : &p.vgt, &sm.full[st], 0,
                            it.lo + t * kN, it.bh);
            }
        } else if (t < it.nband) {
            if (lane == 0) {
                const int y = it.lo + t * kN;
                mbar_arrive_expect_tx(&sm.full[st], bytes);
                tma_load_3d(sm.b1[st], &p.res[tb1][rb], &sm.full[st], 0, y, it.bh);
                if (need_b2) tma_load_3d(sm.b2[st], &p.res[tb2][rb], &sm.full[st], 0, y, it.bh);
            }
        } else {
            const int slot0 = (t - it.nband) * kN;
            if (lane == 0) mbar_arrive_expect_tx(&sm.full[st], bytes);
            __syncwarp();
            for (int rr = lane; rr < kN; rr += 32) {
                const int slot = slot0 + rr;
                const int y = slot < it.g ? it.bh * a.n + a.ws.gidx[size_t(it.b) * a.n + slot]
                                          : p.oob_row;
                tma_load_2d(sm.b1[st] + rr * kRowBytes, &p.krow, &sm.full[st], 0, y);
                if (need_b2) tma_load_2d(sm.b2[st] + rr * kRowBytes, &p.vrow, &sm.full[st], 0, y);
            }
        }
        armed[st] = true;
        armed_ph[st] = ph;
        __syncwarp();
    }
    if (!ok || sm.abort_flag) {
        if (lane == 0) {
            for (int s = 0; s < kStages; ++s)
                if (armed[s]) drain_wait(&sm.full[s], armed_ph[s]);
            drain_wait(&sm.stat_full, 0);
        }
        __syncwarp();
    }
}

// --------------------------------------------------------------------- MMA
template <int kMode>
__device__ __forceinline__ void mma_role(const Params &p, Smem &sm, const Item &it, uint32_t tmem,
                                         bool bf16)
{
    constexpr bool kKeys = keys_side(kMode);
    const AttnArgs &a = p.A.a;
    const uint32_t id_s = make_idesc(kM, kN, bf16, false);
    const uint32_t id_acc = make_idesc(kM, kDHead, bf16, true);
    const uint32_t tT1 = tmem, tT2 = tmem + 64, tA1 = tmem + 128, tA2 = tmem + 192;
    if (!warp_wait(&sm.stat_full, 0, &sm.abort_flag, a.ws.status)) return;
    tc_fence_after();
    const uint64_t a1d = make_sdesc(smem_u32(sm.a1), 16, 1024);
    const uint64_t a2d = make_sdesc(smem_u32(sm.a2), 16, 1024);
    const bool one_pass = single_pass(kMode, p.A);
    const int total = (one_pass ? 1 : 2) * it.ntiles;
    bool first_acc = true;
    for (int u = 0; u < total; ++u) {
        const int st = u % kStages;
        const uint32_t ph = uint32_t(u / kStages) & 1u;
        const bool grad = one_pass || u >= it.ntiles;
        if (!warp_wait(&sm.full[st], ph, &sm.abort_flag, a.ws.status)) return;
        tc_fence_after();
        const uint64_t b1d = make_sdesc(smem_u32(sm.b1[st]), 16, 1024);
        const uint64_t b2d = make_sdesc(smem_u32(sm.b2[st]), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kDHead / 16; ++kk)
            mma_ss_elect(tT1, a1d + uint64_t((kk * 32) >> 4), b1d + uint64_t((kk * 32) >> 4), id_s,
                         kk > 0 ? 1u : 0u);
        if (grad) {
#pragma unroll
            for (int kk = 0; kk < kDHead / 16; ++kk)
                mma_ss_elect(tT2, a2d + uint64_t((kk * 32) >> 4), b2d + uint64_t((kk * 32) >> 4),
                             id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit_elect(&sm.s_full);
        if (!grad) tc_commit_elect(&sm.empty[st]);
        __syncwarp();
        // T1 / T2 are rewritten by the next tile's products only after the
        // row threads have read them and stored P / dS (and the products
        // below, issued first, have read those: the tensor pipe runs in order).
        if (!warp_wait(&sm.p_full, uint32_t(u) & 1u, &sm.abort_flag, a.ws.status)) return;
        tc_fence_after();
        if (grad) {
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk)
                mma_ts_elect(tA1, tT2 + kk * 8, b1d + uint64_t((kk * 2048) >> 4), id_acc,
                             (kk > 0 || !first_acc) ? 1u : 0u);
            if (kKeys) {
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk)
                    mma_ts_elect(tA2, tT1 + kk * 8, b2d + uint64_t((kk * 2048) >> 4), id_acc,
                                 (kk > 0 || !first_acc) ? 1u : 0u);
            }
            first_acc = false;
            tc_commit_elect(&sm.empty[st]);
        }
        __syncwarp();
    }
    tc_commit_elect(&sm.acc_full);
    __syncwarp();
}

// ------------------------------------------------------------- rows side
// Key-column mask of one streamed tile for this thread's query row.
__device__ __forceinline__ void rows_mask(const AttnArgs &a, const Item &it, int t, int lane, int i,
                                          bool active, int tlo, int thi, uint32_t (&mw)[2])
{
    const uint32_t *vb = a.ws.vbits + size_t(it.b) * a.L.nwords;
    if (t < it.nband) {
        const int k0 = it.lo + t * kN;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const int jr = k0 + 32 * w + lane;
            const uint32_t cb =
                __ballot_sync(0xffffffffu, jr < it.n_r && bit_at(vb, jr * it.dil + it.r));
            mw[w] = active ? (range_bits(w, tlo - k0, thi - k0) & cb) : 0u;
        }
        return;
    }
    // Global-token columns: valid tokens that are not already window taps of
    // row i (a tap shares i's residue class and lies within the window span).
    const int slot0 = (t - it.nband) * kN;
    const int span_lo = a.causal ? (a.window - 1) * it.dil : a.half * it.dil;
    const int span_hi = a.causal ? 0 : a.half * it.dil;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const int slot = slot0 + 32 * w + lane;
        const int j = slot < it.g ? a.ws.gidx[size_t(it.b) * a.n + slot] : -1;
        const bool ok = j >= 0 && bit_at(vb, j);
        uint32_t m = __ballot_sync(0xffffffffu, ok);
        uint32_t rest = __ballot_sync(0xffffffffu, ok && (j % it.dil) == it.r);
        while (rest) {
            const int c = __ffs(rest) - 1;
            rest &= rest - 1u;
            const int d = __shfl_sync(0xffffffffu, j, c) - i;
            if (d >= -span_lo && d <= span_hi) m &= ~(1u << c);
        }
        mw[w] = active ? m : 0u;
    }
}

template <typename T>
__device__ __forceinline__ void rows_softmax(const Params &p, Smem &sm, const Item &it,
                                             uint32_t tmem, int tid)
{
    const BwdArgs &A = p.A;
    const AttnArgs &a = A.a;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t tT1 = tmem + (uint32_t(warp * 32) << 16);
    const uint32_t tT2 = tT1 + 64, tA1 = tT1 + 128;
    const float sl2 = a.scale_log2;
    const int n = a.n;
    const int row = it.s0 + tid;
    const bool row_in = row < it.n_r;
    const int i = row * it.dil + it.r;
    const uint32_t *vb = a.ws.vbits + size_t(it.b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(it.b) * a.L.nwords;
    const bool active = row_in && bit_at(vb, i) && !bit_at(gb, i);
    const size_t rowoff = (size_t(it.bh) * n + (row_in ? i : 0)) * kDHead;
    // With the forward's lse, the row statistics (lse, D) are already in
    // A.lse / A.dsum and the keys side may be reading them.
    const bool one_pass = A.lse_in != nullptr;
    const float D = one_pass ? A.dsum[size_t(it.bh) * n + (row_in ? i : 0)]
                    : active ? row_dot(static_cast<const T *>(A.dout) + rowoff,
                                       static_cast<const T *>(A.out) + rowoff)
                             : 0.f;
    const int tlo = row - (a.causal ? a.window - 1 : a.half);
    const int thi = row + (a.causal ? 0 : a.half);
    float m = -INFINITY, l = 0.f, lse = INFINITY;
    if (one_pass && active) lse = A.lse_in[size_t(it.bh) * n + i];

    for (int u = 0; u < (one_pass ? 1 : 2) * it.ntiles; ++u) {
        const int pass = one_pass ? 1 : u / it.ntiles, t = one_pass ? u : u - it.ntiles * pass;
        uint32_t mw[2];
        rows_mask(a, it, t, lane, i, active, tlo, thi, mw);
        if (!warp_wait(&sm.s_full, uint32_t(u) & 1u, &sm.abort_flag, a.ws.status)) return;
        tc_fence_after();
        if (pass == 0) {
            float s[64];
            tmem_ld32(tT1, *reinterpret_cast<float(*)[32]>(&s[0]));
            tmem_ld32(tT1 + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                s[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? s[c] * sl2 : -INFINITY;
                mt = fmaxf(mt, s[c]);
            }
            const float mn = fmaxf(m, mt);
            if (mn != -INFINITY) {
                float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    sum0 += ex2(s[c] - mn);
                    sum1 += ex2(s[c + 1] - mn);
                }
                l = l * ex2(m - mn) + (sum0 + sum1);
                m = mn;
            }
            if (t == it.ntiles - 1) lse = l > 0.f ? m + log2f(l) : INFINITY;
        } else {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float s[32], dp[32];
                tmem_ld32(tT1 + 32 * hf, s);
                tmem_ld32(tT2 + 32 * hf, dp);
                const uint32_t bits = mw[hf];
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float p0 = ((bits >> (2 * c)) & 1u) ? ex2(fmaf(s[2 * c], sl2, -lse)) : 0.f;
                    const float p1 =
                        ((bits >> (2 * c + 1)) & 1u) ? ex2(fmaf(s[2 * c + 1], sl2, -lse)) : 0.f;
                    pk[c] = pack2<T>(p0 * (dp[2 * c] - D), p1 * (dp[2 * c + 1] - D));
                }
                tmem_st16(tT2 + 16 * hf, pk);
            }
            tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
    }
    if (!warp_wait(&sm.acc_full, 0, &sm.abort_flag, a.ws.status)) return;
    tc_fence_after();
    const float inv_sqrt_d = sl2 * 0.69314718055994531f;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float acc[32];
        tmem_ld32(tA1 + 32 * hf, acc);
        if (row_in) store_half_row<T>(static_cast<T *>(A.dq) + rowoff + 32 * hf, acc, inv_sqrt_d);
    }
    if (row_in && !one_pass) {
        A.lse[size_t(it.bh) * n + i] = active ? lse : INFINITY;
        A.dsum[size_t(it.bh) * n + i] = D;
    }
}

// ------------------------------------------------------------- global rows
// Thread = global slot s0 + tid (its Qg and dO rows stationary); the chunk's
// Kg / Vg tiles stream past once with the rows' lse and D from
// row_stats_kernel.  Every valid key of the chunk counts.  dq sums (fp32,
// unscaled) go atomically into A.dqg_acc; gfinal_kernel scales and stores.
template <typename T>
__device__ __forceinline__ void grows_softmax(const Params &p, Smem &sm, const Item &it,
                                              uint32_t tmem, int tid)
{
    const BwdArgs &A = p.A;
    const AttnArgs &a = A.a;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t tT1 = tmem + (uint32_t(warp * 32) << 16);
    const uint32_t tT2 = tT1 + 64, tA1 = tT1 + 128;
    const float sl2 = a.scale_log2;
    const int n = a.n;
    const size_t mg = size_t(a.max_global);
    const int slot = it.s0 + tid;
    const uint32_t *vb = a.ws.vbits + size_t(it.b) * a.L.nwords;
    const bool active = slot < it.g && bit_at(vb, a.ws.gidx[size_t(it.b) * n + slot]);
    const float lse = active ? A.lse_g[size_t(it.bh) * mg + slot] : INFINITY;
    const float D = active ? A.dsum_g[size_t(it.bh) * mg + slot] : 0.f;

    for (int u = 0; u < it.ntiles; ++u) {
        uint32_t mw[2];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const int k = it.lo + u * kN + 32 * w + lane;
            const uint32_t cb = __ballot_sync(0xffffffffu, k < n && bit_at(vb, k));
            mw[w] = active ? cb : 0u;
        }
        if (!warp_wait(&sm.s_full, uint32_t(u) & 1u, &sm.abort_flag, a.ws.status)) return;
        tc_fence_after();
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float s[32], dp[32];
            tmem_ld32(tT1 + 32 * hf, s);
            tmem_ld32(tT2 + 32 * hf, dp);
            const uint32_t bits = mw[hf];
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float p0 = ((bits >> (2 * c)) & 1u) ? ex2(fmaf(s[2 * c], sl2, -lse)) : 0.f;
                const float p1 =
                    ((bits >> (2 * c + 1)) & 1u) ? ex2(fmaf(s[2 * c + 1], sl2, -lse)) : 0.f;
                pk[c] = pack2<T>(p0 * (dp[2 * c] - D), p1 * (dp[2 * c + 1] - D));
            }
            tmem_st16(tT2 + 16 * hf, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
    }
    if (!warp_wait(&sm.acc_full, 0, &sm.abort_flag, a.ws.status)) return;
    tc_fence_after();
    float *dst = A.dqg_acc + (size_t(it.bh) * mg + (active ? slot : 0)) * kDHead;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float acc[32];
        __syncwarp();
        tmem_ld32(tA1 + 32 * hf, acc);
        if (active) {
#pragma unroll
            for (int x = 0; x < 32; ++x) atomicAdd(dst + 32 * hf + x, acc[x]);
        }
    }
}

// ------------------------------------------------------------- keys side
// Slot of global token j in the batch's ascending global index.
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

template <typename T, int kMode>
__device__ __forceinline__ void keys_softmax(const Params &p, Smem &sm, const Item &it,
                                             uint32_t tmem, int tid)
{
    const BwdArgs &A = p.A;
    const AttnArgs &a = A.a;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t tT1 = tmem + (uint32_t(warp * 32) << 16);
    const uint32_t tT2 = tT1 + 64, tA1 = tT1 + 128, tA2 = tT1 + 192;
    const float sl2 = a.scale_log2;
    const int n = a.n;
    const size_t mg = size_t(a.max_global);
    // This thread's key: band keys in residue space, every position of Kg /
    // Vg, or the global token of slot s0 + tid.
    const int key = it.s0 + tid;
    const bool key_in = kMode == kGColsMode ? key < it.g : key < it.n_r;
    const int j = kMode == kGColsMode ? (key_in ? a.ws.gidx[size_t(it.b) * n + key] : 0)
                                      : key * it.dil + it.r;
    const uint32_t *vb = a.ws.vbits + size_t(it.b) * a.L.nwords;
    const uint32_t *gb = a.ws.gbits + size_t(it.b) * a.L.nwords;
    const bool kvalid = key_in && bit_at(vb, j);
    // Band keys: the rows (residue space) that take this key as a window tap.
    const int rlo = a.causal ? key : key - a.half;
    const int rhi = key + (a.causal ? a.window - 1 : a.half);
    // Global columns: the positions that take token j as a window tap.
    const int tlo = j - (a.causal ? 0 : a.half * it.dil);
    const int thi = j + (a.causal ? (a.window - 1) * it.dil : a.half * it.dil);
    const float *lse = kMode == kGKeysMode ? A.lse_g + size_t(it.bh) * mg : A.lse + size_t(it.bh) * n;
    const float *dsum = kMode == kGKeysMode ? A.dsum_g + size_t(it.bh) * mg
                                            : A.dsum + size_t(it.bh) * n;

    for (int u = 0; u < it.ntiles; ++u) {
        const int ir0 = it.lo + u * kN;
        // Lane l holds (lse, D) of the tile's rows l and l + 32; each warp
        // broadcasts them with shuffles (no cross-warp barrier).
        uint32_t mw[2];
        float cl[2], cd[2];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const int ir = ir0 + 32 * w + lane;
            if (kMode == kGKeysMode) {
                // Streamed row = global slot ir: a valid global row takes every
                // valid key.
                const bool act = ir < it.g && bit_at(vb, a.ws.gidx[size_t(it.b) * n + ir]);
                const uint32_t ab = __ballot_sync(0xffffffffu, act);
                mw[w] = kvalid ? ab : 0u;
                cl[w] = act ? lse[ir] : INFINITY;
                cd[w] = act ? dsum[ir] : 0.f;
            } else if (kMode == kGColsMode) {
                // Streamed row = position ir: valid non-global rows that are
                // not window taps of token j (same residue class within the
                // dilated span).
                const bool act = ir < n && bit_at(vb, ir) && !bit_at(gb, ir);
                const uint32_t ab = __ballot_sync(0xffffffffu, act);
                const int c0 = ir0 + 32 * w;
                uint32_t taps = range_bits(0, tlo - c0, thi - c0);
                if (it.dil > 1 && taps) {
                    uint32_t pat = 0u;
                    for (int c = ((j - c0) % it.dil + it.dil) % it.dil; c < 32; c += it.dil)
                        pat |= 1u << c;
                    taps &= pat;
                }
                mw[w] = kvalid ? (ab & ~taps) : 0u;
                cl[w] = act ? lse[ir] : INFINITY;
                cd[w] = act ? dsum[ir] : 0.f;
            } else {
                const int ii = ir * it.dil + it.r;
                const bool act = ir < it.n_r && bit_at(vb, ii) && !bit_at(gb, ii);
                const uint32_t ab = __ballot_sync(0xffffffffu, act);
                mw[w] = kvalid ? (range_bits(w, rlo - ir0, rhi - ir0) & ab) : 0u;
                cl[w] = act ? lse[ii] : INFINITY;
                cd[w] = act ? dsum[ii] : 0.f;
            }
        }
        if (!warp_wait(&sm.s_full, uint32_t(u) & 1u, &sm.abort_flag, a.ws.status)) return;
        tc_fence_after();
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float s[32], dp[32];
            tmem_ld32(tT1 + 32 * hf, s);
            tmem_ld32(tT2 + 32 * hf, dp);
            const uint32_t bits = mw[hf];
            uint32_t pp[16], pd[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float l0 = __shfl_sync(0xffffffffu, cl[hf], 2 * c);
                const float l1 = __shfl_sync(0xffffffffu, cl[hf], 2 * c + 1);
                const float d0 = __shfl_sync(0xffffffffu, cd[hf], 2 * c);
                const float d1 = __shfl_sync(0xffffffffu, cd[hf], 2 * c + 1);
                const float p0 = ((bits >> (2 * c)) & 1u) ? ex2(fmaf(s[2 * c], sl2, -l0)) : 0.f;
                const float p1 =
                    ((bits >> (2 * c + 1)) & 1u) ? ex2(fmaf(s[2 * c + 1], sl2, -l1)) : 0.f;
                pp[c] = pack2<T>(p0, p1);
                pd[c] = pack2<T>(p0 * (dp[2 * c] - d0), p1 * (dp[2 * c + 1] - d1));
            }
            tmem_st16(tT1 + 16 * hf, pp);
            tmem_st16(tT2 + 16 * hf, pd);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
    }
    if (!warp_wait(&sm.acc_full, 0, &sm.abort_flag, a.ws.status)) return;
    tc_fence_after();
    if (kMode == kGColsMode) {
        // Sums over this chunk's rows, unscaled dk then dv, into A.gkv.
        float *dst = A.gkv + (size_t(it.bh) * mg + (key_in ? key : 0)) * (2 * kDHead);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float dk[32], dv[32];
            __syncwarp();
            tmem_ld32(tA1 + 32 * hf, dk);
            tmem_ld32(tA2 + 32 * hf, dv);
            if (kvalid) {
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    atomicAdd(dst + 32 * hf + x, dk[x]);
                    atomicAdd(dst + kDHead + 32 * hf + x, dv[x]);
                }
            }
        }
        return;
    }
    if (kMode == kGKeysMode) {
        const float inv_sqrt_d = sl2 * 0.69314718055994531f;
        const size_t keyoff = (size_t(it.bh) * n + (key_in ? key : 0)) * kDHead;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float dk[32], dv[32];
            __syncwarp();
            tmem_ld32(tA1 + 32 * hf, dk);
            tmem_ld32(tA2 + 32 * hf, dv);
            if (key_in) {
                store_half_row<T>(static_cast<T *>(A.dkg) + keyoff + 32 * hf, dk, inv_sqrt_d);
                store_half_row<T>(static_cast<T *>(A.dvg) + keyoff + 32 * hf, dv, 1.f);
            }
        }
        return;
    }
    const int slot = (kvalid && bit_at(gb, j)) ? global_slot(a, it.b, j) : -1;
    const float *gsum = slot >= 0 ? A.gkv + (size_t(it.bh) * a.max_global + slot) * (2 * kDHead)
                                  : nullptr;
    const float inv_sqrt_d = sl2 * 0.69314718055994531f;
    const size_t keyoff = (size_t(it.bh) * n + (key_in ? j : 0)) * kDHead;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float dk[32], dv[32];
        tmem_ld32(tA1 + 32 * hf, dk);
        tmem_ld32(tA2 + 32 * hf, dv);
        if (gsum) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                dk[x] += gsum[32 * hf + x];
                dv[x] += gsum[kDHead + 32 * hf + x];
            }
        }
        if (key_in) {
            store_half_row<T>(static_cast<T *>(A.dk) + keyoff + 32 * hf, dk, inv_sqrt_d);
            store_half_row<T>(static_cast<T *>(A.dv) + keyoff + 32 * hf, dv, 1.f);
        }
    }
}

// ------------------------------------------------------------------ kernel
template <typename T, int kMode>
__global__ void __launch_bounds__(kThreads) bwd_tc_kernel(const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Item it = decode<kMode>(p.A.a);
    // Items without work leave before any barrier or tensor memory is set up:
    // global columns past the batch's tokens; global keys of a batch without
    // global tokens store zero gradients.
    if ((kMode == kGColsMode || kMode == kGRowsMode) && (it.s0 >= it.g || it.ntiles <= 0)) return;
    if (kMode == kGKeysMode && it.g == 0) {
        const int key = it.s0 + int(threadIdx.x);
        if (threadIdx.x < kM && key < it.n_r) {
            const size_t off = (size_t(it.bh) * it.n_r + key) * kDHead;
            float z[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) z[x] = 0.f;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                store_half_row<T>(static_cast<T *>(p.A.dkg) + off + 32 * hf, z, 1.f);
                store_half_row<T>(static_cast<T *>(p.A.dvg) + off + 32 * hf, z, 1.f);
            }
        }
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(&sm.stat_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, 4);       // one arrival per row warp
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp < 4) {
        if (keys_side(kMode))
            keys_softmax<T, kMode>(p, sm, it, tmem, threadIdx.x);
        else if (kMode == kGRowsMode)
            grows_softmax<T>(p, sm, it, tmem, threadIdx.x);
        else
            rows_softmax<T>(p, sm, it, tmem, threadIdx.x);
    } else if (warp == kWarpProducer) {
        producer_role<kMode>(p, sm, it, lane);
    } else {
        mma_role<kMode>(p, sm, it, tmem, std::is_same<T, __nv_bfloat16>::value);
        // Every MMA this warp issued has completed once this commit lands.
        tc_commit_elect(&sm.drain);
        __syncwarp();
        drain_wait(&sm.drain, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// -------------------------------------------------------------------- host
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

// rows = 0: single rows of the flattened [B*H*n, 64] tensor; otherwise tiles
// of kN rows of residue class r of dilation dil of each (batch*head) slice.
bool encode(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int n, int BH, bool tiles,
            int dil, int r)
{
    auto enc = encoder();
    if (!enc) return false;
    if (!tiles) {
        cuuint64_t dims[2] = {cuuint64_t(kDHead), cuuint64_t(n) * BH};
        cuuint64_t strides[1] = {cuuint64_t(kRowBytes)};
        cuuint32_t box[2] = {kDHead, 1};
        cuuint32_t es[2] = {1, 1};
        return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
               CUDA_SUCCESS;
    }
    const int n_r = (n - r + dil - 1) / dil;
    base = static_cast<const char *>(base) + size_t(r) * kRowBytes;
    cuuint64_t dims[3] = {cuuint64_t(kDHead), cuuint64_t(n_r), cuuint64_t(BH)};
    cuuint64_t strides[2] = {cuuint64_t(dil) * kRowBytes, cuuint64_t(n) * kRowBytes};
    cuuint32_t box[3] = {kDHead, cuuint32_t(kN), 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Encoded maps, reused while the same buffer and shape come back.
bool cached(CUtensorMap *out, const void *base, CUtensorMapDataType dt, int n, int BH, bool tiles,
            int dil = 1, int r = 0)
{
    struct Entry {
        const void *base;
        int dt, n, BH, tiles, dil, r;
        CUtensorMap map;
        bool used;
    };
    constexpr int kCache = 256;
    static std::mutex mu;
    static Entry cache[kCache];
    static unsigned next = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &e : cache)
        if (e.used && e.base == base && e.dt == int(dt) && e.n == n && e.BH == BH &&
            e.tiles == int(tiles) && e.dil == dil && e.r == r) {
            *out = e.map;
            return true;
        }
    CUtensorMap m;
    if (!encode(&m, base, dt, n, BH, tiles, dil, r)) return false;
    cache[next++ % kCache] = Entry{base, int(dt), n, BH, int(tiles), dil, r, m, true};
    *out = m;
    return true;
}

template <typename T, int kMode>
int launch_side(const Params &p, cudaStream_t stream)
{
    const AttnArgs &a = p.A.a;
    const size_t smem = sizeof(Smem) + 1024;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(bwd_tc_kernel<T, kMode>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess)
            return kErrCuda;
        attr_set[dev] = true;
    }
    const int BH = a.B * a.H;
    const int sblocks = (a.max_global + kM - 1) / kM;
    const int grid =
        kMode == kGKeysMode   ? BH * ((a.n + kM - 1) / kM)
        : kMode == kGColsMode ? BH * sblocks * ((a.n + kGColRows - 1) / kGColRows)
        : kMode == kGRowsMode ? BH * sblocks * ((a.n + kGRowKeys - 1) / kGRowKeys)
                              : a.B * a.band_items_per_batch;
    if (grid > 0) bwd_tc_kernel<T, kMode><<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

// Global tokens as keys of the rows outside their window: the streamed
// CUDA-core kernel for at most 8 tokens, else the tensor-core items.
template <typename T>
int launch_global_cols_tc(const Params &p, cudaStream_t stream)
{
    const AttnArgs &a = p.A.a;
    // With the forward's lse and at most 8 tokens the statistics pass has
    // already summed them (launch_row_stats).
    if (a.max_global <= 8) return p.A.lse_in ? kOk : launch_global_cols<T>(p.A, stream);
    const size_t bytes = sizeof(float) * size_t(a.B) * a.H * a.max_global * 2 * kDHead;
    if (cudaMemsetAsync(p.A.gkv, 0, bytes, stream) != cudaSuccess) return kErrCuda;
    return launch_side<T, kGColsMode>(p, stream);
}

// dqg of the global rows: with the forward's lse, the tensor-core items for
// more than 8 global tokens (one pass, fp32 sums, then gfinal_kernel) and
// the streamed CUDA-core pass over the keys for fewer (which also leaves
// dkg, dvg); without it the CUDA-core kernels.
template <typename T>
int launch_global_rows_tc(const Params &p, cudaStream_t stream)
{
    const AttnArgs &a = p.A.a;
    if (a.max_global == 0) return kOk;
    if (p.A.lse_in == nullptr) return launch_global_rows<T>(p.A, stream);
    if (a.max_global <= 8) return launch_global_small<T>(p.A, stream);   // dkg, dvg too
    const size_t mg = size_t(a.max_global), bh = size_t(a.B) * a.H;
    if (cudaMemsetAsync(p.A.dqg_acc, 0, sizeof(float) * bh * mg * kDHead, stream) != cudaSuccess)
        return kErrCuda;
    const int rc = launch_side<T, kGRowsMode>(p, stream);
    if (rc != kOk) return rc;
    return launch_global_final<T>(p.A, stream);
}

// dkg, dvg on the tensor cores for more than 8 global tokens; the CUDA-core
// kernel (zeros without global tokens) below that, where one 64-row tile of
// a few real rows per item costs more than it saves.
template <typename T>
int launch_global_keys_tc(const Params &p, cudaStream_t stream)
{
    const int mg = p.A.a.max_global;
    if (mg > 0 && mg <= 8 && p.A.lse_in) return kOk;    // done by launch_global_small
    if (mg <= 8) return launch_global_keys<T>(p.A, sizeof(T), stream);
    return launch_side<T, kGKeysMode>(p, stream);
}

template <typename T>
int launch_typed(const BwdArgs &A, CUtensorMapDataType dt, cudaStream_t stream)
{
    const AttnArgs &a = A.a;
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.A = A;
    const int BH = a.B * a.H;
    // Residue maps of every distinct dilation; heads beyond the budget send
    // the whole call to the CUDA-core path (nothing launched yet).
    for (int h = 0; h < a.H; ++h) p.res_base[h] = -1;
    int n_res = 0;
    for (int h = 0; h < a.H; ++h) {
        if (p.res_base[h] >= 0) continue;
        const int dil = a.dil[h];
        const int nres = std::min(dil, a.n);
        if (n_res + nres > kMaxResidues) return kErrUnsupported;
        for (int h2 = h; h2 < a.H; ++h2)
            if (a.dil[h2] == dil) p.res_base[h2] = n_res;
        n_res += nres;
    }
    const void *src[4] = {a.q, a.k, a.v, A.dout};
    for (int h = 0; h < a.H; ++h) {
        bool seen = false;                  // an earlier head has this dilation
        for (int h2 = 0; h2 < h; ++h2) seen = seen || a.dil[h2] == a.dil[h];
        if (seen) continue;
        const int dil = a.dil[h];
        for (int r = 0; r < std::min(dil, a.n); ++r)
            for (int tsr = 0; tsr < 4; ++tsr)
                if (!cached(&p.res[tsr][p.res_base[h] + r], src[tsr], dt, a.n, BH, true, dil, r))
                    return kErrCuda;
    }
    if (!cached(&p.krow, a.k, dt, a.n, BH, false) || !cached(&p.vrow, a.v, dt, a.n, BH, false))
        return kErrCuda;
    if (a.max_global > 0 &&
        (!cached(&p.kgt, a.kg, dt, a.n, BH, true) || !cached(&p.vgt, a.vg, dt, a.n, BH, true) ||
         !cached(&p.qgrow, a.qg, dt, a.n, BH, false) ||
         !cached(&p.dorow, A.dout, dt, a.n, BH, false) ||
         !cached(&p.qt, a.q, dt, a.n, BH, true) || !cached(&p.dot, A.dout, dt, a.n, BH, true)))
        return kErrCuda;
    p.oob_row = BH * a.n;
    return backward_schedule<T>(
        A, sizeof(T), stream, [&](cudaStream_t st) { return launch_side<T, kRowsMode>(p, st); },
        [&](cudaStream_t st) { return launch_side<T, kKeysMode>(p, st); },
        [&](cudaStream_t st) { return launch_global_rows_tc<T>(p, st); },
        [&](cudaStream_t st) { return launch_global_cols_tc<T>(p, st); },
        [&](cudaStream_t st) { return launch_global_keys_tc<T>(p, st); }, A.lse_in != nullptr);
}

}  // namespace bwdtc

int launch_backward_tc(lf_dtype dtype, const BwdArgs &A, cudaStream_t stream)
{
    using namespace bwdtc;
    if (dtype == LF_BF16)
        return launch_typed<__nv_bfloat16>(A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, stream);
    if (dtype == LF_F16) return launch_typed<__half>(A, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, stream);
    return kErrUnsupported;
}

}  // namespace lf
