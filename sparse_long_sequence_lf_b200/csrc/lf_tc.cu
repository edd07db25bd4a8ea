// Tensor-core (tcgen05) attention kernel for bf16 / fp16 inputs on sm_100a.
//
// What it computes ("LongFormer: The Long-Document Transformer" notes,
// "Sliding Window", "Dilated Sliding Window", "Global Attention"; the notes
// say the costly part is QK^T and that Longformer only computes a fixed
// number of its diagonals with a banded product; FasterTransformer Longformer
// Encoder guide, "compute flow": local rows softmax over window + global
// tokens, global rows over the whole sequence, masked rows zeroed):
//
//   band items    128 query rows of one (batch, head, residue class of the
//                 head's dilation).  A dilated head is a plain band over each
//                 residue subsequence x[r::dil], so the same tile loop serves
//                 every dilation.  The keys stream as 64-key tiles over the
//                 band's diagonals, then as tiles of the (deduplicated) global
//                 tokens; an online softmax runs over all of them.
//   global items  up to 128 global rows of one (batch, head) against one
//                 512-key chunk of Kg/Vg; each writes fp32 partials (max, sum,
//                 unnormalised output).  While a row spans at most 8 chunks,
//                 the warp that finishes the last chunk of a group of 32 rows
//                 merges them by log-sum-exp into the output rows; beyond
//                 that combine_kernel does, after this kernel.
//
// Layout of one CTA (384 threads, one CTA per SM, persistent over items):
//   warps 0-3   softmax warpgroup of lane 0   (one thread per query row)
//   warps 4-7   softmax warpgroup of lane 1
//   warps 8-9   TMA producers of lanes 0 and 1
//   warps 10-11 MMA issuers of lanes 0 and 1 (warp 10 also owns TMEM)
// The two lanes are independent item streams sharing the SM's tensor core,
// SFU and FMA pipes.
//
// TMEM (512 columns; lane X uses [192X, 192X+192)): two 64-key score
// buffers S0, S1 (fp32, overwritten in place by the 16-bit probabilities P in
// their first 32 columns) and the 64-column output accumulator O.  While the
// softmax works on S(j), the tensor core already computes S(j+1) into the
// other buffer.
//   S = Q K^T      tcgen05.mma kind::f16, A = Q (smem, K-major),
//                  B = K tile (smem, K-major), 128x64 fp32 in TMEM
//   O += P V       tcgen05.mma kind::f16, A = P (TMEM), B = V tile
//                  (smem, MN-major), 128x64 fp32 in TMEM
// Shared-memory tiles have 128-byte rows with the 128-byte swizzle, written
// by TMA: whole tiles from residue-class tensor maps (rows r, r+dil, ...),
// single-row loads for global tokens, gathered Qg rows and heads beyond the
// residue-map budget.  Q is double-buffered per lane, K/V run through a
// 3-stage ring of 64-key tiles per lane.  Every wait on an mbarrier is
// bounded; on expiry the kernel records LF_ERR_DEVICE_TIMEOUT, drains its own
// copies and MMAs, frees its TMEM and returns.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cudaTypedefs.h>

#include "../../include/lf_attention.h"
#include "lf_sm100.cuh"

namespace lf {

using namespace sm100;

constexpr int kRows = 128;                        // query rows per tile (M)
constexpr int kKeys = 64;                         // keys per S tile / K-V stage
constexpr int kStages = 3;                        // K/V ring depth per lane
constexpr int kLanes = 2;
constexpr int kQBytes = kRows * kDHead * 2;       // 16 KB of 16-bit elements
constexpr int kKvBytes = kKeys * kDHead * 2;      // 8 KB
constexpr int kRowBytes = kDHead * 2;             // 128 B
constexpr int kThreads = 384;                     // 3 warpgroups
constexpr int kWarpProducer = 8;                  // warps 8, 9: TMA producers of lanes 0, 1
constexpr int kWarpMma = 10;                      // warps 10, 11: MMA issuers of lanes 0, 1
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemLaneCols = 192;           // S0 (64) | S1 (64) | O (64) per lane
constexpr float kRescaleLog2 = 8.f;               // lazy rescale: P stays below 2^8
// Register split: the softmax warpgroups take registers from the producer /
// MMA warpgroup.  The launch must hold at least kRegsNeeded registers
// (checked on the host against the compiled register count).
constexpr int kRegsSoftmax = 176;
constexpr int kRegsControl = 144;
constexpr int kRegsNeeded = 2 * 128 * kRegsSoftmax + 128 * kRegsControl;
// Of every 8 column pairs of a score tile, the pairs whose bit is set here
// take 2^x from a cubic on the FMA pipe, the others from the SFU; the two
// units then share the exponentials.
constexpr uint32_t kPolyPairs = 0x49u;            // pairs 0, 3, 6 of each 8

enum MapId { kMapKgTile, kMapVgTile, kMapQRow, kMapKRow, kMapVRow, kMapQgRow, kMapCount };

// Residue-class tensor maps: for a head with dilation d, the rows r, r+d,
// r+2d, ... of each (batch, head) slice form a plain sequence (row stride
// d*128 B, first row r), so whole tiles of a dilated window load with one TMA
// copy.  Up to kMaxResidues (dilation, residue) pairs per call; heads beyond
// that load their rows one by one.
constexpr int kMaxResidues = 24;
constexpr int kMergeInKernelChunks = 8;           // longest sequence merged in-kernel: 4096

struct TcParams {
    CUtensorMap maps[kMapCount];              // first: 64-byte aligned
    CUtensorMap res_q[kMaxResidues];          // Q tiles of 128 rows
    CUtensorMap res_k[kMaxResidues];          // K tiles of 64 rows
    CUtensorMap res_v[kMaxResidues];          // V tiles of 64 rows
    AttnArgs a;
    int res_base[kMaxHeads];  // residue map of (head h, residue 0); -1: load rows one by one
    int global_items;     // B*H*gtiles*nchunks, ordered before the band items
    int total_items;
    int gtiles;           // ceil(max_global / 128)
    int oob_row;          // a row coordinate past the end of the row maps (reads zeros)
    int n_res;            // residue maps in use
    int merge_in_kernel;  // global rows merged by the last chunk (else by combine_kernel)
};

// Kernel arguments above 4 KB need CUDA 12.1 or newer (up to 32764 bytes).
static_assert(sizeof(TcParams) <= 32000, "kernel arguments exceed the parameter space");

struct __align__(1024) TcSmem {
    uint8_t q[kLanes][2][kQBytes];
    uint8_t k[kLanes][kStages][kKvBytes];
    uint8_t v[kLanes][kStages][kKvBytes];
    uint64_t q_full[kLanes][2], q_empty[kLanes][2];
    uint64_t kv_full[kLanes][kStages], kv_empty[kLanes][kStages];
    uint64_t s_full[kLanes][2], p_full[kLanes][2], pv_done[kLanes][2];
    uint64_t o_free[kLanes];
    uint64_t drain[kLanes];
    uint32_t tmem_base;
    int abort_flag;
};

// ------------------------------------------------------------- item walk
struct Geom {
    int ntiles;     // 0: nothing to do
    int kind;       // 1 band, 2 global rows
    int b, h, bh, dil, r, n_r;
    int q0;         // band: first residue-space row; global: first global slot
    int klo;        // first key of tile 0 (residue space for band items)
    int nkv;        // key tiles before the global-column tiles
    int key_end;    // global items: end of the key chunk
    int g;          // global tokens of the batch (clamped to max_global)
    int chunk, gtile;
    int has_pad;
};

__device__ __forceinline__ Geom decode_item(const TcParams &p, int item)
{
    const AttnArgs &a = p.a;
    Geom G;
    if (item < p.global_items) {
        const int per_bh = p.gtiles * a.L.nchunks;
        G.bh = item / per_bh;
        const int rem = item - G.bh * per_bh;
        G.gtile = rem / a.L.nchunks;
        G.chunk = rem - G.gtile * a.L.nchunks;
        G.b = G.bh / a.H;
        G.h = G.bh - G.b * a.H;
        G.kind = 2;
        G.dil = 1;
        G.r = 0;
        G.n_r = a.n;
        G.g = min(a.ws.counts[G.b], a.max_global);
        G.q0 = G.gtile * kRows;
        G.klo = G.chunk * kChunkKeys;
        G.key_end = min(a.n, G.klo + kChunkKeys);
        G.nkv = (G.key_end - G.klo + kKeys - 1) / kKeys;
        G.ntiles = (G.g > G.q0) ? G.nkv : 0;
    } else {
        int tile;
        band_item(a, item - p.global_items, G.b, G.h, G.r, tile);
        G.kind = 1;
        G.bh = G.b * a.H + G.h;
        G.dil = a.dil[G.h];
        G.n_r = (a.n - G.r + G.dil - 1) / G.dil;
        G.q0 = tile * kRows;
        const int rows_hi = min(G.q0 + kRows - 1, G.n_r - 1);
        const int lo = max(G.q0 - (a.causal ? a.window - 1 : a.half), 0);
        const int hi = min(rows_hi + (a.causal ? 0 : a.half), G.n_r - 1);
        G.klo = lo;
        G.nkv = (hi - lo + kKeys) / kKeys;
        G.key_end = 0;
        G.g = min(a.ws.counts[G.b], a.max_global);
        G.chunk = G.gtile = 0;
        G.ntiles = G.nkv + (G.g + kKeys - 1) / kKeys;
    }
    G.has_pad = a.ws.flags[G.b] & kFlagHasPadding;
    return G;
}

// Walks the 64-key tiles of the items of one lane: items lane, lane + stride,
// ...  `j` counts the lane's tiles and `k` its items (both from 0); they pick
// the double buffers and the barrier parities.
struct Cursor {
    int item, stride, total;
    int t, j, k;
    Geom G;
    bool valid;

    __device__ __forceinline__ void seek(const TcParams &p)
    {
        while (item < total) {
            G = decode_item(p, item);
            if (G.ntiles > 0) {
                t = 0;
                valid = true;
                return;
            }
            item += stride;
        }
        valid = false;
    }
    __device__ __forceinline__ void init(const TcParams &p, int first, int stride_)
    {
        item = first;
        stride = stride_;
        total = p.total_items;
        j = 0;
        k = 0;
        seek(p);
    }
    __device__ __forceinline__ void advance(const TcParams &p)
    {
        ++j;
        if (++t < G.ntiles) return;
        ++k;
        item += stride;
        seek(p);
    }
    __device__ __forceinline__ bool first() const { return t == 0; }
    __device__ __forceinline__ bool last() const { return t == G.ntiles - 1; }
    __device__ __forceinline__ bool is_global_col_tile() const { return G.kind == 1 && t >= G.nkv; }
    // Keys in this tile (N of QK^T, K of PV): 64, or the global tokens of a
    // global-column tile rounded up to a multiple of 16.
    __device__ __forceinline__ int tile_n() const
    {
        if (!is_global_col_tile()) return kKeys;
        const int left = min(kKeys, G.g - (t - G.nkv) * kKeys);
        return (left + 15) & ~15;
    }
    __device__ __forceinline__ int k0() const { return G.klo + t * kKeys; }
    __device__ __forceinline__ int slot0() const { return (t - G.nkv) * kKeys; }
};

// ------------------------------------------------------------ roles
// Bounded wait taken by a whole warp: either every lane goes on or every lane
// gives up, so no warp-collective instruction runs with a partial warp.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int *status)
{
    const bool ok = mbar_wait(bar, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void advance_ring(int &stage, uint32_t &phase)
{
    if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
    }
}

// Waits (bounded, ignoring the abort flag) for a copy this CTA started, so
// that nothing lands in shared memory after the CTA has exited.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
}

// TMA producer of one lane: Q (double-buffered) and the 64-key K/V ring.
__device__ __forceinline__ void producer_role(const TcParams &p, TcSmem &sm, int X, int lane)
{
    const AttnArgs &a = p.a;
    Cursor cur;
    cur.init(p, blockIdx.x * kLanes + X, gridDim.x * kLanes);
    int stage = 0;
    uint32_t phase = 0;
    bool armed[kStages] = {};
    uint32_t armed_phase[kStages] = {};
    bool q_armed[2] = {false, false};
    uint32_t q_armed_phase[2] = {0u, 0u};
    const int n = a.n;
    bool ok = true;

    while (cur.valid && ok) {
        const Geom &G = cur.G;
        if (cur.first()) {
            const int qb = cur.k & 1;
            const uint32_t use = uint32_t(cur.k >> 1);
            if (!warp_wait(&sm.q_empty[X][qb], (use & 1u) ^ 1u, &sm.abort_flag, a.ws.status)) {
                ok = false;
                break;
            }
            uint8_t *qd = sm.q[X][qb];
            uint64_t *qbar = &sm.q_full[X][qb];
            const int rb = G.kind == 1 ? p.res_base[G.h] : -1;
            if (rb >= 0) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(qbar, kQBytes);
                    tma_load_3d(qd, &p.res_q[rb + G.r], qbar, 0, G.q0, G.bh);
                }
            } else if (G.kind == 1) {
                if (lane == 0) mbar_arrive_expect_tx(qbar, kQBytes);
                __syncwarp();
                for (int rr = lane; rr < kRows; rr += 32) {
                    const int ir = G.q0 + rr;
                    const int y = ir < G.n_r ? G.bh * n + ir * G.dil + G.r : p.oob_row;
                    tma_load_2d(qd + rr * kRowBytes, &p.maps[kMapQRow], qbar, 0, y);
                }
            } else {
                // Only the rows of real global tokens: a query row only feeds
                // its own output row, and rows past the count are never stored.
                const int rows = min(kRows, G.g - G.q0);
                if (lane == 0) mbar_arrive_expect_tx(qbar, rows * kRowBytes);
                __syncwarp();
                for (int rr = lane; rr < rows; rr += 32) {
                    const int y = G.bh * n + a.ws.gidx[size_t(G.b) * n + G.q0 + rr];
                    tma_load_2d(qd + rr * kRowBytes, &p.maps[kMapQgRow], qbar, 0, y);
                }
            }
            q_armed[qb] = true;
            q_armed_phase[qb] = use & 1u;
        }
        if (!warp_wait(&sm.kv_empty[X][stage], phase ^ 1u, &sm.abort_flag, a.ws.status)) {
            ok = false;
            break;
        }
        uint8_t *kd = sm.k[X][stage];
        uint8_t *vd = sm.v[X][stage];
        uint64_t *bar = &sm.kv_full[X][stage];
        const int rb = G.kind == 1 ? p.res_base[G.h] : -1;
        if (G.kind == 2 || (!cur.is_global_col_tile() && rb >= 0)) {
            const CUtensorMap *km = G.kind == 2 ? &p.maps[kMapKgTile] : &p.res_k[rb + G.r];
            const CUtensorMap *vm = G.kind == 2 ? &p.maps[kMapVgTile] : &p.res_v[rb + G.r];
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, 2 * kKvBytes);
                tma_load_3d(kd, km, bar, 0, cur.k0(), G.bh);
                tma_load_3d(vd, vm, bar, 0, cur.k0(), G.bh);
            }
        } else {
            const bool gcol = cur.is_global_col_tile();
            const int rows = gcol ? cur.tile_n() : kKeys;
            if (lane == 0) mbar_arrive_expect_tx(bar, 2 * rows * kRowBytes);
            __syncwarp();
            for (int rr = lane; rr < rows; rr += 32) {
                int y = p.oob_row;
                if (gcol) {
                    const int slot = cur.slot0() + rr;
                    if (slot < G.g) y = G.bh * n + a.ws.gidx[size_t(G.b) * n + slot];
                } else {
                    const int jr = cur.k0() + rr;
                    if (jr < G.n_r) y = G.bh * n + jr * G.dil + G.r;
                }
                tma_load_2d(kd + rr * kRowBytes, &p.maps[kMapKRow], bar, 0, y);
                tma_load_2d(vd + rr * kRowBytes, &p.maps[kMapVRow], bar, 0, y);
            }
        }
        armed[stage] = true;
        armed_phase[stage] = phase;
        advance_ring(stage, phase);
        cur.advance(p);
    }
    if (!ok || sm.abort_flag) {
        for (int s = 0; s < kStages; ++s)
            if (armed[s]) drain_wait(&sm.kv_full[X][s], armed_phase[s]);
        for (int b = 0; b < 2; ++b)
            if (q_armed[b]) drain_wait(&sm.q_full[X][b], q_armed_phase[b]);
    }
}

struct TileInfo {
    int stage, n, j, k;
    bool first, last;
};

// MMA issuer of one lane.  Order: S(0); then for every tile j:
// S(j+1) into the other S buffer (look-ahead), then PV(j) once P(j) is ready.
// S(j+2) reuses the buffer of P(j) and is issued after PV(j), and the tensor
// pipe executes in issue order.
__device__ __forceinline__ void mma_role(const TcParams &p, TcSmem &sm, uint32_t tmem, int X,
                                         bool bf16)
{
    const AttnArgs &a = p.a;
    const uint32_t id_s = make_idesc(128, 0, bf16, false);
    const uint32_t id_pv = make_idesc(128, 64, bf16, true);
    const uint32_t tbase = tmem + X * kTmemLaneCols;
    const uint32_t tO = tbase + 128;
    Cursor cur;
    cur.init(p, blockIdx.x * kLanes + X, gridDim.x * kLanes);
    int stage = 0;
    uint32_t phase = 0;

    // Issues S(j) for the tile under the cursor; returns false on abort.
    auto issue_s = [&](TileInfo &info) -> bool {
        if (cur.first()) {
            const uint32_t use = uint32_t(cur.k >> 1);
            if (!warp_wait(&sm.q_full[X][cur.k & 1], use & 1u, &sm.abort_flag, a.ws.status))
                return false;
        }
        if (!warp_wait(&sm.kv_full[X][stage], phase, &sm.abort_flag, a.ws.status)) return false;
        tc_fence_after();
        const int N = cur.tile_n();
        const uint32_t tS = tbase + (cur.j & 1) * 64;
        const uint64_t qdesc = make_sdesc(smem_u32(sm.q[X][cur.k & 1]), 16, 1024);
        const uint64_t kdesc = make_sdesc(smem_u32(sm.k[X][stage]), 16, 1024);
        const uint32_t idesc = id_s | (uint32_t(N >> 3) << 17);
#pragma unroll
        for (int kk = 0; kk < kDHead / 16; ++kk)
            mma_ss_elect(tS, qdesc + uint64_t((kk * 32) >> 4), kdesc + uint64_t((kk * 32) >> 4),
                         idesc, kk > 0 ? 1u : 0u);
        tc_commit_elect(&sm.s_full[X][cur.j & 1]);
        if (cur.last()) tc_commit_elect(&sm.q_empty[X][cur.k & 1]);
        __syncwarp();
        info.stage = stage;
        info.n = N;
        info.j = cur.j;
        info.k = cur.k;
        info.first = cur.first();
        info.last = cur.last();
        advance_ring(stage, phase);
        cur.advance(p);
        return true;
    };

    if (!cur.valid) return;
    TileInfo pend;
    if (!issue_s(pend)) return;
    for (;;) {
        TileInfo next;
        const bool have_next = cur.valid;
        if (have_next && !issue_s(next)) return;
        // PV of the pending tile.
        const int b = pend.j & 1;
        if (!warp_wait(&sm.p_full[X][b], uint32_t(pend.j >> 1) & 1u, &sm.abort_flag, a.ws.status))
            return;
        if (pend.first && pend.k > 0) {
            if (!warp_wait(&sm.o_free[X], uint32_t(pend.k - 1) & 1u, &sm.abort_flag, a.ws.status))
                return;
        }
        tc_fence_after();
        {
            const uint32_t tP = tbase + b * 64;
            const uint64_t vdesc = make_sdesc(smem_u32(sm.v[X][pend.stage]), 16, 1024);
            const int ksteps = pend.n >> 4;
            for (int kk = 0; kk < ksteps; ++kk)
                mma_ts_elect(tO, tP + kk * 8, vdesc + uint64_t((kk * 2048) >> 4), id_pv,
                             (kk > 0 || !pend.first) ? 1u : 0u);
            tc_commit_elect(&sm.kv_empty[X][pend.stage]);
            tc_commit_elect(&sm.pv_done[X][b]);
        }
        __syncwarp();
        if (!have_next) break;
        pend = next;
    }
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

// Bits of the 64 key columns of a tile that hold real, unpadded keys, built
// by each warp on its own (2 lookups per lane and 2 ballots).  For a
// global-column tile also the token position of column 32w + lane (jpos[w])
// and the columns whose token lies in the row's residue class (res[w]): a
// window tap of row i = ir*dil + r always does.
__device__ __forceinline__ void column_bits(const AttnArgs &a, const Cursor &cur, int lane,
                                            uint32_t (&bits)[2], int (&jpos)[2],
                                            uint32_t (&res)[2])
{
    const Geom &G = cur.G;
    const uint32_t *vb = a.ws.vbits + size_t(G.b) * a.L.nwords;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const int c = w * 32 + lane;
        bool ok;
        if (cur.is_global_col_tile()) {
            const int slot = cur.slot0() + c;
            const int j = slot < G.g ? a.ws.gidx[size_t(G.b) * a.n + slot] : -1;
            ok = j >= 0 && bit_at(vb, j);
            jpos[w] = j;
            res[w] = __ballot_sync(0xffffffffu, ok && (j % G.dil) == G.r);
        } else if (G.kind == 2) {
            const int j = cur.k0() + c;
            ok = j < G.key_end && bit_at(vb, j);
        } else {
            const int jr = cur.k0() + c;
            ok = jr < G.n_r && bit_at(vb, jr * G.dil + G.r);
        }
        bits[w] = __ballot_sync(0xffffffffu, ok);
    }
}

struct RowState {
    float m, l;
};

// Bits of the columns [32q, 32q + 32) that lie inside [clo, chi].
__device__ __forceinline__ uint32_t range_bits(int q, int clo, int chi)
{
    const int lo = min(max(clo - 32 * q, 0), 32);
    const int hi = min(max(chi - 32 * q + 1, 0), 32);
    const uint32_t below_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
    const uint32_t below_lo = lo >= 32 ? 0xffffffffu : ((1u << lo) - 1u);
    return below_hi & ~below_lo;
}

// Maximum of 32 values as a shallow tree of 3-input maxima.
__device__ __forceinline__ float max32(const float *s)
{
    float t[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) t[i] = max3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
    t[10] = fmaxf(s[30], s[31]);
    const float u0 = max3(t[0], t[1], t[2]);
    const float u1 = max3(t[3], t[4], t[5]);
    const float u2 = max3(t[6], t[7], t[8]);
    return max3(u0, u1, max3(u2, t[9], t[10]));
}

// 2^x for a pair of arguments on the FMA pipe.  x = j + f with j = round(x)
// (the 1.5*2^23 addition rounds to an integer in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f is a cubic fitted to minimise the maximum relative
// error on [-1/2, 1/2] (Remez exchange, error below 7.5e-5); 2^j is added to
// the exponent field.  Arguments below -126 are clamped (the result is then
// at most 2^-126, which is zero for every use here).
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float &y0, float &y1)
{
    constexpr float kRound = 12582912.f;     // 1.5 * 2^23
    constexpr float c0 = 0.999928074f, c1 = 0.693260985f, c2 = 0.242611122f,
                    c3 = 0.0551716691f;
    x0 = fmaxf(x0, -126.f);
    x1 = fmaxf(x1, -126.f);
    float t0, t1, j0, j1, f0, f1, p0, p1;
    add2(t0, t1, x0, x1, kRound, kRound);
    add2(j0, j1, t0, t1, -kRound, -kRound);
    fma2(f0, f1, j0, j1, -1.f, -1.f, x0, x1);
    fma2(p0, p1, f0, f1, c3, c3, c2, c2);
    fma2(p0, p1, p0, p1, f0, f1, c1, c1);
    fma2(p0, p1, p0, p1, f0, f1, c0, c0);
    y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Online softmax of one 64-key score tile for this thread's row.  mw marks
// the columns that are keys of this row.  Writes P = 2^(S*scale*log2e - m)
// as 16-bit pairs over the first 32 columns of the tile and adds the row sum.
// O is rescaled in TMEM only when the running maximum grows by more than 2^8
// (after the previous PV has completed).  Returns false on abort.
template <typename T>
__device__ __forceinline__ bool softmax_tile(TcSmem &sm, const AttnArgs &a, int X, uint32_t tS,
                                             uint32_t tO, RowState &st, const Cursor &cur,
                                             const uint32_t (&mw)[2], bool need_mask, float sl2)
{
    float s[64];
    tmem_ld32(tS, *reinterpret_cast<float(*)[32]>(&s[0]));
    tmem_ld32(tS + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
    if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? s[c] : -INFINITY;
    }
    const float mt = fmaxf(max32(&s[0]), max32(&s[32])) * sl2;
    float alpha = 1.f;
    bool rescale = false;
    if (cur.first()) {
        st.m = mt;
        st.l = 0.f;
    } else if (mt > st.m + kRescaleLog2) {
        alpha = ex2(st.m - mt);
        st.m = mt;
        rescale = true;
    }
    const float nb = (st.m == -INFINITY) ? 0.f : -st.m;
    float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        float x0, x1, p0, p1;
        fma2(x0, x1, s[2 * c], s[2 * c + 1], sl2, sl2, nb, nb);
        if ((kPolyPairs >> (c & 7)) & 1u) {
            exp2_poly2(x0, x1, p0, p1);
        } else {
            p0 = ex2(x0);
            p1 = ex2(x1);
        }
        if (c & 1)
            add2(sb0, sb1, sb0, sb1, p0, p1);
        else
            add2(sa0, sa1, sa0, sa1, p0, p1);
        pk[c] = pack2<T>(p0, p1);
    }
    if (__any_sync(0xffffffffu, rescale)) {
        // O must hold every PV before this tile: the previous one may still run.
        const int jp = cur.j - 1;
        if (!warp_wait(&sm.pv_done[X][jp & 1], uint32_t(jp >> 1) & 1u, &sm.abort_flag,
                       a.ws.status))
            return false;
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float o[32];
            tmem_ld32(tO + half * 32, o);
            uint32_t ob[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) ob[x] = __float_as_uint(o[x] * alpha);
            tmem_st32(tO + half * 32, ob);
        }
    }
    tmem_st32(tS, pk);
    st.l = st.l * alpha + ((sa0 + sa1) + (sb0 + sb1));
    tmem_st_wait();
    return true;
}

template <typename T>
__device__ __forceinline__ void store_half_row(T *dst, const float (&o)[32], float inv)
{
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack2<T>(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
        v.y = pack2<T>(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
        v.z = pack2<T>(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
        v.w = pack2<T>(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
        d4[q] = v;
    }
}

template <typename T>
__device__ __forceinline__ void store_row(T *dst, const float (&o)[64], float inv)
{
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint4 v;
        v.x = pack2<T>(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
        v.y = pack2<T>(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
        v.z = pack2<T>(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
        v.w = pack2<T>(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
        d4[q] = v;
    }
}

// Merges the chunk partials of the global rows slot0 .. slot0 + 31 (lane =
// row) by log-sum-exp and writes their output rows.  Called by the warp that
// wrote the last chunk of the group; the partials of the other chunks come
// from other CTAs, so they are read past L1.
template <typename T>
__device__ __noinline__ void merge_global_rows(const AttnArgs &a, int b, int bh, int g, int slot0,
                                               int lane)
{
    const int slot = slot0 + lane;
    if (slot >= g) return;
    const int pos = a.ws.gidx[size_t(b) * a.n + slot];
    if (!bit_at(a.ws.vbits + size_t(b) * a.L.nwords, pos)) return;   // padded: zeros elsewhere
    const size_t mg = size_t(a.max_global);
    const size_t cstride = kPartialFloats * mg;
    const float *P = partial_base(a, bh, 0) + slot;
    const int nch = a.L.nchunks;
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(P + c * cstride));
    float L = 0.f, acc[kDHead];
#pragma unroll
    for (int x = 0; x < kDHead; ++x) acc[x] = 0.f;
    for (int c = 0; c < nch; ++c) {
        const float *pc = P + c * cstride;
        const float mc = __ldcg(pc);
        const float f = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
        L = fmaf(f, __ldcg(pc + mg), L);
#pragma unroll
        for (int x = 0; x < kDHead; ++x) acc[x] = fmaf(f, __ldcg(pc + (2 + x) * mg), acc[x]);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    store_row<T>(static_cast<T *>(a.out) + (size_t(bh) * a.n + pos) * kDHead, acc, inv);
}

template <typename T>
__device__ __forceinline__ void softmax_role(const TcParams &p, TcSmem &sm, uint32_t tmem, int X,
                                             int tid)
{
    const AttnArgs &a = p.a;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const uint32_t tbase = tmem + lane_off + X * kTmemLaneCols;
    const uint32_t tO = tbase + 128;
    const float sl2 = a.scale_log2;
    Cursor cur;
    cur.init(p, blockIdx.x * kLanes + X, gridDim.x * kLanes);
    RowState st{-INFINITY, 0.f};

    while (cur.valid) {
        const Geom &G = cur.G;
        if (cur.first() && tid == 0 && a.ws.counts[G.b] > a.max_global)
            set_status(a.ws.status, kErrGlobalOverflow);
        const int row = G.q0 + tid;     // residue-space row (band) or global slot
        const int bsel = cur.j & 1;
        const uint32_t tS = tbase + bsel * 64;
        const bool gcol = cur.is_global_col_tile();
        uint32_t cbits[2] = {~0u, ~0u}, res[2] = {0u, 0u};
        int jpos[2] = {-1, -1};
        if (gcol || G.has_pad) column_bits(a, cur, lane, cbits, jpos, res);
        uint32_t mw[2];
        bool need_mask;
        if (gcol) {
            // Global-token columns: real, unpadded tokens that are not already
            // window taps of this row.  A tap shares the row's residue class
            // and lies within the (dilated) window span.
            const int i = row * G.dil + G.r;
            const int span_lo = a.causal ? (a.window - 1) * G.dil : a.half * G.dil;
            const int span_hi = a.causal ? 0 : a.half * G.dil;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                uint32_t m = cbits[w];
                uint32_t rest = res[w];
                while (rest) {
                    const int c = __ffs(rest) - 1;
                    rest &= rest - 1u;
                    const int d = __shfl_sync(0xffffffffu, jpos[w], c) - i;
                    if (d >= -span_lo && d <= span_hi) m &= ~(1u << c);
                }
                mw[w] = m;
            }
            need_mask = true;
        } else {
            int clo, chi;
            const int k0 = cur.k0();
            if (G.kind == 2) {
                clo = 0;
                chi = min(kKeys - 1, G.key_end - 1 - k0);
            } else {
                const int lo = max(row - (a.causal ? a.window - 1 : a.half), 0);
                const int hi = min(row + (a.causal ? 0 : a.half), G.n_r - 1);
                clo = lo - k0;
                chi = hi - k0;
            }
            mw[0] = range_bits(0, clo, chi) & cbits[0];
            mw[1] = range_bits(1, clo, chi) & cbits[1];
            need_mask = __any_sync(0xffffffffu, (mw[0] & mw[1]) != 0xffffffffu);
        }

        if (!warp_wait(&sm.s_full[X][bsel], uint32_t(cur.j >> 1) & 1u, &sm.abort_flag,
                       a.ws.status))
            return;
        tc_fence_after();
        if (!softmax_tile<T>(sm, a, X, tS, tO, st, cur, mw, need_mask, sl2)) return;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[X][bsel]);

        if (cur.last()) {
            if (!warp_wait(&sm.pv_done[X][bsel], uint32_t(cur.j >> 1) & 1u, &sm.abort_flag,
                           a.ws.status))
                return;
            tc_fence_after();
            if (G.kind == 1) {
                const bool row_in = row < G.n_r;
                const int i = row * G.dil + G.r;
                const uint32_t *vb = a.ws.vbits + size_t(G.b) * a.L.nwords;
                const uint32_t *gb = a.ws.gbits + size_t(G.b) * a.L.nwords;
                const bool valid = row_in && bit_at(vb, i);
                const bool write = row_in && (!valid || !bit_at(gb, i));
                T *dst = static_cast<T *>(a.out) + (size_t(G.bh) * a.n + (row_in ? i : 0)) * kDHead;
                // A padded row is written as zeros (inv = 0).
                const float inv = valid ? 1.f / st.l : 0.f;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tmem_ld32(tO + half * 32, o);
                    if (write) store_half_row<T>(dst + half * 32, o, inv);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.o_free[X]);
            } else {
                const int slot = row;
                const size_t mg = size_t(a.max_global);
                float *P = a.ws.partials +
                           (size_t(G.bh) * a.L.nchunks + G.chunk) * kPartialFloats * mg +
                           min(slot, a.max_global - 1);
                const bool write = slot < G.g;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tmem_ld32(tO + half * 32, o);
                    if (write) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) P[(2 + half * 32 + x) * mg] = o[x];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.o_free[X]);
                if (write) {
                    P[0] = st.m;
                    P[mg] = st.l;
                }
                // The last chunk to finish this warp's group of 32 global rows
                // merges them and resets the group's arrival counter for the
                // next call on the same workspace.
                const int group = (G.q0 >> 5) + warp;
                if (p.merge_in_kernel && group * 32 < G.g) {
                    __threadfence();
                    __syncwarp();
                    int last = 0;
                    if (lane == 0) {
                        int *ctr = a.ws.counters + size_t(G.bh) * (a.L.ngroups + 1) + group;
                        last = atomicAdd(ctr, 1) == a.L.nchunks - 1;
                        if (last) atomicExch(ctr, 0);
                    }
                    if (__shfl_sync(0xffffffffu, last, 0)) {
                        __threadfence();
                        merge_global_rows<T>(a, G.b, G.bh, G.g, group * 32, lane);
                    }
                }
            }
        }
        cur.advance(p);
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    TcSmem &sm = *reinterpret_cast<TcSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int X = 0; X < kLanes; ++X) {
            for (int b = 0; b < 2; ++b) {
                mbar_init(&sm.q_full[X][b], 1);
                mbar_init(&sm.q_empty[X][b], 1);
                mbar_init(&sm.s_full[X][b], 1);
                mbar_init(&sm.p_full[X][b], 4);     // one arrival per softmax warp
                mbar_init(&sm.pv_done[X][b], 1);
            }
            for (int s = 0; s < kStages; ++s) {
                mbar_init(&sm.kv_full[X][s], 1);
                mbar_init(&sm.kv_empty[X][s], 1);
            }
            mbar_init(&sm.o_free[X], 4);
            mbar_init(&sm.drain[X], 1);
        }
        sm.abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kWarpProducer && lane == 0)
    {
        for (int m = 0; m < kMapCount; ++m) tma_prefetch_map(&p.maps[m]);
        for (int m = 0; m < p.n_res; ++m) {
            tma_prefetch_map(&p.res_q[m]);
            tma_prefetch_map(&p.res_k[m]);
            tma_prefetch_map(&p.res_v[m]);
        }
    }
    if (warp == kWarpMma) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // Everything above overlaps the previous kernel in the stream; the
    // workspace it writes (compacted indices, bitmaps) is read only below.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        softmax_role<T>(p, sm, tmem, warp >> 2, threadIdx.x & 127);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
        if (warp < kWarpMma) {
            producer_role(p, sm, warp - kWarpProducer, lane);
        } else {
            const int X = warp - kWarpMma;
            mma_role(p, sm, tmem, X, std::is_same<T, __nv_bfloat16>::value);
            // Every MMA this warp issued has completed once this commit lands.
            tc_commit_elect(&sm.drain[X]);
            __syncwarp();
            drain_wait(&sm.drain[X], 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merges the chunk partials of every global row into its output row: one
// warp per (batch*head, global slot); lane l handles dimensions 2l, 2l+1.
// Launched after the attention kernel (programmatic dependent launch: its
// prologue overlaps the attention kernel's tail, the wait below orders it).
template <typename T>
__global__ void __launch_bounds__(128) combine_kernel(const AttnArgs a)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int bh = blockIdx.x;
    const int slot = blockIdx.y * 4 + (threadIdx.x >> 5);
    const int b = bh / a.H;
    const int g = min(a.ws.counts[b], a.max_global);
    if (slot >= g) return;
    const int pos = a.ws.gidx[size_t(b) * a.n + slot];
    if (!bit_at(a.ws.vbits + size_t(b) * a.L.nwords, pos)) return;   // padded: zeros elsewhere
    const int nch = a.L.nchunks;
    const size_t mg = size_t(a.max_global);
    const size_t cstride = kPartialFloats * mg;
    const float *P = partial_base(a, bh, 0) + slot;
    float M = -INFINITY;
    for (int c = lane; c < nch; c += 32) M = fmaxf(M, P[c * cstride]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll 4
    for (int c = 0; c < nch; ++c) {
        const float *pc = P + c * cstride;
        const float mc = pc[0];
        const float f = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
        L = fmaf(f, pc[mg], L);
        a0 = fmaf(f, pc[(2 + 2 * lane) * mg], a0);
        a1 = fmaf(f, pc[(3 + 2 * lane) * mg], a1);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    T *dst = static_cast<T *>(a.out) + (size_t(bh) * a.n + pos) * kDHead;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        reinterpret_cast<__nv_bfloat162 *>(dst)[lane] = __floats2bfloat162_rn(a0 * inv, a1 * inv);
    } else {
        reinterpret_cast<__half2 *>(dst)[lane] = __floats2half2_rn(a0 * inv, a1 * inv);
    }
}

// ------------------------------------------------------------------ host
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encoder()
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

// Whole tiles of box_rows rows of the residue class r of dilation dil of each
// (batch*head) slice: rows r, r+dil, ... ; dims {64, ceil((n-r)/dil), B*H}.
bool encode_tile_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int n, int BH,
                     int box_rows, int dil, int r)
{
    auto enc = get_encoder();
    if (!enc) return false;
    const int n_r = (n - r + dil - 1) / dil;
    base = static_cast<const char *>(base) + size_t(r) * kRowBytes;
    cuuint64_t dims[3] = {cuuint64_t(kDHead), cuuint64_t(n_r), cuuint64_t(BH)};
    cuuint64_t strides[2] = {cuuint64_t(dil) * kRowBytes, cuuint64_t(n) * kRowBytes};
    cuuint32_t box[3] = {kDHead, cuuint32_t(box_rows), 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Single rows of the flattened tensor: dims {64, B*H*n}.
bool encode_row_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, long rows)
{
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cuuint64_t(kDHead), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(kRowBytes)};
    cuuint32_t box[2] = {kDHead, 1};
    cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

struct MapCacheEntry {
    const void *base;
    int kind, dt, n, BH, dil, r;
    CUtensorMap map;
    bool used;
};

// Encoded tensor maps, reused while the same buffer and shape come back.
// kind: 0 = tiles of 128 rows, 1 = single rows, 2 = tiles of kKeys rows.
bool cached_map(CUtensorMap *out, int kind, const void *base, CUtensorMapDataType dt, int n, int BH,
                int dil = 1, int r = 0)
{
    constexpr int kCache = 256;
    static std::mutex mu;
    static MapCacheEntry cache[kCache];
    static unsigned next = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &e : cache)
        if (e.used && e.base == base && e.kind == kind && e.dt == int(dt) && e.n == n &&
            e.BH == BH && e.dil == dil && e.r == r) {
            *out = e.map;
            return true;
        }
    CUtensorMap m;
    const bool ok = kind == 1 ? encode_row_map(&m, base, dt, long(n) * BH)
                              : encode_tile_map(&m, base, dt, n, BH, kind == 0 ? kRows : kKeys,
                                                dil, r);
    if (!ok) return false;
    MapCacheEntry &e = cache[next++ % kCache];
    e = MapCacheEntry{base, kind, int(dt), n, BH, dil, r, m, true};
    *out = m;
    return true;
}

int num_sms()
{
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 1;
}

template <typename T>
int launch_typed(const AttnArgs &a, CUtensorMapDataType dt, cudaStream_t stream)
{
    TcParams p;
    std::memset(&p, 0, sizeof(p));
    p.a = a;
    const int BH = a.B * a.H;
    bool ok = true;
    // Residue maps of every distinct dilation, while they fit.
    for (int h = 0; h < a.H; ++h) p.res_base[h] = -1;
    p.n_res = 0;
    for (int h = 0; h < a.H; ++h) {
        if (p.res_base[h] >= 0) continue;
        const int dil = a.dil[h];
        const int nres = std::min(dil, a.n);
        if (p.n_res + nres > kMaxResidues) continue;
        const int base = p.n_res;
        for (int r = 0; r < nres && ok; ++r) {
            ok = ok && cached_map(&p.res_q[base + r], 0, a.q, dt, a.n, BH, dil, r);
            ok = ok && cached_map(&p.res_k[base + r], 2, a.k, dt, a.n, BH, dil, r);
            ok = ok && cached_map(&p.res_v[base + r], 2, a.v, dt, a.n, BH, dil, r);
        }
        p.n_res += nres;
        for (int h2 = h; h2 < a.H; ++h2)
            if (a.dil[h2] == dil) p.res_base[h2] = base;
    }
    ok = ok && cached_map(&p.maps[kMapKgTile], 2, a.kg, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapVgTile], 2, a.vg, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapQRow], 1, a.q, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapKRow], 1, a.k, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapVRow], 1, a.v, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapQgRow], 1, a.qg, dt, a.n, BH);
    if (!ok) return kErrCuda;
    p.gtiles = (a.max_global + kRows - 1) / kRows;
    p.global_items = BH * p.gtiles * a.L.nchunks;
    p.total_items = p.global_items + a.B * a.band_items_per_batch;
    p.oob_row = BH * a.n;
    // One warp merges 32 global rows over every chunk: cheap for a few chunks,
    // a separate wide kernel beyond that.
    p.merge_in_kernel = a.L.nchunks <= kMergeInKernelChunks;
    const size_t smem = sizeof(TcSmem) + 1024;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(attn_tc_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess)
            return kErrCuda;
        // setmaxnreg.inc waits until the registers it asks for are free; refuse
        // to launch if the compiled register count cannot cover the split.
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, attn_tc_kernel<T>) != cudaSuccess) return kErrCuda;
        if (fa.numRegs * kThreads < kRegsNeeded) return kErrUnsupported;
        attr_set[dev] = true;
    }
    const int want = (p.total_items + kLanes - 1) / kLanes;
    const int grid = std::max(1, std::min(num_sms(), want));
    // Programmatic dependent launch: the kernel's prologue (barriers, TMEM,
    // tensor-map prefetch) overlaps the kernel before it in the stream.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attn_tc_kernel<T>, p) != cudaSuccess) return kErrCuda;
    if (a.max_global > 0 && !p.merge_in_kernel) {
        cudaLaunchConfig_t cc = {};
        cc.gridDim = dim3(a.B * a.H, (a.max_global + 3) / 4);
        cc.blockDim = dim3(128);
        cc.stream = stream;
        cc.attrs = attr;
        cc.numAttrs = 1;
        if (cudaLaunchKernelEx(&cc, combine_kernel<T>, a) != cudaSuccess) return kErrCuda;
    }
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

}  // namespace

int launch_tc(lf_dtype dtype, const AttnArgs &a, cudaStream_t stream)
{
    if (dtype == LF_BF16) return launch_typed<__nv_bfloat16>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, stream);
    return launch_typed<__half>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, stream);
}

}  // namespace lf
