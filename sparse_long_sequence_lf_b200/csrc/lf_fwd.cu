// Tensor-core (tcgen05) attention forward for bf16 / fp16 inputs on sm_100a.
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
//                 every dilation.  The keys stream as 96-key tiles over the
//                 band's diagonals, then as tiles of the (deduplicated) global
//                 tokens; an online softmax runs over all of them.
//   global items  up to 128 global rows of one (batch, head) against one
//                 512-key chunk of Kg/Vg; each writes fp32 partials (max, sum,
//                 unnormalised output).  While a row spans at most 8 chunks,
//                 the warp that finishes the last chunk of a group of 32 rows
//                 merges them by log-sum-exp into the output rows; beyond
//                 that combine_kernel does, after this kernel.
//
// Schedule.  A persistent grid, one CTA per SM.  Items are handed out by a
// device-wide atomic counter (band items first and the global items last,
// or the global items first when many global rows are merged in the kernel:
// FwdParams::global_first), so CTAs that finish early take more work; the
// first item of every slot is fixed by its CTA index.  Each CTA runs two item "slots" at once;
// their softmax warpgroups share the tensor core and the exponential units.
//
// Layout of one CTA (384 threads):
//   warps 0-3    softmax warpgroup of slot 0 (thread t owns query row t)
//   warps 4-7    softmax warpgroup of slot 1
//   warps 8, 9   TMA producers of slots 0 and 1: item records two ahead, Q,
//                K and V tiles, and each key tile's column masks (padding
//                bits, global-token positions) in shared memory
//   warps 10, 11 MMA issuers of slots 0 and 1 (lane 0 only: one thread waits
//                on the barriers and issues every MMA and commit); warp 10
//                allocates and frees the tensor memory
//
// TMEM (512 columns, slot X uses [256X, 256X+256)): two 96-column score
// buffers S0, S1 (fp32; the 16-bit probabilities P overwrite the first 48
// columns of a buffer as pairs) and a 64-column output accumulator O.
//   S = Q K^T      tcgen05.mma kind::f16, A = Q (smem, K-major),
//                  B = K tile (smem, K-major), 128x96 fp32 in TMEM
//   O += P V       tcgen05.mma kind::f16, A = P (TMEM), B = V tile
//                  (smem, MN-major), 128x64 fp32 in TMEM
// Per slot and tile the issuer puts PV(j) then S(j+2) into the buffer P(j)
// was read from, so the softmax of tile j+1 finds its scores ready.  The
// epilogue of item k (done by the softmax warps after the first tile of item
// k+1) reads O before the first PV of item k+1 overwrites it.
// Shared-memory tiles have 128-byte rows with the 128-byte swizzle, written
// by TMA: whole tiles from residue-class tensor maps (rows r, r+dil, ...),
// single-row loads for global tokens, gathered Qg rows and heads beyond the
// residue-map budget.  Each slot has two Q buffers and three K and three V
// stages.  Every wait on an mbarrier is bounded; on expiry the kernel records
// LF_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees its TMEM and
// returns.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cudaTypedefs.h>

#include "../../include/lf_attention.h"
#include "lf_sm100.cuh"

namespace lf {

using namespace sm100;

constexpr int kRows = 128;                        // query rows per tile (M)
constexpr int kTileKeys = 96;                     // keys per S tile (N) / K-V stage
constexpr int kChunks = kTileKeys / 32;           // 32-key chunks of a tile (softmax loop)
constexpr int kStages = 3;                        // K and V ring depth per slot
constexpr int kSlots = 2;
constexpr int kRing = 4;                          // item records per slot
// Tile masks per slot: the producer writes the mask of tile j once the K
// stage of tile j-3 is free, i.e. once QK^T of tile j-3, PV of tile j-5 and
// the softmax of tile j-5 are done; the softmax may still read the mask of
// tile j-4, so the ring must hold at least five.
constexpr int kMaskRing = 8;
constexpr int kQBytes = kRows * kDHead * 2;       // 16 KB of 16-bit elements
constexpr int kKvBytes = kTileKeys * kDHead * 2;  // 12 KB
constexpr int kRowBytes = kDHead * 2;             // 128 B
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8;                  // warps 8, 9: TMA producers of slots 0, 1
constexpr int kWarpMma = 10;                      // warps 10, 11: MMA issuers of slots 0, 1
constexpr int kWarpTmem = 10;                     // allocates and frees the tensor memory
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;               // S0 (96) | S1 (96) | O (64)
constexpr uint32_t kColO = 2 * kTileKeys;         // O within a slot's columns
constexpr float kRescaleLog2 = 8.f;               // lazy rescale: P stays below 2^8
// Register split: the two softmax warpgroups take registers from the control
// warpgroup: 256 * 208 + 128 * 88 = 64512 registers, which the launch (384
// threads at the compiled count) must hold (checked on the host).
constexpr int kRegsSoftmax = 208;
constexpr int kRegsControl = 88;
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
constexpr int kBatchCache = 64;                   // per-batch counts / flags kept in smem

struct FwdParams {
    CUtensorMap maps[kMapCount];              // first: 64-byte aligned
    CUtensorMap res_q[kMaxResidues];          // Q tiles of 128 rows
    CUtensorMap res_k[kMaxResidues];          // K tiles of kTileKeys rows
    CUtensorMap res_v[kMaxResidues];          // V tiles of kTileKeys rows
    AttnArgs a;
    int res_base[kMaxHeads];  // residue map of (head h, residue 0); -1: load rows one by one
    int band_items;       // B * band_items_per_batch, numbered first
    int total_items;      // + B*H*gtiles*nchunks global items
    int gtiles;           // ceil(max_global / 128)
    int oob_row;          // a row coordinate past the end of the row maps (reads zeros)
    int n_res;            // residue maps in use
    int merge_in_kernel;  // global rows merged by the last chunk (else by combine_kernel)
    unsigned long long wait_ns;   // limit of every bounded wait
    int stall_first_q;    // test hook: CTA 0 never loads slot 0's first Q tile
    int global_first;     // global items numbered before the band items
};

// Kernel arguments above 4 KB need CUDA 12.1 or newer (up to 32764 bytes).
static_assert(sizeof(FwdParams) <= 32000, "kernel arguments exceed the parameter space");

// An item as the producer decodes it; read by the MMA warp and the softmax
// warpgroup of the slot.
struct ItemInfo {
    int kind;       // 0: no more items, 1 band, 2 global rows
    int b, h, bh, dil, r, n_r;
    int q0;         // band: first residue-space row; global: first global slot
    int klo;        // first key of tile 0 (residue space for band items)
    int nkv;        // key tiles before the global-column tiles
    int ntiles;
    int key_end;    // global items: end of the key chunk
    int g;          // global tokens of the batch (clamped to max_global)
    int chunk;
    int has_pad;
    int res;        // band: residue tensor map of (head, r), -1: rows one by one
};
static_assert(sizeof(ItemInfo) == 64, "item record size");

// Column masks of one key tile, written by the producer: bits of the keys
// that exist and are not padding; for a global-column tile also the token
// position of each column (-1 past the count).
struct TileMask {
    uint32_t bits[4];
    int jpos[kTileKeys];
};

struct __align__(1024) FwdSmem {
    uint8_t q[kSlots][2][kQBytes];
    uint8_t k[kSlots][kStages][kKvBytes];
    uint8_t v[kSlots][kStages][kKvBytes];
    TileMask tmask[kSlots][kMaskRing];
    ItemInfo items[kSlots][kRing];
    uint64_t q_full[kSlots][2], q_empty[kSlots][2];
    uint64_t k_full[kSlots][kStages], k_empty[kSlots][kStages];
    uint64_t v_full[kSlots][kStages], v_empty[kSlots][kStages];
    uint64_t item_full[kSlots][kRing], item_empty[kSlots][kRing];
    uint64_t tm_full[kSlots][kMaskRing];
    // S / P buffer b of slot X: S(j) complete, P(j) stored, for the tiles j
    // with j % 2 == b (the softmax can store P(j+1) before PV(j) is issued).
    uint64_t s_full[kSlots][2], p_full[kSlots][2];
    uint64_t pv_done[kSlots], o_full[kSlots], o_free[kSlots];
    uint64_t drain[kSlots];
    int batch_count[kBatchCache];
    int batch_flags[kBatchCache];
    int head_dil[kMaxHeads];            // per-head tables, copied from the kernel
    int head_prefix[kMaxHeads + 1];     // arguments (indexed per item)
    int head_res[kMaxHeads];
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kFwdSmemBytes = sizeof(FwdSmem) + 1024;
static_assert(kFwdSmemBytes <= 232448, "shared memory per CTA");

// ------------------------------------------------------------ small helpers
// The part of a bounded wait that runs only when the phase is not complete
// at the first test; out of line to keep the roles' code small.
__device__ __forceinline__ bool wait_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                       int *status, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    uint32_t spins = 0;
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++spins & 31u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                set_status(status, kErrDeviceTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Bounded wait taken by a whole warp: either every lane goes on or every lane
// gives up, so no warp-collective instruction runs with a partial warp.
__device__ __forceinline__ bool warp_wait(const FwdParams &p, FwdSmem &sm, uint64_t *bar,
                                          uint32_t parity)
{
    const bool ok = mbar_try_wait(bar, parity) ||
                    wait_slow(bar, parity, &sm.abort_flag, p.a.ws.status, p.wait_ns);
    return __all_sync(0xffffffffu, ok);
}

// Waits (bounded, ignoring the abort flag) for a copy this CTA started, so
// that nothing lands in shared memory after the CTA has exited.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < limit_ns) {
    }
}

// Keys of the tile (N of QK^T, K of PV): 128, or the global tokens of a
// global-column tile rounded up to a multiple of 16.
__device__ __forceinline__ int tile_cols(const ItemInfo &I, int t)
{
    if (I.kind != 1 || t < I.nkv) return kTileKeys;
    const int left = min(kTileKeys, I.g - (t - I.nkv) * kTileKeys);
    return (left + 15) & ~15;
}

__device__ __forceinline__ int batch_count(const FwdSmem &sm, const AttnArgs &a, int b)
{
    return b < kBatchCache ? sm.batch_count[b] : a.ws.counts[b];
}

__device__ __forceinline__ int batch_flags(const FwdSmem &sm, const AttnArgs &a, int b)
{
    return b < kBatchCache ? sm.batch_flags[b] : a.ws.flags[b];
}

// Band item -> (batch, head, residue, tile of 128 rows): the heads' item
// counts are prefix sums in shared memory (binary search), the residues of
// a head are walked in order.
__device__ __forceinline__ void band_item_s(const FwdSmem &sm, const AttnArgs &a, int item, int &b,
                                            int &h, int &r, int &tile)
{
    b = item / a.band_items_per_batch;
    int rem = item - b * a.band_items_per_batch;
    int lo = 0, hi = a.H - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sm.head_prefix[mid] <= rem)
            lo = mid;
        else
            hi = mid - 1;
    }
    h = lo;
    rem -= sm.head_prefix[h];
    const int dil = sm.head_dil[h];
    r = 0;
    for (;;) {
        const int n_r = (a.n - r + dil - 1) / dil;
        const int t = (n_r + kRows - 1) / kRows;
        if (rem < t || r + 1 >= dil) break;
        rem -= t;
        ++r;
    }
    tile = rem;
}

__device__ __forceinline__ ItemInfo decode_item(const FwdParams &p, const FwdSmem &sm, int item)
{
    const AttnArgs &a = p.a;
    ItemInfo I;
    I.res = -1;
    // Band items first (index = band item), or after the global items.
    const int bi = p.global_first ? item - (p.total_items - p.band_items) : item;
    if (bi >= 0 && bi < p.band_items) {
        int tile;
        band_item_s(sm, a, bi, I.b, I.h, I.r, tile);
        I.kind = 1;
        I.bh = I.b * a.H + I.h;
        I.dil = sm.head_dil[I.h];
        I.res = sm.head_res[I.h] >= 0 ? sm.head_res[I.h] + I.r : -1;
        I.n_r = (a.n - I.r + I.dil - 1) / I.dil;
        I.q0 = tile * kRows;
        const int rows_hi = min(I.q0 + kRows - 1, I.n_r - 1);
        const int lo = max(I.q0 - (a.causal ? a.window - 1 : a.half), 0);
        const int hi = min(rows_hi + (a.causal ? 0 : a.half), I.n_r - 1);
        I.klo = lo;
        I.nkv = (hi - lo + kTileKeys) / kTileKeys;
        I.key_end = 0;
        I.g = min(batch_count(sm, a, I.b), a.max_global);
        I.chunk = 0;
        I.ntiles = I.nkv + (I.g + kTileKeys - 1) / kTileKeys;
    } else {
        const int gi = p.global_first ? item : item - p.band_items;
        const int per_bh = p.gtiles * a.L.nchunks;
        I.bh = gi / per_bh;
        const int rem = gi - I.bh * per_bh;
        const int gtile = rem / a.L.nchunks;
        I.chunk = rem - gtile * a.L.nchunks;
        I.b = I.bh / a.H;
        I.h = I.bh - I.b * a.H;
        I.kind = 2;
        I.dil = 1;
        I.r = 0;
        I.n_r = a.n;
        I.g = min(batch_count(sm, a, I.b), a.max_global);
        I.q0 = gtile * kRows;
        I.klo = I.chunk * kChunkKeys;
        I.key_end = min(a.n, I.klo + kChunkKeys);
        I.nkv = (I.key_end - I.klo + kTileKeys - 1) / kTileKeys;
        I.ntiles = (I.g > I.q0) ? I.nkv : 0;   // 0: no global row in this tile: skipped
    }
    I.has_pad = batch_flags(sm, a, I.b) & kFlagHasPadding;
    return I;
}

// ------------------------------------------------------------ producer
// The producer keeps, per slot, two items ahead of the one whose tiles it is
// loading: item records are written to the slot's ring as soon as they are
// claimed, their Q tiles load as soon as a Q buffer frees, and the index of
// the item after them is already being claimed (the atomic's round trip
// overlaps the tile loads), so that an item change stalls neither slot.
struct ProducerSlot {
    int kc;         // item whose tiles are being loaded (count within the slot)
    int t;          // its next tile
    int kw;         // item records written to the ring
    int kq;         // items whose Q load was started (or that need none)
    int claimed;    // index claimed for record kw (lane 0)
    int jt;         // tiles loaded
    bool ended;     // the "no more items" record has been written
};

// Claims the next item index from the device-wide counter (lane 0 only; the
// value is read when the record is written).  The first item of every slot
// is fixed (slot X of CTA c takes item kSlots * c + X), so the counter hands
// out the items after those and no atomic sits on the start of the kernel.
__device__ __forceinline__ int claim_item(int *sched, int lane)
{
    return lane == 0 ? atomicAdd(sched, 1) + int(gridDim.x) * kSlots : 0;
}

// Decodes the claimed index into the slot's next ring record and claims the
// one after.  Items without work (a tile of global rows past the batch's
// count) are skipped.  The end of the items is written as a record of kind 0.
__device__ __forceinline__ bool producer_write_next(const FwdParams &p, FwdSmem &sm, ProducerSlot &S,
                                                    int X, int lane, int *sched)
{
    ItemInfo I;
    I.kind = 0;
    for (;;) {
        const int idx = __shfl_sync(0xffffffffu, S.claimed, 0);
        if (idx >= p.total_items) {
            I.kind = 0;
            S.ended = true;
            break;
        }
        I = decode_item(p, sm, idx);
        S.claimed = claim_item(sched, lane);
        if (I.ntiles > 0) break;
    }
    const int k = S.kw;
    const int rs = k % kRing;
    if (!warp_wait(p, sm, &sm.item_empty[X][rs], (uint32_t(k / kRing) & 1u) ^ 1u)) return false;
    if (lane == 0) sm.items[X][rs] = I;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.item_full[X][rs]);
    ++S.kw;
    return true;
}

// Starts the Q load of record S.kq when its buffer is free (or at once if
// `block`); returns false on abort.
__device__ __forceinline__ bool producer_q(const FwdParams &p, FwdSmem &sm, ProducerSlot &S, int X,
                                           int lane, bool block, uint32_t &q_armed, uint32_t &q_par)
{
    const AttnArgs &a = p.a;
    if (S.kq >= S.kw) return true;
    const int k = S.kq;
    const ItemInfo &I = sm.items[X][k % kRing];
    if (I.kind == 0) {
        ++S.kq;
        return true;
    }
    const int qb = k & 1;
    const uint32_t use = uint32_t(k >> 1);
    const uint32_t want = (use & 1u) ^ 1u;
    if (block) {
        if (!warp_wait(p, sm, &sm.q_empty[X][qb], want)) return false;
    } else if (!__all_sync(0xffffffffu, mbar_try_wait(&sm.q_empty[X][qb], want))) {
        return true;
    }
    uint8_t *qd = sm.q[X][qb];
    uint64_t *qbar = &sm.q_full[X][qb];
    const bool stall = p.stall_first_q && blockIdx.x == 0 && X == 0 && k == 0;
    if (!stall) {
        if (I.kind == 1 && I.res >= 0) {
            if (lane == 0) {
                mbar_arrive_expect_tx(qbar, kQBytes);
                tma_load_3d(qd, &p.res_q[I.res], qbar, 0, I.q0, I.bh);
            }
        } else if (I.kind == 1) {
            if (lane == 0) mbar_arrive_expect_tx(qbar, kQBytes);
            __syncwarp();
            for (int rr = lane; rr < kRows; rr += 32) {
                const int ir = I.q0 + rr;
                const int y = ir < I.n_r ? I.bh * a.n + ir * I.dil + I.r : p.oob_row;
                tma_load_2d(qd + rr * kRowBytes, &p.maps[kMapQRow], qbar, 0, y);
            }
        } else {
            // Only the rows of real global tokens: a query row only feeds its
            // own output row, and rows past the count are never stored.
            const int rows = min(kRows, I.g - I.q0);
            if (lane == 0) mbar_arrive_expect_tx(qbar, rows * kRowBytes);
            __syncwarp();
            for (int rr = lane; rr < rows; rr += 32) {
                const int y = I.bh * a.n + a.ws.gidx[size_t(I.b) * a.n + I.q0 + rr];
                tma_load_2d(qd + rr * kRowBytes, &p.maps[kMapQgRow], qbar, 0, y);
            }
        }
        // Bit qb: a Q copy of that buffer was started; its parity.
        const uint32_t bit = 1u << qb;
        q_armed |= bit;
        q_par = (use & 1u) ? (q_par | bit) : (q_par & ~bit);
    }
    __syncwarp();
    ++S.kq;
    return true;
}

// Loads tile S.t of the slot's current item: its K tile (with the tile's
// column masks in the slot's tile-mask ring) into K stage jt % kStages, then
// its V tile into V stage jt % kStages, each once the stage has been released
// (the K stage by the tile's QK^T two tiles back, the V stage by its PV).
// Returns false on abort; `armed` and `par` record the copies started (bit
// 2*stage + {0: K, 1: V}) for the drain.
__device__ __forceinline__ bool producer_tile(const FwdParams &p, FwdSmem &sm, ProducerSlot &S,
                                              int X, int lane, uint32_t &armed, uint32_t &par)
{
    const AttnArgs &a = p.a;
    const ItemInfo I = sm.items[X][S.kc % kRing];
    const int t = S.t;
    const int stage = S.jt % kStages;
    const uint32_t phase = uint32_t(S.jt / kStages) & 1u;
    uint8_t *kd = sm.k[X][stage];
    uint8_t *vd = sm.v[X][stage];
    uint64_t *kbar = &sm.k_full[X][stage];
    uint64_t *vbar = &sm.v_full[X][stage];
    TileMask &tm = sm.tmask[X][S.jt % kMaskRing];
    const uint32_t *vb = a.ws.vbits + size_t(I.b) * a.L.nwords;
    const int kind = I.kind == 2 ? 2 : (t < I.nkv ? 1 : 3);   // 3: global-token columns
    const int k0 = I.klo + t * kTileKeys;
    const int s0 = (t - I.nkv) * kTileKeys;
    const int rows = tile_cols(I, t);
    if (!warp_wait(p, sm, &sm.k_empty[X][stage], phase ^ 1u)) return false;
    // Column masks.
    if (kind == 2 || (kind == 1 && I.has_pad)) {
#pragma unroll
        for (int w = 0; w < kChunks; ++w) {
            const int j = k0 + 32 * w + lane;
            const bool ok = kind == 2 ? (j < I.key_end && (!I.has_pad || bit_at(vb, j)))
                                      : (j < I.n_r && bit_at(vb, j * I.dil + I.r));
            const uint32_t bits = __ballot_sync(0xffffffffu, ok);
            if (lane == 0) tm.bits[w] = bits;
        }
    } else if (kind == 1) {
        if (lane < kChunks) tm.bits[lane] = 0xffffffffu;
    } else {
#pragma unroll
        for (int w = 0; w < kChunks; ++w) {
            const int c = 32 * w + lane;
            const int slot = s0 + c;
            const int j = slot < I.g ? a.ws.gidx[size_t(I.b) * a.n + slot] : -1;
            tm.jpos[c] = j;
            const bool ok = j >= 0 && bit_at(vb, j);
            const uint32_t bits = __ballot_sync(0xffffffffu, ok);
            if (lane == 0) tm.bits[w] = bits;
        }
    }
    // K (or V when second): a whole tile by one TMA copy, or rows one by one.
    auto load = [&](bool is_v, uint8_t *dst, uint64_t *bar) {
        if (kind == 2 || (kind == 1 && I.res >= 0)) {
            if (lane == 0) {
                const CUtensorMap *m = kind == 2 ? &p.maps[is_v ? kMapVgTile : kMapKgTile]
                                                 : (is_v ? &p.res_v[I.res] : &p.res_k[I.res]);
                mbar_arrive_expect_tx(bar, kKvBytes);
                tma_load_3d(dst, m, bar, 0, k0, I.bh);
            }
        } else {
            const int n_rows = kind == 1 ? kTileKeys : rows;
            if (lane == 0) mbar_arrive_expect_tx(bar, n_rows * kRowBytes);
            __syncwarp();
            const CUtensorMap *m = &p.maps[is_v ? kMapVRow : kMapKRow];
            for (int rr = lane; rr < n_rows; rr += 32) {
                int y = p.oob_row;
                if (kind == 1) {
                    const int jr = k0 + rr;
                    if (jr < I.n_r) y = I.bh * a.n + jr * I.dil + I.r;
                } else if (s0 + rr < I.g) {
                    y = I.bh * a.n + a.ws.gidx[size_t(I.b) * a.n + s0 + rr];
                }
                tma_load_2d(dst + rr * kRowBytes, m, bar, 0, y);
            }
        }
        __syncwarp();
    };
    load(false, kd, kbar);
    if (lane == 0) mbar_arrive(&sm.tm_full[X][S.jt % kMaskRing]);
    const uint32_t kb = 1u << (2 * stage);
    armed |= kb;
    par = phase ? (par | kb) : (par & ~kb);
    if (!warp_wait(p, sm, &sm.v_empty[X][stage], phase ^ 1u)) return false;
    load(true, vd, vbar);
    armed |= kb << 1;
    par = phase ? (par | (kb << 1)) : (par & ~(kb << 1));
    return true;
}

// The producer of slot X: item records two ahead, Q tiles as soon as a Q
// buffer frees, the K and V tiles of the current item.
__device__ __forceinline__ void producer_role(const FwdParams &p, FwdSmem &sm, int X, int lane)
{
    int *sched = p.a.ws.status + 16;
    ProducerSlot A;
    uint32_t kv_armed = 0, kv_par = 0;   // K/V copies started (see producer_tile); parities
    uint32_t qa = 0, qp = 0;             // bit b: Q buffer b was filled; parity
    bool ok = true;
    A.kc = A.t = A.kw = A.kq = A.jt = 0;
    A.ended = false;
    A.claimed = int(blockIdx.x) * kSlots + X;
#pragma unroll 1
    for (;;) {
        // Keep two records ahead of the current item.
        if (!A.ended && A.kw < A.kc + 2) ok = producer_write_next(p, sm, A, X, lane, sched);
        // The Q load of the oldest record without one: at once if it is the
        // current item's, else only if its buffer is already free.
        if (ok) ok = producer_q(p, sm, A, X, lane, A.kq == A.kc, qa, qp);
        if (!ok) break;
        // A slot that is not at its end always has the record of a real item.
        if (sm.items[X][A.kc % kRing].kind == 0) break;
        if (!producer_tile(p, sm, A, X, lane, kv_armed, kv_par)) {
            ok = false;
            break;
        }
        ++A.jt;
        if (++A.t == sm.items[X][A.kc % kRing].ntiles) {
            ++A.kc;
            A.t = 0;
        }
    }
    if (!ok || sm.abort_flag) {
        for (int b = 0; b < 2 * kStages; ++b) {
            if (!((kv_armed >> b) & 1u)) continue;
            uint64_t *bar = (b & 1) ? &sm.v_full[X][b >> 1] : &sm.k_full[X][b >> 1];
            drain_wait(bar, (kv_par >> b) & 1u, p.wait_ns);
        }
        for (int b = 0; b < 2; ++b)
            if ((qa >> b) & 1u) drain_wait(&sm.q_full[X][b], (qp >> b) & 1u, p.wait_ns);
    }
}

// ------------------------------------------------------------ MMA issuer
// The MMA issuer of slot X is one thread (lane 0 of the slot's MMA warp): it
// waits on the barriers itself and issues every tcgen05.mma and commit of the
// slot, so no instruction of the loop is a warp vote or an election.  S is
// double-buffered: QK^T of tile j+2 goes to the buffer of tile j right after
// PV of tile j (which reads P(j) there), so while the softmax works on tile
// j+1 the tensor core has already computed its scores.  Per slot the products
// run in issue order.
struct MmaCursor {
    int k;          // item
    int t;          // tile within the item
    int j;          // tile within the slot
    int kind, ntiles;
    int nkv, g;     // key tiles before the global-column tiles; global tokens
};

// Bounded wait of a single thread.
__device__ __forceinline__ bool thread_wait(const FwdParams &p, FwdSmem &sm, uint64_t *bar,
                                            uint32_t parity)
{
    return mbar_try_wait(bar, parity) ||
           wait_slow(bar, parity, &sm.abort_flag, p.a.ws.status, p.wait_ns);
}

// Keys of tile t of the cursor's item (see tile_cols).
__device__ __forceinline__ int cursor_cols(const MmaCursor &c, int t)
{
    if (c.kind != 1 || t < c.nkv) return kTileKeys;
    const int left = min(kTileKeys, c.g - (t - c.nkv) * kTileKeys);
    return (left + 15) & ~15;
}

// Reads the fields of ring record k the issuer needs.  Returns false on abort.
__device__ __forceinline__ bool mma_load_item(const FwdParams &p, FwdSmem &sm, MmaCursor &c, int X)
{
    const int rs = c.k % kRing;
    if (!thread_wait(p, sm, &sm.item_full[X][rs], uint32_t(c.k / kRing) & 1u)) return false;
    const ItemInfo &I = sm.items[X][rs];
    c.kind = I.kind;
    c.ntiles = I.ntiles;
    c.nkv = I.nkv;
    c.g = I.g;
    return true;
}

// Moves a cursor to its next tile; reads the next item's record from the
// ring when the item ends.  Returns false on abort.
__device__ __forceinline__ bool mma_advance(const FwdParams &p, FwdSmem &sm, MmaCursor &c, int X)
{
    ++c.j;
    if (++c.t < c.ntiles) return true;
    ++c.k;
    c.t = 0;
    return mma_load_item(p, sm, c, X);
}

__device__ __forceinline__ bool mma_issue_s(const FwdParams &p, FwdSmem &sm, uint32_t tS0, int X,
                                            const MmaCursor &c, int &stage, uint32_t &phase,
                                            bool bf16)
{
    if (c.t == 0 && !thread_wait(p, sm, &sm.q_full[X][c.k & 1], uint32_t(c.k >> 1) & 1u))
        return false;
    if (!thread_wait(p, sm, &sm.k_full[X][stage], phase)) return false;
    tc_fence_after();
    const int N = cursor_cols(c, c.t);
    const uint64_t qdesc = make_sdesc(smem_u32(sm.q[X][c.k & 1]), 16, 1024);
    const uint64_t kdesc = make_sdesc(smem_u32(sm.k[X][stage]), 16, 1024);
    const uint32_t idesc = make_idesc(128, 0, bf16, false) | (uint32_t(N >> 3) << 17);
    const uint32_t tS = tS0 + (c.j & 1) * kTileKeys;
#pragma unroll
    for (int kk = 0; kk < kDHead / 16; ++kk)
        mma_ss(tS, qdesc + uint64_t((kk * 32) >> 4), kdesc + uint64_t((kk * 32) >> 4), idesc,
               kk > 0 ? 1u : 0u);
    tc_commit(&sm.k_empty[X][stage]);
    tc_commit(&sm.s_full[X][c.j & 1]);
    if (c.t == c.ntiles - 1) tc_commit(&sm.q_empty[X][c.k & 1]);
    if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
    }
    return true;
}

__device__ __forceinline__ void mma_role(const FwdParams &p, FwdSmem &sm, uint32_t tmem, int X,
                                         bool bf16)
{
    const uint32_t tS0 = tmem + X * kSlotCols;
    const uint32_t tO = tS0 + kColO;
    const uint32_t id_pv = make_idesc(128, 64, bf16, true);
    // cs: the next QK^T to issue; cp: the next PV.  Each walks the K (V)
    // stages in order: stage index and phase parity.
    MmaCursor cs, cp;
    int ks = 0, vs = 0;
    uint32_t kph = 0, vph = 0;
    cs.k = cs.t = cs.j = 0;
    if (!mma_load_item(p, sm, cs, X)) return;
    cp = cs;
    // The first two QK^T of the slot.
    for (int i = 0; i < 2 && cs.kind != 0; ++i) {
        if (!mma_issue_s(p, sm, tS0, X, cs, ks, kph, bf16) || !mma_advance(p, sm, cs, X)) return;
    }
#pragma unroll 1
    while (cp.kind != 0) {
        if (!thread_wait(p, sm, &sm.p_full[X][cp.j & 1], uint32_t(cp.j >> 1) & 1u)) return;
        // The first PV of an item overwrites O: the epilogue of the item
        // before must have read it.
        if (cp.t == 0 && cp.k > 0 && !thread_wait(p, sm, &sm.o_free[X], uint32_t(cp.k - 1) & 1u))
            return;
        if (!thread_wait(p, sm, &sm.v_full[X][vs], vph)) return;
        tc_fence_after();
        const uint64_t vdesc = make_sdesc(smem_u32(sm.v[X][vs]), 16, 1024);
        const uint32_t tP = tS0 + (cp.j & 1) * kTileKeys;
        const int ksteps = cursor_cols(cp, cp.t) >> 4;
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk)
            if (kk < ksteps)
                mma_ts(tO, tP + kk * 8, vdesc + uint64_t((kk * 2048) >> 4), id_pv,
                       (kk > 0 || cp.t > 0) ? 1u : 0u);
        tc_commit(&sm.v_empty[X][vs]);
        tc_commit(&sm.pv_done[X]);
        if (++vs == kStages) {
            vs = 0;
            vph ^= 1u;
        }
        if (cp.t == cp.ntiles - 1) {
            tc_commit(&sm.o_full[X]);
            mbar_arrive(&sm.item_empty[X][cp.k % kRing]);
        }
        if (!mma_advance(p, sm, cp, X)) return;
        // QK^T two tiles ahead, into the buffer P(j) has just been read from.
        if (cs.kind != 0) {
            if (!mma_issue_s(p, sm, tS0, X, cs, ks, kph, bf16) || !mma_advance(p, sm, cs, X)) return;
        }
    }
}

// ------------------------------------------------------------ softmax
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
// the exponent field.  That holds for x >= -125.5; below, the exponent field
// leaves the normal range and the result is only a number in [0, 2^-124]
// (arguments below -126 are clamped), which is zero for every use here.
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

__global__ void exp2_poly_kernel(const float *x, float *y, int n)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (2 * i + 1 < n) {
        exp2_poly2(x[2 * i], x[2 * i + 1], y[2 * i], y[2 * i + 1]);
    } else if (2 * i < n) {
        float y1;
        exp2_poly2(x[2 * i], 0.f, y[2 * i], y1);
    }
}

struct RowState {
    float m, l;
};

template <typename T> __device__ __forceinline__ void unpack2(uint32_t w, float &lo, float &hi);
template <> __device__ __forceinline__ void unpack2<__nv_bfloat16>(uint32_t w, float &lo, float &hi)
{
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w));
    lo = f.x;
    hi = f.y;
}
template <> __device__ __forceinline__ void unpack2<__half>(uint32_t w, float &lo, float &hi)
{
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w));
    lo = f.x;
    hi = f.y;
}

// Online softmax of one 128-key score tile for this thread's row, 32 keys at
// a time (one compact loop: the code stays small enough for the instruction
// caches shared with the producer and MMA warps).  mw[c] marks the keys of
// this row among columns [32c, 32c+32); a chunk that is empty for every row
// of the warp is skipped (its probabilities are zero) and a chunk that is
// full for every row is not masked.  P = 2^(S*scale*log2e - m) goes as 16-bit
// pairs over the first 64 columns of the tile (chunk c to packed columns
// [16c, 16c+16), which hold scores already read).  The running maximum m is
// kept lazily: it moves only when a chunk's maximum exceeds it by more than
// 2^8; then the row sum, the probabilities already written in this tile and,
// at the end of the tile, O (every PV before this tile has completed) are
// scaled by the same factor.
template <typename T>
__device__ __forceinline__ bool softmax_tile(const FwdParams &p, FwdSmem &sm, uint32_t tS,
                                             uint32_t tO, RowState &st, bool first,
                                             const uint32_t (&mw)[4], float sl2, uint64_t *pv_bar,
                                             uint32_t pv_parity)
{
    uint32_t any_m = 0, full_m = 0;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
        any_m |= (__any_sync(0xffffffffu, mw[c] != 0u) ? 1u : 0u) << c;
        full_m |= (__all_sync(0xffffffffu, mw[c] == 0xffffffffu) ? 1u : 0u) << c;
    }
    if (first) {
        st.m = -INFINITY;
        st.l = 0.f;
    }
    float m = st.m, l = st.l;
    float alpha_o = 1.f;        // factor O must take for this tile's new maxima
#pragma unroll 1
    for (int c = 0; c < kChunks; ++c) {
        uint32_t pk[16];
        if ((any_m >> c) & 1u) {
            float s[32];
            tmem_ld32(tS + 32 * c, s);
            if (!((full_m >> c) & 1u)) {
                const uint32_t mc = c == 0 ? mw[0] : c == 1 ? mw[1] : c == 2 ? mw[2] : mw[3];
#pragma unroll
                for (int i = 0; i < 32; ++i) s[i] = ((mc >> i) & 1u) ? s[i] : -INFINITY;
            }
            const float cmax = max32(s) * sl2;
            const bool need = cmax > m + kRescaleLog2;
            if (__any_sync(0xffffffffu, need)) {
                const float a = !need ? 1.f : (m == -INFINITY ? 0.f : ex2(m - cmax));
                if (need) m = cmax;
                l *= a;
                alpha_o *= a;
                // Probabilities of earlier chunks of this tile were taken against
                // the old maximum.  Their stores must land before they are
                // read back.
                if (__any_sync(0xffffffffu, a != 1.f && a != 0.f)) {
                    if (c > 0) tmem_st_wait();
                    for (int c2 = 0; c2 < c; ++c2) {
                        float w[16];
                        tmem_ld16(tS + 16 * c2, w);
                        uint32_t r[16];
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            float lo, hi;
                            unpack2<T>(__float_as_uint(w[x]), lo, hi);
                            r[x] = pack2<T>(lo * a, hi * a);
                        }
                        tmem_st16(tS + 16 * c2, r);
                    }
                }
            }
            const float nb = (m == -INFINITY) ? 0.f : -m;
            float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float x0, x1, p0, p1;
                fma2(x0, x1, s[2 * i], s[2 * i + 1], sl2, sl2, nb, nb);
                if ((kPolyPairs >> (i & 7)) & 1u) {
                    exp2_poly2(x0, x1, p0, p1);
                } else {
                    p0 = ex2(x0);
                    p1 = ex2(x1);
                }
                if (i & 1)
                    add2(sb0, sb1, sb0, sb1, p0, p1);
                else
                    add2(sa0, sa1, sa0, sa1, p0, p1);
                pk[i] = pack2<T>(p0, p1);
            }
            l += (sa0 + sa1) + (sb0 + sb1);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
        }
        tmem_st16(tS + 16 * c, pk);
    }
    if (!first && __any_sync(0xffffffffu, alpha_o != 1.f)) {
        // O must hold every PV before this tile (the previous one may run).
        if (!warp_wait(p, sm, pv_bar, pv_parity)) return false;
        tc_fence_after();
        for (int half = 0; half < 2; ++half) {
            float o[32];
            tmem_ld32(tO + half * 32, o);
            uint32_t ob[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) ob[x] = __float_as_uint(o[x] * alpha_o);
            tmem_st32(tO + half * 32, ob);
        }
    }
    st.m = m;
    st.l = l;
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
__device__ __forceinline__ void merge_global_rows(const AttnArgs &a, int b, int bh, int g, int slot0,
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
    if (a.lse_out && L > 0.f) a.lse_out[size_t(bh) * a.n + pos] = M + log2f(L);
}

// Per-row results an item's epilogue needs after the softmax has moved on;
// the item's record stays in the slot's item ring until the epilogue is done.
// The row's words of the valid-key and global-token bitmaps are loaded when
// the item starts and decoded only in the epilogue, so their latency hides
// behind the item's tiles.
struct RowOut {
    float m, l;
    uint32_t vword, gword;  // band: bitmap words holding the row's position
    int bit;                // band: the row's bit in them
    bool row_in;            // band: the row exists
    __device__ __forceinline__ bool valid() const { return row_in && ((vword >> bit) & 1u); }
    // The row exists and is not a valid global row (those come from the
    // global items).
    __device__ __forceinline__ bool write() const
    {
        return row_in && (!valid() || !((gword >> bit) & 1u));
    }
};

// Writes the output of item `ke` of slot X: band rows O / l (zeros for padded
// rows); for global rows the chunk partials, and the merge when this is the
// last chunk of a group.  O is complete (o_full); the O buffer and the item's
// ring entry are released afterwards.
template <typename T>
__device__ __forceinline__ void epilogue(const FwdParams &p, FwdSmem &sm, uint32_t tmem_row, int X,
                                         int ke, const RowOut &ro, int tid)
{
    const AttnArgs &a = p.a;
    const int warp = tid >> 5, lane = tid & 31;
    const ItemInfo &I = sm.items[X][ke % kRing];
    const int kind = I.kind, bh = I.bh, q0 = I.q0;
    const uint32_t tO = tmem_row + X * kSlotCols + kColO;
    const int row = q0 + tid;
    const bool active = kind == 2 ? q0 + warp * 32 < I.g : q0 + warp * 32 < I.n_r;
    if (active) {
        if (kind == 1) {
            const bool write = ro.write();
            const int pos = write ? row * I.dil + I.r : 0;
            T *dst = static_cast<T *>(a.out) + (size_t(bh) * a.n + pos) * kDHead;
            const float inv = ro.valid() ? __frcp_rn(ro.l) : 0.f;
            if (a.lse_out && write && ro.valid())
                a.lse_out[size_t(bh) * a.n + pos] = ro.m + log2f(ro.l);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[32];
                tmem_ld32(tO + half * 32, o);
                if (write) store_half_row<T>(dst + half * 32, o, inv);
            }
        } else {
            const int slot = row;
            const size_t mg = size_t(a.max_global);
            float *P = a.ws.partials + (size_t(bh) * a.L.nchunks + I.chunk) * kPartialFloats * mg +
                       min(slot, a.max_global - 1);
            const bool write = slot < I.g;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[32];
                tmem_ld32(tO + half * 32, o);
                if (write) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) P[(2 + half * 32 + x) * mg] = o[x];
                }
            }
            if (write) {
                P[0] = ro.m;
                P[mg] = ro.l;
            }
        }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.o_free[X]);
    if (kind == 2 && active && p.merge_in_kernel) {
        // The last chunk to finish this warp's group of 32 global rows merges
        // them and resets the group's arrival counter for the next call on the
        // same workspace.
        const int group = (q0 >> 5) + warp;
        const int b = I.b, g = I.g;
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
            int *ctr = a.ws.counters + size_t(bh) * (a.L.ngroups + 1) + group;
            last = atomicAdd(ctr, 1) == a.L.nchunks - 1;
            if (last) atomicExch(ctr, 0);
        }
        if (__shfl_sync(0xffffffffu, last, 0)) {
            __threadfence();
            merge_global_rows<T>(a, b, bh, g, group * 32, lane);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.item_empty[X][ke % kRing]);
}

// Column masks of this thread's row for one tile: mw[c] marks the keys of
// the row among columns [32c, 32c + 32).
__device__ __forceinline__ void tile_row_mask(const AttnArgs &a, const ItemInfo &I, const TileMask &tm,
                                              int t, int row, int lane, uint32_t (&mw)[4])
{
    if (I.kind == 2) {
#pragma unroll
        for (int c = 0; c < 4; ++c) mw[c] = c < kChunks ? tm.bits[c] : 0u;
    } else if (t < I.nkv) {
        const int k0 = I.klo + t * kTileKeys;
        const int lo = max(row - (a.causal ? a.window - 1 : a.half), 0);
        const int hi = min(row + (a.causal ? 0 : a.half), I.n_r - 1);
#pragma unroll
        for (int c = 0; c < 4; ++c) mw[c] = c < kChunks ? range_bits(c, lo - k0, hi - k0) & tm.bits[c] : 0u;
    } else {
        // Global-token columns: real, unpadded tokens that are not already
        // window taps of this row.  A tap shares the row's residue class and
        // lies within the (dilated) window span; only tokens near the warp's
        // rows are tested.
        const int i = row * I.dil + I.r;
        const int span = a.half * I.dil;
        const int i_lo = __shfl_sync(0xffffffffu, i, 0) - span;
        const int i_hi = __shfl_sync(0xffffffffu, i, 31) + span;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (c >= kChunks) {
                mw[c] = 0u;
                continue;
            }
            uint32_t m = tm.bits[c];
            const int jl = tm.jpos[32 * c + lane];
            const bool near = jl >= i_lo && jl <= i_hi && (jl % I.dil) == I.r;
            uint32_t cand = __ballot_sync(0xffffffffu, near) & m;
            while (cand) {
                const int col = __ffs(cand) - 1;
                cand &= cand - 1u;
                const int d = __shfl_sync(0xffffffffu, jl, col) - i;
                if (d >= -span && d <= span) m &= ~(1u << col);
            }
            mw[c] = m;
        }
    }
}

// The softmax warpgroup of slot X.  Per tile: masks, wait for S, softmax,
// P to TMEM, arrive.  The epilogue of an item runs after the first tile of
// the next one (the issuer waits for it before that item's first PV).
template <typename T>
__device__ __forceinline__ void softmax_role(const FwdParams &p, FwdSmem &sm, uint32_t tmem, int X,
                                             int tid)
{
    const AttnArgs &a = p.a;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t tmem_row = tmem + (uint32_t(warp * 32) << 16);
    const uint32_t tSlot = tmem_row + X * kSlotCols;
    const uint32_t tO = tSlot + kColO;
    const float sl2 = a.scale_log2;
    int k = 0;      // items taken
    int jt = 0;     // tiles taken
    RowOut pend;
    bool pending = false;
    bool ok = true;

    while (ok) {
        const int rs = k % kRing;
        if (!warp_wait(p, sm, &sm.item_full[X][rs], uint32_t(k / kRing) & 1u)) break;
        const ItemInfo I = sm.items[X][rs];
        if (I.kind == 0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.item_empty[X][rs]);
            if (!pending) break;
        }
        const int row = I.q0 + tid;
        const int wrow0 = I.q0 + warp * 32;
        const bool active = I.kind == 2 ? wrow0 < I.g : wrow0 < I.n_r;
        RowOut ro;
        ro.vword = ro.gword = 0u;
        ro.bit = 0;
        ro.row_in = false;
        if (I.kind == 1 && active) {
            ro.row_in = row < I.n_r;
            const int i = row * I.dil + I.r;
            ro.bit = i & 31;
            if (ro.row_in) {
                ro.vword = a.ws.vbits[size_t(I.b) * a.L.nwords + (i >> 5)];
                ro.gword = a.ws.gbits[size_t(I.b) * a.L.nwords + (i >> 5)];
            }
        }
        RowState st{-INFINITY, 0.f};
        // A record of kind 0 (no more items) runs no tile but still flushes
        // the pending epilogue below.
        const int ntiles = I.kind == 0 ? 0 : I.ntiles;
        for (int t = 0; t <= ntiles; ++t) {
            if (t == 1 || (t == 0 && ntiles == 0)) {
                if (pending) {
                    // Every product of the previous item is complete.
                    const int ke = k - 1;
                    if (!warp_wait(p, sm, &sm.o_full[X], uint32_t(ke) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    epilogue<T>(p, sm, tmem_row, X, ke, pend, tid);
                    pending = false;
                }
            }
            if (t == ntiles) break;
            const int rt = jt % kMaskRing;
            if (!warp_wait(p, sm, &sm.tm_full[X][rt], uint32_t(jt / kMaskRing) & 1u)) {
                ok = false;
                break;
            }
            uint32_t mw[4];
            if (active) tile_row_mask(a, I, sm.tmask[X][rt], t, row, lane, mw);
            if (!warp_wait(p, sm, &sm.s_full[X][jt & 1], uint32_t(jt >> 1) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (active && !softmax_tile<T>(p, sm, tSlot + (jt & 1) * kTileKeys, tO, st, t == 0, mw,
                                           sl2, &sm.pv_done[X], uint32_t(jt - 1) & 1u)) {
                ok = false;
                break;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full[X][jt & 1]);
            ++jt;
        }
        if (!ok || I.kind == 0) break;
        ro.m = st.m;
        ro.l = st.l;
        pend = ro;
        pending = true;
        ++k;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdParams p)
{
    extern __shared__ uint8_t smem_raw[];
    FwdSmem &sm = *reinterpret_cast<FwdSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int X = 0; X < kSlots; ++X) {
            for (int b = 0; b < 2; ++b) {
                mbar_init(&sm.q_full[X][b], 1);
                mbar_init(&sm.q_empty[X][b], 1);
                mbar_init(&sm.s_full[X][b], 1);
                mbar_init(&sm.p_full[X][b], 4);           // one arrival per softmax warp
            }
            for (int st = 0; st < kStages; ++st) {
                mbar_init(&sm.k_full[X][st], 1);
                mbar_init(&sm.k_empty[X][st], 1);
                mbar_init(&sm.v_full[X][st], 1);
                mbar_init(&sm.v_empty[X][st], 1);
            }
            for (int r = 0; r < kRing; ++r) {
                mbar_init(&sm.item_full[X][r], 1);
                mbar_init(&sm.item_empty[X][r], 5);   // four softmax warps + the MMA warp
            }
            for (int r = 0; r < kMaskRing; ++r) mbar_init(&sm.tm_full[X][r], 1);
            mbar_init(&sm.pv_done[X], 1);
            mbar_init(&sm.o_full[X], 1);
            mbar_init(&sm.o_free[X], 4);
            mbar_init(&sm.drain[X], 1);
        }
        sm.abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kWarpProducer && lane == 0) {
        for (int m = 0; m < kMapCount; ++m) tma_prefetch_map(&p.maps[m]);
        for (int m = 0; m < p.n_res; ++m) {
            tma_prefetch_map(&p.res_q[m]);
            tma_prefetch_map(&p.res_k[m]);
            tma_prefetch_map(&p.res_v[m]);
        }
    }
    if (warp == kWarpTmem) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // Everything above overlaps the previous kernel in the stream; the
    // workspace it writes (compacted indices, bitmaps, counters) is read
    // only below.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int h = threadIdx.x; h < p.a.H; h += kThreads) {
        sm.head_dil[h] = p.a.dil[h];
        sm.head_prefix[h] = p.a.head_prefix[h];
        sm.head_res[h] = p.res_base[h];
    }
    if (threadIdx.x == 0) sm.head_prefix[p.a.H] = p.a.head_prefix[p.a.H];
    for (int b = threadIdx.x; b < kBatchCache && b < p.a.B; b += kThreads) {
        sm.batch_count[b] = p.a.ws.counts[b];
        sm.batch_flags[b] = p.a.ws.flags[b];
    }
    if (blockIdx.x == 0)
        for (int b = threadIdx.x; b < p.a.B; b += kThreads)
            if (p.a.ws.counts[b] > p.a.max_global) set_status(p.a.ws.status, kErrGlobalOverflow);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
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
            if (lane == 0) {
                mma_role(p, sm, tmem, X, std::is_same<T, __nv_bfloat16>::value);
                // Every MMA this thread issued has completed once this commit lands.
                tc_commit(&sm.drain[X]);
                drain_wait(&sm.drain[X], 0, p.wait_ns);
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpTmem) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    // Every CTA counts itself out, also after an abort; the last one resets
    // the item counter for the next launch on this workspace (no CTA claims
    // items any more by then).
    if (threadIdx.x == 0) {
        int *sched = p.a.ws.status + 16;
        int *finished = p.a.ws.status + 32;
        __threadfence();
        if (atomicAdd(finished, 1) == int(gridDim.x) - 1) {
            atomicExch(sched, 0);
            atomicExch(finished, 0);
        }
    }
}

// Merges the chunk partials of every global row into its output row.  A
// block takes 32 global slots of one (batch*head), lane = slot, so that every
// load is one 128-byte run of a field over the 32 slots; warp w owns the
// output dimensions [4w, 4w + 4).  One pass over the chunks keeps a running
// maximum (log-sum-exp: m in log2 units, the row sum l and the unnormalised
// output are rescaled when it grows).  Launched after the attention kernel
// (programmatic dependent launch: the wait below orders it).
constexpr int kCombineWarps = kDHead / 4;

template <typename T>
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const AttnArgs a)
{
    // The next kernel in the stream may launch now; it waits for this grid.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int d0 = 4 * (threadIdx.x >> 5);
    const int bh = blockIdx.x;
    const int slot = blockIdx.y * 32 + lane;
    const int b = bh / a.H;
    const int g = min(a.ws.counts[b], a.max_global);
    if (int(blockIdx.y) * 32 >= g) return;
    const size_t mg = size_t(a.max_global);
    const size_t cstride = kPartialFloats * mg;
    const float *P = partial_base(a, bh, 0) + min(slot, a.max_global - 1);
    float M = -INFINITY, L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    // Eight chunks per round: all their loads are issued before any is used,
    // so the round costs one memory latency.
    constexpr int kPerRound = 8;
    for (int c0 = 0; c0 < a.L.nchunks; c0 += kPerRound) {
        float mc[kPerRound], lc[kPerRound], oc[kPerRound][4];
#pragma unroll
        for (int u = 0; u < kPerRound; ++u) {
            const bool in = c0 + u < a.L.nchunks;
            const float *pc = P + size_t(in ? c0 + u : 0) * cstride;
            mc[u] = in ? __ldcg(pc) : -INFINITY;
            lc[u] = __ldcg(pc + mg);
#pragma unroll
            for (int x = 0; x < 4; ++x) oc[u][x] = __ldcg(pc + (2 + d0 + x) * mg);
        }
        float mr = M;
#pragma unroll
        for (int u = 0; u < kPerRound; ++u) mr = fmaxf(mr, mc[u]);
        if (mr == -INFINITY) continue;      // no key for this row so far
        const float fo = exp2f(M - mr);     // 0 while M is still -inf
        L *= fo;
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[x] *= fo;
#pragma unroll
        for (int u = 0; u < kPerRound; ++u) {
            const float f = exp2f(mc[u] - mr);   // 0 for a chunk without keys
            L = fmaf(f, lc[u], L);
#pragma unroll
            for (int x = 0; x < 4; ++x) acc[x] = fmaf(f, oc[u][x], acc[x]);
        }
        M = mr;
    }
    if (slot >= g) return;
    const int pos = a.ws.gidx[size_t(b) * a.n + slot];
    if (!bit_at(a.ws.vbits + size_t(b) * a.L.nwords, pos)) return;   // padded: zeros elsewhere
    const float inv = L > 0.f ? 1.f / L : 0.f;
    if (a.lse_out && d0 == 0 && L > 0.f) a.lse_out[size_t(bh) * a.n + pos] = M + log2f(L);
    T *dst = static_cast<T *>(a.out) + (size_t(bh) * a.n + pos) * kDHead + d0;
    uint2 v;
    v.x = pack2<T>(acc[0] * inv, acc[1] * inv);
    v.y = pack2<T>(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2 *>(dst) = v;
}

// ------------------------------------------------------------------ host
namespace {

// Test hooks (lf_test_forward_hooks): the limit of the bounded waits and a
// planted stall; read at every launch.
std::atomic<unsigned long long> g_wait_ns{1000ull * 1000ull * 1000ull};
std::atomic<int> g_stall_first_q{0};

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

// Whole tiles of box_rows rows of the residue class r of dilation dil of
// each (batch*head) slice: rows r, r+dil, ... ; dims {64, ceil((n-r)/dil), B*H}.
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
// kind: 0 = tiles of kRows rows (Q), 1 = single rows, 2 = tiles of kTileKeys
// rows (K, V, Kg, Vg).
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
                              : encode_tile_map(&m, base, dt, n, BH, kind == 0 ? kRows : kTileKeys,
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
    FwdParams p;
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
    p.band_items = a.B * a.band_items_per_batch;
    p.total_items = p.band_items + BH * p.gtiles * a.L.nchunks;
    p.oob_row = BH * a.n;
    // One warp merges 32 global rows over every chunk: cheap for a few chunks,
    // a separate wide kernel beyond that.
    p.merge_in_kernel = a.L.nchunks <= kMergeInKernelChunks;
    // Global items go first when their rows are merged in the kernel and a
    // call allows more than 32 global tokens: the merges (the last chunk's
    // warp reads every chunk's partials) then overlap band work instead of
    // ending the launch.  Measured: fp16 B2 H16 n4096 with 64 tokens 100.5 ->
    // 92.2 us; with 1 token at n4096 and with 32 tokens at n16384 (merged by
    // combine_kernel) global items first were 4 % and 2 % slower, so those
    // keep them last.
    p.global_first = p.merge_in_kernel && a.max_global > 32;
    p.wait_ns = g_wait_ns.load();
    p.stall_first_q = g_stall_first_q.load();
    const size_t smem = kFwdSmemBytes;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(attn_fwd_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem)) != cudaSuccess)
            return kErrCuda;
        // setmaxnreg.inc waits until the registers it asks for are free; refuse
        // to launch if the compiled register count cannot cover the split.
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, attn_fwd_kernel<T>) != cudaSuccess) return kErrCuda;
        if (fa.numRegs * kThreads < kRegsNeeded) return kErrUnsupported;
        attr_set[dev] = true;
    }
    const int want = (p.total_items + kSlots - 1) / kSlots;
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
    if (cudaLaunchKernelEx(&cfg, attn_fwd_kernel<T>, p) != cudaSuccess) return kErrCuda;
    if (a.max_global > 0 && !p.merge_in_kernel) {
        cudaLaunchConfig_t cc = {};
        cc.gridDim = dim3(a.B * a.H, (a.max_global + 31) / 32);
        cc.blockDim = dim3(32 * kCombineWarps);
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

extern "C" int lf_test_forward_hooks(unsigned long long wait_limit_ns, int stall_first_q)
{
    if (wait_limit_ns == 0) return LF_ERR_INVALID_ARG;
    lf::g_wait_ns.store(wait_limit_ns);
    lf::g_stall_first_q.store(stall_first_q ? 1 : 0);
    return LF_OK;
}

extern "C" int lf_exp2_poly_eval(const float *x, float *y, int n, lf_stream_t stream)
{
    if (n < 0 || (n > 0 && (!x || !y))) return LF_ERR_INVALID_ARG;
    if (n == 0) return LF_OK;
    const int pairs = (n + 1) / 2;
    lf::exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}
