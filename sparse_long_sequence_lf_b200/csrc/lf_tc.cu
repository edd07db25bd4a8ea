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
//                 every dilation.  The keys stream as 128-key tiles over the
//                 band's diagonals, then as tiles of the (deduplicated) global
//                 tokens; an online softmax runs over all of them.
//   global items  up to 128 global rows of one (batch, head) against one
//                 512-key chunk of Kg/Vg; each writes fp32 partials (max, sum,
//                 unnormalised output) and the last chunk to finish merges
//                 them by log-sum-exp into the output rows.
//
// Layout of one CTA (384 threads, one CTA per SM, persistent over items):
//   warps 0-3   softmax warpgroup of lane 0   (one thread per query row)
//   warps 4-7   softmax warpgroup of lane 1
//   warp  8     TMA producer of lane 0
//   warp  9     TMA producer of lane 1
//   warp 10     TMEM allocator and MMA issuer for both lanes
//   warp 11     idle (completes the third warpgroup for the register split)
// The two lanes are independent item streams; the MMA warp alternates
// between them so one lane's QK^T / PV runs while the other lane's softmax
// does its exponentials.
//
// TMEM (512 columns): S/P of lane X at columns [128X, 128X+128) (fp32 scores,
// overwritten in place by the 16-bit probabilities P in the first 64
// columns), O of lane X at [256+64X, 320+64X).
//   S = Q K^T      tcgen05.mma kind::f16, A = Q (smem, K-major),
//                  B = K tile (smem, K-major), 128x128 fp32 in TMEM
//   O += P V       tcgen05.mma kind::f16, A = P (TMEM), B = V tile
//                  (smem, MN-major), 128x64 fp32 in TMEM
// Shared-memory tiles are 128 rows x 128 bytes with the 128-byte swizzle,
// written by TMA: whole tiles for undilated rows, single-row loads for dilated
// rows, global tokens and gathered Qg rows.  Every wait on an mbarrier is
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

constexpr int kRows = 128;
constexpr int kKeys = 128;
constexpr int kStages = 2;
constexpr int kLanes = 2;
constexpr int kTileBytes = kRows * kDHead * 2;   // 16 KB of 16-bit elements
constexpr int kRowBytes = kDHead * 2;            // 128 B
constexpr int kThreads = 384;        // 3 warpgroups
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 10;
// Register split: the softmax warpgroups take registers from the producer /
// MMA warpgroup.  The launch must hold at least kRegsNeeded registers
// (checked on the host against the compiled register count).
constexpr int kRegsSoftmax = 216;
constexpr int kRegsControl = 64;
constexpr int kRegsNeeded = 2 * 128 * kRegsSoftmax + 128 * kRegsControl;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;   // lazy rescale: P stays below 2^8

enum MapId {
    kMapQTile, kMapKTile, kMapVTile, kMapKgTile, kMapVgTile,
    kMapQRow, kMapKRow, kMapVRow, kMapQgRow, kMapCount
};

struct TcParams {
    CUtensorMap maps[kMapCount];   // first: 64-byte aligned
    AttnArgs a;
    int global_items;     // B*H*gtiles*nchunks, ordered before the band items
    int total_items;
    int gtiles;           // ceil(max_global / 128)
    int oob_row;          // a row coordinate past the end of the row maps (reads zeros)
};

static_assert(sizeof(AttnArgs) + kMapCount * sizeof(CUtensorMap) + 64 <= 4096,
              "kernel arguments must fit the classic 4 KB parameter space");

struct __align__(1024) TcSmem {
    uint8_t q[kLanes][kTileBytes];
    uint8_t k[kLanes][kStages][kTileBytes];
    uint8_t v[kLanes][kStages][kTileBytes];
    uint64_t q_full[kLanes], q_empty[kLanes];
    uint64_t kv_full[kLanes][kStages], kv_empty[kLanes][kStages];
    uint64_t s_full[kLanes], p_full[kLanes], o_full[kLanes], o_free[kLanes];
    uint64_t drain;
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

// Walks the tiles of the items of one lane: items lane, lane + stride, ...
struct Cursor {
    int item, stride, total;
    int t;
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
        seek(p);
    }
    __device__ __forceinline__ void advance(const TcParams &p)
    {
        if (++t < G.ntiles) return;
        item += stride;
        seek(p);
    }
    __device__ __forceinline__ bool is_global_col_tile() const { return G.kind == 1 && t >= G.nkv; }
    // Keys in this tile (N of QK^T, K of PV): 128, or the global tokens of a
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

// TMA producer of one lane.
__device__ void producer_role(const TcParams &p, TcSmem &sm, int X, int lane)
{
    const AttnArgs &a = p.a;
    Cursor cur;
    cur.init(p, blockIdx.x * kLanes + X, gridDim.x * kLanes);
    int stage = 0;
    uint32_t phase = 0, qe_phase = 1;
    bool armed[kStages] = {};
    uint32_t armed_phase[kStages] = {};
    bool q_armed = false;
    uint32_t q_armed_phase = 0, qf_count = 0;
    const int n = a.n;
    bool ok = true;

    while (cur.valid && ok) {
        const Geom &G = cur.G;
        if (cur.t == 0) {
            if (!warp_wait(&sm.q_empty[X], qe_phase, &sm.abort_flag, a.ws.status)) { ok = false; break; }
            qe_phase ^= 1u;
            const bool tile_load = (G.kind == 1 && G.dil == 1);
            if (lane == 0) mbar_arrive_expect_tx(&sm.q_full[X], kTileBytes);
            __syncwarp();
            if (tile_load) {
                if (lane == 0) tma_load_3d(sm.q[X], &p.maps[kMapQTile], &sm.q_full[X], 0, G.q0, G.bh);
            } else {
                const CUtensorMap *map = G.kind == 1 ? &p.maps[kMapQRow] : &p.maps[kMapQgRow];
                for (int rr = lane; rr < kRows; rr += 32) {
                    int y = p.oob_row;
                    if (G.kind == 1) {
                        const int ir = G.q0 + rr;
                        if (ir < G.n_r) y = G.bh * n + ir * G.dil + G.r;
                    } else {
                        const int slot = G.q0 + rr;
                        if (slot < G.g) y = G.bh * n + a.ws.gidx[size_t(G.b) * n + slot];
                    }
                    tma_load_2d(sm.q[X] + rr * kRowBytes, map, &sm.q_full[X], 0, y);
                }
            }
            q_armed = true;
            q_armed_phase = qf_count & 1u;
            ++qf_count;
        }
        if (!warp_wait(&sm.kv_empty[X][stage], phase ^ 1u, &sm.abort_flag, a.ws.status)) { ok = false; break; }
        uint8_t *kd = sm.k[X][stage];
        uint8_t *vd = sm.v[X][stage];
        uint64_t *bar = &sm.kv_full[X][stage];
        if (G.kind == 2) {
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, 2 * kTileBytes);
                tma_load_3d(kd, &p.maps[kMapKgTile], bar, 0, cur.k0(), G.bh);
                tma_load_3d(vd, &p.maps[kMapVgTile], bar, 0, cur.k0(), G.bh);
            }
        } else if (!cur.is_global_col_tile() && G.dil == 1) {
            if (lane == 0) {
                mbar_arrive_expect_tx(bar, 2 * kTileBytes);
                tma_load_3d(kd, &p.maps[kMapKTile], bar, 0, cur.k0(), G.bh);
                tma_load_3d(vd, &p.maps[kMapVTile], bar, 0, cur.k0(), G.bh);
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
        // Let every copy this warp started land before the CTA exits.
        for (int s = 0; s < kStages; ++s)
            if (armed[s]) {
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(&sm.kv_full[X][s], armed_phase[s]) &&
                       global_timer_ns() - t0 < kWaitLimitNs) {
                }
            }
        if (q_armed) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&sm.q_full[X], q_armed_phase) &&
                   global_timer_ns() - t0 < kWaitLimitNs) {
            }
        }
    }
}

struct MmaLane {
    Cursor cur;
    int stage;
    uint32_t phase, qf_phase, pf_phase, of_phase;
    bool pend;
    int pend_stage, pend_n;
    bool pend_first, pend_last;
};

// One step of the MMA schedule of lane X: the PV of the previous tile, then
// the QK^T of the next one.  Returns false on abort.
__device__ __forceinline__ bool mma_step(const TcParams &p, TcSmem &sm, MmaLane &L, int X,
                                         uint32_t tmem, bool leader, uint32_t id_s,
                                         uint32_t id_pv)
{
    const AttnArgs &a = p.a;
    const uint32_t tS = tmem + X * 128;
    const uint32_t tO = tmem + 256 + X * 64;
    if (L.pend) {
        if (!warp_wait(&sm.p_full[X], L.pf_phase, &sm.abort_flag, a.ws.status)) return false;
        L.pf_phase ^= 1u;
        if (L.pend_first) {
            if (!warp_wait(&sm.o_free[X], L.of_phase, &sm.abort_flag, a.ws.status)) return false;
            L.of_phase ^= 1u;
        }
        tc_fence_after();
        if (leader) {
            const uint32_t vbase = smem_u32(sm.v[X][L.pend_stage]);
            for (int kk = 0; kk < L.pend_n / 16; ++kk) {
                const uint64_t bdesc = make_sdesc(vbase + kk * 2048, 16, 1024);
                mma_ts(tO, tS + kk * 8, bdesc, id_pv, (kk > 0 || !L.pend_first) ? 1u : 0u);
            }
            tc_commit(&sm.kv_empty[X][L.pend_stage]);
            if (L.pend_last) tc_commit(&sm.o_full[X]);
        }
        __syncwarp();
        L.pend = false;
    }
    if (L.cur.valid) {
        if (L.cur.t == 0) {
            if (!warp_wait(&sm.q_full[X], L.qf_phase, &sm.abort_flag, a.ws.status)) return false;
            L.qf_phase ^= 1u;
        }
        if (!warp_wait(&sm.kv_full[X][L.stage], L.phase, &sm.abort_flag, a.ws.status)) return false;
        tc_fence_after();
        const int N = L.cur.tile_n();
        if (leader) {
            const uint32_t qbase = smem_u32(sm.q[X]);
            const uint32_t kbase = smem_u32(sm.k[X][L.stage]);
            const uint32_t idesc = id_s | (uint32_t(N >> 3) << 17);
#pragma unroll
            for (int kk = 0; kk < kDHead / 16; ++kk) {
                const uint64_t adesc = make_sdesc(qbase + kk * 32, 16, 1024);
                const uint64_t bdesc = make_sdesc(kbase + kk * 32, 16, 1024);
                mma_ss(tS, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sm.s_full[X]);
            if (L.cur.t == L.cur.G.ntiles - 1) tc_commit(&sm.q_empty[X]);
        }
        __syncwarp();
        L.pend = true;
        L.pend_stage = L.stage;
        L.pend_n = N;
        L.pend_first = (L.cur.t == 0);
        L.pend_last = (L.cur.t == L.cur.G.ntiles - 1);
        advance_ring(L.stage, L.phase);
        L.cur.advance(p);
    }
    return true;
}

__device__ void mma_role(const TcParams &p, TcSmem &sm, uint32_t tmem, int lane, bool bf16)
{
    // S tiles: M = 128, N set per tile; PV: M = 128, N = 64, B MN-major.
    const uint32_t id_s = make_idesc(128, 0, bf16, false);
    const uint32_t id_pv = make_idesc(128, 64, bf16, true);
    MmaLane L[kLanes];
    for (int X = 0; X < kLanes; ++X) {
        L[X].cur.init(p, blockIdx.x * kLanes + X, gridDim.x * kLanes);
        L[X].stage = 0;
        L[X].phase = 0;
        L[X].qf_phase = 0;
        L[X].pf_phase = 0;
        L[X].of_phase = 1;   // the first item has no previous epilogue to wait for
        L[X].pend = false;
    }
    const bool leader = (lane == 0);
    for (;;) {
        bool any = false;
        for (int X = 0; X < kLanes; ++X) {
            if (!L[X].cur.valid && !L[X].pend) continue;
            any = true;
            if (!mma_step(p, sm, L[X], X, tmem, leader, id_s, id_pv)) return;
        }
        if (!any) break;
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

// Bits of the 128 key columns of a tile that hold real, unpadded keys, built
// by each warp on its own (4 lookups per lane and 4 ballots).
__device__ __forceinline__ void column_bits(const AttnArgs &a, const Cursor &cur, int lane,
                                            uint32_t (&bits)[4])
{
    const Geom &G = cur.G;
    const uint32_t *vb = a.ws.vbits + size_t(G.b) * a.L.nwords;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const int c = w * 32 + lane;
        bool ok;
        if (cur.is_global_col_tile()) {
            const int slot = cur.slot0() + c;
            ok = slot < G.g && bit_at(vb, a.ws.gidx[size_t(G.b) * a.n + slot]);
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

// Softmax of one full 128-key tile for this thread's row.  clo/chi bound the
// columns of the row's key range; cbits (when use_bits) marks real keys.
template <typename T>
__device__ __forceinline__ void softmax_tile128(uint32_t tS, uint32_t tO, RowState &st,
                                                bool first, int clo, int chi, bool use_bits,
                                                const uint32_t (&cbits)[4], float sl2)
{
    float s[128];
    tmem_ld128(tS, s);
    const bool need_mask = (clo > 0) || (chi < 127) || use_bits;
    if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
            bool ok = (c >= clo) && (c <= chi);
            if (use_bits) ok = ok && ((cbits[c >> 5] >> (c & 31)) & 1u);
            s[c] = ok ? s[c] : -INFINITY;
        }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 128; ++c) mx = fmaxf(mx, s[c]);
    const float mt = mx * sl2;
    float alpha = 1.f;
    bool rescale = false;
    if (first) {
        st.m = mt;
        st.l = 0.f;
    } else if (mt > st.m + kRescaleLog2) {
        alpha = ex2(st.m - mt);
        st.m = mt;
        rescale = true;
    }
    const float base = (st.m == -INFINITY) ? 0.f : st.m;
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float p0 = ex2(fmaf(s[32 * q + 2 * c], sl2, -base));
            const float p1 = ex2(fmaf(s[32 * q + 2 * c + 1], sl2, -base));
            sum += p0 + p1;
            pk[c] = pack2<T>(p0, p1);
        }
        tmem_st16(tS + 16 * q, pk);
    }
    if (__any_sync(0xffffffffu, rescale)) {
        // O of the previous tiles is complete: its PV was issued before this S.
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
    st.l = st.l * alpha + sum;
    tmem_st_wait();
}

// Softmax of a global-token column tile with N (multiple of 16) columns.
// Unrolled over the 8 possible 16-column chunks so every mask bit stays in a
// register (N is the same for the whole warp).
template <typename T>
__device__ __forceinline__ void softmax_tile_global_cols(const AttnArgs &a, const Cursor &cur,
                                                         uint32_t tS, uint32_t tO, RowState &st,
                                                         bool first, int i, int dil,
                                                         const uint32_t (&cbits)[4], float sl2)
{
    const Geom &G = cur.G;
    const int N = cur.tile_n();
    const int *gl = a.ws.gidx + size_t(G.b) * a.n + cur.slot0();
    uint32_t okb[4] = {0u, 0u, 0u, 0u};
    float mx = -INFINITY;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        if (ch * 16 < N) {
            float s[16];
            tmem_ld16(tS + ch * 16, s);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int col = ch * 16 + c;
                bool ok = (cbits[col >> 5] >> (col & 31)) & 1u;
                if (ok) ok = !is_tap(i, __ldg(gl + col), a.window, a.half, dil, a.causal);
                okb[col >> 5] |= (ok ? 1u : 0u) << (col & 31);
                mx = ok ? fmaxf(mx, s[c]) : mx;
            }
        }
    }
    const float mt = mx * sl2;
    float alpha = 1.f;
    bool rescale = false;
    if (first) {
        st.m = mt;
        st.l = 0.f;
    } else if (mt > st.m + kRescaleLog2) {
        alpha = ex2(st.m - mt);
        st.m = mt;
        rescale = true;
    }
    const float base = (st.m == -INFINITY) ? 0.f : st.m;
    float sum = 0.f;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        if (ch * 16 < N) {
            float s[16];
            tmem_ld16(tS + ch * 16, s);
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int col = ch * 16 + 2 * c;
                const bool ok0 = (okb[col >> 5] >> (col & 31)) & 1u;
                const bool ok1 = (okb[(col + 1) >> 5] >> ((col + 1) & 31)) & 1u;
                const float p0 = ok0 ? ex2(fmaf(s[2 * c], sl2, -base)) : 0.f;
                const float p1 = ok1 ? ex2(fmaf(s[2 * c + 1], sl2, -base)) : 0.f;
                sum += p0 + p1;
                pk[c] = pack2<T>(p0, p1);
            }
            tmem_st8(tS + ch * 8, pk);
        }
    }
    if (__any_sync(0xffffffffu, rescale)) {
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
    st.l = st.l * alpha + sum;
    tmem_st_wait();
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

// Merges the chunk partials of the global rows of one (bh, 128-row tile); run
// by the warp that arrived last.  Lane l handles rows l, l+32, l+64, l+96.
template <typename T>
__device__ void combine_global_tile(const AttnArgs &a, const Geom &G, int lane)
{
    const int nch = a.L.nchunks;
    const size_t cstride = size_t(a.max_global) * kPartialFloats;
    const uint32_t *vb = a.ws.vbits + size_t(G.b) * a.L.nwords;
    T *Out = static_cast<T *>(a.out) + size_t(G.bh) * a.n * kDHead;
    for (int rr = lane; rr < kRows; rr += 32) {
        const int slot = G.q0 + rr;
        if (slot >= G.g) break;
        const int pos = a.ws.gidx[size_t(G.b) * a.n + slot];
        if (!bit_at(vb, pos)) continue;   // padded global position: written as zeros elsewhere
        const float *P = a.ws.partials + (size_t(G.bh) * nch * a.max_global + slot) * kPartialFloats;
        float M = -INFINITY;
        for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(P + c * cstride));
        float Lsum = 0.f;
        float o[64];
#pragma unroll
        for (int x = 0; x < 64; ++x) o[x] = 0.f;
        for (int c = 0; c < nch; ++c) {
            const float *pc = P + c * cstride;
            const float mc = __ldcg(pc);
            const float f = (mc == -INFINITY) ? 0.f : ex2(mc - M);
            Lsum += f * __ldcg(pc + 1);
#pragma unroll
            for (int x = 0; x < 64; ++x) o[x] = fmaf(f, __ldcg(pc + 2 + x), o[x]);
        }
        store_row<T>(Out + size_t(pos) * kDHead, o, Lsum > 0.f ? 1.f / Lsum : 0.f);
    }
}

template <typename T>
__device__ void softmax_role(const TcParams &p, TcSmem &sm, uint32_t tmem, int X, int tid)
{
    const AttnArgs &a = p.a;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + X * 128;
    const uint32_t tO = tmem + lane_off + 256 + X * 64;
    const float sl2 = a.scale_log2;
    Cursor cur;
    cur.init(p, blockIdx.x * kLanes + X, gridDim.x * kLanes);
    uint32_t sf_phase = 0, of_phase = 0;
    RowState st{-INFINITY, 0.f};

    while (cur.valid) {
        const Geom &G = cur.G;
        const bool first = (cur.t == 0);
        const bool last = (cur.t == G.ntiles - 1);
        if (first && tid == 0 && a.ws.counts[G.b] > a.max_global)
            set_status(a.ws.status, kErrGlobalOverflow);
        const int row = G.q0 + tid;     // residue-space row (band) or global slot
        uint32_t cbits[4] = {~0u, ~0u, ~0u, ~0u};
        const bool gcol = cur.is_global_col_tile();
        const bool use_bits = gcol || G.has_pad;
        if (use_bits) column_bits(a, cur, lane, cbits);

        if (!warp_wait(&sm.s_full[X], sf_phase, &sm.abort_flag, a.ws.status)) return;
        sf_phase ^= 1u;
        tc_fence_after();
        if (gcol) {
            softmax_tile_global_cols<T>(a, cur, tS, tO, st, first, row * G.dil + G.r, G.dil,
                                        cbits, sl2);
        } else {
            int clo, chi;
            const int k0 = cur.k0();
            if (G.kind == 2) {
                clo = 0;
                chi = min(127, G.key_end - 1 - k0);
            } else {
                const int lo = max(row - (a.causal ? a.window - 1 : a.half), 0);
                const int hi = min(row + (a.causal ? 0 : a.half), G.n_r - 1);
                clo = lo - k0;
                chi = hi - k0;
            }
            softmax_tile128<T>(tS, tO, st, first, clo, chi, use_bits, cbits, sl2);
        }
        tc_fence_before();
        mbar_arrive(&sm.p_full[X]);

        if (last) {
            if (!warp_wait(&sm.o_full[X], of_phase, &sm.abort_flag, a.ws.status)) return;
            of_phase ^= 1u;
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
                mbar_arrive(&sm.o_free[X]);
            } else {
                const int slot = row;
                float *P = a.ws.partials +
                           ((size_t(G.bh) * a.L.nchunks + G.chunk) * a.max_global +
                            min(slot, a.max_global - 1)) * kPartialFloats;
                const bool write = slot < G.g;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tmem_ld32(tO + half * 32, o);
                    if (write) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) P[2 + half * 32 + x] = o[x];
                    }
                }
                tc_fence_before();
                mbar_arrive(&sm.o_free[X]);
                if (write) {
                    P[0] = st.m;
                    P[1] = st.l;
                }
                __threadfence();
                __syncwarp();
                int last_warp = 0;
                if (lane == 0) {
                    int *ctr = a.ws.counters + size_t(G.bh) * (a.L.ngroups + 1) + G.gtile;
                    const int target = 4 * a.L.nchunks;
                    const int prev = atomicAdd(ctr, 1);
                    last_warp = (prev == target - 1);
                    if (last_warp) *ctr = 0;
                }
                last_warp = __shfl_sync(0xffffffffu, last_warp, 0);
                if (last_warp) {
                    __threadfence();
                    combine_global_tile<T>(a, G, lane);
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
            mbar_init(&sm.q_full[X], 1);
            mbar_init(&sm.q_empty[X], 1);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(&sm.kv_full[X][s], 1);
                mbar_init(&sm.kv_empty[X][s], 1);
            }
            mbar_init(&sm.s_full[X], 1);
            mbar_init(&sm.p_full[X], kRows);
            mbar_init(&sm.o_full[X], 1);
            mbar_init(&sm.o_free[X], kRows);
        }
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kWarpProducer && lane == 0)
        for (int m = 0; m < kMapCount; ++m) tma_prefetch_map(&p.maps[m]);
    if (warp == kWarpMma) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        softmax_role<T>(p, sm, tmem, warp >> 2, threadIdx.x & 127);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    }
    if (warp < 8) {
    } else if (warp < kWarpMma) {
        producer_role(p, sm, warp - kWarpProducer, lane);
    } else if (warp == kWarpMma) {
        mma_role(p, sm, tmem, lane, std::is_same<T, __nv_bfloat16>::value);
        // Every MMA of this CTA has completed once this commit lands.
        if (lane == 0) tc_commit(&sm.drain);
        __syncwarp();
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&sm.drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
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

// Whole 128-row tiles of one (batch*head) slice: dims {64, n, B*H}.
bool encode_tile_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int n, int BH)
{
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cuuint64_t(kDHead), cuuint64_t(n), cuuint64_t(BH)};
    cuuint64_t strides[2] = {cuuint64_t(kRowBytes), cuuint64_t(n) * kRowBytes};
    cuuint32_t box[3] = {kDHead, kRows, 1};
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
    int kind, dt, n, BH;
    CUtensorMap map;
    bool used;
};

// Encoded tensor maps, reused while the same buffer and shape come back.
bool cached_map(CUtensorMap *out, int kind, const void *base, CUtensorMapDataType dt, int n, int BH)
{
    static std::mutex mu;
    static MapCacheEntry cache[64];
    static unsigned next = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &e : cache)
        if (e.used && e.base == base && e.kind == kind && e.dt == int(dt) && e.n == n && e.BH == BH) {
            *out = e.map;
            return true;
        }
    CUtensorMap m;
    const bool ok = kind == 0 ? encode_tile_map(&m, base, dt, n, BH)
                              : encode_row_map(&m, base, dt, long(n) * BH);
    if (!ok) return false;
    MapCacheEntry &e = cache[next++ % 64];
    e = MapCacheEntry{base, kind, int(dt), n, BH, m, true};
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
    ok = ok && cached_map(&p.maps[kMapQTile], 0, a.q, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapKTile], 0, a.k, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapVTile], 0, a.v, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapKgTile], 0, a.kg, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapVgTile], 0, a.vg, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapQRow], 1, a.q, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapKRow], 1, a.k, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapVRow], 1, a.v, dt, a.n, BH);
    ok = ok && cached_map(&p.maps[kMapQgRow], 1, a.qg, dt, a.n, BH);
    if (!ok) return kErrCuda;
    p.gtiles = (a.max_global + kRows - 1) / kRows;
    p.global_items = BH * p.gtiles * a.L.nchunks;
    p.total_items = p.global_items + a.B * a.band_items_per_batch;
    p.oob_row = BH * a.n;
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
    attn_tc_kernel<T><<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? kOk : kErrCuda;
}

}  // namespace

int launch_tc(lf_dtype dtype, const AttnArgs &a, cudaStream_t stream)
{
    if (dtype == LF_BF16) return launch_typed<__nv_bfloat16>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, stream);
    return launch_typed<__half>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, stream);
}

}  // namespace lf
