// Arguments of the attention backward kernels (lf_bwd.cu).
#pragma once

#include <mutex>

#include "../../include/lf_attention.h"
#include "lf_device.cuh"

namespace lf {

struct BwdArgs {
    AttnArgs a;                 // inputs, prepared workspace, sizes, window
    const void *out, *dout;     // forward output O and its gradient dO
    void *dq, *dk, *dv, *dqg, *dkg, *dvg;
    float *lse, *dsum;          // [B*H*n] per band row: log2-domain lse, D
    const float *lse_in;        // optional: the forward's lse of the band rows
    float *lse_g, *dsum_g;      // [B*H*max_global] per global slot
    // Global tokens as keys of the rows that do not reach them through the
    // window: [B*H*max_global][dk (64, unscaled) | dv (64)] fp32 sums.
    float *gkv;
    // Global rows: (max, sum) per chunk of kGChunk keys
    // [B*H][nchg][max_global] and the fp32 dqg sums [B*H*max_global][64].
    float2 *gpart;
    float *dqg_acc;
    int nchg;
};

constexpr int kGChunk = 128;    // keys per partial of a global row; rows per
                                // chunk of the global-key column pass

// Bytes of the caller scratch of the backward.
inline size_t backward_scratch_bytes(int B, int H, int n, int max_global)
{
    const size_t bh = size_t(B) * H, mg = max_global > 0 ? max_global : 1;
    const size_t nchg = (size_t(n) + kGChunk - 1) / kGChunk;
    return lf_align256(2 * sizeof(float) * bh * n) + lf_align256(2 * sizeof(float) * bh * mg) +
           lf_align256(sizeof(float) * bh * mg * 2 * kDHead) +
           lf_align256(sizeof(float2) * bh * nchg * mg) +
           lf_align256(sizeof(float) * bh * mg * kDHead);
}

// Carves the scratch (256-byte aligned) into the pointers above.
inline void backward_scratch_ptrs(BwdArgs &A, void *scratch, int B, int H, int n, int max_global)
{
    const size_t bh = size_t(B) * H, mg = max_global > 0 ? max_global : 1;
    const size_t nchg = (size_t(n) + kGChunk - 1) / kGChunk;
    char *p = static_cast<char *>(scratch);
    A.lse = reinterpret_cast<float *>(p);
    A.dsum = A.lse + bh * n;
    p += lf_align256(2 * sizeof(float) * bh * n);
    A.lse_g = reinterpret_cast<float *>(p);
    A.dsum_g = A.lse_g + bh * mg;
    p += lf_align256(2 * sizeof(float) * bh * mg);
    A.gkv = reinterpret_cast<float *>(p);
    p += lf_align256(sizeof(float) * bh * mg * 2 * kDHead);
    A.gpart = reinterpret_cast<float2 *>(p);
    p += lf_align256(sizeof(float2) * bh * nchg * mg);
    A.dqg_acc = reinterpret_cast<float *>(p);
    A.nchg = int(nchg);
}

// CUDA-core path: every dtype, any dilations.
template <typename T> int launch_backward_simt(const BwdArgs &A, size_t elem, cudaStream_t stream);
// Global rows (independent of the band) and then the Kg/Vg keys over them,
// and global tokens as keys of the rows outside their window (after the rows'
// lse and D, before the band keys), on the CUDA cores.
template <typename T> int launch_global_rows(const BwdArgs &A, cudaStream_t stream);
template <typename T> int launch_global_keys(const BwdArgs &A, size_t elem, cudaStream_t stream);
// dqg from the fp32 sums in A.dqg_acc (the last step of the global rows).
template <typename T> int launch_global_final(const BwdArgs &A, cudaStream_t stream);
// Global rows and Kg / Vg keys in one streamed pass (at most 8 global
// tokens, given the forward's lse: after launch_row_stats).
template <typename T> int launch_global_small(const BwdArgs &A, cudaStream_t stream);
template <typename T> int launch_global_cols(const BwdArgs &A, cudaStream_t stream);
// lse (from A.lse_in) and D of every band row into A.lse and A.dsum, and of
// every global slot into A.lse_g and A.dsum_g, for the schedule in which the
// band rows and keys run side by side.
template <typename T> int launch_row_stats(const BwdArgs &A, cudaStream_t stream);

// A second stream of the current device, with the events that fork work onto
// it and join it back; the returned lock serialises its use across host
// threads (out = nullptr when it cannot be created).
struct SideStream {
    cudaStream_t stream, stream2;
    cudaEvent_t fork, join, fork2, join2;
};
std::unique_lock<std::mutex> side_stream(SideStream *&out);

// The backward's order on `stream`: zero dqg; fork the global rows and then
// the Kg/Vg keys onto the side stream; band rows; global-token columns; band
// keys; join.  With side_by_side (the tensor-core path given the forward's
// lse), every row's lse and D are written first (launch_row_stats), the side
// stream forks after them, and the global-token columns + band keys run on a
// third stream beside the band rows.  Works under stream capture (the side
// streams join and leave with the events).
template <typename T, typename RowsFn, typename KeysFn, typename GRowsFn, typename GColsFn,
          typename GKeysFn>
int backward_schedule(const BwdArgs &A, size_t elem, cudaStream_t stream, RowsFn &&band_rows,
                      KeysFn &&band_keys, GRowsFn &&global_rows, GColsFn &&global_cols,
                      GKeysFn &&global_keys, bool side_by_side)
{
    const size_t bytes = size_t(A.a.B) * A.a.H * A.a.n * kDHead * elem;
    // Qg gets gradient rows only at global positions.
    if (cudaMemsetAsync(A.dqg, 0, bytes, stream) != cudaSuccess) return kErrCuda;
    SideStream *side = nullptr;
    auto lock = side_stream(side);
    if (!side) return kErrCuda;
    int rc = side_by_side ? launch_row_stats<T>(A, stream) : kOk;
    if (cudaEventRecord(side->fork, stream) != cudaSuccess ||
        cudaStreamWaitEvent(side->stream, side->fork, 0) != cudaSuccess)
        return kErrCuda;
    if (rc == kOk) rc = global_rows(side->stream);
    if (rc == kOk) rc = global_keys(side->stream);
    const bool joined = cudaEventRecord(side->join, side->stream) == cudaSuccess;
    if (!side_by_side) {
        if (rc == kOk) rc = band_rows(stream);
        if (rc == kOk) rc = global_cols(stream);
        if (rc == kOk) rc = band_keys(stream);
    } else if (rc == kOk) {
        // The band rows (dq) and the global-token columns + band keys (dk,
        // dv) need nothing from one another once lse and D are written, so
        // they run on two streams at once and each fills the other's last
        // partial wave of CTAs.
        bool joined2 = false;
        if (cudaEventRecord(side->fork2, stream) == cudaSuccess &&
            cudaStreamWaitEvent(side->stream2, side->fork2, 0) == cudaSuccess) {
            rc = global_cols(side->stream2);
            if (rc == kOk) rc = band_keys(side->stream2);
            joined2 = cudaEventRecord(side->join2, side->stream2) == cudaSuccess;
            if (rc == kOk) rc = band_rows(stream);
            if (!joined2 || cudaStreamWaitEvent(stream, side->join2, 0) != cudaSuccess) rc = kErrCuda;
        } else {
            rc = kErrCuda;
        }
    }
    // Joined on every path, so a capture of `stream` stays well formed.
    if (!joined || cudaStreamWaitEvent(stream, side->join, 0) != cudaSuccess) return kErrCuda;
    return rc;
}
// Tensor-core path for bf16 / fp16; kErrUnsupported (nothing launched) when
// the heads' residue classes exceed its tensor-map budget.
int launch_backward_tc(lf_dtype dtype, const BwdArgs &A, cudaStream_t stream);

}  // namespace lf
