// C ABI of the Longformer attention library: argument checks, workspace
// layout, kernel dispatch.  Declared in include/lf_attention.h.
#include <cmath>
#include <cstring>
#include <initializer_list>

#include "../../include/lf_attention.h"
#include "lf_device.cuh"
#include "lf_bwd.cuh"

namespace lf {
int launch_prepare(const uint8_t *local_mask, const uint8_t *global_mask, int B, int n,
                   int max_global, int32_t *gidx, int32_t *counts, int *flags, uint32_t *vbits,
                   uint32_t *gbits, int *status, int *counters, int counters_per_batch,
                   int fill_tail, cudaStream_t stream);
int launch_f32(const AttnArgs &a, cudaStream_t stream);
int launch_tc(lf_dtype dtype, const AttnArgs &a, cudaStream_t stream);
int launch_projection(lf_dtype dtype, int B, int n, int H, const void *x, const void *w,
                      const void *bias, const void *wqg, const void *bqg, const int32_t *gidx,
                      const int32_t *counts, int max_global, void *const out[6], int32_t *status,
                      cudaStream_t stream);
int launch_output_layer(lf_dtype dtype, int B, int n, int H, const void *attn, const void *wo,
                        const void *bo, const void *residual, const void *gamma,
                        const void *beta, float eps, void *out, float *sum, int32_t *status,
                        cudaStream_t stream);
int launch_ffn(lf_dtype dtype, int B, int n, int hidden, int inter, const void *h,
               const void *w1, const void *b1, const void *w2, const void *b2,
               const void *gamma, const void *beta, float eps, void *out, void *act, float *sum,
               int32_t *status, cudaStream_t stream);
}  // namespace lf

using namespace lf;

namespace {

constexpr int kVersion = 10000;  // 1.0.0

int device_ok()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return kErrNoDevice;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return kErrNoDevice;
    return major == 10 ? kOk : kErrNoDevice;
}

bool sizes_ok(int B, int H, int n)
{
    if (B < 1 || H < 1 || n < 1 || H > kMaxHeads) return false;
    // Offsets inside one tensor are computed in 64-bit, positions in 32-bit.
    return double(B) * H * n * kDHead < 9.0e18 && n < (1 << 30);
}

size_t elem_size(lf_dtype dt)
{
    switch (dt) {
        case LF_F32: return 4;
        case LF_F16: return 2;
        case LF_BF16: return 2;
    }
    return 0;
}

int check_workspace(const void *ws, size_t bytes, const WsLayout &L)
{
    if (ws == nullptr) return kErrWorkspace;
    if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return kErrWorkspace;
    if (bytes < L.total) return kErrWorkspace;
    return kOk;
}

// Checks the arguments shared by the forward run and the backward pass and
// fills the kernel arguments; nothing is launched and the device is not
// queried.
int make_args(lf_dtype dtype, int B, int H, int n, int d_head, const void *q, const void *k,
              const void *v, const void *qg, const void *kg, const void *vg, int max_global,
              int window, const int32_t *dilation, int causal, void *workspace,
              size_t workspace_bytes, std::initializer_list<const void *> outputs, AttnArgs &a)
{
    if (d_head != kDHead) return LF_ERR_UNSUPPORTED;
    if (elem_size(dtype) == 0) return LF_ERR_INVALID_ARG;
    if (!sizes_ok(B, H, n) || max_global < 0 || max_global > n) return LF_ERR_INVALID_ARG;
    if (!q || !k || !v || !qg || !kg || !vg) return LF_ERR_INVALID_ARG;
    // Tiles move as 16-byte pieces (TMA boxes, vector loads).
    for (const void *ptr : {q, k, v, qg, kg, vg})
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return LF_ERR_INVALID_ARG;
    for (const void *ptr : outputs)
        if (!ptr || (reinterpret_cast<uintptr_t>(ptr) & 15u)) return LF_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return LF_ERR_INVALID_ARG;
    if (causal) {
        if (window < 1) return LF_ERR_INVALID_ARG;
        if (max_global != 0) return LF_ERR_UNSUPPORTED;
    } else if (window < 2 || (window % 2) != 0) {
        return LF_ERR_INVALID_ARG;
    }
    if (dilation)
        for (int h = 0; h < H; ++h)
            if (dilation[h] < 1) return LF_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(B, H, n, max_global);
    if (int rc = check_workspace(workspace, workspace_bytes, L)) return rc;

    std::memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.qg = qg; a.kg = kg; a.vg = vg;
    a.L = L;
    a.ws = ws_ptrs(workspace, L);
    a.B = B; a.H = H; a.n = n;
    a.window = window;
    a.half = window / 2;
    a.causal = causal;
    a.max_global = max_global;
    a.scale_log2 = float(1.4426950408889634 / std::sqrt(double(kDHead)));
    int items = 0;
    for (int h = 0; h < H; ++h) {
        const int dil = dilation ? dilation[h] : 1;
        a.dil[h] = dil;
        a.head_prefix[h] = items;
        for (int r = 0; r < dil && r < n; ++r) {
            const int n_r = (n - r + dil - 1) / dil;
            items += (n_r + 127) / 128;
        }
    }
    a.head_prefix[H] = items;
    a.band_items_per_batch = items;
    return kOk;
}

}  // namespace

extern "C" {

int lf_version(void) { return kVersion; }

const char *lf_status_string(int status)
{
    switch (status) {
        case LF_OK: return "ok";
        case LF_ERR_INVALID_ARG: return "invalid argument";
        case LF_ERR_UNSUPPORTED: return "unsupported configuration";
        case LF_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case LF_ERR_CUDA: return "CUDA runtime error";
        case LF_ERR_DEVICE_TIMEOUT: return "bounded device-side wait ran out";
        case LF_ERR_GLOBAL_OVERFLOW: return "more global tokens than max_global";
        case LF_ERR_NO_DEVICE: return "no sm_100 device is current";
        case LF_ERR_SCRATCH_LIMIT:
            return "workspace would exceed the fixed 16 MiB scratch of lf_attention_forward_static";
    }
    return "unknown status";
}

int lf_global_index(const uint8_t *global_mask, int B, int n, int32_t *global_idx,
                    int32_t *counts, lf_stream_t stream)
{
    if (B < 1 || n < 1 || !global_mask || !global_idx || !counts) return LF_ERR_INVALID_ARG;
    if (int rc = device_ok()) return rc;
    return launch_prepare(nullptr, global_mask, B, n, n, global_idx, counts, nullptr, nullptr,
                          nullptr, nullptr, nullptr, 0, 1, static_cast<cudaStream_t>(stream));
}

size_t lf_workspace_size(int B, int H, int n, int d_head, int max_global)
{
    if (!sizes_ok(B, H, n) || d_head != kDHead || max_global < 0 || max_global > n) return 0;
    return ws_layout(B, H, n, max_global).total;
}

int lf_attention_prepare(int B, int H, int n, int d_head, const uint8_t *local_mask,
                         const uint8_t *global_mask, int max_global, void *workspace,
                         size_t workspace_bytes, lf_stream_t stream)
{
    if (d_head != kDHead) return LF_ERR_UNSUPPORTED;
    if (!sizes_ok(B, H, n) || max_global < 0 || max_global > n) return LF_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(B, H, n, max_global);
    if (int rc = check_workspace(workspace, workspace_bytes, L)) return rc;
    if (int rc = device_ok()) return rc;
    WsPtrs p = ws_ptrs(workspace, L);
    return launch_prepare(local_mask, global_mask, B, n, max_global, p.gidx, p.counts, p.flags,
                          p.vbits, p.gbits, p.status, p.counters, H * (L.ngroups + 1), 0,
                          static_cast<cudaStream_t>(stream));
}

namespace {
int attention_run(lf_dtype dtype, int B, int H, int n, int d_head, const void *q, const void *k,
                  const void *v, const void *qg, const void *kg, const void *vg, int max_global,
                  int window, const int32_t *dilation, int causal, void *out, void *workspace,
                  size_t workspace_bytes, float *lse, lf_stream_t stream)
{
    AttnArgs a;
    if (int rc = make_args(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, max_global, window,
                           dilation, causal, workspace, workspace_bytes, {out}, a))
        return rc;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LF_ERR_INVALID_ARG;
    if (int rc = device_ok()) return rc;
    a.out = out;
    a.lse_out = lse;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case LF_F32: return launch_f32(a, s);
        case LF_F16: return launch_tc(LF_F16, a, s);
        case LF_BF16: return launch_tc(LF_BF16, a, s);
    }
    return LF_ERR_INVALID_ARG;
}

int attention_forward(lf_dtype dtype, int B, int H, int n, int d_head, const void *q,
                      const void *k, const void *v, const void *qg, const void *kg,
                      const void *vg, const uint8_t *local_mask, const uint8_t *global_mask,
                      int max_global, int window, const int32_t *dilation, int causal, void *out,
                      void *workspace, size_t workspace_bytes, float *lse, lf_stream_t stream)
{
    // Argument checks of the run come first so nothing is launched on error.
    if (d_head != kDHead) return LF_ERR_UNSUPPORTED;
    if (causal && max_global != 0) return LF_ERR_UNSUPPORTED;
    int rc = lf_attention_prepare(B, H, n, d_head, local_mask, global_mask, max_global,
                                  workspace, workspace_bytes, stream);
    if (rc != LF_OK) return rc;
    return attention_run(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, max_global, window,
                         dilation, causal, out, workspace, workspace_bytes, lse, stream);
}
}  // namespace

int lf_attention_run(lf_dtype dtype, int B, int H, int n, int d_head, const void *q,
                     const void *k, const void *v, const void *qg, const void *kg, const void *vg,
                     int max_global, int window, const int32_t *dilation, int causal, void *out,
                     void *workspace, size_t workspace_bytes, lf_stream_t stream)
{
    return attention_run(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, max_global, window,
                         dilation, causal, out, workspace, workspace_bytes, nullptr, stream);
}

int lf_attention_forward(lf_dtype dtype, int B, int H, int n, int d_head, const void *q,
                         const void *k, const void *v, const void *qg, const void *kg,
                         const void *vg, const uint8_t *local_mask, const uint8_t *global_mask,
                         int max_global, int window, const int32_t *dilation, int causal,
                         void *out, void *workspace, size_t workspace_bytes, lf_stream_t stream)
{
    return attention_forward(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, local_mask,
                             global_mask, max_global, window, dilation, causal, out, workspace,
                             workspace_bytes, nullptr, stream);
}

int lf_attention_forward_lse(lf_dtype dtype, int B, int H, int n, int d_head, const void *q,
                             const void *k, const void *v, const void *qg, const void *kg,
                             const void *vg, const uint8_t *local_mask,
                             const uint8_t *global_mask, int max_global, int window,
                             const int32_t *dilation, int causal, void *out, float *lse,
                             void *workspace, size_t workspace_bytes, lf_stream_t stream)
{
    if (!lse) return LF_ERR_INVALID_ARG;
    if (dtype != LF_BF16 && dtype != LF_F16) return LF_ERR_UNSUPPORTED;
    return attention_forward(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, local_mask,
                             global_mask, max_global, window, dilation, causal, out, workspace,
                             workspace_bytes, lse, stream);
}

size_t lf_host_staging_size(lf_dtype dtype, int B, int H, int n, int d_head)
{
    if (!sizes_ok(B, H, n) || d_head != kDHead || elem_size(dtype) == 0) return 0;
    const size_t t = lf_align256(size_t(B) * H * n * kDHead * elem_size(dtype));
    const size_t m = lf_align256(size_t(B) * n);
    return 7 * t + 2 * m;
}

namespace {

// What lf_attention_forward_host copies from the host: Q, K, V in full, and
// Qg, Kg, Vg in full when the global mask has a global position (the kernels
// read them only then).  Copying only Qg's global rows was measured slower:
// small strided copies from host memory cost more than the bytes they save.
bool has_global_token(const uint8_t *h_global_mask, int B, int n)
{
    if (!h_global_mask) return false;
    for (size_t i = 0; i < size_t(B) * n; ++i)
        if (h_global_mask[i]) return true;
    return false;
}

}  // namespace

size_t lf_host_copy_bytes(lf_dtype dtype, int B, int H, int n, int d_head,
                          const uint8_t *h_local_mask, const uint8_t *h_global_mask)
{
    if (lf_host_staging_size(dtype, B, H, n, d_head) == 0) return 0;
    const size_t tb = size_t(B) * H * n * kDHead * elem_size(dtype);
    const size_t masks = (h_local_mask ? size_t(B) * n : 0) + (h_global_mask ? size_t(B) * n : 0);
    return (has_global_token(h_global_mask, B, n) ? 6 : 3) * tb + masks;
}

int lf_attention_forward_host(lf_dtype dtype, int B, int H, int n, int d_head, const void *h_q,
                              const void *h_k, const void *h_v, const void *h_qg,
                              const void *h_kg, const void *h_vg, const uint8_t *h_local_mask,
                              const uint8_t *h_global_mask, int max_global, int window,
                              const int32_t *dilation, int causal, void *h_out, void *d_staging,
                              size_t staging_bytes, void *workspace, size_t workspace_bytes,
                              lf_stream_t stream)
{
    const size_t need = lf_host_staging_size(dtype, B, H, n, d_head);
    if (need == 0) return d_head != kDHead ? LF_ERR_UNSUPPORTED : LF_ERR_INVALID_ARG;
    if (!h_q || !h_k || !h_v || !h_qg || !h_kg || !h_vg || !h_out) return LF_ERR_INVALID_ARG;
    if (!d_staging || staging_bytes < need || reinterpret_cast<uintptr_t>(d_staging) % 256)
        return LF_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t tb = size_t(B) * H * n * kDHead * elem_size(dtype);
    const size_t t = lf_align256(tb);
    const size_t mb = size_t(B) * n;
    const size_t m = lf_align256(mb);
    char *base = static_cast<char *>(d_staging);
    // Without a global token the kernels read no Qg, Kg, Vg.
    const int ntensors = has_global_token(h_global_mask, B, n) ? 6 : 3;
    const void *src[6] = {h_q, h_k, h_v, h_qg, h_kg, h_vg};
    for (int i = 0; i < ntensors; ++i)
        if (cudaMemcpyAsync(base + i * t, src[i], tb, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return LF_ERR_CUDA;
    uint8_t *d_lm = nullptr, *d_gm = nullptr;
    if (h_local_mask) {
        d_lm = reinterpret_cast<uint8_t *>(base + 7 * t);
        if (cudaMemcpyAsync(d_lm, h_local_mask, mb, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return LF_ERR_CUDA;
    }
    if (h_global_mask) {
        d_gm = reinterpret_cast<uint8_t *>(base + 7 * t + m);
        if (cudaMemcpyAsync(d_gm, h_global_mask, mb, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return LF_ERR_CUDA;
    }
    void *d_out = base + 6 * t;
    int rc = lf_attention_forward(dtype, B, H, n, d_head, base, base + t, base + 2 * t,
                                  base + 3 * t, base + 4 * t, base + 5 * t, d_lm, d_gm, max_global,
                                  window, dilation, causal, d_out, workspace, workspace_bytes,
                                  stream);
    if (rc != LF_OK) return rc;
    if (cudaMemcpyAsync(h_out, d_out, tb, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return LF_ERR_CUDA;
    return lf_workspace_status(workspace, stream);
}

int lf_workspace_status(const void *workspace, lf_stream_t stream)
{
    if (!workspace) return LF_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return LF_ERR_CUDA;
    int status = 0;
    // The status word sits at offset 0 of every workspace layout.
    if (cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LF_ERR_CUDA;
    return status;
}

int lf_qkv_projection(lf_dtype dtype, int B, int n, int H, int d_head, const void *x,
                      const void *w, const void *bias, const void *wqg, const void *bqg,
                      const int32_t *global_idx, const int32_t *counts, int max_global, void *q,
                      void *k, void *v, void *qg, void *kg, void *vg, int32_t *status,
                      lf_stream_t stream)
{
    if (d_head != kDHead) return LF_ERR_UNSUPPORTED;
    if (dtype != LF_BF16 && dtype != LF_F16) return elem_size(dtype) ? LF_ERR_UNSUPPORTED
                                                                   : LF_ERR_INVALID_ARG;
    if (!sizes_ok(B, H, n) || max_global < 0 || max_global > n) return LF_ERR_INVALID_ARG;
    if (!x || !w || !q || !k || !v || !kg || !vg) return LF_ERR_INVALID_ARG;
    const bool with_qg = wqg != nullptr && max_global > 0;
    if (with_qg && (!qg || !global_idx || !counts)) return LF_ERR_INVALID_ARG;
    for (const void *ptr : {x, w, bias, wqg, bqg, static_cast<const void *>(q),
                            static_cast<const void *>(k), static_cast<const void *>(v),
                            static_cast<const void *>(qg), static_cast<const void *>(kg),
                            static_cast<const void *>(vg)})
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return LF_ERR_INVALID_ARG;
    if (int rc = device_ok()) return rc;
    void *const out[6] = {q, k, v, kg, vg, qg};
    return launch_projection(dtype, B, n, H, x, w, bias, with_qg ? wqg : nullptr, bqg, global_idx,
                             counts, with_qg ? max_global : 0, out, status,
                             static_cast<cudaStream_t>(stream));
}

size_t lf_output_workspace_size(int B, int n, int H, int d_head)
{
    if (!sizes_ok(B, H, n) || d_head != kDHead) return 0;
    return lf_align256(sizeof(float) * size_t(B) * n * H * kDHead);
}

int lf_output_layer(lf_dtype dtype, int B, int n, int H, int d_head, const void *attn,
                    const void *wo, const void *bo, const void *residual, const void *gamma,
                    const void *beta, float eps, void *out, void *workspace,
                    size_t workspace_bytes, int32_t *status, lf_stream_t stream)
{
    if (d_head != kDHead) return LF_ERR_UNSUPPORTED;
    if (dtype != LF_BF16 && dtype != LF_F16) return elem_size(dtype) ? LF_ERR_UNSUPPORTED
                                                                   : LF_ERR_INVALID_ARG;
    if (!sizes_ok(B, H, n)) return LF_ERR_INVALID_ARG;
    if (!attn || !wo || !residual || !gamma || !beta || !out) return LF_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return LF_ERR_INVALID_ARG;
    for (const void *ptr : {attn, wo, bo, residual, gamma, beta, static_cast<const void *>(out)})
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return LF_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < lf_output_workspace_size(B, n, H, d_head))
        return LF_ERR_WORKSPACE;
    if (int rc = device_ok()) return rc;
    return launch_output_layer(dtype, B, n, H, attn, wo, bo, residual, gamma, beta, eps, out,
                               static_cast<float *>(workspace), status,
                               static_cast<cudaStream_t>(stream));
}

size_t lf_backward_scratch_size(int B, int H, int n, int d_head, int max_global)
{
    if (!sizes_ok(B, H, n) || d_head != kDHead || max_global < 0 || max_global > n) return 0;
    return backward_scratch_bytes(B, H, n, max_global);
}

namespace {
int attention_backward(lf_dtype dtype, int B, int H, int n, int d_head, const void *q,
                       const void *k, const void *v, const void *qg, const void *kg,
                       const void *vg, const void *out, const void *dout, int max_global,
                       int window, const int32_t *dilation, int causal, void *dq, void *dk,
                       void *dv, void *dqg, void *dkg, void *dvg, const void *workspace,
                       size_t workspace_bytes, void *scratch, size_t scratch_bytes,
                       const float *lse, lf_stream_t stream)
{
    BwdArgs A;
    if (int rc = make_args(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, max_global, window,
                           dilation, causal, const_cast<void *>(workspace), workspace_bytes,
                           {out, dout, dq, dk, dv, dqg, dkg, dvg}, A.a))
        return rc;
    const size_t need = lf_backward_scratch_size(B, H, n, d_head, max_global);
    if (!scratch || scratch_bytes < need || reinterpret_cast<uintptr_t>(scratch) % 256)
        return LF_ERR_WORKSPACE;
    if (int rc = device_ok()) return rc;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LF_ERR_INVALID_ARG;
    A.out = out;
    A.dout = dout;
    A.dq = dq; A.dk = dk; A.dv = dv; A.dqg = dqg; A.dkg = dkg; A.dvg = dvg;
    backward_scratch_ptrs(A, scratch, B, H, n, max_global);
    A.lse_in = lse;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case LF_F32: return launch_backward_simt<float>(A, 4, s);
        case LF_F16:
        case LF_BF16: {
            const int rc = launch_backward_tc(dtype, A, s);
            if (rc != kErrUnsupported) return rc;
            return dtype == LF_F16 ? launch_backward_simt<__half>(A, 2, s)
                                   : launch_backward_simt<__nv_bfloat16>(A, 2, s);
        }
    }
    return LF_ERR_INVALID_ARG;
}
}  // namespace

int lf_attention_backward(lf_dtype dtype, int B, int H, int n, int d_head, const void *q,
                          const void *k, const void *v, const void *qg, const void *kg,
                          const void *vg, const void *out, const void *dout, int max_global,
                          int window, const int32_t *dilation, int causal, void *dq, void *dk,
                          void *dv, void *dqg, void *dkg, void *dvg, const void *workspace,
                          size_t workspace_bytes, void *scratch, size_t scratch_bytes,
                          lf_stream_t stream)
{
    return attention_backward(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, out, dout,
                              max_global, window, dilation, causal, dq, dk, dv, dqg, dkg, dvg,
                              workspace, workspace_bytes, scratch, scratch_bytes, nullptr, stream);
}

int lf_attention_backward_lse(lf_dtype dtype, int B, int H, int n, int d_head, const void *q,
                              const void *k, const void *v, const void *qg, const void *kg,
                              const void *vg, const void *out, const void *dout,
                              const float *lse, int max_global, int window,
                              const int32_t *dilation, int causal, void *dq, void *dk, void *dv,
                              void *dqg, void *dkg, void *dvg, const void *workspace,
                              size_t workspace_bytes, void *scratch, size_t scratch_bytes,
                              lf_stream_t stream)
{
    if (!lse) return LF_ERR_INVALID_ARG;
    if (dtype != LF_BF16 && dtype != LF_F16) return LF_ERR_UNSUPPORTED;
    return attention_backward(dtype, B, H, n, d_head, q, k, v, qg, kg, vg, out, dout,
                              max_global, window, dilation, causal, dq, dk, dv, dqg, dkg, dvg,
                              workspace, workspace_bytes, scratch, scratch_bytes, lse, stream);
}

size_t lf_ffn_workspace_size(int B, int n, int hidden, int inter)
{
    if (B < 1 || n < 1 || hidden < 64 || inter < 64 || hidden % 64 || inter % 64) return 0;
    const size_t rows = size_t(B) * n;
    return lf_align256(2 * rows * inter) + lf_align256(sizeof(float) * rows * hidden);
}

int lf_ffn_block(lf_dtype dtype, int B, int n, int hidden, int inter, const void *h,
                 const void *w1, const void *b1, const void *w2, const void *b2,
                 const void *gamma, const void *beta, float eps, void *out, void *workspace,
                 size_t workspace_bytes, int32_t *status, lf_stream_t stream)
{
    if (dtype != LF_BF16 && dtype != LF_F16) return elem_size(dtype) ? LF_ERR_UNSUPPORTED
                                                                   : LF_ERR_INVALID_ARG;
    if (B < 1 || n < 1 || hidden < 64 || inter < 64) return LF_ERR_INVALID_ARG;
    if (hidden % 64 || inter % 64) return LF_ERR_UNSUPPORTED;
    if (double(B) * n * (inter > hidden ? inter : hidden) > 9.0e18 || double(B) * n >= 2.0e9)
        return LF_ERR_INVALID_ARG;
    if (!h || !w1 || !w2 || !gamma || !beta || !out) return LF_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return LF_ERR_INVALID_ARG;
    for (const void *ptr : {h, w1, b1, w2, b2, gamma, beta, static_cast<const void *>(out)})
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return LF_ERR_INVALID_ARG;
    const size_t need = lf_ffn_workspace_size(B, n, hidden, inter);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return LF_ERR_WORKSPACE;
    if (int rc = device_ok()) return rc;
    char *base = static_cast<char *>(workspace);
    float *sum = reinterpret_cast<float *>(base + lf_align256(2 * size_t(B) * n * inter));
    return launch_ffn(dtype, B, n, hidden, inter, h, w1, b1, w2, b2, gamma, beta, eps, out, base,
                      sum, status, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
