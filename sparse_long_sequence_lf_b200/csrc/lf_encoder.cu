// Longformer encoder stack from the library's own steps: per layer the
// projection prologue, the attention, the output layer and the feed-forward
// block (FasterTransformer Longformer Encoder guide, "compute flow": the two
// preprocessing kernels once, then the per-layer loop), with a window and
// dilations of its own for every layer ("LongFormer: The Long-Document
// Transformer" notes, "Sliding Window": w may differ from layer to layer).
// Host code only: it validates everything up front, then issues the steps on
// one stream; the masks are prepared once for all layers.
#include <cmath>

#include "../../include/lf_attention.h"
#include "lf_device.cuh"

using namespace lf;

namespace {

struct EncLayout {
    size_t attn_ws, tensor, hidden_t, ffn_ws;
    size_t off_proj, off_attn_out, off_h1, off_tmp, off_ffn, total;
};

EncLayout enc_layout(int B, int n, int H, int inter, int max_global)
{
    EncLayout L{};
    const int hid = H * kDHead;
    L.attn_ws = lf_workspace_size(B, H, n, kDHead, max_global);
    L.tensor = lf_align256(2 * size_t(B) * H * n * kDHead);
    L.hidden_t = lf_align256(2 * size_t(B) * n * hid);
    L.ffn_ws = lf_ffn_workspace_size(B, n, hid, inter);
    size_t off = lf_align256(L.attn_ws);     // the attention workspace sits at offset 0
    L.off_proj = off;      off += 6 * L.tensor;
    L.off_attn_out = off;  off += L.tensor;
    L.off_h1 = off;        off += L.hidden_t;
    L.off_tmp = off;       off += L.hidden_t;
    L.off_ffn = off;       off += L.ffn_ws;
    L.total = off;
    return L;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

size_t lf_encoder_workspace_size(int B, int n, int H, int d_head, int inter, int max_global)
{
    if (d_head != kDHead || B < 1 || n < 1 || H < 1 || H > kMaxHeads) return 0;
    if (max_global < 0 || max_global > n || inter < 64 || inter % 64) return 0;
    const EncLayout L = enc_layout(B, n, H, inter, max_global);
    if (L.attn_ws == 0 || L.ffn_ws == 0) return 0;
    return L.total;
}

int lf_encoder_forward(lf_dtype dtype, int B, int n, int H, int d_head, int inter, int layers,
                       const lf_layer_weights *weights, const int32_t *windows,
                       const int32_t *dilations, const void *x, const uint8_t *local_mask,
                       const uint8_t *global_mask, int max_global, float eps, void *out,
                       void *workspace, size_t workspace_bytes, lf_stream_t stream)
{
    if (d_head != kDHead) return LF_ERR_UNSUPPORTED;
    if (dtype != LF_BF16 && dtype != LF_F16)
        return (dtype == LF_F32) ? LF_ERR_UNSUPPORTED : LF_ERR_INVALID_ARG;
    if (B < 1 || n < 1 || H < 1 || H > kMaxHeads || layers < 1) return LF_ERR_INVALID_ARG;
    if (max_global < 0 || max_global > n || inter < 64) return LF_ERR_INVALID_ARG;
    if (inter % 64) return LF_ERR_UNSUPPORTED;
    if (!weights || !windows || !x || !out || !aligned16(x) || !aligned16(out))
        return LF_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return LF_ERR_INVALID_ARG;
    for (int l = 0; l < layers; ++l) {
        const lf_layer_weights &w = weights[l];
        if (windows[l] < 2 || windows[l] % 2) return LF_ERR_INVALID_ARG;
        if (dilations)
            for (int h = 0; h < H; ++h)
                if (dilations[size_t(l) * H + h] < 1) return LF_ERR_INVALID_ARG;
        for (const void *p : {w.w_qkv, w.w_o, w.ln1_gamma, w.ln1_beta, w.w_1, w.w_2,
                              w.ln2_gamma, w.ln2_beta})
            if (!p) return LF_ERR_INVALID_ARG;
        if (max_global > 0 && !w.w_qg) return LF_ERR_INVALID_ARG;
        for (const void *p : {w.w_qkv, w.b_qkv, w.w_qg, w.b_qg, w.w_o, w.b_o, w.ln1_gamma,
                              w.ln1_beta, w.w_1, w.b_1, w.w_2, w.b_2, w.ln2_gamma, w.ln2_beta})
            if (!aligned16(p)) return LF_ERR_INVALID_ARG;
    }
    const size_t need = lf_encoder_workspace_size(B, n, H, d_head, inter, max_global);
    if (need == 0) return LF_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return LF_ERR_WORKSPACE;

    const EncLayout L = enc_layout(B, n, H, inter, max_global);
    const int hid = H * kDHead;
    char *base = static_cast<char *>(workspace);
    const WsPtrs wp = ws_ptrs(workspace, ws_layout(B, H, n, max_global));
    int32_t *status = reinterpret_cast<int32_t *>(wp.status);
    void *proj[6];
    for (int i = 0; i < 6; ++i) proj[i] = base + L.off_proj + i * L.tensor;
    void *q = proj[0], *k = proj[1], *v = proj[2], *qg = proj[3], *kg = proj[4], *vg = proj[5];
    void *attn = base + L.off_attn_out;
    void *h1 = base + L.off_h1;
    void *tmp = base + L.off_tmp;
    void *ffn_ws = base + L.off_ffn;
    // The output layer's fp32 sums reuse the feed-forward block's.
    void *sum_ws = base + L.off_ffn + lf_align256(2 * size_t(B) * n * inter);
    const size_t sum_bytes = L.ffn_ws - lf_align256(2 * size_t(B) * n * inter);

    int rc = lf_attention_prepare(B, H, n, kDHead, local_mask, global_mask, max_global,
                                  workspace, L.attn_ws, stream);
    if (rc != LF_OK) return rc;
    const void *in = x;
    for (int l = 0; l < layers; ++l) {
        const lf_layer_weights &w = weights[l];
        // The last layer writes out; earlier ones alternate so that no step
        // reads the buffer it writes.
        void *dst = ((layers - 1 - l) % 2 == 0) ? out : tmp;
        rc = lf_qkv_projection(dtype, B, n, H, kDHead, in, w.w_qkv, w.b_qkv, w.w_qg, w.b_qg,
                               wp.gidx, wp.counts, max_global, q, k, v, qg, kg, vg, status,
                               stream);
        if (rc != LF_OK) return rc;
        rc = lf_attention_run(dtype, B, H, n, kDHead, q, k, v, qg, kg, vg, max_global,
                              windows[l], dilations ? dilations + size_t(l) * H : nullptr, 0,
                              attn, workspace, L.attn_ws, stream);
        if (rc != LF_OK) return rc;
        rc = lf_output_layer(dtype, B, n, H, kDHead, attn, w.w_o, w.b_o, in, w.ln1_gamma,
                             w.ln1_beta, eps, h1, sum_ws, sum_bytes, status, stream);
        if (rc != LF_OK) return rc;
        rc = lf_ffn_block(dtype, B, n, hid, inter, h1, w.w_1, w.b_1, w.w_2, w.b_2, w.ln2_gamma,
                          w.ln2_beta, eps, dst, ffn_ws, L.ffn_ws, status, stream);
        if (rc != LF_OK) return rc;
        in = dst;
    }
    return LF_OK;
}

}  // extern "C"
