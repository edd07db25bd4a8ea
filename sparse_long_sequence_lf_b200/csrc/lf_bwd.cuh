// Arguments of the attention backward kernels (lf_bwd.cu).
#pragma once

#include "lf_device.cuh"

namespace lf {

struct BwdArgs {
    AttnArgs a;                 // inputs, prepared workspace, sizes, window
    const void *out, *dout;     // forward output O and its gradient dO
    void *dq, *dk, *dv, *dqg, *dkg, *dvg;
    float *lse, *dsum;          // [B*H*n] per band row: log2-domain lse, D
    float *lse_g, *dsum_g;      // [B*H*max_global] per global slot
};

template <typename T> int launch_backward(const BwdArgs &A, size_t elem, cudaStream_t stream);

}  // namespace lf
