// Internal launch interface between the C ABI (ssm_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "ssm_scan.h"

namespace ssm {

struct FwdParams {
    const void *u, *delta;
    const float *A;
    const void *B, *C;
    const float *D;
    const void *z;
    const float *delta_bias;
    void *out;
    float *last_state, *ckpt;
    int batch, dim, L, N, n_ckpt;
    int softplus;
    bool io_bf16;
    bool vec_ok;  // every [.., L] row starts 16-byte aligned
};

struct BwdParams {
    const void *u, *delta;
    const float *A;
    const void *B, *C;
    const float *D;
    const void *z;
    const float *delta_bias;
    const void *dout;
    const float *ckpt;  // [batch][dim][n_ckpt][N] states at chunk ends
    float *du, *ddelta, *dA, *dB, *dC, *dD, *dz, *ddelta_bias;
    int batch, dim, L, N, n_ckpt;
    int softplus;
    bool io_bf16;
    bool vec_ok;
};

cudaError_t launch_fwd(const FwdParams &p, bool states_only, cudaStream_t stream);
cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream);

}  // namespace ssm
