// Backward entry point that allocates nothing.
//
// ssm_selective_scan_bwd needs device scratch for its state checkpoints when
// the caller does not keep the forward's.  Some callers cannot hand it any:
// they have no device allocator at hand, or must not call one (cudaMalloc and
// cudaFree can synchronise the whole device, and some runtimes forbid
// allocation after start-up).  For them this entry point takes the scratch
// from a fixed array compiled into the library; every GPU that loads the
// library holds that array until the process exits.

#include <stdio.h>

#include "ssm_internal.h"

namespace {

constexpr size_t kScratchBytes = SSM_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, not a device address: kernels get the address looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch on the current device.  It is looked
// up on every call (a cheap runtime query) rather than cached, so an address
// from an earlier context of this device (after a cudaDeviceReset in the
// caller's process) is never reused.
cudaError_t scratch_address(void **out) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" ssm_status_t ssm_selective_scan_bwd_noalloc(
    const ssm_shape_t *shape, const void *u, const void *delta, const float *A, const void *B,
    const void *C, const float *D, const void *z, const float *delta_bias, int delta_softplus,
    const void *dout, float *du, float *ddelta, float *dA, float *dB, float *dC, float *dD,
    float *dz, float *ddelta_bias, void *stream) {
    size_t need = 0;
    ssm_status_t st = ssm_selective_scan_bwd_scratch_bytes(shape, 0, &need);
    if (st != SSM_OK) return st;
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "ssm_selective_scan_bwd_noalloc: this shape needs %zu bytes of checkpoint "
                 "scratch, more than the %zu-byte static buffer (SSM_NOALLOC_SCRATCH_BYTES)",
                 need, kScratchBytes);
        return ssm::set_last_error(SSM_ERR_UNSUPPORTED, msg);
    }
    void *scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "ssm_selective_scan_bwd_noalloc: scratch lookup failed: %s",
                 cudaGetErrorString(e));
        return ssm::set_last_error(SSM_ERR_CUDA, msg);
    }
    // The state pre-pass writes every checkpoint before the backward reads
    // it, so the previous call's contents need no clearing.
    return ssm_selective_scan_bwd(shape, u, delta, A, B, C, D, z, delta_bias, delta_softplus, dout,
                                  nullptr, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, scratch,
                                  kScratchBytes, stream);
}
