// C ABI of libssmscan.so: argument checking and dispatch to the kernels.
// Every check happens on the host before anything is launched, so a bad call
// returns an error code instead of reaching the GPU.

#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <string>

#include "ssm_internal.h"

// The device error word (see ssm_device_error_status).
__device__ int g_ssm_device_error = 0;

namespace ssm {

int *device_error_word() {
    // Looked up on every call (a cheap runtime query) rather than cached: no
    // lock is needed between host threads, and an address from an earlier
    // context of this device (after a cudaDeviceReset in the caller's
    // process) is never reused.
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ssm_device_error) != cudaSuccess) return nullptr;
    return static_cast<int *>(p);
}

cudaError_t read_and_clear_device_error(int *value, cudaStream_t stream) {
    int *w = device_error_word();
    if (!w) return cudaErrorInvalidDevice;
    cudaError_t e = cudaMemcpyAsync(value, w, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && *value) e = cudaMemsetAsync(w, 0, sizeof(int), stream);
    if (e == cudaSuccess && *value) e = cudaStreamSynchronize(stream);
    return e;
}

}  // namespace ssm

namespace {

thread_local std::string g_last_error;
thread_local const char *g_kernel_path = "";

ssm_status_t fail(ssm_status_t st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
ssm_status_t fail(ssm_status_t st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

ssm_status_t ok() {
    g_last_error.clear();
    return SSM_OK;
}

ssm_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(SSM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool supported_dstate(int n) {
    return n == 1 || n == 2 || n == 4 || n == 8 || n == 16 || n == 32;
}

ssm_status_t check_shape(const ssm_shape_t *s) {
    if (!s) return fail(SSM_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 1 || s->dim < 1 || s->seqlen < 1 || s->dstate < 1)
        return fail(SSM_ERR_INVALID_ARG, "batch, dim, seqlen, dstate must be >= 1 (got %d, %d, %d, %d)",
                    s->batch, s->dim, s->seqlen, s->dstate);
    if (s->io_dtype != SSM_F32 && s->io_dtype != SSM_BF16)
        return fail(SSM_ERR_INVALID_ARG, "io_dtype %d is not SSM_F32 or SSM_BF16", (int)s->io_dtype);
    if ((long long)s->batch * s->dim * s->seqlen >= (1LL << 31))
        return fail(SSM_ERR_UNSUPPORTED, "batch*dim*seqlen must be < 2^31");
    if ((long long)s->batch * s->dstate * s->seqlen >= (1LL << 31))
        return fail(SSM_ERR_UNSUPPORTED, "batch*dstate*seqlen must be < 2^31");
    if (!supported_dstate(s->dstate))
        return fail(SSM_ERR_UNSUPPORTED, "dstate %d not supported (1, 2, 4, 8, 16, 32)", s->dstate);
    return SSM_OK;
}

// A pointer must be device (or managed) memory on the current device, aligned
// to `align` bytes.  Host pointers are refused: handing one to a kernel would
// fault the GPU.
ssm_status_t check_ptr(const void *p, const char *name, size_t align, bool required) {
    if (!p) {
        if (required) return fail(SSM_ERR_INVALID_ARG, "%s is NULL", name);
        return SSM_OK;
    }
    if ((uintptr_t)p % align)
        return fail(SSM_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(SSM_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name, cudaGetErrorName(e));
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return fail(SSM_ERR_INVALID_ARG, "%s is not device memory", name);
    int dev = -1;
    cudaGetDevice(&dev);
    if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
        return fail(SSM_ERR_INVALID_ARG, "%s lives on device %d, current device is %d", name,
                    attr.device, dev);
    return SSM_OK;
}

#define SSM_TRY(expr)                    \
    do {                                 \
        ssm_status_t st_ = (expr);       \
        if (st_ != SSM_OK) return st_;   \
    } while (0)

size_t esize(ssm_dtype_t t) { return t == SSM_BF16 ? 2 : 4; }

int n_ckpt(const ssm_shape_t *s) { return (s->seqlen + SSM_CKPT_CHUNK - 1) / SSM_CKPT_CHUNK; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

ssm_status_t check_options(const ssm_options_t *o) {
    if (!o) return fail(SSM_ERR_INVALID_ARG, "options is NULL");
    if (o->discretization != SSM_DISC_DELTA_B && o->discretization != SSM_DISC_ZOH)
        return fail(SSM_ERR_INVALID_ARG, "discretization %d is not SSM_DISC_DELTA_B or SSM_DISC_ZOH",
                    (int)o->discretization);
    return SSM_OK;
}

}  // namespace

void ssm::set_kernel_path(const char *path) { g_kernel_path = path ? path : ""; }

ssm_status_t ssm::set_last_error(ssm_status_t status, const char *msg) {
    g_last_error = msg ? msg : "";
    return status;
}

extern "C" {

int ssm_version(void) { return 100; }

const char *ssm_last_error_string(void) { return g_last_error.c_str(); }

const char *ssm_last_kernel_path(void) { return g_kernel_path; }

ssm_status_t ssm_selective_scan_ckpt_bytes(const ssm_shape_t *shape, size_t *bytes) {
    SSM_TRY(check_shape(shape));
    if (!bytes) return fail(SSM_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = (size_t)shape->batch * shape->dim * n_ckpt(shape) * shape->dstate * sizeof(float);
    return ok();
}

ssm_status_t ssm_selective_scan_workspace_size(const ssm_shape_t *shape, size_t *ckpt_bytes) {
    return ssm_selective_scan_ckpt_bytes(shape, ckpt_bytes);
}

ssm_status_t ssm_selective_scan_bwd_scratch_bytes(const ssm_shape_t *shape, int have_ckpt,
                                                  size_t *bytes) {
    SSM_TRY(check_shape(shape));
    if (!bytes) return fail(SSM_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = have_ckpt ? 0
                       : (size_t)shape->batch * shape->dim * n_ckpt(shape) * shape->dstate * sizeof(float);
    return ok();
}

}  // extern "C"

namespace {

// The forward behind ssm_selective_scan_fwd_ex and ssm_selective_scan_fwd_segment.
ssm_status_t fwd_impl(const ssm_shape_t *shape, const ssm_options_t *opts, const void *u,
                      const void *delta, const float *A, const void *B, const void *C,
                      const float *D, const void *z, const float *delta_bias, const float *h0,
                      void *out, float *last_state, float *ckpt, float *delta_sum, void *workspace,
                      size_t workspace_bytes, void *stream) {
    SSM_TRY(check_shape(shape));
    SSM_TRY(check_options(opts));
    const size_t es = esize(shape->io_dtype);
    SSM_TRY(check_ptr(u, "u", es, true));
    SSM_TRY(check_ptr(delta, "delta", es, true));
    SSM_TRY(check_ptr(A, "A", 4, true));
    SSM_TRY(check_ptr(B, "B", es, true));
    SSM_TRY(check_ptr(C, "C", es, true));
    SSM_TRY(check_ptr(D, "D", 4, false));
    SSM_TRY(check_ptr(z, "z", es, false));
    SSM_TRY(check_ptr(delta_bias, "delta_bias", 4, false));
    SSM_TRY(check_ptr(h0, "h0", 4, false));
    SSM_TRY(check_ptr(out, "out", es, true));
    SSM_TRY(check_ptr(last_state, "last_state", 4, false));
    SSM_TRY(check_ptr(ckpt, "ckpt", 4, false));
    SSM_TRY(check_ptr(delta_sum, "delta_sum", 4, false));
    if (out == u || out == delta || out == z || out == B || out == C)
        return fail(SSM_ERR_INVALID_ARG, "out may not alias an input");
    if (h0 && (h0 == last_state || (const void *)h0 == (const void *)ckpt))
        return fail(SSM_ERR_INVALID_ARG, "h0 may not alias last_state or ckpt");

    ssm::FwdParams p{};
    p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z;
    p.delta_bias = delta_bias; p.out = out; p.last_state = last_state; p.ckpt = ckpt; p.h0 = h0;
    p.delta_sum = delta_sum;
    p.batch = shape->batch; p.dim = shape->dim; p.L = shape->seqlen; p.N = shape->dstate;
    p.n_ckpt = n_ckpt(shape);
    p.softplus = opts->delta_softplus != 0;
    p.zoh = opts->discretization == SSM_DISC_ZOH;
    p.io_bf16 = shape->io_dtype == SSM_BF16;
    p.vec_ok = ((size_t)shape->seqlen * es) % 16 == 0 && aligned16(u) && aligned16(delta) &&
               aligned16(B) && aligned16(C) && aligned16(out) && (!z || aligned16(z));
    cudaError_t e;
    const size_t need = workspace ? ssm::fwd_chunk_plan(p, nullptr, nullptr) : 0;
    if (need > 0 && ssm::fwd_kernel_choice() == ssm::FwdKernel::kAuto) {
        if (workspace_bytes < need)
            return fail(SSM_ERR_INVALID_ARG, "workspace_bytes %zu < %zu needed for this shape",
                        workspace_bytes, need);
        SSM_TRY(check_ptr(workspace, "workspace", 16, true));
        e = ssm::launch_fwd_chunked(p, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
    } else {
        e = ssm::launch_fwd(p, false, static_cast<cudaStream_t>(stream));
    }
    if (e == cudaErrorNotSupported && ssm::fwd_kernel_choice() == ssm::FwdKernel::kTma)
        return fail(SSM_ERR_UNSUPPORTED,
                    "SSM_FWD_KERNEL=tma: the TMA-fed forward does not cover this shape");
    if (e != cudaSuccess) return cuda_fail(e, "ssm_selective_scan_fwd launch");
    return ok();
}

}  // namespace

extern "C" {

ssm_status_t ssm_selective_scan_fwd_ex(const ssm_shape_t *shape, const ssm_options_t *opts,
                                       const void *u, const void *delta, const float *A,
                                       const void *B, const void *C, const float *D, const void *z,
                                       const float *delta_bias, void *out, float *last_state,
                                       float *ckpt, void *stream) {
    return fwd_impl(shape, opts, u, delta, A, B, C, D, z, delta_bias, nullptr, out, last_state, ckpt,
                    nullptr, nullptr, 0, stream);
}

ssm_status_t ssm_selective_scan_fwd_workspace_bytes(const ssm_shape_t *shape,
                                                    const ssm_options_t *opts, size_t *bytes) {
    SSM_TRY(check_shape(shape));
    SSM_TRY(check_options(opts));
    if (!bytes) return fail(SSM_ERR_INVALID_ARG, "bytes is NULL");
    ssm::FwdParams p{};
    p.batch = shape->batch; p.dim = shape->dim; p.L = shape->seqlen; p.N = shape->dstate;
    p.zoh = opts->discretization == SSM_DISC_ZOH;
    p.io_bf16 = shape->io_dtype == SSM_BF16;
    p.vec_ok = ((size_t)shape->seqlen * esize(shape->io_dtype)) % 16 == 0;
    *bytes = ssm::fwd_chunk_plan(p, nullptr, nullptr);
    return ok();
}

ssm_status_t ssm_selective_scan_fwd_ws(const ssm_shape_t *shape, const ssm_options_t *opts,
                                       const void *u, const void *delta, const float *A,
                                       const void *B, const void *C, const float *D, const void *z,
                                       const float *delta_bias, void *out, float *last_state,
                                       float *ckpt, void *workspace, size_t workspace_bytes,
                                       void *stream) {
    return fwd_impl(shape, opts, u, delta, A, B, C, D, z, delta_bias, nullptr, out, last_state, ckpt,
                    nullptr, workspace, workspace_bytes, stream);
}

ssm_status_t ssm_selective_scan_fwd_segment(const ssm_shape_t *shape, const ssm_options_t *opts,
                                            const void *u, const void *delta, const float *A,
                                            const void *B, const void *C, const float *D,
                                            const void *z, const float *delta_bias, const float *h0,
                                            void *out, float *last_state, float *ckpt,
                                            float *delta_sum, void *stream) {
    return fwd_impl(shape, opts, u, delta, A, B, C, D, z, delta_bias, h0, out, last_state, ckpt,
                    delta_sum, nullptr, 0, stream);
}

ssm_status_t ssm_scan_combine_carries(int nseg, int batch, int dim, int dstate, const float *A,
                                      const float *delta_sums, const float *h_ends, const float *h0,
                                      float *h_in, void *stream) {
    if (nseg < 1 || batch < 1 || dim < 1 || dstate < 1)
        return fail(SSM_ERR_INVALID_ARG, "nseg, batch, dim, dstate must be >= 1");
    const long long P = (long long)batch * dim;
    if ((long long)nseg * P * dstate >= (1LL << 40))
        return fail(SSM_ERR_UNSUPPORTED, "nseg*batch*dim*dstate too large");
    SSM_TRY(check_ptr(A, "A", 4, true));
    SSM_TRY(check_ptr(delta_sums, "delta_sums", 4, true));
    SSM_TRY(check_ptr(h_ends, "h_ends", 4, true));
    SSM_TRY(check_ptr(h0, "h0", 4, false));
    SSM_TRY(check_ptr(h_in, "h_in", 4, true));
    if ((const void *)h_in == (const void *)h_ends || (const void *)h_in == (const void *)delta_sums ||
        (h0 && h_in == h0))
        return fail(SSM_ERR_INVALID_ARG, "h_in may not alias an input");
    cudaError_t e = ssm::launch_combine_carries(nseg, P, dim, dstate, A, delta_sums, h_ends, h0, h_in,
                                                static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ssm_scan_combine_carries launch");
    return ok();
}

ssm_status_t ssm_selective_scan_bwd_ex(const ssm_shape_t *shape, const ssm_options_t *opts,
                                       const void *u, const void *delta, const float *A,
                                       const void *B, const void *C, const float *D, const void *z,
                                       const float *delta_bias, const void *dout, const float *ckpt,
                                       float *du, float *ddelta, float *dA, float *dB, float *dC,
                                       float *dD, float *dz, float *ddelta_bias, void *scratch,
                                       size_t scratch_bytes, void *stream) {
    SSM_TRY(check_shape(shape));
    SSM_TRY(check_options(opts));
    const size_t es = esize(shape->io_dtype);
    SSM_TRY(check_ptr(u, "u", es, true));
    SSM_TRY(check_ptr(delta, "delta", es, true));
    SSM_TRY(check_ptr(A, "A", 4, true));
    SSM_TRY(check_ptr(B, "B", es, true));
    SSM_TRY(check_ptr(C, "C", es, true));
    SSM_TRY(check_ptr(D, "D", 4, false));
    SSM_TRY(check_ptr(z, "z", es, false));
    SSM_TRY(check_ptr(delta_bias, "delta_bias", 4, false));
    SSM_TRY(check_ptr(dout, "dout", es, true));
    SSM_TRY(check_ptr(ckpt, "ckpt", 4, false));
    SSM_TRY(check_ptr(du, "du", 4, true));
    SSM_TRY(check_ptr(ddelta, "ddelta", 4, true));
    SSM_TRY(check_ptr(dA, "dA", 4, true));
    SSM_TRY(check_ptr(dB, "dB", 4, true));
    SSM_TRY(check_ptr(dC, "dC", 4, true));
    SSM_TRY(check_ptr(dD, "dD", 4, D != nullptr));
    SSM_TRY(check_ptr(dz, "dz", 4, z != nullptr));
    SSM_TRY(check_ptr(ddelta_bias, "ddelta_bias", 4, delta_bias != nullptr));
    if (!D && dD) return fail(SSM_ERR_INVALID_ARG, "dD given without D");
    if (!z && dz) return fail(SSM_ERR_INVALID_ARG, "dz given without z");
    if (!delta_bias && ddelta_bias)
        return fail(SSM_ERR_INVALID_ARG, "ddelta_bias given without delta_bias");

    const int nck = n_ckpt(shape);
    const size_t ck_bytes = (size_t)shape->batch * shape->dim * nck * shape->dstate * sizeof(float);
    float *ck = const_cast<float *>(ckpt);
    if (!ckpt) {
        if (scratch_bytes < ck_bytes)
            return fail(SSM_ERR_INVALID_ARG, "scratch_bytes %zu < required %zu (no ckpt given)",
                        scratch_bytes, ck_bytes);
        SSM_TRY(check_ptr(scratch, "scratch", 16, true));
        ck = static_cast<float *>(scratch);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool vec_ok = ((size_t)shape->seqlen * es) % 16 == 0 && aligned16(u) && aligned16(delta) &&
                        aligned16(B) && aligned16(C) && aligned16(dout) && (!z || aligned16(z));
    if (!ckpt) {
        ssm::FwdParams fp{};
        fp.u = u; fp.delta = delta; fp.A = A; fp.B = B; fp.C = C; fp.D = D; fp.z = z;
        fp.delta_bias = delta_bias; fp.out = nullptr; fp.last_state = nullptr; fp.ckpt = ck;
        fp.batch = shape->batch; fp.dim = shape->dim; fp.L = shape->seqlen; fp.N = shape->dstate;
        fp.n_ckpt = nck; fp.softplus = opts->delta_softplus != 0;
        fp.zoh = opts->discretization == SSM_DISC_ZOH;
        fp.io_bf16 = shape->io_dtype == SSM_BF16; fp.vec_ok = vec_ok;
        cudaError_t e = ssm::launch_fwd(fp, true, st);
        if (e != cudaSuccess) return cuda_fail(e, "ssm_selective_scan_bwd state pass");
    }
    // gradients accumulated with atomics start from zero
    const size_t bcl = (size_t)shape->batch * shape->dstate * shape->seqlen * sizeof(float);
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = cudaMemsetAsync(dA, 0, (size_t)shape->dim * shape->dstate * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, bcl, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dC, 0, bcl, st);
    if (e == cudaSuccess && dD) e = cudaMemsetAsync(dD, 0, (size_t)shape->dim * 4, st);
    if (e == cudaSuccess && ddelta_bias) e = cudaMemsetAsync(ddelta_bias, 0, (size_t)shape->dim * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "ssm_selective_scan_bwd memset");

    ssm::BwdParams p{};
    p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z;
    p.delta_bias = delta_bias; p.dout = dout; p.ckpt = ck;
    p.du = du; p.ddelta = ddelta; p.dA = dA; p.dB = dB; p.dC = dC; p.dD = dD; p.dz = dz;
    p.ddelta_bias = ddelta_bias;
    p.batch = shape->batch; p.dim = shape->dim; p.L = shape->seqlen; p.N = shape->dstate;
    p.n_ckpt = nck; p.softplus = opts->delta_softplus != 0;
    p.zoh = opts->discretization == SSM_DISC_ZOH;
    p.io_bf16 = shape->io_dtype == SSM_BF16; p.vec_ok = vec_ok;
    e = ssm::launch_bwd(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "ssm_selective_scan_bwd launch");
    return ok();
}

ssm_status_t ssm_selective_state_update_ex(const ssm_shape_t *shape, const ssm_options_t *opts,
                                           float *state, const void *u, const void *delta,
                                           const float *A, const void *B, const void *C,
                                           const float *D, const void *z, const float *delta_bias,
                                           void *out, void *stream) {
    SSM_TRY(check_shape(shape));
    SSM_TRY(check_options(opts));
    if (shape->seqlen != 1)
        return fail(SSM_ERR_INVALID_ARG, "a single step needs seqlen == 1 (got %d)", shape->seqlen);
    if (shape->batch > 65535)
        return fail(SSM_ERR_UNSUPPORTED, "batch %d > 65535 for a single step", shape->batch);
    const size_t es = esize(shape->io_dtype);
    SSM_TRY(check_ptr(state, "state", 4, true));
    SSM_TRY(check_ptr(u, "u", es, true));
    SSM_TRY(check_ptr(delta, "delta", es, true));
    SSM_TRY(check_ptr(A, "A", 4, true));
    SSM_TRY(check_ptr(B, "B", es, true));
    SSM_TRY(check_ptr(C, "C", es, true));
    SSM_TRY(check_ptr(D, "D", 4, false));
    SSM_TRY(check_ptr(z, "z", es, false));
    SSM_TRY(check_ptr(delta_bias, "delta_bias", 4, false));
    SSM_TRY(check_ptr(out, "out", es, true));
    const void *ins[] = {state, u, delta, A, B, C, D, z, delta_bias};
    for (const void *q : ins)
        if (out == q) return fail(SSM_ERR_INVALID_ARG, "out may not alias an input or the state");
    ssm::StepParams p{};
    p.state = state; p.u = u; p.delta = delta; p.A = A; p.B = B; p.C = C; p.D = D; p.z = z;
    p.delta_bias = delta_bias; p.out = out;
    p.P = (long long)shape->batch * shape->dim; p.dim = shape->dim; p.N = shape->dstate;
    p.softplus = opts->delta_softplus != 0;
    p.zoh = opts->discretization == SSM_DISC_ZOH;
    p.io_bf16 = shape->io_dtype == SSM_BF16;
    p.vec_ok = aligned16(state) && aligned16(A) && aligned16(B) && aligned16(C);
    cudaError_t e = ssm::launch_state_update(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ssm_selective_state_update launch");
    return ok();
}

ssm_status_t ssm_selective_scan_fwd(const ssm_shape_t *shape, const void *u, const void *delta,
                                    const float *A, const void *B, const void *C, const float *D,
                                    const void *z, const float *delta_bias, int delta_softplus,
                                    void *out, float *last_state, float *ckpt, void *stream) {
    const ssm_options_t o = {delta_softplus, SSM_DISC_DELTA_B};
    return ssm_selective_scan_fwd_ex(shape, &o, u, delta, A, B, C, D, z, delta_bias, out,
                                     last_state, ckpt, stream);
}

ssm_status_t ssm_selective_scan_bwd(const ssm_shape_t *shape, const void *u, const void *delta,
                                    const float *A, const void *B, const void *C, const float *D,
                                    const void *z, const float *delta_bias, int delta_softplus,
                                    const void *dout, const float *ckpt, float *du, float *ddelta,
                                    float *dA, float *dB, float *dC, float *dD, float *dz,
                                    float *ddelta_bias, void *scratch, size_t scratch_bytes,
                                    void *stream) {
    const ssm_options_t o = {delta_softplus, SSM_DISC_DELTA_B};
    return ssm_selective_scan_bwd_ex(shape, &o, u, delta, A, B, C, D, z, delta_bias, dout, ckpt,
                                     du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, scratch,
                                     scratch_bytes, stream);
}

ssm_status_t ssm_selective_state_update(const ssm_shape_t *shape, float *state, const void *u,
                                        const void *delta, const float *A, const void *B,
                                        const void *C, const float *D, const void *z,
                                        const float *delta_bias, int delta_softplus, void *out,
                                        void *stream) {
    const ssm_options_t o = {delta_softplus, SSM_DISC_DELTA_B};
    return ssm_selective_state_update_ex(shape, &o, state, u, delta, A, B, C, D, z, delta_bias,
                                         out, stream);
}

ssm_status_t ssm_selection_projections(const ssm_shape_t *shape, int dt_rank, const void *x,
                                       const void *W_x, const void *W_dt, void *dt_low, void *delta,
                                       void *B, void *C, void *stream) {
    if (!shape) return fail(SSM_ERR_INVALID_ARG, "shape is NULL");
    const ssm_shape_t &s = *shape;
    if (s.batch < 1 || s.dim < 1 || s.seqlen < 1 || s.dstate < 1 || dt_rank < 1)
        return fail(SSM_ERR_INVALID_ARG, "batch, dim, seqlen, dstate, dt_rank must be >= 1");
    if (s.io_dtype != SSM_BF16)
        return fail(SSM_ERR_UNSUPPORTED, "the projections take bfloat16 only");
    if (s.seqlen % 8 || s.dim % 8 || dt_rank % 8)
        return fail(SSM_ERR_INVALID_ARG, "seqlen, dim and dt_rank must be multiples of 8 (got %d, %d, %d)",
                    s.seqlen, s.dim, dt_rank);
    if (s.dstate > 64) return fail(SSM_ERR_UNSUPPORTED, "dstate %d > 64", s.dstate);
    if (s.batch > 65535) return fail(SSM_ERR_UNSUPPORTED, "batch %d > 65535", s.batch);
    const long long M1 = dt_rank + 2LL * s.dstate;
    if ((long long)s.batch * s.dim * s.seqlen >= (1LL << 31) ||
        (long long)s.batch * M1 * s.seqlen >= (1LL << 31) || (long long)s.dim * M1 >= (1LL << 31))
        return fail(SSM_ERR_UNSUPPORTED, "tensor sizes must be < 2^31 elements");
    const void *ptrs[] = {x, W_x, W_dt, dt_low, delta, B, C};
    const char *names[] = {"x", "W_x", "W_dt", "dt_low", "delta", "B", "C"};
    for (int i = 0; i < 7; ++i) SSM_TRY(check_ptr(ptrs[i], names[i], 16, true));
    const size_t bytes[] = {
        (size_t)s.batch * s.dim * s.seqlen * 2, (size_t)M1 * s.dim * 2, (size_t)s.dim * dt_rank * 2,
        (size_t)s.batch * dt_rank * s.seqlen * 2, (size_t)s.batch * s.dim * s.seqlen * 2,
        (size_t)s.batch * s.dstate * s.seqlen * 2, (size_t)s.batch * s.dstate * s.seqlen * 2};
    for (int i = 3; i < 7; ++i)          // every output against every other tensor
        for (int j = 0; j < 7; ++j) {
            if (i == j) continue;
            const uintptr_t a0 = (uintptr_t)ptrs[i], a1 = a0 + bytes[i];
            const uintptr_t b0 = (uintptr_t)ptrs[j], b1 = b0 + bytes[j];
            if (a0 < b1 && b0 < a1)
                return fail(SSM_ERR_INVALID_ARG, "%s overlaps %s", names[i], names[j]);
        }
    if (!ssm::tma_available()) return fail(SSM_ERR_UNSUPPORTED, "the driver has no tensor-map encoder");
    const ssm::ProjShape ps{s.batch, s.dim, s.seqlen, s.dstate, dt_rank};
    cudaError_t e = ssm::launch_projections(ps, x, W_x, W_dt, dt_low, delta, B, C,
                                            static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ssm_selection_projections launch");
    return ok();
}

ssm_status_t ssm_device_error_status(void *stream) {
    int v = 0;
    cudaError_t e = ssm::read_and_clear_device_error(&v, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ssm_device_error_status");
    if (v) return fail(SSM_ERR_TIMEOUT, "a bounded wait inside a kernel gave up (code %d)", v);
    return ok();
}

ssm_status_t ssm_check_device_errors(void *stream) { return ssm_device_error_status(stream); }

}  // extern "C"
