// Internal launch interface between the C ABI (ssm_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
    const float *h0;  // [batch][dim][N] state before step 0; NULL: zeros
    float *delta_sum; // [batch][dim] Σ_t Δ_t, or NULL (sequence segments)
    int batch, dim, L, N, n_ckpt;
    int softplus;
    int zoh;      // zero-order-hold B̄ (general kernels only)
    bool io_bf16;
    bool vec_ok;  // every [.., L] row starts 16-byte aligned
    // Two-level scan along L (TMA forward only): K time chunks of Lc steps
    // (K <= 1: one pass over the whole sequence), `virt` bits as in the
    // kernel (1: h0 per chunk and row; 2: last_state / delta_sum per chunk
    // and row), `summary`: chunk summaries only (end state from h = 0 and
    // Σ Δ; no output).
    int K, Lc, virt;
    bool summary;
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
    int zoh;      // zero-order-hold B̄ (general kernel only)
    bool io_bf16;
    bool vec_ok;
};

struct StepParams {
    float *state;                  // [batch][dim][N], updated in place
    const void *u, *delta;         // [batch][dim]
    const float *A;                // [dim][N]
    const void *B, *C;             // [batch][N]
    const float *D;
    const void *z;
    const float *delta_bias;
    void *out;                     // [batch][dim]
    long long P;                   // batch * dim
    int dim, N;
    int softplus;
    int zoh;                       // zero-order-hold B̄
    bool io_bf16;
    bool vec_ok;                   // state, A, B, C 16-byte aligned (vector access)
};

// Selection projections (ssm_proj.cu): x_proj then dt_proj on the tensor
// cores, bf16 in and out.
struct ProjShape {
    int batch, dim, seqlen, dstate, dt_rank;
};
cudaError_t launch_projections(const ProjShape &s, const void *x, const void *W_x, const void *W_dt,
                               void *dt_low, void *delta, void *B, void *C, cudaStream_t stream);

// Sequence segments (ssm_seg.cu).  delta_sum[b][d] = Σ_t Δ_t over the
// segment; combine_carries turns per-segment (Σ Δ, end state) pairs into the
// state entering each segment.
cudaError_t launch_delta_sum(const FwdParams &p, float *delta_sum, cudaStream_t stream);
cudaError_t launch_combine_carries(int nseg, long long P, int dim, int N, const float *A,
                                   const float *dsums, const float *h_ends, const float *h0,
                                   float *h_in, cudaStream_t stream);

// Single-step recurrent update (ssm_step.cu).
cudaError_t launch_state_update(const StepParams &p, cudaStream_t stream);

enum class FwdKernel { kAuto = 0, kGeneral = 1, kTma = 2 };
FwdKernel fwd_kernel_choice();

cudaError_t launch_fwd(const FwdParams &p, bool states_only, cudaStream_t stream);
// The chunked two-level forward for long sequences over few channel rows:
// fwd_chunk_plan returns the workspace bytes it needs (0: the shape is better
// served by one pass), launch_fwd_chunked runs it (summaries, carry combine,
// full pass from the carries) in `ws`.
size_t fwd_chunk_plan(const FwdParams &p, int *K, int *Lc);
cudaError_t launch_fwd_chunked(const FwdParams &p, void *ws, size_t ws_bytes, cudaStream_t stream);
// Launches the TMA-fed persistent forward when it applies (returns true and
// sets *err); returns false when the general kernel must be used.
bool try_launch_fwd_tma(const FwdParams &p, cudaStream_t stream, cudaError_t *err);
// Records which kernels the last launch on this thread used (the string
// behind ssm_last_kernel_path; a static string literal).
void set_kernel_path(const char *path);

// Records `msg` as this thread's last error (ssm_last_error_string) and
// returns `status`.
ssm_status_t set_last_error(ssm_status_t status, const char *msg);

// Device address of the error word that kernels set when a bounded wait
// gives up (one word per device, looked up on every call); NULL on failure.
int *device_error_word();
// Copies the device error word to *value (after synchronising `stream`) and
// clears it when set.
cudaError_t read_and_clear_device_error(int *value, cudaStream_t stream);
cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream);

// TMA host helpers (ssm_tma_host.cu).  tma_available() is false when the
// driver does not expose the tensor-map encoder.  make_tma_map_2d describes a
// row-major [rows x cols] bf16 or fp32 array with a [box_rows x box_cols] box
// (128-byte swizzle on request).  device_sm_count() caches per device.
bool tma_available();
bool make_tma_map_2d(CUtensorMap *m, const void *base, bool bf16, uint64_t rows, uint64_t cols,
                     uint32_t box_cols, uint32_t box_rows, bool swizzle128);
// make_tma_map_bf16_3d: a bf16 tensor of extents {d0 (contiguous), d1, d2},
// tiles of {box0, box1, 1} with the 128-byte swizzle; out-of-range elements
// of a tile read 0.
bool make_tma_map_bf16_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                          uint32_t box0, uint32_t box1);
int device_sm_count();
// Launches the TMA-fed persistent backward when it applies (dstate 16, 16-byte
// aligned rows and checkpoints, at least one channel row per SM); returns
// false when the general backward must be used.  SSM_BWD_KERNEL=general in
// the environment disables it.
bool try_launch_bwd_tma(const BwdParams &p, cudaStream_t stream, cudaError_t *err);

}  // namespace ssm
