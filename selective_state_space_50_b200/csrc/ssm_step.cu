// Single-step recurrent update (decoding one token): for each (batch b,
// channel d) the state advances by one time step in place,
//   Δ = softplus(delta + bias[d]),  h[n] ← exp(Δ A[d,n]) h[n] + Δ B[n] u,
//   y = Σ_n C[n] h[n] + D[d] u,     out = y · z σ(z),
// the recurrent form of the selective SSM (정보관리기술사 학습 노트, "상태공간
// 모델(SSM)과 Mamba 아키텍처" §2: h_t = Ā h_{t-1} + B̄ x_t, y_t = C h_t;
// booiljung.github.io "3.2 선택적 스캔(Selective Scan) 알고리즘" §1.1 for the
// selective Δ, B, C).
//
// The step is memory-bound: the fp32 state (4 N bytes per channel) is read
// and written once, everything else is a few bytes per channel.  A group of
// TPC = N / SPT consecutive threads owns one channel, SPT <= 4 states each, so
// that a warp's state, A, B and C accesses are contiguous 16-byte vectors;
// the readout is summed over the group with shuffles.

#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

namespace {

template <typename T, int SPT>
__device__ __forceinline__ void load_io(const T *p, float (&f)[SPT]) {
#pragma unroll
    for (int i = 0; i < SPT; ++i) f[i] = IO<T>::to_f(p[i]);
}

template <typename T, int N, bool VEC>
__global__ void __launch_bounds__(256) state_update_kernel(const StepParams p) {
    constexpr int SPT = N < 4 ? N : 4;     // states per thread
    constexpr int TPC = N / SPT;           // threads per channel (a power of two, <= 8)
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long ch_raw = gid / TPC;
    const int q = (int)(gid % TPC);
    const bool ok = ch_raw < p.P;
    const long long ch = ok ? ch_raw : p.P - 1;   // out-of-range threads mirror the last channel
    const int b = (int)(ch / p.dim), d = (int)(ch % p.dim);

    float h[SPT], a2[SPT], bb[SPT], cc[SPT];
    float *st = p.state + ch * N + q * SPT;
    const float *ar = p.A + (size_t)d * N + q * SPT;
    if constexpr (VEC && SPT == 4) {
        const float4 hv = *reinterpret_cast<const float4 *>(st);
        const float4 av = __ldg(reinterpret_cast<const float4 *>(ar));
        h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
        a2[0] = av.x; a2[1] = av.y; a2[2] = av.z; a2[3] = av.w;
    } else {
#pragma unroll
        for (int i = 0; i < SPT; ++i) { h[i] = st[i]; a2[i] = __ldg(ar + i); }
    }
    const T *Bp = static_cast<const T *>(p.B) + (size_t)b * N + q * SPT;
    const T *Cp = static_cast<const T *>(p.C) + (size_t)b * N + q * SPT;
    load_io<T, SPT>(Bp, bb);
    load_io<T, SPT>(Cp, cc);

    const float u = IO<T>::to_f(static_cast<const T *>(p.u)[ch]);
    const float r = IO<T>::to_f(static_cast<const T *>(p.delta)[ch]) + (p.delta_bias ? p.delta_bias[d] : 0.f);
    const float dt = p.softplus ? softplus_fast(r) : r;
    const float du = dt * u;
    float y = 0.f;
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
        const float a = ex2(dt * (a2[i] * SSM_LOG2E));
        h[i] = fmaf(a, h[i], du * bb[i]);
        y = fmaf(cc[i], h[i], y);
    }
#pragma unroll
    for (int m = TPC / 2; m >= 1; m >>= 1) y += __shfl_xor_sync(0xffffffffu, y, m);
    if (!ok) return;
    if constexpr (VEC && SPT == 4) {
        *reinterpret_cast<float4 *>(st) = make_float4(h[0], h[1], h[2], h[3]);
    } else {
#pragma unroll
        for (int i = 0; i < SPT; ++i) st[i] = h[i];
    }
    if (q == 0) {
        y = fmaf(p.D ? p.D[d] : 0.f, u, y);
        if (p.z) {
            const float z = IO<T>::to_f(static_cast<const T *>(p.z)[ch]);
            y *= z * sigmoid(z);
        }
        static_cast<T *>(p.out)[ch] = IO<T>::from_f(y);
    }
}

template <typename T, int N>
cudaError_t launch_step_n(const StepParams &p, cudaStream_t stream) {
    constexpr int SPT = N < 4 ? N : 4;
    constexpr int TPC = N / SPT;
    const long long threads = p.P * TPC;
    const int block = 256;
    const long long grid = (threads + block - 1) / block;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (p.vec_ok) state_update_kernel<T, N, true><<<(unsigned)grid, block, 0, stream>>>(p);
    else state_update_kernel<T, N, false><<<(unsigned)grid, block, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_step_t(const StepParams &p, cudaStream_t stream) {
    switch (p.N) {
    case 1: return launch_step_n<T, 1>(p, stream);
    case 2: return launch_step_n<T, 2>(p, stream);
    case 4: return launch_step_n<T, 4>(p, stream);
    case 8: return launch_step_n<T, 8>(p, stream);
    case 16: return launch_step_n<T, 16>(p, stream);
    case 32: return launch_step_n<T, 32>(p, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_state_update(const StepParams &p, cudaStream_t stream) {
    if (p.P <= 0) return cudaSuccess;
    return p.io_bf16 ? launch_step_t<__nv_bfloat16>(p, stream) : launch_step_t<float>(p, stream);
}

}  // namespace ssm
