// Single-step recurrent update (decoding one token): for each (batch b,
// channel d) the state advances by one time step in place,
//   Δ = softplus(delta + bias[d]),  h[n] ← exp(Δ A[d,n]) h[n] + Δ B[n] u
//   (zero-order hold: (exp(Δ A[d,n]) - 1)/A[d,n] B[n] u in the last term),
//   y = Σ_n C[n] h[n] + D[d] u,     out = y · z σ(z),
// the recurrent form of the selective SSM (정보관리기술사 학습 노트, "상태공간
// 모델(SSM)과 Mamba 아키텍처" §2: h_t = Ā h_{t-1} + B̄ x_t, y_t = C h_t;
// booiljung.github.io "3.2 선택적 스캔(Selective Scan) 알고리즘" §1.1 for the
// selective Δ, B, C).
//
// The step is memory-bound: the fp32 state (4 N bytes per channel) is read
// and written once, everything else is a few bytes per channel.  A group of
// TPC = N / SPT consecutive threads owns one channel, SPT <= 8 states each
// (16-byte vectors, two per thread at SPT = 8), so that a warp's state, A, B
// and C accesses are contiguous; the readout is summed over the group with
// shuffles.

#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

namespace {

// States per thread (at most; a multiple of 4 for vector access).  Eight
// (two threads per channel at N = 16) measured fastest: 14.8 us against 17.3
// with four, for 64 x 5120 x 16.
#ifndef SSM_STEP_SPT
#define SSM_STEP_SPT 8
#endif
constexpr int kStepSpt = SSM_STEP_SPT;

template <typename T, int SPT, bool VEC>
__device__ __forceinline__ void load_io(const T *p, float (&f)[SPT]) {
    if constexpr (VEC && SPT % 4 == 0 && sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < SPT; i += 4) {
            const uint2 q = *reinterpret_cast<const uint2 *>(p + i);
            f[i] = __uint_as_float(q.x << 16); f[i + 1] = __uint_as_float(q.x & 0xffff0000u);
            f[i + 2] = __uint_as_float(q.y << 16); f[i + 3] = __uint_as_float(q.y & 0xffff0000u);
        }
    } else if constexpr (VEC && SPT % 4 == 0 && sizeof(T) == 4) {
#pragma unroll
        for (int i = 0; i < SPT; i += 4) {
            const float4 q = *reinterpret_cast<const float4 *>(p + i);
            f[i] = q.x; f[i + 1] = q.y; f[i + 2] = q.z; f[i + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < SPT; ++i) f[i] = IO<T>::to_f(p[i]);
    }
}

// Channels per thread: all loads of the CPT channels are issued before any
// arithmetic.  One channel per thread (shorter threads, more of them
// resident) measured fastest with eight states per thread.
#ifndef SSM_STEP_CPT
#define SSM_STEP_CPT 1
#endif
#ifndef SSM_STEP_BLOCK
#define SSM_STEP_BLOCK 128
#endif
#ifndef SSM_STEP_MIN_BLOCKS
#define SSM_STEP_MIN_BLOCKS 1
#endif
constexpr int kStepBlock = SSM_STEP_BLOCK, kStepMinBlocks = SSM_STEP_MIN_BLOCKS;
constexpr int kStepCpt = SSM_STEP_CPT;

template <typename T, int N, bool VEC>
__global__ void __launch_bounds__(kStepBlock, kStepMinBlocks) state_update_kernel(const StepParams p) {
    constexpr int SPT = N < kStepSpt ? N : kStepSpt;   // states per thread
    constexpr int TPC = N / SPT;           // threads per channel (a power of two)
    constexpr int CPT = kStepCpt;
    // grid: x covers the channels of one batch row (CPT per thread group,
    // strided by the x extent), y is the batch row
    const unsigned b = blockIdx.y;
    const unsigned t = blockIdx.x * blockDim.x + threadIdx.x;
    const unsigned stride = gridDim.x * blockDim.x / TPC;
    const unsigned dim = (unsigned)p.dim;
    const int q = (int)(t % TPC);

    float h[CPT][SPT], a2[CPT][SPT], bb[SPT], cc[SPT];
    float u[CPT], r[CPT], zz[CPT];
    unsigned ds[CPT];
    bool oks[CPT];
    load_io<T, SPT, VEC>(static_cast<const T *>(p.B) + b * N + q * SPT, bb);
    load_io<T, SPT, VEC>(static_cast<const T *>(p.C) + b * N + q * SPT, cc);
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
        const unsigned d_raw = t / TPC + k * stride;
        oks[k] = d_raw < dim;
        const unsigned d = oks[k] ? d_raw : dim - 1;   // out-of-range groups mirror the last channel
        ds[k] = d;
        const unsigned ch = b * dim + d;
        const float *st = p.state + (size_t)ch * N + q * SPT;   // batch * dim * N may exceed 2^32
        const float *ar = p.A + (size_t)d * N + q * SPT;
        if constexpr (VEC && SPT % 4 == 0) {
#pragma unroll
            for (int i = 0; i < SPT; i += 4) {
                const float4 hv = *reinterpret_cast<const float4 *>(st + i);
                const float4 av = __ldg(reinterpret_cast<const float4 *>(ar + i));
                h[k][i] = hv.x; h[k][i + 1] = hv.y; h[k][i + 2] = hv.z; h[k][i + 3] = hv.w;
                a2[k][i] = av.x; a2[k][i + 1] = av.y; a2[k][i + 2] = av.z; a2[k][i + 3] = av.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < SPT; ++i) { h[k][i] = st[i]; a2[k][i] = __ldg(ar + i); }
        }
        u[k] = IO<T>::to_f(static_cast<const T *>(p.u)[ch]);
        r[k] = IO<T>::to_f(static_cast<const T *>(p.delta)[ch]) + (p.delta_bias ? p.delta_bias[d] : 0.f);
        zz[k] = p.z ? IO<T>::to_f(static_cast<const T *>(p.z)[ch]) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
        const float dt = p.softplus ? softplus_fast(r[k]) : r[k];
        const float du = dt * u[k];
        float y = 0.f;
#pragma unroll
        for (int i = 0; i < SPT; ++i) {
            const float a = ex2(dt * (a2[k][i] * SSM_LOG2E));
            const float coef = p.zoh ? zoh_phi(dt * a2[k][i], a) * du : du;   // B̄ u / B
            h[k][i] = fmaf(a, h[k][i], coef * bb[i]);
            y = fmaf(cc[i], h[k][i], y);
        }
#pragma unroll
        for (int m = TPC / 2; m >= 1; m >>= 1) y += __shfl_xor_sync(0xffffffffu, y, m);
        if (!oks[k]) continue;
        const unsigned ch = b * dim + ds[k];
        float *st = p.state + (size_t)ch * N + q * SPT;
        if constexpr (VEC && SPT % 4 == 0) {
#pragma unroll
            for (int i = 0; i < SPT; i += 4)
                *reinterpret_cast<float4 *>(st + i) = make_float4(h[k][i], h[k][i + 1], h[k][i + 2], h[k][i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < SPT; ++i) st[i] = h[k][i];
        }
        if (q == 0) {
            y = fmaf(p.D ? p.D[ds[k]] : 0.f, u[k], y);
            if (p.z) y *= zz[k] * sigmoid(zz[k]);
            static_cast<T *>(p.out)[ch] = IO<T>::from_f(y);
        }
    }
}

template <typename T, int N>
cudaError_t launch_step_n(const StepParams &p, cudaStream_t stream) {
    constexpr int SPT = N < kStepSpt ? N : kStepSpt;
    constexpr int TPC = N / SPT;
    const int block = kStepBlock;
    const long long groups = ((long long)p.dim + kStepCpt - 1) / kStepCpt;
    const long long gx = (groups * TPC + block - 1) / block;
    const long long batch = p.P / p.dim;
    if (gx > 0x7fffffffLL || batch > 65535) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)gx, (unsigned)batch);
    if (p.vec_ok) state_update_kernel<T, N, true><<<grid, block, 0, stream>>>(p);
    else state_update_kernel<T, N, false><<<grid, block, 0, stream>>>(p);
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
