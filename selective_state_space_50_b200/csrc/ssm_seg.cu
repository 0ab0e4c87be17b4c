// Sequence segments: the two small kernels that let a sequence be scanned in
// pieces (one piece per GPU, or several in turn on one GPU).
//
// The pieces are reassembled with the associative operator of the two-level
// scan (booiljung.github.io, "3.2 선택적 스캔(Selective Scan) 알고리즘", §2.2:
// (a_j, b_j) • (a_i, b_i) = (a_j a_i, a_j b_i + b_j)).  A segment run from a
// zero state ends in state e; its decay product over the segment is
// prod_t exp(Δ_t A) = exp(A Σ_t Δ_t), so the segment is summarised by
// (Σ_t Δ_t, e) per channel, and the state entering segment s + 1 is
// exp(A Σ Δ_s) h_in(s) + e_s.
//
//  * delta_sum_kernel: Σ_t Δ_t per (batch, channel) of one segment, with the
//    scan's own Δ = softplus(delta + bias) (one warp per channel row), after
//    the general forward kernel.  The TMA forward sums Δ itself, in the same
//    pass that forms it.
//  * combine_kernel: the exclusive scan of the summaries across segments,
//    one thread per (channel row, state).

#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

namespace {

template <typename T>
__global__ void __launch_bounds__(256) delta_sum_kernel(const T *__restrict__ delta,
                                                        const float *__restrict__ bias, long long P,
                                                        int dim, int L, int softplus, bool vec_ok,
                                                        float *__restrict__ out) {
    constexpr int V = IO<T>::kVec;
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (row >= P) return;
    const float b = bias ? bias[row % dim] : 0.f;
    const T *src = delta + row * (long long)L;
    float acc = 0.f;
    for (int i = lane * V; i < L; i += 32 * V) {
        float v[V];
        if (vec_ok && i + V <= L) {
            IO<T>::unpack(*reinterpret_cast<const uint4 *>(src + i), v);
        } else {
#pragma unroll
            for (int e = 0; e < V; ++e) v[e] = (i + e < L) ? IO<T>::to_f(src[i + e]) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < V; ++e) {
            if (i + e < L) {
                const float r = v[e] + b;
                acc += softplus ? softplus_fast(r) : r;
            }
        }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (lane == 0) out[row] = acc;
}

__global__ void __launch_bounds__(256) combine_kernel(int nseg, long long P, int dim, int N,
                                                      const float *__restrict__ A,
                                                      const float *__restrict__ dsums,
                                                      const float *__restrict__ h_ends,
                                                      const float *__restrict__ h0,
                                                      float *__restrict__ h_in) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // (row, n)
    if (i >= P * N) return;
    const long long row = i / N;
    const int n = (int)(i % N);
    const float a2 = A[(long long)(row % dim) * N + n] * SSM_LOG2E;
    float h = h0 ? h0[i] : 0.f;
    for (int s = 0; s < nseg; ++s) {
        h_in[(long long)s * P * N + i] = h;
        // the last segment's summary is not needed (and may be absent)
        if (s + 1 < nseg)
            h = fmaf(exp2f(a2 * dsums[(long long)s * P + row]), h, h_ends[(long long)s * P * N + i]);
    }
}

}  // namespace

cudaError_t launch_delta_sum(const FwdParams &p, float *delta_sum, cudaStream_t stream) {
    const long long P = (long long)p.batch * p.dim;
    if (P <= 0) return cudaSuccess;
    const int warps = 8;
    const long long blocks = (P + warps - 1) / warps;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (p.io_bf16)
        delta_sum_kernel<__nv_bfloat16><<<(unsigned)blocks, warps * 32, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(p.delta), p.delta_bias, P, p.dim, p.L, p.softplus,
            p.vec_ok, delta_sum);
    else
        delta_sum_kernel<float><<<(unsigned)blocks, warps * 32, 0, stream>>>(
            static_cast<const float *>(p.delta), p.delta_bias, P, p.dim, p.L, p.softplus, p.vec_ok,
            delta_sum);
    return cudaGetLastError();
}

cudaError_t launch_combine_carries(int nseg, long long P, int dim, int N, const float *A,
                                   const float *dsums, const float *h_ends, const float *h0,
                                   float *h_in, cudaStream_t stream) {
    const long long n = P * N;
    if (n <= 0 || nseg <= 0) return cudaSuccess;
    const long long blocks = (n + 255) / 256;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    combine_kernel<<<(unsigned)blocks, 256, 0, stream>>>(nseg, P, dim, N, A, dsums, h_ends, h0, h_in);
    return cudaGetLastError();
}

}  // namespace ssm
