// Forward selective scan (S6) for sm_100a.
//
// Computes, per batch row b and channel d (booiljung.github.io "3.2 선택적
// 스캔(Selective Scan) 알고리즘" §1.1/§1.2/§2.1; 정보관리기술사 학습 노트
// "상태공간 모델(SSM)과 Mamba 아키텍처" §3):
//   Δ_t = softplus(delta_t + bias[d]);  Ā_t[n] = exp(Δ_t A[d,n])
//   h_t[n] = Ā_t[n] h_{t-1}[n] + Δ_t B_t[n] u_t;  y_t = Σ_n C_t[n] h_t[n] + D[d] u_t
//   out_t = y_t · silu(z_t)
//
// Design (fused as in §3.2 of the scan page: only y, the final state and the
// optional checkpoints reach HBM):
//  * A CTA owns one batch row b and G channels and walks the whole sequence
//    in tiles of TT steps.  Lane (c, g) owns channel c and the NS states
//    g*NS .. g*NS+NS-1 (NT = N / NS lanes per channel) and keeps them in fp32
//    registers for the whole sequence; the recurrence itself runs
//    sequentially inside the lane, so no scan-combine work is spent.
//  * Per tile: (1) all threads stage the tile through shared memory with
//    16-byte coalesced loads, computing Δ (softplus) and Δ·u once per element;
//    B and C (shared by every channel of the row) are staged transposed,
//    [t][n], so a lane reads its NS states with one vector load.
//    (2) Each lane runs its recurrence over the TT steps: one ex2 per
//    (step, state) on A pre-scaled by log2(e), two FMAs, and its partial
//    readout Σ_{own n} C h goes to shared memory.  (3) A fused epilogue sums
//    the NT partials, adds D·u, applies the SiLU gate and stores y with
//    16-byte stores.
//  * Steps past the end of the sequence are staged as Δ = 0, so they leave
//    the state unchanged (Ā = 1, no input) and nothing is stored for them.

#include <stdlib.h>
#include <string.h>

#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

// SSM_FWD_KERNEL=general|tma|auto (default auto) selects the forward kernel:
// "tma" fails with cudaErrorNotSupported where the TMA kernel does not apply.
FwdKernel fwd_kernel_choice() {
    static int cached = -1;
    if (cached < 0) {
        const char *e = getenv("SSM_FWD_KERNEL");
        cached = (e && !strcmp(e, "general")) ? (int)FwdKernel::kGeneral
                 : (e && !strcmp(e, "tma"))   ? (int)FwdKernel::kTma
                                              : (int)FwdKernel::kAuto;
    }
    return (FwdKernel)cached;
}

template <typename T, int NT, int NS, int G, int TT>
struct FwdSmem {
    static constexpr int N = NT * NS;
    static constexpr int RS = TT + 4;   // row stride of per-channel tiles (floats)
    static constexpr int NSB = N + 4;   // row stride of the [t][n] B/C tiles
    static constexpr int kDt = 0;
    static constexpr int kDu = kDt + G * RS;
    static constexpr int kU = kDu + G * RS;
    static constexpr int kZ = kU + G * RS;
    static constexpr int kB = kZ + G * RS;
    static constexpr int kC = kB + TT * NSB;
    static constexpr int kY = kC + TT * NSB;
    static constexpr int kTotal = kY + NT * G * RS;
    static constexpr size_t bytes = sizeof(float) * kTotal;
};

// MODE 0: full forward.  MODE 1: states only (writes ckpt / last_state, no
// readout), used by the backward when no checkpoints were given.  ZOH: the
// zero-order-hold input matrix B̄ = φ(ΔA) Δ B (zoh_phi) instead of Δ B.
template <typename T, int NT, int NS, int G, int TT, int MODE, bool ZOH>
__global__ void __launch_bounds__(NT * G)
fwd_kernel(const FwdParams p) {
    using S = FwdSmem<T, NT, NS, G, TT>;
    constexpr int N = S::N;
    constexpr int RS = S::RS;
    constexpr int NSB = S::NSB;
    constexpr int NTHR = NT * G;
    constexpr int V = IO<T>::kVec;
    constexpr int VPR = TT / V;
    static_assert(TT % V == 0 && TT % 4 == 0, "tile must hold whole vectors");
    static_assert(TT % SSM_CKPT_CHUNK == 0 && SSM_CKPT_CHUNK % 4 == 0, "checkpoint grid");

    extern __shared__ __align__(16) float smem[];
    float *sDt = smem + S::kDt, *sDu = smem + S::kDu, *sU = smem + S::kU, *sZ = smem + S::kZ;
    float *sB = smem + S::kB, *sC = smem + S::kC, *sY = smem + S::kY;

    const int tid = threadIdx.x;
    const int g = tid % NT;   // state group of this lane
    const int c = tid / NT;   // channel of this lane within the CTA
    const int b = blockIdx.y;
    const int d0 = blockIdx.x * G;
    const int d = d0 + c;
    const bool live = d < p.dim;
    const int L = p.L;

    const T *u = static_cast<const T *>(p.u);
    const T *delta = static_cast<const T *>(p.delta);
    const T *z = static_cast<const T *>(p.z);
    const T *Bm = static_cast<const T *>(p.B);
    const T *Cm = static_cast<const T *>(p.C);

    float A2[NS], h[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        A2[s] = live ? p.A[(size_t)d * N + g * NS + s] * SSM_LOG2E : 0.f;
        h[s] = (live && p.h0) ? p.h0[((size_t)b * p.dim + d) * N + g * NS + s] : 0.f;
    }

    const size_t row_bd0 = (size_t)b * p.dim;

    for (int t0 = 0; t0 < L; t0 += TT) {
        const int nvalid = min(TT, L - t0);
        // ---------------- (1) stage the tile
        for (int v = tid; v < G * VPR; v += NTHR) {
            const int cc = v / VPR, j = (v % VPR) * V;
            const int dd = d0 + cc;
            float dr[V], uu[V], zz[V];
            const int n_in = nvalid - j;
            if (dd < p.dim) {
                const size_t off = (row_bd0 + dd) * (size_t)L + t0 + j;
                const float bias = p.delta_bias ? p.delta_bias[dd] : 0.f;
                load_vec_stream(delta + off, n_in, p.vec_ok, 0.f, dr);
                load_vec_stream(u + off, n_in, p.vec_ok, 0.f, uu);
                if (MODE == 0 && z) load_vec_stream(z + off, n_in, p.vec_ok, 0.f, zz);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    float r = dr[i] + bias;
                    float dt = p.softplus ? softplus_fast(r) : r;
                    dr[i] = (i < n_in) ? dt : 0.f;
                }
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) dr[i] = uu[i] = 0.f;
            }
            float *rowDt = sDt + cc * RS + j, *rowDu = sDu + cc * RS + j;
#pragma unroll
            for (int i = 0; i < V; i += 4) {
                *reinterpret_cast<float4 *>(rowDt + i) = make_float4(dr[i], dr[i + 1], dr[i + 2], dr[i + 3]);
                *reinterpret_cast<float4 *>(rowDu + i) =
                    make_float4(dr[i] * uu[i], dr[i + 1] * uu[i + 1], dr[i + 2] * uu[i + 2], dr[i + 3] * uu[i + 3]);
                if (MODE == 0) {
                    *reinterpret_cast<float4 *>(sU + cc * RS + j + i) = make_float4(uu[i], uu[i + 1], uu[i + 2], uu[i + 3]);
                    if (z)
                        *reinterpret_cast<float4 *>(sZ + cc * RS + j + i) = make_float4(zz[i], zz[i + 1], zz[i + 2], zz[i + 3]);
                }
            }
        }
        for (int v = tid; v < N * VPR; v += NTHR) {
            const int n = v / VPR, j = (v % VPR) * V;
            const size_t off = ((size_t)b * N + n) * (size_t)L + t0 + j;
            float bb[V], cv[V];
            load_vec(Bm + off, nvalid - j, p.vec_ok, 0.f, bb);
            if (MODE == 0) load_vec(Cm + off, nvalid - j, p.vec_ok, 0.f, cv);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                sB[(j + i) * NSB + n] = bb[i];
                if (MODE == 0) sC[(j + i) * NSB + n] = cv[i];
            }
        }
        __syncthreads();

        // ---------------- (2) the recurrence, NS states per lane
        const float *rowDt = sDt + c * RS, *rowDu = sDu + c * RS;
#pragma unroll 2
        for (int t = 0; t < TT; t += 4) {
            const float4 dt4 = *reinterpret_cast<const float4 *>(rowDt + t);
            const float4 du4 = *reinterpret_cast<const float4 *>(rowDu + t);
            const float dts[4] = {dt4.x, dt4.y, dt4.z, dt4.w};
            const float dus[4] = {du4.x, du4.y, du4.z, du4.w};
            float yv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float *bp = sB + (t + i) * NSB + g * NS;
                const float *cp = sC + (t + i) * NSB + g * NS;
                float bv[NS], cv[NS];
                if constexpr (NS % 4 == 0) {
#pragma unroll
                    for (int s = 0; s < NS; s += 4) {
                        const float4 q = *reinterpret_cast<const float4 *>(bp + s);
                        bv[s] = q.x; bv[s + 1] = q.y; bv[s + 2] = q.z; bv[s + 3] = q.w;
                        if (MODE == 0) {
                            const float4 r = *reinterpret_cast<const float4 *>(cp + s);
                            cv[s] = r.x; cv[s + 1] = r.y; cv[s + 2] = r.z; cv[s + 3] = r.w;
                        }
                    }
                } else {
#pragma unroll
                    for (int s = 0; s < NS; ++s) {
                        bv[s] = bp[s];
                        if (MODE == 0) cv[s] = cp[s];
                    }
                }
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                    const float arg = dts[i] * A2[s];
                    const float a = ex2(arg);
                    const float k = ZOH ? zoh_phi(arg * 0.69314718f, a) * dus[i] : dus[i];
                    h[s] = fmaf(a, h[s], k * bv[s]);
                    if (MODE == 0) acc = fmaf(cv[s], h[s], acc);
                }
                yv[i] = acc;
            }
            if (MODE == 0)
                *reinterpret_cast<float4 *>(sY + (g * G + c) * RS + t) = make_float4(yv[0], yv[1], yv[2], yv[3]);
            // checkpoint: state at the end of chunk k (steps past L leave it unchanged)
            if (p.ckpt && live && (t + 4) % SSM_CKPT_CHUNK == 0) {
                const int k = (t0 + t + 4) / SSM_CKPT_CHUNK - 1;
                if (k * SSM_CKPT_CHUNK < L) {
                    float *dst = p.ckpt + (((row_bd0 + d) * p.n_ckpt + k) * N + g * NS);
#pragma unroll
                    for (int s = 0; s < NS; ++s) dst[s] = h[s];
                }
            }
        }

        __syncthreads();

        // ---------------- (3) epilogue: Σ partials, D skip, gate, store
        if (MODE == 0) {
            T *out = static_cast<T *>(p.out);
            for (int v = tid; v < G * VPR; v += NTHR) {
                const int cc = v / VPR, j = (v % VPR) * V;
                const int dd = d0 + cc;
                if (dd >= p.dim || j >= nvalid) continue;
                float y[V];
#pragma unroll
                for (int i = 0; i < V; i += 4) {
                    float4 acc = *reinterpret_cast<const float4 *>(sY + cc * RS + j + i);
#pragma unroll
                    for (int gg = 1; gg < NT; ++gg) {
                        const float4 q = *reinterpret_cast<const float4 *>(sY + (gg * G + cc) * RS + j + i);
                        acc.x += q.x; acc.y += q.y; acc.z += q.z; acc.w += q.w;
                    }
                    y[i] = acc.x; y[i + 1] = acc.y; y[i + 2] = acc.z; y[i + 3] = acc.w;
                }
                const float Dd = p.D ? p.D[dd] : 0.f;
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    float yy = fmaf(Dd, sU[cc * RS + j + i], y[i]);
                    if (z) {
                        const float zz = sZ[cc * RS + j + i];
                        if constexpr (sizeof(T) == 2) yy *= silu_tanh(zz);
                        else yy *= zz * sigmoid(zz);
                    }
                    y[i] = yy;
                }
                const size_t off = (row_bd0 + dd) * (size_t)L + t0 + j;
                store_vec(out + off, nvalid - j, p.vec_ok, y);
            }
            __syncthreads();
        }
    }

    if (p.last_state && live) {
        float *dst = p.last_state + (row_bd0 + d) * N + g * NS;
#pragma unroll
        for (int s = 0; s < NS; ++s) dst[s] = h[s];
    }
}

// ---------------------------------------------------------------- launch

template <typename T, int NT, int NS, int G, int TT, int MODE, bool ZOH>
static cudaError_t launch_fwd_cfg(const FwdParams &p, cudaStream_t stream) {
    using S = FwdSmem<T, NT, NS, G, TT>;
    auto kern = fwd_kernel<T, NT, NS, G, TT, MODE, ZOH>;
    static bool attr_done = false;  // per instance; benign race (idempotent)
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)S::bytes);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    dim3 grid((p.dim + G - 1) / G, p.batch);
    kern<<<grid, NT * G, S::bytes, stream>>>(p);
    return cudaGetLastError();
}

// Picks the lane split for dstate N.  With few (b, d) pairs (long sequences,
// small batch) every state gets its own lane to keep enough warps resident.
template <typename T, int MODE, bool ZOH>
static cudaError_t launch_fwd_tz(const FwdParams &p, cudaStream_t stream) {
    const long pairs = (long)p.batch * p.dim;
    const bool few = pairs < 4096;
    constexpr int TT = 32;
    switch (p.N) {
    case 1: return launch_fwd_cfg<T, 1, 1, 128, TT, MODE, ZOH>(p, stream);
    case 2: return launch_fwd_cfg<T, 1, 2, 128, TT, MODE, ZOH>(p, stream);
    case 4: return few ? launch_fwd_cfg<T, 4, 1, 32, TT, MODE, ZOH>(p, stream)
                       : launch_fwd_cfg<T, 1, 4, 128, TT, MODE, ZOH>(p, stream);
    case 8: return few ? launch_fwd_cfg<T, 8, 1, 16, TT, MODE, ZOH>(p, stream)
                       : launch_fwd_cfg<T, 2, 4, 64, TT, MODE, ZOH>(p, stream);
    case 16: return few ? launch_fwd_cfg<T, 16, 1, 8, TT, MODE, ZOH>(p, stream)
                        : launch_fwd_cfg<T, 4, 4, 32, TT, MODE, ZOH>(p, stream);
    case 32: return few ? launch_fwd_cfg<T, 16, 2, 8, TT, MODE, ZOH>(p, stream)
                        : launch_fwd_cfg<T, 8, 4, 16, TT, MODE, ZOH>(p, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T, int MODE>
static cudaError_t launch_fwd_t(const FwdParams &p, cudaStream_t stream) {
    return p.zoh ? launch_fwd_tz<T, MODE, true>(p, stream) : launch_fwd_tz<T, MODE, false>(p, stream);
}

cudaError_t launch_fwd(const FwdParams &p, bool states_only, cudaStream_t stream) {
    const FwdKernel choice = fwd_kernel_choice();
    if (!states_only && choice != FwdKernel::kGeneral) {
        cudaError_t e = cudaSuccess;
        if (try_launch_fwd_tma(p, stream, &e)) {   // also writes delta_sum
            set_kernel_path("fwd:tma");
            return e;
        }
        if (choice == FwdKernel::kTma) return cudaErrorNotSupported;
    }
    set_kernel_path(states_only ? "fwd:general-states" : "fwd:general");
    cudaError_t e;
    if (p.io_bf16)
        e = states_only ? launch_fwd_t<__nv_bfloat16, 1>(p, stream)
                        : launch_fwd_t<__nv_bfloat16, 0>(p, stream);
    else
        e = states_only ? launch_fwd_t<float, 1>(p, stream) : launch_fwd_t<float, 0>(p, stream);
    if (e == cudaSuccess && p.delta_sum) e = launch_delta_sum(p, p.delta_sum, stream);
    return e;
}

}  // namespace ssm
