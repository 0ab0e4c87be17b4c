// Backward selective scan (S6) for sm_100a.
//
// The states are never stored by the forward; they are recomputed here from
// the per-chunk checkpoints (booiljung.github.io "3.2 선택적 스캔(Selective
// Scan) 알고리즘" §3.3: recomputation instead of storing the intermediate
// states).  With g = dout, s = sigmoid(z) and y the pre-gate output, reverse-
// mode differentiation of the forward recurrence gives:
//   gy_t = g_t z_t s_t,  dz_t = g_t y_t s_t (1 + z_t (1 - s_t))
//   λ_t[n] = C_t[n] gy_t + Ā_{t+1}[n] λ_{t+1}[n]                 (reverse scan)
//   du_t = gy_t D + Δ_t Σ_n λ_t[n] B_t[n]
//   dΔ_t = Σ_n λ_t[n] A[n] Ā_t[n] h_{t-1}[n] + u_t Σ_n λ_t[n] B_t[n]
//   ddelta_t = dΔ_t sigmoid(delta_t + bias)   (softplus on)
//   dA[d,n] = Σ_{b,t} λ Δ Ā h_{t-1};  dB[b,n,t] = Σ_d λ Δ u;  dC[b,n,t] = Σ_d gy h_t
//   dD[d] = Σ_{b,t} gy u;  dbias[d] = Σ_{b,t} ddelta
//
// Work split: a CTA owns one batch row and G channels; lane (c, g) owns NS
// states of channel c (as in the forward).  Checkpoint chunks are visited
// last to first.  Per chunk:
//   1. forward over the chunk in windows of W steps from the chunk's starting
//      state: the state at each window start is kept in shared memory, and the
//      readout partials give y, hence dz and gy for the chunk;
//   2. windows last to first: recompute the W steps (Ā and h_{t-1} held in
//      registers), then walk them backwards carrying λ and Ā_{t+1}; the
//      per-(channel, step) sums over states and the per-(state, step) sums over
//      the CTA's channels are reduced through shared memory; dB and dC are then
//      added to global memory with one atomic per (state, step) per CTA.

#include "ssm_common.cuh"
#include "ssm_internal.h"

namespace ssm {

template <int NT, int NS, int G, int W>
struct BwdSmem {
    static constexpr int N = NT * NS;
    static constexpr int CK = SSM_CKPT_CHUNK;
    static constexpr int NW = CK / W;
    static constexpr int WS = W + 4;    // row stride of per-channel window tiles
    static constexpr int CS = CK + 4;   // row stride of the chunk-long gy tile
    static constexpr int NSB = N + 4;
    static constexpr int kDt = 0;
    static constexpr int kDu = kDt + G * WS;
    static constexpr int kU = kDu + G * WS;
    static constexpr int kR = kU + G * WS;
    static constexpr int kGy = kR + G * WS;
    static constexpr int kB = kGy + G * CS;
    static constexpr int kC = kB + W * NSB;
    static constexpr int kHw = kC + W * NSB;
    static constexpr int kP0 = kHw + NW * G * N;
    static constexpr int kP1 = kP0 + NT * G * W;
    static constexpr int kdB = kP1 + NT * G * W;
    static constexpr int kdC = kdB + G * W * N;
    static constexpr int kTotal = kdC + G * W * N;
    static constexpr size_t bytes = sizeof(float) * kTotal;
};

// ZOH: the adjoint of the zero-order-hold forward (B̄ = φ(ΔA) Δ B): du and
// dB use φ Δ, the B term of dΔ carries dk/dΔ = Ā, and dA gains
// λ B u Δ² ψ(ΔA) (zoh_phi, zoh_psi).
template <typename T, int NT, int NS, int G, int W, bool ZOH>
__global__ void __launch_bounds__(NT * G)
bwd_kernel(const BwdParams p) {
    using S = BwdSmem<NT, NS, G, W>;
    constexpr int N = S::N, CK = S::CK, NW = S::NW, WS = S::WS, CS = S::CS, NSB = S::NSB;
    constexpr int NTHR = NT * G;
    constexpr int V = IO<T>::kVec;
    constexpr int VPW = (W + V - 1) / V;  // vectors per channel row of a window
    constexpr int EPL = W / NT;           // elements of its channel each lane finishes
    static_assert(W % NT == 0 && CK % W == 0 && W % 4 == 0, "bad window");

    extern __shared__ __align__(16) float smem[];
    float *sDt = smem + S::kDt, *sDu = smem + S::kDu, *sU = smem + S::kU, *sR = smem + S::kR;
    float *sGy = smem + S::kGy, *sB = smem + S::kB, *sC = smem + S::kC, *sHw = smem + S::kHw;
    float *sP0 = smem + S::kP0, *sP1 = smem + S::kP1, *sdB = smem + S::kdB, *sdC = smem + S::kdC;

    const int tid = threadIdx.x;
    const int g = tid % NT, c = tid / NT;
    const int b = blockIdx.y, d0 = blockIdx.x * G, d = d0 + c;
    const bool live = d < p.dim;
    const int L = p.L;
    const size_t row_bd0 = (size_t)b * p.dim;

    const T *u = static_cast<const T *>(p.u);
    const T *delta = static_cast<const T *>(p.delta);
    const T *z = static_cast<const T *>(p.z);
    const T *dout = static_cast<const T *>(p.dout);
    const T *Bm = static_cast<const T *>(p.B);
    const T *Cm = static_cast<const T *>(p.C);

    float Aw[NS], A2[NS], dA_acc[NS], lam[NS], anext[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        Aw[s] = live ? p.A[(size_t)d * N + g * NS + s] : 0.f;
        A2[s] = Aw[s] * SSM_LOG2E;
        dA_acc[s] = 0.f;
        lam[s] = 0.f;
        anext[s] = 1.f;
    }
    float dD_acc = 0.f, db_acc = 0.f;
    const float Dd = (p.D && live) ? p.D[d] : 0.f;

    // Stages Δ, Δ·u, u, r = delta + bias for the G channels and B, C for the
    // W steps starting at t0; steps >= L read as Δ = u = B = C = 0.
    auto stage_window = [&](int t0) {
        const int nvalid = min(W, L - t0);
        for (int v = tid; v < G * VPW; v += NTHR) {
            const int cc = v / VPW, j = (v % VPW) * V;
            const int dd = d0 + cc;
            float dr[V], uu[V];
            const int n_in = nvalid - j;
            float bias = 0.f;
            if (dd < p.dim) {
                const size_t off = (row_bd0 + dd) * (size_t)L + t0 + j;
                bias = p.delta_bias ? p.delta_bias[dd] : 0.f;
                load_vec(delta + off, n_in, p.vec_ok, 0.f, dr);
                load_vec(u + off, n_in, p.vec_ok, 0.f, uu);
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) dr[i] = uu[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < V; ++i) {
                if (j + i >= W) break;
                const bool ok = (i < n_in) && dd < p.dim;
                const float r = dr[i] + bias;
                const float dt = ok ? (p.softplus ? softplus_fast(r) : r) : 0.f;
                const float x = ok ? uu[i] : 0.f;
                sDt[cc * WS + j + i] = dt;
                sDu[cc * WS + j + i] = dt * x;
                sU[cc * WS + j + i] = x;
                sR[cc * WS + j + i] = r;
            }
        }
        for (int v = tid; v < N * VPW; v += NTHR) {
            const int n = v / VPW, j = (v % VPW) * V;
            const size_t off = ((size_t)b * N + n) * (size_t)L + t0 + j;
            float bb[V], cv[V];
            load_vec(Bm + off, nvalid - j, p.vec_ok, 0.f, bb);
            load_vec(Cm + off, nvalid - j, p.vec_ok, 0.f, cv);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                if (j + i >= W) break;
                sB[(j + i) * NSB + n] = bb[i];
                sC[(j + i) * NSB + n] = cv[i];
            }
        }
    };

    const int nchunk = (L + CK - 1) / CK;
    for (int k = nchunk - 1; k >= 0; --k) {
        const int c0 = k * CK;
        float h[NS];
#pragma unroll
        for (int s = 0; s < NS; ++s)
            h[s] = (k > 0 && live) ? p.ckpt[((row_bd0 + d) * p.n_ckpt + (k - 1)) * N + g * NS + s] : 0.f;

        // ------------------------------------------------ 1. forward over the chunk
        for (int w = 0; w < NW; ++w) {
            const int t0 = c0 + w * W;
            stage_window(t0);
            __syncthreads();
#pragma unroll
            for (int s = 0; s < NS; ++s) sHw[(w * G + c) * N + g * NS + s] = h[s];
#pragma unroll
            for (int t = 0; t < W; ++t) {
                const float dt = sDt[c * WS + t], du = sDu[c * WS + t];
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                    const float a = ex2(dt * A2[s]);
                    const float k = ZOH ? zoh_phi(dt * Aw[s], a) * du : du;
                    h[s] = fmaf(a, h[s], k * sB[t * NSB + g * NS + s]);
                    acc = fmaf(sC[t * NSB + g * NS + s], h[s], acc);
                }
                sP0[(g * G + c) * W + t] = acc;
            }
            __syncthreads();
            // y for EPL steps of this lane's own channel -> dz, gy
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int t = g * EPL + i;
                const int tg = t0 + t;
                float gy = 0.f;
                if (live && tg < L) {
                    float y = 0.f;
#pragma unroll
                    for (int gg = 0; gg < NT; ++gg) y += sP0[(gg * G + c) * W + t];
                    const float x = sU[c * WS + t];
                    y = fmaf(Dd, x, y);
                    const size_t off = (row_bd0 + d) * (size_t)L + tg;
                    const float gv = IO<T>::to_f(dout[off]);
                    if (z) {
                        const float zz = IO<T>::to_f(z[off]);
                        const float sg = sigmoid(zz);
                        p.dz[off] = gv * y * sg * (1.f + zz * (1.f - sg));
                        gy = gv * zz * sg;
                    } else {
                        gy = gv;
                    }
                    dD_acc = fmaf(gy, x, dD_acc);
                }
                sGy[c * CS + w * W + t] = gy;
            }
            __syncthreads();
        }

        // ------------------------------------------------ 2. reverse over windows
        for (int w = NW - 1; w >= 0; --w) {
            const int t0 = c0 + w * W;
            stage_window(t0);
            __syncthreads();
            float ab[W][NS], hp[W][NS];
            {
                float hw[NS];
#pragma unroll
                for (int s = 0; s < NS; ++s) hw[s] = sHw[(w * G + c) * N + g * NS + s];
#pragma unroll
                for (int t = 0; t < W; ++t) {
                    const float dt = sDt[c * WS + t], du = sDu[c * WS + t];
#pragma unroll
                    for (int s = 0; s < NS; ++s) {
                        ab[t][s] = ex2(dt * A2[s]);
                        hp[t][s] = hw[s];
                        const float k = ZOH ? zoh_phi(dt * Aw[s], ab[t][s]) * du : du;
                        hw[s] = fmaf(ab[t][s], hw[s], k * sB[t * NSB + g * NS + s]);
                    }
                }
            }
#pragma unroll
            for (int t = W - 1; t >= 0; --t) {
                const float gy = sGy[c * CS + w * W + t];
                const float dt = sDt[c * WS + t], du = sDu[c * WS + t];
                const float xu = ZOH ? sU[c * WS + t] : 0.f;
                // sa: Σ over the lane's states of the dΔ terms (through Ā, and
                // with ZOH through B̄ too); sb: Σ λ B (ZOH: Σ λ φ B), the du term / Δ
                float sa = 0.f, sb = 0.f;
                float dBv[NS], dCv[NS];
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                    const float Bt = sB[t * NSB + g * NS + s], Ct = sC[t * NSB + g * NS + s];
                    const float l = fmaf(anext[s], lam[s], Ct * gy);
                    const float a = ab[t][s], hv = hp[t][s];
                    const float phi = ZOH ? zoh_phi(dt * Aw[s], a) : 1.f;
                    const float hcur = fmaf(a, hv, phi * du * Bt);
                    const float wv = l * a * hv;
                    dA_acc[s] = fmaf(dt, wv, dA_acc[s]);
                    sa = fmaf(Aw[s], wv, sa);
                    if (ZOH) {
                        const float lB = l * Bt;
                        dA_acc[s] = fmaf(lB * xu, dt * dt * zoh_psi(dt * Aw[s], a), dA_acc[s]);
                        sa = fmaf(xu * a, lB, sa);
                        sb = fmaf(lB, phi, sb);
                    } else {
                        sb = fmaf(l, Bt, sb);
                    }
                    dBv[s] = l * phi * du;
                    dCv[s] = gy * hcur;
                    lam[s] = l;
                    anext[s] = a;
                }
                sP0[(g * G + c) * W + t] = sa;
                sP1[(g * G + c) * W + t] = sb;
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                    sdB[(c * W + t) * N + g * NS + s] = dBv[s];
                    sdC[(c * W + t) * N + g * NS + s] = dCv[s];
                }
            }
            __syncthreads();
            // per-element gradients for this lane's channel
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int t = g * EPL + i;
                const int tg = t0 + t;
                if (live && tg < L) {
                    float sa = 0.f, sb = 0.f;
#pragma unroll
                    for (int gg = 0; gg < NT; ++gg) {
                        sa += sP0[(gg * G + c) * W + t];
                        sb += sP1[(gg * G + c) * W + t];
                    }
                    const float dt = sDt[c * WS + t], x = sU[c * WS + t];
                    const float gy = sGy[c * CS + w * W + t];
                    const float dDelta = ZOH ? sa : fmaf(x, sb, sa);
                    const float ddr = p.softplus ? dDelta * sigmoid(sR[c * WS + t]) : dDelta;
                    const size_t off = (row_bd0 + d) * (size_t)L + tg;
                    p.du[off] = fmaf(gy, Dd, dt * sb);
                    p.ddelta[off] = ddr;
                    db_acc += ddr;
                }
            }
            // per-(state, step) sums over the CTA's channels
            for (int o = tid; o < W * N; o += NTHR) {
                const int t = o / N, n = o % N;
                const int tg = t0 + t;
                if (tg >= L) continue;
                float sb_ = 0.f, sc_ = 0.f;
#pragma unroll 8
                for (int cc = 0; cc < G; ++cc) {
                    sb_ += sdB[(cc * W + t) * N + n];
                    sc_ += sdC[(cc * W + t) * N + n];
                }
                const size_t off = ((size_t)b * N + n) * (size_t)L + tg;
                atomicAdd(p.dB + off, sb_);
                atomicAdd(p.dC + off, sc_);
            }
            __syncthreads();
        }
    }

    // ------------------------------------------------ per-channel reductions
    if (live) {
#pragma unroll
        for (int s = 0; s < NS; ++s) atomicAdd(p.dA + (size_t)d * N + g * NS + s, dA_acc[s]);
    }
#pragma unroll
    for (int m = NT / 2; m >= 1; m /= 2) {
        dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, m);
        db_acc += __shfl_xor_sync(0xffffffffu, db_acc, m);
    }
    if (live && g == 0) {
        if (p.dD) atomicAdd(p.dD + d, dD_acc);
        if (p.ddelta_bias) atomicAdd(p.ddelta_bias + d, db_acc);
    }
}

template <typename T, int NT, int NS, int G, int W, bool ZOH>
static cudaError_t launch_bwd_cfg(const BwdParams &p, cudaStream_t stream) {
    using S = BwdSmem<NT, NS, G, W>;
    auto kern = bwd_kernel<T, NT, NS, G, W, ZOH>;
    static bool attr_done = false;
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

template <typename T, bool ZOH>
static cudaError_t launch_bwd_tz(const BwdParams &p, cudaStream_t stream) {
    switch (p.N) {
    case 1: return launch_bwd_cfg<T, 1, 1, 64, 8, ZOH>(p, stream);
    case 2: return launch_bwd_cfg<T, 1, 2, 64, 8, ZOH>(p, stream);
    case 4: return launch_bwd_cfg<T, 1, 4, 64, 8, ZOH>(p, stream);
    case 8: return launch_bwd_cfg<T, 2, 4, 32, 8, ZOH>(p, stream);
    case 16: return launch_bwd_cfg<T, 4, 4, 32, 8, ZOH>(p, stream);
    case 32: return launch_bwd_cfg<T, 8, 4, 16, 8, ZOH>(p, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T>
static cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t stream) {
    return p.zoh ? launch_bwd_tz<T, true>(p, stream) : launch_bwd_tz<T, false>(p, stream);
}

cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream) {
    cudaError_t err = cudaSuccess;
    if (try_launch_bwd_tma(p, stream, &err)) {
        set_kernel_path("bwd:tma");
        return err;
    }
    set_kernel_path("bwd:general");
    return p.io_bf16 ? launch_bwd_t<__nv_bfloat16>(p, stream) : launch_bwd_t<float>(p, stream);
}

}  // namespace ssm
