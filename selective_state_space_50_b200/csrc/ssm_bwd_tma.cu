// Backward selective scan, TMA-fed persistent kernel for sm_100a.
//
// Same adjoint as the general backward in ssm_bwd.cu (reverse-mode
// differentiation of the forward recurrence, with the hidden states
// recomputed instead of stored: booiljung.github.io, "3.2 선택적 스캔
// (Selective Scan) 알고리즘", §3.3).  With g = dout, s = sigmoid(z) and y the
// output before the gate:
//   gy = g z s,  dz = g y s (1 + z (1 - s)),  λ_t = C_t gy_t + Ā_{t+1} λ_{t+1}
//   du = gy D + Δ Σ_n λ B,  dΔ = Σ_n λ A Ā h_{t-1} + u Σ_n λ B,  ddelta = dΔ σ(r)
//   dA = Σ λ Δ Ā h_{t-1},  dB = Σ_d λ Δ u,  dC = Σ_d gy h,  dD = Σ gy u,  dbias = Σ ddelta
//
// Organisation (mirrors the TMA forward):
//  * One CTA per SM; channel rows (batch x dim) split evenly over the CTAs.
//    Time tiles of 32 steps are visited last to first.  A producer lane
//    streams delta, u, z, dout ([rows x 32] boxes) and B, C ([dstate x 32]
//    per batch row) into a two-stage ring with TMA loads that complete on
//    mbarriers; consumer warps release a stage with an mbarrier arrive.
//  * A consumer warp owns 8 channels x 4 groups of 4 states
//    (lane = group * 8 + channel).  Per tile it first computes Δ, Δu and gy
//    once per element.  Then, for each 8-step window (one checkpoint chunk of
//    the forward) from last to first, it starts from the checkpointed state,
//    recomputes Ā_t (one ex2 per step and state) and Ā_t h_{t-1} into
//    registers, and sweeps the window backwards carrying λ and Ā_{t+1}.
//  * Sums over states for each (channel, step) -- y, Σ λ A Ā h, Σ λ B -- go
//    through a per-warp buffer and are finished per element (dz, du, ddelta;
//    dD and dbias accumulate per lane).  Sums over channels for each
//    (state, step) -- dB, dC -- are reduced over a quarter-warp's 8 channels
//    by a transpose through shared memory, accumulated over the CTA's warps
//    with shared-memory atomics into a per-tile buffer, and flushed by the
//    producer warp once per tile with 16-byte global atomics.

#include <cudaTypedefs.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>

#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_tma.cuh"

namespace ssm {

namespace {

constexpr int bwd_align128(int x) { return (x + 127) / 128 * 128; }
constexpr int bwd_align1024(int x) { return (x + 1023) / 1024 * 1024; }

struct TmaBwdParams {
    const float *A, *D, *delta_bias, *ckpt;
    float *du, *ddelta, *dA, *dB, *dC, *dD, *dz, *ddelta_bias;
    int P, dim, L, n_ckpt;
    int softplus, has_z;
    int rows_max;
    int *err;
};

template <typename T, int NWC, int STAGES>
struct BwdLayout {
    static constexpr int NT = 4, NS = 4, N = 16, TT = 32;
    static constexpr int CPW = 32 / NT;                                // channels per warp
    static constexpr int MAXR = NWC * CPW;
    static constexpr int RAW_ROW = TT * (int)sizeof(T);
    static constexpr int RAW_CH = bwd_align128(MAXR * RAW_ROW);       // delta, u, z, dout
    static constexpr bool SWZ = RAW_ROW >= 128;
    static constexpr int PW = SWZ ? 128 : RAW_ROW;
    static constexpr int NPIECE = RAW_ROW / PW;
    static constexpr int PIECE = 2 * N * PW;                           // [2 batch rows][N][PW]
    static constexpr int RAW_BC = NPIECE * PIECE;
    static constexpr int kBC0 = bwd_align1024(4 * RAW_CH);
    static constexpr int STAGE = bwd_align1024(kBC0 + 2 * RAW_BC);
    static constexpr int W = 8;                                        // window = checkpoint chunk
    static constexpr int NWIN = TT / W;
    static constexpr int WS = TT + 4;                                  // row of wDt / wDu / wGy
    static constexpr int PS = W + 4;                                   // row of the state partials
    static constexpr int XS = W * NS + 4;                              // row of the transpose
    static constexpr int kWdt = 0, kWdu = CPW * WS, kWgy = 2 * CPW * WS;
    static constexpr int kWp = 3 * CPW * WS;                           // [3][NT][CPW][PS]
    static constexpr int kWx = kWp + 3 * NT * CPW * PS;                // [32][XS]
    static constexpr int WBUF = (kWx + 32 * XS) * 4;
    // dB/dC tile accumulator: [B or C][batch row][state, permuted][DS]
    static constexpr int DS = TT + 8;
    static constexpr int DBC_PAR = 2 * 2 * N * DS;
    static constexpr int kW = STAGES * STAGE;
    static constexpr int kDBC = kW + NWC * WBUF;
    static constexpr int kBar = kDBC + 2 * DBC_PAR * 4;
    static constexpr int kTotal = kBar + (2 * STAGES + 4) * 8;
    static constexpr int kAlloc = kTotal + 1024;
    static constexpr int kThreads = (NWC + 1) * 32;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static_assert(CPW * (TT / W) == 32, "one prep item of 8 steps per lane");
    static_assert(SSM_CKPT_CHUNK == W, "windows are checkpoint chunks");
    static_assert(PS % 4 == 0 && XS % 4 == 0 && WS % 4 == 0 && DS % 4 == 0, "16-byte rows");
};

// Row of state n in the dB/dC accumulator.  Lanes of different quarter-warps
// add to different states at once; with this order and a row of DS = 40
// floats they fall in different banks.
__device__ __forceinline__ int dbc_row(int n) { return (n % 4) * 4 + n / 4; }

__device__ __forceinline__ void red_add_v4(float *addr, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

// The 8 steps of one window of one row of B or C, kept packed in registers.
template <typename T> struct BCWin;

// at() unpacks with opaque instructions so that the compiler re-extracts a
// value where it is used instead of keeping all unpacked values alive across
// the recompute and the reverse sweep.
template <> struct BCWin<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ float at(int t) const {
        const uint32_t x = (t < 2) ? v.x : (t < 4) ? v.y : (t < 6) ? v.z : v.w;
        uint32_t r;
        if (t & 1) asm volatile("and.b32 %0, %1, 0xffff0000;" : "=r"(r) : "r"(x));
        else asm volatile("shl.b32 %0, %1, 16;" : "=r"(r) : "r"(x));
        return __uint_as_float(r);
    }
};

template <> struct BCWin<float> {
    uint4 v[2];
    __device__ __forceinline__ float at(int t) const {
        const uint4 &q = v[t / 4];
        const int i = t % 4;
        return __uint_as_float(i == 0 ? q.x : i == 1 ? q.y : i == 2 ? q.z : q.w);
    }
};

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
    const float2 lo = __fadd2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
    const float2 hi = __fadd2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

template <typename T, int NWC, int STAGES>
__global__ void __launch_bounds__((NWC + 1) * 32, 1)
bwd_tma_kernel(const __grid_constant__ CUtensorMap m_delta, const __grid_constant__ CUtensorMap m_u,
               const __grid_constant__ CUtensorMap m_z, const __grid_constant__ CUtensorMap m_g,
               const __grid_constant__ CUtensorMap m_B, const __grid_constant__ CUtensorMap m_C,
               const TmaBwdParams p) {
    using Ly = BwdLayout<T, NWC, STAGES>;
    constexpr int N = Ly::N, NT = Ly::NT, NS = Ly::NS, TT = Ly::TT, CPW = Ly::CPW;
    constexpr int WS = Ly::WS, PS = Ly::PS, XS = Ly::XS, DS = Ly::DS, W = Ly::W;

    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Ly::kBar);
    uint64_t *empty = full + STAGES;
    uint64_t *dfull = empty + STAGES;   // all consumers added their dB/dC of a tile
    uint64_t *dempty = dfull + 2;       // the producer flushed and cleared that buffer
    float *dbc = reinterpret_cast<float *>(smem + Ly::kDBC);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int G = gridDim.x;
    const int r0 = (int)((long long)blockIdx.x * p.P / G);
    const int r1 = (int)((long long)(blockIdx.x + 1) * p.P / G);
    const int R = r1 - r0;
    const int npass = (R + p.rows_max - 1) / p.rows_max;
    const int ntiles = (p.L + TT - 1) / TT;
    const int total = npass * ntiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, NWC);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(dfull + b, NWC);
            mbar_init(dempty + b, 1);
        }
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < 2 * Ly::DBC_PAR; i += blockDim.x) dbc[i] = 0.f;
    __syncthreads();

    auto pass_rows = [&](int q, int &q0, int &q1) {
        q0 = r0 + (int)((long long)q * R / npass);
        q1 = r0 + (int)((long long)(q + 1) * R / npass);
    };

    if (warp == NWC) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&m_delta);
            prefetch_tensormap(&m_u);
            if (p.has_z) prefetch_tensormap(&m_z);
            prefetch_tensormap(&m_g);
            prefetch_tensormap(&m_B);
            prefetch_tensormap(&m_C);
        }
        int is_ = 0, is_s = 0, is_q = 0, is_k = 0, is_q0 = 0, is_q1 = 0;
        auto issue_next = [&]() {   // lane 0 only
            if (is_k == 0) pass_rows(is_q, is_q0, is_q1);
            const int t0 = (ntiles - 1 - is_k) * TT;
            const int b_lo = is_q0 / p.dim, nb = (is_q1 - 1) / p.dim - b_lo + 1;
            uint8_t *st = smem + is_s * Ly::STAGE;
            const uint32_t bytes = (uint32_t)(p.rows_max * Ly::RAW_ROW * (3 + p.has_z) +
                                              2 * nb * N * Ly::RAW_ROW);
            mbar_arrive_expect_tx(full + is_s, bytes);
            tma_load_2d(st, &m_delta, t0, is_q0, full + is_s);
            tma_load_2d(st + Ly::RAW_CH, &m_u, t0, is_q0, full + is_s);
            if (p.has_z) tma_load_2d(st + 2 * Ly::RAW_CH, &m_z, t0, is_q0, full + is_s);
            tma_load_2d(st + 3 * Ly::RAW_CH, &m_g, t0, is_q0, full + is_s);
            for (int bs = 0; bs < nb; ++bs)
                for (int pc = 0; pc < Ly::NPIECE; ++pc) {
                    const int off = Ly::kBC0 + pc * Ly::PIECE + bs * N * Ly::PW;
                    const int x = t0 + pc * (Ly::PW / (int)sizeof(T));
                    tma_load_2d(st + off, &m_B, x, (b_lo + bs) * N, full + is_s);
                    tma_load_2d(st + off + Ly::RAW_BC, &m_C, x, (b_lo + bs) * N, full + is_s);
                }
            ++is_;
            if (++is_s == STAGES) is_s = 0;
            if (++is_k == ntiles) { is_k = 0; ++is_q; }
        };
        if (lane == 0)
            while (is_ < STAGES && is_ < total) issue_next();
        bool ok = true;
        int q = 0, k = 0, q0 = 0, q1 = 0;
        for (int kg = 0; kg < total; ++kg) {
            if (k == 0) pass_rows(q, q0, q1);
            // every consumer is done with tile kg: flush its dB/dC, then refill the stage
            ok = mbar_wait(dfull + (kg & 1), (kg >> 1) & 1, p.err);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            {
                const int t0 = (ntiles - 1 - k) * TT;
                const int b_lo = q0 / p.dim, nb = (q1 - 1) / p.dim - b_lo + 1;
                float *buf = dbc + (kg & 1) * Ly::DBC_PAR;
                constexpr int QPR = TT / 4;                 // float4 per accumulator row
                const int nvec = 2 * nb * N * QPR;
                for (int i = lane; i < nvec; i += 32) {
                    const int tq = i % QPR, n = (i / QPR) % N;
                    const int bs = (i / (QPR * N)) % nb, which = i / (QPR * N * nb);
                    float *src = buf + ((which * 2 + bs) * N + dbc_row(n)) * DS + tq * 4;
                    const float4 v = *reinterpret_cast<const float4 *>(src);
                    *reinterpret_cast<float4 *>(src) = make_float4(0.f, 0.f, 0.f, 0.f);
                    const int tg = t0 + tq * 4;
                    if (tg < p.L) {
                        float *dst = (which == 0 ? p.dB : p.dC) + ((size_t)(b_lo + bs) * N + n) * p.L + tg;
                        red_add_v4(dst, v);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(dempty + (kg & 1));
            }
            if (lane == 0 && is_ < total) {
                ok = mbar_wait(empty + (kg % STAGES), (kg / STAGES) & 1, p.err);
                if (ok) issue_next();
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (++k == ntiles) { k = 0; ++q; }
        }
        if (lane == 0) {
            // never leave while a copy may still write shared memory
            for (int kg = (is_ > STAGES ? is_ - STAGES : 0); kg < is_; ++kg)
                if (!mbar_wait(full + (kg % STAGES), (kg / STAGES) & 1, p.err)) break;
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int c = lane % CPW, g = lane / CPW;                 // scan: channel, state group
    const int it_rl = lane / (TT / W), it_t = (lane % (TT / W)) * W;   // prep: row, step offset
    float *wbase = reinterpret_cast<float *>(smem + Ly::kW + warp * Ly::WBUF);
    float *wDt = wbase + Ly::kWdt, *wDu = wbase + Ly::kWdu, *wGy = wbase + Ly::kWgy;
    float *wP = wbase + Ly::kWp, *wX = wbase + Ly::kWx;
    float *myX = wX + lane * XS;

    float A2[NS], lam[NS], anext[NS], dA_acc[NS];   // A2 = A log2(e)
    float4 hpre = make_float4(0.f, 0.f, 0.f, 0.f);        // checkpoint of the next window
    float dD_acc = 0.f, db_acc = 0.f, Dd = 0.f, bias_c = 0.f, i_bias = 0.f;
    int row = 0, d = 0, bsel = 0, wb = 0, irow = -1;
    bool live = false, straddle = false;
    unsigned b1mask = 0;                                   // channels of the second batch row

    int s = 0, phase = 0, q = 0, k = 0, q0 = 0, q1 = 0;
    for (int kg = 0; kg < total; ++kg) {
        const int t0 = (ntiles - 1 - k) * TT;
        if (k == 0) {
            pass_rows(q, q0, q1);
            const int wrow0 = q0 + warp * CPW;
            row = wrow0 + c;
            live = row < q1;
            d = live ? row % p.dim : 0;
            bsel = live ? row / p.dim - q0 / p.dim : 0;
            const unsigned lmask = __ballot_sync(0xffffffffu, live) & 0xffu;
            b1mask = __ballot_sync(0xffffffffu, bsel == 1) & 0xffu;
            straddle = b1mask != 0 && b1mask != lmask;
            wb = b1mask != 0 ? 1 : 0;
#pragma unroll
            for (int j = 0; j < NS; ++j) {
                A2[j] = live ? p.A[(size_t)d * N + g * NS + j] * SSM_LOG2E : 0.f;
                lam[j] = 0.f;
                anext[j] = 1.f;
                dA_acc[j] = 0.f;
            }
            Dd = (live && p.D) ? p.D[d] : 0.f;
            bias_c = (live && p.delta_bias) ? p.delta_bias[d] : 0.f;
            const int rr = wrow0 + it_rl;
            irow = rr < q1 ? rr : -1;
            i_bias = (irow >= 0 && p.delta_bias) ? p.delta_bias[rr % p.dim] : 0.f;
            dD_acc = 0.f;
            db_acc = 0.f;
            // starting state of the first window visited (the one holding step L-1)
            const int kc0 = (p.L - 1) / W - 1;
            hpre = (live && kc0 >= 0) ? __ldg(reinterpret_cast<const float4 *>(
                                            p.ckpt + ((size_t)row * p.n_ckpt + kc0) * N + g * NS))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int wrow0 = q0 + warp * CPW;
        {
            // every lane waits; the warp leaves together if any wait gave up
            bool ok = mbar_wait(full + s, phase, p.err);
            if (kg >= 2) ok = ok && mbar_wait(dempty + (kg & 1), ((kg - 2) >> 1) & 1, p.err);
            if (!__all_sync(0xffffffffu, ok)) return;
        }
        float *dbuf = dbc + (kg & 1) * Ly::DBC_PAR;

        if (wrow0 < q1) {
            const uint8_t *st = smem + s * Ly::STAGE;
            const T *rawD = reinterpret_cast<const T *>(st) + warp * CPW * TT;
            const T *rawU = reinterpret_cast<const T *>(st + Ly::RAW_CH) + warp * CPW * TT;
            const T *rawZ = reinterpret_cast<const T *>(st + 2 * Ly::RAW_CH) + warp * CPW * TT;
            const T *rawG = reinterpret_cast<const T *>(st + 3 * Ly::RAW_CH) + warp * CPW * TT;
            // (1) Δ, Δu and gy of this lane's 8 steps of one row, once per element
            {
                constexpr int V = IO<T>::kVec;
                float dt[W], du[W], gy[W];
#pragma unroll
                for (int v0 = 0; v0 < W; v0 += V) {
                    float dr[V], uu[V], zz[V], gg[V];
                    const int o = it_rl * TT + it_t + v0;
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawD + o), dr);
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawU + o), uu);
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawG + o), gg);
                    if (p.has_z) IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawZ + o), zz);
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        const bool ok = irow >= 0 && (t0 + it_t + v0 + e) < p.L;
                        const float r = dr[e] + i_bias;
                        const float dtv = p.softplus ? softplus_fast(r) : r;
                        float gyv = gg[e];
                        if (p.has_z) gyv *= zz[e] * sigmoid(zz[e]);
                        dt[v0 + e] = ok ? dtv : 0.f;
                        du[v0 + e] = ok ? dtv * uu[e] : 0.f;
                        gy[v0 + e] = ok ? gyv : 0.f;
                    }
                }
                float *pdt = wDt + it_rl * WS + it_t, *pdu = wDu + it_rl * WS + it_t;
                float *pgy = wGy + it_rl * WS + it_t;
#pragma unroll
                for (int e = 0; e < W; e += 4) {
                    *reinterpret_cast<float4 *>(pdt + e) = make_float4(dt[e], dt[e + 1], dt[e + 2], dt[e + 3]);
                    *reinterpret_cast<float4 *>(pdu + e) = make_float4(du[e], du[e + 1], du[e + 2], du[e + 3]);
                    *reinterpret_cast<float4 *>(pgy + e) = make_float4(gy[e], gy[e + 1], gy[e + 2], gy[e + 3]);
                }
            }
            __syncwarp();

            const uint8_t *rawB = st + Ly::kBC0;
            const uint8_t *rawC = rawB + Ly::RAW_BC;
            auto bc_chunk = [&](const uint8_t *base, int rr, int tb) -> uint4 {
                const int byte = tb * (int)sizeof(T);
                const int pc = byte / Ly::PW, in = byte % Ly::PW;
                int chunk = in >> 4;
                if constexpr (Ly::SWZ) chunk ^= (rr & 7);
                return *reinterpret_cast<const uint4 *>(base + pc * Ly::PIECE + rr * Ly::PW + (chunk << 4));
            };
            const int rr0 = bsel * N + g * NS;
            // Sum of the transpose buffer over the quarter-warp's channels for
            // step c of the window, states 4g..4g+3, added to the tile
            // accumulator `which` (0: dB, 1: dC).
            auto reduce_x = [&](int which, int tw) {
                __syncwarp();
                float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
#pragma unroll
                for (int cc = 0; cc < CPW; ++cc) {
                    const float4 v = *reinterpret_cast<const float4 *>(wX + (g * CPW + cc) * XS + c * NS);
                    if (straddle && ((b1mask >> cc) & 1)) s1 = f4add(s1, v);
                    else s0 = f4add(s0, v);
                }
                __syncwarp();
                float *dst = dbuf + ((which * 2 + (straddle ? 0 : wb)) * N) * DS + tw + c;
                atomicAdd(dst + dbc_row(g * NS + 0) * DS, s0.x);
                atomicAdd(dst + dbc_row(g * NS + 1) * DS, s0.y);
                atomicAdd(dst + dbc_row(g * NS + 2) * DS, s0.z);
                atomicAdd(dst + dbc_row(g * NS + 3) * DS, s0.w);
                if (straddle) {
                    dst += N * DS;
                    atomicAdd(dst + dbc_row(g * NS + 0) * DS, s1.x);
                    atomicAdd(dst + dbc_row(g * NS + 1) * DS, s1.y);
                    atomicAdd(dst + dbc_row(g * NS + 2) * DS, s1.z);
                    atomicAdd(dst + dbc_row(g * NS + 3) * DS, s1.w);
                }
            };

            // (2) 8-step windows, last to first
#pragma unroll 1
            for (int w = Ly::NWIN - 1; w >= 0; --w) {
                const int tw = w * W;                       // window start within the tile
                const int tgw = t0 + tw;                    // and within the sequence
                if (tgw >= p.L) continue;                   // past the end: λ stays 0
                float h[NS] = {hpre.x, hpre.y, hpre.z, hpre.w};
                {
                    const int kc = tgw / W - 2;             // checkpoint of the next window
                    hpre = (live && kc >= 0) ? __ldg(reinterpret_cast<const float4 *>(
                                                   p.ckpt + ((size_t)row * p.n_ckpt + kc) * N + g * NS))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                BCWin<T> Bw[NS], Cw[NS];
#pragma unroll
                for (int j = 0; j < NS; ++j) {
                    if constexpr (sizeof(T) == 2) {
                        Bw[j].v = bc_chunk(rawB, rr0 + j, tw);
                        Cw[j].v = bc_chunk(rawC, rr0 + j, tw);
                    } else {
                        Bw[j].v[0] = bc_chunk(rawB, rr0 + j, tw);
                        Bw[j].v[1] = bc_chunk(rawB, rr0 + j, tw + 4);
                        Cw[j].v[0] = bc_chunk(rawC, rr0 + j, tw);
                        Cw[j].v[1] = bc_chunk(rawC, rr0 + j, tw + 4);
                    }
                }
                // forward recompute, 4 steps at a time: Ā_t, Ā_t h_{t-1}, the y
                // partials, and gy h_t for dC
                float ab[W][NS], ahp[W][NS];
                float *pY = wP + (0 * NT + g) * CPW * PS + c * PS;
#pragma unroll
                for (int t4 = 0; t4 < W; t4 += 4) {
                    const float4 dt4 = *reinterpret_cast<const float4 *>(wDt + c * WS + tw + t4);
                    const float4 du4 = *reinterpret_cast<const float4 *>(wDu + c * WS + tw + t4);
                    const float4 gy4 = *reinterpret_cast<const float4 *>(wGy + c * WS + tw + t4);
                    const float dt[4] = {dt4.x, dt4.y, dt4.z, dt4.w}, du[4] = {du4.x, du4.y, du4.z, du4.w};
                    const float gy[4] = {gy4.x, gy4.y, gy4.z, gy4.w};
                    float yp[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int t = t4 + i;
                        float acc = 0.f, xc[NS];
#pragma unroll
                        for (int j = 0; j < NS; ++j) {
                            const float a = ex2(dt[i] * A2[j]);
                            ab[t][j] = a;
                            ahp[t][j] = a * h[j];
                            h[j] = fmaf(du[i], Bw[j].at(t), ahp[t][j]);
                            acc = fmaf(Cw[j].at(t), h[j], acc);
                            xc[j] = gy[i] * h[j];
                        }
                        yp[i] = acc;
                        *reinterpret_cast<float4 *>(myX + t * NS) = make_float4(xc[0], xc[1], xc[2], xc[3]);
                    }
                    *reinterpret_cast<float4 *>(pY + t4) = make_float4(yp[0], yp[1], yp[2], yp[3]);
                }
                reduce_x(1, tw);
                // reverse sweep, 4 steps at a time.  The A-weighted sum is kept
                // in units of A log2(e) and rescaled per element.
                float *pA = wP + (1 * NT + g) * CPW * PS + c * PS;
                float *pB = wP + (2 * NT + g) * CPW * PS + c * PS;
#pragma unroll
                for (int t4 = W - 4; t4 >= 0; t4 -= 4) {
                    const float4 dt4 = *reinterpret_cast<const float4 *>(wDt + c * WS + tw + t4);
                    const float4 du4 = *reinterpret_cast<const float4 *>(wDu + c * WS + tw + t4);
                    const float4 gy4 = *reinterpret_cast<const float4 *>(wGy + c * WS + tw + t4);
                    const float dt[4] = {dt4.x, dt4.y, dt4.z, dt4.w}, du[4] = {du4.x, du4.y, du4.z, du4.w};
                    const float gy[4] = {gy4.x, gy4.y, gy4.z, gy4.w};
                    float sa[4], sb[4];
#pragma unroll
                    for (int i = 3; i >= 0; --i) {
                        const int t = t4 + i;
                        float a_sa = 0.f, a_sb = 0.f, xb[NS];
#pragma unroll
                        for (int j = 0; j < NS; ++j) {
                            const float Bt = Bw[j].at(t);
                            const float l = fmaf(anext[j], lam[j], Cw[j].at(t) * gy[i]);
                            const float wv = l * ahp[t][j];
                            dA_acc[j] = fmaf(dt[i], wv, dA_acc[j]);
                            a_sa = fmaf(A2[j], wv, a_sa);
                            a_sb = fmaf(l, Bt, a_sb);
                            xb[j] = l * du[i];
                            lam[j] = l;
                            anext[j] = ab[t][j];
                        }
                        sa[i] = a_sa;
                        sb[i] = a_sb;
                        *reinterpret_cast<float4 *>(myX + t * NS) = make_float4(xb[0], xb[1], xb[2], xb[3]);
                    }
                    *reinterpret_cast<float4 *>(pA + t4) = make_float4(sa[0], sa[1], sa[2], sa[3]);
                    *reinterpret_cast<float4 *>(pB + t4) = make_float4(sb[0], sb[1], sb[2], sb[3]);
                }
                reduce_x(0, tw);   // its leading __syncwarp also publishes the partials
                // per-element results: lane (g, c) finishes steps 2g and 2g+1 of channel c
                if (live && tgw + 2 * g < p.L) {
                    const int t = 2 * g;
                    float2 y = make_float2(0.f, 0.f), a_sa = y, a_sb = y;
#pragma unroll
                    for (int gg = 0; gg < NT; ++gg) {
                        y = __fadd2_rn(y, *reinterpret_cast<const float2 *>(wP + (0 * NT + gg) * CPW * PS + c * PS + t));
                        a_sa = __fadd2_rn(a_sa, *reinterpret_cast<const float2 *>(wP + (1 * NT + gg) * CPW * PS + c * PS + t));
                        a_sb = __fadd2_rn(a_sb, *reinterpret_cast<const float2 *>(wP + (2 * NT + gg) * CPW * PS + c * PS + t));
                    }
                    const int o = c * TT + tw + t;
                    const float x[2] = {IO<T>::to_f(rawU[o]), IO<T>::to_f(rawU[o + 1])};
                    const float gv[2] = {IO<T>::to_f(rawG[o]), IO<T>::to_f(rawG[o + 1])};
                    const float2 dtv = *reinterpret_cast<const float2 *>(wDt + c * WS + tw + t);
                    const float2 gyv = *reinterpret_cast<const float2 *>(wGy + c * WS + tw + t);
                    const float yy[2] = {fmaf(Dd, x[0], y.x), fmaf(Dd, x[1], y.y)};
                    const float sa2[2] = {a_sa.x * 0.69314718f, a_sa.y * 0.69314718f};
                    const float sb2[2] = {a_sb.x, a_sb.y};
                    const float dt2[2] = {dtv.x, dtv.y}, gy2[2] = {gyv.x, gyv.y};
                    float dzv[2] = {0.f, 0.f}, duv[2], ddv[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if (p.has_z) {
                            const float zz = IO<T>::to_f(rawZ[o + e]);
                            const float sg = sigmoid(zz);
                            dzv[e] = gv[e] * yy[e] * sg * fmaf(zz, 1.f - sg, 1.f);
                        }
                        const float dDelta = fmaf(x[e], sb2[e], sa2[e]);
                        ddv[e] = p.softplus ? dDelta * sigmoid(IO<T>::to_f(rawD[o + e]) + bias_c) : dDelta;
                        duv[e] = fmaf(gy2[e], Dd, dt2[e] * sb2[e]);
                        dD_acc = fmaf(gy2[e], x[e], dD_acc);
                        db_acc += ddv[e];
                    }
                    const size_t off = (size_t)row * p.L + tgw + t;
                    __stcs(reinterpret_cast<float2 *>(p.du + off), make_float2(duv[0], duv[1]));
                    __stcs(reinterpret_cast<float2 *>(p.ddelta + off), make_float2(ddv[0], ddv[1]));
                    if (p.has_z) __stcs(reinterpret_cast<float2 *>(p.dz + off), make_float2(dzv[0], dzv[1]));
                }
                __syncwarp();   // wP and the transpose buffer are rewritten by the next window
            }
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(empty + s);
            mbar_arrive(dfull + (kg & 1));
        }
        if (++s == STAGES) { s = 0; phase ^= 1; }
        if (++k == ntiles) {
            // end of a pass over this CTA's rows: per-channel sums
            if (live) {
#pragma unroll
                for (int j = 0; j < NS; ++j) atomicAdd(p.dA + (size_t)d * N + g * NS + j, dA_acc[j]);
            }
#pragma unroll
            for (int m = CPW; m < 32; m <<= 1) {    // lanes c, c+8, c+16, c+24 share channel c
                dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, m);
                db_acc += __shfl_xor_sync(0xffffffffu, db_acc, m);
            }
            if (live && g == 0) {
                if (p.dD) atomicAdd(p.dD + d, dD_acc);
                if (p.ddelta_bias) atomicAdd(p.ddelta_bias + d, db_acc);
            }
            k = 0;
            ++q;
        }
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 bwd_get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool bwd_make_map(CUtensorMap *m, const void *base, bool bf16, uint64_t rows, uint64_t cols,
                  uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
    auto enc = bwd_get_encode();
    if (!enc) return false;
    const uint64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * es};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int bwd_sm_count() {
    static int count[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!count[dev]) cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
    return count[dev];
}

template <typename T, int NWC, int STAGES>
cudaError_t launch_bwd_tma_cfg(const BwdParams &bp, int rows_max, cudaStream_t stream) {
    using Ly = BwdLayout<T, NWC, STAGES>;
    const int P = bp.batch * bp.dim;
    const int grid = std::min(bwd_sm_count(), P);
    const bool bf16 = sizeof(T) == 2;
    CUtensorMap md, mu, mz, mg, mB, mC;
    const uint32_t bc_box = Ly::PW / sizeof(T);
    if (!bwd_make_map(&md, bp.delta, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !bwd_make_map(&mu, bp.u, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !bwd_make_map(&mz, bp.z ? bp.z : bp.u, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !bwd_make_map(&mg, bp.dout, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !bwd_make_map(&mB, bp.B, bf16, (uint64_t)bp.batch * Ly::N, bp.L, bc_box, Ly::N, Ly::SWZ) ||
        !bwd_make_map(&mC, bp.C, bf16, (uint64_t)bp.batch * Ly::N, bp.L, bc_box, Ly::N, Ly::SWZ))
        return cudaErrorInvalidValue;
    TmaBwdParams p{};
    p.A = bp.A; p.D = bp.D; p.delta_bias = bp.delta_bias; p.ckpt = bp.ckpt;
    p.du = bp.du; p.ddelta = bp.ddelta; p.dA = bp.dA; p.dB = bp.dB; p.dC = bp.dC;
    p.dD = bp.dD; p.dz = bp.dz; p.ddelta_bias = bp.ddelta_bias;
    p.P = P; p.dim = bp.dim; p.L = bp.L; p.n_ckpt = bp.n_ckpt;
    p.softplus = bp.softplus; p.has_z = bp.z != nullptr; p.rows_max = rows_max;
    p.err = device_error_word();
    if (!p.err) return cudaErrorInvalidDevice;
    auto kern = bwd_tma_kernel<T, NWC, STAGES>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    kern<<<grid, Ly::kThreads, Ly::kAlloc, stream>>>(md, mu, mz, mg, mB, mC, p);
    return cudaGetLastError();
}

bool aligned_to(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

// Consumer warps per CTA.  With the producer warp, 12 (bf16) or 8 (fp32)
// warps keep at most 3 or 2 warps on each SM sub-partition, which leaves 168
// or 255 registers per thread.
#ifndef SSM_BWD_WARPS_BF16
#define SSM_BWD_WARPS_BF16 11
#endif
#ifndef SSM_BWD_WARPS_F32
#define SSM_BWD_WARPS_F32 7
#endif
constexpr int kBwdWarpsBf16 = SSM_BWD_WARPS_BF16, kBwdWarpsF32 = SSM_BWD_WARPS_F32;

}  // namespace

bool try_launch_bwd_tma(const BwdParams &bp, cudaStream_t stream, cudaError_t *err) {
    static const char *force = getenv("SSM_BWD_KERNEL");
    if (force && !strcmp(force, "general")) return false;
    if (!bp.vec_ok || bp.N != 16 || !bp.ckpt) return false;
    if (!aligned_to(bp.ckpt, 16) || !aligned_to(bp.dB, 16) || !aligned_to(bp.dC, 16) ||
        !aligned_to(bp.du, 8) || !aligned_to(bp.ddelta, 8) || (bp.dz && !aligned_to(bp.dz, 8)))
        return false;
    if (!bwd_get_encode()) return false;
    const long long P = (long long)bp.batch * bp.dim;
    const int sms = bwd_sm_count();
    if (P < sms) return false;
    const long long cap = (bp.io_bf16 ? kBwdWarpsBf16 : kBwdWarpsF32) * 8;
    const long long R = (P + sms - 1) / sms;
    const long long npass = (R + cap - 1) / cap;
    const long long rows_max = (R + npass - 1) / npass;
    if (rows_max > bp.dim) return false;   // a pass spans at most two batch rows
    *err = bp.io_bf16 ? launch_bwd_tma_cfg<__nv_bfloat16, kBwdWarpsBf16, 2>(bp, (int)rows_max, stream)
                      : launch_bwd_tma_cfg<float, kBwdWarpsF32, 2>(bp, (int)rows_max, stream);
    return true;
}

}  // namespace ssm
