// Forward selective scan, TMA-fed persistent kernel for sm_100a.
//
// Same arithmetic as ssm_fwd.cu (booiljung.github.io "3.2 선택적 스캔(Selective
// Scan) 알고리즘" §1.1/§1.2/§2.1, fused as in its §3.2): Δ = softplus(delta +
// bias), Ā = exp(Δ A), h = Ā h + Δ B u, y = C·h + D u, out = y silu(z).
//
// Layout of the work:
//  * One CTA per SM.  The batch*dim channel rows are split over the CTAs to
//    within one row, so every SM does the same amount of work; a CTA may run
//    its rows in several passes when they exceed one pass's capacity.
//  * One producer lane streams fixed-size time tiles (TT steps) of delta, u,
//    z (a [rows x TT] box each) and B, C (a [dstate x TT] box per batch row)
//    into a STAGES-deep shared-memory ring with 2-D TMA loads completing on
//    mbarriers.
//  * Consumer warps own 32/NT channels each (whole groups of rows; warps past
//    a pass's rows stay idle); lane (c, g) owns NS = N/NT
//    states of channel c and keeps them in fp32 registers for the whole
//    sequence.  Per tile a warp (1) computes Δ and Δ·u once per element into
//    a warp-private fp32 buffer, (2) runs the recurrence, two time steps per
//    f32x2 instruction and one ex2 per (step, state).  Lanes are numbered
//    state-group-major, so the eight lanes of a quarter-warp read the same
//    B/C row: a broadcast 16-byte shared load.  B and C stay in the io dtype
//    (converted in registers): the SFU is fed through the same MIO queue as
//    shared-memory instructions, so halving the B/C load count matters more
//    than the conversion ALU ops.  Each lane writes its partial readout
//    Σ_{own n} C h to shared memory,
//    (3) sums the NT partials, applies D·u and the SiLU gate and writes y
//    with 16-byte stores.  Warps synchronise only through the ring's
//    mbarriers; every wait is bounded (kWaitBudgetCycles).

#include <cudaTypedefs.h>

#include <stdlib.h>

#include <algorithm>
#include <type_traits>

#include "ssm_common.cuh"
#include "ssm_internal.h"
#include "ssm_tma.cuh"

// Build-time tuning knobs (defaults are the measured best on B200).
#ifndef SSM_TMA_STAGES
#define SSM_TMA_STAGES 3      // depth of the TMA ring for bf16 io
#endif
#ifndef SSM_TMA_POLY_PAIRS
#define SSM_TMA_POLY_PAIRS 0  // (state, step-pair) slots of 16 per block using ex2_poly2
#endif
#ifndef SSM_TMA_F32BC
#define SSM_TMA_F32BC 1       // producer rewrites B/C as fp32 (32-step tiles)
#endif
#ifndef SSM_TMA_CONV_SUBPART3
#define SSM_TMA_CONV_SUBPART3 1   // the B/C converter warp on SM sub-partition 3
#endif
#ifndef SSM_TMA_WAIT_SUSPEND
#define SSM_TMA_WAIT_SUSPEND 0    // waits suspend in the barrier unit instead of polling
#endif
#ifndef SSM_TMA_STEP_MAJOR
#define SSM_TMA_STEP_MAJOR 1      // recurrence loop ordered step-major (fp32 B/C, Δ·B only)
#endif
#ifndef SSM_TMA_SOFTPLUS_1SFU
#define SSM_TMA_SOFTPLUS_1SFU 1   // softplus with one SFU op (log1p on the FMA pipe)
#endif
#ifndef SSM_TMA_SUM_POLY
#define SSM_TMA_SUM_POLY 1        // quarters of a lane's states with FMA-pipe exponentials in chunk summaries
#endif
#ifndef SSM_TMA_UNROLL
#define SSM_TMA_UNROLL 2      // 8-step blocks unrolled in the recurrence loop
#endif

namespace ssm {

namespace {

constexpr int kTmaUnroll = SSM_TMA_UNROLL;
constexpr int kPolyPairs = SSM_TMA_POLY_PAIRS;
constexpr bool kStepMajor = SSM_TMA_STEP_MAJOR != 0;
constexpr int kSumPolyStates = SSM_TMA_SUM_POLY;
constexpr bool kSoftplus1Sfu = SSM_TMA_SOFTPLUS_1SFU != 0;

constexpr int align128(int x) { return (x + 127) / 128 * 128; }

struct TmaFwdParams {
    const float *A, *D, *delta_bias;
    const float *h0;    // [P][N] state before step 0; NULL: zeros
    float *delta_sum;   // [P] Σ_t Δ_t of each row, or NULL
    void *out;
    float *last_state, *ckpt;
    int P;          // batch * dim channel rows
    int dim, L, n_ckpt;
    // Time chunks (the two-level scan along L): the launch covers chunks
    // 0..K-1 of Lc steps each (the last one ends at L); the CTAs are split
    // evenly over the chunks, and a CTA's rows all lie in its chunk.  With
    // K = 1 (Lc = L) the launch is one ordinary pass over the sequence.
    // Chunk k's copy of row r is the virtual row v = k P + r; `virt` says
    // bit 1: h0 is indexed by virtual row; bit 2: last_state and delta_sum
    // are indexed by virtual row (else by row, and last_state is written by
    // the last chunk only).
    int K, Lc, virt;
    int softplus, has_z;
    int rows_max;   // rows of one pass (= box height of the per-channel maps)
    int *err;       // device error word
};

template <typename T, int NT, int NS, int TT, int NWC, int STAGES>
struct TmaLayout {
    static constexpr int N = NT * NS;
    static constexpr int CPW = 32 / NT;            // channels per consumer warp
    static constexpr int MAXR = NWC * CPW;         // rows per pass, at most
    static constexpr int ES = sizeof(T);
    static constexpr int RAW_ROW = TT * ES;
    static constexpr int RAW_CH = align128(MAXR * RAW_ROW);
    // B and C tiles: when a row spans >= 128 bytes it is loaded in 128-byte
    // pieces with the TMA 128B swizzle (16-byte chunk index XOR row % 8), so
    // lanes reading the same chunk of different rows hit different banks.
    static constexpr bool SWZ = RAW_ROW >= 128;
    static constexpr int PW = SWZ ? 128 : RAW_ROW;             // bytes per piece row
    static constexpr int NPIECE = RAW_ROW / PW;
    static constexpr int PIECE = 2 * N * PW;                   // one piece, two batch rows
    static constexpr int RAW_BC = NPIECE * PIECE;
    static constexpr int kBC0 = (3 * RAW_CH + 1023) / 1024 * 1024;
    // With 32-step tiles the producer warp also rewrites each B and C tile as
    // fp32 ([B or C][batch row][state][TT], 16-byte chunks swizzled so that
    // the state groups of a warp read different banks): consumers then load
    // four steps of B or C per 16-byte broadcast load, with no conversion.
    static constexpr bool F32BC = SSM_TMA_F32BC && TT == 32;
    static constexpr int BCF = 2 * 2 * N * TT;                 // floats of the fp32 copy
    static constexpr int kBCF0 = align128(kBC0 + 2 * RAW_BC);
    static constexpr int STAGE = (kBCF0 + (F32BC ? BCF * 4 : 0) + 1023) / 1024 * 1024;
    static constexpr int WS = TT + 4;                          // fp32 row stride (floats)
    static constexpr int WBUF = (2 + NT) * CPW * WS * 4;       // Δ, Δ·u, NT readout partials
    static constexpr int kW = STAGES * STAGE;
    static constexpr int kBar = kW + NWC * WBUF;
    static constexpr int kTotal = kBar + 3 * STAGES * 8;
    static constexpr int kAlloc = kTotal + 1024;   // room to align the base to 1024 B
    // Consumer warps 0..NWC-1, the TMA warp NWC and (with the fp32 B/C copy) a
    // converter warp.  Warp w runs on SM sub-partition w % 4, and the consumers
    // fill sub-partitions 0, 1, 2 first, so the converter takes the first index
    // after the TMA warp on sub-partition 3 (indices between stay idle).
    static constexpr int kConvWarp =
        SSM_TMA_CONV_SUBPART3 ? NWC + 1 + (3 - (NWC + 1) % 4 + 4) % 4 : NWC + 1;
    static constexpr int kThreads = (F32BC ? kConvWarp + 1 : NWC + 1) * 32;
    static constexpr int CHUNK = 8;                            // steps per prep/epilogue item
    static constexpr int ITEMS = CPW * (TT / CHUNK);           // (row, chunk) items per warp
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static_assert(TT % 8 == 0 && ITEMS % 32 == 0, "tile shape");
    static_assert(!SWZ || (RAW_ROW % 128 == 0 && PIECE % 1024 == 0), "swizzle atoms");
    static_assert(NT == 2 || NT == 4 || NT == 8 || NT == 16, "lane split");
};

// Loads 8 consecutive time steps of one B or C row from a raw stage tile
// (io dtype) as four fp32 pairs {t, t+1}.
template <typename T>
__device__ __forceinline__ void load_pairs8(const T *src, float2 (&v)[4]);

template <>
__device__ __forceinline__ void load_pairs8<__nv_bfloat16>(const __nv_bfloat16 *src, float2 (&v)[4]) {
    const uint4 q = *reinterpret_cast<const uint4 *>(src);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        v[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}

template <>
__device__ __forceinline__ void load_pairs8<float>(const float *src, float2 (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(src);
    const float4 b = *reinterpret_cast<const float4 *>(src + 4);
    v[0] = make_float2(a.x, a.y); v[1] = make_float2(a.z, a.w);
    v[2] = make_float2(b.x, b.y); v[3] = make_float2(b.z, b.w);
}

// Same, for chunks at separate addresses (the swizzled layout stores the two
// 16-byte halves of an fp32 8-step group apart; for bf16 `hi` is unused).
template <typename T>
__device__ __forceinline__ void load_pairs8_at(const T *lo, const T *hi, float2 (&v)[4]);

template <>
__device__ __forceinline__ void load_pairs8_at<__nv_bfloat16>(const __nv_bfloat16 *lo, const __nv_bfloat16 *,
                                                              float2 (&v)[4]) {
    load_pairs8<__nv_bfloat16>(lo, v);
}

template <>
__device__ __forceinline__ void load_pairs8_at<float>(const float *lo, const float *hi, float2 (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(lo);
    const float4 b = *reinterpret_cast<const float4 *>(hi);
    v[0] = make_float2(a.x, a.y); v[1] = make_float2(a.z, a.w);
    v[2] = make_float2(b.x, b.y); v[3] = make_float2(b.z, b.w);
}

// FL >= 0: the gate, softplus and checkpoint options are compile-time bits
// (1: gate z, 2: softplus, 4: checkpoints); B̄ = Δ B.  FL = -1: the options
// are read at run time; B̄ = Δ B.  FL = -2: options at run time, zero-order
// hold B̄ = φ(Δ A) Δ B.  FL = -3 / -4: chunk summaries of the two-level scan
// (no readout, no output), with / without softplus: each row's end state
// from a zero state, and Σ Δ.  Only the run-time-option kernels (FL < 0) can also write the per-row
// delta sums: the code is left out of the others, where it measured 4 %
// slower even unused.
template <typename T, int NT, int NS, int TT, int NWC, int STAGES, int FL>
__global__ void __launch_bounds__(TmaLayout<T, NT, NS, TT, NWC, STAGES>::kThreads, 1)
fwd_tma_kernel(const __grid_constant__ CUtensorMap m_delta, const __grid_constant__ CUtensorMap m_u,
               const __grid_constant__ CUtensorMap m_z, const __grid_constant__ CUtensorMap m_B,
               const __grid_constant__ CUtensorMap m_C, const TmaFwdParams p) {
    using Ly = TmaLayout<T, NT, NS, TT, NWC, STAGES>;
    constexpr int N = Ly::N, CPW = Ly::CPW, WS = Ly::WS, CHUNK = Ly::CHUNK;
    constexpr int IPL = Ly::ITEMS / 32;   // prep/epilogue items per lane
    constexpr int CPR = TT / CHUNK;       // chunks per row
    constexpr bool ZOH = FL == -2;
    constexpr bool kSummary = FL == -3 || FL == -4;
    constexpr bool kDsum = FL < 0;   // delta sums only in the run-time-option kernels
    const bool has_z = kSummary ? false : FL < 0 ? p.has_z != 0 : (FL & 1) != 0;
    const bool softplus = kSummary ? FL == -3 : FL < 0 ? p.softplus != 0 : (FL & 2) != 0;
    float *const ckpt = kSummary ? nullptr : (FL < 0 || (FL & 4)) ? p.ckpt : nullptr;

    extern __shared__ __align__(128) uint8_t smem_raw[];
    // 1024-byte aligned base: the 128B-swizzle pattern of the B/C tiles repeats
    // every 1024 bytes of shared-memory address
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Ly::kBar);
    uint64_t *empty = full + STAGES;
    uint64_t *bcready = empty + STAGES;   // the producer wrote the fp32 B/C of a stage

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // this CTA's time chunk kc (CTAs [g0, g1) share it) and its rows [r0, r1)
    const int G = gridDim.x;
    const int kc = (int)((long long)blockIdx.x * p.K / G);
    const int g0 = (int)(((long long)kc * G + p.K - 1) / p.K);
    const int g1 = (int)(((long long)(kc + 1) * G + p.K - 1) / p.K);
    const int r0 = (int)((long long)(blockIdx.x - g0) * p.P / (g1 - g0));
    const int r1 = (int)((long long)(blockIdx.x - g0 + 1) * p.P / (g1 - g0));
    const int R = r1 - r0;
    const int T0 = kc * p.Lc;                     // the chunk's steps [T0, T1)
    const int T1 = min(p.L, T0 + p.Lc);
    const long long voff = (long long)kc * p.P;   // virtual row of row 0
    const int npass = (R + p.rows_max - 1) / p.rows_max;
    const int ntiles = (T1 - T0 + TT - 1) / TT;
    const int total = npass * ntiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, NWC);
            mbar_init(bcready + s, 1);
        }
        fence_barrier_init();
    }
    __syncthreads();

    // rows of pass q: [q0, q1), split evenly
    auto pass_rows = [&](int q, int &q0, int &q1) {
        q0 = r0 + (int)((long long)q * R / npass);
        q1 = r0 + (int)((long long)(q + 1) * R / npass);
    };

    // batch rows [b_lo, b_lo + nb) of the pass that tile kk belongs to
    auto tile_batches = [&](int kk, int &b_lo, int &nb) {
        int a0, a1;
        pass_rows(kk / ntiles, a0, a1);
        b_lo = a0 / p.dim;
        nb = (a1 - 1) / p.dim - b_lo + 1;
    };

    if (warp == NWC) {
        // ------------------------------------------------------- TMA producer
        if (lane != 0) return;
        prefetch_tensormap(&m_delta);
        prefetch_tensormap(&m_u);
        if (has_z) prefetch_tensormap(&m_z);
        prefetch_tensormap(&m_B);
        prefetch_tensormap(&m_C);
        int issued = 0;
        for (; issued < total; ++issued) {
            const int si = issued % STAGES;
            if (issued >= STAGES &&   // wait until every consumer left this stage
                !mbar_wait_sleep(empty + si, ((issued / STAGES) & 1) ^ 1, p.err, 64))
                break;
            int a0, a1, b_lo, nb;
            pass_rows(issued / ntiles, a0, a1);
            tile_batches(issued, b_lo, nb);
            const int t0 = T0 + (issued % ntiles) * TT;
            uint8_t *st = smem + si * Ly::STAGE;
            const uint32_t bytes = (uint32_t)(p.rows_max * Ly::RAW_ROW * (has_z ? 3 : 2) +
                                              2 * nb * N * Ly::RAW_ROW);
            mbar_arrive_expect_tx(full + si, bytes);
            tma_load_2d(st, &m_delta, t0, a0, full + si);
            tma_load_2d(st + Ly::RAW_CH, &m_u, t0, a0, full + si);
            if (has_z) tma_load_2d(st + 2 * Ly::RAW_CH, &m_z, t0, a0, full + si);
            for (int bs = 0; bs < nb; ++bs)
                for (int pc = 0; pc < Ly::NPIECE; ++pc) {
                    const int off = Ly::kBC0 + pc * Ly::PIECE + bs * N * Ly::PW;
                    const int x = t0 + pc * (Ly::PW / (int)sizeof(T));
                    tma_load_2d(st + off, &m_B, x, (b_lo + bs) * N, full + si);
                    tma_load_2d(st + off + Ly::RAW_BC, &m_C, x, (b_lo + bs) * N, full + si);
                }
        }
        // Never leave while a copy may still write shared memory: the last
        // STAGES loads are the only ones no consumer is known to have seen.
        for (int kk = (issued > STAGES ? issued - STAGES : 0); kk < issued; ++kk)
            if (!mbar_wait(full + (kk % STAGES), (kk / STAGES) & 1, p.err)) break;
        return;
    }
    if (warp > NWC && warp != Ly::kConvWarp) return;   // idle slots before the converter
    if constexpr (Ly::F32BC) {
        if (warp == Ly::kConvWarp) {
            // ------------------------------------------------ B/C converter
            // Each tile's B and C, once landed, rewritten as fp32 rows in the
            // stage's fp32 area (16-byte chunks swizzled by row / NS), then
            // announced on bcready.  The stage was refilled only after every
            // consumer left it, so its fp32 area is free.
            constexpr int CH = TT / 4;                 // fp32 16-byte chunks per row
            constexpr int PER_LANE = N * CH / 32;      // (state, chunk) items per lane
            static_assert(N * CH % 32 == 0, "items per lane");
            for (int kk = 0; kk < total; ++kk) {
                const int si = kk % STAGES;
#if SSM_TMA_WAIT_SUSPEND
                if (!__all_sync(0xffffffffu, mbar_wait_suspend(full + si, (kk / STAGES) & 1, p.err))) return;
#else
                if (!__all_sync(0xffffffffu, mbar_wait(full + si, (kk / STAGES) & 1, p.err))) return;
#endif
                int b_lo, nb;
                tile_batches(kk, b_lo, nb);
                const uint8_t *raw = smem + si * Ly::STAGE + Ly::kBC0;
                float *dst = reinterpret_cast<float *>(smem + si * Ly::STAGE + Ly::kBCF0);
                for (int which = 0; which < 2; ++which)
                    for (int bs = 0; bs < nb; ++bs) {
#pragma unroll
                        for (int r = 0; r < PER_LANE; ++r) {
                            const int it = lane + 32 * r;
                            const int ch = it % CH, rr = bs * N + it / CH;
                            constexpr int ES = (int)sizeof(T);
                            const int byte = ch * 4 * ES;
                            const int pc = byte / Ly::PW, in = byte % Ly::PW;
                            int rch = in >> 4;
                            if constexpr (Ly::SWZ) rch ^= (rr & 7);
                            const uint8_t *src = raw + which * Ly::RAW_BC + pc * Ly::PIECE + rr * Ly::PW + rch * 16;
                            float4 v;
                            if constexpr (ES == 2) {
                                const uint2 q2 = *reinterpret_cast<const uint2 *>(src + (in & 15));
                                v = make_float4(__uint_as_float(q2.x << 16), __uint_as_float(q2.x & 0xffff0000u),
                                                __uint_as_float(q2.y << 16), __uint_as_float(q2.y & 0xffff0000u));
                            } else {
                                v = *reinterpret_cast<const float4 *>(src);
                            }
                            float *drow = dst + (which * 2 * N + rr) * TT;
                            *reinterpret_cast<float4 *>(drow + ((ch ^ ((rr / NS) & 7)) << 2)) = v;
                        }
                    }
                __syncwarp();
                if (lane == 0) mbar_arrive(bcready + si);
            }
            return;
        }
    }

    // ---------------------------------------------------------------- consumers
    // Scan mapping: lane = g * CPW + c (a quarter-warp shares one state group,
    // so its B/C reads are one broadcast row).  Prep/epilogue mapping: item
    // lane + 32 i = (row, 8-step chunk), contiguous in shared memory.
    const int c = lane % CPW, g = lane / CPW;
    float *wDt = reinterpret_cast<float *>(smem + Ly::kW + warp * Ly::WBUF);
    float *wDu = wDt + CPW * WS;
    float *wY = wDu + CPW * WS;      // [NT][CPW][WS] readout partials

    float2 A2d[NS];                  // A[d, n] log2(e), duplicated for f32x2 math
    float2 iAd[NS];                  // 1 / A[d, n], duplicated (zero-order hold only)
    float h[NS];
    bool poly_ok = false;            // every A of this warp <= 0 (ex2_poly2 applies)
    int bsel = 0;
    bool live = false;
    // per-item constants for the prep / epilogue rows
    float Dd[IPL], bias[IPL];
    float dsum[IPL];                 // Σ Δ of this lane's prep items over the pass (delta_sum)
    int irow[IPL];

    int s = 0, phase = 0;          // ring slot and its parity for tile kg
    int q = 0, tile = 0, q0 = 0, q1 = 0;
    // Each warp takes a whole group of CPW rows of the pass (the last busy
    // warp may hold fewer); warps past the pass's rows stay idle.  Fewer,
    // fuller warps issue fewer instructions for the same rows than rows
    // spread over every warp.
    constexpr int rpw = CPW;
    for (int kg = 0; kg < total; ++kg) {
        if (tile == 0) {
            pass_rows(q, q0, q1);
        }
        const int t0 = T0 + tile * TT;
        const int wrow0 = q0 + warp * rpw;   // first row of this warp in the pass
        const int wend = min(wrow0 + rpw, q1);
        if (tile == 0) {
            const int row = wrow0 + c;
            live = row < wend;
            const int d = live ? row % p.dim : 0;
            bsel = live ? row / p.dim - q0 / p.dim : 0;
            bool neg = true;
#pragma unroll
            for (int j = 0; j < NS; ++j) {
                const float av = live ? p.A[(size_t)d * N + g * NS + j] : 0.f;
                const float a = av * SSM_LOG2E;
                A2d[j] = make_float2(a, a);
                if constexpr (ZOH) {
                    const float ia = 1.f / av;
                    iAd[j] = make_float2(ia, ia);
                }
                h[j] = (live && p.h0) ? p.h0[(size_t)((p.virt & 1) ? voff + row : row) * N + g * NS + j] : 0.f;
                neg = neg && a <= 0.f;
            }
            poly_ok = __all_sync(0xffffffffu, neg);
#pragma unroll
            for (int i = 0; i < IPL; ++i) {
                const int rr = wrow0 + (lane + 32 * i) / CPR;
                const bool ok = rr < wend;
                const int dd = ok ? rr % p.dim : 0;
                irow[i] = ok ? rr : -1;
                dsum[i] = 0.f;
                Dd[i] = (ok && p.D) ? p.D[dd] : 0.f;
                bias[i] = (ok && p.delta_bias) ? p.delta_bias[dd] : 0.f;
            }
        }
        // every lane waits; the warp leaves together if any wait gave up
        {
#if SSM_TMA_WAIT_SUSPEND
            bool ok = mbar_wait_suspend(full + s, phase, p.err);
            if constexpr (Ly::F32BC) ok = ok && mbar_wait_suspend(bcready + s, phase, p.err);
#else
            bool ok = mbar_wait(full + s, phase, p.err);
            if constexpr (Ly::F32BC) ok = ok && mbar_wait(bcready + s, phase, p.err);
#endif
            if (!__all_sync(0xffffffffu, ok)) return;
        }

        if (wrow0 < wend) {
            const uint8_t *st = smem + s * Ly::STAGE;
            const T *rawD = reinterpret_cast<const T *>(st) + warp * rpw * TT;
            const T *rawU = reinterpret_cast<const T *>(st + Ly::RAW_CH) + warp * rpw * TT;
            const T *rawZ = reinterpret_cast<const T *>(st + 2 * Ly::RAW_CH) + warp * rpw * TT;
            // (1) Δ and Δ·u, once per element (pairs of steps in f32x2 math)
            const bool full_tile = t0 + TT <= T1;
#pragma unroll
            for (int i = 0; i < IPL; ++i) {
                const int it = lane + 32 * i, rl = it / CPR, t = (it % CPR) * CHUNK;
                float dt[CHUNK], du[CHUNK];
#pragma unroll
                for (int v0 = 0; v0 < CHUNK; v0 += IO<T>::kVec) {
                    constexpr int V = IO<T>::kVec;
                    float dr[V], uu[V];
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawD + rl * TT + t + v0), dr);
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawU + rl * TT + t + v0), uu);
#pragma unroll
                    for (int k = 0; k < V; k += 2) {
                        const float2 r = __fadd2_rn(make_float2(dr[k], dr[k + 1]), make_float2(bias[i], bias[i]));
                        float2 d2 = softplus ? (kSoftplus1Sfu ? softplus_fast2_1sfu(r) : softplus_fast2(r)) : r;
                        if (!full_tile) {
                            const bool ok0 = irow[i] >= 0 && (t0 + t + v0 + k) < T1;
                            const bool ok1 = irow[i] >= 0 && (t0 + t + v0 + k + 1) < T1;
                            d2 = make_float2(ok0 ? d2.x : 0.f, ok1 ? d2.y : 0.f);
                        } else if (irow[i] < 0) {
                            d2 = make_float2(0.f, 0.f);
                        }
                        const float2 u2 = __fmul2_rn(d2, make_float2(uu[k], uu[k + 1]));
                        dt[v0 + k] = d2.x; dt[v0 + k + 1] = d2.y;
                        du[v0 + k] = u2.x; du[v0 + k + 1] = u2.y;
                    }
                }
                if (kDsum && p.delta_sum) {
#pragma unroll
                    for (int k = 0; k < CHUNK; ++k) dsum[i] += dt[k];
                }
#pragma unroll
                for (int k = 0; k < CHUNK; k += 4) {
                    *reinterpret_cast<float4 *>(wDt + rl * WS + t + k) = make_float4(dt[k], dt[k + 1], dt[k + 2], dt[k + 3]);
                    *reinterpret_cast<float4 *>(wDu + rl * WS + t + k) = make_float4(du[k], du[k + 1], du[k + 2], du[k + 3]);
                }
            }
            __syncwarp();
            // (2) the recurrence, two time steps per f32x2 op; B and C are read
            // in the io dtype straight from the TMA tile, the eight lanes of a
            // quarter-warp reading the same row (a broadcast load)
            const uint8_t *rawB = st + Ly::kBC0;
            const uint8_t *rawC = rawB + Ly::RAW_BC;
            // byte address of the 16-byte chunk holding steps [tb, tb + 16/size)
            // of state row rr (within the two-batch-row B or C tile)
            auto bc_chunk = [&](const uint8_t *base, int rr, int tb) -> const T * {
                const int byte = tb * (int)sizeof(T);
                const int pc = byte / Ly::PW, in = byte % Ly::PW;
                int chunk = in >> 4;
                if constexpr (Ly::SWZ) chunk ^= (rr & 7);
                return reinterpret_cast<const T *>(base + pc * Ly::PIECE + rr * Ly::PW + (chunk << 4));
            };
            const int rr0 = bsel * N + g * NS;
            // fp32 copy of B and C: rows of this lane's states, and the chunk
            // swizzle key of those rows (one per lane)
            const float *bcfB = reinterpret_cast<const float *>(st + Ly::kBCF0) + rr0 * TT;
            const float *bcfC = bcfB + 2 * N * TT;
            const int bkey = (rr0 / NS) & 7;
            float *myY = wY + (g * CPW + c) * WS;
            float *ck_row = (live && ckpt) ? ckpt + (size_t)(wrow0 + c) * p.n_ckpt * N + g * NS : nullptr;
            static_assert(SSM_CKPT_CHUNK == 8, "checkpoints are written per 8-step block");
            // one 8-step block of the recurrence; USE_POLY evaluates some of the
            // exponentials with ex2_poly2 on the FMA pipe instead of the SFU
            auto run_blocks = [&](auto use_poly) {
                constexpr bool kPoly = decltype(use_poly)::value;
#pragma unroll kTmaUnroll
                for (int tb = 0; tb < TT; tb += 8) {
                    float2 dtp[4], dup[4];
                    {
                        const float4 a = *reinterpret_cast<const float4 *>(wDt + c * WS + tb);
                        const float4 b = *reinterpret_cast<const float4 *>(wDt + c * WS + tb + 4);
                        const float4 e = *reinterpret_cast<const float4 *>(wDu + c * WS + tb);
                        const float4 f = *reinterpret_cast<const float4 *>(wDu + c * WS + tb + 4);
                        dtp[0] = make_float2(a.x, a.y); dtp[1] = make_float2(a.z, a.w);
                        dtp[2] = make_float2(b.x, b.y); dtp[3] = make_float2(b.z, b.w);
                        dup[0] = make_float2(e.x, e.y); dup[1] = make_float2(e.z, e.w);
                        dup[2] = make_float2(f.x, f.y); dup[3] = make_float2(f.z, f.w);
                    }
                    float2 idt[4];           // 1/Δ per step (zero-order hold only)
                    if constexpr (ZOH) {
#pragma unroll
                        for (int pp = 0; pp < 4; ++pp)
                            idt[pp] = make_float2(rcp_approx(dtp[pp].x), rcp_approx(dtp[pp].y));
                    }
                    float2 y2[4];
#pragma unroll
                    for (int pp = 0; pp < 4; ++pp) y2[pp] = make_float2(0.f, 0.f);
                    if constexpr (kSummary) {
                        // chunk summary: the recurrence alone (no readout);
                        // with every A of the warp <= 0, the first
                        // kSumPolyStates quarters of each lane's states take
                        // their exponentials on the FMA pipe (ex2_poly2),
                        // since this pass leaves issue slots free and the SFU
                        // is the bound
#pragma unroll
                        for (int hb = 0; hb < 2; ++hb) {
                            float4 Bv[NS];
#pragma unroll
                            for (int j = 0; j < NS; ++j) {
                                if constexpr (Ly::F32BC) {
                                    const int cc = (((tb >> 2) + hb) ^ bkey) << 2;
                                    Bv[j] = *reinterpret_cast<const float4 *>(bcfB + j * TT + cc);
                                } else {
                                    float2 bq[4];
                                    load_pairs8_at<T>(bc_chunk(rawB, rr0 + j, tb), bc_chunk(rawB, rr0 + j, tb + 4), bq);
                                    Bv[j] = make_float4(bq[2 * hb].x, bq[2 * hb].y, bq[2 * hb + 1].x, bq[2 * hb + 1].y);
                                }
                            }
#pragma unroll
                            for (int pq = 0; pq < 2; ++pq) {
                                const int pp = 2 * hb + pq;
                                float2 a[NS], beta[NS];
#pragma unroll
                                for (int j = 0; j < NS; ++j) {
                                    const float2 arg = __fmul2_rn(dtp[pp], A2d[j]);
                                    if (kPoly && j < (NS * kSumPolyStates + 3) / 4)
                                        a[j] = ex2_poly2(arg);
                                    else
                                        a[j] = make_float2(ex2(arg.x), ex2(arg.y));
                                    const float2 bb = pq ? make_float2(Bv[j].z, Bv[j].w) : make_float2(Bv[j].x, Bv[j].y);
                                    beta[j] = __fmul2_rn(dup[pp], bb);
                                }
#pragma unroll
                                for (int j = 0; j < NS; ++j) h[j] = fmaf(a[j].y, fmaf(a[j].x, h[j], beta[j].x), beta[j].y);
                            }
                        }
                    } else if constexpr (Ly::F32BC && !ZOH && !kPoly && kStepMajor) {
                        // step-major order: per pair of steps, every state's
                        // exponentials, then the NS independent recurrence
                        // chains side by side, then the readout
#pragma unroll
                        for (int hb = 0; hb < 2; ++hb) {
                            const int cc = (((tb >> 2) + hb) ^ bkey) << 2;
                            float4 Bv[NS], Cv[NS];
#pragma unroll
                            for (int j = 0; j < NS; ++j) {
                                Bv[j] = *reinterpret_cast<const float4 *>(bcfB + j * TT + cc);
                                Cv[j] = *reinterpret_cast<const float4 *>(bcfC + j * TT + cc);
                            }
#pragma unroll
                            for (int pq = 0; pq < 2; ++pq) {
                                const int pp = 2 * hb + pq;
                                float2 a[NS], beta[NS];
                                float hA[NS];
#pragma unroll
                                for (int j = 0; j < NS; ++j) {
                                    const float2 arg = __fmul2_rn(dtp[pp], A2d[j]);
                                    a[j] = make_float2(ex2(arg.x), ex2(arg.y));
                                    const float2 bb = pq ? make_float2(Bv[j].z, Bv[j].w) : make_float2(Bv[j].x, Bv[j].y);
                                    beta[j] = __fmul2_rn(dup[pp], bb);
                                }
#pragma unroll
                                for (int j = 0; j < NS; ++j) hA[j] = fmaf(a[j].x, h[j], beta[j].x);
#pragma unroll
                                for (int j = 0; j < NS; ++j) h[j] = fmaf(a[j].y, hA[j], beta[j].y);
                                float2 yy = make_float2(0.f, 0.f);
#pragma unroll
                                for (int j = 0; j < NS; ++j) {
                                    const float2 cv = pq ? make_float2(Cv[j].z, Cv[j].w) : make_float2(Cv[j].x, Cv[j].y);
                                    yy = __ffma2_rn(cv, make_float2(hA[j], h[j]), yy);
                                }
                                y2[pp] = yy;
                            }
                        }
                    } else {
#pragma unroll
                    for (int j = 0; j < NS; ++j) {
                        float2 bq[4], cq[4];
                        if constexpr (Ly::F32BC) {
                            const int c0 = ((tb >> 2) ^ bkey) << 2, c1 = (((tb >> 2) + 1) ^ bkey) << 2;
                            const float4 b0 = *reinterpret_cast<const float4 *>(bcfB + j * TT + c0);
                            const float4 b1 = *reinterpret_cast<const float4 *>(bcfB + j * TT + c1);
                            const float4 e0 = *reinterpret_cast<const float4 *>(bcfC + j * TT + c0);
                            const float4 e1 = *reinterpret_cast<const float4 *>(bcfC + j * TT + c1);
                            bq[0] = make_float2(b0.x, b0.y); bq[1] = make_float2(b0.z, b0.w);
                            bq[2] = make_float2(b1.x, b1.y); bq[3] = make_float2(b1.z, b1.w);
                            cq[0] = make_float2(e0.x, e0.y); cq[1] = make_float2(e0.z, e0.w);
                            cq[2] = make_float2(e1.x, e1.y); cq[3] = make_float2(e1.z, e1.w);
                        } else {
                            load_pairs8_at<T>(bc_chunk(rawB, rr0 + j, tb), bc_chunk(rawB, rr0 + j, tb + 4), bq);
                            load_pairs8_at<T>(bc_chunk(rawC, rr0 + j, tb), bc_chunk(rawC, rr0 + j, tb + 4), cq);
                        }
#pragma unroll
                        for (int pp = 0; pp < 4; ++pp) {
                            const float2 arg = __fmul2_rn(dtp[pp], A2d[j]);
                            float2 a;
                            if (kPoly && (pp * NS + j) % 16 < kPolyPairs) {
                                a = ex2_poly2(arg);
                            } else {
                                a = make_float2(ex2(arg.x), ex2(arg.y));
                            }
                            float2 beta = __fmul2_rn(dup[pp], bq[pp]);
                            if constexpr (ZOH) beta = __fmul2_rn(beta, zoh_phi2(arg, a, idt[pp], iAd[j]));
                            const float h0 = fmaf(a.x, h[j], beta.x);
                            const float h1 = fmaf(a.y, h0, beta.y);
                            h[j] = h1;
                            y2[pp] = __ffma2_rn(cq[pp], make_float2(h0, h1), y2[pp]);
                        }
                    }
                    }
                    if constexpr (!kSummary) {
                        *reinterpret_cast<float4 *>(myY + tb) = make_float4(y2[0].x, y2[0].y, y2[1].x, y2[1].y);
                        *reinterpret_cast<float4 *>(myY + tb + 4) = make_float4(y2[2].x, y2[2].y, y2[3].x, y2[3].y);
                    }
                    // checkpoint: the state after this 8-step block (a chunk)
                    if (ck_row && t0 + tb < T1) {
                        float *dst = ck_row + (size_t)((t0 + tb) / SSM_CKPT_CHUNK) * N;
#pragma unroll
                        for (int j = 0; j < NS; ++j) dst[j] = h[j];
                    }
                }
        
            };
            if ((kPolyPairs > 0 || (kSummary && kSumPolyStates > 0)) && poly_ok)
                run_blocks(std::integral_constant<bool, true>{});
            else
                run_blocks(std::integral_constant<bool, false>{});
            // the final state
            const int row = wrow0 + c;
            if (live && p.last_state && tile == ntiles - 1 && ((p.virt & 2) || kc == p.K - 1)) {
                float *dst = p.last_state + (size_t)((p.virt & 2) ? voff + row : row) * N + g * NS;
#pragma unroll
                for (int j = 0; j < NS; ++j) dst[j] = h[j];
            }
            __syncwarp();
            // (3) Σ of the NT partials, D skip, gate, 16-byte stores
#pragma unroll
            for (int i = 0; i < (kSummary ? 0 : IPL); ++i) {
                const int it = lane + 32 * i, rl = it / CPR, t = (it % CPR) * CHUNK;
                if (irow[i] < 0 || t0 + t >= T1) continue;
                float y[CHUNK];
#pragma unroll
                for (int k = 0; k < CHUNK; k += 4) {
                    float2 lo = make_float2(0.f, 0.f), hi = make_float2(0.f, 0.f);
#pragma unroll
                    for (int gg = 0; gg < NT; ++gg) {
                        const float4 q4 = *reinterpret_cast<const float4 *>(wY + (gg * CPW + rl) * WS + t + k);
                        lo = __fadd2_rn(lo, make_float2(q4.x, q4.y));
                        hi = __fadd2_rn(hi, make_float2(q4.z, q4.w));
                    }
                    y[k] = lo.x; y[k + 1] = lo.y; y[k + 2] = hi.x; y[k + 3] = hi.y;
                }
                T *out = static_cast<T *>(p.out) + (size_t)irow[i] * p.L + t0 + t;
#pragma unroll
                for (int v0 = 0; v0 < CHUNK; v0 += IO<T>::kVec) {
                    constexpr int V = IO<T>::kVec;
                    float uu[V], zz[V], o[V];
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawU + rl * TT + t + v0), uu);
                    if (has_z) IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawZ + rl * TT + t + v0), zz);
#pragma unroll
                    for (int k = 0; k < V; k += 2) {
                        float2 yy = __ffma2_rn(make_float2(Dd[i], Dd[i]), make_float2(uu[k], uu[k + 1]),
                                               make_float2(y[v0 + k], y[v0 + k + 1]));
                        if (has_z) {
                            if constexpr (sizeof(T) == 2) {
                                yy = __fmul2_rn(yy, silu_tanh2(make_float2(zz[k], zz[k + 1])));
                            } else {
                                yy.x *= zz[k] * sigmoid(zz[k]);
                                yy.y *= zz[k + 1] * sigmoid(zz[k + 1]);
                            }
                        }
                        o[k] = yy.x; o[k + 1] = yy.y;
                    }
                    __stcs(reinterpret_cast<uint4 *>(out + v0), IO<T>::pack(o));
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        if (++s == STAGES) { s = 0; phase ^= 1; }
        if (kDsum && tile == ntiles - 1 && p.delta_sum && wrow0 < wend) {
            // end of the pass: the CPR lanes holding a row's chunks (consecutive
            // lanes of one item index) sum their shares; the first one stores
#pragma unroll
            for (int i = 0; i < IPL; ++i) {
                float v = dsum[i];
#pragma unroll
                for (int m = 1; m < CPR; m <<= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
                if (irow[i] >= 0 && (lane % CPR) == 0) p.delta_sum[(p.virt & 2) ? voff + irow[i] : irow[i]] = v;
            }
        }
        if (++tile == ntiles) { tile = 0; ++q; }
    }
}

// ------------------------------------------------------------------ host side


template <typename T, int NT, int NS, int TT, int NWC, int STAGES, int FL>
cudaError_t launch_cfg(const FwdParams &fp, cudaStream_t stream) {
    using Ly = TmaLayout<T, NT, NS, TT, NWC, STAGES>;
    const int P = fp.batch * fp.dim;
    const int K = std::max(1, fp.K);
    const int grid = K > 1 ? device_sm_count() : std::min(device_sm_count(), P);
    const int gk = grid / K;                      // fewest CTAs of a chunk
    const int Lc = fp.Lc > 0 ? fp.Lc : fp.L;     // a chunk plan may cover less than L
    if (gk < 1 || (fp.Lc > 0 && (Lc % TT != 0 || (long long)(K - 1) * Lc >= fp.L)))
        return cudaErrorInvalidValue;   // chunks of whole tiles, each starting inside the sequence
    const int R = (P + gk - 1) / gk;
    const int npass = (R + Ly::MAXR - 1) / Ly::MAXR;
    const int rows_max = (R + npass - 1) / npass;
    const bool bf16 = sizeof(T) == 2;
    CUtensorMap md, mu, mz, mB, mC;
    if (!make_tma_map_2d(&md, fp.delta, bf16, P, fp.L, TT, rows_max, false) ||
        !make_tma_map_2d(&mu, fp.u, bf16, P, fp.L, TT, rows_max, false) ||
        !make_tma_map_2d(&mz, fp.z ? fp.z : fp.u, bf16, P, fp.L, TT, rows_max, false) ||
        !make_tma_map_2d(&mB, fp.B, bf16, (uint64_t)fp.batch * fp.N, fp.L, Ly::PW / sizeof(T), Ly::N, Ly::SWZ) ||
        !make_tma_map_2d(&mC, fp.C, bf16, (uint64_t)fp.batch * fp.N, fp.L, Ly::PW / sizeof(T), Ly::N, Ly::SWZ))
        return cudaErrorInvalidValue;
    TmaFwdParams p{};
    p.A = fp.A; p.D = fp.D; p.delta_bias = fp.delta_bias; p.out = fp.out;
    p.last_state = fp.last_state; p.ckpt = fp.ckpt; p.h0 = fp.h0; p.delta_sum = fp.delta_sum;
    p.P = P; p.dim = fp.dim; p.L = fp.L; p.n_ckpt = fp.n_ckpt;
    p.softplus = fp.softplus; p.has_z = fp.z != nullptr; p.rows_max = rows_max;
    p.K = K; p.Lc = Lc; p.virt = fp.virt;
    p.err = device_error_word();
    if (!p.err) return cudaErrorInvalidDevice;
    auto kern = fwd_tma_kernel<T, NT, NS, TT, NWC, STAGES, FL>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    kern<<<grid, Ly::kThreads, Ly::kAlloc, stream>>>(md, mu, mz, mB, mC, p);
    return cudaGetLastError();
}

// Launch configurations.  For a lane split NT (lanes per channel) the tile
// holds TT = max(32, 8 * NT) steps, so every lane owns one 8-step
// prep/epilogue item; the consumer-warp count NWC and ring depth STAGES are
// the largest the 227 KB shared-memory budget allows (static_assert in
// TmaLayout).
template <typename T, int N, int NT> struct TmaCfg;
#define SSM_TMA_CFG(T_, N_, NT_, NWC_, ST_)                                   \
    template <> struct TmaCfg<T_, N_, NT_> {                                  \
        static constexpr int TT = (8 * NT_ > 32 ? 8 * NT_ : 32);              \
        static constexpr int NWC = NWC_, STAGES = ST_;                        \
        static constexpr int MAXR = NWC_ * (32 / NT_);                        \
    };
using bf16_t = __nv_bfloat16;
SSM_TMA_CFG(bf16_t, 16, 2, 9, SSM_TMA_STAGES)
#ifndef SSM_TMA_NWC_BF16_N16
#define SSM_TMA_NWC_BF16_N16 12
#endif
#ifndef SSM_TMA_STAGES_NT4
#define SSM_TMA_STAGES_NT4 SSM_TMA_STAGES
#endif
SSM_TMA_CFG(bf16_t, 16, 4, SSM_TMA_NWC_BF16_N16, SSM_TMA_STAGES_NT4)
SSM_TMA_CFG(bf16_t, 16, 8, 12, 3)
SSM_TMA_CFG(bf16_t, 16, 16, 7, 3)
SSM_TMA_CFG(bf16_t, 32, 4, 12, SSM_TMA_STAGES)
SSM_TMA_CFG(bf16_t, 32, 8, 10, 3)
SSM_TMA_CFG(bf16_t, 32, 16, 7, 2)
SSM_TMA_CFG(bf16_t, 8, 2, 9, SSM_TMA_STAGES)
SSM_TMA_CFG(bf16_t, 8, 4, 12, 3)
SSM_TMA_CFG(bf16_t, 8, 8, 12, 3)
SSM_TMA_CFG(float, 16, 2, 8, 2)
SSM_TMA_CFG(float, 16, 4, 8, 2)
SSM_TMA_CFG(float, 16, 8, 8, 2)
SSM_TMA_CFG(float, 16, 16, 6, 2)
SSM_TMA_CFG(float, 32, 4, 8, 2)
SSM_TMA_CFG(float, 32, 8, 6, 2)
SSM_TMA_CFG(float, 32, 16, 3, 2)
SSM_TMA_CFG(float, 8, 2, 8, 2)
SSM_TMA_CFG(float, 8, 4, 8, 2)
SSM_TMA_CFG(float, 8, 8, 8, 2)
#undef SSM_TMA_CFG

template <typename T, int N, int NT>
cudaError_t launch_nt(const FwdParams &fp, cudaStream_t stream) {
    using C = TmaCfg<T, N, NT>;
    if (fp.summary)
        return fp.softplus ? launch_cfg<T, NT, N / NT, C::TT, C::NWC, C::STAGES, -3>(fp, stream)
                           : launch_cfg<T, NT, N / NT, C::TT, C::NWC, C::STAGES, -4>(fp, stream);
    if constexpr (N == 16) {   // zero-order hold: dstate 16 only (else the general kernel)
        if (fp.zoh) return launch_cfg<T, NT, N / NT, C::TT, C::NWC, C::STAGES, -2>(fp, stream);
    }
    // the benchmarked bf16 dstate-16 splits get compile-time options for the
    // usual combinations (gate and softplus on, with or without checkpoints;
    // no delta sums)
    if constexpr (sizeof(T) == 2 && N == 16 && (NT == 2 || NT == 4 || NT == 16)) {
        const int fl = (fp.z ? 1 : 0) | (fp.softplus ? 2 : 0) | (fp.ckpt ? 4 : 0);
        if (!fp.delta_sum && fl == 3) return launch_cfg<T, NT, N / NT, C::TT, C::NWC, C::STAGES, 3>(fp, stream);
        if (!fp.delta_sum && fl == 7) return launch_cfg<T, NT, N / NT, C::TT, C::NWC, C::STAGES, 7>(fp, stream);
    }
    return launch_cfg<T, NT, N / NT, C::TT, C::NWC, C::STAGES, -1>(fp, stream);
}

template <typename T, int N, int NT>
constexpr int maxr() { return TmaCfg<T, N, NT>::MAXR; }

// Lane splits available for each dstate, fewest lanes per channel first.
template <typename T, int N>
cudaError_t launch_n(const FwdParams &fp, int nt, cudaStream_t stream) {
    if constexpr (N == 8) {
        if (nt == 2) return launch_nt<T, 8, 2>(fp, stream);
        if (nt == 4) return launch_nt<T, 8, 4>(fp, stream);
        return launch_nt<T, 8, 8>(fp, stream);
    } else if constexpr (N == 16) {
        if (nt == 2) return launch_nt<T, 16, 2>(fp, stream);
        if (nt == 4) return launch_nt<T, 16, 4>(fp, stream);
        if (nt == 8) return launch_nt<T, 16, 8>(fp, stream);
        return launch_nt<T, 16, 16>(fp, stream);
    } else {
        if (nt == 4) return launch_nt<T, 32, 4>(fp, stream);
        if (nt == 8) return launch_nt<T, 32, 8>(fp, stream);
        return launch_nt<T, 32, 16>(fp, stream);
    }
}

template <typename T>
int rows_cap(int N, int nt) {
    if (N == 8) return nt == 2 ? maxr<T, 8, 2>() : nt == 4 ? maxr<T, 8, 4>() : maxr<T, 8, 8>();
    if (N == 16)
        return nt == 2 ? maxr<T, 16, 2>() : nt == 4 ? maxr<T, 16, 4>() : nt == 8 ? maxr<T, 16, 8>()
                                                                              : maxr<T, 16, 16>();
    return nt == 4 ? maxr<T, 32, 4>() : nt == 8 ? maxr<T, 32, 8>() : maxr<T, 32, 16>();
}

bool nt_valid(int N, int nt) {
    if (N == 8) return nt == 2 || nt == 4 || nt == 8;
    if (N == 16) return nt == 2 || nt == 4 || nt == 8 || nt == 16;
    return nt == 4 || nt == 8 || nt == 16;
}

}  // namespace

// Returns true (and launches) when the TMA path applies; false means the
// caller should use the general kernel.
bool try_launch_fwd_tma(const FwdParams &fp, cudaStream_t stream, cudaError_t *err) {
    if (!fp.vec_ok || !(fp.out || fp.summary) || (fp.zoh && fp.N != 16)) return false;   // ZOH: dstate 16 here
    if (fp.summary && fp.zoh) return false;
    if (fp.N != 8 && fp.N != 16 && fp.N != 32) return false;
    if (!tma_available()) return false;
    const long long P = (long long)fp.batch * fp.dim;
    const int sms = device_sm_count();
    const int K = std::max(1, fp.K);
    const long long gk = sms / K;                   // fewest CTAs of a time chunk
    if (gk < 1 || P < gk) return false;             // fewer channels than CTAs
    const long long R = (P + gk - 1) / gk;          // rows per CTA
    // Lane split: the fewest lanes per channel that still give every SM
    // 8 warps of lanes (more states per lane = less per-state overhead);
    // chunk summaries, which carry no readout, settle for 4 warps.
    int nt = 0;
    for (int cand : {2, 4, 8, 16}) {
        if (!nt_valid(fp.N, cand)) continue;
        nt = cand;
        if (R * cand >= (fp.summary ? 128 : 256)) break;
    }
    // SSM_TMA_NT overrides the lane split (tuning knob)
    static const char *force_nt = getenv("SSM_TMA_NT");
    if (force_nt && nt_valid(fp.N, atoi(force_nt))) nt = atoi(force_nt);
    const long long cap = fp.io_bf16 ? rows_cap<__nv_bfloat16>(fp.N, nt) : rows_cap<float>(fp.N, nt);
    const long long npass = (R + cap - 1) / cap;
    const long long rows_pass = (R + npass - 1) / npass;
    if (rows_pass > fp.dim) return false;           // a pass may touch at most two batch rows
    cudaError_t e;
    if (fp.io_bf16) {
        using T = __nv_bfloat16;
        e = fp.N == 8 ? launch_n<T, 8>(fp, nt, stream)
          : fp.N == 16 ? launch_n<T, 16>(fp, nt, stream) : launch_n<T, 32>(fp, nt, stream);
    } else {
        using T = float;
        e = fp.N == 8 ? launch_n<T, 8>(fp, nt, stream)
          : fp.N == 16 ? launch_n<T, 16>(fp, nt, stream) : launch_n<T, 32>(fp, nt, stream);
    }
    *err = e;
    return true;
}

// ------------------------------------------------------------ two-level scan
// For long sequences over few channel rows, one pass leaves most of each SM
// idle: every (row, state) recurrence runs the whole length in one lane.  The
// sequence is then cut into K chunks, and the chunks of a row run side by side
// in three launches (booiljung.github.io, "3.2 선택적 스캔(Selective Scan)
// 알고리즘", §2.2: the pairs (Ā, b) compose with (a_j, b_j) • (a_i, b_i) =
// (a_j a_i, a_j b_i + b_j)):
//  1. summaries of chunks 0..K-2: the end state e_k of each chunk run from a
//     zero state, and Σ Δ over it (its decay product is exp(A Σ Δ));
//  2. the exclusive combine of the summaries in sequence order: the state
//     h_in[k] entering each chunk (launch_combine_carries);
//  3. every chunk run again from h_in[k], writing the output.
// Workspace: e [K-1][P][N], Σ Δ [K-1][P] (rounded up to 16 bytes), h_in
// [K][P][N], all fp32.

namespace {
constexpr int kChunkMinSteps = 512;      // shortest chunk worth a pipeline fill
size_t align16(size_t x) { return (x + 15) / 16 * 16; }

// Modelled time of one launch over K chunks of Lc steps: the passes of its
// busiest CTA times the warps on its busiest SM sub-partition times the
// states each lane carries and the chunk length, weighted by the measured
// cost per element-state of each lane split relative to 4 lanes per channel
// (16 lanes 1.55x, from the long-context forward; 2 lanes 0.85x, from a
// 128-row-per-SM chunked pass; 8 lanes taken as 1.3x).
double launch_cost(long long P, int dim, long long K, long long Lc, int N, bool bf16, int sms,
                   bool summary) {
    const long long gk = sms / K;
    if (gk < 1 || P < gk) return 1e300;        // a launch the TMA forward refuses
    const long long R = (P + gk - 1) / gk;
    int nt = 0;
    for (int cand : {2, 4, 8, 16}) {
        if (!nt_valid(N, cand)) continue;
        nt = cand;
        if (R * cand >= (summary ? 128 : 256)) break;
    }
    const long long cap = bf16 ? rows_cap<__nv_bfloat16>(N, nt) : rows_cap<float>(N, nt);
    const long long npass = (R + cap - 1) / cap, rp = (R + npass - 1) / npass;
    if (rp > dim) return 1e300;                 // a pass may touch at most two batch rows
    const long long warps = (rp + 32 / nt - 1) / (32 / nt);
    const double w = nt >= 16 ? 1.55 : nt == 8 ? 1.3 : nt == 2 ? 0.85 : 1.0;
    return (double)npass * (double)((warps + 3) / 4) * (N / nt) * (double)Lc * w;
}
}  // namespace

// The chunk plan: the K (and chunk length, whole 128-step blocks) that
// minimises the modelled time of the two-level scan (a summary pass counted at
// 0.7 of a full pass), taken only when that is below 0.85 of the one-pass
// forward's modelled time.  SSM_FWD_CHUNKS=K in the environment forces K.
size_t fwd_chunk_plan(const FwdParams &fp, int *Kp, int *Lcp) {
    if (!fp.vec_ok || fp.zoh || fp.delta_sum) return 0;
    if (fp.N != 8 && fp.N != 16 && fp.N != 32) return 0;
    if (!tma_available()) return 0;
    const long long P = (long long)fp.batch * fp.dim;
    const int sms = device_sm_count();
    if (sms < 2) return 0;
    static const char *force = getenv("SSM_FWD_CHUNKS");
    const long long forced = force ? atoll(force) : 0;
    long long bestK = 0, bestLc = 0;
    double best = 0.85 * launch_cost(P, fp.dim, 1, fp.L, fp.N, fp.io_bf16, sms, false);
    const long long kmax = std::min<long long>(sms, fp.L / kChunkMinSteps);
    for (long long K = 2; K <= kmax; ++K) {
        const long long Lc = ((fp.L + K - 1) / K + 127) / 128 * 128;
        const long long K2 = (fp.L + Lc - 1) / Lc;
        if (K2 < 2 || (forced >= 2 && K != forced)) continue;
        const double c = launch_cost(P, fp.dim, K2, Lc, fp.N, fp.io_bf16, sms, false) +
                         0.7 * launch_cost(P, fp.dim, K2 - 1, Lc, fp.N, fp.io_bf16, sms, true);
        if (c < best || (forced >= 2 && !bestK && c < 1e299)) {
            best = c;
            bestK = K2;
            bestLc = Lc;
        }
    }
    if (bestK < 2) return 0;
    if (Kp) *Kp = (int)bestK;
    if (Lcp) *Lcp = (int)bestLc;
    const size_t PN = (size_t)P * fp.N * sizeof(float);
    return (size_t)(bestK - 1) * PN + align16((size_t)(bestK - 1) * P * sizeof(float)) +
           (size_t)bestK * PN;
}

cudaError_t launch_fwd_chunked(const FwdParams &fp, void *ws, size_t ws_bytes, cudaStream_t stream) {
    int K = 0, Lc = 0;
    const size_t need = fwd_chunk_plan(fp, &K, &Lc);
    if (need == 0 || ws_bytes < need || !ws || (reinterpret_cast<uintptr_t>(ws) & 15)) return cudaErrorInvalidValue;
    const long long P = (long long)fp.batch * fp.dim;
    float *h_ends = static_cast<float *>(ws);
    float *dsums = h_ends + (size_t)(K - 1) * P * fp.N;
    float *h_in = reinterpret_cast<float *>(reinterpret_cast<char *>(dsums) +
                                           align16((size_t)(K - 1) * P * sizeof(float)));
    cudaError_t e = cudaSuccess;
    // 1. summaries of chunks 0..K-2 (end states from zero, Σ Δ), per virtual row
    FwdParams s = fp;
    s.out = nullptr; s.z = nullptr; s.ckpt = nullptr; s.h0 = nullptr;
    s.last_state = h_ends; s.delta_sum = dsums;
    s.K = K - 1; s.Lc = Lc; s.virt = 2; s.summary = true;
    if (!try_launch_fwd_tma(s, stream, &e)) return cudaErrorNotSupported;
    if (e != cudaSuccess) return e;
    // 2. the state entering each chunk (the caller's h0 enters chunk 0)
    e = launch_combine_carries(K, P, fp.dim, fp.N, fp.A, dsums, h_ends, fp.h0, h_in, stream);
    if (e != cudaSuccess) return e;
    // 3. every chunk from its carry-in; last_state from the last chunk
    FwdParams f = fp;
    f.h0 = h_in; f.K = K; f.Lc = Lc; f.virt = 1; f.summary = false;
    if (!try_launch_fwd_tma(f, stream, &e)) return cudaErrorNotSupported;
    set_kernel_path("fwd:chunked");
    return e;
}

}  // namespace ssm
