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
//  * One CTA per SM; channel rows (batch x dim) split evenly over the CTAs, in
//    units of 8 rows when dim is a multiple of 8.
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
//  * Sums over states for each (channel, step) -- y, Σ λ A Ā h, Σ λ B -- are
//    reduced over the channel's 4 state groups with warp shuffles, per 4-step
//    half-window, and finished per element by the lane that holds the total
//    (dz, du, ddelta; dD and dbias accumulate per lane).  Sums over channels for each
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

// Unroll factor of the loop over the 8-step windows of a tile.
#ifndef SSM_BWD_RECOMPUTE_A
#define SSM_BWD_RECOMPUTE_A 1       // Δ·B: form Ā again in the sweep too
#endif
#ifndef SSM_BWD_RECOMPUTE_A_ZOH
#define SSM_BWD_RECOMPUTE_A_ZOH 1   // zero-order hold: form Ā again in the sweep
#endif
#ifndef SSM_BWD_WIN_UNROLL
#define SSM_BWD_WIN_UNROLL 1
#endif
constexpr int kWinUnroll = SSM_BWD_WIN_UNROLL;

constexpr int bwd_align128(int x) { return (x + 127) / 128 * 128; }
constexpr int bwd_align1024(int x) { return (x + 1023) / 1024 * 1024; }

struct TmaBwdParams {
    const float *A, *D, *delta_bias, *ckpt;
    float *du, *ddelta, *dA, *dB, *dC, *dD, *dz, *ddelta_bias;
    int P, dim, L, n_ckpt;
    int softplus, has_z;
    int rows_max;
    int vec_out;     // du, ddelta, dz 16-byte aligned and L % 4 == 0
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
    // B and C of a tile in fp32, [B or C][batch row][state][TT]: rows of
    // BRS floats and a 16-byte pad after the first 8 states of a batch row,
    // so that the rows a warp reads at once (states 4g + j and, with the
    // neighbour-channel pairing, 4g + (j ^ 2)) start in 8 different banks;
    // two buffers (tiles alternate)
    static constexpr int BRS = TT + 4;
    static constexpr int BROW = N * BRS + 4;                           // one batch row of B or C
    static constexpr int BCF = 2 * 2 * BROW;                           // floats per buffer
    static constexpr int W = 8;                                        // window = checkpoint chunk
    static constexpr int NWIN = TT / W;
    static constexpr int WS = TT + 4;                                  // row of wDt / wDu / wGy
    static constexpr int XS = W * NS + 4;                              // row of the transpose
    // the same after the pairing: 16 floats, 16-byte chunk kk of lane 8g + c
    // stored at chunk kk ^ ((c >> 1) & 3), so that the stores and the
    // channel-sum reads both meet 8 different banks per quarter-warp
    static constexpr int XP = W * NS / 2;
    static constexpr int kWdt = 0, kWdu = CPW * WS, kWgy = 2 * CPW * WS;
    // per-element sums over the states, written by the windows and read by
    // the tile's epilogue: y, Σ λ A Ā h (scaled to units of A), Σ λ B, and
    // with zero-order hold Σ λ B Ā
    static constexpr int kWy = 3 * CPW * WS, kWsa = 4 * CPW * WS, kWsb = 5 * CPW * WS;
    static constexpr int kWsq = 6 * CPW * WS;
    static constexpr int kWx = 7 * CPW * WS;                           // [32][XS]
    static constexpr int WBUF = (kWx + 32 * XS) * 4;
    // dB/dC tile accumulator: [B or C][batch row][state][TT], rows rotated
    static constexpr int DBC_PAR = 2 * 2 * N * TT;
    static constexpr int kBCF = STAGES * STAGE;
    static constexpr int kW = kBCF + 2 * BCF * 4;
    static constexpr int kDBC = kW + NWC * WBUF;
    static constexpr int kBar = kDBC + 2 * DBC_PAR * 4;
    static constexpr int kTotal = kBar + (2 * STAGES + 6) * 8;
    static constexpr int kAlloc = kTotal + 1024;
    static constexpr int kThreads = (NWC + 1) * 32;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static_assert(CPW * (TT / W) == 32, "one prep item of 8 steps per lane");
    static_assert(SSM_CKPT_CHUNK == W, "windows are checkpoint chunks");
    static_assert(WS % 4 == 0 && XS == 36 && XP == 16 && TT == 32 && NT == 4 && W == 8, "row shapes");
    static_assert(BROW % 4 == 0, "16-byte rows");
};

// Column of step t of state n in the dB/dC accumulator.  The rotation puts
// the 32 (state, step) cells that one atomic instruction of a warp touches
// into 32 different banks.
__device__ __forceinline__ int dbc_col(int n, int t) { return (t + 8 * (n >> 2) + (n & 3)) & 31; }

// Offset (floats) of state row n of one batch row in the fp32 B/C tile.
template <int BRS>
__device__ __forceinline__ int bcf_row(int n) { return n * BRS + (n >> 3) * 4; }

__device__ __forceinline__ void red_add_v4(float *addr, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

// Read-only 16-byte load issued where it stands in the program, so that a
// prefetch is not moved next to its use.
__device__ __forceinline__ float4 ldg_f4_now(const float *ptr) {
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(ptr));
    return v;
}

__device__ __forceinline__ float2 ldg_f2_now(const float *ptr) {
    float2 v;
    asm volatile("ld.global.nc.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(ptr));
    return v;
}

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
    const float2 lo = __fadd2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
    const float2 hi = __fadd2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Sum over the 4 state groups of a channel (lanes c, c+8, c+16, c+24) of the
// partials of a 4-step half-window, held as (steps 0,1) and (steps 2,3):
// two butterfly rounds (xor 16, then xor 8) leave lane group g with the
// total of step g.
__device__ __forceinline__ float group_reduce4(float2 p01, float2 p23, int g) {
    const bool g1 = (g & 2) != 0, g0 = (g & 1) != 0;
    float2 keep = g1 ? p23 : p01;
    const float2 send = g1 ? p01 : p23;
    keep.x += __shfl_xor_sync(0xffffffffu, send.x, 16);
    keep.y += __shfl_xor_sync(0xffffffffu, send.y, 16);
    const float k = g0 ? keep.y : keep.x, o = g0 ? keep.x : keep.y;
    return k + __shfl_xor_sync(0xffffffffu, o, 8);
}

// ALN: the channel count is a multiple of 8 and CTAs and passes start on
// multiples of 8 rows, so that no warp's 8 channels span two batch rows.
// ZOH: zero-order hold, B̄ = φ(Δ A) Δ B with φ(x) = (e^x - 1)/x
// (booiljung.github.io, "3.2 선택적 스캔(Selective Scan) 알고리즘" §2.1), whose
// derivatives are d(φ Δ)/dΔ = Ā and d(φ Δ)/dA = Δ² ψ(Δ A); φ and ψ come from
// Ā, 1/Δ and 1/A (zoh_phi2, zoh_psi2), with no division per element-state.
template <typename T, int NWC, int STAGES, bool HZ, bool SP, bool ALN, bool ZOH>
__global__ void __launch_bounds__((NWC + 1) * 32, 1)
bwd_tma_kernel(const __grid_constant__ CUtensorMap m_delta, const __grid_constant__ CUtensorMap m_u,
               const __grid_constant__ CUtensorMap m_z, const __grid_constant__ CUtensorMap m_g,
               const __grid_constant__ CUtensorMap m_B, const __grid_constant__ CUtensorMap m_C,
               const TmaBwdParams p) {
    using Ly = BwdLayout<T, NWC, STAGES>;
    constexpr int N = Ly::N, NS = Ly::NS, TT = Ly::TT, CPW = Ly::CPW;
    // the reverse sweep forms Ā again instead of keeping it (frees 32
    // registers per lane for the zero-order-hold factors)
    constexpr bool kRecomputeA = ZOH ? SSM_BWD_RECOMPUTE_A_ZOH != 0 : SSM_BWD_RECOMPUTE_A != 0;
    constexpr int WS = Ly::WS, XS = Ly::XS, W = Ly::W;

    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Ly::kBar);
    uint64_t *empty = full + STAGES;
    uint64_t *dfull = empty + STAGES;   // all consumers added their dB/dC of a tile
    uint64_t *dempty = dfull + 2;       // the producer flushed and cleared that buffer
    uint64_t *bcready = dempty + 2;     // the producer converted B/C of a tile to fp32
    float *dbc = reinterpret_cast<float *>(smem + Ly::kDBC);
    float *bcf = reinterpret_cast<float *>(smem + Ly::kBCF);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int G = gridDim.x;
    constexpr int RU = ALN ? CPW : 1;   // rows are split in units of RU
    const int r0 = RU * (int)((long long)blockIdx.x * (p.P / RU) / G);
    const int r1 = RU * (int)((long long)(blockIdx.x + 1) * (p.P / RU) / G);
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
            mbar_init(bcready + b, 1);
        }
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < 2 * Ly::DBC_PAR; i += blockDim.x) dbc[i] = 0.f;
    __syncthreads();

    auto pass_rows = [&](int q, int &q0, int &q1) {
        q0 = r0 + RU * (int)((long long)q * (R / RU) / npass);
        q1 = r0 + RU * (int)((long long)(q + 1) * (R / RU) / npass);
    };
    // batch rows [b_lo, b_lo + nb) touched by pass q
    auto pass_batches = [&](int q, int &b_lo, int &nb) {
        int q0, q1;
        pass_rows(q, q0, q1);
        b_lo = q0 / p.dim;
        nb = (q1 - 1) / p.dim - b_lo + 1;
    };

    if (warp == NWC) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&m_delta);
            prefetch_tensormap(&m_u);
            if constexpr (HZ) prefetch_tensormap(&m_z);
            prefetch_tensormap(&m_g);
            prefetch_tensormap(&m_B);
            prefetch_tensormap(&m_C);
        }
        int is_ = 0;
        auto issue = [&](int kk) {   // lane 0: TMA loads of tile kk into stage kk % STAGES
            const int q = kk / ntiles, k = kk - q * ntiles, st_i = kk % STAGES;
            int q0, q1, b_lo, nb;
            pass_rows(q, q0, q1);
            pass_batches(q, b_lo, nb);
            const int t0 = (ntiles - 1 - k) * TT;
            uint8_t *st = smem + st_i * Ly::STAGE;
            const uint32_t bytes = (uint32_t)(p.rows_max * Ly::RAW_ROW * (3 + (HZ ? 1 : 0)) +
                                              2 * nb * N * Ly::RAW_ROW);
            mbar_arrive_expect_tx(full + st_i, bytes);
            tma_load_2d(st, &m_delta, t0, q0, full + st_i);
            tma_load_2d(st + Ly::RAW_CH, &m_u, t0, q0, full + st_i);
            if constexpr (HZ) tma_load_2d(st + 2 * Ly::RAW_CH, &m_z, t0, q0, full + st_i);
            tma_load_2d(st + 3 * Ly::RAW_CH, &m_g, t0, q0, full + st_i);
            for (int bs = 0; bs < nb; ++bs)
                for (int pc = 0; pc < Ly::NPIECE; ++pc) {
                    const int off = Ly::kBC0 + pc * Ly::PIECE + bs * N * Ly::PW;
                    const int x = t0 + pc * (Ly::PW / (int)sizeof(T));
                    tma_load_2d(st + off, &m_B, x, (b_lo + bs) * N, full + st_i);
                    tma_load_2d(st + off + Ly::RAW_BC, &m_C, x, (b_lo + bs) * N, full + st_i);
                }
        };
        // B/C of tile kk (landed in its stage) to fp32 in buffer kk & 1
        auto convert = [&](int kk) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait_sleep(full + kk % STAGES, (kk / STAGES) & 1, p.err, 64)))
                return false;
            int b_lo, nb;
            pass_batches(kk / ntiles, b_lo, nb);
            const uint8_t *st = smem + (kk % STAGES) * Ly::STAGE + Ly::kBC0;
            float *dstb = bcf + (kk & 1) * Ly::BCF;
            constexpr int CH = TT / 4;                      // fp32 chunks per row
            const int nitems = 2 * nb * N * CH;             // (B or C, batch row, state, chunk)
            for (int i = lane; i < nitems; i += 32) {
                const int ch = i % CH, rr = (i / CH) % (nb * N), which = i / (CH * nb * N);
                const int byte = ch * 4 * (int)sizeof(T);
                const int pc = byte / Ly::PW, in = byte % Ly::PW;
                int rch = in >> 4;
                if constexpr (Ly::SWZ) rch ^= (rr & 7);
                const uint8_t *src = st + which * Ly::RAW_BC + pc * Ly::PIECE + rr * Ly::PW;
                float v[4];
                if constexpr (sizeof(T) == 2) {
                    const uint2 q2 = *reinterpret_cast<const uint2 *>(src + rch * 16 + (in & 15));
                    v[0] = __uint_as_float(q2.x << 16); v[1] = __uint_as_float(q2.x & 0xffff0000u);
                    v[2] = __uint_as_float(q2.y << 16); v[3] = __uint_as_float(q2.y & 0xffff0000u);
                } else {
                    const float4 f = *reinterpret_cast<const float4 *>(src + rch * 16);
                    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
                }
                float *drow = dstb + (which * 2 + rr / N) * Ly::BROW + bcf_row<Ly::BRS>(rr % N);
                *reinterpret_cast<float4 *>(drow + ch * 4) = make_float4(v[0], v[1], v[2], v[3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bcready + (kk & 1));
            return true;
        };
        if (lane == 0)
            while (is_ < STAGES && is_ < total) issue(is_++);
        bool ok = convert(0);
        for (int kg = 0; ok && kg < total; ++kg) {
            // B/C of the next tile while the consumers work on this one; its
            // buffer was last read by tile kg - 1, whose dfull was awaited
            if (kg + 1 < total && !convert(kg + 1)) break;
            // every consumer is done with tile kg: flush its dB/dC, then refill the stage
            ok = __all_sync(0xffffffffu, mbar_wait_sleep(dfull + (kg & 1), (kg >> 1) & 1, p.err, 256));
            if (!ok) break;
            {
                const int q = kg / ntiles, k = kg - q * ntiles;
                const int t0 = (ntiles - 1 - k) * TT;
                int b_lo, nb;
                pass_batches(q, b_lo, nb);
                float *buf = dbc + (kg & 1) * Ly::DBC_PAR;
                constexpr int QPR = TT / 4;                 // float4 per accumulator row
                const int nvec = 2 * nb * N * QPR;
                for (int i = lane; i < nvec; i += 32) {
                    const int tq = i % QPR, n = (i / QPR) % N;
                    const int bs = (i / (QPR * N)) % nb, which = i / (QPR * N * nb);
                    const float *src = buf + ((which * 2 + bs) * N + n) * TT;
                    const int t = tq * 4;
                    const float4 v = make_float4(src[dbc_col(n, t)], src[dbc_col(n, t + 1)],
                                                 src[dbc_col(n, t + 2)], src[dbc_col(n, t + 3)]);
                    const int tg = t0 + t;
                    if (tg < p.L) {
                        float *dst = (which == 0 ? p.dB : p.dC) + ((size_t)(b_lo + bs) * N + n) * p.L + tg;
                        red_add_v4(dst, v);
                    }
                }
                __syncwarp();
                for (int i = lane; i < Ly::DBC_PAR / 4; i += 32)
                    reinterpret_cast<float4 *>(buf)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                __syncwarp();
                if (lane == 0) mbar_arrive(dempty + (kg & 1));
            }
            if (lane == 0 && is_ < total) {
                ok = mbar_wait_sleep(empty + (kg % STAGES), (kg / STAGES) & 1, p.err, 64);
                if (ok) issue(is_++);
            }
            ok = __all_sync(0xffffffffu, ok);
        }
        if (lane == 0) {
            // never leave while a copy may still write shared memory
            for (int kk = (is_ > STAGES ? is_ - STAGES : 0); kk < is_; ++kk)
                if (!mbar_wait(full + (kk % STAGES), (kk / STAGES) & 1, p.err)) break;
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int c = lane % CPW, g = lane / CPW;                 // scan: channel, state group
    // Pairing of neighbour channels (8-row aligned passes, where a warp's
    // channels share one batch row): lane c holds state 4g + (j ^ rot) in
    // register j, so that lanes c and c ^ 1 keep the same two states in
    // registers 2 and 3 and trade registers 0 and 1 when they sum their dB/dC
    // partials over the pair.
    constexpr bool PAIR = ALN;
    const int rot = PAIR ? (c & 1) << 1 : 0;
    const int it_rl = lane / (TT / W), it_t = (lane % (TT / W)) * W;   // prep: row, step offset
    float *wbase = reinterpret_cast<float *>(smem + Ly::kW + warp * Ly::WBUF);
    float *wDt = wbase + Ly::kWdt, *wDu = wbase + Ly::kWdu, *wGy = wbase + Ly::kWgy;
    float *wY = wbase + Ly::kWy, *wSa = wbase + Ly::kWsa, *wSb = wbase + Ly::kWsb;
    float *wSq = wbase + Ly::kWsq;
    float *wX = wbase + Ly::kWx;
    float *myX = wX + lane * (PAIR ? Ly::XP : XS);

    float2 A2p[NS], dA2[NS];                                   // (A log2 e) twice; dA partials
    float2 iA2[NS];                                            // 1 / A twice (zero-order hold)
    float lam[NS], anext[NS];
    float4 hpre = make_float4(0.f, 0.f, 0.f, 0.f);             // checkpoint of the next window
    float dD_acc = 0.f, db_acc = 0.f, i_D = 0.f, i_bias = 0.f;
    int row = 0, d = 0, bsel = 0, wb = 0, irow = -1;
    bool live = false, straddle = false;
    unsigned b1mask = 0;                                       // channels of the second batch row
    // checkpoint kc of this lane's 4 states, in its register order
    auto load_ckpt = [&](int kc) -> float4 {
        if (!(live && kc >= 0)) return make_float4(0.f, 0.f, 0.f, 0.f);
        const float *b = p.ckpt + ((size_t)row * p.n_ckpt + kc) * N + g * NS;
        if constexpr (PAIR) {
            const float2 lo = ldg_f2_now(b + rot), hi = ldg_f2_now(b + (rot ^ 2));
            return make_float4(lo.x, lo.y, hi.x, hi.y);
        } else {
            return ldg_f4_now(b);
        }
    };

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
            straddle = !ALN && b1mask != 0 && b1mask != lmask;
            wb = b1mask != 0 ? 1 : 0;
#pragma unroll
            for (int j = 0; j < NS; ++j) {
                const float av = live ? p.A[(size_t)d * N + g * NS + (j ^ rot)] : 0.f;
                const float a2 = av * SSM_LOG2E;
                A2p[j] = make_float2(a2, a2);
                if constexpr (ZOH) {
                    const float ia = 1.f / av;
                    iA2[j] = make_float2(ia, ia);
                }
                dA2[j] = make_float2(0.f, 0.f);
                lam[j] = 0.f;
                anext[j] = 1.f;
            }
            const int rr = wrow0 + it_rl;
            irow = rr < q1 ? rr : -1;
            i_bias = (irow >= 0 && p.delta_bias) ? p.delta_bias[rr % p.dim] : 0.f;
            i_D = (irow >= 0 && p.D) ? p.D[rr % p.dim] : 0.f;
            dD_acc = 0.f;
            db_acc = 0.f;
            // starting state of the first window visited (the one holding step L-1)
            const int kc0 = (p.L - 1) / W - 1;
            hpre = load_ckpt(kc0);
        }
        const int wrow0 = q0 + warp * CPW;
        {
            // every lane waits; the warp leaves together if any wait gave up
            bool ok = mbar_wait(full + s, phase, p.err);
            ok = ok && mbar_wait(bcready + (kg & 1), (kg >> 1) & 1, p.err);
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
                    if constexpr (HZ) IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawZ + o), zz);
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        const bool ok = irow >= 0 && (t0 + it_t + v0 + e) < p.L;
                        const float r = dr[e] + i_bias;
                        const float dtv = SP ? softplus_fast(r) : r;
                        float gyv = gg[e];
                        if constexpr (HZ) gyv *= zz[e] * sigmoid(zz[e]);
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

            const float *bcfB = bcf + (kg & 1) * Ly::BCF + bsel * Ly::BROW;
            const float *bcfC = bcfB + 2 * Ly::BROW;
            auto bc4 = [&](const float *base, int j, int tb) -> float4 {
                return *reinterpret_cast<const float4 *>(base + bcf_row<Ly::BRS>(g * NS + (j ^ rot)) + tb);
            };
            // Sum of the transpose buffer over the quarter-warp's 8 channels:
            // lane (g, c) takes state 4g + c/2, steps 4(c&1)..4(c&1)+3 of the
            // window, and adds them to accumulator `which` (0: dB, 1: dC).
            auto reduce_x = [&](int which, int tw) {
                __syncwarp();
                const int nl = c >> 1, n = g * NS + nl, tb = tw + (c & 1) * 4;
                float *dst = dbuf + (which * 2 * N + n) * TT;
                auto add4 = [&](float *row, float4 v) {
                    atomicAdd(row + dbc_col(n, tb + 0), v.x);
                    atomicAdd(row + dbc_col(n, tb + 1), v.y);
                    atomicAdd(row + dbc_col(n, tb + 2), v.z);
                    atomicAdd(row + dbc_col(n, tb + 3), v.w);
                };
                if constexpr (PAIR) {
                    // after the pairing, state nl of the group is held by the
                    // lanes of parity 1 (states 0, 1) or 0 (states 2, 3), at
                    // chunk 2 (half) + (nl & 1) of their rows; row par + 2i
                    // stores it at that chunk ^ i
                    const int par = nl < 2 ? 1 : 0, kk = (c & 1) * 2 + (nl & 1);
                    const float *src = wX + (g * CPW + par) * Ly::XP;
                    float4 s0 = *reinterpret_cast<const float4 *>(src + kk * 4);
#pragma unroll
                    for (int i = 1; i < CPW / 2; ++i)
                        s0 = f4add(s0, *reinterpret_cast<const float4 *>(src + 2 * i * Ly::XP + (kk ^ i) * 4));
                    __syncwarp();
                    add4(dst + wb * N * TT, s0);
                } else {
                    const float *src = wX + g * CPW * XS + c * 4;
                    if (!straddle) {
                        float4 s0 = *reinterpret_cast<const float4 *>(src);
#pragma unroll
                        for (int cc = 1; cc < CPW; ++cc) s0 = f4add(s0, *reinterpret_cast<const float4 *>(src + cc * XS));
                        __syncwarp();
                        add4(dst + wb * N * TT, s0);
                    } else {
                        // channels of two batch rows: one sum per batch row
                        float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
#pragma unroll
                        for (int cc = 0; cc < CPW; ++cc) {
                            const float4 v = *reinterpret_cast<const float4 *>(src + cc * XS);
                            if ((b1mask >> cc) & 1) s1 = f4add(s1, v);
                            else s0 = f4add(s0, v);
                        }
                        __syncwarp();
                        add4(dst, s0);
                        add4(dst + N * TT, s1);
                    }
                }
            };
            // The dB/dC partials of a half-window (4 states x 4 steps, as
            // (state, step pair) float2) into this lane's transpose row; with
            // the pairing, summed with the neighbour channel's first.
            auto put_x = [&](const float2 (&xv)[NS][2], int hh) {
                if constexpr (PAIR) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        float2 o0 = xv[r][0], o1 = xv[r][1];
                        o0.x = __shfl_xor_sync(0xffffffffu, o0.x, 1);
                        o0.y = __shfl_xor_sync(0xffffffffu, o0.y, 1);
                        o1.x = __shfl_xor_sync(0xffffffffu, o1.x, 1);
                        o1.y = __shfl_xor_sync(0xffffffffu, o1.y, 1);
                        const float2 k0 = __fadd2_rn(xv[r + 2][0], o0), k1 = __fadd2_rn(xv[r + 2][1], o1);
                        *reinterpret_cast<float4 *>(myX + ((2 * hh + r) ^ ((c >> 1) & 3)) * 4) =
                            make_float4(k0.x, k0.y, k1.x, k1.y);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < NS; ++j)
                        *reinterpret_cast<float4 *>(myX + (2 * j + hh) * 4) =
                            make_float4(xv[j][0].x, xv[j][0].y, xv[j][1].x, xv[j][1].y);
                }
            };

            // (2) 8-step windows, last to first
#pragma unroll kWinUnroll
            for (int w = Ly::NWIN - 1; w >= 0; --w) {
                const int tw = w * W;                       // window start within the tile
                const int tgw = t0 + tw;                    // and within the sequence
                if (tgw >= p.L) continue;                   // past the end: λ stays 0
                float h[NS] = {hpre.x, hpre.y, hpre.z, hpre.w};
                {
                    const int kc = tgw / W - 2;             // checkpoint of the next window
                    hpre = load_ckpt(kc);
                }
                // Forward recompute over pairs of steps (f32x2 arithmetic):
                // Ā_t, Ā_t h_{t-1}, the y partials and gy h_t (for dC).
                float2 ab2[W / 2][NS], ahp2[W / 2][NS];
                // per half-window, summed over the state groups: y, Σ λ A Ā h
                // (units of A log2 e) and Σ λ B at step 4 hh + g of channel c
                float yv[2], sav[2], sbv[2], sqv[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int tb = tw + 4 * hh;
                    const float4 dt4 = *reinterpret_cast<const float4 *>(wDt + c * WS + tb);
                    const float4 du4 = *reinterpret_cast<const float4 *>(wDu + c * WS + tb);
                    const float4 gy4 = *reinterpret_cast<const float4 *>(wGy + c * WS + tb);
                    const float2 dtp[2] = {make_float2(dt4.x, dt4.y), make_float2(dt4.z, dt4.w)};
                    const float2 dup[2] = {make_float2(du4.x, du4.y), make_float2(du4.z, du4.w)};
                    const float2 gyp[2] = {make_float2(gy4.x, gy4.y), make_float2(gy4.z, gy4.w)};
                    float2 idt[2];                          // 1/Δ (zero-order hold)
                    if constexpr (ZOH) {
#pragma unroll
                        for (int pp = 0; pp < 2; ++pp)
                            idt[pp] = make_float2(rcp_approx(dtp[pp].x), rcp_approx(dtp[pp].y));
                    }
                    float2 y2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    float2 xc[NS][2];                       // gy h (dC partials)
#pragma unroll
                    for (int j = 0; j < NS; ++j) {
                        const float4 B4 = bc4(bcfB, j, tb), C4 = bc4(bcfC, j, tb);
                        const float2 Bp[2] = {make_float2(B4.x, B4.y), make_float2(B4.z, B4.w)};
                        const float2 Cp[2] = {make_float2(C4.x, C4.y), make_float2(C4.z, C4.w)};
#pragma unroll
                        for (int pp = 0; pp < 2; ++pp) {
                            const int P = 2 * hh + pp;
                            const float2 arg = __fmul2_rn(dtp[pp], A2p[j]);
                            const float2 a = make_float2(ex2(arg.x), ex2(arg.y));
                            float2 beta = __fmul2_rn(dup[pp], Bp[pp]);
                            if constexpr (ZOH) beta = __fmul2_rn(beta, zoh_phi2(arg, a, idt[pp], iA2[j]));
                            const float h0 = fmaf(a.x, h[j], beta.x);
                            const float h1 = fmaf(a.y, h0, beta.y);
                            h[j] = h1;
                            const float2 hv = make_float2(h0, h1);
                            if constexpr (!kRecomputeA) ab2[P][j] = a;
                            ahp2[P][j] = __ffma2_rn(beta, make_float2(-1.f, -1.f), hv);   // Ā_t h_{t-1}
                            y2[pp] = __ffma2_rn(Cp[pp], hv, y2[pp]);
                            xc[j][pp] = __fmul2_rn(gyp[pp], hv);
                        }
                    }
                    put_x(xc, hh);
                    yv[hh] = group_reduce4(y2[0], y2[1], g);
                }
                reduce_x(1, tw);
                // Reverse sweep over pairs of steps.  The A-weighted sum is
                // kept in units of A log2(e) and rescaled per element.
#pragma unroll
                for (int hh = 1; hh >= 0; --hh) {
                    const int tb = tw + 4 * hh;
                    const float4 dt4 = *reinterpret_cast<const float4 *>(wDt + c * WS + tb);
                    const float4 du4 = *reinterpret_cast<const float4 *>(wDu + c * WS + tb);
                    const float4 gy4 = *reinterpret_cast<const float4 *>(wGy + c * WS + tb);
                    const float2 dtp[2] = {make_float2(dt4.x, dt4.y), make_float2(dt4.z, dt4.w)};
                    const float2 dup[2] = {make_float2(du4.x, du4.y), make_float2(du4.z, du4.w)};
                    const float2 gyp[2] = {make_float2(gy4.x, gy4.y), make_float2(gy4.z, gy4.w)};
                    float2 sa2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    float2 sb2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    // zero-order hold: Σ λ B Ā (the B term of dΔ); sb2 holds Σ λ B φ
                    float2 sq2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                    float2 idt[2];
                    if constexpr (ZOH) {
#pragma unroll
                        for (int pp = 0; pp < 2; ++pp)
                            idt[pp] = make_float2(rcp_approx(dtp[pp].x), rcp_approx(dtp[pp].y));
                    }
                    float2 xb[NS][2];                       // λ Δu (dB partials)
#pragma unroll
                    for (int j = 0; j < NS; ++j) {
                        const float4 B4 = bc4(bcfB, j, tb), C4 = bc4(bcfC, j, tb);
                        const float2 Bp[2] = {make_float2(B4.x, B4.y), make_float2(B4.z, B4.w)};
                        const float2 Cp[2] = {make_float2(C4.x, C4.y), make_float2(C4.z, C4.w)};
#pragma unroll
                        for (int pp = 1; pp >= 0; --pp) {
                            const int P = 2 * hh + pp;
                            // Ā of this pair: kept from the recompute, or (with
                            // zero-order hold, short of registers) formed again,
                            // bit for bit the same
                            float2 aP;
                            if constexpr (kRecomputeA) {
                                const float2 argA = __fmul2_rn(dtp[pp], A2p[j]);
                                aP = make_float2(ex2(argA.x), ex2(argA.y));
                            } else {
                                aP = ab2[P][j];
                            }
                            const float2 cg = __fmul2_rn(Cp[pp], gyp[pp]);
                            const float l1 = fmaf(anext[j], lam[j], cg.y);      // λ of the later step
                            const float l0 = fmaf(aP.y, l1, cg.x);              // λ of the earlier step
                            const float2 l2 = make_float2(l0, l1);
                            const float2 wv = __fmul2_rn(l2, ahp2[P][j]);
                            sa2[pp] = __ffma2_rn(A2p[j], wv, sa2[pp]);
                            if constexpr (ZOH) {
                                // β = φ Δ B u: dβ/dΔ = Ā B u, dβ/dA = Δ² ψ B u,
                                // dβ/du = φ Δ B, dβ/dB = φ Δ u
                                const float2 arg = __fmul2_rn(dtp[pp], A2p[j]);
                                const float2 phi = zoh_phi2(arg, aP, idt[pp], iA2[j]);
                                const float2 psi = zoh_psi2(arg, aP, phi, idt[pp], iA2[j]);
                                const float2 lB = __fmul2_rn(l2, Bp[pp]);
                                sb2[pp] = __ffma2_rn(lB, phi, sb2[pp]);
                                sq2[pp] = __ffma2_rn(lB, aP, sq2[pp]);
                                const float2 w2 = __ffma2_rn(lB, __fmul2_rn(dup[pp], psi), wv);
                                dA2[j] = __ffma2_rn(dtp[pp], w2, dA2[j]);
                                xb[j][pp] = __fmul2_rn(__fmul2_rn(l2, dup[pp]), phi);
                            } else {
                                dA2[j] = __ffma2_rn(dtp[pp], wv, dA2[j]);
                                sb2[pp] = __ffma2_rn(l2, Bp[pp], sb2[pp]);
                                xb[j][pp] = __fmul2_rn(l2, dup[pp]);
                            }
                            lam[j] = l0;
                            anext[j] = aP.x;
                        }
                    }
                    put_x(xb, hh);
                    sav[hh] = group_reduce4(sa2[0], sa2[1], g);
                    sbv[hh] = group_reduce4(sb2[0], sb2[1], g);
                    if constexpr (ZOH) sqv[hh] = group_reduce4(sq2[0], sq2[1], g);
                }
                reduce_x(0, tw);
                // per-element sums of the window for the epilogue: lane (g, c)
                // holds steps g and g + 4 of channel c (rows of WS floats:
                // the 32 lanes write 32 different banks)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int o = c * WS + tw + g + 4 * e;
                    wY[o] = yv[e];
                    wSa[o] = sav[e] * 0.69314718f;
                    wSb[o] = sbv[e];
                    if constexpr (ZOH) wSq[o] = sqv[e];
                }
                __syncwarp();   // the transpose buffer is rewritten by the next window
            }
            // (3) Epilogue of the tile: lane (it_rl, it_t) finishes steps
            // it_t .. it_t + 7 of its row (the prep's items): du, dΔ and dz
            // from the per-element sums, 16-byte loads and streaming stores.
            if (irow >= 0) {
                constexpr int V = IO<T>::kVec;
                float xu[W], xz[W], xd[W], xg[W];
#pragma unroll
                for (int v0 = 0; v0 < W; v0 += V) {
                    const int o = it_rl * TT + it_t + v0;
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawU + o), xu + v0);
                    IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawG + o), xg + v0);
                    if constexpr (SP) IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawD + o), xd + v0);
                    if constexpr (HZ) IO<T>::unpack(*reinterpret_cast<const uint4 *>(rawZ + o), xz + v0);
                }
                const int ro = it_rl * WS + it_t;
                float rdu[W], rdd[W], rdz[W];
#pragma unroll
                for (int e = 0; e < W; e += 4) {
                    const float4 dt4 = *reinterpret_cast<const float4 *>(wDt + ro + e);
                    const float4 gy4 = *reinterpret_cast<const float4 *>(wGy + ro + e);
                    const float4 y4 = *reinterpret_cast<const float4 *>(wY + ro + e);
                    const float4 sa4 = *reinterpret_cast<const float4 *>(wSa + ro + e);
                    const float4 sb4 = *reinterpret_cast<const float4 *>(wSb + ro + e);
                    float4 sq4 = sb4;
                    if constexpr (ZOH) sq4 = *reinterpret_cast<const float4 *>(wSq + ro + e);
                    const float dt[4] = {dt4.x, dt4.y, dt4.z, dt4.w}, gy[4] = {gy4.x, gy4.y, gy4.z, gy4.w};
                    const float yv4[4] = {y4.x, y4.y, y4.z, y4.w}, sa[4] = {sa4.x, sa4.y, sa4.z, sa4.w};
                    const float sb[4] = {sb4.x, sb4.y, sb4.z, sb4.w}, sq[4] = {sq4.x, sq4.y, sq4.z, sq4.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float x = xu[e + i];
                        if constexpr (HZ) {
                            const float zz = xz[e + i], sg = sigmoid(zz);
                            const float yy = fmaf(i_D, x, yv4[i]);
                            rdz[e + i] = xg[e + i] * yy * sg * fmaf(zz, 1.f - sg, 1.f);
                        }
                        // dΔ: the A term, and u times Σ λ B (Δ·B) or Σ λ B Ā (zero-order hold)
                        const float dDelta = fmaf(x, sq[i], sa[i]);
                        rdd[e + i] = SP ? dDelta * sigmoid(xd[e + i] + i_bias) : dDelta;
                        rdu[e + i] = fmaf(gy[i], i_D, dt[i] * sb[i]);
                        // prep zeroed gy past the end of the sequence
                        dD_acc = fmaf(gy[i], x, dD_acc);
                        if ((t0 + it_t + e + i) < p.L) db_acc += rdd[e + i];
                    }
                }
                const size_t off = (size_t)irow * p.L + t0 + it_t;
                if (p.vec_out && t0 + it_t + W <= p.L) {
#pragma unroll
                    for (int e = 0; e < W; e += 4) {
                        __stcs(reinterpret_cast<float4 *>(p.du + off + e), make_float4(rdu[e], rdu[e + 1], rdu[e + 2], rdu[e + 3]));
                        __stcs(reinterpret_cast<float4 *>(p.ddelta + off + e), make_float4(rdd[e], rdd[e + 1], rdd[e + 2], rdd[e + 3]));
                        if constexpr (HZ)
                            __stcs(reinterpret_cast<float4 *>(p.dz + off + e), make_float4(rdz[e], rdz[e + 1], rdz[e + 2], rdz[e + 3]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < W; ++e) {
                        if (t0 + it_t + e < p.L) {
                            __stcs(p.du + off + e, rdu[e]);
                            __stcs(p.ddelta + off + e, rdd[e]);
                            if constexpr (HZ) __stcs(p.dz + off + e, rdz[e]);
                        }
                    }
                }
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
                for (int j = 0; j < NS; ++j)
                    atomicAdd(p.dA + (size_t)d * N + g * NS + (j ^ rot), dA2[j].x + dA2[j].y);
            }
#pragma unroll
            for (int m = 1; m < TT / W; m <<= 1) {   // the epilogue's 4 lanes of a row
                dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, m);
                db_acc += __shfl_xor_sync(0xffffffffu, db_acc, m);
            }
            if (irow >= 0 && it_t == 0) {
                if (p.dD) atomicAdd(p.dD + irow % p.dim, dD_acc);
                if (p.ddelta_bias) atomicAdd(p.ddelta_bias + irow % p.dim, db_acc);
            }
            k = 0;
            ++q;
        }
    }
}

// ------------------------------------------------------------------ host side


template <typename T, int NWC, int STAGES, bool HZ, bool SP, bool ALN, bool ZOH>
cudaError_t launch_bwd_tma_cfg(const BwdParams &bp, int rows_max, cudaStream_t stream) {
    using Ly = BwdLayout<T, NWC, STAGES>;
    const int P = bp.batch * bp.dim;
    const int grid = std::min(device_sm_count(), ALN ? P / Ly::CPW : P);
    const bool bf16 = sizeof(T) == 2;
    CUtensorMap md, mu, mz, mg, mB, mC;
    const uint32_t bc_box = Ly::PW / sizeof(T);
    if (!make_tma_map_2d(&md, bp.delta, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !make_tma_map_2d(&mu, bp.u, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !make_tma_map_2d(&mz, bp.z ? bp.z : bp.u, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !make_tma_map_2d(&mg, bp.dout, bf16, P, bp.L, Ly::TT, rows_max, false) ||
        !make_tma_map_2d(&mB, bp.B, bf16, (uint64_t)bp.batch * Ly::N, bp.L, bc_box, Ly::N, Ly::SWZ) ||
        !make_tma_map_2d(&mC, bp.C, bf16, (uint64_t)bp.batch * Ly::N, bp.L, bc_box, Ly::N, Ly::SWZ))
        return cudaErrorInvalidValue;
    TmaBwdParams p{};
    p.A = bp.A; p.D = bp.D; p.delta_bias = bp.delta_bias; p.ckpt = bp.ckpt;
    p.du = bp.du; p.ddelta = bp.ddelta; p.dA = bp.dA; p.dB = bp.dB; p.dC = bp.dC;
    p.dD = bp.dD; p.dz = bp.dz; p.ddelta_bias = bp.ddelta_bias;
    p.P = P; p.dim = bp.dim; p.L = bp.L; p.n_ckpt = bp.n_ckpt;
    p.softplus = bp.softplus; p.has_z = bp.z != nullptr; p.rows_max = rows_max;
    p.vec_out = bp.L % 4 == 0 && reinterpret_cast<uintptr_t>(bp.du) % 16 == 0 &&
                reinterpret_cast<uintptr_t>(bp.ddelta) % 16 == 0 &&
                (!bp.z || reinterpret_cast<uintptr_t>(bp.dz) % 16 == 0);
    p.err = device_error_word();
    if (!p.err) return cudaErrorInvalidDevice;
    auto kern = bwd_tma_kernel<T, NWC, STAGES, HZ, SP, ALN, ZOH>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    kern<<<grid, Ly::kThreads, Ly::kAlloc, stream>>>(md, mu, mz, mg, mB, mC, p);
    return cudaGetLastError();
}

// Depth of the ring of input tiles.
#ifndef SSM_BWD_STAGES
#define SSM_BWD_STAGES 2
#endif
constexpr int kBwdStages = SSM_BWD_STAGES;

// The gate, the softplus, the 8-row alignment and the discretisation are
// compile-time switches of the kernel.
template <typename T, int NWC, bool ALN, bool ZOH>
cudaError_t launch_bwd_tma_flags(const BwdParams &bp, int rows_max, cudaStream_t stream) {
    const bool hz = bp.z != nullptr, sp = bp.softplus != 0;
    constexpr int S = kBwdStages;
    if (hz && sp) return launch_bwd_tma_cfg<T, NWC, S, true, true, ALN, ZOH>(bp, rows_max, stream);
    if (hz) return launch_bwd_tma_cfg<T, NWC, S, true, false, ALN, ZOH>(bp, rows_max, stream);
    if (sp) return launch_bwd_tma_cfg<T, NWC, S, false, true, ALN, ZOH>(bp, rows_max, stream);
    return launch_bwd_tma_cfg<T, NWC, S, false, false, ALN, ZOH>(bp, rows_max, stream);
}

template <typename T, int NWC>
cudaError_t launch_bwd_tma_aln(const BwdParams &bp, int rows_max, bool aln, cudaStream_t stream) {
    if (bp.zoh)
        return aln ? launch_bwd_tma_flags<T, NWC, true, true>(bp, rows_max, stream)
                   : launch_bwd_tma_flags<T, NWC, false, true>(bp, rows_max, stream);
    return aln ? launch_bwd_tma_flags<T, NWC, true, false>(bp, rows_max, stream)
               : launch_bwd_tma_flags<T, NWC, false, false>(bp, rows_max, stream);
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
    if (!tma_available()) return false;
    const long long P = (long long)bp.batch * bp.dim;
    const int sms = device_sm_count();
    if (P < sms) return false;
    // rows are split over the CTAs in units of 8 when the channel count
    // allows it (one unit per consumer warp), else one by one
    const bool aln = bp.dim % 8 == 0;
    const long long unit = aln ? 8 : 1;
    const long long cap = (bp.io_bf16 ? kBwdWarpsBf16 : kBwdWarpsF32) * 8 / unit;
    const long long U = P / unit;
    const long long R = (U + sms - 1) / sms;
    const long long npass = (R + cap - 1) / cap;
    const long long rows_max = unit * ((R + npass - 1) / npass);
    if (rows_max > bp.dim) return false;   // a pass spans at most two batch rows
    *err = bp.io_bf16 ? launch_bwd_tma_aln<__nv_bfloat16, kBwdWarpsBf16>(bp, (int)rows_max, aln, stream)
                      : launch_bwd_tma_aln<float, kBwdWarpsF32>(bp, (int)rows_max, aln, stream);
    return true;
}

}  // namespace ssm
