// Selection projections on the 5th-generation tensor cores (tcgen05).
//
// The selection mechanism makes B, C and the step size functions of the
// input: B_t = Linear_N(x_t), C_t = Linear_N(x_t) and
// Δ_t = softplus(Parameter + Linear_1(x_t)) (booiljung.github.io, "3.2 선택적
// 스캔(Selective Scan) 알고리즘", §1.2; honbul.tistory.com, "Mamba" §2,
// s_B, s_C, s_Δ).  The step-size projection is the rank-R factorisation
// Linear_D(Linear_R(x)); R = 1 with an all-ones up-projection is the pages'
// broadcast Linear_1.  The Parameter (delta_bias) and the softplus are applied
// by the scan.  Two products, batched over the batch rows, with the scan's
// [batch, rows, L] layouts on both sides:
//
//   x_proj:  xdbl[b] = W_x [R+2N, D] · x[b] [D, L]       rows 0..R-1 -> dt_low,
//                                                        R..R+N-1 -> B, the rest -> C
//   dt_proj: delta[b] = W_dt [D, R] · dt_low[b] [R, L]
//
// Both are C[m, n] = Σ_k A[m, k] Bm[k, n] with A K-major (row-major weights)
// and Bm N-major (the activations, contiguous along L), bf16 in, fp32
// accumulated in tensor memory, bf16 out.
//
// Kernel: one 128 x 128 output tile per CTA, 4 warps.  Lane 0 of warp 0
// streams 64-deep K slices of A and Bm into a shared-memory ring with TMA
// (128-byte swizzle; 6 stages for x_proj, 1 or 3 for dt_proj whose K is one
// to three slices); lane 0 of warp 1 issues tcgen05.mma (M 128, N 128, K 16) on
// shared-memory descriptors and frees each stage with tcgen05.commit; warp 2
// owns the tensor-memory allocation.  After the last commit all four warps
// read the accumulator (warp w reads lanes 32w..32w+31, i.e. output rows),
// convert to bf16, turn rows into 128-byte row pieces through shared memory
// and store them into the output segment that holds each row.  Tiles past M,
// K or L read zeros (TMA out-of-range fill) and are not stored.  Every wait
// is bounded; a wait that gives up sets the device error word.

#include <cuda_bf16.h>

#include "ssm_internal.h"
#include "ssm_tma.cuh"

namespace ssm {

namespace {

constexpr int kBM = 128, kBK = 64;                    // output tile rows, K slice
constexpr int kATile = kBM * kBK * 2;                 // [128 rows][64 k] bf16
constexpr int kBChunk = kBK * 64 * 2;                 // [64 k][64 columns] bf16
constexpr int kThreads = 128;
// Epilogue staging (reuses the ring): per warp 32 rows x 64 columns of bf16,
// rows padded to 72 elements so that row-wise 16-byte writes spread over the
// banks.
constexpr int kStgRow = 72;
constexpr int kStgWarp = 32 * kStgRow * 2;
static_assert(kATile % 1024 == 0 && kBChunk % 1024 == 0, "swizzle atoms stay aligned");

// An output tile of kBM x BN columns: the ring stage that feeds it and the
// instruction descriptor of kind::f16 (fp32 accumulator, bf16 A and B,
// A K-major, B N-major, N = BN, M = kBM).
template <int BN>
struct ProjTile {
    static constexpr int kBTile = (BN / 64) * kBChunk;
    static constexpr int kStage = kATile + kBTile;
    static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                       ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "whole 64-column chunks; UMMA N <= 256");
    static_assert(4 * kStgWarp <= kStage, "epilogue staging fits in one stage");
};

// Shared memory of a STAGES-deep ring: the ring, then the barriers and the
// tensor-memory address.  A kernel asks for at least a 512/BN share of the
// SM's 228 KB (less the 1 KB the SM keeps per CTA), so that at most 512/BN
// CTAs share an SM: their BN-column accumulators fill its 512 tensor-memory
// columns, and no allocation has to wait (one-stage 128-column tiles: 56 KB,
// four CTAs; 64-column tiles: eight).  Deeper rings fit at most two (3
// stages) or one (6 stages) 128-column CTA per SM.
template <int STAGES, int BN>
struct ProjSmem {
    static constexpr int kBars = STAGES * ProjTile<BN>::kStage;
    static constexpr int kUsed = kBars + (2 * STAGES + 1) * 8 + 16 + 1024;
    static constexpr int kMin = 228 * 1024 / (512 / BN) - 1024;
    static constexpr int kAlloc = kUsed > kMin ? kUsed : kMin;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    // CTAs that can share an SM, by shared memory, never need more tensor
    // memory than its 512 columns (BN each), so no allocation has to wait
    static_assert((228 * 1024 / kAlloc) * BN <= 512, "tensor-memory columns of co-resident CTAs");
};

struct ProjSeg {
    void *ptr;      // [batch][rows][L] bf16
    int row0, rows; // output rows row0 .. row0 + rows - 1 of this product
};

struct ProjParams {
    ProjSeg seg[3];
    int nseg;
    int M, K, L;
    int tma_out;    // one output (seg[0] is the whole product): TMA stores through mO
    int *err;
};

// TMA-store epilogue: each warp stages 32 rows x 64 columns of bf16 (128-byte
// rows, 16-byte chunks XOR-swizzled by row as the tensor map's 128B swizzle
// expects) and one lane stores the box.
constexpr int kOutStg = 32 * 128;

// ------------------------------------------------------------ tcgen05 helpers

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Whole-warp tensor-memory allocation of `cols` columns; the address is
// written to *slot (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(slot)), "r"(cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
                 : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100
// descriptor version 1: start address, leading and stride byte offsets, all
// in 16-byte units.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    const uint32_t mask0 = 0, mask1 = 0, mask2 = 0, mask3 = 0;   // no output lanes disabled
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate),
          "r"(mask0), "r"(mask1), "r"(mask2), "r"(mask3)
        : "memory");
}

// Arrives on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// 16 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t *>(&v);
}

template <int kStages, int kBN>
__global__ void __launch_bounds__(kThreads, 1)
proj_gemm_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB,
                 const __grid_constant__ CUtensorMap mO, const ProjParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    using Tile = ProjTile<kBN>;
    constexpr int kStage = Tile::kStage;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + ProjSmem<kStages, kBN>::kBars);
    uint64_t *empty = full + kStages;
    uint64_t *accum = empty + kStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM, b = blockIdx.z;
    const int nk = (p.K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(accum, 1);
        fence_barrier_init();
    }
    if (warp == 2) tmem_alloc(tmem_slot, kBN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- TMA producer
            prefetch_tensormap(&mA);
            prefetch_tensormap(&mB);
            int issued = 0;
            for (int kt = 0; kt < nk; ++kt) {
                const int s = kt % kStages;
                if (kt >= kStages && !mbar_wait(empty + s, ((kt / kStages) - 1) & 1, p.err)) break;
                uint8_t *st = smem + s * kStage;
                mbar_arrive_expect_tx(full + s, kStage);
                tma_load_2d(st, &mA, kt * kBK, m0, full + s);
#pragma unroll
                for (int c = 0; c < kBN / 64; ++c)
                    tma_load_3d(st + kATile + c * kBChunk, &mB, n0 + 64 * c, kt * kBK, b, full + s);
                ++issued;
            }
            // never leave while a copy may still write shared memory
            for (int kk = (issued > kStages ? issued - kStages : 0); kk < issued; ++kk)
                if (!mbar_wait(full + kk % kStages, (kk / kStages) & 1, p.err)) break;
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------- MMA issuer
            for (int kt = 0; kt < nk; ++kt) {
                const int s = kt % kStages;
                if (!mbar_wait(full + s, (kt / kStages) & 1, p.err)) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * kStage), b0 = a0 + kATile;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    // A: K-major rows of 128 bytes, 8-row groups 1024 bytes apart,
                    //    K step of 16 = 32 bytes along the row.
                    // B: N-major rows of 64 columns (128 bytes) per chunk, chunks
                    //    kBChunk apart (LBO), 8-row K groups 1024 bytes apart
                    //    (SBO), K step of 16 = 16 rows.
                    const uint64_t da = sw128_desc(a0 + kk * 32, 16, 1024);
                    const uint64_t db = sw128_desc(b0 + kk * 16 * 128, kBChunk, 1024);
                    umma_bf16(tmem, da, db, Tile::kIdesc, (kt | kk) != 0);
                }
                umma_commit(empty + s);   // the stage is free once these MMAs are done
            }
            umma_commit(accum);           // also when a wait gave up: the epilogue must not hang
        }
        __syncwarp();
    }

    // -------------------------------------------------------- epilogue (4 warps)
    // Warp w holds output rows m0 + 32w .. m0 + 32w + 31 (tensor-memory lanes).
    // Per 64 columns: each lane converts its row to bf16 into the warp's
    // staging rows, then the warp writes 4 rows x 128 bytes per instruction.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(accum, 0, p.err));
    tc_fence_after();
    if (ok && p.tma_out) {
        static_assert(4 * kOutStg <= kStage && kOutStg % 1024 == 0, "output staging fits one stage");
        uint8_t *stg = smem + warp * kOutStg;            // 1024-byte aligned: the swizzle atom
        const int m = m0 + warp * 32;
#pragma unroll 1
        for (int h = 0; h < kBN / 64; ++h) {
            if (h > 0) {                                 // the previous box has left the staging
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[16];
                tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(h * 64 + c * 16), r);
                uint4 v0, v1;
                v0.x = pack_bf16x2(r[0], r[1]);   v0.y = pack_bf16x2(r[2], r[3]);
                v0.z = pack_bf16x2(r[4], r[5]);   v0.w = pack_bf16x2(r[6], r[7]);
                v1.x = pack_bf16x2(r[8], r[9]);   v1.y = pack_bf16x2(r[10], r[11]);
                v1.z = pack_bf16x2(r[12], r[13]); v1.w = pack_bf16x2(r[14], r[15]);
                uint8_t *row = stg + lane * 128;
                *reinterpret_cast<uint4 *>(row + (((2 * c) ^ (lane & 7)) << 4)) = v0;
                *reinterpret_cast<uint4 *>(row + (((2 * c + 1) ^ (lane & 7)) << 4)) = v1;
            }
            fence_proxy_async();                          // the staging, seen by the TMA unit
            __syncwarp();
            const int n = n0 + h * 64;
            if (lane == 0 && n < p.L && m < p.M) {
                tma_store_3d(&mO, stg, n, m, b);
                bulk_commit_group();
            }
        }
        if (lane == 0) bulk_wait_group<0>();              // stores done before the CTA leaves
        __syncwarp();
    } else if (ok) {
        __nv_bfloat16 *stg = reinterpret_cast<__nv_bfloat16 *>(smem + warp * kStgWarp);
        const int srow = lane / 8, schunk = lane % 8;     // write-out: row within 4, 16-byte chunk
#pragma unroll 1
        for (int h = 0; h < kBN / 64; ++h) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[16];
                tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(h * 64 + c * 16), r);
                uint4 v0, v1;
                v0.x = pack_bf16x2(r[0], r[1]);   v0.y = pack_bf16x2(r[2], r[3]);
                v0.z = pack_bf16x2(r[4], r[5]);   v0.w = pack_bf16x2(r[6], r[7]);
                v1.x = pack_bf16x2(r[8], r[9]);   v1.y = pack_bf16x2(r[10], r[11]);
                v1.z = pack_bf16x2(r[12], r[13]); v1.w = pack_bf16x2(r[14], r[15]);
                *reinterpret_cast<uint4 *>(stg + lane * kStgRow + c * 16) = v0;
                *reinterpret_cast<uint4 *>(stg + lane * kStgRow + c * 16 + 8) = v1;
            }
            __syncwarp();
            const int n = n0 + h * 64 + schunk * 8;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int rl = it * 4 + srow;                 // row within the warp's 32
                const int m = m0 + warp * 32 + rl;
                __nv_bfloat16 *row = nullptr;
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int r0 = p.seg[i].row0, nr = p.seg[i].rows;
                    if (i < p.nseg && m < p.M && m >= r0 && m < r0 + nr)
                        row = static_cast<__nv_bfloat16 *>(p.seg[i].ptr) + ((size_t)b * nr + (m - r0)) * (size_t)p.L;
                }
                if (row && n + 8 <= p.L)
                    *reinterpret_cast<uint4 *>(row + n) =
                        *reinterpret_cast<const uint4 *>(stg + rl * kStgRow + schunk * 8);
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) tmem_dealloc(tmem, kBN);
}

template <int STAGES, int BN>
cudaError_t launch_proj_gemm(const CUtensorMap &mA, const CUtensorMap &mB, const CUtensorMap &mO,
                             const ProjParams &p, int batch, cudaStream_t stream) {
    constexpr int smem = ProjSmem<STAGES, BN>::kAlloc;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(proj_gemm_kernel<STAGES, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    const dim3 grid((unsigned)((p.L + BN - 1) / BN), (unsigned)((p.M + kBM - 1) / kBM), (unsigned)batch);
    proj_gemm_kernel<STAGES, BN><<<grid, kThreads, smem, stream>>>(mA, mB, mO, p);
    return cudaGetLastError();
}

// dt_proj's output through TMA stores (1) or the row-store epilogue (0).
#ifndef SSM_PROJ_TMA_STORE
#define SSM_PROJ_TMA_STORE 1
#endif

// Tile width of the one-slice contraction (dt_proj at rank <= 64).
#ifndef SSM_PROJ_SHORT_BN
#define SSM_PROJ_SHORT_BN 128
#endif

// Ring depth and tile width of the long contraction (x_proj).
#ifndef SSM_PROJ_LONG_STAGES
#define SSM_PROJ_LONG_STAGES 6
#endif
#ifndef SSM_PROJ_LONG_BN
#define SSM_PROJ_LONG_BN 128
#endif

// Ring depth by contraction length.  One K slice (dt_proj at rank <= 64): a
// single stage, with up to four CTAs per SM overlapping each other's loads,
// MMAs and stores.  Two or three slices (larger ranks): the whole contraction
// in flight at once, two CTAs per SM.  Longer (x_proj streams the
// activations): a 6-stage ring.
cudaError_t launch_proj_any(const CUtensorMap &mA, const CUtensorMap &mB, const CUtensorMap &mO,
                            const ProjParams &p, int batch, cudaStream_t stream) {
    const int nk = (p.K + kBK - 1) / kBK;
    if (nk <= 1) return launch_proj_gemm<1, SSM_PROJ_SHORT_BN>(mA, mB, mO, p, batch, stream);
    if (nk <= 3) return launch_proj_gemm<3, 128>(mA, mB, mO, p, batch, stream);
    return launch_proj_gemm<SSM_PROJ_LONG_STAGES, SSM_PROJ_LONG_BN>(mA, mB, mO, p, batch, stream);
}

}  // namespace

cudaError_t launch_projections(const ProjShape &s, const void *x, const void *W_x, const void *W_dt,
                               void *dt_low, void *delta, void *B, void *C, cudaStream_t stream) {
    if (!tma_available()) return cudaErrorNotSupported;
    int *err = device_error_word();
    if (!err) return cudaErrorInvalidDevice;
    const int R = s.dt_rank, N = s.dstate, M1 = s.dt_rank + 2 * s.dstate;
    CUtensorMap mA, mB;
    // x_proj: A = W_x [M1 x D], Bm = x [batch][D][L]
    if (!make_tma_map_2d(&mA, W_x, true, (uint64_t)M1, (uint64_t)s.dim, kBK, kBM, true) ||
        !make_tma_map_bf16_3d(&mB, x, (uint64_t)s.seqlen, (uint64_t)s.dim, (uint64_t)s.batch, 64, kBK))
        return cudaErrorInvalidValue;
    ProjParams p{};
    p.seg[0] = {dt_low, 0, R};
    p.seg[1] = {B, R, N};
    p.seg[2] = {C, R + N, N};
    p.nseg = 3;
    p.M = M1; p.K = s.dim; p.L = s.seqlen; p.err = err;
    p.tma_out = 0;   // three outputs (dt_low, B, C): the row-store epilogue
    cudaError_t e = launch_proj_any(mA, mB, mA, p, s.batch, stream);
    if (e != cudaSuccess) return e;
    // dt_proj: A = W_dt [D x R], Bm = dt_low [batch][R][L]
    if (!make_tma_map_2d(&mA, W_dt, true, (uint64_t)s.dim, (uint64_t)R, kBK, kBM, true) ||
        !make_tma_map_bf16_3d(&mB, dt_low, (uint64_t)s.seqlen, (uint64_t)R, (uint64_t)s.batch, 64, kBK))
        return cudaErrorInvalidValue;
    // delta [batch][D][L] written by TMA stores of 64-column x 32-row boxes
    CUtensorMap mO;
    if (!make_tma_map_bf16_3d(&mO, delta, (uint64_t)s.seqlen, (uint64_t)s.dim, (uint64_t)s.batch, 64, 32))
        return cudaErrorInvalidValue;
    ProjParams q{};
    q.seg[0] = {delta, 0, s.dim};
    q.nseg = 1;
    q.M = s.dim; q.K = R; q.L = s.seqlen; q.err = err;
    q.tma_out = SSM_PROJ_TMA_STORE;
    return launch_proj_any(mA, mB, mO, q, s.batch, stream);
}

}  // namespace ssm
