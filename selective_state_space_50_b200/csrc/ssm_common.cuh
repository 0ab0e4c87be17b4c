// Device helpers shared by the selective-scan kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define SSM_LOG2E 1.4426950408889634f

namespace ssm {

// 2^x on the MUFU (SFU) pipe: the PTX instruction ex2.approx.ftz.f32.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float sigmoid(float v) {
    return __fdividef(1.f, 1.f + __expf(-v));
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(r) = ln(1 + e^r) from the hardware base-2 units:
//   x = e^r = 2^(r log2 e);  ln(1 + x) = lg2(1 + x) ln 2  for x >= 1/32,
//   and below that the Taylor series ln(1+x) = x - x^2/2 + x^3/3 - x^4/4
//   (truncation error under x^5/5, i.e. relative 2e-7 at x = 1/32), which
//   avoids the cancellation of 1 + x.  Above r = 15, ln(1 + e^r) - r < 3.1e-7
//   is below half an ulp of r, so r is returned.
__device__ __forceinline__ float softplus_fast(float r) {
    const float x = ex2(r * SSM_LOG2E);
    const float series = x * fmaf(x, fmaf(x, fmaf(x, -0.25f, 0.33333334f), -0.5f), 1.f);
    const float viaLog = lg2(1.f + x) * 0.69314718f;
    const float v = x < 0.03125f ? series : viaLog;
    return r > 15.f ? r : v;
}

// softplus_fast on a pair of values, with the polynomial and scalings in
// f32x2 arithmetic.
__device__ __forceinline__ float2 softplus_fast2(float2 r) {
    const float2 a = __fmul2_rn(r, make_float2(SSM_LOG2E, SSM_LOG2E));
    const float2 x = make_float2(ex2(a.x), ex2(a.y));
    float2 s = __ffma2_rn(x, make_float2(-0.25f, -0.25f), make_float2(0.33333334f, 0.33333334f));
    s = __ffma2_rn(x, s, make_float2(-0.5f, -0.5f));
    s = __ffma2_rn(x, s, make_float2(1.f, 1.f));
    s = __fmul2_rn(x, s);
    const float2 one_x = __fadd2_rn(x, make_float2(1.f, 1.f));
    const float2 lv = __fmul2_rn(make_float2(lg2(one_x.x), lg2(one_x.y)),
                                 make_float2(0.69314718f, 0.69314718f));
    float2 v;
    v.x = r.x > 15.f ? r.x : (x.x < 0.03125f ? s.x : lv.x);
    v.y = r.y > 15.f ? r.y : (x.y < 0.03125f ? s.y : lv.y);
    return v;
}

// log1p(x) for a pair of x in [0, 1] on the FMA pipe: x q(x), with q a
// degree-8 polynomial fitted to log1p(x)/x on [0, 1] for minimax relative
// error (Lawson's iteration on a least-squares fit; 2.3e-7 relative when
// evaluated in fp32 Horner form).  q(0) = 1, so tiny x keep full relative
// accuracy.
__device__ __forceinline__ float2 log1p_poly2(float2 x) {
    constexpr float Q0 = 0.99999994f, Q1 = -0.499994934f, Q2 = 0.333190978f;
    constexpr float Q3 = -0.248429865f, Q4 = 0.191060171f, Q5 = -0.136632651f;
    constexpr float Q6 = 0.0782261342f, Q7 = -0.0295053348f, Q8 = 0.00523271505f;
    float2 q = __ffma2_rn(x, make_float2(Q8, Q8), make_float2(Q7, Q7));
    q = __ffma2_rn(x, q, make_float2(Q6, Q6));
    q = __ffma2_rn(x, q, make_float2(Q5, Q5));
    q = __ffma2_rn(x, q, make_float2(Q4, Q4));
    q = __ffma2_rn(x, q, make_float2(Q3, Q3));
    q = __ffma2_rn(x, q, make_float2(Q2, Q2));
    q = __ffma2_rn(x, q, make_float2(Q1, Q1));
    q = __ffma2_rn(x, q, make_float2(Q0, Q0));
    return __fmul2_rn(x, q);
}

// softplus on a pair with one SFU op per value: softplus(r) = max(r, 0) +
// log1p(e^-|r|), the exponential by ex2 on the SFU and log1p by
// log1p_poly2 on the FMA pipe (softplus_fast2 spends two SFU ops per value).
__device__ __forceinline__ float2 softplus_fast2_1sfu(float2 r) {
    const float2 na = make_float2(-fabsf(r.x) * SSM_LOG2E, -fabsf(r.y) * SSM_LOG2E);
    const float2 l = log1p_poly2(make_float2(ex2(na.x), ex2(na.y)));
    return __fadd2_rn(make_float2(fmaxf(r.x, 0.f), fmaxf(r.y, 0.f)), l);
}

// SiLU gate z * sigmoid(z) with sigmoid(z) = (1 + tanh(z/2)) / 2 on the
// hardware tanh (one SFU op; relative error of tanh.approx ~2^-11, below the
// rounding of a bf16 result).
__device__ __forceinline__ float silu_tanh(float z) {
    const float hz = 0.5f * z;
    return fmaf(hz, tanh_approx(hz), hz);
}

__device__ __forceinline__ float2 silu_tanh2(float2 z) {
    const float2 hz = __fmul2_rn(z, make_float2(0.5f, 0.5f));
    return __ffma2_rn(hz, make_float2(tanh_approx(hz.x), tanh_approx(hz.y)), hz);
}

// 2^x for a pair of x <= 0 on the FMA pipe (no SFU op), for offloading part of
// the discretisation's exponentials from the SFU.  Method: Cody-Waite style
// range reduction x = j + r with j = round(x) (adding 1.5 * 2^23 rounds to an
// integer held in the low mantissa bits), r in [-1/2, 1/2]; 2^r from a degree-5
// polynomial fitted for minimax relative error on [-1/2, 1/2] (Lawson's
// iteration, constant term fixed at 1; max relative error 2.4e-7 = 2^-22.0
// when evaluated in fp32 Horner form); 2^j applied by adding j to the
// exponent field.  Inputs below -126 are clamped (2^-126 ~ 1.2e-38 instead of
// 0).  Valid for x <= 0 only: callers check that A <= 0.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
    x.x = fmaxf(x.x, -126.f);
    x.y = fmaxf(x.y, -126.f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
    const float2 j = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 r = __ffma2_rn(j, make_float2(-1.f, -1.f), x);
    float2 p = __ffma2_rn(make_float2(0.0013276467f, 0.0013276467f), r,
                          make_float2(0.009675542f, 0.009675542f));
    p = __ffma2_rn(p, r, make_float2(0.055507135f, 0.055507135f));
    p = __ffma2_rn(p, r, make_float2(0.2402212f, 0.2402212f));
    p = __ffma2_rn(p, r, make_float2(0.69314694f, 0.69314694f));
    p = __ffma2_rn(p, r, make_float2(1.f, 1.f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// ---- zero-order-hold discretisation ----------------------------------------
// With diagonal A the ZOH input matrix is B̄ = (Ā - 1)/A · B = φ(x) Δ B with
// x = Δ A and φ(x) = (e^x - 1)/x (→ 1 as A → 0, the B̄ = ΔB limit).  Given
// a = e^x, φ is (a - 1)/x except near 0, where that difference cancels and
// the Taylor series 1 + x/2 + x²/6 + ... + x⁵/720 is used (truncation below
// 3e-10 for |x| < 0.1).
__device__ __forceinline__ float zoh_phi(float x, float a) {
    if (fabsf(x) < 0.1f)
        return fmaf(x, fmaf(x, fmaf(x, fmaf(x, fmaf(x, 1.f / 720.f, 1.f / 120.f), 1.f / 24.f), 1.f / 6.f),
                            0.5f), 1.f);
    return __fdividef(a - 1.f, x);
}

// ψ(x) = (x e^x - (e^x - 1)) / x², so that d/dA of the ZOH factor
// (e^{ΔA} - 1)/A is Δ² ψ(ΔA); its series near 0 is
// 1/2 + x/3 + x²/8 + x³/30 + x⁴/144 (truncation below 2e-8 for |x| < 0.1).
__device__ __forceinline__ float zoh_psi(float x, float a) {
    if (fabsf(x) < 0.1f)
        return fmaf(x, fmaf(x, fmaf(x, fmaf(x, 1.f / 144.f, 1.f / 30.f), 1.f / 8.f), 1.f / 3.f), 0.5f);
    return __fdividef(fmaf(x, a, 1.f - a), x * x);
}

// Zero-order-hold factor φ = (Ā - 1)/(Δ A) for a pair of steps of one state,
// with arg = Δ A log2(e), a = 2^arg = Ā, idt = 1/Δ per step and ia = 1/A:
// (a - 1) · idt · ia, or, for |Δ A| < 0.1 where a - 1 cancels, the Taylor
// series 1 + x/2 + x²/6 + x³/24 + x⁴/120 + x⁵/720 in x = arg ln 2 (its
// coefficients below are pre-scaled by powers of ln 2, so it runs in arg).
// Exact zeros (Δ = 0 or A = 0) take the series: φ = 1, the Δ·B limit.
__device__ __forceinline__ float2 zoh_phi2(float2 arg, float2 a, float2 idt, float2 ia) {
    constexpr float L1 = 0.34657359f;      // ln2 / 2
    constexpr float L2 = 0.080075502f;     // ln2^2 / 6
    constexpr float L3 = 0.013876027f;     // ln2^3 / 24
    constexpr float L4 = 0.0019236258f;    // ln2^4 / 120
    constexpr float L5 = 0.00022222597f;   // ln2^5 / 720
    float2 ser = __ffma2_rn(arg, make_float2(L5, L5), make_float2(L4, L4));
    ser = __ffma2_rn(arg, ser, make_float2(L3, L3));
    ser = __ffma2_rn(arg, ser, make_float2(L2, L2));
    ser = __ffma2_rn(arg, ser, make_float2(L1, L1));
    ser = __ffma2_rn(arg, ser, make_float2(1.f, 1.f));
    const float2 em1 = __fadd2_rn(a, make_float2(-1.f, -1.f));
    const float2 q = __fmul2_rn(__fmul2_rn(em1, idt), ia);
    constexpr float kSmall = 0.14426950f;  // |Δ A| < 0.1  <=>  |arg| < 0.1 log2(e)
    return make_float2(fabsf(arg.x) < kSmall ? ser.x : q.x, fabsf(arg.y) < kSmall ? ser.y : q.y);
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ψ = (Ā - φ)/(Δ A) for a pair of steps of one state (the factor of Δ² in the
// derivative of the zero-order-hold input matrix with respect to A, with
// ψ(x) = (x e^x - (e^x - 1))/x²), in the same units as zoh_phi2: arg = Δ A
// log2(e), a = Ā, phi = φ, idt = 1/Δ, ia = 1/A.  For |Δ A| < 0.1, where
// Ā - φ cancels, its Taylor series 1/2 + x/3 + x²/8 + x³/30 + x⁴/144 in
// x = arg ln 2 (coefficients pre-scaled by powers of ln 2; truncation below
// 2e-8).  Exact zeros (Δ = 0 or A = 0) take the series: ψ = 1/2.
__device__ __forceinline__ float2 zoh_psi2(float2 arg, float2 a, float2 phi, float2 idt, float2 ia) {
    constexpr float M1 = 0.23104906f;      // ln2 / 3
    constexpr float M2 = 0.060056627f;     // ln2^2 / 8
    constexpr float M3 = 0.011100822f;     // ln2^3 / 30
    constexpr float M4 = 0.0016030215f;    // ln2^4 / 144
    float2 ser = __ffma2_rn(arg, make_float2(M4, M4), make_float2(M3, M3));
    ser = __ffma2_rn(arg, ser, make_float2(M2, M2));
    ser = __ffma2_rn(arg, ser, make_float2(M1, M1));
    ser = __ffma2_rn(arg, ser, make_float2(0.5f, 0.5f));
    const float2 d = __fadd2_rn(a, make_float2(-phi.x, -phi.y));
    const float2 q = __fmul2_rn(__fmul2_rn(d, idt), ia);
    constexpr float kSmallPsi = 0.14426950f;  // |Δ A| < 0.1
    return make_float2(fabsf(arg.x) < kSmallPsi ? ser.x : q.x, fabsf(arg.y) < kSmallPsi ? ser.y : q.y);
}

// ---- io element types -------------------------------------------------------

template <typename T> struct IO;

template <> struct IO<float> {
    static constexpr int kVec = 4;  // elements per 16-byte vector
    __device__ __forceinline__ static float to_f(float v) { return v; }
    __device__ __forceinline__ static float from_f(float v) { return v; }
    // 16-byte vector <-> 4 floats
    __device__ __forceinline__ static void unpack(const uint4 &q, float *f) {
        f[0] = __uint_as_float(q.x); f[1] = __uint_as_float(q.y);
        f[2] = __uint_as_float(q.z); f[3] = __uint_as_float(q.w);
    }
    __device__ __forceinline__ static uint4 pack(const float *f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

template <> struct IO<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ __forceinline__ static __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
    __device__ __forceinline__ static void unpack(const uint4 &q, float *f) {
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
    __device__ __forceinline__ static uint4 pack(const float *f) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                          pack2(f[6], f[7]));
    }
};

// Loads kVec consecutive elements starting at p[0] into f (as fp32).  Elements
// at index >= n (n < kVec at a ragged end) read as `fill`.  `vec` says the
// 16-byte load is legal (aligned and fully in range).
template <typename T>
__device__ __forceinline__ void load_vec(const T *p, int n, bool vec, float fill, float *f) {
    constexpr int V = IO<T>::kVec;
    if (vec && n >= V) {
        uint4 q = __ldg(reinterpret_cast<const uint4 *>(p));
        IO<T>::unpack(q, f);
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) f[i] = i < n ? IO<T>::to_f(p[i]) : fill;
    }
}

// Streaming variant (evict-first): for data read exactly once.
template <typename T>
__device__ __forceinline__ void load_vec_stream(const T *p, int n, bool vec, float fill, float *f) {
    constexpr int V = IO<T>::kVec;
    if (vec && n >= V) {
        uint4 q = __ldcs(reinterpret_cast<const uint4 *>(p));
        IO<T>::unpack(q, f);
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) f[i] = i < n ? IO<T>::to_f(p[i]) : fill;
    }
}

template <typename T>
__device__ __forceinline__ void store_vec(T *p, int n, bool vec, const float *f) {
    constexpr int V = IO<T>::kVec;
    if (vec && n >= V) {
        __stcs(reinterpret_cast<uint4 *>(p), IO<T>::pack(f));
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i)
            if (i < n) p[i] = IO<T>::from_f(f[i]);
    }
}

}  // namespace ssm
