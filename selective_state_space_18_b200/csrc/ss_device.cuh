// ss_device.cuh -- small device helpers shared by the scan and decode kernels.
//
// Element access for the two storage types (fp32, bf16), the MUFU base-2
// exponential, and the two pointwise functions of the S6 step: softplus for the
// step size (a series form, and the polynomial form that the prompt scan and the
// segment decay share, scalar and packed) and silu for the output gate (nnterp
// "selective_scan" component: dt = softplus(dt_proj(x) + dt_bias); the output is y
// gated by silu(z)).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ss {

constexpr float kLog2e = 1.4426950408889634f;

// ---- debug build with index checks (compile with -DSS_BOUNDS_CHECK) ----------------
//
// SS_IN_BOUNDS(cond, site) is `cond` in the checked build and `true` otherwise.  In
// the checked build a false condition records the site's number in g_ss_bounds_site
// (the first one wins) and the caller skips the access it guards: no trap, so the
// kernel finishes and the host reads the site with ss_debug_bounds_status.
#ifdef SS_BOUNDS_CHECK
__device__ uint32_t g_ss_bounds_site;
__device__ __forceinline__ bool ss_bounds_ok(bool ok, uint32_t site)
{
    if (!ok)
        atomicCAS(&g_ss_bounds_site, 0u, site);
    return ok;
}
#define SS_IN_BOUNDS(cond, site) ::ss::ss_bounds_ok((cond), (site))
#else
#define SS_IN_BOUNDS(cond, site) true
#endif

// 2^x on the MUFU unit (flush-to-zero: results below 2^-126 become +0, and
// 2^-inf = +0, which the reset fold relies on).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log(1 + e) for e in [0, 1], from log(1 + e) = 2 atanh(s) with s = e / (2 + e)
// in [0, 1/3]:  2 atanh(s) = 2 s (1 + s^2/3 + s^4/5 + ... + s^12/13).  The first
// omitted term is below 1.5e-8 relative, and the form keeps full relative
// accuracy as e -> 0 (where log(1 + e) -> e).
__device__ __forceinline__ float log1p_unit(float e)
{
    const float s = __fdividef(e, 2.0f + e);
    const float w = s * s;
    float p = 1.0f / 13.0f;
    p = fmaf(p, w, 1.0f / 11.0f);
    p = fmaf(p, w, 1.0f / 9.0f);
    p = fmaf(p, w, 1.0f / 7.0f);
    p = fmaf(p, w, 1.0f / 5.0f);
    p = fmaf(p, w, 1.0f / 3.0f);
    p = fmaf(p, w, 1.0f);
    return (2.0f * s) * p;
}

// softplus(r) = log(1 + e^r) = max(r, 0) + log(1 + e^{-|r|}).
__device__ __forceinline__ float softplus(float r)
{
    return fmaxf(r, 0.0f) + log1p_unit(ex2(-fabsf(r) * kLog2e));
}

// softplus(r) = max(r, 0) + log(1 + e), e = exp(-|r|) in (0, 1].  log(1 + e) = e Q(e)
// with Q a degree-8 polynomial fitted to log1p(e)/e on [0, 1] for relative error
// (1.5e-7 in fp32 Horner form): no division, one MUFU op.
__device__ __forceinline__ float softplus_poly(float r)
{
    const float e = ex2(-fabsf(r) * kLog2e);
    float q = 5.232690697e-03f;
    q = fmaf(q, e, -2.950522892e-02f);
    q = fmaf(q, e, 7.822594434e-02f);
    q = fmaf(q, e, -1.366324604e-01f);
    q = fmaf(q, e, 1.910600743e-01f);
    q = fmaf(q, e, -2.484298259e-01f);
    q = fmaf(q, e, 3.331909690e-01f);
    q = fmaf(q, e, -4.999949315e-01f);
    q = fmaf(q, e, 9.999999699e-01f);
    return fmaxf(r, 0.0f) + e * q;
}

// The same for two tokens at once with packed fp32x2 arithmetic; the polynomial
// and the final e Q(e) + max(r, 0) run as fp32x2 fused multiply-adds.
__device__ __forceinline__ float2 softplus_poly2(float2 r)
{
    const float2 t = __fmul2_rn(make_float2(-fabsf(r.x), -fabsf(r.y)), make_float2(kLog2e, kLog2e));
    const float2 e = make_float2(ex2(t.x), ex2(t.y));
    float2 q = make_float2(5.232690697e-03f, 5.232690697e-03f);
    q = __ffma2_rn(q, e, make_float2(-2.950522892e-02f, -2.950522892e-02f));
    q = __ffma2_rn(q, e, make_float2(7.822594434e-02f, 7.822594434e-02f));
    q = __ffma2_rn(q, e, make_float2(-1.366324604e-01f, -1.366324604e-01f));
    q = __ffma2_rn(q, e, make_float2(1.910600743e-01f, 1.910600743e-01f));
    q = __ffma2_rn(q, e, make_float2(-2.484298259e-01f, -2.484298259e-01f));
    q = __ffma2_rn(q, e, make_float2(3.331909690e-01f, 3.331909690e-01f));
    q = __ffma2_rn(q, e, make_float2(-4.999949315e-01f, -4.999949315e-01f));
    q = __ffma2_rn(q, e, make_float2(9.999999699e-01f, 9.999999699e-01f));
    return __ffma2_rn(e, q, make_float2(fmaxf(r.x, 0.0f), fmaxf(r.y, 0.0f)));
}

// silu(v) = v / (1 + e^{-v}).
__device__ __forceinline__ float silu(float v)
{
    return __fdividef(v, 1.0f + ex2(-v * kLog2e));
}

// ---- storage types ---------------------------------------------------------------

template <typename T> struct Elem;

template <> struct Elem<float> {
    static constexpr int kBytes = 4;
    static __device__ __forceinline__ float load(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ float load_smem(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
};

template <> struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p)
    {
        return __bfloat162float(__ldg(p));
    }
    static __device__ __forceinline__ float load_smem(const __nv_bfloat16 *p)
    {
        return __uint_as_float(uint32_t(*reinterpret_cast<const unsigned short *>(p)) << 16);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v)
    {
        *p = __float2bfloat16_rn(v);
    }
};

// Eight consecutive elements held in registers in their storage form: one 16-byte
// vector of bf16 or two of fp32.
template <typename T> struct Raw8;

template <> struct Raw8<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void load_smem(const __nv_bfloat16 *p)
    {
        v = *reinterpret_cast<const uint4 *>(p);
    }
    __device__ __forceinline__ float get(int j) const
    {
        const uint32_t w = (&v.x)[j >> 1];
        return __uint_as_float((j & 1) ? (w & 0xffff0000u) : (w << 16));
    }
    // Vector load of elements [t, t+8) of a row; the row length is a multiple of 8,
    // so either the whole vector is in range or none of it is.
    __device__ __forceinline__ void load_vec_stream(const __nv_bfloat16 *row, int64_t t, int64_t len)
    {
        if (t < len)
            v = __ldcs(reinterpret_cast<const uint4 *>(row + t));
        else
            zero();
    }
    __device__ __forceinline__ void load_vec(const __nv_bfloat16 *row, int64_t t, int64_t len)
    {
        if (t < len)
            v = __ldg(reinterpret_cast<const uint4 *>(row + t));
        else
            zero();
    }
    __device__ __forceinline__ void load_scalar(const __nv_bfloat16 *row, int64_t t, int64_t len)
    {
        const unsigned short *r = reinterpret_cast<const unsigned short *>(row);
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t lo = (t + 2 * k < len) ? (uint32_t)__ldg(r + t + 2 * k) : 0u;
            const uint32_t hi = (t + 2 * k + 1 < len) ? (uint32_t)__ldg(r + t + 2 * k + 1) : 0u;
            w[k] = lo | (hi << 16);
        }
        v = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <> struct Raw8<float> {
    uint4 v[2];
    __device__ __forceinline__ void zero() { v[0] = v[1] = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void load_smem(const float *p)
    {
        v[0] = reinterpret_cast<const uint4 *>(p)[0];
        v[1] = reinterpret_cast<const uint4 *>(p)[1];
    }
    __device__ __forceinline__ float get(int j) const
    {
        return __uint_as_float((&v[j >> 2].x)[j & 3]);
    }
    // The row length is a multiple of 4: each half is wholly in range or not.
    __device__ __forceinline__ void load_vec_stream(const float *row, int64_t t, int64_t len)
    {
#pragma unroll
        for (int h = 0; h < 2; ++h)
            v[h] = (t + 4 * h < len) ? __ldcs(reinterpret_cast<const uint4 *>(row + t + 4 * h))
                                     : make_uint4(0, 0, 0, 0);
    }
    __device__ __forceinline__ void load_vec(const float *row, int64_t t, int64_t len)
    {
#pragma unroll
        for (int h = 0; h < 2; ++h)
            v[h] = (t + 4 * h < len) ? __ldg(reinterpret_cast<const uint4 *>(row + t + 4 * h))
                                     : make_uint4(0, 0, 0, 0);
    }
    __device__ __forceinline__ void load_scalar(const float *row, int64_t t, int64_t len)
    {
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            w[k] = (t + k < len) ? __float_as_uint(__ldg(row + t + k)) : 0u;
        v[0] = make_uint4(w[0], w[1], w[2], w[3]);
        v[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
};

// Store eight outputs to elements [t, t+8) of a row (round-to-nearest-even for bf16).
template <typename T, bool VEC>
__device__ __forceinline__ void store8(T *row, int64_t t, int64_t len, const float (&o)[8]);

// Two floats rounded to bf16 (nearest-even) and packed, `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <>
__device__ __forceinline__ void store8<__nv_bfloat16, true>(__nv_bfloat16 *row, int64_t t,
                                                            int64_t len, const float (&o)[8])
{
    if (t < len)
        __stcs(reinterpret_cast<uint4 *>(row + t),
               make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                          pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7])));
}

template <>
__device__ __forceinline__ void store8<float, true>(float *row, int64_t t, int64_t len,
                                                    const float (&o)[8])
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
        if (t + 4 * h < len)
            __stcs(reinterpret_cast<float4 *>(row + t + 4 * h),
                   make_float4(o[4 * h], o[4 * h + 1], o[4 * h + 2], o[4 * h + 3]));
}

template <>
__device__ __forceinline__ void store8<__nv_bfloat16, false>(__nv_bfloat16 *row, int64_t t,
                                                             int64_t len, const float (&o)[8])
{
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (t + k < len)
            row[t + k] = __float2bfloat16_rn(o[k]);
}

template <>
__device__ __forceinline__ void store8<float, false>(float *row, int64_t t, int64_t len,
                                                     const float (&o)[8])
{
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (t + k < len)
            row[t + k] = o[k];
}

} // namespace ss
