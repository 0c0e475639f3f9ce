// ss_state_update.cuh -- single-token decode update of the selective scan.
//
// For one token (nnterp "selective_scan" component: mamba_selective_state_update on
// a decode step, the state [batch, channels, state_dim] updated in place):
//   dt       = softplus(dt_raw[b,c] + dt_bias[c])
//   s[b,c,n] = exp(dt A[c,n]) s[b,c,n] + dt B[b,n] x[b,c]
//   y[b,c]   = (sum_n C[b,n] s[b,c,n] + D[c] x[b,c]) silu(z[b,c])
//
// The fp32 state is the only large operand (8 bytes moved per state element: one
// read, one write), so this kernel is bound by HBM bandwidth.  N/4 adjacent lanes
// share one (b, c) row, each owning four states as one 16-byte vector.  A CTA
// covers kUpdateItems * 256 row quarters of one batch row (so B and C are one
// broadcast load per CTA and no index needs a division); each thread issues the
// loads of all its quarters before computing, to keep enough bytes in flight.  The
// per-lane partial outputs are summed with warp shuffles.
#pragma once

#include "ss_device.cuh"

namespace ss {

struct UpdateArgs {
    int64_t batch, channels;
    float *state;
    const void *x, *dt, *B, *C, *z;
    const float *A, *D, *dt_bias;
    void *y;
    int softplus;
    int blocks_per_row; // CTAs per batch row
};

constexpr int kUpdateThreads = 256;
constexpr int kUpdateItems = 8; // row quarters per thread: 128 B of state in flight each

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float *p, bool vec)
    {
        if (vec)
            return __ldg(reinterpret_cast<const float4 *>(p));
        return make_float4(__ldg(p), __ldg(p + 1), __ldg(p + 2), __ldg(p + 3));
    }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16 *p, bool vec)
    {
        if (vec) {
            const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
            return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                               __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
        }
        return make_float4(__bfloat162float(__ldg(p)), __bfloat162float(__ldg(p + 1)),
                           __bfloat162float(__ldg(p + 2)), __bfloat162float(__ldg(p + 3)));
    }
};

template <int N, typename T, bool VEC>
__global__ void __launch_bounds__(kUpdateThreads)
ss_state_update_kernel(const UpdateArgs p)
{
    constexpr int Q = N / 4;                       // lanes per (b, c) row
    constexpr int kQShift = Q == 4 ? 2 : (Q == 2 ? 1 : 0);
    const int64_t b = blockIdx.x / p.blocks_per_row;
    const int64_t cblk = blockIdx.x - b * p.blocks_per_row;
    const int64_t j0 = cblk * (kUpdateThreads * kUpdateItems) + threadIdx.x;
    const T *Bb = static_cast<const T *>(p.B) + b * N;
    const T *Cb = static_cast<const T *>(p.C) + b * N;
    const int lane_q = threadIdx.x & (Q - 1);      // quarter within the row
    const float4 bv = Vec4<T>::load(Bb + 4 * lane_q, VEC);
    const float4 cv = Vec4<T>::load(Cb + 4 * lane_q, VEC);

    // channel of item `it` (clamped: lanes past the end compute on a valid row and
    // store nothing)
    auto chan = [&](int it) -> int64_t {
        const int64_t c = (j0 + it * kUpdateThreads) >> kQShift;
        return c < p.channels ? c : p.channels - 1;
    };
    // all state loads first (the HBM stream), then the small per-row operands
    float4 s[kUpdateItems];
#pragma unroll
    for (int it = 0; it < kUpdateItems; ++it) {
        const float *sp = p.state + (b * p.channels + chan(it)) * N + 4 * lane_q;
        s[it] = VEC ? __ldcs(reinterpret_cast<const float4 *>(sp)) : make_float4(sp[0], sp[1], sp[2], sp[3]);
    }
    float xs[kUpdateItems], ds[kUpdateItems];
#pragma unroll
    for (int it = 0; it < kUpdateItems; ++it) {
        const int64_t row = b * p.channels + chan(it);
        xs[it] = Elem<T>::load(static_cast<const T *>(p.x) + row);
        ds[it] = Elem<T>::load(static_cast<const T *>(p.dt) + row);
    }
#pragma unroll
    for (int it = 0; it < kUpdateItems; ++it) {
        const int64_t c = chan(it);
        const int64_t row = b * p.channels + c;
        const bool valid = ((j0 + it * kUpdateThreads) >> kQShift) < p.channels;
        const float4 a = Vec4<float>::load(p.A + c * N + 4 * lane_q, VEC);
        const float bias = p.dt_bias ? __ldg(p.dt_bias + c) : 0.0f;
        const float r = ds[it] + bias;
        const float d = p.softplus ? softplus(r) : r;
        const float dx = d * xs[it];
        const float dl = d * kLog2e;
        float4 st = s[it];
        st.x = fmaf(ex2(dl * a.x), st.x, dx * bv.x);
        st.y = fmaf(ex2(dl * a.y), st.y, dx * bv.y);
        st.z = fmaf(ex2(dl * a.z), st.z, dx * bv.z);
        st.w = fmaf(ex2(dl * a.w), st.w, dx * bv.w);
        float yp = cv.x * st.x;
        yp = fmaf(cv.y, st.y, yp);
        yp = fmaf(cv.z, st.z, yp);
        yp = fmaf(cv.w, st.w, yp);
#pragma unroll
        for (int off = Q / 2; off >= 1; off >>= 1)
            yp += __shfl_xor_sync(0xffffffffu, yp, off);
        if (valid) {
            float *sp = p.state + row * N + 4 * lane_q;
            if (VEC)
                __stcs(reinterpret_cast<float4 *>(sp), st);
            else {
                sp[0] = st.x;
                sp[1] = st.y;
                sp[2] = st.z;
                sp[3] = st.w;
            }
            if (lane_q == 0) {
                float v = fmaf(p.D ? __ldg(p.D + c) : 0.0f, xs[it], yp);
                if (p.z)
                    v *= silu(Elem<T>::load(static_cast<const T *>(p.z) + row));
                Elem<T>::store(static_cast<T *>(p.y) + row, v);
            }
        }
    }
}

} // namespace ss
