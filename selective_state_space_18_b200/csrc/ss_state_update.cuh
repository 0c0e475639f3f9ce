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
#include "ss_sync.cuh"

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

// ---------------------------------------------------------------------------------------
// Streaming form for a 16-byte aligned state (the common case)
// ---------------------------------------------------------------------------------------
//
// The state is the only large operand, and the kernel above keeps at most its
// registers' worth of it in flight (about 64 KB per SM at its occupancy), below what
// HBM needs to run at full rate.  Here persistent CTAs stream the state through a
// ring of shared-memory stages filled by bulk asynchronous copies (one per tile, no
// multicast), so kDecStages tiles of every CTA are always on their way regardless of
// the registers the arithmetic needs.  A tile is 1024 row quarters (16 KB of state)
// of one batch row; thread t owns quarters t, t + 256, t + 512, t + 768 of it.  The
// updated state goes straight back to global memory with streaming stores.
constexpr int kDecThreads = 256;
constexpr int kDecItems = 4;                              // quarters per thread per tile
constexpr int kDecQuarters = kDecThreads * kDecItems;     // 1024 quarters = 16 KB
constexpr int kDecStages = 5;
constexpr int kDecTileBytes = kDecQuarters * 16;
constexpr size_t kDecSmem = size_t(kDecStages) * kDecTileBytes + 8 * kDecStages;

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

template <int N, typename T>
__global__ void __launch_bounds__(kDecThreads)
ss_state_update_stream_kernel(const UpdateArgs p, int64_t ntiles, uint32_t *status)
{
    constexpr int Q = N / 4;                  // quarters per (b, c) row
    constexpr int kChanPerTile = kDecQuarters / Q;
    extern __shared__ __align__(128) unsigned char dsm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(dsm + size_t(kDecStages) * kDecTileBytes);
    const int tid = threadIdx.x;
    const int64_t tiles_per_row = (p.channels + kChanPerTile - 1) / kChanPerTile;

    // bytes of tile `tile` and where its state starts
    auto tile_span = [&](int64_t tile, int64_t &b, int64_t &c0) -> uint32_t {
        b = tile / tiles_per_row;
        c0 = (tile - b * tiles_per_row) * kChanPerTile;
        const int64_t nch = p.channels - c0 < kChanPerTile ? p.channels - c0 : kChanPerTile;
        return uint32_t(nch * N * 4);
    };
    auto issue = [&](int64_t tile, int stage) {
        int64_t b, c0;
        const uint32_t bytes = tile_span(tile, b, c0);
        mbar_arrive_expect_tx(full + stage, bytes);
        bulk_load(dsm + size_t(stage) * kDecTileBytes, p.state + (b * p.channels + c0) * N, bytes, full + stage);
    };

    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s)
            mbar_init(full + s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    int64_t issued = 0; // tiles of this CTA handed to the copy engine (thread 0's count)
    if (tid == 0) {
        for (int s = 0; s < kDecStages - 1; ++s) {
            const int64_t tile = blockIdx.x + int64_t(s) * gridDim.x;
            if (tile < ntiles) {
                issue(tile, s);
                ++issued;
            }
        }
    }
    bool ok = true;
    int64_t it = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        // every thread is done with the stage of tile it - 1: refill it with tile
        // it + kDecStages - 1
        __syncthreads();
        if (tid == 0) {
            const int64_t nt = tile + int64_t(kDecStages - 1) * gridDim.x;
            if (nt < ntiles) {
                issue(nt, int((it + kDecStages - 1) % kDecStages));
                ++issued;
            }
        }
        int64_t b, c0;
        const uint32_t bytes = tile_span(tile, b, c0);
        const int nq = int(bytes / 16); // valid quarters in this tile
        // the small operands first: their latency overlaps the wait for the state
        const int lane_q = tid & (Q - 1);
        const float4 bv = Vec4<T>::load(static_cast<const T *>(p.B) + b * N + 4 * lane_q, false);
        const float4 cv = Vec4<T>::load(static_cast<const T *>(p.C) + b * N + 4 * lane_q, false);
        float xs[kDecItems], ds[kDecItems], zs[kDecItems], bias[kDecItems], dd[kDecItems];
        float4 av[kDecItems];
#pragma unroll
        for (int k = 0; k < kDecItems; ++k) {
            const int q = tid + k * kDecThreads;
            const int qq = q < nq ? q : nq - 1;
            const int64_t c = c0 + qq / Q;
            const int64_t row = b * p.channels + c;
            xs[k] = Elem<T>::load(static_cast<const T *>(p.x) + row);
            ds[k] = Elem<T>::load(static_cast<const T *>(p.dt) + row);
            zs[k] = p.z ? Elem<T>::load(static_cast<const T *>(p.z) + row) : 0.0f;
            bias[k] = p.dt_bias ? __ldg(p.dt_bias + c) : 0.0f;
            dd[k] = p.D ? __ldg(p.D + c) : 0.0f;
            av[k] = __ldg(reinterpret_cast<const float4 *>(p.A + c * N) + lane_q);
        }
        const int stage = int(it % kDecStages);
        if (!mbar_wait(full + stage, uint32_t(it / kDecStages) & 1u, status)) {
            ok = false;
            break;
        }
        const float4 *sv = reinterpret_cast<const float4 *>(dsm + size_t(stage) * kDecTileBytes);
#pragma unroll
        for (int k = 0; k < kDecItems; ++k) {
            const int q = tid + k * kDecThreads;
            const bool valid = q < nq;
            const int qq = valid ? q : nq - 1;
            float4 st = sv[qq];
            const float r = ds[k] + bias[k];
            const float d = p.softplus ? softplus(r) : r;
            const float dx = d * xs[k];
            const float dl = d * kLog2e;
            st.x = fmaf(ex2(dl * av[k].x), st.x, dx * bv.x);
            st.y = fmaf(ex2(dl * av[k].y), st.y, dx * bv.y);
            st.z = fmaf(ex2(dl * av[k].z), st.z, dx * bv.z);
            st.w = fmaf(ex2(dl * av[k].w), st.w, dx * bv.w);
            float yp = cv.x * st.x;
            yp = fmaf(cv.y, st.y, yp);
            yp = fmaf(cv.z, st.z, yp);
            yp = fmaf(cv.w, st.w, yp);
#pragma unroll
            for (int off = Q / 2; off >= 1; off >>= 1)
                yp += __shfl_xor_sync(0xffffffffu, yp, off);
            if (valid) {
                const int64_t c = c0 + q / Q;
                const int64_t row = b * p.channels + c;
                __stcs(reinterpret_cast<float4 *>(p.state + row * N) + lane_q, st);
                if (lane_q == 0) {
                    float v = fmaf(dd[k], xs[k], yp);
                    if (p.z)
                        v *= silu(zs[k]);
                    Elem<T>::store(static_cast<T *>(p.y) + row, v);
                }
            }
        }
    }
    if (!ok && tid == 0) {
        // gave up (SS_ERR_TIMEOUT recorded): let the copies still in flight land
        for (int64_t k = it; k < issued; ++k)
            mbar_wait(full + int(k % kDecStages), uint32_t(k / kDecStages) & 1u, nullptr);
    }
}

} // namespace ss
