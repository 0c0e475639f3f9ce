// ss_probe.cu -- throughput probe of the special-function (MUFU) unit.
//
// The prompt scan is bound by its exponentials, so its roofline's denominator is the
// rate at which an SM retires ex2 (and tanh, which the bf16 output gate uses).  One
// CTA per SM runs many independent chains of the instruction; the SM's cycle counter
// brackets the loop, so the result is in results per clock per SM, independent of the
// clock the GPU happens to run at.
#include "ss_scan.h"

#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kProbeThreads = 512;
constexpr int kChains = 8;

template <int OP> __device__ __forceinline__ float probe_op(float x)
{
    float y;
    if (OP == 0)
        asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    else
        asm volatile("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Each thread runs kChains independent chains of `iters` operations; the values stay in
// (0, 1] (ex2 of a negative number, tanh of a small one), so nothing overflows.
template <int OP> __global__ void __launch_bounds__(kProbeThreads, 1)
ss_mufu_probe_kernel(int64_t iters, long long *cycles, float *sink)
{
    float v[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c)
        v[c] = -0.25f - 0.01f * float(c + (threadIdx.x & 7));
    __syncthreads();
    const long long t0 = clock64();
    for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
        for (int c = 0; c < kChains; ++c)
            v[c] = -probe_op<OP>(v[c]);
    }
    __syncthreads();
    const long long t1 = clock64();
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < kChains; ++c)
        s += v[c];
    if (s == 12345.0f) // never true; keeps the chains live
        sink[threadIdx.x] = s;
    if (threadIdx.x == 0)
        cycles[blockIdx.x] = t1 - t0;
}

} // namespace

extern "C" {

int ss_debug_mufu_probe(int op, int64_t iters, int64_t blocks, long long *cycles, float *sink,
                        int64_t *ops_per_block, ss_stream_t stream)
{
    if (!cycles || !sink || !ops_per_block)
        return SS_ERR_NULL;
    if (op < 0 || op > 1)
        return SS_ERR_UNSUPPORTED;
    if (iters <= 0 || blocks <= 0 || blocks > 0x7fffffffLL || iters > (int64_t(1) << 40))
        return SS_ERR_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (op == 0)
        ss_mufu_probe_kernel<0><<<unsigned(blocks), kProbeThreads, 0, s>>>(iters, cycles, sink);
    else
        ss_mufu_probe_kernel<1><<<unsigned(blocks), kProbeThreads, 0, s>>>(iters, cycles, sink);
    *ops_per_block = int64_t(kProbeThreads) * kChains * iters;
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

} // extern "C"
