// ss_gated_scan.cuh -- the Mamba-2 gated state scan in recurrent form.
//
// "Mamba 2 Gated State Scan" (exercise page): per batch item b, with a scalar gate
//   S_t = gamma_t S_{t-1} + k_t v_t^T          (S: Dk x Dv, fp32)
//   y_t = q_t^T S_t                             (the updated state is read)
// each state starting at zero (or at an optional h0), outputs and the final state
// cast to the dtype of q, all intermediate arithmetic in fp32.
//
// Work split.  A CTA owns one batch item and a tile of 64 value columns; thread
// (rg, cg) keeps the 8 x 8 block S[8 rg .. 8 rg + 8, 8 cg .. 8 cg + 8] in registers
// for the whole sequence.  Tokens are staged in chunks of kGChunk through shared
// memory as fp32 (q and k rows, the tile's v columns, gamma).  Per token a thread
// reads 8 k, 8 q and 8 v values (broadcast reads, each reused 8 times) and updates
// its 64 elements with packed fp32x2 operations (gamma S, then + k v, then the
// partial readout q S); the partial readouts of the Dk/8 row groups are summed once
// per chunk from shared memory.  The cost per element and token is three fp32 lane
// operations, so the kernel is bound by the FP32 pipe (and the shared-memory pipe
// close behind); the dense chunked form for tensor cores is a different algorithm.
#pragma once

#include "ss_device.cuh"

namespace ss {

struct GatedArgs {
    int64_t batch, seq, dk, dv;
    const void *q, *k, *v;
    const float *gamma, *h0; // gamma [batch, seq]; h0 [batch, dk, dv] fp32 (nullable)
    void *y, *final_state;   // [batch, seq, dv], [batch, dk, dv] in the dtype of q
    int col_tiles;           // value-column tiles per batch item
};

constexpr int kGChunk = 8; // tokens staged per round
constexpr int kGCols = 64; // value columns per CTA

// RG row groups of 8 rows (Dk <= 8 RG) and 8 column groups of 8 columns: 8 RG threads.
template <int RG> struct GatedShape {
    static constexpr int kRows = 8 * RG;                 // padded Dk
    static constexpr int kCG = kGCols / 8;
    static constexpr int kCols = kGCols;
    static constexpr int kThreads = RG * kCG;
    // shared memory (floats): q, k [chunk][kRowStride]; v [chunk][kCols]; gamma
    // [chunk]; partial readouts [chunk][RG][kPStride].  Rows are padded by 4 floats
    // every 32 (and partial rows by 4) so the row groups a warp reads or writes at once
    // fall into distinct banks.
    static constexpr int kRowStride = kRows + 4 * (kRows / 32);
    static constexpr int kPStride = kCols + 4;
    static constexpr int kQOff = 0, kKOff = kGChunk * kRowStride, kVOff = 2 * kGChunk * kRowStride;
    static constexpr int kGOff = kVOff + kGChunk * kCols;
    static constexpr int kPOff = kGOff + kGChunk;
    static constexpr int kFloats = kPOff + kGChunk * RG * kPStride;
    static __device__ __forceinline__ int row_pos(int i) { return i + 4 * (i / 32); }
    static constexpr size_t kSmem = size_t(kFloats) * 4;
};

template <typename T> __device__ __forceinline__ float gload(const T *p, int64_t i);
template <> __device__ __forceinline__ float gload<float>(const float *p, int64_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float gload<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i)
{
    return __bfloat162float(__ldg(p + i));
}

// Eight consecutive elements of a q, k or v row as fp32, from one 16-byte load (bf16)
// or two (fp32).
template <typename T> __device__ __forceinline__ void load8(const T *src, float (&o)[8]);
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *src, float (&o)[8])
{
    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(src));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        o[2 * h] = __uint_as_float(u[h] << 16);
        o[2 * h + 1] = __uint_as_float(u[h] & 0xffff0000u);
    }
}
template <> __device__ __forceinline__ void load8<float>(const float *src, float (&o)[8])
{
    const float4 a = __ldg(reinterpret_cast<const float4 *>(src)), b = __ldg(reinterpret_cast<const float4 *>(src) + 1);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

// VEC: dk equals the padded row count and dv is a multiple of 8, with 16-byte aligned
// rows, so a chunk is staged with 8-element vector loads (a few per thread) instead
// of one scalar load per element.
template <int RG, typename T, bool VEC>
__global__ void __launch_bounds__(GatedShape<RG>::kThreads, 512 / GatedShape<RG>::kThreads)
ss_gated_scan_kernel(const GatedArgs p)
{
    using G = GatedShape<RG>;
    extern __shared__ __align__(16) float gsm[];
    const int64_t b = blockIdx.x / p.col_tiles;
    const int64_t j0 = int64_t(blockIdx.x % p.col_tiles) * G::kCols; // first value column
    const int tid = threadIdx.x, rg = tid % RG, cg = tid / RG;
    const T *q = static_cast<const T *>(p.q) + b * p.seq * p.dk;
    const T *k = static_cast<const T *>(p.k) + b * p.seq * p.dk;
    const T *v = static_cast<const T *>(p.v) + b * p.seq * p.dv;
    const float *gamma = p.gamma + b * p.seq;

    // the thread's 8 x 8 block, as 8 rows of 4 column pairs
    float2 S[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t i = 8 * rg + r, j = j0 + 8 * cg + 2 * c;
            float2 s = make_float2(0.f, 0.f);
            if (p.h0 && i < p.dk) {
                const float *h = p.h0 + (b * p.dk + i) * p.dv;
                s.x = j < p.dv ? __ldg(h + j) : 0.f;
                s.y = j + 1 < p.dv ? __ldg(h + j + 1) : 0.f;
            }
            S[r][c] = s;
        }

    for (int64_t t0 = 0; t0 < p.seq; t0 += kGChunk) {
        const int nt = p.seq - t0 < kGChunk ? int(p.seq - t0) : kGChunk;
        __syncthreads(); // the previous chunk's staging and partials are consumed
        if constexpr (VEC) {
            for (int e8 = tid; e8 < kGChunk * G::kRows / 8; e8 += G::kThreads) {
                const int t = (8 * e8) / G::kRows, i = (8 * e8) % G::kRows;
                const int pos = t * G::kRowStride + G::row_pos(i);
                float a[8], c[8];
                if (t < nt) {
                    load8<T>(q + (t0 + t) * p.dk + i, a);
                    load8<T>(k + (t0 + t) * p.dk + i, c);
                } else {
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        a[u] = c[u] = 0.f;
                }
                float4 *dq = reinterpret_cast<float4 *>(gsm + G::kQOff + pos);
                float4 *dk4 = reinterpret_cast<float4 *>(gsm + G::kKOff + pos);
                dq[0] = make_float4(a[0], a[1], a[2], a[3]);
                dq[1] = make_float4(a[4], a[5], a[6], a[7]);
                dk4[0] = make_float4(c[0], c[1], c[2], c[3]);
                dk4[1] = make_float4(c[4], c[5], c[6], c[7]);
            }
            for (int e8 = tid; e8 < kGChunk * G::kCols / 8; e8 += G::kThreads) {
                const int t = (8 * e8) / G::kCols, cc = (8 * e8) % G::kCols;
                float a[8];
                if (t < nt && j0 + cc < p.dv) {
                    load8<T>(v + (t0 + t) * p.dv + j0 + cc, a);
                } else {
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        a[u] = 0.f;
                }
                float4 *dv4 = reinterpret_cast<float4 *>(gsm + G::kVOff + 8 * e8);
                dv4[0] = make_float4(a[0], a[1], a[2], a[3]);
                dv4[1] = make_float4(a[4], a[5], a[6], a[7]);
            }
        }
        for (int e = tid; e < (VEC ? 0 : kGChunk * G::kRows); e += G::kThreads) {
            const int t = e / G::kRows, i = e % G::kRows;
            const bool in = t < nt && i < p.dk;
            const int64_t off = (t0 + t) * p.dk + i;
            const int pos = t * G::kRowStride + G::row_pos(i);
            gsm[G::kQOff + pos] = in ? gload<T>(q, off) : 0.f;
            gsm[G::kKOff + pos] = in ? gload<T>(k, off) : 0.f;
        }
        for (int e = tid; e < (VEC ? 0 : kGChunk * G::kCols); e += G::kThreads) {
            const int t = e / G::kCols, c = e % G::kCols;
            const bool in = t < nt && j0 + c < p.dv;
            gsm[G::kVOff + e] = in ? gload<T>(v, (t0 + t) * p.dv + j0 + c) : 0.f;
        }
        if (tid < kGChunk)
            gsm[G::kGOff + tid] = tid < nt ? __ldg(gamma + t0 + tid) : 1.f;
        __syncthreads();
        for (int t = 0; t < nt; ++t) {
            const float g = gsm[G::kGOff + t];
            const float2 gg = make_float2(g, g);
            const float4 *kr = reinterpret_cast<const float4 *>(gsm + G::kKOff + t * G::kRowStride + G::row_pos(8 * rg));
            const float4 *qr = reinterpret_cast<const float4 *>(gsm + G::kQOff + t * G::kRowStride + G::row_pos(8 * rg));
            const float4 *vr = reinterpret_cast<const float4 *>(gsm + G::kVOff + t * G::kCols + 8 * cg);
            const float4 k0 = kr[0], k1 = kr[1], q0 = qr[0], q1 = qr[1], v0 = vr[0], v1 = vr[1];
            const float kk[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
            const float qq[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            const float2 vv[4] = {make_float2(v0.x, v0.y), make_float2(v0.z, v0.w), make_float2(v1.x, v1.y),
                                  make_float2(v1.z, v1.w)};
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float2 kr2 = make_float2(kk[r], kk[r]), qr2 = make_float2(qq[r], qq[r]);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    S[r][c] = __ffma2_rn(kr2, vv[c], __fmul2_rn(gg, S[r][c]));
                    acc[c] = __ffma2_rn(qr2, S[r][c], acc[c]);
                }
            }
            float4 *pp = reinterpret_cast<float4 *>(gsm + G::kPOff + (t * RG + rg) * G::kPStride + 8 * cg);
            pp[0] = make_float4(acc[0].x, acc[0].y, acc[1].x, acc[1].y);
            pp[1] = make_float4(acc[2].x, acc[2].y, acc[3].x, acc[3].y);
        }
        __syncthreads();
        // outputs of the chunk, four columns per thread: the sum over row groups
        for (int e = tid; e < nt * (G::kCols / 4); e += G::kThreads) {
            const int t = e / (G::kCols / 4), c4 = 4 * (e % (G::kCols / 4));
            float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int g2 = 0; g2 < RG; ++g2) {
                const float4 v4 = *reinterpret_cast<const float4 *>(gsm + G::kPOff + (t * RG + g2) * G::kPStride + c4);
                s4.x += v4.x;
                s4.y += v4.y;
                s4.z += v4.z;
                s4.w += v4.w;
            }
            T *yr = static_cast<T *>(p.y) + (b * p.seq + t0 + t) * p.dv + j0 + c4;
            const float o[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (j0 + c4 + u < p.dv)
                    Elem<T>::store(yr + u, o[u]);
        }
    }
    // the final state, in the dtype of q
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int64_t i = 8 * rg + r;
        if (i >= p.dk)
            continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t j = j0 + 8 * cg + 2 * c;
            T *fs = static_cast<T *>(p.final_state) + (b * p.dk + i) * p.dv;
            if (j < p.dv)
                Elem<T>::store(fs + j, S[r][c].x);
            if (j + 1 < p.dv)
                Elem<T>::store(fs + j + 1, S[r][c].y);
        }
    }
}

} // namespace ss
