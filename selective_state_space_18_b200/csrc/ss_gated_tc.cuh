// ss_gated_tc.cuh -- the gated state scan in chunked form on the tensor cores (tcgen05).
//
// What it computes ("Mamba 2 Gated State Scan" exercise page: S_t = gamma_t S_{t-1} +
// k_t v_t^T, y_t = q_t^T S_t, fp32 intermediates), for one batch item and a tile of 64
// value columns, 128 tokens (a chunk) at a time.  With the entering state H and, inside
// the chunk (tokens i, j = 0..127),
//   P_i    = prod_{s <= i} gamma_s                  (decay from the chunk start to i)
//   L[i,j] = prod_{j < s <= i} gamma_s  for j <= i, 0 above the diagonal
//   w_j    = L[127, j]                              (decay from j to the chunk end)
// the recurrence unrolls to
//   y_i  = sum_j L[i,j] (q_i . k_j) v_j  +  P_i q_i^T H
//   H'   = P_127 H  +  sum_j w_j k_j v_j^T
// i.e. four matrix products per chunk:
//   S  = Q K^T          [128 x 128, K = dk]      scores
//   Yi = (L o S) V      [128 x 64,  K = 128]     within the chunk
//   Yh = Q H            [128 x 64,  K = dk]      from the entering state
//   dH = K^T (w o V)    [dk x 64,   K = 128]     the state's increment
// run as tcgen05.mma (bf16 operands staged in shared memory by TMA or by the CUDA
// cores, fp32 accumulators in tensor memory), and the element-wise parts on the CUDA
// cores: the decay mask from a block scan of log2(gamma), y = Yi + P o Yh, and the
// fp32 state H' = P_127 H + dH, which each thread keeps in registers for one row.
// The decays are exact products in log space: L[i,j] = exp2(sum_{j<s<=i} log2 gamma_s),
// and exactly 0 where a gate of 0 lies in (j, i] (tracked as the last zero's index).
//
// Precision: the operands of the products are bf16 -- q, k, v exactly (they are bf16
// inputs); L o S, w o V and H rounded to bf16 -- with fp32 accumulation; the state
// itself stays fp32.  The result is within the bf16 output tolerance of the fp32
// recurrence (tested against the float64 oracle); fp32 inputs use the recurrent kernel.
#pragma once

#include <cuda.h>
#include "ss_device.cuh"
#include "ss_sync.cuh"

namespace ss {

constexpr int kGtChunk = 128;   // tokens per chunk (the MMA's M)
constexpr int kGtDk = 128;      // key size of this kernel
constexpr int kGtNv = 64;       // value columns per CTA
constexpr int kGtThreads = 128; // thread i owns score/output row i and state row i
constexpr uint32_t kGtTmemCols = 512;
// tensor-memory columns of the accumulators
constexpr uint32_t kGtColS = 0, kGtColYi = 128, kGtColYh = 192, kGtColDH = 256;

// shared memory (bytes from a 1024-byte aligned base): every tile is 128 rows of 128
// bytes per 64-element block, written with the 128-byte swizzle
struct GtSmem {
    static constexpr int kQ = 0;              // q chunk: 2 blocks [128 tokens x 64 keys]
    static constexpr int kK = kQ + 32768;     // k chunk: 2 blocks
    static constexpr int kV = kK + 32768;     // v chunk: [128 tokens x 64 values]
    static constexpr int kM = kV + 16384;     // L o S: 2 blocks [128 rows i x 64 cols j]
    static constexpr int kH = kM + 32768;     // H in bf16: [128 keys x 64 values]
    static constexpr int kW = kH + 16384;     // w o V: [128 tokens x 64 values]
    static constexpr int kLam = kW + 16384;   // log2 prefix of the chunk's gates [128] fp32
    static constexpr int kZ = kLam + 512;     // index of the last zero gate <= i [128] int
    static constexpr int kRed = kZ + 512;     // block-scan partials [4 warps x 2]
    static constexpr int kBar = kRed + 64;    // mbarriers: load, mma1, mma2
    static constexpr int kTmem = kBar + 32;   // tensor-memory base address
    static constexpr int kBytes = kTmem + 16 + 1024; // + alignment slack
};

struct GatedTcArgs {
    int64_t batch, seq, dv;
    const float *gamma;       // [batch, seq]
    const float *h0;          // [batch, dk, dv] or null
    __nv_bfloat16 *y;         // [batch, seq, dv]
    __nv_bfloat16 *final_state; // [batch, dk, dv]
    int col_tiles;            // ceil(dv / 64)
};

struct GatedTcMaps {
    CUtensorMap q, k, v; // 3-D: (inner, seq, batch), boxes (64, 128, 1), 128-byte swizzle
};

// ---- tcgen05 and tensor-memory primitives (PTX ISA: tcgen05.*) ---------------------

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] B[smem]; issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 tensor-memory lanes: thread t gets lane
// (warp's first lane + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor (the tcgen05 "smem descriptor"): start address, leading
// and stride byte offsets (all in 16-byte units), version 1, the 128-byte swizzle
// (layout type 2 in bits 61..63).  Bit ranges: start [0,14), LBO [16,30), SBO [32,46),
// version [46,48), base offset [49,52) = 0, LBO mode [52] = 0.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}

// Instruction descriptor of a dense bf16 x bf16 -> fp32 MMA of shape M x N: D format F32
// (bits 4..5 = 1), A and B format BF16 (bits 7..9 and 10..12 = 1), A / B major (bit 15 /
// 16: 0 = K-major, 1 = MN-major), N / 8 in bits 17..22, M / 16 in bits 24..28.
constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
           (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Byte offset of 16-byte chunk c16 (0..7) of row r in a [rows x 128 B] tile with the
// 128-byte swizzle (address bits 4..6 XOR bits 7..9).
__device__ __forceinline__ uint32_t sw128_off(int r, int c16) { return uint32_t(r) * 128u + (uint32_t(c16 ^ (r & 7)) << 4); }

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int32_t c0, int32_t c1, int32_t c2,
                                            uint64_t *bar)
{
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
                 : "memory");
}

// One CTA per (batch item, 64-column value tile); 128 threads; thread 0 issues the
// tile loads and the MMAs.  `status` records a timeout of a bounded wait.
__global__ void __launch_bounds__(kGtThreads, 1)
ss_gated_tc_kernel(const GatedTcArgs a, const __grid_constant__ GatedTcMaps maps, uint32_t *status)
{
    extern __shared__ unsigned char gt_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(gt_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + GtSmem::kBar);
    uint64_t *bar_load = bars, *bar_mma1 = bars + 1, *bar_mma2 = bars + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + GtSmem::kTmem);
    float *s_lam = reinterpret_cast<float *>(sm + GtSmem::kLam);
    int *s_z = reinterpret_cast<int *>(sm + GtSmem::kZ);
    float *s_red = reinterpret_cast<float *>(sm + GtSmem::kRed);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t b = blockIdx.x / a.col_tiles;
    const int n0 = int(blockIdx.x % a.col_tiles) * kGtNv;
    const int64_t nchunks = (a.seq + kGtChunk - 1) / kGtChunk;
    const uint32_t s_base = smem_u32(sm);

    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma1, 1);
        mbar_init(bar_mma2, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kGtTmemCols);
        tmem_relinquish();
    }
    // the entering state: this thread's row d = tid, fp32, in registers
    float H[kGtNv];
#pragma unroll
    for (int n = 0; n < kGtNv; ++n) {
        const int col = n0 + n;
        H[n] = (a.h0 && col < a.dv) ? __ldg(a.h0 + (b * kGtDk + tid) * a.dv + col) : 0.0f;
    }
    // and its bf16 copy, the B operand of Q H
    auto store_h = [&]() {
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {
            const float *h = H + 8 * c16;
            *reinterpret_cast<uint4 *>(sm + GtSmem::kH + sw128_off(tid, c16)) =
                make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]),
                           pack_bf16x2(h[6], h[7]));
        }
    };
    store_h();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); // generic writes -> MMA reads
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    const uint32_t lane_base = uint32_t(32 * warp) << 16; // this warp's tensor-memory lanes

    constexpr uint32_t kLoadBytes = 2 * 16384 + 2 * 16384 + 16384;
    auto issue_loads = [&](int64_t c) {
        mbar_arrive_expect_tx(bar_load, kLoadBytes);
        const int32_t t0 = int32_t(c * kGtChunk), bb = int32_t(b);
        tma_load_3d(sm + GtSmem::kQ, &maps.q, 0, t0, bb, bar_load);
        tma_load_3d(sm + GtSmem::kQ + 16384, &maps.q, 64, t0, bb, bar_load);
        tma_load_3d(sm + GtSmem::kK, &maps.k, 0, t0, bb, bar_load);
        tma_load_3d(sm + GtSmem::kK + 16384, &maps.k, 64, t0, bb, bar_load);
        tma_load_3d(sm + GtSmem::kV, &maps.v, n0, t0, bb, bar_load);
    };
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.v)) : "memory");
        issue_loads(0);
    }

    // (thread 0's record of the asynchronous work in flight, for draining after a timeout)
    int64_t loads_issued = tid == 0 ? 1 : 0, loads_done = 0, mma_issued = 0, mma_done = 0;
    constexpr uint32_t kIdS = idesc_bf16(128, 128, 0, 0);  // Q (K-major) x K (K-major)
    constexpr uint32_t kIdY = idesc_bf16(128, kGtNv, 0, 1); // (L o S) or Q (K-major) x V or H (MN-major)
    constexpr uint32_t kIdH = idesc_bf16(128, kGtNv, 1, 1); // K^T (MN-major) x (w o V) (MN-major)
    bool ok = true;
    for (int64_t c = 0; c < nchunks && ok; ++c) {
        const uint32_t ph = uint32_t(c & 1);
        const int64_t t0 = c * kGtChunk;
        // ---- gates: block scan of log2(gamma) and of the last zero gate --------------
        const int64_t t = t0 + tid;
        const float gm = t < a.seq ? __ldg(a.gamma + b * a.seq + t) : 1.0f; // past the end: no decay
        float lg = gm > 0.0f ? __log2f(gm) : 0.0f;
        int zl = gm == 0.0f ? tid : -1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float up = __shfl_up_sync(0xffffffffu, lg, o);
            const int uz = __shfl_up_sync(0xffffffffu, zl, o);
            if (lane >= o) {
                lg += up;
                zl = max(zl, uz);
            }
        }
        if (lane == 31) {
            s_red[2 * warp] = lg;
            s_red[2 * warp + 1] = __int_as_float(zl);
        }
        // ---- the chunk's tiles (every thread observes the load), then S = Q K^T and
        // Yh = Q H ------------------------------------------------------------------------
        if (!mbar_wait(bar_load, ph, status))
            ok = false;
        else if (tid == 0)
            loads_done = c + 1;
        if (tid == 0 && ok) {
            {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) { // K = 128 keys in slices of 16
                    const uint32_t qa = s_base + GtSmem::kQ + (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint32_t ka = s_base + GtSmem::kK + (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_bf16(tmem + kGtColS, sw128_desc(qa, 16, 1024), sw128_desc(ka, 16, 1024), kIdS, ks > 0);
                    const uint32_t ha = s_base + GtSmem::kH + ks * 2048; // 16 key rows of H
                    umma_bf16(tmem + kGtColYh, sw128_desc(qa, 16, 1024), sw128_desc(ha, 16384, 1024), kIdY, ks > 0);
                }
                umma_commit(bar_mma1);
                mma_issued = c + 1;
            }
        }
        __syncthreads();
        {
            float off = 0.0f;
            int zoff = -1;
            for (int w = 0; w < warp; ++w) {
                off += s_red[2 * w];
                zoff = max(zoff, __float_as_int(s_red[2 * w + 1]));
            }
            lg += off;
            zl = max(zl, zoff);
            s_lam[tid] = lg;
            s_z[tid] = zl;
        }
        if (!__syncthreads_and(ok ? 1 : 0)) { // thread 0 could not get the tiles
            ok = false;
            break;
        }
        const float lam_i = lg;
        const int z_i = zl;
        const float p_i = z_i >= 0 ? 0.0f : ex2(lam_i);                 // P_i
        const float lam_end = s_lam[kGtChunk - 1];
        const int z_end = s_z[kGtChunk - 1];
        const float p_end = z_end >= 0 ? 0.0f : ex2(lam_end);           // P_127
        // ---- w o V: thread j scales row j of v by w_j ---------------------------------
        {
            const float w_j = z_end > tid ? 0.0f : ex2(lam_end - lam_i);
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
                const uint4 vv = *reinterpret_cast<const uint4 *>(sm + GtSmem::kV + sw128_off(tid, c16));
                const uint32_t in[4] = {vv.x, vv.y, vv.z, vv.w};
                uint32_t out[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    out[e] = pack_bf16x2(__uint_as_float(in[e] << 16) * w_j, __uint_as_float(in[e] & 0xffff0000u) * w_j);
                *reinterpret_cast<uint4 *>(sm + GtSmem::kW + sw128_off(tid, c16)) =
                    make_uint4(out[0], out[1], out[2], out[3]);
            }
        }
        // ---- L o S: thread i masks and decays row i of the scores -------------------
        if (!mbar_wait(bar_mma1, ph, status)) {
            ok = false;
        }
        tc_fence_after();
        if (ok) {
#pragma unroll 1
            for (int jb = 0; jb < 4; ++jb) { // 32 columns at a time
                float s[32];
                tmem_ld32(tmem + lane_base + kGtColS + 32 * jb, s);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * jb + 8 * q8 + e;
                        const bool valid = j <= tid && z_i <= j;
                        m[e] = valid ? s[8 * q8 + e] * ex2(lam_i - s_lam[j]) : 0.0f;
                    }
                    const int j0 = 32 * jb + 8 * q8;
                    *reinterpret_cast<uint4 *>(sm + GtSmem::kM + (j0 >> 6) * 16384 + sw128_off(tid, (j0 & 63) >> 3)) =
                        make_uint4(pack_bf16x2(m[0], m[1]), pack_bf16x2(m[2], m[3]), pack_bf16x2(m[4], m[5]),
                                   pack_bf16x2(m[6], m[7]));
                }
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        if (!__syncthreads_and(ok ? 1 : 0)) {
            ok = false;
            break;
        }
        // ---- Yi = (L o S) V and dH = K^T (w o V) ---------------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) { // K = 128 tokens in slices of 16
                const uint32_t ma = s_base + GtSmem::kM + (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint32_t va = s_base + GtSmem::kV + ks * 2048;
                umma_bf16(tmem + kGtColYi, sw128_desc(ma, 16, 1024), sw128_desc(va, 16384, 1024), kIdY, ks > 0);
                const uint32_t kt = s_base + GtSmem::kK + ks * 2048; // keys x 16 tokens (MN-major)
                const uint32_t wa = s_base + GtSmem::kW + ks * 2048;
                umma_bf16(tmem + kGtColDH, sw128_desc(kt, 16384, 1024), sw128_desc(wa, 16384, 1024), kIdH, ks > 0);
            }
            umma_commit(bar_mma2);
        }
        if (!mbar_wait(bar_mma2, ph, status))
            ok = false;
        else if (tid == 0)
            mma_done = c + 1;
        tc_fence_after();
        // the chunk's tiles are free: start the next chunk's loads now
        if (tid == 0 && ok && c + 1 < nchunks) {
            issue_loads(c + 1);
            loads_issued = c + 2;
        }
        if (ok) {
            // ---- y = Yi + P o Yh for this thread's row i ----------------------------------
            const bool row_ok = t0 + tid < a.seq;
#pragma unroll 1
            for (int nb = 0; nb < 2; ++nb) {
                float yi[32], yh[32];
                tmem_ld32(tmem + lane_base + kGtColYi + 32 * nb, yi);
                tmem_ld32(tmem + lane_base + kGtColYh + 32 * nb, yh);
                if (row_ok) {
                    __nv_bfloat16 *dst = a.y + (b * a.seq + t0 + tid) * a.dv + n0 + 32 * nb;
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            o[e] = fmaf(p_i, yh[8 * q8 + e], yi[8 * q8 + e]);
                        const int col = n0 + 32 * nb + 8 * q8;
                        if (col + 8 <= a.dv)
                            *reinterpret_cast<uint4 *>(dst + 8 * q8) =
                                make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                           pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
                    }
                }
            }
            // ---- H' = P_127 H + dH for this thread's key row ------------------------------
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                float dh[32];
                tmem_ld32(tmem + lane_base + kGtColDH + 32 * nb, dh);
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    H[32 * nb + e] = fmaf(p_end, H[32 * nb + e], dh[e]);
            }
            store_h();
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        if (!__syncthreads_and(ok ? 1 : 0)) {
            ok = false;
            break;
        }
    }
    if (ok) {
#pragma unroll
        for (int n = 0; n < kGtNv; n += 2) {
            const int col = n0 + n;
            if (col < a.dv) {
                __nv_bfloat16 *dst = a.final_state + (b * kGtDk + tid) * a.dv + col;
                *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(H[n], H[n + 1]);
            }
        }
    } else if (tid == 0) {
        // a wait gave up: let the loads and MMAs still in flight finish (the drain waits
        // keep the default limit) before the tensor memory is freed
        if (loads_issued > loads_done)
            mbar_wait(bar_load, uint32_t((loads_issued - 1) & 1), nullptr);
        if (mma_issued > mma_done) {
            mbar_wait(bar_mma1, uint32_t((mma_issued - 1) & 1), nullptr);
            mbar_wait(bar_mma2, uint32_t((mma_issued - 1) & 1), nullptr);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, kGtTmemCols);
}

} // namespace ss
