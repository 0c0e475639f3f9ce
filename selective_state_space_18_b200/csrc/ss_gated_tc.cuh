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
//   Yh = Q H            [128 x 64,  K = dk]      from the entering state
//   Yi = (L o S) V      [128 x 64,  K = 128]     within the chunk
//   dH = K^T (w o V)    [dk x 64,   K = 128]     the state's increment
// run as tcgen05.mma (bf16 x bf16 -> fp32 accumulators in tensor memory), and the
// element-wise parts on the CUDA cores: the decay mask from a block scan of the gates,
// y = Yi + P o Yh, and the fp32 state H' = P_127 H + dH, kept in registers.
//
// Decays.  The gates are scanned in log space with the zero gates and the signs kept
// apart, so every real gate is taken as the recurrence takes it: lam_i = sum of
// log2|gamma_s| over s <= i (zero gates add 0), z_i = index of the last zero gate <= i,
// par_i = parity of the negative gates <= i.  Then L[i,j] = 0 if z_i > j, else
// (-1)^(par_i ^ par_j) exp2(lam_i - lam_j).  (A gate below the smallest normal float
// counts as zero: the terms it scales are below 1e-38 of the others.)  For a 32-column
// block below the diagonal block (every j before every i of the row block) the decay
// factors through the block's last column j1: L[i,j] = L[i,j1] L[j1,j], one
// exponential per row and one per column instead of one per element -- used when every
// gate of the chunk has |gamma| <= 1, so that neither factor can overflow (otherwise
// every element takes the direct form).
//
// Precision.  q, k, v are bf16 inputs and enter the products exactly.  The fp32
// intermediates that are operands (L o S, w o V and the state H) are each split into a
// bf16 high part and a bf16 residual (x = hi + lo to about 2^-17 relative), and each of
// their products runs as two MMAs into the same fp32 accumulator: the result follows
// fp32 intermediate arithmetic far below the bf16 rounding of the outputs.
//
// One CTA: 16 compute warps and one issuer warp.  Compute warp w works on tensor-memory
// lanes 32 (w % 4) .. +31 (rows of the scores, outputs and state) and on column group
// w / 4 (a quarter of the value columns and one 32-column block of the scores).  The issuer warp's lane 0 issues every tile load (TMA) and every MMA, each as
// soon as its inputs are ready; the compute warps tell it through two mbarriers (L o S
// and w o V written; the epilogue done) and wait only for products to complete, so the
// scores of a chunk are computed while the previous chunk's epilogue runs and Q H while
// the mask is built.  (Issuing an MMA blocks the issuing thread for about as long as
// the tensor core takes to run it.)  The k and v tiles are double-buffered (the next
// chunk's are in flight during this one); the q tile is reloaded as soon as the
// products that read it are done.  L o S goes to tensor memory (tcgen05.st) and enters
// Yi as the A operand from there.
#pragma once

#include <cuda.h>
#include "ss_device.cuh"
#include "ss_sync.cuh"

namespace ss {

constexpr int kGtChunk = 128;   // tokens per chunk (the MMA's M)
constexpr int kGtDk = 128;      // key size of this kernel
constexpr int kGtNv = 64;       // value columns per CTA
constexpr int kGtComputeWarps = 16; // warp w: tensor-memory lane quarter w % 4, column group w / 4
constexpr int kGtComputeThreads = 32 * kGtComputeWarps;
constexpr int kGtColGroups = kGtComputeWarps / 4;     // column groups per lane quarter
constexpr int kGtVCols = 64 / kGtColGroups;           // value columns per compute thread
constexpr int kGtSBlocks = 4 / kGtColGroups;          // 32-column score blocks per compute thread
static_assert(kGtColGroups == 2 || kGtColGroups == 4, "compute warps: 8 or 16");
constexpr int kGtThreads = kGtComputeThreads + 32; // + the issuer warp
constexpr uint32_t kGtTmemCols = 512;
// tensor-memory columns: fp32 accumulators S, Yi, Yh, and dH as two 64-column halves
// (the products with the high and the low part of w o V, summed in the epilogue); L o S
// as packed bf16 pairs (high and low parts, 64 columns = 128 elements each)
constexpr uint32_t kGtColS = 0, kGtColMhi = 128, kGtColMlo = 192, kGtColYi = 256, kGtColYh = 320,
                   kGtColDH = 384;

// shared memory (bytes from a 1024-byte aligned base): every tile is rows of 128 bytes
// per 64-element block, written with the 128-byte swizzle
struct GtSmem {
    static constexpr int kQ = 0;                // q chunk: 2 blocks [128 tokens x 64 keys]
    static constexpr int kK = kQ + 32768;       // k chunk: 2 stages of 2 blocks
    static constexpr int kV = kK + 2 * 32768;   // v chunk: 2 stages of [128 tokens x 64 values]
    static constexpr int kHhi = kV + 2 * 16384; // H, high and low bf16 parts: [128 keys x 64 values]
    static constexpr int kHlo = kHhi + 16384;
    static constexpr int kWhi = kHlo + 16384;   // w o V, high and low parts: [128 tokens x 64 values]
    static constexpr int kWlo = kWhi + 16384;
    static constexpr int kLam = kWlo + 16384;   // lam_j [128] fp32
    static constexpr int kG = kLam + 512;       // L[j1(j), j] [128] fp32 (column factors)
    static constexpr int kZ = kG + 512;         // z_j [128] int
    static constexpr int kSg = kZ + 512;        // (-1)^par_j [128] fp32
    static constexpr int kRed = kSg + 512;      // per lane quarter: log sum, last zero, parity, |gamma| > 1
    static constexpr int kBar = kRed + 64;      // mbarriers: q, kv[2], s, yh, mma2, mw, epi
    static constexpr int kTmem = kBar + 64;     // tensor-memory base address
    static constexpr int kBytes = kTmem + 16 + 1024; // + alignment slack
};
static_assert(GtSmem::kBytes <= 227 * 1024, "shared memory of the gated tensor-core kernel");

struct GatedTcArgs {
    int64_t batch, seq, dv;
    const float *gamma;       // [batch, seq]
    const float *h0;          // [batch, dk, dv] or null
    __nv_bfloat16 *y;         // [batch, seq, dv]
    __nv_bfloat16 *final_state; // [batch, dk, dv]
    int col_tiles;            // dv / 64
    int hold_first_mw;        // failure-path test aid: withhold the first "L o S written" arrival
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
// D[tmem] (+)= A[tmem] B[smem]: A is M x 16 with row m in lane m and its 16 bf16
// elements packed in pairs (lower index in the low half) into 8 columns from a_tmem.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 tensor-memory lanes (thread t gets lane
// (warp's first lane + t)), as raw 32-bit words, without waiting: several loads go out
// together and one tmem_ld_wait(), followed by tmem_ld_fence() on each destination,
// completes them.
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 16 consecutive 32-bit columns, as tmem_ld32_issue.
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_fence(uint32_t (&r)[16])
{
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]));
}
// NC (16 or 32) consecutive columns of this warp's lanes (issue only).
template <int NC> __device__ __forceinline__ void tmem_ld_n_issue(uint32_t taddr, uint32_t (&r)[NC])
{
    if constexpr (NC == 16)
        tmem_ld16_issue(taddr, r);
    else
        tmem_ld32_issue(taddr, r);
}
// Ties every later use of `r` to a point after the wait (the registers a tcgen05.ld
// writes are only valid once the wait has returned).
__device__ __forceinline__ void tmem_ld_fence(uint32_t (&r)[32])
{
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// 16 consecutive 32-bit columns of this warp's 32 lanes from registers (thread t writes
// lane (warp's first lane + t)); complete once tmem_st_wait returns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
                 "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi), for a pair of values, as packed
// pairs (element 0 in the low half).  x - hi is exact in fp32.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    hi = pack_bf16x2(x0, x1);
    lo = pack_bf16x2(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xffff0000u));
}

// The 8 bf16 values of a 16-byte chunk, scaled by w, split into high and low parts.
__device__ __forceinline__ void scale_split8(uint4 v, float w, uint4 &hi, uint4 &lo)
{
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        split_bf16x2(__uint_as_float(in[e] << 16) * w, __uint_as_float(in[e] & 0xffff0000u) * w, h[e], l[e]);
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Named barrier 1 over the compute warps (the issuer warp takes no part): plain, and
// with an AND over every thread's predicate, so the compute warps leave the chunk loop
// together (a warp that left alone would strand the others at the barrier).
__device__ __forceinline__ void gt_compute_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kGtComputeThreads) : "memory");
}
__device__ __forceinline__ bool gt_compute_sync_and(bool v)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"(uint32_t(v)), "n"(kGtComputeThreads)
                 : "memory");
    return r != 0;
}

// One CTA per (batch item, 64-column value tile).  `status` records a timeout of a
// bounded wait.
__global__ void __launch_bounds__(kGtThreads, 1)
ss_gated_tc_kernel(const GatedTcArgs a, const __grid_constant__ GatedTcMaps maps, uint32_t *status)
{
    extern __shared__ unsigned char gt_raw[];
    // the 1024-byte aligned base, as an offset into the shared array (a pointer that went
    // through an integer would lose its address space: every access through it would
    // compile to a generic load or store)
    unsigned char *sm = gt_raw + ((1024u - (smem_u32(gt_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + GtSmem::kBar);
    uint64_t *bar_q = bars, *bar_kv = bars + 1 /* [2] */, *bar_s = bars + 3, *bar_yh = bars + 4, *bar_2 = bars + 5;
    uint64_t *bar_mw = bars + 6, *bar_epi = bars + 7;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + GtSmem::kTmem);
    float *s_lam = reinterpret_cast<float *>(sm + GtSmem::kLam);
    float *s_g = reinterpret_cast<float *>(sm + GtSmem::kG);
    int *s_z = reinterpret_cast<int *>(sm + GtSmem::kZ);
    float *s_sg = reinterpret_cast<float *>(sm + GtSmem::kSg);
    uint32_t *s_red = reinterpret_cast<uint32_t *>(sm + GtSmem::kRed);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool issuer = warp == kGtComputeWarps;
    const int q4 = warp & 3, cg = (warp >> 2) % kGtColGroups; // lane quarter, column group
    const int r = 32 * q4 + lane; // this thread's row: a token of the chunk, a key of the state
    const int64_t b = blockIdx.x / a.col_tiles;
    const int n0 = int(blockIdx.x % a.col_tiles) * kGtNv;
    const int64_t nchunks = (a.seq + kGtChunk - 1) / kGtChunk;
    const uint32_t s_base = smem_u32(sm);

    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_kv, 1);
        mbar_init(bar_kv + 1, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_yh, 1);
        mbar_init(bar_2, 1);
        mbar_init(bar_mw, kGtComputeWarps);  // one arrival per compute warp
        mbar_init(bar_epi, kGtComputeWarps);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kGtTmemCols);
        tmem_relinquish();
    }
    // the entering state: key row r, value columns kGtVCols cg .. + kGtVCols - 1 of the
    // tile, fp32
    float H[kGtVCols];
#pragma unroll
    for (int e = 0; e < kGtVCols; ++e)
        H[e] = 0.0f;
    if (!issuer && a.h0) {
        const float *src = a.h0 + (b * kGtDk + r) * a.dv + n0 + kGtVCols * cg;
#pragma unroll
        for (int e = 0; e < kGtVCols; e += 4) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(src + e));
            H[e] = v.x;
            H[e + 1] = v.y;
            H[e + 2] = v.z;
            H[e + 3] = v.w;
        }
    }
    // and its high and low bf16 parts, the B operands of Q H
    auto store_h = [&]() {
#pragma unroll
        for (int cc = 0; cc < kGtVCols / 8; ++cc) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                split_bf16x2(H[8 * cc + 2 * e], H[8 * cc + 2 * e + 1], hi[e], lo[e]);
            const uint32_t off = sw128_off(r, (kGtVCols / 8) * cg + cc);
            *reinterpret_cast<uint4 *>(sm + GtSmem::kHhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(sm + GtSmem::kHlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
    };
    if (!issuer)
        store_h();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    const uint32_t lane_base = uint32_t(32 * q4) << 16; // this warp's tensor-memory lanes
    if (!issuer) {
        // L o S is 0 above the diagonal in every chunk: those blocks of its tensor-memory
        // copy are written once, here, and never again
#pragma unroll
        for (int bb = 0; bb < kGtSBlocks; ++bb) {
            const int jb = kGtSBlocks * cg + bb;
            if (jb > q4) {
                const uint32_t zero[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                tmem_st16(tmem + lane_base + kGtColMhi + 16 * jb, zero);
                tmem_st16(tmem + lane_base + kGtColMlo + 16 * jb, zero);
            }
        }
        tmem_st_wait();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); // H writes -> MMA reads
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    constexpr uint32_t kIdS = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
    constexpr uint32_t kIdY = idesc_bf16(128, kGtNv, 0, 1); // Q or L o S (K-major) x H or V (MN-major)
    // K^T (MN-major) x [w o V high | w o V low] (MN-major, N = 128: the low part's tile lies
    // one 64-column block after the high part's, the stride between N blocks)
    constexpr uint32_t kIdH = idesc_bf16(128, 2 * kGtNv, 1, 1);
    static_assert(GtSmem::kWlo == GtSmem::kWhi + 16384, "w o V high and low parts one block apart");
    bool ok = true;
    if (issuer) {
        // ======================= the issuer warp (lane 0 works) =======================
        // Per chunk c, in order: S(c) once the chunk's tiles have landed and the mask of
        // chunk c-1 is done with the score columns; Yh(c) once the epilogue of c-1 has
        // stored H(c) and read its accumulators; the k / v tiles of c+1 into the stage
        // chunk c-1 used, once that chunk's products are done; the q tile of c+1 once
        // Yh(c) (the last reader of q) is done; dH(c) and Yi(c) once the compute warps
        // have written L o S and w o V.  The compute warps never wait for an issue, only
        // for products to complete.
        if (lane == 0) {
            const int32_t b32 = int32_t(b);
            auto issue_q = [&](int64_t c) {
                mbar_arrive_expect_tx(bar_q, 32768);
                const int32_t t0 = int32_t(c * kGtChunk);
                tma_load_3d(sm + GtSmem::kQ, &maps.q, 0, t0, b32, bar_q);
                tma_load_3d(sm + GtSmem::kQ + 16384, &maps.q, 64, t0, b32, bar_q);
            };
            auto issue_kv = [&](int64_t c) {
                const int st = int(c & 1);
                mbar_arrive_expect_tx(bar_kv + st, 32768 + 16384);
                const int32_t t0 = int32_t(c * kGtChunk);
                tma_load_3d(sm + GtSmem::kK + st * 32768, &maps.k, 0, t0, b32, bar_kv + st);
                tma_load_3d(sm + GtSmem::kK + st * 32768 + 16384, &maps.k, 64, t0, b32, bar_kv + st);
                tma_load_3d(sm + GtSmem::kV + st * 16384, &maps.v, n0, t0, b32, bar_kv + st);
            };
            // phases issued (or committed) per barrier, for draining after a timeout
            int64_t nq = 0, nkv0 = 0, nkv1 = 0, ns = 0, nyh = 0, n2 = 0;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.q)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.v)) : "memory");
            issue_q(0);
            nq = 1;
            issue_kv(0);
            nkv0 = 1;
            if (nchunks > 1) {
                issue_kv(1);
                nkv1 = 1;
            }
            for (int64_t c = 0; c < nchunks; ++c) {
                const int st = int(c & 1);
                const uint32_t ph = uint32_t(c & 1), pp = uint32_t((c - 1) & 1);
                if (!mbar_wait(bar_q, ph, status) || !mbar_wait(bar_kv + st, uint32_t((c >> 1) & 1), status) ||
                    (c > 0 && !mbar_wait(bar_mw, pp, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t qb = s_base + GtSmem::kQ, kb = s_base + GtSmem::kK + st * 32768;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) { // K = 128 keys in slices of 16
                    const uint32_t o = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_bf16(tmem + kGtColS, sw128_desc(qb + o, 16, 1024), sw128_desc(kb + o, 16, 1024), kIdS,
                              ks > 0);
                }
                umma_commit(bar_s);
                ns = c + 1;
                if (c > 0 && !mbar_wait(bar_epi, pp, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t qd = sw128_desc(qb + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    const uint32_t ho = ks * 2048; // 16 key rows of H
                    umma_bf16(tmem + kGtColYh, qd, sw128_desc(s_base + GtSmem::kHhi + ho, 16384, 1024), kIdY,
                              ks > 0);
                    umma_bf16(tmem + kGtColYh, qd, sw128_desc(s_base + GtSmem::kHlo + ho, 16384, 1024), kIdY, 1);
                }
                umma_commit(bar_yh);
                nyh = c + 1;
                if (c > 0 && c + 1 < nchunks) {
                    if (!mbar_wait(bar_2, pp, status)) { // chunk c-1's products: its stage is free
                        ok = false;
                        break;
                    }
                    issue_kv(c + 1);
                    ((c + 1) & 1 ? nkv1 : nkv0) = ((c + 1) >> 1) + 1;
                }
                if (!mbar_wait(bar_yh, ph, status)) {
                    ok = false;
                    break;
                }
                if (c + 1 < nchunks) {
                    issue_q(c + 1);
                    nq = c + 2;
                }
                if (!mbar_wait(bar_mw, ph, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t vb = s_base + GtSmem::kV + st * 16384;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) { // K = 128 tokens in slices of 16
                    const uint64_t kd = sw128_desc(kb + ks * 2048, 16384, 1024); // keys x 16 tokens (MN-major)
                    umma_bf16(tmem + kGtColDH, kd, sw128_desc(s_base + GtSmem::kWhi + ks * 2048, 16384, 1024),
                              kIdH, ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t vd = sw128_desc(vb + ks * 2048, 16384, 1024);
                    umma_bf16_ts(tmem + kGtColYi, tmem + kGtColMhi + 8 * ks, vd, kIdY, ks > 0);
                    umma_bf16_ts(tmem + kGtColYi, tmem + kGtColMlo + 8 * ks, vd, kIdY, 1);
                }
                umma_commit(bar_2);
                n2 = c + 1;
            }
            // Let every load and product still in flight finish before the tensor memory
            // is freed: the latest phase of each barrier (already complete on the normal
            // path; the drain waits keep the default limit)
            if (nq)
                mbar_wait(bar_q, uint32_t((nq - 1) & 1), nullptr);
            if (nkv0)
                mbar_wait(bar_kv, uint32_t((nkv0 - 1) & 1), nullptr);
            if (nkv1)
                mbar_wait(bar_kv + 1, uint32_t((nkv1 - 1) & 1), nullptr);
            if (ns)
                mbar_wait(bar_s, uint32_t((ns - 1) & 1), nullptr);
            if (nyh)
                mbar_wait(bar_yh, uint32_t((nyh - 1) & 1), nullptr);
            if (n2)
                mbar_wait(bar_2, uint32_t((n2 - 1) & 1), nullptr);
        }
    } else {
        // ======================= the compute warps =======================================
        // Per chunk c: w o V(c) and L o S(c) (then the issuer runs dH(c) and Yi(c)); while
        // those products run, the gate scan of chunk c+1; then the epilogue of chunk c.
        constexpr float kTiny = 1.17549435e-38f; // smallest normal float
        const float *gam = a.gamma + b * a.seq;
        float gm_next = r < a.seq ? __ldg(gam + r) : 1.0f; // past the end: no decay
        // chunk values of this row from the gate scan
        float lam_r = 0.0f, sg_r = 1.0f, p_r = 0.0f, p_end = 0.0f, lam_end = 0.0f;
        int z_r = -1, z_end = -1;
        uint32_t par_r = 0, par_end = 0, any_big = 0;
        // The gate scan of chunk c: scans of log2|gamma|, of the last zero gate and of the
        // sign parity over each lane quarter's 32 tokens (both column halves compute the
        // same), then the prefixes of row r, the chunk's totals and the arrays the mask
        // reads.  Between two barriers of the compute warps: the first comes after every
        // compute warp has finished the previous chunk's mask (the last reader of those
        // arrays), and ends the loop for all of them at once when any has seen a failed
        // wait (false).
        auto scan_gates = [&](int64_t c) -> bool {
            const int64_t t0 = c * kGtChunk;
            const float gm = gm_next;
            gm_next = t0 + kGtChunk + r < a.seq ? __ldg(gam + t0 + kGtChunk + r) : 1.0f; // the next chunk's
            const bool zero_gate = fabsf(gm) < kTiny;
            float lg = zero_gate ? 0.0f : __log2f(fabsf(gm));
            int zl = zero_gate ? r : -1;
            uint32_t par = (!zero_gate && gm < 0.0f) ? 1u : 0u;
            const uint32_t big = __any_sync(0xffffffffu, !(fabsf(gm) <= 1.0f)) ? 1u : 0u; // |gamma| > 1, or NaN
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, lg, o);
                const int uz = __shfl_up_sync(0xffffffffu, zl, o);
                const uint32_t upar = __shfl_up_sync(0xffffffffu, par, o);
                if (lane >= o) {
                    lg += up;
                    zl = max(zl, uz);
                    par ^= upar;
                }
            }
            if (cg == 0 && lane == 31) {
                s_red[4 * q4] = __float_as_uint(lg);
                s_red[4 * q4 + 1] = uint32_t(zl);
                s_red[4 * q4 + 2] = par;
                s_red[4 * q4 + 3] = big;
            }
            if (!gt_compute_sync_and(ok))
                return false;
            float off = 0.0f;
            int zoff = -1;
            uint32_t poff = 0;
            z_end = -1;
            par_end = 0;
            any_big = 0;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int wz = int(s_red[4 * w + 1]);
                const uint32_t wp = s_red[4 * w + 2];
                if (w < q4) {
                    off += __uint_as_float(s_red[4 * w]);
                    zoff = max(zoff, wz);
                    poff ^= wp;
                }
                z_end = max(z_end, wz);
                par_end ^= wp;
                any_big |= s_red[4 * w + 3];
            }
            lam_r = lg + off;
            z_r = max(zl, zoff);
            par_r = par ^ poff;
            sg_r = par_r ? -1.0f : 1.0f;
            // lam of token 127, summed in the order its own row prefix was
            lam_end = __uint_as_float(s_red[12]) +
                      ((__uint_as_float(s_red[0]) + __uint_as_float(s_red[4])) + __uint_as_float(s_red[8]));
            if (cg == 0) {
                // the column factor L[j1, r], j1 the last token of this lane quarter
                const float lam_j1 = __uint_as_float(s_red[4 * q4]) + off;
                const int z_j1 = max(int(s_red[4 * q4 + 1]), zoff);
                const uint32_t par_j1 = s_red[4 * q4 + 2] ^ poff;
                s_lam[r] = lam_r;
                s_z[r] = z_r;
                s_sg[r] = sg_r;
                s_g[r] = z_j1 > r ? 0.0f : ((par_j1 ^ par_r) ? -1.0f : 1.0f) * ex2(lam_j1 - lam_r);
            }
            p_r = z_r >= 0 ? 0.0f : sg_r * ex2(lam_r);                            // P_r
            p_end = z_end >= 0 ? 0.0f : (par_end ? -1.0f : 1.0f) * ex2(lam_end); // P_127
            gt_compute_sync();
            return true;
        };
        bool run = scan_gates(0);
        for (int64_t c = 0; run && c < nchunks; ++c) {
            const int st = int(c & 1);
            const uint32_t ph = uint32_t(c & 1), ph_kv = uint32_t((c >> 1) & 1);
            const int64_t t0 = c * kGtChunk;
            // ---- w o V: token row r, this thread's kGtVCols value columns, high / low parts
            // (the v tile has landed; dH of the previous chunk, the last reader of w o V,
            // completed before that chunk's epilogue) --------------------------------------
            if (!mbar_wait(bar_kv + st, ph_kv, status))
                ok = false;
            if (ok) {
                const float w_r = z_end > r ? 0.0f : ((par_end ^ par_r) ? -1.0f : 1.0f) * ex2(lam_end - lam_r);
#pragma unroll
                for (int cc = 0; cc < kGtVCols / 8; ++cc) {
                    const uint32_t o = sw128_off(r, (kGtVCols / 8) * cg + cc);
                    uint4 hi, lo;
                    scale_split8(*reinterpret_cast<const uint4 *>(sm + GtSmem::kV + st * 16384 + o), w_r, hi, lo);
                    *reinterpret_cast<uint4 *>(sm + GtSmem::kWhi + o) = hi;
                    *reinterpret_cast<uint4 *>(sm + GtSmem::kWlo + o) = lo;
                }
            }
            // ---- L o S: row r, this thread's 32 kGtSBlocks columns, into tensor memory
            if (!mbar_wait(bar_s, ph, status))
                ok = false;
            ok = __all_sync(0xffffffffu, ok); // the tensor-memory accesses below are warp-collective
            tc_fence_after();
            if (ok) {
#pragma unroll 1
                for (int bb = 0; bb < kGtSBlocks; ++bb) {
                    const int jb = kGtSBlocks * cg + bb;
                    if (jb > q4)
                        continue; // above the diagonal: the zeros written once
                    uint32_t sr[32];
                    tmem_ld32_issue(tmem + lane_base + kGtColS + 32 * jb, sr);
                    tmem_ld_wait();
                    tmem_ld_fence(sr);
                    float s[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        s[e] = __uint_as_float(sr[e]);
                    uint32_t hi[16], lo[16];
                    if (jb < q4 && !any_big) {
                        // below the diagonal block: L[r, j] = L[r, j1] L[j1, j]
                        const int j1 = 32 * jb + 31;
                        const float f = z_r > j1 ? 0.0f : sg_r * s_sg[j1] * ex2(lam_r - s_lam[j1]);
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 gv = *reinterpret_cast<const float4 *>(s_g + 32 * jb + e);
                            split_bf16x2(s[e] * gv.x * f, s[e + 1] * gv.y * f, hi[e / 2], lo[e / 2]);
                            split_bf16x2(s[e + 2] * gv.z * f, s[e + 3] * gv.w * f, hi[e / 2 + 1], lo[e / 2 + 1]);
                        }
                    } else {
                        // the diagonal block (or a chunk with gates above 1 in magnitude):
                        // element by element
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const int j = 32 * jb + e;
                            const float4 lj = *reinterpret_cast<const float4 *>(s_lam + j);
                            const float4 sj = *reinterpret_cast<const float4 *>(s_sg + j);
                            const float ljv[4] = {lj.x, lj.y, lj.z, lj.w}, sjv[4] = {sj.x, sj.y, sj.z, sj.w};
                            float m[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const bool valid = j + u <= r && z_r <= j + u;
                                m[u] = valid ? s[e + u] * (sg_r * sjv[u]) * ex2(lam_r - ljv[u]) : 0.0f;
                            }
                            split_bf16x2(m[0], m[1], hi[e / 2], lo[e / 2]);
                            split_bf16x2(m[2], m[3], hi[e / 2 + 1], lo[e / 2 + 1]);
                        }
                    }
                    tmem_st16(tmem + lane_base + kGtColMhi + 16 * jb, hi);
                    tmem_st16(tmem + lane_base + kGtColMlo + 16 * jb, lo);
                }
                tmem_st_wait();
            }
            // L o S and w o V of this warp are written: tell the issuer (after a failed
            // wait too, so that it does not wait in vain; the loop ends at the next barrier)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); // w o V writes -> MMA reads
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !(a.hold_first_mw && c == 0))
                mbar_arrive(bar_mw);
            // ---- while dH(c) and Yi(c) run: the gate scan of the next chunk -----------
            const float p_rc = p_r, p_endc = p_end; // this chunk's, for its epilogue
            run = c + 1 < nchunks ? scan_gates(c + 1) : gt_compute_sync_and(ok);
            if (!run) {
                ok = false;
                break;
            }
            // ---- the chunk's products: y = Yi + P o Yh and H' = P_127 H + dH ------------
            if (!mbar_wait(bar_2, ph, status))
                ok = false;
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok) {
                {
                    uint32_t yir[kGtVCols], yhr[kGtVCols];
                    tmem_ld_n_issue<kGtVCols>(tmem + lane_base + kGtColYi + kGtVCols * cg, yir);
                    tmem_ld_n_issue<kGtVCols>(tmem + lane_base + kGtColYh + kGtVCols * cg, yhr);
                    tmem_ld_wait();
                    tmem_ld_fence(yir);
                    tmem_ld_fence(yhr);
                    if (t0 + r < a.seq) {
                        __nv_bfloat16 *dst = a.y + (b * a.seq + t0 + r) * a.dv + n0 + kGtVCols * cg;
#pragma unroll
                        for (int q8 = 0; q8 < kGtVCols / 8; ++q8) {
                            float o[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                o[e] = fmaf(p_rc, __uint_as_float(yhr[8 * q8 + e]), __uint_as_float(yir[8 * q8 + e]));
                            *reinterpret_cast<uint4 *>(dst + 8 * q8) =
                                make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                           pack_bf16x2(o[6], o[7]));
                        }
                    }
                }
                {
                    uint32_t dhr[kGtVCols], dlr[kGtVCols];
                    tmem_ld_n_issue<kGtVCols>(tmem + lane_base + kGtColDH + kGtVCols * cg, dhr);
                    tmem_ld_n_issue<kGtVCols>(tmem + lane_base + kGtColDH + kGtNv + kGtVCols * cg, dlr);
                    tmem_ld_wait();
                    tmem_ld_fence(dhr);
                    tmem_ld_fence(dlr);
#pragma unroll
                    for (int e = 0; e < kGtVCols; ++e)
                        H[e] = fmaf(p_endc, H[e], __uint_as_float(dhr[e]) + __uint_as_float(dlr[e]));
                }
                store_h();
            }
            // this warp has read its accumulators and stored its part of H(c+1)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); // H writes -> MMA reads
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_epi);
        }
        if (!run)
            ok = false;
        if (ok) {
            __nv_bfloat16 *dst = a.final_state + (b * kGtDk + r) * a.dv + n0 + kGtVCols * cg;
#pragma unroll
            for (int q8 = 0; q8 < kGtVCols / 8; ++q8) {
                const float *h = H + 8 * q8;
                *reinterpret_cast<uint4 *>(dst + 8 * q8) = make_uint4(
                    pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tmem, kGtTmemCols);
}

} // namespace ss
