// ss_scan_fwd.cuh -- prompt-scan kernel of the Mamba-1 selective scan (S6).
//
// Recurrence (nnterp "selective_scan" component, SelectiveScan description;
// TransformerLens "ssm_mixer", compute_ssm_state):
//   h_t[n] = exp(dt_t A[c,n]) h_{t-1}[n] + dt_t B[b,n,t] x[b,c,t]
//   y_t    = sum_n C[b,n,t] h_t[n] + D[c] x[b,c,t],   out_t = y_t silu(z_t)
// with an enforced reset ("s6_reset" blog draft, Enforced Boundary Resetting)
// folded into the decay: at a flagged token exp(dt A) is replaced by exactly 0 --
// the zero of the (decay, increment) operator -- so h_t = dt_t B_t x_t there.
//
// Cost model.  The N exponentials per (b, t, c) are the bound (MUFU ex2, 16 per
// clock per SM); the HBM traffic is about 8 bytes per (b, t, c).  The design keeps
// the exponential unit fed:
//
//  * Work split.  A scan lane owns TWO states of one channel and walks the tokens
//    in order, so each exponential is computed once and the state never leaves
//    registers.  A scan warp covers 32 / (N/2) channels (4 at N = 16).
//  * Warp specialisation.  Each CTA has four scan warps (one per SM sub-partition,
//    so all four MUFU units work), two producer warps and two epilogue warps.  The
//    producers stream x, dt_raw, z, B and C (B, C shared by every channel of a
//    batch row) into a two-stage shared-memory ring -- as 2-D TMA tile loads several
//    chunks ahead on aligned shapes -- computing dt = softplus(dt_raw + dt_bias) and
//    dt*x on the way.  The epilogue warps sum the scan lanes' partial outputs over
//    the N/2 state pairs, apply D*x and the silu(z) gate and store y.  The scan warps therefore run an
//    uninterrupted stream of packed fp32x2 multiplies, MUFU ex2 and fused
//    multiply-adds.  The roles hand chunks of 32 tokens over through mbarriers
//    (bounded waits).
//  * Chained segments.  The sequence is cut into segments; a work unit is (channel
//    group, segment).  Persistent CTAs take units from a global counter in
//    segment-major order; the scan carry (the state at a segment's end) is passed
//    to the next segment's CTA through the workspace under an epoch-tagged flag --
//    the "carry between chunks" of a two-level scan, applied at segment
//    granularity.  Without a workspace each CTA runs one channel group over the
//    whole sequence.
#pragma once

#include "ss_device.cuh"
#include "ss_sync.cuh"

namespace ss {

struct ScanArgs {
    int64_t batch, channels, seq;
    const void *x, *dt, *B, *C, *z;
    const float *A, *D, *dt_bias, *h0;
    const uint8_t *reset;
    void *y;
    float *h_last;
    float *h_all;             // nullable: the state after every token [b, c, L, N] fp32
    float *betas;             // nullable: the step size dt of every token [b, c, L] fp32
    // fused causal conv + SiLU prologue (x above is then the conv's input u):
    const float *conv_w;      // [channels, conv_k] taps
    const float *conv_b;      // [channels] bias (nullable)
    const float *conv_state;  // [b, c, conv_k - 1] inputs before the sequence (nullable: 0)
    float *conv_state_out;    // [b, c, conv_k - 1] the last conv_k - 1 inputs (nullable)
    void *x_out;              // [b, c, L] the scan input x = silu(conv) (nullable)
    int conv_k;               // taps, 1..4
    int softplus;
    int64_t groups_per_batch; // channel groups per batch row
    int64_t groups;           // batch * groups_per_batch
    int64_t seg_len;          // tokens per segment (a multiple of the chunk)
    int64_t segments;         // ceil(seq / seg_len); 1 without a workspace
    uint8_t *workspace;       // nullptr: one CTA per channel group, one segment
    uint32_t *status;         // status word when there is no workspace
    // In-GPU two-level scan over the sequence (no carries between segments):
    //  pass 1: every segment starts from zero, no outputs; its end state goes to
    //          seg_state[s * seg_stride + (b * channels + c) * N + n];
    //  pass 2: every segment starts from seg_in[s * seg_stride + ...] (the joined
    //          entering state) and writes y; h_last comes from the join.
    // pass 0 is the single-pass scan (chained segments, or one CTA per group).
    int pass;
    float *seg_state;
    const float *seg_in;
    int64_t seg_stride;
};

// Tensor maps of the TMA path: x, dt (and z) as [batch * channels rows][seq] and B, C
// as [batch * state_dim rows][seq], boxes of one chunk of tokens.  z is not loaded into
// shared memory: the issuer only prefetches each chunk's z tile into L2, several chunks
// before the epilogue reads it with plain loads.
struct TmaMaps {
    CUtensorMap x, dt, B, C, z;
};

// Workspace layout (bytes): the caller zeroes it once; every call leaves it ready for
// the next one -- also a call whose waits gave up, since every warp counts itself
// out on every exit path and the last one resets the counters.
struct WsHeader {
    uint32_t counter; // next work unit of this call
    uint32_t status;  // sticky error bits (1 << SS_ERR_TIMEOUT)
    uint32_t done;    // warps finished in this call
    uint32_t pad0;
    uint64_t epoch;   // advanced by the last warp of every call; tags the carry flags
    uint32_t pad[10];
};
static_assert(sizeof(WsHeader) == 64, "workspace header is 64 bytes");

// A carry flag holds (epoch << 24) | segment: 40 bits of epoch (a flag left by an
// earlier call never matches a later one) and 24 bits of segment index (the host
// keeps segments below 2^24).
constexpr int kFlagSegBits = 24;
__device__ __forceinline__ uint64_t carry_tag(uint64_t epoch, int64_t s)
{
    return ((epoch & ((uint64_t(1) << 40) - 1)) << kFlagSegBits) | uint64_t(s);
}

// Geometry of the prompt-scan kernel for state_dim N with SPL states per scan lane.
// A channel's N states are spread over kLanes = N / SPL lanes of one warp; a warp
// covers 32 / kLanes channels, a CTA (four scan warps) kChanPerCta.  SPL = 2 (eight
// lanes per channel at N = 16) gives the most independent warps, for shapes with few
// channel groups.  SPL = 4 (four lanes per channel, 32 channels per CTA, one CTA per
// SM) halves the lanes that read each token's dt and dt*x and the partial outputs
// the epilogue stores, reads and sums, per (b, t, c): the scan is bound by the
// exponential unit, and those shared-memory bytes and instructions are what keeps it
// from running at that unit's rate.
template <int N, int SPL> struct ScanShape {
    static_assert(N == 4 || N == 8 || N == 16, "state_dim must be 4, 8 or 16");
    static_assert(SPL == 2 || (SPL == 4 && N == 16), "states per lane: 2, or 4 at state_dim 16");
    static constexpr int kSpl = SPL;
    static constexpr int kLanes = N / SPL;             // lanes per channel
    static constexpr int kChanPerWarp = 32 / kLanes;
    // Roles: warps 0-3 scan (one per SM sub-partition, so all four MUFU units work),
    // then kIoWarps producer warps, kIoWarps epilogue warps and one issuer warp.  Warp
    // w executes on sub-partition w % 4, so the producers and the epilogue warps are
    // spread evenly over the sub-partitions.
    static constexpr int kScanWarps = 4;
    static constexpr int kIoWarps = SPL == 4 ? 4 : 2;  // warps per IO role
    static constexpr int kWarps = kScanWarps + 2 * kIoWarps + 1;
    static constexpr int kIssuerWarp = kWarps - 1;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kIoThreads = 32 * kIoWarps;   // threads per IO role
    static constexpr int kChanPerCta = kScanWarps * kChanPerWarp;
    static constexpr int kChunk = 32;                  // tokens per pipeline stage
    static constexpr int kBlocks = kChunk / 8;         // 8-token blocks per chunk
    static constexpr int kRow = kChunk + 4;            // padded row (floats)
    // ring depths: at N = 16 four input and three output stages (measured 5% faster
    // than three and two) still leave room for two CTAs per SM with SPL = 2 (one CTA
    // per SM with SPL = 4); N = 4 and 8 put 2-4x more channels in a CTA and keep the
    // rings short to fit
    static constexpr int kStages = N == 16 ? 4 : 2, kYStages = N == 16 ? 3 : 2;
    // input stage (floats): meta | dt rows | dt*x rows | reset bias
    static constexpr int kMeta = 8;
    static constexpr int kDTOff = kMeta;
    static constexpr int kDXOff = kDTOff + kChanPerCta * kRow;
    static constexpr int kRBOff = kDXOff + kChanPerCta * kRow;
    static constexpr int kInStage = kRBOff + kChunk;
    // output stage (floats): meta | partial outputs
    static constexpr int kYChan = kLanes * kRow + 4;   // per-channel block, bank-skewed
    static constexpr int kYPOff = kMeta;
    // then x of the chunk in storage type [channels][chunk] (the fused conv form hands
    // it from the producers to the epilogue here)
    static constexpr int kYXOff = kYPOff + kChanPerCta * kYChan;
    template <typename T> static constexpr int y_stage() { return kYXOff + kChanPerCta * kChunk * int(sizeof(T)) / 4; }
    template <typename T> static constexpr int floats() { return kStages * kInStage + kYStages * y_stage<T>(); }
    // IO work per chunk
    static constexpr int kTokTasks = kChanPerCta * kBlocks;       // (channel, 8 tokens)
    static constexpr int kTokPerLane = kTokTasks / kIoThreads;
    static constexpr int kBCTasks = 2 * N * kBlocks;              // (B/C row, 8 tokens)
    static constexpr int kBCPerLane = (kBCTasks + kIoThreads - 1) / kIoThreads;
    // raw ring: x, dt tiles [channels][chunk] and B, C tiles [N][chunk] in storage
    // type (z is only needed by the epilogue, which reads it from global memory).  On aligned shapes TMA fills whole slots; the issuer warp keeps every
    // slot its readers have released loading, so up to kRawStages chunks are in
    // flight.  The scan warps read B and C straight from the slot, in storage type
    // (bf16 halves their shared-memory traffic), from tiles swizzled by TMA so the
    // kLanes state rows a warp reads at once fall into distinct banks.  On the ragged
    // path the producers write the B and C tiles themselves in the same layout.
    static constexpr int kRawStages = N == 16 ? 8 : 4;
    // mbarriers: in_full, in_empty [kStages]; y_full, y_empty [kYStages]; raw_full,
    // raw_empty [kRawStages]
    static constexpr int kBarInFull = 0, kBarInEmpty = kStages;
    static constexpr int kBarYFull = 2 * kStages, kBarYEmpty = 2 * kStages + kYStages;
    static constexpr int kBarRawFull = 2 * (kStages + kYStages), kBarRawEmpty = kBarRawFull + kRawStages;
    static constexpr int kBars = kBarRawEmpty + kRawStages;
    static constexpr int align1k(int b) { return (b + 1023) / 1024 * 1024; }
    template <typename T> static constexpr int raw_x_off() { return 0; }
    template <typename T> static constexpr int raw_dt_off() { return kChanPerCta * kChunk * int(sizeof(T)); }
    // B and C tiles start on 1024-byte boundaries (the swizzle pattern's period)
    template <typename T> static constexpr int raw_b_off() { return align1k(2 * kChanPerCta * kChunk * int(sizeof(T))); }
    template <typename T> static constexpr int raw_c_off() { return raw_b_off<T>() + align1k(N * kChunk * int(sizeof(T))); }
    template <typename T> static constexpr int raw_stage_bytes()
    {
        return raw_c_off<T>() + align1k(N * kChunk * int(sizeof(T)));
    }
    // shared memory: [raw ring] [input stages] [output stages] [barriers] [raw meta]
    template <typename T, bool TMA> static constexpr size_t smem_bytes()
    {
        return size_t(kRawStages * raw_stage_bytes<T>()) + size_t(floats<T>()) * 4 + 8 * size_t(kBars) +
               32 * size_t(kRawStages);
    }
    // The lane with state group g owns states g, g + kLanes, g + 2 kLanes, ...; the B and
    // C tiles are swizzled by TMA with the swizzle whose span is exactly one tile row
    // (64 bytes for bf16 rows of 32 tokens, 128 bytes for fp32 rows), so the rows a
    // warp reads at once fall into distinct banks: with 64-byte rows, rows g and g + 1
    // lie in different halves of the banks and rows g and g + 2 differ in the chunk the
    // swizzle selects; with 128-byte rows, the swizzle alone separates eight rows.  (A
    // swizzle span wider than the row is not used: TMA lays such a box out at the span's
    // pitch, not the row's.)
    template <typename T> static constexpr int swizzle() { return sizeof(T) == 2 ? 64 : 128; }
    template <typename T> static __device__ __forceinline__ int state(int g, int j) { return g + kLanes * j; }
    static_assert(kTokTasks % kIoThreads == 0, "token tasks fill whole IO lanes");
    static_assert(kInStage % 4 == 0 && kYXOff % 4 == 0, "16-byte aligned stages");
};

struct ChunkMeta {
    int64_t t0;   // first token of the chunk
    int64_t g;    // channel group (b * groups_per_batch + group)
    int32_t s;    // segment
    int32_t flags;
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

// Chunk descriptors live in the first 32 bytes of each stage, field by field.
__device__ __forceinline__ void write_meta(float *stage, int64_t t0, int64_t g, int32_t s, int32_t flags)
{
    int64_t *w = reinterpret_cast<int64_t *>(stage);
    w[0] = t0;
    w[1] = g;
    int32_t *v = reinterpret_cast<int32_t *>(stage + 4);
    v[0] = s;
    v[1] = flags;
}

__device__ __forceinline__ ChunkMeta read_meta(const float *stage)
{
    const int64_t *w = reinterpret_cast<const int64_t *>(stage);
    const int32_t *v = reinterpret_cast<const int32_t *>(stage + 4);
    ChunkMeta m;
    m.t0 = w[0];
    m.g = w[1];
    m.s = v[0];
    m.flags = v[1];
    return m;
}

// Byte offset of 16-byte chunk `c16` of row `row` in a B or C tile of the raw ring.
// The tile is a dense [N rows][chunk tokens] box (64-byte rows for bf16, 128-byte rows
// for fp32) that TMA writes with a swizzle: the 16-byte chunk index (address bits
// 4..6) is XORed with address bits 7.. -- two bits of them for the 64-byte swizzle,
// three for the 128-byte one.
template <typename T, int SWZ> __device__ __forceinline__ int bc_offset(int row, int c16)
{
    const int lin = row * (32 * int(sizeof(T))) + (c16 << 4);
    return SWZ == 64 ? lin ^ (((lin >> 7) & 3) << 4) : lin ^ (((lin >> 7) & 7) << 4);
}

// silu on the output gate: the exact form for fp32 outputs; for bf16 outputs the
// MUFU tanh form 0.5 v (1 + tanh(v / 2)) (one MUFU op instead of two, error in the
// gate below 2.5e-4 |v|, inside the bf16 output tolerance).
template <typename T> __device__ __forceinline__ float gate(float v);
template <> __device__ __forceinline__ float gate<float>(float v) { return silu(v); }
template <> __device__ __forceinline__ float gate<__nv_bfloat16>(float v)
{
    float t;
    const float h = 0.5f * v;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
}

// ---------------------------------------------------------------------------------------
// producer warp: global -> registers (one chunk ahead) -> shared-memory stage
// ---------------------------------------------------------------------------------------

template <int N, int SPL, typename T, bool HAS_RESET, bool VEC, bool CONV>
struct IoPrefetch {
    using S = ScanShape<N, SPL>;
    Raw8<T> bc[S::kBCPerLane];
    Raw8<T> xr[S::kTokPerLane], dr[S::kTokPerLane];
    float bias[S::kTokPerLane];
    int64_t bias_g = -1; // channel group whose dt_bias values `bias` holds
    uint32_t rbyte;
    // fused conv: taps and bias of each task's channel (cached with dt_bias), and the
    // three conv inputs before each task's first token
    float cw[CONV ? S::kTokPerLane : 1][4], cb[CONV ? S::kTokPerLane : 1];
    float halo[CONV ? S::kTokPerLane : 1][3];
    // (TMA path) the last three inputs of each task's block in the previous chunk, and
    // which chunk that was: the next chunk of the same rows takes its first block's halo
    // from them
    float tail[CONV ? S::kTokPerLane : 1][3] = {};
    int64_t tail_g = -1, tail_t0 = -1;

    __device__ __forceinline__ void load_bias(const ScanArgs &p, int lane, int64_t g)
    {
        if (g == bias_g)
            return;
        bias_g = g;
        const int64_t c0 = (g % p.groups_per_batch) * S::kChanPerCta;
#pragma unroll
        for (int m = 0; m < S::kTokPerLane; ++m) {
            int64_t c = c0 + (lane + S::kIoThreads * m) / S::kBlocks;
            c = c < p.channels ? c : p.channels - 1;
            bias[m] = p.dt_bias ? __ldg(p.dt_bias + c) : 0.0f;
            if constexpr (CONV) {
                // taps aligned to the newest input: cw[m][3] multiplies u_t
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int kk = k - (4 - p.conv_k);
                    cw[m][k] = kk >= 0 ? __ldg(p.conv_w + c * p.conv_k + kk) : 0.0f;
                }
                cb[m] = p.conv_b ? __ldg(p.conv_b + c) : 0.0f;
            }
        }
    }

    __device__ __forceinline__ void load(const ScanArgs &p, int lane, int64_t g, int64_t t0)
    {
        const int64_t L = p.seq;
        const uint32_t gpb = uint32_t(p.groups_per_batch), b32 = uint32_t(g) / gpb;
        const int64_t b = b32;
        const int64_t c0 = int64_t(uint32_t(g) - b32 * gpb) * S::kChanPerCta;
        const T *Bb = static_cast<const T *>(p.B) + b * N * L;
        const T *Cb = static_cast<const T *>(p.C) + b * N * L;
#pragma unroll
        for (int m = 0; m < S::kBCPerLane; ++m) {
            const int q = lane + S::kIoThreads * m;
            if (q < S::kBCTasks) {
                const int r = q % (2 * N), tb = q / (2 * N);
                const T *src = r < N ? Bb + r * L : Cb + (r - N) * L;
                if (!SS_IN_BOUNDS(b < p.batch, 120))
                    continue;
                if (VEC)
                    bc[m].load_vec(src, t0 + tb * 8, L);
                else
                    bc[m].load_scalar(src, t0 + tb * 8, L);
            }
        }
#pragma unroll
        for (int m = 0; m < S::kTokPerLane; ++m) {
            const int q = lane + S::kIoThreads * m;
            const int cl = q / S::kBlocks, tb = q % S::kBlocks;
            int64_t c = c0 + cl;
            c = c < p.channels ? c : p.channels - 1;
            const int64_t row = b * p.channels + c;
            const int64_t t = t0 + tb * 8;
            if (!SS_IN_BOUNDS(row < p.batch * p.channels && t0 < L, 121))
                continue;
            const T *xrow = static_cast<const T *>(p.x) + row * L;
            const T *drow = static_cast<const T *>(p.dt) + row * L;
            if (VEC) {
                xr[m].load_vec_stream(xrow, t, L);
                dr[m].load_vec_stream(drow, t, L);
            } else {
                xr[m].load_scalar(xrow, t, L);
                dr[m].load_scalar(drow, t, L);
            }
        }
        load_bias(p, lane, g);
        if constexpr (CONV)
            load_halo(p, lane, g, t0);
        if (HAS_RESET)
            rbyte = (lane < S::kChunk && t0 + lane < L) ? uint32_t(__ldg(p.reset + b * L + t0 + lane)) : 0u;
    }

    // The three conv inputs before each task's first token t: u[t-3 .. t-1] from global
    // memory (L2 hits: the same rows are being tiled in), or from the caller's conv
    // state before the sequence start (zeros without one).
    __device__ __forceinline__ void load_halo(const ScanArgs &p, int lane, int64_t g, int64_t t0)
    {
        const uint32_t gpb = uint32_t(p.groups_per_batch), b32 = uint32_t(g) / gpb;
        const int64_t c0 = int64_t(uint32_t(g) - b32 * gpb) * S::kChanPerCta;
        const int64_t H = p.conv_k - 1;
#pragma unroll
        for (int m = 0; m < S::kTokPerLane; ++m) {
            const int q = lane + S::kIoThreads * m;
            const int cl = q / S::kBlocks, tb = q % S::kBlocks;
            int64_t c = c0 + cl;
            c = c < p.channels ? c : p.channels - 1;
            const int64_t row = int64_t(b32) * p.channels + c;
            const int64_t t = t0 + tb * 8;
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const int64_t pos = t - 3 + k;
                float v = 0.0f;
                if (pos >= 0)
                    v = Elem<T>::load(static_cast<const T *>(p.x) + row * p.seq + pos);
                else if (p.conv_state && H + pos >= 0)
                    v = __ldg(p.conv_state + row * H + H + pos);
                halo[m][k] = v;
            }
        }
    }

    // x and dt_raw from a raw TMA stage (B and C stay in the stage for the scan
    // warps; the reset byte is loaded by the caller).
    __device__ __forceinline__ void load_smem(const ScanArgs &p, int lane, int64_t g, const unsigned char *raw,
                                              int64_t t0)
    {
        const T *rx = reinterpret_cast<const T *>(raw + S::template raw_x_off<T>());
        const T *rd = reinterpret_cast<const T *>(raw + S::template raw_dt_off<T>());
#pragma unroll
        for (int m = 0; m < S::kTokPerLane; ++m) {
            const int q = lane + S::kIoThreads * m;
            const int cl = q / S::kBlocks, tb = q % S::kBlocks;
            xr[m].load_smem(rx + cl * S::kChunk + tb * 8);
            dr[m].load_smem(rd + cl * S::kChunk + tb * 8);
        }
        load_bias(p, lane, g);
        if constexpr (CONV) {
            // The halo of a task's block: the block before it in the same row of the tile,
            // or, for the first block, the previous chunk's last block -- held by lane
            // (lane | kBlocks - 1) of this warp one chunk ago when that chunk was this
            // row group's previous one (chunks of a unit reach the producers in order);
            // only the first chunk of a unit reads global memory (or the conv state).
            static_assert(S::kBlocks == 4 && S::kIoThreads % S::kBlocks == 0, "task (channel, block) layout");
            const bool follows = g == tail_g && t0 == tail_t0 + S::kChunk;
            if (!follows)
                load_halo(p, lane, g, t0);
#pragma unroll
            for (int m = 0; m < S::kTokPerLane; ++m) {
                const int q = lane + S::kIoThreads * m;
                const int cl = q / S::kBlocks, tb = q % S::kBlocks;
                float prev[3];
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    prev[k] = __shfl_sync(0xffffffffu, tail[m][k], (lane & 31) | (S::kBlocks - 1));
                if (tb > 0) {
#pragma unroll
                    for (int k = 0; k < 3; ++k)
                        halo[m][k] = Elem<T>::load_smem(rx + cl * S::kChunk + tb * 8 - 3 + k);
                } else if (follows) {
#pragma unroll
                    for (int k = 0; k < 3; ++k)
                        halo[m][k] = prev[k];
                }
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    tail[m][k] = xr[m].get(5 + k);
            }
            tail_g = g;
            tail_t0 = t0;
        }
    }
};

// Eight values to shared memory in storage type (one 16-byte store for bf16).
template <typename T> __device__ __forceinline__ void smem_store8(T *dst, const float (&o)[8]);
template <> __device__ __forceinline__ void smem_store8<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&o)[8])
{
    *reinterpret_cast<uint4 *>(dst) = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                                 pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
}
template <> __device__ __forceinline__ void smem_store8<float>(float *dst, const float (&o)[8])
{
    reinterpret_cast<float4 *>(dst)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4 *>(dst)[1] = make_float4(o[4], o[5], o[6], o[7]);
}

// CONV (fused causal conv + SiLU): x of each token is silu(cb + sum_k w_k u_{t-3+k})
// from the task's eight inputs u (the raw x tile) and the three before them; x also
// goes to the chunk's output stage (`ystage`, already free) for the epilogue, and the
// last conv_k - 1 inputs of each row to conv_state_out.
template <int N, int SPL, typename T, bool HAS_RESET, bool VEC, bool CONV, int EMIT>
__device__ __forceinline__ void produce_chunk(const ScanArgs &p, int lane,
                                              const IoPrefetch<N, SPL, T, HAS_RESET, VEC, CONV> &f, float *stage,
                                              unsigned char *raw, int64_t t0, int64_t g, float *ystage)
{
    using S = ScanShape<N, SPL>;
    const int64_t L = p.seq;
    if constexpr (!VEC) { // ragged path: B and C tiles into the raw slot, as TMA would lay them out
#pragma unroll
        for (int m = 0; m < S::kBCPerLane; ++m) {
            const int q = lane + S::kIoThreads * m;
            if (q < S::kBCTasks) {
                const int r = q % (2 * N), tb = q / (2 * N);
                unsigned char *tile = raw + (r < N ? S::template raw_b_off<T>() : S::template raw_c_off<T>());
                const int row = r < N ? r : r - N;
                constexpr int kChunksPer8 = int(sizeof(T)) / 2; // 16-byte chunks per 8 tokens
#pragma unroll
                for (int h = 0; h < kChunksPer8; ++h) {
                    const int o = bc_offset<T, S::template swizzle<T>()>(row, tb * kChunksPer8 + h);
                    if (SS_IN_BOUNDS(o >= 0 && o + 16 <= N * S::kChunk * int(sizeof(T)), 123))
                        *reinterpret_cast<uint4 *>(tile + o) = reinterpret_cast<const uint4 *>(&f.bc[m])[h];
                }
            }
        }
    }
    if (HAS_RESET && lane < S::kChunk)
        stage[S::kRBOff + lane] = f.rbyte ? -INFINITY : 0.0f;
    const bool softplus_on = p.softplus != 0;
#pragma unroll
    for (int m = 0; m < S::kTokPerLane; ++m) {
        const int q = lane + S::kIoThreads * m;
        const int cl = q / S::kBlocks, tb = q % S::kBlocks;
        const int64_t tl = t0 + tb * 8;
        float xv[8];
        if constexpr (CONV) {
            float U[11];
#pragma unroll
            for (int k = 0; k < 3; ++k)
                U[k] = f.halo[m][k];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                U[3 + j] = f.xr[m].get(j);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float acc = f.cb[m];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    acc = fmaf(f.cw[m][k], U[j + k], acc);
                xv[j] = tl + j < L ? gate<T>(acc) : 0.0f;
            }
            smem_store8<T>(reinterpret_cast<T *>(ystage + S::kYXOff) + cl * S::kChunk + tb * 8, xv);
            // the last conv_k - 1 inputs of the row (before the sequence start: from the
            // conv state, for sequences shorter than the window)
            const int64_t H = p.conv_k - 1;
            if (p.conv_state_out && H > 0 && tl + 8 > L - H && tl <= L) {
                const uint32_t gpb = uint32_t(p.groups_per_batch), b32 = uint32_t(g) / gpb;
                const int64_t c = int64_t(uint32_t(g) - b32 * gpb) * S::kChanPerCta + cl;
                if (c < p.channels) {
                    const int64_t row = int64_t(b32) * p.channels + c;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int64_t pos = tl + j;
                        if (pos >= L - H && pos < L && SS_IN_BOUNDS(row < p.batch * p.channels, 125))
                            p.conv_state_out[row * H + (pos - (L - H))] = U[3 + j];
                    }
                    if (tl == 0)
                        for (int64_t pos = L - H; pos < 0; ++pos)
                            p.conv_state_out[row * H + (pos - (L - H))] =
                                p.conv_state ? __ldg(p.conv_state + row * H + H + pos) : 0.0f;
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                xv[j] = f.xr[m].get(j);
        }
        float2 dtv[4], dxv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 r = __fadd2_rn(make_float2(f.dr[m].get(2 * k), f.dr[m].get(2 * k + 1)),
                                        make_float2(f.bias[m], f.bias[m]));
            float2 d = softplus_on ? softplus_poly2(r) : r;
            if (tl + 8 > L) { // past the end: decay 1, increment 0
                d.x = (tl + 2 * k < L) ? d.x : 0.0f;
                d.y = (tl + 2 * k + 1 < L) ? d.y : 0.0f;
            }
            dtv[k] = d;
            dxv[k] = __fmul2_rn(d, make_float2(xv[2 * k], xv[2 * k + 1]));
        }
        float4 *pd = reinterpret_cast<float4 *>(stage + S::kDTOff + cl * S::kRow + tb * 8);
        float4 *px = reinterpret_cast<float4 *>(stage + S::kDXOff + cl * S::kRow + tb * 8);
        pd[0] = make_float4(dtv[0].x, dtv[0].y, dtv[1].x, dtv[1].y);
        pd[1] = make_float4(dtv[2].x, dtv[2].y, dtv[3].x, dtv[3].y);
        px[0] = make_float4(dxv[0].x, dxv[0].y, dxv[1].x, dxv[1].y);
        px[1] = make_float4(dxv[2].x, dxv[2].y, dxv[3].x, dxv[3].y);
        if constexpr (EMIT != 0) {
            // the step sizes of this block's tokens, as the scan uses them
            const uint32_t gpb = uint32_t(p.groups_per_batch), b32 = uint32_t(g) / gpb;
            const int64_t c = int64_t(uint32_t(g) - b32 * gpb) * S::kChanPerCta + cl;
            if (p.betas && c < p.channels && tl < L &&
                SS_IN_BOUNDS(int64_t(b32) < p.batch && (int64_t(b32) * p.channels + c) * L + tl < p.batch * p.channels * L, 126)) {
                float *dst = p.betas + (int64_t(b32) * p.channels + c) * L + tl;
                if (tl + 8 <= L && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
                    __stcs(reinterpret_cast<float4 *>(dst), make_float4(dtv[0].x, dtv[0].y, dtv[1].x, dtv[1].y));
                    __stcs(reinterpret_cast<float4 *>(dst) + 1, make_float4(dtv[2].x, dtv[2].y, dtv[3].x, dtv[3].y));
                } else {
                    const float v[8] = {dtv[0].x, dtv[0].y, dtv[1].x, dtv[1].y, dtv[2].x, dtv[2].y, dtv[3].x, dtv[3].y};
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (tl + j < L)
                            __stcs(dst + j, v[j]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// epilogue warp: partial outputs -> sum over state pairs, D*x, gate -> y
// ---------------------------------------------------------------------------------------

template <typename T> __device__ __forceinline__ float2 gate2(float2 v);
template <> __device__ __forceinline__ float2 gate2<float>(float2 v)
{
    return make_float2(silu(v.x), silu(v.y));
}
template <> __device__ __forceinline__ float2 gate2<__nv_bfloat16>(float2 v)
{
    const float2 h = __fmul2_rn(v, make_float2(0.5f, 0.5f));
    float2 t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.x) : "f"(h.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.y) : "f"(h.y));
    return __ffma2_rn(h, t, h);
}

// Per-thread state of the epilogue that depends only on the channel group: the rows
// of x, z and y of this thread's channels and their D values.  Refreshed when the
// group changes (once per work unit), so a chunk costs no index arithmetic.
template <int N, int SPL, typename T> struct EpiCache {
    const T *x[ScanShape<N, SPL>::kTokPerLane];
    const T *z[ScanShape<N, SPL>::kTokPerLane];
    T *y[ScanShape<N, SPL>::kTokPerLane];
    T *xo[ScanShape<N, SPL>::kTokPerLane]; // fused conv form: rows of x_out (or null)
    float d[ScanShape<N, SPL>::kTokPerLane];
    int64_t g = -1;
};

// x and z are re-read from global memory (the producers' tile loads brought them into
// L2 a few chunks earlier), issued first so their latency overlaps the partial sums.
// In the fused conv form x is not an input: the producers left it in the output
// stage, and it is also stored to x_out when the caller asks for it.
template <int N, int SPL, typename T, bool VEC, bool CONV>
__device__ __forceinline__ void epilogue_chunk(const ScanArgs &p, int lane, const float *ystage, int64_t g, int64_t t0,
                                               EpiCache<N, SPL, T> &ec)
{
    using S = ScanShape<N, SPL>;
    const int64_t L = p.seq;
    if (ec.g != g) {
        const int64_t b = g / p.groups_per_batch;
        const int64_t c0 = (g - b * p.groups_per_batch) * S::kChanPerCta;
#pragma unroll
        for (int m = 0; m < S::kTokPerLane; ++m) {
            const int cl = (lane + S::kIoThreads * m) / S::kBlocks;
            const int64_t c_raw = c0 + cl;
            const bool valid = c_raw < p.channels;
            const int64_t c = valid ? c_raw : p.channels - 1;
            const int64_t off = (b * p.channels + c) * L;
            (void)SS_IN_BOUNDS(b < p.batch && c < p.channels && t0 < L, 130);
            ec.x[m] = static_cast<const T *>(p.x) + off;
            ec.z[m] = p.z ? static_cast<const T *>(p.z) + off : nullptr;
            ec.y[m] = valid ? static_cast<T *>(p.y) + off : nullptr;
            ec.xo[m] = (CONV && valid && p.x_out) ? static_cast<T *>(p.x_out) + off : nullptr;
            ec.d[m] = p.D ? __ldg(p.D + c) : 0.0f;
        }
        ec.g = g;
    }
    Raw8<T> xs[S::kTokPerLane], zs[S::kTokPerLane];
#pragma unroll
    for (int m = 0; m < S::kTokPerLane; ++m) {
        const int q = lane + S::kIoThreads * m;
        const int tb = q % S::kBlocks;
        if constexpr (CONV) {
            xs[m].load_smem(reinterpret_cast<const T *>(ystage + S::kYXOff) + (q / S::kBlocks) * S::kChunk + tb * 8);
            if (p.z) {
                if (VEC)
                    zs[m].load_vec(ec.z[m], t0 + tb * 8, L);
                else
                    zs[m].load_scalar(ec.z[m], t0 + tb * 8, L);
            }
        } else if (VEC) {
            xs[m].load_vec(ec.x[m], t0 + tb * 8, L);
            if (p.z)
                zs[m].load_vec(ec.z[m], t0 + tb * 8, L);
        } else {
            xs[m].load_scalar(ec.x[m], t0 + tb * 8, L);
            if (p.z)
                zs[m].load_scalar(ec.z[m], t0 + tb * 8, L);
        }
    }
#pragma unroll
    for (int m = 0; m < S::kTokPerLane; ++m) {
        const int q = lane + S::kIoThreads * m;
        const int cl = q / S::kBlocks, tb = q % S::kBlocks;
        float2 o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            o[k] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int pr = 0; pr < S::kLanes; ++pr) {
            const float4 *src = reinterpret_cast<const float4 *>(ystage + S::kYPOff + cl * S::kYChan + pr * S::kRow + tb * 8);
            const float4 v0 = src[0], v1 = src[1];
            o[0] = __fadd2_rn(o[0], make_float2(v0.x, v0.y));
            o[1] = __fadd2_rn(o[1], make_float2(v0.z, v0.w));
            o[2] = __fadd2_rn(o[2], make_float2(v1.x, v1.y));
            o[3] = __fadd2_rn(o[3], make_float2(v1.z, v1.w));
        }
        if (!ec.y[m])
            continue;
        const float Dc = ec.d[m];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            o[k] = __ffma2_rn(make_float2(Dc, Dc), make_float2(xs[m].get(2 * k), xs[m].get(2 * k + 1)), o[k]);
        if (p.z) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                o[k] = __fmul2_rn(o[k], gate2<T>(make_float2(zs[m].get(2 * k), zs[m].get(2 * k + 1))));
        }
        const float out[8] = {o[0].x, o[0].y, o[1].x, o[1].y, o[2].x, o[2].y, o[3].x, o[3].y};
        store8<T, VEC>(ec.y[m], t0 + tb * 8, L, out);
        if (CONV && ec.xo[m]) {
            float xo[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                xo[j] = xs[m].get(j);
            store8<T, VEC>(ec.xo[m], t0 + tb * 8, L, xo);
        }
    }
}

// ---------------------------------------------------------------------------------------
// producer loops
// ---------------------------------------------------------------------------------------

// Shared context of the roles of one CTA.
struct CtaCtx {
    float *in_base, *y_base;
    unsigned char *raw_base;
    uint64_t *in_full, *in_empty, *y_full, *y_empty, *raw_full, *raw_empty;
    int64_t *raw_meta; // per raw stage: t0, g, (s | flags << 32)
    WsHeader *ws;
    uint32_t *status;
};

constexpr uint32_t kNoUnit = 0xffffffffu;

// Next unit of this CTA: from the work counter (chained) or blockIdx.x (static).
__device__ __forceinline__ uint32_t take_unit(const ScanArgs &p, WsHeader *ws, bool first)
{
    if (!ws)
        return first ? uint32_t(blockIdx.x) : kNoUnit;
    const uint32_t u = grab_unit(&ws->counter);
    return int64_t(u) >= p.groups * p.segments ? kNoUnit : u;
}

// Where work unit u = segment * groups + group lies: computed once per unit (the
// divisions are not cheap), then advanced chunk by chunk.
struct UnitPos {
    int64_t g, s, t_begin; // channel group, segment, first token
    int64_t nck;           // chunks in the unit
    int32_t xrow, brow;    // first x / dt row and first B / C row of the group
};

template <int N, int SPL> __device__ __forceinline__ UnitPos unit_pos(const ScanArgs &p, uint32_t u)
{
    UnitPos up;
    // units, groups and rows all fit in 32 bits (checked on the host)
    const uint32_t groups = uint32_t(p.groups), gpb = uint32_t(p.groups_per_batch);
    const uint32_t g = u % groups, s = u / groups, b = g / gpb;
    up.g = g;
    up.s = s;
    up.t_begin = int64_t(s) * p.seg_len;
    const int64_t rest = p.seq - up.t_begin;
    const int64_t len = rest < p.seg_len ? rest : p.seg_len;
    up.nck = (len + ScanShape<N, SPL>::kChunk - 1) / ScanShape<N, SPL>::kChunk;
    up.xrow = int32_t(int64_t(b) * p.channels + int64_t(g - b * gpb) * ScanShape<N, SPL>::kChanPerCta);
    up.brow = int32_t(b * N);
    return up;
}

// Token pair `pi` of a 16-byte chunk of a B or C row, widened to fp32: bf16 rows hold
// 8 tokens (pairs are 32-bit words), fp32 rows 4.
template <typename T> __device__ __forceinline__ float2 bc_pair(const uint4 &w, int pi);
template <> __device__ __forceinline__ float2 bc_pair<__nv_bfloat16>(const uint4 &w, int pi)
{
    const uint32_t u = pi == 0 ? w.x : (pi == 1 ? w.y : (pi == 2 ? w.z : w.w));
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
template <> __device__ __forceinline__ float2 bc_pair<float>(const uint4 &w, int pi)
{
    return pi == 0 ? make_float2(__uint_as_float(w.x), __uint_as_float(w.y))
                   : make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
}

// Decays and increments of one group of four tokens for the lane's SPL states:
// [state][token pair] as (token t, token t + 1).
template <int SPL> struct GroupTerms {
    float2 a[SPL][2], v[SPL][2];
};

// One chunk of the recurrence for this lane's SPL states nn[] of channel `cl`: dt and
// dt*x from the input stage, B and C from the raw slot (storage type), the partial
// outputs C.h over the lane's states to `ys`.  Per pair of tokens and state: one
// packed multiply for the exponent arguments, two MUFU ex2, one packed multiply for
// the increments, two FMAs along the sequence and one packed op for the readout.
//
// Software pipelined over groups of four tokens: the exponentials and increments of
// group k + 1 are issued before the sequential FMA chain of group k, so the MUFU
// latency of one group hides behind the chain of the previous one (with one or two
// scan warps per sub-partition there is little other work to switch to).
//
// EMIT == 1: also store the state after every token to `hrow` (this channel's row of
// h_all at the chunk's first token, N floats per token), for the first `valid` tokens.
template <int N, int SPL, typename T, bool HAS_RESET, int EMIT>
__device__ __forceinline__ void scan_chunk(const float *stage, const unsigned char *raw, float *ys, int cl,
                                           const int (&nn)[SPL], const float2 (&A2)[SPL], float (&hs)[SPL],
                                           float *hrow, int64_t valid)
{
    using S = ScanShape<N, SPL>;
    constexpr int kTok = 16 / int(sizeof(T)); // tokens per 16-byte chunk of a B/C row
    constexpr int kGroups = S::kChunk / 4;
    constexpr int SWZ = S::template swizzle<T>();
    const unsigned char *Bt = raw + S::template raw_b_off<T>();
    const unsigned char *Ct = raw + S::template raw_c_off<T>();
    const float *rbs = stage + S::kRBOff;
    const float *dts = stage + S::kDTOff + cl * S::kRow;
    const float *dxs = stage + S::kDXOff + cl * S::kRow;
    uint4 wb[SPL], wc[SPL];
#pragma unroll
    for (int j = 0; j < SPL; ++j)
        wb[j] = wc[j] = make_uint4(0, 0, 0, 0);
    GroupTerms<SPL> gt[2];
    // decays and increments of group k into `f`
    auto front = [&](int k, GroupTerms<SPL> &f) {
        const int t = 4 * k;
        if (t % kTok == 0) {
#pragma unroll
            for (int j = 0; j < SPL; ++j) {
                const int o = bc_offset<T, SWZ>(nn[j], t / kTok);
                if (SS_IN_BOUNDS(o >= 0 && o + 16 <= N * S::kChunk * int(sizeof(T)), 112))
                    wb[j] = *reinterpret_cast<const uint4 *>(Bt + o);
            }
        }
        const float4 d4 = *reinterpret_cast<const float4 *>(dts + t);
        const float4 u4 = *reinterpret_cast<const float4 *>(dxs + t);
        float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (HAS_RESET)
            r4 = *reinterpret_cast<const float4 *>(rbs + t);
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
            const int pi = (t % kTok) / 2 + pr;
            const float2 dd = pr ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
            const float2 uu = pr ? make_float2(u4.z, u4.w) : make_float2(u4.x, u4.y);
            const float2 rr = pr ? make_float2(r4.z, r4.w) : make_float2(r4.x, r4.y);
#pragma unroll
            for (int j = 0; j < SPL; ++j) {
                const float2 g = HAS_RESET ? __ffma2_rn(dd, A2[j], rr) : __fmul2_rn(dd, A2[j]);
                f.a[j][pr] = make_float2(ex2(g.x), ex2(g.y));
                f.v[j][pr] = __fmul2_rn(uu, bc_pair<T>(wb[j], pi));
            }
        }
    };
    front(0, gt[0]);
#pragma unroll
    for (int k = 0; k < kGroups; ++k) {
        const int t = 4 * k;
        if (t % kTok == 0) {
#pragma unroll
            for (int j = 0; j < SPL; ++j) {
                const int o = bc_offset<T, SWZ>(nn[j], t / kTok);
                if (SS_IN_BOUNDS(o >= 0 && o + 16 <= N * S::kChunk * int(sizeof(T)), 113))
                    wc[j] = *reinterpret_cast<const uint4 *>(Ct + o);
            }
        }
        uint4 cc[SPL];
#pragma unroll
        for (int j = 0; j < SPL; ++j)
            cc[j] = wc[j];
        if (k + 1 < kGroups)
            front(k + 1, gt[(k + 1) & 1]);
        const GroupTerms<SPL> &f = gt[k & 1];
        float2 yo[2];
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
            const int pi = (t % kTok) / 2 + pr;
            float hm[SPL]; // the states after token t + 2 pr (hs: after the next token)
#pragma unroll
            for (int j = 0; j < SPL; ++j) {
                hm[j] = fmaf(f.a[j][pr].x, hs[j], f.v[j][pr].x);
                hs[j] = fmaf(f.a[j][pr].y, hm[j], f.v[j][pr].y);
            }
            float2 yy = __fmul2_rn(bc_pair<T>(cc[0], pi), make_float2(hm[0], hs[0]));
#pragma unroll
            for (int j = 1; j < SPL; ++j)
                yy = __ffma2_rn(bc_pair<T>(cc[j], pi), make_float2(hm[j], hs[j]), yy);
            yo[pr] = yy;
            if (EMIT == 1) {
                const int tt = t + 2 * pr;
#pragma unroll
                for (int j = 0; j < SPL; ++j) {
                    if (tt < valid)
                        __stcs(hrow + tt * N + nn[j], hm[j]);
                    if (tt + 1 < valid)
                        __stcs(hrow + (tt + 1) * N + nn[j], hs[j]);
                }
            }
        }
        *reinterpret_cast<float4 *>(ys + t) = make_float4(yo[0].x, yo[0].y, yo[1].x, yo[1].y);
    }
}

// The issuer warp (one lane works): takes work units, writes one chunk descriptor per
// raw-ring slot as far ahead as the ring allows and, on the TMA path (VEC), starts the
// chunk's 2-D tile loads of x, dt, z, B and C into the slot.  Every lane returns
// normally, so the warp reaches the kernel's end-of-call accounting as a whole.
template <int N, int SPL, typename T, bool VEC>
__device__ __forceinline__ bool issuer_warp(const ScanArgs &p, const TmaMaps &maps, const CtaCtx &cx, int lane)
{
    using S = ScanShape<N, SPL>;
    constexpr int RS = S::kRawStages;
    if (lane != 0)
        return true;
    if constexpr (VEC) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.dt)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.B)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.C)) : "memory");
        if (p.z)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.z)) : "memory");
    }
    constexpr uint32_t tx_bytes = uint32_t((2 * S::kChanPerCta + 2 * N) * S::kChunk * sizeof(T));
    uint32_t u = take_unit(p, cx.ws, true);
    UnitPos up;
    if (u != kNoUnit)
        up = unit_pos<N, SPL>(p, u);
    int64_t k = 0;
    for (uint32_t j = 0;; ++j) {
        const int r = int(j % RS);
        if (j >= uint32_t(RS) && !mbar_wait(cx.raw_empty + r, ((j / RS) & 1u) ^ 1u, cx.status)) {
            // the converters gave up: let the loads still in flight land, then leave
            for (uint32_t c = j > uint32_t(RS) ? j - RS : 0; c < j; ++c)
                mbar_wait(cx.raw_full + c % RS, (c / RS) & 1u, nullptr);
            return false;
        }
        int64_t *m = cx.raw_meta + 3 * r;
        if (u == kNoUnit) {
            m[2] = int64_t(kEnd) << 32;
            mbar_arrive(cx.raw_full + r);
            return true;
        }
        const int64_t t0 = up.t_begin + k * S::kChunk;
        const int32_t fl = (k == 0 ? kFirst : 0) | (k + 1 == up.nck ? kLast : 0);
        m[0] = t0;
        m[1] = up.g;
        m[2] = (int64_t(fl) << 32) | int64_t(up.s);
        if constexpr (VEC) {
            unsigned char *dst = cx.raw_base + r * S::template raw_stage_bytes<T>();
            uint64_t *bar = cx.raw_full + r;
            mbar_arrive_expect_tx(bar, tx_bytes);
            const int32_t tt = int32_t(t0), xrow = up.xrow, brow = up.brow;
            (void)SS_IN_BOUNDS(t0 < p.seq && int64_t(xrow) < p.batch * p.channels &&
                                   int64_t(brow) + N <= p.batch * N && r < S::kRawStages,
                               140);
            tma_load_2d(dst + S::template raw_x_off<T>(), &maps.x, tt, xrow, bar);
            tma_load_2d(dst + S::template raw_dt_off<T>(), &maps.dt, tt, xrow, bar);
            tma_load_2d(dst + S::template raw_b_off<T>(), &maps.B, tt, brow, bar);
            tma_load_2d(dst + S::template raw_c_off<T>(), &maps.C, tt, brow, bar);
            if (p.z && p.pass != 1) // the epilogue's z, from HBM into L2 ahead of time
                tma_prefetch_l2_2d(&maps.z, tt, xrow);
        } else {
            mbar_arrive(cx.raw_full + r);
        }
        if (++k == up.nck) {
            u = take_unit(p, cx.ws, false);
            k = 0;
            if (u != kNoUnit)
                up = unit_pos<N, SPL>(p, u);
        }
    }
}

// The two producer warps: each thread converts its share of every chunk (from the
// raw slot, or straight from global memory on the ragged path) into the input stage.
template <int N, int SPL, typename T, bool HAS_RESET, bool VEC, bool CONV, int EMIT>
__device__ __forceinline__ bool producer(const ScanArgs &p, const CtaCtx &cx, int pi, int lane)
{
    using S = ScanShape<N, SPL>;
    constexpr int RS = S::kRawStages;
    constexpr int kRawBytes = S::template raw_stage_bytes<T>();
    const int tl = pi * 32 + lane; // producer thread index
    IoPrefetch<N, SPL, T, HAS_RESET, VEC, CONV> pf;
    int64_t reset_g = -1;
    const uint8_t *reset_row = p.reset;
    for (uint32_t i = 0;; ++i) {
        const int r = int(i % RS);
        if (!mbar_wait(cx.raw_full + r, (i / RS) & 1u, cx.status))
            return false;
        const int64_t *m = cx.raw_meta + 3 * r;
        const int64_t t0 = m[0], g = m[1];
        const int32_t s = int32_t(m[2] & 0xffffffff), fl = int32_t(m[2] >> 32);
        const bool end = (fl & kEnd) != 0;
        if (!end) {
            if constexpr (VEC)
                pf.load_smem(p, tl, g, cx.raw_base + r * kRawBytes, t0);
            else
                pf.load(p, tl, g, t0);
            if (HAS_RESET) {
                if (g != reset_g) { // the reset row of the batch entry, once per unit
                    reset_g = g;
                    reset_row = p.reset + int64_t(uint32_t(g) / uint32_t(p.groups_per_batch)) * p.seq;
                }
                pf.rbyte = (tl < S::kChunk && t0 + tl < p.seq &&
                            SS_IN_BOUNDS(uint32_t(g) / uint32_t(p.groups_per_batch) < uint64_t(p.batch), 122))
                               ? uint32_t(__ldg(reset_row + t0 + tl))
                               : 0u;
            }
        }
        mbar_arrive(cx.raw_empty + r); // this thread's reads of slot r are done
        const int st = int(i % S::kStages);
        // the input stage is free once the scan warps are done with chunk i - kStages
        if (!mbar_wait(cx.in_empty + st, ((i / S::kStages) & 1u) ^ 1u, cx.status))
            return false;
        float *stage = cx.in_base + st * S::kInStage;
        // The chunk's output stage must be free as well (the epilogue is done with
        // chunk i - kYStages).  Waiting for it here, and for the raw slot above, makes
        // in_full the one barrier the scan warps wait on per chunk: a satisfied wait
        // still costs on the order of a hundred cycles, on the critical warps.  (The
        // fused conv form writes x into the output stage, so it waits first.)
        const int ys = int(i % S::kYStages);
        float *ystage = cx.y_base + ys * S::template y_stage<T>();
        if (CONV && !mbar_wait(cx.y_empty + ys, ((i / S::kYStages) & 1u) ^ 1u, cx.status))
            return false;
        if (!end)
            produce_chunk<N, SPL, T, HAS_RESET, VEC, CONV, EMIT>(p, tl, pf, stage, cx.raw_base + r * kRawBytes, t0, g,
                                                                 ystage);
        if (tl == 0)
            write_meta(stage, t0, g, s, fl);
        if (!CONV && !mbar_wait(cx.y_empty + ys, ((i / S::kYStages) & 1u) ^ 1u, cx.status))
            return false;
        if (tl == 0) // the epilogue warps learn the chunk from its output stage
            write_meta(ystage, t0, g, s, fl);
        mbar_arrive(cx.in_full + st);
        if (end)
            return true;
    }
}

// The two epilogue warps: partial outputs of each chunk -> y.  False on a timeout.
template <int N, int SPL, typename T, bool VEC, bool CONV>
__device__ __forceinline__ bool epilogue_role(const ScanArgs &p, const float *y_base, uint64_t *y_full,
                                              uint64_t *y_empty, uint32_t *status, int tl)
{
    using S = ScanShape<N, SPL>;
    EpiCache<N, SPL, T> ec;
    for (uint32_t j = 0;; ++j) {
        const int ys = int(j % S::kYStages);
        if (!mbar_wait(y_full + ys, (j / S::kYStages) & 1u, status))
            return false;
        const float *ystage = y_base + ys * S::template y_stage<T>();
        const ChunkMeta meta = read_meta(ystage);
        if (meta.flags & kEnd)
            return true;
        if (p.pass != 1) // (the first pass of the two-level scan has no outputs)
            epilogue_chunk<N, SPL, T, VEC, CONV>(p, tl, ystage, meta.g, meta.t0, ec);
        mbar_arrive(y_empty + ys);
    }
}

// ---------------------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------------------

// CTAs per SM to plan registers for: the states and conv forms need more registers
// than the plain form and are bounded to two CTAs per SM wherever shared memory fits
// two (about 113 KB each); the plain form gets there at its natural allocation.
template <int N, int SPL, typename T, int EMIT, bool CONV> constexpr int scan_min_ctas()
{
    return (EMIT != 0 || CONV) && ScanShape<N, SPL>::template smem_bytes<T, true>() <= 113 * 1024 ? 2 : 1;
}

template <int N, int SPL, typename T, bool HAS_RESET, bool VEC, int EMIT, bool CONV>
__global__ void __launch_bounds__(ScanShape<N, SPL>::kThreads, (scan_min_ctas<N, SPL, T, EMIT, CONV>()))
ss_scan_fwd_kernel(const ScanArgs p, const __grid_constant__ TmaMaps maps)
{
    using S = ScanShape<N, SPL>;
    constexpr int kRawRing = S::kRawStages * S::template raw_stage_bytes<T>();
    extern __shared__ __align__(1024) unsigned char smem_bytes[];
    float *const in_base = reinterpret_cast<float *>(smem_bytes + kRawRing);
    float *const y_base = in_base + S::kStages * S::kInStage;
    uint64_t *const bars = reinterpret_cast<uint64_t *>(in_base + S::template floats<T>());
    uint64_t *const in_full = bars + S::kBarInFull, *const in_empty = bars + S::kBarInEmpty;
    uint64_t *const y_full = bars + S::kBarYFull, *const y_empty = bars + S::kBarYEmpty;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    WsHeader *const ws = reinterpret_cast<WsHeader *>(p.workspace);
    const bool chained = ws != nullptr;
    uint32_t *const status = chained ? &ws->status : p.status;
    const uint64_t epoch = chained ? *reinterpret_cast<volatile uint64_t *>(&ws->epoch) : 0u;
    uint64_t *const flags = chained ? reinterpret_cast<uint64_t *>(p.workspace + sizeof(WsHeader)) : nullptr;
    // carries: SPL floats per lane and (channel group, scan warp) slot
    float *const carry = chained
        ? reinterpret_cast<float *>(p.workspace + sizeof(WsHeader) + 8 * p.groups * S::kScanWarps)
        : nullptr;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S::kStages; ++s) {
            mbar_init(in_full + s, S::kIoThreads);          // the producer warps
            mbar_init(in_empty + s, 32 * S::kScanWarps);
        }
        for (int s = 0; s < S::kYStages; ++s) {
            mbar_init(y_full + s, 32 * S::kScanWarps);
            mbar_init(y_empty + s, S::kIoThreads);          // the epilogue warps
        }
        for (int r = 0; r < S::kRawStages; ++r) {
            mbar_init(bars + S::kBarRawFull + r, 1);              // the issuer
            mbar_init(bars + S::kBarRawEmpty + r, S::kIoThreads + 32 * S::kScanWarps); // producers, scan
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp >= S::kScanWarps) {
        // ============================== IO warps ==============================
        CtaCtx cx;
        cx.in_base = in_base;
        cx.y_base = y_base;
        cx.raw_base = smem_bytes;
        cx.in_full = in_full;
        cx.in_empty = in_empty;
        cx.y_full = y_full;
        cx.y_empty = y_empty;
        cx.raw_full = bars + S::kBarRawFull;
        cx.raw_empty = bars + S::kBarRawEmpty;
        cx.raw_meta = reinterpret_cast<int64_t *>(bars + S::kBars);
        cx.ws = ws;
        cx.status = status;
        // IO role of this warp and its index within the role: with two warps per role
        // they alternate (sub-partitions 0 and 2 produce, 1 and 3 finish outputs), with
        // four per role each role takes four consecutive warps (one per sub-partition)
        const int io = warp - S::kScanWarps;
        const bool prod = S::kIoWarps == 4 ? io < 4 : (io & 1) == 0;
        const int ri = S::kIoWarps == 4 ? (io & 3) : (io >> 1);
        bool ok;
        if (warp == S::kIssuerWarp)
            ok = issuer_warp<N, SPL, T, VEC>(p, maps, cx, lane);
        else if (prod)
            ok = producer<N, SPL, T, HAS_RESET, VEC, CONV, EMIT>(p, cx, ri, lane);
        else
            ok = epilogue_role<N, SPL, T, VEC, CONV>(p, y_base, y_full, y_empty, status, ri * 32 + lane);
        (void)ok; // false: gave up on a wait (SS_ERR_TIMEOUT recorded); counted out below
    } else {
        // =============================== scan warps ==============================
        const int cw = lane / S::kLanes;    // channel within the warp
        const int sub = lane % S::kLanes;   // state group within the channel
        // the lane's states (the same lane-to-state map in every form of this layout, so
        // outputs are bit-identical across the plain, states and segmented forms)
        int nn[SPL];
#pragma unroll
        for (int j = 0; j < SPL; ++j)
            nn[j] = S::template state<T>(sub, j);
        const int cl = warp * S::kChanPerWarp + cw;  // channel within the CTA
        float hs[SPL];
        float2 A2[SPL];
#pragma unroll
        for (int j = 0; j < SPL; ++j) {
            hs[j] = 0.0f;
            A2[j] = make_float2(0.f, 0.f);
        }
        int64_t row = 0;
        bool cvalid = false;
        for (uint32_t j = 0;; ++j) {
            const int st = int(j % S::kStages);
            if (!mbar_wait(in_full + st, (j / S::kStages) & 1u, status))
                break; // timeout recorded; counted out below
            // (in_full also means: the chunk's raw slot has landed and its output
            // stage is free -- the producers waited for both before arriving)
            const float *stage = in_base + st * S::kInStage;
            const ChunkMeta meta = read_meta(stage);
            const uint32_t ysi = j % S::kYStages;
            if (meta.flags & kEnd) {
                mbar_arrive(y_full + ysi); // lets the epilogue warp see the end marker
                break;
            }
            if (meta.flags & kFirst) {
                if (!SS_IN_BOUNDS(meta.g < p.groups && meta.s < p.segments && meta.t0 < p.seq, 101))
                    break;
                const int64_t b = meta.g / p.groups_per_batch;
                const int64_t c_raw = (meta.g % p.groups_per_batch) * S::kChanPerCta + cl;
                cvalid = c_raw < p.channels;
                const int64_t c = cvalid ? c_raw : p.channels - 1;
                row = b * p.channels + c;
                if (!SS_IN_BOUNDS(c < p.channels && row < p.batch * p.channels && nn[SPL - 1] < N, 109))
                    break;
#pragma unroll
                for (int q = 0; q < SPL; ++q) {
                    const float a = __ldg(p.A + c * N + nn[q]) * kLog2e;
                    A2[q] = make_float2(a, a);
                }
                if (p.pass == 1) {
#pragma unroll
                    for (int q = 0; q < SPL; ++q)
                        hs[q] = 0.0f;
                } else if (p.pass == 2) {
                    if (!SS_IN_BOUNDS(p.seg_stride >= p.batch * p.channels * N, 107))
                        break;
                    const float *src = p.seg_in + meta.s * p.seg_stride + row * N;
#pragma unroll
                    for (int q = 0; q < SPL; ++q)
                        hs[q] = __ldcg(src + nn[q]);
                } else if (meta.s == 0) {
#pragma unroll
                    for (int q = 0; q < SPL; ++q)
                        hs[q] = p.h0 ? __ldg(p.h0 + row * N + nn[q]) : 0.0f;
                } else {
                    const int64_t slot = meta.g * S::kScanWarps + warp;
                    if (!SS_IN_BOUNDS(slot < p.groups * S::kScanWarps, 103))
                        break;
                    const uint64_t want = carry_tag(epoch, meta.s);
                    if (!flag_wait(flags + slot, want, status))
                        break; // timeout recorded; counted out below
                    const float *cs = carry + (slot * 32 + lane) * SPL;
#pragma unroll
                    for (int q = 0; q < SPL; ++q)
                        hs[q] = __ldcg(cs + q);
                }
            }
            const int rs = int(j % S::kRawStages);
            float *hrow = nullptr;
            if (EMIT == 1 && p.h_all) {
                if (!SS_IN_BOUNDS(row < p.batch * p.channels && meta.t0 < p.seq, 110))
                    break;
                hrow = p.h_all + (row * p.seq + meta.t0) * N;
            }
            scan_chunk<N, SPL, T, HAS_RESET, EMIT>(stage, smem_bytes + rs * S::template raw_stage_bytes<T>(),
                                                   y_base + ysi * S::template y_stage<T>() + S::kYPOff +
                                                       cl * S::kYChan + sub * S::kRow,
                                                   cl, nn, A2, hs, hrow,
                                                   (cvalid && hrow) ? p.seq - meta.t0 : int64_t(0));
            mbar_arrive(bars + S::kBarRawEmpty + rs);
            mbar_arrive(in_empty + st);
            mbar_arrive(y_full + ysi);
            if (meta.flags & kLast) {
                if (p.pass == 1) {
                    if (cvalid && SS_IN_BOUNDS(p.seg_stride >= p.batch * p.channels * N, 106)) {
                        float *dst = p.seg_state + meta.s * p.seg_stride + row * N;
#pragma unroll
                        for (int q = 0; q < SPL; ++q)
                            __stcg(dst + nn[q], hs[q]);
                    }
                } else if (p.pass == 2) {
                    // the final state was produced by the join
                } else if (int64_t(meta.s) + 1 < p.segments) {
                    const int64_t slot = meta.g * S::kScanWarps + warp;
                    if (!SS_IN_BOUNDS(slot < p.groups * S::kScanWarps, 104))
                        continue;
                    float *cs = carry + (slot * 32 + lane) * SPL;
#pragma unroll
                    for (int q = 0; q < SPL; ++q)
                        __stcg(cs + q, hs[q]);
                    __threadfence();
                    __syncwarp();
                    if (lane == 0)
                        st_release_gpu(flags + slot, carry_tag(epoch, meta.s + 1));
                } else if (p.h_last && cvalid && SS_IN_BOUNDS(row < p.batch * p.channels, 105)) {
#pragma unroll
                    for (int q = 0; q < SPL; ++q)
                        p.h_last[row * N + nn[q]] = hs[q];
                }
            }
        }
    }

    // The last warp of a chained call to finish resets the work counter and advances
    // the epoch for the next call.  Each warp counts itself, so no CTA-wide barrier is
    // needed after the roles have diverged; a warp that gave up on a wait counts itself
    // too (every wait is bounded, so every warp gets here), so even a call that timed
    // out leaves the workspace ready: its carry flags hold the old epoch and can never
    // satisfy a later call's wait, and the status word says what happened.
    if (chained) {
        if (lane == 0) {
            __threadfence();
            const uint32_t done = atomicAdd(&ws->done, 1u);
            if (done + 1 == gridDim.x * uint32_t(S::kWarps)) {
                ws->done = 0;
                ws->counter = 0;
                __threadfence();
                atomicAdd(reinterpret_cast<unsigned long long *>(&ws->epoch), 1ull);
            }
        }
    }
}

// Bytes of workspace a chained call needs for `groups` channel groups.
template <int N, int SPL> constexpr int64_t scan_workspace_bytes(int64_t groups)
{
    return int64_t(sizeof(WsHeader)) + groups * ScanShape<N, SPL>::kScanWarps * (8 + 32 * SPL * 4);
}

} // namespace ss
