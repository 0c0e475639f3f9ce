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
    static __device__ __forceinline__ float4 load_smem(const float *p) { return *reinterpret_cast<const float4 *>(p); }
    static __device__ __forceinline__ float4 load(const float *p, bool vec)
    {
        if (vec)
            return __ldg(reinterpret_cast<const float4 *>(p));
        return make_float4(__ldg(p), __ldg(p + 1), __ldg(p + 2), __ldg(p + 3));
    }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load_smem(const __nv_bfloat16 *p)
    {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
    }
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
        s[it] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (SS_IN_BOUNDS(b < p.batch && chan(it) < p.channels, 210))
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
        if (valid && SS_IN_BOUNDS(row < p.batch * p.channels, 211)) {
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
// ring of shared-memory stages filled by bulk asynchronous copies (no multicast), so
// kDecStages tiles of every CTA are always on their way regardless of the registers
// the arithmetic needs.  A tile is 1024 row quarters (16 KB of state) of one batch
// row, plus -- when their rows are 16-byte aligned -- the tile's x, dt_raw and z and
// the row's B and C in the same stage, so a tile's arithmetic waits on nothing but
// its stage.  Thread t owns quarters t, t + 256, t + 512, t + 768 of a tile.
// When the grid is a multiple of the channel blocks per row, every CTA keeps one
// channel block and walks batch rows, so A, dt_bias and D are loaded once per CTA.
// One extra warp issues the copies: it refills a stage as soon as the eight consumer
// warps have each released it (an "empty" mbarrier per stage), so consumer warps never
// wait for one another.
// The updated state goes straight back to global memory with streaming stores.
constexpr int kDecThreads = 256;                          // consumer threads (8 warps)
constexpr int kDecBlock = kDecThreads + 32;               // + one copy-issuing warp
constexpr int kDecItems = 4;                              // quarters per thread per tile
constexpr int kDecQuarters = kDecThreads * kDecItems;     // 1024 quarters = 16 KB
constexpr int kDecStages = 4;
constexpr int kDecTileBytes = kDecQuarters * 16;

template <int N, typename T> struct DecShape {
    static constexpr int kQ = N / 4;                           // quarters per (b, c) row
    static constexpr int kChanPerTile = kDecQuarters / kQ;
    static constexpr int kVecBytes = kChanPerTile * int(sizeof(T)); // x, dt or z of a tile
    static constexpr int kBCOff = kDecTileBytes + 3 * kVecBytes;  // B then C of the row
    static constexpr int kStageBytes = kBCOff + 2 * 64;
    static constexpr size_t kSmem = size_t(kDecStages) * kStageBytes + 16 * kDecStages; // + full, empty
    // the fused conv form also copies the tile's conv-state rows (up to 3 inputs each)
    static constexpr int kCSOff = kStageBytes;
    static constexpr int kStageBytesConv = kCSOff + kChanPerTile * 3 * 4;
    template <bool CONV> static constexpr int stage_bytes() { return CONV ? kStageBytesConv : kStageBytes; }
    template <bool CONV> static constexpr size_t smem()
    {
        return size_t(kDecStages) * stage_bytes<CONV>() + 16 * kDecStages;
    }
    static_assert(kStageBytes % 16 == 0 && kStageBytesConv % 16 == 0, "16-byte aligned stages");
};

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

struct DecArgs {
    UpdateArgs u;
    int64_t ncb;     // channel blocks per batch row
    int fixed_cb;    // grid is a multiple of ncb: CTA i keeps channel block i % ncb
    int bulk_xdz;    // x, dt_raw (and z) rows are copied with the state
    int bulk_bc;     // B and C rows are copied with the state
    int bulk_cs;     // conv form: the tile's conv-state rows are copied with the state
    // conv form: x above is the conv input u; x = silu(conv_b + conv_w . [state, u])
    const float *conv_w, *conv_b; // [channels, conv_k], [channels] (nullable)
    float *conv_state;            // [batch, channels, conv_k - 1] in/out
    int conv_k;
};

// CONV: the decode step of the fused conv form -- x is silu of the causal conv over the
// row's conv state and the new input u, and the conv state shifts by one input.
template <int N, typename T, bool CONV>
__global__ void __launch_bounds__(kDecBlock, 2)
ss_state_update_stream_kernel(const DecArgs da, uint32_t *status)
{
    using D = DecShape<N, T>;
    constexpr int Q = D::kQ;
    constexpr int kStage = D::template stage_bytes<CONV>();
    const UpdateArgs &p = da.u;
    extern __shared__ __align__(128) unsigned char dsm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(dsm + size_t(kDecStages) * kStage);
    uint64_t *empty = full + kDecStages;
    const int tid = threadIdx.x, lane_q = tid & (Q - 1);

    // Tile k of this CTA is tile blockIdx.x + k * gridDim.x of the (batch row, channel
    // block) order; walked incrementally, without a division per tile.  (With fixed_cb
    // the grid is a multiple of the channel blocks, so the CTA keeps its channel block.)
    struct TileWalk {
        int64_t b, cb, db, dcb, ncb;
        __device__ __forceinline__ void start(int64_t n)
        {
            ncb = n;
            b = int64_t(blockIdx.x) / n;
            cb = int64_t(blockIdx.x) - b * n;
            db = int64_t(gridDim.x) / n;
            dcb = int64_t(gridDim.x) - db * n;
        }
        __device__ __forceinline__ void next()
        {
            b += db;
            cb += dcb;
            if (cb >= ncb) {
                cb -= ncb;
                ++b;
            }
        }
    };
    auto nchan = [&](int64_t cb) -> int64_t {
        const int64_t rest = p.channels - cb * D::kChanPerTile;
        return rest < D::kChanPerTile ? rest : D::kChanPerTile;
    };
    auto issue = [&](const TileWalk &w, int stage) -> bool {
        const int64_t b = w.b, cb = w.cb;
        if (b >= p.batch)
            return false;
        const int64_t nch = nchan(cb), row0 = b * p.channels + cb * D::kChanPerTile;
        const uint32_t sbytes = uint32_t(nch * N * 4), vbytes = uint32_t(nch * int64_t(sizeof(T)));
        const int nvec = da.bulk_xdz ? (p.z ? 3 : 2) : 0;
        const uint32_t bcbytes = da.bulk_bc ? uint32_t(2 * N * sizeof(T)) : 0u;
        // (bulk_cs: channels % 4 == 0, so row0 * H * 4 and nch * H * 4 are multiples of 16)
        const uint32_t csbytes = (CONV && da.bulk_cs) ? uint32_t(nch * (da.conv_k - 1) * 4) : 0u;
        unsigned char *dst = dsm + size_t(stage) * kStage;
        if (!SS_IN_BOUNDS(b < p.batch && nch > 0 && row0 + nch <= p.batch * p.channels && stage < kDecStages &&
                              nch * N * 4 <= kDecTileBytes,
                          202))
            return false;
        mbar_arrive_expect_tx(full + stage, sbytes + nvec * vbytes + bcbytes + csbytes);
        bulk_load(dst, p.state + row0 * N, sbytes, full + stage);
        if (nvec) {
            bulk_load(dst + kDecTileBytes, static_cast<const T *>(p.x) + row0, vbytes, full + stage);
            bulk_load(dst + kDecTileBytes + D::kVecBytes, static_cast<const T *>(p.dt) + row0, vbytes, full + stage);
            if (p.z)
                bulk_load(dst + kDecTileBytes + 2 * D::kVecBytes, static_cast<const T *>(p.z) + row0, vbytes,
                          full + stage);
        }
        if (bcbytes) {
            bulk_load(dst + D::kBCOff, static_cast<const T *>(p.B) + b * N, bcbytes / 2, full + stage);
            bulk_load(dst + D::kBCOff + 64, static_cast<const T *>(p.C) + b * N, bcbytes / 2, full + stage);
        }
        if (csbytes)
            bulk_load(dst + D::kCSOff, da.conv_state + row0 * (da.conv_k - 1), csbytes, full + stage);
        return true;
    };

    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, kDecThreads / 32); // one arrival per consumer warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid >= kDecThreads) {
        // the copy-issuing warp: tile k goes into stage k % kDecStages once the
        // consumers have released tile k - kDecStages
        if (tid == kDecThreads) {
            TileWalk w;
            w.start(da.ncb);
            for (int64_t k = 0;; ++k, w.next()) {
                const int s = int(k % kDecStages);
                if (k >= kDecStages &&
                    !mbar_wait(empty + s, (uint32_t(k / kDecStages) & 1u) ^ 1u, status)) {
                    // the consumers gave up (SS_ERR_TIMEOUT recorded): let the copies
                    // still in flight land, then leave
                    for (int64_t j = k - kDecStages + 1; j < k; ++j)
                        mbar_wait(full + int(j % kDecStages), uint32_t(j / kDecStages) & 1u, nullptr);
                    break;
                }
                if (!issue(w, s))
                    break;
            }
        }
        return;
    }

    float4 av[kDecItems];
    float bias[kDecItems], dco[kDecItems];
    // conv taps of the items this lane evaluates (item v * Q + lane_q, see below):
    // cs_w[e] multiplies conv-state entry e (the input H - e back; 0 for e >= H), cu_w
    // the new input u.  Every index is a compile-time constant, so they stay in registers.
    constexpr int kMine = CONV ? kDecItems / Q : 1;
    float cs_w[kMine][3], cu_w[kMine], cbi[kMine];
    const int H = CONV ? da.conv_k - 1 : 0;
    int64_t cached_cb = -1;
    bool ok = true;
    TileWalk w;
    w.start(da.ncb);
    for (int64_t k = 0;; ++k, w.next()) {
        const int64_t b = w.b, cb = w.cb;
        if (b >= p.batch)
            break;
        const int64_t c0 = cb * D::kChanPerTile;
        const int nq = int(nchan(cb) * Q); // valid quarters in this tile
        if (!SS_IN_BOUNDS(cb < da.ncb && nq > 0 && nq <= kDecQuarters, 201)) {
            ok = false;
            break;
        }
        if (cb != cached_cb) {
            cached_cb = cb;
#pragma unroll
            for (int it = 0; it < kDecItems; ++it) {
                const int q = tid + it * kDecThreads;
                const int64_t c = c0 + (q < nq ? q : nq - 1) / Q;
                av[it] = __ldg(reinterpret_cast<const float4 *>(p.A + c * N) + lane_q);
                bias[it] = p.dt_bias ? __ldg(p.dt_bias + c) : 0.0f;
                dco[it] = p.D ? __ldg(p.D + c) : 0.0f;
            }
            if constexpr (CONV) {
                // tap k of a row multiplies the input K-1-k back: taps 0..H-1 the conv
                // state (oldest first), tap H = K-1 the new input
#pragma unroll
                for (int v = 0; v < kMine; ++v) {
                    const int q = tid + (v * Q + lane_q) * kDecThreads;
                    const int64_t c = c0 + (q < nq ? q : nq - 1) / Q;
#pragma unroll
                    for (int e = 0; e < 3; ++e)
                        cs_w[v][e] = e < H ? __ldg(da.conv_w + c * da.conv_k + e) : 0.0f;
                    cu_w[v] = __ldg(da.conv_w + c * da.conv_k + H);
                    cbi[v] = da.conv_b ? __ldg(da.conv_b + c) : 0.0f;
                }
            }
        }
        // the conv state of each item's row (read by the row's lanes before its first
        // lane writes the shifted state back, below)
        // conv form: each lane evaluates, and shifts the conv state of, its own items
        // (item v * Q + lane_q of its row group for v < kMine): their state rows only
        float csm[kMine][3];
        int own_cl[kMine];
        if constexpr (CONV) {
#pragma unroll
            for (int v = 0; v < kMine; ++v) {
                const int q = tid + (v * Q + lane_q) * kDecThreads;
                own_cl[v] = (q < nq ? q : nq - 1) / Q;
                if (!da.bulk_cs) {
                    const int64_t row = b * p.channels + c0 + own_cl[v];
#pragma unroll
                    for (int j = 0; j < 3; ++j)
                        csm[v][j] = j < H ? __ldg(da.conv_state + row * H + j) : 0.0f;
                }
            }
        }
        // the small operands first: their latency overlaps the wait for the state
        float4 bv = make_float4(0.f, 0.f, 0.f, 0.f), cv = bv;
        if (!da.bulk_bc) {
            bv = Vec4<T>::load(static_cast<const T *>(p.B) + b * N + 4 * lane_q, true);
            cv = Vec4<T>::load(static_cast<const T *>(p.C) + b * N + 4 * lane_q, true);
        }
        float xs[kDecItems], ds[kDecItems], zs[kDecItems];
        if (!da.bulk_xdz) {
#pragma unroll
            for (int it = 0; it < kDecItems; ++it) {
                const int q = tid + it * kDecThreads;
                const int64_t row = b * p.channels + c0 + (q < nq ? q : nq - 1) / Q;
                xs[it] = Elem<T>::load(static_cast<const T *>(p.x) + row);
                ds[it] = Elem<T>::load(static_cast<const T *>(p.dt) + row);
                zs[it] = p.z ? Elem<T>::load(static_cast<const T *>(p.z) + row) : 0.0f;
            }
        }
        const int stage = int(k % kDecStages);
        if (!mbar_wait(full + stage, uint32_t(k / kDecStages) & 1u, status)) {
            ok = false;
            break;
        }
        const unsigned char *sb = dsm + size_t(stage) * kStage;
        const float4 *sv = reinterpret_cast<const float4 *>(sb);
        if (da.bulk_bc) {
            bv = Vec4<T>::load_smem(reinterpret_cast<const T *>(sb + D::kBCOff) + 4 * lane_q);
            cv = Vec4<T>::load_smem(reinterpret_cast<const T *>(sb + D::kBCOff + 64) + 4 * lane_q);
        }
        if (da.bulk_xdz) {
            const T *sx = reinterpret_cast<const T *>(sb + kDecTileBytes);
            const T *sd = reinterpret_cast<const T *>(sb + kDecTileBytes + D::kVecBytes);
            const T *sz = reinterpret_cast<const T *>(sb + kDecTileBytes + 2 * D::kVecBytes);
#pragma unroll
            for (int it = 0; it < kDecItems; ++it) {
                const int q = tid + it * kDecThreads;
                const int cl = (q < nq ? q : nq - 1) / Q;
                xs[it] = Elem<T>::load_smem(sx + cl);
                ds[it] = Elem<T>::load_smem(sd + cl);
                zs[it] = p.z ? Elem<T>::load_smem(sz + cl) : 0.0f;
            }
        }
        if constexpr (CONV) {
            if (da.bulk_cs) { // the conv state arrived with the tile
                const float *scs = reinterpret_cast<const float *>(sb + D::kCSOff);
#pragma unroll
                for (int v = 0; v < kMine; ++v)
#pragma unroll
                    for (int j = 0; j < 3; ++j)
                        csm[v][j] = j < H ? scs[own_cl[v] * H + j] : 0.0f;
            }
        }
        if constexpr (CONV) {
            // x = silu(conv over [state, u]); xs held u until here.  The Q lanes of a row
            // share each item's x: lane j evaluates the items it with it % Q == j and the
            // row's lanes exchange (as for the softplus below)
            float xm[kMine];
#pragma unroll
            for (int v = 0; v < kMine; ++v) {
                // this lane's item v * Q + lane_q: its input, selected with compile-time
                // indices
                float uu = xs[v * Q];
#pragma unroll
                for (int j = 1; j < Q; ++j)
                    if (lane_q == j)
                        uu = xs[v * Q + j];
                float a = fmaf(cu_w[v], uu, cbi[v]); // entries e >= H hold 0, and so do their taps
                a = fmaf(cs_w[v][0], csm[v][0], a);
                a = fmaf(cs_w[v][1], csm[v][1], a);
                a = fmaf(cs_w[v][2], csm[v][2], a);
                xm[v] = silu(a);
                // the row's conv state shifts by one input: drop the oldest, append u
                // (only this lane reads or writes this row's conv state)
                const int q = tid + (v * Q + lane_q) * kDecThreads;
                if (q < nq && H > 0 && SS_IN_BOUNDS(c0 + own_cl[v] < p.channels, 207)) {
                    float *csr = da.conv_state + (b * p.channels + c0 + own_cl[v]) * H;
#pragma unroll
                    for (int j = 0; j < 3; ++j)
                        if (j < H)
                            csr[j] = j + 1 < H ? csm[v][j + 1 < 3 ? j + 1 : 0] : uu;
                }
            }
            const int xbase = (tid & 31) & ~(Q - 1);
#pragma unroll
            for (int it = 0; it < kDecItems; ++it)
                xs[it] = Q == 1 ? xm[it] : __shfl_sync(0xffffffffu, xm[it / Q], xbase | (it % Q));
        }
        // dt of the four items: the Q lanes of a row share them, so lane j computes
        // the softplus of the items it with it % Q == j and the row's lanes exchange
        float dsp[kDecItems];
        if (p.softplus) {
            float mine[kDecItems / Q];
#pragma unroll
            for (int u = 0; u < kDecItems / Q; ++u) {
                float r = ds[u * Q] + bias[u * Q];
#pragma unroll
                for (int j = 1; j < Q; ++j)
                    r = lane_q == j ? ds[u * Q + j] + bias[u * Q + j] : r;
                mine[u] = softplus(r);
            }
            const int base = (tid & 31) & ~(Q - 1);
#pragma unroll
            for (int it = 0; it < kDecItems; ++it)
                dsp[it] = Q == 1 ? mine[it] : __shfl_sync(0xffffffffu, mine[it / Q], base | (it % Q));
        } else {
#pragma unroll
            for (int it = 0; it < kDecItems; ++it)
                dsp[it] = ds[it] + bias[it];
        }
        // the tile's rows start at row0: item it of this thread is quarter
        // q = tid + it * kDecThreads, i.e. float4 q of the tile's state and row q / Q
        const int64_t row0 = b * p.channels + c0;
        float4 *const st_tile = reinterpret_cast<float4 *>(p.state) + row0 * Q;
        float ysum[kDecItems];
#pragma unroll
        for (int it = 0; it < kDecItems; ++it) {
            const int q = tid + it * kDecThreads;
            const bool valid = q < nq;
            float4 st = sv[valid ? q : nq - 1];
            const float d = dsp[it];
            const float dx = d * xs[it];
            const float dl = d * kLog2e;
            st.x = fmaf(ex2(dl * av[it].x), st.x, dx * bv.x);
            st.y = fmaf(ex2(dl * av[it].y), st.y, dx * bv.y);
            st.z = fmaf(ex2(dl * av[it].z), st.z, dx * bv.z);
            st.w = fmaf(ex2(dl * av[it].w), st.w, dx * bv.w);
            float yp = cv.x * st.x;
            yp = fmaf(cv.y, st.y, yp);
            yp = fmaf(cv.z, st.z, yp);
            yp = fmaf(cv.w, st.w, yp);
#pragma unroll
            for (int off = Q / 2; off >= 1; off >>= 1)
                yp += __shfl_xor_sync(0xffffffffu, yp, off);
            ysum[it] = yp; // (every lane of the row holds the row's sum)
            if (valid && SS_IN_BOUNDS(c0 + q / Q < p.channels && b < p.batch, 204))
                __stcs(st_tile + q, st);
        }
        // y of the items' rows: the Q lanes of a row finish one item each in turn (lane
        // j the items it with it % Q == j), instead of one lane finishing them all
#pragma unroll
        for (int m = 0; m < kDecItems / Q; ++m) {
            float yv = ysum[m * Q], xv = xs[m * Q], zv = zs[m * Q], dv = dco[m * Q];
#pragma unroll
            for (int j = 1; j < Q; ++j)
                if (lane_q == j) {
                    yv = ysum[m * Q + j];
                    xv = xs[m * Q + j];
                    zv = zs[m * Q + j];
                    dv = dco[m * Q + j];
                }
            const int q = tid + (m * Q + lane_q) * kDecThreads;
            if (q < nq && SS_IN_BOUNDS(c0 + q / Q < p.channels && b < p.batch, 208)) {
                float v = fmaf(dv, xv, yv);
                if (p.z)
                    v *= silu(zv);
                Elem<T>::store(static_cast<T *>(p.y) + row0 + q / Q, v);
            }
        }
        // this warp is done reading the stage
        __syncwarp();
        if ((tid & 31) == 0)
            mbar_arrive(empty + stage);
    }
    (void)ok;
}

} // namespace ss
