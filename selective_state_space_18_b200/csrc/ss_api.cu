// ss_api.cu -- the C ABI of libssscan.so (declarations and contracts: ss_scan.h).
//
// Host-side validation, dispatch on (state_dim, dtype, reset present, vector path)
// and launch on the caller's stream.  No allocation, no synchronisation.
#include "ss_scan.h"

#include <atomic>
#include <type_traits>
#include <cstring>
#include <cstdint>
#include <cudaTypedefs.h> // PFN_cuTensorMapEncodeTiled

#include "ss_scan_fwd.cuh"
#include "ss_state_update.cuh"
#include "ss_gated_scan.cuh"
#include "ss_gated_tc.cuh"
#include "ss_segment.cuh"

namespace {

constexpr int kAbiMajor = 3, kAbiMinor = 0;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// [p, p + n) and [q, q + m) intersect (NULL or empty ranges never do).
bool overlaps(const void *p, size_t n, const void *q, size_t m)
{
    if (!p || !q || n == 0 || m == 0)
        return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + m && b < a + n;
}

bool mul_ok(int64_t a, int64_t b, int64_t *out) { return !__builtin_mul_overflow(a, b, out); }

// Raise the dynamic shared-memory limit of a kernel once per device; `done_mask`
// is owned by the caller's kernel instantiation.
template <typename K> int ensure_smem(K kernel, size_t bytes, std::atomic<uint64_t> &done_mask)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return SS_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (bit && (done_mask.load(std::memory_order_acquire) & bit))
        return SS_OK;
    if (bytes > 48 * 1024 &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) != cudaSuccess)
        return SS_ERR_CUDA;
    done_mask.fetch_or(bit, std::memory_order_acq_rel);
    return SS_OK;
}

int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

// Status word of calls made without a workspace (one per device that loads the
// library); read and cleared by ss_scan_status(NULL, ...).
__device__ uint32_t g_ss_status_word;

int status_word_address(uint32_t **out)
{
    static std::atomic<uintptr_t> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return SS_ERR_CUDA;
    if (dev < 64) {
        const uintptr_t v = cache[dev].load(std::memory_order_acquire);
        if (v) {
            *out = reinterpret_cast<uint32_t *>(v);
            return SS_OK;
        }
    }
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_ss_status_word) != cudaSuccess)
        return SS_ERR_CUDA;
    if (dev < 64)
        cache[dev].store(reinterpret_cast<uintptr_t>(ptr), std::memory_order_release);
    *out = static_cast<uint32_t *>(ptr);
    return SS_OK;
}

int device_sm_count(int *sms)
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return SS_ERR_CUDA;
    int v = dev < 64 ? cache[dev].load(std::memory_order_acquire) : 0;
    if (!v) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SS_ERR_CUDA;
        if (dev < 64)
            cache[dev].store(v, std::memory_order_release);
    }
    *sms = v;
    return SS_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled tensor_map_encoder()
{
    static std::atomic<void *> fn{nullptr};
    void *f = fn.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn.store(f, std::memory_order_release);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled>(f);
}

// 2-D map over `rows` rows of `inner` contiguous elements, box = chunk x box_rows.
template <typename T>
bool encode_rows(CUtensorMap *map, const void *base, int64_t inner, int64_t rows, uint32_t box_inner,
                 uint32_t box_rows, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE)
{
    PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
    if (!enc)
        return false;
    const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(inner) * sizeof(T)};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N, int SPL, typename T>
bool build_maps(const ss::ScanArgs &a, ss::TmaMaps *m)
{
    using S = ss::ScanShape<N, SPL>;
    const int64_t rows = a.batch * a.channels, brows = a.batch * N;
    // B and C tiles are read by the scan warps in place: their 16-byte chunks are
    // swizzled across the banks (the swizzle the layout's lane-to-state map needs)
    // (the kernel reads the tiles at a pitch of one row: the swizzle span must be that row)
    static_assert(S::kChunk * sizeof(T) == size_t(S::template swizzle<T>()), "swizzle span = tile row");
    const CUtensorMapSwizzle bc_swizzle =
        S::template swizzle<T>() == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    return encode_rows<T>(&m->x, a.x, a.seq, rows, S::kChunk, S::kChanPerCta) &&
           encode_rows<T>(&m->dt, a.dt, a.seq, rows, S::kChunk, S::kChanPerCta) &&
           (!a.z || encode_rows<T>(&m->z, a.z, a.seq, rows, S::kChunk, S::kChanPerCta)) &&
           encode_rows<T>(&m->B, a.B, a.seq, brows, S::kChunk, N, bc_swizzle) &&
           encode_rows<T>(&m->C, a.C, a.seq, brows, S::kChunk, N, bc_swizzle);
}

// Launch plan of the scan kernel instance <N, SPL, T, R, V, E, C> for the shape in `a`
// (groups, segments, segment length and grid filled in); also what ss_scan_plan
// reports.
template <int N, int SPL, typename T, bool R, bool V, int E, bool C>
int plan_scan(ss::ScanArgs &a, int64_t *grid_out, int *occ_out, int *sms_out)
{
    using S = ss::ScanShape<N, SPL>;
    constexpr size_t kSmem = S::template smem_bytes<T, V>();
    auto kernel = ss::ss_scan_fwd_kernel<N, SPL, T, R, V, E, C>;
    static std::atomic<uint64_t> smem_done{0};
    static std::atomic<int> occ_cache[64];
    a.groups_per_batch = (a.channels + S::kChanPerCta - 1) / S::kChanPerCta;
    if (!mul_ok(a.batch, a.groups_per_batch, &a.groups) || a.groups > 0x7fffffffLL)
        return SS_ERR_SHAPE;
    int st = ensure_smem(kernel, kSmem, smem_done);
    if (st != SS_OK)
        return st;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || device_sm_count(&sms) != SS_OK)
        return SS_ERR_CUDA;
    int occ = dev < 64 ? occ_cache[dev].load(std::memory_order_acquire) : 0;
    if (!occ) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, S::kThreads, kSmem) != cudaSuccess)
            return SS_ERR_CUDA;
        occ = occ > 0 ? occ : 1;
        if (dev < 64)
            occ_cache[dev].store(occ, std::memory_order_release);
    }
    *occ_out = occ;
    *sms_out = sms;
    const int64_t nchunks = (a.seq + S::kChunk - 1) / S::kChunk;
    int64_t grid = a.groups;
    if (a.pass != 0) {
        // two-level passes: the segmentation comes with the call (it fixes the layout of
        // the composites); every unit is independent, so all resident CTAs take them
        const int64_t units = a.groups * a.segments;
        const int64_t resident = int64_t(sms) * occ;
        grid = units < resident ? units : resident;
    } else if (a.workspace) {
        const int64_t resident = int64_t(sms) * occ;
        // about sixteen units per resident CTA (finer units balance the tail), segments
        // of at least sixteen chunks (each unit start costs a carry hand-off)
        int64_t segs = (16 * resident + a.groups - 1) / a.groups;
        // (segment indices stay below 2^24: the carry flags keep 24 bits for them)
        int64_t max_segs = nchunks / 16 > 1 ? nchunks / 16 : 1;
        max_segs = max_segs < (int64_t(1) << 24) - 1 ? max_segs : (int64_t(1) << 24) - 1;
        segs = segs < 1 ? 1 : (segs > max_segs ? max_segs : segs);
        const int64_t seg_chunks = (nchunks + segs - 1) / segs;
        a.seg_len = seg_chunks * S::kChunk;
        a.segments = (nchunks + seg_chunks - 1) / seg_chunks;
        const int64_t units = a.groups * a.segments;
        grid = units < resident ? units : resident;
    } else {
        a.seg_len = nchunks * S::kChunk;
        a.segments = 1;
    }
    if (grid > 0x7fffffffLL)
        return SS_ERR_SHAPE;
    *grid_out = grid;
    return SS_OK;
}

template <int N, int SPL, typename T, bool R, bool V, int E, bool C>
int launch_scan(ss::ScanArgs a, size_t ws_bytes, cudaStream_t stream)
{
    using S = ss::ScanShape<N, SPL>;
    constexpr size_t kSmem = S::template smem_bytes<T, V>();
    auto kernel = ss::ss_scan_fwd_kernel<N, SPL, T, R, V, E, C>;
    int64_t grid = 0;
    int occ = 0, sms = 0;
    int st = plan_scan<N, SPL, T, R, V, E, C>(a, &grid, &occ, &sms);
    if (st != SS_OK)
        return st;
    if (!a.workspace && status_word_address(&a.status) != SS_OK)
        return SS_ERR_CUDA;
    ss::TmaMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (V && !build_maps<N, SPL, T>(a, &maps))
        return SS_ERR_CUDA;
    kernel<<<unsigned(grid), S::kThreads, kSmem, stream>>>(a, maps);
    return launch_status();
}

template <int N, int SPL, typename T, int E, bool C>
int dispatch_scan_e(const ss::ScanArgs &a, bool vec, size_t ws, cudaStream_t s)
{
    const bool r = a.reset != nullptr;
    if (r)
        return vec ? launch_scan<N, SPL, T, true, true, E, C>(a, ws, s)
                   : launch_scan<N, SPL, T, true, false, E, C>(a, ws, s);
    return vec ? launch_scan<N, SPL, T, false, true, E, C>(a, ws, s)
               : launch_scan<N, SPL, T, false, false, E, C>(a, ws, s);
}

// forms: plain (E 0); with per-token states and optionally step sizes (E 1); with the
// step sizes alone (E 2); with the fused conv prologue (C)
template <int N, int SPL, typename T>
int dispatch_scan_t(const ss::ScanArgs &a, bool vec, size_t ws, cudaStream_t s)
{
    if (a.conv_w)
        return dispatch_scan_e<N, SPL, T, 0, true>(a, vec, ws, s);
    if (a.h_all) // the states (and the step sizes when asked for)
        return dispatch_scan_e<N, SPL, T, 1, false>(a, vec, ws, s);
    return a.betas ? dispatch_scan_e<N, SPL, T, 2, false>(a, vec, ws, s) // the step sizes alone
                   : dispatch_scan_e<N, SPL, T, 0, false>(a, vec, ws, s);
}

template <int N, int SPL> int64_t scan_groups(int64_t batch, int64_t channels)
{
    const int64_t per = ss::ScanShape<N, SPL>::kChanPerCta;
    return batch * ((channels + per - 1) / per);
}

// States per scan lane: two.  Four per lane (32 channels per CTA, one CTA per SM)
// moves fewer shared-memory bytes and issues fewer instructions per state, but leaves
// one scan warp per SM sub-partition for the 2.8B-layer shape, and measured slower
// (0.738 against 0.637 ms): a lone warp cannot hide the exponential unit's throttling
// and the FMA chains' latency as two warps do.  It stays selectable
// (ss_debug_set_scan_layout) and tested.
std::atomic<int> g_forced_spl{0};     // ss_debug_set_scan_layout: 0 = choose per shape
std::atomic<int> g_gated_path{0};     // ss_debug_set_gated_path: 0 auto, 1 recurrent, 2 auto, 3 auto + held arrival
std::atomic<int> g_two_level_mode{0}; // ss_debug_set_scan_two_level: 0 auto, 1 never, 2 always

int scan_spl(int64_t batch, int64_t channels, int64_t state_dim)
{
    if (state_dim != 16)
        return 2;
    const int forced = g_forced_spl.load(std::memory_order_relaxed);
    if (forced)
        return forced;
    (void)batch;
    (void)channels;
    return 2;
}

template <int N, int SPL>
int dispatch_scan_s(const ss::ScanArgs &a, ss_dtype_t dtype, bool vec, size_t ws_bytes, cudaStream_t s)
{
    if (dtype == SS_BF16)
        return dispatch_scan_t<N, SPL, __nv_bfloat16>(a, vec, ws_bytes, s);
    return dispatch_scan_t<N, SPL, float>(a, vec, ws_bytes, s);
}

// ------------------------------------------------------------------------------------
// In-GPU two-level scan over the sequence ("s6_reset" blog draft, Associative Boundary
// Resetting: the recurrence composes associatively, so a sequence can be cut into
// segments scanned in parallel).  For shapes with too few channel groups to fill the
// GPU through the chained schedule (whose segments of one group run one after
// another), every segment of every group runs at once, twice:
//   pass 1  each segment from zero, no outputs: its end state;
//   decay   exp(A * sum of the segment's steps), 0 where the segment holds a reset;
//   join    each segment's entering state, h_in[s+1] = decay[s] h_in[s] + state[s],
//           and the final state;
//   pass 2  each segment from its entering state, with outputs.
// This costs twice the exponentials of one pass and wins when the chained schedule
// would leave more than half of the GPU idle.
// ------------------------------------------------------------------------------------

// Workspace of the chained (single-pass) schedule: the larger of the two layouts'
// needs, so the size does not depend on which one the call picks on the device.
int64_t chained_workspace_bytes(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq)
{
    if (batch <= 0 || channels <= 0 || seq <= 0)
        return 0;
    switch (state_dim) {
    case 4: return ss::scan_workspace_bytes<4, 2>(scan_groups<4, 2>(batch, channels));
    case 8: return ss::scan_workspace_bytes<8, 2>(scan_groups<8, 2>(batch, channels));
    case 16: {
        const int64_t a = ss::scan_workspace_bytes<16, 2>(scan_groups<16, 2>(batch, channels));
        const int64_t b = ss::scan_workspace_bytes<16, 4>(scan_groups<16, 4>(batch, channels));
        return a > b ? a : b;
    }
    default: return 0;
    }
}

struct TwoLevelPlan {
    bool use = false;
    int spl = 4;
    int64_t groups = 0, segs = 0, seg_len = 0, count = 0;
    int64_t chained_bytes = 0, bytes = 0; // workspace: chained part, then 3 x segs x count floats
};

int64_t align256(int64_t b) { return (b + 255) / 256 * 256; }

TwoLevelPlan two_level_plan(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq)
{
    TwoLevelPlan t;
    if (state_dim != 16)
        return t;
    int sms = 0;
    if (device_sm_count(&sms) != SS_OK || sms <= 0)
        sms = 148;
    const int64_t groups16 = scan_groups<16, 2>(batch, channels);
    const int64_t nchunks = (seq + 31) / 32;
    const int mode = g_two_level_mode.load(std::memory_order_relaxed);
    // worth it when the chained schedule (two CTAs per SM of 16-channel groups) would
    // keep fewer than half its CTA slots busy, on sequences of 64 chunks or more
    if (mode == 1 || (mode == 0 && (groups16 >= int64_t(sms) || nchunks < 64)))
        return t;
    const int forced = g_forced_spl.load(std::memory_order_relaxed);
    t.spl = forced ? forced : 2;
    t.groups = t.spl == 4 ? scan_groups<16, 4>(batch, channels) : groups16;
    const int64_t resident = int64_t(sms) * (t.spl == 4 ? 1 : 2);
    int64_t segs = (8 * resident + t.groups - 1) / t.groups; // about eight units per CTA
    const int64_t max_segs = nchunks / 16 < (int64_t(1) << 24) - 1 ? nchunks / 16 : (int64_t(1) << 24) - 1;
    segs = segs > max_segs ? max_segs : segs;
    if (segs < 2)
        return t;
    const int64_t seg_chunks = (nchunks + segs - 1) / segs;
    t.seg_len = seg_chunks * 32;
    t.segs = (nchunks + seg_chunks - 1) / seg_chunks;
    if (t.segs < 2)
        return t;
    t.count = batch * channels * 16;
    t.chained_bytes = t.spl == 4 ? ss::scan_workspace_bytes<16, 4>(t.groups) : ss::scan_workspace_bytes<16, 2>(t.groups);
    t.bytes = align256(t.chained_bytes) + 3 * t.segs * t.count * 4;
    t.use = true;
    return t;
}

template <typename T>
void launch_segment_decay(bool vec, bool sp, unsigned grid, const ss::SegDecayArgs &a, cudaStream_t s);

template <int SPL, typename T>
int launch_two_level(const ss::ScanArgs &a0, const TwoLevelPlan &t, bool vec, cudaStream_t s)
{
    uint8_t *base = a0.workspace;
    float *state = reinterpret_cast<float *>(base + align256(t.chained_bytes));
    float *decay = state + t.segs * t.count;
    float *h_in = decay + t.segs * t.count;
    ss::ScanArgs a = a0;
    a.seg_len = t.seg_len;
    a.segments = t.segs;
    a.seg_stride = t.count;
    a.seg_state = state;
    a.seg_in = h_in;
    const bool r = a.reset != nullptr;
    // pass 1: the segments' end states from zero
    a.pass = 1;
    int st = r ? (vec ? launch_scan<16, SPL, T, true, true, false, false>(a, 0, s)
                      : launch_scan<16, SPL, T, true, false, false, false>(a, 0, s))
               : (vec ? launch_scan<16, SPL, T, false, true, false, false>(a, 0, s)
                      : launch_scan<16, SPL, T, false, false, false, false>(a, 0, s));
    if (st != SS_OK)
        return st;
    // the segments' decays
    ss::SegDecayArgs d{};
    d.dt = a.dt;
    d.A = a.A;
    d.dt_bias = a.dt_bias;
    d.reset = a.reset;
    d.decay = decay;
    d.batch = a.batch;
    d.channels = a.channels;
    d.seq = a.seq;
    d.seg_len = t.seg_len;
    d.segments = t.segs;
    d.out_stride = t.count;
    d.state_dim = 16;
    d.reset_vec = a.reset && aligned(a.reset, 16) && a.seq % 16 == 0;
    int sms = 0;
    if (device_sm_count(&sms) != SS_OK)
        return SS_ERR_CUDA;
    const int64_t items = a.batch * a.channels * t.segs;
    const int64_t dblocks = (items + ss::kSegWarps - 1) / ss::kSegWarps;
    const bool dvec = a.seq % 8 == 0 && aligned(a.dt, 16);
    launch_segment_decay<T>(dvec, a.softplus != 0, unsigned(dblocks < int64_t(sms) * 8 ? dblocks : int64_t(sms) * 8),
                            d, s);
    if (launch_status() != SS_OK)
        return SS_ERR_CUDA;
    // the join: every segment's entering state, and the final state
    ss::JoinAllArgs j{};
    j.decay = decay;
    j.state = state;
    j.h0 = a.h0;
    j.h_in = h_in;
    j.h_last = a.h_last;
    j.count = t.count;
    j.segments = t.segs;
    const int64_t jblocks = (t.count + 255) / 256;
    ss::ss_join_all_kernel<<<unsigned(jblocks < int64_t(sms) * 8 ? jblocks : int64_t(sms) * 8), 256, 0, s>>>(j);
    if (launch_status() != SS_OK)
        return SS_ERR_CUDA;
    // pass 2: every segment from its entering state, with outputs
    a.pass = 2;
    return r ? (vec ? launch_scan<16, SPL, T, true, true, false, false>(a, 0, s)
                    : launch_scan<16, SPL, T, true, false, false, false>(a, 0, s))
             : (vec ? launch_scan<16, SPL, T, false, true, false, false>(a, 0, s)
                    : launch_scan<16, SPL, T, false, false, false, false>(a, 0, s));
}

template <int N>
int dispatch_scan_n(ss::ScanArgs a, ss_dtype_t dtype, bool vec, size_t ws_bytes, bool allow_two_level,
                    cudaStream_t s)
{
    // (a host-side check, before anything touches the device: the size the query
    // reports -- or, where the two-level schedule is ruled out, the chained one's)
    if (a.workspace) {
        const int64_t need = allow_two_level ? ss_scan_workspace_bytes(a.batch, a.channels, N, a.seq)
                                             : chained_workspace_bytes(a.batch, a.channels, N, a.seq);
        if (int64_t(ws_bytes) < need)
            return SS_ERR_WORKSPACE;
    }
    if constexpr (N == 16) {
        // the two-level schedule for the plain form, when the shape asks for it and the
        // workspace holds its composites
        if (allow_two_level && a.workspace && !a.h_all && !a.betas && !a.conv_w) {
            const TwoLevelPlan t = two_level_plan(a.batch, a.channels, N, a.seq);
            if (t.use && int64_t(ws_bytes) >= t.bytes) {
                if (t.spl == 4)
                    return dtype == SS_BF16 ? launch_two_level<4, __nv_bfloat16>(a, t, vec, s)
                                            : launch_two_level<4, float>(a, t, vec, s);
                return dtype == SS_BF16 ? launch_two_level<2, __nv_bfloat16>(a, t, vec, s)
                                        : launch_two_level<2, float>(a, t, vec, s);
            }
        }
        if (scan_spl(a.batch, a.channels, N) == 4)
            return dispatch_scan_s<16, 4>(a, dtype, vec, ws_bytes, s);
    }
    return dispatch_scan_s<N, 2>(a, dtype, vec, ws_bytes, s);
}

// The conv form of the decode step (w NULL: none).
struct UpdConv {
    const float *w = nullptr, *b = nullptr;
    float *state = nullptr;
    int k = 0;
};

template <int N, typename T, bool V, bool CV>
int launch_update(ss::UpdateArgs a, cudaStream_t stream, const UpdConv &cv)
{
    if constexpr (V) {
        // aligned state: persistent CTAs streaming the state through shared memory
        using D = ss::DecShape<N, T>;
        auto kernel = ss::ss_state_update_stream_kernel<N, T, CV>;
        static std::atomic<uint64_t> smem_done{0};
        static std::atomic<int> occ_cache[64];
        constexpr size_t kSmem = D::template smem<CV>();
        int st = ensure_smem(kernel, kSmem, smem_done);
        if (st != SS_OK)
            return st;
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || device_sm_count(&sms) != SS_OK)
            return SS_ERR_CUDA;
        int occ = dev < 64 ? occ_cache[dev].load(std::memory_order_acquire) : 0;
        if (!occ) {
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, ss::kDecBlock, kSmem) != cudaSuccess)
                return SS_ERR_CUDA;
            occ = occ > 0 ? occ : 1;
            if (dev < 64)
                occ_cache[dev].store(occ, std::memory_order_release);
        }
        ss::DecArgs da{};
        da.u = a;
        da.ncb = (a.channels + D::kChanPerTile - 1) / D::kChanPerTile;
        const int64_t tiles = a.batch * da.ncb;
        const int64_t resident = int64_t(sms) * occ;
        int64_t grid = tiles < resident ? tiles : resident;
        // with more tiles than CTAs, a grid that is a multiple of the channel blocks
        // lets every CTA keep one channel block (A, dt_bias, D loaded once)
        if (tiles > resident && resident >= da.ncb) {
            grid = resident / da.ncb * da.ncb;
            da.fixed_cb = 1;
        }
        // x, dt_raw, z rows ride along with the state when every tile's rows are
        // 16-byte aligned
        const size_t es = sizeof(T);
        da.bulk_xdz = aligned(a.x, 16) && aligned(a.dt, 16) && (!a.z || aligned(a.z, 16)) &&
                      (size_t(a.channels) * es) % 16 == 0;
        da.bulk_bc = aligned(a.B, 16) && aligned(a.C, 16) && (N * es) % 16 == 0;
        da.conv_w = cv.w;
        da.conv_b = cv.b;
        da.conv_state = cv.state;
        da.conv_k = cv.k;
        // conv-state rows ride along too when every tile's rows start and end on 16 bytes
        da.bulk_cs = CV && cv.k > 1 && aligned(cv.state, 16) && a.channels % 4 == 0;
        uint32_t *status = nullptr;
        if (status_word_address(&status) != SS_OK)
            return SS_ERR_CUDA;
        kernel<<<unsigned(grid), ss::kDecBlock, kSmem, stream>>>(da, status);
        return launch_status();
    }
    if constexpr (CV)
        return SS_ERR_ALIGN; // the conv form runs on the streaming kernel only
    const int64_t per_block = int64_t(ss::kUpdateThreads) * ss::kUpdateItems; // row quarters
    const int64_t quarters = a.channels * (N / 4);
    a.blocks_per_row = int((quarters + per_block - 1) / per_block);
    const int64_t blocks = a.batch * a.blocks_per_row;
    if (blocks > 0x7fffffffLL)
        return SS_ERR_SHAPE;
    ss::ss_state_update_kernel<N, T, V><<<unsigned(blocks), ss::kUpdateThreads, 0, stream>>>(a);
    return launch_status();
}

template <int N, bool CV>
int dispatch_update_c(const ss::UpdateArgs &a, ss_dtype_t dtype, bool vec, cudaStream_t s, const UpdConv &cv)
{
    if (dtype == SS_BF16)
        return vec ? launch_update<N, __nv_bfloat16, true, CV>(a, s, cv)
                   : launch_update<N, __nv_bfloat16, false, CV>(a, s, cv);
    return vec ? launch_update<N, float, true, CV>(a, s, cv) : launch_update<N, float, false, CV>(a, s, cv);
}

template <int N>
int dispatch_update_n(const ss::UpdateArgs &a, ss_dtype_t dtype, bool vec, cudaStream_t s, const UpdConv &cv)
{
    return cv.w ? dispatch_update_c<N, true>(a, dtype, vec, s, cv) : dispatch_update_c<N, false>(a, dtype, vec, s, cv);
}

// Scratch of ss_scan_fwd_static_scratch: a fixed workspace in device memory, one per
// device that loads the library.  Zero at module load; every scan that completes
// leaves it ready for the next.
static_assert(SS_STATIC_SCRATCH_BYTES % 256 == 0, "scratch size");
static __device__ __align__(256) uint8_t g_ss_static_scratch[SS_STATIC_SCRATCH_BYTES];

// Device address of this device's scratch, looked up (with the device current) on
// the first call and cached per device.
int static_scratch_address(void **out)
{
    static std::atomic<uintptr_t> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return SS_ERR_CUDA;
    if (dev < 64) {
        const uintptr_t v = cache[dev].load(std::memory_order_acquire);
        if (v) {
            *out = reinterpret_cast<void *>(v);
            return SS_OK;
        }
    }
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_ss_static_scratch) != cudaSuccess || !ptr)
        return SS_ERR_CUDA;
    if (dev < 64)
        cache[dev].store(reinterpret_cast<uintptr_t>(ptr), std::memory_order_release);
    *out = ptr;
    return SS_OK;
}

} // namespace

extern "C" {

int ss_abi_version(void) { return (kAbiMajor << 16) | kAbiMinor; }

const char *ss_status_string(int status)
{
    switch (status) {
    case SS_OK: return "SS_OK";
    case SS_ERR_NULL: return "SS_ERR_NULL: a required pointer is NULL";
    case SS_ERR_SHAPE: return "SS_ERR_SHAPE: a size is <= 0 or too large";
    case SS_ERR_DTYPE: return "SS_ERR_DTYPE: dtype must be SS_F32 or SS_BF16";
    case SS_ERR_ALIGN: return "SS_ERR_ALIGN: a pointer is not aligned to its element size";
    case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED: state_dim must be 4, 8 or 16; unknown flag bit";
    case SS_ERR_CUDA: return "SS_ERR_CUDA: the CUDA runtime reported an error";
    case SS_ERR_TIMEOUT: return "SS_ERR_TIMEOUT: a bounded device-side wait gave up";
    case SS_ERR_ALIAS: return "SS_ERR_ALIAS: an output overlaps an input";
    case SS_ERR_WORKSPACE: return "SS_ERR_WORKSPACE: the workspace is smaller than ss_scan_workspace_bytes()";
    case SS_ERR_SCRATCH_LIMIT:
        return "SS_ERR_SCRATCH_LIMIT: the shape needs more workspace than the static scratch holds "
               "(SS_STATIC_SCRATCH_BYTES); use ss_scan_fwd with a workspace";
    default: return "unknown status";
    }
}

int ss_debug_set_scan_layout(int states_per_lane)
{
    if (states_per_lane != 0 && states_per_lane != 2 && states_per_lane != 4)
        return SS_ERR_UNSUPPORTED;
    g_forced_spl.store(states_per_lane, std::memory_order_relaxed);
    return SS_OK;
}

int ss_debug_bounds_status(ss_stream_t stream, int *site)
{
    if (!site)
        return SS_ERR_NULL;
#ifdef SS_BOUNDS_CHECK
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    const uint32_t zero = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpyFromSymbol(&v, ss::g_ss_bounds_site, sizeof(v)) != cudaSuccess ||
        cudaMemcpyToSymbol(ss::g_ss_bounds_site, &zero, sizeof(zero)) != cudaSuccess)
        return SS_ERR_CUDA;
    *site = int(v);
    return SS_OK;
#else
    (void)stream;
    *site = -1;
    return SS_ERR_UNSUPPORTED;
#endif
}

int ss_debug_set_gated_path(int mode)
{
    if (mode < 0 || mode > 3)
        return SS_ERR_UNSUPPORTED;
    g_gated_path.store(mode, std::memory_order_relaxed);
    return SS_OK;
}

int ss_debug_set_scan_two_level(int mode)
{
    if (mode < 0 || mode > 2)
        return SS_ERR_UNSUPPORTED;
    g_two_level_mode.store(mode, std::memory_order_relaxed);
    return SS_OK;
}

int ss_debug_set_wait_limit(uint32_t microseconds)
{
    return cudaMemcpyToSymbol(ss::g_ss_wait_limit_us, &microseconds, sizeof(microseconds)) == cudaSuccess
               ? SS_OK
               : SS_ERR_CUDA;
}

int64_t ss_scan_workspace_bytes(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq)
{
    const int64_t chained = chained_workspace_bytes(batch, channels, state_dim, seq);
    if (chained <= 0)
        return chained;
    const TwoLevelPlan t = two_level_plan(batch, channels, state_dim, seq);
    return t.use && t.bytes > chained ? t.bytes : chained;
}

int ss_scan_status(const void *workspace, ss_stream_t stream, int *status)
{
    if (!status)
        return SS_ERR_NULL;
    uint32_t *word = nullptr;
    if (workspace) {
        if (!aligned(workspace, 16))
            return SS_ERR_ALIGN;
        word = &static_cast<ss::WsHeader *>(const_cast<void *>(workspace))->status;
    } else if (status_word_address(&word) != SS_OK) {
        return SS_ERR_CUDA;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return SS_ERR_CUDA;
    if (v && (cudaMemsetAsync(word, 0, sizeof(v), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess))
        return SS_ERR_CUDA;
    *status = (v & (1u << ss::kStatusTimeout)) ? SS_ERR_TIMEOUT : SS_OK;
    return SS_OK;
}

int ss_scan_plan(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq, ss_dtype_t dtype,
                 int has_reset, int with_workspace, ss_scan_plan_t *plan)
{
    if (!plan)
        return SS_ERR_NULL;
    if (batch <= 0 || channels <= 0 || seq <= 0)
        return SS_ERR_SHAPE;
    if (dtype != SS_F32 && dtype != SS_BF16)
        return SS_ERR_DTYPE;
    if (state_dim != 4 && state_dim != 8 && state_dim != 16)
        return SS_ERR_UNSUPPORTED;
    ss::ScanArgs a{};
    a.batch = batch;
    a.channels = channels;
    a.seq = seq;
    // any non-null value: the plan only asks whether a workspace is given
    a.workspace = with_workspace ? reinterpret_cast<uint8_t *>(uintptr_t(256)) : nullptr;
    int64_t grid = 0;
    int occ = 0, sms = 0, st = SS_OK;
    const bool r = has_reset != 0;
    auto run = [&](auto n_tag, auto spl_tag) -> int {
        constexpr int N = decltype(n_tag)::value, SPL = decltype(spl_tag)::value;
        if (dtype == SS_BF16)
            return r ? plan_scan<N, SPL, __nv_bfloat16, true, true, false, false>(a, &grid, &occ, &sms)
                     : plan_scan<N, SPL, __nv_bfloat16, false, true, false, false>(a, &grid, &occ, &sms);
        return r ? plan_scan<N, SPL, float, true, true, false, false>(a, &grid, &occ, &sms)
                 : plan_scan<N, SPL, float, false, true, false, false>(a, &grid, &occ, &sms);
    };
    using I2 = std::integral_constant<int, 2>;
    switch (state_dim) {
    case 4: st = run(std::integral_constant<int, 4>(), I2()); break;
    case 8: st = run(std::integral_constant<int, 8>(), I2()); break;
    default:
        st = scan_spl(batch, channels, 16) == 4 ? run(std::integral_constant<int, 16>(), std::integral_constant<int, 4>())
                                                  : run(std::integral_constant<int, 16>(), I2());
        break;
    }
    if (st != SS_OK)
        return st;
    plan->grid = grid;
    plan->ctas_per_sm = occ;
    plan->states_per_lane = state_dim == 16 ? scan_spl(batch, channels, 16) : 2;
    plan->two_level = 0;
    if (with_workspace) {
        const TwoLevelPlan t = two_level_plan(batch, channels, state_dim, seq);
        if (t.use) { // (the plain form with a workspace of ss_scan_workspace_bytes)
            const int64_t resident = int64_t(sms) * (t.spl == 4 ? 1 : 2);
            plan->two_level = 1;
            plan->states_per_lane = t.spl;
            plan->ctas_per_sm = t.spl == 4 ? 1 : 2;
            plan->groups = t.groups;
            plan->segments = t.segs;
            plan->seg_len = t.seg_len;
            plan->grid = t.groups * t.segs < resident ? t.groups * t.segs : resident;
            plan->states_per_lane = t.spl;
        }
    }
    plan->sms = sms;
    plan->groups = a.groups;
    plan->segments = a.segments;
    plan->seg_len = a.seg_len;
    return SS_OK;
}

int ss_debug_status(ss_stream_t stream)
{
    int st = SS_OK;
    const int q = ss_scan_status(nullptr, stream, &st);
    return q != SS_OK ? q : st;
}

} // extern "C"

namespace {

// ss_scan_fwd and ss_scan_fwd_states: validation, then the launch.  h_all (nullable)
// receives the state after every token, betas (nullable) every token's step size.
// Fused conv prologue of ss_scan_fwd_conv (w NULL: none); x is then the conv input.
struct ConvArgs {
    const float *w = nullptr, *b = nullptr, *state = nullptr;
    float *state_out = nullptr;
    void *x_out = nullptr;
    int k = 0;
};

int scan_impl(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq, ss_dtype_t dtype,
              const void *x, const void *dt_raw, const float *A, const void *B, const void *C,
              const float *D, const void *z, const float *dt_bias, const uint8_t *reset,
              const float *h0, uint32_t flags, void *y, float *h_last, float *h_all, float *betas,
              void *workspace, size_t workspace_bytes, ss_stream_t stream, const ConvArgs &cv = ConvArgs(),
              bool allow_two_level = true)
{
    if (!x || !dt_raw || !A || !B || !C || !y)
        return SS_ERR_NULL;
    if (batch <= 0 || channels <= 0 || state_dim <= 0 || seq <= 0)
        return SS_ERR_SHAPE;
    if (dtype != SS_F32 && dtype != SS_BF16)
        return SS_ERR_DTYPE;
    if (state_dim != 4 && state_dim != 8 && state_dim != 16)
        return SS_ERR_UNSUPPORTED;
    if (flags & ~uint32_t(SS_DT_SOFTPLUS))
        return SS_ERR_UNSUPPORTED;
    const size_t es = dtype == SS_BF16 ? 2 : 4;
    int64_t rows = 0, elems = 0, bn = 0, bcel = 0, stel = 0, rsel = 0;
    if (!mul_ok(batch, channels, &rows) || !mul_ok(rows, seq, &elems) || !mul_ok(batch, state_dim, &bn) ||
        !mul_ok(bn, seq, &bcel) || !mul_ok(rows, state_dim, &stel) || !mul_ok(batch, seq, &rsel) ||
        elems > (INT64_MAX / 8) || bcel > (INT64_MAX / 8) || stel > (INT64_MAX / 8))
        return SS_ERR_SHAPE;
    const void *typed[] = {x, dt_raw, B, C, z, y};
    for (const void *p : typed)
        if (p && !aligned(p, es))
            return SS_ERR_ALIGN;
    const void *f32s[] = {A, D, dt_bias, h0, h_last};
    for (const void *p : f32s)
        if (p && !aligned(p, 4))
            return SS_ERR_ALIGN;
    // outputs must not overlap inputs (h_last may BE h0: each lane reads its own
    // h0 entries before it writes the same h_last entries)
    const size_t ybytes = size_t(elems) * es, hbytes = size_t(stel) * 4;
    const void *in_p[] = {x, dt_raw, z, B, C, A, D, dt_bias, reset, h0};
    const size_t in_n[] = {ybytes, ybytes, z ? ybytes : 0, size_t(bcel) * es, size_t(bcel) * es,
                           size_t(channels * state_dim) * 4, D ? size_t(channels) * 4 : 0,
                           dt_bias ? size_t(channels) * 4 : 0, reset ? size_t(rsel) : 0,
                           h0 ? hbytes : 0};
    for (int i = 0; i < 10; ++i) {
        if (overlaps(y, ybytes, in_p[i], in_n[i]))
            return SS_ERR_ALIAS;
        if (h_last && !(i == 9 && in_p[i] == h_last) && overlaps(h_last, hbytes, in_p[i], in_n[i]))
            return SS_ERR_ALIAS;
    }
    if (h_last && overlaps(h_last, hbytes, y, ybytes))
        return SS_ERR_ALIAS;
    size_t abytes = 0; // h_all
    if (h_all) {
        int64_t ael = 0;
        if (!mul_ok(elems, state_dim, &ael) || ael > (INT64_MAX / 8))
            return SS_ERR_SHAPE;
        abytes = size_t(ael) * 4;
        if (!aligned(h_all, 4))
            return SS_ERR_ALIGN;
        for (int i = 0; i < 10; ++i)
            if (overlaps(h_all, abytes, in_p[i], in_n[i]))
                return SS_ERR_ALIAS;
        if (overlaps(h_all, abytes, y, ybytes) || (h_last && overlaps(h_all, abytes, h_last, hbytes)))
            return SS_ERR_ALIAS;
    }
    const size_t bbytes = betas ? size_t(elems) * 4 : 0; // betas
    if (betas) {
        if (!aligned(betas, 4))
            return SS_ERR_ALIGN;
        for (int i = 0; i < 10; ++i)
            if (overlaps(betas, bbytes, in_p[i], in_n[i]))
                return SS_ERR_ALIAS;
        if (overlaps(betas, bbytes, y, ybytes) || (h_last && overlaps(betas, bbytes, h_last, hbytes)) ||
            (h_all && overlaps(betas, bbytes, h_all, abytes)))
            return SS_ERR_ALIAS;
    }
    size_t cbytes = 0; // conv state
    if (cv.w) {
        if (cv.k < 1 || cv.k > 4 || h_all || betas)
            return SS_ERR_UNSUPPORTED;
        const float *f32c[] = {cv.w, cv.b, cv.state, cv.state_out};
        for (const float *q : f32c)
            if (q && !aligned(q, 4))
                return SS_ERR_ALIGN;
        if (cv.x_out && !aligned(cv.x_out, es))
            return SS_ERR_ALIGN;
        cbytes = size_t(rows) * size_t(cv.k - 1) * 4;
        const size_t wbytes = size_t(channels) * size_t(cv.k) * 4;
        const void *cin[] = {cv.w, cv.b, cv.state};
        const size_t cin_n[] = {wbytes, cv.b ? size_t(channels) * 4 : 0, cv.state ? cbytes : 0};
        // the outputs (y, h_last, x_out, state_out) overlap no input and no other output
        const void *outs[] = {y, h_last, cv.x_out, cv.state_out};
        const size_t out_n[] = {ybytes, h_last ? hbytes : 0, cv.x_out ? ybytes : 0, cv.state_out ? cbytes : 0};
        for (int o = 0; o < 4; ++o) {
            for (int i = 0; i < 10; ++i)
                if (!(o == 1 && i == 9 && in_p[i] == h_last) && overlaps(outs[o], out_n[o], in_p[i], in_n[i]))
                    return SS_ERR_ALIAS;
            for (int i = 0; i < 3; ++i)
                if (overlaps(outs[o], out_n[o], cin[i], cin_n[i]))
                    return SS_ERR_ALIAS;
            for (int o2 = o + 1; o2 < 4; ++o2)
                if (overlaps(outs[o], out_n[o], outs[o2], out_n[o2]))
                    return SS_ERR_ALIAS;
        }
    }
    if (workspace) {
        if (!aligned(workspace, 16))
            return SS_ERR_ALIGN;
        for (int i = 0; i < 10; ++i)
            if (overlaps(workspace, workspace_bytes, in_p[i], in_n[i]))
                return SS_ERR_ALIAS;
        if (overlaps(workspace, workspace_bytes, y, ybytes) ||
            (h_last && overlaps(workspace, workspace_bytes, h_last, hbytes)) ||
            (h_all && overlaps(workspace, workspace_bytes, h_all, abytes)) ||
            (betas && overlaps(workspace, workspace_bytes, betas, bbytes)) ||
            (cv.x_out && overlaps(workspace, workspace_bytes, cv.x_out, ybytes)) ||
            (cv.state_out && overlaps(workspace, workspace_bytes, cv.state_out, cbytes)))
            return SS_ERR_ALIAS;
    }

    const int vec_elems = 16 / int(es);
    // the vector path loads tiles through TMA tensor maps: 32-bit coordinates
    bool vec = (seq % vec_elems) == 0 && seq < (int64_t(1) << 31) && rows < (int64_t(1) << 31) &&
               batch * state_dim < (int64_t(1) << 31);
    for (const void *p : typed)
        if (p && !aligned(p, 16))
            vec = false;
    if (cv.x_out && !aligned(cv.x_out, 16))
        vec = false;

    ss::ScanArgs a{};
    a.batch = batch;
    a.channels = channels;
    a.seq = seq;
    a.x = x; a.dt = dt_raw; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.dt_bias = dt_bias; a.h0 = h0;
    a.reset = reset;
    a.y = y;
    a.h_last = h_last;
    a.h_all = h_all;
    a.betas = betas;
    a.conv_w = cv.w;
    a.conv_b = cv.b;
    a.conv_state = cv.state;
    a.conv_state_out = cv.state_out;
    a.x_out = cv.x_out;
    a.conv_k = cv.k;
    a.softplus = (flags & SS_DT_SOFTPLUS) ? 1 : 0;
    a.workspace = static_cast<uint8_t *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (state_dim) {
    case 4: return dispatch_scan_n<4>(a, dtype, vec, workspace_bytes, allow_two_level, s);
    case 8: return dispatch_scan_n<8>(a, dtype, vec, workspace_bytes, allow_two_level, s);
    default: return dispatch_scan_n<16>(a, dtype, vec, workspace_bytes, allow_two_level, s);
    }
}

template <int RG, typename T, bool VEC> int launch_gated(ss::GatedArgs a, cudaStream_t stream)
{
    using G = ss::GatedShape<RG>;
    auto kernel = ss::ss_gated_scan_kernel<RG, T, VEC>;
    static std::atomic<uint64_t> smem_done{0};
    const int st = ensure_smem(kernel, G::kSmem, smem_done);
    if (st != SS_OK)
        return st;
    a.col_tiles = int((a.dv + G::kCols - 1) / G::kCols);
    int64_t grid = 0;
    if (!mul_ok(a.batch, a.col_tiles, &grid) || grid > 0x7fffffffLL)
        return SS_ERR_SHAPE;
    kernel<<<unsigned(grid), G::kThreads, G::kSmem, stream>>>(a);
    return launch_status();
}

template <int RG, typename T> int dispatch_gated_v(const ss::GatedArgs &a, cudaStream_t s)
{
    // 8-element vector staging: whole rows (dk equals the padded row count), dv a
    // multiple of 8, rows 16-byte aligned
    const bool vec = a.dk == 8 * RG && a.dv % 8 == 0 && aligned(a.q, 16) && aligned(a.k, 16) && aligned(a.v, 16);
    return vec ? launch_gated<RG, T, true>(a, s) : launch_gated<RG, T, false>(a, s);
}

// 3-D map over [batch][seq][inner] bf16 with boxes of 64 x 128 x 1 and the 128-byte
// swizzle (rows past seq read as zeros, per batch item).
bool encode_bsi(CUtensorMap *map, const void *base, int64_t batch, int64_t seq, int64_t inner)
{
    PFN_cuTensorMapEncodeTiled enc = tensor_map_encoder();
    if (!enc)
        return false;
    const cuuint64_t dims[3] = {cuuint64_t(inner), cuuint64_t(seq), cuuint64_t(batch)};
    const cuuint64_t strides[2] = {cuuint64_t(inner) * 2, cuuint64_t(seq) * cuuint64_t(inner) * 2};
    const cuuint32_t box[3] = {64, uint32_t(ss::kGtChunk), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The chunked tensor-core form: bf16, dk = 128, dv a multiple of 64, 16-byte aligned
// rows (the tile loads, the vector loads of h0 and the vector stores).
bool gated_tc_eligible(const ss::GatedArgs &a, bool bf16)
{
    const int mode = g_gated_path.load(std::memory_order_relaxed);
    if (mode == 1 || !bf16)
        return false;
    return a.dk == ss::kGtDk && a.dv % ss::kGtNv == 0 && a.seq < (int64_t(1) << 31) &&
           a.batch < (int64_t(1) << 31) && aligned(a.q, 16) && aligned(a.k, 16) && aligned(a.v, 16) &&
           aligned(a.y, 16) && aligned(a.final_state, 16) && (!a.h0 || aligned(a.h0, 16));
}

int launch_gated_tc(const ss::GatedArgs &g, cudaStream_t stream)
{
    static std::atomic<uint64_t> smem_done{0};
    const int st = ensure_smem(ss::ss_gated_tc_kernel, size_t(ss::GtSmem::kBytes), smem_done);
    if (st != SS_OK)
        return st;
    ss::GatedTcArgs a{};
    a.batch = g.batch;
    a.seq = g.seq;
    a.dv = g.dv;
    a.gamma = g.gamma;
    a.h0 = g.h0;
    a.y = static_cast<__nv_bfloat16 *>(g.y);
    a.final_state = static_cast<__nv_bfloat16 *>(g.final_state);
    a.col_tiles = int(g.dv / ss::kGtNv);
    a.hold_first_mw = g_gated_path.load(std::memory_order_relaxed) == 3 ? 1 : 0;
    int64_t grid = 0;
    if (!mul_ok(g.batch, a.col_tiles, &grid) || grid > 0x7fffffffLL)
        return SS_ERR_SHAPE;
    ss::GatedTcMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (!encode_bsi(&maps.q, g.q, g.batch, g.seq, g.dk) || !encode_bsi(&maps.k, g.k, g.batch, g.seq, g.dk) ||
        !encode_bsi(&maps.v, g.v, g.batch, g.seq, g.dv))
        return SS_ERR_CUDA;
    uint32_t *status = nullptr;
    if (status_word_address(&status) != SS_OK)
        return SS_ERR_CUDA;
    ss::ss_gated_tc_kernel<<<unsigned(grid), ss::kGtThreads, ss::GtSmem::kBytes, stream>>>(a, maps, status);
    return launch_status();
}

template <typename T> int dispatch_gated(const ss::GatedArgs &a, cudaStream_t s)
{
    if (gated_tc_eligible(a, sizeof(T) == 2))
        return launch_gated_tc(a, s);
    if (a.dk <= 32)
        return dispatch_gated_v<4, T>(a, s);
    if (a.dk <= 64)
        return dispatch_gated_v<8, T>(a, s);
    return dispatch_gated_v<16, T>(a, s);
}

template <typename T>
void launch_segment_decay(bool vec, bool sp, unsigned grid, const ss::SegDecayArgs &a, cudaStream_t s)
{
    const unsigned threads = ss::kSegWarps * 32;
    if (vec && sp)
        ss::ss_segment_decay_kernel<T, true, true><<<grid, threads, 0, s>>>(a);
    else if (vec)
        ss::ss_segment_decay_kernel<T, true, false><<<grid, threads, 0, s>>>(a);
    else if (sp)
        ss::ss_segment_decay_kernel<T, false, true><<<grid, threads, 0, s>>>(a);
    else
        ss::ss_segment_decay_kernel<T, false, false><<<grid, threads, 0, s>>>(a);
}

} // namespace

extern "C" {

int ss_gated_scan(int64_t batch, int64_t seq, int64_t dk, int64_t dv, ss_dtype_t dtype, const void *q,
                  const void *k, const void *v, const float *gamma, const float *h0, void *outputs,
                  void *final_state, ss_stream_t stream)
{
    if (!q || !k || !v || !gamma || !outputs || !final_state)
        return SS_ERR_NULL;
    if (batch <= 0 || seq <= 0 || dk <= 0 || dv <= 0)
        return SS_ERR_SHAPE;
    if (dtype != SS_F32 && dtype != SS_BF16)
        return SS_ERR_DTYPE;
    if (dk > 128)
        return SS_ERR_UNSUPPORTED;
    const size_t es = dtype == SS_BF16 ? 2 : 4;
    int64_t bs = 0, qel = 0, vel = 0, bk = 0, sel = 0;
    if (!mul_ok(batch, seq, &bs) || !mul_ok(bs, dk, &qel) || !mul_ok(bs, dv, &vel) || !mul_ok(batch, dk, &bk) ||
        !mul_ok(bk, dv, &sel) || qel > (INT64_MAX / 8) || vel > (INT64_MAX / 8) || sel > (INT64_MAX / 8))
        return SS_ERR_SHAPE;
    const void *typed[] = {q, k, v, outputs, final_state};
    for (const void *p : typed)
        if (!aligned(p, es))
            return SS_ERR_ALIGN;
    if (!aligned(gamma, 4) || (h0 && !aligned(h0, 4)))
        return SS_ERR_ALIGN;
    const void *in_p[] = {q, k, v, gamma, h0};
    const size_t in_n[] = {size_t(qel) * es, size_t(qel) * es, size_t(vel) * es, size_t(bs) * 4,
                           h0 ? size_t(sel) * 4 : 0};
    const size_t ybytes = size_t(vel) * es, fbytes = size_t(sel) * es;
    for (int i = 0; i < 5; ++i)
        if (overlaps(outputs, ybytes, in_p[i], in_n[i]) || overlaps(final_state, fbytes, in_p[i], in_n[i]))
            return SS_ERR_ALIAS;
    if (overlaps(outputs, ybytes, final_state, fbytes))
        return SS_ERR_ALIAS;
    ss::GatedArgs a{};
    a.batch = batch;
    a.seq = seq;
    a.dk = dk;
    a.dv = dv;
    a.q = q; a.k = k; a.v = v;
    a.gamma = gamma;
    a.h0 = h0;
    a.y = outputs;
    a.final_state = final_state;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return dtype == SS_BF16 ? dispatch_gated<__nv_bfloat16>(a, s) : dispatch_gated<float>(a, s);
}

int ss_scan_fwd(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq, ss_dtype_t dtype,
                const void *x, const void *dt_raw, const float *A, const void *B, const void *C,
                const float *D, const void *z, const float *dt_bias, const uint8_t *reset,
                const float *h0, uint32_t flags, void *y, float *h_last, void *workspace,
                size_t workspace_bytes, ss_stream_t stream)
{
    return scan_impl(batch, channels, state_dim, seq, dtype, x, dt_raw, A, B, C, D, z, dt_bias, reset, h0, flags, y,
                     h_last, nullptr, nullptr, workspace, workspace_bytes, stream);
}

int ss_scan_fwd_conv(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq, ss_dtype_t dtype,
                     const void *u, const float *conv_w, const float *conv_b, int64_t conv_k,
                     const float *conv_state, float *conv_state_out, void *x_out, const void *dt_raw,
                     const float *A, const void *B, const void *C, const float *D, const void *z,
                     const float *dt_bias, const uint8_t *reset, const float *h0, uint32_t flags, void *y,
                     float *h_last, void *workspace, size_t workspace_bytes, ss_stream_t stream)
{
    if (!conv_w)
        return SS_ERR_NULL;
    if (conv_k < 1 || conv_k > 4)
        return SS_ERR_UNSUPPORTED;
    ConvArgs cv;
    cv.w = conv_w;
    cv.b = conv_b;
    cv.state = conv_state;
    cv.state_out = conv_state_out;
    cv.x_out = x_out;
    cv.k = int(conv_k);
    return scan_impl(batch, channels, state_dim, seq, dtype, u, dt_raw, A, B, C, D, z, dt_bias, reset, h0, flags, y,
                     h_last, nullptr, nullptr, workspace, workspace_bytes, stream, cv);
}

int ss_scan_fwd_states(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq, ss_dtype_t dtype,
                       const void *x, const void *dt_raw, const float *A, const void *B, const void *C,
                       const float *D, const void *z, const float *dt_bias, const uint8_t *reset,
                       const float *h0, uint32_t flags, void *y, float *h_last, float *h_all, float *betas,
                       void *workspace, size_t workspace_bytes, ss_stream_t stream)
{
    if (!h_all && !betas)
        return SS_ERR_NULL;
    return scan_impl(batch, channels, state_dim, seq, dtype, x, dt_raw, A, B, C, D, z, dt_bias, reset, h0, flags, y,
                     h_last, h_all, betas, workspace, workspace_bytes, stream);
}

} // extern "C"

namespace {

int update_impl(int64_t batch, int64_t channels, int64_t state_dim, ss_dtype_t dtype, float *state,
                const void *x, const void *dt_raw, const float *A, const void *B, const void *C, const float *D,
                const void *z, const float *dt_bias, uint32_t flags, void *y, ss_stream_t stream,
                const UpdConv &cv = UpdConv())
{
    if (!state || !x || !dt_raw || !A || !B || !C || !y)
        return SS_ERR_NULL;
    if (batch <= 0 || channels <= 0 || state_dim <= 0)
        return SS_ERR_SHAPE;
    if (dtype != SS_F32 && dtype != SS_BF16)
        return SS_ERR_DTYPE;
    if (state_dim != 4 && state_dim != 8 && state_dim != 16)
        return SS_ERR_UNSUPPORTED;
    if (flags & ~uint32_t(SS_DT_SOFTPLUS))
        return SS_ERR_UNSUPPORTED;
    const size_t es = dtype == SS_BF16 ? 2 : 4;
    int64_t rows = 0, stel = 0, bnel = 0;
    if (!mul_ok(batch, channels, &rows) || !mul_ok(rows, state_dim, &stel) ||
        !mul_ok(batch, state_dim, &bnel) || stel > (INT64_MAX / 8))
        return SS_ERR_SHAPE;
    const void *typed[] = {x, dt_raw, B, C, z, y};
    for (const void *p : typed)
        if (p && !aligned(p, es))
            return SS_ERR_ALIGN;
    const void *f32s[] = {state, A, D, dt_bias};
    for (const void *p : f32s)
        if (p && !aligned(p, 4))
            return SS_ERR_ALIGN;
    const size_t sbytes = size_t(stel) * 4, ybytes = size_t(rows) * es;
    const void *in_p[] = {x, dt_raw, z, B, C, A, D, dt_bias};
    const size_t in_n[] = {ybytes, ybytes, z ? ybytes : 0, size_t(bnel) * es, size_t(bnel) * es,
                           size_t(channels * state_dim) * 4, D ? size_t(channels) * 4 : 0,
                           dt_bias ? size_t(channels) * 4 : 0};
    for (int i = 0; i < 8; ++i)
        if (overlaps(y, ybytes, in_p[i], in_n[i]) || overlaps(state, sbytes, in_p[i], in_n[i]))
            return SS_ERR_ALIAS;
    if (overlaps(y, ybytes, state, sbytes))
        return SS_ERR_ALIAS;
    if (cv.w) {
        if (cv.k < 1 || cv.k > 4)
            return SS_ERR_UNSUPPORTED;
        if (cv.k > 1 && !cv.state)
            return SS_ERR_NULL;
        const float *f32c[] = {cv.w, cv.b, cv.state};
        for (const float *q : f32c)
            if (q && !aligned(q, 4))
                return SS_ERR_ALIGN;
        // the conv state is updated in place: it overlaps no other buffer
        const size_t cbytes = size_t(rows) * size_t(cv.k - 1) * 4;
        const void *oth[] = {x, dt_raw, z, B, C, A, D, dt_bias, y, state, cv.w, cv.b};
        const size_t oth_n[] = {ybytes, ybytes, z ? ybytes : 0, size_t(bnel) * es, size_t(bnel) * es,
                                size_t(channels * state_dim) * 4, D ? size_t(channels) * 4 : 0,
                                dt_bias ? size_t(channels) * 4 : 0, ybytes, sbytes, size_t(channels) * cv.k * 4,
                                cv.b ? size_t(channels) * 4 : 0};
        for (int i = 0; i < 12; ++i)
            if (overlaps(cv.state, cbytes, oth[i], oth_n[i]))
                return SS_ERR_ALIAS;
    }

    const bool vec = aligned(state, 16) && aligned(A, 16) && aligned(B, 4 * es) && aligned(C, 4 * es);
    ss::UpdateArgs a{};
    a.batch = batch;
    a.channels = channels;
    a.state = state;
    a.x = x; a.dt = dt_raw; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.dt_bias = dt_bias;
    a.y = y;
    a.softplus = (flags & SS_DT_SOFTPLUS) ? 1 : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (state_dim) {
    case 4: return dispatch_update_n<4>(a, dtype, vec, s, cv);
    case 8: return dispatch_update_n<8>(a, dtype, vec, s, cv);
    default: return dispatch_update_n<16>(a, dtype, vec, s, cv);
    }
}

} // namespace

extern "C" {

int ss_state_update(int64_t batch, int64_t channels, int64_t state_dim, ss_dtype_t dtype,
                    float *state, const void *x, const void *dt_raw, const float *A,
                    const void *B, const void *C, const float *D, const void *z,
                    const float *dt_bias, uint32_t flags, void *y, ss_stream_t stream)
{
    return update_impl(batch, channels, state_dim, dtype, state, x, dt_raw, A, B, C, D, z, dt_bias, flags, y, stream);
}

int ss_state_update_conv(int64_t batch, int64_t channels, int64_t state_dim, ss_dtype_t dtype, float *state,
                         float *conv_state, const float *conv_w, const float *conv_b, int64_t conv_k,
                         const void *u, const void *dt_raw, const float *A, const void *B, const void *C,
                         const float *D, const void *z, const float *dt_bias, uint32_t flags, void *y,
                         ss_stream_t stream)
{
    if (!conv_w)
        return SS_ERR_NULL;
    if (conv_k < 1 || conv_k > 4)
        return SS_ERR_UNSUPPORTED;
    UpdConv cv;
    cv.w = conv_w;
    cv.b = conv_b;
    cv.state = conv_state;
    cv.k = int(conv_k);
    return update_impl(batch, channels, state_dim, dtype, state, u, dt_raw, A, B, C, D, z, dt_bias, flags, y, stream,
                       cv);
}

// The scratch stands in for the caller's workspace: the shape is checked against its
// size first, then the scan is exactly ss_scan_fwd's segmented schedule.
int ss_scan_fwd_static_scratch(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq,
                               ss_dtype_t dtype, const void *x, const void *dt_raw, const float *A,
                               const void *B, const void *C, const float *D, const void *z,
                               const float *dt_bias, const uint8_t *reset, const float *h0,
                               uint32_t flags, void *y, float *h_last, const void **scratch,
                               ss_stream_t stream)
{
    if (!x || !dt_raw || !A || !B || !C || !y)
        return SS_ERR_NULL;
    if (flags & ~uint32_t(SS_DT_SOFTPLUS | SS_SCRATCH_ZERO))
        return SS_ERR_UNSUPPORTED;
    // (the chained schedule: the static scratch does not hold the two-level one's
    // composites)
    const int64_t need = chained_workspace_bytes(batch, channels, state_dim, seq);
    if (need > int64_t(SS_STATIC_SCRATCH_BYTES))
        return SS_ERR_SCRATCH_LIMIT;
    // (need == 0: an invalid shape, which ss_scan_fwd reports with its own status)
    void *ws = nullptr;
    if (static_scratch_address(&ws) != SS_OK)
        return SS_ERR_CUDA;
    if (scratch)
        *scratch = ws;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the whole scratch: carry flags beyond this shape's part, left by an earlier call
    // with more channel groups, must not survive the epoch going back to zero
    if (need > 0 && (flags & SS_SCRATCH_ZERO) &&
        cudaMemsetAsync(ws, 0, size_t(SS_STATIC_SCRATCH_BYTES), s) != cudaSuccess)
        return SS_ERR_CUDA;
    return scan_impl(batch, channels, state_dim, seq, dtype, x, dt_raw, A, B, C, D, z, dt_bias, reset, h0,
                     flags & uint32_t(SS_DT_SOFTPLUS), y, h_last, nullptr, nullptr, ws, SS_STATIC_SCRATCH_BYTES, stream,
                     ConvArgs(), false);
}


int ss_segment_decay(int64_t batch, int64_t channels, int64_t state_dim, int64_t seq, ss_dtype_t dtype,
                     const void *dt_raw, const float *A, const float *dt_bias, const uint8_t *reset,
                     uint32_t flags, float *decay, ss_stream_t stream)
{
    if (!dt_raw || !A || !decay)
        return SS_ERR_NULL;
    if (batch <= 0 || channels <= 0 || state_dim <= 0 || seq <= 0)
        return SS_ERR_SHAPE;
    if (dtype != SS_F32 && dtype != SS_BF16)
        return SS_ERR_DTYPE;
    if ((state_dim != 4 && state_dim != 8 && state_dim != 16) || (flags & ~uint32_t(SS_DT_SOFTPLUS)))
        return SS_ERR_UNSUPPORTED;
    const size_t es = dtype == SS_BF16 ? 2 : 4;
    int64_t rows = 0, el = 0, st = 0, bs = 0, an = 0;
    if (!mul_ok(batch, channels, &rows) || !mul_ok(rows, seq, &el) || !mul_ok(rows, state_dim, &st) ||
        !mul_ok(batch, seq, &bs) || !mul_ok(channels, state_dim, &an) || el > INT64_MAX / 8 ||
        st > INT64_MAX / 8)
        return SS_ERR_SHAPE;
    if (!aligned(dt_raw, es) || !aligned(A, 4) || !aligned(decay, 4) || (dt_bias && !aligned(dt_bias, 4)))
        return SS_ERR_ALIGN;
    const void *in_p[] = {dt_raw, A, dt_bias, reset};
    const size_t in_n[] = {size_t(el) * es, size_t(an) * 4, dt_bias ? size_t(channels) * 4 : 0,
                           reset ? size_t(bs) : 0};
    for (int i = 0; i < 4; ++i)
        if (overlaps(decay, size_t(st) * 4, in_p[i], in_n[i]))
            return SS_ERR_ALIAS;
    ss::SegDecayArgs a{};
    a.dt = dt_raw;
    a.A = A;
    a.dt_bias = dt_bias;
    a.reset = reset;
    a.decay = decay;
    a.batch = batch;
    a.channels = channels;
    a.seq = seq;
    a.state_dim = int(state_dim);
    a.seg_len = seq;
    a.segments = 1;
    a.out_stride = 0;
    a.reset_vec = reset && aligned(reset, 16) && seq % 16 == 0;
    int sms = 0;
    if (device_sm_count(&sms) != SS_OK)
        return SS_ERR_CUDA;
    // one warp per row; at most 8 blocks of 8 warps per SM, grid-strided beyond that
    const int64_t blocks = (rows + ss::kSegWarps - 1) / ss::kSegWarps;
    const unsigned grid = unsigned(blocks < int64_t(sms) * 8 ? blocks : int64_t(sms) * 8);
    const bool vec = seq % 8 == 0 && aligned(dt_raw, 16);
    const bool sp = (flags & SS_DT_SOFTPLUS) != 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == SS_BF16)
        launch_segment_decay<__nv_bfloat16>(vec, sp, grid, a, s);
    else
        launch_segment_decay<float>(vec, sp, grid, a, s);
    return launch_status();
}

int ss_join_segments(int64_t segments, int64_t count, const float *composites, int64_t rank, float *carry,
                     float *final_state, ss_stream_t stream)
{
    if (!composites || (!carry && !final_state))
        return SS_ERR_NULL;
    if (segments <= 0 || count <= 0 || segments > 0x7fffffffLL)
        return SS_ERR_SHAPE;
    if (carry && (rank < 1 || rank >= segments))
        return SS_ERR_SHAPE;
    int64_t per = 0, total = 0;
    if (!mul_ok(count, 2, &per) || !mul_ok(per, segments, &total) || total > INT64_MAX / 4)
        return SS_ERR_SHAPE;
    if (!aligned(composites, 4) || (carry && !aligned(carry, 4)) || (final_state && !aligned(final_state, 4)))
        return SS_ERR_ALIGN;
    const size_t cb = size_t(total) * 4, ob = size_t(count) * 4;
    if (overlaps(carry, ob, composites, cb) || overlaps(final_state, ob, composites, cb) ||
        overlaps(carry, ob, final_state, ob))
        return SS_ERR_ALIAS;
    ss::JoinArgs a{};
    a.comp = composites;
    a.carry = carry;
    a.final_state = final_state;
    a.count = count;
    a.segments = int(segments);
    a.rank = carry ? int(rank) : 0;
    int sms = 0;
    if (device_sm_count(&sms) != SS_OK)
        return SS_ERR_CUDA;
    const int64_t blocks = (count + 255) / 256;
    const unsigned grid = unsigned(blocks < int64_t(sms) * 8 ? blocks : int64_t(sms) * 8);
    ss::ss_join_segments_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
    return launch_status();
}

} // extern "C"
