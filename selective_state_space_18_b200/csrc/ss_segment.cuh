// ss_segment.cuh -- joining a sequence that was cut into segments scanned apart.
//
// The recurrence h_t = a_t * h_{t-1} + u_t composes associatively ("s6_reset" blog
// draft, Associative Boundary Resetting: pairs (a, u) combine as
// (a_i, u_i) o (a_j, u_j) = (a_i a_j, a_j u_i + u_j), and a reset inside a segment
// makes it discard the state that enters it).  A whole segment therefore acts on
// its entering state as one map h -> decay * h + state, where
//
//   decay = prod_t exp(dt_t * A[c,n]) = exp(A[c,n] * sum_t dt_t), or 0 when the
//           segment holds a reset for its batch row;
//   state = the segment's end state entered from zero (a plain scan's h_last).
//
// Two kernels live here: the decay of one segment (the state comes from the scan
// kernel itself), and the join of gathered composites into the state that enters
// a given segment.  Both are small next to the scan: the first reads dt once (HBM
// bound, 2 or 4 bytes per (b, c, t)), the second touches 2 floats per segment and
// state element.
#pragma once

#include "ss_device.cuh"

namespace ss {

struct SegDecayArgs {
    const void *dt;          // [batch, channels, seq] T
    const float *A;          // [channels, state_dim]
    const float *dt_bias;    // [channels] or null
    const uint8_t *reset;    // [batch, seq] or null
    float *decay;            // [segments][batch, channels, state_dim], out_stride apart
    int64_t batch, channels, seq;
    int64_t seg_len;         // tokens per segment (a multiple of 32; seq for one segment)
    int64_t segments;        // ceil(seq / seg_len)
    int64_t out_stride;      // floats between the decays of consecutive segments
    int state_dim;
    int reset_vec;           // reset rows are 16-byte aligned and seq % 16 == 0
};

constexpr int kSegWarps = 8;
constexpr int kSegBatch = 8; // 16-byte loads in flight per lane (a 2048-token bf16 row in one round trip)

// One warp per (b, c) row and segment, grid-strided: the lanes sum the segment's
// step sizes (8 elements per 16-byte vector when VEC), OR the batch row's reset flags
// in the segment, reduce across the warp, and lanes n < state_dim write
// exp2(A log2(e) sum).  SP: the step is softplus(dt_raw + dt_bias), computed exactly as
// the prompt scan's producers compute it (the same polynomial, packed two tokens at a
// time).
template <typename T, bool VEC, bool SP>
__global__ void __launch_bounds__(kSegWarps * 32) ss_segment_decay_kernel(SegDecayArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t items = a.batch * a.channels * a.segments;
    const int64_t stride = int64_t(gridDim.x) * kSegWarps;
    for (int64_t item = int64_t(blockIdx.x) * kSegWarps + (threadIdx.x >> 5); item < items; item += stride) {
        const int64_t row = item / a.segments, s = item - row * a.segments;
        const int64_t b = row / a.channels, c = row - b * a.channels;
        const int64_t t_begin = s * a.seg_len;
        const int64_t t_end = t_begin + a.seg_len < a.seq ? t_begin + a.seg_len : a.seq;
        const T *dr = static_cast<const T *>(a.dt) + row * a.seq;
        const float bias = a.dt_bias ? __ldg(a.dt_bias + c) : 0.0f;
        float sum = 0.0f;
        if (VEC) {
            // seq and the segment start are multiples of 8, so each vector lies wholly
            // inside the segment or wholly past it.  The loads of a batch are all
            // issued before any of them is used, so each lane keeps kSegBatch 16-byte
            // loads in flight.
            float2 acc = make_float2(0.0f, 0.0f);
            for (int64_t t0 = t_begin + int64_t(lane) * 8; t0 < t_end; t0 += 256 * kSegBatch) {
                Raw8<T> v[kSegBatch];
#pragma unroll
                for (int i = 0; i < kSegBatch; ++i)
                    v[i].load_vec_stream(dr, t0 + 256 * i, t_end);
#pragma unroll
                for (int i = 0; i < kSegBatch; ++i) {
                    if (t0 + 256 * i >= t_end)
                        break;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 r = __fadd2_rn(make_float2(v[i].get(2 * k), v[i].get(2 * k + 1)),
                                                    make_float2(bias, bias));
                        acc = __fadd2_rn(acc, SP ? softplus_poly2(r) : r);
                    }
                }
            }
            sum = acc.x + acc.y;
        } else {
#pragma unroll 8
            for (int64_t t = t_begin + lane; t < t_end; t += 32) {
                const float r = Elem<T>::load(dr + t) + bias;
                sum += SP ? softplus_poly(r) : r;
            }
        }
        uint32_t any = 0;
        if (a.reset) {
            const uint8_t *rr = a.reset + b * a.seq;
            if (a.reset_vec) { // (segment starts are multiples of 16 as well)
                for (int64_t t = t_begin + int64_t(lane) * 16; t < t_end; t += 512) {
                    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(rr + t));
                    any |= w.x | w.y | w.z | w.w;
                }
            } else {
                for (int64_t t = t_begin + lane; t < t_end; t += 32)
                    any |= __ldg(rr + t);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const bool discard = __any_sync(0xffffffffu, any != 0);
        if (lane < a.state_dim) {
            const float An = __ldg(a.A + c * a.state_dim + lane);
            a.decay[s * a.out_stride + row * a.state_dim + lane] = discard ? 0.0f : ex2(An * kLog2e * sum);
        }
    }
}

struct JoinArgs {
    const float *comp;  // [segments][2][count]: decay then end state of each segment
    float *carry;       // [count] or null: the state entering segment `rank`
    float *final_state; // [count] or null: the state after the last segment
    int64_t count;
    int segments, rank;
};

// Element-wise fold of the composites in segment order.  Segment 0 was scanned from
// the true initial state, so its end state starts the fold and its decay is unread.
__global__ void __launch_bounds__(256) ss_join_segments_kernel(JoinArgs a)
{
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.count; i += stride) {
        float h = __ldg(a.comp + a.count + i);
        for (int s = 1; s < a.segments; ++s) {
            if (s == a.rank && a.carry)
                a.carry[i] = h;
            const float *cs = a.comp + int64_t(2 * s) * a.count;
            h = fmaf(__ldg(cs + i), h, __ldg(cs + a.count + i));
        }
        if (a.final_state)
            a.final_state[i] = h;
    }
}

struct JoinAllArgs {
    const float *decay; // [segments][count]
    const float *state; // [segments][count]: each segment's end state entered from zero
    const float *h0;    // [count] or null (zeros): the state entering segment 0
    float *h_in;        // [segments][count]: the state entering each segment
    float *h_last;      // [count] or null: the state after the last segment
    int64_t count;
    int64_t segments;
};

// Element-wise fold of every segment's composite in order, keeping each entering
// state: h_in[0] = h0, h_in[s + 1] = decay[s] h_in[s] + state[s].  (The in-GPU
// two-level scan: the segments' composites are computed in parallel, this joins them,
// and each segment is then rescanned from its entering state.)
__global__ void __launch_bounds__(256) ss_join_all_kernel(JoinAllArgs a)
{
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.count; i += stride) {
        float h = a.h0 ? __ldg(a.h0 + i) : 0.0f;
        for (int64_t s = 0; s < a.segments; ++s) {
            a.h_in[s * a.count + i] = h;
            h = fmaf(__ldg(a.decay + s * a.count + i), h, __ldg(a.state + s * a.count + i));
        }
        if (a.h_last)
            a.h_last[i] = h;
    }
}

} // namespace ss
