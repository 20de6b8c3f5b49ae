// streaming.cuh -- the weight-streaming path of the routed MoE FFN for 1..8
// rows (decode).
//
// Only the picked experts' weights are read, each exactly once for all the
// tokens that picked it, with 1-D bulk copies (cp.async.bulk) into a ring of
// shared-memory slots that a producer warp keeps full while consumer warps
// compute on CUDA cores.  Products are bf16 x bf16 (or fp32 x bf16) folded in
// fp32; the SwiGLU activations stay fp32 between the two projections.
//
// Two kernels:
//  * stream_gate_up: per (picked expert, row i of I) task, the dots of the
//    expert's W_gate and W_up rows with the x of every token that picked it,
//    then h = silu(g) * u (expertSwiGLU, fak note "GLM-5.2 multi-GPU: expert-
//    parallel sharding", "What is not yet" update).
//  * stream_down_fold: each CTA owns a contiguous slice of the H output
//    features and walks the picked experts in ascending (id, repeat) order,
//    then the shared expert, folding w * (W_down h) into one fp32 running sum
//    per (feature, token).  That walk is the bands in rank order with the
//    carry passed along (TensorFold issue #310, maintainer's reply: one fixed
//    sum order however the slices fall over ranks), so y does not depend on
//    the plan; the shared expert enters after the routed sum (the GLM shared-
//    expert wrapper of the fak note's gate table).
#pragma once

#include "common.cuh"

namespace epk {

constexpr int kStreamMaxT = 8;
constexpr int kStreamMaxK = 16;
constexpr int kStreamMaxPairs = kStreamMaxT * kStreamMaxK;

// The picks of up to 8 tokens grouped by expert, in fold order.  A group is
// one (expert, repeat) pair: a token that picks the same expert twice has its
// second pick in a second group of that expert, so a group never holds a
// token twice.
struct StreamPlan {
    int n_groups;
    int n_pairs;
    int16_t group_expert[kStreamMaxPairs];
    int16_t group_first[kStreamMaxPairs + 1];   // first pair of each group
    int8_t pair_token[kStreamMaxPairs];
    uint8_t pair_is_first[kStreamMaxPairs];     // the token's first pick in fold order
    uint8_t token_has_pick[kStreamMaxT];
    float pair_weight[kStreamMaxPairs];
    int keys[kStreamMaxPairs];
    int sorted_key[kStreamMaxPairs];
    int sorted_src[kStreamMaxPairs];
};

// Built by every CTA from ids (<= 128 picks): sort key (expert, repeat, token).
// Needs blockDim.x >= kStreamMaxPairs.  Ends with __syncthreads().
__device__ void build_stream_plan(StreamPlan &P, const int32_t *__restrict__ ids,
                                  const float *__restrict__ weights, int T, int k, int E) {
    const int tid = threadIdx.x;
    const int np = T * k;
    int key = 0x7fffffff;
    if (tid < np) {
        const int e = ids[tid];
        const int t = tid / k, j = tid - t * k;
        if (e >= 0 && e < E) {
            int rep = 0;
            for (int q = 0; q < j; ++q)
                rep += ids[t * k + q] == e;
            key = (e * kStreamMaxK + rep) * kStreamMaxT + t;
        } else {
            flag_status(kStatusBadId);
        }
    }
    if (tid < kStreamMaxPairs)
        P.keys[tid] = key;
    const int nvalid = __syncthreads_count(tid < np && key != 0x7fffffff);
    if (tid < np && key != 0x7fffffff) {
        int r = 0;
        for (int q = 0; q < np; ++q)
            r += P.keys[q] < key;
        P.sorted_key[r] = key;
        P.sorted_src[r] = tid;
    }
    __syncthreads();
    if (tid < 32) {
        const int lane = tid;
        int base = 0;
        for (int r0 = 0; r0 < nvalid; r0 += 32) {
            const int r = r0 + lane;
            const bool start = r < nvalid && (r == 0 || P.sorted_key[r] / kStreamMaxT !=
                                                            P.sorted_key[r - 1] / kStreamMaxT);
            const uint32_t m = __ballot_sync(0xffffffffu, start);
            if (start) {
                const int gid = base + __popc(m & ((1u << lane) - 1u));
                P.group_expert[gid] = (int16_t)(P.sorted_key[r] / (kStreamMaxT * kStreamMaxK));
                P.group_first[gid] = (int16_t)r;
            }
            base += __popc(m);
        }
        if (lane == 0) {
            P.n_groups = base;
            P.group_first[base] = (int16_t)nvalid;
            P.n_pairs = nvalid;
        }
    }
    if (tid < nvalid) {
        const int src = P.sorted_src[tid];
        const int t = src / k;
        P.pair_token[tid] = (int8_t)t;
        P.pair_weight[tid] = weights[src];
        bool first = true;
        for (int q = 0; q < tid; ++q)
            first &= (P.sorted_key[q] % kStreamMaxT) != t;
        P.pair_is_first[tid] = first;
    }
    if (tid < T) {
        bool has = false;
        for (int q = 0; q < nvalid; ++q)
            has |= (P.sorted_key[q] % kStreamMaxT) == tid;
        P.token_has_pick[tid] = has;
    }
    __syncthreads();
}

template <bool XF32>
__device__ __forceinline__ void x8_from_smem(const uint8_t *xs_row, int c, float (&xf)[8]) {
    if constexpr (XF32) {
        const float4 *p = reinterpret_cast<const float4 *>(xs_row) + 2 * c;
        const float4 a = p[0], b = p[1];
        xf[0] = a.x; xf[1] = a.y; xf[2] = a.z; xf[3] = a.w;
        xf[4] = b.x; xf[5] = b.y; xf[6] = b.z; xf[7] = b.w;
    } else {
        const uint4 v = reinterpret_cast<const uint4 *>(xs_row)[c];
        xf[0] = bf16_lo(v.x); xf[1] = bf16_hi(v.x); xf[2] = bf16_lo(v.y); xf[3] = bf16_hi(v.y);
        xf[4] = bf16_lo(v.z); xf[5] = bf16_hi(v.z); xf[6] = bf16_lo(v.w); xf[7] = bf16_hi(v.w);
    }
}

__device__ __forceinline__ void w8_unpack(const uint4 v, float (&wf)[8]) {
    wf[0] = bf16_lo(v.x); wf[1] = bf16_hi(v.x); wf[2] = bf16_lo(v.y); wf[3] = bf16_hi(v.y);
    wf[4] = bf16_lo(v.z); wf[5] = bf16_hi(v.z); wf[6] = bf16_lo(v.w); wf[7] = bf16_hi(v.w);
}

__host__ __device__ inline size_t align_up_sz(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------------ gate / up
constexpr int kGUConsumerWarps = 4;
constexpr int kGUThreads = 32 * (1 + kGUConsumerWarps);
constexpr int kGUMaxSlots = 8;

struct StreamGateUpArgs {
    const void *x;
    int T, H, E, I, I_s, top_k, n_slots;
    const uint16_t *w_gate, *w_up, *ws_gate, *ws_up;
    const int32_t *ids;
    const float *weights;
    float *h_routed;  // [pairs, I], pairs in plan order
    float *h_shared;  // [T, I_s]
};

struct GateUpSmem {
    size_t plan, x, slots, bars, total;
};

__host__ __device__ inline GateUpSmem gate_up_smem_layout(int T, int H, int x_bytes, int n_slots) {
    GateUpSmem s;
    size_t o = 0;
    s.plan = o;  o = align_up_sz(o + sizeof(StreamPlan), 128);
    s.x = o;     o = align_up_sz(o + (size_t)T * H * x_bytes, 128);
    s.slots = o; o = align_up_sz(o + (size_t)n_slots * 4 * H, 128);
    s.bars = o;  o = align_up_sz(o + (size_t)2 * kGUMaxSlots * 8 + 16, 128);
    s.total = o;
    return s;
}

template <bool XF32>
__global__ void __launch_bounds__(kGUThreads, 1) stream_gate_up_kernel(const StreamGateUpArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int XB = XF32 ? 4 : 2;
    const GateUpSmem L = gate_up_smem_layout(a.T, a.H, XB, a.n_slots);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + L.plan);
    uint8_t *xs = smem + L.x;
    uint8_t *slots = smem + L.slots;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + kGUMaxSlots;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kGUMaxSlots);
    const int H = a.H, I = a.I, I_s = a.I_s, NS = a.n_slots;
    const uint32_t slot_bytes = 4u * (uint32_t)H;

    build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E);
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.x);
        uint4 *dst = reinterpret_cast<uint4 *>(xs);
        const int n16 = a.T * H * XB / 16;
        for (int i = threadIdx.x; i < n16; i += blockDim.x)
            dst[i] = src[i];
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // tasks: the shared expert's rows first, then (group, row) in plan order
    const int64_t total = (int64_t)I_s + (int64_t)P.n_groups * I;
    const int64_t lo = total * blockIdx.x / gridDim.x;
    const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
    const int ntask = (int)(hi - lo);
    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();

    if (warp == 0) {
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            int issued = 0;
            for (int n = 0; n < ntask; ++n) {
                const int s = n % NS;
                if (n >= NS && !mbar_wait(&empty[s], (uint32_t)((n / NS) - 1) & 1u, abort_flag))
                    break;
                const int64_t tau = lo + n;
                const uint16_t *g, *u;
                if (tau < I_s) {
                    g = a.ws_gate + (size_t)tau * H;
                    u = a.ws_up + (size_t)tau * H;
                } else {
                    const int64_t q = tau - I_s;
                    const int grp = (int)(q / I), i = (int)(q - (int64_t)grp * I);
                    const size_t row = (size_t)P.group_expert[grp] * I + i;
                    g = a.w_gate + row * H;
                    u = a.w_up + row * H;
                }
                uint8_t *dst = slots + (size_t)s * slot_bytes;
                mbar_arrive_expect_tx(&full[s], slot_bytes);
                bulk_g2s(dst, g, 2u * H, &full[s], pol);
                bulk_g2s(dst + 2 * H, u, 2u * H, &full[s], pol);
                ++issued;
            }
            // no copy may still be writing this CTA's shared memory at exit
            for (int n = issued > NS ? issued - NS : 0; n < issued; ++n)
                mbar_wait(&full[n % NS], (uint32_t)(n / NS) & 1u, nullptr);
        }
        return;
    }

    const int c_warp = warp - 1;
    const int nck = H >> 3;
    for (int n = c_warp; n < ntask; n += kGUConsumerWarps) {
        const int s = n % NS;
        if (!mbar_wait(&full[s], (uint32_t)(n / NS) & 1u, abort_flag))
            break;
        const int64_t tau = lo + n;
        int cnt, first = 0, i;
        bool shared_task;
        if (tau < I_s) {
            shared_task = true;
            cnt = a.T;
            i = (int)tau;
        } else {
            shared_task = false;
            const int64_t q = tau - I_s;
            const int grp = (int)(q / I);
            i = (int)(q - (int64_t)grp * I);
            first = P.group_first[grp];
            cnt = P.group_first[grp + 1] - first;
        }
        int tok[kStreamMaxT];
#pragma unroll
        for (int j = 0; j < kStreamMaxT; ++j)
            tok[j] = j < cnt ? (shared_task ? j : (int)P.pair_token[first + j]) : 0;
        const uint4 *sg = reinterpret_cast<const uint4 *>(slots + (size_t)s * slot_bytes);
        const uint4 *su = reinterpret_cast<const uint4 *>(slots + (size_t)s * slot_bytes + 2 * H);
        float ga[kStreamMaxT], ua[kStreamMaxT];
#pragma unroll
        for (int j = 0; j < kStreamMaxT; ++j) { ga[j] = 0.f; ua[j] = 0.f; }
        for (int c = lane; c < nck; c += 32) {
            float gf[8], uf[8];
            w8_unpack(sg[c], gf);
            w8_unpack(su[c], uf);
#pragma unroll
            for (int j = 0; j < kStreamMaxT; ++j) {
                if (j < cnt) {
                    float xf[8];
                    x8_from_smem<XF32>(xs + (size_t)tok[j] * H * XB, c, xf);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        ga[j] = fmaf(gf[q], xf[q], ga[j]);
                        ua[j] = fmaf(uf[q], xf[q], ua[j]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);  // slot contents are in registers now
#pragma unroll
        for (int j = 0; j < kStreamMaxT; ++j) {
            if (j < cnt) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    ga[j] += __shfl_xor_sync(0xffffffffu, ga[j], off);
                    ua[j] += __shfl_xor_sync(0xffffffffu, ua[j], off);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kStreamMaxT; ++j) {
            if (j < cnt && lane == j) {
                const float h = silu_f32(ga[j]) * ua[j];
                if (shared_task)
                    a.h_shared[(size_t)j * I_s + i] = h;
                else
                    a.h_routed[(size_t)(first + j) * I + i] = h;
            }
        }
    }
}

// ------------------------------------------------------------- down + fold
constexpr int kDownConsumerWarps = 8;
constexpr int kDownRowsPerSlot = kDownConsumerWarps;
constexpr int kDownThreads = 32 * (1 + kDownConsumerWarps);
constexpr int kDownMaxSlots = 8;

struct StreamDownArgs {
    int T, H, E, I, I_s, top_k, n_slots, rows_max;
    const uint16_t *w_down, *ws_down;
    const int32_t *ids;
    const float *weights;
    const float *h_routed, *h_shared;
    float *y;
};

struct DownSmem {
    size_t plan, slots, acc, bars, total;
};

__host__ __device__ inline DownSmem down_smem_layout(int I_max, int n_slots, int rows_max) {
    DownSmem s;
    size_t o = 0;
    s.plan = o;  o = align_up_sz(o + sizeof(StreamPlan), 128);
    s.slots = o; o = align_up_sz(o + (size_t)n_slots * kDownRowsPerSlot * I_max * 2, 128);
    s.acc = o;   o = align_up_sz(o + (size_t)rows_max * kStreamMaxT * 4, 128);
    s.bars = o;  o = align_up_sz(o + (size_t)2 * kDownMaxSlots * 8 + 16, 128);
    s.total = o;
    return s;
}

__global__ void __launch_bounds__(kDownThreads, 1) stream_down_fold_kernel(const StreamDownArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int I_max = a.I > a.I_s ? a.I : a.I_s;
    const DownSmem L = down_smem_layout(I_max, a.n_slots, a.rows_max);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + L.plan);
    uint8_t *slots = smem + L.slots;
    float *yacc = reinterpret_cast<float *>(smem + L.acc);  // [row][token]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + kDownMaxSlots;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kDownMaxSlots);
    const int H = a.H, NS = a.n_slots;
    const size_t slot_bytes = (size_t)kDownRowsPerSlot * I_max * 2;

    build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDownConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int r0 = (int)((int64_t)H * blockIdx.x / gridDim.x);
    const int r1 = (int)((int64_t)H * (blockIdx.x + 1) / gridDim.x);
    const int nrows = r1 - r0;
    const int nsub = (nrows + kDownRowsPerSlot - 1) / kDownRowsPerSlot;
    const int ngroups = P.n_groups + (a.I_s > 0 ? 1 : 0);
    const int ntask = ngroups * nsub;
    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();

    if (warp == 0) {
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            int issued = 0;
            for (int n = 0; n < ntask; ++n) {
                const int s = n % NS;
                if (n >= NS && !mbar_wait(&empty[s], (uint32_t)((n / NS) - 1) & 1u, abort_flag))
                    break;
                const int gi = n / nsub, q = n - gi * nsub;
                const bool shared_task = gi >= P.n_groups;
                const int width = shared_task ? a.I_s : a.I;
                const uint16_t *mat = shared_task
                                          ? a.ws_down
                                          : a.w_down + (size_t)P.group_expert[gi] * H * a.I;
                const int row = r0 + q * kDownRowsPerSlot;
                const int nr = min(kDownRowsPerSlot, r1 - row);
                const uint32_t bytes = (uint32_t)nr * (uint32_t)width * 2u;
                mbar_arrive_expect_tx(&full[s], bytes);
                bulk_g2s(slots + (size_t)s * slot_bytes, mat + (size_t)row * width, bytes, &full[s],
                         pol);
                ++issued;
            }
            for (int n = issued > NS ? issued - NS : 0; n < issued; ++n)
                mbar_wait(&full[n % NS], (uint32_t)(n / NS) & 1u, nullptr);
        }
    } else {
        const int w = warp - 1;
        for (int n = 0; n < ntask; ++n) {
            const int s = n % NS;
            if (!mbar_wait(&full[s], (uint32_t)(n / NS) & 1u, abort_flag))
                break;
            const int gi = n / nsub, q = n - gi * nsub;
            const int rl = q * kDownRowsPerSlot + w;  // this warp's row, local to the CTA
            if (rl < nrows) {
                const bool shared_task = gi >= P.n_groups;
                const int width = shared_task ? a.I_s : a.I;
                int cnt, first = 0;
                const float *hbase;
                if (shared_task) {
                    cnt = a.T;
                    hbase = a.h_shared;
                } else {
                    first = P.group_first[gi];
                    cnt = P.group_first[gi + 1] - first;
                    hbase = a.h_routed + (size_t)first * a.I;
                }
                const uint4 *wrow = reinterpret_cast<const uint4 *>(
                    slots + (size_t)s * slot_bytes + (size_t)w * width * 2);
                float acc[kStreamMaxT];
#pragma unroll
                for (int j = 0; j < kStreamMaxT; ++j)
                    acc[j] = 0.f;
                const int nck = width >> 3;
                for (int c = lane; c < nck; c += 32) {
                    float wf[8];
                    w8_unpack(wrow[c], wf);
#pragma unroll
                    for (int j = 0; j < kStreamMaxT; ++j) {
                        if (j < cnt) {
                            const float4 *hp =
                                reinterpret_cast<const float4 *>(hbase + (size_t)j * width) + 2 * c;
                            const float4 h0 = __ldg(hp), h1 = __ldg(hp + 1);
                            acc[j] = fmaf(wf[0], h0.x, acc[j]);
                            acc[j] = fmaf(wf[1], h0.y, acc[j]);
                            acc[j] = fmaf(wf[2], h0.z, acc[j]);
                            acc[j] = fmaf(wf[3], h0.w, acc[j]);
                            acc[j] = fmaf(wf[4], h1.x, acc[j]);
                            acc[j] = fmaf(wf[5], h1.y, acc[j]);
                            acc[j] = fmaf(wf[6], h1.z, acc[j]);
                            acc[j] = fmaf(wf[7], h1.w, acc[j]);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < kStreamMaxT; ++j) {
                    if (j < cnt) {
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1)
                            acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
                    }
                }
#pragma unroll
                for (int j = 0; j < kStreamMaxT; ++j) {
                    if (j < cnt && lane == j) {
                        if (shared_task) {
                            float &ya = yacc[rl * kStreamMaxT + j];
                            ya = P.token_has_pick[j] ? ya + acc[j] : 0.0f + acc[j];
                        } else {
                            const int p = first + j;
                            const int t = P.pair_token[p];
                            const float c = P.pair_weight[p] * acc[j];
                            float &ya = yacc[rl * kStreamMaxT + t];
                            ya = P.pair_is_first[p] ? c : ya + c;
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[s]);
        }
    }
    __syncthreads();
    if (*abort_flag)
        return;
    for (int idx = threadIdx.x; idx < a.T * nrows; idx += blockDim.x) {
        const int t = idx / nrows, r = idx - t * nrows;
        const bool any = P.token_has_pick[t] || a.I_s > 0;
        a.y[(size_t)t * H + r0 + r] = any ? yacc[r * kStreamMaxT + t] : 0.0f;
    }
}

}  // namespace epk
