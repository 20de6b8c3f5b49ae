// streaming.cuh -- the weight-streaming path of the routed MoE FFN for 1..8
// rows (decode) on the CUDA cores: one token, fp32 activations, or a forced
// choice (the tensor-core kernels of decode_tc.cuh take 2..8 tokens of bf16
// activations by default).  The expert grouping (build_stream_plan) serves
// both.
//
// Only the picked experts' weights are read, each exactly once for all the
// tokens that picked it, with 1-D bulk copies (cp.async.bulk) into a ring of
// shared-memory slots that a producer warp keeps full while consumer warps
// compute with packed fp32 FMAs (fma.rn.f32x2).  Products are bf16 x bf16 (or
// fp32 x bf16) folded in fp32; the SwiGLU activations stay fp32 between the
// two projections.
//
// Two kernels:
//  * stream_gate_up: per (picked expert, unit i of I) task, the dots of the
//    expert's W_gate row and W_up row with the x of every token that picked
//    it, then h = silu(g) * u (expertSwiGLU, fak note "GLM-5.2 multi-GPU:
//    expert-parallel sharding", "What is not yet" update).  Each task's
//    inner loop is specialised on its token count (1..8).
//  * stream_down_fold: each CTA owns a contiguous slice of the H output
//    features.  It computes the shared expert's share first, then walks the
//    picked experts in ascending (id, repeat) order, folding w * (W_down h)
//    into one fp32 running sum per (feature, token); y = routed + shared.
//    The walk is the bands in rank order with the carry passed along
//    (TensorFold issue #310, maintainer's reply: the order of the sums does
//    not depend on where the slices live), so y does not depend on the plan; the
//    shared expert enters after the routed sum (the GLM shared-expert wrapper
//    of the fak note's gate table).
//
// Both kernels are launched as programmatic dependents: before
// griddepcontrol.wait they only prefetch the shared expert's weight rows
// (which no kernel writes) into their rings; every read of x, ids, routing
// weights or h, and every global write, comes after the wait.
#pragma once

#include "common.cuh"

namespace epk {

constexpr int kStreamMaxT = 8;
constexpr int kStreamMaxK = 16;
constexpr int kStreamMaxPairs = kStreamMaxT * kStreamMaxK;
constexpr int kChunkUnroll = 4;  // 16-byte chunks in flight per lane

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

// Built from ids (<= 128 picks) by `nthr` (>= 128) threads with local ids
// ltid, synchronised on named barrier `bar`; sort key (expert, repeat, token).
// Each valid pick finds its rank and whether it is its token's first pick in
// one pass over the keys, and writes its own row of the sorted tables.
__device__ void build_stream_plan(StreamPlan &P, const int32_t *__restrict__ ids,
                                  const float *__restrict__ weights, int T, int k, int E,
                                  int ltid, uint32_t nthr, uint32_t bar) {
    const int np = T * k;
    int key = 0x7fffffff, t = 0;
    float w = 0.f;
    if (ltid < np) {
        const int e = ids[ltid];
        w = weights[ltid];  // in flight with the id
        t = ltid / k;
        const int j = ltid - t * k;
        if (e >= 0 && e < E) {
            int rep = 0;
            for (int q = 0; q < j; ++q)
                rep += ids[t * k + q] == e;
            key = (e * kStreamMaxK + rep) * kStreamMaxT + t;
        } else if (e != kIdNone) {
            flag_status(kStatusBadId);
        }
    }
    if (ltid < kStreamMaxPairs)
        P.keys[ltid] = key;
    if (ltid < T)
        P.token_has_pick[ltid] = 0;
    const bool valid = ltid < np && key != 0x7fffffff;
    const int nvalid = named_count(bar, nthr, valid);
    if (valid) {
        int r = 0;
        bool first = true;  // no smaller key of the same token
#pragma unroll 4
        for (int q = 0; q < np; ++q) {
            const int kq = P.keys[q];
            const bool below = kq < key;
            r += below;
            first &= !(below && kq % kStreamMaxT == t);
        }
        P.sorted_key[r] = key;
        P.sorted_src[r] = ltid;
        P.pair_token[r] = (int8_t)t;
        P.pair_weight[r] = w;
        P.pair_is_first[r] = first;
        if (first)
            P.token_has_pick[t] = 1;
    }
    named_sync(bar, nthr);
    if (ltid < 32) {
        const int lane = ltid;
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
    named_sync(bar, nthr);
}

__host__ __device__ inline size_t align_up_sz(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Eight bf16 weights as four fp32 pairs.
__device__ __forceinline__ void w_pairs(const uint4 v, float2 (&wp)[4]) {
    wp[0] = bf16x2_to_f2(v.x);
    wp[1] = bf16x2_to_f2(v.y);
    wp[2] = bf16x2_to_f2(v.z);
    wp[3] = bf16x2_to_f2(v.w);
}

// Eight activations of 16-byte weight chunk c as four fp32 pairs, from a row
// held in shared memory as fp32 (XS_F32) or bf16.
template <bool XS_F32>
__device__ __forceinline__ void x_pairs(const uint8_t *xrow, int c, float2 (&xp)[4]) {
    if constexpr (XS_F32) {
        const float4 *p = reinterpret_cast<const float4 *>(xrow) + 2 * c;
        const float4 a = p[0], b = p[1];
        xp[0] = make_float2(a.x, a.y);
        xp[1] = make_float2(a.z, a.w);
        xp[2] = make_float2(b.x, b.y);
        xp[3] = make_float2(b.z, b.w);
    } else {
        const uint4 v = reinterpret_cast<const uint4 *>(xrow)[c];
        xp[0] = bf16x2_to_f2(v.x);
        xp[1] = bf16x2_to_f2(v.y);
        xp[2] = bf16x2_to_f2(v.z);
        xp[3] = bf16x2_to_f2(v.w);
    }
}

__device__ __forceinline__ float pair_sum(float2 a, float2 b) { return (a.x + a.y) + (b.x + b.y); }

// One gate/up task for TE tokens: the dots of the W_gate row and the W_up row
// (16-byte chunks, lane-strided, four chunks in flight per lane, two packed
// accumulators per token and row), a butterfly reduction, then lane j writes
// h = silu(g) * u of token j.
template <int TE, bool XS_F32>
__device__ __forceinline__ void gate_up_task(const uint4 *__restrict__ wg,
                                             const uint4 *__restrict__ wu, int nck,
                                             const uint8_t *xs, size_t xrow_bytes,
                                             const int (&tok)[kStreamMaxT], uint64_t *empty_bar,
                                             float *__restrict__ hout, size_t hstride) {
    const int lane = (int)lane_id();
    float2 ag[TE][2], au[TE][2];
#pragma unroll
    for (int t = 0; t < TE; ++t)
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            ag[t][b] = make_float2(0.f, 0.f);
            au[t][b] = make_float2(0.f, 0.f);
        }
    const uint8_t *xr[TE];
#pragma unroll
    for (int t = 0; t < TE; ++t)
        xr[t] = xs + (size_t)tok[t] * xrow_bytes;
    const int full_end = nck - nck % (32 * kChunkUnroll);
    int base = 0;
    for (; base < full_end; base += 32 * kChunkUnroll) {
        uint4 vg[kChunkUnroll], vu[kChunkUnroll];
#pragma unroll
        for (int q = 0; q < kChunkUnroll; ++q) {
            vg[q] = wg[base + lane + 32 * q];
            vu[q] = wu[base + lane + 32 * q];
        }
#pragma unroll
        for (int q = 0; q < kChunkUnroll; ++q) {
            const int c = base + lane + 32 * q;
            float2 gp[4], up[4];
            w_pairs(vg[q], gp);
            w_pairs(vu[q], up);
#pragma unroll
            for (int t = 0; t < TE; ++t) {
                float2 xp[4];
                x_pairs<XS_F32>(xr[t], c, xp);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    ag[t][q & 1] = ffma2(gp[p], xp[p], ag[t][q & 1]);
                    au[t][q & 1] = ffma2(up[p], xp[p], au[t][q & 1]);
                }
            }
        }
    }
    for (int c = base + lane; c < nck; c += 32) {
        float2 gp[4], up[4];
        w_pairs(wg[c], gp);
        w_pairs(wu[c], up);
#pragma unroll
        for (int t = 0; t < TE; ++t) {
            float2 xp[4];
            x_pairs<XS_F32>(xr[t], c, xp);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                ag[t][0] = ffma2(gp[p], xp[p], ag[t][0]);
                au[t][0] = ffma2(up[p], xp[p], au[t][0]);
            }
        }
    }
    __syncwarp();
    if (lane == 0)
        mbar_arrive(empty_bar);  // the slot's contents are in registers now
    float g[TE], u[TE];
#pragma unroll
    for (int t = 0; t < TE; ++t) {
        g[t] = pair_sum(ag[t][0], ag[t][1]);
        u[t] = pair_sum(au[t][0], au[t][1]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            g[t] += __shfl_xor_sync(0xffffffffu, g[t], off);
            u[t] += __shfl_xor_sync(0xffffffffu, u[t], off);
        }
    }
#pragma unroll
    for (int t = 0; t < TE; ++t)
        if (lane == t)
            hout[(size_t)t * hstride] = silu_f32(g[t]) * u[t];
}

// RW down-projection rows for TE tokens: the dots of bf16 W_down rows with the
// group's fp32 activations in shared memory; each activation chunk is loaded
// once for all RW rows.
template <int TE, int RW>
__device__ __forceinline__ void down_rows(const uint4 *__restrict__ w0, size_t row_stride16,
                                          int nck, const float *hg, int width,
                                          float (&acc)[RW][TE]) {
    const int lane = (int)lane_id();
    float2 a[RW][TE][2];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int t = 0; t < TE; ++t) {
            a[r][t][0] = make_float2(0.f, 0.f);
            a[r][t][1] = make_float2(0.f, 0.f);
        }
    const int full_end = nck - nck % (32 * kChunkUnroll);
    int base = 0;
    for (; base < full_end; base += 32 * kChunkUnroll) {
        uint4 v[RW][kChunkUnroll];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int q = 0; q < kChunkUnroll; ++q)
                v[r][q] = w0[r * row_stride16 + base + lane + 32 * q];
#pragma unroll
        for (int q = 0; q < kChunkUnroll; ++q) {
            const int c = base + lane + 32 * q;
            float2 wp[RW][4];
#pragma unroll
            for (int r = 0; r < RW; ++r)
                w_pairs(v[r][q], wp[r]);
#pragma unroll
            for (int t = 0; t < TE; ++t) {
                const float4 *hp = reinterpret_cast<const float4 *>(hg + (size_t)t * width) + 2 * c;
                const float4 h0 = hp[0], h1 = hp[1];
                const float2 hx[4] = {make_float2(h0.x, h0.y), make_float2(h0.z, h0.w),
                                      make_float2(h1.x, h1.y), make_float2(h1.z, h1.w)};
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        a[r][t][q & 1] = ffma2(wp[r][p], hx[p], a[r][t][q & 1]);
            }
        }
    }
    for (int c = base + lane; c < nck; c += 32) {
        float2 wp[RW][4];
#pragma unroll
        for (int r = 0; r < RW; ++r)
            w_pairs(w0[r * row_stride16 + c], wp[r]);
#pragma unroll
        for (int t = 0; t < TE; ++t) {
            const float4 *hp = reinterpret_cast<const float4 *>(hg + (size_t)t * width) + 2 * c;
            const float4 h0 = hp[0], h1 = hp[1];
            const float2 hx[4] = {make_float2(h0.x, h0.y), make_float2(h0.z, h0.w),
                                  make_float2(h1.x, h1.y), make_float2(h1.z, h1.w)};
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    a[r][t][0] = ffma2(wp[r][p], hx[p], a[r][t][0]);
        }
    }
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int t = 0; t < TE; ++t) {
            acc[r][t] = pair_sum(a[r][t][0], a[r][t][1]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                acc[r][t] += __shfl_xor_sync(0xffffffffu, acc[r][t], off);
        }
}

// ------------------------------------------------------------------ gate / up
constexpr int kGUConsumerWarps = 8;
constexpr int kGUThreads = 32 * (1 + kGUConsumerWarps);
constexpr int kGUMaxSlots = 16;
constexpr uint32_t kGUBarPlan = 1;  // named barrier of the 256 consumer threads

struct StreamGateUpArgs {
    const void *x;
    int T, H, E, I, I_s, top_k, n_slots;
    const uint16_t *w_gate, *w_up, *ws_gate, *ws_up;
    const int32_t *ids;
    const float *weights;
    float *h_routed;  // [pairs, I], pairs in plan order
    float *h_shared;  // [T, I_s]
};

// Consumer warps of the gate/up kernel for NS slots: the most, up to
// kGUConsumerWarps, that divide NS (task n goes to warp n % A and slot n % NS).
__host__ __device__ inline int gate_up_consumers(int NS) {
    for (int a = kGUConsumerWarps; a > 1; --a)
        if (NS % a == 0)
            return a;
    return 1;
}

struct GateUpSmem {
    size_t plan, x, slots, bars, total;
};

// xs_bytes: bytes per activation in shared memory (4: fp32, 2: bf16)
__host__ __device__ inline GateUpSmem gate_up_smem_layout(int T, int H, int xs_bytes, int n_slots) {
    GateUpSmem s;
    size_t o = 0;
    s.plan = o;  o = align_up_sz(o + sizeof(StreamPlan), 128);
    s.x = o;     o = align_up_sz(o + (size_t)T * H * xs_bytes, 128);
    s.slots = o; o = align_up_sz(o + (size_t)n_slots * 4 * H, 128);
    s.bars = o;  o = align_up_sz(o + (size_t)(2 * kGUMaxSlots + 2) * 8 + 16, 128);
    s.total = o;
    return s;
}

// XIN_F32: x is fp32 in global memory; XS_F32: x is held as fp32 in shared
// memory (converted from bf16 when XIN_F32 is false).
template <bool XIN_F32, bool XS_F32>
__global__ void __launch_bounds__(kGUThreads, 1) stream_gate_up_kernel(const StreamGateUpArgs a) {
    static_assert(XS_F32 || !XIN_F32, "fp32 activations stay fp32");
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int XSB = XS_F32 ? 4 : 2;
    const GateUpSmem L = gate_up_smem_layout(a.T, a.H, XSB, a.n_slots);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + L.plan);
    uint8_t *xs = smem + L.x;
    uint8_t *slots = smem + L.slots;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + kGUMaxSlots;
    uint64_t *xbar = empty + kGUMaxSlots;
    uint64_t *planbar = xbar + 1;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(planbar + 1);
    const int H = a.H, I = a.I, I_s = a.I_s, NS = a.n_slots;
    const uint32_t slot_bytes = 4u * (uint32_t)H;
    const int warp = (int)(threadIdx.x >> 5);
    constexpr bool kBulkX = XIN_F32 == XS_F32;  // x lands in shared memory as stored

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(xbar, 1);
        mbar_init(planbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    grid_dependents_launch();

    // shared-expert rows [s_lo, s_hi) first, then routed (group, unit) tasks
    const int64_t G = gridDim.x, c = blockIdx.x;
    const int64_t s_lo = (int64_t)I_s * c / G, s_hi = (int64_t)I_s * (c + 1) / G;
    const int n_shared = (int)(s_hi - s_lo);

    if (warp == 0) {
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            int issued = 0;
            int ntask = n_shared;        // grows once the plan is known
            bool have_plan = false;
            int64_t r_lo = 0;
            for (int n = 0; n < ntask || !have_plan; ++n) {
                if (n >= n_shared && !have_plan) {
                    // routed tasks need the plan the consumers build
                    if (!mbar_wait(planbar, 0, abort_flag))
                        break;
                    have_plan = true;
                    const int64_t R = (int64_t)P.n_groups * I;
                    r_lo = R * c / G;
                    ntask = n_shared + (int)(R * (c + 1) / G - r_lo);
                    if (n >= ntask)
                        break;
                }
                const int s = n % NS;
                if (n >= NS && !mbar_wait(&empty[s], (uint32_t)((n / NS) - 1) & 1u, abort_flag))
                    break;
                const uint16_t *g, *u;
                if (n < n_shared) {
                    const int64_t row = s_lo + n;
                    g = a.ws_gate + (size_t)row * H;
                    u = a.ws_up + (size_t)row * H;
                } else {
                    const int64_t q = r_lo + (n - n_shared);
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
            if (kBulkX)
                mbar_wait(xbar, 0, nullptr);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int ltid = (int)threadIdx.x - 32;
    const int w = warp - 1;
    grid_dependency_wait();  // ids, weights and x may come from the previous kernel
    if (kBulkX) {
        if (ltid == 0) {
            const uint32_t xbytes = (uint32_t)(a.T * H * XSB);
            mbar_arrive_expect_tx(xbar, xbytes);
            bulk_g2s(xs, a.x, xbytes, xbar, policy_evict_last());
        }
    } else {
        // bf16 x widened to fp32 on the way in (exact)
        const uint4 *src = reinterpret_cast<const uint4 *>(a.x);
        float4 *dst = reinterpret_cast<float4 *>(xs);
        const int n16 = a.T * H / 8;
        for (int i = ltid; i < n16; i += 32 * kGUConsumerWarps) {
            const uint4 v = src[i];
            dst[2 * i] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
            dst[2 * i + 1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
        }
    }
    // (the plan's closing barrier also publishes the widened x)
    build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E, ltid, 32 * kGUConsumerWarps,
                      kGUBarPlan);
    if (ltid == 0)
        mbar_arrive(planbar);
    const int64_t R = (int64_t)P.n_groups * I;
    const int64_t r_lo = R * c / G;
    const int ntask = n_shared + (int)(R * (c + 1) / G - r_lo);
    if (kBulkX && !mbar_wait(xbar, 0, abort_flag))
        return;

    // Task n uses slot n % NS and goes to consumer warp n % A, where A
    // divides NS: every slot then has one consumer, which waits for the
    // slot's phases in order.  (Were a slot shared by two warps, one could
    // wait for phase k + 1 while phase k is still in flight, and the parity
    // test would pass at once on the stale phase.)
    // (the host sizes NS so that such an A of several warps exists)
    const int A = gate_up_consumers(NS);
    const int nck = H >> 3;
    const size_t xrow_bytes = (size_t)H * XSB;
    for (int n = w; w < A && n < ntask; n += A) {
        const int s = n % NS;
        if (!mbar_wait(&full[s], (uint32_t)(n / NS) & 1u, abort_flag))
            break;
        int cnt, first = 0;
        float *hout;
        size_t hstride;
        bool shared_task = n < n_shared;
        if (shared_task) {
            cnt = a.T;
            hout = a.h_shared + (s_lo + n);
            hstride = (size_t)I_s;
        } else {
            const int64_t q = r_lo + (n - n_shared);
            const int grp = (int)(q / I);
            const int i = (int)(q - (int64_t)grp * I);
            first = P.group_first[grp];
            cnt = P.group_first[grp + 1] - first;
            hout = a.h_routed + (size_t)first * I + i;
            hstride = (size_t)I;
        }
        int tok[kStreamMaxT];
#pragma unroll
        for (int j = 0; j < kStreamMaxT; ++j)
            tok[j] = j < cnt ? (shared_task ? j : (int)P.pair_token[first + j]) : 0;
        const uint4 *wg = reinterpret_cast<const uint4 *>(slots + (size_t)s * slot_bytes);
        const uint4 *wu = reinterpret_cast<const uint4 *>(slots + (size_t)s * slot_bytes + 2 * H);
        switch (cnt) {
        case 1: gate_up_task<1, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        case 2: gate_up_task<2, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        case 3: gate_up_task<3, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        case 4: gate_up_task<4, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        case 5: gate_up_task<5, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        case 6: gate_up_task<6, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        case 7: gate_up_task<7, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        default: gate_up_task<8, XS_F32>(wg, wu, nck, xs, xrow_bytes, tok, &empty[s], hout, hstride); break;
        }
    }
}

// ------------------------------------------------------------- down + fold
constexpr int kDownConsumerWarps = 8;
constexpr int kDownMaxRowsPerWarp = 2;
constexpr int kDownThreads = 32 * (1 + kDownConsumerWarps);
constexpr int kDownMaxSlots = 8;
constexpr int kDownHGroups = 8;  // groups whose activations may be in the arena at once
constexpr uint32_t kDownBarPlan = 1;

struct StreamDownArgs {
    int T, H, E, I, I_s, top_k, n_slots, rows_max;
    int rw;  // rows per consumer warp per slot (1 or 2)
    int h_arena;  // bytes of the h arena, >= T * max(I, I_s) * 4
    const uint16_t *w_down, *ws_down;
    const int32_t *ids;
    const float *weights;
    const float *h_routed, *h_shared;
    float *y;
};

struct DownSmem {
    size_t plan, hbuf, slots, acc, sacc, bars, total;
};

// The h arena holds the activations of the groups in flight, each group's
// rows (count x width fp32) contiguous at a 128-byte boundary.
__host__ __device__ inline DownSmem down_smem_layout(int T, int I_max, int n_slots, int rows_max,
                                                    int rw, size_t h_arena) {
    DownSmem s;
    size_t o = 0;
    (void)T;
    (void)I_max;
    s.plan = o;  o = align_up_sz(o + sizeof(StreamPlan), 128);
    s.hbuf = o;  o = align_up_sz(o + h_arena, 128);
    s.slots = o; o = align_up_sz(o + (size_t)n_slots * kDownConsumerWarps * rw * I_max * 2, 128);
    s.acc = o;   o = align_up_sz(o + (size_t)rows_max * kStreamMaxT * 4, 128);
    s.sacc = o;  o = align_up_sz(o + (size_t)rows_max * kStreamMaxT * 4, 128);
    s.bars = o;
    o = align_up_sz(o + (size_t)(2 * kDownMaxSlots + 2 * kDownHGroups + 1) * 8 +
                        (size_t)kDownHGroups * 4 + 16, 128);
    s.total = o;
    return s;
}

// What a consumer warp needs to walk one group's slots.
struct DownGroup {
    const StreamPlan *P;
    uint8_t *slots;
    size_t slot_bytes;
    uint64_t *full, *empty, *hempty;
    volatile int *abort_flag;
    float *yacc, *sacc;
    const float *hg;
    int NS, nsub, rows_per_slot, nrows, w, gi, width, cnt, first, rw;
    bool shared_group;
};

// The values of one row for the group's tokens (lane j holds token j's)
// folded into the per-(row, token) accumulators.
template <int TE>
__device__ __forceinline__ void fold_row(const DownGroup &g, int rl, const float (&v)[TE]) {
    const int lane = (int)lane_id();
#pragma unroll
    for (int j = 0; j < TE; ++j) {
        if (lane == j) {
            if (g.shared_group) {
                g.sacc[rl * kStreamMaxT + j] = v[j];
            } else {
                const int p = g.first + j;
                const int t = g.P->pair_token[p];
                const float cval = g.P->pair_weight[p] * v[j];
                float &ya = g.yacc[rl * kStreamMaxT + t];
                ya = g.P->pair_is_first[p] ? cval : ya + cval;
            }
        }
    }
}

// One row for TE tokens whose activations sit in registers: lane l holds
// chunks c = l + 32 i (i < NCL) of every token.
template <int TE, int NCL>
__device__ __forceinline__ void down_row_reg(const uint4 *__restrict__ wrow,
                                             const float2 (&hr)[TE][NCL][4], float (&acc)[TE]) {
    const int lane = (int)lane_id();
    float2 a[TE][2];
#pragma unroll
    for (int t = 0; t < TE; ++t) {
        a[t][0] = make_float2(0.f, 0.f);
        a[t][1] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < NCL; ++i) {
        float2 wp[4];
        w_pairs(wrow[lane + 32 * i], wp);
#pragma unroll
        for (int t = 0; t < TE; ++t)
#pragma unroll
            for (int p = 0; p < 4; ++p)
                a[t][i & 1] = ffma2(wp[p], hr[t][i][p], a[t][i & 1]);
    }
#pragma unroll
    for (int t = 0; t < TE; ++t) {
        acc[t] = pair_sum(a[t][0], a[t][1]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    }
}

// A group of TE (1, or 2 when NCL <= 6) tokens with width = 256 NCL: each warp
// copies its slice of h into registers once, then walks the group's slots.
// The h buffer is freed only after the group's last slot: an arrive does not
// wait for shared-memory loads still in flight, and the next group's h is
// written by a bulk copy (the async proxy), so freeing it right after the
// loads let that copy overwrite values not yet read.  Returns false when a
// wait gave up.
template <int TE, int NCL>
__device__ bool down_group_reg(const DownGroup &g) {
    const int lane = (int)lane_id();
    float2 hr[TE][NCL][4];
#pragma unroll
    for (int t = 0; t < TE; ++t)
#pragma unroll
        for (int i = 0; i < NCL; ++i) {
            const float4 *hp =
                reinterpret_cast<const float4 *>(g.hg + (size_t)t * g.width) + 2 * (lane + 32 * i);
            const float4 h0 = hp[0], h1 = hp[1];
            hr[t][i][0] = make_float2(h0.x, h0.y);
            hr[t][i][1] = make_float2(h0.z, h0.w);
            hr[t][i][2] = make_float2(h1.x, h1.y);
            hr[t][i][3] = make_float2(h1.z, h1.w);
        }
    const size_t stride16 = (size_t)kDownConsumerWarps * g.width / 8;
    for (int q = 0; q < g.nsub; ++q) {
        const int n = g.gi * g.nsub + q;
        const int s = n % g.NS;
        if (!mbar_wait(&g.full[s], (uint32_t)(n / g.NS) & 1u, g.abort_flag))
            return false;
        const int rl0 = q * g.rows_per_slot + g.w;
        const int nmine =
            rl0 >= g.nrows ? 0 : (g.rw == 2 && rl0 + kDownConsumerWarps < g.nrows ? 2 : 1);
        const uint4 *wrow =
            reinterpret_cast<const uint4 *>(g.slots + (size_t)s * g.slot_bytes + (size_t)g.w * g.width * 2);
        float acc0[TE], acc1[TE];
        if (nmine >= 1)
            down_row_reg<TE, NCL>(wrow, hr, acc0);
        if (nmine == 2)
            down_row_reg<TE, NCL>(wrow + stride16, hr, acc1);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&g.empty[s]);
        if (nmine >= 1)
            fold_row<TE>(g, rl0, acc0);
        if (nmine == 2)
            fold_row<TE>(g, rl0 + kDownConsumerWarps, acc1);
    }
    __syncwarp();
    if (lane == 0)
        mbar_arrive(g.hempty);
    return true;
}

// Any other group: h is read from shared memory for every row; the h
// buffer is freed after the group's last slot.
template <int TE>
__device__ bool down_group_smem(const DownGroup &g) {
    const int lane = (int)lane_id();
    const int nck = g.width >> 3;
    const size_t stride16 = (size_t)kDownConsumerWarps * g.width / 8;
    bool ok = true;
    for (int q = 0; q < g.nsub; ++q) {
        const int n = g.gi * g.nsub + q;
        const int s = n % g.NS;
        if (!mbar_wait(&g.full[s], (uint32_t)(n / g.NS) & 1u, g.abort_flag)) {
            ok = false;
            break;
        }
        const int rl0 = q * g.rows_per_slot + g.w;
        const int nmine =
            rl0 >= g.nrows ? 0 : (g.rw == 2 && rl0 + kDownConsumerWarps < g.nrows ? 2 : 1);
        const uint4 *wrow =
            reinterpret_cast<const uint4 *>(g.slots + (size_t)s * g.slot_bytes + (size_t)g.w * g.width * 2);
        if (nmine == 2) {
            float acc[2][TE];
            down_rows<TE, 2>(wrow, stride16, nck, g.hg, g.width, acc);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&g.empty[s]);
            fold_row<TE>(g, rl0, acc[0]);
            fold_row<TE>(g, rl0 + kDownConsumerWarps, acc[1]);
        } else if (nmine == 1) {
            float acc[1][TE];
            down_rows<TE, 1>(wrow, stride16, nck, g.hg, g.width, acc);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&g.empty[s]);
            fold_row<TE>(g, rl0, acc[0]);
        } else {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&g.empty[s]);
        }
    }
    __syncwarp();
    if (lane == 0)
        mbar_arrive(g.hempty);
    return ok;
}

__device__ __forceinline__ bool down_group(const DownGroup &g) {
    // small groups keep h in registers, the rest read it from shared memory
    const int ncl = (g.width % 256 == 0) ? g.width / 256 : 0;
    if (g.cnt == 1 && (ncl == 4 || ncl == 6 || ncl == 8))
        return ncl == 4 ? down_group_reg<1, 4>(g)
                        : (ncl == 6 ? down_group_reg<1, 6>(g) : down_group_reg<1, 8>(g));
    if (g.cnt == 2 && (ncl == 4 || ncl == 6))
        return ncl == 4 ? down_group_reg<2, 4>(g) : down_group_reg<2, 6>(g);
    switch (g.cnt) {
    case 1: return down_group_smem<1>(g);
    case 2: return down_group_smem<2>(g);
    case 3: return down_group_smem<3>(g);
    case 4: return down_group_smem<4>(g);
    case 5: return down_group_smem<5>(g);
    case 6: return down_group_smem<6>(g);
    case 7: return down_group_smem<7>(g);
    default: return down_group_smem<8>(g);
    }
}

__global__ void __launch_bounds__(kDownThreads, 1) stream_down_fold_kernel(const StreamDownArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int I_max = a.I > a.I_s ? a.I : a.I_s;
    const DownSmem L = down_smem_layout(a.T, I_max, a.n_slots, a.rows_max, a.rw,
                                        (size_t)a.h_arena);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + L.plan);
    float *hbuf = reinterpret_cast<float *>(smem + L.hbuf);   // the h arena
    uint8_t *slots = smem + L.slots;
    float *yacc = reinterpret_cast<float *>(smem + L.acc);    // routed fold [row][token]
    float *sacc = reinterpret_cast<float *>(smem + L.sacc);   // shared expert [row][token]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + kDownMaxSlots;
    uint64_t *hfull = empty + kDownMaxSlots;      // [kDownHGroups]
    uint64_t *hempty = hfull + kDownHGroups;      // [kDownHGroups]
    uint64_t *planbar = hempty + kDownHGroups;
    int *hoff = reinterpret_cast<int *>(planbar + 1);  // [kDownHGroups] arena offsets (floats)
    volatile int *abort_flag = reinterpret_cast<volatile int *>(hoff + kDownHGroups);
    const int H = a.H, NS = a.n_slots;
    constexpr int HK = kDownHGroups;
    const int HA = a.h_arena / 4;  // arena capacity in floats
    const int rows_per_slot = kDownConsumerWarps * a.rw;
    const size_t slot_bytes = (size_t)rows_per_slot * I_max * 2;
    const int warp = (int)(threadIdx.x >> 5);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDownConsumerWarps);
        }
        for (int b = 0; b < HK; ++b) {
            mbar_init(&hfull[b], 1);
            mbar_init(&hempty[b], kDownConsumerWarps);
        }
        mbar_init(planbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    grid_dependents_launch();

    const int r0 = (int)((int64_t)H * blockIdx.x / gridDim.x);
    const int r1 = (int)((int64_t)H * (blockIdx.x + 1) / gridDim.x);
    const int nrows = r1 - r0;
    const int nsub = (nrows + rows_per_slot - 1) / rows_per_slot;
    const int has_shared = a.I_s > 0 ? 1 : 0;

    if (warp == 0) {
        if (elect_one()) {
            const uint64_t pol = policy_evict_first();
            const uint64_t pol_h = policy_evict_last();
            int issued = 0, h_issued = 0;
            bool waited = false;
            // arena ring: the live groups [g_old, h_issued) occupy [head, tail),
            // or [head, HA) and [0, tail) once wrapped
            int g_old = 0, head = 0, tail = 0;
            bool wrapped = false;
            int ngroups = has_shared;  // the routed groups are added once the plan is known
            bool have_plan = false;
            bool stop = false;
            for (int gi = 0; (gi < ngroups || !have_plan) && !stop; ++gi) {
                if (gi >= has_shared && !have_plan) {
                    if (!mbar_wait(planbar, 0, abort_flag))
                        break;
                    have_plan = true;
                    ngroups = has_shared + P.n_groups;
                    if (gi >= ngroups)
                        break;
                }
                const bool shared_group = gi < has_shared;
                const int width = shared_group ? a.I_s : a.I;
                const uint16_t *mat;
                const float *hsrc;
                uint32_t hbytes;
                if (shared_group) {
                    mat = a.ws_down;
                    hsrc = a.h_shared;
                    hbytes = (uint32_t)(a.T * a.I_s * 4);
                } else {
                    const int g = gi - has_shared;
                    mat = a.w_down + (size_t)P.group_expert[g] * H * a.I;
                    const int first = P.group_first[g];
                    hsrc = a.h_routed + (size_t)first * a.I;
                    hbytes = (uint32_t)((P.group_first[g + 1] - first) * a.I * 4);
                }
                // the first group's weights are prefetched into the empty ring
                // before its activations can be waited for
                const int q_h = gi == 0 ? min(nsub, NS) - 1 : 0;
                for (int q = 0; q < nsub; ++q) {
                    const int n = gi * nsub + q;
                    const int s = n % NS;
                    if (n >= NS && !mbar_wait(&empty[s], (uint32_t)((n / NS) - 1) & 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    const int row = r0 + q * rows_per_slot;
                    const int nr = min(rows_per_slot, r1 - row);
                    const uint32_t bytes = (uint32_t)nr * (uint32_t)width * 2u;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    bulk_g2s(slots + (size_t)s * slot_bytes, mat + (size_t)row * width, bytes,
                             &full[s], pol);
                    ++issued;
                    if (q == q_h) {
                        // this group's activations (written by the previous kernel)
                        if (!waited) {
                            grid_dependency_wait();
                            waited = true;
                        }
                        // a contiguous place in the arena, freeing the oldest
                        // groups (in order) until one exists
                        const int need = (int)((hbytes / 4 + 31) & ~31u);
                        int off = -1;
                        for (;;) {
                            if (g_old == gi) {
                                head = tail = 0;
                                wrapped = false;
                            }
                            if (gi - g_old < HK) {
                                if (!wrapped) {
                                    if (tail + need <= HA) {
                                        off = tail;
                                    } else if (need <= head) {
                                        off = 0;
                                        wrapped = true;
                                    }
                                } else if (tail + need <= head) {
                                    off = tail;
                                }
                                if (off >= 0)
                                    break;
                            }
                            if (!mbar_wait(&hempty[g_old % HK], (uint32_t)(g_old / HK) & 1u,
                                           abort_flag)) {
                                stop = true;
                                break;
                            }
                            ++g_old;
                            if (g_old < gi) {
                                head = hoff[g_old % HK];
                                wrapped = head >= tail;
                            }
                        }
                        if (stop)
                            break;
                        tail = off + need;
                        const int hb = gi % HK;
                        hoff[hb] = off;
                        mbar_arrive_expect_tx(&hfull[hb], hbytes);
                        bulk_g2s(hbuf + off, hsrc, hbytes, &hfull[hb], pol_h);
                        ++h_issued;
                    }
                }
            }
            for (int n = issued > NS ? issued - NS : 0; n < issued; ++n)
                mbar_wait(&full[n % NS], (uint32_t)(n / NS) & 1u, nullptr);
            for (int n = h_issued > HK ? h_issued - HK : 0; n < h_issued; ++n)
                mbar_wait(&hfull[n % HK], (uint32_t)(n / HK) & 1u, nullptr);
        }
    } else {
        const int ltid = (int)threadIdx.x - 32;
        // ids and weights are read only after griddepcontrol.wait: the
        // gate/up kernel lets this one start early, possibly while the kernel
        // that wrote the ids (the router) is still running
        grid_dependency_wait();
        build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E, ltid, 32 * kDownConsumerWarps,
                          kDownBarPlan);
        if (ltid == 0)
            mbar_arrive(planbar);
        DownGroup g;
        g.P = &P;
        g.slots = slots;
        g.slot_bytes = slot_bytes;
        g.full = full;
        g.empty = empty;
        g.abort_flag = abort_flag;
        g.yacc = yacc;
        g.sacc = sacc;
        g.NS = NS;
        g.nsub = nsub;
        g.rows_per_slot = rows_per_slot;
        g.nrows = nrows;
        g.w = warp - 1;
        g.rw = a.rw;
        const int ngroups = has_shared + P.n_groups;
        for (int gi = 0; gi < ngroups; ++gi) {
            g.gi = gi;
            g.shared_group = gi < has_shared;
            g.width = g.shared_group ? a.I_s : a.I;
            if (g.shared_group) {
                g.cnt = a.T;
                g.first = 0;
            } else {
                const int grp = gi - has_shared;
                g.first = P.group_first[grp];
                g.cnt = P.group_first[grp + 1] - g.first;
            }
            if (!mbar_wait(&hfull[gi % HK], (uint32_t)(gi / HK) & 1u, abort_flag))
                break;
            g.hg = hbuf + hoff[gi % HK];
            g.hempty = &hempty[gi % HK];
            if (!down_group(g))
                break;
        }
    }
    __syncthreads();
    if (*abort_flag)
        return;
    // y = routed fold + shared expert; a token with no routed pick gets 0 + s
    for (int idx = threadIdx.x; idx < a.T * nrows; idx += blockDim.x) {
        const int t = idx / nrows, r = idx - t * nrows;
        const float routed = P.token_has_pick[t] ? yacc[r * kStreamMaxT + t] : 0.0f;
        a.y[(size_t)t * H + r0 + r] = has_shared ? routed + sacc[r * kStreamMaxT + t] : routed;
    }
}

}  // namespace epk
