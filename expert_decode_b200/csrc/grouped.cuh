// grouped.cuh -- the tensor-core path of the routed MoE FFN (more than 8 rows).
//
//  1. group_plan    (one CTA): the picks grouped by expert with a warp-level
//                   histogram (__match_any_sync) and prefix scans; a stable
//                   scatter keeps each expert's rows in (token, slot) order.
//                   The fak note "GLM-5.2 multi-GPU" batches its expert
//                   dispatch the same way (hostBatchedGLMExperts: each
//                   expert runs once over the rows that picked it).
//  2. gather_rows:  the picked activation rows, expert by expert, as bf16,
//                   followed by every token's row for the shared expert.
//  3. grouped GEMM, gate/up: per (expert, 64 units of I, up to 256 rows) tile
//                   one 128-row tcgen05 MMA stack whose A tile stacks 64
//                   W_gate rows over the 64 W_up rows of the same units (the
//                   fused gate/up operand of TensorFold #593's packGateUp),
//                   loaded as two boxes; the epilogue warp holding a unit's g
//                   and the one holding its u swap half their columns through
//                   shared memory, form h = silu(g) * u and round it to bf16.
//  4. grouped GEMM, down: per (expert, 128 output features, up to 256 rows)
//                   tile; the epilogue scales by the routing weight and writes
//                   each pick's fp32 contribution to its (token, slot) row.
//  5. combine:      y[t] = fold of the contributions in ascending (expert id,
//                   slot) -- the band partials in rank order with the carry
//                   passed along, one fixed order whatever the plan -- then
//                   plus the shared expert's output.
//
// The GEMMs are persistent and warp specialised: warp 0 issues the weight
// tiles' TMA loads (cp.async.bulk.tensor, 128-byte swizzle, one CTA per copy)
// into a 6-stage ring of 16 KB and warp 6 the activation tiles' into a
// 3-stage ring of 32 KB, so that a tile with few rows (whose weights are most
// of its bytes) keeps 96 KB of weights in flight; warp 1 issues tcgen05.mma
// with the fp32 accumulator in tensor memory (two accumulators, so the
// epilogue of one tile overlaps the MMAs of the next), and warps 2..5 drain
// the accumulator with tcgen05.ld.
// Weights sit on the MMA's M side (128 rows) and the expert's tokens on the
// N side (16..256), so a tile is never padded to 128 tokens.
#pragma once

#include <cudaTypedefs.h>
#include <cstdio>

#include "common.cuh"

namespace epk {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 64;
constexpr int kGemmAStages = 6;   // weight tiles
constexpr int kGemmBStages = 3;   // activation tiles
constexpr int kGemmThreads = 224;
constexpr int kGemmWarpB = 6;     // the activation-tile producer
constexpr int kGateUpRows = 64;  // units of I per gate/up tile (64 gate + 64 up rows)
// The activation tile is one box per stage, of the smallest of these heights
// (capped at the tensor's rows rounded up to 32) that covers the tile's rows:
// one copy instruction instead of one per 32 rows.
constexpr int kBoxLevels = 4;
constexpr int kBoxRowsB[kBoxLevels] = {32, 64, 128, 256};
constexpr uint32_t kTileABytes = kGemmBM * kGemmBK * 2;
constexpr uint32_t kTileBBytes = kGemmBN * kGemmBK * 2;
constexpr uint32_t kRingBOff = kGemmAStages * kTileABytes;
constexpr uint32_t kRingBytes = kRingBOff + kGemmBStages * kTileBBytes;
constexpr int kTmemCols = 2 * kGemmBN;
constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kMaxGroups = 1025;

struct GroupedWorkspace {
    size_t group_offset = 0, perm_pair = 0, units_gu = 0, units_dn = 0, chunk_count = 0;
    size_t x_perm = 0, h_perm = 0, h_shared = 0, c = 0, s = 0;
    size_t end = 0;
};

inline size_t g_align256(size_t v) { return (v + 255) / 256 * 256; }

inline GroupedWorkspace grouped_workspace_layout(size_t base, int64_t T, int64_t H, int64_t E,
                                                 int64_t k, int64_t I, int64_t I_s) {
    GroupedWorkspace w;
    const size_t P = (size_t)T * k;
    size_t o = g_align256(base);
    w.group_offset = o; o = g_align256(o + (size_t)(E + 2) * 4);
    w.perm_pair = o;    o = g_align256(o + P * 4);
    w.units_gu = o;     o = g_align256(o + (size_t)(E + 2) * 4);
    w.units_dn = o;     o = g_align256(o + (size_t)(E + 2) * 4);
    w.chunk_count = o;  o = g_align256(o + (P + kPlanThreads - 1) / kPlanThreads * (size_t)E * 4);
    w.x_perm = o;       o = g_align256(o + (P + (size_t)T) * H * 2);
    w.h_perm = o;       o = g_align256(o + P * I * 2);
    w.h_shared = o;     o = g_align256(o + (size_t)T * I_s * 2);
    w.c = o;            o = g_align256(o + P * H * 4);
    w.s = o;            o = g_align256(o + (size_t)T * H * 4);
    w.end = o;
    return w;
}

// ------------------------------------------------------------- block scans
// Exclusive scan of up to 2 * blockDim.x values held two per thread
// (elements 2 tid, 2 tid + 1); returns the total.  blockDim.x == 1024.
__device__ int block_exclusive_scan2(int &v0, int &v1, int *warp_sums) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int local = v0 + v1;
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off)
            incl += n;
    }
    if (lane == 31)
        warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
        int inc = s;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off)
                inc += n;
        }
        warp_sums[32 + lane] = inc - s;   // exclusive prefix of the warp totals
        if (lane == 31)
            warp_sums[64] = inc;
    }
    __syncthreads();
    const int excl = warp_sums[32 + warp] + incl - local;
    const int total = warp_sums[64];
    v1 = excl + v0;
    v0 = excl;
    __syncthreads();
    return total;
}

// ------------------------------------------------------------- group plan
// The picks are grouped by expert in two launches over chunks of
// kPlanThreads picks, one CTA per chunk: group_count_kernel counts each
// chunk's picks per expert; group_plan_kernel then gives every CTA its
// chunk's first row in each expert's group (the experts before it, plus the
// same expert's picks in earlier chunks) and scatters the chunk stably, so
// the grouped order is a stable sort of the picks by expert id.
struct PlanArgs {
    const int32_t *ids;
    int64_t T, P;
    int top_k, E, H, I, I_s;
    int32_t *group_offset;  // [E + 2]: routed row offsets, [E] = valid picks, [E+1] = P
    int32_t *perm_pair;     // [P]: permuted row -> pick index t * top_k + j
    int32_t *units_gu;      // [G + 1] exclusive prefix of gate/up tiles per group
    int32_t *units_dn;      // [G + 1] same for the down projection
    int32_t *chunk_count;   // [chunks][E]: valid picks of expert e in chunk c
};

__global__ void __launch_bounds__(kPlanThreads, 1) group_count_kernel(const PlanArgs a) {
    extern __shared__ __align__(16) int hist[];  // [E]
    grid_dependents_launch();
    grid_dependency_wait();  // ids come from the router
    const int E = a.E, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += kPlanThreads)
        hist[e] = 0;
    __syncthreads();
    const int64_t p = (int64_t)blockIdx.x * kPlanThreads + threadIdx.x;
    int e = -1;
    bool valid = false;
    if (p < a.P) {
        e = a.ids[p];
        valid = e >= 0 && e < E;
        if (!valid && e != kIdNone)
            flag_status(kStatusBadId);
    }
    const int key = valid ? e : -(lane + 2);
    const uint32_t m = __match_any_sync(0xffffffffu, key);
    if (valid && lane == __ffs(m) - 1)
        atomicAdd(&hist[e], __popc(m));
    __syncthreads();
    for (int f = threadIdx.x; f < E; f += kPlanThreads)
        a.chunk_count[(size_t)blockIdx.x * E + f] = hist[f];
}

__global__ void __launch_bounds__(kPlanThreads, 1) group_plan_kernel(const PlanArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    grid_dependents_launch();
    grid_dependency_wait();  // the chunk counts come from group_count_kernel
    int *cnt = reinterpret_cast<int *>(smem);            // [kPlanWarps][E]
    int *total = cnt + kPlanWarps * a.E;                 // [E]
    int *goff = total + a.E;                             // [E]
    int *wsum = goff + a.E;                              // [65]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E;
    const int64_t P = a.P;
    const int chunk = (int)blockIdx.x, n_chunks = (int)gridDim.x;
    // this chunk's picks, 32 per warp, in pick order
    const int64_t p_lo = (int64_t)chunk * kPlanThreads + 32 * warp;
    const int64_t p_hi = min(P, p_lo + 32);

    for (int i = tid; i < kPlanWarps * E; i += kPlanThreads)
        cnt[i] = 0;
    // every expert's total, and its picks in the chunks before this one
    // (summed in chunk order)
    for (int e = tid; e < E; e += kPlanThreads) {
        int all = 0, before = 0;
        for (int c = 0; c < n_chunks; ++c) {
            const int v = a.chunk_count[(size_t)c * E + e];
            before += c < chunk ? v : 0;
            all += v;
        }
        total[e] = all;
        goff[e] = before;
    }
    __syncthreads();
    // per-warp histogram of the chunk's picks
    {
        const int64_t p = p_lo + lane;
        int e = -1;
        bool valid = false;
        if (p < p_hi) {
            e = a.ids[p];
            valid = e >= 0 && e < E;
        }
        const int key = valid ? e : -(lane + 2);
        const uint32_t m = __match_any_sync(0xffffffffu, key);
        if (valid && lane == __ffs(m) - 1)
            cnt[warp * E + e] = __popc(m);
    }
    // exclusive scan of the per-expert totals (E <= 1024 <= 2 * threads)
    {
        int v0 = 2 * tid < E ? total[2 * tid] : 0;
        int v1 = 2 * tid + 1 < E ? total[2 * tid + 1] : 0;
        const int all = block_exclusive_scan2(v0, v1, wsum);
        // each expert's first row for this chunk: its group's start plus the
        // earlier chunks' picks of it
        if (2 * tid < E)
            goff[2 * tid] += v0;
        if (2 * tid + 1 < E)
            goff[2 * tid + 1] += v1;
        if (chunk == 0 && tid == 0) {
            a.group_offset[E] = all;
            a.group_offset[E + 1] = (int)P;
        }
        if (chunk == 0) {
            if (2 * tid < E)
                a.group_offset[2 * tid] = v0;
            if (2 * tid + 1 < E)
                a.group_offset[2 * tid + 1] = v1;
        }
    }
    __syncthreads();
    // each warp's first row per expert: the chunk's start plus the earlier
    // warps' picks of it
    for (int e = tid; e < E; e += kPlanThreads) {
        int run = goff[e];
        for (int w = 0; w < kPlanWarps; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    // stable scatter: lane order inside a warp, warp order inside the chunk
    {
        const int64_t p = p_lo + lane;
        int e = -1;
        bool valid = false;
        if (p < p_hi) {
            e = a.ids[p];
            valid = e >= 0 && e < E;
        }
        const int key = valid ? e : -(lane + 2);
        const uint32_t m = __match_any_sync(0xffffffffu, key);
        if (valid)
            a.perm_pair[cnt[warp * E + e] + __popc(m & ((1u << lane) - 1u))] = (int32_t)p;
    }
    if (chunk != 0)
        return;
    // tiles per group: routed groups, then the shared expert (all T rows)
    const int G = E + (a.I_s > 0 ? 1 : 0);
    {
        int gu[2], dn[2];
        for (int q = 0; q < 2; ++q) {
            const int g = 2 * tid + q;
            gu[q] = dn[q] = 0;
            if (g < G) {
                const int64_t rows = g < E ? total[g] : a.T;
                const int nb = (int)((rows + kGemmBN - 1) / kGemmBN);
                const int m_rows = g < E ? a.I : a.I_s;
                gu[q] = nb * ((m_rows + kGateUpRows - 1) / kGateUpRows);
                dn[q] = nb * ((a.H + kGemmBM - 1) / kGemmBM);
            }
        }
        const int all_gu = block_exclusive_scan2(gu[0], gu[1], wsum);
        const int all_dn = block_exclusive_scan2(dn[0], dn[1], wsum);
        for (int q = 0; q < 2; ++q) {
            const int g = 2 * tid + q;
            if (g < G) {
                a.units_gu[g] = gu[q];
                a.units_dn[g] = dn[q];
            }
        }
        if (tid == 0) {
            a.units_gu[G] = all_gu;
            a.units_dn[G] = all_dn;
        }
    }
}

// ----------------------------------------------------------- row gather
__global__ void __launch_bounds__(256) gather_rows_kernel(const void *__restrict__ x, int x_f32,
                                                          int64_t T, int H, int top_k, int64_t P,
                                                          int E, int with_shared,
                                                          const int32_t *__restrict__ group_offset,
                                                          const int32_t *__restrict__ perm_pair,
                                                          uint16_t *__restrict__ x_perm) {
    grid_dependents_launch();
    grid_dependency_wait();  // the grouping comes from group_plan_kernel
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_valid = group_offset[E];
    const int64_t rows = n_valid + (with_shared ? T : 0);
    const int nck = H >> 3;
    for (int64_t r = warp_global; r < rows; r += nwarps) {
        int64_t t, dst;
        if (r < n_valid) {
            t = perm_pair[r] / top_k;
            dst = r;
        } else {
            t = r - n_valid;
            dst = P + t;
        }
        uint4 *out = reinterpret_cast<uint4 *>(x_perm + (size_t)dst * H);
        if (x_f32) {
            const float4 *in = reinterpret_cast<const float4 *>(
                reinterpret_cast<const float *>(x) + (size_t)t * H);
            for (int c = lane; c < nck; c += 32) {
                const float4 a = in[2 * c], b = in[2 * c + 1];
                uint4 v;
                v.x = (uint32_t)f32_to_bf16_rne(a.x) | ((uint32_t)f32_to_bf16_rne(a.y) << 16);
                v.y = (uint32_t)f32_to_bf16_rne(a.z) | ((uint32_t)f32_to_bf16_rne(a.w) << 16);
                v.z = (uint32_t)f32_to_bf16_rne(b.x) | ((uint32_t)f32_to_bf16_rne(b.y) << 16);
                v.w = (uint32_t)f32_to_bf16_rne(b.z) | ((uint32_t)f32_to_bf16_rne(b.w) << 16);
                out[c] = v;
            }
        } else {
            const uint4 *in = reinterpret_cast<const uint4 *>(
                reinterpret_cast<const uint16_t *>(x) + (size_t)t * H);
            for (int c = lane; c < nck; c += 32)
                out[c] = in[c];
        }
    }
}

// ------------------------------------------------------------ grouped GEMM
struct GemmMaps {
    CUtensorMap a, a2;               // routed weights (gate/up: W_gate, W_up; down: W_down)
    CUtensorMap a_shared, a2_shared; // shared expert weights
    CUtensorMap b[kBoxLevels];       // activations of the routed rows, one map per box height
    CUtensorMap b_shared[kBoxLevels];  // the shared expert's rows (down only)
};

struct GemmParams {
    int E, G;
    int64_t T, P;
    int top_k;
    int m_routed, m_shared;   // rows of the weight matrices: gate/up I, I_s; down H, H
    int k_routed, k_shared;   // reduction length: gate/up H, H; down I, I_s
    const int32_t *group_offset, *units, *perm_pair;
    const float *weights;
    uint16_t *h_out, *h_shared_out;   // gate/up outputs
    int I, I_s;
    float *c_out, *s_out;             // down outputs
    int H;
    int b_rows[kBoxLevels], bs_rows[kBoxLevels];  // box heights of maps.b and maps.b_shared
};

struct GemmSmem {
    static constexpr uint32_t bars = kRingBytes;
    static constexpr uint32_t misc = bars + 256;
    static constexpr uint32_t units = misc + 64;
    static constexpr uint32_t offsets = units + kMaxGroups * 4 + 4;
    // gate/up: the column exchange of the two epilogue warp pairs, 2 x 2 x [16][32]
    static constexpr uint32_t xchg = (offsets + (kMaxGroups + 2) * 4 + 15) / 16 * 16;
    static constexpr uint32_t total = xchg + 2 * 2 * 16 * 32 * 4;
    static constexpr uint32_t alloc = total + 1024;  // room to align the base to 1024
};

template <bool GATE_UP>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
    using Smem = GemmSmem;
    constexpr int SA = kGemmAStages, SB = kGemmBStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_a = reinterpret_cast<uint64_t *>(smem + Smem::bars);
    uint64_t *empty_a = full_a + SA;
    uint64_t *full_b = empty_a + SA;
    uint64_t *empty_b = full_b + SB;
    uint64_t *tfull = empty_b + SB;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Smem::misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Smem::misc + 8);
    int *units = reinterpret_cast<int *>(smem + Smem::units);
    int *offsets = reinterpret_cast<int *>(smem + Smem::offsets);

    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int G = p.G;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&empty_a[s], 1);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&maps.a);
        for (int l = 0; l < kBoxLevels; ++l)
            prefetch_tensormap(&maps.b[l]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    // the set-up above overlaps the previous kernel's tail; everything below
    // reads what the earlier kernels of the call wrote
    grid_dependency_wait();
    grid_dependents_launch();
    for (int i = threadIdx.x; i <= G; i += blockDim.x)
        units[i] = p.units[i];
    for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x)
        offsets[i] = p.group_offset[i];
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    const int total_units = units[G];

    // unit -> (group, m block, n block); m-major inside a group so that
    // consecutive units reuse the same weight tile from L2.
    auto decode = [&](int u, int &g, int &mb, int &nb, int &rows, int &n_blocks) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {  // largest g with units[g] <= u
            const int mid = (lo + hi + 1) >> 1;
            if (units[mid] <= u)
                lo = mid;
            else
                hi = mid - 1;
        }
        g = lo;
        rows = g < p.E ? offsets[g + 1] - offsets[g] : (int)p.T;
        n_blocks = (rows + kGemmBN - 1) / kGemmBN;
        const int local = u - units[g];
        mb = local / n_blocks;
        nb = local - mb * n_blocks;
    };

    if (warp == 0) {
        // -------------------------------------------- TMA producer: weights
        if (elect_one()) {
            // a weight tile read by one n block streams through L2 once; one
            // read by several (an expert with more than 256 rows, whose n
            // blocks run on neighbouring CTAs at about the same time) stays
            // at normal priority so that the other n blocks find it there
            const uint64_t pol_once = policy_evict_first();
            const uint64_t pol_again = policy_evict_normal();
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool stop = false;
            for (int u = blockIdx.x; u < total_units && !stop; u += gridDim.x) {
                int g, mb, nb, rows, n_blocks;
                decode(u, g, mb, nb, rows, n_blocks);
                const uint64_t pol_w = n_blocks > 1 ? pol_again : pol_once;
                const bool shared = g >= p.E;
                const int K = shared ? p.k_shared : p.k_routed;
                const int kblocks = (K + kGemmBK - 1) / kGemmBK;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty_a[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sa = smem + stage * kTileABytes;
                    mbar_arrive_expect_tx(&full_a[stage], kTileABytes);
                    const int k0 = kb * kGemmBK;
                    if (GATE_UP) {
                        // rows 0..63: W_gate of the tile's 64 units, 64..127: W_up
                        const int row = mb * kGateUpRows;
                        uint8_t *sa_up = sa + kGateUpRows * kGemmBK * 2;
                        if (shared) {
                            tma_load_2d(sa, &maps.a_shared, k0, row, &full_a[stage], pol_w);
                            tma_load_2d(sa_up, &maps.a2_shared, k0, row, &full_a[stage], pol_w);
                        } else {
                            tma_load_3d(sa, &maps.a, k0, row, g, &full_a[stage], pol_w);
                            tma_load_3d(sa_up, &maps.a2, k0, row, g, &full_a[stage], pol_w);
                        }
                    } else {
                        if (shared)
                            tma_load_2d(sa, &maps.a_shared, k0, mb * kGemmBM, &full_a[stage],
                                        pol_w);
                        else
                            tma_load_3d(sa, &maps.a, k0, mb * kGemmBM, g, &full_a[stage], pol_w);
                    }
                    ++issued;
                    if (++stage == SA) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int n = issued > SA ? issued - SA : 0; n < issued; ++n)
                mbar_wait(&full_a[n % SA], (uint32_t)(n / SA) & 1u, nullptr);
        }
    } else if (warp == kGemmWarpB) {
        // ---------------------------------------- TMA producer: activations
        if (elect_one()) {
            const uint64_t pol_x = policy_evict_last();
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool stop = false;
            for (int u = blockIdx.x; u < total_units && !stop; u += gridDim.x) {
                int g, mb, nb, rows, n_blocks;
                decode(u, g, mb, nb, rows, n_blocks);
                const bool shared = g >= p.E;
                const int K = shared ? p.k_shared : p.k_routed;
                const int n0 = nb * kGemmBN;
                const int n_valid = min(kGemmBN, rows - n0);
                int brow;
                if (GATE_UP)
                    brow = (shared ? (int)p.P : offsets[g]) + n0;
                else
                    brow = (shared ? 0 : offsets[g]) + n0;
                const bool bs = !GATE_UP && shared;
                const int *box_rows = bs ? p.bs_rows : p.b_rows;
                int lvl = 0;
                while (lvl + 1 < kBoxLevels && box_rows[lvl] < n_valid)
                    ++lvl;
                const CUtensorMap *bmap = bs ? &maps.b_shared[lvl] : &maps.b[lvl];
                const uint32_t b_bytes = (uint32_t)box_rows[lvl] * kGemmBK * 2;
                const int kblocks = (K + kGemmBK - 1) / kGemmBK;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty_b[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sb = smem + kRingBOff + stage * kTileBBytes;
                    mbar_arrive_expect_tx(&full_b[stage], b_bytes);
                    tma_load_2d(sb, bmap, kb * kGemmBK, brow, &full_b[stage], pol_x);
                    ++issued;
                    if (++stage == SB) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int n = issued > SB ? issued - SB : 0; n < issued; ++n)
                mbar_wait(&full_b[n % SB], (uint32_t)(n / SB) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t sa = 0, pa = 0, sb = 0, pb = 0;
            uint32_t acc = 0, acc_phase = 0;
            bool stop = false;
            for (int u = blockIdx.x; u < total_units && !stop; u += gridDim.x) {
                int g, mb, nb, rows, n_blocks;
                decode(u, g, mb, nb, rows, n_blocks);
                const bool shared = g >= p.E;
                const int K = shared ? p.k_shared : p.k_routed;
                const int n_valid = min(kGemmBN, rows - nb * kGemmBN);
                const uint32_t n_mma = (uint32_t)((n_valid + 15) / 16 * 16);
                const uint32_t idesc = idesc_bf16_f32(kGemmBM, n_mma);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kGemmBN;
                const int kblocks = (K + kGemmBK - 1) / kGemmBK;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&full_a[sa], pa, abort_flag) ||
                        !mbar_wait(&full_b[sb], pb, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(smem + sa * kTileABytes);
                    const uint32_t b_addr = smem_u32(smem + kRingBOff + sb * kTileBBytes);
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_bf16(d_tmem, smem_desc_sw128_kmajor(a_addr + kk * 32),
                                  smem_desc_sw128_kmajor(b_addr + kk * 32), idesc,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
                    // each frees its slot once these MMAs are done
                    umma_commit(&empty_a[sa]);
                    umma_commit(&empty_b[sb]);
                    if (++sa == SA) {
                        sa = 0;
                        pa ^= 1u;
                    }
                    if (++sb == SB) {
                        sb = 0;
                        pb ^= 1u;
                    }
                }
                if (stop)
                    break;
                umma_commit(&tfull[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // every MMA issued by this thread has completed before TMEM is freed
            umma_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
    } else if (warp >= 2 && warp < 6) {
        // ------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        // gate/up: quarters 0, 1 hold the gate rows of units 0..31, 32..63 and
        // quarters 2, 3 the up rows of the same units; the two warps of a pair
        // (same units) swap half their columns through shared memory:
        // xg = gate values of columns 16..31, xu = up values of columns 0..15,
        // each [16][32 lanes]
        const bool gate_warp = q < 2;
        const int pair = q & 1;
        float *xg = reinterpret_cast<float *>(smem + Smem::xchg) + pair * 2 * 16 * 32;
        float *xu = xg + 16 * 32;
        uint32_t acc = 0, acc_phase = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
            int g, mb, nb, rows, n_blocks;
            decode(u, g, mb, nb, rows, n_blocks);
            const bool shared = g >= p.E;
            const int n0 = nb * kGemmBN;
            const int n_valid = min(kGemmBN, rows - n0);
            // down: the pick index and routing weight of column 32 c + lane in
            // mp[c], mw[c], loaded while the accumulator fills and handed to the
            // other lanes by shuffles, so that no load waits behind a store
            int mp[kGemmBN / 32];
            float mw[kGemmBN / 32];
#pragma unroll
            for (int c = 0; c < kGemmBN / 32; ++c) {
                mp[c] = 0;
                mw[c] = 0.f;
            }
            if (!GATE_UP && !shared) {
#pragma unroll
                for (int c = 0; c < kGemmBN / 32; ++c)
                    if (32 * c + lane < n_valid)
                        mp[c] = p.perm_pair[offsets[g] + n0 + 32 * c + lane];
#pragma unroll
                for (int c = 0; c < kGemmBN / 32; ++c)
                    if (32 * c + lane < n_valid)
                        mw[c] = p.weights[mp[c]];
            }
            bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag);
            // the two warps of a pair leave together or not at all (their
            // exchange below synchronises on a named barrier)
            if (GATE_UP)
                ok = named_count(1 + pair, 64, ok) == 64;
            if (!ok)
                break;
            tc_fence_after_sync();
            const uint32_t t_row = tmem_base + ((uint32_t)(32 * q) << 16) + acc * kGemmBN;
#pragma unroll
            for (int c = 0; c < kGemmBN / 32; ++c) {
                const int c0 = 32 * c;
                if (c0 >= n_valid)
                    break;
                uint32_t v[32];
                tmem_load_32cols(t_row + (uint32_t)c0, v);
                tmem_load_wait();
                if (GATE_UP) {
                    // lane = unit; the gate warp finishes columns 0..15 of the
                    // chunk, the up warp columns 16..31
                    const int M = shared ? p.I_s : p.I;
                    const int unit = mb * kGateUpRows + 32 * pair + lane;
                    uint16_t *hrow_base = shared ? p.h_shared_out : p.h_out;
                    const int ld = shared ? p.I_s : p.I;
                    const int64_t row0 = (shared ? 0 : offsets[g]) + n0 + c0;
                    if (gate_warp) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            xg[j * 32 + lane] = __uint_as_float(v[16 + j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            xu[j * 32 + lane] = __uint_as_float(v[j]);
                    }
                    named_sync(1 + pair, 64);
                    // the partner's half, into registers before any store
                    float xo[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        xo[j] = gate_warp ? xu[j * 32 + lane] : xg[j * 32 + lane];
                    named_sync(1 + pair, 64);  // the buffers are free for the next chunk
                    const int cb = gate_warp ? 0 : 16;
                    uint16_t *dst = hrow_base + (size_t)(row0 + cb) * ld + unit;
                    // whole half-chunks store without a test per column
                    if (unit < M) {
                        if (c0 + cb + 16 <= n_valid) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const float gv = gate_warp ? __uint_as_float(v[j]) : xo[j];
                                const float uv = gate_warp ? xo[j] : __uint_as_float(v[16 + j]);
                                dst[(size_t)j * ld] = f32_to_bf16_rne(silu_fast_f32(gv) * uv);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const float gv = gate_warp ? __uint_as_float(v[j]) : xo[j];
                                const float uv = gate_warp ? xo[j] : __uint_as_float(v[16 + j]);
                                if (c0 + cb + j < n_valid)
                                    dst[(size_t)j * ld] = f32_to_bf16_rne(silu_fast_f32(gv) * uv);
                            }
                        }
                    }
                } else {
                    const int row = mb * kGemmBM + 32 * q + lane;
                    // whole chunks store without a test per column; the pick
                    // metadata of column c0 + j comes from lane j
                    float wv[32];
                    int pk[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        pk[j] = __shfl_sync(0xffffffffu, mp[c], j);
                        wv[j] = __shfl_sync(0xffffffffu, mw[c], j);
                    }
                    if (row < p.H) {
                        if (shared) {
                            float *dst = p.s_out + (size_t)(n0 + c0) * p.H + row;
                            if (c0 + 32 <= n_valid) {
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    dst[(size_t)j * p.H] = __uint_as_float(v[j]);
                            } else {
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (c0 + j < n_valid)
                                        dst[(size_t)j * p.H] = __uint_as_float(v[j]);
                            }
                        } else {
                            float *dst = p.c_out + row;
                            if (c0 + 32 <= n_valid) {
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    dst[(size_t)pk[j] * p.H] = wv[j] * __uint_as_float(v[j]);
                            } else {
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (c0 + j < n_valid)
                                        dst[(size_t)pk[j] * p.H] = wv[j] * __uint_as_float(v[j]);
                            }
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&tempty[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------- combine
// y[t] = contributions of t's picks folded in ascending (expert id, slot),
// then + the shared expert's output.  Skipped (invalid) picks add nothing.
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ c,
                                                      const float *__restrict__ s,
                                                      const int32_t *__restrict__ ids, int64_t T,
                                                      int H, int top_k, int E,
                                                      float *__restrict__ y) {
    __shared__ int pick_e[16];
    __shared__ int order[16];
    __shared__ int n_valid;
    const int64_t t = blockIdx.x;
    // the token's picks in ascending (expert id, slot): each valid pick's
    // place is the number of valid picks before it in that order (blockDim.x
    // >= top_k; the ids are read once, in parallel)
    const int j = (int)threadIdx.x;
    if (j < top_k)
        pick_e[j] = ids[t * top_k + j];
    __syncthreads();
    if (j < top_k) {
        const int e = pick_e[j];
        if (e >= 0 && e < E) {
            int r = 0;
            for (int q = 0; q < top_k; ++q) {
                const int f = pick_e[q];
                r += f >= 0 && f < E && (f < e || (f == e && q < j));
            }
            order[r] = j;
        }
    }
    if (j == 0) {
        int n = 0;
        for (int q = 0; q < top_k; ++q)
            n += pick_e[q] >= 0 && pick_e[q] < E;
        n_valid = n;
    }
    __syncthreads();
    // The ids were written before the previous kernel began (every kernel
    // that launches this one early has passed its own wait on its
    // predecessor, back to the router), so the order above was formed while
    // the previous kernel ran; c and s come from that kernel.
    grid_dependency_wait();
    const int h4 = blockIdx.y * blockDim.x + threadIdx.x;  // float4 column
    if (h4 * 4 >= H)
        return;
    const int n = n_valid;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < n; ++q) {
        const float4 v =
            reinterpret_cast<const float4 *>(c + ((size_t)t * top_k + order[q]) * H)[h4];
        if (q == 0) {
            acc = v;
        } else {
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
    }
    if (s != nullptr) {
        const float4 v = reinterpret_cast<const float4 *>(s + (size_t)t * H)[h4];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    reinterpret_cast<float4 *>(y + (size_t)t * H)[h4] = acc;
}

// ================================================================== host side
struct GroupedArgs {
    const void *x;
    bool x_f32;
    int64_t T, H, E, I, I_s;
    int top_k;
    const int32_t *ids;
    const float *weights;
    const void *w_gate, *w_up, *w_down, *ws_gate, *ws_up, *ws_down;
    float *y;
    int sm_count, smem_optin;
    bool pdl;  // launch as programmatic dependents
};

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// bf16 tensor map: dims innermost first; box (64 elements of K) x box_rows (x 1).
inline bool make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
                     const uint64_t *strides_bytes, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (enc == nullptr)
        return false;
    cuuint64_t gdim[3], gstride[2];
    cuuint32_t box[3], estride[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i)
        gdim[i] = dims[i];
    for (int i = 0; i < rank - 1; ++i)
        gstride[i] = strides_bytes[i];
    box[0] = kGemmBK;
    box[1] = box_rows;
    box[2] = 1;
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                           const_cast<void *>(base), gdim, gstride, box, estride,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline bool map_2d(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                   uint32_t box_rows) {
    const uint64_t dims[2] = {cols, rows};
    const uint64_t strides[1] = {cols * 2};
    return make_map(m, base, 2, dims, strides, box_rows);
}

inline bool map_3d(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t mats,
                   uint32_t box_rows) {
    const uint64_t dims[3] = {cols, rows, mats};
    const uint64_t strides[2] = {cols * 2, cols * rows * 2};
    return make_map(m, base, 3, dims, strides, box_rows);
}

// The activation maps of every box height; a height is capped at the rows
// rounded up to 32, so that no box is taller than the tensor needs.
inline bool map_b_levels(CUtensorMap *maps, int *box_rows, const void *base, uint64_t cols,
                         int64_t rows) {
    const int64_t cap = (rows + 31) / 32 * 32;
    for (int l = 0; l < kBoxLevels; ++l) {
        box_rows[l] = (int)std::min<int64_t>(kBoxRowsB[l], cap);
        if (!map_2d(&maps[l], base, cols, (uint64_t)rows, (uint32_t)box_rows[l]))
            return false;
    }
    return true;
}

inline size_t plan_smem_bytes(int64_t E) { return (size_t)(kPlanWarps * E + 2 * E + 65) * 4; }

inline ep_status grouped_set_attributes(int smem_optin) {
    if (cudaFuncSetAttribute(group_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_optin) != cudaSuccess)
        return EP_ECUDA;
    if (cudaFuncSetAttribute(grouped_gemm_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(grouped_gemm_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_optin) != cudaSuccess)
        return EP_ECUDA;
    return EP_OK;
}

// Launch with programmatic dependent launch (pdl = true) or as a plain launch.
template <typename... KArgs, typename... Args>
inline cudaError_t grouped_launch(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                  size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Records events[2j] / events[2j+1] around kernel j when a timing hook is set.
inline void bracket_event(void *const *events, int n, int idx, cudaStream_t st) {
    if (events != nullptr && idx < n && (idx | 1) < n)
        cudaEventRecord(static_cast<cudaEvent_t>(events[idx]), st);
}

inline ep_status grouped_forward(const GroupedArgs &g, const GroupedWorkspace &W, uint8_t *ws,
                                 cudaStream_t st, int *launches, char *why, size_t why_len,
                                 void *const *ev, int n_ev) {
    *launches = 0;
    const int64_t T = g.T, H = g.H, E = g.E, I = g.I, I_s = g.I_s;
    const int k = g.top_k;
    const int64_t P = T * k;
    const int G = (int)E + (I_s > 0 ? 1 : 0);
    const uint32_t gemm_smem = GemmSmem::alloc;
    if (gemm_smem > (uint32_t)g.smem_optin || plan_smem_bytes(E) > (size_t)g.smem_optin) {
        snprintf(why, why_len, "not enough shared memory per block for the tensor path");
        return EP_EINVAL;
    }
    if (tensor_map_encoder() == nullptr) {
        snprintf(why, why_len, "cuTensorMapEncodeTiled is not available from the driver");
        return EP_ECUDA;
    }
    int32_t *group_offset = reinterpret_cast<int32_t *>(ws + W.group_offset);
    int32_t *perm_pair = reinterpret_cast<int32_t *>(ws + W.perm_pair);
    int32_t *units_gu = reinterpret_cast<int32_t *>(ws + W.units_gu);
    int32_t *units_dn = reinterpret_cast<int32_t *>(ws + W.units_dn);
    uint16_t *x_perm = reinterpret_cast<uint16_t *>(ws + W.x_perm);
    uint16_t *h_perm = reinterpret_cast<uint16_t *>(ws + W.h_perm);
    uint16_t *h_shared = reinterpret_cast<uint16_t *>(ws + W.h_shared);
    float *c = reinterpret_cast<float *>(ws + W.c);
    float *s = reinterpret_cast<float *>(ws + W.s);

    // 1. plan
    PlanArgs pa;
    pa.ids = g.ids; pa.T = T; pa.P = P; pa.top_k = k; pa.E = (int)E; pa.H = (int)H;
    pa.I = (int)I; pa.I_s = (int)I_s;
    pa.group_offset = group_offset; pa.perm_pair = perm_pair;
    pa.units_gu = units_gu; pa.units_dn = units_dn;
    pa.chunk_count = reinterpret_cast<int32_t *>(ws + W.chunk_count);
    const unsigned n_chunks = (unsigned)((P + kPlanThreads - 1) / kPlanThreads);
    bracket_event(ev, n_ev, 0, st);
    cudaError_t e_plan = grouped_launch(g.pdl, group_count_kernel, dim3(n_chunks),
                                        dim3(kPlanThreads), (size_t)E * 4, st, pa);
    if (e_plan == cudaSuccess)
        e_plan = grouped_launch(g.pdl, group_plan_kernel, dim3(n_chunks), dim3(kPlanThreads),
                                plan_smem_bytes(E), st, pa);
    bracket_event(ev, n_ev, 1, st);
    if (e_plan != cudaSuccess) {
        snprintf(why, why_len, "group_plan launch failed");
        return EP_ECUDA;
    }
    // 2. gather
    {
        const int64_t rows = P + (I_s > 0 ? T : 0);
        const int64_t blocks = std::min<int64_t>((rows + 7) / 8, (int64_t)g.sm_count * 8);
        bracket_event(ev, n_ev, 2, st);
        const cudaError_t e_gather = grouped_launch(
            g.pdl, gather_rows_kernel, dim3((unsigned)std::max<int64_t>(blocks, 1)), dim3(256), 0,
            st, g.x, (int)(g.x_f32 ? 1 : 0), T, (int)H, k, P, (int)E, (int)(I_s > 0 ? 1 : 0),
            (const int32_t *)group_offset, (const int32_t *)perm_pair, x_perm);
        bracket_event(ev, n_ev, 3, st);
        if (e_gather != cudaSuccess) {
            snprintf(why, why_len, "gather_rows launch failed");
            return EP_ECUDA;
        }
    }
    // 3. gate/up
    GemmMaps gm;
    memset(&gm, 0, sizeof gm);
    GemmParams gp;
    memset(&gp, 0, sizeof gp);
    bool okm = map_3d(&gm.a, g.w_gate, H, I, E, kGateUpRows) &&
               map_3d(&gm.a2, g.w_up, H, I, E, kGateUpRows) &&
               map_b_levels(gm.b, gp.b_rows, x_perm, H, P + T);
    if (I_s > 0)
        okm = okm && map_2d(&gm.a_shared, g.ws_gate, H, I_s, kGateUpRows) &&
              map_2d(&gm.a2_shared, g.ws_up, H, I_s, kGateUpRows);
    if (!okm) {
        snprintf(why, why_len, "encoding a gate/up tensor map failed");
        return EP_ECUDA;
    }
    gp.E = (int)E; gp.G = G; gp.T = T; gp.P = P; gp.top_k = k;
    gp.m_routed = (int)I; gp.m_shared = (int)I_s; gp.k_routed = (int)H; gp.k_shared = (int)H;
    gp.group_offset = group_offset; gp.units = units_gu; gp.perm_pair = perm_pair;
    gp.weights = g.weights;
    gp.h_out = h_perm; gp.h_shared_out = h_shared; gp.I = (int)I; gp.I_s = (int)I_s;
    gp.c_out = c; gp.s_out = s; gp.H = (int)H;
    bracket_event(ev, n_ev, 4, st);
    const cudaError_t e_gu = grouped_launch(g.pdl, grouped_gemm_kernel<true>, dim3(g.sm_count),
                                            dim3(kGemmThreads), gemm_smem, st, gm, gp);
    bracket_event(ev, n_ev, 5, st);
    if (e_gu != cudaSuccess) {
        snprintf(why, why_len, "gate/up GEMM launch failed");
        return EP_ECUDA;
    }
    // 4. down
    memset(&gm, 0, sizeof gm);
    okm = map_3d(&gm.a, g.w_down, I, H, E, kGemmBM) &&
          map_b_levels(gm.b, gp.b_rows, h_perm, I, std::max<int64_t>(P, 1));
    if (I_s > 0)
        okm = okm && map_2d(&gm.a_shared, g.ws_down, I_s, H, kGemmBM) &&
              map_b_levels(gm.b_shared, gp.bs_rows, h_shared, I_s, T);
    if (!okm) {
        snprintf(why, why_len, "encoding a down tensor map failed");
        return EP_ECUDA;
    }
    gp.m_routed = (int)H; gp.m_shared = (int)H; gp.k_routed = (int)I; gp.k_shared = (int)I_s;
    gp.units = units_dn;
    bracket_event(ev, n_ev, 6, st);
    const cudaError_t e_dn = grouped_launch(g.pdl, grouped_gemm_kernel<false>, dim3(g.sm_count),
                                            dim3(kGemmThreads), gemm_smem, st, gm, gp);
    bracket_event(ev, n_ev, 7, st);
    if (e_dn != cudaSuccess) {
        snprintf(why, why_len, "down GEMM launch failed");
        return EP_ECUDA;
    }
    // 5. combine
    {
        const dim3 grid((unsigned)T, (unsigned)((H / 4 + 255) / 256));
        bracket_event(ev, n_ev, 8, st);
        const cudaError_t e_comb = grouped_launch(
            g.pdl, combine_kernel, grid, dim3(256), 0, st, (const float *)c,
            (const float *)(I_s > 0 ? s : nullptr), g.ids, T, (int)H, k, (int)E, g.y);
        bracket_event(ev, n_ev, 9, st);
        if (e_comb != cudaSuccess) {
            snprintf(why, why_len, "combine launch failed");
            return EP_ECUDA;
        }
    }
    *launches = 6;
    return EP_OK;
}

}  // namespace epk
