// router.cuh -- replicated softmax router with top-k and renormalisation.
//
// fak note "GLM-5.2 multi-GPU: expert-parallel sharding + the resident-fit
// benchmark", "What landed": the router runs replicated and every rank picks
// the same top-k.  Softmax over the logits, top_k by logit with ties to the
// lower expert id, weights renormalised over the picked set.
//
// One thread-block cluster of kRouterCluster CTAs handles a block of up to
// kRouterMaxTB tokens; CTA r owns a contiguous slice of the experts.
//  1. Each CTA holds the block's activations in shared memory as fp32.
//  2. Each warp computes, for one expert row of its CTA's slice at a time,
//     the fp32 logits of all the block's tokens (the row streams from HBM
//     with one round of 16-byte loads per lane) and a rigorous bound on each
//     logit's rounding error; both go to CTA 0 through distributed shared
//     memory.
//  3. CTA 0 finds, per token, every expert whose exact logit could reach the
//     k-th largest under those bounds (the candidates).
//  4. Every CTA recomputes its own candidates' logits in fp64 and sends them
//     back to CTA 0.
//  5. CTA 0 picks the top_k on the fp64 logits (ties to the lower id), orders
//     them by descending logit and renormalises the softmax over them in fp64.
// The selection and the weights are therefore those of exact arithmetic up to
// fp64 rounding.
#pragma once

#include "common.cuh"

namespace epk {

constexpr int kRouterCluster = 8;
constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;
constexpr int kRouterMaxTB = 8;        // tokens per cluster
constexpr int kRouterMaxK = 16;
constexpr int kRouterMaxCand = 64;     // fp64 candidates per token handled in parallel
constexpr int kRouterXBudget = 128 * 1024;  // fp32 activations of one token block
constexpr int kRouterRowChunks = 16;   // 16-byte chunks of a router row per lane per round

struct RouterSmem {
    // byte offsets into dynamic shared memory
    uint32_t x, logit, bound, xnorm2, ncand, cand, cval, list_val, list_id, total;
};

__host__ __device__ inline uint32_t align_up_u32(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline RouterSmem router_smem_layout(int tb_max, int H, int E) {
    RouterSmem s;
    uint32_t o = 0;
    s.x = o;        o = align_up_u32(o + (uint32_t)tb_max * H * 4, 16);
    s.logit = o;    o = align_up_u32(o + (uint32_t)kRouterMaxTB * E * 4, 16);
    s.bound = o;    o = align_up_u32(o + (uint32_t)kRouterMaxTB * E * 4, 16);
    s.xnorm2 = o;   o = align_up_u32(o + kRouterMaxTB * 4, 16);
    s.ncand = o;    o = align_up_u32(o + kRouterMaxTB * 4, 16);
    s.cand = o;     o = align_up_u32(o + kRouterMaxTB * kRouterMaxCand * 4, 16);
    s.cval = o;     o = align_up_u32(o + kRouterMaxTB * kRouterMaxCand * 8, 16);
    s.list_val = o; o = align_up_u32(o + kRouterMaxTB * kRouterMaxK * 8, 16);
    s.list_id = o;  o = align_up_u32(o + kRouterMaxTB * kRouterMaxK * 4, 16);
    s.total = o;
    return s;
}

__device__ __forceinline__ void unpack_w8(uint4 v, float (&wf)[8]) {
    wf[0] = bf16_lo(v.x); wf[1] = bf16_hi(v.x); wf[2] = bf16_lo(v.y); wf[3] = bf16_hi(v.y);
    wf[4] = bf16_lo(v.z); wf[5] = bf16_hi(v.z); wf[6] = bf16_lo(v.w); wf[7] = bf16_hi(v.w);
}

// fp64 logit of expert e for the token whose fp32 activations are at xrow.
__device__ double logit_fp64(const float *xrow, const uint16_t *__restrict__ w_router,
                             const float *__restrict__ bias, int H, int e) {
    const int lane = (int)lane_id();
    const int nck = H >> 3;
    const uint4 *wrow = reinterpret_cast<const uint4 *>(w_router + (size_t)e * H);
    double acc = 0.0;
    for (int base = 0; base < nck; base += 32 * kRouterRowChunks) {
        uint4 wv[kRouterRowChunks];
#pragma unroll
        for (int u = 0; u < kRouterRowChunks; ++u) {
            const int c = base + lane + 32 * u;
            wv[u] = c < nck ? wrow[c] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kRouterRowChunks; ++u) {
            const int c = base + lane + 32 * u;
            if (c < nck) {
                float wf[8];
                unpack_w8(wv[u], wf);
                const float4 *xp = reinterpret_cast<const float4 *>(xrow) + 2 * c;
                const float4 a = xp[0], b = xp[1];
                acc = fma((double)a.x, (double)wf[0], acc);
                acc = fma((double)a.y, (double)wf[1], acc);
                acc = fma((double)a.z, (double)wf[2], acc);
                acc = fma((double)a.w, (double)wf[3], acc);
                acc = fma((double)b.x, (double)wf[4], acc);
                acc = fma((double)b.y, (double)wf[5], acc);
                acc = fma((double)b.z, (double)wf[6], acc);
                acc = fma((double)b.w, (double)wf[7], acc);
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (bias != nullptr)
        acc += (double)bias[e];
    return acc;
}

// Index of the k-th largest fp32 logit of one token (ties to the lower id),
// computed by a warp; `chosen` keeps the picked lanes' bits.
__device__ float kth_logit(const float *lt, int E, int top_k) {
    const int lane = (int)lane_id();
    const int per_lane = (E + 31) / 32;  // <= 32
    uint32_t chosen = 0;
    float vk = -INFINITY;
    for (int r = 0; r < top_k; ++r) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
        for (int i = 0; i < per_lane; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((chosen >> i) & 1u)) {
                const float v = lt[e];
                if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
        if (be != 0x7fffffff && (be & 31) == lane)
            chosen |= 1u << (be >> 5);
        vk = bv;
    }
    return vk;
}

template <bool XF32>
__global__ void __cluster_dims__(kRouterCluster, 1, 1) __launch_bounds__(kRouterThreads, 1)
router_topk_kernel(const void *__restrict__ x, int64_t T, int H,
                   const uint16_t *__restrict__ w_router, const float *__restrict__ bias, int E,
                   int top_k, int tb_max, int32_t *__restrict__ ids, float *__restrict__ weights) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int XB = XF32 ? 4 : 2;
    const RouterSmem L = router_smem_layout(tb_max, H, E);
    float *xs = reinterpret_cast<float *>(smem + L.x);            // [tb][H] fp32
    float *logit = reinterpret_cast<float *>(smem + L.logit);     // [kRouterMaxTB][E], CTA 0
    float *bound = reinterpret_cast<float *>(smem + L.bound);     // [kRouterMaxTB][E], CTA 0
    float *xnorm2 = reinterpret_cast<float *>(smem + L.xnorm2);
    int *ncand = reinterpret_cast<int *>(smem + L.ncand);         // CTA 0
    int *cand = reinterpret_cast<int *>(smem + L.cand);           // CTA 0
    double *cval = reinterpret_cast<double *>(smem + L.cval);     // CTA 0
    double *list_val = reinterpret_cast<double *>(smem + L.list_val);
    int *list_id = reinterpret_cast<int *>(smem + L.list_id);

    grid_dependents_launch();
    grid_dependency_wait();  // x may come from the previous kernel; ids / weights are read there

    const uint32_t rank = cluster_ctarank();
    const int64_t t0 = (int64_t)(blockIdx.x / kRouterCluster) * tb_max;
    const int tb = (T - t0 < (int64_t)tb_max) ? (int)(T - t0) : tb_max;
    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int nck = H >> 3;
    const int per_cta = (E + kRouterCluster - 1) / kRouterCluster;
    const int e_lo = (int)rank * per_cta;
    const int e_hi = min(E, e_lo + per_cta);

    // ---- 1. this block's activations as fp32, ||x_t||^2
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            reinterpret_cast<const uint8_t *>(x) + (size_t)t0 * H * XB);
        const int n16 = tb * H * XB / 16;
        for (int i0 = threadIdx.x; i0 < n16; i0 += 4 * kRouterThreads) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kRouterThreads;
                v[u] = i < n16 ? src[i] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kRouterThreads;
                if (i < n16) {
                    if constexpr (XF32) {
                        reinterpret_cast<uint4 *>(xs)[i] = v[u];
                    } else {
                        float f[8];
                        unpack_w8(v[u], f);
                        float4 *d = reinterpret_cast<float4 *>(xs) + 2 * i;
                        d[0] = make_float4(f[0], f[1], f[2], f[3]);
                        d[1] = make_float4(f[4], f[5], f[6], f[7]);
                    }
                }
            }
        }
    }
    __syncthreads();
    if (warp < tb) {
        const float4 *row = reinterpret_cast<const float4 *>(xs + (size_t)warp * H);
        float s = 0.f;
        for (int c = lane; c < H / 4; c += 32) {
            const float4 v = row[c];
            s = fmaf(v.x, v.x, s);
            s = fmaf(v.y, v.y, s);
            s = fmaf(v.z, v.z, s);
            s = fmaf(v.w, v.w, s);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0)
            xnorm2[warp] = s;
    }
    cluster_sync();  // every CTA of the cluster is running; x block and norms visible

    // ---- 2. fp32 logits of this CTA's experts, with error bounds, to CTA 0
    {
        const uint32_t r_logit = map_shared_rank(logit, 0);
        const uint32_t r_bound = map_shared_rank(bound, 0);
        // Each lane folds at most n_lane products with fused multiply-adds,
        // then five butterfly additions and the bias add: the classic bound
        // |fl(s) - s| <= gamma_n * sum |x_h w_h| + u |l|, gamma_n = n u / (1 - n u),
        // with sum |x_h w_h| <= ||x|| ||w|| (Cauchy-Schwarz).
        const int n_lane = 8 * ((nck + 31) / 32) + 6;
        const float u = 5.9604644775390625e-8f;  // 2^-24
        const float gam = (float)n_lane * u / (1.0f - (float)n_lane * u);
        for (int e = e_lo + warp; e < e_hi; e += kRouterWarps) {
            float acc[kRouterMaxTB];
#pragma unroll
            for (int t = 0; t < kRouterMaxTB; ++t)
                acc[t] = 0.f;
            float wsq = 0.f;
            const uint4 *wrow = reinterpret_cast<const uint4 *>(w_router + (size_t)e * H);
            for (int base = 0; base < nck; base += 32 * kRouterRowChunks) {
                uint4 wv[kRouterRowChunks];
#pragma unroll
                for (int q = 0; q < kRouterRowChunks; ++q) {
                    const int c = base + lane + 32 * q;
                    wv[q] = c < nck ? ld_stream_16(wrow + c) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int q = 0; q < kRouterRowChunks; ++q) {
                    const int c = base + lane + 32 * q;
                    if (c < nck) {
                        float wf[8];
                        unpack_w8(wv[q], wf);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            wsq = fmaf(wf[j], wf[j], wsq);
#pragma unroll
                        for (int t = 0; t < kRouterMaxTB; ++t) {
                            if (t < tb) {
                                const float4 *xp =
                                    reinterpret_cast<const float4 *>(xs + (size_t)t * H) + 2 * c;
                                const float4 a = xp[0], b = xp[1];
                                acc[t] = fmaf(a.x, wf[0], acc[t]);
                                acc[t] = fmaf(a.y, wf[1], acc[t]);
                                acc[t] = fmaf(a.z, wf[2], acc[t]);
                                acc[t] = fmaf(a.w, wf[3], acc[t]);
                                acc[t] = fmaf(b.x, wf[4], acc[t]);
                                acc[t] = fmaf(b.y, wf[5], acc[t]);
                                acc[t] = fmaf(b.z, wf[6], acc[t]);
                                acc[t] = fmaf(b.w, wf[7], acc[t]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                wsq += __shfl_xor_sync(0xffffffffu, wsq, off);
#pragma unroll
                for (int t = 0; t < kRouterMaxTB; ++t)
                    acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
            }
            const float b = bias != nullptr ? bias[e] : 0.f;
            const float wnorm = sqrtf(wsq);
#pragma unroll
            for (int t = 0; t < kRouterMaxTB; ++t) {
                if (t < tb && lane == t) {
                    const float l = acc[t] + b;
                    const float d = 1.5f * (gam * sqrtf(xnorm2[t]) * wnorm + u * fabsf(l)) + 1e-30f;
                    st_cluster_f32(r_logit + 4u * (uint32_t)(t * E + e), l);
                    st_cluster_f32(r_bound + 4u * (uint32_t)(t * E + e), d);
                }
            }
        }
    }
    cluster_sync();  // all logits and bounds are in CTA 0

    // ---- 3. CTA 0: candidates per token
    if (rank == 0 && warp < tb) {
        const int t = warp;
        const float *lt = logit + t * E;
        const float *bt = bound + t * E;
        const float vk = kth_logit(lt, E, top_k);
        float dmax = 0.f;
        for (int e = lane; e < E; e += 32)
            dmax = fmaxf(dmax, bt[e]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
        // every expert whose exact logit could reach the k-th one
        const double thr = (double)vk - 2.0 * (double)dmax * 1.0001;
        int count = 0;
        for (int i = 0; i < (E + 31) / 32; ++i) {
            const int e = lane + 32 * i;
            const bool c = e < E && (double)lt[e] >= thr;
            const uint32_t m = __ballot_sync(0xffffffffu, c);
            const int pos = count + __popc(m & ((1u << lane) - 1u));
            if (c && pos < kRouterMaxCand)
                cand[t * kRouterMaxCand + pos] = e;
            count += __popc(m);
        }
        if (lane == 0)
            ncand[t] = count;
    }
    cluster_sync();  // candidate lists visible to every CTA

    // ---- 4. every CTA: fp64 logits of the candidates in its expert slice
    {
        // CTAs other than 0 copy CTA 0's candidate lists into their own arrays
        const uint32_t r_ncand = map_shared_rank(ncand, 0);
        const uint32_t r_cand = map_shared_rank(cand, 0);
        const uint32_t r_cval = map_shared_rank(cval, 0);
        if (rank != 0) {
            if (threadIdx.x < (unsigned)tb)
                ncand[threadIdx.x] = ld_cluster_s32(r_ncand + 4u * threadIdx.x);
            for (int i = threadIdx.x; i < tb * kRouterMaxCand; i += kRouterThreads)
                cand[i] = ld_cluster_s32(r_cand + 4u * (uint32_t)i);
        }
        __syncthreads();
        int nc[kRouterMaxTB];
        int total = 0;
#pragma unroll
        for (int t = 0; t < kRouterMaxTB; ++t) {
            nc[t] = 0;
            if (t < tb)
                nc[t] = ncand[t] <= kRouterMaxCand ? ncand[t] : 0;  // larger sets: CTA 0 fallback
            total += nc[t];
        }
        // (token, candidate) pairs, token by token; the warps of the CTA that
        // owns the expert split them by the expert's place in the slice
        for (int p = 0; p < total; ++p) {
            int t = 0, ci = p;
#pragma unroll
            for (int q = 0; q < kRouterMaxTB; ++q) {
                if (t == q && ci >= nc[q]) {
                    ci -= nc[q];
                    ++t;
                }
            }
            const int e = cand[t * kRouterMaxCand + ci];
            if (e < e_lo || e >= e_hi || ((e - e_lo) % kRouterWarps) != warp)
                continue;
            const double v = logit_fp64(xs + (size_t)t * H, w_router, bias, H, e);
            if (lane == 0)
                st_cluster_f64(r_cval + 8u * (uint32_t)(t * kRouterMaxCand + ci), v);
        }
    }
    cluster_sync();  // fp64 logits are in CTA 0
    if (rank != 0)
        return;

    // ---- 5. CTA 0: pick top_k on the fp64 logits, renormalise, write
    if (warp < tb) {
        const int t = warp;
        const int nc = ncand[t];
        double *lv = list_val + t * kRouterMaxK;
        int *li = list_id + t * kRouterMaxK;
        if (nc <= kRouterMaxCand) {
            uint32_t chosen = 0;  // bit i: candidate lane + 32 i taken (nc <= 64)
            for (int r = 0; r < top_k; ++r) {
                double bv = -INFINITY;
                int be = 0x7fffffff, bi = -1;
                for (int i = 0; i < 2; ++i) {
                    const int ci = lane + 32 * i;
                    if (ci < nc && !((chosen >> i) & 1u)) {
                        const double v = cval[t * kRouterMaxCand + ci];
                        const int e = cand[t * kRouterMaxCand + ci];
                        if (v > bv || (v == bv && e < be)) { bv = v; be = e; bi = ci; }
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                    if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; bi = oi; }
                }
                if (bi >= 0 && (bi & 31) == lane)
                    chosen |= 1u << (bi >> 5);
                if (lane == 0) { lv[r] = bv; li[r] = be; }
            }
        } else {
            // Degenerate input (more than kRouterMaxCand experts within the
            // bound of the k-th logit): stream every candidate, in ascending
            // id, through a sorted top_k list.
            const float *lt = logit + t * E;
            float dmax = 0.f;
            for (int e = lane; e < E; e += 32)
                dmax = fmaxf(dmax, bound[t * E + e]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
            const double thr = (double)kth_logit(lt, E, top_k) - 2.0 * (double)dmax * 1.0001;
            int n = 0;
            for (int e = 0; e < E; ++e) {
                if ((double)lt[e] < thr)
                    continue;
                const double v = logit_fp64(xs + (size_t)t * H, w_router, bias, H, e);
                if (lane == 0) {
                    if (n < top_k || v > lv[top_k - 1]) {
                        int pos = n < top_k ? n : top_k - 1;
                        while (pos > 0 && v > lv[pos - 1]) {  // equal values keep the lower id first
                            lv[pos] = lv[pos - 1];
                            li[pos] = li[pos - 1];
                            --pos;
                        }
                        lv[pos] = v;
                        li[pos] = e;
                        if (n < top_k)
                            ++n;
                    }
                }
                __syncwarp();
            }
        }
        __syncwarp();
        if (lane < top_k) {
            const double m = lv[0];
            double s = 0.0;
            for (int j = 0; j < top_k; ++j)
                s += exp(lv[j] - m);
            ids[(t0 + t) * top_k + lane] = li[lane];
            weights[(t0 + t) * top_k + lane] = (float)(exp(lv[lane] - m) / s);
        }
    }
}

}  // namespace epk
