// router.cuh -- replicated softmax router with top-k and renormalisation.
//
// fak note "GLM-5.2 multi-GPU: expert-parallel sharding + the resident-fit
// benchmark", "What landed": the router runs replicated and every rank picks
// the same top-k.  Softmax over the logits, top_k by logit with ties to the
// lower expert id, weights renormalised over the picked set.
//
// One thread-block cluster of kRouterCluster CTAs handles a block of up to
// kRouterMaxTB tokens.  CTA r of the cluster computes the fp32 logits of its
// slice of experts for those tokens (the x block sits in its shared memory,
// the router rows stream from HBM with 16-byte loads), together with a
// rigorous bound on each logit's rounding error, and stores both into the
// shared memory of CTA 0 (distributed shared memory).  CTA 0 then finds, per
// token, every expert that could belong to the exact top-k under those bounds,
// recomputes exactly those logits in fp64, and makes the pick and the weights
// from the fp64 values.  The selection and the weights are therefore those of
// exact arithmetic up to fp64 rounding.
#pragma once

#include "common.cuh"

namespace epk {

constexpr int kRouterCluster = 8;
constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;
constexpr int kRouterMaxTB = 8;        // tokens per cluster
constexpr int kRouterMaxK = 16;
constexpr int kRouterMaxCand = 64;     // fp64 candidates per token handled in parallel
constexpr int kRouterXBudget = 96 * 1024;

struct RouterSmem {
    // byte offsets into dynamic shared memory
    uint32_t x, logit, bound, xnorm2, ncand, cand, cval, list_val, list_id, total;
};

__host__ __device__ inline uint32_t align_up_u32(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline RouterSmem router_smem_layout(int tb_max, int H, int x_bytes, int E) {
    RouterSmem s;
    uint32_t o = 0;
    s.x = o;        o = align_up_u32(o + (uint32_t)tb_max * H * x_bytes, 16);
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

// Eight activations of token row `xs_row` at 16-byte chunk c, as floats.
template <bool XF32>
__device__ __forceinline__ void load_x8(const uint8_t *xs_row, int c, float (&xf)[8]) {
    if constexpr (XF32) {
        const float4 *p = reinterpret_cast<const float4 *>(xs_row) + 2 * c;
        float4 a = p[0], b = p[1];
        xf[0] = a.x; xf[1] = a.y; xf[2] = a.z; xf[3] = a.w;
        xf[4] = b.x; xf[5] = b.y; xf[6] = b.z; xf[7] = b.w;
    } else {
        uint4 v = reinterpret_cast<const uint4 *>(xs_row)[c];
        xf[0] = bf16_lo(v.x); xf[1] = bf16_hi(v.x); xf[2] = bf16_lo(v.y); xf[3] = bf16_hi(v.y);
        xf[4] = bf16_lo(v.z); xf[5] = bf16_hi(v.z); xf[6] = bf16_lo(v.w); xf[7] = bf16_hi(v.w);
    }
}

__device__ __forceinline__ void unpack_w8(uint4 v, float (&wf)[8]) {
    wf[0] = bf16_lo(v.x); wf[1] = bf16_hi(v.x); wf[2] = bf16_lo(v.y); wf[3] = bf16_hi(v.y);
    wf[4] = bf16_lo(v.z); wf[5] = bf16_hi(v.z); wf[6] = bf16_lo(v.w); wf[7] = bf16_hi(v.w);
}

// fp64 logit of expert e for the token whose activations are at xs_row.
template <bool XF32>
__device__ double logit_fp64(const uint8_t *xs_row, const uint16_t *__restrict__ w_router,
                             const float *__restrict__ bias, int H, int e) {
    const int lane = (int)lane_id();
    const int nck = H >> 3;
    const uint16_t *wrow = w_router + (size_t)e * H;
    double acc = 0.0;
    for (int c = lane; c < nck; c += 32) {
        uint4 wv = *reinterpret_cast<const uint4 *>(wrow + (size_t)c * 8);
        float wf[8], xf[8];
        unpack_w8(wv, wf);
        load_x8<XF32>(xs_row, c, xf);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            acc = fma((double)xf[j], (double)wf[j], acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (bias != nullptr)
        acc += (double)bias[e];
    return acc;
}

template <bool XF32>
__global__ void __cluster_dims__(kRouterCluster, 1, 1) __launch_bounds__(kRouterThreads, 1)
router_topk_kernel(const void *__restrict__ x, int64_t T, int H,
                   const uint16_t *__restrict__ w_router, const float *__restrict__ bias, int E,
                   int top_k, int tb_max, int32_t *__restrict__ ids, float *__restrict__ weights) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int XB = XF32 ? 4 : 2;
    const RouterSmem L = router_smem_layout(tb_max, H, XB, E);
    uint8_t *xs = smem + L.x;
    float *logit = reinterpret_cast<float *>(smem + L.logit);     // [kRouterMaxTB][E], CTA 0
    float *bound = reinterpret_cast<float *>(smem + L.bound);     // [kRouterMaxTB][E], CTA 0
    float *xnorm2 = reinterpret_cast<float *>(smem + L.xnorm2);
    int *ncand = reinterpret_cast<int *>(smem + L.ncand);
    int *cand = reinterpret_cast<int *>(smem + L.cand);
    double *cval = reinterpret_cast<double *>(smem + L.cval);
    double *list_val = reinterpret_cast<double *>(smem + L.list_val);
    int *list_id = reinterpret_cast<int *>(smem + L.list_id);

    const uint32_t rank = cluster_ctarank();
    const int64_t t0 = (int64_t)(blockIdx.x / kRouterCluster) * tb_max;
    const int tb = (T - t0 < (int64_t)tb_max) ? (int)(T - t0) : tb_max;
    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int nck = H >> 3;

    // ---- phase 1: this block's activations into shared memory, ||x_t||^2
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            reinterpret_cast<const uint8_t *>(x) + (size_t)t0 * H * XB);
        uint4 *dst = reinterpret_cast<uint4 *>(xs);
        const int n16 = tb * H * XB / 16;
        for (int i = threadIdx.x; i < n16; i += kRouterThreads)
            dst[i] = src[i];
    }
    __syncthreads();
    if (warp < tb) {
        const uint8_t *row = xs + (size_t)warp * H * XB;
        float s = 0.f;
        for (int c = lane; c < nck; c += 32) {
            float xf[8];
            load_x8<XF32>(row, c, xf);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                s = fmaf(xf[j], xf[j], s);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0)
            xnorm2[warp] = s;
    }
    cluster_sync();  // every CTA of the cluster is running; x block and norms visible

    // ---- phase 2: fp32 logits of this CTA's experts, with error bounds
    {
        const int per_cta = (E + kRouterCluster - 1) / kRouterCluster;
        const int e_lo = (int)rank * per_cta;
        const int e_hi = min(E, e_lo + per_cta);
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
            const uint16_t *wrow = w_router + (size_t)e * H;
#pragma unroll 2
            for (int c = lane; c < nck; c += 32) {
                float wf[8];
                unpack_w8(ld_stream_16(wrow + (size_t)c * 8), wf);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    wsq = fmaf(wf[j], wf[j], wsq);
#pragma unroll
                for (int t = 0; t < kRouterMaxTB; ++t) {
                    if (t < tb) {
                        float xf[8];
                        load_x8<XF32>(xs + (size_t)t * H * XB, c, xf);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            acc[t] = fmaf(xf[j], wf[j], acc[t]);
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
    if (rank != 0)
        return;

    // ---- phase 3 (CTA 0): candidates per token
    if (warp < tb) {
        const int t = warp;
        const float *lt = logit + t * E;
        const float *bt = bound + t * E;
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
        float dmax = 0.f;
        for (int e = lane; e < E; e += 32)
            dmax = fmaxf(dmax, bt[e]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
        // every expert whose exact logit could reach the k-th one
        const double thr = (double)vk - 2.0 * (double)dmax * 1.0001;
        int count = 0;
        for (int i = 0; i < per_lane; ++i) {
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
    __syncthreads();

    // ---- fp64 logits of the candidates, all warps in parallel
    {
        // (token, candidate) pairs of the tokens with at most kRouterMaxCand
        // candidates, enumerated token by token
        int total = 0;
        for (int t = 0; t < tb; ++t)
            total += ncand[t] <= kRouterMaxCand ? ncand[t] : 0;
        for (int p = warp; p < total; p += kRouterWarps) {
            int t = 0, ci = p;
            while (true) {
                const int c = ncand[t] <= kRouterMaxCand ? ncand[t] : 0;
                if (ci < c)
                    break;
                ci -= c;
                ++t;
            }
            const int e = cand[t * kRouterMaxCand + ci];
            const double v = logit_fp64<XF32>(xs + (size_t)t * H * XB, w_router, bias, H, e);
            if (lane == 0)
                cval[t * kRouterMaxCand + ci] = v;
        }
    }
    __syncthreads();

    // ---- pick top_k on the fp64 logits, renormalise, write
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
            // bound of the k-th logit): stream every candidate through a
            // sorted top_k list, in ascending expert id.
            const float *lt = logit + t * E;
            float dmax = 0.f;
            for (int e = lane; e < E; e += 32)
                dmax = fmaxf(dmax, bound[t * E + e]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
            // the k-th fp32 logit again (the candidate test of phase 3)
            float vk = -INFINITY;
            {
                uint32_t chosen = 0;
                const int per_lane = (E + 31) / 32;
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
            }
            const double thr = (double)vk - 2.0 * (double)dmax * 1.0001;
            int n = 0;
            for (int e = 0; e < E; ++e) {
                if ((double)lt[e] < thr)
                    continue;
                const double v = logit_fp64<XF32>(xs + (size_t)t * H * XB, w_router, bias, H, e);
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
        if (lane == 0) {
            const double m = lv[0];
            double s = 0.0;
            for (int j = 0; j < top_k; ++j)
                s += exp(lv[j] - m);
            for (int j = 0; j < top_k; ++j) {
                ids[(t0 + t) * top_k + j] = li[j];
                weights[(t0 + t) * top_k + j] = (float)(exp(lv[j] - m) / s);
            }
        }
    }
}

}  // namespace epk
