// router.cuh -- replicated softmax router with top-k and renormalisation.
//
// fak note "GLM-5.2 multi-GPU: expert-parallel sharding + the resident-fit
// benchmark", "What landed": each rank holds a copy of the router and runs it
// on the same rows, so the ranks agree on the picks.  Softmax over the logits, top_k by logit with ties to the
// lower expert id, weights renormalised over the picked set.
//
// Two kernels, both launched as clusters of CTAs that split the experts and
// meet in CTA 0's shared memory (distributed shared memory):
//  * router_dot2_kernel (up to 32 tokens): every logit as a compensated
//    (Dot2) fp32 dot product, accurate to about 1e-9 (bound below).
//  * router_tiled_kernel (more tokens): register-tiled fp32 logits with a
//    rigorous bound on each logit's rounding error; every expert whose exact
//    logit could reach the k-th largest under those bounds is recomputed by
//    Dot2 before the pick.
// Either way the selection and its order are those of exact arithmetic
// except between logits closer than the Dot2 bound, and the weights carry
// the error of that bound plus one fp32 rounding.
#pragma once

#include "common.cuh"

namespace epk {

constexpr int kRouterCluster = 8;
constexpr int kRouterMaxCand = 64;     // refined candidates per token handled in parallel
constexpr int kRouterRowChunks = 16;   // 16-byte chunks of a router row per lane per round

__host__ __device__ inline uint32_t align_up_u32(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__device__ __forceinline__ void unpack_w8(uint4 v, float (&wf)[8]) {
    wf[0] = bf16_lo(v.x); wf[1] = bf16_hi(v.x); wf[2] = bf16_lo(v.y); wf[3] = bf16_hi(v.y);
    wf[4] = bf16_lo(v.z); wf[5] = bf16_hi(v.z); wf[6] = bf16_lo(v.w); wf[7] = bf16_hi(v.w);
}

// The k-th largest fp32 logit of one token (counted with multiplicity; NaN
// never counts), computed by a warp.  Up to 256 experts the logits sit in
// registers as order-preserving 32-bit keys (NaN and empty slots 0): each
// round takes the warp's largest key and how many lanes' keys equal it by two
// warp reductions, and clears them, until top_k are counted.  Above 256 the
// logits are re-read each round.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t b = __float_as_uint(v);
    return v != v ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ float kth_logit(const float *lt, int E, int top_k) {
    const int lane = (int)lane_id();
    if (E <= 256) {
        uint32_t key[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            key[i] = e < E ? order_key(lt[e]) : 0u;
        }
        int counted = 0;
        for (int r = 0; r < top_k; ++r) {
            uint32_t m = key[0];
#pragma unroll
            for (int i = 1; i < 8; ++i)
                m = max(m, key[i]);
            m = __reduce_max_sync(0xffffffffu, m);
            if (m == 0u)
                return -INFINITY;  // fewer than top_k orderable logits
            uint32_t c = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c += key[i] == m ? 1u : 0u;
                key[i] = key[i] == m ? 0u : key[i];
            }
            counted += (int)__reduce_add_sync(0xffffffffu, c);
            if (counted >= top_k)
                return key_value(m);
        }
        return -INFINITY;
    }
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

// The k-th largest logits of two tokens at once (E <= 256), as kth_logit
// computes each: the two selections interleave, so that each round's warp
// reductions of one token overlap those of the other.
__device__ void kth_logit2(const float *la, const float *lb, int E, int top_k, float &va,
                           float &vb) {
    const int lane = (int)lane_id();
    uint32_t ka[8], kb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        ka[i] = e < E ? order_key(la[e]) : 0u;
        kb[i] = e < E ? order_key(lb[e]) : 0u;
    }
    int ca = 0, cb = 0;
    bool da = false, db = false;
    va = vb = -INFINITY;
    for (int r = 0; r < top_k && !(da && db); ++r) {
        uint32_t ma = ka[0], mb = kb[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            ma = max(ma, ka[i]);
            mb = max(mb, kb[i]);
        }
        ma = __reduce_max_sync(0xffffffffu, ma);
        mb = __reduce_max_sync(0xffffffffu, mb);
        uint32_t na = 0, nb = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            na += ka[i] == ma ? 1u : 0u;
            ka[i] = ka[i] == ma ? 0u : ka[i];
            nb += kb[i] == mb ? 1u : 0u;
            kb[i] = kb[i] == mb ? 0u : kb[i];
        }
        ca += (int)__reduce_add_sync(0xffffffffu, na);
        cb += (int)__reduce_add_sync(0xffffffffu, nb);
        if (!da && (ma == 0u || ca >= top_k)) {
            da = true;
            va = ma == 0u ? -INFINITY : key_value(ma);
        }
        if (!db && (mb == 0u || cb >= top_k)) {
            db = true;
            vb = mb == 0u ? -INFINITY : key_value(mb);
        }
    }
}

// ------------------------------------------------------ compensated logits
// A logit is a dot product of H terms x_h w_h.  With bf16 activations every
// product is exact in fp32 (8 + 8 significant bits); with fp32 activations
// the rounding error of each product is recovered exactly by an FMA.  The
// terms are summed as an unevaluated pair (s, c): s the running fp32 sum and
// c the sum of the exact rounding errors of the additions into s (Knuth's
// TwoSum), the compensated dot product "Dot2" of Ogita, Rump and Oishi
// ("Accurate sum and dot product", SIAM J. Sci. Comput. 26(6), 2005).  Each
// lane sums its terms in two packed chains and the 32 lanes are combined by
// the same error-free step, so the pair differs from the exact dot product
// by at most about gamma_n^2 sum_h |x_h w_h|, gamma_n = n u / (1 - n u),
// u = 2^-24, n = H/64 + 6: about 1e-9 at H = 4096 for unit activations and
// weights of scale 0.02.  fp64 arithmetic is not used for the sums: on this
// part its throughput is a small fraction of fp32's.

// s + p as the pair (s, c): s takes the rounded sum, c the exact error.
__device__ __forceinline__ void dot2_add(float2 &s, float2 &c, float2 p) {
    const float2 sn = add2(s, p);
    const float2 bb = sub2(sn, s);
    c = add2(c, add2(sub2(s, sub2(sn, bb)), sub2(p, bb)));
    s = sn;
}

// Eight terms of one 16-byte weight chunk: wp the weights as fp32 pairs, wn
// their negations (used only for fp32 activations), xp the activations.
template <bool XF32>
__device__ __forceinline__ void dot2_chunk(const float2 (&wp)[4], const float2 (&wn)[4],
                                           const float2 (&xp)[4], float2 &s, float2 &c) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 prod = mul2(wp[p], xp[p]);
        if constexpr (XF32)
            c = sub2(c, ffma2(wn[p], xp[p], prod));  // + (w x - prod), exact
        dot2_add(s, c, prod);
    }
}

__device__ __forceinline__ void dot2_unpack_w(uint4 v, float2 (&wp)[4], float2 (&wn)[4]) {
    wp[0] = bf16x2_to_f2(v.x); wp[1] = bf16x2_to_f2(v.y);
    wp[2] = bf16x2_to_f2(v.z); wp[3] = bf16x2_to_f2(v.w);
    wn[0] = bf16x2_to_f2(v.x ^ 0x80008000u); wn[1] = bf16x2_to_f2(v.y ^ 0x80008000u);
    wn[2] = bf16x2_to_f2(v.z ^ 0x80008000u); wn[3] = bf16x2_to_f2(v.w ^ 0x80008000u);
}

__device__ __forceinline__ float two_sum(float a, float b, float &err) {
    const float s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    err = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
    return s;
}

// The warp's pairs summed into one value (identical in every lane).
__device__ __forceinline__ double dot2_warp_total(float2 s, float2 c) {
    float r;
    float S = two_sum(s.x, s.y, r);
    float C = __fadd_rn(__fadd_rn(c.x, c.y), r);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float So = __shfl_xor_sync(0xffffffffu, S, off);
        const float Co = __shfl_xor_sync(0xffffffffu, C, off);
        S = two_sum(S, So, r);
        C = __fadd_rn(__fadd_rn(C, Co), r);
    }
    return (double)S + (double)C;
}

// An fp64 value and an expert id as one unsigned key that orders by value,
// then by lower id: the value's bits made order-preserving as an unsigned
// integer, with the lowest 10 bits replaced by 1023 - id.  Values closer than
// about 2^-42 of their size (far inside the Dot2 logits' error bound) are
// thereby ordered by id, as exact ties are.  E <= 1024.
__device__ __forceinline__ unsigned long long topk_key(double v, int e) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(v);
    const unsigned long long ord = (b >> 63) ? ~b : (b | 0x8000000000000000ull);
    return (ord & ~0x3ffull) | (unsigned long long)(1023 - e);
}

// One warp: the top_k of E values of one token by value, ties to the lower
// id; lane r < top_k receives the r-th pick's id and value.
__device__ void topk_select_warp(const double *v, int E, int top_k, int &pick_e, double &pick_v) {
    const int lane = (int)lane_id();
    const int per_lane = (E + 31) / 32;
    uint32_t chosen = 0;
    pick_v = 0.0;
    pick_e = 0;
    for (int r = 0; r < top_k; ++r) {
        unsigned long long best = 0ull;  // below every key of a finite value
        for (int i = 0; i < per_lane; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((chosen >> i) & 1u)) {
                const unsigned long long k = topk_key(v[e], e);
                best = k > best ? k : best;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, best, off);
            best = o > best ? o : best;
        }
        const int be = 1023 - (int)(best & 0x3ffull);
        if ((be & 31) == lane)
            chosen |= 1u << (be >> 5);
        if (lane == r) {
            pick_e = be;
            pick_v = v[be];
        }
    }
}

// Softmax weights of a token's picks (lane r < top_k holds the r-th pick's
// id and logit): softmax over the picked set, summed in pick order.
__device__ void softmax_finish_warp(int pick_e, double pick_v, int top_k, int32_t *ids_row,
                                    float *w_row) {
    const int lane = (int)lane_id();
    const double top = __shfl_sync(0xffffffffu, pick_v, 0);
    const double ev = lane < top_k ? exp(pick_v - top) : 0.0;
    double sum = 0.0;
    for (int j = 0; j < top_k; ++j)
        sum += __shfl_sync(0xffffffffu, ev, j);
    if (lane < top_k) {
        ids_row[lane] = pick_e;
        w_row[lane] = (float)(ev / sum);
    }
}

// Softmax router: the picks by logit, weights = softmax over the picked set.
__device__ void topk_softmax_warp(const double *lt, int E, int top_k, int32_t *ids_row,
                                  float *w_row) {
    int pick_e;
    double pick_v;
    topk_select_warp(lt, E, top_k, pick_e, pick_v);
    softmax_finish_warp(pick_e, pick_v, top_k, ids_row, w_row);
}

// Sigmoid router (the GLM variant: sigmoid scores, a bias used in the selection only, weights from the unbiased scores;
// TensorFold #593, "What exists now", glm_route.cu): the picks by key =
// score + bias, weights = scale * score, or scale * score / (sum of the
// picked scores) with normalize.
__device__ void sigmoid_finish_warp(const double *score, int pick_e, int top_k, int normalize,
                                    float scale, int32_t *ids_row, float *w_row) {
    const int lane = (int)lane_id();
    const double sc = lane < top_k ? score[pick_e] : 0.0;
    double sum = 0.0;
    for (int j = 0; j < top_k; ++j)
        sum += __shfl_sync(0xffffffffu, sc, j);
    if (lane < top_k) {
        ids_row[lane] = pick_e;
        w_row[lane] = (float)((double)scale * (normalize ? sc / sum : sc));
    }
}

__device__ void topk_sigmoid_warp(const double *key, const double *score, int E, int top_k,
                                  int normalize, float scale, int32_t *ids_row, float *w_row) {
    int pick_e;
    double pick_v;
    topk_select_warp(key, E, top_k, pick_e, pick_v);
    sigmoid_finish_warp(score, pick_e, top_k, normalize, scale, ids_row, w_row);
}

__device__ __forceinline__ double sigmoid_f64(double l) { return 1.0 / (1.0 + exp(-l)); }

// ------------------------------------------------------ small-batch router
// Up to 32 tokens: every logit by Dot2.  A cluster of 8 CTAs takes TB tokens
// (one or two), CTA r the experts [r E/8, (r+1) E/8); 16 warps per CTA, one
// expert row per warp at a time, each lane 16-byte chunks lane + 32 j of the
// row.  The first chunks of each warp's first row are loaded before
// griddepcontrol.wait (the router weights never come from the previous
// kernel).  Logits go to CTA 0 by distributed shared memory, where one warp
// per token picks and normalises.
constexpr int kRdThreads = 512;
constexpr int kRdWarps = kRdThreads / 32;
constexpr int kRdMaxTB = 2;

struct RdSmem {
    uint32_t x, vals, logit, total;
};

// Up to this many experts the small-batch router picks with the token's keys
// in registers, two warp reductions a round; above, one warp per token
// selects the top_k in top_k rounds of shuffles over shared memory.
constexpr int kRdRankMaxE = 256;

__host__ __device__ inline RdSmem rd_smem_layout(int tb_max, int H, int E) {
    RdSmem s;
    uint32_t o = 0;
    const int per_cta = (E + kRouterCluster - 1) / kRouterCluster;
    s.x = o;     o = align_up_u32(o + (uint32_t)tb_max * H * 4, 16);
    // [2][tb][per_cta] and [2][tb][E]: the logit (softmax) or the key and the
    // score (sigmoid)
    s.vals = o;  o = align_up_u32(o + 2u * tb_max * per_cta * 8, 16);
    s.logit = o; o = align_up_u32(o + 2u * tb_max * E * 8, 16);
    s.total = o;
    return s;
}

__device__ __forceinline__ void rd_load_chunks(const uint4 *__restrict__ wrow, int base, int nck,
                                               uint4 (&wv)[kRouterRowChunks]) {
    const int lane = (int)lane_id();
#pragma unroll
    for (int q = 0; q < kRouterRowChunks; ++q) {
        const int c = base + lane + 32 * q;
        wv[q] = c < nck ? ld_stream_16(wrow + c) : make_uint4(0u, 0u, 0u, 0u);
    }
}

template <bool XF32, int TB, bool SIG>
__global__ void __cluster_dims__(kRouterCluster, 1, 1) __launch_bounds__(kRdThreads, 1)
router_dot2_kernel(const void *__restrict__ x, int64_t T, int H,
                   const uint16_t *__restrict__ w_router, const float *__restrict__ bias, int E,
                   int top_k, int32_t *__restrict__ ids, float *__restrict__ weights,
                   int normalize, float scale) {
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int XB = XF32 ? 4 : 2;
    const RdSmem L = rd_smem_layout(TB, H, E);
    float *xs = reinterpret_cast<float *>(smem + L.x);          // [TB][H]
    double *vals = reinterpret_cast<double *>(smem + L.vals);   // [2][TB][per_cta]
    double *logit = reinterpret_cast<double *>(smem + L.logit); // [2][TB][E], CTA 0

    const uint32_t rank = cluster_ctarank();
    const int64_t t0 = (int64_t)(blockIdx.x / kRouterCluster) * TB;
    const int tb = (T - t0 < (int64_t)TB) ? (int)(T - t0) : TB;
    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int nck = H >> 3;
    const int per_cta = (E + kRouterCluster - 1) / kRouterCluster;
    const int e_lo = (int)rank * per_cta;
    const int e_hi = min(E, e_lo + per_cta);
    const int e_first = e_lo + warp;

    uint4 wv[kRouterRowChunks];
    if (e_first < e_hi)
        rd_load_chunks(reinterpret_cast<const uint4 *>(w_router + (size_t)e_first * H), 0, nck, wv);
    grid_dependents_launch();
    grid_dependency_wait();
    cluster_arrive_relaxed();  // "this CTA runs"; waited for before the first remote store

    // activations of the block as fp32 (bf16 widens exactly)
    {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(x) + (size_t)t0 * H * XB;
        const int n8 = tb * H / 8;
        for (int i = threadIdx.x; i < n8; i += kRdThreads) {
            float4 a, b;
            if constexpr (XF32) {
                a = reinterpret_cast<const float4 *>(src)[2 * i];
                b = reinterpret_cast<const float4 *>(src)[2 * i + 1];
            } else {
                const uint4 v = reinterpret_cast<const uint4 *>(src)[i];
                a = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
                b = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
            }
            reinterpret_cast<float4 *>(xs)[2 * i] = a;
            reinterpret_cast<float4 *>(xs)[2 * i + 1] = b;
        }
    }
    __syncthreads();

    bool have = true;  // wv holds the first chunks of the warp's first row
    for (int e = e_first; e < e_hi; e += kRdWarps) {
        float2 s[TB], c[TB];
#pragma unroll
        for (int t = 0; t < TB; ++t) {
            s[t] = make_float2(0.f, 0.f);
            c[t] = make_float2(0.f, 0.f);
        }
        const uint4 *wrow = reinterpret_cast<const uint4 *>(w_router + (size_t)e * H);
        for (int base = 0; base < nck; base += 32 * kRouterRowChunks) {
            if (!have)
                rd_load_chunks(wrow, base, nck, wv);
            have = false;
#pragma unroll
            for (int q = 0; q < kRouterRowChunks; ++q) {
                const int ch = base + lane + 32 * q;
                if (ch < nck) {
                    float2 wp[4], wn[4];
                    dot2_unpack_w(wv[q], wp, wn);
#pragma unroll
                    for (int t = 0; t < TB; ++t) {
                        if (t < tb) {
                            const float4 *xp4 = reinterpret_cast<const float4 *>(xs + (size_t)t * H) + 2 * ch;
                            const float4 a = xp4[0], b = xp4[1];
                            const float2 xp[4] = {make_float2(a.x, a.y), make_float2(a.z, a.w),
                                                  make_float2(b.x, b.y), make_float2(b.z, b.w)};
                            dot2_chunk<XF32>(wp, wn, xp, s[t], c[t]);
                        }
                    }
                }
            }
        }
        const double b = bias != nullptr ? (double)bias[e] : 0.0;
#pragma unroll
        for (int t = 0; t < TB; ++t) {
            if (t < tb) {
                const double l = dot2_warp_total(s[t], c[t]);
                if (lane == 0) {
                    if constexpr (SIG) {
                        const double sc = sigmoid_f64(l);
                        vals[t * per_cta + (e - e_lo)] = sc + b;
                        vals[(TB + t) * per_cta + (e - e_lo)] = sc;
                    } else {
                        vals[t * per_cta + (e - e_lo)] = l + b;
                    }
                }
            }
        }
    }
    __syncthreads();
    cluster_wait();  // every CTA of the cluster runs: CTA 0's shared memory may be written
    {
        const uint32_t r_logit = map_shared_rank(logit, 0);
        const int n = e_hi - e_lo;
        for (int i = threadIdx.x; i < tb * n; i += kRdThreads) {
            const int t = i / n, j = i - t * n;
            st_cluster_f64(r_logit + 8u * (uint32_t)(t * E + e_lo + j), vals[t * per_cta + j]);
            if (SIG)
                st_cluster_f64(r_logit + 8u * (uint32_t)((TB + t) * E + e_lo + j),
                               vals[(TB + t) * per_cta + j]);
        }
    }
    cluster_sync();  // all logits are in CTA 0
    if (rank != 0)
        return;
    if (E <= kRdRankMaxE) {
        // the pick by warp reductions: warp t holds token t's keys (value,
        // id) in registers, eight per lane, and round r takes the largest
        // (its high half by one reduction, then its low half among the lanes
        // whose largest key shares that high half), which lane r keeps
        if (warp >= tb)
            return;
        const double *lt = logit + warp * E;
        unsigned long long key[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            key[i] = e < E ? topk_key(lt[e], e) : 0ull;
        }
        int pick_e = 0;
        for (int r = 0; r < top_k; ++r) {
            unsigned long long m = key[0];
#pragma unroll
            for (int i = 1; i < 8; ++i)
                m = key[i] > m ? key[i] : m;
            const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(m >> 32));
            const uint32_t lo =
                __reduce_max_sync(0xffffffffu, (uint32_t)(m >> 32) == hi ? (uint32_t)m : 0u);
            const unsigned long long best = ((unsigned long long)hi << 32) | lo;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                key[i] = key[i] == best ? 0ull : key[i];
            if (lane == r)
                pick_e = 1023 - (int)(lo & 0x3ffu);
        }
        if constexpr (SIG) {
            sigmoid_finish_warp(logit + (TB + warp) * E, pick_e, top_k, normalize, scale,
                                ids + (t0 + warp) * top_k, weights + (t0 + warp) * top_k);
        } else {
            const double pick_v = lane < top_k ? lt[pick_e] : 0.0;
            softmax_finish_warp(pick_e, pick_v, top_k, ids + (t0 + warp) * top_k,
                                weights + (t0 + warp) * top_k);
        }
        return;
    }
    if (warp >= tb)
        return;
    if constexpr (SIG)
        topk_sigmoid_warp(logit + warp * E, logit + (TB + warp) * E, E, top_k, normalize, scale,
                          ids + (t0 + warp) * top_k, weights + (t0 + warp) * top_k);
    else
        topk_softmax_warp(logit + warp * E, E, top_k, ids + (t0 + warp) * top_k,
                          weights + (t0 + warp) * top_k);
}

// ------------------------------------------------------- tiled fp32 router
// For larger batches the fp32 logits are a register-tiled SIMT product.  A
// cluster of CE x CK CTAs covers one block of BT tokens: CE = ceil(E / 128)
// expert slices times CK slices of H (CE CK <= 8).  CTA (e, k) accumulates
// the experts [128 e, 128 e + 128) over its k-tiles of 32 values of H; both
// operand tiles are widened to fp32 in shared memory (double-buffered), and
// each thread keeps TM tokens x 4 experts of packed accumulators.  The CK
// partial tiles are then added in a fixed order, each CTA taking a share of
// the tokens.  Every 32-term block is summed on its own (two 16-term packed
// halves) before it joins the running total, which bounds the rounding error
// of a logit by gamma_n sum_h |x_h w_h| + u |l|, n = 32 + (k-tiles per CTA)
// + CK + 2, with sum |x_h w_h| <= ||x|| ||w||.  Each token's logits and bounds
// then go to one CTA of the cluster (token t to CTA t mod CE CK), which picks
// its candidates, refines them by Dot2 and writes its ids and weights.
constexpr int kRtBE = 128;
constexpr int kRtBK = 32;
constexpr int kRtPad = 4;
constexpr int kRtThreads = 256;
constexpr int kRtMaxBT = 32;

__host__ __device__ inline int rt_block_tokens(int E) {
    // the logits and bounds of the block live in CTA 0: BT * E * 8 <= 64 KB
    return E <= 256 ? 32 : (E <= 512 ? 16 : 8);
}

struct RtSmem {
    uint32_t xs, ws, xsq, wsq, part, logit, bound, ncand, cand, cval, cscore, total;
};

__host__ __device__ inline RtSmem rt_smem_layout(int BT, int E) {
    RtSmem s;
    uint32_t o = 0;
    s.xs = o;    o = align_up_u32(o + 2u * BT * (kRtBK + kRtPad) * 4, 16);
    s.ws = o;    o = align_up_u32(o + 2u * kRtBE * (kRtBK + kRtPad) * 4, 16);
    s.xsq = o;   o = align_up_u32(o + (uint32_t)BT * 4, 16);
    s.wsq = o;   o = align_up_u32(o + kRtBE * 4, 16);
    s.part = o;  o = align_up_u32(o + (uint32_t)BT * kRtBE * 4, 16);
    s.logit = o; o = align_up_u32(o + (uint32_t)BT * E * 4, 16);
    s.bound = o; o = align_up_u32(o + (uint32_t)BT * E * 4, 16);
    s.ncand = o; o = align_up_u32(o + (uint32_t)BT * 4, 16);
    s.cand = o;  o = align_up_u32(o + (uint32_t)BT * kRouterMaxCand * 4, 16);
    s.cval = o;  o = align_up_u32(o + (uint32_t)BT * kRouterMaxCand * 8, 16);
    s.cscore = o; o = align_up_u32(o + (uint32_t)BT * kRouterMaxCand * 8, 16);
    s.total = o;
    return s;
}

// Dot2 logit of expert e for one token whose activations are in global
// memory (one warp); eight chunks per lane are loaded before they are used.
template <bool XF32>
__device__ double logit_dot2_global(const void *xrow, const uint16_t *__restrict__ w_router,
                                    const float *__restrict__ bias, int H, int e) {
    constexpr int U = 8;
    const int lane = (int)lane_id();
    const int nck = H >> 3;
    const uint4 *wrow = reinterpret_cast<const uint4 *>(w_router + (size_t)e * H);
    float2 s = make_float2(0.f, 0.f), c = make_float2(0.f, 0.f);
    for (int base = 0; base < nck; base += 32 * U) {
        uint4 wv[U], xv[U][XF32 ? 2 : 1];
#pragma unroll
        for (int q = 0; q < U; ++q) {
            const int ch = base + lane + 32 * q;
            const bool ok = ch < nck;
            wv[q] = ok ? wrow[ch] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int h = 0; h < (XF32 ? 2 : 1); ++h)
                xv[q][h] = ok ? reinterpret_cast<const uint4 *>(xrow)[(XF32 ? 2 : 1) * ch + h]
                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < U; ++q) {
            float2 wp[4], wn[4], xp[4];
            dot2_unpack_w(wv[q], wp, wn);
            if constexpr (XF32) {
                xp[0] = make_float2(__uint_as_float(xv[q][0].x), __uint_as_float(xv[q][0].y));
                xp[1] = make_float2(__uint_as_float(xv[q][0].z), __uint_as_float(xv[q][0].w));
                xp[2] = make_float2(__uint_as_float(xv[q][1].x), __uint_as_float(xv[q][1].y));
                xp[3] = make_float2(__uint_as_float(xv[q][1].z), __uint_as_float(xv[q][1].w));
            } else {
                xp[0] = bf16x2_to_f2(xv[q][0].x); xp[1] = bf16x2_to_f2(xv[q][0].y);
                xp[2] = bf16x2_to_f2(xv[q][0].z); xp[3] = bf16x2_to_f2(xv[q][0].w);
            }
            dot2_chunk<XF32>(wp, wn, xp, s, c);  // zero chunks add exact zeros
        }
    }
    double acc = dot2_warp_total(s, c);
    if (bias != nullptr)
        acc += (double)bias[e];
    return acc;
}

// Dot2 logits of up to NC experts for one token (one warp): the token's
// activation chunks are loaded once per round and the experts' weight chunks
// beside them, so that NC rows are in flight at once instead of one.  Lane
// results are combined as in logit_dot2_global; out[i] (all lanes) includes
// the bias when bias is not NULL.
template <bool XF32, int NC>
__device__ void logit_dot2_multi(const void *xrow, const uint16_t *__restrict__ w_router,
                                 const float *__restrict__ bias, int H, const int *es, int n,
                                 double (&out)[NC]) {
    constexpr int U = 8;
    const int lane = (int)lane_id();
    const int nck = H >> 3;
    float2 s[NC], c[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        s[i] = make_float2(0.f, 0.f);
        c[i] = make_float2(0.f, 0.f);
    }
    const uint4 *wrow[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i)
        wrow[i] = reinterpret_cast<const uint4 *>(w_router + (size_t)es[i < n ? i : 0] * H);
    for (int base = 0; base < nck; base += 32 * U) {
        uint4 wv[NC][U], xv[U][XF32 ? 2 : 1];
#pragma unroll
        for (int q = 0; q < U; ++q) {
            const int ch = base + lane + 32 * q;
            const bool ok = ch < nck;
#pragma unroll
            for (int h = 0; h < (XF32 ? 2 : 1); ++h)
                xv[q][h] = ok ? reinterpret_cast<const uint4 *>(xrow)[(XF32 ? 2 : 1) * ch + h]
                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int i = 0; i < NC; ++i)
                wv[i][q] = (ok && i < n) ? wrow[i][ch] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < U; ++q) {
            float2 xp[4];
            if constexpr (XF32) {
                xp[0] = make_float2(__uint_as_float(xv[q][0].x), __uint_as_float(xv[q][0].y));
                xp[1] = make_float2(__uint_as_float(xv[q][0].z), __uint_as_float(xv[q][0].w));
                xp[2] = make_float2(__uint_as_float(xv[q][1].x), __uint_as_float(xv[q][1].y));
                xp[3] = make_float2(__uint_as_float(xv[q][1].z), __uint_as_float(xv[q][1].w));
            } else {
                xp[0] = bf16x2_to_f2(xv[q][0].x); xp[1] = bf16x2_to_f2(xv[q][0].y);
                xp[2] = bf16x2_to_f2(xv[q][0].z); xp[3] = bf16x2_to_f2(xv[q][0].w);
            }
#pragma unroll
            for (int i = 0; i < NC; ++i) {
                float2 wp[4], wn[4];
                dot2_unpack_w(wv[i][q], wp, wn);
                dot2_chunk<XF32>(wp, wn, xp, s[i], c[i]);  // zero chunks add exact zeros
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        double acc = dot2_warp_total(s[i], c[i]);
        if (bias != nullptr && i < n)
            acc += (double)bias[es[i]];
        out[i] = acc;
    }
}

// The pick of the tokens a CTA owns, shared by the routers that first form
// fp32 logits with an error bound (router_tiled_kernel, router_tc_kernel).
// Owned token j (0 <= j < n_local) is token t0 + tbase + tstride j of the
// batch; logit [n_local][E] (the selection key for the sigmoid variant) is in
// shared memory and bound_at(j, e) gives the bound of its error.  For every
// owned token: its candidates (every expert whose exact value could reach the
// k-th largest under the bounds), their Dot2 logits (one warp per candidate),
// the pick on those values and the weights.  More than max_cand candidates
// (a degenerate input) take a slower path over every expert that clears the
// threshold, in ascending id.
template <bool XF32, bool SIG, int NWARPS, typename BoundAt>
__device__ void router_pick_owned(int n_local, int tbase, int tstride, int64_t t0, const void *x,
                                  int H, const uint16_t *__restrict__ w_router,
                                  const float *__restrict__ bias, int E, int top_k,
                                  int32_t *__restrict__ ids, float *__restrict__ weights,
                                  int normalize, float scale, const float *logit, int *ncand,
                                  int *cand, double *cval, double *cscore, int max_cand,
                                  BoundAt bound_at) {
    constexpr int XB = XF32 ? 4 : 2;
    const int warp = (int)(threadIdx.x >> 5), lane = (int)lane_id();
    // candidates per owned token (one warp each): every expert whose exact
    // logit could reach the k-th largest under the bounds.  A warp's tokens
    // j and j + NWARPS find their k-th logits together.
    float vk_next = 0.f;
    for (int j = warp; j < n_local; j += NWARPS) {
        const float *lt = logit + j * E;
        float vk;
        if (E <= 256 && ((j - warp) / NWARPS) % 2 == 1) {
            vk = vk_next;  // found with the previous token's
        } else if (E <= 256 && j + NWARPS < n_local) {
            kth_logit2(lt, logit + (j + NWARPS) * E, E, top_k, vk, vk_next);
        } else {
            vk = kth_logit(lt, E, top_k);
        }
        float dmax = 0.f;
        for (int e = lane; e < E; e += 32)
            dmax = fmaxf(dmax, bound_at(j, e));
        // bounds are positive (or NaN, dropped by fmaxf): their bits order as integers
        dmax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(dmax)));
        // the largest float not above the threshold: the same experts pass,
        // and at most those equal to it besides
        const float thr = __double2float_rd((double)vk - 2.0 * (double)dmax * 1.0001);
        int count = 0;
        for (int i = 0; i < (E + 31) / 32; ++i) {
            const int e = lane + 32 * i;
            const bool c = e < E && lt[e] >= thr;
            const uint32_t m = __ballot_sync(0xffffffffu, c);
            const int pos = count + __popc(m & ((1u << lane) - 1u));
            if (c && pos < max_cand)
                cand[j * max_cand + pos] = e;
            count += __popc(m);
        }
        if (lane == 0)
            ncand[j] = count;
    }
    __syncthreads();

    // Dot2 logits of the owned tokens' candidates, spread over the warps in
    // groups of up to NG candidates of one token (one warp refines a group
    // at once: its rows stream side by side; a short group's missing rows
    // add zeros, cheaper than more code variants in the instruction cache)
    {
        constexpr int NG = XF32 ? 2 : 4;
        int mine = 0;
        for (int j = 0; j < n_local; ++j) {
            const int t = tbase + tstride * j;
            const int nc = ncand[j] <= max_cand ? ncand[j] : 0;
            const uint8_t *xrow = reinterpret_cast<const uint8_t *>(x) + (size_t)(t0 + t) * H * XB;
            for (int c0 = 0; c0 < nc; c0 += NG) {
                if ((mine++ % NWARPS) != warp)
                    continue;
                const int n = nc - c0 < NG ? nc - c0 : NG;
                const int *es = cand + j * max_cand + c0;
                double v[NG];
                logit_dot2_multi<XF32, NG>(xrow, w_router, SIG ? nullptr : bias, H, es, n, v);
                if (lane == 0) {
                    for (int i = 0; i < n; ++i) {
                        if (SIG) {
                            const double sc = sigmoid_f64(v[i]);
                            cval[j * max_cand + c0 + i] =
                                sc + (bias != nullptr ? (double)bias[es[i]] : 0.0);
                            cscore[j * max_cand + c0 + i] = sc;
                        } else {
                            cval[j * max_cand + c0 + i] = v[i];
                        }
                    }
                }
            }
        }
    }
    __syncthreads();

    // pick top_k on the refined values of each owned token, weigh, write
    for (int j = warp; j < n_local; j += NWARPS) {
        const int t = tbase + tstride * j;
        const int nc = ncand[j];
        double bv_list = 0.0, top = 0.0, bs_list = 0.0;  // lane r: the r-th pick's value, score
        int be_list = 0;
        if (nc <= 32 && nc <= max_cand) {
            // lane ci holds candidate ci; its rank among the orderable ones
            // (larger value first, ties to the lower id; NaN never picked)
            // sends it to slot rank of the token's lists
            const int base = j * max_cand;
            const bool ok0 = lane < nc;
            const double v = ok0 ? cval[base + lane] : 0.0;
            const int e = ok0 ? cand[base + lane] : 0x7fffffff;
            const double sc = (SIG && ok0) ? cscore[base + lane] : 0.0;
            const bool ok = ok0 && v == v;
            int rank = 0;
            for (int q = 0; q < nc; ++q) {
                const double ov = __shfl_sync(0xffffffffu, v, q);
                const int oe = __shfl_sync(0xffffffffu, e, q);
                rank += (ov > v || (ov == v && oe < e)) ? 1 : 0;  // NaN ov: false
            }
            const int n_ok = __popc(__ballot_sync(0xffffffffu, ok));
            __syncwarp();
            if (ok && rank < top_k) {
                cval[base + rank] = v;
                cand[base + rank] = e;
                if (SIG)
                    cscore[base + rank] = sc;
            }
            __syncwarp();
            if (lane < top_k) {
                if (lane < n_ok) {
                    bv_list = cval[base + lane];
                    be_list = cand[base + lane];
                    if (SIG)
                        bs_list = cscore[base + lane];
                } else {
                    bv_list = -INFINITY;
                    be_list = 0x7fffffff;
                }
            }
            top = __shfl_sync(0xffffffffu, bv_list, 0);
        } else if (nc <= max_cand) {
            uint32_t chosen = 0;
            for (int r = 0; r < top_k; ++r) {
                double bv = -INFINITY;
                int be = 0x7fffffff, bi = -1;
                for (int i = 0; i < (max_cand + 31) / 32; ++i) {
                    const int ci = lane + 32 * i;
                    if (ci < nc && !((chosen >> i) & 1u)) {
                        const double v = cval[j * max_cand + ci];
                        const int e = cand[j * max_cand + ci];
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
                if (r == 0)
                    top = bv;
                if (lane == r) {
                    bv_list = bv;
                    be_list = be;
                    if (SIG && bi >= 0)
                        bs_list = cscore[j * max_cand + bi];
                }
            }
        } else {
            // degenerate input: every candidate in ascending id through a
            // sorted top_k list kept in registers of lanes 0..top_k-1
            const float *lt = logit + j * E;
            float dmax = 0.f;
            for (int e = lane; e < E; e += 32)
                dmax = fmaxf(dmax, bound_at(j, e));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
            const double thr = (double)kth_logit(lt, E, top_k) - 2.0 * (double)dmax * 1.0001;
            const uint8_t *xrow = reinterpret_cast<const uint8_t *>(x) + (size_t)(t0 + t) * H * XB;
            double lv = -INFINITY;  // lane j holds the j-th best so far
            double ls = 0.0;        // and its score (sigmoid)
            int li = 0x7fffffff;
            for (int e = 0; e < E; ++e) {
                if ((double)lt[e] < thr)
                    continue;
                double v, sc = 0.0;
                if (SIG) {
                    sc = sigmoid_f64(logit_dot2_global<XF32>(xrow, w_router, nullptr, H, e));
                    v = sc + (bias != nullptr ? (double)bias[e] : 0.0);
                } else {
                    v = logit_dot2_global<XF32>(xrow, w_router, bias, H, e);
                }
                // insert: lanes whose value ranks below v shift down by one
                const bool below = !(lv > v || (lv == v && li < e));
                const uint32_t m = __ballot_sync(0xffffffffu, below && lane < top_k);
                const int pos = m ? __ffs(m) - 1 : top_k;
                const double pv = __shfl_up_sync(0xffffffffu, lv, 1);
                const double ps = __shfl_up_sync(0xffffffffu, ls, 1);
                const int pi = __shfl_up_sync(0xffffffffu, li, 1);
                if (lane < top_k && pos < top_k) {
                    if (lane == pos) { lv = v; ls = sc; li = e; }
                    else if (lane > pos) { lv = pv; ls = ps; li = pi; }
                }
            }
            top = __shfl_sync(0xffffffffu, lv, 0);
            bv_list = lv;
            bs_list = ls;
            be_list = li;
        }
        double wv;
        if (SIG) {
            double ssum = 0.0;
            for (int jj = 0; jj < top_k; ++jj)
                ssum += __shfl_sync(0xffffffffu, lane < top_k ? bs_list : 0.0, jj);
            wv = (double)scale * (normalize ? bs_list / ssum : bs_list);
        } else {
            const double ev = lane < top_k ? exp(bv_list - top) : 0.0;
            double ssum = 0.0;
            for (int jj = 0; jj < top_k; ++jj)
                ssum += __shfl_sync(0xffffffffu, ev, jj);
            wv = ev / ssum;
        }
        if (lane < top_k) {
            ids[(t0 + t) * top_k + lane] = be_list;
            weights[(t0 + t) * top_k + lane] = (float)wv;
        }
    }
}

template <bool XF32, int TM, bool SIG>
__global__ void __launch_bounds__(kRtThreads, 1)
router_tiled_kernel(const void *__restrict__ x, int64_t T, int H,
                    const uint16_t *__restrict__ w_router, const float *__restrict__ bias, int E,
                    int top_k, int32_t *__restrict__ ids, float *__restrict__ weights, int CE,
                    int CK, int normalize, float scale, float *__restrict__ dump_logit,
                    float *__restrict__ dump_bound) {
    constexpr int BT = 8 * TM;             // tokens per cluster
    constexpr int XB = XF32 ? 4 : 2;
    constexpr int LD = kRtBK + kRtPad;     // padded row of a k-tile, in floats
    extern __shared__ __align__(1024) uint8_t smem[];
    const RtSmem L = rt_smem_layout(BT, E);
    float *xs = reinterpret_cast<float *>(smem + L.xs);       // [2][BT][LD]
    float *ws = reinterpret_cast<float *>(smem + L.ws);       // [2][kRtBE][LD]
    float *xsq = reinterpret_cast<float *>(smem + L.xsq);
    float *wsq = reinterpret_cast<float *>(smem + L.wsq);
    float *part = reinterpret_cast<float *>(smem + L.part);   // [BT][kRtBE], this CTA's k-slice
    float *logit = reinterpret_cast<float *>(smem + L.logit); // [BT][E], CTA 0
    float *bound = reinterpret_cast<float *>(smem + L.bound); // [BT][E], CTA 0
    int *ncand = reinterpret_cast<int *>(smem + L.ncand);
    int *cand = reinterpret_cast<int *>(smem + L.cand);
    double *cval = reinterpret_cast<double *>(smem + L.cval);      // refined logit or key
    double *cscore = reinterpret_cast<double *>(smem + L.cscore);  // refined score (sigmoid)

    grid_dependents_launch();
    grid_dependency_wait();

    const uint32_t rank = cluster_ctarank();
    const int64_t t0 = (int64_t)blockIdx.y * BT;
    const int tb = (T - t0 < (int64_t)BT) ? (int)(T - t0) : BT;
    const int e_part = (int)rank % CE, k_part = (int)rank / CE;
    const int e0 = e_part * kRtBE;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int tx = lane, ty = warp;        // experts tx + 32 j, tokens TM ty + i

    // global -> registers for one k-tile: x (BT x 32) and w (128 x 32) as
    // 16-byte chunks of 8 bf16 (x fp32: 8 floats in two chunks)
    constexpr int XCH = BT * (kRtBK / 8);          // 8-value chunks of the x tile
    constexpr int WCH = kRtBE * (kRtBK / 8);       // 512
    float xr[(XCH + kRtThreads - 1) / kRtThreads][8];
    float wr[WCH / kRtThreads][8];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int q = 0; q < (XCH + kRtThreads - 1) / kRtThreads; ++q) {
            const int ch = tid + q * kRtThreads;
            const int row = ch / (kRtBK / 8), kc = (ch % (kRtBK / 8)) * 8;
            bool ok = ch < XCH && row < tb && k0 + kc < H;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                xr[q][j] = 0.f;
            if (ok) {
                const uint8_t *src = reinterpret_cast<const uint8_t *>(x) +
                                     ((size_t)(t0 + row) * H + k0 + kc) * XB;
                if constexpr (XF32) {
                    const float4 a = reinterpret_cast<const float4 *>(src)[0];
                    const float4 b = reinterpret_cast<const float4 *>(src)[1];
                    xr[q][0] = a.x; xr[q][1] = a.y; xr[q][2] = a.z; xr[q][3] = a.w;
                    xr[q][4] = b.x; xr[q][5] = b.y; xr[q][6] = b.z; xr[q][7] = b.w;
                } else {
                    unpack_w8(*reinterpret_cast<const uint4 *>(src), xr[q]);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < WCH / kRtThreads; ++q) {
            const int ch = tid + q * kRtThreads;
            const int row = ch / (kRtBK / 8), kc = (ch % (kRtBK / 8)) * 8;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                wr[q][j] = 0.f;
            if (e0 + row < E && k0 + kc < H)
                unpack_w8(ld_stream_16(w_router + (size_t)(e0 + row) * H + k0 + kc), wr[q]);
        }
    };
    // A thread stashes the same rows' chunks in every k-tile, so it also
    // keeps their running sums of squares (for the error bound).
    constexpr int XQ = (XCH + kRtThreads - 1) / kRtThreads;
    constexpr int WQ = WCH / kRtThreads;
    float2 x2[XQ], w2[WQ];
#pragma unroll
    for (int q = 0; q < XQ; ++q)
        x2[q] = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < WQ; ++q)
        w2[q] = make_float2(0.f, 0.f);
    auto stash = [&](int buf) {
#pragma unroll
        for (int q = 0; q < XQ; ++q) {
            const int ch = tid + q * kRtThreads;
            if (ch < XCH) {
                const int row = ch / (kRtBK / 8), kc = (ch % (kRtBK / 8)) * 8;
                float4 *d = reinterpret_cast<float4 *>(xs + (size_t)(buf * BT + row) * LD + kc);
                d[0] = make_float4(xr[q][0], xr[q][1], xr[q][2], xr[q][3]);
                d[1] = make_float4(xr[q][4], xr[q][5], xr[q][6], xr[q][7]);
#pragma unroll
                for (int j = 0; j < 8; j += 2)
                    x2[q] = ffma2(make_float2(xr[q][j], xr[q][j + 1]),
                                  make_float2(xr[q][j], xr[q][j + 1]), x2[q]);
            }
        }
#pragma unroll
        for (int q = 0; q < WQ; ++q) {
            const int ch = tid + q * kRtThreads;
            const int row = ch / (kRtBK / 8), kc = (ch % (kRtBK / 8)) * 8;
            float4 *d = reinterpret_cast<float4 *>(ws + (size_t)(buf * kRtBE + row) * LD + kc);
            d[0] = make_float4(wr[q][0], wr[q][1], wr[q][2], wr[q][3]);
            d[1] = make_float4(wr[q][4], wr[q][5], wr[q][6], wr[q][7]);
#pragma unroll
            for (int j = 0; j < 8; j += 2)
                w2[q] = ffma2(make_float2(wr[q][j], wr[q][j + 1]),
                              make_float2(wr[q][j], wr[q][j + 1]), w2[q]);
        }
    };

    float acc[TM][4];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.f;
    const int nkt = (H + kRtBK - 1) / kRtBK;
    const int kt_lo = nkt * k_part / CK, kt_hi = nkt * (k_part + 1) / CK;
    if (kt_lo < kt_hi) {
        fetch(kt_lo * kRtBK);
        stash(0);
    }
    __syncthreads();
    for (int kt = kt_lo; kt < kt_hi; ++kt) {
        const int buf = (kt - kt_lo) & 1;
        if (kt + 1 < kt_hi)
            fetch((kt + 1) * kRtBK);
        // two 16-term packed halves per 32-term block
        float2 blk[TM][4];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                blk[i][j] = make_float2(0.f, 0.f);
        const float *xb = xs + (size_t)buf * BT * LD;
        const float *wb = ws + (size_t)buf * kRtBE * LD;
#pragma unroll
        for (int k = 0; k < kRtBK; k += 4) {
            float4 xv[TM], wv[4];
#pragma unroll
            for (int i = 0; i < TM; ++i)
                xv[i] = *reinterpret_cast<const float4 *>(xb + (size_t)(TM * ty + i) * LD + k);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                wv[j] = *reinterpret_cast<const float4 *>(wb + (size_t)(tx + 32 * j) * LD + k);
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    blk[i][j] = ffma2(make_float2(xv[i].x, xv[i].y), make_float2(wv[j].x, wv[j].y),
                                      blk[i][j]);
                    blk[i][j] = ffma2(make_float2(xv[i].z, xv[i].w), make_float2(wv[j].z, wv[j].w),
                                      blk[i][j]);
                }
        }
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc[i][j] += blk[i][j].x + blk[i][j].y;
        // the other buffer was last read before the previous barrier
        if (kt + 1 < kt_hi) {
            stash(buf ^ 1);
            __syncthreads();
        }
    }
    // this CTA's k-slice: partial sums and sums of squares
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            part[(TM * ty + i) * kRtBE + tx + 32 * j] = acc[i][j];
    // a row's chunks sit in 4 adjacent lanes (ch = 4 row + c)
#pragma unroll
    for (int q = 0; q < XQ; ++q) {
        float v = x2[q].x + x2[q].y;
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        const int ch = tid + q * kRtThreads;
        if (ch < XCH && (ch & 3) == 0)
            xsq[ch >> 2] = v;
    }
#pragma unroll
    for (int q = 0; q < WQ; ++q) {
        float v = w2[q].x + w2[q].y;
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        const int ch = tid + q * kRtThreads;
        if ((ch & 3) == 0)
            wsq[ch >> 2] = v;
    }
    __syncthreads();
    cluster_sync();  // every CTA runs and has its partial tile in place
    // Token t of the block belongs to CTA t mod NC of the cluster (local row
    // t / NC): its logits and bounds are delivered there, and that CTA picks
    // its candidates, refines them and writes its ids and weights.
    const int NC = CE * CK;
    const int n_local = (tb - (int)rank + NC - 1) / NC;  // tokens this CTA owns
    {
        // CTA (e, k) adds the CK partials of tokens [BT k / CK, BT (k+1) / CK)
        // of expert slice e, in ascending k-slice order
        const float u = 5.9604644775390625e-8f;  // 2^-24
        const float n = (float)(kRtBK + (nkt + CK - 1) / CK + CK + 2);
        const float gam = n * u / (1.0f - n * u);
        const int t_lo = BT * k_part / CK, t_hi = BT * (k_part + 1) / CK;
        for (int idx = tid; idx < (t_hi - t_lo) * kRtBE; idx += kRtThreads) {
            const int t = t_lo + idx / kRtBE, el = idx % kRtBE;
            const int e = e0 + el;
            if (t >= tb || e >= E)
                continue;
            float sum = 0.f, x2 = 0.f, w2 = 0.f;
            for (int j = 0; j < CK; ++j) {
                const uint32_t r = (uint32_t)(e_part + CE * j);
                sum += ld_cluster_f32(map_shared_rank(part + t * kRtBE + el, r));
                x2 += ld_cluster_f32(map_shared_rank(xsq + t, r));
                w2 += ld_cluster_f32(map_shared_rank(wsq + el, r));
            }
            const float b = bias != nullptr ? bias[e] : 0.f;
            float l, d;
            if (SIG) {
                // key = sigmoid(l) + b; the sigmoid's slope is at most 1/4, and
                // 4e-7 (1 + |key|) covers its fp32 evaluation and the sum
                const float d_l = 1.5f * (gam * sqrtf(x2) * sqrtf(w2) + u * fabsf(sum)) + 1e-30f;
                l = 1.0f / (1.0f + expf(-sum)) + b;
                d = 0.25f * d_l + 4e-7f * (1.0f + fabsf(l));
            } else {
                l = sum + b;
                d = 1.5f * (gam * sqrtf(x2) * sqrtf(w2) + u * fabsf(l)) + 1e-30f;
            }
            const uint32_t owner = (uint32_t)(t % NC), row = (uint32_t)(t / NC);
            st_cluster_f32(map_shared_rank(logit + row * E + e, owner), l);
            st_cluster_f32(map_shared_rank(bound + row * E + e, owner), d);
        }
    }
    cluster_sync();  // every token's logits and bounds are with its owner; no
                     // shared memory of another CTA is used after this point
    if (dump_logit != nullptr) {
        // inspection (moe_route_logits): the fp32 logits and their bounds
        for (int idx = tid; idx < n_local * E; idx += kRtThreads) {
            const int j = idx / E, e = idx - j * E;
            const int64_t t = t0 + (int)rank + NC * j;
            dump_logit[t * E + e] = logit[j * E + e];
            dump_bound[t * E + e] = bound[j * E + e];
        }
        return;
    }
    router_pick_owned<XF32, SIG, kRtThreads / 32>(
        n_local, (int)rank, NC, t0, x, H, w_router, bias, E, top_k, ids, weights, normalize,
        scale, logit, ncand, cand, cval, cscore, kRouterMaxCand,
        [&](int j, int e) { return bound[j * E + e]; });
}

}  // namespace epk
