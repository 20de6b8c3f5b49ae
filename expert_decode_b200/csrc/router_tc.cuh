// router_tc.cuh -- the router for batches of more than 32 tokens of bf16
// activations (E <= 256) with its logits on the tensor cores.
//
// The same operation as router_tiled_kernel (fak note "GLM-5.2 multi-GPU",
// "What landed": every rank runs the router on the same rows), with the
// logit contraction l = W_router x moved from fp32 CUDA-core FMAs to tcgen05:
//
//  * A cluster of CK CTAs (2 <= CK <= 8) takes a tile of 64 tokens; CTA k of
//    the cluster contracts the k-th of CK slices of H.  Warp 0 issues TMA
//    loads (128-byte swizzle, each CTA its own copy) of the router weights,
//    one 128-expert box per MMA M tile (MT = 1 or 2), and of the 64 token
//    rows; warp 1 issues tcgen05.mma (M = 128 experts, N = 64 tokens) into
//    fp32 TMEM accumulators; warps 2..15 add up, from the same shared-memory
//    stages, each expert's and each token's sum of squares over the slice
//    (a row's sum does not depend on the swizzle's order of its chunks).
//  * Once every CTA of the cluster has finished its slice, warps 2..5 drain
//    the accumulators (tcgen05.ld) and push each token's partial row, and
//    every CTA its sums of squares, into the shared memory of the CTA that
//    owns the token (CK owners per tile, 64 / CK tokens each; stores over
//    distributed shared memory, no remote loads).  The owner adds the CK
//    partials in ascending slice order and forms the error bounds.
//  * The owner then picks as router_tiled_kernel does (router_pick_owned):
//    every expert that could reach the k-th largest under the bounds is
//    recomputed by Dot2 and the pick and the weights are made on those
//    values, so the result is that of the other routers.
//
// Error bound of a tensor-core logit.  The products x_h w_h of bf16 values
// are exact in fp32; only the accumulation rounds.  The tensor core's fp32
// accumulation order and rounding are not specified, so the bound assumes
// little: each MMA instruction (16 products added to the accumulator) may
// err by up to 2^-19 of the magnitudes it adds (|acc| + sum |p|), which
// covers aligning 17 operands to the largest and truncating each to 25 bits,
// and a final rounding.  Over n instructions along one accumulator that is at
// most 2 n 2^-19 S, S = sum_h |x_h w_h| <= ||x|| ||w||; the CK partials are
// then added in fp32 ((CK + 2) u S more, u = 2^-24) and the bias (u |l|).
// A test checks the tensor core's actual error against this bound.
#pragma once

#include "common.cuh"
#include "grouped.cuh"
#include "router.cuh"

namespace epk {

constexpr int kRcNT = 64;         // tokens per tile: the MMA's N
constexpr int kRcThreads = 512;
constexpr int kRcMaxE = 256;      // two 128-expert M tiles at most
constexpr int kRcMaxCand = 32;    // refined candidates per token
constexpr int kRcMinCK = 2;
constexpr int kRcMaxCK = 8;
constexpr uint32_t kRcWBox = kGemmBM * kGemmBK * 2;  // 128 experts x 64 of H, 16 KB
constexpr uint32_t kRcXBox = kRcNT * kGemmBK * 2;    // 64 tokens x 64 of H, 8 KB
constexpr int kRcNormWarps = 14;                     // warps 2..15

struct RcMaps {
    CUtensorMap w;  // W_router [E, H]: box 64 x 128
    CUtensorMap x;  // x [T, H]: box 64 x 64
};

// Shared memory: the stage ring, later reused for the partials pushed to
// this CTA by the cluster (its owned tokens' rows from every slice, and every
// slice's sums of squares), then the owned tokens' logits and bounds (in place
// of slices 0 and 1) and candidates.  The row sums of squares of this CTA's
// own slice wait beyond the ring (nsq) until the ring may be written.
struct RcSmem {
    uint32_t stage_bytes, stages, ring;            // ring = stages * stage_bytes
    uint32_t recv, wsq, xsq;                       // written by the cluster's CTAs
    uint32_t xn, wn, ncand, cand, cval, cscore, end;  // this CTA's only
    uint32_t bars, nsq, pbase, total, alloc;
};

__host__ __device__ inline RcSmem rc_smem_layout(int MT, int E, int CK) {
    RcSmem s;
    s.stage_bytes = MT * kRcWBox + kRcXBox;
    s.stages = 200u * 1024u / s.stage_bytes;
    if (s.stages > 8)
        s.stages = 8;
    s.ring = s.stages * s.stage_bytes;
    const uint32_t own = (kRcNT + CK - 1) / CK;  // tokens a CTA owns at most
    uint32_t o = 0;
    s.recv = o;   o = align_up_u32(o + (uint32_t)CK * own * E * 4, 16);  // [CK][own][E]
    s.wsq = o;    o = align_up_u32(o + (uint32_t)CK * E * 4, 16);        // [CK][E]
    s.xsq = o;    o = align_up_u32(o + (uint32_t)CK * own * 4, 16);      // [CK][own]
    s.xn = o;     o = align_up_u32(o + own * 4, 16);
    s.wn = o;     o = align_up_u32(o + (uint32_t)E * 4, 16);
    s.ncand = o;  o = align_up_u32(o + own * 4, 16);
    s.cand = o;   o = align_up_u32(o + own * kRcMaxCand * 4, 16);
    s.cval = o;   o = align_up_u32(o + own * kRcMaxCand * 8, 16);
    s.cscore = o; o = align_up_u32(o + own * kRcMaxCand * 8, 16);
    s.end = o;
    s.bars = align_up_u32(s.ring > s.end ? s.ring : s.end, 1024);
    // full[S], empty[S], tdone; tmem holder, abort flag
    s.nsq = align_up_u32(s.bars + (2 * s.stages + 1) * 8 + 16, 16);
    s.pbase = s.nsq + (uint32_t)(MT * kGemmBM + kRcNT) * 4;  // nsq: [MT 128 + 64]
    s.total = s.pbase + kRcMaxCK * 4;
    s.alloc = s.total + 1024;
    return s;
}

template <bool SIG>
__global__ void __launch_bounds__(kRcThreads, 1)
router_tc_kernel(const __grid_constant__ RcMaps maps, const uint16_t *__restrict__ x,
                 int64_t T, int H, const uint16_t *__restrict__ w_router,
                 const float *__restrict__ bias, int E, int top_k, int32_t *__restrict__ ids,
                 float *__restrict__ weights, int CK, int normalize, float scale,
                 float *__restrict__ dump_logit, float *__restrict__ dump_bound) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int MT = (E + kGemmBM - 1) / kGemmBM;
    const RcSmem L = rc_smem_layout(MT, E, CK);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + L.stages;
    uint64_t *tdone = empty + L.stages;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tdone + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tdone + 1) + 2;
    float *recv = reinterpret_cast<float *>(smem + L.recv);    // [CK][own][E]
    float *wsq = reinterpret_cast<float *>(smem + L.wsq);      // [CK][E]
    float *xsq = reinterpret_cast<float *>(smem + L.xsq);      // [CK][own]
    float *nsq = reinterpret_cast<float *>(smem + L.nsq);      // [MT 128 + 64]
    uint32_t *pbase = reinterpret_cast<uint32_t *>(smem + L.pbase);  // [CK]
    float *xn = reinterpret_cast<float *>(smem + L.xn);        // [own] ||x_t||
    float *wn = reinterpret_cast<float *>(smem + L.wn);        // [E] ||w_e||
    int *ncand = reinterpret_cast<int *>(smem + L.ncand);
    int *cand = reinterpret_cast<int *>(smem + L.cand);
    double *cval = reinterpret_cast<double *>(smem + L.cval);
    double *cscore = reinterpret_cast<double *>(smem + L.cscore);

    const int warp = (int)(threadIdx.x >> 5), lane = (int)lane_id();
    const uint32_t rank = cluster_ctarank();
    const int64_t t0 = (int64_t)blockIdx.y * kRcNT;
    const int tb = (T - t0 < (int64_t)kRcNT) ? (int)(T - t0) : kRcNT;
    const int nkb = (H + kGemmBK - 1) / kGemmBK;
    const int kb_lo = nkb * (int)rank / CK, kb_hi = nkb * ((int)rank + 1) / CK;
    const uint32_t tcols = MT * kRcNT <= 64 ? 64u : 128u;
    const int own = (kRcNT + CK - 1) / CK;
    float *logit = recv;            // [own][E], in place of slice 0's rows
    float *bound = recv + own * E;  // [own][E], in place of slice 1's rows
    bool have = false;              // the partial tile is in TMEM (warps 2..15)

    if (warp == 0 && lane < CK) {
        // where this CTA's rows of owner `lane` begin there, less the owner's
        // first token's rows (so that token t of the tile adds t E floats)
        const int lo = kRcNT * lane / CK;
        pbase[lane] = remote_shared(smem_u32(recv) + (uint32_t)(rank * own * E) * 4, (uint32_t)lane) -
                      (uint32_t)(lo * E) * 4;
    }
    if (warp == 0 && lane == 0) {
        for (uint32_t s = 0; s < L.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kRcNormWarps);
        }
        mbar_init(tdone, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&maps.w);
        prefetch_tensormap(&maps.x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, tcols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    grid_dependents_launch();
    // x may come from the previous kernel, which may also still read the ids
    // and weights this call overwrites
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            const uint64_t pol = policy_evict_last();  // every tile rereads W
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag))
                    break;
                uint8_t *sa = smem + stage * L.stage_bytes;
                mbar_arrive_expect_tx(&full[stage], L.stage_bytes);
                const int k0 = kb * kGemmBK;
                for (int m = 0; m < MT; ++m)
                    tma_load_2d(sa + m * kRcWBox, &maps.w, k0, m * kGemmBM, &full[stage], pol);
                tma_load_2d(sa + MT * kRcWBox, &maps.x, k0, (int32_t)t0, &full[stage], pol);
                ++issued;
                if (++stage == L.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // no copy may still be landing in shared memory when the stages
            // are reused below
            for (int n = issued > (int)L.stages ? issued - (int)L.stages : 0; n < issued; ++n)
                mbar_wait(&full[n % L.stages], (uint32_t)(n / L.stages) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            const uint32_t idesc = idesc_bf16_f32(kGemmBM, kRcNT);
            for (int kb = kb_lo; kb < kb_hi; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t a0 = smem_u32(smem + stage * L.stage_bytes);
                const uint32_t b0 = a0 + MT * kRcWBox;
                for (int m = 0; m < MT; ++m)
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_bf16(tmem_base + m * kRcNT,
                                  smem_desc_sw128_kmajor(a0 + m * kRcWBox + kk * 32),
                                  smem_desc_sw128_kmajor(b0 + kk * 32), idesc,
                                  (kb > kb_lo || kk > 0) ? 1u : 0u);
                umma_commit(&empty[stage]);
                if (++stage == L.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            umma_commit(tdone);  // every MMA of the slice has completed
        }
    } else {
        // ---------------------------------- sums of squares from the stages
        // The stage's rows (the W tiles' rows, then the token rows) are 128
        // bytes each and contiguous (the swizzle only permutes the chunks of
        // a row), so a warp reads four rows at once, lane l taking chunk
        // l % 8 of row l / 8: 512 contiguous bytes, free of bank conflicts.
        // Row quad g (rows 4g .. 4g + 3) goes to norm warp g mod 14; a lane
        // keeps one partial sum per quad it reads, and the eight lanes of a
        // row add theirs at the end.
        constexpr int kMaxQuads = (2 * kGemmBM + kRcNT) / 4 / kRcNormWarps + 1;
        const int nw = warp - 2;  // 0 .. 13
        const int rows = MT * kGemmBM + kRcNT;
        const int quads = rows / 4;
        float2 sq[kMaxQuads];
#pragma unroll
        for (int i = 0; i < kMaxQuads; ++i)
            sq[i] = make_float2(0.f, 0.f);
        uint32_t stage = 0, phase = 0;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag))
                break;
            const uint4 *sa = reinterpret_cast<const uint4 *>(smem + stage * L.stage_bytes);
#pragma unroll
            for (int i = 0; i < kMaxQuads; ++i) {
                const int g = nw + kRcNormWarps * i;
                if (g < quads) {
                    const uint4 v = sa[g * 32 + lane];  // rows 4g.., 16-byte chunk lane
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float2 f = bf16x2_to_f2(w4[h]);
                        sq[i] = ffma2(f, f, sq[i]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[stage]);
            if (++stage == L.stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        have = __all_sync(0xffffffffu, mbar_wait(tdone, 0, abort_flag));
        // a row's eight chunks sit in lanes 8 (l / 8) .. 8 (l / 8) + 7
#pragma unroll
        for (int i = 0; i < kMaxQuads; ++i) {
            float v = sq[i].x + sq[i].y;
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            const int g = nw + kRcNormWarps * i;
            if (g < quads && (lane & 7) == 0)
                nsq[4 * g + (lane >> 3)] = v;
        }
    }
    // this CTA's stages are free (every copy landed, every MMA completed,
    // every norm read done); after the cluster barrier every CTA's are, and
    // the partials are pushed to the CTAs that own their tokens
    tc_fence_before_sync();
    __syncthreads();
    // an execution barrier only: what it orders (the copies into the stages
    // and the MMAs reading them) has completed, as the mbarriers showed
    cluster_arrive_relaxed();
    cluster_wait();
    tc_fence_after_sync();
    // the owner of token t of the tile and t's row there
    static_assert(kRcNT == 64, "owner_of divides by 64");
    auto owner_of = [&](int t) { return (t * CK + CK - 1) >> 6; };
    if (have && warp >= 2 && warp < 6) {
        // warps 2..5 hold TMEM lane quarters 2, 3, 0, 1: expert e's partials
        // of 32 tokens per load, each sent to row (rank, t - lo) of t's owner
        const int q = warp & 3;
        for (int m = 0; m < MT; ++m) {
            const int e = m * kGemmBM + 32 * q + lane;
            for (int c0 = 0; c0 < kRcNT; c0 += 32) {
                uint32_t v[32];
                tmem_load_32cols(tmem_base + ((uint32_t)(32 * q) << 16) + m * kRcNT + c0, v);
                tmem_load_wait();
                if (e < E) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = c0 + j;
                        st_cluster_f32(pbase[owner_of(t)] + (uint32_t)(t * E + e) * 4,
                                       __uint_as_float(v[j]));
                    }
                }
            }
        }
    }
    // this slice's sums of squares: every expert's to every CTA, every
    // token's to its owner
    for (int i = threadIdx.x; i < E + kRcNT; i += kRcThreads) {
        if (i < E) {
            const float v = nsq[i];
            const uint32_t addr = smem_u32(wsq + rank * E + i);
            for (int o = 0; o < CK; ++o)
                st_cluster_f32(remote_shared(addr, (uint32_t)o), v);
        } else {
            const int t = i - E, o = owner_of(t);
            const int tl = t - kRcNT * o / CK;
            st_cluster_f32(remote_shared(smem_u32(xsq + rank * own + tl), (uint32_t)o),
                           nsq[MT * kGemmBM + t]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, tcols);
    }
    cluster_sync();  // every push has landed; no CTA's shared memory is written by another after this

    // The owner of tokens [64 rank / CK, 64 (rank + 1) / CK) adds the CK
    // partials of each (token, expert) in ascending slice order, then its
    // bound: 1.5 (gam ||x|| ||w|| + u |l|) with gam for the longest slice.
    const int own_lo = kRcNT * (int)rank / CK, own_hi = kRcNT * ((int)rank + 1) / CK;
    const int n_local = max(0, min(own_hi, tb) - own_lo);
    for (int i = threadIdx.x; i < E + n_local; i += kRcThreads) {
        float s2 = 0.f;
        for (int r = 0; r < CK; ++r)
            s2 += i < E ? wsq[r * E + i] : xsq[r * own + (i - E)];
        if (i < E)
            wn[i] = sqrtf(s2);
        else
            xn[i - E] = sqrtf(s2);
    }
    __syncthreads();
    {
        const float u = 5.9604644775390625e-8f;  // 2^-24
        const float n_instr = (float)(4 * ((nkb + CK - 1) / CK));
        const float gam = 2.0f * n_instr * 1.9073486328125e-6f + (float)(CK + 2) * u;  // 2^-19
        // thread (j0, e) takes tokens j0, j0 + js, ... of expert e
        const int js = kRcThreads / E;  // >= 1: E <= 256
        const int e = (int)threadIdx.x % E, j0 = (int)threadIdx.x / E;
        const float b = (bias != nullptr && j0 < js) ? bias[e] : 0.f;
        for (int j = j0 < js ? j0 : n_local; j < n_local; j += js) {
            float sum = 0.f;
            for (int r = 0; r < CK; ++r)
                sum += recv[(r * own + j) * E + e];
            float l, d;
            if (SIG) {
                // key = sigmoid(l) + b; the sigmoid's slope is at most 1/4, and
                // 4e-7 (1 + |key|) covers its fp32 evaluation and the sum
                const float d_l = 1.5f * (gam * xn[j] * wn[e] + u * fabsf(sum)) + 1e-30f;
                l = 1.0f / (1.0f + expf(-sum)) + b;
                d = 0.25f * d_l + 4e-7f * (1.0f + fabsf(l));
            } else {
                l = sum + b;
                d = 1.5f * (gam * xn[j] * wn[e] + u * fabsf(l)) + 1e-30f;
            }
            logit[j * E + e] = l;  // the element just read of slice 0
            bound[j * E + e] = d;  // and of slice 1
        }
    }
    __syncthreads();
    if (dump_logit != nullptr) {
        // inspection (moe_route_logits): the fp32 logits and their bounds
        for (int idx = threadIdx.x; idx < n_local * E; idx += kRcThreads) {
            const int j = idx / E, e = idx - j * E;
            const int64_t t = t0 + own_lo + j;
            dump_logit[t * E + e] = logit[j * E + e];
            dump_bound[t * E + e] = bound[j * E + e];
        }
        return;
    }

    router_pick_owned<false, SIG, kRcThreads / 32>(
        n_local, own_lo, 1, t0, x, H, w_router, bias, E, top_k, ids, weights, normalize, scale,
        logit, ncand, cand, cval, cscore, kRcMaxCand,
        [&](int j, int e) { return bound[j * E + e]; });
}

}  // namespace epk
