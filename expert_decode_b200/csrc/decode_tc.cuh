// decode_tc.cuh -- gate/up and down projections of the weight-streaming
// (decode, T <= 8) path on the tensor cores.
//
// stream_gate_up_tc_kernel: the contraction of stream_gate_up_kernel
// (h = silu(W_gate x) * (W_up x) for every picked expert and the shared
// expert; fak note "GLM-5.2 multi-GPU", expertSwiGLU), laid out for tcgen05.
// A tile is 64 units of I: 128 weight rows on the MMA's M side, the 64 W_gate
// rows over the 64 W_up rows of the same units (TensorFold #593's packGateUp
// operand), and all T <= 8 tokens on its N side (N = 16; the tensor map
// zero-fills the rows after T).  Every tile therefore computes every token,
// and the epilogue keeps the tokens that picked the tile's expert, so no
// activation gather is needed.
//
// Persistent and warp specialised, one CTA per SM:
//   warp 0     TMA producer: per 64-wide k block the A tile (two boxes of 64
//              weight rows, 16 KB) and the x tile (16 rows, 2 KB) into a
//              ring of kTcStages stages, 128-byte swizzle, each CTA loading
//              its own copy: three copy instructions per stage, as few as the
//              operands allow;
//   warp 1     tcgen05.mma issuer (M = 128, N = 16, K = 16 per instruction),
//              fp32 accumulators in TMEM, two of them so that the epilogue
//              of one tile overlaps the MMAs of the next;
//   warps 2-5  build the expert grouping from ids (the streaming plan), then
//              drain each accumulator with tcgen05.ld: the warps of TMEM
//              quarters 2 and 3 (up rows) pass their values through shared
//              memory to those of quarters 0 and 1 (gate rows of the same
//              units), which write h = silu(g) * u: as bf16 hi/lo rows for
//              stream_down_tc_kernel, or in fp32 for stream_down_fold_kernel.
// Tiles go round-robin over the CTAs: the shared expert's first, then each
// routed group's in ascending expert id.  While it waits for the router,
// each CTA prefetches a share of the shared expert's three matrices into L2.
//
// stream_down_tc_kernel (below): the down projection with the same machinery.
#pragma once

#include "common.cuh"
#include "grouped.cuh"
#include "streaming.cuh"

namespace epk {

constexpr int kTcN = 16;                                   // MMA N: tokens, zero rows after T
constexpr int kTcStages = 10;
constexpr int kTcThreads = 224;  // warp 6: the gate/up kernel's group publisher
constexpr uint32_t kTcABytes = kGemmBM * kGemmBK * 2;      // 64 gate + 64 up rows, 16 KB
constexpr uint32_t kTcBBytes = kTcN * kGemmBK * 2;         // 16 token rows, 2 KB
constexpr uint32_t kTcStageBytes = kTcABytes + kTcBBytes;  // 18 KB, a multiple of 1024
constexpr int kTcTmemCols = 2 * kTcN;                      // two accumulators
constexpr uint32_t kTcBarPlan = 1;                         // named barrier of the epilogue warps
constexpr uint32_t kTcBarPair = 2;                         // + pair: the two warps of one pair
constexpr int kTcMaxGroups = kStreamMaxPairs + 1;          // routed groups + the shared expert

struct TcMaps {
    CUtensorMap wg, wu;  // W_gate, W_up [E, I, H]: box 64 x 64 x 1
    CUtensorMap sg, su;  // shared expert [I_s, H]: box 64 x 64
    CUtensorMap x;       // activations [T, H]: box 64 x 16
};

struct TcArgs {
    int T, H, E, I, I_s, top_k;
    const int32_t *ids;
    const float *weights;
    // the shared expert's weights (no routing decides them), prefetched into
    // L2 while the kernel waits for the router: Ws_gate, Ws_up, Ws_down
    const void *pf[3];
    size_t pf_bytes[3];
    float *h_routed;  // [pairs, I] in plan order
    float *h_shared;  // [T, I_s]
    // When set, h goes out instead as bf16 hi/lo pairs for the tensor-core
    // down projection, in hb_routed [2 * pairs + 16][I]: a group of cnt picks
    // takes 2 cnt rows, cut into slices of up to 8 picks; a slice of n picks
    // at row b holds hi(h) of its picks in rows b .. b+n-1 and lo(h) =
    // h - hi(h) in rows b+n .. b+2n-1.  The shared expert's T tokens likewise
    // in hb_shared [16][I_s] (hi in rows 0..T-1, lo in T..2T-1).
    uint16_t *hb_routed;
    uint16_t *hb_shared;
    // When set, one word per group (the shared expert first, then the routed
    // groups in plan order) counting the gate warps that have written their
    // tile's h, for stream_down_tc_kernel of the same call (group_done_add)
    unsigned long long *grp_done;
    unsigned long long epoch;  // this call's number, 1 .. 2^48 - 1
};

constexpr int kTcSlice = 8;  // picks per slice of the bf16 hi/lo activations

// Per-group completion words between the two decode kernels of a call.  The
// word holds the call's epoch in its high 48 bits and the number of the
// group's gate/up tiles done in its low 16, so a word left by an earlier call
// (or never written) counts as zero without any reset: the first add of a
// call replaces it.  The gate/up kernel adds one per tile once its h stores
// are fenced; the down kernel starts a group's slices when the word reads
// (epoch, the group's tile count).
// Called by one thread after a __threadfence that follows the tile's h
// stores (seen through a barrier): the fence is cumulative over them.
__device__ __forceinline__ void group_done_add(unsigned long long *w, unsigned long long epoch) {
    unsigned long long old = *reinterpret_cast<volatile unsigned long long *>(w);
    for (int tries = 0; tries < (1 << 20); ++tries) {
        const unsigned long long nw = (old >> 16) == epoch ? old + 1 : (epoch << 16) | 1ull;
        const unsigned long long got = atomicCAS(w, old, nw);
        if (got == old)
            return;
        old = got;
    }
    flag_status(kStatusTimeout);
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// The count a group reaches: its gate/up tiles (`width` units of I, 64 per tile).
__host__ __device__ inline int group_done_target(int width) {
    return (width + kGateUpRows - 1) / kGateUpRows;
}

// h as the two bf16 parts hi = bf16(h), lo = bf16(h - hi): together they
// carry h to about 16 significant bits, so that a bf16 x bf16 contraction of
// both parts loses next to nothing against fp32 h.
__device__ __forceinline__ void store_hi_lo(uint16_t *hi_p, uint16_t *lo_p, float h) {
    const uint16_t hi = f32_to_bf16_rne(h);
    *hi_p = hi;
    *lo_p = f32_to_bf16_rne(h - __uint_as_float((uint32_t)hi << 16));
}

struct TcSmem {
    static constexpr uint32_t stages = 0;
    static constexpr uint32_t bars = kTcStages * kTcStageBytes;
    // full[S], empty[S], tfull[2], tempty[2], drain, planbar, hdone[2],
    // hfree[2]; tmem holder, abort flag
    static constexpr uint32_t misc = bars + (2 * kTcStages + 10) * 8;
    // up values handed to the gate warps: [pair][accumulator][token][lane]
    static constexpr uint32_t xchg = (misc + 16 + 15) / 16 * 16;
    static constexpr uint32_t plan = (xchg + 2 * 2 * kStreamMaxT * 32 * 4 + 127) / 128 * 128;
    static constexpr uint32_t total = plan + (uint32_t)sizeof(StreamPlan);
    static constexpr uint32_t alloc = total + 1024;  // room to align the base to 1024
};

__device__ __forceinline__ void tmem_load_16cols(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__global__ void __launch_bounds__(kTcThreads, 1)
stream_gate_up_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + TcSmem::bars);
    uint64_t *empty = full + kTcStages;
    uint64_t *tfull = empty + kTcStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *planbar = drain + 1;
    uint64_t *hdone = planbar + 1;  // [2]: both gate warps have stored a tile's h
    uint64_t *hfree = hdone + 2;    // [2]: the publisher has taken hdone's phase
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + TcSmem::misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + TcSmem::misc + 8);
    float *xchg = reinterpret_cast<float *>(smem + TcSmem::xchg);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + TcSmem::plan);

    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int has_shared = a.I_s > 0 ? 1 : 0;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(drain, 1);
        mbar_init(planbar, 1);
        mbar_init(&hdone[0], 2);
        mbar_init(&hdone[1], 2);
        mbar_init(&hfree[0], 1);
        mbar_init(&hfree[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&maps.wg);
        prefetch_tensormap(&maps.wu);
        prefetch_tensormap(&maps.x);
        for (int i = 0; i < 3; ++i)
            prefetch_l2_share(a.pf[i], a.pf_bytes[i]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;

    // tile u -> (group index gi, first unit m0): tiles of kGateUpRows units,
    // the shared expert's first (gi = 0, when there is one), then each routed
    // group's, every routed group being I units wide
    const int tiles_s = has_shared ? (a.I_s + kGateUpRows - 1) / kGateUpRows : 0;
    const int tiles_r = (a.I + kGateUpRows - 1) / kGateUpRows;
    auto n_tiles = [&]() { return tiles_s + P.n_groups * tiles_r; };
    auto decode = [&](int u, int &gi, int &m0) {
        if (u < tiles_s) {
            gi = 0;
            m0 = u * kGateUpRows;
        } else {
            const int v = u - tiles_s, g = v / tiles_r;
            gi = has_shared + g;
            m0 = (v - g * tiles_r) * kGateUpRows;
        }
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            grid_dependency_wait();  // x may come from the previous kernel
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : n_tiles();
            const int kblocks = (a.H + kGemmBK - 1) / kGemmBK;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                int gi, m0;
                decode(u, gi, m0);
                const bool shared = gi < has_shared;
                const int e = shared ? 0 : (int)P.group_expert[gi - has_shared];
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sa = smem + stage * kTcStageBytes;
                    uint8_t *sb = sa + kTcABytes;
                    mbar_arrive_expect_tx(&full[stage], kTcStageBytes);
                    const int k0 = kb * kGemmBK;
                    // rows 0..63: W_gate of the tile's units, 64..127: W_up
                    uint8_t *sa_up = sa + kGateUpRows * kGemmBK * 2;
                    if (shared) {
                        tma_load_2d(sa, &maps.sg, k0, m0, &full[stage], pol_w);
                        tma_load_2d(sa_up, &maps.su, k0, m0, &full[stage], pol_w);
                    } else {
                        tma_load_3d(sa, &maps.wg, k0, m0, e, &full[stage], pol_w);
                        tma_load_3d(sa_up, &maps.wu, k0, m0, e, &full[stage], pol_w);
                    }
                    tma_load_2d(sb, &maps.x, k0, 0, &full[stage], pol_x);
                    ++issued;
                    if (++stage == kTcStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int n = issued > kTcStages ? issued - kTcStages : 0; n < issued; ++n)
                mbar_wait(&full[n % kTcStages], (uint32_t)(n / kTcStages) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            uint32_t acc = 0, acc_phase = 0;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : n_tiles();
            const int kblocks = (a.H + kGemmBK - 1) / kGemmBK;
            const uint32_t idesc = idesc_bf16_f32(kGemmBM, kTcN);
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kTcN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(smem + stage * kTcStageBytes);
                    const uint32_t b_addr = a_addr + kTcABytes;
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_bf16(d_tmem, smem_desc_sw128_kmajor(a_addr + kk * 32),
                                  smem_desc_sw128_kmajor(b_addr + kk * 32), idesc,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);  // frees the stage once these MMAs are done
                    if (++stage == kTcStages) {
                        stage = 0;
                        phase ^= 1u;
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
    } else if (warp == 6) {
        // ---------------------------------------------------- group publisher
        // After both gate warps have stored a tile's h (hdone), a gpu-scope
        // fence (cumulative over those stores, seen through the barrier) and
        // the group's count; kept off the epilogue, where the fence's wait
        // would hold both warps of a pair.
        if (a.grp_done != nullptr && elect_one()) {
            const bool planned = mbar_wait(planbar, 0, abort_flag);
            const int total = planned ? n_tiles() : 0;
            uint32_t acc = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                int gi, m0;
                decode(u, gi, m0);
                if (!mbar_wait(&hdone[acc], acc_phase, abort_flag))
                    break;
                mbar_arrive(&hfree[acc]);  // the gate warps may arrive on it again
                __threadfence();
                group_done_add(&a.grp_done[gi], a.epoch);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------ plan, then epilogue
        const int ltid = (int)threadIdx.x - 64;
        grid_dependency_wait();  // ids and weights may come from the previous kernel
        // the next kernel is let launch only once every CTA of this one has
        // passed its wait, so that it may read the ids (and x) before its own
        grid_dependents_launch();
        build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E, ltid, 128, kTcBarPlan);
        if (ltid == 0)
            mbar_arrive(planbar);  // release: the plan is written
        // the planning warps agree on the plan wait, so the pairs below either
        // all enter the tile loop or none does
        const bool planned =
            named_count(kTcBarPlan, 128, mbar_wait(planbar, 0, abort_flag)) == 128;
        if (planned) {
            const int q = warp & 3;  // TMEM lane quarter this warp may access
            // quarters 0, 1: gate rows of units 0..31, 32..63; 2, 3: their up rows
            const bool gate_warp = q < 2;
            const int pair = q & 1;
            const int total = n_tiles();
            uint32_t acc = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                int gi, m0;
                decode(u, gi, m0);
                const bool shared = gi < has_shared;
                // the two warps of a pair leave together or not at all
                const bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag);
                if (named_count(kTcBarPair + pair, 64, ok) != 64)
                    break;
                tc_fence_after_sync();
                uint32_t v[16];
                tmem_load_16cols(tmem_base + ((uint32_t)(32 * q) << 16) + acc * kTcN, v);
                tmem_load_wait();
                // [token][lane] of this pair and accumulator; a buffer is written
                // again two tiles later, after the pair's next barrier, which the
                // gate warp reaches only once it has read this one
                float *xb = xchg + (pair * 2 + acc) * kStreamMaxT * 32;
                if (!gate_warp) {
#pragma unroll
                    for (int t = 0; t < kStreamMaxT; ++t)
                        xb[t * 32 + lane] = __uint_as_float(v[t]);
                }
                named_sync(kTcBarPair + pair, 64);
                const int unit = m0 + 32 * pair + lane;
                if (gate_warp && shared) {
#pragma unroll
                    for (int t = 0; t < kStreamMaxT; ++t)
                        if (t < a.T && unit < a.I_s) {
                            const float h = silu_f32(__uint_as_float(v[t])) * xb[t * 32 + lane];
                            if (a.hb_shared != nullptr)
                                store_hi_lo(a.hb_shared + (size_t)t * a.I_s + unit,
                                            a.hb_shared + (size_t)(a.T + t) * a.I_s + unit, h);
                            else
                                a.h_shared[(size_t)t * a.I_s + unit] = h;
                        }
                } else if (gate_warp) {
                    const int g = gi - has_shared;
                    const int first = P.group_first[g];
                    const int cnt = P.group_first[g + 1] - first;
                    for (int j = 0; j < cnt; ++j) {
                        const int tok = P.pair_token[first + j];
                        float mine = 0.f;
#pragma unroll
                        for (int t = 0; t < kStreamMaxT; ++t)
                            mine = t == tok ? __uint_as_float(v[t]) : mine;
                        if (unit < a.I) {
                            const float h = silu_f32(mine) * xb[tok * 32 + lane];
                            if (a.hb_routed != nullptr) {
                                const int j0 = j / kTcSlice * kTcSlice;
                                const int n = min(kTcSlice, cnt - j0);
                                const size_t b = 2 * (size_t)first + 2 * j0;  // 2 rows (hi, lo) per pick
                                uint16_t *hb = a.hb_routed + unit;
                                store_hi_lo(hb + (b + (j - j0)) * a.I,
                                            hb + (b + n + (j - j0)) * a.I, h);
                            } else {
                                a.h_routed[(size_t)(first + j) * a.I + unit] = h;
                            }
                        }
                    }
                }
                tc_fence_before_sync();
                __syncwarp();  // the warp's h stores before lane 0's arrive
                if (lane == 0) {
                    mbar_arrive(&tempty[acc]);
                    // the publisher has taken this barrier's previous phase
                    // (it runs far ahead of the tiles: this wait normally
                    // returns at once)
                    if (gate_warp && a.grp_done != nullptr &&
                        mbar_wait(&hfree[acc], acc_phase ^ 1u, abort_flag))
                        mbar_arrive(&hdone[acc]);
                }
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTcTmemCols);
    }
}

// ---------------------------------------------------------------------------
// The down projection of the weight-streaming path on the tensor cores:
// c[pick] = w * (W_down[e] h) for every pick, s[t] = Ws_down h_s[t] for the
// shared expert.  A tile is 128 rows of W_down (the MMA's M side) against one
// slice of n <= 8 picks of one expert, whose h enters as the bf16 parts hi
// (B rows 0..n-1) and lo (rows n..2n-1) written by stream_gate_up_tc_kernel,
// so that D[:, r] + D[:, n + r] is W_down h for pick r (the box's other rows
// belong to the next slice and land in columns nobody reads).  Two copy instructions
// per 64-wide k block (one 128-row weight box, one 16-row activation box).
// The contributions are written per (token, slot) and folded afterwards by
// combine_kernel in ascending (expert id, slot), then + s: the same fold as
// the other paths.
struct DtMaps {
    CUtensorMap wd;  // W_down [E, H, I]: box 64 x 128 x 1
    CUtensorMap sd;  // shared W_down [H, I_s]: box 64 x 128
    CUtensorMap hr;  // routed h, bf16 hi/lo rows [2 * pairs + 16, I]: box 64 x 16
    CUtensorMap hs;  // shared h [16, I_s] bf16: box 64 x 16
};

struct DtArgs {
    int T, H, E, I, I_s, top_k;
    const int32_t *ids;
    const float *weights;
    float *c;  // [T * top_k, H]: weighted contribution of pick t * top_k + j
    float *s;  // [T, H]: the shared expert's output
    // the gate/up kernel's per-group completion words and the call's epoch;
    // without them the kernel waits for the whole gate/up kernel instead
    const unsigned long long *grp_done;
    unsigned long long epoch;
};

struct DtSmem {
    static constexpr uint32_t bars = kTcStages * kTcStageBytes;
    // full[S], empty[S], tfull[2], tempty[2], drain, planbar; tmem holder, abort flag
    static constexpr uint32_t misc = bars + (2 * kTcStages + 6) * 8;
    static constexpr uint32_t slice_group = misc + 16;                        // [kStreamMaxPairs]
    static constexpr uint32_t slice_j0 = slice_group + kStreamMaxPairs * 4;    // [kStreamMaxPairs]
    static constexpr uint32_t n_slices = slice_j0 + kStreamMaxPairs * 4;
    // a slice's first pair p0 = group_first[g] + j0 is also its first h row / 2
    static constexpr uint32_t plan = (n_slices + 4 + 127) / 128 * 128;
    static constexpr uint32_t total = plan + (uint32_t)sizeof(StreamPlan);
    static constexpr uint32_t alloc = total + 1024;  // room to align the base to 1024
};

__global__ void __launch_bounds__(kTcThreads, 1)
stream_down_tc_kernel(const __grid_constant__ DtMaps maps, const DtArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + DtSmem::bars);
    uint64_t *empty = full + kTcStages;
    uint64_t *tfull = empty + kTcStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *planbar = drain + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + DtSmem::misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + DtSmem::misc + 8);
    int *slice_group = reinterpret_cast<int *>(smem + DtSmem::slice_group);
    int *slice_j0 = reinterpret_cast<int *>(smem + DtSmem::slice_j0);
    int *n_slices = reinterpret_cast<int *>(smem + DtSmem::n_slices);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + DtSmem::plan);

    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int has_shared = a.I_s > 0 ? 1 : 0;
    const int n_mb = (a.H + kGemmBM - 1) / kGemmBM;  // 128-row blocks of H

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(drain, 1);
        mbar_init(planbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&maps.wd);
        prefetch_tensormap(&maps.hr);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    grid_dependents_launch();
    const uint32_t tmem_base = *tmem_holder;

    // tile u -> (slice si, 128-row block mb); si = 0 is the shared expert when
    // there is one, then the routed slices in plan order

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        // The plan comes from ids, which the kernel before the previous one
        // wrote (the previous kernel lets this one launch only after its own
        // wait), so the weights of the first kTcStages stages are requested
        // before griddepcontrol.wait; their h boxes, written by the previous
        // kernel, follow once it has completed.  A stage's full barrier takes
        // the weight bytes by expect_tx and the h bytes with its one arrive.
        if (a.grp_done != nullptr && elect_one()) {
            // Each slice starts once its group's gate/up tiles have published
            // their h (group_done_add): the slices of groups finished early
            // stream while the gate/up kernel's last tiles still run.
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_h = policy_evict_last();
            uint32_t stage = 0, phase = 0;
            int issued = 0, ready_group = -1;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : (has_shared + *n_slices) * n_mb;
            auto group_ready = [&](int gidx, int width) -> bool {
                const unsigned long long want =
                    (a.epoch << 16) | (unsigned long long)group_done_target(width);
                if (ld_acquire_u64(&a.grp_done[gidx]) == want)
                    return true;
                const uint64_t t0 = global_timer_ns();
                for (uint32_t spin = 1;; ++spin) {
                    if (ld_acquire_u64(&a.grp_done[gidx]) == want)
                        return true;
                    if (*abort_flag)
                        return false;
                    if ((spin & 255u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
                        *abort_flag = 1;
                        flag_status(kStatusTimeout);
                        return false;
                    }
                }
            };
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const int si = u / n_mb, mb = u - si * n_mb;
                const bool shared = si < has_shared;
                const int slice = si - has_shared;
                const int g = shared ? 0 : slice_group[slice];
                const int gidx = shared ? 0 : has_shared + g;
                const int e = shared ? 0 : (int)P.group_expert[g];
                const int row = shared ? -1 : 2 * ((int)P.group_first[g] + slice_j0[slice]);
                const int kblocks = ((shared ? a.I_s : a.I) + kGemmBK - 1) / kGemmBK;
                if (gidx != ready_group) {
                    if (!group_ready(gidx, shared ? a.I_s : a.I)) {
                        stop = true;
                        break;
                    }
                    // the h boxes are read by the copy engine (async proxy)
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    ready_group = gidx;
                }
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sa = smem + stage * kTcStageBytes;
                    uint8_t *sb = sa + kTcABytes;
                    const int k0 = kb * kGemmBK;
                    mbar_arrive_expect_tx(&full[stage], kTcStageBytes);
                    if (shared) {
                        tma_load_2d(sa, &maps.sd, k0, mb * kGemmBM, &full[stage], pol_w);
                        tma_load_2d(sb, &maps.hs, k0, 0, &full[stage], pol_h);
                    } else {
                        tma_load_3d(sa, &maps.wd, k0, mb * kGemmBM, e, &full[stage], pol_w);
                        tma_load_2d(sb, &maps.hr, k0, row, &full[stage], pol_h);
                    }
                    ++issued;
                    if (++stage == kTcStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int n = issued > kTcStages ? issued - kTcStages : 0; n < issued; ++n)
                mbar_wait(&full[n % kTcStages], (uint32_t)(n / kTcStages) & 1u, nullptr);
        } else if (a.grp_done == nullptr && elect_one()) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_h = policy_evict_last();
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool waited = false;
            int pend_row[kTcStages], pend_k0[kTcStages];  // h boxes not yet requested
            auto load_h = [&](int st, int k0, int row) {
                uint8_t *sb = smem + st * kTcStageBytes + kTcABytes;
                if (row < 0)
                    tma_load_2d(sb, &maps.hs, k0, 0, &full[st], pol_h);
                else
                    tma_load_2d(sb, &maps.hr, k0, row, &full[st], pol_h);
            };
            auto finish_wait = [&]() {
                grid_dependency_wait();  // h comes from the previous kernel
                waited = true;
                for (int n = 0; n < issued; ++n) {
                    mbar_arrive_expect_tx(&full[n], kTcBBytes);
                    load_h(n, pend_k0[n], pend_row[n]);
                }
            };
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : (has_shared + *n_slices) * n_mb;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const int si = u / n_mb, mb = u - si * n_mb;
                const bool shared = si < has_shared;
                const int slice = si - has_shared;
                const int e = shared ? 0 : (int)P.group_expert[slice_group[slice]];
                // h row of the slice's first pick (-1: the shared expert's rows)
                const int row =
                    shared ? -1 : 2 * ((int)P.group_first[slice_group[slice]] + slice_j0[slice]);
                const int kblocks = ((shared ? a.I_s : a.I) + kGemmBK - 1) / kGemmBK;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!waited && issued == kTcStages)
                        finish_wait();  // the ring is full: the stages need their h now
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *sa = smem + stage * kTcStageBytes;
                    const int k0 = kb * kGemmBK;
                    if (waited)
                        mbar_arrive_expect_tx(&full[stage], kTcStageBytes);
                    else
                        mbar_expect_tx(&full[stage], kTcABytes);
                    if (shared)
                        tma_load_2d(sa, &maps.sd, k0, mb * kGemmBM, &full[stage], pol_w);
                    else
                        tma_load_3d(sa, &maps.wd, k0, mb * kGemmBM, e, &full[stage], pol_w);
                    if (waited) {
                        load_h(stage, k0, row);
                    } else {
                        pend_k0[stage] = k0;
                        pend_row[stage] = row;
                    }
                    ++issued;
                    if (++stage == kTcStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!waited)
                finish_wait();  // fewer stages than the ring holds, or none, or a stop
            // no copy may still be landing in shared memory when the CTA exits
            for (int n = issued > kTcStages ? issued - kTcStages : 0; n < issued; ++n)
                mbar_wait(&full[n % kTcStages], (uint32_t)(n / kTcStages) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            uint32_t acc = 0, acc_phase = 0;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : (has_shared + *n_slices) * n_mb;
            const uint32_t idesc = idesc_bf16_f32(kGemmBM, kTcN);
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const bool shared = u / n_mb < has_shared;
                const int kblocks = ((shared ? a.I_s : a.I) + kGemmBK - 1) / kGemmBK;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kTcN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(smem + stage * kTcStageBytes);
                    const uint32_t b_addr = a_addr + kTcABytes;
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_bf16(d_tmem, smem_desc_sw128_kmajor(a_addr + kk * 32),
                                  smem_desc_sw128_kmajor(b_addr + kk * 32), idesc,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);  // frees the stage once these MMAs are done
                    if (++stage == kTcStages) {
                        stage = 0;
                        phase ^= 1u;
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
    } else if (warp < 6) {
        // ------------------------------------------------ plan, then epilogue
        const int ltid = (int)threadIdx.x - 64;
        // ids and weights come from the kernel before the previous one, which
        // has completed: the previous kernel let this one launch only after
        // passing its own griddepcontrol.wait
        build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E, ltid, 128, kTcBarPlan);
        if (ltid == 0) {
            int sl = 0;
            for (int g = 0; g < P.n_groups; ++g) {
                const int cnt = P.group_first[g + 1] - P.group_first[g];
                for (int j0 = 0; j0 < cnt; j0 += kTcSlice) {
                    slice_group[sl] = g;
                    slice_j0[sl] = j0;
                    ++sl;
                }
            }
            *n_slices = sl;
            mbar_arrive(planbar);  // release: the plan and the slice table are written
        }
        // Without the completion words, nothing is written before the gate/up
        // kernel has completed.  With them, the outputs c and s are read only
        // by the next kernel, and their earlier readers (the previous call's)
        // completed before this call's router did.
        if (a.grp_done == nullptr)
            grid_dependency_wait();
        if (mbar_wait(planbar, 0, abort_flag)) {
            const int q = warp & 3;  // TMEM lane quarter this warp may access
            const int total = (has_shared + *n_slices) * n_mb;
            uint32_t acc = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                const int si = u / n_mb, mb = u - si * n_mb;
                const bool shared = si < has_shared;
                if (!mbar_wait(&tfull[acc], acc_phase, abort_flag))
                    break;
                tc_fence_after_sync();
                uint32_t v[16];
                tmem_load_16cols(tmem_base + ((uint32_t)(32 * q) << 16) + acc * kTcN, v);
                tmem_load_wait();
                const int row = mb * kGemmBM + 32 * q + lane;
                if (row < a.H) {
                    // column r + n holds the lo part of column r (n picks)
                    const int slice = si - has_shared;
                    const int g = shared ? 0 : slice_group[slice];
                    const int p0 = shared ? 0 : P.group_first[g] + slice_j0[slice];
                    const int n = shared ? a.T : min(kTcSlice, (int)P.group_first[g + 1] - p0);
                    // lo[r] = column r + n, picked with constant register indices
                    float lo[kTcSlice];
#pragma unroll
                    for (int r = 0; r < kTcSlice; ++r)
                        lo[r] = 0.f;
#pragma unroll
                    for (int nn = 1; nn <= kTcSlice; ++nn)
                        if (n == nn) {
#pragma unroll
                            for (int r = 0; r < nn; ++r)
                                lo[r] = __uint_as_float(v[r + nn]);
                        }
#pragma unroll
                    for (int r = 0; r < kTcSlice; ++r) {
                        const float d = __uint_as_float(v[r]) + lo[r];
                        if (r < n) {
                            if (shared) {
                                a.s[(size_t)r * a.H + row] = d;
                            } else {
                                const int pair = p0 + r;
                                a.c[(size_t)P.sorted_src[pair] * a.H + row] = P.pair_weight[pair] * d;
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
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTcTmemCols);
    }
}

}  // namespace epk
