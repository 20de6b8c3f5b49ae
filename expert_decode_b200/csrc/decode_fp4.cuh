// decode_fp4.cuh -- the decode (T <= 8) routed FFN with NVFP4 expert weights,
// 4-bit weights and 16-bit activations, on the tensor cores.
//
// TensorFold #593, "Checkpoint formats on that family": NVIDIA's NVFP4
// checkpoint used as stored, 4-bit weights against 16-bit activations.  The
// format (NVIDIA's public definition; the page names it only): FP4 E2M1
// elements, two per byte (element 2i in the low nibble), one FP8 E4M3 scale
// per 16 consecutive elements of a row along the reduction dimension, one
// fp32 scale per tensor; a weight is tensor scale x block scale x element.
//
// Streaming the weights as stored cuts the bytes a decode call reads to
// 4.5 bits per weight.  The two kernels are those of decode_tc.cuh with a
// dequantising step between the copy and the MMA:
//
//   warp 0      TMA: per 256-wide k stage the raw codes of the tile's 128
//               rows (128 bytes each, 128-byte swizzled) and the stage's four
//               16-bit activation (or h) boxes, into an 8-stage ring;
//   warps 6-13  dequantise, 64-wide k block by k block, into a ring of fp16
//               A tiles held in tensor memory: thread (row, half) takes 32
//               codes of its row (cvt of E2M1 pairs to fp16 pairs, exact),
//               multiplies them by their two block scales (E4M3 to fp16,
//               exact: every product has at most 6 significant bits and lies
//               in fp16's range) and stores the 16 fp16 pairs to its row's
//               TMEM lane with tcgen05.st;
//   warp 1      tcgen05.mma kind::f16 with A from tensor memory and B (fp16)
//               from shared memory, fp32 accumulators in TMEM;
//   warps 2-5   the epilogue of decode_tc.cuh, with the tensor scale applied
//               to the fp32 accumulator first.
//
// The A tiles live in tensor memory rather than shared memory for two
// reasons.  A tile is released only when the MMAs reading it complete, and
// that latency must be covered by tiles already dequantised: tensor memory
// holds fifteen 64-wide A tiles (480 of its 512 columns) where shared memory
// could spare four.  And shared memory then carries only the codes and the
// activations, whose 24 KB stages keep 192 KB of codes in flight per SM.
//
// The activations enter as fp16: x is converted once per call (exact for
// bf16 values of magnitude 2^-14 .. 65504, which covers activations in
// practice), and h goes from the gate/up kernel to the down kernel as fp16
// hi/lo pairs (hi = fp16(h), lo = fp16(h - hi): about 22 significant bits).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "grouped.cuh"
#include "streaming.cuh"
#include "decode_tc.cuh"

namespace epk {

constexpr int kF4KS = 256;                               // k extent of one stage
constexpr int kF4Sub = kF4KS / kGemmBK;                  // 64-wide k blocks per stage
constexpr int kF4Stages = 8;
constexpr int kF4ASlots = 15;                            // A tiles in TMEM
constexpr int kF4Threads = 448;                          // warps 0..13
constexpr uint32_t kF4CodeBytes = kGemmBM * kF4KS / 2;   // 128 rows x 128 code bytes, 16 KB
constexpr uint32_t kF4BBox = kTcN * kGemmBK * 2;         // 16 fp16 rows x 64, 2 KB
constexpr uint32_t kF4BOff = kF4CodeBytes;               // four B boxes after the codes
constexpr uint32_t kF4StageBytes = kF4CodeBytes + kF4Sub * kF4BBox;   // 24 KB
constexpr uint32_t kF4Bars = kF4Stages * kF4StageBytes;
// tensor memory: two accumulators of kTcN columns, then the A ring, 32
// columns (64 fp16 of k, two per 32-bit column) per tile
constexpr uint32_t kF4TmemCols = 512;
constexpr uint32_t kF4ACol0 = 2 * kTcN;
constexpr uint32_t kF4ACols = kGemmBK / 2;
// full[S], empty[S], afull[A], aempty[A], tfull[2], tempty[2], drain, planbar
constexpr uint32_t kF4Misc = kF4Bars + (2 * kF4Stages + 2 * kF4ASlots + 6) * 8;
constexpr int kF4DeqWarp0 = 6;                           // warps 6..13 dequantise
constexpr int kF4DeqWarps = 8;

// Instruction descriptor: fp16 A and B, fp32 D, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t M, uint32_t N) {
    return (1u << 4)                 // D format: f32
           | ((N >> 3) << 17)        // N / 8 (A and B format 0: f16)
           | ((M >> 4) << 24);       // M / 16
}

// One NVFP4 matrix set as the kernels take it: codes [mats][rows][cols / 2],
// scales [mats][rows][cols / 16], one tensor scale.
struct F4Mat {
    const uint8_t *scales;
    float ts;
    int64_t rows, cols;  // per matrix
};

// The eight E2M1 codes of a 32-bit word as four fp16 pairs: byte k (elements
// 2k, 2k + 1) into d[k].  The word is split into its four bytes by one
// vector move, which the conversions take directly (measured 1.7x the
// conversion rate of a shift and mask per byte).
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&d)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(w));
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t d;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(d) : "r"(two));
    return d;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_store_16cols(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_store_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One MMA with A (M x 16 of k) from tensor memory and B from shared memory.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// k block `sub` of a stage, half h of row r: 32 codes (chunk 2 sub + h of the
// row's 128 code bytes, which the copy stored 128-byte swizzled at position
// (2 sub + h) ^ (r mod 8)) times their two block scales (bytes 2h, 2h + 1 of
// s4, the row's four scale bytes of this k block), as 16 fp16 pairs in the
// order of k (element 2i in the low half of pair i).  A warp takes 32
// consecutive rows: each eight lanes read eight distinct bank groups.
__device__ __forceinline__ void dequant_half(const uint8_t *codes, int sub, uint32_t s4, int r,
                                             int h, uint32_t (&out)[16]) {
    const uint4 c =
        reinterpret_cast<const uint4 *>(codes + 128 * r)[(2 * sub + h) ^ (r & 7)];
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    const uint32_t s2 = e4m3x2_to_f16x2(h ? (s4 >> 16) : (s4 & 0xffffu));
    // each block scale broadcast to both halves of an fp16 pair
    const uint32_t sb[2] = {__byte_perm(s2, 0, 0x1010), __byte_perm(s2, 0, 0x3232)};
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {  // code word jj: elements 8 jj .. 8 jj + 7, block jj / 2
        uint32_t d[4];
        e2m1x8_to_f16x2x4(cw[jj], d);
        const uint32_t sc = sb[jj >> 1];
#pragma unroll
        for (int m = 0; m < 4; ++m)
            out[4 * jj + m] = hmul2_u32(d[m], sc);
    }
}

// The row and half a dequantiser warp takes: warps 6..13; a warp may store
// only to its lane quarter of tensor memory (warp mod 4), so warp w takes
// rows 32 (w mod 4) + lane, half (w - 6) / 4 of each k block.
__device__ __forceinline__ void dequant_row_of(int warp, int lane, int &r, int &h) {
    r = 32 * (warp & 3) + lane;
    h = (warp - kF4DeqWarp0) >> 2;
}

// Scale rows past a matrix read this zero row instead.
constexpr int kF4MaxKBlocks = 16384 / kGemmBK;  // reduction dims up to 16384
__device__ const uint32_t kZeroScales[kF4MaxKBlocks] = {};

// One stage as a dequantiser sees it: its k blocks' scale words (this
// thread's row) and how many of its four k blocks exist.
struct F4StageScales {
    uint32_t s[kF4Sub];
    int n_sub;
};

// The stages one dequantiser thread consumes, in order of (tile, stage).
// row_of(u, p, kbn) gives tile u's scale row (left at the zero row past the
// matrix) and its count of 64-wide k blocks; fetch() loads the next stage's
// scale words (each index clamped into the row: no branch around a load).
template <class RowOf>
struct ScaleCursor {
    int u, ks, kbn, total, step;
    const uint32_t *p;
    RowOf row_of;

    __device__ __forceinline__ ScaleCursor(int u0, int total_, int step_, RowOf f)
        : u(u0), ks(0), kbn(1), total(total_), step(step_), p(kZeroScales), row_of(f) {
        if (u < total)
            row_of(u, p, kbn);
    }
    __device__ __forceinline__ F4StageScales fetch() {
        F4StageScales o;
        const int kb0 = ks * kF4Sub;
#pragma unroll
        for (int i = 0; i < kF4Sub; ++i)
            o.s[i] = __ldg(p + min(kb0 + i, kbn - 1));
        o.n_sub = min(kF4Sub, kbn - kb0);
        if (kb0 + kF4Sub >= kbn) {
            ks = 0;
            u += step;
            p = kZeroScales;
            kbn = 1;
            if (u < total)
                row_of(u, p, kbn);
        } else {
            ++ks;
        }
        return o;
    }
};

// Stages of a tile whose reduction spans kbn 64-wide k blocks.
__device__ __forceinline__ int f4_stages_of(int kbn) { return (kbn + kF4Sub - 1) / kF4Sub; }

// The dequantisers' loop over the n_stages stages this CTA consumes: wait for
// a stage's codes, then per k block wait for a free A tile, write this
// thread's half-row and release the tile to the MMA.  Each stage's scales are
// loaded kScaleAhead stages before their use; the loop is unrolled by that
// distance so each stays in its registers from load to use.
constexpr int kScaleAhead = 2;

template <class RowOf>
__device__ __forceinline__ void dequant_stages(uint8_t *smem, uint64_t *full, uint64_t *afull,
                                               uint64_t *aempty, volatile int *abort_flag,
                                               int n_stages, ScaleCursor<RowOf> &cur, int r,
                                               int h, int lane, uint32_t tmem_base) {
    F4StageScales q[kScaleAhead];
#pragma unroll
    for (int j = 0; j < kScaleAhead; ++j)
        q[j] = cur.fetch();
    // this warp's lane quarter and k half of every A tile
    const uint32_t t_own = tmem_base + ((uint32_t)(r & ~31) << 16) + kF4ACol0 + 16u * (uint32_t)h;
    uint32_t stage = 0, phase = 0, slot = 0, aphase = 0;
    for (int n0 = 0; n0 < n_stages; n0 += kScaleAhead) {
#pragma unroll
        for (int j = 0; j < kScaleAhead; ++j) {
            if (n0 + j < n_stages) {
                if (!mbar_wait(&full[stage], phase, abort_flag))
                    return;
                const uint8_t *codes = smem + stage * kF4StageBytes;
#pragma unroll
                for (int sub = 0; sub < kF4Sub; ++sub) {
                    if (sub < q[j].n_sub) {
                        uint32_t v[16];
                        dequant_half(codes, sub, q[j].s[sub], r, h, v);
                        if (!mbar_wait(&aempty[slot], aphase ^ 1u, abort_flag))
                            return;
                        tc_fence_after_sync();
                        tmem_store_16cols(t_own + slot * kF4ACols, v);
                        tmem_store_wait();
                        tc_fence_before_sync();  // the MMA reads the tile after the arrive
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(&afull[slot]);
                        if (++slot == kF4ASlots) {
                            slot = 0;
                            aphase ^= 1u;
                        }
                    }
                }
                q[j] = cur.fetch();
                if (++stage == kF4Stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }
}

// The MMA issuer's loop, common to both kernels: per tile one accumulator
// (of two in TMEM), per stage its k blocks, each from the next A tile of the
// ring and the stage's B box of that k block.
template <class KbnOf>
__device__ __forceinline__ void f4_mma_loop(uint8_t *smem, uint64_t *full, uint64_t *empty,
                                            uint64_t *afull, uint64_t *aempty, uint64_t *tfull,
                                            uint64_t *tempty, volatile int *abort_flag,
                                            uint32_t tmem_base, int total, KbnOf kbn_of) {
    uint32_t stage = 0, phase = 0, slot = 0, aphase = 0;
    uint32_t acc = 0, acc_phase = 0;
    const uint32_t idesc = idesc_f16_f32(kGemmBM, kTcN);
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag))
            return;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + acc * kTcN;
        const int kbn = kbn_of(u);
        const int n_st = f4_stages_of(kbn);
        for (int ks = 0; ks < n_st; ++ks) {
            if (!mbar_wait(&full[stage], phase, abort_flag))
                return;
            const uint32_t b_base = smem_u32(smem + stage * kF4StageBytes + kF4BOff);
            const int n_sub = min(kF4Sub, kbn - ks * kF4Sub);
            for (int sub = 0; sub < n_sub; ++sub) {
                if (!mbar_wait(&afull[slot], aphase, abort_flag))
                    return;
                tc_fence_after_sync();
                const uint32_t a_tmem = tmem_base + kF4ACol0 + slot * kF4ACols;
                const uint32_t b_addr = b_base + sub * kF4BBox;
#pragma unroll
                for (int kk = 0; kk < kGemmBK / 16; ++kk)  // 16 of k: 8 columns of A
                    umma_f16_tmem_a(d_tmem, a_tmem + 8 * kk,
                                    smem_desc_sw128_kmajor(b_addr + kk * 32), idesc,
                                    (ks > 0 || sub > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&aempty[slot]);
                if (++slot == kF4ASlots) {
                    slot = 0;
                    aphase ^= 1u;
                }
            }
            umma_commit(&empty[stage]);
            if (++stage == kF4Stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
        }
    }
}

// Barrier set of both kernels, at kF4Bars.
struct F4Bars {
    uint64_t *full, *empty, *afull, *aempty, *tfull, *tempty, *drain, *planbar;
    __device__ __forceinline__ explicit F4Bars(uint8_t *smem) {
        full = reinterpret_cast<uint64_t *>(smem + kF4Bars);
        empty = full + kF4Stages;
        afull = empty + kF4Stages;
        aempty = afull + kF4ASlots;
        tfull = aempty + kF4ASlots;
        tempty = tfull + 2;
        drain = tempty + 2;
        planbar = drain + 1;
    }
    __device__ __forceinline__ void init() const {
        for (int s = 0; s < kF4Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kF4ASlots; ++s) {
            mbar_init(&afull[s], kF4DeqWarps);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(drain, 1);
        mbar_init(planbar, 1);
    }
};

// h as fp16 hi/lo: hi = fp16(h), lo = fp16(h - hi).
__device__ __forceinline__ void store_hi_lo_f16(uint16_t *hi_p, uint16_t *lo_p, float h) {
    const __half hi = __float2half_rn(h);
    *hi_p = __half_as_ushort(hi);
    *lo_p = __half_as_ushort(__float2half_rn(h - __half2float(hi)));
}

// ------------------------------------------------------------------ gate/up
// Tiles as in decode_tc.cuh: 64 units of one expert's W_gate (A rows 0..63)
// and the same units of W_up (rows 64..127) against the 16 token rows of x.
struct F4GuMaps {
    CUtensorMap cg, cu;  // routed W_gate / W_up codes [E, I, H/2] u8: box 128 x 64 x 1, SW128
    CUtensorMap sg, su;  // shared codes [I_s, H/2] u8: box 128 x 64, SW128
    CUtensorMap x;       // x fp16 [T, H]: box 64 x 16, SW128
};

struct F4GuArgs {
    int T, H, E, I, I_s, top_k;
    const int32_t *ids;
    const float *weights;
    F4Mat wg, wu, sg, su;   // scales and tensor scales
    uint16_t *hb_routed;    // fp16 hi/lo rows, as TcArgs::hb_routed
    uint16_t *hb_shared;
};

struct F4Smem {
    static constexpr uint32_t misc = kF4Misc;  // tmem holder, abort flag
    static constexpr uint32_t xchg = (misc + 16 + 15) / 16 * 16;
    static constexpr uint32_t plan = (xchg + 2 * 2 * kStreamMaxT * 32 * 4 + 127) / 128 * 128;
    static constexpr uint32_t total = plan + (uint32_t)sizeof(StreamPlan);
    static constexpr uint32_t alloc = total + 1024;
};

__global__ void __launch_bounds__(kF4Threads, 1)
stream_gate_up_fp4_kernel(const __grid_constant__ F4GuMaps maps, const F4GuArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const F4Bars B(smem);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + F4Smem::misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + F4Smem::misc + 8);
    float *xchg = reinterpret_cast<float *>(smem + F4Smem::xchg);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + F4Smem::plan);

    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int has_shared = a.I_s > 0 ? 1 : 0;

    if (warp == 0 && lane == 0) {
        B.init();
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&maps.cg);
        prefetch_tensormap(&maps.cu);
        prefetch_tensormap(&maps.x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kF4TmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;

    // tiles of kGateUpRows units: the shared expert's first, then each routed
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
    const int kblocks = (a.H + kGemmBK - 1) / kGemmBK;
    const int n_st = f4_stages_of(kblocks);

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            grid_dependency_wait();  // x16 comes from the previous kernel
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool stop = !mbar_wait(B.planbar, 0, abort_flag);
            const int total = stop ? 0 : n_tiles();
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                int gi, m0;
                decode(u, gi, m0);
                const bool shared = gi < has_shared;
                const int e = shared ? 0 : (int)P.group_expert[gi - has_shared];
                for (int ks = 0; ks < n_st; ++ks) {
                    if (!mbar_wait(&B.empty[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *st = smem + stage * kF4StageBytes;
                    const int n_sub = min(kF4Sub, kblocks - ks * kF4Sub);
                    mbar_arrive_expect_tx(&B.full[stage], kF4CodeBytes + n_sub * kF4BBox);
                    const int kc = ks * (kF4KS / 2);  // byte column of the codes
                    // rows 0..63: W_gate codes of the tile's units, 64..127: W_up
                    uint8_t *cg = st, *cu = st + kF4CodeBytes / 2;
                    if (shared) {
                        tma_load_2d(cg, &maps.sg, kc, m0, &B.full[stage], pol_w);
                        tma_load_2d(cu, &maps.su, kc, m0, &B.full[stage], pol_w);
                    } else {
                        tma_load_3d(cg, &maps.cg, kc, m0, e, &B.full[stage], pol_w);
                        tma_load_3d(cu, &maps.cu, kc, m0, e, &B.full[stage], pol_w);
                    }
                    for (int sub = 0; sub < n_sub; ++sub)
                        tma_load_2d(st + kF4BOff + sub * kF4BBox, &maps.x,
                                    (ks * kF4Sub + sub) * kGemmBK, 0, &B.full[stage], pol_x);
                    ++issued;
                    if (++stage == kF4Stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int n = issued > kF4Stages ? issued - kF4Stages : 0; n < issued; ++n)
                mbar_wait(&B.full[n % kF4Stages], (uint32_t)(n / kF4Stages) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            const bool planned = mbar_wait(B.planbar, 0, abort_flag);
            const int total = planned ? n_tiles() : 0;
            f4_mma_loop(smem, B.full, B.empty, B.afull, B.aempty, B.tfull, B.tempty, abort_flag,
                        tmem_base, total, [&](int) { return kblocks; });
            umma_commit(B.drain);
            mbar_wait(B.drain, 0, nullptr);
        }
    } else if (warp >= kF4DeqWarp0) {
        // ---------------------------------------------------- dequantisers
        int r, h;  // row of the A tile, half of its k block
        dequant_row_of(warp, lane, r, h);
        const bool planned = mbar_wait(B.planbar, 0, abort_flag);
        const int total = planned ? n_tiles() : 0;
        // the row's unit and its scale row (zeros past the matrix)
        auto row_of = [&](int u, const uint32_t *&p, int &kbn) {
            int gi, m0;
            decode(u, gi, m0);
            const bool shared = gi < has_shared;
            const int e = shared ? 0 : (int)P.group_expert[gi - has_shared];
            const bool up = r >= kGateUpRows;
            const int unit = m0 + (r & (kGateUpRows - 1));
            const F4Mat &m = shared ? (up ? a.su : a.sg) : (up ? a.wu : a.wg);
            if (unit < m.rows)
                p = reinterpret_cast<const uint32_t *>(
                    m.scales + ((size_t)e * m.rows + unit) * (size_t)(m.cols / 16));
            kbn = kblocks;
        };
        const int mine = (int)blockIdx.x < total
                             ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                             : 0;
        ScaleCursor<decltype(row_of)> cur((int)blockIdx.x, total, (int)gridDim.x, row_of);
        dequant_stages(smem, B.full, B.afull, B.aempty, abort_flag, mine * n_st, cur, r, h,
                       lane, tmem_base);
    } else {
        // ------------------------------------------------ plan, then epilogue
        const int ltid = (int)threadIdx.x - 64;
        grid_dependency_wait();  // ids and weights may come from the previous kernel
        grid_dependents_launch();
        build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E, ltid, 128, kTcBarPlan);
        if (ltid == 0)
            mbar_arrive(B.planbar);  // release: the plan is written
        const bool planned =
            named_count(kTcBarPlan, 128, mbar_wait(B.planbar, 0, abort_flag)) == 128;
        if (planned) {
            const int q = warp & 3;
            const bool gate_warp = q < 2;
            const int pair = q & 1;
            const int total = n_tiles();
            uint32_t acc = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                int gi, m0;
                decode(u, gi, m0);
                const bool shared = gi < has_shared;
                const bool ok = mbar_wait(&B.tfull[acc], acc_phase, abort_flag);
                if (named_count(kTcBarPair + pair, 64, ok) != 64)
                    break;
                tc_fence_after_sync();
                uint32_t v[16];
                tmem_load_16cols(tmem_base + ((uint32_t)(32 * q) << 16) + acc * kTcN, v);
                tmem_load_wait();
                // the tensor scale of this warp's rows (gate or up, routed or shared)
                const float ts = shared ? (gate_warp ? a.sg.ts : a.su.ts)
                                        : (gate_warp ? a.wg.ts : a.wu.ts);
                float *xb = xchg + (pair * 2 + acc) * kStreamMaxT * 32;
                if (!gate_warp) {
#pragma unroll
                    for (int t = 0; t < kStreamMaxT; ++t)
                        xb[t * 32 + lane] = ts * __uint_as_float(v[t]);
                }
                named_sync(kTcBarPair + pair, 64);
                const int unit = m0 + 32 * pair + lane;
                if (gate_warp && shared) {
#pragma unroll
                    for (int t = 0; t < kStreamMaxT; ++t)
                        if (t < a.T && unit < a.I_s) {
                            const float hv =
                                silu_f32(ts * __uint_as_float(v[t])) * xb[t * 32 + lane];
                            store_hi_lo_f16(a.hb_shared + (size_t)t * a.I_s + unit,
                                            a.hb_shared + (size_t)(a.T + t) * a.I_s + unit, hv);
                        }
                } else if (gate_warp) {
                    const int g = gi - has_shared;
                    const int first = P.group_first[g];
                    const int cnt = P.group_first[g + 1] - first;
                    for (int j = 0; j < cnt; ++j) {
                        const int tok = P.pair_token[first + j];
                        float mv = 0.f;
#pragma unroll
                        for (int t = 0; t < kStreamMaxT; ++t)
                            mv = t == tok ? __uint_as_float(v[t]) : mv;
                        if (unit < a.I) {
                            const float hv = silu_f32(ts * mv) * xb[tok * 32 + lane];
                            const int j0 = j / kTcSlice * kTcSlice;
                            const int n = min(kTcSlice, cnt - j0);
                            const size_t b = 2 * (size_t)first + 2 * j0;  // 2 rows (hi, lo) per pick
                            uint16_t *hb = a.hb_routed + unit;
                            store_hi_lo_f16(hb + (b + (j - j0)) * a.I,
                                            hb + (b + n + (j - j0)) * a.I, hv);
                        }
                    }
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&B.tempty[acc]);
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
        tmem_dealloc(tmem_base, kF4TmemCols);
    }
}

// --------------------------------------------------------------------- down
// Tiles as in decode_tc.cuh: 128 rows of W_down against one slice of <= 8
// picks of one expert (h as fp16 hi/lo rows), or against the shared h.
struct F4DnMaps {
    CUtensorMap cd;  // routed W_down codes [E, H, I/2] u8: box 128 x 128 x 1, SW128
    CUtensorMap sd;  // shared W_down codes [H, I_s/2] u8: box 128 x 128, SW128
    CUtensorMap hr;  // routed h fp16 hi/lo rows [2 pairs + 16, I]: box 64 x 16, SW128
    CUtensorMap hs;  // shared h fp16 [16, I_s]: box 64 x 16, SW128
};

struct F4DnArgs {
    int T, H, E, I, I_s, top_k;
    const int32_t *ids;
    const float *weights;
    F4Mat wd, sd;
    float *c;  // [T * top_k, H]
    float *s;  // [T, H]
};

struct F4DnSmem {
    static constexpr uint32_t misc = kF4Misc;
    static constexpr uint32_t slice_group = misc + 16;
    static constexpr uint32_t slice_j0 = slice_group + kStreamMaxPairs * 4;
    static constexpr uint32_t n_slices = slice_j0 + kStreamMaxPairs * 4;
    static constexpr uint32_t plan = (n_slices + 4 + 127) / 128 * 128;
    static constexpr uint32_t total = plan + (uint32_t)sizeof(StreamPlan);
    static constexpr uint32_t alloc = total + 1024;
};

__global__ void __launch_bounds__(kF4Threads, 1)
stream_down_fp4_kernel(const __grid_constant__ F4DnMaps maps, const F4DnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const F4Bars B(smem);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + F4DnSmem::misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + F4DnSmem::misc + 8);
    int *slice_group = reinterpret_cast<int *>(smem + F4DnSmem::slice_group);
    int *slice_j0 = reinterpret_cast<int *>(smem + F4DnSmem::slice_j0);
    int *n_slices = reinterpret_cast<int *>(smem + F4DnSmem::n_slices);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + F4DnSmem::plan);

    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int has_shared = a.I_s > 0 ? 1 : 0;
    const int n_mb = (a.H + kGemmBM - 1) / kGemmBM;
    const int kb_routed = (a.I + kGemmBK - 1) / kGemmBK;
    const int kb_shared = (a.I_s + kGemmBK - 1) / kGemmBK;
    auto kbn_of = [&](int u) { return u / n_mb < has_shared ? kb_shared : kb_routed; };

    if (warp == 0 && lane == 0) {
        B.init();
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&maps.cd);
        prefetch_tensormap(&maps.hr);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kF4TmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    grid_dependents_launch();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_h = policy_evict_last();
            grid_dependency_wait();  // h comes from the previous kernel
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool stop = !mbar_wait(B.planbar, 0, abort_flag);
            const int total = stop ? 0 : (has_shared + *n_slices) * n_mb;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const int si = u / n_mb, mb = u - si * n_mb;
                const bool shared = si < has_shared;
                const int slice = si - has_shared;
                const int e = shared ? 0 : (int)P.group_expert[slice_group[slice]];
                const int row =
                    shared ? 0 : 2 * ((int)P.group_first[slice_group[slice]] + slice_j0[slice]);
                const int kbn = kbn_of(u);
                const int n_st = f4_stages_of(kbn);
                for (int ks = 0; ks < n_st; ++ks) {
                    if (!mbar_wait(&B.empty[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *st = smem + stage * kF4StageBytes;
                    const int n_sub = min(kF4Sub, kbn - ks * kF4Sub);
                    mbar_arrive_expect_tx(&B.full[stage], kF4CodeBytes + n_sub * kF4BBox);
                    const int kc = ks * (kF4KS / 2);
                    if (shared)
                        tma_load_2d(st, &maps.sd, kc, mb * kGemmBM, &B.full[stage], pol_w);
                    else
                        tma_load_3d(st, &maps.cd, kc, mb * kGemmBM, e, &B.full[stage], pol_w);
                    for (int sub = 0; sub < n_sub; ++sub)
                        tma_load_2d(st + kF4BOff + sub * kF4BBox, shared ? &maps.hs : &maps.hr,
                                    (ks * kF4Sub + sub) * kGemmBK, row, &B.full[stage], pol_h);
                    ++issued;
                    if (++stage == kF4Stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int n = issued > kF4Stages ? issued - kF4Stages : 0; n < issued; ++n)
                mbar_wait(&B.full[n % kF4Stages], (uint32_t)(n / kF4Stages) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            const bool planned = mbar_wait(B.planbar, 0, abort_flag);
            const int total = planned ? (has_shared + *n_slices) * n_mb : 0;
            f4_mma_loop(smem, B.full, B.empty, B.afull, B.aempty, B.tfull, B.tempty, abort_flag,
                        tmem_base, total, kbn_of);
            umma_commit(B.drain);
            mbar_wait(B.drain, 0, nullptr);
        }
    } else if (warp >= kF4DeqWarp0) {
        // ---------------------------------------------------- dequantisers
        int r, h;  // row of the 128-row tile, half of its k block
        dequant_row_of(warp, lane, r, h);
        const bool planned = mbar_wait(B.planbar, 0, abort_flag);
        const int total = planned ? (has_shared + *n_slices) * n_mb : 0;
        auto row_of = [&](int u, const uint32_t *&p, int &kbn) {
            const int si = u / n_mb, mb = u - si * n_mb;
            const bool shared = si < has_shared;
            const int e = shared ? 0 : (int)P.group_expert[slice_group[si - has_shared]];
            const F4Mat &m = shared ? a.sd : a.wd;
            const int hrow = mb * kGemmBM + r;
            if (hrow < m.rows)
                p = reinterpret_cast<const uint32_t *>(
                    m.scales + ((size_t)e * m.rows + hrow) * (size_t)(m.cols / 16));
            kbn = kbn_of(u);
        };
        int n_stages = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x)
            n_stages += f4_stages_of(kbn_of(u));
        ScaleCursor<decltype(row_of)> cur((int)blockIdx.x, total, (int)gridDim.x, row_of);
        dequant_stages(smem, B.full, B.afull, B.aempty, abort_flag, n_stages, cur, r, h, lane,
                       tmem_base);
    } else {
        // ------------------------------------------------ plan, then epilogue
        const int ltid = (int)threadIdx.x - 64;
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
            mbar_arrive(B.planbar);
        }
        grid_dependency_wait();  // before any output is written
        if (mbar_wait(B.planbar, 0, abort_flag)) {
            const int q = warp & 3;
            const int total = (has_shared + *n_slices) * n_mb;
            uint32_t acc = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                const int si = u / n_mb, mb = u - si * n_mb;
                const bool shared = si < has_shared;
                if (!mbar_wait(&B.tfull[acc], acc_phase, abort_flag))
                    break;
                tc_fence_after_sync();
                uint32_t v[16];
                tmem_load_16cols(tmem_base + ((uint32_t)(32 * q) << 16) + acc * kTcN, v);
                tmem_load_wait();
                const int row = mb * kGemmBM + 32 * q + lane;
                if (row < a.H) {
                    const float ts = shared ? a.sd.ts : a.wd.ts;
                    const int slice = si - has_shared;
                    const int g = shared ? 0 : slice_group[slice];
                    const int p0 = shared ? 0 : P.group_first[g] + slice_j0[slice];
                    const int n = shared ? a.T : min(kTcSlice, (int)P.group_first[g + 1] - p0);
                    float lo[kTcSlice];
#pragma unroll
                    for (int i = 0; i < kTcSlice; ++i)
                        lo[i] = 0.f;
#pragma unroll
                    for (int nn = 1; nn <= kTcSlice; ++nn)
                        if (n == nn) {
#pragma unroll
                            for (int i = 0; i < nn; ++i)
                                lo[i] = __uint_as_float(v[i + nn]);
                        }
#pragma unroll
                    for (int i = 0; i < kTcSlice; ++i) {
                        const float dv = ts * (__uint_as_float(v[i]) + lo[i]);
                        if (i < n) {
                            if (shared) {
                                a.s[(size_t)i * a.H + row] = dv;
                            } else {
                                const int pair = p0 + i;
                                a.c[(size_t)P.sorted_src[pair] * a.H + row] =
                                    P.pair_weight[pair] * dv;
                            }
                        }
                    }
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&B.tempty[acc]);
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
        tmem_dealloc(tmem_base, kF4TmemCols);
    }
}

// ---------------------------------------------------------------- host side
// A tiled tensor map of another element type than bf16: dims innermost
// first, box (box0 x box1 x 1).
inline bool make_map_typed(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
                           const uint64_t *strides_bytes, uint32_t box0, uint32_t box1,
                           CUtensorMapDataType dt, CUtensorMapSwizzle sw) {
    auto enc = tensor_map_encoder();
    if (enc == nullptr)
        return false;
    cuuint64_t gdim[3], gstride[2];
    cuuint32_t box[3] = {box0, box1, 1}, estride[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i)
        gdim[i] = dims[i];
    for (int i = 0; i < rank - 1; ++i)
        gstride[i] = strides_bytes[i];
    return enc(m, dt, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Codes of `mats` matrices of [rows][cols] NVFP4 elements: 128-byte (one
// stage's 256 elements) by box_rows boxes, 128-byte swizzled.
inline bool map_codes(CUtensorMap *m, const void *codes, uint64_t cols, uint64_t rows,
                      uint64_t mats, uint32_t box_rows) {
    const uint64_t dims[3] = {cols / 2, rows, mats};
    const uint64_t strides[2] = {cols / 2, rows * cols / 2};
    return make_map_typed(m, codes, mats > 1 ? 3 : 2, dims, strides, kF4KS / 2, box_rows,
                          CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_128B);
}

// fp16 [rows][cols]: 64 x box_rows boxes, 128-byte swizzle (an MMA operand).
inline bool map_f16(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                    uint32_t box_rows) {
    const uint64_t dims[2] = {cols, rows};
    const uint64_t strides[1] = {cols * 2};
    return make_map_typed(m, base, 2, dims, strides, kGemmBK, box_rows,
                          CU_TENSOR_MAP_DATA_TYPE_FLOAT16, CU_TENSOR_MAP_SWIZZLE_128B);
}

// x (bf16) -> fp16, round to nearest (T x H values; a few KB).
__global__ void __launch_bounds__(256) to_f16_kernel(const uint16_t *__restrict__ x, int64_t n,
                                                     uint16_t *__restrict__ out) {
    grid_dependents_launch();
    grid_dependency_wait();  // x may come from the previous kernel
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = __half_as_ushort(__float2half_rn(bf16_lo(x[i])));
}

}  // namespace epk
