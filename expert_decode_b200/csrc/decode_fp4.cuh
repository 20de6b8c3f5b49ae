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
// dequantising stage between the copy and the MMA:
//
//   warp 0     TMA: per 64-wide k block the raw codes of the tile's 128 rows
//              (32 bytes each) and the 16-bit activation (or h) tile;
//   warps 6-9  dequantise: thread r takes row r's 64 codes (cvt of E2M1
//              pairs to fp16 pairs, exact), multiplies them by the row's four
//              block scales (E4M3 to fp16, exact: every product has at most 6
//              significant bits and lies in fp16's normal range) and writes
//              the row into the stage's fp16 A tile in the 128-byte swizzled
//              K-major layout the MMA reads;
//   warp 1     tcgen05.mma kind::f16 with fp16 A and B, fp32 accumulators in
//              TMEM;
//   warps 2-5  the epilogue of decode_tc.cuh, with the tensor scale applied
//              to the fp32 accumulator first (an exact power of two for the
//              usual per-tensor scales).
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

constexpr int kF4Stages = 8;
constexpr int kF4Threads = 320;                           // warps 0..9
constexpr uint32_t kF4ABytes = kGemmBM * kGemmBK * 2;    // dequantised fp16 A, 16 KB
constexpr uint32_t kF4CodeBytes = kGemmBM * kGemmBK / 2; // 128 rows x 32 code bytes, 4 KB
constexpr uint32_t kF4BBytes = kTcN * kGemmBK * 2;       // 16 fp16 rows, 2 KB
constexpr uint32_t kF4CodeOff = kF4ABytes;
constexpr uint32_t kF4BOff = kF4ABytes + kF4CodeBytes;   // 20 KB, 1024-aligned
constexpr uint32_t kF4StageBytes = kF4ABytes + kF4CodeBytes + kF4BBytes;  // 22 KB
constexpr int kF4DeqWarp0 = 6;

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

__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t d;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(d) : "r"(byte));
    return d;
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

// Row r of a stage: its 64 codes (32 bytes at codes + 32 r) times its four
// block scales (s4: the scale bytes of k block kb, scales 4 kb .. 4 kb + 3
// of the row) into row r of the fp16 A tile, 128-byte swizzled: 16-byte
// chunk j of the row at position j ^ (r mod 8).
__device__ __forceinline__ void dequant_row(const uint8_t *codes, uint32_t s4, uint8_t *a_tile,
                                            int r) {
    const uint4 c0 = reinterpret_cast<const uint4 *>(codes + 32 * r)[0];
    const uint4 c1 = reinterpret_cast<const uint4 *>(codes + 32 * r)[1];
    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const uint32_t s01 = e4m3x2_to_f16x2(s4 & 0xffffu), s23 = e4m3x2_to_f16x2(s4 >> 16);
    // each block scale broadcast to both halves of an fp16 pair
    const uint32_t sb[4] = {__byte_perm(s01, 0, 0x1010), __byte_perm(s01, 0, 0x3232),
                            __byte_perm(s23, 0, 0x1010), __byte_perm(s23, 0, 0x3232)};
    uint4 *row = reinterpret_cast<uint4 *>(a_tile + 128 * r);
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // chunk j: elements 8 j .. 8 j + 7, code word j
        const uint32_t w = cw[j];
        const uint32_t s = sb[j >> 1];  // 16 elements per block: two chunks
        uint4 out;
        out.x = hmul2_u32(e2m1x2_to_f16x2(w & 0xffu), s);
        out.y = hmul2_u32(e2m1x2_to_f16x2((w >> 8) & 0xffu), s);
        out.z = hmul2_u32(e2m1x2_to_f16x2((w >> 16) & 0xffu), s);
        out.w = hmul2_u32(e2m1x2_to_f16x2(w >> 24), s);
        row[j ^ (r & 7)] = out;
    }
}

// h as fp16 hi/lo: hi = fp16(h), lo = fp16(h - hi).
__device__ __forceinline__ void store_hi_lo_f16(uint16_t *hi_p, uint16_t *lo_p, float h) {
    const __half hi = __float2half_rn(h);
    *hi_p = __half_as_ushort(hi);
    *lo_p = __half_as_ushort(__float2half_rn(h - __half2float(hi)));
}

// ------------------------------------------------------------------ gate/up
struct F4GuMaps {
    CUtensorMap cg, cu;  // routed W_gate / W_up codes [E, I, H/2] u8: box 32 x 64 x 1
    CUtensorMap sg, su;  // shared codes [I_s, H/2] u8: box 32 x 64
    CUtensorMap x;       // x fp16 [T, H]: box 64 x 16
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
    static constexpr uint32_t bars = kF4Stages * kF4StageBytes;
    // full[S], deq[S], empty[S], tfull[2], tempty[2], drain, planbar; holder, abort
    static constexpr uint32_t misc = bars + (3 * kF4Stages + 6) * 8;
    static constexpr uint32_t tile_first = misc + 16;
    static constexpr uint32_t row_first = tile_first + (kTcMaxGroups + 1) * 4;
    static constexpr uint32_t xchg = (row_first + kTcMaxGroups * 4 + 15) / 16 * 16;
    static constexpr uint32_t plan = (xchg + 2 * 2 * kStreamMaxT * 32 * 4 + 127) / 128 * 128;
    static constexpr uint32_t total = plan + (uint32_t)sizeof(StreamPlan);
    static constexpr uint32_t alloc = total + 1024;
};

__global__ void __launch_bounds__(kF4Threads, 1)
stream_gate_up_fp4_kernel(const __grid_constant__ F4GuMaps maps, const F4GuArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + F4Smem::bars);
    uint64_t *deq = full + kF4Stages;
    uint64_t *empty = deq + kF4Stages;
    uint64_t *tfull = empty + kF4Stages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *planbar = drain + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + F4Smem::misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + F4Smem::misc + 8);
    int *tile_first = reinterpret_cast<int *>(smem + F4Smem::tile_first);
    int *row_first = reinterpret_cast<int *>(smem + F4Smem::row_first);
    float *xchg = reinterpret_cast<float *>(smem + F4Smem::xchg);
    StreamPlan &P = *reinterpret_cast<StreamPlan *>(smem + F4Smem::plan);

    const int warp = (int)(threadIdx.x >> 5);
    const int lane = (int)lane_id();
    const int has_shared = a.I_s > 0 ? 1 : 0;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kF4Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&deq[s], 4);
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
        prefetch_tensormap(&maps.cg);
        prefetch_tensormap(&maps.cu);
        prefetch_tensormap(&maps.x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;

    auto decode = [&](int u, int &gi, int &m0) {
        const int G = has_shared + P.n_groups;
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tile_first[mid] <= u)
                lo = mid;
            else
                hi = mid - 1;
        }
        gi = lo;
        m0 = (u - tile_first[gi]) * kGateUpRows;
    };
    const int kblocks = (a.H + kGemmBK - 1) / kGemmBK;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            grid_dependency_wait();  // x16 comes from the previous kernel
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : tile_first[has_shared + P.n_groups];
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
                    uint8_t *st = smem + stage * kF4StageBytes;
                    mbar_arrive_expect_tx(&full[stage], kF4CodeBytes + kF4BBytes);
                    const int kc = kb * (kGemmBK / 2);  // byte column of the codes
                    // rows 0..63: W_gate codes of the tile's units, 64..127: W_up
                    uint8_t *cg = st + kF4CodeOff, *cu = cg + kF4CodeBytes / 2;
                    if (shared) {
                        tma_load_2d(cg, &maps.sg, kc, m0, &full[stage], pol_w);
                        tma_load_2d(cu, &maps.su, kc, m0, &full[stage], pol_w);
                    } else {
                        tma_load_3d(cg, &maps.cg, kc, m0, e, &full[stage], pol_w);
                        tma_load_3d(cu, &maps.cu, kc, m0, e, &full[stage], pol_w);
                    }
                    tma_load_2d(st + kF4BOff, &maps.x, kb * kGemmBK, 0, &full[stage], pol_x);
                    ++issued;
                    if (++stage == kF4Stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int n = issued > kF4Stages ? issued - kF4Stages : 0; n < issued; ++n)
                mbar_wait(&full[n % kF4Stages], (uint32_t)(n / kF4Stages) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            uint32_t acc = 0, acc_phase = 0;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : tile_first[has_shared + P.n_groups];
            const uint32_t idesc = idesc_f16_f32(kGemmBM, kTcN);
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kTcN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&deq[stage], phase, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(smem + stage * kF4StageBytes);
                    const uint32_t b_addr = a_addr + kF4BOff;
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_bf16(d_tmem, smem_desc_sw128_kmajor(a_addr + kk * 32),
                                  smem_desc_sw128_kmajor(b_addr + kk * 32), idesc,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);
                    if (++stage == kF4Stages) {
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
            umma_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
    } else if (warp >= kF4DeqWarp0) {
        // ---------------------------------------------------- dequantisers
        const int r = (int)threadIdx.x - 32 * kF4DeqWarp0;  // 0..127: row of the A tile
        const bool planned = mbar_wait(planbar, 0, abort_flag);
        const int total = planned ? tile_first[has_shared + P.n_groups] : 0;
        uint32_t stage = 0, phase = 0;
        bool stop = false;
        for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
            int gi, m0;
            decode(u, gi, m0);
            const bool shared = gi < has_shared;
            const int e = shared ? 0 : (int)P.group_expert[gi - has_shared];
            // the row's unit and its scales row (zero past the matrix)
            const bool up = r >= kGateUpRows;
            const int unit = m0 + (r & (kGateUpRows - 1));
            const F4Mat &m = shared ? (up ? a.su : a.sg) : (up ? a.wu : a.wg);
            const bool in = unit < m.rows;
            const uint32_t *srow = reinterpret_cast<const uint32_t *>(
                m.scales + ((size_t)e * m.rows + (in ? unit : 0)) * (size_t)(m.cols / 16));
            for (int kb = 0; kb < kblocks; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort_flag)) {
                    stop = true;
                    break;
                }
                uint8_t *st = smem + stage * kF4StageBytes;
                const uint32_t s4 = in ? __ldg(srow + kb) : 0u;
                dequant_row(st + kF4CodeOff, s4, st, r);
                fence_proxy_async_smem();  // the MMA reads the tile through the async proxy
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&deq[stage]);
                if (++stage == kF4Stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------ plan, then epilogue
        const int ltid = (int)threadIdx.x - 64;
        grid_dependency_wait();  // ids and weights may come from the previous kernel
        grid_dependents_launch();
        build_stream_plan(P, a.ids, a.weights, a.T, a.top_k, a.E, ltid, 128, kTcBarPlan);
        if (ltid == 0) {
            const int G = has_shared + P.n_groups;
            int t = 0;
            for (int gi = 0; gi < G; ++gi) {
                tile_first[gi] = t;
                const int width = gi < has_shared ? a.I_s : a.I;
                t += (width + kGateUpRows - 1) / kGateUpRows;
            }
            tile_first[G] = t;
            for (int g = 0; g < P.n_groups; ++g)
                row_first[g] = 2 * P.group_first[g];
            mbar_arrive(planbar);
        }
        const bool planned =
            named_count(kTcBarPlan, 128, mbar_wait(planbar, 0, abort_flag)) == 128;
        if (planned) {
            const int q = warp & 3;
            const bool gate_warp = q < 2;
            const int pair = q & 1;
            const int total = tile_first[has_shared + P.n_groups];
            uint32_t acc = 0, acc_phase = 0;
            for (int u = blockIdx.x; u < total; u += gridDim.x) {
                int gi, m0;
                decode(u, gi, m0);
                const bool shared = gi < has_shared;
                const bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag);
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
                            const float h =
                                silu_f32(ts * __uint_as_float(v[t])) * xb[t * 32 + lane];
                            store_hi_lo_f16(a.hb_shared + (size_t)t * a.I_s + unit,
                                            a.hb_shared + (size_t)(a.T + t) * a.I_s + unit, h);
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
                            const float h = silu_f32(ts * mine) * xb[tok * 32 + lane];
                            const int j0 = j / kTcSlice * kTcSlice;
                            const int n = min(kTcSlice, cnt - j0);
                            const size_t b = (size_t)row_first[g] + 2 * j0;
                            uint16_t *hb = a.hb_routed + unit;
                            store_hi_lo_f16(hb + (b + (j - j0)) * a.I,
                                            hb + (b + n + (j - j0)) * a.I, h);
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

// --------------------------------------------------------------------- down
struct F4DnMaps {
    CUtensorMap cd;  // routed W_down codes [E, H, I/2] u8: box 32 x 128 x 1
    CUtensorMap sd;  // shared W_down codes [H, I_s/2] u8: box 32 x 128
    CUtensorMap hr;  // routed h fp16 hi/lo rows [2 pairs + 16, I]: box 64 x 16
    CUtensorMap hs;  // shared h fp16 [16, I_s]: box 64 x 16
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
    static constexpr uint32_t bars = kF4Stages * kF4StageBytes;
    static constexpr uint32_t misc = bars + (3 * kF4Stages + 6) * 8;
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
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + F4DnSmem::bars);
    uint64_t *deq = full + kF4Stages;
    uint64_t *empty = deq + kF4Stages;
    uint64_t *tfull = empty + kF4Stages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *planbar = drain + 1;
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

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kF4Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&deq[s], 4);
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
        prefetch_tensormap(&maps.cd);
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

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_h = policy_evict_last();
            grid_dependency_wait();  // h comes from the previous kernel
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : (has_shared + *n_slices) * n_mb;
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const int si = u / n_mb, mb = u - si * n_mb;
                const bool shared = si < has_shared;
                const int slice = si - has_shared;
                const int e = shared ? 0 : (int)P.group_expert[slice_group[slice]];
                const int row =
                    shared ? -1 : 2 * ((int)P.group_first[slice_group[slice]] + slice_j0[slice]);
                const int kblocks = ((shared ? a.I_s : a.I) + kGemmBK - 1) / kGemmBK;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *st = smem + stage * kF4StageBytes;
                    mbar_arrive_expect_tx(&full[stage], kF4CodeBytes + kF4BBytes);
                    const int kc = kb * (kGemmBK / 2);
                    if (shared) {
                        tma_load_2d(st + kF4CodeOff, &maps.sd, kc, mb * kGemmBM, &full[stage], pol_w);
                        tma_load_2d(st + kF4BOff, &maps.hs, kb * kGemmBK, 0, &full[stage], pol_h);
                    } else {
                        tma_load_3d(st + kF4CodeOff, &maps.cd, kc, mb * kGemmBM, e, &full[stage],
                                    pol_w);
                        tma_load_2d(st + kF4BOff, &maps.hr, kb * kGemmBK, row, &full[stage], pol_h);
                    }
                    ++issued;
                    if (++stage == kF4Stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int n = issued > kF4Stages ? issued - kF4Stages : 0; n < issued; ++n)
                mbar_wait(&full[n % kF4Stages], (uint32_t)(n / kF4Stages) & 1u, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            uint32_t acc = 0, acc_phase = 0;
            bool stop = !mbar_wait(planbar, 0, abort_flag);
            const int total = stop ? 0 : (has_shared + *n_slices) * n_mb;
            const uint32_t idesc = idesc_f16_f32(kGemmBM, kTcN);
            for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
                const bool shared = u / n_mb < has_shared;
                const int kblocks = ((shared ? a.I_s : a.I) + kGemmBK - 1) / kGemmBK;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag))
                    break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * kTcN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&deq[stage], phase, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(smem + stage * kF4StageBytes);
                    const uint32_t b_addr = a_addr + kF4BOff;
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_bf16(d_tmem, smem_desc_sw128_kmajor(a_addr + kk * 32),
                                  smem_desc_sw128_kmajor(b_addr + kk * 32), idesc,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);
                    if (++stage == kF4Stages) {
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
            umma_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
    } else if (warp >= kF4DeqWarp0) {
        // ---------------------------------------------------- dequantisers
        const int r = (int)threadIdx.x - 32 * kF4DeqWarp0;  // row of the 128-row tile
        const bool planned = mbar_wait(planbar, 0, abort_flag);
        const int total = planned ? (has_shared + *n_slices) * n_mb : 0;
        uint32_t stage = 0, phase = 0;
        bool stop = false;
        for (int u = blockIdx.x; u < total && !stop; u += gridDim.x) {
            const int si = u / n_mb, mb = u - si * n_mb;
            const bool shared = si < has_shared;
            const int e = shared ? 0 : (int)P.group_expert[slice_group[si - has_shared]];
            const F4Mat &m = shared ? a.sd : a.wd;
            const int hrow = mb * kGemmBM + r;
            const bool in = hrow < m.rows;
            const uint32_t *srow = reinterpret_cast<const uint32_t *>(
                m.scales + ((size_t)e * m.rows + (in ? hrow : 0)) * (size_t)(m.cols / 16));
            const int kblocks = ((int)m.cols + kGemmBK - 1) / kGemmBK;
            for (int kb = 0; kb < kblocks; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort_flag)) {
                    stop = true;
                    break;
                }
                uint8_t *st = smem + stage * kF4StageBytes;
                const uint32_t s4 = in ? __ldg(srow + kb) : 0u;
                dequant_row(st + kF4CodeOff, s4, st, r);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&deq[stage]);
                if (++stage == kF4Stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
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
            mbar_arrive(planbar);
        }
        grid_dependency_wait();  // before any output is written
        if (mbar_wait(planbar, 0, abort_flag)) {
            const int q = warp & 3;
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
                    const float ts = shared ? a.sd.ts : a.wd.ts;
                    const int slice = si - has_shared;
                    const int g = shared ? 0 : slice_group[slice];
                    const int p0 = shared ? 0 : P.group_first[g] + slice_j0[slice];
                    const int n = shared ? a.T : min(kTcSlice, (int)P.group_first[g + 1] - p0);
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
                        const float d = ts * (__uint_as_float(v[r]) + lo[r]);
                        if (r < n) {
                            if (shared) {
                                a.s[(size_t)r * a.H + row] = d;
                            } else {
                                const int pair = p0 + r;
                                a.c[(size_t)P.sorted_src[pair] * a.H + row] =
                                    P.pair_weight[pair] * d;
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

// Codes of `mats` matrices of [rows][cols] NVFP4 elements: 32-byte (64
// element) by box_rows boxes, no swizzle (the dequantisers read them).
inline bool map_codes(CUtensorMap *m, const void *codes, uint64_t cols, uint64_t rows,
                      uint64_t mats, uint32_t box_rows) {
    const uint64_t dims[3] = {cols / 2, rows, mats};
    const uint64_t strides[2] = {cols / 2, rows * cols / 2};
    return make_map_typed(m, codes, mats > 1 ? 3 : 2, dims, strides, kGemmBK / 2, box_rows,
                          CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_NONE);
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
