// ep.cuh -- the expert-parallel form of the routed FFN across ranks.
//
// fak note "GLM-5.2 multi-GPU: expert-parallel sharding + the resident-fit
// benchmark", "What landed": the experts are split into contiguous bands
// (ExpertParallelPlan), every rank computes the partial FFN output of the
// picks that fall in its band, and the partials are summed in rank order.
// TensorFold #310's maintainer's reply: the sum is taken in one order that
// does not depend on which rank holds which slice.
//
//  * ep_band_ids_kernel: a rank's view of the picks.  Ids inside its band
//    [e_lo, e_hi) become band-local ids (e - e_lo, matching weights that hold
//    only the band's experts); every other pick becomes an empty slot.  Ids
//    outside [0, E) are reported (the sticky status word) and dropped.
//  * ep_combine_kernel: y[t] = the partials of the bands that hold at least
//    one of t's picks, left-folded in rank order (each partial is that band's
//    fold in ascending (expert id, slot), starting from its first term), then
//    + the shared expert's output.  A token without a valid pick gets the
//    shared expert's output (or 0).
#pragma once

#include "common.cuh"

namespace epk {

constexpr int kEpMaxBands = 64;

struct EpBands {
    int32_t start[kEpMaxBands + 1];
};

__global__ void __launch_bounds__(256)
ep_band_ids_kernel(const int32_t *__restrict__ ids, int64_t n, int32_t E, int32_t e_lo,
                   int32_t e_hi, int32_t *__restrict__ local) {
    grid_dependents_launch();
    grid_dependency_wait();  // the ids may come from the previous kernel (the router)
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t e = ids[i];
        if (e >= e_lo && e < e_hi) {
            local[i] = e - e_lo;
        } else {
            if ((e < 0 || e >= E) && e != kIdNone)
                flag_status(kStatusBadId);
            local[i] = kIdNone;
        }
    }
}

constexpr int kEpCombineThreads = 256;

// Grid (ceil(H / 256), T); partials [R][T][H].
__global__ void __launch_bounds__(kEpCombineThreads)
ep_combine_kernel(const float *__restrict__ partials, int64_t T, int H,
                  const int32_t *__restrict__ ids, int top_k, int E, const EpBands bands, int R,
                  const float *__restrict__ shared, float *__restrict__ y) {
    __shared__ unsigned long long mask;
    grid_dependents_launch();
    grid_dependency_wait();  // the partials come from earlier kernels
    const int64_t t = blockIdx.y;
    if (threadIdx.x < 32) {
        // lane j < top_k marks the band of pick j; the marks are OR-ed over the warp
        const int j = (int)threadIdx.x;
        unsigned long long m = 0ull;
        if (j < top_k) {
            const int32_t e = ids[t * top_k + j];
            if (e >= 0 && e < E) {
                int r = 0;
                while (r + 1 < R && bands.start[r + 1] <= e)
                    ++r;
                m = 1ull << r;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m |= __shfl_xor_sync(0xffffffffu, m, off);
        if (j == 0)
            mask = m;
    }
    __syncthreads();
    const int col = (int)blockIdx.x * kEpCombineThreads + (int)threadIdx.x;
    if (col >= H)
        return;
    // the partials are loaded eight bands at a time before they are added, so
    // that the loads' latencies overlap; the adds run in rank order
    float acc = 0.f;
    bool first = true;
    for (int r0 = 0; r0 < R; r0 += 8) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (r0 + i < R && ((mask >> (r0 + i)) & 1ull))
                v[i] = partials[((size_t)(r0 + i) * T + t) * H + col];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (r0 + i < R && ((mask >> (r0 + i)) & 1ull)) {
                acc = first ? v[i] : acc + v[i];
                first = false;
            }
    }
    y[t * H + col] = shared != nullptr ? acc + shared[t * H + col] : acc;
}

}  // namespace epk
