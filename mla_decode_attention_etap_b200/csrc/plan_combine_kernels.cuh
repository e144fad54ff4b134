// Split-KV plan kernel and the log-sum-exp combine kernel.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "merge.cuh"
#include "plan_core.h"

namespace mla {

// One CTA: tile prefix sums, per-CTA flattened ranges, per-sequence split info.
// Writes the header (and clears the status word) so that the decode kernel can
// check that it runs on a plan for its own grid.
__global__ void plan_kernel(const int32_t *__restrict__ seqlens, int batch, int ctas, int groups, int ncols,
                            int32_t *__restrict__ ws, WsLayout lay) {
    int32_t *tile_off = ws + lay.tile_off / 4;
    int32_t *ranges = ws + lay.cta_ranges / 4;
    int32_t *seq_info = ws + lay.seq_info / 4;
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int b = 0; b < batch; ++b) {
            tile_off[b] = (int32_t)acc;
            acc += tiles_of(seqlens[b]);
        }
        tile_off[batch] = (int32_t)acc;
    }
    __syncthreads();
    const int64_t total = tile_off[batch];
    const int used = used_ctas(total, ctas);
    for (int c = threadIdx.x; c < ctas; c += blockDim.x) {
        ranges[2 * c] = (int32_t)cta_begin(total, used, c);
        ranges[2 * c + 1] = (int32_t)cta_begin(total, used, c + 1);
    }
    int32_t *counters = ws + lay.counters / 4;
    for (int i = threadIdx.x; i < 2 * batch * groups; i += blockDim.x) counters[i] = 0;
    for (int b = threadIdx.x; b < batch; b += blockDim.x) {
        const int t0 = tile_off[b], t1 = tile_off[b + 1];
        int first = -1, nsplit = 0;
        if (t1 > t0) {
            first = cta_of(total, used, t0);
            nsplit = cta_of(total, used, t1 - 1) - first + 1;
        }
        seq_info[4 * b + 0] = t1 - t0;
        seq_info[4 * b + 1] = first;
        seq_info[4 * b + 2] = nsplit;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int slots = 0;
        for (int b = 0; b < batch; ++b) {
            seq_info[4 * b + 3] = slots;
            if (seq_info[4 * b + 2] >= 2) slots += seq_info[4 * b + 2];
        }
        ws[kHdrStatus] = 0;
        ws[kHdrCtas] = ctas;
        ws[kHdrGroups] = groups;
        ws[kHdrBatch] = batch;
        ws[kHdrTotalTiles] = (int32_t)total;
        ws[kHdrCols] = ncols;
        ws[kHdrSlotsUsed] = slots;
        ws[kHdrSlotsMax] = lay.slots;
    }
}

// grid (ncols, batch), 128 threads: each thread merges 4 of the 512 output columns.
__global__ void __launch_bounds__(128) combine_kernel(const int32_t *__restrict__ ws, const float *__restrict__ opart,
                                                      const float *__restrict__ lsepart, int ncols, WsLayout lay,
                                                      __nv_bfloat16 *__restrict__ o, float *__restrict__ lse) {
    const int n = blockIdx.x, b = blockIdx.y;
    const int32_t *seq_info = ws + lay.seq_info / 4;
    const int nsplit = seq_info[4 * b + 2];
    if (nsplit == 1) return;  // written by the decode kernel
    const int64_t orow = ((int64_t)b * ncols + n) * kDv + 4 * threadIdx.x;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float lse_tot = -INFINITY;
    if (nsplit >= 2) {
        const int s0 = seq_info[4 * b + 3];
        const float *l = lsepart + (int64_t)s0 * ncols + n;
        lse_tot = merged_lse([&](int s) { return __ldcg(l + (int64_t)s * ncols); }, nsplit);
        if (lse_tot != -INFINITY) {
            for (int s = 0; s < nsplit; ++s) {
                const float w = merge_weight(__ldcg(l + (int64_t)s * ncols), lse_tot);
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(opart + ((int64_t)(s0 + s) * ncols + n) * kDv +
                                                                          4 * threadIdx.x));
                acc[0] = fmaf(w, v.x, acc[0]);
                acc[1] = fmaf(w, v.y, acc[1]);
                acc[2] = fmaf(w, v.z, acc[2]);
                acc[3] = fmaf(w, v.w, acc[3]);
            }
        }
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t *>(&lo);
    packed.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(o + orow) = packed;
    if (threadIdx.x == 0) lse[(int64_t)b * ncols + n] = lse_tot;
}

}  // namespace mla
