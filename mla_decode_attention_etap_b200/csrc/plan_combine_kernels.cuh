// Split-KV plan kernel and the log-sum-exp combine kernel.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "merge.cuh"
#include "plan_core.h"

namespace mla {

constexpr int kPlanThreads = 1024;

// Exclusive prefix sum of one int64 per thread over the block; *total gets the block sum.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t x, int64_t *smem32, int64_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int64_t incl = x;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) smem32[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int64_t w = lane < nwarps ? smem32[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, w, d);
            if (lane >= d) w += y;
        }
        smem32[lane] = w;  // inclusive prefix of the warp sums
    }
    __syncthreads();
    const int64_t base = warp > 0 ? smem32[warp - 1] : 0;
    *total = smem32[nwarps - 1];
    __syncthreads();  // smem32 is free for the next scan
    return base + incl - x;
}

// One CTA: tile prefix sums, per-CTA flattened ranges, per-sequence split info, and
// zeroed merge counters.  Writes the header (and clears the status word) so that the
// decode kernel can check that it runs on a plan for its own grid.  kPlanThreads
// threads; thread i owns the consecutive sequences [i*per, (i+1)*per).
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t *__restrict__ seqlens, int batch, int ctas,
                                                            int groups, int ncols, int32_t *__restrict__ ws,
                                                            WsLayout lay) {
    // Launched as a programmatic dependent: nothing is read (seqlens may come from the
    // preceding kernel) or written (that kernel may still read the workspace) before it
    // completes.  Then the decode kernel may start its prologue: it waits for this grid in
    // turn before reading the workspace.  Both are no-ops without programmatic launch.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int64_t scan_smem[32];
    int32_t *tile_off = ws + lay.tile_off / 4;
    int32_t *ranges = ws + lay.cta_ranges / 4;
    int32_t *seq_info = ws + lay.seq_info / 4;
    int32_t *counters = ws + lay.counters / 4;
    int32_t *cta_seq = ws + lay.cta_seq / 4;
    const int per = (batch + kPlanThreads - 1) / kPlanThreads;
    const int b0 = min(batch, (int)threadIdx.x * per), b1 = min(batch, b0 + per);
    // flattened tile offsets: exclusive prefix sum of tiles per sequence
    int64_t mine = 0;
    for (int b = b0; b < b1; ++b) mine += tiles_of(seqlens[b]);
    int64_t total;
    int64_t f = block_exclusive_scan(mine, scan_smem, &total);
    const int used = used_ctas(total, ctas);
    // splits per sequence (the consecutive CTAs its tiles fall on)
    int64_t split_slots = 0;
    for (int b = b0; b < b1; ++b) {
        const int64_t t0 = f, t1 = f + tiles_of(seqlens[b]);
        int first = -1, nsplit = 0;
        if (t1 > t0) {
            first = cta_of(total, used, t0);
            nsplit = cta_of(total, used, t1 - 1) - first + 1;
        }
        tile_off[b] = (int32_t)t0;
        // the units whose range starts inside this sequence start their walk here
        for (int c = first; c >= 0 && c < first + nsplit; ++c)
            if (cta_begin(total, used, c) >= t0) cta_seq[c] = b;
        seq_info[4 * b + 0] = (int32_t)(t1 - t0);
        seq_info[4 * b + 1] = first;
        seq_info[4 * b + 2] = nsplit;
        if (nsplit >= 2) split_slots += nsplit;
        f = t1;
    }
    // partial-output slots: exclusive prefix sum of the split counts of split sequences
    int64_t slots;
    int64_t sl = block_exclusive_scan(split_slots, scan_smem, &slots);
    for (int b = b0; b < b1; ++b) {
        seq_info[4 * b + 3] = (int32_t)sl;
        if (seq_info[4 * b + 2] >= 2) sl += seq_info[4 * b + 2];
    }
    for (int c = threadIdx.x; c < ctas; c += kPlanThreads) {
        ranges[2 * c] = (int32_t)cta_begin(total, used, c);
        ranges[2 * c + 1] = (int32_t)cta_begin(total, used, c + 1);
        if (c >= used) cta_seq[c] = batch;  // no tiles
    }
    for (int i = threadIdx.x; i < 2 * batch * groups; i += kPlanThreads) counters[i] = 0;
    if (threadIdx.x == 0) {
        tile_off[batch] = (int32_t)total;
        ws[kHdrStatus] = 0;
        ws[kHdrCtas] = ctas;
        ws[kHdrGroups] = groups;
        ws[kHdrBatch] = batch;
        ws[kHdrTotalTiles] = (int32_t)total;
        ws[kHdrCols] = ncols;
        ws[kHdrSlotsUsed] = (int32_t)slots;
        ws[kHdrSlotsMax] = lay.slots;
    }
}

// Stand-alone split merge: one CTA of 128 threads per (column, sequence), 4 latent rows
// per thread.  Also writes O = 0, LSE = -inf for sequences without rows.
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
