// Split-KV plan kernel and the log-sum-exp combine kernel.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "etap_common.cuh"
#include "merge.cuh"
#include "plan_core.h"
#include "plan_cut.h"

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

// Minimum of one int per thread over the block (all threads call it).
__device__ __forceinline__ int block_min(int x, int *smem32) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, d));
    if (lane == 0) smem32[warp] = x;
    __syncthreads();
    int r = smem32[0];
    for (int w = 1; w < nwarps; ++w) r = min(r, smem32[w]);
    __syncthreads();
    return r;
}

// One schedule: unit prefix sums, per-CTA flattened ranges (cut by cost, see plan_core.h),
// per-sequence split info and zeroed merge counters, plus its header words.  Every thread of the
// block calls it; thread i owns the consecutive sequences [b0, b1).
__device__ void plan_schedule(const int32_t *__restrict__ seqlens, int batch, int b0, int b1, int ctas, int groups,
                              int unit_rows, int gcols, int mode, int32_t *__restrict__ ws, const Sched &sc, int hdr,
                              int64_t *scan_smem) {
    int32_t *tile_off = ws + sc.tile_off / 4;
    int32_t *ranges = ws + sc.cta_ranges / 4;
    int32_t *seq_info = ws + sc.seq_info / 4;
    int32_t *counters = ws + sc.counters / 4;
    int32_t *cta_seq = ws + sc.cta_seq / 4;
    const int E = end_cost_units(unit_rows);
    // flattened unit offsets and cost offsets: exclusive prefix sums per sequence
    int64_t mine = 0, mine_cost = 0;
    for (int b = b0; b < b1; ++b) {
        const int u = units_of(seqlens[b], unit_rows);
        mine += u;
        mine_cost += u + (u > 0 ? E : 0);
    }
    int64_t total, total_cost;
    int64_t f = block_exclusive_scan(mine, scan_smem, &total);
    int64_t g = block_exclusive_scan(mine_cost, scan_smem, &total_cost);
    const int used = used_ctas(total, ctas);
    for (int c = threadIdx.x; c < ctas; c += blockDim.x) {
        cta_seq[c] = batch;  // no units, unless a sequence below claims it
        if (c >= used) ranges[2 * c] = (int32_t)total;
    }
    // range starts that fall inside each sequence's cost interval, and its split CTAs
    int64_t split_slots = 0;
    for (int b = b0; b < b1; ++b) {
        const int64_t units = units_of(seqlens[b], unit_rows);
        const int64_t t0 = f, t1 = f + units;
        const int64_t gend = g + units + (units > 0 ? E : 0);
        int first = -1, nsplit = 0;
        if (units > 0) {
            first = cta_of(total_cost, used, g);
            nsplit = cta_of(total_cost, used, g + units - 1) - first + 1;
            for (int c = first_range_at_or_after(total_cost, used, g); c < used; ++c) {
                const int64_t x = cta_begin(total_cost, used, c);
                if (x >= gend) break;
                ranges[2 * c] = (int32_t)unit_at_cost(x, g, t0, units);
            }
        }
        tile_off[b] = (int32_t)t0;
        seq_info[4 * b + 0] = (int32_t)units;
        seq_info[4 * b + 1] = first;
        seq_info[4 * b + 2] = nsplit;
        if (nsplit >= 2) split_slots += nsplit;
        f = t1;
        g = gend;
    }
    // partial-output slots: exclusive prefix sum of the split counts of split sequences (the scan's
    // barriers also publish every range start written above)
    int64_t slots;
    int64_t sl = block_exclusive_scan(split_slots, scan_smem, &slots);
    for (int b = b0; b < b1; ++b) {
        seq_info[4 * b + 3] = (int32_t)sl;
        const int nsplit = seq_info[4 * b + 2];
        if (nsplit >= 2) sl += nsplit;
        // the units whose range starts inside this sequence start their walk here
        const int first = seq_info[4 * b + 1];
        for (int c = first; c >= 0 && c < first + nsplit; ++c)
            if (ranges[2 * c] >= tile_off[b]) cta_seq[c] = b;
    }
    for (int c = threadIdx.x; c < ctas; c += blockDim.x)
        ranges[2 * c + 1] = c + 1 < ctas ? ranges[2 * (c + 1)] : (int32_t)total;
    for (int i = threadIdx.x; i < 2 * batch * groups; i += blockDim.x) counters[i] = 0;
    for (int i = threadIdx.x; i < batch; i += blockDim.x) ws[sc.done / 4 + i] = 0;
    if (threadIdx.x == 0) {
        tile_off[batch] = (int32_t)total;
        ws[hdr + kSchCtas] = ctas;
        ws[hdr + kSchGroups] = groups;
        ws[hdr + kSchTotal] = (int32_t)total;
        ws[hdr + kSchSlotsUsed] = (int32_t)slots;
        ws[hdr + kSchGroupCols] = gcols;
        ws[hdr + kSchMode] = mode;
    }
}

// One CTA of kPlanThreads threads: the pair schedule and, for more than 16 query columns, the duo
// schedule (whose column-group width depends on the shortest nonempty sequence).  Writes the header
// (and clears the status word) so that the decode kernels can check that they run on a plan for
// their own grid.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t *__restrict__ seqlens, int batch, int ncols,
                                                            int num_sms, int32_t *__restrict__ ws, WsLayout lay) {
    // Launched as a programmatic dependent: nothing is read (seqlens may come from the
    // preceding kernel) or written (that kernel may still read the workspace) before it
    // completes.  Then the decode kernel may start its prologue: it waits for this grid in
    // turn before reading the workspace.  Both are no-ops without programmatic launch.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int64_t scan_smem[32];
    __shared__ int min_smem[32];
    const int per = (batch + kPlanThreads - 1) / kPlanThreads;
    const int b0 = min(batch, (int)threadIdx.x * per), b1 = min(batch, b0 + per);
    plan_schedule(seqlens, batch, b0, b1, lay.ctas, lay.groups, kTileRows, group_cols(ncols), 0, ws, lay.pair,
                  kHdrPair, scan_smem);
    if (lay.has_duo) {
        int mn = 0x7fffffff;
        for (int b = b0; b < b1; ++b) {
            const int L = seqlens[b];
            if (L > 0) mn = min(mn, L);
        }
        mn = block_min(mn, min_smem);
        const int mode = duo_mode(ncols, mn == 0x7fffffff ? 0 : mn);
        const int groups = duo_groups(ncols, mode);
        plan_schedule(seqlens, batch, b0, b1, num_ctas(num_sms, groups), groups, kDuoRows, duo_group_cols(mode), mode,
                      ws, lay.duo, kHdrDuo, scan_smem);
    }
    if (threadIdx.x == 0) {
        ws[kHdrStatus] = 0;
        ws[kHdrBatch] = batch;
        ws[kHdrCols] = ncols;
        ws[kHdrSlotsMax] = lay.slots;
        ws[kHdrSchedUsed] = 0;
    }
}

// Stand-alone split merge: one CTA of 128 threads per (column, sequence), 4 latent rows per
// thread.  Up to 8 splits' partial LSEs and outputs are loaded at once, so that a sequence with
// at most 8 splits costs one round trip to L2 once its partials are complete.  Also writes
// O = 0, LSE = -inf for sequences without rows.
//   spin = 0: launched after the decode (or by the caller after MLA_FLAG_SKIP_COMBINE): waits
//             for the whole previous grid (griddepcontrol.wait) and reads the schedule the
//             decode recorded.
//   spin = 1: a programmatic dependent of the duo decode kernel that starts on the SMs its CTAs
//             leave: each CTA waits only for the split counters of its own sequence and column
//             group (both CTAs of every split add 1 with release semantics once their partials
//             are stored), so early sequences merge while the decode still runs.
// Either way, for the duo schedule the last combine CTA of a sequence rearms its counters.
constexpr int kCombineBatch = 8;
__device__ __forceinline__ int ld_acquire_gpu(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__global__ void __launch_bounds__(128) combine_kernel(int32_t *__restrict__ ws, const float *__restrict__ opart,
                                                      const float *__restrict__ lsepart, int ncols, WsLayout lay,
                                                      __nv_bfloat16 *__restrict__ o, float *__restrict__ lse, int spin,
                                                      unsigned long long wait_limit_ns) {
    if (!spin) asm volatile("griddepcontrol.wait;" ::: "memory");
    const int n = blockIdx.x, b = blockIdx.y;
    // the schedule of the decode that wrote the partials (the plan's tables: complete before the
    // decode started)
    const bool duo = spin || __ldcg(ws + kHdrSchedUsed) == 1;
    const Sched &sc = duo ? lay.duo : lay.pair;
    const int32_t *seq_info = ws + sc.seq_info / 4;
    const int nsplit = __ldcg(seq_info + 4 * b + 2);
    if (nsplit == 1) return;  // written by the decode kernel
    int32_t *cnt = nullptr;
    if (duo && nsplit >= 2) {
        const int gcols = __ldcg(ws + kHdrDuo + kSchGroupCols), groups = __ldcg(ws + kHdrDuo + kSchGroups);
        cnt = ws + sc.counters / 4 + ((int64_t)b * groups + n / gcols) * 2;
    }
    if (spin && nsplit >= 2) {
        __shared__ int ready;
        if (threadIdx.x == 0) {
            const uint64_t t0 = global_timer_ns();
            int ok = 1;
            while (ld_acquire_gpu(cnt) < nsplit || ld_acquire_gpu(cnt + 1) < nsplit) {
                if (global_timer_ns() - t0 > wait_limit_ns) {
                    atomicCAS(ws + kHdrStatus, 0, kStatusTimeout);
                    ok = 0;
                    break;
                }
                __nanosleep(256);
            }
            ready = ok;
        }
        __syncthreads();  // with thread 0's acquire, orders every thread's reads of the partials
        if (!ready) return;
    }
    const int64_t orow = ((int64_t)b * ncols + n) * kDv + 4 * threadIdx.x;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float lse_tot = -INFINITY;
    if (nsplit >= 2) {
        const int s0 = seq_info[4 * b + 3];
        const float *l = lsepart + (int64_t)s0 * ncols + n;
        const float *op = opart + ((int64_t)s0 * ncols + n) * kDv + 4 * threadIdx.x;
        float ls[kCombineBatch];
        float4 v[kCombineBatch];
#pragma unroll
        for (int u = 0; u < kCombineBatch; ++u) {
            const int su = u < nsplit ? u : nsplit - 1;
            ls[u] = __ldcg(l + (int64_t)su * ncols);
            v[u] = __ldcg(reinterpret_cast<const float4 *>(op + (int64_t)su * ncols * kDv));
        }
        if (nsplit <= kCombineBatch) {
            lse_tot = merged_lse([&](int s) { return ls[s]; }, nsplit);
        } else {
            lse_tot = merged_lse([&](int s) { return __ldcg(l + (int64_t)s * ncols); }, nsplit);
        }
        // the sum runs in split order, as in the decode kernel's own merge
        if (lse_tot != -INFINITY) {
#pragma unroll
            for (int u = 0; u < kCombineBatch; ++u) {
                if (u < nsplit) {
                    const float w = merge_weight(ls[u], lse_tot);
                    acc[0] = fmaf(w, v[u].x, acc[0]);
                    acc[1] = fmaf(w, v[u].y, acc[1]);
                    acc[2] = fmaf(w, v[u].z, acc[2]);
                    acc[3] = fmaf(w, v[u].w, acc[3]);
                }
            }
            for (int s = kCombineBatch; s < nsplit; ++s) {
                const float w = merge_weight(__ldcg(l + (int64_t)s * ncols), lse_tot);
                const float4 vs = __ldcg(reinterpret_cast<const float4 *>(op + (int64_t)s * ncols * kDv));
                acc[0] = fmaf(w, vs.x, acc[0]);
                acc[1] = fmaf(w, vs.y, acc[1]);
                acc[2] = fmaf(w, vs.z, acc[2]);
                acc[3] = fmaf(w, vs.w, acc[3]);
            }
        }
    }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t *>(&lo);
    packed.y = *reinterpret_cast<const uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(o + orow) = packed;
    if (threadIdx.x == 0) {
        lse[(int64_t)b * ncols + n] = lse_tot;
        if (cnt && atomicAdd(ws + sc.done / 4 + b, 1) == ncols - 1) {
            // every combine CTA of this sequence is past its wait: rearm for the next decode
            const int groups = __ldcg(ws + kHdrDuo + kSchGroups);
            for (int i = 0; i < 2 * groups; ++i) ws[sc.counters / 4 + (int64_t)b * groups * 2 + i] = 0;
            ws[sc.done / 4 + b] = 0;
        }
    }
}

}  // namespace mla
