// Streaming probe: the decode kernel's KV read pattern without its computation, to measure the
// read bandwidth that pattern can reach on this GPU (the "attainable" line beside the roofline).
//
// Same grid and split as the decode: one 2-CTA cluster per work unit, rank r of a pair loads
// latent chunks 4r..4r+3 of every 128-row tile (two 32 KB V-pair slots, 64-row TMA boxes of 64
// columns, 128B swizzle) and 32 rope columns (64B swizzle), with an L2 prefetch one tile ahead.
// A single consumer thread frees each tile's slots as soon as they land.  Every wait is bounded.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "ptx_sm100.cuh"

namespace mla {

constexpr int kProbeSlots = 5;  // V-pair slots, as the decode's 16-column configuration

struct ProbeParams {
    int64_t rows;   // rows of the [rows, 576] matrix streamed (a multiple of 128)
    int units;      // CTA pairs
    int32_t *err;   // set to 1 when a wait ran out
};

__device__ __forceinline__ bool probe_wait(uint32_t bar, uint32_t parity, int32_t *err) {
    for (uint32_t i = 0; i < (1u << 22); ++i)
        if (mbar_try_wait(bar, parity)) return true;
    atomicExch(err, 1);
    return false;
}

__global__ void __launch_bounds__(64, 1) stream_probe_kernel(const __grid_constant__ CUtensorMap tm_kv,
                                                             const __grid_constant__ CUtensorMap tm_kvr,
                                                             const ProbeParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    constexpr uint32_t V_SLOT = 32768, R_SLOT = 8192;
    constexpr uint32_t OFF_R = kProbeSlots * V_SLOT, OFF_BAR = OFF_R + 2 * R_SLOT;
    auto bar = [&](int i) { return sb + OFF_BAR + 8u * (uint32_t)i; };
    constexpr int VF = 0, VE = kProbeSlots, RF = 2 * kProbeSlots, RE = RF + 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < RE + 2; ++i) mbar_init(bar(i), 1);
        fence_barrier_init();
    }
    __syncthreads();
    const int u = blockIdx.x >> 1, rank = blockIdx.x & 1;
    const int64_t tiles = p.rows / 128;
    const int64_t t0 = tiles * u / p.units, t1 = tiles * (u + 1) / p.units;
    const int rope_x = 512 + 32 * rank;
    if (warp == 0 && lane == 0) {
        if (t0 < t1)
            for (int h = 0; h < 2; ++h) {
                for (int c = 0; c < 4; ++c) tma_prefetch_l2_2d(&tm_kv, (4 * rank + c) * 64, (int)(t0 * 128 + 64 * h));
                tma_prefetch_l2_2d(&tm_kvr, rope_x, (int)(t0 * 128 + 64 * h));
            }
        int issued_v[kProbeSlots] = {}, issued_r[2] = {};
        bool ok = true;
        int k = 0;
        for (int64_t t = t0; t < t1 && ok; ++t, ++k) {
            if (t + 1 < t1)
                for (int h = 0; h < 2; ++h) {
                    for (int c = 0; c < 4; ++c)
                        tma_prefetch_l2_2d(&tm_kv, (4 * rank + c) * 64, (int)((t + 1) * 128 + 64 * h));
                    tma_prefetch_l2_2d(&tm_kvr, rope_x, (int)((t + 1) * 128 + 64 * h));
                }
            const int rs = k & 1;
            ok = probe_wait(bar(RE + rs), ((k >> 1) & 1) ^ 1, p.err);
            if (!ok) break;
            mbar_arrive_expect_tx(bar(RF + rs), R_SLOT);
            for (int h = 0; h < 2; ++h)
                tma_load_2d(sb + OFF_R + rs * R_SLOT + h * 4096u, &tm_kvr, bar(RF + rs), rope_x, (int)(t * 128 + 64 * h));
            ++issued_r[rs];
            for (int i = 0; i < 2 && ok; ++i) {
                const int g = 2 * k + i, vs = g % kProbeSlots;
                ok = probe_wait(bar(VE + vs), ((g / kProbeSlots) & 1) ^ 1, p.err);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(VF + vs), V_SLOT);
                for (int hc = 0; hc < 2; ++hc)
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d(sb + vs * V_SLOT + hc * 16384u + h * 8192u, &tm_kv, bar(VF + vs),
                                    (4 * rank + 2 * i + hc) * 64, (int)(t * 128 + 64 * h));
                ++issued_v[vs];
            }
        }
        // no load may still be in flight when the CTA exits: wait for the last one of every slot
        for (int i = 0; i < kProbeSlots; ++i)
            if (issued_v[i] > 0) probe_wait(bar(VF + i), (issued_v[i] - 1) & 1, p.err);
        for (int i = 0; i < 2; ++i)
            if (issued_r[i] > 0) probe_wait(bar(RF + i), (issued_r[i] - 1) & 1, p.err);
    } else if (warp == 1 && lane == 0) {
        int k = 0;
        bool ok = true;
        for (int64_t t = t0; t < t1 && ok; ++t, ++k) {
            const int rs = k & 1;
            ok = probe_wait(bar(RF + rs), (k >> 1) & 1, p.err);
            if (!ok) break;
            mbar_arrive(bar(RE + rs));
            for (int i = 0; i < 2 && ok; ++i) {
                const int g = 2 * k + i, vs = g % kProbeSlots;
                ok = probe_wait(bar(VF + vs), (g / kProbeSlots) & 1, p.err);
                if (ok) mbar_arrive(bar(VE + vs));
            }
        }
    }
    __syncthreads();
}

constexpr uint32_t kProbeSmem = kProbeSlots * 32768 + 2 * 8192 + 1024 + 1024;

}  // namespace mla
