// Ablation of the two forms of the decode's contractions on the tensor cores (the pages' padding
// argument, FlashMLA-ETAP technical summary, "Problem Statement" and "Methodology"): per 128-row KV tile
// and h query heads (one query token), with d_qk = 576 and d_v = 512, bf16 operands, fp32 accumulators:
//
//   transposed (ETAP):   S^T = K Q^T   M = 128 KV rows,  N = h,        K = 576  (36 MMAs of K = 16)
//                        O^T = V^T P^T M = 128 latent x4, N = h,       K = 128  (32 MMAs)
//   untransposed:        S   = Q K^T   M = h padded to 64 or 128, N = 128 KV rows, K = 576 (36 MMAs)
//                        O   = P V     M = h padded,  N = 256 latent x2, K = 128 (16 MMAs)
//
// Only the MMA instructions are timed: the operands are zero-filled shared memory laid out as the
// real operands would be (K-major Q, K, P; MN-major V), with chunk addresses wrapped inside a 96 KB
// area per operand (a whole bf16 tile is 147 KB; the values are never used), and accumulators in
// TMEM columns that some M-tiles share (the sums are not read).  Thread 0 issues the score MMAs of every
// tile and thread 32 the output MMAs (as the decode kernel splits them between two issuing threads),
// or one of the two streams alone.  Every wait is bounded.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace mla {

constexpr uint32_t kAblSmem = 200 * 1024;  // operand area (zero-filled) + alignment slack

struct AblationParams {
    int form;       // 0 transposed (ETAP), 1 untransposed (heads padded to M = 64 or 128)
    int heads;      // 16, 32, 64 or 128
    int streams;    // 1 scores only, 2 outputs only, 3 both (two issuing threads)
    int tiles;      // tiles per CTA
    unsigned long long *cycles;  // [gridDim.x]: clock cycles of the CTA's MMA work
    int32_t *err;   // set to 1 when a wait ran out
};

__global__ void __launch_bounds__(64, 1) form_ablation_kernel(const AblationParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_slot;
    __shared__ __align__(8) uint64_t bars[2];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sb - raw);
    // zero the operands: A area [0, 96 KB), B area [96 KB, 192 KB)
    for (int i = threadIdx.x; i < 192 * 1024 / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bars[0]), 1);
        mbar_init(smem_addr(&bars[1]), 1);
        fence_barrier_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(smem_addr(&tmem_slot), 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t a0 = sb, b0 = sb + 96 * 1024;
    const int h = p.heads;
    const int hpad = h <= 64 ? 64 : 128;
    const bool run = lane == 0 && ((warp == 0 && (p.streams & 1)) || (warp == 1 && (p.streams & 2)));
    uint64_t t0 = 0, t1 = 0;
    if (run) {
        t0 = clock64();
        for (int t = 0; t < p.tiles; ++t) {
            if (warp == 0) {
                if (p.form == 0) {
                    // S^T: A = K tile [128 x 576] K-major (9 chunks of 64 columns), B = Q^T [h x 576] K-major
                    const uint32_t idesc = idesc_bf16_f32(128, h, 0, 0);
                    for (int k = 0; k < 36; ++k) {
                        const uint32_t c = (uint32_t)(k >> 2) % 5u, j = (uint32_t)(k & 3);
                        const uint64_t a = smem_desc(a0 + c * 16384u + 32u * j, 16, 1024, kSwizzle128B);
                        const uint64_t b = smem_desc(b0 + c * 128u * h + 32u * j, 16, 1024, kSwizzle128B);
                        umma_bf16(tmem + 256, a, b, idesc, k > 0 ? 1u : 0u);
                    }
                } else {
                    // S: A = Q [hpad x 576] K-major, B = K tile [128 x 576] K-major
                    const uint32_t idesc = idesc_bf16_f32(hpad, 128, 0, 0);
                    for (int k = 0; k < 36; ++k) {
                        const uint32_t c = (uint32_t)(k >> 2) % 5u, j = (uint32_t)(k & 3);
                        const uint64_t a = smem_desc(a0 + c * 128u * hpad + 32u * j, 16, 1024, kSwizzle128B);
                        const uint64_t b = smem_desc(b0 + c * 16384u + 32u * j, 16, 1024, kSwizzle128B);
                        umma_bf16(tmem + 384, a, b, idesc, k > 0 ? 1u : 0u);
                    }
                }
            } else {
                if (p.form == 0) {
                    // O^T: A = V^T (MN-major, 4 M-tiles of 128 latent columns), B = P^T [128 rows x h] MN-major
                    const uint32_t idesc = idesc_bf16_f32(128, h, 1, 1);
                    const uint32_t ppitch = h * 2u < 128u ? h * 2u : 128u;  // bytes per KV row of P^T
                    const uint32_t pswz = ppitch == 128 ? kSwizzle128B : ppitch == 64 ? kSwizzle64B : kSwizzle32B;
                    // M-tile accumulators: 4 x 64 columns for h <= 64; two shared 128-column ones for h = 128
                    for (int mt = 0; mt < 4; ++mt)
                        for (int s = 0; s < 8; ++s) {
                            const uint64_t a = smem_desc(a0 + (uint32_t)(mt & 1) * 32768u + 2048u * s, 16384, 1024,
                                                         kSwizzle128B);
                            const uint64_t b = smem_desc(b0 + 16u * ppitch * s, 128u * ppitch, 8u * ppitch, pswz);
                            const uint32_t d = h <= 64 ? (uint32_t)mt * 64u : (uint32_t)(mt & 1) * 128u;
                            umma_bf16(tmem + d, a, b, idesc, s > 0 ? 1u : 0u);
                        }
                } else {
                    // O: A = P [hpad x 128 rows] K-major (2 chunks of 64), B = V [128 rows x 256] MN-major
                    const uint32_t idesc = idesc_bf16_f32(hpad, 256, 0, 1);
                    for (int half = 0; half < 2; ++half)
                        for (int s = 0; s < 8; ++s) {
                            const uint32_t c = (uint32_t)(s >> 2), j = (uint32_t)(s & 3);
                            const uint64_t a = smem_desc(a0 + c * 128u * hpad + 32u * j, 16, 1024, kSwizzle128B);
                            const uint64_t b = smem_desc(b0 + 2048u * s, 16384, 1024, kSwizzle128B);
                            umma_bf16(tmem, a, b, idesc, s > 0 ? 1u : 0u);
                        }
                }
            }
        }
        // one commit: it arrives once every MMA this thread issued has completed
        const uint32_t bar = smem_addr(&bars[warp]);
        umma_commit(bar);
        bool done = false;
        for (uint32_t it = 0; it < (1u << 26) && !done; ++it) done = mbar_test_wait(bar, 0);
        if (!done) atomicExch(p.err, 1);
        t1 = clock64();
    }
    __shared__ unsigned long long dt[2];
    if (lane == 0) dt[warp] = run ? t1 - t0 : 0ull;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) p.cycles[blockIdx.x] = dt[0] > dt[1] ? dt[0] : dt[1];
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace mla
