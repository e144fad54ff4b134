// ETAP decode kernel for sm_100a (FlashMLA-ETAP technical summary, "Methodology",
// ETAP steps 1-4, and "Integration and Implementation": producer/consumer roles
// around a circular shared-memory buffer, block-wise KV processing with online
// softmax statistics).  Re-designed for Blackwell:
//
//   * one CTA per SM; CTA (c, g) handles column group g (16 query columns,
//     heads x tokens) over the flattened KV tile range the plan gave CTA c;
//   * warp 0 (producer) streams each 128-row KV tile with TMA into a ring of
//     32 KB "pair" slots (two 64-column chunks = 128 V columns) plus a 16 KB
//     slot for the 64 rope columns; Q (16 x 576) is loaded once per segment;
//   * warp 1, lane 0 (MMA issuer) runs tcgen05.mma:
//       step 1  S^T[128 x 16]  = K_tile[128 x 576] . Q^T          (K-major A and B)
//       step 3  O^T[512 x 32] += V^T[512 x 128] . [P_hi^T | P_lo^T] (MN-major A and B)
//     with fp32 accumulators in TMEM (S^T double-buffered, O^T as 4 M-tiles);
//   * warps 2-5 (softmax) own one TMEM lane = one KV row each: step 2 is a
//     column softmax of S^T, i.e. a reduction ACROSS threads (butterfly
//     shuffles + an exchange through shared memory), with the running maximum
//     raised only when a column's maximum grows by more than 2^8 (O^T is then
//     rescaled in TMEM); P^T is written to shared memory as bf16 hi + lo parts
//     so the second contraction keeps ~16 mantissa bits of P;
//   * the same warps run the epilogue (step 4): O = (O^T)^T / l, LSE, written
//     as final bf16/fp32 outputs or as fp32 split partials.
//
// Every wait is bounded (a few seconds); on expiry the CTA records
// MLA_ERR_TIMEOUT in the workspace status word, drains its own asynchronous
// work and returns.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "plan_core.h"
#include "ptx_sm100.cuh"

namespace mla {

constexpr int kStatusTimeout = -6;      // MLA_ERR_TIMEOUT
constexpr int kStatusBlockTable = -7;   // MLA_ERR_BLOCK_TABLE
constexpr int kStatusInvalid = -1;      // MLA_ERR_INVALID_ARG
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p = 2^(x - m) stays <= 256

struct DecodeParams {
    const int32_t *seqlens;
    const int32_t *block_table;
    int32_t *ws;  // workspace (int32 view)
    float *opart;
    float *lsepart;
    __nv_bfloat16 *o;
    float *lse;
    int64_t kv_rows;  // contiguous: rows per sequence; paged: total rows of the pool
    int batch, q_len, num_heads, ncols, ctas, groups, max_blocks, paged, causal;
    float scale_log2;  // softmax_scale * log2(e)
    int cta_ranges_off, tile_off_off, seq_info_off;  // int32 offsets into ws
};

// Shared memory / TMEM plan for a 16-column group with split P.
struct Cfg16 {
    static constexpr int NG = 16;              // query columns per CTA (UMMA N of step 1)
    static constexpr int NP = 32;              // UMMA N of step 3: P_hi | P_lo
    static constexpr int NV = 5;               // V pair slots
    static constexpr int NR = 1;               // rope slots
    static constexpr int PB = 2;               // P^T buffers
    static constexpr int EARLY = NV - 4;       // pairs of tile k+1 whose slots never overlap tile k
    static constexpr uint32_t CHUNK = 16384;   // 128 rows x 64 bf16 columns, 128B-swizzled
    static constexpr uint32_t HALF = 8192;     // 64 rows of a chunk (one TMA box)
    static constexpr uint32_t V_SLOT = 2 * CHUNK;
    static constexpr uint32_t R_SLOT = CHUNK;
    static constexpr uint32_t Q_CHUNK = NG * 128;  // NG rows x 64 columns
    static constexpr uint32_t P_ROW = NP * 2;      // bytes per KV row of P^T
    static constexpr uint32_t P_BUF = 128 * P_ROW;
    static constexpr uint32_t OFF_V = 0;
    static constexpr uint32_t OFF_R = OFF_V + NV * V_SLOT;
    static constexpr uint32_t OFF_Q = OFF_R + NR * R_SLOT;
    static constexpr uint32_t OFF_P = OFF_Q + 9 * Q_CHUNK;
    static constexpr uint32_t OFF_BAR = OFF_P + PB * P_BUF;
    static constexpr uint32_t OFF_RED = OFF_BAR + 512;  // float [2][4][16] column max exchange
    static constexpr uint32_t OFF_REDL = OFF_RED + 512; // float [4][16] column sum exchange
    static constexpr uint32_t OFF_MISC = OFF_REDL + 256;
    static constexpr uint32_t BYTES = OFF_MISC + 64;
    static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
    // TMEM columns
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t O_COL = 0;       // 4 M-tiles x NP columns
    static constexpr uint32_t S_COL = 128;     // 2 buffers x NG columns
    // P^T B-operand swizzle: rows of 64 bytes -> 64B swizzle
    static constexpr uint32_t P_SWIZZLE = kSwizzle64B;
    static constexpr uint32_t P_SWZ_MASK = 3;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, NG, 0, 0);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, NP, 1, 1);
};
static_assert(Cfg16::SMEM_ALLOC <= 232448, "shared memory plan exceeds 227 KB");
static_assert(Cfg16::OFF_R % 1024 == 0 && Cfg16::OFF_Q % 1024 == 0 && Cfg16::OFF_P % 1024 == 0, "alignment");
static_assert(4 * Cfg16::NP + 2 * Cfg16::NG <= (int)Cfg16::TMEM_COLS, "TMEM plan");

// barrier indices
template <class C>
struct Bars {
    static constexpr int VFULL = 0;
    static constexpr int VEMPTY = VFULL + C::NV;
    static constexpr int RFULL = VEMPTY + C::NV;
    static constexpr int REMPTY = RFULL + C::NR;
    static constexpr int QFULL = REMPTY + C::NR;
    static constexpr int QEMPTY = QFULL + 1;
    static constexpr int SFULL = QEMPTY + 1;
    static constexpr int SEMPTY = SFULL + 2;
    static constexpr int PFULL = SEMPTY + 2;
    static constexpr int PEMPTY = PFULL + C::PB;
    static constexpr int TAIL = PEMPTY + C::PB;
    static constexpr int FINAL = TAIL + 1;
    static constexpr int RED = FINAL + 1;
    static constexpr int REDL = RED + 1;
    static constexpr int COUNT = REDL + 1;
};
static_assert(Bars<Cfg16>::COUNT * 8 <= 512, "barrier area");

// Bounded wait on an mbarrier phase.  Returns false (and raises the CTA abort
// flag) when the wait ran past kWaitLimitNs, or when another role aborted.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                           int32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((spin & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
}
// Wait used only while draining after an abort: bounded, ignores the abort flag.
__device__ __forceinline__ void drain_phase(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kDrainLimitNs) return;
    }
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Walks the (sequence, tile range) segments of flattened tiles [fb, fe).
struct SegIter {
    int64_t f, fe;
    int b;
    __device__ void init(const int32_t *tile_off, int batch, int64_t fb, int64_t fe_) {
        f = fb;
        fe = fe_;
        // last b with tile_off[b] <= fb
        int lo = 0, hi = batch;  // tile_off[batch] = total > fb when fb < fe
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (tile_off[mid] <= fb) lo = mid; else hi = mid;
        }
        b = lo;
    }
    __device__ bool next(const int32_t *tile_off, int &ob, int &t0, int &t1) {
        if (f >= fe) return false;
        while (tile_off[b + 1] <= f) ++b;
        ob = b;
        t0 = (int)(f - tile_off[b]);
        int64_t e = fe < (int64_t)tile_off[b + 1] ? fe : (int64_t)tile_off[b + 1];
        t1 = (int)(e - tile_off[b]);
        f = e;
        return true;
    }
};

// Column reduction of 16 values per lane across the 32 lanes of a warp
// (recursive halving: 16 shuffles instead of 5 per column).  Lane l ends with
// the reduction of column col16(l); lanes l and l^1 hold the same column.
__device__ __forceinline__ int col16(int lane) {
    return (((lane >> 4) & 1) << 3) | (((lane >> 3) & 1) << 2) | (((lane >> 2) & 1) << 1) | ((lane >> 1) & 1);
}
template <bool IS_MAX>
__device__ __forceinline__ float op2(float a, float b) {
    return IS_MAX ? fmaxf(a, b) : a + b;
}
template <bool IS_MAX>
__device__ __forceinline__ float warp_colreduce16(const float (&v)[16], int lane) {
    float a8[8], a4[4], a2[2];
    bool up = (lane & 16) != 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float send = up ? v[j] : v[j + 8];
        float keep = up ? v[j + 8] : v[j];
        a8[j] = op2<IS_MAX>(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
    up = (lane & 8) != 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float send = up ? a8[j] : a8[j + 4];
        float keep = up ? a8[j + 4] : a8[j];
        a4[j] = op2<IS_MAX>(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
    up = (lane & 4) != 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        float send = up ? a4[j] : a4[j + 2];
        float keep = up ? a4[j + 2] : a4[j];
        a2[j] = op2<IS_MAX>(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    }
    up = (lane & 2) != 0;
    float a1 = op2<IS_MAX>(up ? a2[1] : a2[0], __shfl_xor_sync(0xffffffffu, up ? a2[0] : a2[1], 2));
    return op2<IS_MAX>(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}

template <class C>
__global__ void __launch_bounds__(192, 1)
    etap_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                       const __grid_constant__ DecodeParams p) {
    using BR = Bars<C>;
    constexpr int NG = C::NG;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - raw_addr);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x / p.groups;
    const int grp = blockIdx.x % p.groups;
    int32_t *status = p.ws + kHdrStatus;

    // The schedule must come from a plan for this same grid.
    if (p.ws[kHdrCtas] != p.ctas || p.ws[kHdrGroups] != p.groups || p.ws[kHdrBatch] != p.batch) {
        if (threadIdx.x == 0) atomicCAS(status, 0, kStatusInvalid);
        return;
    }

    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NV; ++i) {
            mbar_init(bar(BR::VFULL + i), 1);
            mbar_init(bar(BR::VEMPTY + i), 1);
        }
        for (int i = 0; i < C::NR; ++i) {
            mbar_init(bar(BR::RFULL + i), 1);
            mbar_init(bar(BR::REMPTY + i), 1);
        }
        mbar_init(bar(BR::QFULL), 1);
        mbar_init(bar(BR::QEMPTY), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BR::SFULL + i), 1);
            mbar_init(bar(BR::SEMPTY + i), 128);
        }
        for (int i = 0; i < C::PB; ++i) {
            mbar_init(bar(BR::PFULL + i), 128);
            mbar_init(bar(BR::PEMPTY + i), 1);
        }
        mbar_init(bar(BR::TAIL), 1);
        mbar_init(bar(BR::FINAL), 1);
        mbar_init(bar(BR::RED), 128);
        mbar_init(bar(BR::REDL), 128);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_kv);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int32_t *ranges = p.ws + p.cta_ranges_off;
    const int32_t *tile_off = p.ws + p.tile_off_off;
    const int32_t *seq_info = p.ws + p.seq_info_off;
    const int64_t fb = ranges[2 * cta], fe = ranges[2 * cta + 1];
    const int64_t l_cap = p.paged ? (int64_t)p.max_blocks * kPage : p.kv_rows;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // Completed-phase bookkeeping for the abort drain: only the latest TMA
        // fill of a slot can still be in flight (the previous one was consumed
        // before the slot's empty barrier let this one start).
        int phases_v[C::NV], arms_r[C::NR];
        bool tma_v[C::NV];
#pragma unroll
        for (int i = 0; i < C::NV; ++i) {
            phases_v[i] = 0;
            tma_v[i] = false;
        }
#pragma unroll
        for (int i = 0; i < C::NR; ++i) arms_r[i] = 0;
        int arms_q = 0, tail_uses = 0;
        bool ok = true;
        if (fb < fe) {
            SegIter it;
            it.init(tile_off, p.batch, fb, fe);
            int b, t0, t1, seg = 0, k = 0;
            while (ok && it.next(tile_off, b, t0, t1)) {
                int L = p.seqlens[b];
                if ((int64_t)L > l_cap) {
                    if (lane == 0) atomicCAS(status, 0, kStatusInvalid);
                    L = (int)l_cap;
                }
                if (L < 0) L = 0;
                if (seg > 0) ok = wait_phase(bar(BR::QEMPTY), (seg - 1) & 1, abort_flag, status);
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(BR::QFULL), 9 * C::Q_CHUNK);
                    const int qrow = b * p.ncols + grp * NG;
                    for (int c = 0; c < 9; ++c)
                        tma_load_2d(sbase + C::OFF_Q + c * C::Q_CHUNK, &tm_q, bar(BR::QFULL), c * 64, qrow);
                }
                ++arms_q;
                for (int t = t0; t < t1 && ok; ++t, ++k) {
                    const int row0 = t * kTileRows;
                    int valid = L - row0;
                    valid = valid < 0 ? 0 : (valid > kTileRows ? kTileRows : valid);
                    int y[2];
                    bool loaded[2];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        loaded[hh] = valid > 64 * hh;
                        y[hh] = 0;
                        if (loaded[hh]) {
                            if (p.paged) {
                                const int pg = (row0 >> 6) + hh;
                                const int blk = p.block_table[(int64_t)b * p.max_blocks + pg];
                                if (blk < 0 || (int64_t)blk * kPage >= p.kv_rows) {
                                    if (lane == 0) atomicCAS(status, 0, kStatusBlockTable);
                                    loaded[hh] = false;
                                } else {
                                    y[hh] = blk * kPage;
                                }
                            } else {
                                y[hh] = (int)((int64_t)b * p.kv_rows + row0 + 64 * hh);
                            }
                        }
                    }
                    const int nload = (int)loaded[0] + (int)loaded[1];
                    const bool tail = !(loaded[0] && loaded[1] && valid == kTileRows);
                    // rope chunk (columns 512..575): rows past the end are masked in S^T, no zeroing needed
                    {
                        const int rs = k % C::NR;
                        ok = wait_phase(bar(BR::REMPTY + rs), ((k / C::NR) & 1) ^ 1, abort_flag, status);
                        if (!ok) break;
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar(BR::RFULL + rs), nload * C::HALF);
                            for (int hh = 0; hh < 2; ++hh)
                                if (loaded[hh])
                                    tma_load_2d(sbase + C::OFF_R + rs * C::R_SLOT + hh * C::HALF, &tm_kv,
                                                bar(BR::RFULL + rs), 512, y[hh]);
                        }
                        ++arms_r[rs];
                    }
                    // V pairs: chunks (2i, 2i+1) = latent columns [128 i, 128 i + 128)
                    for (int i = 0; i < 4 && ok; ++i) {
                        const int g4 = 4 * k + i;
                        const int vs = g4 % C::NV;
                        ok = wait_phase(bar(BR::VEMPTY + vs), ((g4 / C::NV) & 1) ^ 1, abort_flag, status);
                        if (!ok) break;
                        const uint32_t dst = sbase + C::OFF_V + vs * C::V_SLOT;
                        if (!tail) {
                            if (lane == 0) {
                                mbar_arrive_expect_tx(bar(BR::VFULL + vs), C::V_SLOT);
                                for (int hc = 0; hc < 2; ++hc)
                                    for (int hh = 0; hh < 2; ++hh)
                                        tma_load_2d(dst + hc * C::CHUNK + hh * C::HALF, &tm_kv, bar(BR::VFULL + vs),
                                                    (2 * i + hc) * 64, y[hh]);
                            }
                            ++phases_v[vs];
                            tma_v[vs] = true;
                        } else {
                            // Tail tile: land the valid rows, zero every other row so that
                            // whatever the cache holds past L_b (NaN included) meets P = 0 as 0.
                            if (nload > 0) {
                                if (lane == 0) {
                                    mbar_arrive_expect_tx(bar(BR::TAIL), 2 * nload * C::HALF);
                                    for (int hc = 0; hc < 2; ++hc)
                                        for (int hh = 0; hh < 2; ++hh)
                                            if (loaded[hh])
                                                tma_load_2d(dst + hc * C::CHUNK + hh * C::HALF, &tm_kv, bar(BR::TAIL),
                                                            (2 * i + hc) * 64, y[hh]);
                                }
                                ok = wait_phase(bar(BR::TAIL), tail_uses & 1, abort_flag, status);
                                ++tail_uses;
                                if (!ok) break;
                            }
                            for (int idx = lane; idx < 2 * kTileRows * 8; idx += 32) {
                                const int hc = idx / (kTileRows * 8);
                                const int r = (idx / 8) % kTileRows;
                                const int c16 = idx % 8;
                                if (r < valid && loaded[r >> 6]) continue;
                                uint4 *ptr = reinterpret_cast<uint4 *>(smem + C::OFF_V + vs * C::V_SLOT + hc * C::CHUNK +
                                                                       r * 128 + c16 * 16);
                                *ptr = make_uint4(0u, 0u, 0u, 0u);
                            }
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar(BR::VFULL + vs));
                            ++phases_v[vs];
                            tma_v[vs] = false;
                        }
                    }
                }
                ++seg;
            }
        }
        if (!ok) {
            // drain this warp's own copies still in flight
            for (int i = 0; i < C::NV; ++i)
                if (tma_v[i]) drain_phase(bar(BR::VFULL + i), (phases_v[i] - 1) & 1);
            for (int i = 0; i < C::NR; ++i)
                if (arms_r[i] > 0) drain_phase(bar(BR::RFULL + i), (arms_r[i] - 1) & 1);
            if (arms_q > 0) drain_phase(bar(BR::QFULL), (arms_q - 1) & 1);
            if (tail_uses > 0) drain_phase(bar(BR::TAIL), (tail_uses - 1) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && fb < fe) {
            bool ok = true;
            const uint32_t q_base = sbase + C::OFF_Q;
            auto qk_chunk = [&](uint32_t d_s, uint32_t a_base, int qchunk, bool first_acc) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t a = smem_desc(a_base + 32u * j, 16, 1024, kSwizzle128B);
                    const uint64_t bq = smem_desc(q_base + qchunk * C::Q_CHUNK + 32u * j, 16, 1024, kSwizzle128B);
                    umma_bf16(d_s, a, bq, C::IDESC_QK, (first_acc && j == 0) ? 0u : 1u);
                }
            };
            auto qk_pair = [&](int k, int i) -> bool {
                const int g4 = 4 * k + i;
                const int vs = g4 % C::NV;
                if (!wait_phase(bar(BR::VFULL + vs), (g4 / C::NV) & 1, abort_flag, status)) return false;
                tc_fence_after();
                const uint32_t d_s = tmem + C::S_COL + (k & 1) * NG;
                const uint32_t slot = sbase + C::OFF_V + vs * C::V_SLOT;
                qk_chunk(d_s, slot, 2 * i, false);
                qk_chunk(d_s, slot + C::CHUNK, 2 * i + 1, false);
                return true;
            };
            auto pv = [&](int k, bool first) -> bool {
                const int pb = k % C::PB;
                if (!wait_phase(bar(BR::PFULL + pb), (k / C::PB) & 1, abort_flag, status)) return false;
                tc_fence_after();
                const uint32_t p_base = sbase + C::OFF_P + pb * C::P_BUF;
                for (int i = 0; i < 4; ++i) {
                    const int g4 = 4 * k + i;
                    const int vs = g4 % C::NV;
                    const uint32_t v_base = sbase + C::OFF_V + vs * C::V_SLOT;
                    const uint32_t d_o = tmem + C::O_COL + i * C::NP;
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        // A = V^T: M = 128 latent columns (two 64-column chunks, LBO apart), K = 16 KV rows
                        const uint64_t a = smem_desc(v_base + 2048u * s, C::CHUNK, 1024, kSwizzle128B);
                        // B = P^T: K = 16 KV rows, N = NP columns contiguous (MN-major)
                        const uint64_t bp = smem_desc(p_base + 16u * C::P_ROW * s, C::P_BUF, 8 * C::P_ROW, C::P_SWIZZLE);
                        umma_bf16(d_o, a, bp, C::IDESC_PV, (first && s == 0) ? 0u : 1u);
                    }
                    umma_commit(bar(BR::VEMPTY + vs));
                }
                umma_commit(bar(BR::PEMPTY + pb));
                return true;
            };

            SegIter it;
            it.init(tile_off, p.batch, fb, fe);
            int b, t0, t1, seg = 0, k = 0, prev_k = -1;
            bool prev_first = false;
            while (ok && it.next(tile_off, b, t0, t1)) {
                ok = wait_phase(bar(BR::QFULL), seg & 1, abort_flag, status);
                for (int t = t0; t < t1 && ok; ++t, ++k) {
                    const bool first = (t == t0), last = (t == t1 - 1);
                    // step 1 for tile k: rope chunk first (frees its slot early) ...
                    ok = wait_phase(bar(BR::SEMPTY + (k & 1)), ((k >> 1) & 1) ^ 1, abort_flag, status);
                    if (!ok) break;
                    const int rs = k % C::NR;
                    ok = wait_phase(bar(BR::RFULL + rs), (k / C::NR) & 1, abort_flag, status);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d_s = tmem + C::S_COL + (k & 1) * NG;
                    qk_chunk(d_s, sbase + C::OFF_R + rs * C::R_SLOT, 8, true);
                    umma_commit(bar(BR::REMPTY + rs));
                    // ... then the V pairs whose slots do not overlap tile k-1 ...
                    for (int i = 0; i < C::EARLY && ok; ++i) ok = qk_pair(k, i);
                    if (!ok) break;
                    // ... step 3 for tile k-1 (needs its P^T from the softmax warps) ...
                    if (prev_k >= 0) ok = pv(prev_k, prev_first);
                    if (!ok) break;
                    // ... and the rest of tile k, whose slots step 3 of tile k-1 releases.
                    for (int i = C::EARLY; i < 4 && ok; ++i) ok = qk_pair(k, i);
                    if (!ok) break;
                    umma_commit(bar(BR::SFULL + (k & 1)));
                    if (last) umma_commit(bar(BR::QEMPTY));
                    prev_k = k;
                    prev_first = first;
                }
                ++seg;
            }
            if (ok && prev_k >= 0) ok = pv(prev_k, prev_first);
            // every MMA this thread issued must finish before TMEM is released
            umma_commit(bar(BR::FINAL));
            drain_phase(bar(BR::FINAL), 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue (warps 2..5)
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *red = reinterpret_cast<float *>(smem + C::OFF_RED);    // [2][4][16]
        float *redl = reinterpret_cast<float *>(smem + C::OFF_REDL);  // [4][16]
        bool ok = true;
        if (fb < fe) {
            SegIter it;
            it.init(tile_off, p.batch, fb, fe);
            int b, t0, t1, k = 0, seg = 0;
            while (ok && it.next(tile_off, b, t0, t1)) {
                int L = p.seqlens[b];
                if ((int64_t)L > l_cap) L = (int)l_cap;
                if (L < 0) L = 0;
                int vis[NG];
                float m[NG], lpart[NG];
#pragma unroll
                for (int n = 0; n < NG; ++n) {
                    const int ng = grp * NG + n;
                    const int tok = ng / p.num_heads;
                    int v = p.causal ? (L - p.q_len + tok + 1) : L;
                    vis[n] = (ng < p.ncols) ? (v < 0 ? 0 : v) : 0;
                    m[n] = -INFINITY;
                    lpart[n] = 0.f;
                }
                for (int t = t0; t < t1 && ok; ++t, ++k) {
                    const bool first = (t == t0);
                    ok = wait_phase(bar(BR::SFULL + (k & 1)), (k >> 1) & 1, abort_flag, status);
                    if (!ok) break;
                    tc_fence_after();
                    float x[NG];
                    tmem_ld16(tmem + lane_addr + C::S_COL + (k & 1) * NG, x);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(bar(BR::SEMPTY + (k & 1)));
                    const int rg = t * kTileRows + row;
#pragma unroll
                    for (int n = 0; n < NG; ++n) x[n] = (rg < vis[n]) ? x[n] * p.scale_log2 : -INFINITY;
                    // column maximum of this tile: across lanes, then across the 4 warps
                    const float wmax = warp_colreduce16<true>(x, lane);
                    float *rb = red + (k & 1) * 64;
                    if ((lane & 1) == 0) rb[quad * 16 + col16(lane)] = wmax;
                    mbar_arrive(bar(BR::RED));
                    ok = wait_phase(bar(BR::RED), k & 1, abort_flag, status);
                    if (!ok) break;
                    float mt[NG];
#pragma unroll
                    for (int n4 = 0; n4 < NG; n4 += 4) {
                        float4 a = *reinterpret_cast<const float4 *>(rb + 0 * 16 + n4);
                        float4 bq = *reinterpret_cast<const float4 *>(rb + 1 * 16 + n4);
                        float4 c = *reinterpret_cast<const float4 *>(rb + 2 * 16 + n4);
                        float4 d = *reinterpret_cast<const float4 *>(rb + 3 * 16 + n4);
                        mt[n4 + 0] = fmaxf(fmaxf(a.x, bq.x), fmaxf(c.x, d.x));
                        mt[n4 + 1] = fmaxf(fmaxf(a.y, bq.y), fmaxf(c.y, d.y));
                        mt[n4 + 2] = fmaxf(fmaxf(a.z, bq.z), fmaxf(c.z, d.z));
                        mt[n4 + 3] = fmaxf(fmaxf(a.w, bq.w), fmaxf(c.w, d.w));
                    }
                    // running maximum: raised on the first tile, or when a column grew by > 2^8
                    float alpha[NG];
                    bool rescale = false;
#pragma unroll
                    for (int n = 0; n < NG; ++n) {
                        alpha[n] = 1.f;
                        if (first) {
                            m[n] = mt[n];
                        } else if (mt[n] > m[n] + kRescaleThreshold) {
                            alpha[n] = fast_exp2(m[n] - mt[n]);
                            m[n] = mt[n];
                            rescale = true;
                        }
                    }
                    float pv[NG];
#pragma unroll
                    for (int n = 0; n < NG; ++n) {
                        const float mu = (m[n] == -INFINITY) ? 0.f : m[n];
                        pv[n] = fast_exp2(x[n] - mu);
                        lpart[n] = lpart[n] * alpha[n] + pv[n];
                    }
                    // P^T row (this thread's KV row) -> shared memory, bf16 hi | lo, MN-major swizzled
                    const int pb = k % C::PB;
                    ok = wait_phase(bar(BR::PEMPTY + pb), ((k / C::PB) & 1) ^ 1, abort_flag, status);
                    if (!ok) break;
                    {
                        uint32_t w[NG];  // [0, NG/2): hi pairs, [NG/2, NG): lo pairs
#pragma unroll
                        for (int n = 0; n < NG; n += 2) {
                            const __nv_bfloat16 h0 = __float2bfloat16_rn(pv[n]);
                            const __nv_bfloat16 h1 = __float2bfloat16_rn(pv[n + 1]);
                            const float l0 = pv[n] - __bfloat162float(h0);
                            const float l1 = pv[n + 1] - __bfloat162float(h1);
                            w[n / 2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                            w[NG / 2 + n / 2] = pack_bf16x2(l0, l1);
                        }
                        uint8_t *prow = smem + C::OFF_P + pb * C::P_BUF + row * C::P_ROW;
                        const uint32_t swz = ((uint32_t)(row * C::P_ROW) >> 7) & C::P_SWZ_MASK;
#pragma unroll
                        for (int j = 0; j < (int)(C::P_ROW / 16); ++j) {
                            uint4 *dst = reinterpret_cast<uint4 *>(prow + (((uint32_t)j ^ swz) << 4));
                            *dst = make_uint4(w[4 * j + 0], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                        }
                    }
                    fence_proxy_async_smem();
                    if (rescale) {
                        // O^T holds step 3 up to tile k-1: wait for it, then scale its columns in TMEM
                        const int kp = k - 1;
                        ok = wait_phase(bar(BR::PEMPTY + (kp % C::PB)), (kp / C::PB) & 1, abort_flag, status);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
#pragma unroll
                            for (int half = 0; half < C::NP / 16; ++half) {
                                float v[16];
                                const uint32_t addr = tmem + lane_addr + C::O_COL + i * C::NP + half * 16;
                                tmem_ld16(addr, v);
                                tmem_wait_ld();
#pragma unroll
                                for (int n = 0; n < 16; ++n) v[n] *= alpha[n];
                                tmem_st16(addr, v);
                            }
                        }
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    mbar_arrive(bar(BR::PFULL + pb));
                }
                if (!ok) break;
                // ---------------------------------------------------- epilogue: step 4
                const int kl = k - 1;
                ok = wait_phase(bar(BR::PEMPTY + (kl % C::PB)), (kl / C::PB) & 1, abort_flag, status);
                if (!ok) break;
                tc_fence_after();
                const float wsum = warp_colreduce16<false>(lpart, lane);
                if ((lane & 1) == 0) redl[quad * 16 + col16(lane)] = wsum;
                mbar_arrive(bar(BR::REDL));
                ok = wait_phase(bar(BR::REDL), seg & 1, abort_flag, status);
                if (!ok) break;
                float inv_l[NG], lse_n[NG];
#pragma unroll
                for (int n = 0; n < NG; ++n) {
                    const float l = redl[n] + redl[16 + n] + redl[32 + n] + redl[48 + n];
                    const bool empty = !(l > 0.f) || m[n] == -INFINITY;
                    inv_l[n] = empty ? 0.f : 1.f / l;
                    lse_n[n] = empty ? -INFINITY : (m[n] + __log2f(l)) * 0.69314718055994531f;
                }
                const int nsplit = seq_info[4 * b + 2];
                const int slot = seq_info[4 * b + 3] + (cta - seq_info[4 * b + 1]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float hi[16], lo[16];
                    tmem_ld16(tmem + lane_addr + C::O_COL + i * C::NP, hi);
                    tmem_ld16(tmem + lane_addr + C::O_COL + i * C::NP + 16, lo);
                    tmem_wait_ld();
                    const int d = i * 128 + row;
#pragma unroll
                    for (int n = 0; n < NG; ++n) {
                        const int ng = grp * NG + n;
                        if (ng >= p.ncols) continue;
                        const float val = (hi[n] + lo[n]) * inv_l[n];
                        if (nsplit == 1) {
                            p.o[((int64_t)b * p.ncols + ng) * kDv + d] = __float2bfloat16_rn(val);
                        } else {
                            p.opart[((int64_t)slot * p.ncols + ng) * kDv + d] = val;
                        }
                    }
                }
                if (quad == 0 && lane < NG) {
                    const int ng = grp * NG + lane;
                    float my = lse_n[0];
#pragma unroll
                    for (int n = 1; n < NG; ++n)
                        if (lane == n) my = lse_n[n];
                    if (ng < p.ncols) {
                        if (nsplit == 1) p.lse[(int64_t)b * p.ncols + ng] = my;
                        else p.lsepart[(int64_t)slot * p.ncols + ng] = my;
                    }
                }
                tc_fence_before();
                ++seg;
            }
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace mla
