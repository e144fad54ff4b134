// The untransposed decode: S = Q K^T with the query columns (heads x tokens) on the MMA's M
// dimension, a row softmax, and O = P V.  This is the form the pages set ETAP against ([TS]
// Problem Statement: with few heads per GPU, M has to be padded up to the tensor core's minimum;
// Methodology: ETAP moves the KV length onto M instead).  It exists to measure that comparison on
// tcgen05 and is built for it, not for speed:
//   - M = the column group padded to 64 (q_len * h <= 64) or 128: the tensor core's M for
//     cta_group::1, so h = 16 pays 4x padding and h = 128 none;
//   - a CTA holds S (M x 128 KV rows, double buffered) and the O accumulator of one latent half
//     (M x 256): the whole 512 TMEM columns, so two CTAs share a work unit, each computing all of
//     S and the softmax and its own 256 latent columns of O;
//   - K tiles stream through a ring of 16 KB chunks for S; the value columns of the CTA's latent
//     half come through the same ring a second time (from L2) for O;
//   - one issuing thread runs S of tile t + 1 before O of tile t, so the softmax of tile t
//     overlaps the next tile's scores;
//   - P as bf16 hi + lo for M = 64 (one bf16 term for the 128-column groups of long sequences),
//     as in the ETAP kernels, so that both forms meet the same error bar.
// Split-KV, the schedules and the partial-output layout are those of the ETAP kernels; the
// combine kernel merges the splits.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "etap_common.cuh"
#include "plan_core.h"
#include "ptx_sm100.cuh"

namespace mla {

// P is stored as bf16 hi + lo (two accumulated MMAs) in the 64-row configuration, as the ETAP
// kernels do for groups of up to 64 columns; the 128-row one serves the 128-column groups, which
// the plan only forms when every sequence is long enough for one bf16 P term.
template <int M_, int NS_, bool SPLIT_>
struct UtCfg {
    static constexpr int M = M_;    // query rows per MMA
    static constexpr int NS = NS_;  // ring slots of 16 KB (128 KV rows x 64 latent columns)
    static constexpr bool SPLIT = SPLIT_;
    static constexpr int P_TERMS = SPLIT ? 2 : 1;
    static constexpr uint32_t CHUNK = 128 * 128;
    static constexpr uint32_t Q_CHUNK = M * 128;  // 64 latent columns of the M query rows
    static constexpr uint32_t P_CHUNK = M * 128;  // 64 KV rows of P for the M query rows
    static constexpr uint32_t OFF_RING = 1024;    // after the control block
    static constexpr uint32_t OFF_Q = OFF_RING + NS * CHUNK;
    static constexpr uint32_t OFF_P = OFF_Q + 9 * Q_CHUNK;  // [term][KV chunk][M rows x 128 B]
    static constexpr uint32_t BYTES = OFF_P + 2 * P_CHUNK * P_TERMS;
    static constexpr uint32_t S_COL = 0;    // TMEM: S double buffer at 0 and 128
    static constexpr uint32_t O_COL = 256;  // TMEM: O of this CTA's 256 latent columns
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(M, 128, 0, 0);  // A = Q, B = K (both K-major)
    static constexpr uint32_t IDESC_O = idesc_bf16_f32(M, 64, 0, 1);   // A = P (K-major), B = V (N-major)
};
using UtCfg64 = UtCfg<64, 7, true>;
using UtCfg128 = UtCfg<128, 3, false>;
constexpr int kUtThreads = 256;
constexpr uint32_t kUtSmemAlloc = (UtCfg64::BYTES > UtCfg128::BYTES ? UtCfg64::BYTES : UtCfg128::BYTES) + 1024;
static_assert(UtCfg64::BYTES + 1024 <= 232448 && UtCfg128::BYTES + 1024 <= 232448, "shared memory plan");

// mbarriers in the control block
struct UtBars {
    static constexpr int FULL = 0, EMPTY = 8, QF = 16, QE = 17, SF = 18, SE = 20, PF = 22, OD = 23, TAIL = 24,
                         FINAL = 25, COUNT = 26;
};
constexpr uint32_t kUtCtlTmem = 512;   // TMEM base address
constexpr uint32_t kUtCtlWait = 528;   // WaitCtl

struct UtMaps {
    CUtensorMap q64;  // Q rows [B * ncols, 576], 64 x 64 boxes
    CUtensorMap kv;   // cache rows [rows, 576], 64 x 64 boxes
};

// Which schedule the untransposed kernel runs on: the pair schedule (128-row units) when the
// query columns fit one 16-column group, else the M = 256 schedule (256-row units, groups of 64
// or 128 columns) with M = the group width.
struct UtSched {
    int ctas, groups, gcols, unit_rows, duo;
    const int32_t *ranges, *tile_off, *seq_info, *cta_seq;
};

// Tiles of 128 KV rows over the work units [fb, fe): the units' tiles in order, skipping tiles
// that start at or past the sequence's end (the second tile of a 256-row unit can).
struct UtWalk {
    SegIter it;
    int b, u0, u, u1, sub, L, row0;
    bool valid, seg_first, seg_last;
    int unit_rows;
    const int32_t *seqlens;
    int64_t l_cap;
    __device__ int len(int bb) const {
        int64_t L_ = seqlens[bb];
        if (L_ > l_cap) L_ = l_cap;
        return L_ < 0 ? 0 : (int)L_;
    }
    __device__ void settle(const int32_t *tile_off) {
        // move to the next tile that starts inside its sequence
        for (;;) {
            if (!valid) return;
            if (u >= u1) {
                valid = it.next(tile_off, b, u0, u1);
                if (!valid) return;
                u = u0;
                sub = 0;
                L = len(b);
                seg_first = true;
                continue;
            }
            row0 = u * unit_rows + 128 * sub;
            if (row0 < L) return;
            ++u;
            sub = 0;
        }
    }
    __device__ void compute_last(const int32_t *tile_off) {
        // the current tile is its segment's last when no later tile of the segment starts before L
        const int next_row = sub + 1 < unit_rows / 128 ? u * unit_rows + 128 * (sub + 1) : (u + 1) * unit_rows;
        seg_last = !(next_row < L && (sub + 1 < unit_rows / 128 ? u < u1 : u + 1 < u1));
    }
    __device__ void init(const int32_t *tile_off, int seq0, int64_t fb, int64_t fe, int unit_rows_,
                         const int32_t *seqlens_, int64_t l_cap_) {
        unit_rows = unit_rows_;
        seqlens = seqlens_;
        l_cap = l_cap_;
        it.init_at(seq0, fb, fe);
        valid = it.next(tile_off, b, u0, u1);
        u = u0;
        sub = 0;
        seg_first = true;
        L = valid ? len(b) : 0;
        settle(tile_off);
        if (valid) compute_last(tile_off);
    }
    __device__ void advance(const int32_t *tile_off) {
        seg_first = false;
        if (sub + 1 < unit_rows / 128) {
            ++sub;
        } else {
            ++u;
            sub = 0;
        }
        const int b_prev = b;
        settle(tile_off);
        if (valid && b != b_prev) seg_first = true;
        if (valid) compute_last(tile_off);
    }
};

template <class C>
__device__ __forceinline__ void ut_body(const UtMaps &tm, const DecodeParams &p, const UtSched &sc, uint8_t *smem,
                                        uint32_t sbase, uint32_t tmem, int hv, int unit, int grp, bool has_work,
                                        volatile WaitCtl *wc, int32_t *status, bool &mma_pending) {
    using BR = UtBars;
    constexpr int M = C::M;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return sbase + 8u * (uint32_t)i; };
    const int64_t fb = has_work ? sc.ranges[2 * unit] : 0, fe = has_work ? sc.ranges[2 * unit + 1] : 0;
    const int seq0 = has_work ? sc.cta_seq[unit] : 0;
    const int64_t l_cap = p.paged ? (int64_t)p.max_blocks * kPage : p.kv_rows;
    if (fb >= fe) return;

    // cache rows of the two 64-row boxes of tile rows [row0, row0 + 128) of sequence b
    auto locate = [&](int b, int row0, int L, int (&y)[2], bool (&loaded)[2]) -> int {
        int valid = L - row0;
        valid = valid < 0 ? 0 : (valid > 128 ? 128 : valid);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            loaded[hh] = valid > 64 * hh;
            y[hh] = 0;
            if (loaded[hh]) {
                if (p.paged) {
                    const int blk = p.block_table[(int64_t)b * p.max_blocks + (row0 >> 6) + hh];
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
        return valid;
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // Ring order: K chunks of tile t, then the value chunks of tile t - 1.
        bool ok = true;
        UtWalk kw, vw;
        kw.init(sc.tile_off, seq0, fb, fe, sc.unit_rows, p.seqlens, l_cap);
        vw = kw;
        uint32_t g = 0;
        int seg = 0, tail_uses = 0;
        bool v_pending = false;
        while (ok && (kw.valid || v_pending)) {
            if (kw.valid) {
                if (kw.seg_first) {
                    if (lane == 0) {
                        if (seg > 0) ok = wait_phase(bar(BR::QE), (seg - 1) & 1, wc, status);
                        if (ok && !p.withhold_q) {
                            mbar_arrive_expect_tx(bar(BR::QF), 9 * C::Q_CHUNK);
                            const int qrow = kw.b * p.ncols + grp * sc.gcols;
                            for (int c = 0; c < 9; ++c)
                                for (int r = 0; r < M; r += 64)
                                    tma_load_2d(sbase + C::OFF_Q + c * C::Q_CHUNK + r * 128, &tm.q64, bar(BR::QF),
                                                64 * c, qrow + r);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    ++seg;
                }
                int y[2];
                bool loaded[2];
                locate(kw.b, kw.row0, kw.L, y, loaded);
                const int nload = (int)loaded[0] + (int)loaded[1];
                for (int c = 0; c < 9 && ok; ++c, ++g) {
                    const int s = (int)(g % C::NS);
                    if (lane == 0) {
                        ok = wait_phase(bar(BR::EMPTY + s), ((g / C::NS) & 1) ^ 1, wc, status);
                        if (ok) {
                            // rows past the end, or of a page not loaded, are masked in the softmax
                            mbar_arrive_expect_tx(bar(BR::FULL + s), (uint32_t)nload * (C::CHUNK / 2));
                            for (int hh = 0; hh < 2; ++hh)
                                if (loaded[hh])
                                    tma_load_2d(sbase + C::OFF_RING + s * C::CHUNK + hh * (C::CHUNK / 2), &tm.kv,
                                                bar(BR::FULL + s), 64 * c, y[hh]);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                }
            }
            if (v_pending && ok) {
                // the value columns of this CTA's latent half, rows of tile vw
                int y[2];
                bool loaded[2];
                const int valid = locate(vw.b, vw.row0, vw.L, y, loaded);
                for (int j = 0; j < 4 && ok; ++j, ++g) {
                    const int s = (int)(g % C::NS);
                    const uint32_t dst = sbase + C::OFF_RING + s * C::CHUNK;
                    const int x = 256 * hv + 64 * j;
                    if (lane == 0) ok = wait_phase(bar(BR::EMPTY + s), ((g / C::NS) & 1) ^ 1, wc, status);
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) break;
                    if (valid == 128 && loaded[0] && loaded[1]) {
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar(BR::FULL + s), C::CHUNK);
                            for (int hh = 0; hh < 2; ++hh)
                                tma_load_2d(dst + hh * (C::CHUNK / 2), &tm.kv, bar(BR::FULL + s), x, y[hh]);
                        }
                    } else {
                        // a tail: land the valid rows and zero the others, so that P = 0 meets exact zeros
                        const int nload = (int)loaded[0] + (int)loaded[1];
                        if (nload > 0) {
                            if (lane == 0) {
                                mbar_arrive_expect_tx(bar(BR::TAIL), (uint32_t)nload * (C::CHUNK / 2));
                                for (int hh = 0; hh < 2; ++hh)
                                    if (loaded[hh])
                                        tma_load_2d(dst + hh * (C::CHUNK / 2), &tm.kv, bar(BR::TAIL), x, y[hh]);
                                ok = wait_phase(bar(BR::TAIL), tail_uses & 1, wc, status);
                            }
                            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                            ++tail_uses;
                            if (!ok) break;
                        }
                        for (int idx = lane; idx < 128 * 8; idx += 32) {
                            const int r = idx >> 3, c16 = idx & 7;
                            if (r < valid && loaded[r >> 6]) continue;
                            *reinterpret_cast<uint4 *>(smem + C::OFF_RING + s * C::CHUNK + r * 128 + c16 * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(BR::FULL + s));
                    }
                }
                vw.advance(sc.tile_off);
            }
            v_pending = kw.valid;
            if (kw.valid) kw.advance(sc.tile_off);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            bool ok = true;
            UtWalk kw, vw;
            kw.init(sc.tile_off, seq0, fb, fe, sc.unit_rows, p.seqlens, l_cap);
            vw = kw;
            const uint64_t q_desc0 = smem_desc(sbase + C::OFF_Q, 16, 1024, kSwizzle128B);
            const uint64_t r_desc0 = smem_desc(sbase + C::OFF_RING, 16, 1024, kSwizzle128B);
            const uint64_t v_desc0 = smem_desc(sbase + C::OFF_RING, C::CHUNK, 1024, kSwizzle128B);
            const uint64_t p_desc0 = smem_desc(sbase + C::OFF_P, 16, 1024, kSwizzle128B);
            uint32_t g = 0;
            int t = 0, seg = 0;
            bool v_pending = false;
            bool v_first = false;
            while (ok && (kw.valid || v_pending)) {
                if (kw.valid) {
                    if (kw.seg_first) {
                        ok = wait_phase(bar(BR::QF), seg & 1, wc, status);
                        ++seg;
                    }
                    // S buffer t & 1 is free once the softmax read tile t - 2 from it
                    ok = ok && wait_phase(bar(BR::SE + (t & 1)), ((t >> 1) & 1) ^ 1, wc, status);
                    tc_fence_after();
                    const uint32_t d_s = tmem + C::S_COL + (uint32_t)(t & 1) * 128;
                    for (int c = 0; c < 9 && ok; ++c, ++g) {
                        const int s = (int)(g % C::NS);
                        ok = wait_phase(bar(BR::FULL + s), (g / C::NS) & 1, wc, status);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t a = q_desc0 + ((uint32_t)(c * C::Q_CHUNK + 32 * k) >> 4);
                            const uint64_t bk = r_desc0 + ((uint32_t)(s * C::CHUNK + 32 * k) >> 4);
                            umma_bf16(d_s, a, bk, C::IDESC_S, (c == 0 && k == 0) ? 0u : 1u);
                        }
                        umma_commit(bar(BR::EMPTY + s));
                    }
                    if (!ok) break;
                    umma_commit(bar(BR::SF + (t & 1)));
                    if (kw.seg_last) umma_commit(bar(BR::QE));
                }
                if (v_pending && ok) {
                    // O of tile t - 1 once its P is written
                    ok = wait_phase(bar(BR::PF), (t - 1) & 1, wc, status);
                    tc_fence_after();
                    for (int j = 0; j < 4 && ok; ++j, ++g) {
                        const int s = (int)(g % C::NS);
                        ok = wait_phase(bar(BR::FULL + s), (g / C::NS) & 1, wc, status);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t d_o = tmem + C::O_COL + 64u * (uint32_t)j;
#pragma unroll
                        for (int term = 0; term < C::P_TERMS; ++term) {
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                // A = P (term): K = 16 KV rows (chunk k / 4, 32 B steps inside it)
                                const uint64_t a = p_desc0 + ((uint32_t)(term * 2 * C::P_CHUNK + (k >> 2) * C::P_CHUNK +
                                                                         32 * (k & 3)) >> 4);
                                // B = V: K = 16 KV rows of the slot, N = 64 latent columns
                                const uint64_t bv = v_desc0 + ((uint32_t)(s * C::CHUNK + 2048 * k) >> 4);
                                umma_bf16(d_o, a, bv, C::IDESC_O, (v_first && term == 0 && k == 0) ? 0u : 1u);
                            }
                        }
                        umma_commit(bar(BR::EMPTY + s));
                    }
                    if (!ok) break;
                    umma_commit(bar(BR::OD));
                    vw.advance(sc.tile_off);
                }
                v_pending = kw.valid;
                v_first = kw.valid && kw.seg_first;
                if (kw.valid) {
                    kw.advance(sc.tile_off);
                    ++t;
                }
            }
            mma_pending = true;  // FINAL is committed and drained at the end of the kernel
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- softmax (one thread per query row)
        const int q4 = warp & 3;  // TMEM lane quadrant of this warp
        // row of this thread: M = 128 -> lane 32 q4 + lane; M = 64 -> rows 16 q4 + lane in the low 16 lanes
        const int row = M == 128 ? 32 * q4 + lane : 16 * q4 + lane;
        const bool has_row = M == 128 || lane < 16;
        const uint32_t lane_addr = (uint32_t)(32 * q4) << 16;
        const int32_t *seq_info = sc.seq_info;
        bool ok = true;
        UtWalk w;
        w.init(sc.tile_off, seq0, fb, fe, sc.unit_rows, p.seqlens, l_cap);
        float m_run = -INFINITY, l_run = 0.f;
        int vis = 0;
        int t = 0;
        const int ng = grp * sc.gcols + row;  // query column of this row
        while (ok && w.valid) {
            const int b = w.b;
            if (w.seg_first) {
                m_run = -INFINITY;
                l_run = 0.f;
                vis = 0;
                if (has_row && row < sc.gcols && ng < p.ncols) {
                    const int tok = ng / p.num_heads;
                    vis = p.causal ? (w.L - p.q_len + tok + 1) : w.L;
                    vis = vis < 0 ? 0 : vis;
                }
            }
            ok = wait_phase(bar(BR::SF + (t & 1)), (t >> 1) & 1, wc, status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_addr = tmem + lane_addr + C::S_COL + (uint32_t)(t & 1) * 128;
            // pass 1: the tile maximum of this row (log2 units, masked)
            float tmax = -INFINITY;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float x[32];
                tmem_ld32_wait(s_addr + 32 * cc, x);
#pragma unroll
                for (int n = 0; n < 32; ++n) {
                    const int j = w.row0 + 32 * cc + n;
                    tmax = fmaxf(tmax, j < vis ? x[n] * p.scale_log2 : -INFINITY);
                }
            }
            // lazy running maximum: move it (with headroom) only when a score exceeds it by the threshold
            bool resc = false;
            float alpha = 1.f;
            if (tmax != -INFINITY && (m_run == -INFINITY || tmax > m_run + kRescaleThreshold)) {
                const float mn = tmax + kRescaleHeadroom;
                if (m_run != -INFINITY) {
                    alpha = fast_exp2(m_run - mn);
                    resc = true;
                }
                m_run = mn;
            }
            // O of the previous tile is complete (P buffer free; O consistent for a rescale)
            if (t > 0) ok = wait_phase(bar(BR::OD), (t - 1) & 1, wc, status);
            if (!ok) break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, resc) && !w.seg_first) {
                // rescale this row's O (256 latent columns); rows without a change multiply by 1
#pragma unroll 1
                for (int cc = 0; cc < 16; ++cc) {
                    float v[16];
                    const uint32_t addr = tmem + lane_addr + C::O_COL + 16 * cc;
                    tmem_ld16(addr, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int n = 0; n < 16; ++n) v[n] *= alpha;
                    tmem_st16(addr, v);
                }
                tmem_wait_st();
            }
            l_run *= alpha;
            // pass 2: P = 2^(s - m) as bf16 into the K-major A operand, row sum in fp32
            const float mv = m_run == -INFINITY ? 0.f : m_run;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float x[32];
                tmem_ld32_wait(s_addr + 32 * cc, x);
                uint32_t pk[C::P_TERMS][16];
#pragma unroll
                for (int n = 0; n < 32; n += 2) {
                    const int j = w.row0 + 32 * cc + n;
                    const float p0 = j < vis ? fast_exp2(x[n] * p.scale_log2 - mv) : 0.f;
                    const float p1 = j + 1 < vis ? fast_exp2(x[n + 1] * p.scale_log2 - mv) : 0.f;
                    l_run += p0 + p1;
                    const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
                    pk[0][n / 2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                    if constexpr (C::SPLIT)
                        pk[C::P_TERMS - 1][n / 2] = pack_bf16x2(p0 - __bfloat162float(h0), p1 - __bfloat162float(h1));
                }
                if (has_row) {
                    // KV rows 32 cc .. + 31: chunk cc / 2, 16-byte units 4 (cc & 1) .. + 3, swizzled by row
#pragma unroll
                    for (int term = 0; term < C::P_TERMS; ++term) {
                        uint8_t *prow = smem + C::OFF_P + (2 * term + (cc >> 1)) * C::P_CHUNK + row * 128;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int unit16 = 4 * (cc & 1) + u;
                            *reinterpret_cast<uint4 *>(prow + ((unit16 ^ (row & 7)) << 4)) =
                                make_uint4(pk[term][4 * u], pk[term][4 * u + 1], pk[term][4 * u + 2],
                                           pk[term][4 * u + 3]);
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(BR::PF));
                mbar_arrive(bar(BR::SE + (t & 1)));
            }
            if (w.seg_last) {
                // epilogue: O of the segment's last tile, divided by the row sum
                ok = wait_phase(bar(BR::OD), t & 1, wc, status);
                if (!ok) break;
                tc_fence_after();
                const int nsplit = seq_info[4 * b + 2];
                const int slot = seq_info[4 * b + 3] + (unit - seq_info[4 * b + 1]);
                const bool live = has_row && row < sc.gcols && ng < p.ncols;
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    float v[32];
                    tmem_ld32_wait(tmem + lane_addr + C::O_COL + 32 * cc, v);
                    if (live) {
                        const int d0 = 256 * hv + 32 * cc;
                        if (nsplit == 1) {
                            __nv_bfloat16 *dst = p.o + ((int64_t)b * p.ncols + ng) * kDv + d0;
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                uint4 pk;
                                pk.x = pack_bf16x2(v[8 * u] * inv, v[8 * u + 1] * inv);
                                pk.y = pack_bf16x2(v[8 * u + 2] * inv, v[8 * u + 3] * inv);
                                pk.z = pack_bf16x2(v[8 * u + 4] * inv, v[8 * u + 5] * inv);
                                pk.w = pack_bf16x2(v[8 * u + 6] * inv, v[8 * u + 7] * inv);
                                *reinterpret_cast<uint4 *>(dst + 8 * u) = pk;
                            }
                        } else {
                            float *dst = p.opart + ((int64_t)slot * p.ncols + ng) * kDv + d0;
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                *reinterpret_cast<float4 *>(dst + 4 * u) =
                                    make_float4(v[4 * u] * inv, v[4 * u + 1] * inv, v[4 * u + 2] * inv,
                                                v[4 * u + 3] * inv);
                        }
                    }
                }
                if (live && hv == 0) {
                    const float lse = (l_run > 0.f && m_run != -INFINITY)
                                          ? (m_run + __log2f(l_run)) * 0.69314718055994531f
                                          : -INFINITY;
                    if (nsplit == 1)
                        p.lse[(int64_t)b * p.ncols + ng] = lse;
                    else
                        p.lsepart[(int64_t)slot * p.ncols + ng] = lse;
                }
                tc_fence_before();
            }
            w.advance(sc.tile_off);
            ++t;
        }
        if (!ok) wc->abort = 1;
        __syncwarp();
    }
}

__global__ void __launch_bounds__(kUtThreads, 1)
    untransposed_kernel(const __grid_constant__ UtMaps tm, const __grid_constant__ DecodeParams p, WsLayout lay) {
    using BR = UtBars;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - raw_addr);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int32_t *status = p.ws + kHdrStatus;
    auto bar = [&](int i) -> uint32_t { return sbase + 8u * (uint32_t)i; };
    volatile WaitCtl *wc = reinterpret_cast<volatile WaitCtl *>(smem + kUtCtlWait);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kUtCtlTmem);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 8; ++i) {
            mbar_init(bar(BR::FULL + i), 1);
            mbar_init(bar(BR::EMPTY + i), 1);
        }
        mbar_init(bar(BR::QF), 1);
        mbar_init(bar(BR::QE), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BR::SF + i), 1);
            mbar_init(bar(BR::SE + i), 4);  // one arrival per softmax warp
        }
        mbar_init(bar(BR::PF), 4);
        mbar_init(bar(BR::OD), 1);
        mbar_init(bar(BR::TAIL), 1);
        mbar_init(bar(BR::FINAL), 1);
        wc->abort = 0;
        wc->limit_ns = p.wait_limit_ns;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm.q64);
        tma_prefetch_desc(&tm.kv);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // a programmatic dependent of the plan: nothing above read global memory
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // the schedule: the pair schedule for up to 16 query columns, else the M = 256 one
    UtSched sc;
    sc.duo = p.ncols > 16;
    const Sched &s = sc.duo ? lay.duo : lay.pair;
    const int hdr = sc.duo ? kHdrDuo : kHdrPair;
    sc.ctas = p.ws[hdr + kSchCtas];
    sc.groups = p.ws[hdr + kSchGroups];
    sc.gcols = p.ws[hdr + kSchGroupCols];
    sc.unit_rows = sc.duo ? kDuoRows : kTileRows;
    sc.ranges = p.ws + s.cta_ranges / 4;
    sc.tile_off = p.ws + s.tile_off / 4;
    sc.seq_info = p.ws + s.seq_info / 4;
    sc.cta_seq = p.ws + s.cta_seq / 4;
    const int m_rows = sc.gcols <= 64 ? 64 : 128;
    const bool plan_ok = p.ws[kHdrBatch] == p.batch && p.ws[kHdrCols] == p.ncols && sc.ctas >= 1 &&
                         sc.groups >= 1 && sc.gcols >= 1 && sc.gcols <= 128 &&
                         (int64_t)sc.ctas * sc.groups <= (int64_t)(gridDim.x >> 1);
    if (!plan_ok && threadIdx.x == 0) atomicCAS(status, 0, kStatusInvalid);
    if (blockIdx.x == 0 && threadIdx.x == 0) p.ws[kHdrSchedUsed] = sc.duo ? 1 : 0;
    const int cl = (int)(blockIdx.x >> 1);
    const int hv = (int)(blockIdx.x & 1);
    const int unit = plan_ok ? cl / sc.groups : 0;
    const int grp = plan_ok ? cl % sc.groups : 0;
    const bool has_work = plan_ok && unit < sc.ctas;
    bool mma_pending = false;
    if (m_rows == 64)
        ut_body<UtCfg64>(tm, p, sc, smem, sbase, tmem, hv, unit, grp, has_work, wc, status, mma_pending);
    else
        ut_body<UtCfg128>(tm, p, sc, smem, sbase, tmem, hv, unit, grp, has_work, wc, status, mma_pending);
    if (mma_pending) {
        // every MMA issued completes before TMEM is released
        umma_commit(bar(BR::FINAL));
        drain_phase(bar(BR::FINAL), 0);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (wc->abort) {
        // after an abort a bulk copy may still be landing: let it finish before the CTA leaves
        const uint64_t t_q = global_timer_ns();
        while (global_timer_ns() - t_q < 20000ull) {
        }
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace mla
