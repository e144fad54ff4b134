// ETAP decode on a pair of SMs with M = 256 KV rows per tensor-core instruction, sm_100a.
//
// Computation (FlashMLA-ETAP technical summary, "Methodology", ETAP steps 1-4): S^T = K Q^T with
// the KV rows as the UMMA M dimension and the query columns (heads x tokens) as N; P^T = softmax
// of S^T down each column; O^T = V^T P^T; O = (O^T)^T.  The pages keep a producer that streams
// KV into a circular shared-memory buffer and consumers that compute scores and softmax
// statistics block by block ("Integration and Implementation"); this kernel keeps those roles
// and lays the two contractions out for Blackwell's CTA-pair tensor cores:
//
//   * A cluster of two CTAs owns 256-row units of one sequence: CTA r holds rows 128r..128r+127
//     of every unit.  Step 1 is tcgen05.mma.cta_group::2 with M = 256: each CTA supplies its 128
//     K rows (A) and half of the group's query columns (B = Q^T, split by columns, so that a
//     128-column group costs each CTA 72 KB of Q); each CTA's TMEM receives S^T of its own rows
//     for all columns.
//   * Step 3 is also M = 256 across the pair, now over latent rows: CTA r accumulates O^T for
//     latent rows 256r..256r+255 (two M-blocks of 128, paired with the peer's) and supplies, as
//     B, P^T of its half of the columns for all 256 KV rows of the unit.  So each CTA sends the
//     peer P^T of its rows for the peer's columns (st.async, 16 KB per unit) and loads, from L2,
//     the value columns of the peer's rows that its M-blocks need (the scores pass streamed its
//     own rows through a separate ring: nothing is held between the two steps).
//   * The softmax is taken down each column over the rows of both CTAs with one running maximum
//     per column, kept identical in both CTAs: it moves only when some score exceeds it by
//     2^THRESH; the vote travels with the P^T exchange, so the common case needs no extra
//     round trip.  When a vote is raised, both CTAs exchange their tile maxima, rescale their
//     O^T in TMEM and redo the tile's P^T.
//   * Column groups of 64 store P as bf16 hi + lo (N = 128 for step 3: [hi | lo] per CTA);
//     groups of 128 store one bf16 term, used when every sequence of the batch is long enough
//     (the plan decides; see plan_core.h).
//
// Warp roles per CTA (12 warps): 0 loads K tiles and Q (TMA; the bytes of both CTAs count on
// the even CTA's barriers), 1 issues step 1 (even CTA only) and owns TMEM, 2 loads the value
// columns for step 3, 3..10 run the softmax and the epilogue (two warps per TMEM lane quadrant,
// one KV row and half of the columns per thread), 11 issues step 3 in the even CTA (a thread that
// issues MMAs blocks while the tensor pipe drains, so step 1's chunks are not queued behind it) and
// in the odd CTA tells the even one when the even CTA's P^T part has landed here.
// Every wait is bounded; see etap_common.cuh.
#pragma once

#include "etap_common.cuh"

namespace mla {

// Shared-memory control block (identical in both configurations, so that one prologue serves both).
constexpr uint32_t kDuoCtlBar = 0;        // mbarriers
constexpr uint32_t kDuoCtlMisc = 512;     // +0 TMEM address, +16 WaitCtl, +64 received votes (2 x 16 B)
constexpr uint32_t kDuoCtlM = 1024;       // float[128] running maximum per column (log2 units)
constexpr uint32_t kDuoCtlAlpha = 1536;   // float[128] rescale factor of the current tile pair
constexpr uint32_t kDuoCtlRed = 2048;     // float[4][128] per-quadrant partial maxima / sums
constexpr uint32_t kDuoCtlMx = 4096;      // float[128] peer's tile maxima (received)
constexpr uint32_t kDuoCtlLx = 4608;      // float[128] peer's row sums (received)
constexpr uint32_t kDuoCtlMt = 5120;      // float[128] this CTA's tile maxima / row sums
constexpr uint32_t kDuoCtlVis = 5632;     // int[128] visible rows per column of the current sequence
constexpr uint32_t kDuoCtlEnd = 6144;     // data regions start here (1024-aligned)
constexpr int kDuoThreads = 384;

// NC query columns per cluster, P as hi + lo (SPLIT), NS1 K-chunk slots, NS3 value-pair slots.
template <int NC_, bool SPLIT_, int NS1_, int NS3_>
struct DuoCfg {
    static constexpr int NC = NC_;
    static constexpr bool SPLIT = SPLIT_;
    static constexpr int NH = NC / 2;               // columns of Q^T / P^T this CTA holds (its half)
    static constexpr int NP = SPLIT ? 2 * NC : NC;  // UMMA N of step 3
    static constexpr int NPH = NP / 2;              // step-3 B columns per CTA
    static constexpr int NS1 = NS1_, NS3 = NS3_;
    static constexpr uint32_t CHUNK = 16384;        // 128 rows x 64 bf16, 128B swizzle
    static constexpr uint32_t HALF = 8192;          // 64 rows of a chunk: one TMA box
    static constexpr uint32_t VPAIR = 2 * CHUNK;    // 128 rows x 128 latent columns (two chunks)
    static constexpr uint32_t Q_CHUNK = NH * 128;   // NH rows x 64 columns
    static constexpr uint32_t P_PITCH = NPH * 2;    // bytes per KV row of a P^T buffer
    static constexpr uint32_t P_BUF = 128 * P_PITCH;
    static constexpr uint32_t OFF_S1 = kDuoCtlEnd;
    static constexpr uint32_t OFF_S3 = OFF_S1 + NS1 * CHUNK;
    static constexpr uint32_t OFF_Q = OFF_S3 + NS3 * VPAIR;
    static constexpr uint32_t OFF_P = OFF_Q + 9 * Q_CHUNK;  // P^T buffer of K-half 0 (rows of CTA 0), then 1
    static constexpr uint32_t BYTES = OFF_P + 2 * P_BUF;
    static constexpr uint32_t O_COL = 0;                   // 2 M-blocks x NP columns
    static constexpr uint32_t S_COL = 2 * NP;              // 2 buffers x NC columns
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(256, NC, 0, 0);
    static constexpr uint32_t IDESC_O = idesc_bf16_f32(256, NP, 1, 1);
};
using DuoCfg64 = DuoCfg<64, true, 3, 3>;     // 64 columns, P as bf16 hi + lo
using DuoCfg128 = DuoCfg<128, false, 3, 2>;  // 128 columns, one bf16 P term
constexpr uint32_t kDuoSmemAlloc =
    (DuoCfg64::BYTES > DuoCfg128::BYTES ? DuoCfg64::BYTES : DuoCfg128::BYTES) + 1024;  // + alignment slack

template <class C>
constexpr bool duo_cfg_fits() {
    return C::BYTES + 1024 <= 232448 && kDuoCtlVis + 512 <= kDuoCtlEnd && C::S_COL + 2 * C::NC <= 512 && C::P_PITCH == 128 && C::NS1 <= 3 &&
           C::NS3 <= 3 && C::OFF_Q % 1024 == 0 && C::OFF_P % 1024 == 0 && C::NC <= 128 && C::NH % 16 == 0;
}
static_assert(duo_cfg_fits<DuoCfg64>() && duo_cfg_fits<DuoCfg128>(), "shared memory / TMEM plan");

// Barrier indices (the same in both configurations; slot barriers sized for 3 slots).  Barriers
// that gather both CTAs (S1F, S3F, QF, SE, PF0, PF1) are used in the even CTA only.  Step 3 runs in
// two K-halves: K-half h reads the P^T buffers that CTA h's softmax fills (its own columns in place,
// the peer's columns through st.async), so PF_h / PE_h track them separately and CTA h refills
// them as soon as the previous unit's K-half h is done.
struct DuoBars {
    static constexpr int S1F = 0, S1E = 3, S3F = 6, S3E = 9, QF = 12, QE = 13, SF = 14, SE = 16, PF0 = 18, PF1 = 19,
                         PE0 = 20, PE1 = 21, XF = 22, XV = 23, XM = 24, XL = 25, TAIL = 26, FINAL = 27, FINAL3 = 28,
                         COUNT = 29;
};
static_assert(DuoBars::COUNT * 8 <= kDuoCtlMisc, "barrier area");

struct DuoMaps {
    CUtensorMap q32, q64, kv;  // Q with 32- and 64-row boxes; the latent cache with 64 x 64 boxes
};

// Trace events (mla_decode_fwd_trace): role 0 K-tile producer, 1 step-1 issuer, 2 value producer,
// 3 softmax (its first thread), 4 step-3 issuer.
enum : int {
    kEvKChunk = 1,      // a K chunk's slot is free and its loads are issued (index: chunk count)
    kEvQ = 2,           // a segment's Q loads are issued
    kEvS1Begin = 10,    // step 1 of a unit may start (S^T buffer free, Q landed)
    kEvS1Chunk = 11,    // step-1 MMAs of one chunk issued (index: chunk 0..8)
    kEvS1Done = 12,     // step 1 of a unit committed (index: unit count)
    kEvPReady = 13,     // both CTAs' P^T of a unit observed
    kEvS3Pair = 14,     // step-3 MMAs of one value pair issued (index 0..3)
    kEvS3Done = 15,     // step 3 of a unit committed
    kEvVPair = 20,      // a value pair's slot is free and its loads are issued (index: pair count)
    kEvSmS = 30,        // softmax: S^T of a unit observed
    kEvSmVote = 31,     // softmax: vote taken
    kEvSmPe = 32,       // softmax: previous unit's step 3 observed complete
    kEvSmX = 33,        // softmax: exchange round complete
    kEvSmSlow = 34,     // softmax: the slow path begins
    kEvSmDone = 35,     // softmax: P^T ready and S^T released
    kEvSmEpi = 36,      // softmax: epilogue begins
    kEvSmEpiDone = 37,  // softmax: epilogue ends
    kEvEpiS3 = 38,      // epilogue: the segment's last step 3 observed complete
    kEvEpiL = 39,       // epilogue: column sums of both CTAs known
    kEvEpiO = 40        // epilogue: outputs (or partials) stored
};

template <class C, bool TR>
__device__ __forceinline__ void duo_body(const DuoMaps &tm, const DecodeParams &p, uint8_t *smem, uint32_t sbase,
                                         uint32_t tmem, uint32_t rank, int unit, int grp, int groups, bool has_work,
                                         volatile WaitCtl *wc, int32_t *status, bool &pv_pending) {
    using BR = DuoBars;
    constexpr int NC = C::NC, NH = C::NH;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t peer = rank ^ 1u;
    const bool leader = rank == 0;
    auto bar = [&](int i) -> uint32_t { return sbase + kDuoCtlBar + 8u * (uint32_t)i; };
    // the even CTA's barrier i as a cluster address (its own barrier when this is the even CTA)
    auto bar0 = [&](int i) -> uint32_t { return map_to_rank(bar(i), 0); };
    // announce transaction bytes on the even CTA's barrier i
    auto expect0 = [&](int i, uint32_t bytes) {
        if (leader)
            mbar_arrive_expect_tx(bar(i), bytes);
        else
            mbar_arrive_expect_tx_remote(bar0(i), bytes);
    };
    // plain arrival on the even CTA's barrier i, ordering this thread's (and, after a barrier,
    // its CTA's) earlier shared-memory accesses before the even CTA's acquire
    auto arrive0 = [&](int i) {
        if (leader) {
            mbar_arrive(bar(i));
        } else {
            mbar_arrive_remote(bar0(i));
        }
    };
    const int32_t *ranges = p.ws + p.cta_ranges_off;
    const int32_t *tile_off = p.ws + p.tile_off_off;
    const int32_t *seq_info = p.ws + p.seq_info_off;
    const int64_t fb = has_work ? ranges[2 * unit] : 0, fe = has_work ? ranges[2 * unit + 1] : 0;
    const int seq0 = has_work ? p.ws[p.cta_seq_off + unit] : 0;
    const int64_t l_cap = p.paged ? (int64_t)p.max_blocks * kPage : p.kv_rows;
    const CUtensorMap *tm_q = NH == 32 ? &tm.q32 : &tm.q64;

    // Cache rows of the 64-row boxes [row0, row0 + 128) of sequence b: y coordinates, which boxes
    // exist, and how many rows are valid.  A block-table entry outside the pool is not used and
    // raises the status word.
    auto locate = [&](int b, int row0, int L, int (&y)[2], bool (&loaded)[2]) -> int {
        int valid = L - row0;
        valid = valid < 0 ? 0 : (valid > kTileRows ? kTileRows : valid);
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
    auto seq_len = [&](int b) -> int {
        int L = p.seqlens[b];
        if ((int64_t)L > l_cap) {
            if (lane == 0) atomicCAS(status, 0, kStatusInvalid);
            L = (int)l_cap;
        }
        return L < 0 ? 0 : L;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ K tiles and Q (step-1 operands)
        if (lane == 0 && fb < fe) {
            bool ok = true;
            TraceRowT<TR> tr;
            tr.init(p, 0);
            SegIter it;
            it.init_at(seq0, fb, fe);
            int b, t0, t1, seg = 0;
            uint32_t g1 = 0;
            while (ok && it.next(tile_off, b, t0, t1)) {
                const int L = seq_len(b);
                if (seg > 0) ok = poll_phase(bar(BR::QE), (seg - 1) & 1, wc, status);
                if (!ok) break;
                if (!p.withhold_q) {
                    expect0(BR::QF, 9 * C::Q_CHUNK);
                    const int qrow = b * p.ncols + grp * NC + (int)rank * NH;
                    for (int i = 0; i < 9; ++i)
                        tma_load_2d_pair(sbase + C::OFF_Q + i * C::Q_CHUNK, tm_q, bar0(BR::QF), 64 * i, qrow);
                    tr.put(kEvQ, seg);
                }
                for (int tp = t0; tp < t1 && ok; ++tp) {
                    int y[2];
                    bool loaded[2];
                    locate(b, tp * kDuoRows + kTileRows * (int)rank, L, y, loaded);
                    const int nload = (int)loaded[0] + (int)loaded[1];
                    // rows past the end need no zeroing here: their scores are masked to -inf
                    for (int i = 0; i < 9 && ok; ++i, ++g1) {
                        const int s = (int)(g1 % C::NS1);
                        ok = poll_phase(bar(BR::S1E + s), ((g1 / C::NS1) & 1) ^ 1, wc, status);
                        if (!ok) break;
                        expect0(BR::S1F + s, nload * C::HALF);
                        for (int hh = 0; hh < 2; ++hh)
                            if (loaded[hh])
                                tma_load_2d_pair(sbase + C::OFF_S1 + s * C::CHUNK + hh * C::HALF, &tm.kv,
                                                 bar0(BR::S1F + s), 64 * i, y[hh]);
                        tr.put(kEvKChunk, (int)g1);
                    }
                }
                ++seg;
            }
            // Tail: the last releases of the slots and of Q arrive by multicast commit; wait for them
            // so that nothing lands in this CTA's shared memory after it leaves.
            for (uint32_t g = g1; ok && g < g1 + C::NS1; ++g)
                ok = poll_phase(bar(BR::S1E + g % C::NS1), ((g / C::NS1) & 1) ^ 1, wc, status);
            if (ok && seg > 0) ok = poll_phase(bar(BR::QE), (seg - 1) & 1, wc, status);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------------------ value columns (step-3 operands)
        // Unit tp, K-half h (rows 256 tp + 128 h ..), M-block j: this CTA's latent columns
        // 256 rank + 128 j .. + 127 of those rows, as one 32 KB slot of two 64-column chunks.
        if (fb < fe) {
            bool ok = true;
            TraceRowT<TR> tr;
            tr.init(p, 2);
            SegIter it;
            it.init_at(seq0, fb, fe);
            int b, t0, t1, tail_uses = 0;
            uint32_t g3 = 0;
            while (ok && it.next(tile_off, b, t0, t1)) {
                const int L = seq_len(b);
                for (int tp = t0; tp < t1 && ok; ++tp) {
                    for (int v = 0; v < 4 && ok; ++v, ++g3) {
                        const int h = v >> 1, j = v & 1;
                        const int s = (int)(g3 % C::NS3);
                        // lane 0 polls; the warp follows (it zeroes tails together)
                        if (lane == 0) ok = poll_phase(bar(BR::S3E + s), ((g3 / C::NS3) & 1) ^ 1, wc, status);
                        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                        if (!ok) break;
                        int y[2];
                        bool loaded[2];
                        const int valid = locate(b, tp * kDuoRows + kTileRows * h, L, y, loaded);
                        const int x0 = 256 * (int)rank + 128 * j;
                        const uint32_t dst = sbase + C::OFF_S3 + s * C::VPAIR;
                        if (valid == kTileRows && loaded[0] && loaded[1]) {
                            if (lane == 0) {
                                expect0(BR::S3F + s, C::VPAIR);
                                for (int hc = 0; hc < 2; ++hc)
                                    for (int hh = 0; hh < 2; ++hh)
                                        tma_load_2d_pair(dst + hc * C::CHUNK + hh * C::HALF, &tm.kv, bar0(BR::S3F + s),
                                                         x0 + 64 * hc, y[hh]);
                                tr.put(kEvVPair, (int)g3);
                            }
                        } else {
                            // a tail: land the valid rows, zero all others, so that whatever the cache (or
                            // the slot) holds there meets P = 0 as an exact 0
                            const int nload = (int)loaded[0] + (int)loaded[1];
                            if (nload > 0) {
                                if (lane == 0) {
                                    mbar_arrive_expect_tx(bar(BR::TAIL), 2 * nload * C::HALF);
                                    for (int hc = 0; hc < 2; ++hc)
                                        for (int hh = 0; hh < 2; ++hh)
                                            if (loaded[hh])
                                                tma_load_2d(dst + hc * C::CHUNK + hh * C::HALF, &tm.kv, bar(BR::TAIL),
                                                            x0 + 64 * hc, y[hh]);
                                }
                                if (lane == 0) ok = wait_phase(bar(BR::TAIL), tail_uses & 1, wc, status);
                                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                                ++tail_uses;
                                if (!ok) break;
                            }
                            for (int idx = lane; idx < 2 * kTileRows * 8; idx += 32) {
                                const int hc = idx / (kTileRows * 8);
                                const int r = (idx / 8) % kTileRows;
                                const int c16 = idx % 8;
                                if (r < valid && loaded[r >> 6]) continue;
                                *reinterpret_cast<uint4 *>(smem + C::OFF_S3 + s * C::VPAIR + hc * C::CHUNK + r * 128 +
                                                           c16 * 16) = make_uint4(0u, 0u, 0u, 0u);
                            }
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) arrive0(BR::S3F + s);
                        }
                    }
                }
            }
            // Tail: the last slot releases (multicast commits) land before this CTA leaves.
            for (uint32_t g = g3; ok && g < g3 + C::NS3; ++g) {
                if (lane == 0) ok = poll_phase(bar(BR::S3E + g % C::NS3), ((g / C::NS3) & 1) ^ 1, wc, status);
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ step-1 issuer (even CTA)
        // Step 1 of each unit chunk by chunk as its K tiles land in both CTAs.
        if (leader && lane == 0 && fb < fe) {
            const uint64_t q_desc0 = smem_desc(sbase + C::OFF_Q, 16, 1024, kSwizzle128B);
            const uint64_t k_desc0 = smem_desc(sbase + C::OFF_S1, 16, 1024, kSwizzle128B);
            TileCursor qc;
            qc.init(tile_off, seq0, fb, fe);
            int kq = 0, seg_q = 0, qstage = 0;
            uint32_t g1 = 0;
            TraceRowT<TR> tr;
            tr.init(p, 1);
            uint64_t t_last = global_timer_ns();
            while (qc.valid) {
                bool progressed = false;
                const uint32_t d_s = tmem + C::S_COL + (uint32_t)(kq & 1) * NC;
                if (qstage == 0) {
                    bool ready = mbar_test_wait_cluster(bar(BR::SE + (kq & 1)), ((kq >> 1) & 1) ^ 1);
                    if (ready && qc.first()) ready = mbar_test_wait_cluster(bar(BR::QF), seg_q & 1);
                    if (ready) {
                        fence_acquire_cluster_smem();
                        tr.put(kEvS1Begin, kq);
                        qstage = 1;
                        progressed = true;
                    }
                }
                if (qstage >= 1) {
                    const int i = qstage - 1;
                    const int s = (int)(g1 % C::NS1);
                    if (mbar_test_wait_cluster(bar(BR::S1F + s), (g1 / C::NS1) & 1)) {
                        fence_acquire_cluster_smem();
                        tc_fence_after();
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            // A = K tile chunk (K-major, 128 rows per CTA), B = Q^T chunk (K-major, NH per CTA)
                            const uint64_t a = k_desc0 + ((uint32_t)(s * C::CHUNK + 32 * j) >> 4);
                            const uint64_t bq = q_desc0 + ((uint32_t)(i * C::Q_CHUNK + 32 * j) >> 4);
                            umma_bf16_pair(d_s, a, bq, C::IDESC_S, (i == 0 && j == 0) ? 0u : 1u);
                        }
                        umma_commit_pair_both(bar(BR::S1E + s));
                        tr.put(kEvS1Chunk, i);
                        ++g1;
                        progressed = true;
                        if (++qstage > 9) {
                            umma_commit_pair_both(bar(BR::SF + (kq & 1)));
                            tr.put(kEvS1Done, kq);
                            if (qc.last()) {
                                umma_commit_pair_both(bar(BR::QE));
                                ++seg_q;
                            }
                            qc.advance(tile_off);
                            ++kq;
                            qstage = 0;
                        }
                    }
                }
                if (progressed) {
                    t_last = global_timer_ns();
                } else if (wc->abort) {
                    break;
                } else if (global_timer_ns() - t_last > wc->limit_ns) {
                    wc->abort = 1;
                    atomicCAS(status, 0, kStatusTimeout);
                    break;
                }
            }
            // Tail: both CTAs' last releases of the score buffers (the odd CTA's arrive is remote)
            // land before this CTA leaves.
            for (int k = kq; k < kq + 2 && !wc->abort; ++k)
                if (!poll_phase(bar(BR::SE + (k & 1)), ((k >> 1) & 1) ^ 1, wc, status)) break;
            pv_pending = true;  // FINAL is committed (and drained) at the end of the kernel
        }
        __syncwarp();
    } else if (warp == 11) {
        if (leader) {
            // -------------------------------------------------------- step-3 issuer (even CTA)
            // Per unit: K-half 0 once PF0 (both CTAs hold the even CTA's P^T part), value pair by value
            // pair as they land, then PE0; K-half 1 once PF1 and this CTA's XF (the odd CTA's part
            // landed here), then PE1.  Each value slot is freed as its MMAs complete.
            if (lane == 0 && fb < fe) {
                const uint64_t v_desc0 = smem_desc(sbase + C::OFF_S3, C::CHUNK, 1024, kSwizzle128B);
                const uint64_t p_desc0 = smem_desc(sbase + C::OFF_P, C::P_BUF, 1024, kSwizzle128B);
                TileCursor pc;
                pc.init(tile_off, seq0, fb, fe);
                int kp = 0, pstage = 0;
                bool armed = false;
                uint32_t g3 = 0;
                TraceRowT<TR> tr;
                tr.init(p, 4);
                uint64_t t_last = global_timer_ns();
                while (pc.valid) {
                    bool progressed = false;
                    if (!armed) {
                        mbar_arrive_expect_tx(bar(BR::XF), C::P_BUF);  // the odd CTA's part of unit kp
                        armed = true;
                    }
                    if (pstage == 0 && mbar_test_wait_cluster(bar(BR::PF0), kp & 1)) {
                        fence_acquire_cluster_smem();
                        tr.put(kEvPReady, 2 * kp);
                        pstage = 1;
                        progressed = true;
                    } else if (pstage == 3 && mbar_test_wait_cluster(bar(BR::PF1), kp & 1) &&
                               mbar_test_wait_cluster(bar(BR::XF), kp & 1)) {
                        fence_acquire_cluster_smem();
                        fence_proxy_async_smem();  // the st.async writes are read by the tensor core next
                        tr.put(kEvPReady, 2 * kp + 1);
                        pstage = 4;
                        progressed = true;
                    }
                    if (pstage != 0 && pstage != 3) {
                        const int v = pstage <= 2 ? pstage - 1 : pstage - 2;  // value pair 0..3
                        const int h = v >> 1, j = v & 1;
                        const int s = (int)(g3 % C::NS3);
                        if (mbar_test_wait_cluster(bar(BR::S3F + s), (g3 / C::NS3) & 1)) {
                            fence_acquire_cluster_smem();
                            tc_fence_after();
                            const uint32_t d_o = tmem + C::O_COL + (uint32_t)j * C::NP;
                            const bool init = pc.first() && h == 0;
#pragma unroll
                            for (int k8 = 0; k8 < 8; ++k8) {
                                // A = V^T: M = 128 latent rows of this CTA (two chunks), K = 16 KV rows
                                const uint64_t a = v_desc0 + ((uint32_t)(s * C::VPAIR + 2048 * k8) >> 4);
                                // B = P^T of K-half h: K = 16 KV rows, N = this CTA's NPH columns
                                const uint64_t bp = p_desc0 + ((uint32_t)(h * C::P_BUF + 2048 * k8) >> 4);
                                umma_bf16_pair(d_o, a, bp, C::IDESC_O, (init && k8 == 0) ? 0u : 1u);
                            }
                            umma_commit_pair_both(bar(BR::S3E + s));
                            tr.put(kEvS3Pair, v);
                            ++g3;
                            progressed = true;
                            if (v == 1) {
                                umma_commit_pair_both(bar(BR::PE0));
                                pstage = 3;
                            } else if (v == 3) {
                                umma_commit_pair_both(bar(BR::PE1));
                                tr.put(kEvS3Done, kp);
                                pc.advance(tile_off);
                                ++kp;
                                pstage = 0;
                                armed = false;
                            } else {
                                ++pstage;
                            }
                        }
                    }
                    if (progressed) {
                        t_last = global_timer_ns();
                    } else if (wc->abort) {
                        break;
                    } else if (global_timer_ns() - t_last > wc->limit_ns) {
                        wc->abort = 1;
                        atomicCAS(status, 0, kStatusTimeout);
                        break;
                    }
                }
                pv_pending = true;  // FINAL3 is committed (and drained) at the end of the kernel
            }
        } else if (lane == 0 && fb < fe) {
            // -------------------------------------------------------- relay (odd CTA)
            // The even CTA's P^T part of each unit lands here through st.async; once it has, tell the
            // even CTA (its PF0 counts this arrival and its own softmax's).
            TileCursor rc;
            rc.init(tile_off, seq0, fb, fe);
            const uint32_t pf0_remote = map_to_rank(bar(BR::PF0), 0);
            int kr = 0;
            bool ok = true;
            while (rc.valid && ok) {
                mbar_arrive_expect_tx(bar(BR::XF), C::P_BUF);
                if (!mbar_test_wait_cluster(bar(BR::XF), kr & 1)) {
                    const uint64_t t0 = global_timer_ns();
                    for (uint32_t spin = 1;; ++spin) {
                        if (mbar_test_wait_cluster(bar(BR::XF), kr & 1)) break;
                        if ((spin & 255u) == 0) {
                            if (wc->abort || global_timer_ns() - t0 > wc->limit_ns) {
                                if (!wc->abort) atomicCAS(status, 0, kStatusTimeout);
                                wc->abort = 1;
                                ok = false;
                                break;
                            }
                        }
                    }
                }
                if (!ok) break;
                fence_acquire_cluster_smem();
                fence_proxy_async_smem();  // the st.async writes are read by the tensor core next
                mbar_arrive_remote(pf0_remote);
                rc.advance(tile_off);
                ++kr;
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue (warps 3..10)
        constexpr uint32_t SMX = 1, NSM = 256;
        const int sw = warp - 3;
        const int quad = warp & 3;                // TMEM lane quadrant this warp may access
        const int half = sw >> 2;                 // columns [half*NH, half*NH + NH) of the group
        const int row = quad * 32 + lane;         // KV row within this CTA's 128-row tile (= TMEM lane)
        const int tid = sw * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const bool own = half == (int)rank;       // these columns are this CTA's half of step 3's B operand
        float *m_s = reinterpret_cast<float *>(smem + kDuoCtlM);
        float *alpha_s = reinterpret_cast<float *>(smem + kDuoCtlAlpha);
        float *red = reinterpret_cast<float *>(smem + kDuoCtlRed);
        const float *mx = reinterpret_cast<const float *>(smem + kDuoCtlMx);
        const float *lx = reinterpret_cast<const float *>(smem + kDuoCtlLx);
        float *mt = reinterpret_cast<float *>(smem + kDuoCtlMt);
        int *vis_s = reinterpret_cast<int *>(smem + kDuoCtlVis);
        // the peer's vote of unit k lands in slot k & 1 (its vote of unit k + 1 may arrive before this
        // CTA has read that of unit k)
        const volatile uint32_t *vote_in = reinterpret_cast<const volatile uint32_t *>(smem + kDuoCtlMisc + 64);
        // this thread's P^T row goes to K-half `rank` of the CTA that owns its columns
        const uint32_t p_row_local = C::OFF_P + rank * C::P_BUF + (uint32_t)row * C::P_PITCH;
        const uint32_t p_row_remote = map_to_rank(sbase + p_row_local, peer);
        const uint32_t xf_remote = map_to_rank(bar(BR::XF), peer);
        const uint32_t xv_remote = map_to_rank(bar(BR::XV), peer);
        const uint32_t xm_remote = map_to_rank(bar(BR::XM), peer);
        const uint32_t xl_remote = map_to_rank(bar(BR::XL), peer);
        const uint32_t vote_remote = map_to_rank(sbase + kDuoCtlMisc + 64, peer);
        const uint32_t mx_remote = map_to_rank(sbase + kDuoCtlMx, peer);
        const uint32_t lx_remote = map_to_rank(sbase + kDuoCtlLx, peer);
        bool ok = true, stop = false;
        int k = 0, xmr = 0, xlr = 0;
        TraceRowT<TR> tr;
        tr.init(p, 3);
        if (tid != 0) tr.row = nullptr;
        // Scores of 32 columns of this thread's row (block cc of its half), scaled to log2 units
        // and masked; one TMEM round trip.
        auto load_scores = [&](int cc, bool full, int rg, float (&x)[32]) {
            tmem_ld32_wait(tmem + lane_addr + C::S_COL + (uint32_t)(k & 1) * NC + half * NH + 32 * cc, x);
            if (full) {
#pragma unroll
                for (int n = 0; n < 32; ++n) x[n] *= p.scale_log2;
            } else {
                const int4 *v4 = reinterpret_cast<const int4 *>(vis_s + half * NH + 32 * cc);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int4 vv = v4[q];
                    x[4 * q] = rg < vv.x ? x[4 * q] * p.scale_log2 : -INFINITY;
                    x[4 * q + 1] = rg < vv.y ? x[4 * q + 1] * p.scale_log2 : -INFINITY;
                    x[4 * q + 2] = rg < vv.z ? x[4 * q + 2] * p.scale_log2 : -INFINITY;
                    x[4 * q + 3] = rg < vv.w ? x[4 * q + 3] * p.scale_log2 : -INFINITY;
                }
            }
        };
        // P^T of this thread's row for its columns, with the final maxima of the unit: into this
        // CTA's buffer (own columns) or the peer's (st.async, counted on its XF barrier); the
        // probabilities are added to lpart.
        float lpart[NH];
        auto write_p = [&](bool full, int rg) {
#pragma unroll
            for (int cc = 0; cc < NH / 32; ++cc) {
                float x[32];
                load_scores(cc, full, rg, x);
                const float4 *m4 = reinterpret_cast<const float4 *>(m_s + half * NH + 32 * cc);
                // one 16-byte chunk (8 columns) at a time: hi at chunk 4cc+u, lo (split) at NH/8 + that
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float4 mm = m4[2 * u + q];
                        const float mv[4] = {mm.x == -INFINITY ? 0.f : mm.x, mm.y == -INFINITY ? 0.f : mm.y,
                                             mm.z == -INFINITY ? 0.f : mm.z, mm.w == -INFINITY ? 0.f : mm.w};
#pragma unroll
                        for (int e = 0; e < 4; e += 2) {
                            const int n = 8 * u + 4 * q + e;
                            const float p0 = fast_exp2(x[n] - mv[e]);
                            const float p1 = fast_exp2(x[n + 1] - mv[e + 1]);
                            lpart[32 * cc + n] += p0;
                            lpart[32 * cc + n + 1] += p1;
                            const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
                            hi[2 * q + e / 2] =
                                (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                            if constexpr (C::SPLIT)
                                lo[2 * q + e / 2] = pack_bf16x2(p0 - __bfloat162float(h0), p1 - __bfloat162float(h1));
                        }
                    }
#pragma unroll
                    for (int hl = 0; hl < (C::SPLIT ? 2 : 1); ++hl) {
                        const uint32_t *w = hl == 0 ? hi : lo;
                        const uint32_t j16 = (uint32_t)(hl * (NH / 8) + 4 * cc + u);
                        const uint32_t off = (j16 ^ ((uint32_t)row & 7u)) << 4;
                        if (own) {
                            *reinterpret_cast<uint4 *>(smem + p_row_local + off) = make_uint4(w[0], w[1], w[2], w[3]);
                        } else if (ok) {
                            st_async_v4(p_row_remote + off, w[0], w[1], w[2], w[3], xf_remote);
                        }
                    }
                }
            }
        };
        if (fb < fe) {
            SegIter it;
            it.init_at(seq0, fb, fe);
            int b, t0, t1;
            while (!stop && it.next(tile_off, b, t0, t1)) {
                int L = p.seqlens[b];
                if ((int64_t)L > l_cap) L = (int)l_cap;
                if (L < 0) L = 0;
                const int seg_nsplit = seq_info[4 * b + 2];
                const int seg_slot = seq_info[4 * b + 3] + (unit - seq_info[4 * b + 1]);
                int qlen_b = p.q_len;
                if (p.q_lens) {
                    qlen_b = p.q_lens[b];
                    if (qlen_b < 0 || qlen_b > p.q_len) {
                        if (tid == 0) atomicCAS(status, 0, kStatusInvalid);
                        qlen_b = qlen_b < 0 ? 0 : p.q_len;
                    }
                }
                // per-column visible rows and a fresh running maximum (after everyone is done with the
                // previous segment's values)
                named_bar_sync(SMX, NSM);
                if (tid < NC) {
                    const int ng = grp * NC + tid;
                    int vis = 0;
                    if (ng < p.ncols) {
                        const int tok = ng / p.num_heads;
                        vis = tok >= qlen_b ? 0 : (p.causal ? (L - qlen_b + tok + 1) : L);
                        vis = vis < 0 ? 0 : vis;
                    }
                    vis_s[tid] = vis;
                    m_s[tid] = -INFINITY;
                }
                named_bar_sync(SMX, NSM);
#pragma unroll
                for (int n = 0; n < NH; ++n) lpart[n] = 0.f;
                for (int tp = t0; tp < t1 && !stop; ++tp, ++k) {
                    const bool first = tp == t0;
                    ok = ok && spin_phase<false>(bar(BR::SF + (k & 1)), (k >> 1) & 1, wc, status);
                    tc_fence_after();
                    tr.put(kEvSmS, k);
                    const int rg = tp * kDuoRows + kTileRows * (int)rank + row;
                    // every row of this CTA's tile visible to every column: no per-column mask
                    const bool full =
                        qlen_b == p.q_len && tp * kDuoRows + kTileRows * ((int)rank + 1) <= (p.causal ? L - qlen_b + 1 : L) &&
                        grp * NC + NC <= p.ncols;
                    // ---- pass 1: does any score exceed its column's running maximum by > 2^THRESH?
                    bool need = first || !ok;
                    // rolled: one copy of the score read and test (instruction cache; measured faster)
#pragma unroll 1
                    for (int cc = 0; cc < NH / 32; ++cc) {
                        float x[32];
                        load_scores(cc, full, rg, x);
                        const float4 *m4 = reinterpret_cast<const float4 *>(m_s + half * NH + 32 * cc);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 mm = m4[q];
                            need |= (x[4 * q] > mm.x + kRescaleThreshold) | (x[4 * q + 1] > mm.y + kRescaleThreshold) |
                                    (x[4 * q + 2] > mm.z + kRescaleThreshold) | (x[4 * q + 3] > mm.w + kRescaleThreshold);
                        }
                    }
                    const bool vote = named_bar_or(SMX, NSM, need);
                    // ---- votes of both CTAs (a small exchange ahead of P^T, so that P^T is final when written)
                    if (tid == 0) {
                        mbar_arrive_expect_tx(bar(BR::XV), 16);
                        if (ok) st_async_v4(vote_remote + 16u * (uint32_t)(k & 1), vote ? 1u : 0u, (uint32_t)k, 0u, 0u, xv_remote);
                    }
                    ok = ok && spin_phase<true>(bar(BR::XV), k & 1, wc, status);
                    tr.put(kEvSmVote, k);
                    const bool peer_vote = vote_in[4 * (k & 1)] != 0u;
                    // a timed-out wait stops every warp here, before any branch on the peer's vote
                    if (!named_bar_and(SMX, NSM, ok)) {
                        stop = true;
                        break;
                    }
                    if (named_bar_or(SMX, NSM, vote || peer_vote)) {
                        tr.put(kEvSmSlow, k);
                        // ---- slow path, taken by both CTAs together: tile maxima over all 256 rows
#pragma unroll 1
                        for (int cc = 0; cc < NH / 32; ++cc) {
                            float x[32];
                            load_scores(cc, full, rg, x);
#pragma unroll
                            for (int g = 0; g < 2; ++g) {
                                float x16[16];
#pragma unroll
                                for (int n = 0; n < 16; ++n) x16[n] = x[16 * g + n];
                                const float wmax = warp_colreduce16<true>(x16, lane);
                                if ((lane & 1) == 0) red[quad * NC + half * NH + 32 * cc + 16 * g + col16(lane)] = wmax;
                            }
                        }
                        named_bar_sync(SMX, NSM);
                        if (tid == 0) mbar_arrive_expect_tx(bar(BR::XM), 4 * NC);
                        if (tid < NC) {
                            const float v = fmaxf(fmaxf(red[tid], red[NC + tid]), fmaxf(red[2 * NC + tid], red[3 * NC + tid]));
                            mt[tid] = v;
                            if (ok) st_async_b32(mx_remote + 4u * tid, __float_as_uint(v), xm_remote);
                        }
                        ok = ok && spin_phase<true>(bar(BR::XM), xmr & 1, wc, status);
                        ++xmr;
                        bool resc = false;
                        if (tid < NC) {
                            // the same inputs and arithmetic in both CTAs: identical maxima and factors
                            const float mtot = fmaxf(mt[tid], mx[tid]);
                            const float mo = m_s[tid];
                            float a = 1.f;
                            if (mo == -INFINITY) {
                                m_s[tid] = mtot == -INFINITY ? -INFINITY : mtot + kRescaleHeadroom;
                            } else if (mtot > mo + kRescaleThreshold) {
                                const float mn = mtot + kRescaleHeadroom;
                                a = fast_exp2(mo - mn);
                                m_s[tid] = mn;
                                resc = true;
                            }
                            alpha_s[tid] = a;
                        }
                        const bool any_resc = named_bar_or(SMX, NSM, resc);
                        if (any_resc) {
                            // O^T holds step 3 up to the previous unit once both of its K-halves completed;
                            // rescale this thread's lane of both M-blocks for its half's columns
                            if (k > 0) {
                                ok = ok && spin_phase<false>(bar(BR::PE0), (k - 1) & 1, wc, status);
                                ok = ok && spin_phase<false>(bar(BR::PE1), (k - 1) & 1, wc, status);
                            }
                            tc_fence_after();
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
#pragma unroll
                                for (int g = 0; g < 4; ++g) {
                                    float v[16];
                                    const uint32_t addr = tmem + lane_addr + C::O_COL + (uint32_t)j * C::NP + half * 64 + 16 * g;
                                    tmem_ld16(addr, v);
                                    tmem_wait_ld();
#pragma unroll
                                    for (int n = 0; n < 16; ++n) v[n] *= alpha_s[half * NH + ((16 * g + n) % NH)];
                                    tmem_st16(addr, v);
                                }
                            }
                            tmem_wait_st();
#pragma unroll
                            for (int n = 0; n < NH; ++n) lpart[n] *= alpha_s[half * NH + n];
                        }
                    }
                    // ---- P^T of this CTA's rows (K-half `rank`) once step 3 of the previous unit released that
                    // K-half's buffers in both CTAs
                    if (k > 0)
                        ok = ok && spin_phase<false>(bar(rank == 0 ? BR::PE0 : BR::PE1), (k - 1) & 1, wc, status);
                    tc_fence_after();
                    tr.put(kEvSmPe, k);
                    write_p(full, rg);
                    // this CTA's P^T writes are seen by the tensor core's reads; the S^T reads are complete
                    fence_proxy_async_smem();
                    tc_fence_before();
                    if (!named_bar_and(SMX, NSM, ok)) {
                        stop = true;
                        break;
                    }
                    if (tid == 0) {
                        // K-half `rank` is ready on this side (the receiving side reports its part)
                        if (leader)
                            mbar_arrive(bar(BR::PF0));
                        else
                            mbar_arrive_remote(map_to_rank(bar(BR::PF1), 0));
                        arrive0(BR::SE + (k & 1));
                        tr.put(kEvSmDone, k);
                    }
                }
                if (stop) break;
                // ---------------------------------------------------- epilogue for this CTA's 256 latent rows
                const int kl = k - 1;  // the segment's last unit: its step 3 has completed
                tr.put(kEvSmEpi, kl);
                ok = ok && spin_phase<false>(bar(BR::PE0), kl & 1, wc, status);
                ok = ok && spin_phase<false>(bar(BR::PE1), kl & 1, wc, status);
                tc_fence_after();
                tr.put(kEvEpiS3, kl);
#pragma unroll
                for (int ch = 0; ch < NH / 16; ++ch) {
                    float v16[16];
#pragma unroll
                    for (int n = 0; n < 16; ++n) v16[n] = lpart[16 * ch + n];
                    const float wsum = warp_colreduce16<false>(v16, lane);
                    if ((lane & 1) == 0) red[quad * NC + half * NH + 16 * ch + col16(lane)] = wsum;
                }
                named_bar_sync(SMX, NSM);
                if (tid == 0) mbar_arrive_expect_tx(bar(BR::XL), 4 * NC);
                if (tid < NC) {
                    const float v = (red[tid] + red[NC + tid]) + (red[2 * NC + tid] + red[3 * NC + tid]);
                    mt[tid] = v;
                    if (ok) st_async_b32(lx_remote + 4u * tid, __float_as_uint(v), xl_remote);
                }
                ok = ok && spin_phase<true>(bar(BR::XL), xlr & 1, wc, status);
                ++xlr;
                if (!named_bar_and(SMX, NSM, ok)) {  // also orders the mt writes before the reads
                    stop = true;
                    break;
                }
                tr.put(kEvEpiL, kl);
                const int nsplit = seg_nsplit;
                const int slot = seg_slot;
                // column sum over both CTAs, rank 0's part first in both (identical values)
                auto col_l = [&](int c) -> float { return rank == 0 ? mt[c] + lx[c] : lx[c] + mt[c]; };
                // 1 / l per column (0 for a column that saw no row), once, in the idle alpha area
                if (tid < NC) {
                    const float l = col_l(tid);
                    alpha_s[tid] = (!(l > 0.f) || m_s[tid] == -INFINITY) ? 0.f : 1.f / l;
                }
                named_bar_sync(SMX, NSM);
                auto store_o = [&](int c, int j, float val) {
                    const int d = 256 * (int)rank + 128 * j + row;
                    const int ng = grp * NC + c;
                    if (ng >= p.ncols) return;
                    if (nsplit == 1)
                        p.o[((int64_t)b * p.ncols + ng) * kDv + d] = __float2bfloat16_rn(val);
                    else
                        p.opart[((int64_t)slot * p.ncols + ng) * kDv + d] = val;
                };
#pragma unroll 1
                for (int j = 0; j < 2; ++j) {
#pragma unroll 1
                    for (int g = 0; g < NH / 16; ++g) {
                        float hi[16], lo[16];
                        tmem_ld16(tmem + lane_addr + C::O_COL + (uint32_t)j * C::NP + half * 64 + 16 * g, hi);
                        if constexpr (C::SPLIT)
                            tmem_ld16(tmem + lane_addr + C::O_COL + (uint32_t)j * C::NP + half * 64 + NH + 16 * g, lo);
                        tmem_wait_ld();
#pragma unroll
                        for (int n = 0; n < 16; ++n) {
                            const int c = half * NH + 16 * g + n;
                            const float val = C::SPLIT ? hi[n] + lo[n] : hi[n];
                            store_o(c, j, val * alpha_s[c]);
                        }
                    }
                }
                if (rank == 0 && tid < NC) {
                    const int ng = grp * NC + tid;
                    if (ng < p.ncols) {
                        const float l = col_l(tid);
                        const bool empty = !(l > 0.f) || m_s[tid] == -INFINITY;
                        const float lse = empty ? -INFINITY : (m_s[tid] + __log2f(l)) * 0.69314718055994531f;
                        if (nsplit == 1)
                            p.lse[(int64_t)b * p.ncols + ng] = lse;
                        else
                            p.lsepart[((int64_t)rank * p.slots + slot) * p.ncols + ng] = lse;
                    }
                }
                tr.put(kEvEpiO, nsplit);
                if (nsplit >= 2 && p.signal_combine) {
                    // this CTA's partial of the split is stored: count it for the combine kernel
                    // (release: the CTA barrier and one thread's release add cover every thread's
                    // stores)
                    named_bar_sync(SMX, NSM);
                    if (tid == 0) red_add_release_gpu(p.counters + ((int64_t)b * groups + grp) * 2 + rank, 1);
                }
                tr.put(kEvSmEpiDone, kl);
                tc_fence_before();
            }
        }
        if (stop || !ok) wc->abort = 1;
        __syncwarp();
    }
}

template <class C64, class C128, bool TR = false>
__global__ void __launch_bounds__(kDuoThreads, 1)
    etap_duo_kernel(const __grid_constant__ DuoMaps tm, const __grid_constant__ DecodeParams p) {
    using BR = DuoBars;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - raw_addr);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    int32_t *status = p.ws + kHdrStatus;
    auto bar = [&](int i) -> uint32_t { return sbase + kDuoCtlBar + 8u * (uint32_t)i; };
    volatile WaitCtl *wc = reinterpret_cast<volatile WaitCtl *>(smem + kDuoCtlMisc + 16);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kDuoCtlMisc);
    // trace: every CTA's entry, start of work (after the plan), end of work and exit
    unsigned long long *span = trace_span<TR>(p);
    if (span && threadIdx.x == 0) span[0] = global_timer_ns();

    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; ++i) {
            mbar_init(bar(BR::S1F + i), 2);  // both CTAs' producers (expect_tx) + their TMA bytes
            mbar_init(bar(BR::S1E + i), 1);  // the MMA commit
            mbar_init(bar(BR::S3F + i), 2);
            mbar_init(bar(BR::S3E + i), 1);
        }
        mbar_init(bar(BR::QF), 2);
        mbar_init(bar(BR::QE), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BR::SF + i), 1);
            mbar_init(bar(BR::SE + i), 2);  // one arrival per CTA once its softmax warps read S^T
        }
        // K-half 0: the even CTA's softmax (its writes) + the odd CTA's relay (it received the rest);
        // K-half 1: the odd CTA's softmax; the step-3 issuer checks its own XF for the rest
        mbar_init(bar(BR::PF0), 2);
        mbar_init(bar(BR::PF1), 1);
        mbar_init(bar(BR::PE0), 1);
        mbar_init(bar(BR::PE1), 1);
        mbar_init(bar(BR::XF), 1);  // the peer's P^T part: armed by this CTA's step-3 issuer or relay
        mbar_init(bar(BR::XV), 1);  // the peer's vote
        mbar_init(bar(BR::XM), 1);
        mbar_init(bar(BR::XL), 1);
        mbar_init(bar(BR::TAIL), 1);
        mbar_init(bar(BR::FINAL), 1);
        mbar_init(bar(BR::FINAL3), 1);
        wc->abort = 0;
        wc->limit_ns = p.wait_limit_ns;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm.q32);
        tma_prefetch_desc(&tm.q64);
        tma_prefetch_desc(&tm.kv);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(tmem_slot), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers and TMEM exist before any remote operation
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Launched as a programmatic dependent of the plan: nothing above read global memory.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // The schedule must come from a plan for this same shape (uniform in the whole cluster).
    const int mode = p.ws[kHdrDuo + kSchMode];
    const int groups = p.ws[kHdrDuo + kSchGroups];
    const int ctas = p.ws[kHdrDuo + kSchCtas];
    const bool plan_ok = p.ws[kHdrBatch] == p.batch && p.ws[kHdrCols] == p.ncols && (mode == 0 || mode == 1) &&
                         p.ws[kHdrDuo + kSchGroupCols] == duo_group_cols(mode) &&
                         groups == duo_groups(p.ncols, mode) && ctas >= 1 && ctas * groups <= (int)(gridDim.x >> 1);
    if (!plan_ok && threadIdx.x == 0) atomicCAS(status, 0, kStatusInvalid);
    if (blockIdx.x == 0 && threadIdx.x == 0) p.ws[kHdrSchedUsed] = 1;  // the partials follow the duo schedule
    const int cluster = (int)(blockIdx.x >> 1);
    const int unit = plan_ok ? cluster / groups : 0;
    const int grp = plan_ok ? cluster % groups : 0;
    const bool has_work = plan_ok && unit < ctas;
    bool pv_pending = false;
    if (span && threadIdx.x == 0) span[1] = global_timer_ns();
    if (mode == 1)
        duo_body<C128, TR>(tm, p, smem, sbase, tmem, rank, unit, grp, groups, has_work, wc, status, pv_pending);
    else
        duo_body<C64, TR>(tm, p, smem, sbase, tmem, rank, unit, grp, groups, has_work, wc, status, pv_pending);
    if (pv_pending) {
        // every MMA issued completes before TMEM is released (one barrier per issuing thread)
        const int fin = warp == 1 ? BR::FINAL : BR::FINAL3;
        umma_commit_pair_local(bar(fin));
        drain_phase(bar(fin), 0);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (span && threadIdx.x == 0) span[2] = global_timer_ns();
    // No CTA leaves while its peer may still write into its shared memory.  Every operation that
    // targets a CTA's shared memory (TMA bytes, st.async, remote and multicast arrivals) has been
    // waited for by that CTA above (the producers' tails included), so the barrier needs no
    // ordering of its own.
    cluster_sync_relaxed_arrive();
    if (wc->abort) {
        // After an abort a peer's last st.async or bulk copy may not have been waited for: let it
        // land before either CTA leaves (no thread sends after the barrier above).
        const uint64_t t_q = global_timer_ns();
        while (global_timer_ns() - t_q < 20000ull) {
        }
    }
    cluster_sync_relaxed_arrive();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, 512);
    if (span && threadIdx.x == 32) span[3] = global_timer_ns();
}

}  // namespace mla
