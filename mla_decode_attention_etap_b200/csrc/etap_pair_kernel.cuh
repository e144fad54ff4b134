// ETAP decode kernel on a pair of SMs (a 2-CTA cluster), sm_100a.
//
// Computation (FlashMLA-ETAP technical summary, "Methodology", ETAP steps 1-4):
// S^T = K Q^T with the 128 KV rows of a tile as the UMMA M dimension and the
// query columns (heads x tokens) as N; P^T = softmax(S^T) down each column;
// O^T = V^T P^T; O = (O^T)^T.  "Integration and Implementation" describes a
// producer that streams KV from HBM into a circular shared-memory buffer and
// consumers that compute the scores and the softmax statistics block by block;
// this kernel keeps those roles but lays them out for Blackwell:
//
//   * The two CTAs of a cluster split every KV row by latent columns: rank r
//     holds value columns 256r..256r+255 and rope columns 512+32r..512+32r+31.
//     A 128-row tile then needs 72 KB of shared memory per CTA instead of
//     144 KB, so each CTA's ring keeps ~2.5 tiles in flight and
//     the loads of tile k+1 overlap the softmax and the second contraction of
//     tile k.  Each CTA computes a partial S^T over its own columns; the 256
//     softmax threads send their part of it to the peer CTA (st.async into the
//     peer's shared memory, counted on the peer's per-warp mbarriers) and add
//     the peer's part, so both CTAs hold the same S^T (fp32 addition commutes),
//     run the same softmax and each accumulates O^T for its own 256 value columns.
//   * warp 0: TMA producer (Q once per segment, KV tiles into 32 KB slots of
//     two 64-column chunks plus 8 KB slots for the 32 rope columns; tail rows
//     zeroed; L2 prefetch one tile ahead);
//   * warp 1 lane 0: tcgen05.mma issuer, an event loop over the score MMAs of
//     the next tile (in stages, as their operands land);
//   * warps 2..9: two warps per TMEM lane quadrant, one KV row and half of the
//     columns per thread; the column softmax reduces ACROSS threads; P^T goes
//     to shared memory as bf16 hi | lo; one or two softmax threads issue O^T
//     right after the barrier that ends the tile; at the end of a split the
//     last CTA of a sequence merges the split partials (log-sum-exp).
//
// The E4M3-cache configuration (PairCfg16E4) keeps the roles but not the column
// split: see PairCfg.  Every wait is bounded; see etap_common.cuh.
#pragma once

#include "etap_common.cuh"
#include "merge.cuh"

namespace mla {

__host__ __device__ constexpr uint32_t align1024(uint32_t x) { return (x + 1023u) & ~1023u; }
__host__ __device__ constexpr uint32_t pow2_at_least(uint32_t x) {
    return x <= 32 ? 32 : x <= 64 ? 64 : x <= 128 ? 128 : x <= 256 ? 256 : 512;
}

// NG query columns per cluster; NV V slots, NR rope slots, PB P^T buffers per CTA.
//
// KV8: the cache holds E4M3 codes plus one fp32 scale per row, and both contractions run as
// kind::f8f6f4 MMAs (Q and P each split into two E4M3 terms).  A whole 576-code tile then takes
// the shared memory a bf16 half tile takes, so the two CTAs of a cluster do not split tiles by
// columns: each takes every other tile of the pair's range with all 576 columns (no per-tile
// score exchange) and the two partial results of a segment are merged once, at its end,
// through distributed shared memory.
template <int NG_, int NV_, int NR_, int PB_, bool KV8_ = false>
struct PairCfg {
    static constexpr bool KV8 = KV8_;
    static constexpr int NG = NG_;
    static constexpr int NP = 2 * NG;             // UMMA N of step 3: [P_hi | P_lo]
    static constexpr int NS = KV8 ? 2 * NG : NG;  // UMMA N of step 1 (E4M3: [Q_hi | Q_lo] products)
    static constexpr int CH = NG / 16;  // 16-column chunks of softmax and exchange
    static constexpr int NV = NV_, NR = NR_, PB = PB_;
    // V slots of a tile in one CTA: a slot is two 128-row chunks of 128 bytes per row
    // (bf16: 2 x 64 latent columns, a "V pair"; E4M3: 2 x 128, the CTA's whole V half)
    static constexpr int PAIRS = 2;
    static constexpr int MB = KV8 ? 4 : 2;        // M-tiles of O^T (128 latent rows each) per CTA
    static constexpr int TSTEP = KV8 ? 2 : 1;     // tiles of a segment taken by one CTA: every TSTEP-th
    static constexpr int CHUNK_COLS = KV8 ? 128 : 64;
    static constexpr int VCOLS = KV8 ? 512 : 256;  // latent (V) columns of a tile this CTA loads
    static constexpr int XS = CH > 2 ? CH : 2;                         // exchange slots (8 KB each)
    // bf16: the per-tile score exchange slots.  E4M3: none; the segment merge receives 2 M-tiles x
    // 128 rows x NG fp32 plus NG/2 (m, l) pairs per softmax warp into the Q and P^T area, idle by then.
    static constexpr uint32_t X_BYTES = KV8 ? 0 : XS * 128 * 16 * 4;
    static constexpr uint32_t XM_ROW = NG * 4;                          // bytes per row of a merge M-tile
    static constexpr uint32_t XM_TILE = 128 * XM_ROW;
    static constexpr uint32_t XM_BYTES = 2 * XM_TILE + 8 * NG * 4;
    // The softmax warps issue step 3 themselves, right after the barrier that ends the tile, instead
    // of handing P^T to the MMA warp (its polling and the score MMAs it may be issuing would delay
    // it); for 32-column groups and the E4M3 cache two threads share it, one V slot each.
    static constexpr bool PV_BY_SOFTMAX = CH <= 2;
    // threads that issue step 3 (one V slot each when two, so that neither blocks for a whole tile)
    static constexpr int PV_SPLIT = (KV8 || CH == 2) ? 2 : 1;
    static constexpr int PREFETCH = 1;                                 // tiles the L2 prefetch runs ahead of the loads
    static constexpr uint32_t CHUNK = 16384;                           // 128 rows x 128 bytes, 128B swizzle
    static constexpr uint32_t HALF = 8192;                             // 64 rows of a chunk = one TMA box
    static constexpr uint32_t V_SLOT = 2 * CHUNK;
    // bytes of a row's rope codes in this CTA: bf16 32 columns (its half), E4M3 all 64
    static constexpr uint32_t R_ROW = 64;
    static constexpr uint32_t R_DATA = 128 * R_ROW;
    // E4M3: the rope slot also receives the tile's 128 row scales
    static constexpr uint32_t R_SLOT = KV8 ? align1024(R_DATA + 128 * 4) : R_DATA;
    static constexpr uint32_t R_HALF = 64 * R_ROW;                     // 64 rows of it = one TMA box
    static constexpr uint32_t R_SWIZZLE = kSwizzle64B;
    static constexpr int R_KSTEPS = 2;                                 // 32-byte K-steps over the rope
    static constexpr int QROWS = KV8 ? 2 * NG : NG;                    // B operand rows of step 1
    static constexpr int Q_CHUNKS = 4;                                 // 128-byte chunks of the V columns
    static constexpr uint32_t Q_CHUNK = QROWS * 128;
    static constexpr uint32_t Q_ROPE = QROWS * R_ROW;
    static constexpr int PE = KV8 ? 1 : 2;                             // bytes per P^T element
    static constexpr uint32_t P_PITCH = NP * PE < 128 ? NP * PE : 128; // bytes per KV row inside an atom
    static constexpr int AW = P_PITCH / PE;                            // P^T swizzle atom width (columns)
    static constexpr int NA = NP / AW;                                 // atoms along N
    static constexpr uint32_t P_ATOM = 128 * P_PITCH;
    static constexpr uint32_t P_BUF = NA * P_ATOM;
    static constexpr uint32_t P_SWIZZLE = P_PITCH == 128 ? kSwizzle128B : P_PITCH == 64 ? kSwizzle64B : kSwizzle32B;
    static constexpr uint32_t P_SWZ_MASK = P_PITCH == 128 ? 7u : P_PITCH == 64 ? 3u : 1u;
    static constexpr int P_ROWS_MMA = KV8 ? 32 : 16;                   // KV rows (K) per step-3 MMA
    static constexpr uint32_t X_SLOT = 128 * 16 * 4;                   // 128 rows x 16 fp32 partial scores
    static constexpr uint32_t OFF_V = 0;
    static constexpr uint32_t OFF_R = OFF_V + NV * V_SLOT;
    static constexpr uint32_t OFF_Q = OFF_R + NR * R_SLOT;
    static constexpr uint32_t OFF_QR = OFF_Q + Q_CHUNKS * Q_CHUNK;
    static constexpr uint32_t OFF_P = align1024(OFF_QR + Q_ROPE);
    static constexpr uint32_t OFF_X = OFF_P + PB * P_BUF;
    static constexpr uint32_t OFF_XM = KV8 ? OFF_Q : OFF_X;            // E4M3: segment-merge receive area
    // the in-kernel split merge stages (splits + 1) x NG floats: E4M3 in the Q area, else in the P^T buffers
    static constexpr uint32_t OFF_STAGE = KV8 ? OFF_Q : OFF_P;
    static constexpr uint32_t STAGE_BYTES = KV8 ? OFF_P - OFF_Q : PB * P_BUF;
    static constexpr uint32_t OFF_BAR = OFF_X + X_BYTES;
    static constexpr uint32_t OFF_RED = OFF_BAR + 512;                 // float [2][4][NG] column max exchange
    static constexpr uint32_t OFF_REDL = OFF_RED + 32 * NG;               // float [4][NG] column sum exchange
    static constexpr uint32_t OFF_QSC = OFF_REDL + 16 * NG;            // E4M3: float [2][NG] Q column factors
    static constexpr uint32_t OFF_MISC = OFF_QSC + 8 * NG;
    static constexpr uint32_t BYTES = OFF_MISC + 64;
    static constexpr uint32_t SMEM_ALLOC = BYTES + 1024;               // slack for 1024-byte alignment
    static constexpr uint32_t O_COL = 0;                               // MB M-tiles x NP columns
    static constexpr uint32_t S_COL = MB * NP;                         // 2 buffers x NS columns
    static constexpr uint32_t TMEM_COLS = pow2_at_least(MB * NP + 2 * NS);
    static constexpr uint32_t IDESC_QK = KV8 ? idesc_e4m3_f32(128, NS, 0, 0) : idesc_bf16_f32(128, NG, 0, 0);
    static constexpr uint32_t IDESC_PV = KV8 ? idesc_e4m3_f32(128, NP, 1, 1) : idesc_bf16_f32(128, NP, 1, 1);
    static constexpr float THRESH = KV8 ? kRescaleThreshold8 : kRescaleThreshold;
    static constexpr float HEADROOM = KV8 ? kRescaleHeadroom8 : kRescaleHeadroom;
    // The in-kernel split merge stages (splits + 1) x NG floats in the idle P^T buffers.
    static constexpr int MERGE_MAX_SPLITS = (int)(STAGE_BYTES / 4) / NG - 1;
};

using PairCfg16 = PairCfg<16, 5, 2, 2>;  // h*q_len <= 16
using PairCfg32 = PairCfg<32, 5, 1, 1>;  // 16 < h*q_len, in groups of 32 columns
// E4M3 cache, h*q_len <= 16: whole tiles per CTA, 2.5 tiles in flight
using PairCfg16E4 = PairCfg<16, 5, 2, 2, true>;
// E4M3 cache, groups of 32 columns: one P^T buffer (N = 64, 8 KB)
using PairCfg32E4 = PairCfg<32, 5, 2, 1, true>;

template <class C>
constexpr bool pair_cfg_fits() {
    return C::SMEM_ALLOC <= 232448 && C::TMEM_COLS <= 512 && C::OFF_P % 1024 == 0 && C::OFF_QR % 512 == 0 &&
           C::OFF_R % 1024 == 0 && C::R_SLOT % 256 == 0 && C::OFF_Q % 1024 == 0 && (!C::KV8 || C::CH <= 2) &&
           (!C::KV8 || (C::OFF_P + C::PB * C::P_BUF - C::OFF_Q >= C::XM_BYTES &&
                        C::OFF_P == C::OFF_Q + 4 * C::Q_CHUNK + C::Q_ROPE));
}
static_assert(pair_cfg_fits<PairCfg16>() && pair_cfg_fits<PairCfg32>() && pair_cfg_fits<PairCfg16E4>() &&
                  pair_cfg_fits<PairCfg32E4>(),
              "shared memory / TMEM plan");

template <class C>
struct PairBars {
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
    static constexpr int SFIN = FINAL + 1;  // drain of the step-3 MMAs a softmax thread issued
    static constexpr int RED = SFIN + 1;
    static constexpr int REDL = RED + 1;
    // Exchange barriers are per softmax warp: warp w only needs (and only frees) the partial
    // scores of the peer's warp w (same rows, same columns), and one barrier per warp keeps the
    // transaction counts of the 16-byte remote stores off a single shared barrier.
    static constexpr int XFULL = REDL + 1;       // [XS][8]
    static constexpr int XFREE = XFULL + 8 * C::XS;  // [8], used when CH > 1: the peer consumed our last tile
    static constexpr int COUNT = XFREE + 8;
};
static_assert(PairBars<PairCfg16>::COUNT * 8 <= 512 && PairBars<PairCfg32>::COUNT * 8 <= 512 &&
                  PairBars<PairCfg16E4>::COUNT * 8 <= 512 && PairBars<PairCfg32E4>::COUNT * 8 <= 512,
              "barrier area");

// Byte offset of 16-byte chunk j of row r in a row-major buffer of `pitch`-byte
// rows swizzled like the MMA operand (chunk index XOR address bits 7+).
__device__ __forceinline__ uint32_t swz_off(uint32_t r, uint32_t j, uint32_t pitch, uint32_t mask) {
    const uint32_t off = r * pitch;
    return off + ((j ^ ((off >> 7) & mask)) << 4);
}

template <class C, bool TR = false>
__global__ void __launch_bounds__(320, 1)
    etap_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_qr, const __grid_constant__ CUtensorMap tm_kvr,
                     const __grid_constant__ DecodeParams p) {
    using BR = PairBars<C>;
    constexpr int NG = C::NG;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - raw_addr);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const int cluster = blockIdx.x >> 1;
    const int unit = cluster / p.groups;
    const int grp = cluster % p.groups;
    int32_t *status = p.ws + kHdrStatus;

    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
    volatile WaitCtl *wc = reinterpret_cast<volatile WaitCtl *>(smem + C::OFF_MISC + 16);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    // trace: every CTA's entry, start of work (after the plan), end of work and exit
    unsigned long long *span = trace_span<TR>(p);
    if (span && threadIdx.x == 0) span[0] = global_timer_ns();

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NV; ++i) {
            mbar_init(bar(BR::VFULL + i), 1);
            mbar_init(bar(BR::VEMPTY + i), 1);
        }
        for (int i = 0; i < C::NR; ++i) {
            // E4M3: the rope TMA (one arrival) and the 32 producer lanes' row-scale copies; the slot
            // is freed by the 8 softmax warps once they have read the scales
            mbar_init(bar(BR::RFULL + i), C::KV8 ? 33 : 1);
            mbar_init(bar(BR::REMPTY + i), C::KV8 ? 8 : 1);
        }
        // E4M3: the softmax warps write the quantised Q operand themselves
        mbar_init(bar(BR::QFULL), C::KV8 ? 8 : 1);
        mbar_init(bar(BR::QEMPTY), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BR::SFULL + i), 1);
            mbar_init(bar(BR::SEMPTY + i), 8);
        }
        for (int i = 0; i < C::PB; ++i) {
            mbar_init(bar(BR::PFULL + i), 8);
            mbar_init(bar(BR::PEMPTY + i), C::PV_BY_SOFTMAX ? C::PV_SPLIT : 1);
        }
        mbar_init(bar(BR::TAIL), 1);
        mbar_init(bar(BR::FINAL), 1);
        mbar_init(bar(BR::SFIN), C::PV_SPLIT);
        mbar_init(bar(BR::RED), 4);
        mbar_init(bar(BR::REDL), 4);
        for (int i = 0; i < 8 * C::XS; ++i) mbar_init(bar(BR::XFULL + i), 1);
        for (int i = 0; i < 8; ++i) mbar_init(bar(BR::XFREE + i), 1);
        wc->abort = 0;
        wc->limit_ns = p.wait_limit_ns;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        if constexpr (!C::KV8) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_qr);
        }
        tma_prefetch_desc(&tm_kv);
        tma_prefetch_desc(&tm_kvr);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before any remote arrive or st.async
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Step 3 of tile kk: O^T (+)= V^T P^T for the CTA's 256 latent rows (two M-tiles); frees each
    // V slot and then the P^T buffer as the MMAs complete.
    // part: which V slots (all with PV_SPLIT == 1); every issuing part commits PEMPTY once.
    auto issue_pv = [&](int kk, bool first, int part) {
        const int pb = kk % C::PB;
        const uint32_t p_base = sbase + C::OFF_P + pb * C::P_BUF;
        for (int i = part * C::PAIRS / C::PV_SPLIT; i < (part + 1) * C::PAIRS / C::PV_SPLIT; ++i) {
            const int g2 = C::PAIRS * kk + i;
            const int vs = g2 % C::NV;
            const uint32_t v_base = sbase + C::OFF_V + vs * C::V_SLOT;
            if constexpr (C::KV8) {
                // slot i = M-tiles 2i, 2i+1: chunk mt of the slot holds latent columns 256 i + 128 mt..
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
                    for (int s = 0; s < 128 / C::P_ROWS_MMA; ++s) {
                        // A = V^T: M = 128 latent columns (one 128-byte swizzle row), K = 32 KV rows (MN-major)
                        const uint64_t a = smem_desc(v_base + mt * C::CHUNK + 4096u * s, C::CHUNK, 1024, kSwizzle128B);
                        // B = [P_hi | P_lo]^T: K = 32 KV rows, N = NP columns (MN-major)
                        const uint64_t bp = smem_desc(p_base + 32u * C::P_PITCH * s, C::P_ATOM, 8 * C::P_PITCH,
                                                      C::P_SWIZZLE);
                        umma_e4m3(tmem + C::O_COL + (2 * i + mt) * C::NP, a, bp, C::IDESC_PV,
                                  (first && s == 0) ? 0u : 1u);
                    }
                }
            } else {
                const uint32_t d_o = tmem + C::O_COL + i * C::NP;
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    // A = V^T: M = 128 latent columns (two chunks CHUNK apart), K = 16 KV rows (MN-major)
                    const uint64_t a = smem_desc(v_base + 2048u * s, C::CHUNK, 1024, kSwizzle128B);
                    // B = [P_hi | P_lo]^T: K = 16 KV rows, N = NP columns (MN-major)
                    const uint64_t bp =
                        smem_desc(p_base + 16u * C::P_PITCH * s, C::P_ATOM, 8 * C::P_PITCH, C::P_SWIZZLE);
                    umma_bf16(d_o, a, bp, C::IDESC_PV, (first && s == 0) ? 0u : 1u);
                }
            }
            umma_commit(bar(BR::VEMPTY + vs));
        }
        umma_commit(bar(BR::PEMPTY + pb));
    };
    // Launched as a programmatic dependent of the plan: everything above overlapped it; no
    // global memory is read before the preceding grid has completed.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // A programmatic dependent launched next (the next plan) may be scheduled from now on; it
    // waits for this grid to complete before touching memory.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (span && threadIdx.x == 0) span[1] = global_timer_ns();

    // The schedule must come from a plan for this same grid (uniform in the whole cluster).
    const bool plan_ok = p.ws[kHdrPair + kSchCtas] == p.ctas && p.ws[kHdrPair + kSchGroups] == p.groups &&
                         p.ws[kHdrBatch] == p.batch;
    if (blockIdx.x == 0 && threadIdx.x == 0) p.ws[kHdrSchedUsed] = 0;  // the partials follow the pair schedule

    const int32_t *ranges = p.ws + p.cta_ranges_off;
    const int32_t *tile_off = p.ws + p.tile_off_off;
    const int32_t *seq_info = p.ws + p.seq_info_off;
    const int64_t fb = plan_ok ? ranges[2 * unit] : 0, fe = plan_ok ? ranges[2 * unit + 1] : 0;
    const int seq0 = plan_ok ? p.ws[p.cta_seq_off + unit] : 0;  // the sequence holding tile fb
    if (!plan_ok && threadIdx.x == 0) atomicCAS(status, 0, kStatusInvalid);
    const int64_t l_cap = p.paged ? (int64_t)p.max_blocks * kPage : p.kv_rows;
    // first rope column of this CTA (E4M3: all 64 rope columns, every CTA)
    const int rope_x = C::KV8 ? 512 : 512 + 32 * (int)rank;
    const int kv_x0 = C::KV8 ? 0 : 256 * (int)rank;  // first latent column of this CTA
    const int toff = C::KV8 ? (int)rank : 0;        // first tile of a segment this CTA takes

    if (warp == 0) {
        // ------------------------------------------------------------ producer
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
        TraceRowT<TR> trp;  // cluster 0: Q and value-pair loads issued
        trp.init(p, 0);
        if (lane != 0) trp.row = nullptr;
        // L2 prefetch of this CTA's columns of a future tile, so that the load that
        // refills a freed slot hits L2 instead of waiting on HBM.
        auto prefetch_tile = [&](int pb_, int pt_) {
            int Lp = p.seqlens[pb_];
            if ((int64_t)Lp > l_cap) Lp = (int)l_cap;
            const int r0 = pt_ * kTileRows;
            for (int hh = 0; hh < 2; ++hh) {
                if (Lp - r0 <= 64 * hh) break;
                int yp;
                if (p.paged) {
                    const int blk = p.block_table[(int64_t)pb_ * p.max_blocks + (r0 >> 6) + hh];
                    if (blk < 0 || (int64_t)blk * kPage >= p.kv_rows) continue;
                    yp = blk * kPage;
                } else {
                    yp = (int)((int64_t)pb_ * p.kv_rows + r0 + 64 * hh);
                }
                for (int c = 0; c < C::VCOLS / C::CHUNK_COLS; ++c)
                    tma_prefetch_l2_2d(&tm_kv, kv_x0 + C::CHUNK_COLS * c, yp);
                tma_prefetch_l2_2d(&tm_kvr, rope_x, yp);
            }
        };
        TileCursorT<C::TSTEP> ahead;
        if (fb < fe && lane == 0) {
            ahead.init(tile_off, seq0, fb, fe, toff);
            for (int d = 0; d < C::PREFETCH && ahead.valid; ++d) {
                prefetch_tile(ahead.b, ahead.t);
                ahead.advance(tile_off);
            }
        }
        if (fb < fe) {
            SegIter it;
            it.init_at(seq0, fb, fe);
            int b, t0, t1, seg = 0, k = 0;
            while (ok && it.next(tile_off, b, t0, t1)) {
                int L = p.seqlens[b];
                if ((int64_t)L > l_cap) {
                    if (lane == 0) atomicCAS(status, 0, kStatusInvalid);
                    L = (int)l_cap;
                }
                if (L < 0) L = 0;
                if (!C::KV8 && seg > 0) ok = wait_phase(bar(BR::QEMPTY), (seg - 1) & 1, wc, status);
                if (!ok) break;
                if (!C::KV8 && lane == 0 && !p.withhold_q) {
                    mbar_arrive_expect_tx(bar(BR::QFULL), 4 * C::Q_CHUNK + C::Q_ROPE);
                    const int qrow = b * p.ncols + grp * NG;
                    for (int j = 0; j < 4; ++j)
                        tma_load_2d(sbase + C::OFF_Q + j * C::Q_CHUNK, &tm_q, bar(BR::QFULL), (4 * (int)rank + j) * 64,
                                    qrow);
                    tma_load_2d(sbase + C::OFF_QR, &tm_qr, bar(BR::QFULL), rope_x, qrow);
                }
                trp.put(kPairEvQ, seg);
                if (!C::KV8 && !p.withhold_q) ++arms_q;
                for (int t = t0 + toff; t < t1 && ok; t += C::TSTEP, ++k) {
                    if (lane == 0 && ahead.valid) {
                        prefetch_tile(ahead.b, ahead.t);
                        ahead.advance(tile_off);
                    }
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
                    const int nload = (int)loaded[0] + (int)loaded[1];
                    const bool tail = !(loaded[0] && loaded[1] && valid == kTileRows);
                    {
                        // this CTA's 32 rope columns: rows past the end are masked in S^T, no zeroing needed
                        const int rs = k % C::NR;
                        ok = wait_phase(bar(BR::REMPTY + rs), ((k / C::NR) & 1) ^ 1, wc, status);
                        if (!ok) break;
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar(BR::RFULL + rs), nload * C::R_HALF);
                            for (int hh = 0; hh < 2; ++hh)
                                if (loaded[hh])
                                    tma_load_2d(sbase + C::OFF_R + rs * C::R_SLOT + hh * C::R_HALF, &tm_kvr,
                                                bar(BR::RFULL + rs), rope_x, y[hh]);
                        }
                        if constexpr (C::KV8) {
                            // the tile's row scales behind the rope codes: lane l copies rows 4l..4l+3
                            const uint32_t sdst = sbase + C::OFF_R + rs * C::R_SLOT + C::R_DATA;
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int r = 4 * lane + u;
                                if (r < valid && loaded[r >> 6])
                                    cp_async4(sdst + 4u * r, p.kv_scale + (int64_t)y[r >> 6] + (r & 63));
                            }
                            cp_async_mbar_arrive(bar(BR::RFULL + rs));
                        }
                        ++arms_r[rs];
                    }
                    for (int i = 0; i < C::PAIRS && ok; ++i) {
                        const int g2 = C::PAIRS * k + i;
                        const int vs = g2 % C::NV;
                        const int x0 = kv_x0 + C::CHUNK_COLS * 2 * i;  // first latent column of the slot
                        ok = wait_phase(bar(BR::VEMPTY + vs), ((g2 / C::NV) & 1) ^ 1, wc, status);
                        if (!ok) break;
                        const uint32_t dst = sbase + C::OFF_V + vs * C::V_SLOT;
                        if (!tail) {
                            if (lane == 0) {
                                mbar_arrive_expect_tx(bar(BR::VFULL + vs), C::V_SLOT);
                                for (int hc = 0; hc < 2; ++hc)
                                    for (int hh = 0; hh < 2; ++hh)
                                        tma_load_2d(dst + hc * C::CHUNK + hh * C::HALF, &tm_kv, bar(BR::VFULL + vs),
                                                    x0 + C::CHUNK_COLS * hc, y[hh]);
                            }
                            trp.put(kPairEvPair, g2);
                            ++phases_v[vs];
                            tma_v[vs] = true;
                        } else {
                            // tail tile: land the valid rows, zero all others so whatever the cache holds
                            // past L_b (NaN included) meets P = 0 as an exact 0
                            if (nload > 0) {
                                if (lane == 0) {
                                    mbar_arrive_expect_tx(bar(BR::TAIL), 2 * nload * C::HALF);
                                    for (int hc = 0; hc < 2; ++hc)
                                        for (int hh = 0; hh < 2; ++hh)
                                            if (loaded[hh])
                                                tma_load_2d(dst + hc * C::CHUNK + hh * C::HALF, &tm_kv, bar(BR::TAIL),
                                                            x0 + C::CHUNK_COLS * hc, y[hh]);
                                }
                                ok = wait_phase(bar(BR::TAIL), tail_uses & 1, wc, status);
                                ++tail_uses;
                                if (!ok) break;
                            }
                            for (int idx = lane; idx < 2 * kTileRows * 8; idx += 32) {
                                const int hc = idx / (kTileRows * 8);
                                const int r = (idx / 8) % kTileRows;
                                const int c16 = idx % 8;
                                if (r < valid && loaded[r >> 6]) continue;
                                *reinterpret_cast<uint4 *>(smem + C::OFF_V + vs * C::V_SLOT + hc * C::CHUNK + r * 128 +
                                                           c16 * 16) = make_uint4(0u, 0u, 0u, 0u);
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
        // An event loop: step 1 of the next tile goes as soon as its KV and Q are
        // in shared memory, step 3 of the oldest pending tile (unless the softmax
        // warps issue it) as soon as its P^T is; "S^T ready" is committed right
        // after the scores' MMAs, so the softmax of tile k overlaps step 3 of
        // tile k-1 on the tensor pipe.
        if (lane == 0 && fb < fe) {
            TraceRowT<TR> tri;  // cluster 0: score MMAs of a tile issued and committed
            tri.init(p, 1);
            const uint32_t q_base = sbase + C::OFF_Q;
            // one 128-byte chunk of K-major operands: four 32-byte K-steps (16 bf16 or 32 E4M3)
            auto qk_chunk = [&](uint32_t d_s, uint32_t a_base, int qchunk, bool init) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t a = smem_desc(a_base + 32u * j, 16, 1024, kSwizzle128B);
                    const uint64_t bq = smem_desc(q_base + qchunk * C::Q_CHUNK + 32u * j, 16, 1024, kSwizzle128B);
                    if constexpr (C::KV8)
                        umma_e4m3(d_s, a, bq, C::IDESC_QK, (init && j == 0) ? 0u : 1u);
                    else
                        umma_bf16(d_s, a, bq, C::IDESC_QK, (init && j == 0) ? 0u : 1u);
                }
            };
            TileCursorT<C::TSTEP> qc, pc;
            qc.init(tile_off, seq0, fb, fe, toff);
            pc.init(tile_off, seq0, fb, fe, toff);
            int kq = 0, kp = 0, seg_q = 0;
            int qstage = 0;  // scores of tile kq: 0 = rope columns next, 1 + i = V pair i next
            uint64_t t_last = global_timer_ns();
            while (C::PV_BY_SOFTMAX ? qc.valid : pc.valid) {
                bool progressed = false;
                // step 3 first when its P^T is ready: it frees V slots for later tiles
                if constexpr (!C::PV_BY_SOFTMAX) {
                    if (kp < kq && mbar_test_wait(bar(BR::PFULL + kp % C::PB), (kp / C::PB) & 1)) {
                        tc_fence_after();
                        issue_pv(kp, pc.first(), 0);
                        pc.advance(tile_off);
                        ++kp;
                        progressed = true;
                    }
                }
                // step 1 in stages, each as soon as its operands have landed
                if (qc.valid) {
                    const uint32_t d_s = tmem + C::S_COL + (kq & 1) * C::NS;
                    if (qstage == 0) {
                        const int rs = kq % C::NR;
                        bool ready = mbar_test_wait(bar(BR::SEMPTY + (kq & 1)), ((kq >> 1) & 1) ^ 1);
                        if (ready && qc.first()) ready = mbar_test_wait(bar(BR::QFULL), seg_q & 1);
                        if (ready) ready = mbar_test_wait(bar(BR::RFULL + rs), (kq / C::NR) & 1);
                        if (ready) {
                            tc_fence_after();
                            // 32 rope columns (K-major rows of R_ROW bytes): 32-byte K-steps; the first
                            // (re)initialises S^T
#pragma unroll
                            for (int j = 0; j < C::R_KSTEPS; ++j) {
                                const uint64_t a = smem_desc(sbase + C::OFF_R + rs * C::R_SLOT + 32u * j, 16,
                                                             8 * C::R_ROW, C::R_SWIZZLE);
                                const uint64_t bq =
                                    smem_desc(sbase + C::OFF_QR + 32u * j, 16, 8 * C::R_ROW, C::R_SWIZZLE);
                                if constexpr (C::KV8)
                                    umma_e4m3(d_s, a, bq, C::IDESC_QK, j == 0 ? 0u : 1u);
                                else
                                    umma_bf16(d_s, a, bq, C::IDESC_QK, j == 0 ? 0u : 1u);
                            }
                            // E4M3: the softmax warps free the slot after reading its row scales
                            if constexpr (!C::KV8) umma_commit(bar(BR::REMPTY + rs));
                            qstage = 1;
                            progressed = true;
                        }
                    }
                    if (qstage >= 1) {
                        const int i = qstage - 1;
                        const int g2 = C::PAIRS * kq + i;
                        if (mbar_test_wait(bar(BR::VFULL + g2 % C::NV), (g2 / C::NV) & 1)) {
                            tc_fence_after();
                            const uint32_t slot = sbase + C::OFF_V + (g2 % C::NV) * C::V_SLOT;
                            qk_chunk(d_s, slot, 2 * i, false);
                            qk_chunk(d_s, slot + C::CHUNK, 2 * i + 1, false);
                            progressed = true;
                            if (++qstage > C::PAIRS) {
                                umma_commit(bar(BR::SFULL + (kq & 1)));
                                tri.put(kPairEvScores, kq);
                                if (qc.last()) {
                                    umma_commit(bar(BR::QEMPTY));
                                    ++seg_q;
                                }
                                qc.advance(tile_off);
                                ++kq;
                                qstage = 0;
                            }
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
            umma_commit(bar(BR::FINAL));
            drain_phase(bar(BR::FINAL), 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue (warps 2..9)
        // Two warps per TMEM lane quadrant: the thread owning KV row `row` handles 8 of every 16
        // columns (`half` picks which).  The eight warps synchronise through named barrier 1; a
        // failed (timed out) wait only clears this thread's `ok`, and the next bar.red turns that
        // into a uniform stop, so no thread is left waiting at a barrier.
        constexpr uint32_t SMX = 1, NSM = 256;
        constexpr int NH = NG / 2;  // columns of the group this thread handles
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int row = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float *red = reinterpret_cast<float *>(smem + C::OFF_RED);    // [2][4][NG]
        float *redl = reinterpret_cast<float *>(smem + C::OFF_REDL);  // [4][NG]
        const uint32_t x_remote = map_to_rank(sbase + C::OFF_X, peer);
        const int sw = warp - 2;  // softmax warp index: its exchange barriers
        const uint32_t xfull_remote = map_to_rank(bar(BR::XFULL + sw), peer);
        const uint32_t xfree_remote = map_to_rank(bar(BR::XFREE + sw), peer);
        const int k_total = (int)(fe - fb);
        bool ok = true, stop = false, pv_issued = false;
        TraceRowT<TR> tr;  // cluster 0: one softmax thread stamps the tile and epilogue events
        tr.init(p, 3);
        if (warp != 2 || lane != 0) tr.row = nullptr;
        // Exchange slots hold 128 rows x 16 fp32; this thread's 8 values are 16-byte chunks 2*half, 2*half+1.
        auto x_off = [&](int j) -> uint32_t { return swz_off(row, 2 * half + j, 64, 3); };
        // CH > 1: whole-tile exchange, one tile ahead.  Our partial S^T of tile kk goes to the
        // peer's slots 0..CH-1 once the peer has combined tile kk-1 (XFREE).
        auto send_tile = [&](int kk) {
            ok = ok && spin_phase<false>(bar(BR::SFULL + (kk & 1)), (kk >> 1) & 1, wc, status);
            tc_fence_after();
            ok = ok && spin_phase<true>(bar(BR::XFREE + sw), (kk & 1) ^ 1, wc, status);
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) {
                float xs8[8];
                tmem_ld8(tmem + lane_addr + C::S_COL + (kk & 1) * NG + 16 * ch + 8 * half, xs8);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 2 && ok; ++j)
                    st_async_v4(x_remote + ch * C::X_SLOT + x_off(j), __float_as_uint(xs8[4 * j]),
                                __float_as_uint(xs8[4 * j + 1]), __float_as_uint(xs8[4 * j + 2]),
                                __float_as_uint(xs8[4 * j + 3]), xfull_remote);
            }
        };
        if (fb < fe) {
            SegIter it;
            it.init_at(seq0, fb, fe);
            int b, t0, t1, k = 0, seg = 0, e = 0, red_uses = 0;
            int qseg = 0;  // E4M3: segments with a tile for this CTA (Q operands written so far)
            int mseg = 0;  // E4M3: segment merges with the peer so far
            while (!stop && it.next(tile_off, b, t0, t1)) {
                const bool has_tiles = t0 + toff < t1;  // E4M3: the peer may hold the only tile
                int L = p.seqlens[b];
                if ((int64_t)L > l_cap) L = (int)l_cap;
                if (L < 0) L = 0;
                // split bookkeeping of this sequence, read now so that the epilogue does not wait for it
                const int seg_nsplit = seq_info[4 * b + 2];
                const int seg_slot = seq_info[4 * b + 3] + (unit - seq_info[4 * b + 1]);
                // query tokens of this sequence: all q_len, or q_lens[b] of them (ragged batch; the
                // rest are padding columns that see no row)
                int qlen_b = p.q_len;
                if (p.q_lens) {
                    qlen_b = p.q_lens[b];
                    if (qlen_b < 0 || qlen_b > p.q_len) {
                        if (row == 0 && half == 0) atomicCAS(status, 0, kStatusInvalid);
                        qlen_b = qlen_b < 0 ? 0 : p.q_len;
                    }
                }
                float m[NH], lpart[NH];  // index 8*ch + n  <->  column 16*ch + 8*half + n
                // visible rows of this warp's columns (0 for padding and absent columns): lane li holds
                // that of the warp's li-th column (all lanes of a warp handle the same columns)
                static_assert(NH <= 32, "one column per lane");
                int vis_lane = 0;
                if (lane < NH) {
                    const int ng = grp * NG + 16 * (lane >> 3) + 8 * half + (lane & 7);
                    if (ng < p.ncols) {
                        const int tok = ng / p.num_heads;
                        vis_lane = tok >= qlen_b ? 0 : (p.causal ? (L - qlen_b + tok + 1) : L);
                        vis_lane = vis_lane < 0 ? 0 : vis_lane;
                    }
                }
#pragma unroll
                for (int n = 0; n < NH; ++n) {
                    m[n] = -INFINITY;
                    lpart[n] = 0.f;
                }
                float qv[NH];  // E4M3: 2^-c of this thread's columns (their Q codes hold q * 2^c)
                if constexpr (C::KV8) {
                    // ---- step 1's B operand for this segment: E4M3 codes [Q_hi ; Q_lo] of all 576 columns,
                    //      query column n scaled by 2^c_n with 128 < max|q_n| 2^c_n <= 256 (Q_lo holds the
                    //      rounding residual of Q_hi, so that Q_hi + Q_lo keeps the 8 bits of bf16)
                    float *qsc = reinterpret_cast<float *>(smem + C::OFF_QSC);  // [NG] 2^c, then [NG] 2^-c
                    const int tid = (warp - 2) * 32 + lane;
                    if (has_tiles) {
                        if (qseg > 0) ok = ok && spin_phase<false>(bar(BR::QEMPTY), (qseg - 1) & 1, wc, status);
                        {
                            // TPC threads per column (16 or 8), each 2 * WPT of the 576 values
                            constexpr int TPC = NSM / NG, WPT = kDqk / 2 / TPC;
                            const int n = tid / TPC, part = tid % TPC;
                            const int ng = grp * NG + n;
                            float amax = 0.f;
                            if (ng < p.ncols) {
                                const uint32_t *qw =
                                    reinterpret_cast<const uint32_t *>(p.q + ((int64_t)b * p.ncols + ng) * kDqk) +
                                    WPT * part;
#pragma unroll 6
                                for (int i = 0; i < WPT; ++i) {
                                    const uint32_t w2 = __ldg(qw + i);
                                    amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w2 << 16)),
                                                             fabsf(__uint_as_float(w2 & 0xFFFF0000u))));
                                }
                            }
#pragma unroll
                            for (int o = TPC / 2; o >= 1; o >>= 1)
                                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                            int c = 0;
                            if (amax > 0.f && amax < INFINITY) {
                                // c = 8 - ceil(log2 amax), read off the fp32 exponent and mantissa fields
                                const uint32_t bits = __float_as_uint(amax);
                                c = 8 - ((int)(bits >> 23) - 127 + ((bits & 0x7FFFFFu) != 0u ? 1 : 0));
                                c = c < -100 ? -100 : (c > 100 ? 100 : c);
                            }
                            if (part == 0) {
                                qsc[n] = __uint_as_float((uint32_t)(127 + c) << 23);
                                qsc[NG + n] = __uint_as_float((uint32_t)(127 - c) << 23);
                            }
                        }
                        named_bar_sync(SMX, NSM);
                        // 8 columns at a time: hi codes to operand row n, lo codes to row NG + n
                        for (int u = tid; u < NG * 72; u += NSM) {
                            const int n = u / 72, w = u - 72 * n;
                            const int ng = grp * NG + n;
                            uint4 raw = make_uint4(0u, 0u, 0u, 0u);
                            if (ng < p.ncols)
                                raw = __ldg(reinterpret_cast<const uint4 *>(p.q + ((int64_t)b * p.ncols + ng) * kDqk +
                                                                            8 * w));
                            const float sc = qsc[n];
                            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
                            uint32_t hi[2] = {0u, 0u}, lo[2] = {0u, 0u};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float a0 = __uint_as_float(wv[i] << 16) * sc;
                                const float a1 = __uint_as_float(wv[i] & 0xFFFF0000u) * sc;
                                const uint16_t h = f32x2_to_e4m3x2(a0, a1);
                                const float2 hf = e4m3x2_to_f32x2(h);
                                const uint16_t l = f32x2_to_e4m3x2(a0 - hf.x, a1 - hf.y);
                                hi[i >> 1] |= (uint32_t)h << (16 * (i & 1));
                                lo[i >> 1] |= (uint32_t)l << (16 * (i & 1));
                            }
                            uint32_t dh, dl;
                            if (w < 64) {  // latent columns 8w..: chunk w / 16 (128 codes, 128B swizzle)
                                const uint32_t base = C::OFF_Q + (uint32_t)(w >> 4) * C::Q_CHUNK;
                                const uint32_t j16 = (uint32_t)(w & 15) >> 1, sub = (uint32_t)(w & 1) * 8u;
                                dh = base + swz_off(n, j16, 128, 7) + sub;
                                dl = base + swz_off(NG + n, j16, 128, 7) + sub;
                            } else {  // rope columns: 64-byte rows, 64B swizzle
                                const uint32_t w2 = (uint32_t)(w - 64), j16 = w2 >> 1, sub = (w2 & 1u) * 8u;
                                dh = C::OFF_QR + swz_off(n, j16, C::R_ROW, 3) + sub;
                                dl = C::OFF_QR + swz_off(NG + n, j16, C::R_ROW, 3) + sub;
                            }
                            *reinterpret_cast<uint2 *>(smem + dh) = make_uint2(hi[0], hi[1]);
                            *reinterpret_cast<uint2 *>(smem + dl) = make_uint2(lo[0], lo[1]);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0 && !p.withhold_q) mbar_arrive(bar(BR::QFULL));
                        ++qseg;
                    }
#pragma unroll
                    for (int n = 0; n < NH; ++n) qv[n] = qsc[NG + 16 * (n >> 3) + 8 * half + (n & 7)];
                } else {
#pragma unroll
                    for (int n = 0; n < NH; ++n) qv[n] = 1.f;
                }
                for (int t = t0 + toff; t < t1 && !stop; t += C::TSTEP, ++k) {
                    const bool first = (t == t0 + toff);
                    const int pb = k % C::PB;
                    ok = ok && spin_phase<false>(bar(BR::SFULL + (k & 1)), (k >> 1) & 1, wc, status);
                    tc_fence_after();
                    tr.put(kPairEvTile, k);
                    const int rg = t * kTileRows + row;
                    // E4M3: this row's scale s (from the rope slot, which the warps then free); the row's scores
                    // are s * (K codes . Q terms) * 2^-c_n, and the maximum tracks them plus log2 s
                    float rsq[NH], lgs = 0.f, inv16 = 1.f;
                    if constexpr (C::KV8) {
                        const int rsl = k % C::NR;
                        ok = ok && spin_phase<false>(bar(BR::RFULL + rsl), (k / C::NR) & 1, wc, status);
                        float sig = *reinterpret_cast<const float *>(smem + C::OFF_R + rsl * C::R_SLOT + C::R_DATA +
                                                                     4 * row);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(BR::REMPTY + rsl));
                        sig = rg < L ? fmaxf(sig, 0x1p-100f) : 1.f;
                        lgs = __log2f(sig);
                        inv16 = 0.0625f / sig;  // 2^-4 / s: turns a stored p back into 2^(score - m)
                        const float rsc = sig * p.scale_log2;
#pragma unroll
                        for (int n = 0; n < NH; ++n) rsq[n] = rsc * qv[n];
                    } else {
#pragma unroll
                        for (int n = 0; n < NH; ++n) rsq[n] = p.scale_log2;
                    }
                    // every row of the tile visible to every column: no per-column mask needed
                    const bool full_tile =
                        qlen_b == p.q_len && (t + 1) * kTileRows <= (p.causal ? L - qlen_b + 1 : L);
                    bool waited_prev = false, rescale_any = false, sent_next = false;
                    float xc[C::CH][8];  // CH > 1: full scores of this thread's columns, in registers
                    if constexpr (C::KV8) {
                        // scores against Q_hi and against Q_lo, added; each CTA holds whole rows (no exchange)
                        float xl[C::CH][8];
#pragma unroll
                        for (int ch = 0; ch < C::CH; ++ch) {
                            tmem_ld8(tmem + lane_addr + C::S_COL + (k & 1) * C::NS + 16 * ch + 8 * half, xc[ch]);
                            tmem_ld8(tmem + lane_addr + C::S_COL + (k & 1) * C::NS + NG + 16 * ch + 8 * half, xl[ch]);
                        }
                        tmem_wait_ld();
#pragma unroll
                        for (int ch = 0; ch < C::CH; ++ch)
#pragma unroll
                            for (int n = 0; n < 8; ++n) xc[ch][n] += xl[ch][n];
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(BR::SEMPTY + (k & 1)));
                    } else if constexpr (C::CH > 1) {
                        // (a) add the peer's partial S^T of tile k to ours in registers; free the TMEM
                        //     buffer and the peer's slots; (b) send our partial of tile k+1 so it travels
                        //     while tile k's softmax runs.
                        if (k == 0) send_tile(0);
#pragma unroll
                        for (int ch = 0; ch < C::CH; ++ch)
                            tmem_ld8(tmem + lane_addr + C::S_COL + (k & 1) * NG + 16 * ch + 8 * half, xc[ch]);
                        tmem_wait_ld();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(BR::SEMPTY + (k & 1)));
                        if (lane == 0) mbar_arrive_expect_tx(bar(BR::XFULL + sw), C::CH * C::X_SLOT / 8);
                        ok = ok && spin_phase<true>(bar(BR::XFULL + sw), k & 1, wc, status);
#pragma unroll
                        for (int ch = 0; ch < C::CH; ++ch) {
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float4 v =
                                    *reinterpret_cast<const float4 *>(smem + C::OFF_X + ch * C::X_SLOT + x_off(j));
                                xc[ch][4 * j] += v.x;
                                xc[ch][4 * j + 1] += v.y;
                                xc[ch][4 * j + 2] += v.z;
                                xc[ch][4 * j + 3] += v.w;
                            }
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(xfree_remote);
                        // Send now only if S^T of tile k+1 is already there: with few V slots its
                        // scores can depend on step 3 of tile k, i.e. on this tile's softmax.
                        // (one probe per warp, so that the warp-collective TMEM loads and the
                        // lane-0 wait inside send_tile see the same decision in every lane)
                        const bool next_ready =
                            k + 1 < k_total &&
                            __shfl_sync(0xffffffffu,
                                        mbar_test_wait(bar(BR::SFULL + ((k + 1) & 1)), ((k + 1) >> 1) & 1) ? 1 : 0,
                                        0) != 0;
                        if (next_ready) {
                            send_tile(k + 1);
                            sent_next = true;
                        }
                    }
                    // ---- pass 1: full scores of this thread's columns (exchange for CH == 1), scale + mask
                    bool need = first || !ok;
#pragma unroll
                    for (int ch = 0; ch < C::CH; ++ch) {
                        float(&x)[8] = xc[ch];
                        if constexpr (C::CH == 1 && !C::KV8) {
                            tmem_ld8(tmem + lane_addr + C::S_COL + (k & 1) * C::NS + 8 * half, x);
                            tmem_wait_ld();
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar(BR::SEMPTY + (k & 1)));
                        }
                        if constexpr (C::CH == 1 && !C::KV8) {
                            // Exchange of the partial scores with the peer CTA.  Slot xs is free for
                            // exchange e without a handshake: the peer overwrites it (exchange e + XS) only
                            // after receiving our exchange e + XS - 1, which we send after consuming e.
                            static_assert(C::XS >= 2, "slot reuse relies on at least two exchange slots");
                            const int xs = e % C::XS, xu = e / C::XS;
                            ++e;
#pragma unroll
                            for (int j = 0; j < 2 && ok; ++j)
                                st_async_v4(x_remote + xs * C::X_SLOT + x_off(j), __float_as_uint(x[4 * j]),
                                            __float_as_uint(x[4 * j + 1]), __float_as_uint(x[4 * j + 2]),
                                            __float_as_uint(x[4 * j + 3]), xfull_remote + 64u * xs);
                            if (lane == 0) mbar_arrive_expect_tx(bar(BR::XFULL + 8 * xs + sw), C::X_SLOT / 8);
                            ok = ok && spin_phase<true>(bar(BR::XFULL + 8 * xs + sw), xu & 1, wc, status);
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float4 v =
                                    *reinterpret_cast<const float4 *>(smem + C::OFF_X + xs * C::X_SLOT + x_off(j));
                                x[4 * j] += v.x;
                                x[4 * j + 1] += v.y;
                                x[4 * j + 2] += v.z;
                                x[4 * j + 3] += v.w;
                            }
                        }
                        if constexpr (C::KV8) {
                            if (full_tile) {
#pragma unroll
                                for (int n = 0; n < 8; ++n) x[n] = fmaf(x[n], rsq[8 * ch + n], lgs);
                            } else {
#pragma unroll
                                for (int n = 0; n < 8; ++n) {
                                    const int vis = __shfl_sync(0xffffffffu, vis_lane, 8 * ch + n);
                                    x[n] = (rg < vis) ? fmaf(x[n], rsq[8 * ch + n], lgs) : -INFINITY;
                                }
                            }
                        } else if (full_tile) {
#pragma unroll
                            for (int n = 0; n < 8; ++n) x[n] *= p.scale_log2;
                        } else {
#pragma unroll
                            for (int n = 0; n < 8; ++n) {
                                const int vis = __shfl_sync(0xffffffffu, vis_lane, 8 * ch + n);
                                x[n] = (rg < vis) ? x[n] * p.scale_log2 : -INFINITY;
                            }
                        }
                        // running maximum: kept unless some row of the tile exceeds it by > 2^THRESH
#pragma unroll
                        for (int n = 0; n < 8; ++n) need = need || (x[n] > m[8 * ch + n] + C::THRESH);
                    }
                    // ---- one vote per tile; the slow path takes the column maxima of all chunks
                    float alpha[C::CH][8];
                    bool rescale = false;
#pragma unroll
                    for (int ch = 0; ch < C::CH; ++ch)
#pragma unroll
                        for (int n = 0; n < 8; ++n) alpha[ch][n] = 1.f;
                    if (named_bar_or(SMX, NSM, need)) {
                        if (!named_bar_and(SMX, NSM, ok)) {
                            stop = true;
                            break;
                        }
                        float *rb = red + (red_uses & 1) * (4 * NG);  // [4 quadrants][NG columns]
                        ++red_uses;
#pragma unroll
                        for (int ch = 0; ch < C::CH; ++ch) {
                            const float wmax = warp_colreduce8<true>(xc[ch], lane);
                            if ((lane & 3) == 0) rb[quad * NG + 16 * ch + 8 * half + col8(lane)] = wmax;
                        }
                        named_bar_sync(SMX, NSM);
#pragma unroll
                        for (int ch = 0; ch < C::CH; ++ch) {
#pragma unroll
                            for (int n4 = 0; n4 < 8; n4 += 4) {
                                const int c0 = 16 * ch + 8 * half + n4;
                                const float4 a = *reinterpret_cast<const float4 *>(rb + 0 * NG + c0);
                                const float4 bq = *reinterpret_cast<const float4 *>(rb + 1 * NG + c0);
                                const float4 c = *reinterpret_cast<const float4 *>(rb + 2 * NG + c0);
                                const float4 d = *reinterpret_cast<const float4 *>(rb + 3 * NG + c0);
                                const float mt4[4] = {fmaxf(fmaxf(a.x, bq.x), fmaxf(c.x, d.x)),
                                                      fmaxf(fmaxf(a.y, bq.y), fmaxf(c.y, d.y)),
                                                      fmaxf(fmaxf(a.z, bq.z), fmaxf(c.z, d.z)),
                                                      fmaxf(fmaxf(a.w, bq.w), fmaxf(c.w, d.w))};
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const int n = n4 + u, li = 8 * ch + n;
                                    if (first) {
                                        m[li] = mt4[u] + C::HEADROOM;
                                    } else if (mt4[u] > m[li] + C::THRESH) {
                                        alpha[ch][n] = fast_exp2(m[li] - (mt4[u] + C::HEADROOM));
                                        m[li] = mt4[u] + C::HEADROOM;
                                        rescale = true;
                                    }
                                }
                            }
                        }
                    }
                    // ---- pass 2: probabilities, P^T (hi + lo) into shared memory, O^T rescale
#pragma unroll
                    for (int ch = 0; ch < C::CH; ++ch) {
                        float pv[8];
#pragma unroll
                        for (int n = 0; n < 8; ++n) {
                            const int li = 8 * ch + n;
                            const float mu = (m[li] == -INFINITY) ? 0.f : m[li];
                            if constexpr (C::KV8) {
                                // stored p = 2^(score + log2 s - m + 4); the sum takes 2^(score - m)
                                pv[n] = fast_exp2(xc[ch][n] - (mu - kPScaleLog2_8));
                                lpart[li] = fmaf(pv[n], inv16, lpart[li] * alpha[ch][n]);
                            } else {
                                pv[n] = fast_exp2(xc[ch][n] - mu);
                                lpart[li] = lpart[li] * alpha[ch][n] + pv[n];
                            }
                        }
                        // ---- P^T row chunk -> shared memory: bf16 hi into column 16ch+8half.., lo into NG + that
                        if (ch == 0)
                            ok = ok && spin_phase<false>(bar(BR::PEMPTY + pb), ((k / C::PB) & 1) ^ 1, wc, status);
                        if constexpr (C::KV8) {
                            // P^T row chunk: E4M3 hi codes into columns 16ch+8half.., the residual's codes into NG + that
                            uint32_t hi[2] = {0u, 0u}, lo[2] = {0u, 0u};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint16_t h = f32x2_to_e4m3x2(pv[2 * i], pv[2 * i + 1]);
                                const float2 hf = e4m3x2_to_f32x2(h);
                                const uint16_t l = f32x2_to_e4m3x2(pv[2 * i] - hf.x, pv[2 * i + 1] - hf.y);
                                hi[i >> 1] |= (uint32_t)h << (16 * (i & 1));
                                lo[i >> 1] |= (uint32_t)l << (16 * (i & 1));
                            }
                            uint8_t *pbuf = smem + C::OFF_P + pb * C::P_BUF;
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl) {
                                const int col0 = hl * NG + 16 * ch + 8 * half;  // first P^T column (= byte) of these 8
                                *reinterpret_cast<uint2 *>(pbuf + swz_off(row, col0 / 16, C::P_PITCH, C::P_SWZ_MASK) +
                                                           (col0 % 16)) =
                                    hl == 0 ? make_uint2(hi[0], hi[1]) : make_uint2(lo[0], lo[1]);
                            }
                        } else {
                            uint32_t hi[4], lo[4];
#pragma unroll
                            for (int n = 0; n < 8; n += 2) {
                                const __nv_bfloat16 h0 = __float2bfloat16_rn(pv[n]);
                                const __nv_bfloat16 h1 = __float2bfloat16_rn(pv[n + 1]);
                                hi[n / 2] =
                                    (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                                lo[n / 2] = pack_bf16x2(pv[n] - __bfloat162float(h0), pv[n + 1] - __bfloat162float(h1));
                            }
                            uint8_t *pbuf = smem + C::OFF_P + pb * C::P_BUF;
#pragma unroll
                            for (int hl = 0; hl < 2; ++hl) {
                                const uint32_t *w = hl == 0 ? hi : lo;
                                const int col0 = hl * NG + 16 * ch + 8 * half;  // first P^T column of these 8
                                const int atom = col0 / C::AW;
                                const int j0 = (col0 % C::AW) / 8;  // 16-byte chunk within the atom row
                                *reinterpret_cast<uint4 *>(pbuf + atom * C::P_ATOM +
                                                           swz_off(row, j0, C::P_PITCH, C::P_SWZ_MASK)) =
                                    make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                        if (rescale) {
                            // O^T holds step 3 up to tile k-1: wait for it, then scale these columns in TMEM
                            if (!waited_prev) {
                                const int kp = k - 1;
                                ok = ok && spin_phase<false>(bar(BR::PEMPTY + (kp % C::PB)), (kp / C::PB) & 1, wc,
                                                             status);
                                tc_fence_after();
                                waited_prev = true;
                            }
                            rescale_any = true;
#pragma unroll
                            for (int i = 0; i < C::MB; ++i) {
#pragma unroll
                                for (int hl = 0; hl < 2; ++hl) {
                                    float v[8];
                                    const uint32_t addr =
                                        tmem + lane_addr + C::O_COL + i * C::NP + hl * NG + 16 * ch + 8 * half;
                                    tmem_ld8(addr, v);
                                    tmem_wait_ld();
#pragma unroll
                                    for (int n = 0; n < 8; ++n) v[n] *= alpha[ch][n];
                                    tmem_st8(addr, v);
                                }
                            }
                        }
                    }
                    if (stop) break;
                    if (rescale_any) tmem_wait_st();
                    fence_proxy_async_smem();
                    tc_fence_before();
                    if constexpr (C::PV_BY_SOFTMAX) {
                        // every P^T row written and every O^T rescale done: one thread issues step 3
                        named_bar_sync(SMX, NSM);
                        if (lane == 0 && (warp == 2 || (C::PV_SPLIT == 2 && warp == 6))) {
                            tc_fence_after();
                            issue_pv(k, first, warp == 2 ? 0 : 1);
                            pv_issued = true;
                        }
                    } else {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(BR::PFULL + pb));
                    }
                    tr.put(kPairEvTileDone, k);
                    if constexpr (C::CH > 1 && !C::KV8) {
                        if (k + 1 < k_total && !sent_next) send_tile(k + 1);
                    }
                }
                if (stop) break;
                // ---------------------------------------------------- epilogue: step 4 for this CTA's 256 columns
                const int kl = k - 1;
                tr.put(kPairEvEpi, seg);
                if (has_tiles)  // the last step 3 of this segment has completed
                    ok = ok && spin_phase<false>(bar(BR::PEMPTY + (kl % C::PB)), (kl / C::PB) & 1, wc, status);
                tc_fence_after();
                tr.put(kPairEvEpiS3, seg);
#pragma unroll
                for (int ch = 0; ch < C::CH; ++ch) {
                    float v8[8];
#pragma unroll
                    for (int n = 0; n < 8; ++n) v8[n] = lpart[8 * ch + n];
                    const float wsum = warp_colreduce8<false>(v8, lane);
                    if ((lane & 3) == 0) redl[quad * NG + 16 * ch + 8 * half + col8(lane)] = wsum;
                }
                if (!named_bar_and(SMX, NSM, ok)) {  // also orders the redl writes before the reads
                    stop = true;
                    break;
                }
                const int nsplit = seg_nsplit;
                const int slot = seg_slot;
                // this CTA's result for latent row d = 256 rank + 128 i + row of column 16 ch + 8 half + n
                auto store_o = [&](int ch, int i, int n, float val) {
                    const int d = 256 * (int)rank + 128 * i + row;
                    const int ng = grp * NG + 16 * ch + 8 * half + n;
                    if (ng >= p.ncols) return;
                    if (nsplit == 1)
                        p.o[((int64_t)b * p.ncols + ng) * kDv + d] = __float2bfloat16_rn(val);
                    else
                        p.opart[((int64_t)slot * p.ncols + ng) * kDv + d] = val;
                };
                auto store_lse = [&](int ch, const float (&lse_n)[8]) {
                    if (quad == 0 && lane < 8) {
                        const int ng = grp * NG + 16 * ch + 8 * half + lane;
                        float my = lse_n[0];
#pragma unroll
                        for (int n = 1; n < 8; ++n)
                            if (lane == n) my = lse_n[n];
                        if (ng < p.ncols) {
                            if (nsplit == 1) {
                                if (rank == 0) p.lse[(int64_t)b * p.ncols + ng] = my;
                            } else {
                                p.lsepart[((int64_t)rank * p.slots + slot) * p.ncols + ng] = my;
                            }
                        }
                    }
                };
                if constexpr (C::KV8) {
                    // ---- merge of the two CTAs' partials of this segment (disjoint tiles, all 512 latent rows
                    //      each): send the peer the two M-tiles it writes and this CTA's (m, l) of these columns,
                    //      receive the same, and combine by the log-sum-exp rule.
                    float ms[NH], ls[NH], own[2][NH];
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
                        const int cn = 16 * (n >> 3) + 8 * half + (n & 7);
                        ls[n] = redl[cn] + redl[NG + cn] + redl[2 * NG + cn] + redl[3 * NG + cn];
                        ms[n] = has_tiles ? m[n] : -INFINITY;
                    }
                    const uint32_t x_peer = map_to_rank(sbase + C::OFF_XM, peer);
                    const uint32_t xml = 2u * C::XM_TILE + (uint32_t)sw * (2u * NH * 4u);
                    // This CTA's merge area (its Q and P^T buffers) is idle now: every thread has passed
                    // the barrier after the segment's last step 3, whose completion it waited for, and
                    // the score MMAs completed before their last S^T was read.  Tell the peer's warp,
                    // then wait until the peer says the same of its area.
                    if (lane == 0) mbar_arrive_remote(xfree_remote);
                    ok = ok && spin_phase<true>(bar(BR::XFREE + sw), mseg & 1, wc, status);
#pragma unroll
                    for (int ch = 0; ch < C::CH; ++ch) {
                        // O^T of the 4 M-tiles for this thread's row and 8 columns (hi + lo)
                        const uint32_t xcol = (uint32_t)row * C::XM_ROW + (uint32_t)(16 * ch + 8 * half) * 4u;
#pragma unroll
                        for (int mt = 0; mt < 4; ++mt) {
                            float hi[8], lo[8];
                            if (has_tiles) {
                                tmem_ld8(tmem + lane_addr + C::O_COL + mt * C::NP + 16 * ch + 8 * half, hi);
                                tmem_ld8(tmem + lane_addr + C::O_COL + mt * C::NP + NG + 16 * ch + 8 * half, lo);
                                tmem_wait_ld();
                            }
                            float v[8];
#pragma unroll
                            for (int n = 0; n < 8; ++n) v[n] = has_tiles ? hi[n] + lo[n] : 0.f;
                            // M-tiles 2 rank, 2 rank + 1 stay here, the other two go to the peer (selects,
                            // so that nothing is indexed by the rank at run time)
                            const bool mine = (mt >> 1) == (int)rank;
                            if (mine) {
#pragma unroll
                                for (int n = 0; n < 8; ++n) own[mt & 1][8 * ch + n] = v[n];
                            } else if (ok) {
                                const uint32_t dst = x_peer + (uint32_t)(mt & 1) * C::XM_TILE + xcol;
                                st_async_v4(dst, __float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                                            __float_as_uint(v[3]), xfull_remote);
                                st_async_v4(dst + 16u, __float_as_uint(v[4]), __float_as_uint(v[5]),
                                            __float_as_uint(v[6]), __float_as_uint(v[7]), xfull_remote);
                            }
                        }
                    }
                    tc_fence_before();
                    if (ok && lane == 0) {
#pragma unroll
                        for (int n4 = 0; n4 < NH; n4 += 4) {
                            st_async_v4(x_peer + xml + 4u * n4, __float_as_uint(ms[n4]), __float_as_uint(ms[n4 + 1]),
                                        __float_as_uint(ms[n4 + 2]), __float_as_uint(ms[n4 + 3]), xfull_remote);
                            st_async_v4(x_peer + xml + 4u * (NH + n4), __float_as_uint(ls[n4]),
                                        __float_as_uint(ls[n4 + 1]), __float_as_uint(ls[n4 + 2]),
                                        __float_as_uint(ls[n4 + 3]), xfull_remote);
                        }
                    }
                    if (lane == 0) mbar_arrive_expect_tx(bar(BR::XFULL + sw), 32 * 2 * NH * 4 + 2 * NH * 4);
                    ok = ok && spin_phase<true>(bar(BR::XFULL + sw), mseg & 1, wc, status);
                    ++mseg;
                    // (the area is written again only by the next segment's Q quantisation, after a
                    // barrier of all softmax warps, i.e. after every warp has read its part)
                    if (!named_bar_and(SMX, NSM, ok)) {
                        stop = true;
                        break;
                    }
                    const float *xs = reinterpret_cast<const float *>(smem + C::OFF_XM);
#pragma unroll
                    for (int ch = 0; ch < C::CH; ++ch) {
                        const uint32_t xcol = (uint32_t)row * C::XM_ROW + (uint32_t)(16 * ch + 8 * half) * 4u;
                        float lse_n[8];
#pragma unroll
                        for (int n = 0; n < 8; ++n) {
                            const int li = 8 * ch + n;
                            const float mp = xs[xml / 4 + li], lp = xs[xml / 4 + NH + li];
                            const float mm = fmaxf(ms[li], mp);
                            const float as = ms[li] == -INFINITY ? 0.f : fast_exp2(ms[li] - mm);
                            const float ap = mp == -INFINITY ? 0.f : fast_exp2(mp - mm);
                            // rank 0's term first in both CTAs, so that both compute the same l (and LSE)
                            const float l = rank == 0 ? __fmaf_rn(ls[li], as, __fmul_rn(lp, ap))
                                                      : __fmaf_rn(lp, ap, __fmul_rn(ls[li], as));
                            const bool empty = !(l > 0.f) || mm == -INFINITY;
                            // the stored p carried a factor 2^4
                            const float inv = empty ? 0.f : 0.0625f / l;
                            lse_n[n] = empty ? -INFINITY : (mm + __log2f(l)) * 0.69314718055994531f;
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float op = xs[(j * C::XM_TILE + xcol) / 4 + n];
                                store_o(ch, j, n, (own[j][li] * as + op * ap) * inv);
                            }
                        }
                        store_lse(ch, lse_n);
                    }
                } else {
#pragma unroll
                for (int ch = 0; ch < C::CH; ++ch) {
                    float inv_l[8], lse_n[8];

#pragma unroll
                    for (int n = 0; n < 8; ++n) {
                        const int cn = 16 * ch + 8 * half + n, li = 8 * ch + n;
                        const float l = redl[cn] + redl[NG + cn] + redl[2 * NG + cn] + redl[3 * NG + cn];
                        const bool empty = !(l > 0.f) || m[li] == -INFINITY;
                        inv_l[n] = empty ? 0.f : 1.f / l;
                        lse_n[n] = empty ? -INFINITY : (m[li] + __log2f(l)) * 0.69314718055994531f;
                    }
#pragma unroll
                    for (int i = 0; i < C::MB; ++i) {
                        float hi[8], lo[8];
                        tmem_ld8(tmem + lane_addr + C::O_COL + i * C::NP + 16 * ch + 8 * half, hi);
                        tmem_ld8(tmem + lane_addr + C::O_COL + i * C::NP + NG + 16 * ch + 8 * half, lo);
                        tmem_wait_ld();
#pragma unroll
                        for (int n = 0; n < 8; ++n) store_o(ch, i, n, (hi[n] + lo[n]) * inv_l[n]);
                    }
                    store_lse(ch, lse_n);
                }
                }
                tr.put(kPairEvEpiO, nsplit);
                if (nsplit >= 2 && p.fuse_merge) {
                    // Split-KV merge in the kernel: the last CTA (of this rank) to finish a split of
                    // sequence b merges all splits for its 256 latent rows and this column group.
                    // Release the partials of all 256 threads (ordered before the fence by the
                    // barrier), count this split, and acquire the others' if it was the last one.
                    named_bar_sync(SMX, NSM);
                    volatile int *merge_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 32);
                    int32_t *cnt = p.counters + ((int64_t)b * p.groups + grp) * 2 + rank;
                    if (row == 0 && half == 0) {
                        __threadfence();
                        const bool last = atomicAdd(cnt, 1) == nsplit - 1;
                        if (last) __threadfence();
                        *merge_flag = last;
                    }
                    named_bar_sync(SMX, NSM);
                    if (*merge_flag) {
                        tr.put(kPairEvMerge, nsplit);
                        // thread = 4 consecutive latent rows (one float4) x NG/4 columns.  The first
                        // U splits' partial outputs are in flight while the LSE partials are staged in
                        // an idle buffer (bf16: the P^T buffers, whose last step 3 has completed; E4M3:
                        // the Q area, read by no MMA before the next segment) and merged per column.
                        constexpr int NQ = NG / 4, U = 16 / NQ;
                        const int s0 = seq_info[4 * b + 3];
                        const int tid = (warp - 2) * 32 + lane;
                        const int d4 = 256 * (int)rank + 4 * (tid & 63), nq0 = (tid >> 6) * NQ;
                        const int nn = p.ncols - grp * NG < NG ? p.ncols - grp * NG : NG;
                        const float *op = p.opart + ((int64_t)s0 * p.ncols + grp * NG + nq0) * kDv + d4;
                        float *ls = reinterpret_cast<float *>(smem + C::OFF_STAGE);  // [nsplit][NG]
                        float *lt = ls + nsplit * NG;                             // [NG]
                        float4 v[U][NQ];
                        auto load_batch = [&](int sp0) {
#pragma unroll
                            for (int u = 0; u < U; ++u)
#pragma unroll
                                for (int j = 0; j < NQ; ++j)
                                    v[u][j] = (sp0 + u < nsplit && nq0 + j < nn)
                                                  ? __ldcg(reinterpret_cast<const float4 *>(
                                                        op + ((int64_t)(sp0 + u) * p.ncols + j) * kDv))
                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                        };
                        load_batch(0);
                        const float *lsrc = p.lsepart + ((int64_t)rank * p.slots + s0) * p.ncols + grp * NG;
                        for (int i = tid; i < nsplit * NG; i += NSM) {
                            const int sp = i / NG, n = i - sp * NG;
                            ls[i] = grp * NG + n < p.ncols ? __ldcg(lsrc + (int64_t)sp * p.ncols + n) : -INFINITY;
                        }
                        named_bar_sync(SMX, NSM);
                        if (tid < NG) lt[tid] = merged_lse([&](int sp) { return ls[sp * NG + tid]; }, nsplit);
                        named_bar_sync(SMX, NSM);
                        float acc[NQ][4];
#pragma unroll
                        for (int j = 0; j < NQ; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
                        for (int sp0 = 0; sp0 < nsplit; sp0 += U) {
                            if (sp0 > 0) load_batch(sp0);
#pragma unroll
                            for (int u = 0; u < U; ++u)
#pragma unroll
                                for (int j = 0; j < NQ; ++j) {
                                    const float lv = lt[nq0 + j];
                                    if (sp0 + u < nsplit && nq0 + j < nn && lv != -INFINITY) {
                                        const float w = merge_weight(ls[(sp0 + u) * NG + nq0 + j], lv);
                                        acc[j][0] = fmaf(w, v[u][j].x, acc[j][0]);
                                        acc[j][1] = fmaf(w, v[u][j].y, acc[j][1]);
                                        acc[j][2] = fmaf(w, v[u][j].z, acc[j][2]);
                                        acc[j][3] = fmaf(w, v[u][j].w, acc[j][3]);
                                    }
                                }
                        }
#pragma unroll
                        for (int j = 0; j < NQ; ++j) {
                            if (nq0 + j >= nn) break;
                            const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j][0], acc[j][1]);
                            const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j][2], acc[j][3]);
                            uint2 packed;
                            packed.x = *reinterpret_cast<const uint32_t *>(&lo);
                            packed.y = *reinterpret_cast<const uint32_t *>(&hi);
                            *reinterpret_cast<uint2 *>(p.o + ((int64_t)b * p.ncols + grp * NG + nq0 + j) * kDv + d4) = packed;
                            if (rank == 0 && (tid & 63) == 0) p.lse[(int64_t)b * p.ncols + grp * NG + nq0 + j] = lt[nq0 + j];
                        }
                        // ls/lt are next overwritten after a barrier of all softmax warps: as P^T (bf16)
                        // or by the next segment's Q quantisation (E4M3)
                        if (row == 0 && half == 0) *cnt = 0;  // ready for the next call
                    }
                }
                tc_fence_before();
                tr.put(kPairEvEpiDone, seg);
                ++seg;
            }
        }
        if (span && warp == 2 && lane == 0) span[2] = global_timer_ns();
        if (p.fuse_merge && !stop && ok) {
            // Sequences without a single KV row get no split: O = 0 and LSE = -inf, written by
            // cluster b mod (number of clusters), each CTA for its 256 latent rows.
            const int ncl = (int)(gridDim.x >> 1);
            const int d = 256 * (int)rank + (warp - 2) * 32 + lane;
            for (int bb = (int)(blockIdx.x >> 1); bb < p.batch; bb += ncl) {
                if (seq_info[4 * bb + 2] != 0) continue;
                for (int n = 0; n < p.ncols; ++n) p.o[((int64_t)bb * p.ncols + n) * kDv + d] = __float2bfloat16_rn(0.f);
                if (rank == 0 && warp == 2)
                    for (int n = lane; n < p.ncols; n += 32) p.lse[(int64_t)bb * p.ncols + n] = -INFINITY;
            }
        }
        if (stop || !ok) wc->abort = 1;
        if (pv_issued) {
            // the step-3 MMAs this thread issued complete before TMEM is released
            umma_commit(bar(BR::SFIN));
            drain_phase(bar(BR::SFIN), 0);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its peer may still write into its shared memory
    if (wc->abort) {
        // After an abort a peer's last st.async may not have been waited for: let it land
        // before either CTA leaves (no thread sends after the barrier above).
        const uint64_t t_q = global_timer_ns();
        while (global_timer_ns() - t_q < 20000ull) {
        }
    }
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
    if (span && threadIdx.x == 32) span[3] = global_timer_ns();
}

}  // namespace mla
