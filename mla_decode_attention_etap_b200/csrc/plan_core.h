// Split-KV schedules and workspace layout, shared by the device plan kernel,
// the decode/combine kernels and the host mirror (mla_decode_plan_host).
//
// The KV units of all sequences are concatenated in sequence order and cut into one
// contiguous range per work unit and column group, balanced by cost (plan_cut.h).  A
// sequence touched by several ranges is "split": each writes an fp32 partial (O_s,
// lse_s) into its slot and the merge (in the decode kernel, or the combine kernel)
// combines them.  Not on the pages: it exists so that a batch of few long
// sequences still spreads over every SM.
//
// Two schedules live in one workspace:
//   pair  128-row units, column groups of 16 or 32: the CTA-pair kernel (etap_pair_kernel),
//         used by the FP8 cache for every shape and by the bf16 cache when q_len*h <= 16;
//   duo   256-row units (a tile of 128 rows per CTA of the pair), column groups of 64 (P as
//         bf16 hi + lo) or 128 (one bf16 P term): the M = 256 kernel (etap_duo_kernel), used
//         by the bf16 cache when q_len*h > 16.  Groups of 128 are chosen by the plan, on the
//         device, when q_len*h > 64 and every nonempty sequence holds at least
//         kSingleP_MinRows rows; the decode kernel reads the choice from the header.
#pragma once

#include <cstddef>
#include <cstdint>

#ifdef __CUDACC__
#define MLA_HD __host__ __device__ __forceinline__
#else
#define MLA_HD inline
#endif

namespace mla {

constexpr int kTileRows = 128;   // KV rows per tile = UMMA M of S^T = K Q^T in one CTA
constexpr int kDuoRows = 256;    // KV rows per unit of the duo kernel = UMMA M across the CTA pair
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kPage = 64;
// One bf16 P term is accurate enough when the softmax spreads over many rows: its rounding
// error in O shrinks like 1/sqrt(rows); at 8192 N(0,1) rows an emulation of the pipeline gives
// RMSE 1.78e-3 x RMS(O_ref) against the 2e-3 bar (bf16 rounding of O alone takes 1.65e-3).
constexpr int kSingleP_MinRows = 8192;

// header words (int32) at the start of the workspace
enum : int {
    kHdrStatus = 0,
    kHdrBatch = 1,
    kHdrCols = 2,
    kHdrSlotsMax = 3,
    kHdrSchedUsed = 4,   // written by the decode kernel: 0 pair, 1 duo (the partials' schedule)
    kHdrPair = 8,        // + kSch*: the pair schedule
    kHdrDuo = 16,        // + kSch*: the duo schedule
    kHdrWords = 64
};
enum : int { kSchCtas = 0, kSchGroups = 1, kSchTotal = 2, kSchSlotsUsed = 3, kSchGroupCols = 4, kSchMode = 5 };

// Column groups of the pair kernel: one group of 16 when they fit, otherwise groups of 32.
MLA_HD int group_cols(int ncols) { return ncols <= 16 ? 16 : 32; }
MLA_HD int num_groups(int ncols) { return (ncols + group_cols(ncols) - 1) / group_cols(ncols); }
// The bf16 cache runs the duo kernel for more than 16 query columns.
MLA_HD bool uses_duo(int ncols) { return ncols > 16; }
// Duo column group: mode 0 = 64 columns (P as bf16 hi + lo), mode 1 = 128 columns (one bf16 P term).
MLA_HD int duo_group_cols(int mode) { return mode ? 128 : 64; }
MLA_HD bool duo_mode1_possible(int ncols) { return ncols > 64; }
MLA_HD int duo_groups(int ncols, int mode) { return (ncols + duo_group_cols(mode) - 1) / duo_group_cols(mode); }
// Work units per column group: one per pair of SMs (a 2-CTA cluster).
MLA_HD int num_ctas(int num_sms, int groups) {
    int c = num_sms / 2 / groups;
    return c < 1 ? 1 : c;
}
MLA_HD int units_of(int L, int unit_rows) { return L <= 0 ? 0 : (L + unit_rows - 1) / unit_rows; }
MLA_HD int tiles_of(int L) { return units_of(L, kTileRows); }
// The duo mode the plan picks for these lengths (min_len: shortest nonempty sequence, 0 if none).
MLA_HD int duo_mode(int ncols, int min_len) { return duo_mode1_possible(ncols) && min_len >= kSingleP_MinRows ? 1 : 0; }

// Work units that receive ranges: never more than there are units.
MLA_HD int used_ctas(int64_t total, int ctas) { return total < (int64_t)ctas ? (int)total : ctas; }
// Near-equal cut of [0, total) into `used` ranges: range c is [cta_begin(c), cta_begin(c+1)).
// The plan cuts the cost axis of plan_cut.h this way.
MLA_HD int64_t cta_begin(int64_t total, int used, int c) {
    return c >= used ? total : total * (int64_t)c / used;
}
// The range that holds position f (0 <= f < total, used >= 1).
MLA_HD int cta_of(int64_t total, int used, int64_t f) { return (int)(((f + 1) * (int64_t)used - 1) / total); }

MLA_HD size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// One schedule's tables (byte offsets into the workspace), sized for its largest grouping.
struct Sched {
    size_t cta_ranges;  // int32 [ctas][2] (one range per work unit = SM pair)
    size_t cta_seq;     // int32 [ctas]: the sequence that holds the unit's first tile (batch if none)
    size_t tile_off;    // int32 [batch + 1]: first flattened unit of each sequence
    size_t seq_info;    // int32 [batch][4]: units, first CTA, splits, slot offset
    size_t counters;    // int32 [batch][groups][2 ranks]: split CTAs done (in-kernel merge, or the combine's wait)
    size_t done;        // int32 [batch]: combine CTAs done with a sequence (the last one rearms its counters)
    int ctas_max, groups_max, unit_rows;
};

struct WsLayout {
    Sched pair, duo;  // duo is meaningful only when has_duo
    int has_duo;
    size_t opart;    // fp32 [slots][ncols][512] (shared: one decode runs per plan at a time)
    size_t lsepart;  // fp32 [2 ranks][slots][ncols] (the two CTAs of a pair compute equal values)
    size_t total;
    int slots;       // batch + the most work units any schedule can have
    // pair schedule grouping (fixed by the shape)
    int ctas, groups;
};

MLA_HD size_t sched_tables(Sched &s, size_t off, int batch, int ctas_max, int groups_max, int unit_rows) {
    s.ctas_max = ctas_max;
    s.groups_max = groups_max;
    s.unit_rows = unit_rows;
    s.cta_ranges = off;
    off += align256(sizeof(int32_t) * 2 * (size_t)ctas_max);
    s.cta_seq = off;
    off += align256(sizeof(int32_t) * (size_t)ctas_max);
    s.tile_off = off;
    off += align256(sizeof(int32_t) * ((size_t)batch + 1));
    s.seq_info = off;
    off += align256(sizeof(int32_t) * 4 * (size_t)batch);
    s.counters = off;
    off += align256(sizeof(int32_t) * 2 * (size_t)batch * groups_max);
    s.done = off;
    off += align256(sizeof(int32_t) * (size_t)batch);
    return off;
}

MLA_HD WsLayout ws_layout(int batch, int q_len, int num_heads, int num_sms) {
    WsLayout w{};
    const int ncols = q_len * num_heads;
    w.groups = num_groups(ncols);
    w.ctas = num_ctas(num_sms, w.groups);
    w.has_duo = uses_duo(ncols) ? 1 : 0;
    size_t off = align256(sizeof(int32_t) * kHdrWords);
    off = sched_tables(w.pair, off, batch, w.ctas, w.groups, kTileRows);
    int units_max = w.ctas;
    if (w.has_duo) {
        // mode 0 has the most groups; mode 1 (when possible) the most units per group
        const int g0 = duo_groups(ncols, 0);
        const int c_max = num_ctas(num_sms, duo_mode1_possible(ncols) ? duo_groups(ncols, 1) : g0);
        off = sched_tables(w.duo, off, batch, c_max, g0, kDuoRows);
        if (c_max > units_max) units_max = c_max;
    }
    w.slots = batch + units_max;  // sum over split sequences of their split counts is < batch + units
    w.opart = off;
    off += align256(sizeof(float) * (size_t)w.slots * ncols * kDv);
    w.lsepart = off;
    off += align256(sizeof(float) * 2 * (size_t)w.slots * ncols);
    w.total = off;
    return w;
}

}  // namespace mla
