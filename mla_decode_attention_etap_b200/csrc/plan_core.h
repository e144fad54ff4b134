// Split-KV schedule and workspace layout, shared by the device plan kernel,
// the decode/combine kernels and the host mirror (mla_decode_plan_host).
//
// The KV tiles (128 cache rows) of all sequences are concatenated in sequence
// order; CTA c of a column group takes the flattened tile range
// [T*c/G, T*(c+1)/G).  A sequence touched by several CTAs is "split": each CTA
// writes an fp32 partial (O_s, lse_s) into its slot and the combine kernel
// merges them.  Not on the pages: it exists so that a batch of few long
// sequences still spreads over every SM.
#pragma once

#include <cstddef>
#include <cstdint>

#ifdef __CUDACC__
#define MLA_HD __host__ __device__ __forceinline__
#else
#define MLA_HD inline
#endif

namespace mla {

constexpr int kTileRows = 128;   // KV rows per tile = UMMA M of S^T = K Q^T
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kPage = 64;

// header words (int32) at the start of the workspace
enum : int {
    kHdrStatus = 0,
    kHdrCtas = 1,
    kHdrGroups = 2,
    kHdrBatch = 3,
    kHdrTotalTiles = 4,
    kHdrCols = 5,
    kHdrSlotsUsed = 6,
    kHdrSlotsMax = 7,
    kHdrWords = 64
};

// Query columns (heads x tokens) per cluster = UMMA N of S^T: one group of 16
// when they fit, otherwise groups of 32 (whose kernel keeps a 5-slot ring).
MLA_HD int group_cols(int ncols) { return ncols <= 16 ? 16 : 32; }
MLA_HD int num_groups(int ncols) { return (ncols + group_cols(ncols) - 1) / group_cols(ncols); }
// Work units per column group: one per pair of SMs (a 2-CTA cluster).
MLA_HD int num_ctas(int num_sms, int groups) {
    int c = num_sms / 2 / groups;
    return c < 1 ? 1 : c;
}
MLA_HD int tiles_of(int L) { return L <= 0 ? 0 : (L + kTileRows - 1) / kTileRows; }

// CTAs that receive work: never more than there are tiles, so that every CTA
// in [0, used) owns at least one tile and the idle ones all come last (a
// sequence's splits are then exactly the consecutive CTAs that touch it).
MLA_HD int used_ctas(int64_t total, int ctas) { return total < (int64_t)ctas ? (int)total : ctas; }
// First flattened tile of CTA c: CTA c covers [cta_begin(c), cta_begin(c+1)).
MLA_HD int64_t cta_begin(int64_t total, int used, int c) {
    return c >= used ? total : total * (int64_t)c / used;
}
// The CTA whose range holds flattened tile f (0 <= f < total, used >= 1).
MLA_HD int cta_of(int64_t total, int used, int64_t f) { return (int)(((f + 1) * (int64_t)used - 1) / total); }

MLA_HD size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct WsLayout {
    size_t cta_ranges;  // int32 [ctas][2] (one range per work unit = SM pair)
    size_t cta_seq;     // int32 [ctas]: the sequence that holds the unit's first tile (batch if none)
    size_t tile_off;    // int32 [batch + 1]
    size_t seq_info;    // int32 [batch][4]: tiles, first CTA, splits, slot offset
    size_t opart;       // fp32  [slots][ncols][512]
    size_t lsepart;     // fp32  [2 ranks][slots][ncols] (the two CTAs of a pair compute equal values)
    size_t counters;    // int32 [batch][groups][2 ranks]: split CTAs done, for the in-kernel merge
    size_t total;
    int ctas, groups, slots;
};

MLA_HD WsLayout ws_layout(int batch, int q_len, int num_heads, int num_sms) {
    WsLayout w{};
    int ncols = q_len * num_heads;
    w.groups = num_groups(ncols);
    w.ctas = num_ctas(num_sms, w.groups);
    w.slots = batch + w.ctas;  // sum over split sequences of their split counts is < batch + ctas
    size_t off = align256(sizeof(int32_t) * kHdrWords);
    w.cta_ranges = off;
    off += align256(sizeof(int32_t) * 2 * (size_t)w.ctas);
    w.cta_seq = off;
    off += align256(sizeof(int32_t) * (size_t)w.ctas);
    w.tile_off = off;
    off += align256(sizeof(int32_t) * ((size_t)batch + 1));
    w.seq_info = off;
    off += align256(sizeof(int32_t) * 4 * (size_t)batch);
    w.opart = off;
    off += align256(sizeof(float) * (size_t)w.slots * ncols * kDv);
    w.lsepart = off;
    off += align256(sizeof(float) * 2 * (size_t)w.slots * ncols);
    w.counters = off;
    off += align256(sizeof(int32_t) * 2 * (size_t)batch * w.groups);
    w.total = off;
    return w;
}

}  // namespace mla
