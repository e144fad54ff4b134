// Cost-balanced split-KV ranges, shared by the device plan kernel and the host mirror
// (mla_decode_plan_host).  Not on the pages: it refines the schedule of plan_core.h.
//
// The end of a nonempty sequence costs its epilogue (and, when split, the merge) on the work unit
// that holds it, so each sequence end counts as end_cost_units() extra units.  On the cost axis
// sequence b occupies [cost_off(b), cost_off(b) + units_b) for its units and the next
// end_cost_units() positions for its end.  The cost axis is cut near-equally (cta_begin of
// plan_core.h over the total cost); a cut that falls among a sequence's end positions lands on
// that sequence's last unit boundary, so a work unit can receive no KV unit (its range is then
// empty, and it idles).  Measured ends: ~7 us (epilogue + merge) against a ~1.85 us tile on the
// CTA-pair kernel, ~10 us against a ~5 us unit on the M = 256 kernel.
#pragma once

#include <cstdint>

#include "plan_core.h"

namespace mla {

MLA_HD int end_cost_units(int unit_rows) { return unit_rows == kTileRows ? 4 : 2; }
// First flattened unit of the range that starts at cost position x, given the sequence that holds
// x (cost_off_b <= x < cost_off_b + units_b + its end cost) and its first flattened unit t0_b.
MLA_HD int64_t unit_at_cost(int64_t x, int64_t cost_off_b, int64_t t0_b, int64_t units_b) {
    const int64_t d = x - cost_off_b;
    return t0_b + (d < units_b ? d : units_b);
}
// The first range whose cost start is >= x (0 <= x <= total_cost, total_cost > 0).
MLA_HD int first_range_at_or_after(int64_t total_cost, int used, int64_t x) {
    return (int)((x * (int64_t)used + total_cost - 1) / total_cost);
}

}  // namespace mla
