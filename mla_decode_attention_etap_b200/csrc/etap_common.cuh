// Helpers shared by the ETAP decode kernels: launch parameters, bounded
// mbarrier waits, the segment iterator over a CTA's flattened tile range, the
// cross-lane column reduction and bf16 packing.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "plan_core.h"
#include "ptx_sm100.cuh"

namespace mla {

constexpr int kStatusTimeout = -6;      // MLA_ERR_TIMEOUT
constexpr int kStatusBlockTable = -7;   // MLA_ERR_BLOCK_TABLE
constexpr int kStatusInvalid = -1;      // MLA_ERR_INVALID_ARG
constexpr uint64_t kWaitLimitNs = 4000000000ull;     // default bound of every wait
constexpr uint64_t kTestWaitLimitNs = 100000000ull;  // bound used by the expired-wait test hook
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p = 2^(x - m) stays <= 256
// When the running maximum of a column moves, it is set this far (log2 units) above the tile's
// maximum, so that later tiles rarely cross the threshold again (each crossing costs a cross-warp
// reduction and an O^T rescale).  p then starts at 2^-24 for the row of the maximum: fp32 and the
// bf16 hi + lo split keep their relative precision there, and only rows more than ~100 octaves
// below the maximum underflow to 0, as they would in any fp32 softmax.
constexpr float kRescaleHeadroom = 24.0f;
// E4M3 cache: P is stored as two E4M3 terms, whose absolute resolution is fixed (2^-9 at the
// bottom of the subnormal range), so p must stay close to the maximum: the running maximum is
// reset to 2 above the tile maximum and moves once a row exceeds it by 4, and p is stored times
// 2^4 (at most 2^8, inside the E4M3 range of 448).
constexpr float kRescaleThreshold8 = 4.0f;
constexpr float kRescaleHeadroom8 = 2.0f;
constexpr float kPScaleLog2_8 = 4.0f;

// Per-CTA wait control in shared memory: the abort flag every role polls and
// the bound after which a wait gives up.
struct WaitCtl {
    int abort;
    int pad;
    unsigned long long limit_ns;
};

struct DecodeParams {
    const __nv_bfloat16 *q;   // [B, q_len, h, 576] (read directly only by the E4M3-cache kernel)
    const float *kv_scale;    // E4M3 cache: one fp32 scale per cache row, indexed like the rows
    const int32_t *seqlens;
    const int32_t *q_lens;  // ragged batch: query tokens per sequence (<= q_len), or NULL
    const int32_t *block_table;
    int32_t *ws;  // workspace (int32 view)
    float *opart;
    float *lsepart;
    __nv_bfloat16 *o;
    float *lse;
    int64_t kv_rows;  // contiguous: rows per sequence; paged: total rows of the pool
    int batch, q_len, num_heads, ncols, ctas, groups, max_blocks, paged, causal;
    float scale_log2;  // softmax_scale * log2(e)
    unsigned long long wait_limit_ns;
    int withhold_q;    // test hook: never load Q, so that the bounded waits expire
    int cta_ranges_off, tile_off_off, seq_info_off, cta_seq_off;  // int32 offsets into ws
    int32_t *counters;  // [batch][groups][2]: split CTAs done per (sequence, column group, rank)
    int slots;          // partial slots (stride between the two ranks' LSE partial arrays)
    int fuse_merge;     // the last split CTA of a sequence merges the partials (no combine launch)
    int signal_combine; // count stored split partials for the combine kernel that follows
    unsigned long long *trace;  // measurement: event stamps of cluster 0's roles, or NULL
    int trace_cap;              // stamps per (CTA, role) in `trace`
};

// Event stamps for the tracing entry point: (code << 56) | (index << 40) | (globaltimer ns mod 2^40),
// written by one thread per (CTA, role) of cluster 0 into its own row of the trace buffer.
enum : int { kTraceRoles = 5 };
// Events of the CTA-pair kernel (softmax role, row 3): tile k's scores in / its P^T handed to
// step 3 (index: tile), a segment's epilogue begins / its last step 3 is complete / its outputs or
// partials are stored (index: splits) / this CTA merges the splits (index: splits) / it ends.
enum : int {
    kPairEvTile = 50,
    kPairEvTileDone = 51,
    kPairEvEpi = 52,
    kPairEvEpiS3 = 53,
    kPairEvEpiO = 54,
    kPairEvMerge = 55,
    kPairEvEpiDone = 56,
    kPairEvQ = 57,       // producer (row 0): a segment's Q loads issued (index: segment)
    kPairEvPair = 58,    // producer (row 0): a value pair's loads issued (index: pair)
    kPairEvScores = 59   // MMA issuer (row 1): a tile's score MMAs issued and committed (index: tile)
};
// ON = false (the kernels the decode entry points launch) compiles every stamp away; the traced
// instances are separate kernels, launched only by the tracing entry point.
template <bool ON>
struct TraceRowT {
    unsigned long long *row;
    int n, cap;
    __device__ void init(const DecodeParams &p, int role) {
        n = 0;
        cap = p.trace_cap;
        row = (ON && p.trace && blockIdx.x < 2) ? p.trace + ((size_t)blockIdx.x * kTraceRoles + role) * (size_t)cap
                                                : nullptr;
    }
    __device__ __forceinline__ void put(int code, int index) {
        if constexpr (ON) {
            if (row && n < cap) {
                row[n++] = ((unsigned long long)code << 56) | ((unsigned long long)(index & 0xFFFF) << 40) |
                           (global_timer_ns() & 0xFFFFFFFFFFull);
            }
        }
    }
};
// Per-CTA stamps (entry, start of work, end of work, exit) after the role rows; nullptr unless traced.
template <bool ON>
__device__ __forceinline__ unsigned long long *trace_span(const DecodeParams &p) {
    if constexpr (ON) {
        return p.trace ? p.trace + (size_t)2 * kTraceRoles * p.trace_cap + 4 * (size_t)blockIdx.x : nullptr;
    } else {
        return nullptr;
    }
}

// Bounded wait on an mbarrier phase.  Returns false (and raises the CTA abort
// flag) when the wait ran past kWaitLimitNs, or when another role aborted.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile WaitCtl *wc,
                                           int32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((spin & 63u) == 0) {
            if (wc->abort) return false;
            if (global_timer_ns() - t0 > wc->limit_ns) {
                wc->abort = 1;
                atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
}
// Bounded wait that polls instead of suspending: for phases that the other CTA of a pair completes
// (a multicast tcgen05.commit, a remote arrive), where a suspended try_wait can resume microseconds
// late.  Same abort and timeout handling as wait_phase.
__device__ __forceinline__ bool poll_phase(uint32_t bar, uint32_t parity, volatile WaitCtl *wc, int32_t *status) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((spin & 255u) == 0) {
            if (wc->abort) return false;
            if (global_timer_ns() - t0 > wc->limit_ns) {
                wc->abort = 1;
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
    // Same, starting from the sequence b0 that holds tile fb (from the plan): no search.
    __device__ void init_at(int b0, int64_t fb, int64_t fe_) {
        f = fb;
        fe = fe_;
        b = b0;
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

// Tile-by-tile cursor over the same segments (the MMA issuer keeps one for
// the scores and one for the output contraction).  STEP > 1: only tiles
// t0 + off, t0 + off + STEP, ... of each segment, skipping segments that have none.
template <int STEP = 1>
struct TileCursorT {
    SegIter it;
    int b, t0, t, t1, off;
    bool valid;
    __device__ void skip_empty(const int32_t *tile_off) {
        if constexpr (STEP > 1) {
            while (valid && t >= t1) {
                valid = it.next(tile_off, b, t0, t1);
                t = t0 + off;
            }
        }
    }
    __device__ void init(const int32_t *tile_off, int b0, int64_t fb, int64_t fe, int off_ = 0) {
        it.init_at(b0, fb, fe);
        off = STEP > 1 ? off_ : 0;
        b = t0 = t = t1 = 0;
        valid = it.next(tile_off, b, t0, t1);
        t = t0 + off;
        skip_empty(tile_off);
    }
    __device__ void advance(const int32_t *tile_off) {
        if (t + STEP < t1) {
            t += STEP;
            return;
        }
        valid = it.next(tile_off, b, t0, t1);
        t = t0 + off;
        skip_empty(tile_off);
    }
    __device__ bool first() const { return t == t0 + off; }
    __device__ bool last() const { return t + STEP >= t1; }
};
using TileCursor = TileCursorT<1>;

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

// Same for 8 values per lane: lane l ends with column col8(l); lanes l..l+3 (l % 4 == 0) share it.
__device__ __forceinline__ int col8(int lane) {
    return (((lane >> 4) & 1) << 2) | (((lane >> 3) & 1) << 1) | ((lane >> 2) & 1);
}
template <bool IS_MAX>
__device__ __forceinline__ float warp_colreduce8(const float (&v)[8], int lane) {
    float a4[4], a2[2];
    bool up = (lane & 16) != 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float send = up ? v[j] : v[j + 4];
        float keep = up ? v[j + 4] : v[j];
        a4[j] = op2<IS_MAX>(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
    up = (lane & 8) != 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        float send = up ? a4[j] : a4[j + 2];
        float keep = up ? a4[j + 2] : a4[j];
        a2[j] = op2<IS_MAX>(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
    up = (lane & 4) != 0;
    float a1 = op2<IS_MAX>(up ? a2[1] : a2[0], __shfl_xor_sync(0xffffffffu, up ? a2[0] : a2[1], 4));
    a1 = op2<IS_MAX>(a1, __shfl_xor_sync(0xffffffffu, a1, 2));
    return op2<IS_MAX>(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}

// Spinning variants for the softmax warps: a non-blocking probe in a loop
// resumes the moment the phase completes (a suspended try_wait can wake late,
// and the slowest of the 128 threads sets the pace of the next named barrier).
// A phase that the peer CTA completes (CLUSTER) is polled by lane 0 alone with relaxed
// cluster-scope probes; a restricted acquire fence then synchronises with the peer's release,
// and __syncwarp orders the other lanes after lane 0.  Call it from all 32 lanes of a warp.
template <bool CLUSTER>
__device__ __forceinline__ bool spin_phase(uint32_t bar, uint32_t parity, volatile WaitCtl *wc,
                                           int32_t *status) {
    if constexpr (CLUSTER) {
        bool ok = true;
        if ((threadIdx.x & 31) == 0) {
            if (!mbar_test_wait_cluster(bar, parity)) {
                const uint64_t t0 = global_timer_ns();
                for (uint32_t spin = 1;; ++spin) {
                    if (mbar_test_wait_cluster(bar, parity)) break;
                    if ((spin & 255u) == 0) {
                        if (wc->abort) {
                            ok = false;
                            break;
                        }
                        if (global_timer_ns() - t0 > wc->limit_ns) {
                            wc->abort = 1;
                            atomicCAS(status, 0, kStatusTimeout);
                            ok = false;
                            break;
                        }
                    }
                }
            }
            fence_acquire_cluster_smem();
        }
        __syncwarp();
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    } else {
        if (mbar_test_wait(bar, parity)) return true;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t spin = 1;; ++spin) {
            if (mbar_test_wait(bar, parity)) return true;
            if ((spin & 255u) == 0) {
                if (wc->abort) return false;
                if (global_timer_ns() - t0 > wc->limit_ns) {
                    wc->abort = 1;
                    atomicCAS(status, 0, kStatusTimeout);
                    return false;
                }
            }
        }
    }
}

}  // namespace mla
