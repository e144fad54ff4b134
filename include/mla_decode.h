/*
 * mla_decode.h — C ABI of libmla_decode.so: Multi-Head Latent Attention decode
 * in the Efficient Transpose Attention Pipeline (ETAP) form, for NVIDIA B200 (sm_100a).
 *
 * Operation (FlashMLA-ETAP technical summary, "Methodology"): for every sequence
 * b, query token t and head hd, with the N = q_len*h query columns ordered
 * n = t*h + hd,
 *     S^T = K Q^T          (KV rows are the MMA M dimension, query columns are N)
 *     P^T = softmax(S^T)   over the KV rows of each column, after multiplying by softmax_scale
 *     O^T = V^T P^T,  O = (O^T)^T
 * K is the full 576-column latent row and V its first 512 columns (one shared
 * latent KV head, the pages' "low-rank joint compression"). LSE is the natural
 * log of the softmax denominator, scale included: LSE = ln sum_j exp(scale*q.k_j).
 *
 * Visible rows: j < L_b; with `causal` set, query token t sees rows
 * j <= L_b - q_len + t (the q_len new tokens are the last q_len cache rows).
 * A column with no visible row yields O = 0 and LSE = -inf.
 *
 * Conventions shared by every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller; no call
 *    allocates or frees memory and no call synchronises the host, except
 *    mla_decode_read_status which waits for its own copy.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns an error code and launches nothing.
 *  - Device-side problems (a wait that ran out of time, an out-of-range block
 *    table entry) are recorded in a status word inside the workspace; read it
 *    with mla_decode_read_status.
 *  - Layouts are row-major; bf16 tensors are passed as void*.
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mla_status {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = -1,   /* null pointer, bad size, bad scale, inconsistent arguments */
    MLA_ERR_UNSUPPORTED = -2,   /* a shape this library does not implement */
    MLA_ERR_ALIGNMENT = -3,     /* a pointer misses its required alignment */
    MLA_ERR_WORKSPACE = -4,     /* workspace too small for (batch, q_len, num_heads, num_sms) */
    MLA_ERR_CUDA = -5,          /* a CUDA runtime/driver call failed (see mla_last_cuda_error) */
    MLA_ERR_TIMEOUT = -6,       /* device status: a bounded wait inside a kernel ran out */
    MLA_ERR_BLOCK_TABLE = -7    /* device status: a block-table entry was outside [0, kv_rows) */
} mla_status;

enum {
    MLA_D_QK = 576,      /* latent row width: 512 "nope" (also V) + 64 rope columns */
    MLA_D_V = 512,       /* value width: the first 512 latent columns */
    MLA_PAGE_SIZE = 64,  /* tokens per page of a paged cache */
    MLA_MAX_BATCH = 65536,
    MLA_MAX_COLUMNS = 1024, /* max q_len * num_heads */
    MLA_STATIC_WORKSPACE_BYTES = 16777216 /* scratch of mla_decode_fwd_static_ws: 16 MiB per GPU */
};

/* Flags for mla_decode_fwd. */
enum {
    MLA_FLAG_SKIP_COMBINE = 1, /* leave split partials in the workspace; call mla_combine yourself */
    /* Test hook for failure detection: the kernel never loads Q, so its bounded waits run out
     * (after 100 ms instead of the normal 4 s); the call still returns MLA_OK and
     * mla_decode_read_status then reports MLA_ERR_TIMEOUT. Outputs are undefined. */
    MLA_FLAG_TEST_EXPIRE_WAITS = 0x40000000
};

/*
 * Bytes of device workspace the plan/fwd/combine calls need for this shape.
 * num_sms is the number of SMs to spread the work over (148 on a B200).
 * Returns 0 for invalid arguments.
 *
 * Workspace layout (owned by the caller, 256-byte aligned): a small header
 * (status word, plan sizes), the split-KV schedule written by mla_decode_plan,
 * then fp32 partial outputs [slots, q_len*h, 512] and partial LSEs for
 * sequences whose KV range is split over several CTAs.
 */
MLA_API size_t mla_decode_workspace_size(int batch, int q_len, int num_heads, int num_sms);

/*
 * Split-KV scheduling metadata (not on the pages: needed so that a batch with
 * few sequences still fills every SM). Reads seqlens (device int32[batch]),
 * concatenates the KV units of all sequences (128 rows each for the CTA-pair
 * kernel, 256 for the M = 256 kernel), cuts them into one contiguous range per
 * work unit and column group, balanced by cost (each sequence end counts as the
 * units its epilogue and merge take, so a range may be empty), and records for
 * each sequence how many ranges touch it and where its partial results go. One
 * small kernel; no host synchronisation, so the call can be captured in a CUDA
 * graph. Also clears the workspace status word.
 */
MLA_API int mla_decode_plan(const int32_t *seqlens, int batch, int q_len, int num_heads, int num_sms,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * The decode itself (ETAP steps 1-4 of the pages, plus the split-KV partial
 * outputs and, unless MLA_FLAG_SKIP_COMBINE is set, their merge).  Without that
 * flag the merge is part of the call, with the arithmetic of mla_combine (so the
 * results are bitwise equal), and sequences with L_b = 0 get O = 0, LSE = -inf.
 * With 16 query columns or fewer (and for mla_decode_fwd_fp8) the last CTA to
 * finish a split of a sequence merges all of its splits inside the decode kernel
 * (when num_sms allows more splits per sequence than that merge's buffer holds,
 * the combine kernel runs after the decode instead).  With more columns on the
 * bf16 cache the combine kernel is launched behind the decode and starts on the
 * SMs the decode leaves: each of its CTAs waits for the split counters of its
 * own sequence, so early sequences are merged while the decode still runs.
 *   q            bf16 [batch, q_len, num_heads, 576], 16-byte aligned
 *   kv           contiguous: bf16 [batch, kv_rows, 576];
 *                paged (block_table != NULL): bf16 [kv_rows / 64, 64, 576], i.e. kv_rows = num_blocks*64
 *   seqlens      int32 [batch], device, 0 <= L_b (<= kv_rows when contiguous;
 *                <= max_blocks*64 when paged)
 *   block_table  int32 [batch, max_blocks] of physical block ids, or NULL for a contiguous cache.
 *                Entries past ceil(L_b/64) are never read. An entry outside
 *                [0, kv_rows/64) is not dereferenced: that page is not loaded, the
 *                sequence's output is unspecified, and MLA_ERR_BLOCK_TABLE is set in
 *                the status word.
 *   softmax_scale  > 0 and finite (576^-0.5 for the DeepSeek-R1 shape)
 *   causal       0 or 1 (see the header comment)
 *   o            bf16 [batch, q_len, num_heads, 512], 16-byte aligned
 *   lse          fp32 [batch, q_len, num_heads], 4-byte aligned
 *   workspace    the buffer mla_decode_plan filled for the same seqlens and shape
 * Rows of the cache past L_b may hold anything (NaN included): they are masked
 * out and never multiply into O.
 */
MLA_API int mla_decode_fwd(const void *q, const void *kv, const int32_t *seqlens, const int32_t *block_table,
                   int batch, int q_len, int num_heads, int64_t kv_rows, int max_blocks,
                   float softmax_scale, int causal, void *o, float *lse,
                   void *workspace, size_t workspace_bytes, int num_sms, unsigned flags, void *stream);

/*
 * Ragged multi-token decode: as mla_decode_fwd, with a different number of new
 * query tokens per sequence.  The pages decode one token per forward and name
 * more as a limitation (FlashMLA-ETAP Chinese abstract page, "Limitations"); this is
 * the speculative-verify shape with per-sequence draft lengths.
 *   q_lens   int32 [batch], device, 0 <= q_lens[b] <= q_len, or NULL (all q_len).
 *            Sequence b's real query tokens are rows t < q_lens[b] of its q_len
 *            query rows; they are the last q_lens[b] cache rows, so with causal = 1
 *            token t sees cache rows j <= L_b - q_lens[b] + t (else j < L_b).
 *            Rows t >= q_lens[b] are padding: O = 0, LSE = -inf.  A q_lens entry
 *            outside [0, q_len] is clamped and sets MLA_ERR_INVALID_ARG in the
 *            status word.
 * All other arguments, layouts and errors as for mla_decode_fwd (which is this
 * call with q_lens = NULL); q_lens must be 4-byte aligned.
 */
MLA_API int mla_decode_fwd_ragged(const void *q, const void *kv, const int32_t *seqlens, const int32_t *q_lens,
                          const int32_t *block_table, int batch, int q_len, int num_heads, int64_t kv_rows,
                          int max_blocks, float softmax_scale, int causal, void *o, float *lse,
                          void *workspace, size_t workspace_bytes, int num_sms, unsigned flags, void *stream);

/*
 * Decode over an FP8 latent cache (a storage format next to the pages' bf16
 * cache: half the bytes per cached token for the HBM-bound decode).  Every cache
 * row holds 576 OCP E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; 0x7F/0xFF are NaN) and one fp32 scale; element k of row r stands for
 * kv_scale[r] * e4m3(kv8[r][k]), and the result is the attention of
 * mla_decode_fwd over those values (same definition, outputs and tolerances).
 *   kv8        uint8 codes, laid out like mla_decode_fwd's kv (contiguous
 *              [batch, kv_rows, 576] or paged [kv_rows / 64, 64, 576]), 16-byte aligned
 *   kv_scale   fp32, one scale per cache row, indexed like the rows ([batch, kv_rows]
 *              or [kv_rows / 64, 64]), 4-byte aligned, must not be NULL; a scale must be
 *              finite and >= 0 (values below 2^-100 count as 2^-100 in the maximum)
 *   q_lens     as for mla_decode_fwd_ragged, or NULL
 * Any q_len * num_heads up to MLA_MAX_COLUMNS, in groups of 16 or 32 query columns
 * as for mla_decode_fwd.  The kernel stores Q per query column as two E4M3 terms
 * times a power of two, and P as two E4M3 terms; the fp32 accumulation, the
 * split-KV merge and the outputs are those of mla_decode_fwd.  All other
 * arguments, layouts and errors as there.
 */
MLA_API int mla_decode_fwd_fp8(const void *q, const void *kv8, const float *kv_scale, const int32_t *seqlens,
                       const int32_t *q_lens, const int32_t *block_table, int batch, int q_len, int num_heads,
                       int64_t kv_rows, int max_blocks, float softmax_scale, int causal, void *o, float *lse,
                       void *workspace, size_t workspace_bytes, int num_sms, unsigned flags, void *stream);

/*
 * The same decode in the untransposed form the pages set ETAP against ([TS]
 * Problem Statement: S = Q K^T puts the heads on the MMA's M dimension, which the
 * tensor core pads to its minimum; Methodology: ETAP puts the KV length there
 * instead).  Built for the A/B comparison of the two forms on tcgen05, not for
 * speed: M = the query-column group padded to 64 (q_len * num_heads <= 64, so
 * 16 heads pay 4x padding) or 128, a row softmax, O = P V; two CTAs per work unit
 * each compute all of S and one 256-column half of O (S and that half fill the
 * TMEM).  Same plan, workspace, split-KV partials and combine as mla_decode_fwd,
 * whose arguments, layouts, masking, outputs and errors it shares, with two
 * limits: the bf16 cache only and one q_len for every sequence.  Any q_len *
 * num_heads up to MLA_MAX_COLUMNS (groups of 16, 64 or 128 columns as the plan
 * picks for mla_decode_fwd).
 */
MLA_API int mla_decode_fwd_untransposed(const void *q, const void *kv, const int32_t *seqlens,
                                const int32_t *block_table, int batch, int q_len, int num_heads,
                                int64_t kv_rows, int max_blocks, float softmax_scale, int causal, void *o,
                                float *lse, void *workspace, size_t workspace_bytes, int num_sms,
                                unsigned flags, void *stream);

/*
 * Log-sum-exp merge of the split-KV partials that mla_decode_fwd left in the
 * workspace: lse = ln sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s, for
 * every sequence split over several CTAs; also writes O = 0, LSE = -inf for
 * empty sequences. Sequences handled by one CTA were already written by fwd.
 * Runs after everything before it on the stream.  It also rearms the split
 * counters in the workspace, which is why the workspace is writable here.
 */
MLA_API int mla_combine(void *workspace, int batch, int q_len, int num_heads, int num_sms,
                void *o, float *lse, void *stream);

/*
 * Measurement helper, not part of the decode (the pages have no counterpart): streams
 * rows x 576 bf16 (kv, 16-byte aligned, rows a multiple of 128, < 2^31) with exactly
 * the decode kernel's TMA read pattern (2*units CTAs, each CTA pair splitting every
 * 128-row tile by latent columns, 5 V-pair slots, L2 prefetch one tile ahead) and no
 * computation, so that timing it gives the read bandwidth that pattern can reach.
 * err: device int32, zeroed by the caller, set to 1 if a bounded wait ran out.
 * Asynchronous on `stream`; allocates nothing.
 */
MLA_API int mla_stream_probe(const void *kv, int64_t rows, int units, int32_t *err, void *stream);

/*
 * Measurement helper, not part of the decode (the pages have no counterpart): mla_decode_fwd
 * (flags 0, bf16 cache) that also records when each role of the two CTAs of cluster 0 reached its
 * events, so that a kernel's pipeline can be read off one launch.
 *   trace      device uint64 [2 CTAs][5 roles][trace_cap], then [num_sms][4]: 8-byte aligned,
 *              zeroed by the caller.  Roles of the M = 256 kernel (q_len*h > 16): 0 K-tile
 *              producer, 1 step-1 MMA issuer (CTA 0 only), 2 value producer, 3 softmax, 4 step-3
 *              MMA issuer (CTA 0 only); of the CTA-pair kernel (q_len*h <= 16): 0 producer,
 *              1 MMA issuer, 3 softmax.  The trailing rows hold each CTA's %globaltimer (ns) at
 *              entry, start of work (the plan read), end of work and exit.
 *              Entry = (event code << 56) | (index << 40) | (%globaltimer ns mod 2^40); a role
 *              stops recording after trace_cap events.  The event codes are listed in
 *              etap_duo_kernel.cuh and etap_common.cuh (the pair kernel's).
 *   trace_cap  1 .. 2^20
 * All other arguments, results and errors as for mla_decode_fwd.  The traced kernels are
 * separate instances of the decode kernels; the ones the other entry points launch carry no
 * stamps at all.
 */
MLA_API int mla_decode_fwd_trace(const void *q, const void *kv, const int32_t *seqlens, const int32_t *block_table,
                                 int batch, int q_len, int num_heads, int64_t kv_rows, int max_blocks,
                                 float softmax_scale, int causal, void *o, float *lse, void *workspace,
                                 size_t workspace_bytes, int num_sms, unsigned long long *trace, int trace_cap,
                                 void *stream);

/*
 * Measurement helper for the pages' argument for the transposed form (FlashMLA-ETAP technical
 * summary, "Problem Statement": with few heads the untransposed S = Q K^T pads the query heads up
 * to the tensor core's minimum M; "Methodology": S^T = K Q^T puts the KV rows on M instead).  Issues,
 * on each of `ctas` CTAs, the tensor-core instructions of `tiles` 128-row KV tiles for h = `heads`
 * query heads (d_qk 576, d_v 512, bf16 operands, fp32 accumulators) in one form:
 *   form 0 transposed:   S^T M=128 N=h K=576; O^T 4 x (M=128 N=h K=128)
 *   form 1 untransposed: S M=hpad N=128 K=576; O 2 x (M=hpad N=256 K=128), hpad = 64 (h <= 64) or 128
 * streams: 1 the score MMAs only, 2 the output MMAs only, 3 both (from two issuing threads).
 * cycles: device [ctas] uint64, written with each CTA's clock cycles from the first issue to the
 * completion of its last MMA.  err: device int32, zeroed by the caller, set to 1 if the bounded wait
 * for completion ran out.  The operands are zero-filled shared memory (no data is read from or
 * written to global memory besides these two).  Asynchronous on `stream`; allocates nothing.
 */
MLA_API int mla_form_ablation(int form, int heads, int streams, int tiles, int ctas, unsigned long long *cycles,
                      int32_t *err, void *stream);

/*
 * Copy the workspace status word to the host (waits for that copy only).
 * *status_out receives MLA_OK or the first device-side error recorded.
 */
MLA_API int mla_decode_read_status(const void *workspace, int *status_out, void *stream);

/*
 * Host mirror of the split-KV schedules, for testing and for callers that want to inspect
 * them. seqlens is a HOST int32[batch]. `schedule` 0 is the one mla_decode_fwd_fp8 uses (and
 * mla_decode_fwd for q_len*h <= 16): 128-row units, column groups of 16 or 32. `schedule` 1
 * is the one mla_decode_fwd uses: for q_len*h > 16, 256-row units (one 128-row tile per CTA of
 * a pair) and column groups of 64, or of 128 when q_len*h > 64 and every nonempty sequence
 * holds at least 8192 rows (the plan picks this on the device from the same lengths); for
 * q_len*h <= 16 it is schedule 0. Writes, when the pointers are non-NULL:
 *   cta_ranges  int32[num_ctas*2]  flattened unit range [begin, end) of each work unit (cut by
 *                                  cost as mla_decode_plan does; possibly empty)
 *   seq_info    int32[batch*4]     per sequence: unit count, first work unit, number of splits, partial slot offset
 * and returns the work units per column group, the column groups, the rows per unit and the
 * columns per group through the output pointers (each may be NULL).
 */
MLA_API int mla_decode_plan_host(const int32_t *seqlens, int batch, int q_len, int num_heads, int num_sms,
                                 int schedule, int32_t *cta_ranges, int32_t *seq_info, int *num_ctas_out,
                                 int *num_groups_out, int *unit_rows_out, int *group_cols_out);

/*
 * The whole decode (schedule, ETAP decode, combine) for callers that cannot
 * allocate device memory: a plugin or extension running inside a host
 * framework that owns the GPU's memory and hands its guests no allocator, or a
 * latency-critical serving loop that must not call cudaMalloc/cudaFree because
 * they can synchronise the whole device. The caller still passes every input
 * and output; the scratch (schedule + fp32 split partials) lives in one static
 * device array of MLA_STATIC_WORKSPACE_BYTES inside this library, which every
 * GPU that loads the library keeps until the process exits. The paper has no
 * counterpart: this is a deployment convenience.
 *
 * Arguments are those of mla_decode_fwd minus the workspace and flags.
 * Returns MLA_ERR_WORKSPACE, launching nothing, when
 * mla_decode_workspace_size(batch, q_len, num_heads, num_sms) exceeds
 * MLA_STATIC_WORKSPACE_BYTES (on 148 SMs: B=16, h=16 needs about 3 MB and
 * B=16, q_len=4, h=16 about 12 MB; B=32, h=128 does not fit). No call allocates memory.
 *
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address once and keeps it for the life of the process; make
 * that first call before any stream capture. The library must not be used on a
 * device across a cudaDeviceReset (the array then moves and the kept address is
 * stale). Every call shares the one array and it keeps the last call's contents
 * (the schedule rewrites everything later reads, status word included), so calls
 * that overlap on the GPU, on different streams or host threads, race: order
 * them on one stream. Read the device status word of the last call (a wait that
 * ran out, an out-of-range block-table entry) with mla_decode_static_ws_status.
 */
MLA_API int mla_decode_fwd_static_ws(const void *q, const void *kv, const int32_t *seqlens,
                                     const int32_t *block_table, int batch, int q_len, int num_heads,
                                     int64_t kv_rows, int max_blocks, float softmax_scale, int causal,
                                     void *o, float *lse, int num_sms, void *stream);

/*
 * The device status word of the last mla_decode_fwd_static_ws call on the current
 * device, copied to the host on `stream` (waits for that copy only): MLA_OK, or the
 * first device-side error the call recorded (MLA_ERR_TIMEOUT, MLA_ERR_BLOCK_TABLE,
 * MLA_ERR_INVALID_ARG). It plays the part of mla_decode_read_status for the static
 * array, whose address callers never see. The paper has no counterpart. Allocates
 * nothing; the same set-up rule as mla_decode_fwd_static_ws applies.
 */
MLA_API int mla_decode_static_ws_status(int *status_out, void *stream);

/* Human-readable name of a status code. */
MLA_API const char *mla_status_string(int status);

/* The last CUDA error string seen by this thread (after MLA_ERR_CUDA). */
MLA_API const char *mla_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
