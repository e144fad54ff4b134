// C ABI of libmla_decode.so (declared in include/mla_decode.h): argument
// validation, TMA tensor-map encoding and the three launches (plan, ETAP
// decode, combine).  No call allocates device memory or synchronises the host
// (except mla_decode_read_status, which waits for its own 4-byte copy).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "mla_decode.h"
#include "etap_pair_kernel.cuh"
#include "etap_duo_kernel.cuh"
#include "plan_combine_kernels.cuh"
#include "untransposed_kernel.cuh"
#include "plan_core.h"
#include "plan_cut.h"
#include "form_ablation.cuh"
#include "stream_probe.cuh"

namespace {

thread_local std::string g_last_cuda_error;

int cuda_fail(cudaError_t e, const char *what) {
    g_last_cuda_error = std::string(what) + ": " + cudaGetErrorString(e);
    return MLA_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D tensor map over a [rows, 576] row-major matrix of bf16 (elem_bytes 2) or E4M3 codes
// (elem_bytes 1); box = box_cols columns x box_rows rows, swizzled by the box's row width
// (128 bytes: 128B swizzle, 64: 64B, 32: 32B), as the MMA operand descriptors expect.
int encode_rows_576(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows, uint32_t box_cols = 64,
                    uint32_t elem_bytes = 2) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) {
        g_last_cuda_error = "cuTensorMapEncodeTiled unavailable";
        return MLA_ERR_CUDA;
    }
    cuuint64_t dims[2] = {(cuuint64_t)mla::kDqk, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)mla::kDqk * elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const uint32_t row_bytes = box_cols * elem_bytes;
    CUresult r = enc(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                     const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     row_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                     : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                       : CU_TENSOR_MAP_SWIZZLE_32B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
        return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

int check_shape(int batch, int q_len, int num_heads, int num_sms) {
    if (batch < 1 || batch > MLA_MAX_BATCH) return MLA_ERR_INVALID_ARG;
    if (q_len < 1 || num_heads < 1) return MLA_ERR_INVALID_ARG;
    if ((int64_t)q_len * num_heads > MLA_MAX_COLUMNS) return MLA_ERR_UNSUPPORTED;
    if (num_sms < 1 || num_sms > 4096) return MLA_ERR_INVALID_ARG;
    return MLA_OK;
}

// Per-device one-time opt-in to the kernels' dynamic shared memory sizes.
int ensure_smem_attr() {
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return MLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        e = cudaFuncSetAttribute(mla::etap_pair_kernel<mla::PairCfg16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mla::PairCfg16::SMEM_ALLOC);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        e = cudaFuncSetAttribute(mla::etap_pair_kernel<mla::PairCfg16E4>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::PairCfg16E4::SMEM_ALLOC);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        e = cudaFuncSetAttribute(mla::etap_pair_kernel<mla::PairCfg32E4>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::PairCfg32E4::SMEM_ALLOC);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        e = cudaFuncSetAttribute(mla::etap_duo_kernel<mla::DuoCfg64, mla::DuoCfg128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::kDuoSmemAlloc);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        e = cudaFuncSetAttribute(mla::etap_duo_kernel<mla::DuoCfg64, mla::DuoCfg128, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::kDuoSmemAlloc);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        e = cudaFuncSetAttribute(mla::etap_pair_kernel<mla::PairCfg16, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::PairCfg16::SMEM_ALLOC);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        e = cudaFuncSetAttribute(mla::untransposed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mla::kUtSmemAlloc);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        done[dev] = true;
    }
    return MLA_OK;
}

// One 2-CTA cluster per work unit and column group.
template <class C>
cudaError_t launch_pair(const CUtensorMap &tm_q, const CUtensorMap &tm_kv, const CUtensorMap &tm_qr,
                        const CUtensorMap &tm_kvr, const mla::DecodeParams &p, int clusters, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(320, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_ALLOC;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // Programmatic dependent launch: the prologue (barriers, TMEM, descriptor prefetch)
    // overlaps the preceding kernel; the kernel waits for it before any global read.
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    // the traced instance only for the tracing entry point (bf16 configurations)
    if constexpr (!C::KV8) {
        if (p.trace) return cudaLaunchKernelEx(&cfg, mla::etap_pair_kernel<C, true>, tm_q, tm_kv, tm_qr, tm_kvr, p);
    }
    return cudaLaunchKernelEx(&cfg, mla::etap_pair_kernel<C>, tm_q, tm_kv, tm_qr, tm_kvr, p);
}

// The duo kernel: one 2-CTA cluster per (work unit, column group); the grid covers the largest
// grouping the plan may pick (the clusters past the plan's own count find no work).
cudaError_t launch_duo(const mla::DuoMaps &maps, const mla::DecodeParams &p, int clusters, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(mla::kDuoThreads, 1, 1);
    cfg.dynamicSmemBytes = mla::kDuoSmemAlloc;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (p.trace) return cudaLaunchKernelEx(&cfg, mla::etap_duo_kernel<mla::DuoCfg64, mla::DuoCfg128, true>, maps, p);
    return cudaLaunchKernelEx(&cfg, mla::etap_duo_kernel<mla::DuoCfg64, mla::DuoCfg128>, maps, p);
}

// The combine kernel, launched as a programmatic dependent of what precedes it on the stream:
// with spin = 0 it waits for that whole grid; with spin = 1 (after the duo kernel only) its CTAs
// wait for their own sequence's split counters.
int launch_combine(void *workspace, int batch, int q_len, int num_heads, int num_sms, void *o, float *lse, int spin,
                   unsigned long long wait_limit_ns, cudaStream_t s) {
    const mla::WsLayout lay = mla::ws_layout(batch, q_len, num_heads, num_sms);
    const int ncols = q_len * num_heads;
    char *ws = reinterpret_cast<char *>(workspace);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ncols, batch, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, mla::combine_kernel, reinterpret_cast<int32_t *>(ws),
                                       reinterpret_cast<const float *>(ws + lay.opart),
                                       reinterpret_cast<const float *>(ws + lay.lsepart), ncols, lay,
                                       reinterpret_cast<__nv_bfloat16 *>(o), lse, spin, wait_limit_ns);
    if (e != cudaSuccess) return cuda_fail(e, "combine_kernel launch");
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "combine_kernel launch");
    return MLA_OK;
}

}  // namespace

extern "C" {

const char *mla_status_string(int status) {
    switch (status) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
        case MLA_ERR_ALIGNMENT: return "MLA_ERR_ALIGNMENT";
        case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
        case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
        case MLA_ERR_BLOCK_TABLE: return "MLA_ERR_BLOCK_TABLE";
        default: return "MLA_ERR_UNKNOWN";
    }
}

const char *mla_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

size_t mla_decode_workspace_size(int batch, int q_len, int num_heads, int num_sms) {
    if (check_shape(batch, q_len, num_heads, num_sms) != MLA_OK) return 0;
    return mla::ws_layout(batch, q_len, num_heads, num_sms).total;
}

int mla_decode_plan_host(const int32_t *seqlens, int batch, int q_len, int num_heads, int num_sms, int schedule,
                         int32_t *cta_ranges, int32_t *seq_info, int *num_ctas_out, int *num_groups_out,
                         int *unit_rows_out, int *group_cols_out) {
    int st = check_shape(batch, q_len, num_heads, num_sms);
    if (st != MLA_OK) return st;
    if (!seqlens || (schedule != 0 && schedule != 1)) return MLA_ERR_INVALID_ARG;
    const mla::WsLayout lay = mla::ws_layout(batch, q_len, num_heads, num_sms);
    const int ncols = q_len * num_heads;
    // schedule 1 (the bf16 cache) is the duo schedule when the shape has one, else the pair schedule
    const bool duo = schedule == 1 && lay.has_duo;
    int ctas = lay.ctas, groups = lay.groups, unit_rows = mla::kTileRows, gcols = mla::group_cols(ncols);
    if (duo) {
        int mn = 0;
        for (int b = 0; b < batch; ++b)
            if (seqlens[b] > 0 && (mn == 0 || seqlens[b] < mn)) mn = seqlens[b];
        const int mode = mla::duo_mode(ncols, mn);
        groups = mla::duo_groups(ncols, mode);
        ctas = mla::num_ctas(num_sms, groups);
        unit_rows = mla::kDuoRows;
        gcols = mla::duo_group_cols(mode);
    }
    // the cost-balanced cut of plan_core.h, sequence by sequence as the plan kernel does it
    const int E = mla::end_cost_units(unit_rows);
    int64_t total = 0, total_cost = 0;
    for (int b = 0; b < batch; ++b) {
        const int u = mla::units_of(seqlens[b], unit_rows);
        total += u;
        total_cost += u + (u > 0 ? E : 0);
    }
    if (total > INT32_MAX) return MLA_ERR_UNSUPPORTED;
    const int used = mla::used_ctas(total, ctas);
    std::vector<int32_t> begin((size_t)ctas + 1, (int32_t)total);
    int64_t f = 0, g = 0;
    int slots = 0;
    for (int b = 0; b < batch; ++b) {
        const int64_t units = mla::units_of(seqlens[b], unit_rows);
        const int64_t gend = g + units + (units > 0 ? E : 0);
        int first = -1, nsplit = 0;
        if (units > 0) {
            first = mla::cta_of(total_cost, used, g);
            nsplit = mla::cta_of(total_cost, used, g + units - 1) - first + 1;
            for (int c = mla::first_range_at_or_after(total_cost, used, g); c < used; ++c) {
                const int64_t x = mla::cta_begin(total_cost, used, c);
                if (x >= gend) break;
                begin[c] = (int32_t)mla::unit_at_cost(x, g, f, units);
            }
        }
        if (seq_info) {
            seq_info[4 * b + 0] = (int32_t)units;
            seq_info[4 * b + 1] = first;
            seq_info[4 * b + 2] = nsplit;
            seq_info[4 * b + 3] = slots;
        }
        if (nsplit >= 2) slots += nsplit;
        f += units;
        g = gend;
    }
    if (cta_ranges)
        for (int c = 0; c < ctas; ++c) {
            cta_ranges[2 * c] = begin[c];
            cta_ranges[2 * c + 1] = begin[c + 1];
        }
    if (num_ctas_out) *num_ctas_out = ctas;
    if (num_groups_out) *num_groups_out = groups;
    if (unit_rows_out) *unit_rows_out = unit_rows;
    if (group_cols_out) *group_cols_out = gcols;
    return MLA_OK;
}

int mla_decode_plan(const int32_t *seqlens, int batch, int q_len, int num_heads, int num_sms, void *workspace,
                    size_t workspace_bytes, void *stream) {
    int st = check_shape(batch, q_len, num_heads, num_sms);
    if (st != MLA_OK) return st;
    if (!seqlens || !workspace) return MLA_ERR_INVALID_ARG;
    if (!aligned(seqlens, 4) || !aligned(workspace, 256)) return MLA_ERR_ALIGNMENT;
    const mla::WsLayout lay = mla::ws_layout(batch, q_len, num_heads, num_sms);
    if (workspace_bytes < lay.total) return MLA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // Programmatic dependent launch: the plan is scheduled while the preceding kernel drains
    // and waits for it to complete before its first global read.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(mla::kPlanThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, mla::plan_kernel, seqlens, batch, q_len * num_heads, num_sms,
                                       reinterpret_cast<int32_t *>(workspace), lay);
    if (e != cudaSuccess) return cuda_fail(e, "plan_kernel launch");
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "plan_kernel launch");
    return MLA_OK;
}

int mla_combine(void *workspace, int batch, int q_len, int num_heads, int num_sms, void *o, float *lse,
                void *stream) {
    int st = check_shape(batch, q_len, num_heads, num_sms);
    if (st != MLA_OK) return st;
    if (!workspace || !o || !lse) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || !aligned(o, 16) || !aligned(lse, 4)) return MLA_ERR_ALIGNMENT;
    return launch_combine(workspace, batch, q_len, num_heads, num_sms, o, lse, 0, mla::kWaitLimitNs,
                          reinterpret_cast<cudaStream_t>(stream));
}

int mla_decode_fwd(const void *q, const void *kv, const int32_t *seqlens, const int32_t *block_table, int batch,
                   int q_len, int num_heads, int64_t kv_rows, int max_blocks, float softmax_scale, int causal,
                   void *o, float *lse, void *workspace, size_t workspace_bytes, int num_sms, unsigned flags,
                   void *stream) {
    return mla_decode_fwd_ragged(q, kv, seqlens, nullptr, block_table, batch, q_len, num_heads, kv_rows, max_blocks,
                                 softmax_scale, causal, o, lse, workspace, workspace_bytes, num_sms, flags, stream);
}

}  // extern "C"

namespace {

// Validation, tensor maps and launch shared by the bf16 and E4M3 cache entry points
// (kv_scale != NULL selects the E4M3 cache).
int decode_fwd_impl(const void *q, const void *kv, const float *kv_scale, const int32_t *seqlens,
                    const int32_t *q_lens, const int32_t *block_table, int batch, int q_len, int num_heads,
                    int64_t kv_rows, int max_blocks, float softmax_scale, int causal, void *o, float *lse,
                    void *workspace, size_t workspace_bytes, int num_sms, unsigned flags, void *stream,
                    unsigned long long *trace = nullptr, int trace_cap = 0, bool untransposed = false) {
    const bool fp8 = kv_scale != nullptr;
    if (untransposed && (fp8 || q_lens || trace)) return MLA_ERR_UNSUPPORTED;
    int st = check_shape(batch, q_len, num_heads, num_sms);
    if (st != MLA_OK) return st;
    if (!q || !kv || !seqlens || !o || !lse || !workspace) return MLA_ERR_INVALID_ARG;
    if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return MLA_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)(MLA_FLAG_SKIP_COMBINE | MLA_FLAG_TEST_EXPIRE_WAITS)) != 0) return MLA_ERR_INVALID_ARG;
    if (kv_rows < 1) return MLA_ERR_INVALID_ARG;
    const bool paged = block_table != nullptr;
    if (paged) {
        if (kv_rows % MLA_PAGE_SIZE != 0 || max_blocks < 1) return MLA_ERR_INVALID_ARG;
        if (kv_rows > INT32_MAX) return MLA_ERR_UNSUPPORTED;
        if (!aligned(block_table, 4)) return MLA_ERR_ALIGNMENT;
    } else {
        if ((int64_t)batch * kv_rows > INT32_MAX) return MLA_ERR_UNSUPPORTED;
    }
    if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(o, 16) || !aligned(lse, 4) || !aligned(seqlens, 4) ||
        !aligned(workspace, 256) || !aligned(q_lens, 4) || !aligned(kv_scale, 4))
        return MLA_ERR_ALIGNMENT;
    const mla::WsLayout lay = mla::ws_layout(batch, q_len, num_heads, num_sms);
    if (workspace_bytes < lay.total) return MLA_ERR_WORKSPACE;
    const int ncols = q_len * num_heads;

    st = ensure_smem_attr();
    if (st != MLA_OK) return st;
    CUtensorMap tm_q, tm_kv, tm_qr, tm_kvr;
    const int ng = mla::group_cols(ncols);
    const uint64_t kv_total_rows = paged ? (uint64_t)kv_rows : (uint64_t)batch * kv_rows;
    // the bf16 cache with more than 16 query columns runs the M = 256 kernel on the duo schedule
    const bool duo = !fp8 && lay.has_duo;
    if (fp8) {
        // the E4M3 kernel quantises Q itself (no Q maps): 128-code boxes of the latent part, 64-code rope boxes
        st = encode_rows_576(&tm_kv, kv, kv_total_rows, 64, 128, 1);
        if (st != MLA_OK) return st;
        st = encode_rows_576(&tm_kvr, kv, kv_total_rows, 64, 64, 1);
        if (st != MLA_OK) return st;
        tm_q = tm_kv;
        tm_qr = tm_kvr;
    } else if (duo) {
        tm_q = tm_qr = tm_kvr = CUtensorMap{};
    } else {
        st = encode_rows_576(&tm_q, q, (uint64_t)batch * ncols, (uint32_t)ng);
        if (st != MLA_OK) return st;
        st = encode_rows_576(&tm_kv, kv, kv_total_rows, 64);
        if (st != MLA_OK) return st;
        st = encode_rows_576(&tm_qr, q, (uint64_t)batch * ncols, (uint32_t)ng, 32);
        if (st != MLA_OK) return st;
        st = encode_rows_576(&tm_kvr, kv, kv_total_rows, 64, 32);
        if (st != MLA_OK) return st;
    }

    char *ws = reinterpret_cast<char *>(workspace);
    mla::DecodeParams p{};
    p.q = reinterpret_cast<const __nv_bfloat16 *>(q);
    p.kv_scale = kv_scale;
    p.seqlens = seqlens;
    p.q_lens = q_lens;
    p.block_table = block_table;
    p.ws = reinterpret_cast<int32_t *>(ws);
    p.opart = reinterpret_cast<float *>(ws + lay.opart);
    p.lsepart = reinterpret_cast<float *>(ws + lay.lsepart);
    p.o = reinterpret_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.kv_rows = kv_rows;
    p.batch = batch;
    p.q_len = q_len;
    p.num_heads = num_heads;
    p.ncols = ncols;
    p.ctas = lay.ctas;
    p.groups = lay.groups;
    p.max_blocks = paged ? max_blocks : 0;
    p.paged = paged ? 1 : 0;
    p.causal = causal;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.wait_limit_ns = (flags & MLA_FLAG_TEST_EXPIRE_WAITS) ? mla::kTestWaitLimitNs : mla::kWaitLimitNs;
    p.withhold_q = (flags & MLA_FLAG_TEST_EXPIRE_WAITS) ? 1 : 0;
    p.cta_ranges_off = (int)(lay.pair.cta_ranges / 4);
    p.tile_off_off = (int)(lay.pair.tile_off / 4);
    p.seq_info_off = (int)(lay.pair.seq_info / 4);
    p.cta_seq_off = (int)(lay.pair.cta_seq / 4);
    p.counters = reinterpret_cast<int32_t *>(ws + lay.pair.counters);
    p.slots = lay.slots;
    p.trace = trace;
    p.trace_cap = trace ? trace_cap : 0;
    // splits of a sequence are at most the work units (CTA pairs per column group); the bf16 cache
    // reaches the pair kernel only with 16 columns (more run the M = 256 kernel)
    const int max_splits = fp8 ? (ng == 16 ? mla::PairCfg16E4::MERGE_MAX_SPLITS : mla::PairCfg32E4::MERGE_MAX_SPLITS)
                               : mla::PairCfg16::MERGE_MAX_SPLITS;
    const bool separate_combine = !(flags & MLA_FLAG_SKIP_COMBINE) && lay.ctas > max_splits;
    p.fuse_merge = ((flags & MLA_FLAG_SKIP_COMBINE) || separate_combine) ? 0 : 1;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (untransposed) {
        // S = Q K^T form: two CTAs per work unit of the pair schedule (<= 16 columns) or the duo one
        mla::UtMaps maps;
        st = encode_rows_576(&maps.q64, q, (uint64_t)batch * ncols, 64);
        if (st != MLA_OK) return st;
        st = encode_rows_576(&maps.kv, kv, kv_total_rows, 64);
        if (st != MLA_OK) return st;
        p.fuse_merge = 0;
        p.signal_combine = 0;
        int units = lay.ctas * lay.groups;
        if (lay.has_duo) {
            units = 0;
            for (int mode = 0; mode < 2; ++mode) {
                if (mode == 1 && !mla::duo_mode1_possible(ncols)) break;
                const int g = mla::duo_groups(ncols, mode), c = mla::num_ctas(num_sms, g) * g;
                if (c > units) units = c;
            }
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * units, 1, 1);
        cfg.blockDim = dim3(mla::kUtThreads, 1, 1);
        cfg.dynamicSmemBytes = mla::kUtSmemAlloc;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, mla::untransposed_kernel, maps, p, lay);
        if (e != cudaSuccess) return cuda_fail(e, "untransposed_kernel launch");
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "untransposed_kernel launch");
        if (flags & MLA_FLAG_SKIP_COMBINE) return MLA_OK;
        return launch_combine(workspace, batch, q_len, num_heads, num_sms, o, lse, 0, p.wait_limit_ns, s);
    }
    if (duo) {
        mla::DuoMaps maps;
        st = encode_rows_576(&maps.q32, q, (uint64_t)batch * ncols, 32);
        if (st != MLA_OK) return st;
        st = encode_rows_576(&maps.q64, q, (uint64_t)batch * ncols, 64);
        if (st != MLA_OK) return st;
        st = encode_rows_576(&maps.kv, kv, kv_total_rows, 64);
        if (st != MLA_OK) return st;
        // the plan picks the grouping on the device (see plan_core.h); the kernel reads it from the header
        p.ctas = lay.duo.ctas_max;
        p.groups = lay.duo.groups_max;
        p.cta_ranges_off = (int)(lay.duo.cta_ranges / 4);
        p.tile_off_off = (int)(lay.duo.tile_off / 4);
        p.seq_info_off = (int)(lay.duo.seq_info / 4);
        p.cta_seq_off = (int)(lay.duo.cta_seq / 4);
        p.counters = reinterpret_cast<int32_t *>(ws + lay.duo.counters);
        // The splits are merged by the combine kernel: spread over all SMs it costs less than the
        // in-kernel merge of the pair kernel, which would fall on the last split's CTA pair.
        p.fuse_merge = 0;
        p.signal_combine = (flags & MLA_FLAG_SKIP_COMBINE) ? 0 : 1;
        int clusters = 0;
        for (int mode = 0; mode < 2; ++mode) {
            if (mode == 1 && !mla::duo_mode1_possible(ncols)) break;
            const int g = mla::duo_groups(ncols, mode), c = mla::num_ctas(num_sms, g) * g;
            if (c > clusters) clusters = c;
        }
        e = launch_duo(maps, p, clusters, s);
        if (e != cudaSuccess) return cuda_fail(e, "etap_duo_kernel launch");
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "etap_duo_kernel launch");
        if (flags & MLA_FLAG_SKIP_COMBINE) return MLA_OK;
        return launch_combine(workspace, batch, q_len, num_heads, num_sms, o, lse, 1, p.wait_limit_ns, s);
    }
    const int clusters = lay.ctas * lay.groups;
    if (fp8)
        e = ng == 16 ? launch_pair<mla::PairCfg16E4>(tm_q, tm_kv, tm_qr, tm_kvr, p, clusters, s)
                     : launch_pair<mla::PairCfg32E4>(tm_q, tm_kv, tm_qr, tm_kvr, p, clusters, s);
    else
        e = launch_pair<mla::PairCfg16>(tm_q, tm_kv, tm_qr, tm_kvr, p, clusters, s);
    if (e != cudaSuccess) return cuda_fail(e, "etap_pair_kernel launch");
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "etap_pair_kernel launch");
    if (separate_combine) return mla_combine(workspace, batch, q_len, num_heads, num_sms, o, lse, stream);
    return MLA_OK;
}

}  // namespace

extern "C" {

int mla_decode_fwd_untransposed(const void *q, const void *kv, const int32_t *seqlens, const int32_t *block_table,
                                int batch, int q_len, int num_heads, int64_t kv_rows, int max_blocks,
                                float softmax_scale, int causal, void *o, float *lse, void *workspace,
                                size_t workspace_bytes, int num_sms, unsigned flags, void *stream) {
    return decode_fwd_impl(q, kv, nullptr, seqlens, nullptr, block_table, batch, q_len, num_heads, kv_rows,
                           max_blocks, softmax_scale, causal, o, lse, workspace, workspace_bytes, num_sms, flags,
                           stream, nullptr, 0, true);
}

int mla_decode_fwd_ragged(const void *q, const void *kv, const int32_t *seqlens, const int32_t *q_lens,
                          const int32_t *block_table, int batch, int q_len, int num_heads, int64_t kv_rows,
                          int max_blocks, float softmax_scale, int causal, void *o, float *lse, void *workspace,
                          size_t workspace_bytes, int num_sms, unsigned flags, void *stream) {
    return decode_fwd_impl(q, kv, nullptr, seqlens, q_lens, block_table, batch, q_len, num_heads, kv_rows, max_blocks,
                           softmax_scale, causal, o, lse, workspace, workspace_bytes, num_sms, flags, stream);
}

int mla_decode_fwd_fp8(const void *q, const void *kv8, const float *kv_scale, const int32_t *seqlens,
                       const int32_t *q_lens, const int32_t *block_table, int batch, int q_len, int num_heads,
                       int64_t kv_rows, int max_blocks, float softmax_scale, int causal, void *o, float *lse,
                       void *workspace, size_t workspace_bytes, int num_sms, unsigned flags, void *stream) {
    if (!kv_scale) return MLA_ERR_INVALID_ARG;
    return decode_fwd_impl(q, kv8, kv_scale, seqlens, q_lens, block_table, batch, q_len, num_heads, kv_rows,
                           max_blocks, softmax_scale, causal, o, lse, workspace, workspace_bytes, num_sms, flags,
                           stream);
}

int mla_decode_fwd_trace(const void *q, const void *kv, const int32_t *seqlens, const int32_t *block_table, int batch,
                         int q_len, int num_heads, int64_t kv_rows, int max_blocks, float softmax_scale, int causal,
                         void *o, float *lse, void *workspace, size_t workspace_bytes, int num_sms,
                         unsigned long long *trace, int trace_cap, void *stream) {
    if (!trace || trace_cap < 1 || trace_cap > (1 << 20)) return MLA_ERR_INVALID_ARG;
    if (!aligned(trace, 8)) return MLA_ERR_ALIGNMENT;
    return decode_fwd_impl(q, kv, nullptr, seqlens, nullptr, block_table, batch, q_len, num_heads, kv_rows, max_blocks,
                           softmax_scale, causal, o, lse, workspace, workspace_bytes, num_sms, 0, stream, trace,
                           trace_cap);
}

int mla_stream_probe(const void *kv, int64_t rows, int units, int32_t *err, void *stream) {
    if (!kv || !err) return MLA_ERR_INVALID_ARG;
    if (rows < 128 || rows % 128 != 0 || rows > INT32_MAX || units < 1 || units > 4096) return MLA_ERR_INVALID_ARG;
    if (!aligned(kv, 16) || !aligned(err, 4)) return MLA_ERR_ALIGNMENT;
    CUtensorMap tm_kv, tm_kvr;
    int st = encode_rows_576(&tm_kv, kv, (uint64_t)rows, 64);
    if (st != MLA_OK) return st;
    st = encode_rows_576(&tm_kvr, kv, (uint64_t)rows, 64, 32);
    if (st != MLA_OK) return st;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(mla::stream_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)mla::kProbeSmem);
    });
    if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute");
    mla::ProbeParams pp{rows, units, err};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    mla::stream_probe_kernel<<<2 * units, 64, mla::kProbeSmem, s>>>(tm_kv, tm_kvr, pp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "stream_probe_kernel launch");
    return MLA_OK;
}

int mla_form_ablation(int form, int heads, int streams, int tiles, int ctas, unsigned long long *cycles, int32_t *err,
                      void *stream) {
    if (form != 0 && form != 1) return MLA_ERR_INVALID_ARG;
    if (heads != 16 && heads != 32 && heads != 64 && heads != 128) return MLA_ERR_INVALID_ARG;
    if (streams < 1 || streams > 3 || tiles < 1 || tiles > 65536 || ctas < 1 || ctas > 4096) return MLA_ERR_INVALID_ARG;
    if (!cycles || !err) return MLA_ERR_INVALID_ARG;
    if (!aligned(cycles, 8) || !aligned(err, 4)) return MLA_ERR_ALIGNMENT;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(mla::form_ablation_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)mla::kAblSmem);
    });
    if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute");
    mla::AblationParams ap{form, heads, streams, tiles, cycles, err};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    mla::form_ablation_kernel<<<ctas, 64, mla::kAblSmem, s>>>(ap);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "form_ablation_kernel launch");
    return MLA_OK;
}

int mla_decode_read_status(const void *workspace, int *status_out, void *stream) {
    if (!workspace || !status_out) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MLA_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "status copy");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "status copy sync");
    *status_out = v;
    return MLA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Entry point that allocates nothing: the scratch of plan/decode/combine is a
// file-scope device array (see mla_decode_fwd_static_ws in mla_decode.h).
namespace {

static __device__ __align__(256) unsigned char g_static_ws[MLA_STATIC_WORKSPACE_BYTES];

std::mutex g_static_ws_mu;
void *g_static_ws_addr[64] = {};  // device address of g_static_ws, per device, looked up once

// The argument checks of mla_decode_fwd, done before anything is launched.
int check_static_ws_args(const void *q, const void *kv, const int32_t *seqlens, const int32_t *block_table,
                         int batch, int q_len, int num_heads, int64_t kv_rows, int max_blocks, float softmax_scale,
                         int causal, const void *o, const float *lse, int num_sms) {
    int st = check_shape(batch, q_len, num_heads, num_sms);
    if (st != MLA_OK) return st;
    if (!q || !kv || !seqlens || !o || !lse) return MLA_ERR_INVALID_ARG;
    if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return MLA_ERR_INVALID_ARG;
    if (kv_rows < 1) return MLA_ERR_INVALID_ARG;
    if (block_table) {
        if (kv_rows % MLA_PAGE_SIZE != 0 || max_blocks < 1) return MLA_ERR_INVALID_ARG;
        if (kv_rows > INT32_MAX) return MLA_ERR_UNSUPPORTED;
        if (!aligned(block_table, 4)) return MLA_ERR_ALIGNMENT;
    } else if ((int64_t)batch * kv_rows > INT32_MAX) {
        return MLA_ERR_UNSUPPORTED;
    }
    if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(o, 16) || !aligned(lse, 4) || !aligned(seqlens, 4))
        return MLA_ERR_ALIGNMENT;
    if (mla::ws_layout(batch, q_len, num_heads, num_sms).total > (size_t)MLA_STATIC_WORKSPACE_BYTES)
        return MLA_ERR_WORKSPACE;
    return MLA_OK;
}

// Device address of g_static_ws on the current device, looked up once per device with that
// device current (in host code the name g_static_ws is a host-side stand-in, not a device address).
int static_ws_device_addr(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return MLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_static_ws_mu);
    if (!g_static_ws_addr[dev]) {
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_static_ws);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
        g_static_ws_addr[dev] = addr;
    }
    *out = g_static_ws_addr[dev];
    return MLA_OK;
}

}  // namespace

extern "C" int mla_decode_fwd_static_ws(const void *q, const void *kv, const int32_t *seqlens,
                                        const int32_t *block_table, int batch, int q_len, int num_heads,
                                        int64_t kv_rows, int max_blocks, float softmax_scale, int causal, void *o,
                                        float *lse, int num_sms, void *stream) {
    int st = check_static_ws_args(q, kv, seqlens, block_table, batch, q_len, num_heads, kv_rows, max_blocks,
                                  softmax_scale, causal, o, lse, num_sms);
    if (st != MLA_OK) return st;
    void *ws = nullptr;
    st = static_ws_device_addr(&ws);
    if (st != MLA_OK) return st;
    // The schedule rewrites the header (status word included) and the tables the
    // decode kernel reads; partial slots are written before the combine reads them.
    st = mla_decode_plan(seqlens, batch, q_len, num_heads, num_sms, ws, MLA_STATIC_WORKSPACE_BYTES, stream);
    if (st != MLA_OK) return st;
    return mla_decode_fwd(q, kv, seqlens, block_table, batch, q_len, num_heads, kv_rows, max_blocks, softmax_scale,
                          causal, o, lse, ws, MLA_STATIC_WORKSPACE_BYTES, num_sms, 0, stream);
}

extern "C" int mla_decode_static_ws_status(int *status_out, void *stream) {
    if (!status_out) return MLA_ERR_INVALID_ARG;
    void *ws = nullptr;
    int st = static_ws_device_addr(&ws);
    if (st != MLA_OK) return st;
    return mla_decode_read_status(ws, status_out, stream);
}
