// C ABI of libsfa: argument validation, workspace sizing and kernel dispatch.
// The argument set follows the SparseFlashAttentionGrad README (参数说明) and the
// two-phase aclnn convention of aclnnFlashAttentionUnpaddingScoreGrad (函数原型).
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <vector>
#include <string>

#include "sfa_internal.cuh"

using namespace sfa;

namespace {

thread_local std::string g_last_error;
thread_local uint64_t g_wait_ns = 0;  // 0: the default limit
thread_local cudaEvent_t g_ev_before = nullptr, g_ev_after = nullptr;

// Records the timing-hook events (if set) around the main kernel launch.
struct KernelEvents {
    cudaEvent_t a, b;
    cudaStream_t s;
    KernelEvents(cudaStream_t st) : a(g_ev_before), b(g_ev_after), s(st) {
        g_ev_before = g_ev_after = nullptr;
        if (a) cudaEventRecord(a, s);
    }
    ~KernelEvents() {
        if (b) cudaEventRecord(b, s);
    }
};

sfa_status fail(sfa_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

sfa_status cuda_fail(cudaError_t e, const char* where) {
    return fail(SFA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define SFA_CUDA(expr, where)                              \
    do {                                                   \
        cudaError_t _e = (expr);                           \
        if (_e != cudaSuccess) return cuda_fail(_e, where); \
    } while (0)

bool n1_supported(int64_t n) {
    // 1/2/4/.../128 (SparseFlashAttentionGrad 约束说明) plus 3/6/12/24/48 (Ascend 950 list)
    static const int64_t ok[] = {1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 48, 64, 128};
    for (int64_t v : ok)
        if (v == n) return true;
    return false;
}

struct Sizes {
    int64_t T1, T2;
};

sfa_status check_shape(const sfa_shape* s, int64_t bs, int64_t mode, Sizes* out) {
    if (!s) return fail(SFA_ERR_NULLPTR, "shape is NULL");
    if (s->layout != SFA_LAYOUT_BSND && s->layout != SFA_LAYOUT_TND)
        return fail(SFA_ERR_INVALID, "layout %d: only BSND (0) or TND (1)", s->layout);
    if (s->dtype != SFA_DTYPE_BF16 && s->dtype != SFA_DTYPE_FP16)
        return fail(SFA_ERR_INVALID, "dtype %d: only bf16 (0) or fp16 (1)", s->dtype);
    if (s->N2 != 1) return fail(SFA_ERR_INVALID, "N2=%lld: only 1 is supported", (long long)s->N2);
    if (s->D != kD) return fail(SFA_ERR_INVALID, "D=%lld: only 512 is supported", (long long)s->D);
    if (s->Dr != kDr) return fail(SFA_ERR_INVALID, "Dr=%lld: only 64 is supported", (long long)s->Dr);
    if (!n1_supported(s->N1)) return fail(SFA_ERR_INVALID, "N1=%lld not supported", (long long)s->N1);
    if (s->B < 1 || s->B > 256) return fail(SFA_ERR_INVALID, "B=%lld outside [1,256]", (long long)s->B);
    if (s->topk < 1) return fail(SFA_ERR_INVALID, "topk=%lld < 1", (long long)s->topk);
    if (bs < 1 || bs > (1 << 20)) return fail(SFA_ERR_INVALID, "sparse_block_size=%lld", (long long)bs);
    if (mode != 0 && mode != 3) return fail(SFA_ERR_INVALID, "sparse_mode=%lld: only 0 or 3", (long long)mode);
    const int64_t kMaxS = 128 * 1024;
    if (s->layout == SFA_LAYOUT_BSND) {
        if (s->S1 < 1 || s->S1 > kMaxS || s->S2 < 1 || s->S2 > kMaxS)
            return fail(SFA_ERR_INVALID, "S1=%lld S2=%lld outside [1,128K]", (long long)s->S1, (long long)s->S2);
        out->T1 = s->B * s->S1;
        out->T2 = s->B * s->S2;
    } else {
        if (s->T1 < 1 || s->T2 < 1 || s->T1 > s->B * kMaxS || s->T2 > s->B * kMaxS)
            return fail(SFA_ERR_INVALID, "T1=%lld T2=%lld out of range", (long long)s->T1, (long long)s->T2);
        out->T1 = s->T1;
        out->T2 = s->T2;
    }
    if (out->T1 * s->topk > (int64_t)INT32_MAX * 64)
        return fail(SFA_ERR_INVALID, "T1*topk too large");
    return SFA_OK;
}

SeqDesc seq_desc(const sfa_shape* s, const Sizes& z, const int32_t* sq, const int32_t* skv) {
    SeqDesc d;
    d.layout = s->layout;
    d.B = (int32_t)s->B;
    d.S1 = s->S1;
    d.S2 = s->S2;
    d.T1 = z.T1;
    d.T2 = z.T2;
    d.seq_q = sq;
    d.seq_kv = skv;
    return d;
}

}  // namespace

void sfa::set_last_error(const char* msg) { g_last_error = msg; }

uint64_t sfa::wait_limit_ns() { return g_wait_ns ? g_wait_ns : 4000000000ull; }

extern "C" {

const char* sfa_version(void) { return "0.1.0"; }

const char* sfa_last_error_string(void) { return g_last_error.c_str(); }

sfa_status sfa_set_wait_limit(uint64_t limit_ns) {
    g_wait_ns = limit_ns;
    return SFA_OK;
}

sfa_status sfa_workspace_status(const void* workspace, sfa_stream_t stream, int32_t* site_out) {
    g_last_error.clear();
    if (!workspace) return fail(SFA_ERR_NULLPTR, "workspace is NULL");
    SFA_CUDA(cudaStreamSynchronize((cudaStream_t)stream), "synchronize stream");
    int32_t word = 0;
    SFA_CUDA(cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost), "read error word");
    if (site_out) *site_out = word;
    if (word != 0)
        return fail(SFA_ERR_TIMEOUT, "a device-side wait exceeded its limit (wait site %d); the outputs of that call "
                    "are invalid", word);
    return SFA_OK;
}

sfa_status sfa_set_kernel_events(void* event_before, void* event_after) {
    g_ev_before = (cudaEvent_t)event_before;
    g_ev_after = (cudaEvent_t)event_after;
    return SFA_OK;
}

const char* sfa_status_string(sfa_status st) {
    switch (st) {
        case SFA_OK: return "SFA_OK";
        case SFA_ERR_NULLPTR: return "SFA_ERR_NULLPTR";
        case SFA_ERR_INVALID: return "SFA_ERR_INVALID";
        case SFA_ERR_WORKSPACE: return "SFA_ERR_WORKSPACE";
        case SFA_ERR_CUDA: return "SFA_ERR_CUDA";
        case SFA_ERR_TIMEOUT: return "SFA_ERR_TIMEOUT";
        default: return "SFA_ERR_UNKNOWN";
    }
}

sfa_status sfa_grad_workspace_size(const sfa_shape* shape, int64_t sparse_block_size, int64_t sparse_mode,
                                   int32_t deterministic, size_t* workspace_bytes) {
    g_last_error.clear();
    if (!workspace_bytes) return fail(SFA_ERR_NULLPTR, "workspace_bytes is NULL");
    Sizes z;
    sfa_status st = check_shape(shape, sparse_block_size, sparse_mode, &z);
    if (st != SFA_OK) return st;
    *workspace_bytes = grad_ws_layout(z.T1, z.T2, shape->N1, shape->topk, sparse_block_size, deterministic != 0,
                                      fused_supported(shape->N1)).total;
    return SFA_OK;
}

}  // extern "C"

namespace {

// Shared body of sfa_grad and sfa_grad_rows: rows [row_begin, row_end) of the
// backward, with the dK/dV contributions added into `acc` (the workspace's own
// accumulator when `acc` is null, which is then zeroed first and cast into the
// three key-side outputs at the end).
sfa_status grad_impl(const void* query, const void* key, const void* value, const int32_t* sparse_indices,
                     const void* d_out, const void* out, const float* softmax_max, const float* softmax_sum,
                     const int32_t* actual_seq_lengths_q, const int32_t* actual_seq_lengths_kv,
                     const void* query_rope, const void* key_rope, float scale, int64_t sparse_block_size,
                     int64_t sparse_mode, int32_t deterministic, const sfa_shape* shape, void* workspace,
                     size_t workspace_bytes, sfa_stream_t stream, int64_t row_begin, int64_t row_end, void* acc,
                     const float* dout_absmax, void* d_query, void* d_key, void* d_value, void* d_query_rope,
                     void* d_key_rope) {
    g_last_error.clear();
    Sizes z;
    sfa_status st = check_shape(shape, sparse_block_size, sparse_mode, &z);
    if (st != SFA_OK) return st;
    const bool own_acc = acc == nullptr;
    if (!query || !key || !value || !sparse_indices || !d_out || !out || !softmax_max || !softmax_sum ||
        !query_rope || !key_rope || !d_query || !d_query_rope || !workspace ||
        (own_acc && (!d_key || !d_value || !d_key_rope)))
        return fail(SFA_ERR_NULLPTR, "a required tensor pointer is NULL");
    if (shape->layout == SFA_LAYOUT_TND && (!actual_seq_lengths_q || !actual_seq_lengths_kv))
        return fail(SFA_ERR_NULLPTR, "TND needs actual_seq_lengths_q and actual_seq_lengths_kv");
    if (!(scale == scale)) return fail(SFA_ERR_INVALID, "scale is NaN");
    if (row_begin < 0 || row_end < row_begin || row_end > z.T1)
        return fail(SFA_ERR_INVALID, "row range [%lld, %lld) outside [0, %lld]", (long long)row_begin,
                    (long long)row_end, (long long)z.T1);
    if (((uintptr_t)workspace & 255u) != 0) return fail(SFA_ERR_INVALID, "workspace not 256-byte aligned");
    if (!own_acc && ((uintptr_t)acc & 255u) != 0) return fail(SFA_ERR_INVALID, "dkv_accum not 256-byte aligned");
    const bool det = deterministic != 0;
    if (det && !own_acc && !dout_absmax)
        return fail(SFA_ERR_NULLPTR, "deterministic: dout_absmax (max|d_out| over every row of the accumulator) is NULL");
    const bool fused_shape = fused_supported(shape->N1);
    const GradWs ws = grad_ws_layout(z.T1, z.T2, shape->N1, shape->topk, sparse_block_size, det, fused_shape);
    if (workspace_bytes < ws.total)
        return fail(SFA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, ws.total);
    cudaStream_t s = (cudaStream_t)stream;
    char* w = (char*)workspace;

    GradArgs a;
    memset(&a, 0, sizeof a);
    a.q = query; a.qr = query_rope; a.k = key; a.kr = key_rope; a.v = value;
    a.dout = d_out; a.out = out; a.smax = softmax_max; a.ssum = softmax_sum; a.idx = sparse_indices;
    a.sd = seq_desc(shape, z, actual_seq_lengths_q, actual_seq_lengths_kv);
    a.N1 = shape->N1; a.topk = shape->topk; a.bs = (int)sparse_block_size; a.mode = (int)sparse_mode;
    a.scale = scale; a.det = det;
    a.blocks = (int32_t*)(w + ws.blocks); a.nblk = (int32_t*)(w + ws.nblk); a.nrows = (int32_t*)(w + ws.nrows);
    a.order = (int32_t*)(w + ws.order); a.rowsum = (float*)(w + ws.rowsum);
    a.dkv_acc = own_acc ? (void*)(w + ws.dkv) : acc;
    a.dq_acc = (float*)(w + ws.dq); a.ctrl = (int32_t*)(w + ws.ctrl);
    a.dq = d_query; a.dqr = d_query_rope;
    a.dtype = shape->dtype; a.rowlist = (int32_t*)(w + ws.rowlist); a.rowcap = shape->topk * sparse_block_size;
    a.row_begin = row_begin; a.row_end = row_end;
    // deterministic mode: the fixed-point grid follows max|dOut| (the workspace's own copy for a
    // whole-problem call, computed below; the caller's for a row range)
    float* own_dmax = (float*)(w + ws.ctrl + kCtrlDmax);
    a.dout_absmax = own_acc ? own_dmax : dout_absmax;

    SFA_CUDA(cudaMemsetAsync(w + ws.ctrl, 0, 256, s), "zero control word");
    if (own_acc)
        SFA_CUDA(cudaMemsetAsync(a.dkv_acc, 0, (size_t)z.T2 * kAccW * (det ? 8 : 4), s), "zero dK/dV accumulator");
    float* rowsum_dmax = own_acc && det ? own_dmax : nullptr;  // max|dO| taken by the rowsum pass
    SFA_CUDA(launch_compact(sparse_indices, a.sd, a.topk, a.bs, a.mode, (int32_t*)a.blocks, (int32_t*)a.nblk,
                            (int32_t*)a.nrows, row_begin, row_end, s), "index compaction");
    const bool fused = fused_shape && value == key;
    if (fused) {
        SFA_CUDA(launch_rowsum(shape->dtype, d_out, out, row_begin, row_end, shape->N1, (float*)a.rowsum, s,
                               rowsum_dmax), "rowsum(dO*O)");
        SFA_CUDA(launch_order(a.nrows, row_begin, row_end, (int32_t*)a.order, a.ctrl, s), "work order");
        // block-sparse lists sorted: consecutive selected blocks become contiguous key tiles
        if (a.bs > 1 && a.topk <= kSortMaxTopk)
            SFA_CUDA(launch_sort_blocks((int32_t*)a.blocks, a.nblk, a.topk, row_begin, row_end, s), "block sort");
        SFA_CUDA(launch_expand(a.blocks, a.nblk, a.sd, a.topk, a.bs, a.mode, a.rowcap, (int32_t*)a.rowlist, row_begin,
                               row_end, s),
                 "key row expansion");
        if (shape->N1 == 128) {
            // adjacent rows with identical block lists go to the paired kernel (two CTAs of a
            // cluster share each key tile); the other rows, if any, to the single-row kernel
            int32_t* counts = (int32_t*)(w + ws.ctrl + kCtrlCounts);
            int32_t* pairs = (int32_t*)(w + ws.pairs);
            SFA_CUDA(launch_pair_lists(a.blocks, a.nblk, a.sd, a.topk, row_begin, row_end, (int32_t*)(w + ws.pflags),
                                       pairs, (int32_t*)a.order, counts, s), "row pairs");
            PairArgs pa;
            memset(&pa, 0, sizeof pa);
            pa.q = query; pa.qr = query_rope; pa.k = key; pa.kr = key_rope; pa.dout = d_out;
            pa.sd = a.sd; pa.topk = a.topk; pa.bs = a.bs; pa.mode = a.mode; pa.scale = scale; pa.det = det;
            pa.dtype = shape->dtype; pa.blocks = a.blocks; pa.nblk = a.nblk; pa.pairs = pairs; pa.npairs = counts;
            pa.smax = softmax_max; pa.ssum = softmax_sum; pa.rowsum = a.rowsum; pa.dkv_acc = a.dkv_acc;
            pa.dq_acc = a.dq_acc; pa.dq = d_query; pa.dqr = d_query_rope; pa.err = a.ctrl;
            pa.dout_absmax = a.dout_absmax;
            a.nwork_dev = counts + 1;
            KernelEvents ev(s);
            SFA_CUDA(launch_bwd_pair(shape->dtype, pa, s), "paired backward");
            SFA_CUDA(launch_bwd_fused(shape->dtype, a, s), "fused backward");
        } else {
            KernelEvents ev(s);
            SFA_CUDA(launch_bwd_fused(shape->dtype, a, s), "fused backward");
        }
    } else {
        if (rowsum_dmax)
            SFA_CUDA(launch_absmax(shape->dtype, d_out, z.T1 * shape->N1 * kD, own_dmax, s), "max|dOut|");
        KernelEvents ev(s);
        SFA_CUDA(launch_bwd_generic(shape->dtype, a, s), "backward");
    }
    if (own_acc)
        SFA_CUDA(launch_cast_dkv(shape->dtype, det, a.dkv_acc, z.T2, d_key, d_key_rope, d_value, s, own_dmax, scale,
                                 z.T1, shape->N1), "cast dKey/dValue");
    return SFA_OK;
}

}  // namespace

extern "C" {

sfa_status sfa_grad(const void* query, const void* key, const void* value, const int32_t* sparse_indices,
                    const void* d_out, const void* out, const float* softmax_max, const float* softmax_sum,
                    const int32_t* actual_seq_lengths_q, const int32_t* actual_seq_lengths_kv,
                    const void* query_rope, const void* key_rope, float scale, int64_t sparse_block_size,
                    int64_t sparse_mode, int64_t pre_tokens, int64_t next_tokens, int32_t deterministic,
                    const sfa_shape* shape, void* workspace, size_t workspace_bytes, sfa_stream_t stream,
                    void* d_query, void* d_key, void* d_value, void* d_query_rope, void* d_key_rope) {
    (void)pre_tokens;
    (void)next_tokens;
    Sizes z;
    g_last_error.clear();
    sfa_status st = check_shape(shape, sparse_block_size, sparse_mode, &z);
    if (st != SFA_OK) return st;
    return grad_impl(query, key, value, sparse_indices, d_out, out, softmax_max, softmax_sum, actual_seq_lengths_q,
                     actual_seq_lengths_kv, query_rope, key_rope, scale, sparse_block_size, sparse_mode, deterministic,
                     shape, workspace, workspace_bytes, stream, 0, z.T1, nullptr, nullptr, d_query, d_key, d_value,
                     d_query_rope, d_key_rope);
}

sfa_status sfa_dkv_accum_size(const sfa_shape* shape, int32_t deterministic, size_t* accum_bytes) {
    g_last_error.clear();
    if (!accum_bytes) return fail(SFA_ERR_NULLPTR, "accum_bytes is NULL");
    Sizes z;
    sfa_status st = check_shape(shape, 1, 0, &z);
    if (st != SFA_OK) return st;
    *accum_bytes = (size_t)z.T2 * kAccW * (deterministic ? 8 : 4);
    return SFA_OK;
}

sfa_status sfa_grad_rows(const void* query, const void* key, const void* value, const int32_t* sparse_indices,
                         const void* d_out, const void* out, const float* softmax_max, const float* softmax_sum,
                         const int32_t* actual_seq_lengths_q, const int32_t* actual_seq_lengths_kv,
                         const void* query_rope, const void* key_rope, float scale, int64_t sparse_block_size,
                         int64_t sparse_mode, int32_t deterministic, int64_t row_begin, int64_t row_end,
                         const sfa_shape* shape, void* workspace, size_t workspace_bytes, sfa_stream_t stream,
                         void* dkv_accum, const float* dout_absmax, void* d_query, void* d_query_rope) {
    if (!dkv_accum) {
        g_last_error = "dkv_accum is NULL";
        return SFA_ERR_NULLPTR;
    }
    return grad_impl(query, key, value, sparse_indices, d_out, out, softmax_max, softmax_sum, actual_seq_lengths_q,
                     actual_seq_lengths_kv, query_rope, key_rope, scale, sparse_block_size, sparse_mode, deterministic,
                     shape, workspace, workspace_bytes, stream, row_begin, row_end, dkv_accum, dout_absmax, d_query,
                     nullptr, nullptr, d_query_rope, nullptr);
}

sfa_status sfa_dout_absmax(const void* d_out, const sfa_shape* shape, int64_t row_begin, int64_t row_end,
                           sfa_stream_t stream, float* dout_absmax) {
    g_last_error.clear();
    Sizes z;
    sfa_status st = check_shape(shape, 1, 0, &z);
    if (st != SFA_OK) return st;
    if (!d_out || !dout_absmax) return fail(SFA_ERR_NULLPTR, "a required pointer is NULL");
    if (row_begin < 0 || row_end < row_begin || row_end > z.T1)
        return fail(SFA_ERR_INVALID, "row range [%lld, %lld) outside [0, %lld]", (long long)row_begin,
                    (long long)row_end, (long long)z.T1);
    const int64_t per_row = shape->N1 * kD;
    const char* base = (const char*)d_out + (size_t)row_begin * per_row * 2;
    SFA_CUDA(launch_absmax(shape->dtype, base, (row_end - row_begin) * per_row, dout_absmax, (cudaStream_t)stream),
             "max|dOut|");
    return SFA_OK;
}

sfa_status sfa_dkv_finalize(const void* dkv_accum, const sfa_shape* shape, int32_t deterministic,
                            const float* dout_absmax, float scale, sfa_stream_t stream, void* d_key, void* d_value,
                            void* d_key_rope) {
    g_last_error.clear();
    Sizes z;
    sfa_status st = check_shape(shape, 1, 0, &z);
    if (st != SFA_OK) return st;
    if (!dkv_accum || !d_key || !d_value || !d_key_rope) return fail(SFA_ERR_NULLPTR, "a required pointer is NULL");
    if (deterministic && !dout_absmax) return fail(SFA_ERR_NULLPTR, "deterministic: dout_absmax is NULL");
    if (((uintptr_t)dkv_accum & 255u) != 0) return fail(SFA_ERR_INVALID, "dkv_accum not 256-byte aligned");
    SFA_CUDA(launch_cast_dkv(shape->dtype, deterministic != 0, dkv_accum, z.T2, d_key, d_key_rope, d_value,
                             (cudaStream_t)stream, dout_absmax, scale, z.T1, shape->N1), "cast dKey/dValue");
    return SFA_OK;
}

sfa_status sfa_fwd_workspace_size(const sfa_shape* shape, int64_t sparse_block_size, int64_t sparse_mode,
                                  size_t* workspace_bytes) {
    g_last_error.clear();
    if (!workspace_bytes) return fail(SFA_ERR_NULLPTR, "workspace_bytes is NULL");
    Sizes z;
    sfa_status st = check_shape(shape, sparse_block_size, sparse_mode, &z);
    if (st != SFA_OK) return st;
    *workspace_bytes = fwd_ws_layout(z.T1, shape->N1, shape->topk, sparse_block_size).total;
    return SFA_OK;
}

sfa_status sfa_fwd(const void* query, const void* key, const void* value, const int32_t* sparse_indices,
                   const int32_t* actual_seq_lengths_q, const int32_t* actual_seq_lengths_kv,
                   const void* query_rope, const void* key_rope, float scale, int64_t sparse_block_size,
                   int64_t sparse_mode, const sfa_shape* shape, void* workspace, size_t workspace_bytes,
                   sfa_stream_t stream, void* out, float* softmax_max, float* softmax_sum) {
    g_last_error.clear();
    Sizes z;
    sfa_status st = check_shape(shape, sparse_block_size, sparse_mode, &z);
    if (st != SFA_OK) return st;
    if (!query || !key || !value || !sparse_indices || !query_rope || !key_rope || !out || !softmax_max ||
        !softmax_sum || !workspace)
        return fail(SFA_ERR_NULLPTR, "a required tensor pointer is NULL");
    if (shape->layout == SFA_LAYOUT_TND && (!actual_seq_lengths_q || !actual_seq_lengths_kv))
        return fail(SFA_ERR_NULLPTR, "TND needs actual_seq_lengths_q and actual_seq_lengths_kv");
    const FwdWs ws = fwd_ws_layout(z.T1, shape->N1, shape->topk, sparse_block_size);
    if (workspace_bytes < ws.total)
        return fail(SFA_ERR_WORKSPACE, "workspace %zu < %zu", workspace_bytes, ws.total);
    if (((uintptr_t)workspace & 255u) != 0) return fail(SFA_ERR_INVALID, "workspace not 256-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    char* w = (char*)workspace;
    FwdArgs a;
    a.q = query; a.qr = query_rope; a.k = key; a.kr = key_rope; a.v = value;
    a.sd = seq_desc(shape, z, actual_seq_lengths_q, actual_seq_lengths_kv);
    a.N1 = shape->N1; a.topk = shape->topk; a.bs = (int)sparse_block_size; a.mode = (int)sparse_mode;
    a.scale = scale;
    int32_t* blocks = (int32_t*)(w + ws.blocks);
    int32_t* nblk = (int32_t*)(w + ws.nblk);
    int32_t* nrows = (int32_t*)(w + ws.nrows);
    SFA_CUDA(cudaMemsetAsync(w + ws.ctrl, 0, 256, s), "zero control word");
    a.blocks = blocks; a.nblk = nblk;
    a.out = out; a.smax = softmax_max; a.ssum = softmax_sum;
    SFA_CUDA(launch_compact(sparse_indices, a.sd, a.topk, a.bs, a.mode, blocks, nblk, nrows, 0, z.T1, s),
             "index compaction");
    if (ws.rowlist && value == key) {
        // tensor-core path: expanded key-row lists, longest rows first
        FwdFusedArgs f;
        f.q = query; f.qr = query_rope; f.k = key; f.kr = key_rope;
        f.rowlist = (int32_t*)(w + ws.rowlist); f.nrows = nrows; f.order = (int32_t*)(w + ws.order);
        f.out = out; f.smax = softmax_max; f.ssum = softmax_sum; f.err = (int*)(w + ws.ctrl);
        f.T1 = z.T1; f.T2 = z.T2; f.rowcap = shape->topk * sparse_block_size; f.scale = scale; f.dtype = shape->dtype;
        SFA_CUDA(launch_order(nrows, 0, z.T1, (int32_t*)f.order, (int32_t*)(w + ws.ctrl), s), "work order");
        // block-sparse lists sorted: consecutive selected blocks become contiguous key tiles
        if (a.bs > 1 && a.topk <= kSortMaxTopk)
            SFA_CUDA(launch_sort_blocks(blocks, nblk, a.topk, 0, z.T1, s), "block sort");
        f.blk16 = a.bs % 16 == 0 ? 1 : 0;
        if (f.blk16) {  // runs of 16 contiguous key rows: 16-row 2-D tile loads instead of row gathers
            f.nrows = (int32_t*)(w + ws.nslots);
            SFA_CUDA(launch_expand_blocks(blocks, nblk, a.sd, a.topk, a.bs, a.mode, f.rowcap, (int32_t*)f.rowlist,
                                          (int32_t*)f.nrows, s), "key row expansion");
        } else {
            SFA_CUDA(launch_expand(blocks, nblk, a.sd, a.topk, a.bs, a.mode, f.rowcap, (int32_t*)f.rowlist, 0, z.T1, s),
                     "key row expansion");
        }
        KernelEvents ev(s);
        SFA_CUDA(launch_fwd_fused(shape->dtype, f, s), "fused forward");
        return SFA_OK;
    }
    {
        KernelEvents ev(s);
        SFA_CUDA(launch_fwd_generic(shape->dtype, a, s), "forward");
    }
    return SFA_OK;
}

sfa_status sfa_compact_indices(const int32_t* sparse_indices, const int32_t* actual_seq_lengths_q,
                               const int32_t* actual_seq_lengths_kv, int64_t sparse_block_size, int64_t sparse_mode,
                               const sfa_shape* shape, sfa_stream_t stream, int32_t* blocks_out, int32_t* nblocks_out,
                               int32_t* nrows_out) {
    g_last_error.clear();
    Sizes z;
    sfa_status st = check_shape(shape, sparse_block_size, sparse_mode, &z);
    if (st != SFA_OK) return st;
    if (!sparse_indices || !blocks_out || !nblocks_out || !nrows_out)
        return fail(SFA_ERR_NULLPTR, "a required pointer is NULL");
    if (shape->layout == SFA_LAYOUT_TND && (!actual_seq_lengths_q || !actual_seq_lengths_kv))
        return fail(SFA_ERR_NULLPTR, "TND needs actual_seq_lengths_q and actual_seq_lengths_kv");
    SeqDesc sd = seq_desc(shape, z, actual_seq_lengths_q, actual_seq_lengths_kv);
    SFA_CUDA(launch_compact(sparse_indices, sd, shape->topk, (int)sparse_block_size, (int)sparse_mode, blocks_out,
                            nblocks_out, nrows_out, 0, z.T1, (cudaStream_t)stream), "index compaction");
    return SFA_OK;
}

sfa_status sfa_key_rows(const int32_t* sparse_indices, const int32_t* actual_seq_lengths_q,
                        const int32_t* actual_seq_lengths_kv, int64_t sparse_block_size, int64_t sparse_mode,
                        const sfa_shape* shape, int32_t sorted, int32_t block_aligned, sfa_stream_t stream,
                        int32_t* blocks_out, int32_t* nblocks_out, int32_t* rows_out, int32_t* count_out) {
    g_last_error.clear();
    Sizes z;
    sfa_status st = check_shape(shape, sparse_block_size, sparse_mode, &z);
    if (st != SFA_OK) return st;
    if (!sparse_indices || !blocks_out || !nblocks_out || !rows_out || !count_out)
        return fail(SFA_ERR_NULLPTR, "a required pointer is NULL");
    if (shape->layout == SFA_LAYOUT_TND && (!actual_seq_lengths_q || !actual_seq_lengths_kv))
        return fail(SFA_ERR_NULLPTR, "TND needs actual_seq_lengths_q and actual_seq_lengths_kv");
    if (sorted && shape->topk > kSortMaxTopk)
        return fail(SFA_ERR_INVALID, "sorted lists need topk <= %lld", (long long)kSortMaxTopk);
    cudaStream_t s = (cudaStream_t)stream;
    SeqDesc sd = seq_desc(shape, z, actual_seq_lengths_q, actual_seq_lengths_kv);
    const int bs = (int)sparse_block_size;
    const int64_t cap = shape->topk * sparse_block_size;
    SFA_CUDA(launch_compact(sparse_indices, sd, shape->topk, bs, (int)sparse_mode, blocks_out, nblocks_out, count_out,
                            0, z.T1, s), "index compaction");
    if (sorted) SFA_CUDA(launch_sort_blocks(blocks_out, nblocks_out, shape->topk, 0, z.T1, s), "block sort");
    if (block_aligned)
        SFA_CUDA(launch_expand_blocks(blocks_out, nblocks_out, sd, shape->topk, bs, (int)sparse_mode, cap, rows_out,
                                      count_out, s), "key row expansion");
    else
        SFA_CUDA(launch_expand(blocks_out, nblocks_out, sd, shape->topk, bs, (int)sparse_mode, cap, rows_out, 0, z.T1, s),
                 "key row expansion");
    return SFA_OK;
}

sfa_status sfa_softmax_grad_rowsum(const void* d_out, const void* out, const sfa_shape* shape, sfa_stream_t stream,
                                   float* rowsum_out) {
    g_last_error.clear();
    Sizes z;
    sfa_status st = check_shape(shape, 1, 0, &z);
    if (st != SFA_OK) return st;
    if (!d_out || !out || !rowsum_out) return fail(SFA_ERR_NULLPTR, "a required pointer is NULL");
    SFA_CUDA(launch_rowsum(shape->dtype, d_out, out, 0, z.T1, shape->N1, rowsum_out, (cudaStream_t)stream),
             "rowsum(dO*O)");
    return SFA_OK;
}

// ---------------------------------------------------------------------------
// Dense varlen FlashAttention (TND)
// ---------------------------------------------------------------------------
static sfa_status check_fa(const fa_shape* s, int64_t mode) {
    if (!s) return fail(SFA_ERR_NULLPTR, "shape is NULL");
    if (s->dtype != SFA_DTYPE_BF16 && s->dtype != SFA_DTYPE_FP16)
        return fail(SFA_ERR_INVALID, "dtype %d: only bf16 (0) or fp16 (1)", s->dtype);
    if (s->B < 1) return fail(SFA_ERR_INVALID, "B=%lld < 1", (long long)s->B);
    if (s->T1 < 1 || s->T2 < 1 || s->T1 > (1 << 20) || s->T2 > (1 << 20))
        return fail(SFA_ERR_INVALID, "T1=%lld T2=%lld outside [1,1M]", (long long)s->T1, (long long)s->T2);
    if (s->Nq < 1 || s->Nq > 256 || s->Nkv < 1 || s->Nq % s->Nkv != 0)
        return fail(SFA_ERR_INVALID, "Nq=%lld Nkv=%lld: need 1<=Nq<=256 and Nq%%Nkv==0", (long long)s->Nq,
                    (long long)s->Nkv);
    if (s->D < 8 || s->D > 256 || s->D % 8 != 0) return fail(SFA_ERR_INVALID, "D=%lld: multiple of 8 in [8,256]",
                                                             (long long)s->D);
    if (mode != 0 && mode != 3) return fail(SFA_ERR_INVALID, "sparse_mode=%lld: only 0 or 3", (long long)mode);
    return SFA_OK;
}

static sfa_status check_cu(const int64_t* cu, int64_t B, int64_t T, const char* name) {
    if (!cu) return fail(SFA_ERR_NULLPTR, "%s is NULL", name);
    int64_t prev = 0;
    for (int64_t b = 0; b < B; ++b) {
        if (cu[b] < prev) return fail(SFA_ERR_INVALID, "%s not non-decreasing at %lld", name, (long long)b);
        prev = cu[b];
    }
    if (prev != T) return fail(SFA_ERR_INVALID, "%s last entry %lld != T %lld", name, (long long)prev, (long long)T);
    return SFA_OK;
}

// FA workspaces start with the 256-byte control area (device error word), then the
// two cumulative-length arrays
constexpr size_t kCtrl = 256;
static size_t fa_cu_bytes(int64_t B) { return kCtrl + 2 * align256((size_t)B * 8); }

// Workspace of the tensor-core dense backward (head dims 64 and 128): cumulative lengths,
// work list, rowsum(dY o O), dQ accumulator, control word.
struct FaFusedWs {
    size_t items, rowsum, dq, ctrl, total;
};
static FaFusedWs fa_fused_ws(const fa_shape* s, bool det) {
    FaFusedWs w;
    size_t o = fa_cu_bytes(s->B);
    w.items = o;  o = align256(o + fa_fused_max_items(s->B, s->T2, s->Nkv) * 16);
    w.rowsum = o; o = align256(o + (size_t)s->T1 * s->Nq * 4);
    w.dq = o;     o = align256(o + (size_t)s->T1 * s->Nq * s->D * (det ? 8 : 4));
    w.ctrl = 0;
    w.total = o;
    return w;
}

sfa_status fa_grad_workspace_size(const fa_shape* shape, int64_t sparse_mode, int32_t deterministic,
                                  size_t* workspace_bytes) {
    g_last_error.clear();
    if (!workspace_bytes) return fail(SFA_ERR_NULLPTR, "workspace_bytes is NULL");
    sfa_status st = check_fa(shape, sparse_mode);
    if (st != SFA_OK) return st;
    *workspace_bytes = fa_cu_bytes(shape->B) +
                       align256((size_t)2 * shape->T2 * shape->Nkv * shape->D * (deterministic ? 8 : 4));
    if (fa_fused_supported(shape->D)) {
        const size_t f = fa_fused_ws(shape, deterministic != 0).total;
        if (f > *workspace_bytes) *workspace_bytes = f;
    }
    return SFA_OK;
}

sfa_status fa_grad(const void* q, const void* k, const void* v, const void* dy, const float* softmax_max,
                   const float* softmax_sum, const void* attention_in, const int64_t* actual_seq_qlen,
                   const int64_t* actual_seq_kvlen, double scale, double keep_prob, int64_t pre_tokens,
                   int64_t next_tokens, int64_t head_num, int64_t sparse_mode, int32_t deterministic,
                   const fa_shape* shape, void* workspace, size_t workspace_bytes, sfa_stream_t stream, void* dq,
                   void* dk, void* dv) {
    (void)pre_tokens;
    (void)next_tokens;
    g_last_error.clear();
    sfa_status st = check_fa(shape, sparse_mode);
    if (st != SFA_OK) return st;
    if (!q || !k || !v || !dy || !softmax_max || !softmax_sum || !attention_in || !dq || !dk || !dv || !workspace)
        return fail(SFA_ERR_NULLPTR, "a required tensor pointer is NULL");
    if ((st = check_cu(actual_seq_qlen, shape->B, shape->T1, "actual_seq_qlen")) != SFA_OK) return st;
    if ((st = check_cu(actual_seq_kvlen, shape->B, shape->T2, "actual_seq_kvlen")) != SFA_OK) return st;
    if (keep_prob != 1.0) return fail(SFA_ERR_INVALID, "keep_prob=%g: only 1 (no dropout)", keep_prob);
    if (head_num != shape->Nq) return fail(SFA_ERR_INVALID, "head_num %lld != Nq %lld", (long long)head_num,
                                           (long long)shape->Nq);
    const bool det = deterministic != 0;
    size_t acc_bytes = (size_t)2 * shape->T2 * shape->Nkv * shape->D * (det ? 8 : 4);
    size_t need = fa_cu_bytes(shape->B) + align256(acc_bytes);
    const bool fused = fa_fused_supported(shape->D);
    if (fused) need = std::max(need, fa_fused_ws(shape, det).total);
    if (workspace_bytes < need) return fail(SFA_ERR_WORKSPACE, "workspace %zu < %zu", workspace_bytes, need);
    cudaStream_t s = (cudaStream_t)stream;
    char* w = (char*)workspace;
    int64_t* cuq = (int64_t*)(w + kCtrl);
    int64_t* cukv = (int64_t*)(w + kCtrl + align256((size_t)shape->B * 8));
    void* acc = w + fa_cu_bytes(shape->B);
    SFA_CUDA(cudaMemsetAsync(w, 0, kCtrl, s), "zero control word");
    SFA_CUDA(cudaMemcpyAsync(cuq, actual_seq_qlen, shape->B * 8, cudaMemcpyHostToDevice, s), "copy seqlens");
    SFA_CUDA(cudaMemcpyAsync(cukv, actual_seq_kvlen, shape->B * 8, cudaMemcpyHostToDevice, s), "copy seqlens");
    if (fused) {
        const FaFusedWs fw = fa_fused_ws(shape, det);
        std::vector<int32_t> items;
        const size_t nitems = fa_fused_items(actual_seq_qlen, actual_seq_kvlen, shape->B, shape->Nq, shape->Nkv,
                                             (int)sparse_mode, &items);
        if (nitems)
            SFA_CUDA(cudaMemcpyAsync(w + fw.items, items.data(), nitems * 16, cudaMemcpyHostToDevice, s),
                     "copy work list");
        SFA_CUDA(cudaMemsetAsync(w + fw.dq, 0, (size_t)shape->T1 * shape->Nq * shape->D * (det ? 8 : 4), s),
                 "zero dQ accumulator");
        SFA_CUDA(cudaMemsetAsync(w + fw.ctrl, 0, 256, s), "zero control word");
        FaFusedArgs f;
        memset(&f, 0, sizeof f);
        f.q = q; f.k = k; f.v = v; f.dy = dy; f.o = attention_in; f.smax = softmax_max; f.ssum = softmax_sum;
        f.cu_q = cuq; f.cu_kv = cukv; f.B = shape->B; f.T1 = shape->T1; f.T2 = shape->T2; f.Nq = shape->Nq;
        f.Nkv = shape->Nkv; f.D = shape->D; f.mode = (int)sparse_mode; f.scale = (float)scale; f.det = det; f.dtype = shape->dtype;
        f.items = w + fw.items; f.nitems = (int)nitems; f.rowsum = (float*)(w + fw.rowsum); f.dq_acc = w + fw.dq;
        f.err = (int*)(w + fw.ctrl); f.dq = dq; f.dk = dk; f.dv = dv;
        f.dout_absmax = (const float*)(w + fw.ctrl + kCtrlDmax);
        if (det)
            SFA_CUDA(launch_absmax(shape->dtype, dy, shape->T1 * shape->Nq * shape->D, (float*)f.dout_absmax, s),
                     "max|dY|");
        KernelEvents ev(s);
        SFA_CUDA(launch_fa_bwd_fused(shape->dtype, f, s), "fa backward (tensor cores)");
        return SFA_OK;
    }
    SFA_CUDA(cudaMemsetAsync(acc, 0, acc_bytes, s), "zero dK/dV accumulator");
    FaArgs a;
    memset(&a, 0, sizeof a);
    a.q = q; a.k = k; a.v = v; a.dy = dy; a.o = attention_in; a.smax = softmax_max; a.ssum = softmax_sum;
    a.cu_q = cuq; a.cu_kv = cukv; a.B = shape->B; a.T1 = shape->T1; a.T2 = shape->T2; a.Nq = shape->Nq;
    a.Nkv = shape->Nkv; a.D = shape->D; a.mode = (int)sparse_mode; a.scale = (float)scale; a.det = det;
    a.dkv_acc = acc; a.dq = dq; a.dk = dk; a.dv = dv;
    a.dout_absmax = (const float*)(w + kCtrlDmax);
    if (det)
        SFA_CUDA(launch_absmax(shape->dtype, dy, shape->T1 * shape->Nq * shape->D, (float*)a.dout_absmax, s),
                 "max|dY|");
    KernelEvents ev(s);
    SFA_CUDA(launch_fa_bwd(shape->dtype, a, s), "fa backward");
    return SFA_OK;
}

sfa_status fa_fwd_workspace_size(const fa_shape* shape, int64_t sparse_mode, size_t* workspace_bytes) {
    g_last_error.clear();
    if (!workspace_bytes) return fail(SFA_ERR_NULLPTR, "workspace_bytes is NULL");
    sfa_status st = check_fa(shape, sparse_mode);
    if (st != SFA_OK) return st;
    *workspace_bytes = fa_cu_bytes(shape->B);
    return SFA_OK;
}

sfa_status fa_fwd(const void* q, const void* k, const void* v, const int64_t* actual_seq_qlen,
                  const int64_t* actual_seq_kvlen, double scale, int64_t sparse_mode, const fa_shape* shape,
                  void* workspace, size_t workspace_bytes, sfa_stream_t stream, void* out, float* softmax_max,
                  float* softmax_sum) {
    g_last_error.clear();
    sfa_status st = check_fa(shape, sparse_mode);
    if (st != SFA_OK) return st;
    if (!q || !k || !v || !out || !softmax_max || !softmax_sum || !workspace)
        return fail(SFA_ERR_NULLPTR, "a required tensor pointer is NULL");
    if ((st = check_cu(actual_seq_qlen, shape->B, shape->T1, "actual_seq_qlen")) != SFA_OK) return st;
    if ((st = check_cu(actual_seq_kvlen, shape->B, shape->T2, "actual_seq_kvlen")) != SFA_OK) return st;
    size_t need = fa_cu_bytes(shape->B);
    if (workspace_bytes < need) return fail(SFA_ERR_WORKSPACE, "workspace %zu < %zu", workspace_bytes, need);
    cudaStream_t s = (cudaStream_t)stream;
    char* w = (char*)workspace;
    int64_t* cuq = (int64_t*)(w + kCtrl);
    int64_t* cukv = (int64_t*)(w + kCtrl + align256((size_t)shape->B * 8));
    SFA_CUDA(cudaMemsetAsync(w, 0, kCtrl, s), "zero control word");
    SFA_CUDA(cudaMemcpyAsync(cuq, actual_seq_qlen, shape->B * 8, cudaMemcpyHostToDevice, s), "copy seqlens");
    SFA_CUDA(cudaMemcpyAsync(cukv, actual_seq_kvlen, shape->B * 8, cudaMemcpyHostToDevice, s), "copy seqlens");
    FaArgs a;
    memset(&a, 0, sizeof a);
    a.q = q; a.k = k; a.v = v;
    a.cu_q = cuq; a.cu_kv = cukv; a.B = shape->B; a.T1 = shape->T1; a.T2 = shape->T2; a.Nq = shape->Nq;
    a.Nkv = shape->Nkv; a.D = shape->D; a.mode = (int)sparse_mode; a.scale = (float)scale;
    a.out = out; a.smax_out = softmax_max; a.ssum_out = softmax_sum;
    SFA_CUDA(launch_fa_fwd(shape->dtype, a, s), "fa forward");
    return SFA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Dense lightning-indexer gradient with KL loss
// ---------------------------------------------------------------------------
namespace {

struct LigWs {
    size_t ctrl, sq, skv, nkeys, kvrow, order, loss, dki, total;
};

LigWs lig_ws_layout(const lig_shape* s) {
    LigWs w;
    size_t o = 0;
    w.ctrl = o;  o += 256;
    w.sq = o;    o = align256(o + (size_t)s->B * 4);
    w.skv = o;   o = align256(o + (size_t)s->B * 4);
    w.nkeys = o; o = align256(o + (size_t)s->T1 * 4);
    w.kvrow = o; o = align256(o + (size_t)s->T1 * 4);
    w.order = o; o = align256(o + (size_t)s->T1 * 4);
    w.loss = o;  o = align256(o + (size_t)s->T1 * 4);
    w.dki = o;   o = align256(o + (size_t)s->T2 * s->Di * 4);
    w.total = o;
    return w;
}

// Validates a lig_shape (filling T1 / T2 for BSND) into `z`.
sfa_status check_lig(const lig_shape* in, int64_t sparse_mode, lig_shape* z) {
    if (!in) return fail(SFA_ERR_NULLPTR, "shape is NULL");
    *z = *in;
    if (z->layout != SFA_LAYOUT_BSND && z->layout != SFA_LAYOUT_TND)
        return fail(SFA_ERR_INVALID, "layout %d", (int)z->layout);
    if (z->dtype != SFA_DTYPE_BF16 && z->dtype != SFA_DTYPE_FP16) return fail(SFA_ERR_INVALID, "dtype %d", (int)z->dtype);
    if (z->D != kD || z->Dr != kDr) return fail(SFA_ERR_INVALID, "D=%lld Dr=%lld: only 512 / 64", (long long)z->D,
                                                (long long)z->Dr);
    if (z->N1 != 64 && z->N1 != 128) return fail(SFA_ERR_INVALID, "N1=%lld: 64 or 128", (long long)z->N1);
    if (z->G != kLigG || z->Di != kLigDi)
        return fail(SFA_ERR_INVALID, "G=%lld Di=%lld: only %d / %d", (long long)z->G, (long long)z->Di, kLigG, kLigDi);
    if (z->B < 1 || z->B > 256) return fail(SFA_ERR_INVALID, "B=%lld outside [1,256]", (long long)z->B);
    if (sparse_mode != 0 && sparse_mode != 3) return fail(SFA_ERR_INVALID, "sparse_mode %lld", (long long)sparse_mode);
    if (z->layout == SFA_LAYOUT_BSND) {
        if (z->S1 < 1 || z->S2 < 1 || z->S1 > (1 << 17) || z->S2 > (1 << 17))
            return fail(SFA_ERR_INVALID, "S1=%lld S2=%lld outside [1,128K]", (long long)z->S1, (long long)z->S2);
        z->T1 = z->B * z->S1;
        z->T2 = z->B * z->S2;
    } else if (z->T1 < 1 || z->T2 < 1) {
        return fail(SFA_ERR_INVALID, "T1=%lld T2=%lld", (long long)z->T1, (long long)z->T2);
    }
    if (z->T1 * (int64_t)kLigG >= ((int64_t)1 << 31) || z->T1 * z->N1 >= ((int64_t)1 << 31) ||
        z->T2 >= ((int64_t)1 << 31))
        return fail(SFA_ERR_INVALID, "T1=%lld T2=%lld too large", (long long)z->T1, (long long)z->T2);
    return SFA_OK;
}

}  // namespace

extern "C" {

sfa_status lig_kl_grad_workspace_size(const lig_shape* shape, int64_t sparse_mode, size_t* workspace_bytes) {
    g_last_error.clear();
    if (!workspace_bytes) return fail(SFA_ERR_NULLPTR, "workspace_bytes is NULL");
    lig_shape z;
    sfa_status st = check_lig(shape, sparse_mode, &z);
    if (st != SFA_OK) return st;
    *workspace_bytes = lig_ws_layout(&z).total;
    return SFA_OK;
}

sfa_status lig_kl_grad(const void* query, const void* key, const void* query_index, const void* key_index,
                       const void* weights, const float* softmax_max, const float* softmax_sum,
                       const float* softmax_max_index, const float* softmax_sum_index, const void* query_rope,
                       const void* key_rope, const int64_t* actual_seq_lengths_query,
                       const int64_t* actual_seq_lengths_key, double scale, int64_t sparse_mode, int64_t pre_tokens,
                       int64_t next_tokens, const lig_shape* shape, void* workspace, size_t workspace_bytes,
                       sfa_stream_t stream, void* d_query_index, void* d_key_index, void* d_weights, float* loss) {
    (void)pre_tokens;
    (void)next_tokens;
    g_last_error.clear();
    lig_shape z;
    sfa_status st = check_lig(shape, sparse_mode, &z);
    if (st != SFA_OK) return st;
    if (!query || !key || !query_index || !key_index || !weights || !softmax_max || !softmax_sum ||
        !softmax_max_index || !softmax_sum_index || !query_rope || !key_rope || !workspace || !d_query_index ||
        !d_key_index || !d_weights || !loss)
        return fail(SFA_ERR_NULLPTR, "a required pointer is NULL");
    if (z.layout == SFA_LAYOUT_TND && (!actual_seq_lengths_query || !actual_seq_lengths_key))
        return fail(SFA_ERR_NULLPTR, "TND needs actual_seq_lengths_query and actual_seq_lengths_key");
    if (!(scale == scale) || scale > 1e30 || scale < -1e30) return fail(SFA_ERR_INVALID, "scale is not finite");
    const void* tma_ptrs[] = {query, key, query_index, key_index, query_rope, key_rope};
    for (const void* ptr : tma_ptrs)
        if (((uintptr_t)ptr & 15u) != 0) return fail(SFA_ERR_INVALID, "16-bit tensors must be 16-byte aligned");
    if (((uintptr_t)workspace & 255u) != 0) return fail(SFA_ERR_INVALID, "workspace not 256-byte aligned");
    const LigWs ws = lig_ws_layout(&z);
    if (workspace_bytes < ws.total)
        return fail(SFA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, ws.total);
    cudaStream_t s = (cudaStream_t)stream;
    char* w = (char*)workspace;

    sfa_shape ss;
    memset(&ss, 0, sizeof ss);
    ss.layout = z.layout; ss.dtype = z.dtype; ss.B = z.B; ss.S1 = z.S1; ss.S2 = z.S2;
    Sizes sz;
    sz.T1 = z.T1;
    sz.T2 = z.T2;
    const SeqDesc sd = seq_desc(&ss, sz, nullptr, nullptr);

    LigArgs a;
    memset(&a, 0, sizeof a);
    a.q = query; a.qr = query_rope; a.k = key; a.kr = key_rope; a.qi = query_index; a.ki = key_index;
    a.weights = weights; a.smax = softmax_max; a.ssum = softmax_sum; a.smax_i = softmax_max_index;
    a.ssum_i = softmax_sum_index;
    a.nkeys = (int32_t*)(w + ws.nkeys); a.kvrow = (int32_t*)(w + ws.kvrow); a.order = (int32_t*)(w + ws.order);
    a.dki_acc = (float*)(w + ws.dki); a.loss_rows = (float*)(w + ws.loss);
    a.dqi = d_query_index; a.dw = d_weights; a.err = (int*)(w + ws.ctrl);
    a.T1 = z.T1; a.T2 = z.T2; a.N1 = z.N1; a.scale = (float)scale; a.dtype = z.dtype;

    SFA_CUDA(cudaMemsetAsync(w + ws.ctrl, 0, 256, s), "zero control word");
    SFA_CUDA(cudaMemsetAsync(a.dki_acc, 0, (size_t)z.T2 * z.Di * 4, s), "zero dKeyIndex accumulator");
    SFA_CUDA(launch_lig_prep(sd, (int)sparse_mode, actual_seq_lengths_query, actual_seq_lengths_key,
                             (int32_t*)(w + ws.sq), (int32_t*)(w + ws.skv), (int32_t*)a.nkeys, (int32_t*)a.kvrow, s),
             "row bookkeeping");
    SFA_CUDA(launch_order(a.nkeys, 0, z.T1, (int32_t*)a.order, a.err, s), "work order");
    {
        KernelEvents ev(s);
        SFA_CUDA(launch_lig_fused(a, s), "fused indexer gradient");
    }
    SFA_CUDA(launch_lig_finish(z.dtype, a.dki_acc, z.T2, d_key_index, a.loss_rows, z.T1, loss, s),
             "dKeyIndex cast and loss sum");
    return SFA_OK;
}

}  // extern "C"

