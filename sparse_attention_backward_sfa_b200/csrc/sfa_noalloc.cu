// sfa_grad_noalloc: the sparse attention backward for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs
// inside another framework's allocator (where a raw cudaMalloc would bypass its
// memory accounting and can fail or fragment its pool), plugins and embedded
// runtimes that are given only input and output buffers, and code paths where
// allocation is forbidden or would synchronize the device.  This entry point
// takes only inputs and outputs and keeps its scratch in a fixed-size device
// array that is part of the library image.
//
// The scratch array holds the fp32 / fixed-point dKey|dKeyRope|dValue
// accumulator and the index-compaction tables of the CUDA-core backward
// kernel.  It is shared by every call on a device and keeps the previous call's
// contents; the accumulator is cleared on the call's stream before use.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "sfa_internal.cuh"

using namespace sfa;

namespace {

// Maximum scratch of one call.  Every GPU that loads the library reserves this
// much device memory until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};  // device address of g_noalloc_scratch per device

// errors are reported through sfa_last_error_string()
sfa_status nfail(sfa_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    set_last_error(buf);
    return st;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with cudaGetSymbolAddress (with that device current).
sfa_status scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return nfail(SFA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return nfail(SFA_ERR_INVALID, "device %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return nfail(SFA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SFA_OK;
}

}  // namespace

extern "C" {

sfa_status sfa_grad_noalloc(const void* query, const void* key, const void* value, const int32_t* sparse_indices,
                            const void* d_out, const void* out, const float* softmax_max, const float* softmax_sum,
                            const int32_t* actual_seq_lengths_q, const int32_t* actual_seq_lengths_kv,
                            const void* query_rope, const void* key_rope, float scale, int64_t sparse_block_size,
                            int64_t sparse_mode, int64_t pre_tokens, int64_t next_tokens, int32_t deterministic,
                            const sfa_shape* shape, sfa_stream_t stream, void* d_query, void* d_key, void* d_value,
                            void* d_query_rope, void* d_key_rope) {
    (void)pre_tokens;
    (void)next_tokens;
    // argument validation shared with sfa_grad (host only)
    size_t ignored = 0;
    sfa_status st = sfa_grad_workspace_size(shape, sparse_block_size, sparse_mode, deterministic, &ignored);
    if (st != SFA_OK) return st;  // message already set by the validation
    if (!query || !key || !value || !sparse_indices || !d_out || !out || !softmax_max || !softmax_sum ||
        !query_rope || !key_rope || !d_query || !d_key || !d_value || !d_query_rope || !d_key_rope)
        return nfail(SFA_ERR_NULLPTR, "a required tensor pointer is NULL");
    if (shape->layout == SFA_LAYOUT_TND && (!actual_seq_lengths_q || !actual_seq_lengths_kv))
        return nfail(SFA_ERR_NULLPTR, "TND needs actual_seq_lengths_q and actual_seq_lengths_kv");
    if (!(scale == scale)) return nfail(SFA_ERR_INVALID, "scale is NaN");
    const int64_t T1 = shape->layout == SFA_LAYOUT_BSND ? shape->B * shape->S1 : shape->T1;
    const int64_t T2 = shape->layout == SFA_LAYOUT_BSND ? shape->B * shape->S2 : shape->T2;
    const bool det = deterministic != 0;
    const GradWs ws = grad_ws_layout(T1, T2, shape->N1, shape->topk, sparse_block_size, det, false);
    if (ws.total > kNoAllocScratchBytes)
        return nfail(SFA_ERR_WORKSPACE,
                     "problem needs %zu bytes of scratch; sfa_grad_noalloc is limited to %zu bytes "
                     "(use sfa_grad with a caller workspace)",
                     ws.total, kNoAllocScratchBytes);
    void* scratch = nullptr;
    if ((st = scratch_for_current_device(&scratch)) != SFA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    char* w = (char*)scratch;

    GradArgs a;
    memset(&a, 0, sizeof a);
    a.q = query; a.qr = query_rope; a.k = key; a.kr = key_rope; a.v = value;
    a.dout = d_out; a.out = out; a.smax = softmax_max; a.ssum = softmax_sum; a.idx = sparse_indices;
    a.sd.layout = shape->layout; a.sd.B = (int32_t)shape->B; a.sd.S1 = shape->S1; a.sd.S2 = shape->S2;
    a.sd.T1 = T1; a.sd.T2 = T2; a.sd.seq_q = actual_seq_lengths_q; a.sd.seq_kv = actual_seq_lengths_kv;
    a.N1 = shape->N1; a.topk = shape->topk; a.bs = (int)sparse_block_size; a.mode = (int)sparse_mode;
    a.scale = scale; a.det = det;
    a.blocks = (int32_t*)(w + ws.blocks); a.nblk = (int32_t*)(w + ws.nblk); a.nrows = (int32_t*)(w + ws.nrows);
    a.order = (int32_t*)(w + ws.order); a.rowsum = (float*)(w + ws.rowsum);
    a.dkv_acc = w + ws.dkv; a.dq_acc = nullptr; a.ctrl = (int32_t*)(w + ws.ctrl);
    a.dq = d_query; a.dqr = d_query_rope;
    a.dtype = shape->dtype; a.rowlist = nullptr; a.rowcap = 0;
    a.row_begin = 0; a.row_end = T1;
    float* dmax = (float*)(w + ws.ctrl + kCtrlDmax);  // max|dOut|: the deterministic fixed-point grid
    a.dout_absmax = dmax;

    cudaError_t e;
    // the accumulator must start at zero; the rest of the scratch is fully rewritten
    if ((e = cudaMemsetAsync(w + ws.ctrl, 0, 256, s)) != cudaSuccess)
        return nfail(SFA_ERR_CUDA, "clear scratch: %s", cudaGetErrorString(e));
    if ((e = cudaMemsetAsync(a.dkv_acc, 0, (size_t)T2 * kAccW * (det ? 8 : 4), s)) != cudaSuccess)
        return nfail(SFA_ERR_CUDA, "clear scratch: %s", cudaGetErrorString(e));
    if ((e = launch_compact(sparse_indices, a.sd, a.topk, a.bs, a.mode, (int32_t*)a.blocks, (int32_t*)a.nblk,
                            (int32_t*)a.nrows, 0, T1, s)) != cudaSuccess)
        return nfail(SFA_ERR_CUDA, "index compaction: %s", cudaGetErrorString(e));
    if (det && (e = launch_absmax(shape->dtype, d_out, T1 * shape->N1 * kD, dmax, s)) != cudaSuccess)
        return nfail(SFA_ERR_CUDA, "max|dOut|: %s", cudaGetErrorString(e));
    if ((e = launch_bwd_generic(shape->dtype, a, s)) != cudaSuccess)
        return nfail(SFA_ERR_CUDA, "backward: %s", cudaGetErrorString(e));
    if ((e = launch_cast_dkv(shape->dtype, det, a.dkv_acc, T2, d_key, d_key_rope, d_value, s, dmax, scale, T1,
                             shape->N1)) != cudaSuccess)
        return nfail(SFA_ERR_CUDA, "cast dKey/dValue: %s", cudaGetErrorString(e));
    return SFA_OK;
}

}  // extern "C"
