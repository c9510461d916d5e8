// Internal declarations shared by the libsfa translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/sfa.h"

namespace sfa {

constexpr int kD = 512;    // latent head dim (SparseFlashAttentionGrad 约束说明: D only 512)
constexpr int kDr = 64;    // rope dim (Drope only 64)
constexpr int kDK = kD + kDr;   // 576: width of a gathered key row [key || keyRope]
constexpr int kAccW = kDK + kD; // 1088: fp32/int64 accumulator row = [dKey | dKeyRope | dValue]

// ---------------------------------------------------------------------------
// Deterministic scatter: 64-bit fixed point with a per-call power-of-two scale.
//
// A key-side gradient element is a sum over query rows t and heads h of
// P[t,h,j] * dO[t,h,d] (dValue) or scale * dS[t,h,j] * Q~[t,h,d] (dKey); a
// query-side FA element (dQ) a sum over keys of scale * dS * K.  With the
// forward's statistics every (t,h) has sum_j P = 1, so
//   |dValue| <= T1 * G * max|dO|                       (G = heads per key head)
//   |dKey|   <= T1 * G * max|dO| * |scale| * C,  |dQ| <= max|dO| * |scale| * C,
// where C = (||dO_th|| / max|dO|) * (||V_j|| + ||O_th||) * max|Q~| (or max|K|)
// is about 2^12.3 for D = 512 with N(0,1) activations.  Each contribution is
// rounded to the grid 2^-e with
//   e_V = 54 - L - E(max|dO|)              L = ceil(log2(T1 * G))
//   e_K = 42 - L - E(max|dO|) - E(|scale|),  e_Q = 42 - E(max|dO|) - E(|scale|)
// (E(x) = the least k with x <= 2^k), which leaves 2^8 of headroom below the
// 2^62 range for dValue (a sum of P up to 256 per row) and about 2^11 for
// dKey / dQ beyond the N(0,1) case.  The grid follows max|dO|, so a gradient
// scaled by 2^k gives results scaled by exactly 2^k: the relative precision does
// not depend on the scale of dOut.  Integer addition is associative, so the
// result does not depend on the order of the atomics.
// ---------------------------------------------------------------------------
__host__ __device__ inline int ceil_log2_pos(double x) {
    // least k with x <= 2^k (x > 0, finite); 0 for zero, negative or non-finite x
    if (!(x > 0.0) || !(x < 1e300)) return 0;
    int k = 0;
    const double m = frexp(x, &k);  // x = m * 2^k, m in [0.5, 1)
    return m == 0.5 ? k - 1 : k;
}
__host__ __device__ inline int fix_clamp(int e) { return e < -60 ? -60 : (e > 100 ? 100 : e); }
struct FixExp {
    int k, v, q;  // fraction bits of dKey (and dKeyRope), dValue, FA dQ
};
__host__ __device__ inline FixExp fix_exponents(float dout_absmax, float scale, int64_t T1, int64_t G) {
    const int L = ceil_log2_pos((double)T1 * (double)(G > 0 ? G : 1));
    const int ed = ceil_log2_pos((double)dout_absmax);
    const int es = ceil_log2_pos(fabs((double)scale));
    FixExp f;
    f.v = fix_clamp(54 - L - ed);
    f.k = fix_clamp(42 - L - ed - es);
    f.q = fix_clamp(42 - ed - es);
    return f;
}
// 2^e as a float (exact for the clamped range) and its inverse as a double
__host__ __device__ inline float fix_mul(int e) { return ldexpf(1.0f, e); }
__host__ __device__ inline double fix_inv(int e) { return ldexp(1.0, -e); }
__device__ __forceinline__ unsigned long long fix_round(float v, float mul) {
    return (unsigned long long)__float2ll_rn(v * mul);
}

// Largest |x| over `n` 16-bit elements, max-merged into *absmax (a non-negative
// fp32 value compared as its bit pattern; *absmax starts at 0).
cudaError_t launch_absmax(int dtype, const void* x, int64_t n, float* absmax, cudaStream_t st);

// ---------------------------------------------------------------------------
// 16-bit element access
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f<__half>(__half x) { return __half2float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

// ---------------------------------------------------------------------------
// Query row -> batch / sequence span
// ---------------------------------------------------------------------------
struct SeqDesc {
    int32_t layout;   // SFA_LAYOUT_BSND | SFA_LAYOUT_TND
    int32_t B;
    int64_t S1, S2;   // BSND padded lengths
    int64_t T1, T2;
    const int32_t* seq_q;   // BSND: per-batch lengths or null; TND: cumulative ends
    const int32_t* seq_kv;
};

struct TokInfo {
    int64_t kv_start;  // first key row of the span in the flattened [T2] view
    int32_t pos;       // position of the query inside its span
    int32_t q_len;     // S1_b
    int32_t kv_len;    // S2_b (clamped to the tensor)
    bool valid;        // false for BSND padding rows / rows beyond the TND total
};

__device__ __forceinline__ int64_t clamp64(int64_t x, int64_t lo, int64_t hi) {
    return x < lo ? lo : (x > hi ? hi : x);
}

// Inconsistent lengths are clamped into the tensors, never trusted for addressing.
__device__ __forceinline__ TokInfo tok_info(const SeqDesc& s, int64_t t) {
    TokInfo r;
    if (s.layout == SFA_LAYOUT_BSND) {
        int64_t b = t / s.S1;
        r.pos = (int32_t)(t - b * s.S1);
        int64_t lq = s.seq_q ? clamp64(s.seq_q[b], 0, s.S1) : s.S1;
        int64_t lk = s.seq_kv ? clamp64(s.seq_kv[b], 0, s.S2) : s.S2;
        r.q_len = (int32_t)lq;
        r.kv_len = (int32_t)lk;
        r.kv_start = b * s.S2;
        r.valid = r.pos < lq;
        return r;
    }
    // TND: first b with cum_q[b] > t
    int lo = 0, hi = s.B;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)s.seq_q[mid] > t) hi = mid; else lo = mid + 1;
    }
    if (lo >= s.B) { r.valid = false; r.pos = 0; r.q_len = 0; r.kv_len = 0; r.kv_start = 0; return r; }
    int b = lo;
    int64_t qs = b ? clamp64(s.seq_q[b - 1], 0, s.T1) : 0;
    int64_t qe = clamp64(s.seq_q[b], 0, s.T1);
    int64_t ks = b ? clamp64(s.seq_kv[b - 1], 0, s.T2) : 0;
    int64_t ke = clamp64(s.seq_kv[b], 0, s.T2);
    r.pos = (int32_t)(t - qs);
    r.q_len = (int32_t)(qe > qs ? qe - qs : 0);
    r.kv_start = ks;
    r.kv_len = (int32_t)(ke > ks ? ke - ks : 0);
    r.valid = t >= qs && t < qe;
    return r;
}

// Number of leading rows of block `blk` (bs rows) a query keeps: rows past S2_b
// and, in sparse mode 3, rows past pos + S2_b - S1_b are dropped.
__device__ __forceinline__ int block_rows(int64_t blk, int bs, const TokInfo& ti, int mode) {
    int64_t start = blk * (int64_t)bs;
    int64_t end = start + bs;
    if (end > ti.kv_len) end = ti.kv_len;
    if (mode == 3) {
        int64_t lim = (int64_t)ti.pos + ti.kv_len - ti.q_len;  // last kept row
        if (end > lim + 1) end = lim + 1;
    }
    int64_t n = end - start;
    return n > 0 ? (int)n : 0;
}

// ---------------------------------------------------------------------------
// Workspace layout of sfa_grad
// ---------------------------------------------------------------------------
struct GradWs {
    size_t dkv;     // [T2][1088] fp32 (atomic) or int64 (deterministic)
    size_t dq;      // [kMaxFusedGrid][N1][576] fp32 per-CTA dQ~ partial sums, fused path only
    size_t blocks;  // [T1][topk] int32 compacted block indices
    size_t nblk;    // [T1] int32
    size_t nrows;   // [T1] int32
    size_t order;   // [T1] int32 work order (longest first)
    size_t rowsum;  // [T1][N1] fp32 FlashSoftmaxGrad
    size_t rowlist; // [T1][topk*bs] int32 gathered key rows, fused path only
    size_t pflags;  // [T1/2+1] int32 flags of the candidate pairs (2m, 2m+1) (N1 = 128 fused path)
    size_t pairs;   // [T1/2+1] int32 first rows of the row pairs (N1 = 128 fused path)
    size_t ctrl;    // 256 B of counters / flags (offset 0: the device error word)
    size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Offset of the fp32 max|dOut| inside a workspace's 256-byte control area (the
// error word is at offset 0; the area is zeroed at the start of every call).
constexpr size_t kCtrlDmax = 128;
// Offset of the int32 [2] (row pairs, remaining rows) counts of the paired backward.
constexpr size_t kCtrlCounts = 64;

constexpr int kMaxFusedGrid = 256;  // persistent CTAs of the fused kernel (one per SM)

inline GradWs grad_ws_layout(int64_t T1, int64_t T2, int64_t N1, int64_t topk, int64_t bs, bool det, bool fused) {
    GradWs w;
    size_t o = 0;
    w.ctrl = o;   o = 256;  // error word first: sfa_workspace_status reads offset 0
    w.dkv = o;    o = align256(o + (size_t)T2 * kAccW * (det ? 8 : 4));
    w.dq = o;     o = align256(o + (fused ? (size_t)kMaxFusedGrid * N1 * kDK * 4 : 0));
    w.blocks = o; o = align256(o + (size_t)T1 * topk * 4);
    w.nblk = o;   o = align256(o + (size_t)T1 * 4);
    w.nrows = o;  o = align256(o + (size_t)T1 * 4);
    w.order = o;  o = align256(o + (size_t)T1 * 4);
    w.rowsum = o; o = align256(o + (size_t)T1 * N1 * 4);
    w.rowlist = o; o = align256(o + (fused ? (size_t)T1 * topk * bs * 4 : 0));
    const bool pair = fused && N1 == 128;
    w.pflags = o;  o = align256(o + (pair ? (size_t)(T1 / 2 + 1) * 4 : 0));
    w.pairs = o;   o = align256(o + (pair ? (size_t)(T1 / 2 + 1) * 4 : 0));
    w.total = o;
    return w;
}

// Workspace layout of sfa_fwd (the expanded row lists, order and control word only
// on the tensor-core path, N1 = 128)
struct FwdWs {
    size_t blocks, nblk, nrows, order, rowlist, nslots, ctrl, total;
};
inline FwdWs fwd_ws_layout(int64_t T1, int64_t N1, int64_t topk, int64_t bs) {
    FwdWs w;
    const bool fused = N1 == 128;
    size_t o = 0;
    w.ctrl = o;    o = 256;  // error word first
    w.blocks = o;  o = align256(o + (size_t)T1 * topk * 4);
    w.nblk = o;    o = align256(o + (size_t)T1 * 4);
    w.nrows = o;   o = align256(o + (size_t)T1 * 4);
    w.order = o;   o = align256(o + (fused ? (size_t)T1 * 4 : 0));
    w.rowlist = fused ? o : 0; o = align256(o + (fused ? (size_t)T1 * topk * bs * 4 : 0));
    w.nslots = o;  o = align256(o + (fused ? (size_t)T1 * 4 : 0));
    w.total = o;
    return w;
}

// ---------------------------------------------------------------------------
// Launchers (defined in the .cu files; all return cudaGetLastError())
// ---------------------------------------------------------------------------
// index compaction of query rows [row_begin, row_end) (only those rows' indices are read and
// only their entries of blocks / nblk / nrows written)
cudaError_t launch_compact(const int32_t* idx, const SeqDesc& sd, int64_t topk, int bs, int mode, int32_t* blocks,
                           int32_t* nblk, int32_t* nrows, int64_t row_begin, int64_t row_end, cudaStream_t st);
// rowsum(dO o O) of query rows [row_begin, row_end) (rows outside are not written)
// (when `absmax` is non-null, max|dO| over the range is max-merged into it too)
cudaError_t launch_rowsum(int dtype, const void* dout, const void* out, int64_t row_begin, int64_t row_end, int64_t N1,
                          float* rowsum, cudaStream_t st, float* absmax = nullptr);
// work order of the fused kernel over query rows [row_begin, row_end) (row_end - row_begin entries)
cudaError_t launch_order(const int32_t* nrows, int64_t row_begin, int64_t row_end, int32_t* order, int32_t* ctrl,
                         cudaStream_t st);
// Sorts the kept block indices of rows [row_begin, row_end) ascending, in place
// (topk <= kSortMaxTopk: the row is sorted in shared memory).
constexpr int64_t kSortMaxTopk = 4096;
cudaError_t launch_sort_blocks(int32_t* blocks, const int32_t* nblk, int64_t topk, int64_t row_begin, int64_t row_end,
                               cudaStream_t st);
// key-row lists of query rows [row_begin, row_end)
cudaError_t launch_expand(const int32_t* blocks, const int32_t* nblk, const SeqDesc& sd, int64_t topk, int bs, int mode,
                          int64_t cap, int32_t* rowlist, int64_t row_begin, int64_t row_end, cudaStream_t st);
// block-aligned key-row lists for sparse_block_size % 16 == 0 (invalid slots: bit 31 set)
cudaError_t launch_expand_blocks(const int32_t* blocks, const int32_t* nblk, const SeqDesc& sd, int64_t topk, int bs,
                                 int mode, int64_t cap, int32_t* rowlist, int32_t* nslots, cudaStream_t st);
// det: the fixed-point grid follows fix_exponents(*dout_absmax, scale, T1, N1)
cudaError_t launch_cast_dkv(int dtype, bool det, const void* acc, int64_t T2, void* dk, void* dkr, void* dv,
                            cudaStream_t st, const float* dout_absmax = nullptr, float scale = 1.f, int64_t T1 = 1,
                            int64_t N1 = 1);
cudaError_t launch_cast_dq(int dtype, const float* acc, int64_t T1, int64_t N1, void* dq, void* dqr,
                           cudaStream_t st);

struct GradArgs {
    const void* q; const void* qr; const void* k; const void* kr; const void* v;
    const void* dout; const void* out; const float* smax; const float* ssum;
    const int32_t* idx; SeqDesc sd; int64_t N1; int64_t topk; int bs; int mode; float scale; bool det;
    const int32_t* blocks; const int32_t* nblk; const int32_t* nrows; const int32_t* order;
    const float* rowsum; void* dkv_acc; float* dq_acc; int32_t* ctrl;
    void* dq; void* dqr;
    int dtype; const int32_t* rowlist; int64_t rowcap;
    int64_t row_begin, row_end;  // query rows [row_begin, row_end) of the flattened [T1] view are processed
    const float* dout_absmax;    // deterministic mode: max|dOut| over every row added into dkv_acc (device)
    const int32_t* nwork_dev;    // fused kernel: when set, the device count of `order` entries to process
};

// Paired-row tensor-core backward (N1 = 128, value == key): rows t, t + 1 of each pair share
// their kept blocks; the two CTAs of a cluster exchange P / dS (sfa_pair.cu).
struct PairArgs {
    const void* q; const void* qr; const void* k; const void* kr; const void* dout;
    SeqDesc sd; int64_t topk; int bs; int mode; float scale; bool det; int dtype;
    const int32_t* blocks; const int32_t* nblk;
    const int32_t* pairs; const int32_t* npairs;  // first rows of the pairs, device count
    const float* smax; const float* ssum; const float* rowsum;
    void* dkv_acc; float* dq_acc; void* dq; void* dqr; int* err;
    const float* dout_absmax;
};
// Pairs of rows (2m, 2m + 1) inside [row_begin, row_end) with identical non-empty block lists in
// one batch / sequence; pair first rows and the other rows listed in descending order, counts
// [pairs, rows] in counts[0..1] (device).  `flags` holds one entry per candidate pair.
cudaError_t launch_pair_lists(const int32_t* blocks, const int32_t* nblk, const SeqDesc& sd, int64_t topk,
                              int64_t row_begin, int64_t row_end, int32_t* flags, int32_t* pairs, int32_t* solo,
                              int32_t* counts, cudaStream_t st);
cudaError_t launch_bwd_pair(int dtype, const PairArgs& a, cudaStream_t st);
cudaError_t launch_bwd_generic(int dtype, const GradArgs& a, cudaStream_t st);
cudaError_t launch_bwd_fused(int dtype, const GradArgs& a, cudaStream_t st);
bool fused_supported(int64_t N1);

struct FwdArgs {
    const void* q; const void* qr; const void* k; const void* kr; const void* v;
    SeqDesc sd; int64_t N1; int64_t topk; int bs; int mode; float scale;
    const int32_t* blocks; const int32_t* nblk;
    void* out; float* smax; float* ssum;
};
cudaError_t launch_fwd_generic(int dtype, const FwdArgs& a, cudaStream_t st);

// Tensor-core forward (N1 = 128, value == key) over the expanded key-row lists.
struct FwdFusedArgs {
    const void* q; const void* qr; const void* k; const void* kr;
    const int32_t* rowlist; const int32_t* nrows; const int32_t* order;
    void* out; float* smax; float* ssum; int* err;
    int64_t T1, T2, rowcap; float scale; int dtype;
    int blk16;  // row lists are block-aligned runs of 16 contiguous rows (nrows = slots; invalid slots: bit 31)
};
bool fwd_fused_supported(int64_t N1);
cudaError_t launch_fwd_fused(int dtype, const FwdFusedArgs& a, cudaStream_t st);

struct FaArgs {
    const void* q; const void* k; const void* v; const void* dy; const void* o;
    const float* smax; const float* ssum;  // [T1][Nq][8]
    const int64_t* cu_q; const int64_t* cu_kv;  // device copies, length B
    int64_t B, T1, T2, Nq, Nkv, D; int mode; float scale; bool det;
    void* dkv_acc;  // [2][T2][Nkv][D] fp32 or int64
    void* dq; void* dk; void* dv;
    void* out; float* smax_out; float* ssum_out;
    const float* dout_absmax;  // deterministic mode: max|dY| (device)
};
cudaError_t launch_fa_bwd(int dtype, const FaArgs& a, cudaStream_t st);

// Tensor-core dense backward (head dims 64 and 128): work list of (sequence, kv head,
// 128-key block) items, built on the host and copied into the workspace.
struct FaFusedArgs {
    const void* q; const void* k; const void* v; const void* dy; const void* o;
    const float* smax; const float* ssum;
    const int64_t* cu_q; const int64_t* cu_kv;
    int64_t B, T1, T2, Nq, Nkv, D; int mode; float scale; bool det; int dtype;
    const void* items; int nitems;
    float* rowsum;   // [T1][Nq]
    void* dq_acc;    // [T1][Nq][D] fp32 or int64 (zeroed by the caller)
    int* err;
    void* dq; void* dk; void* dv;
    const float* dout_absmax;  // deterministic mode: max|dY| (device)
};
bool fa_fused_supported(int64_t D);
// Builds the work list (4 int32 per item) for the given host cumulative lengths
// (when `out` is non-null) and returns the number of items.
size_t fa_fused_items(const int64_t* cu_q, const int64_t* cu_kv, int64_t B, int64_t Nq, int64_t Nkv, int mode,
                      std::vector<int32_t>* out);
inline size_t fa_fused_max_items(int64_t B, int64_t T2, int64_t Nkv) { return (size_t)Nkv * (T2 / 128 + B + 1); }
cudaError_t launch_fa_bwd_fused(int dtype, const FaFusedArgs& a, cudaStream_t st);
// Sets the message returned by sfa_last_error_string() on the calling thread.
// ---------------------------------------------------------------------------
// Dense lightning-indexer gradient with KL loss (DenseLightningIndexerGradKLLoss)
constexpr int kLigG = 64;    // indexer query heads the fused kernel supports
constexpr int kLigDi = 128;  // indexer head dim the fused kernel supports
struct LigArgs {
    const void *q, *qr, *k, *kr, *qi, *ki, *weights;
    const float *smax, *ssum, *smax_i, *ssum_i;
    const int32_t *nkeys, *kvrow, *order;
    float* dki_acc;   // [T2][Di] fp32, zeroed by the caller
    float* loss_rows; // [T1]
    void *dqi, *dw;
    int* err;
    int64_t T1, T2, N1;
    float scale;
    int dtype;
};
// Row bookkeeping: int64 sequence lengths (null for BSND full lengths) copied to
// int32, then per query row its visible key count and first key row.
cudaError_t launch_lig_prep(const SeqDesc& sd, int mode, const int64_t* sq64, const int64_t* skv64, int32_t* sq32,
                            int32_t* skv32, int32_t* nkeys, int32_t* kvrow, cudaStream_t st);
cudaError_t launch_lig_fused(const LigArgs& a, cudaStream_t st);
// dKeyIndex from the fp32 accumulator, and the loss as the fixed-order sum of the rows' losses.
cudaError_t launch_lig_finish(int dtype, const float* dki_acc, int64_t T2, void* dki, const float* loss_rows,
                              int64_t T1, float* loss, cudaStream_t st);

void set_last_error(const char* msg);
// Limit of every device-side mbarrier wait of the fused kernels launched from the
// calling thread (sfa_set_wait_limit; 4 s by default).
uint64_t wait_limit_ns();
cudaError_t launch_fa_fwd(int dtype, const FaArgs& a, cudaStream_t st);

}  // namespace sfa
