// Preparation and finishing kernels of the sparse attention backward:
//   - index compaction (the Gather of SparseFlashAttentionGrad README, 功能说明, with
//     the sparseMode 3 mask of 约束说明),
//   - FlashSoftmaxGrad(dO, O) = rowsum(dO o O) of stage 2,
//   - the work order of the fused kernel,
//   - the final fp32 / fixed-point -> 16-bit casts of the scattered gradients.
#include "sfa_internal.cuh"

namespace sfa {

// One warp per query row of [row_begin, row_end): keep the valid block indices in their original
// order (no other row's indices are read).
__global__ void compact_kernel(const int32_t* __restrict__ idx, SeqDesc sd, int64_t topk, int bs, int mode,
                               int32_t* __restrict__ blocks, int32_t* __restrict__ nblk,
                               int32_t* __restrict__ nrows, int64_t row_begin, int64_t row_end) {
    const int lane = threadIdx.x & 31;
    const int64_t t = row_begin + (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= row_end) return;
    TokInfo ti = tok_info(sd, t);
    int count = 0, rows = 0;
    if (ti.valid) {
        const int32_t* src = idx + t * topk;
        int32_t* dst = blocks + t * topk;
        for (int64_t c = 0; c < topk; c += 32) {
            int64_t i = c + lane;
            int n = 0;
            int32_t b = -1;
            if (i < topk) {
                b = src[i];
                if (b >= 0) n = block_rows(b, bs, ti, mode);
            }
            // a block is kept iff it has at least one row before the cuts
            bool keep = n > 0;
            unsigned m = __ballot_sync(0xffffffffu, keep);
            int before = __popc(m & ((1u << lane) - 1u));
            if (keep) dst[count + before] = b;
            count += __popc(m);
            rows += n;
        }
    }
    for (int o = 16; o; o >>= 1) rows += __shfl_xor_sync(0xffffffffu, rows, o);
    if (lane == 0) {
        nblk[t] = count;
        nrows[t] = rows;
    }
}

cudaError_t launch_compact(const int32_t* idx, const SeqDesc& sd, int64_t topk, int bs, int mode, int32_t* blocks,
                           int32_t* nblk, int32_t* nrows, int64_t row_begin, int64_t row_end, cudaStream_t st) {
    const int warps = 8;
    int64_t grid = (row_end - row_begin + warps - 1) / warps;
    if (grid > 0)
        compact_kernel<<<(unsigned)grid, warps * 32, 0, st>>>(idx, sd, topk, bs, mode, blocks, nblk, nrows, row_begin,
                                                              row_end);
    return cudaGetLastError();
}

// Max-merge of a non-negative float into *dst: for x >= 0 the IEEE bit patterns
// order like the values, so an unsigned atomicMax on the bits is a float max.
__device__ __forceinline__ void absmax_merge(float* dst, float x) {
    atomicMax(reinterpret_cast<unsigned int*>(dst), __float_as_uint(x));
}

// Block-wide max of one value per thread (every thread gets the result in lane 0 of warp 0).
__device__ __forceinline__ float block_max(float v) {
    __shared__ float red[32];
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    if (w == 0) {
        v = l < (int)(blockDim.x >> 5) ? red[l] : 0.f;
        for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    }
    return v;
}

// One warp per (row, head): sum over the 512 value dims of dO * O in fp32.
// Grid-stride over the rows; with `absmax` set, max|dO| is max-merged into it
// (one atomic per CTA).
template <typename T>
__global__ void rowsum_kernel(const T* __restrict__ dout, const T* __restrict__ out, int64_t rows,
                              float* __restrict__ res, float* __restrict__ absmax) {
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    float am = 0.f;
    for (int64_t r = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += (int64_t)gridDim.x * wpb) {
        const uint4* a = reinterpret_cast<const uint4*>(dout + r * kD);
        const uint4* b = reinterpret_cast<const uint4*>(out + r * kD);
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < kD / 8 / 32; ++c) {
            uint4 x = a[c * 32 + lane], y = b[c * 32 + lane];
            const T* xp = reinterpret_cast<const T*>(&x);
            const T* yp = reinterpret_cast<const T*>(&y);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float xv = to_f(xp[e]);
                s = fmaf(xv, to_f(yp[e]), s);
                am = fmaxf(am, fabsf(xv));
            }
        }
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) res[r] = s;
    }
    if (absmax) {
        am = block_max(am);
        if (threadIdx.x == 0) absmax_merge(absmax, am);
    }
}

cudaError_t launch_rowsum(int dtype, const void* dout, const void* out, int64_t row_begin, int64_t row_end, int64_t N1,
                          float* rowsum, cudaStream_t st, float* absmax) {
    const int64_t rows = (row_end - row_begin) * N1;
    const int64_t first = row_begin * N1;  // (row, head) pairs before the range
    const size_t elem = 2;                  // bf16 / fp16
    dout = (const char*)dout + first * kD * elem;
    out = (const char*)out + first * kD * elem;
    rowsum += first;
    const int warps = 8;
    if (rows == 0) return cudaGetLastError();
    int64_t need = (rows + warps - 1) / warps;
    unsigned grid = (unsigned)(need < 148 * 16 ? need : 148 * 16);
    if (dtype == SFA_DTYPE_BF16)
        rowsum_kernel<__nv_bfloat16><<<grid, warps * 32, 0, st>>>((const __nv_bfloat16*)dout,
                                                                  (const __nv_bfloat16*)out, rows, rowsum, absmax);
    else
        rowsum_kernel<__half><<<grid, warps * 32, 0, st>>>((const __half*)dout, (const __half*)out, rows, rowsum,
                                                           absmax);
    return cudaGetLastError();
}

// max|x| over n 16-bit elements (8 per 16-byte load, then a scalar tail).
template <typename T>
__global__ void absmax_kernel(const T* __restrict__ x, int64_t n, float* __restrict__ absmax) {
    float am = 0.f;
    const int64_t nv = n / 8;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
        const uint4 u = xv[i];
        const T* p = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(to_f(p[e])));
    }
    for (int64_t i = nv * 8 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        am = fmaxf(am, fabsf(to_f(x[i])));
    am = block_max(am);
    if (threadIdx.x == 0) absmax_merge(absmax, am);
}

cudaError_t launch_absmax(int dtype, const void* x, int64_t n, float* absmax, cudaStream_t st) {
    if (n <= 0) return cudaGetLastError();
    int64_t need = (n / 8 + 255) / 256;
    unsigned grid = (unsigned)(need < 1 ? 1 : (need < 148 * 8 ? need : 148 * 8));
    if (dtype == SFA_DTYPE_BF16)
        absmax_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, n, absmax);
    else
        absmax_kernel<__half><<<grid, 256, 0, st>>>((const __half*)x, n, absmax);
    return cudaGetLastError();
}

// Work order for the persistent fused kernel: later rows first (under the causal
// masks they carry the most keys, so the largest work items start first).
__global__ void order_kernel(int64_t row_begin, int64_t row_end, int32_t* __restrict__ order,
                             int32_t* __restrict__ ctrl) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    (void)ctrl;
    if (i < row_end - row_begin) order[i] = (int32_t)(row_end - 1 - i);
}

cudaError_t launch_order(const int32_t* nrows, int64_t row_begin, int64_t row_end, int32_t* order, int32_t* ctrl,
                         cudaStream_t st) {
    (void)nrows;
    const int64_t cnt = row_end - row_begin;
    int64_t n = cnt > 64 ? cnt : 64;
    order_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(row_begin, row_end, order, ctrl);
    return cudaGetLastError();
}

// Expand each query row's compacted block list into its gathered key rows
// (global row ids, in index order), one warp per query row.
__global__ void expand_kernel(const int32_t* __restrict__ blocks, const int32_t* __restrict__ nblk, SeqDesc sd,
                              int64_t topk, int bs, int mode, int64_t cap, int32_t* __restrict__ rowlist,
                              int64_t row_begin, int64_t row_end) {
    const int lane = threadIdx.x & 31;
    const int64_t t = row_begin + (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= row_end) return;
    const TokInfo ti = tok_info(sd, t);
    const int nb = nblk[t];
    int32_t* dst = rowlist + t * cap;
    int64_t base = 0;
    for (int c = 0; c < nb; c += 32) {
        const int i = c + lane;
        const int64_t blk = i < nb ? blocks[t * topk + i] : 0;
        const int n = i < nb ? block_rows(blk, bs, ti, mode) : 0;
        int x = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const int total = __shfl_sync(0xffffffffu, x, 31);
        const int64_t first = ti.kv_start + blk * bs;
        for (int r = 0; r < n; ++r) dst[base + (x - n) + r] = (int32_t)(first + r);
        base += total;
    }
}

// Block-aligned expansion (sparse_block_size a multiple of 16): block i of row t
// takes slots [i*bs, i*bs+bs) with the block's consecutive rows, so every
// 16-slot group is one run of contiguous key rows (loadable as one 2-D tile);
// slots past the block's kept rows (sequence end, causal bound) hold the row id
// with bit 31 set.  nslots[t] = blocks x bs.
__global__ void expand_blocks_kernel(const int32_t* __restrict__ blocks, const int32_t* __restrict__ nblk, SeqDesc sd,
                                     int64_t topk, int bs, int mode, int64_t cap, int32_t* __restrict__ rowlist,
                                     int32_t* __restrict__ nslots) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= sd.T1) return;
    const TokInfo ti = tok_info(sd, t);
    const int nb = nblk[t];
    int32_t* dst = rowlist + t * cap;
    for (int i = 0; i < nb; ++i) {
        const int64_t blk = blocks[t * topk + i];
        const int keep = block_rows(blk, bs, ti, mode);
        const int64_t first = ti.kv_start + blk * bs;
        for (int o = lane; o < bs; o += 32)
            dst[(int64_t)i * bs + o] = (int32_t)((uint32_t)(first + o) | (o < keep ? 0u : 0x80000000u));
    }
    if (lane == 0) nslots[t] = (int32_t)(nb * bs);
}

cudaError_t launch_expand_blocks(const int32_t* blocks, const int32_t* nblk, const SeqDesc& sd, int64_t topk, int bs,
                                 int mode, int64_t cap, int32_t* rowlist, int32_t* nslots, cudaStream_t st) {
    const int warps = 8;
    const int64_t grid = (sd.T1 + warps - 1) / warps;
    if (grid > 0)
        expand_blocks_kernel<<<(unsigned)grid, warps * 32, 0, st>>>(blocks, nblk, sd, topk, bs, mode, cap, rowlist,
                                                                    nslots);
    return cudaGetLastError();
}

// Sorts each query row's kept block indices ascending (rows [row_begin, row_end)).
// The sum over a row's keys does not depend on their order; sorted, the
// expanded key rows form runs of consecutive rows, and a tile of 128 of them is
// loaded as one 2-D tile instead of 32 four-row gathers.  One CTA per row, a
// bitonic network over the next power of two >= the row's count in shared memory
// (padding sorts last).
__global__ void sort_blocks_kernel(int32_t* __restrict__ blocks, const int32_t* __restrict__ nblk, int64_t topk,
                                   int64_t row_begin) {
    extern __shared__ int32_t v[];
    const int64_t t = row_begin + blockIdx.x;
    const int n = nblk[t];
    if (n <= 1) return;  // uniform over the CTA
    int p = 1;
    while (p < n) p <<= 1;
    int32_t* row = blocks + t * topk;
    for (int i = threadIdx.x; i < p; i += blockDim.x) v[i] = i < n ? row[i] : 0x7fffffff;
    __syncthreads();
    for (int k = 2; k <= p; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < p; i += blockDim.x) {
                const int l = i ^ j;
                if (l > i) {
                    const int32_t a = v[i], b = v[l];
                    if ((a > b) == ((i & k) == 0)) {
                        v[i] = b;
                        v[l] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < n; i += blockDim.x) row[i] = v[i];
}

cudaError_t launch_sort_blocks(int32_t* blocks, const int32_t* nblk, int64_t topk, int64_t row_begin, int64_t row_end,
                               cudaStream_t st) {
    if (row_end <= row_begin || topk <= 1) return cudaGetLastError();
    int p = 1;
    while (p < topk) p <<= 1;
    sort_blocks_kernel<<<(unsigned)(row_end - row_begin), 256, (size_t)p * 4, st>>>(blocks, nblk, topk, row_begin);
    return cudaGetLastError();
}

cudaError_t launch_expand(const int32_t* blocks, const int32_t* nblk, const SeqDesc& sd, int64_t topk, int bs, int mode,
                          int64_t cap, int32_t* rowlist, int64_t row_begin, int64_t row_end, cudaStream_t st) {
    const int warps = 8;
    int64_t grid = (row_end - row_begin + warps - 1) / warps;
    if (grid > 0)
        expand_kernel<<<(unsigned)grid, warps * 32, 0, st>>>(blocks, nblk, sd, topk, bs, mode, cap, rowlist, row_begin,
                                                             row_end);
    return cudaGetLastError();
}

// [T2][1088] accumulator -> dKey [T2][512], dKeyRope [T2][64], dValue [T2][512].
// Fixed point (deterministic mode) is scaled back by the call's grid (see fix_exponents).
template <typename T, bool DET>
__global__ void cast_dkv_kernel(const void* __restrict__ acc, int64_t T2, T* __restrict__ dk, T* __restrict__ dkr,
                                T* __restrict__ dv, const float* __restrict__ dmax, float scale, int64_t T1,
                                int64_t N1) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // group of 4 columns
    const int64_t per_row = kAccW / 4;
    if (i >= T2 * per_row) return;
    int64_t r = i / per_row;
    int c = (int)(i - r * per_row) * 4;
    float v[4];
    if (DET) {
        const FixExp fe = fix_exponents(*dmax, scale, T1, N1);
        const double inv = fix_inv(c < kDK ? fe.k : fe.v);  // a 4-column group never straddles 576
        const long long* a = reinterpret_cast<const long long*>(acc) + r * kAccW + c;
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = (float)((double)a[e] * inv);
    } else {
        float4 x = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(acc) + r * kAccW + c);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
    T* dst;
    if (c < kD) dst = dk + r * kD + c;
    else if (c < kDK) dst = dkr + r * kDr + (c - kD);
    else dst = dv + r * kD + (c - kDK);
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[e] = from_f<T>(v[e]);
}

cudaError_t launch_cast_dkv(int dtype, bool det, const void* acc, int64_t T2, void* dk, void* dkr, void* dv,
                            cudaStream_t st, const float* dmax, float scale, int64_t T1, int64_t N1) {
    int64_t n = T2 * (kAccW / 4);
    if (n == 0) return cudaGetLastError();
    if (det && !dmax) return cudaErrorInvalidValue;
    unsigned grid = (unsigned)((n + 255) / 256);
    if (dtype == SFA_DTYPE_BF16) {
        using T = __nv_bfloat16;
        if (det) cast_dkv_kernel<T, true><<<grid, 256, 0, st>>>(acc, T2, (T*)dk, (T*)dkr, (T*)dv, dmax, scale, T1, N1);
        else cast_dkv_kernel<T, false><<<grid, 256, 0, st>>>(acc, T2, (T*)dk, (T*)dkr, (T*)dv, dmax, scale, T1, N1);
    } else {
        using T = __half;
        if (det) cast_dkv_kernel<T, true><<<grid, 256, 0, st>>>(acc, T2, (T*)dk, (T*)dkr, (T*)dv, dmax, scale, T1, N1);
        else cast_dkv_kernel<T, false><<<grid, 256, 0, st>>>(acc, T2, (T*)dk, (T*)dkr, (T*)dv, dmax, scale, T1, N1);
    }
    return cudaGetLastError();
}

// [T1][N1][576] fp32 -> dQuery [T1][N1][512], dQueryRope [T1][N1][64].
template <typename T>
__global__ void cast_dq_kernel(const float* __restrict__ acc, int64_t rows, T* __restrict__ dq, T* __restrict__ dqr) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_row = kDK / 4;
    if (i >= rows * per_row) return;
    int64_t r = i / per_row;
    int c = (int)(i - r * per_row) * 4;
    float4 x = *reinterpret_cast<const float4*>(acc + r * kDK + c);
    T* dst = c < kD ? dq + r * kD + c : dqr + r * kDr + (c - kD);
    dst[0] = from_f<T>(x.x); dst[1] = from_f<T>(x.y); dst[2] = from_f<T>(x.z); dst[3] = from_f<T>(x.w);
}

cudaError_t launch_cast_dq(int dtype, const float* acc, int64_t T1, int64_t N1, void* dq, void* dqr,
                           cudaStream_t st) {
    int64_t rows = T1 * N1;
    int64_t n = rows * (kDK / 4);
    if (n == 0) return cudaGetLastError();
    unsigned grid = (unsigned)((n + 255) / 256);
    if (dtype == SFA_DTYPE_BF16)
        cast_dq_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(acc, rows, (__nv_bfloat16*)dq, (__nv_bfloat16*)dqr);
    else
        cast_dq_kernel<__half><<<grid, 256, 0, st>>>(acc, rows, (__half*)dq, (__half*)dqr);
    return cudaGetLastError();
}

}  // namespace sfa
