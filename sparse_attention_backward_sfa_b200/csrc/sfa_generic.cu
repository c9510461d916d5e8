// Warp-per-(query row, head) CUDA-core kernels for sparse attention.
//
// These serve every shape the fused tensor-core kernel does not (N1 < 64, value
// distinct from key) and the forward that produces `out` and the softmax
// statistics.  One warp owns one (row t, head h) pair; lane l holds dims
// l, l+32, ... of the 576-wide [q || qRope] row and of the 512-wide dO row.
//
// Backward per gathered key row j (SparseFlashAttentionGrad README, 功能说明):
//   s = scale * q~.k~_j, p = exp(s - softmaxMax) / softmaxSum,
//   dp = dO.v_j, ds = p * (dp - rowsum(dO o O))            (stages 1, 2)
//   dq~ += scale * ds * k~_j                                (stage 3, registers)
//   dk~_j += scale * ds * q~, dv_j += p * dO                (red to the fp32 or
//                                                           fixed-point accumulator)
#include "sfa_internal.cuh"

namespace sfa {

constexpr int kQC = kDK / 32;  // 18 chunks of the 576-wide row per lane
constexpr int kVC = kD / 32;   // 16 chunks of the 512-wide row per lane

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <bool DET>
__device__ __forceinline__ void scatter_add(void* acc, int64_t off, float x, float fmul) {
    if (DET) {
        atomicAdd(reinterpret_cast<unsigned long long*>(acc) + off, fix_round(x, fmul));
    } else {
        atomicAdd(reinterpret_cast<float*>(acc) + off, x);
    }
}

template <typename T, bool DET>
__global__ void __launch_bounds__(256) sfa_bwd_generic_kernel(GradArgs a) {
    const int lane = threadIdx.x & 31;
    // (row, head) pair within the processed rows [row_begin, row_end)
    const int64_t pair = a.row_begin * a.N1 + (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (pair >= a.row_end * a.N1) return;
    const int64_t t = pair / a.N1;
    const int h = (int)(pair - t * a.N1);
    const TokInfo ti = tok_info(a.sd, t);
    const T* q = (const T*)a.q + pair * kD;
    const T* qr = (const T*)a.qr + pair * kDr;
    const T* k = (const T*)a.k;
    const T* kr = (const T*)a.kr;
    const T* v = (const T*)a.v;
    float dq[kQC];
#pragma unroll
    for (int c = 0; c < kQC; ++c) dq[c] = 0.f;
    float fmul_k = 0.f, fmul_v = 0.f;  // fixed-point grids of dK~ and dV (deterministic mode)
    if (DET) {
        const FixExp fe = fix_exponents(*a.dout_absmax, a.scale, a.sd.T1, a.N1);
        fmul_k = fix_mul(fe.k);
        fmul_v = fix_mul(fe.v);
    }

    if (ti.valid) {
        float qv[kQC], dov[kVC];
#pragma unroll
        for (int c = 0; c < kVC; ++c) qv[c] = to_f(q[c * 32 + lane]);
#pragma unroll
        for (int c = kVC; c < kQC; ++c) qv[c] = to_f(qr[(c - kVC) * 32 + lane]);
        const T* dop = (const T*)a.dout + pair * kD;
        const T* op = (const T*)a.out + pair * kD;
        float dsum = 0.f;
#pragma unroll
        for (int c = 0; c < kVC; ++c) {
            dov[c] = to_f(dop[c * 32 + lane]);
            dsum = fmaf(dov[c], to_f(op[c * 32 + lane]), dsum);
        }
        dsum = warp_sum(dsum);  // FlashSoftmaxGrad(dO, O)
        const float m = a.smax[pair];
        const float l = a.ssum[pair];
        const float inv_l = l == 0.f ? 0.f : 1.f / l;
        const int nb = a.nblk[t];
        const int32_t* blist = a.blocks + t * a.topk;
        for (int ib = 0; ib < nb; ++ib) {
            const int64_t blk = blist[ib];
            const int nr = block_rows(blk, a.bs, ti, a.mode);
            for (int r = 0; r < nr; ++r) {
                const int64_t g = ti.kv_start + blk * a.bs + r;
                const T* kg = k + g * kD;
                const T* krg = kr + g * kDr;
                const T* vg = v + g * kD;
                float kv[kQC];
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int c = 0; c < kVC; ++c) {
                    kv[c] = to_f(kg[c * 32 + lane]);
                    s = fmaf(qv[c], kv[c], s);
                    dp = fmaf(dov[c], to_f(vg[c * 32 + lane]), dp);
                }
#pragma unroll
                for (int c = kVC; c < kQC; ++c) {
                    kv[c] = to_f(krg[(c - kVC) * 32 + lane]);
                    s = fmaf(qv[c], kv[c], s);
                }
                s = warp_sum(s) * a.scale;
                dp = warp_sum(dp);
                const float p = expf(s - m) * inv_l;
                const float ds = p * (dp - dsum);
                const float sds = a.scale * ds;
                void* acc = a.dkv_acc;
                const int64_t rowoff = g * kAccW;
#pragma unroll
                for (int c = 0; c < kQC; ++c) {
                    dq[c] = fmaf(ds, kv[c], dq[c]);
                    scatter_add<DET>(acc, rowoff + c * 32 + lane, sds * qv[c], fmul_k);
                }
#pragma unroll
                for (int c = 0; c < kVC; ++c) scatter_add<DET>(acc, rowoff + kDK + c * 32 + lane, p * dov[c], fmul_v);
            }
        }
    }
    T* dqo = (T*)a.dq + pair * kD;
    T* dqro = (T*)a.dqr + pair * kDr;
#pragma unroll
    for (int c = 0; c < kVC; ++c) dqo[c * 32 + lane] = from_f<T>(a.scale * dq[c]);
#pragma unroll
    for (int c = kVC; c < kQC; ++c) dqro[(c - kVC) * 32 + lane] = from_f<T>(a.scale * dq[c]);
    (void)h;
}

cudaError_t launch_bwd_generic(int dtype, const GradArgs& a, cudaStream_t st) {
    const int64_t pairs = (a.row_end - a.row_begin) * a.N1;
    if (pairs == 0) return cudaGetLastError();
    const int warps = 8;
    unsigned grid = (unsigned)((pairs + warps - 1) / warps);
    if (dtype == SFA_DTYPE_BF16) {
        if (a.det) sfa_bwd_generic_kernel<__nv_bfloat16, true><<<grid, warps * 32, 0, st>>>(a);
        else sfa_bwd_generic_kernel<__nv_bfloat16, false><<<grid, warps * 32, 0, st>>>(a);
    } else {
        if (a.det) sfa_bwd_generic_kernel<__half, true><<<grid, warps * 32, 0, st>>>(a);
        else sfa_bwd_generic_kernel<__half, false><<<grid, warps * 32, 0, st>>>(a);
    }
    return cudaGetLastError();
}

// Forward with an online softmax over the gathered rows (same warp mapping).
template <typename T>
__global__ void __launch_bounds__(256) sfa_fwd_generic_kernel(FwdArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t pair = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (pair >= a.sd.T1 * a.N1) return;
    const int64_t t = pair / a.N1;
    const TokInfo ti = tok_info(a.sd, t);
    float acc[kVC];
#pragma unroll
    for (int c = 0; c < kVC; ++c) acc[c] = 0.f;
    float m = -INFINITY, l = 0.f;
    if (ti.valid) {
        const T* q = (const T*)a.q + pair * kD;
        const T* qr = (const T*)a.qr + pair * kDr;
        float qv[kQC];
#pragma unroll
        for (int c = 0; c < kVC; ++c) qv[c] = to_f(q[c * 32 + lane]);
#pragma unroll
        for (int c = kVC; c < kQC; ++c) qv[c] = to_f(qr[(c - kVC) * 32 + lane]);
        const int nb = a.nblk[t];
        const int32_t* blist = a.blocks + t * a.topk;
        for (int ib = 0; ib < nb; ++ib) {
            const int64_t blk = blist[ib];
            const int nr = block_rows(blk, a.bs, ti, a.mode);
            for (int r = 0; r < nr; ++r) {
                const int64_t g = ti.kv_start + blk * a.bs + r;
                const T* kg = (const T*)a.k + g * kD;
                const T* krg = (const T*)a.kr + g * kDr;
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < kVC; ++c) s = fmaf(qv[c], to_f(kg[c * 32 + lane]), s);
#pragma unroll
                for (int c = kVC; c < kQC; ++c) s = fmaf(qv[c], to_f(krg[(c - kVC) * 32 + lane]), s);
                s = warp_sum(s) * a.scale;
                const float mn = fmaxf(m, s);
                const float corr = expf(m - mn);  // exp(-inf) = 0 on the first row
                const float e = expf(s - mn);
                l = l * corr + e;
                const T* vg = (const T*)a.v + g * kD;
#pragma unroll
                for (int c = 0; c < kVC; ++c) acc[c] = fmaf(e, to_f(vg[c * 32 + lane]), acc[c] * corr);
                m = mn;
            }
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    T* o = (T*)a.out + pair * kD;
#pragma unroll
    for (int c = 0; c < kVC; ++c) o[c * 32 + lane] = from_f<T>(acc[c] * inv);
    if (lane == 0) {
        a.smax[pair] = l > 0.f ? m : 0.f;
        a.ssum[pair] = l;
    }
}

cudaError_t launch_fwd_generic(int dtype, const FwdArgs& a, cudaStream_t st) {
    const int64_t pairs = a.sd.T1 * a.N1;
    if (pairs == 0) return cudaGetLastError();
    const int warps = 8;
    unsigned grid = (unsigned)((pairs + warps - 1) / warps);
    if (dtype == SFA_DTYPE_BF16) sfa_fwd_generic_kernel<__nv_bfloat16><<<grid, warps * 32, 0, st>>>(a);
    else sfa_fwd_generic_kernel<__half><<<grid, warps * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace sfa
