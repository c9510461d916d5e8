// Dense varlen FlashAttention forward / backward (TND, GQA, sparseMode 0 / 3),
// warp per (query row, query head).  aclnnFlashAttentionUnpaddingScoreGrad
// (计算公式): dV = P^T.dY, dQ = scale*dS.K, dK = scale*dS^T.Q with
// dS = P o (dY.V^T - rowsum(dY o attentionIn)) and P = exp(scale*Q.K^T - max)/sum.
// Lane l holds dims l, l+32, ... of the head dim; the key-side sums go to an fp32
// (or 64-bit fixed-point) accumulator [2][T2][Nkv][D] and are cast at the end.
#include "sfa_internal.cuh"

namespace sfa {

namespace {

__device__ __forceinline__ float wsum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

struct FaTok {
    int64_t kv_start;
    int64_t n_keys;  // keys 0 .. n_keys-1 of the sequence are kept
    bool valid;
};

__device__ __forceinline__ FaTok fa_tok(const FaArgs& a, int64_t t, int mode) {
    FaTok r{0, 0, false};
    int lo = 0, hi = (int)a.B;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (a.cu_q[mid] > t) hi = mid; else lo = mid + 1;
    }
    if (lo >= a.B) return r;
    const int b = lo;
    int64_t qs = b ? clamp64(a.cu_q[b - 1], 0, a.T1) : 0;
    int64_t qe = clamp64(a.cu_q[b], 0, a.T1);
    int64_t ks = b ? clamp64(a.cu_kv[b - 1], 0, a.T2) : 0;
    int64_t ke = clamp64(a.cu_kv[b], 0, a.T2);
    if (t < qs || t >= qe) return r;
    int64_t kl = ke > ks ? ke - ks : 0;
    int64_t n = kl;
    if (mode == 3) {
        int64_t lim = (t - qs) + kl - (qe - qs);  // last kept key
        n = lim + 1 < kl ? lim + 1 : kl;
        if (n < 0) n = 0;
    }
    r.kv_start = ks;
    r.n_keys = n;
    r.valid = true;
    return r;
}

template <bool DET>
__device__ __forceinline__ void acc_add(void* acc, int64_t off, float x, float fmul) {
    if (DET) atomicAdd(reinterpret_cast<unsigned long long*>(acc) + off, fix_round(x, fmul));
    else atomicAdd(reinterpret_cast<float*>(acc) + off, x);
}

template <typename T, int NC, bool DET>
__global__ void __launch_bounds__(256) fa_bwd_kernel(FaArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t pair = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (pair >= a.T1 * a.Nq) return;
    const int64_t t = pair / a.Nq;
    const int h = (int)(pair - t * a.Nq);
    const int hk = h / (int)(a.Nq / a.Nkv);
    const int D = (int)a.D;
    const FaTok ti = fa_tok(a, t, a.mode);
    float fmul_k = 0.f, fmul_v = 0.f;  // fixed-point grids of dK and dV (deterministic mode)
    if (DET) {
        const FixExp fe = fix_exponents(*a.dout_absmax, a.scale, a.T1, a.Nq / a.Nkv);
        fmul_k = fix_mul(fe.k);
        fmul_v = fix_mul(fe.v);
    }
    float dq[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) dq[c] = 0.f;
    if (ti.valid) {
        float qv[NC], dyv[NC];
        float dsum = 0.f;
        const T* q = (const T*)a.q + pair * D;
        const T* dy = (const T*)a.dy + pair * D;
        const T* o = (const T*)a.o + pair * D;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int d = c * 32 + lane;
            qv[c] = d < D ? to_f(q[d]) : 0.f;
            dyv[c] = d < D ? to_f(dy[d]) : 0.f;
            dsum = fmaf(dyv[c], d < D ? to_f(o[d]) : 0.f, dsum);
        }
        dsum = wsum(dsum);
        const float m = a.smax[pair * 8];
        const float l = a.ssum[pair * 8];
        const float inv_l = l == 0.f ? 0.f : 1.f / l;
        const int64_t kvD = a.T2 * a.Nkv * D;
        for (int64_t j = 0; j < ti.n_keys; ++j) {
            const int64_t g = ((ti.kv_start + j) * a.Nkv + hk) * D;
            const T* kg = (const T*)a.k + g;
            const T* vg = (const T*)a.v + g;
            float kv[NC];
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int d = c * 32 + lane;
                kv[c] = d < D ? to_f(kg[d]) : 0.f;
                s = fmaf(qv[c], kv[c], s);
                dp = fmaf(dyv[c], d < D ? to_f(vg[d]) : 0.f, dp);
            }
            s = wsum(s) * a.scale;
            dp = wsum(dp);
            const float p = expf(s - m) * inv_l;
            const float ds = p * (dp - dsum);
            const float sds = a.scale * ds;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int d = c * 32 + lane;
                dq[c] = fmaf(ds, kv[c], dq[c]);
                if (d < D) {
                    acc_add<DET>(a.dkv_acc, g + d, sds * qv[c], fmul_k);
                    acc_add<DET>(a.dkv_acc, kvD + g + d, p * dyv[c], fmul_v);
                }
            }
        }
    }
    T* dqo = (T*)a.dq + pair * D;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int d = c * 32 + lane;
        if (d < D) dqo[d] = from_f<T>(a.scale * dq[c]);
    }
}

template <typename T, bool DET>
__global__ void fa_cast_kernel(const void* __restrict__ acc, int64_t n, T* __restrict__ dk, T* __restrict__ dv,
                               const float* __restrict__ dmax, float scale, int64_t T1, int64_t G) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * n) return;
    float x;
    if (DET) {
        const FixExp fe = fix_exponents(*dmax, scale, T1, G);
        x = (float)((double)reinterpret_cast<const long long*>(acc)[i] * fix_inv(i < n ? fe.k : fe.v));
    } else {
        x = reinterpret_cast<const float*>(acc)[i];
    }
    if (i < n) dk[i] = from_f<T>(x);
    else dv[i - n] = from_f<T>(x);
}

template <typename T, int NC>
__global__ void __launch_bounds__(256) fa_fwd_kernel(FaArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t pair = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (pair >= a.T1 * a.Nq) return;
    const int64_t t = pair / a.Nq;
    const int h = (int)(pair - t * a.Nq);
    const int hk = h / (int)(a.Nq / a.Nkv);
    const int D = (int)a.D;
    const FaTok ti = fa_tok(a, t, a.mode);
    float acc[NC], qv[NC];
    float m = -INFINITY, l = 0.f;
    const T* q = (const T*)a.q + pair * D;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        acc[c] = 0.f;
        const int d = c * 32 + lane;
        qv[c] = d < D ? to_f(q[d]) : 0.f;
    }
    if (ti.valid) {
        for (int64_t j = 0; j < ti.n_keys; ++j) {
            const int64_t g = ((ti.kv_start + j) * a.Nkv + hk) * D;
            const T* kg = (const T*)a.k + g;
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int d = c * 32 + lane;
                s = fmaf(qv[c], d < D ? to_f(kg[d]) : 0.f, s);
            }
            s = wsum(s) * a.scale;
            const float mn = fmaxf(m, s);
            const float corr = expf(m - mn);
            const float e = expf(s - mn);
            l = l * corr + e;
            const T* vg = (const T*)a.v + g;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int d = c * 32 + lane;
                acc[c] = fmaf(e, d < D ? to_f(vg[d]) : 0.f, acc[c] * corr);
            }
            m = mn;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    T* o = (T*)a.out + pair * D;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int d = c * 32 + lane;
        if (d < D) o[d] = from_f<T>(acc[c] * inv);
    }
    if (lane < 8) {
        a.smax_out[pair * 8 + lane] = l > 0.f ? m : 0.f;
        a.ssum_out[pair * 8 + lane] = l;
    }
}

template <typename T, bool DET>
cudaError_t fa_bwd_dispatch(const FaArgs& a, cudaStream_t st) {
    const int64_t pairs = a.T1 * a.Nq;
    const int warps = 8;
    if (pairs > 0) {
        unsigned grid = (unsigned)((pairs + warps - 1) / warps);
        const int nc = (int)((a.D + 31) / 32);
        switch (nc) {
            case 1: fa_bwd_kernel<T, 1, DET><<<grid, warps * 32, 0, st>>>(a); break;
            case 2: fa_bwd_kernel<T, 2, DET><<<grid, warps * 32, 0, st>>>(a); break;
            case 3: case 4: fa_bwd_kernel<T, 4, DET><<<grid, warps * 32, 0, st>>>(a); break;
            default: fa_bwd_kernel<T, 8, DET><<<grid, warps * 32, 0, st>>>(a); break;
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = a.T2 * a.Nkv * a.D;
    if (n > 0)
        fa_cast_kernel<T, DET><<<(unsigned)((2 * n + 255) / 256), 256, 0, st>>>(a.dkv_acc, n, (T*)a.dk, (T*)a.dv,
                                                                            a.dout_absmax, a.scale, a.T1,
                                                                            a.Nq / a.Nkv);
    return cudaGetLastError();
}

template <typename T>
cudaError_t fa_fwd_dispatch(const FaArgs& a, cudaStream_t st) {
    const int64_t pairs = a.T1 * a.Nq;
    const int warps = 8;
    if (pairs == 0) return cudaGetLastError();
    unsigned grid = (unsigned)((pairs + warps - 1) / warps);
    const int nc = (int)((a.D + 31) / 32);
    switch (nc) {
        case 1: fa_fwd_kernel<T, 1><<<grid, warps * 32, 0, st>>>(a); break;
        case 2: fa_fwd_kernel<T, 2><<<grid, warps * 32, 0, st>>>(a); break;
        case 3: case 4: fa_fwd_kernel<T, 4><<<grid, warps * 32, 0, st>>>(a); break;
        default: fa_fwd_kernel<T, 8><<<grid, warps * 32, 0, st>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fa_bwd(int dtype, const FaArgs& a, cudaStream_t st) {
    if (dtype == SFA_DTYPE_BF16)
        return a.det ? fa_bwd_dispatch<__nv_bfloat16, true>(a, st) : fa_bwd_dispatch<__nv_bfloat16, false>(a, st);
    return a.det ? fa_bwd_dispatch<__half, true>(a, st) : fa_bwd_dispatch<__half, false>(a, st);
}

cudaError_t launch_fa_fwd(int dtype, const FaArgs& a, cudaStream_t st) {
    if (dtype == SFA_DTYPE_BF16) return fa_fwd_dispatch<__nv_bfloat16>(a, st);
    return fa_fwd_dispatch<__half>(a, st);
}

}  // namespace sfa
