// Tensor-core dense varlen FlashAttention backward for sm_100a, head dims 64 and 128
// (aclnnFlashAttentionUnpaddingScoreGrad, 计算公式: dV = P^T.dY, dQ = scale*dS.K,
// dK = scale*dS^T.Q with dS = P o (dY.V^T - rowsum(dY o attentionIn)) and
// P = exp(scale*Q.K^T - softmaxMax) / softmaxSum; TND layout, GQA, sparseMode 0 / 3).
//
// Key-major: a work item is one 128-key block of one KV head of one sequence.
// The CTA loops over the query heads of that KV head's group and over the
// 128-row query blocks that can see the key block, and accumulates dK and dV
// for its keys in TMEM (so they are written once, without atomics).  Per
// (query head, query block):
//   S^T  = K . Q^T,  dP^T = V . dY^T        [128 keys x 128 queries] in TMEM
//   P (16-bit, written back into S^T's columns) and dS (scale folded in, SW128
//        smem) by the softmax warps (TMEM lane = key)
//   dV  += P  . dY  (A operand read from TMEM),   dK += dS . Q     [128 keys x 128 dims]
//   dQ^T = K^T . dS^T                        [128 dims x 128 queries], reusing
//        dP^T's columns, reduced into an fp32 (or 64-bit fixed point) dQ buffer
//        by the flush warps (TMEM lane = dim: 128-byte coalesced reductions).
// Q / dY are double-buffered, so the next pair's load overlaps this pair, and the
// next S^T is issued as soon as this pair's gradient MMAs have read P.
// Warps: 0-7 softmax (two per TMEM lane quarter, each taking half of the query
// columns), 0-3 also the dK/dV write-out, 4-11 dQ flush (two per lane quarter,
// halves of the query columns), 12 TMA producer, 13 MMA.
// Head dim 64 runs the same schedule with half-width K / V / Q / dY tiles (one SW128
// half each), S^T / dP^T over 4 K-steps, dK / dV accumulators of 64 TMEM columns, and
// dQ^T formed with M = 128 over the key block's 64 valid dims (the upper 64 TMEM lanes
// are not written out).
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <type_traits>
#include <vector>

#include "sfa_internal.cuh"
#include "tc_common.cuh"

namespace sfa {

namespace {

using namespace tc;

constexpr int kFaDMax = 128;  // largest head dim of the tensor-core path (the smem / TMEM plan)
constexpr int kBlk = 128;
constexpr int kFaThreads = 448;
// K, V, then Q / dY of slot x at kOffQ / kOffO + x * 65536, dS, constants, barriers
constexpr int kOffK = 0, kOffV = 32768, kOffQ = 65536, kOffO = 98304, kOffDS = 196608;
constexpr int kOffCst = 229376;                     // float [2][2][128]: max*log2e + log2(sum), rowsum(dY o O)
constexpr int kOffBar = kOffCst + 2 * 2 * 128 * 4;  // 17 mbarriers
constexpr int kOffMisc = kOffBar + 18 * 8;
constexpr int kFaSmem = kOffMisc + 16;

struct FaItem {
    int b, hk, kb, cost;
};

struct FaParams {
    CUtensorMap mapQ, mapK, mapV, mapO;  // mapO = dY
    const FaItem* items;
    int nitems;
    const int64_t* cu_q;
    const int64_t* cu_kv;
    const float* smax;    // [T1][Nq][8]
    const float* ssum;
    const float* rowsum;  // [T1][Nq]
    void* dq_acc;         // [T1][Nq][D] fp32 or int64
    void* dk;             // [T2][Nkv][D]
    void* dv;
    int* err;
    const float* dmax;    // deterministic mode: max|dY| that sets the dQ fixed-point grid
    int64_t T1;
    int B, Nq, Nkv, mode;
    float scale;
    uint64_t wait_ns;  // limit of every mbarrier wait
};

struct Seq {
    int64_t qs, ql, ks, kl;
};
__device__ __forceinline__ Seq seq_of(const FaParams& p, int b) {
    Seq s;
    s.qs = b ? p.cu_q[b - 1] : 0;
    s.ql = p.cu_q[b] - s.qs;
    s.ks = b ? p.cu_kv[b - 1] : 0;
    s.kl = p.cu_kv[b] - s.ks;
    return s;
}
// first query block that can see key block kb (bottom-right causal in mode 3)
__device__ __forceinline__ int first_qb(const Seq& s, int kb, int mode) {
    if (mode != 3) return 0;
    const int64_t lo = (int64_t)kb * kBlk - (s.kl - s.ql);  // smallest query row seeing the block's first key
    return lo <= 0 ? 0 : (int)(lo / kBlk);
}

template <typename T, bool DET, int D>
__global__ void __launch_bounds__(kFaThreads, 1) fa_bwd_fused_kernel(const __grid_constant__ FaParams prm) {
    static_assert(D == 64 || D == 128, "head dims 64 and 128");
    constexpr bool kF16 = std::is_same<T, __half>::value;
    constexpr int kHalves = D / 64;       // SW128 halves (64 dims each) of a K / V / Q / dY tile
    constexpr uint32_t kTileTx = kHalves * kBlk * 128u;  // bytes of one such tile
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) atomicCAS(prm.err, 0, 7);
        return;
    }
    float* cst = reinterpret_cast<float*>(smem + kOffCst);
    const uint32_t bar0 = sbase + kOffBar;
    const uint32_t KV_FULL = bar0, KV_EMPTY = bar0 + 8, SDP_FULL = bar0 + 16, PDS_FULL = bar0 + 24,
                   PDS_FREE = bar0 + 32, DQ_FULL = bar0 + 40, DQ_FREE = bar0 + 48, ACC_FULL = bar0 + 56,
                   ACC_EMPTY = bar0 + 64, DONE = bar0 + 72;
    auto CST_FULL = [&](int x) { return bar0 + 80 + 8u * x; };   // per-pair softmax constants written
    auto QDO_FULL = [&](int x) { return bar0 + 96 + 8u * x; };   // Q / dY slot loaded
    auto QDO_EMPTY = [&](int x) { return bar0 + 112 + 8u * x; }; // ... and consumed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    // bounded mbarrier wait: past prm.wait_ns it records `code` in the error word and every role exits
    auto WAIT = [&](uint32_t bar, uint32_t parity, int code) {
        return wait_bar(bar, parity, abort_flag, prm.err, code, prm.wait_ns);
    };
    if (threadIdx.x == 0) {
        mbar_init(KV_FULL, 1);
        mbar_init(KV_EMPTY, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(QDO_FULL(x), 1);
            mbar_init(QDO_EMPTY(x), 1);
        }
        mbar_init(SDP_FULL, 1);
        mbar_init(PDS_FULL, 256);
        mbar_init(CST_FULL(0), 128);
        mbar_init(CST_FULL(1), 128);
        mbar_init(PDS_FREE, 1);
        mbar_init(DQ_FULL, 1);
        mbar_init(DQ_FREE, 256);
        mbar_init(ACC_FULL, 1);
        mbar_init(ACC_EMPTY, 128);
        mbar_init(DONE, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {  // S^T / P [0,128), dP^T / dQ^T [128,256), dK [256,384), dV [384,512)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t T_S = tmem, T_DP = tmem + 128, T_DK = tmem + 256, T_DV = tmem + 384;
    const int G = prm.Nq / prm.Nkv;
    const float scale = prm.scale;

    if (warp == 12) {
        // =================== TMA producer ===================
        int item_ctr = 0, pair_ctr = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < prm.nitems && ok; w += gridDim.x, ++item_ctr) {
            const FaItem it = prm.items[w];
            const Seq s = seq_of(prm, it.b);
            if (lane == 0) {
                ok = WAIT(KV_EMPTY, (item_ctr & 1) ^ 1, 21);
                if (ok) {
                    mbar_expect_tx(KV_FULL, 2 * kTileTx);
                    const int row = (int)(s.ks + (int64_t)it.kb * kBlk);
                    for (int h = 0; h < kHalves; ++h) {
                        tma_load_2d(sbase + kOffK + h * 16384, &prm.mapK, it.hk * D + h * 64, row, KV_FULL);
                        tma_load_2d(sbase + kOffV + h * 16384, &prm.mapV, it.hk * D + h * 64, row, KV_FULL);
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            const int q0 = first_qb(s, it.kb, prm.mode), nqb = (int)((s.ql + kBlk - 1) / kBlk);
            for (int h = it.hk * G; h < it.hk * G + G && ok; ++h) {
                for (int qb = q0; qb < nqb && ok; ++qb, ++pair_ctr) {
                    const int x = pair_ctr & 1;
                    if (lane == 0) {
                        ok = WAIT(QDO_EMPTY(x), ((pair_ctr >> 1) & 1) ^ 1, 22);
                        if (ok) {
                            mbar_expect_tx(QDO_FULL(x), 2 * kTileTx);
                            const int row = (int)(s.qs + (int64_t)qb * kBlk);
                            for (int hh = 0; hh < kHalves; ++hh) {
                                tma_load_2d(sbase + kOffQ + x * 65536 + hh * 16384, &prm.mapQ, h * D + hh * 64, row,
                                            QDO_FULL(x));
                                tma_load_2d(sbase + kOffO + x * 65536 + hh * 16384, &prm.mapO, h * D + hh * 64, row,
                                            QDO_FULL(x));
                            }
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                }
            }
        }
        if (lane == 0) {  // drain the last loads before exiting
            uint64_t t0 = globaltimer();
            if (item_ctr > 0)
                while (!mbar_try(KV_FULL, (item_ctr - 1) & 1) && globaltimer() - t0 < 1000000000ull) {
                }
            for (int k = 1; k <= 2; ++k) {
                const int p = pair_ctr - k;
                if (p >= 0)
                    while (!mbar_try(QDO_FULL(p & 1), (p >> 1) & 1) && globaltimer() - t0 < 1000000000ull) {
                    }
            }
        }
    } else if (warp == 13) {
        // =================== MMA issuer ===================
        const uint32_t ID_S = idesc(128, 128, false, false, kF16);  // S^T, dP^T (A = K/V, B = Q/dY, both K-major)
        const uint32_t ID_A = idesc(128, D, false, true, kF16);     // dV (A = P in TMEM), dK (A = dS K-major); B MN-major
        // dQ^T (A = K MN-major, B = dS MN-major); M = 128 also for head dim 64 (its upper 64 rows
        // read the unused second half of the K tile and are never written out)
        const uint32_t ID_Q = idesc(128, 128, true, true, kF16);
        const uint32_t sK = sbase + kOffK, sV = sbase + kOffV, sDS = sbase + kOffDS;
        int item_ctr = 0, pair_ctr = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < prm.nitems && ok; w += gridDim.x, ++item_ctr) {
            const FaItem it = prm.items[w];
            const Seq s = seq_of(prm, it.b);
            if (lane == 0) ok = WAIT(KV_FULL, item_ctr & 1, 23);
            if (lane == 0 && ok) ok = WAIT(ACC_EMPTY, (item_ctr & 1) ^ 1, 24);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const int q0 = first_qb(s, it.kb, prm.mode), nqb = (int)((s.ql + kBlk - 1) / kBlk);
            bool first = true;
            for (int h = it.hk * G; h < it.hk * G + G && ok; ++h) {
                for (int qb = q0; qb < nqb && ok; ++qb, ++pair_ctr) {
                    const int x = pair_ctr & 1;
                    const uint32_t sQ = sbase + kOffQ + x * 65536, sO = sbase + kOffO + x * 65536;
                    if (lane == 0) {
                        ok = WAIT(QDO_FULL(x), (pair_ctr >> 1) & 1, 25);
                        // S^T overwrites P of the previous pair: its gradient MMAs must have completed
                        if (ok && pair_ctr > 0) ok = WAIT(PDS_FREE, (pair_ctr - 1) & 1, 26);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                            mma(T_S, sdesc(sK + off, 16, 1024), sdesc(sQ + off, 16, 1024), ID_S, ks > 0);
                        }
                        // dP^T overwrites the previous pair's dQ^T once the flush has read it
                        ok = WAIT(DQ_FREE, (pair_ctr & 1) ^ 1, 33);
                        if (ok) {
                            tc_fence_after();
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                                mma(T_DP, sdesc(sV + off, 16, 1024), sdesc(sO + off, 16, 1024), ID_S, ks > 0);
                            }
                            mma_commit(SDP_FULL);
                            ok = WAIT(PDS_FULL, pair_ctr & 1, 27);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        for (int ks = 0; ks < 8; ++ks) {  // K = 128 queries, 16 per step
                            // P of queries 16ks..16ks+15: TMEM columns 64*(ks/4) + 8*(ks%4) (16-bit pairs)
                            const uint32_t aP = T_S + 64u * (ks >> 2) + 8u * (ks & 3);
                            const uint64_t aS = sdesc(sDS + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                            mma_ts(T_DV, aP, sdesc(sO + ks * 2048, 16384, 1024), ID_A, (!first || ks > 0));
                            mma(T_DK, aS, sdesc(sQ + ks * 2048, 16384, 1024), ID_A, (!first || ks > 0));
                        }
                        for (int ks = 0; ks < 8; ++ks)  // K = 128 keys
                            mma(T_DP, sdesc(sK + ks * 2048, 16384, 1024), sdesc(sDS + ks * 2048, 16384, 1024), ID_Q,
                                ks > 0);
                        mma_commit(QDO_EMPTY(x));
                        mma_commit(PDS_FREE);
                        mma_commit(DQ_FULL);
                    }
                    __syncwarp();
                    first = false;
                }
            }
            if (!ok) break;
            if (lane == 0) {
                mma_commit(KV_EMPTY);
                mma_commit(ACC_FULL);
            }
        }
        if (lane == 0) {
            mma_commit(DONE);
            uint64_t t0 = globaltimer();
            while (!mbar_try(DONE, 0) && globaltimer() - t0 < 1000000000ull) {
            }
        }
    } else {
        // ====== warps 0-7: softmax / dS (TMEM lane = key; warp w takes query columns 64*(w/4)..+64);
        // ====== warps 0-3: dK / dV write-out; warps 4-11: dQ flush (TMEM lane = dim) ======
        const bool do_softmax = warp < 8, do_flush = warp >= 4, do_out = warp < 4;
        const int quarter = warp & 3;                 // TMEM lane quarter of this warp
        const int j = quarter * 32 + lane;            // key (softmax / write-out) or dim (flush)
        const int cs = warp >> 2;                     // softmax: which half of the query columns
        const int hsel = (warp - 4) >> 2;             // flush: which half of the query columns
        const float fmul_q = DET ? fix_mul(fix_exponents(*prm.dmax, prm.scale, prm.T1, prm.Nq / prm.Nkv).q) : 0.f;
        const float c1 = scale * 1.4426950408889634f;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        int item_ctr = 0, pair_ctr = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < prm.nitems && ok; w += gridDim.x, ++item_ctr) {
            const FaItem it = prm.items[w];
            const Seq s = seq_of(prm, it.b);
            const int q0 = first_qb(s, it.kb, prm.mode), nqb = (int)((s.ql + kBlk - 1) / kBlk);
            const int64_t jl = (int64_t)it.kb * kBlk + j;  // key position in the sequence
            const bool key_ok = jl < s.kl;
            const int64_t off = s.kl - s.ql;
            int npairs = 0;
            for (int h = it.hk * G; h < it.hk * G + G && ok; ++h) {
                for (int qb = q0; qb < nqb && ok; ++qb, ++pair_ctr, ++npairs) {
                    if (do_softmax) {
                        const int x = pair_ctr & 1, use = pair_ctr >> 1;
                        float* cx = cst + x * 256;
                        if (do_out) {
                            // constants of query row j of this block (the buffer's previous pair,
                            // pair_ctr - 2, finished its softmax before the gradients of pair_ctr - 1)
                            const int64_t il = (int64_t)qb * kBlk + j;
                            // P = exp2(S*scale*log2e - (max*log2e + log2(sum))); an empty row (sum 0)
                            // gets +inf, so P = 0
                            if (il < s.ql) {
                                const int64_t sidx = (s.qs + il) * prm.Nq + h;
                                const float l = prm.ssum[sidx * 8];
                                cx[j] = l > 0.f ? fmaf(prm.smax[sidx * 8], 1.4426950408889634f, log2f(l)) : INFINITY;
                                cx[128 + j] = prm.rowsum[sidx];
                            } else {
                                cx[j] = INFINITY;
                                cx[128 + j] = 0.f;
                            }
                            mbar_arrive(CST_FULL(x));
                        }
                        // queries i of this block that keep this key: lo <= i < hi (i < ql, and in
                        // mode 3 jl <= qb*128 + i + off); none when the key is past the sequence
                        const int64_t ibase = (int64_t)qb * kBlk;
                        int64_t lo64 = prm.mode == 3 ? jl - off - ibase : 0;
                        int64_t hi64 = s.ql - ibase;
                        lo64 = lo64 < 0 ? 0 : (lo64 > kBlk ? kBlk : lo64);
                        hi64 = hi64 > kBlk ? kBlk : hi64;
                        const int lo = (int)lo64;
                        const uint32_t span = key_ok && hi64 > lo64 ? (uint32_t)(hi64 - lo64) : 0u;
                        ok = WAIT(CST_FULL(x), use & 1, 32);
                        if (ok) ok = WAIT(SDP_FULL, pair_ctr & 1, 28);
                        if (ok && pair_ctr > 0) ok = WAIT(PDS_FREE, (pair_ctr - 1) & 1, 29);
                        ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-collective
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll 1
                        for (int cc = 4 * cs; cc < 4 * cs + 4; ++cc) {  // 16 query columns at a time
                            float sv[16], dp[16];
                            tmem_ld16(T_S + lane_base + cc * 16, sv);
                            tmem_ld16(T_DP + lane_base + cc * 16, dp);
                            tmem_wait_ld();
                            uint32_t pw[8], dw[8];
                            const float4* cm = reinterpret_cast<const float4*>(cx + cc * 16);        // log2 offset
                            const float4* cd = reinterpret_cast<const float4*>(cx + 128 + cc * 16);  // rowsum(dY o O)
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                const float4 m4 = cm[g], d4 = cd[g];
                                const float mm[4] = {m4.x, m4.y, m4.z, m4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
                                float pv[4], dv[4];
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const int e = 4 * g + k;
                                    const bool v = (uint32_t)(cc * 16 + e - lo) < span;
                                    // a select (not a product): masked scores may overflow exp2
                                    pv[k] = v ? ex2_approx(fmaf(sv[e], c1, -mm[k])) : 0.f;
                                    dv[k] = pv[k] * (dp[e] - dd[k]) * scale;
                                }
                                pw[2 * g] = pack2<T>(pv[0], pv[1]);
                                pw[2 * g + 1] = pack2<T>(pv[2], pv[3]);
                                dw[2 * g] = pack2<T>(dv[0], dv[1]);
                                dw[2 * g + 1] = pack2<T>(dv[2], dv[3]);
                            }
                            // P -> TMEM columns 64*(cc/4) + 8*(cc%4): inside the S^T columns this warp
                            // group reads, at or behind the ones it has already read
                            tmem_st8(T_S + lane_base + 64u * (cc >> 2) + 8u * (cc & 3), pw);
                            // dS columns [16cc, 16cc+16): SW128 half cc/4, 16-byte units 2(cc%4) and 2(cc%4)+1
                            const int half = cc >> 2, u0 = (cc & 3) * 2;
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const uint32_t o = half * 16384 + j * 128 + (((u0 + u) ^ (j & 7)) << 4);
                                *reinterpret_cast<uint4*>(smem + kOffDS + o) =
                                    make_uint4(dw[4 * u], dw[4 * u + 1], dw[4 * u + 2], dw[4 * u + 3]);
                            }
                        }
                        tmem_wait_st();
                        fence_view_async_shared();
                        tc_fence_before();
                        mbar_arrive(PDS_FULL);
                    }
                    if (do_flush) {
                        ok = __all_sync(0xffffffffu, WAIT(DQ_FULL, pair_ctr & 1, 31));
                        if (!ok) break;
                        tc_fence_after();
                        const int dim = j;
                        const bool dim_ok = quarter * 32 < D;  // (warp-uniform) lane quarter holds real dims
                        const int64_t nq = min((int64_t)kBlk, s.ql - (int64_t)qb * kBlk);
                        const int64_t row0 = s.qs + (int64_t)qb * kBlk;
#pragma unroll 1
                        for (int cc = 2 * hsel; cc < 2 * hsel + 2 && dim_ok; ++cc) {
                            float v[32];
                            tmem_ld32(T_DP + lane_base + cc * 32, v);
                            tmem_wait_ld();
                            const int lim = (int)min((int64_t)32, nq - cc * 32);
                            const size_t base = ((size_t)(row0 + cc * 32) * prm.Nq + h) * D + dim;
                            const uint32_t step = (uint32_t)prm.Nq * D;  // elements between query rows
                            // one running pointer (not 32 precomputed addresses) keeps the loop in registers
                            if (DET) {
                                unsigned long long* d = reinterpret_cast<unsigned long long*>(prm.dq_acc) + base;
#pragma unroll
                                for (int e = 0; e < 32; ++e, d += step)
                                    if (e < lim) atomicAdd(d, fix_round(v[e], fmul_q));
                            } else {
                                float* d = reinterpret_cast<float*>(prm.dq_acc) + base;
#pragma unroll
                                for (int e = 0; e < 32; ++e, d += step)
                                    if (e < lim) atomicAdd(d, v[e]);
                            }
                        }
                        tc_fence_before();
                        mbar_arrive(DQ_FREE);
                    }
                }
            }
            if (!ok) break;
            if (!do_out) continue;
            // dK / dV rows of this key block (zero when no query sees the block)
            ok = __all_sync(0xffffffffu, WAIT(ACC_FULL, item_ctr & 1, 30));
            if (!ok) break;
            tc_fence_after();
            const int64_t orow = ((s.ks + jl) * prm.Nkv + it.hk) * D;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                T* dst = reinterpret_cast<T*>(which ? prm.dv : prm.dk) + orow;
                const uint32_t src = which ? T_DV : T_DK;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    float v[32];
                    tmem_ld32(src + lane_base + cc * 32, v);
                    tmem_wait_ld();
                    if (key_ok) {
                        uint32_t wv[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2)
                            wv[e >> 1] = npairs ? pack2<T>(v[e], v[e + 1]) : 0u;
                        uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
                        for (int u = 0; u < 4; ++u) d4[u] = make_uint4(wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(ACC_EMPTY);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

template <typename T, int D>
__global__ void fa_rowsum_kernel(const T* __restrict__ dy, const T* __restrict__ o, int64_t rows,
                                 float* __restrict__ res) {
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    constexpr int kPer = D / 32;  // elements per lane
    const T* ap = dy + r * D + lane * kPer;
    const T* bp = o + r * D + lane * kPer;
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) sum = fmaf(to_f(ap[e]), to_f(bp[e]), sum);
#pragma unroll
    for (int k = 16; k; k >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, k);
    if (lane == 0) res[r] = sum;
}

template <typename T, bool DET>
__global__ void fa_cast_dq_kernel(const void* __restrict__ acc, int64_t n, T* __restrict__ dq,
                                  const float* __restrict__ dmax, float scale, int64_t T1, int64_t G) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float x = DET ? (float)((double)reinterpret_cast<const long long*>(acc)[i] *
                                  fix_inv(fix_exponents(*dmax, scale, T1, G).q))
                        : reinterpret_cast<const float*>(acc)[i];
    dq[i] = from_f<T>(x);
}

template <typename T, bool DET, int D>
cudaError_t launch_fa_t(const FaFusedArgs& a, cudaStream_t st) {
    FaParams p;
    memset(&p, 0, sizeof p);
    const uint64_t qcols = (uint64_t)a.Nq * D, kcols = (uint64_t)a.Nkv * D;
    if (!make_map(&p.mapQ, a.q, a.dtype, qcols, a.T1, qcols, kBlk) ||
        !make_map(&p.mapO, a.dy, a.dtype, qcols, a.T1, qcols, kBlk) ||
        !make_map(&p.mapK, a.k, a.dtype, kcols, a.T2, kcols, kBlk) ||
        !make_map(&p.mapV, a.v, a.dtype, kcols, a.T2, kcols, kBlk))
        return cudaErrorInvalidValue;
    p.items = reinterpret_cast<const FaItem*>(a.items);
    p.nitems = a.nitems;
    p.cu_q = a.cu_q;
    p.cu_kv = a.cu_kv;
    p.smax = a.smax;
    p.ssum = a.ssum;
    p.rowsum = a.rowsum;
    p.dq_acc = a.dq_acc;
    p.dk = a.dk;
    p.dv = a.dv;
    p.err = a.err;
    p.dmax = a.dout_absmax;
    p.T1 = a.T1;
    p.B = (int)a.B;
    p.Nq = (int)a.Nq;
    p.Nkv = (int)a.Nkv;
    p.mode = a.mode;
    p.scale = a.scale;
    p.wait_ns = wait_limit_ns();
    const int64_t rows = a.T1 * a.Nq;
    if (rows > 0)
        fa_rowsum_kernel<T, D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>((const T*)a.dy, (const T*)a.o, rows,
                                                                           (float*)a.rowsum);
    auto kern = fa_bwd_fused_kernel<T, DET, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFaSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(sms, a.nitems);
    if (grid > 0) kern<<<grid, kFaThreads, kFaSmem, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t n = a.T1 * a.Nq * D;
    if (n > 0)
        fa_cast_dq_kernel<T, DET><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.dq_acc, n, (T*)a.dq, a.dout_absmax,
                                                                            a.scale, a.T1, a.Nq / a.Nkv);
    return cudaGetLastError();
}

}  // namespace

size_t fa_fused_items(const int64_t* cu_q, const int64_t* cu_kv, int64_t B, int64_t Nq, int64_t Nkv, int mode,
                      std::vector<int32_t>* out) {
    std::vector<FaItem> items;
    const int64_t G = Nq / Nkv;
    int64_t pq = 0, pk = 0;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t ql = cu_q[b] - pq, kl = cu_kv[b] - pk;
        pq = cu_q[b];
        pk = cu_kv[b];
        const int64_t nkb = (kl + kBlk - 1) / kBlk, nqb = (ql + kBlk - 1) / kBlk;
        for (int64_t kb = 0; kb < nkb; ++kb) {
            int64_t q0 = 0;
            if (mode == 3) {
                const int64_t lo = kb * kBlk - (kl - ql);
                q0 = lo <= 0 ? 0 : lo / kBlk;
            }
            const int cost = (int)(G * std::max<int64_t>(0, nqb - q0));
            for (int64_t hk = 0; hk < Nkv; ++hk) items.push_back(FaItem{(int)b, (int)hk, (int)kb, cost});
        }
    }
    // longest first, so the persistent CTAs finish together
    std::stable_sort(items.begin(), items.end(), [](const FaItem& x, const FaItem& y) { return x.cost > y.cost; });
    if (out) {
        out->resize(items.size() * 4);
        memcpy(out->data(), items.data(), items.size() * sizeof(FaItem));
    }
    return items.size();
}

bool fa_fused_supported(int64_t D) { return D == 64 || D == kFaDMax; }

template <typename T, int D>
cudaError_t launch_fa_d(const FaFusedArgs& a, cudaStream_t st) {
    return a.det ? launch_fa_t<T, true, D>(a, st) : launch_fa_t<T, false, D>(a, st);
}

cudaError_t launch_fa_bwd_fused(int dtype, const FaFusedArgs& a, cudaStream_t st) {
    if (dtype == SFA_DTYPE_BF16)
        return a.D == 64 ? launch_fa_d<__nv_bfloat16, 64>(a, st) : launch_fa_d<__nv_bfloat16, 128>(a, st);
    return a.D == 64 ? launch_fa_d<__half, 64>(a, st) : launch_fa_d<__half, 128>(a, st);
}

}  // namespace sfa
