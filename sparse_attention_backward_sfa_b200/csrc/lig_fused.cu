// Fused tensor-core dense lightning-indexer gradient with its KL loss for sm_100a
// (tcgen05 MMA, TMEM accumulators, TMA 2-D tile loads, mbarrier pipelines).
//
// What it computes (DenseLightningIndexerGradKLLoss README, 功能说明 formulas
// 1-4), per query row t over the key rows j it sees (the whole sequence, or the
// causal prefix j <= pos + S2_b - S1_b), one 128-key tile at a time:
//   S~^T  = K~ . Q~_t^T        [keys x N1 heads], K = 576 (main attention, MLA shape)
//   SI^T  = K~I . q~I_t^T      [keys x G heads],  K = Di (indexer scores)
//   p_j   = (1/N1) sum_h exp2(S~*scale*log2e - max_h*log2e) / sum_h   (target distribution)
//   I_j   = sum_g W_g ReLU(SI_gj),  sI_j = exp(I_j - maxI) / sumI
//   loss_t += p_j (log p_j - log sI_j),   dI_j = sI_j - p_j
//   dW_g  += dI_j ReLU(SI_gj),   dS_gj = dI_j W_g [SI_gj > 0]
//   dq~I_t^T += K~I^T . dS^T   [Di x G], K = keys    (accumulated in TMEM over the row)
//   dK~I^T    = q~I_t^T . dS   [Di x keys], K = G    -> red.add into an fp32 [T2][Di] buffer
//
// Layout decisions (B200):
//  * Work item = one query row (all N1 main heads and G indexer heads share one
//    key head each); keys are consecutive rows, so every operand chunk is a 2-D
//    TMA tile (128 key rows, or the row's N1 / G head rows) of 128 (64 for the
//    rope) dims, held as two 128-byte-row SW128 halves 16 KB apart in a ring of
//    32 KB slots that carries K0 Q0 .. K4 Q4 (S~^T) and is released chunk by chunk
//    as the S~^T MMAs read it, so it prefetches the next tile while the compute
//    warps work; the K~I tile (double-buffered) and the row's q~I have buffers of
//    their own, held until the gradient MMAs have read them.
//  * TMEM (512 columns): S~^T [0,N1), SI^T [128,192), dq~I^T [256,320) (kept
//    over the row's tiles), dK~I^T [384,512).  TMEM lane = key while the scores
//    are read (each thread owns one key: the head sums stay in registers) and
//    lane = dim for the dK~I / dq~I write-out (coalesced reductions and stores).
//  * dS is stored 16-bit, [keys x G] in one SW128 block: K-major B operand of
//    dK~I^T and MN-major B operand of dq~I^T.
//  * Warp roles: 0-3 compute (scores, loss, dS, dK~I flush, row write-out),
//    4 TMA producer, 5 MMA issuer.  Every mbarrier wait is bounded; on timeout
//    the kernel records an error word, stops issuing, drains what it issued and
//    frees its TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <type_traits>

#include "sfa_internal.cuh"
#include "tc_common.cuh"

namespace sfa {

namespace {

using namespace tc;

constexpr int kThreads = 192;
constexpr int kSlots = 4;
constexpr int kSlotBytes = 32768;
constexpr int kHalf = 16384;
constexpr int kKeys = 128;
constexpr int kOffKI = kSlots * kSlotBytes;   // K~I tiles, double-buffered [2][128 keys x Di]
constexpr int kOffQI = kOffKI + 2 * kSlotBytes;  // q~I of the row [G heads x Di]: two 8 KB SW128 halves
constexpr int kQIHalf = 8192;
constexpr int kOffDS = kOffQI + 16384;        // dS [128 keys x 64 heads] 16-bit, one SW128 block
constexpr int kOffConst = kOffDS + 16384;     // float constants, see below
// constants: [0,128) max*log2e, [128,256) 1/sum of the main heads, [256,320) W,
// [320,576) dW partials [4 warps][64], [576,580) loss partials, [580] maxI*log2e,
// [581] 1/sumI, [582] log(sumI), [583] maxI
constexpr int kNumConst = 584;
constexpr int kOffBar = kOffConst + kNumConst * 4;
constexpr int kNumBars = 2 * kSlots + 14;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 16;
static_assert(kOffBar % 8 == 0, "mbarrier alignment");
static_assert(kSmem <= 227 * 1024, "shared memory budget");

struct LigParams {
    CUtensorMap mapQ, mapQr, mapK, mapKr, mapQI, mapKI;
    const int32_t* nkeys;    // [T1] visible key count of each query row
    const int32_t* kvrow;    // [T1] global row of the first visible key
    const int32_t* order;    // [T1] work order
    const float* smax;       // [T1][N1] main attention statistics
    const float* ssum;
    const float* smax_i;     // [T1] indexer statistics
    const float* ssum_i;
    const void* weights;     // [T1][G] 16-bit
    float* dki_acc;          // [T2][Di] fp32
    void* dqi_out;           // [T1][G][Di] 16-bit
    void* dw_out;            // [T1][G] 16-bit
    float* loss_rows;        // [T1] per-row loss
    int* err;                // device error word
    int64_t T1;
    float scale;
    uint64_t wait_ns;        // limit of every mbarrier wait
};

template <typename T> __device__ __forceinline__ float ld16(const void* p, int64_t i);
template <> __device__ __forceinline__ float ld16<__nv_bfloat16>(const void* p, int64_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}
template <> __device__ __forceinline__ float ld16<__half>(const void* p, int64_t i) {
    return __half2float(reinterpret_cast<const __half*>(p)[i]);
}
template <typename T> __device__ __forceinline__ T cvt16(float x);
template <> __device__ __forceinline__ __nv_bfloat16 cvt16<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half cvt16<__half>(float x) { return __float2half_rn(x); }

// Named barrier 1 over the 128 compute threads that also ANDs a flag across them,
// so a thread that gave up waiting takes the others with it to the same exit.
__device__ __forceinline__ bool compute_all(bool v) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((int)v)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// One halving step of a warp transpose-reduction: lanes with bit `o` set keep the
// upper half of v[0, LEN), the others the lower half, each adding the partner's
// copy of the half it keeps.  After the steps for o = 16, 8, 4, 2, 1 on 64
// values, lane L holds the warp sums of entries 2L and 2L + 1 in v[0], v[1].
template <int LEN>
__device__ __forceinline__ void fold_half(float* v, int lane, int o) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < LEN / 2; ++i) {
        const float send = up ? v[i] : v[i + LEN / 2];
        const float keep = up ? v[i + LEN / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
}

template <typename T, int N1>
__global__ void __launch_bounds__(kThreads, 1) lig_fused_kernel(const __grid_constant__ LigParams prm) {
    constexpr bool kF16 = std::is_same<T, __half>::value;
    constexpr int kG = kLigG, kDi = kLigDi;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) atomicCAS(prm.err, 0, 7);
        return;
    }
    const uint32_t bar0 = sbase + kOffBar;
    auto FULL = [&](int s) { return bar0 + 8u * s; };
    auto EMPTY = [&](int s) { return bar0 + 8u * (kSlots + s); };
    const uint32_t S_FULL = bar0 + 8u * (2 * kSlots + 0);
    const uint32_t DS_FULL = bar0 + 8u * (2 * kSlots + 1);
    const uint32_t DS_FREE = bar0 + 8u * (2 * kSlots + 2);
    const uint32_t DKI_FULL = bar0 + 8u * (2 * kSlots + 3);
    const uint32_t DKI_EMPTY = bar0 + 8u * (2 * kSlots + 4);
    const uint32_t DQI_FULL = bar0 + 8u * (2 * kSlots + 5);
    const uint32_t DQI_FREE = bar0 + 8u * (2 * kSlots + 6);
    const uint32_t DONE = bar0 + 8u * (2 * kSlots + 7);
    auto KI_FULL = [&](int b) { return bar0 + 8u * (2 * kSlots + 8 + b); };
    auto KI_EMPTY = [&](int b) { return bar0 + 8u * (2 * kSlots + 10 + b); };
    const uint32_t QI_FULL = bar0 + 8u * (2 * kSlots + 12);
    const uint32_t QI_EMPTY = bar0 + 8u * (2 * kSlots + 13);
    float* cst = reinterpret_cast<float*>(smem + kOffConst);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    // bounded mbarrier wait: past prm.wait_ns it records `code` in the error word and every role exits
    auto WAIT = [&](uint32_t bar, uint32_t parity, int code) {
        return wait_bar(bar, parity, abort_flag, prm.err, code, prm.wait_ns);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(FULL(s), 1);
            mbar_init(EMPTY(s), 1);
        }
        mbar_init(S_FULL, 1);
        mbar_init(DS_FULL, 128);
        mbar_init(DS_FREE, 1);
        mbar_init(DKI_FULL, 1);
        mbar_init(DKI_EMPTY, 128);
        mbar_init(DQI_FULL, 1);
        mbar_init(DQI_FREE, 128);
        mbar_init(DONE, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(KI_FULL(b), 1);
            mbar_init(KI_EMPTY(b), 1);
        }
        mbar_init(QI_FULL, 1);
        mbar_init(QI_EMPTY, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t T_SM = tmem, T_SI = tmem + 128, T_DQI = tmem + 256, T_DKI = tmem + 384;
    const int nwork = (int)prm.T1;

    if (warp == 4) {
        // =================== TMA producer ===================
        // per tile: the K~I tile into its double buffer, then K0 Q0 .. K4 Q4 through the ring;
        // the row's q~I after its first tile's chunks (it is first read by that tile's SI MMA)
        int slot = 0;
        uint32_t sphase = 0;
        int tile_ctr = 0, row_ctr = 0;
        bool ok = true;
        uint32_t issued_mask = 0;
        int ki_loads = 0, qi_loads = 0;  // loads issued into the K~I buffers / the q~I buffer
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nkeys[t];
            if (n <= 0) continue;
            const int kv0 = prm.kvrow[t];
            const int ntiles = (n + kKeys - 1) / kKeys;
            for (int tile = 0; tile < ntiles && ok; ++tile, ++tile_ctr) {
                const int krow = kv0 + tile * kKeys;
                const int kb = tile_ctr & 1;
                if (lane == 0) ok = WAIT(KI_EMPTY(kb), ((tile_ctr >> 1) & 1) ^ 1, 60);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t dst = sbase + kOffKI + kb * kSlotBytes;
                    mbar_expect_tx(KI_FULL(kb), 2 * kKeys * 128u);
                    for (int h = 0; h < 2; ++h) tma_load_2d(dst + h * kHalf, &prm.mapKI, h * 64, krow, KI_FULL(kb));
                }
                ++ki_loads;
                for (int it = 0; it < 10 && ok; ++it) {  // K0 Q0 K1 Q1 ... K4 Q4 (chunk 4 = the 64 rope dims)
                    if (lane == 0) ok = WAIT(EMPTY(slot), sphase ^ 1, 61);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    if (lane == 0) {
                        const uint32_t dst = sbase + slot * kSlotBytes;
                        const int c = it >> 1;
                        const int halves = c < 4 ? 2 : 1;
                        const bool is_q = it & 1;
                        mbar_expect_tx(FULL(slot), halves * (is_q ? N1 : kKeys) * 128u);
                        for (int h = 0; h < halves; ++h) {
                            const int col = c < 4 ? c * 128 + h * 64 : 0;
                            if (is_q)
                                tma_load_2d(dst + h * kHalf, c < 4 ? &prm.mapQ : &prm.mapQr, col, t * N1, FULL(slot));
                            else
                                tma_load_2d(dst + h * kHalf, c < 4 ? &prm.mapK : &prm.mapKr, col, krow, FULL(slot));
                        }
                        issued_mask |= 1u << slot;
                    }
                    __syncwarp();
                    if (++slot == kSlots) { slot = 0; sphase ^= 1; }
                }
                if (ok && tile == 0) {
                    // the previous row's last gradient MMAs have read its q~I
                    if (lane == 0) ok = WAIT(QI_EMPTY, (row_ctr & 1) ^ 1, 59);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (ok && lane == 0) {
                        mbar_expect_tx(QI_FULL, 2 * kG * 128u);
                        for (int h = 0; h < 2; ++h)
                            tma_load_2d(sbase + kOffQI + h * kQIHalf, &prm.mapQI, h * 64, t * kG, QI_FULL);
                    }
                    if (ok) ++qi_loads;
                }
            }
            ++row_ctr;
        }
        if (lane == 0) {  // drain: every issued load must land before the CTA exits
            for (int k = 0; k < kSlots; ++k) {
                const int s = (slot + k) % kSlots;
                const uint32_t ph = s < slot ? sphase : sphase ^ 1;
                if (issued_mask & (1u << s)) {
                    uint64_t t0 = globaltimer();
                    while (!mbar_try(FULL(s), ph) && globaltimer() - t0 < 1000000000ull) {
                    }
                }
            }
            // the last load into each K~I buffer and the last q~I load
            for (int k = 1; k <= 2; ++k) {
                const int c = ki_loads - k;
                if (c >= 0) {
                    uint64_t t0 = globaltimer();
                    while (!mbar_try(KI_FULL(c & 1), (c >> 1) & 1) && globaltimer() - t0 < 1000000000ull) {
                    }
                }
            }
            if (qi_loads > 0) {
                uint64_t t0 = globaltimer();
                while (!mbar_try(QI_FULL, (qi_loads - 1) & 1) && globaltimer() - t0 < 1000000000ull) {
                }
            }
        }
    } else if (warp == 5) {
        // =================== MMA issuer ===================
        const uint32_t ID_S = idesc(128, N1, false, false, kF16);   // S~^T: A = key chunk, B = q chunk (K-major)
        const uint32_t ID_SI = idesc(128, kG, false, false, kF16);  // SI^T: A = K~I, B = q~I (K-major)
        const uint32_t ID_DQ = idesc(128, kG, true, true, kF16);    // dq~I^T: A = K~I (MN), B = dS (MN, N = heads)
        const uint32_t ID_DK = idesc(128, 128, true, false, kF16);  // dK~I^T: A = q~I (MN), B = dS (K-major, N = keys)
        const uint32_t sDS = sbase + kOffDS;
        int slot = 0;
        uint32_t sphase = 0;
        int tile_ctr = 0, row_ctr = 0;
        bool ok = true;
        auto wait_full = [&](int code) -> bool {
            bool r = true;
            if (lane == 0) r = WAIT(FULL(slot), sphase, code);
            r = __shfl_sync(0xffffffffu, r, 0);
            if (r) tc_fence_after();
            return r;
        };
        auto advance = [&]() {
            if (++slot == kSlots) { slot = 0; sphase ^= 1; }
        };
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nkeys[t];
            if (n <= 0) continue;
            const int ntiles = (n + kKeys - 1) / kKeys;
            for (int tile = 0; tile < ntiles && ok; ++tile, ++tile_ctr) {
                // ---- S~^T over the five chunks ----
                for (int c = 0; c < 5 && ok; ++c) {
                    ok = wait_full(62);
                    if (!ok) break;
                    const uint32_t sk = sbase + slot * kSlotBytes;
                    const int kslot = slot;
                    advance();
                    ok = wait_full(63);
                    if (!ok) break;
                    const uint32_t sq = sbase + slot * kSlotBytes;
                    if (lane == 0) {
                        const int ksteps = c < 4 ? 8 : 4;
                        for (int ks = 0; ks < ksteps; ++ks) {
                            const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                            mma(T_SM, sdesc(sk + off, 16, 1024), sdesc(sq + off, 16, 1024), ID_S,
                                (c > 0 || ks > 0) ? 1u : 0u);
                        }
                        mma_commit(EMPTY(slot));
                        mma_commit(EMPTY(kslot));
                    }
                    __syncwarp();
                    advance();
                }
                if (!ok) break;
                // ---- SI^T from this tile's K~I buffer and the row's q~I ----
                const int kb = tile_ctr & 1;
                const uint32_t ski = sbase + kOffKI + kb * kSlotBytes;
                const uint32_t sqi = sbase + kOffQI;
                if (lane == 0) ok = WAIT(KI_FULL(kb), (tile_ctr >> 1) & 1, 64);
                if (lane == 0 && ok && tile == 0) ok = WAIT(QI_FULL, row_ctr & 1, 65);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    for (int ks = 0; ks < kDi / 16; ++ks) {
                        const uint32_t oa = (ks >> 2) * kHalf + (ks & 3) * 32;
                        const uint32_t ob = (ks >> 2) * kQIHalf + (ks & 3) * 32;
                        mma(T_SI, sdesc(ski + oa, 16, 1024), sdesc(sqi + ob, 16, 1024), ID_SI, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(S_FULL);
                }
                __syncwarp();
                // ---- gradients ----
                if (lane == 0) ok = WAIT(DS_FULL, tile_ctr & 1, 66);
                // the first tile of a row overwrites dq~I^T: the previous row's must have been read
                if (lane == 0 && ok && tile == 0) ok = WAIT(DQI_FREE, (row_ctr & 1) ^ 1, 67);
                if (lane == 0 && ok) ok = WAIT(DKI_EMPTY, (tile_ctr & 1) ^ 1, 68);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    // dq~I^T [Di x G] += K~I^T . dS^T (K = keys, 16 per step)
                    for (int ks = 0; ks < kKeys / 16; ++ks)
                        mma(T_DQI, sdesc(ski + ks * 2048, kHalf, 1024), sdesc(sDS + ks * 2048, kHalf, 1024), ID_DQ,
                            (tile > 0 || ks > 0) ? 1u : 0u);
                    // dK~I^T [Di x keys] = q~I^T . dS (K = G heads, 16 per step)
                    for (int ks = 0; ks < kG / 16; ++ks)
                        mma(T_DKI, sdesc(sqi + ks * 2048, kQIHalf, 1024), sdesc(sDS + ks * 32, 16, 1024), ID_DK,
                            ks > 0 ? 1u : 0u);
                    mma_commit(DKI_FULL);
                    mma_commit(DS_FREE);
                    mma_commit(KI_EMPTY(kb));
                    if (tile == ntiles - 1) {
                        mma_commit(DQI_FULL);
                        mma_commit(QI_EMPTY);
                    }
                }
                __syncwarp();
            }
            ++row_ctr;
        }
        if (lane == 0) {  // drain: the last MMAs complete before TMEM is freed
            mma_commit(DONE);
            uint64_t t0 = globaltimer();
            while (!mbar_try(DONE, 0) && globaltimer() - t0 < 1000000000ull) {
            }
        }
    } else if (warp < 4) {
        // =================== compute: scores, loss, dS, dK~I flush, row write-out ===================
        const int j = threadIdx.x;  // key slot of the tile (scores) / dim (write-out)
        const float c1 = prm.scale * 1.4426950408889634f;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        uint8_t* sDSp = smem + kOffDS;
        const float inv_n1 = 1.f / (float)N1;
        int tile_ctr = 0, row_ctr = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nkeys[t];
            if (n <= 0) {
                // no visible key: zero dq~I and dW rows, zero loss
                T* dq = reinterpret_cast<T*>(prm.dqi_out) + (int64_t)t * kG * kDi;
                for (int i = j; i < kG * kDi; i += 128) dq[i] = cvt16<T>(0.f);
                if (j < kG) reinterpret_cast<T*>(prm.dw_out)[(int64_t)t * kG + j] = cvt16<T>(0.f);
                if (j == 0) prm.loss_rows[t] = 0.f;
                continue;
            }
            const int kv0 = prm.kvrow[t];
            compute_sync();
            if (j < N1) {
                const float l = prm.ssum[(int64_t)t * N1 + j];
                cst[j] = prm.smax[(int64_t)t * N1 + j] * 1.4426950408889634f;
                cst[128 + j] = l == 0.f ? 0.f : 1.f / l;
            }
            if (j < kG) cst[256 + j] = ld16<T>(prm.weights, (int64_t)t * kG + j);
            if (j == 0) {
                const float li = prm.ssum_i[t];
                cst[580] = prm.smax_i[t] * 1.4426950408889634f;
                cst[581] = li > 0.f ? 1.f / li : 0.f;
                cst[582] = li > 0.f ? logf(li) : 0.f;
                cst[583] = prm.smax_i[t];
            }
            compute_sync();
            const float mi2 = cst[580], inv_li = cst[581], log_li = cst[582], mi = cst[583];
            float dw[kG];
#pragma unroll
            for (int g = 0; g < kG; ++g) dw[g] = 0.f;
            float loss = 0.f;
            const int ntiles = (n + kKeys - 1) / kKeys;
            for (int tile = 0; tile < ntiles && ok; ++tile, ++tile_ctr) {
                const bool kv = tile * kKeys + j < n;
                ok = WAIT(S_FULL, tile_ctr & 1, 69);
                if (ok && tile_ctr > 0) ok = WAIT(DS_FREE, (tile_ctr - 1) & 1, 70);
                ok = compute_all(ok);
                if (!ok) break;
                tc_fence_after();
                // indexer score I_j = sum_g W_g ReLU(SI_gj)
                float I = 0.f;
#pragma unroll 1
                for (int cc = 0; cc < kG / 32; ++cc) {
                    float s[32];
                    tmem_ld32(T_SI + lane_base + cc * 32, s);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) I = fmaf(cst[256 + cc * 32 + e], fmaxf(s[e], 0.f), I);
                }
                // target p_j = mean over heads of exp(scale*S - max) / sum
                float p = 0.f;
#pragma unroll 1
                for (int cc = 0; cc < N1 / 32; ++cc) {
                    float s[32];
                    tmem_ld32(T_SM + lane_base + cc * 32, s);
                    tmem_wait_ld();
                    const float4* cm = reinterpret_cast<const float4*>(cst + cc * 32);
                    const float4* cl = reinterpret_cast<const float4*>(cst + 128 + cc * 32);
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const float4 m4 = cm[g], l4 = cl[g];
                        p = fmaf(ex2_approx(fmaf(s[4 * g + 0], c1, -m4.x)), l4.x, p);
                        p = fmaf(ex2_approx(fmaf(s[4 * g + 1], c1, -m4.y)), l4.y, p);
                        p = fmaf(ex2_approx(fmaf(s[4 * g + 2], c1, -m4.z)), l4.z, p);
                        p = fmaf(ex2_approx(fmaf(s[4 * g + 3], c1, -m4.w)), l4.w, p);
                    }
                }
                // padding keys of the last tile (rows past the row's visible keys) are selected out
                p = kv ? p * inv_n1 : 0.f;
                const float si = kv ? ex2_approx(fmaf(I, 1.4426950408889634f, -mi2)) * inv_li : 0.f;
                const float di = si - p;
                if (kv && p > 0.f) loss += p * (logf(p) - ((I - mi) - log_li));
                // dW partials and dS (16-bit, row j of the [keys x G] SW128 block)
#pragma unroll 1
                for (int cc = 0; cc < kG / 32; ++cc) {
                    float s[32];
                    tmem_ld32(T_SI + lane_base + cc * 32, s);
                    tmem_wait_ld();
                    uint32_t pw[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float w0 = cst[256 + cc * 32 + e], w1 = cst[256 + cc * 32 + e + 1];
                        const float d0 = s[e] > 0.f ? di * w0 : 0.f;
                        const float d1 = s[e + 1] > 0.f ? di * w1 : 0.f;
                        pw[e >> 1] = pack2<T>(d0, d1);
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        // dw[] is indexed statically: cc selects one of two unrolled halves
                        const float r = fmaxf(s[e], 0.f) * di;
                        if (cc == 0) dw[e] += r;
                        else dw[32 + e] += r;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t off = j * 128 + (((cc * 4 + u) ^ (j & 7)) << 4);
                        *reinterpret_cast<uint4*>(sDSp + off) =
                            make_uint4(pw[4 * u], pw[4 * u + 1], pw[4 * u + 2], pw[4 * u + 3]);
                    }
                }
                fence_view_async_shared();
                tc_fence_before();
                mbar_arrive(DS_FULL);
                // dK~I^T of this tile: lane = dim, column = key
                ok = compute_all(WAIT(DKI_FULL, tile_ctr & 1, 71));
                if (!ok) break;
                tc_fence_after();
                const int nvalid = min(kKeys, n - tile * kKeys);
                float* acc = prm.dki_acc + (int64_t)(kv0 + tile * kKeys) * kDi + j;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    if (cc * 32 >= nvalid) break;  // uniform over the warp
                    float v[32];
                    tmem_ld32(T_DKI + lane_base + cc * 32, v);
                    tmem_wait_ld();
                    const int lim = nvalid - cc * 32;
                    float* d = acc + (int64_t)cc * 32 * kDi;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e < lim) atomicAdd(d + (int64_t)e * kDi, v[e]);
                }
                tc_fence_before();
                mbar_arrive(DKI_EMPTY);
            }
            if (!ok) break;
            // ---- row end: dq~I (lane = dim), dW and the row's loss ----
            ok = compute_all(WAIT(DQI_FULL, row_ctr & 1, 72));
            if (!ok) break;
            tc_fence_after();
            {
                T* dq = reinterpret_cast<T*>(prm.dqi_out) + (int64_t)t * kG * kDi + j;
#pragma unroll 1
                for (int cc = 0; cc < kG / 32; ++cc) {
                    float v[32];
                    tmem_ld32(T_DQI + lane_base + cc * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) dq[(int64_t)(cc * 32 + e) * kDi] = cvt16<T>(v[e]);
                }
            }
            tc_fence_before();
            mbar_arrive(DQI_FREE);
            fold_half<64>(dw, lane, 16);
            fold_half<32>(dw, lane, 8);
            fold_half<16>(dw, lane, 4);
            fold_half<8>(dw, lane, 2);
            fold_half<4>(dw, lane, 1);
            for (int o = 16; o; o >>= 1) loss += __shfl_xor_sync(0xffffffffu, loss, o);
            cst[320 + warp * 64 + 2 * lane] = dw[0];
            cst[320 + warp * 64 + 2 * lane + 1] = dw[1];
            if (lane == 0) cst[576 + warp] = loss;
            compute_sync();
            if (j < kG) {
                const float s = cst[320 + j] + cst[384 + j] + cst[448 + j] + cst[512 + j];
                reinterpret_cast<T*>(prm.dw_out)[(int64_t)t * kG + j] = cvt16<T>(s);
            }
            if (j == 0) prm.loss_rows[t] = cst[576] + cst[577] + cst[578] + cst[579];
            ++row_ctr;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

template <typename T, int N1>
cudaError_t launch_t(const LigArgs& a, cudaStream_t st) {
    LigParams p;
    memset(&p, 0, sizeof p);
    const int64_t T1 = a.T1, T2 = a.T2;
    if (!make_map(&p.mapQ, a.q, a.dtype, kD, (uint64_t)T1 * N1, kD, N1) ||
        !make_map(&p.mapQr, a.qr, a.dtype, kDr, (uint64_t)T1 * N1, kDr, N1) ||
        !make_map(&p.mapK, a.k, a.dtype, kD, (uint64_t)T2, kD, kKeys) ||
        !make_map(&p.mapKr, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, kKeys) ||
        !make_map(&p.mapQI, a.qi, a.dtype, kLigDi, (uint64_t)T1 * kLigG, kLigDi, kLigG) ||
        !make_map(&p.mapKI, a.ki, a.dtype, kLigDi, (uint64_t)T2, kLigDi, kKeys))
        return cudaErrorInvalidValue;
    p.nkeys = a.nkeys;
    p.kvrow = a.kvrow;
    p.order = a.order;
    p.smax = a.smax;
    p.ssum = a.ssum;
    p.smax_i = a.smax_i;
    p.ssum_i = a.ssum_i;
    p.weights = a.weights;
    p.dki_acc = a.dki_acc;
    p.dqi_out = a.dqi;
    p.dw_out = a.dw;
    p.loss_rows = a.loss_rows;
    p.err = a.err;
    p.T1 = T1;
    p.scale = a.scale;
    p.wait_ns = wait_limit_ns();
    auto kern = lig_fused_kernel<T, N1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (int)(T1 < sms ? T1 : sms);
    if (grid < 1) return cudaSuccess;
    kern<<<grid, kThreads, kSmem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

// Per query row: the number of key rows it sees (the whole sequence in sparseMode
// 0, the causal prefix j <= pos + S2_b - S1_b in mode 3, none for a BSND padding
// row) and the global row of the first one.
__global__ void lig_rows_kernel(SeqDesc sd, int mode, int32_t* __restrict__ nkeys, int32_t* __restrict__ kvrow) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= sd.T1) return;
    const TokInfo ti = tok_info(sd, t);
    int64_t n = 0;
    if (ti.valid) {
        n = ti.kv_len;
        if (mode == 3) n = clamp64((int64_t)ti.pos + 1 + ti.kv_len - ti.q_len, 0, ti.kv_len);
    }
    nkeys[t] = (int32_t)n;
    kvrow[t] = (int32_t)ti.kv_start;
}

// int64 sequence lengths (as the indexer gradient takes them) -> the int32 form the
// row bookkeeping reads, clamped to [0, 2^31 - 1].
__global__ void lig_seqlens_kernel(const int64_t* __restrict__ in, int32_t* __restrict__ out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = (int32_t)clamp64(in[i], 0, 0x7fffffff);
}

// fp32 [T2][Di] accumulator -> 16-bit dKeyIndex.
template <typename T>
__global__ void lig_cast_kernel(const float* __restrict__ acc, int64_t n, T* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = cvt16<T>(acc[i]);
}

// Sum of the per-row losses in a fixed order (one CTA): a deterministic scalar.
__global__ void lig_loss_kernel(const float* __restrict__ rows, int64_t n, float* __restrict__ loss) {
    __shared__ double part[256];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += 256) s += rows[i];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int o = 128; o; o >>= 1) {
        if ((int)threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *loss = (float)part[0];
}

cudaError_t launch_lig_prep(const SeqDesc& sd, int mode, const int64_t* sq64, const int64_t* skv64, int32_t* sq32,
                            int32_t* skv32, int32_t* nkeys, int32_t* kvrow, cudaStream_t st) {
    if (sq64) lig_seqlens_kernel<<<1, 256, 0, st>>>(sq64, sq32, sd.B);
    if (skv64) lig_seqlens_kernel<<<1, 256, 0, st>>>(skv64, skv32, sd.B);
    SeqDesc d = sd;
    d.seq_q = sq64 ? sq32 : nullptr;
    d.seq_kv = skv64 ? skv32 : nullptr;
    if (d.T1 > 0) lig_rows_kernel<<<(unsigned)((d.T1 + 255) / 256), 256, 0, st>>>(d, mode, nkeys, kvrow);
    return cudaGetLastError();
}

cudaError_t launch_lig_finish(int dtype, const float* dki_acc, int64_t T2, void* dki, const float* loss_rows,
                              int64_t T1, float* loss, cudaStream_t st) {
    const int64_t n = T2 * kLigDi;
    const unsigned grid = (unsigned)std::min<int64_t>((n + 255) / 256, 4096);
    if (n > 0) {
        if (dtype == SFA_DTYPE_BF16) lig_cast_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(dki_acc, n, (__nv_bfloat16*)dki);
        else lig_cast_kernel<__half><<<grid, 256, 0, st>>>(dki_acc, n, (__half*)dki);
    }
    lig_loss_kernel<<<1, 256, 0, st>>>(loss_rows, T1, loss);
    return cudaGetLastError();
}

cudaError_t launch_lig_fused(const LigArgs& a, cudaStream_t st) {
    if (a.dtype == SFA_DTYPE_BF16)
        return a.N1 == 128 ? launch_t<__nv_bfloat16, 128>(a, st) : launch_t<__nv_bfloat16, 64>(a, st);
    return a.N1 == 128 ? launch_t<__half, 128>(a, st) : launch_t<__half, 64>(a, st);
}

}  // namespace sfa
