// Fused tensor-core sparse attention forward for sm_100a, N1 = 128 query heads
// sharing one KV head, value == key (first 512 dims).
//
// What it computes (FlashAttentionUnpaddingScoreGrad page, 计算公式: S = scale *
// Q.K^T, P = Softmax(S), Y = P.V; over each query row's gathered key rows as in
// the SparseFlashAttentionGrad README, 功能说明 Gather):
//   softmaxMax = max_j scale * Q~.K~_j          (per head)
//   softmaxSum = sum_j exp(scale * Q~.K~_j - softmaxMax)
//   out        = sum_j exp(scale * Q~.K~_j - softmaxMax) / softmaxSum * V_j
//
// Work item = one query row.  Two passes over its 128-key tiles reuse the same
// S = Q~.K~^T MMA ([128 heads x 128 keys], K = 576, TMEM lane = head):
//   pass 1: a per-head running max m_run; P = exp2(S*scale*log2e - m_used) to shared
//   memory (16-bit, SW128) and out[:, 0, 256) += P . V in TMEM, where m_used follows
//   m_run lazily: only when m_run exceeds it by more than 8 (log2 units) are the
//   accumulated half and the running sum rescaled, so P stays below 2^8; the half is
//   divided by the sum when written out, and the statistics are taken relative to the
//   true max;
//   pass 2: P = exp2(S*scale*log2e - (m_used + log2 sum)), out[:, 256, 512) += P . V.
// V's two 128-dim chunks are the key chunks the S MMA just read.  Recomputing S once
// (2x 19 MFLOP per tile against 17 MFLOP of P.V) keeps the 512-dim fp32 output half
// (256 TMEM columns) and two S buffers within TMEM.
// Key rows arrive by TMA tile::gather4, or, when the row lists are block-aligned
// runs of 16 contiguous rows (block size a multiple of 16; padding slots flagged
// with bit 31), as one 16-row 2-D tile per run (~2.7x the gather rate on B200), or,
// when all 128 rows of a tile are consecutive (sorted block lists), as one 128-row
// 2-D tile per 64-column half.
// Warps: 0-3 softmax / output write-out (thread = head), 4 TMA producer, 5 MMA.
// Every mbarrier wait is bounded; on timeout the kernel records an error word,
// stops issuing, drains its loads and frees its TMEM.
#include <cuda.h>

#include <cstring>
#include <type_traits>

#include "sfa_internal.cuh"
#include "tc_common.cuh"

namespace sfa {

namespace {

using namespace tc;

constexpr int kN1 = 128;
constexpr int kThreads = 192;
constexpr int kSlots = 6;
constexpr int kSlotBytes = 32768;
constexpr int kHalf = 16384;
constexpr int kKeys = 128;
constexpr float kLazy = 8.f;  // log2 headroom of P before the output half is rescaled
constexpr int kOffP = kSlots * kSlotBytes;       // P [128 heads x 128 keys] 16-bit, two SW128 halves
constexpr int kOffBar = kOffP + 32768;
constexpr int kNumBars = 2 * kSlots + 11;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 16;

struct FwdParams {
    CUtensorMap mapQ, mapQr, mapK, mapKr;
    CUtensorMap mapK16, mapKr16;    // 16-row boxes (block-aligned row lists)
    CUtensorMap mapK128, mapKr128;  // 128-row boxes (tiles of consecutive key rows)
    const int32_t* rowlist;  // [T1][cap] global key rows of each query row
    const int32_t* nrows;    // [T1]
    const int32_t* order;    // [T1] work order
    void* out;               // [T1][N1][512]
    float* smax;             // [T1][N1]
    float* ssum;
    int* err;
    int64_t T1;
    int64_t cap;
    float scale;
    int blk16;
    uint64_t wait_ns;  // limit of every mbarrier wait
};

// Chunk order of a pass: pass 0 any order; pass 1 / 2 put the two value chunks of
// their output half (2h, 2h+1) last, so those key slots are held shortest.
__device__ __forceinline__ int chunk_of(int pass, int i) {
    if (pass == 1) return (i + 2) % 5;           // 2 3 4 0 1
    if (pass == 2) return i < 2 ? i : (i == 2 ? 4 : i - 1);  // 0 1 4 2 3
    return i;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) sfa_fwd_fused_kernel(const __grid_constant__ FwdParams prm) {
    constexpr bool kF16 = std::is_same<T, __half>::value;
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
    auto S_FULL = [&](int b) { return bar0 + 8u * (2 * kSlots + b); };
    auto S_FREE = [&](int b) { return bar0 + 8u * (2 * kSlots + 2 + b); };
    const uint32_t P_FULL = bar0 + 8u * (2 * kSlots + 4);
    const uint32_t P_FREE = bar0 + 8u * (2 * kSlots + 5);
    const uint32_t O_FULL = bar0 + 8u * (2 * kSlots + 6);
    const uint32_t O_EMPTY = bar0 + 8u * (2 * kSlots + 7);
    const uint32_t DONE = bar0 + 8u * (2 * kSlots + 8);
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
        for (int b = 0; b < 2; ++b) {
            mbar_init(S_FULL(b), 1);
            mbar_init(S_FREE(b), 128);
        }
        mbar_init(P_FULL, 128);
        mbar_init(P_FREE, 1);
        mbar_init(O_FULL, 1);
        mbar_init(O_EMPTY, 128);
        mbar_init(DONE, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {  // S buffers [0,128) and [128,256), output half [256,512)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto T_S = [&](int b) { return tmem + 128u * b; };
    const uint32_t T_O = tmem + 256;
    const int nwork = (int)prm.T1;

    if (warp == 4) {
        // =================== TMA producer ===================
        int slot = 0;
        uint32_t sphase = 0;
        bool ok = true;
        uint32_t issued_mask = 0;
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nrows[t];
            if (n <= 0) continue;
            const int32_t* rl = prm.rowlist + (int64_t)t * prm.cap;
            const int ntiles = (n + kKeys - 1) / kKeys;
            const int first = rl[0] & 0x7fffffff;
            for (int pass = 1; pass < 3 && ok; ++pass) {
                for (int tile = 0; tile < ntiles && ok; ++tile) {
                    int32_t my[4];  // lane L gathers key rows 4L..4L+3 of the tile
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = tile * kKeys + 4 * lane + e;
                        my[e] = s < n ? rl[s] & 0x7fffffff : first;
                    }
                    // block-aligned lists: lane L < 16 loads half L/8, 16-row group L%8 from the
                    // group's first row (always a kept row; groups past the list reload the first)
                    int gfirst = first;
                    if (prm.blk16) {
                        const int s = tile * kKeys + 16 * (lane & 7);
                        gfirst = s < n ? rl[s] & 0x7fffffff : first;
                    }
                    // a tile whose slots hold rows run0, run0+1, ... (padding flags aside) is one
                    // 128-row 2-D tile; its slots past the list then hold rows run0+s, masked
                    const int run0 = rl[tile * kKeys] & 0x7fffffff;
                    bool contig = true;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = tile * kKeys + 4 * lane + e;
                        if (s < n && my[e] != run0 + 4 * lane + e) contig = false;
                    }
                    contig = __all_sync(0xffffffffu, contig);
                    for (int i = 0; i < 10 && ok; ++i) {
                        const int c = chunk_of(pass, i >> 1);
                        const bool is_key = (i & 1) == 0;
                        if (lane == 0) ok = WAIT(EMPTY(slot), sphase ^ 1, 41);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        const uint32_t dst = sbase + slot * kSlotBytes;
                        const int halves = c < 4 ? 2 : 1;
                        if (lane == 0) mbar_expect_tx(FULL(slot), halves * 128u * 128u);
                        __syncwarp();
                        if (is_key && contig) {
                            if (lane == 0) {
                                const CUtensorMap* map = c < 4 ? &prm.mapK128 : &prm.mapKr128;
                                for (int h = 0; h < halves; ++h)
                                    tma_load_2d(dst + h * kHalf, map, c < 4 ? c * 128 + h * 64 : 0, run0, FULL(slot));
                            }
                        } else if (is_key && prm.blk16) {
                            const int h = lane >> 3;
                            if (lane < 8 * halves)
                                tma_load_2d(dst + h * kHalf + (lane & 7) * 2048, c < 4 ? &prm.mapK16 : &prm.mapKr16,
                                            c < 4 ? c * 128 + h * 64 : 0, gfirst, FULL(slot));
                        } else if (is_key) {
                            const CUtensorMap* map = c < 4 ? &prm.mapK : &prm.mapKr;
                            for (int h = 0; h < halves; ++h)
                                tma_gather4(dst + h * kHalf + lane * 512, map, c < 4 ? c * 128 + h * 64 : 0, my[0],
                                            my[1], my[2], my[3], FULL(slot));
                        } else if (lane == 0) {
                            const CUtensorMap* map = c < 4 ? &prm.mapQ : &prm.mapQr;
                            for (int h = 0; h < halves; ++h)
                                tma_load_2d(dst + h * kHalf, map, c < 4 ? c * 128 + h * 64 : 0, t * kN1, FULL(slot));
                        }
                        if (lane == 0) issued_mask |= 1u << slot;
                        if (++slot == kSlots) { slot = 0; sphase ^= 1; }
                    }
                }
            }
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
        }
    } else if (warp == 5) {
        // =================== MMA issuer ===================
        const uint32_t ID_S = idesc(128, 128, false, false, kF16);  // S = Q~.K~^T (A = q chunk, B = key chunk)
        const uint32_t ID_O = idesc(128, 128, false, true, kF16);   // out += P.V (A = P K-major, B = V MN-major)
        const uint32_t sP = sbase + kOffP;
        int slot = 0;
        uint32_t sphase = 0;
        int s_ctr = 0, p_ctr = 0, o_ctr = 0;
        bool ok = true;
        auto wait_full = [&]() -> bool {
            bool r = true;
            if (lane == 0) r = WAIT(FULL(slot), sphase, 42);
            r = __shfl_sync(0xffffffffu, r, 0);
            if (r) tc_fence_after();
            return r;
        };
        auto advance = [&]() {
            if (++slot == kSlots) { slot = 0; sphase ^= 1; }
        };
        // S of one tile into buffer s_ctr & 1; returns the slots of the value chunks
        // (the last two key chunks of an output pass), still held
        auto issue_s = [&](int pass, uint32_t (&vslot)[2]) -> bool {
            const int b = s_ctr & 1;
            bool r = true;
            if (lane == 0) r = WAIT(S_FREE(b), ((s_ctr >> 1) & 1) ^ 1, 43);
            r = __shfl_sync(0xffffffffu, r, 0);
            if (!r) return false;
            tc_fence_after();
            for (int i = 0; i < 5; ++i) {
                const int c = chunk_of(pass, i);
                if (!wait_full()) return false;
                const uint32_t sk = sbase + slot * kSlotBytes;
                const int kslot = slot;
                advance();
                if (!wait_full()) return false;
                const uint32_t sq = sbase + slot * kSlotBytes;
                if (lane == 0) {
                    const int ksteps = c < 4 ? 8 : 4;
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                        mma(T_S(b), sdesc(sq + off, 16, 1024), sdesc(sk + off, 16, 1024), ID_S,
                            (i > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(EMPTY(slot));                     // q chunk
                    if (pass == 0 || i < 3) mma_commit(EMPTY(kslot));  // key chunk not needed as a value
                }
                if (pass > 0 && i >= 3) vslot[i - 3] = (uint32_t)kslot;
                __syncwarp();
                advance();
            }
            if (lane == 0) mma_commit(S_FULL(b));
            __syncwarp();
            ++s_ctr;
            return true;
        };
        // out half += P . V of one tile (P from the softmax warps; V = the held key chunks)
        auto issue_o = [&](bool first_tile, const uint32_t (&vslot)[2]) -> bool {
            bool r = true;
            if (lane == 0) r = WAIT(P_FULL, p_ctr & 1, 44);
            r = __shfl_sync(0xffffffffu, r, 0);
            if (!r) return false;
            tc_fence_after();
            if (lane == 0) {
                for (int v = 0; v < 2; ++v) {
                    const uint32_t sv = sbase + vslot[v] * kSlotBytes;
                    for (int ks = 0; ks < kKeys / 16; ++ks) {
                        const uint64_t a = sdesc(sP + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
                        const uint64_t bdesc = sdesc(sv + ks * 2048, kHalf, 1024);
                        mma(T_O + 128u * v, a, bdesc, ID_O, (!first_tile || ks > 0) ? 1u : 0u);
                    }
                }
                mma_commit(P_FREE);
                mma_commit(EMPTY(vslot[0]));
                mma_commit(EMPTY(vslot[1]));
            }
            __syncwarp();
            ++p_ctr;
            return true;
        };
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nrows[t];
            if (n <= 0) continue;
            const int ntiles = (n + kKeys - 1) / kKeys;
            for (int pass = 1; pass < 3 && ok; ++pass) {
                // the previous output half has been written out
                if (lane == 0) ok = WAIT(O_EMPTY, (o_ctr & 1) ^ 1, 45);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after();
                // S then P.V per tile, in ring order: the value chunks stay in their key slots
                // until the output MMA reads them, and the producer's next loads wait for those
                // slots, so the next tile's S must not be issued before this tile's output MMA
                for (int tile = 0; tile < ntiles && ok; ++tile) {
                    uint32_t vs[2];
                    ok = issue_s(pass, vs);
                    if (ok) ok = issue_o(tile == 0, vs);
                }
                if (!ok) break;
                if (lane == 0) mma_commit(O_FULL);
                __syncwarp();
                ++o_ctr;
            }
        }
        if (lane == 0) {
            mma_commit(DONE);
            uint64_t t0 = globaltimer();
            while (!mbar_try(DONE, 0) && globaltimer() - t0 < 1000000000ull) {
            }
        }
    } else {
        // =================== softmax / output (TMEM lane = head) ===================
        const int h = threadIdx.x;  // head
        const float c1 = prm.scale * 1.4426950408889634f;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        uint8_t* sPp = smem + kOffP;
        int s_ctr = 0, p_ctr = 0, o_ctr = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nrows[t];
            const int64_t row = (int64_t)t * kN1 + h;
            if (n <= 0) {  // no key for this query row (or a BSND padding row)
                uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<T*>(prm.out) + row * kD);
                for (int i = 0; i < kD / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
                prm.smax[row] = 0.f;
                prm.ssum[row] = 0.f;
                continue;
            }
            const int ntiles = (n + kKeys - 1) / kKeys;
            const int32_t* rl = prm.rowlist + (int64_t)t * prm.cap;
            // kept keys of a tile as four 32-bit masks (slot < n and not a block-padding slot)
            auto tile_mask = [&](int tile, uint32_t (&mk)[4]) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int s = tile * kKeys + 32 * k + lane;
                    mk[k] = __ballot_sync(0xffffffffu, s < n && rl[s] >= 0);
                }
            };
            // pass 1: output half 0 with a running max (lazy rescaling); pass 2: half 1 with the
            // final statistics.  m_run = max * log2e so far; P is taken relative to m_used, which
            // moves up (rescaling the accumulated half and the sum) only when m_run exceeds it by
            // more than kLazy, so P stays below 2^kLazy.
            float m_run = -INFINITY, m_used = -INFINITY, l = 0.f, mc = 0.f;
            for (int pass = 1; pass < 3 && ok; ++pass, ++o_ctr) {
                for (int tile = 0; tile < ntiles && ok; ++tile, ++s_ctr, ++p_ctr) {
                    const int b = s_ctr & 1;
                    ok = WAIT(S_FULL(b), (s_ctr >> 1) & 1, 47);
                    // P of the previous tile has been read by its output MMA (the half is stable)
                    if (ok) ok = WAIT(P_FREE, (p_ctr & 1) ^ 1, 48);
                    ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-collective
                    if (!ok) break;
                    tc_fence_after();
                    uint32_t mk[4];
                    tile_mask(tile, mk);
                    float msub = mc;  // pass 2: P = exp2(S*c1 - (m_used + log2 l)), normalised
                    if (pass == 1) {
                        float tmax = -INFINITY;
#pragma unroll 1
                        for (int cc = 0; cc < 4; ++cc) {
                            float sv[32];
                            tmem_ld32(T_S(b) + lane_base + cc * 32, sv);
                            tmem_wait_ld();
                            const uint32_t mw = cc == 0 ? mk[0] : cc == 1 ? mk[1] : cc == 2 ? mk[2] : mk[3];
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if ((mw >> e) & 1u) tmax = fmaxf(tmax, sv[e]);
                        }
                        m_run = fmaxf(m_run, tmax * c1);
                        // the decision is per head (thread); the TMEM loads / stores below are
                        // warp-collective, so a warp rescales when any of its heads needs it and
                        // the other heads apply a factor of 1
                        const bool need = m_run > m_used + kLazy;
                        const float f = need ? ex2_approx(m_used - m_run) : 1.f;  // 0 on the first tile
                        if (tile > 0 && __any_sync(0xffffffffu, need)) {
                            // rescale the accumulated output half (TMEM lane = head)
#pragma unroll 1
                            for (int cc = 0; cc < 8; ++cc) {
                                float v[32];
                                tmem_ld32(T_O + lane_base + cc * 32, v);
                                tmem_wait_ld();
                                uint32_t r[32];
#pragma unroll
                                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(v[e] * f);
#pragma unroll
                                for (int q = 0; q < 4; ++q) tmem_st8(T_O + lane_base + cc * 32 + 8 * q, r + 8 * q);
                            }
                            tmem_wait_st();
                        }
                        if (need) {
                            l *= f;
                            m_used = m_run;
                        }
                        msub = m_used;
                    }
                    float psum = 0.f;
#pragma unroll 1
                    for (int cc = 0; cc < 4; ++cc) {
                        float sv[32];
                        tmem_ld32(T_S(b) + lane_base + cc * 32, sv);
                        tmem_wait_ld();
                        uint32_t pw[16];
                        const uint32_t mw = cc == 0 ? mk[0] : cc == 1 ? mk[1] : cc == 2 ? mk[2] : mk[3];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float p0 = (mw >> e) & 1u ? ex2_approx(fmaf(sv[e], c1, -msub)) : 0.f;
                            const float p1 = (mw >> (e + 1)) & 1u ? ex2_approx(fmaf(sv[e + 1], c1, -msub)) : 0.f;
                            psum += p0 + p1;
                            pw[e >> 1] = pack2<T>(p0, p1);
                        }
                        // keys [32cc, 32cc+32) of head row h: SW128 half cc/2, 16-byte units 4(cc%2)..+4
                        const int half = cc >> 1, u0 = (cc & 1) * 4;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t off = half * kHalf + h * 128 + (((u0 + u) ^ (h & 7)) << 4);
                            *reinterpret_cast<uint4*>(sPp + off) =
                                make_uint4(pw[4 * u], pw[4 * u + 1], pw[4 * u + 2], pw[4 * u + 3]);
                        }
                    }
                    if (pass == 1) l += psum;
                    fence_view_async_shared();
                    tc_fence_before();
                    mbar_arrive(S_FREE(b));
                    mbar_arrive(P_FULL);
                }
                if (pass == 1 && ok) {
                    // statistics relative to the true max (natural-log units for softmaxMax)
                    prm.smax[row] = m_run * 0.6931471805599453f;
                    prm.ssum[row] = l * ex2_approx(m_used - m_run);
                    mc = m_used + log2f(l);
                }
                if (!ok) break;
                ok = __all_sync(0xffffffffu, WAIT(O_FULL, o_ctr & 1, 49));
                if (!ok) break;
                tc_fence_after();
                T* o = reinterpret_cast<T*>(prm.out) + row * kD + 256 * (pass - 1);
                const float inv = pass == 1 ? 1.f / l : 1.f;  // half 0 holds P relative to m_used, unnormalised
#pragma unroll 1
                for (int cc = 0; cc < 8; ++cc) {
                    float v[32];
                    tmem_ld32(T_O + lane_base + cc * 32, v);
                    tmem_wait_ld();
                    uint32_t wv[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) wv[e >> 1] = pack2<T>(v[e] * inv, v[e + 1] * inv);
                    uint4* d4 = reinterpret_cast<uint4*>(o + cc * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u) d4[u] = make_uint4(wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
                }
                tc_fence_before();
                mbar_arrive(O_EMPTY);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

template <typename T>
cudaError_t launch_t(const FwdFusedArgs& a, cudaStream_t st) {
    FwdParams p;
    memset(&p, 0, sizeof p);
    const int64_t T1 = a.T1, T2 = a.T2;
    if (!make_map(&p.mapQ, a.q, a.dtype, kD, (uint64_t)T1 * kN1, kD, kN1) ||
        !make_map(&p.mapQr, a.qr, a.dtype, kDr, (uint64_t)T1 * kN1, kDr, kN1) ||
        !make_map(&p.mapK, a.k, a.dtype, kD, (uint64_t)T2, kD, 1) ||
        !make_map(&p.mapKr, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, 1) ||
        !make_map(&p.mapK16, a.k, a.dtype, kD, (uint64_t)T2, kD, 16) ||
        !make_map(&p.mapKr16, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, 16) ||
        !make_map(&p.mapK128, a.k, a.dtype, kD, (uint64_t)T2, kD, kKeys) ||
        !make_map(&p.mapKr128, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, kKeys))
        return cudaErrorInvalidValue;
    p.rowlist = a.rowlist;
    p.nrows = a.nrows;
    p.order = a.order;
    p.out = a.out;
    p.smax = a.smax;
    p.ssum = a.ssum;
    p.err = a.err;
    p.T1 = T1;
    p.cap = a.rowcap;
    p.scale = a.scale;
    p.blk16 = a.blk16;
    p.wait_ns = wait_limit_ns();
    auto kern = sfa_fwd_fused_kernel<T>;
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

bool fwd_fused_supported(int64_t N1) { return N1 == kN1; }

cudaError_t launch_fwd_fused(int dtype, const FwdFusedArgs& a, cudaStream_t st) {
    return dtype == SFA_DTYPE_BF16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<__half>(a, st);
}

}  // namespace sfa
