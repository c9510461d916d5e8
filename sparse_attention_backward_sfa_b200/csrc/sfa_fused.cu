// Fused tensor-core sparse attention backward for sm_100a (tcgen05 MMA, TMEM
// accumulators, TMA tile and gather4 loads, mbarrier pipelines).
//
// What it computes (SparseFlashAttentionGrad README, 功能说明, stages 1-3), per
// query row t with its gathered key rows j (value == key, first 512 dims):
//   S^T  = K~ . Q~^T                      [keys x heads], K = 576
//   dP^T = V  . dO^T                      [keys x heads], K = 512
//   P    = exp2(S*scale*log2e - max*log2e) / sum,  dS = P o (dP - rowsum(dO o O))
//   dV^T = dO^T . P^T  -> red into dValue rows      [dims x keys], K = heads
//   dK~^T= Q~^T . dS^T -> red into dKey||dKeyRope   [dims x keys], K = heads
//   dQ~^T= K~^T . dS   -> red into the dQuery rows  [dims x heads], K = keys
//
// Layout decisions (B200):
//  * Work item = one query row (all N1 heads share the single KV head), key
//    tiles of 128 gathered rows.  MMA M is always 128: keys for S^T/dP^T, output
//    dims for every gradient block, so TMEM lane = key during the softmax (per
//    thread masking) and lane = output dim during the flush (each warp-level red
//    covers 32 consecutive fp32 = one 128-byte line).
//  * Every operand is a "chunk" of 128 dims (64 for the rope) held as two
//    128-byte-row SW128 halves 16 KB apart; the same bytes serve as a K-major
//    operand (S^T, dP^T) and as an MN-major one (gradients).  Chunks stream
//    through a ring of 32 KB slots: key rows by TMA tile::gather4 (or one
//    128-row 2-D tile when the tile's rows are consecutive), the query row's
//    q / qRope / dO by 2-D TMA tiles.
//  * The producer and MMA warps run a cross-tile software pipeline: the next
//    tile's S^T / dP^T items are interleaved into this tile's last gradient
//    blocks, so the next scores are formed while this tile's reductions flush.
//  * P and dS live in shared memory as bf16 [keys x heads] (SW128 halves of 64
//    heads); S^T / dP^T and two 128-column staging accumulators live in TMEM
//    (all 512 columns).
//  * Warp roles: 0-3 softmax/dS (TMEM lanes = keys), 4-11 flush (TMEM lanes =
//    dims; two warps per lane quarter, each taking half of a block's columns),
//    12 TMA producer, 13 MMA issuer.  dS is stored pre-multiplied by scale so
//    the flush is a bare reduction.  Every mbarrier wait is bounded; on
//    timeout the kernel records an error word, stops issuing, drains what it
//    issued and frees its TMEM.
#include <cuda.h>

#include <cstring>
#include <type_traits>

#include "sfa_internal.cuh"
#include "tc_common.cuh"

namespace sfa {

namespace {

using namespace tc;

constexpr int kThreads = 448;   // 4 softmax + 8 flush + 1 TMA + 1 MMA warps
constexpr int kSlotBytes = 32768;
constexpr int kHalf = 16384;
constexpr int kKeys = 128;          // key rows per tile (MMA M)

// N1 = 128: every chunk streams through a 5-slot ring of 32 KB.  N1 = 64: the tile's key rows stay
// resident (5 chunks, 144 KB) from the S^T / dP^T items to the dQ~ blocks, so each tile gathers
// them once instead of twice (gathered loads are the slowest TMA operations); q / dO chunks
// (16 KB at 64 heads) stream through a 3-slot ring of 16 KB.
template <int N1> struct Cfg {
    static constexpr bool kResident = N1 == 64;
    static constexpr int kKeyBytes = 4 * kSlotBytes + kHalf;                // resident key tile
    static constexpr int kSlots = N1 == 128 ? 5 : 3;
    static constexpr int kRingSlot = N1 == 128 ? kSlotBytes : 16384;
    static constexpr int kQHalf = N1 * 128;                                 // 64-dim halves of a q / dO chunk
    static constexpr int kOffRing = kResident ? kKeyBytes : 0;
    static constexpr int kOffP = kOffRing + kSlots * kRingSlot;
    static constexpr int kOffDS = kOffP + (N1 == 128 ? 32768 : 16384);
    static constexpr int kOffRows = kOffDS + (N1 == 128 ? 32768 : 16384);  // int32 [2][128]
    static constexpr int kOffConst = kOffRows + 2 * kKeys * 4;              // float [3][128]
    static constexpr int kOffBar = kOffConst + 3 * 128 * 4;
    static constexpr int kNumBars = 2 * kSlots + 12 + (kResident ? 10 : 0);
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmem = kOffMisc + 16;
};
static_assert(Cfg<64>::kSmem <= 232448 && Cfg<128>::kSmem <= 232448, "shared memory per CTA");

struct FusedParams {
    CUtensorMap mapQ, mapQr, mapO, mapK, mapKr;  // dO shares mapO; key maps: 1-row boxes (gather4)
    CUtensorMap mapK128, mapKr128;                // key maps with 128-row boxes (contiguous tiles)
    const int32_t* rowlist;  // [T1][cap] global key rows of each query row
    const int32_t* nrows;    // [T1]
    const int32_t* order;    // [T1] work order
    const float* smax;       // [T1][N1]
    const float* ssum;
    const float* rowsum;     // [T1][N1]
    void* dkv_acc;           // [T2][1088] fp32 or int64
    float* dq_scratch;       // [gridDim.x][N1][576] fp32 per-CTA partial dQ~ of the current row
    void* dq_out;            // dQuery [T1][N1][512]
    void* dqr_out;           // dQueryRope [T1][N1][64]
    int* err;                // device error word
    const float* dmax;       // deterministic mode: max|dOut| that sets the fixed-point grid
    int64_t T1;
    int64_t nwork;           // entries of `order` (query rows processed by this launch)
    const int32_t* nwork_dev;  // when set: the entry count, read on the device
    int64_t cap;
    float scale;
    int det;
    uint64_t wait_ns;        // limit of every mbarrier wait (error word + clean exit past it)
};

// Schedule of a tile's loads and MMAs (kind 0 key chunk, 1 q chunk, 2 dO chunk; chunk c):
//   S / dP items j = 0..13: K0 Q0 O0 K1 Q1 O1 K2 Q2 O2 K3 Q3 O3 K4 Q4;
//   gradient blocks k = 0..13: dQ~ 0..4 (A = key chunk k), dK~ 0..4 (A = q chunk), dV 0..3
//   (A = dO chunk), each loading its own chunk; the output kind equals the chunk's kind.
// Software pipeline: after gradient block k >= kInterleave of tile i come the S / dP items
// 2(k - kInterleave) and 2(k - kInterleave) + 1 of tile i + 1, so the next tile's S^T / dP^T
// loads and MMAs run while this tile's reduction flush (the SM's reduction path is the bound
// of the gradient phase) continues; the first tile's S / dP items come first.
constexpr int kInterleave = 7;
__device__ __forceinline__ void sdp_item(int j, int& kind, int& c) {
    c = j / 3;
    kind = j - 3 * c;
}
__device__ __forceinline__ void block_of(int k, int& kind, int& b) {
    if (k < 5) { kind = 0; b = k; return; }
    if (k < 10) { kind = 1; b = k - 5; return; }
    kind = 2;
    b = k - 10;
}

// Named barrier 1 over the 128 softmax threads that also ANDs a flag across them:
// a thread that gave up waiting takes the others with it, so none of them is
// left at a later barrier of this group.
__device__ __forceinline__ bool softmax_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Reductions of one 32-column chunk of a staged gradient block held by this
// thread (its TMEM lane = output dim `dim`).  kind 0: dQ~ (column = head);
// kind 1 / 2: dK~ / dV (column = key, padding keys of the last tile skipped).
enum { DQ_SINGLE = 0, DQ_FIRST = 1, DQ_MID = 2, DQ_LAST = 3 };

__device__ __forceinline__ void st_relaxed(float* a, float v) {
    asm volatile("st.relaxed.gpu.global.f32 [%0], %1;" ::"l"(a), "f"(v) : "memory");
}
__device__ __forceinline__ float ld_relaxed(const float* a) {
    float v;
    asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(a) : "memory");
    return v;
}

// dQ~ of one query row accumulates across its key tiles in this CTA's scratch:
// the first tile stores, middle tiles reduce, the last tile reads back, adds and
// writes the 16-bit dQuery / dQueryRope; a single-tile row is written directly.
// Every element is handled by the same thread in tile order.
template <typename T, int N1>
__device__ __forceinline__ void flush_dq(const float (&v)[32], int mode, int cc, int t, int dim, const FusedParams& prm) {
    float* sc = prm.dq_scratch + ((size_t)blockIdx.x * N1 + cc * 32) * kDK + dim;
    if (mode == DQ_FIRST) {
#pragma unroll
        for (int e = 0; e < 32; ++e) st_relaxed(sc + e * kDK, v[e]);
        return;
    }
    if (mode == DQ_MID) {
#pragma unroll
        for (int e = 0; e < 32; ++e) atomicAdd(sc + e * kDK, v[e]);
        return;
    }
    float x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = v[e];
    if (mode == DQ_LAST) {
#pragma unroll
        for (int h = 0; h < 32; h += 16) {
            float y[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = ld_relaxed(sc + (h + e) * kDK);
#pragma unroll
            for (int e = 0; e < 16; ++e) x[h + e] += y[e];
        }
    }
    const int64_t row0 = (int64_t)t * N1 + cc * 32;
    if (dim < kD) {
        T* o = reinterpret_cast<T*>(prm.dq_out) + row0 * kD + dim;
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e * kD] = from_f<T>(x[e]);
    } else {
        T* o = reinterpret_cast<T*>(prm.dqr_out) + row0 * kDr + (dim - kD);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e * kDr] = from_f<T>(x[e]);
    }
}

template <bool DET, int N1>
__device__ __forceinline__ void flush_chunk(const float (&v)[32], int kind, int cc, int t, int dim, const int32_t* rid,
                                            int nvalid, const FusedParams& prm, float fmul) {
    const size_t col = kind == 2 ? kDK + dim : dim;
    const int32_t* r = rid + cc * 32;
    const int lim = nvalid - cc * 32;
    float* d32 = reinterpret_cast<float*>(prm.dkv_acc) + col;
    unsigned long long* d64 = reinterpret_cast<unsigned long long*>(prm.dkv_acc) + col;
    if (lim >= 32) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const size_t off = (size_t)(uint32_t)r[e] * kAccW;
            if (DET) atomicAdd(d64 + off, fix_round(v[e], fmul));
            else atomicAdd(d32 + off, v[e]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            if (e < lim) {
                const size_t off = (size_t)(uint32_t)r[e] * kAccW;
                if (DET) atomicAdd(d64 + off, fix_round(v[e], fmul));
                else atomicAdd(d32 + off, v[e]);
            }
        }
    }
}

template <typename T, int N1, bool DET>
__global__ void __launch_bounds__(kThreads, 1) sfa_bwd_fused_kernel(const __grid_constant__ FusedParams prm) {
    using C = Cfg<N1>;
    constexpr bool kF16 = std::is_same<T, __half>::value;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {  // the SW128 layouts need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicCAS(prm.err, 0, 7);
        return;
    }
    int32_t* rowids = reinterpret_cast<int32_t*>(smem + C::kOffRows);
    float* cst = reinterpret_cast<float*>(smem + C::kOffConst);
    const uint32_t bar0 = sbase + C::kOffBar;
    auto FULL = [&](int s) { return bar0 + 8u * s; };
    auto EMPTY = [&](int s) { return bar0 + 8u * (C::kSlots + s); };
    const uint32_t SDP_FULL = bar0 + 8u * (2 * C::kSlots + 0);
    const uint32_t PDS_FULL = bar0 + 8u * (2 * C::kSlots + 1);
    const uint32_t PDS_FREE = bar0 + 8u * (2 * C::kSlots + 2);
    auto STG_FULL = [&](int s) { return bar0 + 8u * (2 * C::kSlots + 3 + s); };
    auto STG_EMPTY = [&](int s) { return bar0 + 8u * (2 * C::kSlots + 5 + s); };
    auto ROWS_FULL = [&](int s) { return bar0 + 8u * (2 * C::kSlots + 7 + s); };
    auto ROWS_EMPTY = [&](int s) { return bar0 + 8u * (2 * C::kSlots + 9 + s); };
    const uint32_t DONE = bar0 + 8u * (2 * C::kSlots + 11);
    // resident key tile (N1 = 64): chunk c loaded / free for the next tile's load
    auto KFULL = [&](int c) { return bar0 + 8u * (2 * C::kSlots + 12 + c); };
    auto KEMPTY = [&](int c) { return bar0 + 8u * (2 * C::kSlots + 17 + c); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    // bounded mbarrier wait: past prm.wait_ns it records `code` in the error word and every role exits
    auto WAIT = [&](uint32_t bar, uint32_t parity, int code) {
        return wait_bar(bar, parity, abort_flag, prm.err, code, prm.wait_ns);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(FULL(s), 1);
            mbar_init(EMPTY(s), 1);
        }
        mbar_init(SDP_FULL, 1);
        mbar_init(PDS_FULL, 128);
        mbar_init(PDS_FREE, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(STG_FULL(s), 1);
            mbar_init(STG_EMPTY(s), 256);
            mbar_init(ROWS_FULL(s), 1);
            mbar_init(ROWS_EMPTY(s), 256);
        }
        mbar_init(DONE, 1);
        if (C::kResident)
            for (int c = 0; c < 5; ++c) {
                mbar_init(KFULL(c), 1);
                mbar_init(KEMPTY(c), 1);
            }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {  // whole TMEM: S^T [0,128), dP^T [128,256), staging [256,384) and [384,512)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t T_S = tmem, T_DP = tmem + 128;
    auto T_STG = [&](int s) { return tmem + 256u + 128u * s; };

    const int nwork = prm.nwork_dev ? *prm.nwork_dev : (int)prm.nwork;
    const float scale = prm.scale;

    if (warp == 12) {
        // =================== TMA producer ===================
        int slot = 0;
        uint32_t sphase = 0;
        int tile_ctr = 0;  // tiles whose row ids have been staged
        bool ok = true;
        uint32_t issued_mask = 0;  // slots that have received loads
        uint32_t kbits = 0;        // resident key chunks: parity of their loads so far
        // the CTA's tiles in order: row w (stepping by gridDim.x, rows without keys skipped), tile
        struct Tile {
            int t, n, tile, first, run0;
            bool contig;
            int32_t my[4];
            const int32_t* rl;
        };
        int w_next = blockIdx.x, tile_next = 0;
        // advances to the next tile of the CTA and stages its key row ids (for the flush warps);
        // returns false at the end of the work
        auto next_tile = [&](Tile& x) -> bool {
            while (w_next < nwork) {
                const int t = prm.order[w_next];
                const int n = prm.nrows[t];
                if (tile_next * kKeys >= n) {  // row done (or without keys): next row
                    w_next += gridDim.x;
                    tile_next = 0;
                    continue;
                }
                x.t = t;
                x.n = n;
                x.tile = tile_next++;
                x.rl = prm.rowlist + (int64_t)t * prm.cap;
                const int rb = tile_ctr & 1;
                if (lane == 0) ok = WAIT(ROWS_EMPTY(rb), ((tile_ctr >> 1) & 1) ^ 1, 1);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) return false;
                int32_t* rid = rowids + rb * kKeys;
                x.first = x.rl[0];
                x.run0 = x.rl[x.tile * kKeys];
                // lane L owns key rows 4L..4L+3 of the tile (one gather4 per 64-dim half); a tile
                // whose rows are run0, run0+1, ... is loaded as one 128-row 2-D tile instead (its
                // slots past the row's end then hold rows run0+s, masked like any padding key)
                bool contig = true;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s = x.tile * kKeys + 4 * lane + e;
                    x.my[e] = s < n ? x.rl[s] : x.first;
                    if (s < n && x.my[e] != x.run0 + 4 * lane + e) contig = false;
                    rid[4 * lane + e] = x.my[e];
                }
                x.contig = __all_sync(0xffffffffu, contig);
                __syncwarp();
                if (lane == 0) mbar_arrive(ROWS_FULL(rb));
                ++tile_ctr;
                return true;
            }
            return false;
        };
        // one chunk of tile x into the next ring slot
        auto load = [&](const Tile& x, int kind, int c) -> bool {
            const bool resident = C::kResident && kind == 0;  // into the key tile's chunk c
            if (lane == 0)
                ok = resident ? WAIT(KEMPTY(c), ((kbits >> c) & 1u) ^ 1u, 12) : WAIT(EMPTY(slot), sphase ^ 1, 2);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) return false;
            const uint32_t dst = resident ? sbase + c * kSlotBytes : sbase + C::kOffRing + slot * C::kRingSlot;
            const uint32_t bar = resident ? KFULL(c) : FULL(slot);
            const int halves = c < 4 ? 2 : 1;
            if (lane == 0) {
                const uint32_t rows = kind == 0 ? kKeys : N1;
                mbar_expect_tx(bar, halves * rows * 128u);
            }
            __syncwarp();
            if (kind == 0 && x.contig) {
                if (lane == 0) {
                    const CUtensorMap* map = c < 4 ? &prm.mapK128 : &prm.mapKr128;
                    for (int h = 0; h < halves; ++h)
                        tma_load_2d(dst + h * kHalf, map, c < 4 ? c * 128 + h * 64 : 0, x.run0, bar);
                }
            } else if (kind == 0) {
                // key rows: every lane gathers its own four rows, in parallel
                const CUtensorMap* map = c < 4 ? &prm.mapK : &prm.mapKr;
                for (int h = 0; h < halves; ++h)
                    tma_gather4(dst + h * kHalf + lane * 512, map, c < 4 ? c * 128 + h * 64 : 0, x.my[0], x.my[1],
                                x.my[2], x.my[3], bar);
            } else if (lane == 0) {
                const CUtensorMap* map = kind == 1 ? (c < 4 ? &prm.mapQ : &prm.mapQr) : &prm.mapO;
                for (int h = 0; h < halves; ++h)
                    tma_load_2d(dst + h * C::kQHalf, map, c < 4 ? c * 128 + h * 64 : 0, x.t * N1, bar);
            }
            if (resident) {
                kbits ^= 1u << c;
                if (lane == 0) issued_mask |= 1u << (16 + c);
            } else {
                if (lane == 0) issued_mask |= 1u << slot;
                if (++slot == C::kSlots) { slot = 0; sphase ^= 1; }
            }
            return true;
        };
        Tile cur, nxt;
        bool have = next_tile(cur);
        for (int j = 0; j < 14 && have && ok; ++j) {  // the first tile's S / dP items
            int kind, c;
            sdp_item(j, kind, c);
            ok = load(cur, kind, c);
        }
        while (have && ok) {
            bool have_next = false;
            for (int k = 0; k < 14 && ok; ++k) {
                int kind, b;
                block_of(k, kind, b);
                if (!(C::kResident && kind == 0)) ok = load(cur, kind, b);  // dQ~ blocks read the key tile
                if (ok && k == kInterleave) have_next = next_tile(nxt);
                if (ok && have_next && k >= kInterleave) {
                    for (int q = 0; q < 2 && ok; ++q) {
                        int kd, c;
                        sdp_item(2 * (k - kInterleave) + q, kd, c);
                        ok = load(nxt, kd, c);
                    }
                }
            }
            cur = nxt;
            have = have_next;
        }
        // drain: every issued load must land before the CTA can exit
        if (lane == 0) {
            for (int k = 0; k < C::kSlots; ++k) {
                // the most recent use of each slot is the one still possibly in flight
                const int s = (slot + k) % C::kSlots;
                const uint32_t ph = s < slot ? sphase : sphase ^ 1;
                if (issued_mask & (1u << s)) {
                    uint64_t t0 = globaltimer();
                    while (!mbar_try(FULL(s), ph) && globaltimer() - t0 < 1000000000ull) {
                    }
                }
            }
            for (int c = 0; c < 5; ++c)  // resident key chunks: their last load
                if (issued_mask & (1u << (16 + c))) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try(KFULL(c), ((kbits >> c) & 1u) ^ 1u) && globaltimer() - t0 < 1000000000ull) {
                    }
                }
        }
    } else if (warp == 13) {
        // =================== MMA issuer ===================
        const uint32_t ID_S = idesc(128, N1, false, false, kF16);      // S^T, dP^T
        const uint32_t ID_G = idesc(128, 128, true, false, kF16);      // dV^T, dK~^T (N = keys)
        const uint32_t ID_Q = idesc(128, N1, true, true, kF16);        // dQ~^T (N = heads)
        const uint32_t sP = sbase + C::kOffP, sDS = sbase + C::kOffDS;
        int slot = 0;
        uint32_t sphase = 0;
        int tile_ctr = 0;
        int blk_ctr = 0;
        bool ok = true;
        uint32_t slotK = 0;  // key chunk of the S / dP item pair in progress
        int sdp_tiles = 0;   // tiles whose S / dP items were issued (resident key tile: load parity)
        auto ring_addr = [&](int s) { return sbase + C::kOffRing + (uint32_t)s * C::kRingSlot; };
        auto wait_full = [&](int code) -> bool {
            bool r = true;
            if (lane == 0) r = WAIT(FULL(slot), sphase, code);
            r = __shfl_sync(0xffffffffu, r, 0);
            if (r) tc_fence_after();
            return r;
        };
        // S / dP item j of a tile (S^T, dP^T accumulate into their TMEM columns)
        auto sdp = [&](int j) -> bool {
            int kind, c;
            sdp_item(j, kind, c);
            if (C::kResident && kind == 0) {  // the key chunk lands in the resident key tile
                bool r = true;
                if (lane == 0) r = WAIT(KFULL(c), (uint32_t)sdp_tiles & 1u, 13);
                r = __shfl_sync(0xffffffffu, r, 0);
                if (!r) return false;
                tc_fence_after();
                slotK = sbase + (uint32_t)c * kSlotBytes;
                return true;
            }
            if (!wait_full(3)) return false;
            const uint32_t sa = ring_addr(slot);
            if (kind == 0) slotK = sa;
            if (lane == 0 && kind != 0) {
                const uint32_t dst = kind == 1 ? T_S : T_DP;
                const int ksteps = c < 4 ? 8 : 4;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint32_t offk = (ks >> 2) * kHalf + (ks & 3) * 32;      // key chunk halves
                    const uint32_t offq = (ks >> 2) * C::kQHalf + (ks & 3) * 32;  // q / dO chunk halves
                    mma(dst, sdesc(slotK + offk, 16, 1024), sdesc(sa + offq, 16, 1024), ID_S,
                        (c > 0 || ks > 0) ? 1u : 0u);
                }
                // a slot is released once the MMAs that read it have completed; a resident key
                // chunk stays for the dQ~ block that reads it again
                mma_commit(EMPTY(slot));
                if (!C::kResident && (kind == 2 || c == 4))
                    mma_commit(EMPTY((slotK - sbase - C::kOffRing) / C::kRingSlot));
                if (j == 13) mma_commit(SDP_FULL);
            }
            __syncwarp();
            if (j == 13) ++sdp_tiles;
            if (++slot == C::kSlots) { slot = 0; sphase ^= 1; }
            return true;
        };
        // the CTA's tile count per row, in the producer's order
        int w_next = blockIdx.x, tile_next = 0;
        auto next_tile = [&]() -> bool {
            while (w_next < nwork) {
                const int n = prm.nrows[prm.order[w_next]];
                if (tile_next * kKeys >= n) {
                    w_next += gridDim.x;
                    tile_next = 0;
                    continue;
                }
                ++tile_next;
                return true;
            }
            return false;
        };
        bool have = next_tile();
        for (int j = 0; j < 14 && have && ok; ++j) ok = sdp(j);  // the first tile's S / dP
        while (have && ok) {
            // ---- gradient blocks of this tile, the next tile's S / dP interleaved ----
            if (lane == 0) ok = WAIT(PDS_FULL, tile_ctr & 1, 4);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            bool have_next = false;
            for (int k = 0; k < 14 && ok; ++k, ++blk_ctr) {
                const int stg = blk_ctr & 1;
                int kind, b;
                block_of(k, kind, b);
                const bool resident = C::kResident && kind == 0;  // A = the resident key chunk b
                if (lane == 0) ok = WAIT(STG_EMPTY(stg), ((blk_ctr >> 1) & 1) ^ 1, 5);
                if (lane == 0 && ok && !resident) ok = WAIT(FULL(slot), sphase, 6);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sa = resident ? sbase + (uint32_t)b * kSlotBytes : ring_addr(slot);
                if (lane == 0) {
                    const uint32_t dst = T_STG(stg);
                    if (kind != 0) {
                        // dV^T (A = dO chunk) or dK~^T (A = q chunk): [128 dims x 128 keys], K = heads
                        const uint32_t bsrc = kind == 2 ? sP : sDS;
                        for (int ks = 0; ks < N1 / 16; ++ks) {
                            const uint64_t a = sdesc(sa + ks * 2048, C::kQHalf, 1024);
                            const uint64_t bd = sdesc(bsrc + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
                            mma(dst, a, bd, ID_G, ks > 0 ? 1u : 0u);
                        }
                    } else {
                        // dQ~^T: A = key chunk [128 dims x 128 keys] (MN), B = dS [heads x keys] (MN)
                        for (int ks = 0; ks < kKeys / 16; ++ks) {
                            const uint64_t a = sdesc(sa + ks * 2048, kHalf, 1024);
                            const uint64_t bd = sdesc(sDS + ks * 2048, kHalf, 1024);
                            mma(dst, a, bd, ID_Q, ks > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(resident ? KEMPTY(b) : EMPTY(slot));  // the key chunk's last read
                    mma_commit(STG_FULL(stg));
                    if (k == 13) mma_commit(PDS_FREE);
                }
                __syncwarp();
                if (!resident && ++slot == C::kSlots) { slot = 0; sphase ^= 1; }
                // the next tile's S^T / dP^T overwrite this tile's: the softmax warps have read
                // them (PDS_FULL above), and P / dS stay in shared memory until PDS_FREE
                if (k == kInterleave) have_next = next_tile();
                if (have_next && k >= kInterleave)
                    for (int q = 0; q < 2 && ok; ++q) ok = sdp(2 * (k - kInterleave) + q);
            }
            ++tile_ctr;
            have = have_next;
        }
        if (lane == 0) {
            mma_commit(DONE);
            uint64_t t0 = globaltimer();
            while (!mbar_try(DONE, 0) && globaltimer() - t0 < 1000000000ull) {
            }
        }
    } else if (warp < 4) {
        // =================== softmax / dS (TMEM lane = key) ===================
        const int j = threadIdx.x;  // key slot within the tile
        const float c1 = scale * 1.4426950408889634f;
        uint8_t* sPp = smem + C::kOffP;
        uint8_t* sDSp = smem + C::kOffDS;
        int tile_ctr = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nrows[t];
            if (n <= 0) continue;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (j < N1) {
                const float m = prm.smax[(int64_t)t * N1 + j];
                const float l = prm.ssum[(int64_t)t * N1 + j];
                cst[j] = m * 1.4426950408889634f;
                cst[128 + j] = l == 0.f ? 0.f : 1.f / l;
                cst[256 + j] = prm.rowsum[(int64_t)t * N1 + j];
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            const int ntiles = (n + kKeys - 1) / kKeys;
            for (int tile = 0; tile < ntiles && ok; ++tile, ++tile_ctr) {
                // padding keys of the last tile get P = dS = 0 (selected, not multiplied: a padding
                // slot of a 2-D tile holds an arbitrary row whose score may exceed the row max)
                const bool kv = tile * kKeys + j < n;
                ok = WAIT(SDP_FULL, tile_ctr & 1, 8);
                if (ok && tile_ctr > 0) ok = WAIT(PDS_FREE, (tile_ctr - 1) & 1, 9);
                ok = softmax_all(ok);
                if (!ok) break;
                tc_fence_after();
                const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
                for (int cc = 0; cc < N1 / 32; ++cc) {
                    float s[32], dp[32];
                    tmem_ld32(T_S + lane_base + cc * 32, s);
                    tmem_ld32(T_DP + lane_base + cc * 32, dp);
                    tmem_wait_ld();
                    uint32_t pw[16], dw[16];
                    const float4* cm = reinterpret_cast<const float4*>(cst + cc * 32);        // max * log2e
                    const float4* cl = reinterpret_cast<const float4*>(cst + 128 + cc * 32);  // 1 / sum
                    const float4* cd = reinterpret_cast<const float4*>(cst + 256 + cc * 32);  // rowsum(dO o O)
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const float4 m4 = cm[g], l4 = cl[g], d4 = cd[g];
                        const float mm[4] = {m4.x, m4.y, m4.z, m4.w}, ll[4] = {l4.x, l4.y, l4.z, l4.w},
                                    dd[4] = {d4.x, d4.y, d4.z, d4.w};
                        float pv[4], dv[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int e = 4 * g + k;
                            pv[k] = kv ? ex2_approx(fmaf(s[e], c1, -mm[k])) * ll[k] : 0.f;
                            dv[k] = pv[k] * (dp[e] - dd[k]) * scale;
                        }
                        pw[2 * g] = pack2<T>(pv[0], pv[1]);
                        pw[2 * g + 1] = pack2<T>(pv[2], pv[3]);
                        dw[2 * g] = pack2<T>(dv[0], dv[1]);
                        dw[2 * g + 1] = pack2<T>(dv[2], dv[3]);
                    }
                    const int half = cc >> 1;
                    const int u0 = (cc & 1) * 4;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t off = half * kHalf + j * 128 + (((u0 + u) ^ (j & 7)) << 4);
                        *reinterpret_cast<uint4*>(sPp + off) =
                            make_uint4(pw[4 * u], pw[4 * u + 1], pw[4 * u + 2], pw[4 * u + 3]);
                        *reinterpret_cast<uint4*>(sDSp + off) =
                            make_uint4(dw[4 * u], dw[4 * u + 1], dw[4 * u + 2], dw[4 * u + 3]);
                    }
                }
                fence_view_async_shared();
                tc_fence_before();
                mbar_arrive(PDS_FULL);
            }
        }
    } else {
        // =================== flush (TMEM lane = output dim) ===================
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int hsel = (warp - 4) >> 2;       // which half of each block's columns
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int tile_ctr = 0;
        int blk_ctr = 0;
        bool ok = true;
        const int ep = threadIdx.x - 128;  // 0..255 across the flush warps
        float fmul_k = 0.f, fmul_v = 0.f;  // fixed-point grids of dK~ and dV (deterministic mode)
        if (DET) {
            const FixExp fe = fix_exponents(*prm.dmax, prm.scale, prm.T1, N1);
            fmul_k = fix_mul(fe.k);
            fmul_v = fix_mul(fe.v);
        }
        for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
            const int t = prm.order[w];
            const int n = prm.nrows[t];
            if (n <= 0) {
                // no key for this query row (or a BSND padding row): dQuery = 0
                uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<T*>(prm.dq_out) + (int64_t)t * N1 * kD);
                uint4* orp = reinterpret_cast<uint4*>(reinterpret_cast<T*>(prm.dqr_out) + (int64_t)t * N1 * kDr);
                for (int i = ep; i < N1 * kD / 8; i += 256) o[i] = make_uint4(0, 0, 0, 0);
                for (int i = ep; i < N1 * kDr / 8; i += 256) orp[i] = make_uint4(0, 0, 0, 0);
                continue;
            }
            const int ntiles = (n + kKeys - 1) / kKeys;
            for (int tile = 0; tile < ntiles && ok; ++tile, ++tile_ctr) {
                const int dqmode = ntiles == 1 ? DQ_SINGLE
                                   : (tile == 0 ? DQ_FIRST : (tile == ntiles - 1 ? DQ_LAST : DQ_MID));
                const int rb = tile_ctr & 1;
                ok = __all_sync(0xffffffffu, WAIT(ROWS_FULL(rb), (tile_ctr >> 1) & 1, 10));
                if (!ok) break;
                const int32_t* rid = rowids + rb * kKeys;
                const int nvalid = min(kKeys, n - tile * kKeys);
                for (int bi = 0; bi < 14 && ok; ++bi, ++blk_ctr) {
                    const int stg = blk_ctr & 1;
                    ok = __all_sync(0xffffffffu, WAIT(STG_FULL(stg), (blk_ctr >> 1) & 1, 11));
                    if (!ok) break;
                    tc_fence_after();
                    // which output block and which dims this lane quarter holds
                    int kind, b;
                    block_of(bi, kind, b);
                    const bool active = b < 4 || q < 2;  // rope blocks: 64 valid dims
                    const int dim = (b < 4 ? b * 128 : kD) + q * 32 + lane;
                    if (active) {
                        const int nch = (kind == 0 ? N1 : kKeys) / 32;
                        const int c0 = hsel * (nch >> 1);
                        const int c1 = c0 + (nch >> 1);
                        for (int cc = c0; cc < c1; ++cc) {
                            float v[32];
                            tmem_ld32(T_STG(stg) + lane_base + cc * 32, v);
                            tmem_wait_ld();
                            if (kind == 0) flush_dq<T, N1>(v, dqmode, cc, t, dim, prm);
                            else flush_chunk<DET, N1>(v, kind, cc, t, dim, rid, nvalid, prm, kind == 2 ? fmul_v : fmul_k);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(STG_EMPTY(stg));
                }
                if (ok) mbar_arrive(ROWS_EMPTY(rb));
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

// ---------------------------------------------------------------------------
// Host side: launch
// ---------------------------------------------------------------------------
template <typename T, int N1, bool DET>
cudaError_t launch_t(const GradArgs& a, cudaStream_t st) {
    FusedParams p;
    memset(&p, 0, sizeof p);
    const int64_t T1 = a.sd.T1, T2 = a.sd.T2;
    if (!make_map(&p.mapQ, a.q, a.dtype, kD, (uint64_t)T1 * N1, kD, N1) ||
        !make_map(&p.mapQr, a.qr, a.dtype, kDr, (uint64_t)T1 * N1, kDr, N1) ||
        !make_map(&p.mapO, a.dout, a.dtype, kD, (uint64_t)T1 * N1, kD, N1) ||
        !make_map(&p.mapK, a.k, a.dtype, kD, (uint64_t)T2, kD, 1) ||
        !make_map(&p.mapKr, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, 1) ||
        !make_map(&p.mapK128, a.k, a.dtype, kD, (uint64_t)T2, kD, kKeys) ||
        !make_map(&p.mapKr128, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, kKeys))
        return cudaErrorInvalidValue;
    p.rowlist = a.rowlist;
    p.nrows = a.nrows;
    p.order = a.order;
    p.smax = a.smax;
    p.ssum = a.ssum;
    p.rowsum = a.rowsum;
    p.dkv_acc = a.dkv_acc;
    p.dq_scratch = a.dq_acc;
    p.dq_out = a.dq;
    p.dqr_out = a.dqr;
    p.err = a.ctrl;
    p.dmax = a.dout_absmax;
    p.T1 = T1;
    p.nwork = a.row_end - a.row_begin;
    p.nwork_dev = a.nwork_dev;
    p.cap = a.rowcap;
    p.scale = a.scale;
    p.det = DET ? 1 : 0;
    p.wait_ns = wait_limit_ns();

    auto kern = sfa_bwd_fused_kernel<T, N1, DET>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<N1>::kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int grid = (int)(p.nwork < sms ? p.nwork : sms);  // (an upper bound when the count is on the device)
    if (grid > kMaxFusedGrid) grid = kMaxFusedGrid;
    if (grid < 1) return cudaSuccess;
    kern<<<grid, kThreads, Cfg<N1>::kSmem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool fused_supported(int64_t N1) { return N1 == 64 || N1 == 128; }

template <typename T>
cudaError_t launch_n1(const GradArgs& a, cudaStream_t st) {
    if (a.N1 == 128) return a.det ? launch_t<T, 128, true>(a, st) : launch_t<T, 128, false>(a, st);
    return a.det ? launch_t<T, 64, true>(a, st) : launch_t<T, 64, false>(a, st);
}

cudaError_t launch_bwd_fused(int dtype, const GradArgs& a, cudaStream_t st) {
    return dtype == SFA_DTYPE_BF16 ? launch_n1<__nv_bfloat16>(a, st) : launch_n1<__half>(a, st);
}

}  // namespace sfa
