// Paired-row tensor-core sparse attention backward for sm_100a: two query rows
// whose selected key blocks are identical are processed by the two CTAs of a
// thread-block cluster, which exchange P / dS through distributed shared memory
// so that each key tile's dK~ / dV sums over both rows before they are reduced
// into the accumulator.
//
// What it computes (SparseFlashAttentionGrad README, 功能说明, stages 1-3) is the
// same as the single-row fused kernel: per query row t with its gathered key
// rows j (value == key, first 512 dims), S^T = K~.Q~^T, dP^T = V.dO^T, P from the
// given statistics, dS = P o (dP - rowsum(dO o O)), dV += P^T.dO, dK~ += dS^T.Q~
// (both scattered to the key rows), dQ~ = dS.K~.  A key's dK~ / dV are sums over
// every (row, head) that selected it; adjacent rows of block-sparse attention
// usually select the same blocks (under the causal mask every row of a 16-row
// block sees the same causal blocks), so a pair of such rows shares every key
// tile and their contributions can be added on chip first.
//
// Layout decisions (B200):
//  * Cluster of two CTAs (one per SM), rank r owns row t0 + r of the pair.  Both
//    load the same key tiles (TMA 2-D tiles for runs of consecutive rows, else
//    tile::gather4) and form S^T / dP^T of their own row (M = 128 keys, N = 128
//    heads, TMEM lane = key), and P / dS of their own row (bf16, shared memory,
//    per-row masks: each row keeps its own causal cut of the shared blocks).
//  * The gradient work of the pair is split by output, not by row: rank 0 owns
//    dV (4 blocks of 128 dims), rank 1 owns dK~ (4 blocks + the 64 rope dims);
//    each block contracts over both rows' heads (K = 256) in one TMEM
//    accumulator, so the reduction of a key tile into dKey / dValue carries both
//    rows: half the reduction bytes per (row, key) pair of the single-row kernel.
//    For that, rank 0 sends its dS (32 KB per tile) with a bulk copy shared::cta
//    -> shared::cluster that completes on rank 1's mbarrier, and rank 1 stores its
//    P straight into rank 0's receive buffer (distributed shared memory stores,
//    a proxy fence, one remote arrive): rank 1 keeps no P of its own, and that
//    buffer is a fifth operand slot.  Each rank also loads the partner row's dO
//    (rank 0) or q (rank 1) chunks.
//    dQ~ is formed per row, dQ~^T = K~^T.dS^T, and accumulated across the row's
//    tiles in a per-CTA fp32 scratch: rank 0 its row's dims 0-383 and the rope,
//    rank 1 its whole row and rank 0's dims 384-511 (from the dS it receives).
//  * Shared memory: 32 KB operand slots (4 on rank 0, 5 on rank 1) split into the
//    two rings, P (X, rank 0 only), dS (Y) and the received tile (R), 32 KB each,
//    row ids and masks, constants, barriers: the same offsets in both CTAs, so an
//    offset names the same object in the peer.
//  * Hand-over of the single received buffer R: a rank grants its partner the
//    next tile's copy (remote arrive on the partner's PEER_FREE) once its own
//    gradient MMAs of the previous tile completed (they read R); the sender
//    overwrites its copy source only after that grant, which also proves the
//    previous copy was consumed.  Rank 1 arms its RECV barrier with the expected
//    bytes when it grants; rank 0's RECV completes on the partner's arrive; each
//    MMA warp waits on RECV before the first MMA that reads R.
//  * Warp roles per CTA: 0-3 softmax/dS, 4-11 flush, 12 / 14 TMA producers and
//    13 / 15 MMA issuers of the gradient blocks / the S^T and dP^T items, each
//    pair with its own ring, so the next tile's S^T / dP^T are formed while this
//    tile's gradient blocks run.  Every wait is bounded; on timeout the CTA
//    records an error word and leaves, after waiting (bounded) for copies still
//    addressed to it and meeting its partner at the final cluster barrier.
#include <cuda.h>

#include <cstring>
#include <type_traits>

#include "sfa_internal.cuh"
#include "tc_common.cuh"

namespace sfa {

namespace {

using namespace tc;

constexpr int kThreads = 512;       // 4 softmax + 8 flush + 2 TMA + 2 MMA warps
constexpr int kSlots = 4;           // operand slots of rank 0
constexpr int kSlotsMax = 5;        // rank 1: its P goes straight to the partner, X is a fifth slot
constexpr int kSRing0 = 3, kSRing1 = 3;  // S / dP ring slots of rank 0 / 1 (the rest carry the gradient blocks)
constexpr int kSlotBytes = 32768;
constexpr int kHalf = 16384;
constexpr int kKeys = 128;          // key rows per tile (MMA M)
constexpr int kN1 = 128;            // query heads (MMA N of S^T / dP^T, K of the gradient blocks per row)
constexpr uint32_t kTileBytes = 32768;  // P or dS of one row and one tile, bf16 [128 keys x 128 heads]

constexpr int kOffX = kSlots * kSlotBytes;        // P of the own row (rank 0); rank 1: ring slot 4
constexpr int kOffY = kOffX + 32768;              // dS of the own row
constexpr int kOffR = kOffY + 32768;              // the partner's P (rank 0) or dS (rank 1)
constexpr int kOffRows = kOffR + 32768;           // int32 [2][128] key row ids, bit 31: invalid for both rows
constexpr int kOffMask = kOffRows + 2 * kKeys * 4;  // uint32 [2][4] own row's valid slots
constexpr int kOffConst = kOffMask + 2 * 4 * 4;   // float [3][128] max*log2e, 1/sum, rowsum(dO o O)
constexpr int kOffBar = kOffConst + 3 * kN1 * 4;
enum {
    BAR_FULL = 0,
    BAR_EMPTY = BAR_FULL + kSlotsMax,
    BAR_SDP = BAR_EMPTY + kSlotsMax,
    BAR_PDS_FULL,
    BAR_PDS_FREE,
    BAR_STG_FULL,
    BAR_STG_EMPTY = BAR_STG_FULL + 2,
    BAR_ROWS_FULL = BAR_STG_EMPTY + 2,
    BAR_ROWS_EMPTY = BAR_ROWS_FULL + 2,
    BAR_DONE = BAR_ROWS_EMPTY + 2,
    BAR_RECV,
    BAR_PEER_FREE,
    BAR_COUNT
};
constexpr int kOffMisc = kOffBar + BAR_COUNT * 8;  // u32: TMEM base, abort flag, copies granted, copies consumed
constexpr int kSmem = kOffMisc + 16;
static_assert(kSmem <= 232448, "shared memory per CTA");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");

struct PairParams {
    CUtensorMap mapQ, mapQr, mapO, mapK, mapKr;  // dO shares mapO; key maps: 1-row boxes (gather4)
    CUtensorMap mapK128, mapKr128;                // key maps with 128-row boxes (contiguous tiles)
    const int32_t* blocks;   // [T1][topk] compacted (sorted) block indices
    const int32_t* nblk;     // [T1]
    const int32_t* pairs;    // first row of each pair (the pair is t, t + 1), longest first
    const int32_t* npairs;   // device count of `pairs`
    const float* smax;       // [T1][N1]
    const float* ssum;
    const float* rowsum;     // [T1][N1]
    void* dkv_acc;           // [T2][1088] fp32 or int64
    float* dq_scratch;       // [gridDim.x][N1][576] fp32 per-CTA partial dQ~ of the current row
    void* dq_out;            // dQuery [T1][N1][512]
    void* dqr_out;           // dQueryRope [T1][N1][64]
    int* err;                // device error word
    const float* dmax;       // deterministic mode: max|dOut| that sets the fixed-point grid
    SeqDesc sd;
    int64_t topk;
    int32_t bs, mode;
    int64_t T2;
    float scale;
    uint64_t wait_ns;
};

// Gradient blocks of a tile: k < 5 dQ~ block k of the own row (one key chunk); k >= 5 the rank's
// key-side block k - 5 (rank 0 dV, rank 1 dK~) over both rows (the own row's chunk, then the partner's).
// dQ~ block (dims 384-511) of rank 0's row that rank 1 computes: rank 1 holds that row's dS (it
// receives it for dK~) and the tile's key chunk, so the block costs it no load, and rank 0, the
// rank that waits at the exchange, gets one block less.  Rank 1 also keeps those dims' partial
// sums, in rank 0's scratch (which rank 0 leaves unused there) and writes them to dQuery.
constexpr int kDqMoved = 3;
__device__ __forceinline__ int num_blocks(uint32_t rank) { return rank ? 11 : 8; }
// Block bi of a tile in the flush order: dQ~ blocks first (rank 0: chunks 0, 1, 2, 4; rank 1:
// chunks 0-3, then rank 0's chunk 3, then chunk 4), then the key-side blocks.
__device__ __forceinline__ void block_of(uint32_t rank, int bi, bool& dq, bool& moved, int& b) {
    const int ndq = rank ? 6 : 4;
    dq = bi < ndq;
    moved = rank && bi == kDqMoved + 1;
    if (!dq) b = bi - ndq;
    else if (rank) b = bi <= kDqMoved ? bi : (bi == kDqMoved + 1 ? kDqMoved : bi - 1);
    else b = bi < kDqMoved ? bi : bi + 1;
}
// Two rings and two MMA warps per CTA.  The gradient ring (1 slot on rank 0, 2 on rank 1) carries,
// per tile, the five key chunks of the dQ~ blocks, then each key-side block's own-row and partner
// chunk, consumed in that order by the gradient MMA warp.  The S / dP ring (3 slots) carries each
// tile's S items (K_c, q_c) and dP items (the same K_c, dO_c), consumed by the S / dP MMA warp, which
// starts a tile's items once the softmax has read the previous tile's S^T / dP^T.  So the gradient
// blocks never wait for the next tile's S / dP operands, and the flush (the reductions, the
// throughput bound of the gradient phase) is fed back to back; per tile 27 (rank 0) / 29 (rank 1)
// chunks are loaded.  A ring slot holds a chunk only until the MMAs of its item or block complete,
// so neither ring can deadlock (checked by a CPU model of both CTAs).  Slot splits measured on the
// 16K-token block-sparse workload: gradient / S 1+3 and 2+3 (rank 0, rank 1) 73.8 ms, 2+2 and 2+3
// (key chunk reloaded for the dP item) 74.6-75.8 ms, one ring for both 78.3 ms.

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

__device__ __forceinline__ void st_relaxed(float* a, float v) {
    asm volatile("st.relaxed.gpu.global.f32 [%0], %1;" ::"l"(a), "f"(v) : "memory");
}
__device__ __forceinline__ float ld_relaxed(const float* a) {
    float v;
    asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(a) : "memory");
    return v;
}

// Bounded wait with acquire at cluster scope (arrivals made by the partner CTA)
__device__ __noinline__ bool wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err, int code,
                                          uint64_t limit_ns) {
    if (mbar_try_cluster(bar, parity)) return true;
    uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_cluster(bar, parity)) return true;
        if ((it & 63) == 1) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicCAS(err, 0, code);
                return false;
            }
        }
    }
}

// dQ~ of the own row across its tiles in this CTA's scratch (first tile stores, middle tiles
// reduce, the last reads back, adds and writes the 16-bit dQuery / dQueryRope; a one-tile row is
// written directly); every element is handled by the same thread in tile order.
enum { DQ_SINGLE = 0, DQ_FIRST = 1, DQ_MID = 2, DQ_LAST = 3 };
template <typename T>
__device__ __forceinline__ void flush_dq(const float (&v)[32], int mode, int cc, int t, int dim,
                                         const PairParams& prm, int cta) {
    float* sc = prm.dq_scratch + ((size_t)cta * kN1 + cc * 32) * kDK + dim;
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
    const int64_t row0 = (int64_t)t * kN1 + cc * 32;
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

// Reductions of one 32-key chunk of a staged dK~ / dV block (this thread's TMEM lane = output
// column `col` of the accumulator); keys invalid for both rows (bit 31) are skipped.
template <bool DET>
__device__ __forceinline__ void flush_keys(const float (&v)[32], size_t col, const int32_t* rid,
                                           const PairParams& prm, float fmul) {
    float* d32 = reinterpret_cast<float*>(prm.dkv_acc) + col;
    unsigned long long* d64 = reinterpret_cast<unsigned long long*>(prm.dkv_acc) + col;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int32_t r = rid[e];
        if (r >= 0) {
            const size_t off = (size_t)r * kAccW;
            if (DET) atomicAdd(d64 + off, fix_round(v[e], fmul));
            else atomicAdd(d32 + off, v[e]);
        }
    }
}

template <typename T, bool DET>
__global__ void __launch_bounds__(kThreads, 1) sfa_bwd_pair_kernel(const __grid_constant__ PairParams prm) {
    constexpr bool kF16 = std::is_same<T, __half>::value;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t rank = cluster_ctarank();   // 0 or 1: row t0 + rank of each pair
    const uint32_t peer = rank ^ 1u;
    const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
    if (sbase & 1023u) {  // the SW128 layouts need a 1024-byte aligned base (uniform over the grid)
        if (threadIdx.x == 0) atomicCAS(prm.err, 0, 7);
        return;
    }
    int32_t* rowids = reinterpret_cast<int32_t*>(smem + kOffRows);
    uint32_t* masks = reinterpret_cast<uint32_t*>(smem + kOffMask);
    float* cst = reinterpret_cast<float*>(smem + kOffConst);
    const uint32_t bar0 = sbase + kOffBar;
    auto BAR = [&](int i) { return bar0 + 8u * i; };
    auto FULL = [&](int s) { return BAR(BAR_FULL + s); };
    auto EMPTY = [&](int s) { return BAR(BAR_EMPTY + s); };
    const uint32_t SDP_FULL = BAR(BAR_SDP), PDS_FULL = BAR(BAR_PDS_FULL), PDS_FREE = BAR(BAR_PDS_FREE);
    auto STG_FULL = [&](int s) { return BAR(BAR_STG_FULL + s); };
    auto STG_EMPTY = [&](int s) { return BAR(BAR_STG_EMPTY + s); };
    auto ROWS_FULL = [&](int s) { return BAR(BAR_ROWS_FULL + s); };
    auto ROWS_EMPTY = [&](int s) { return BAR(BAR_ROWS_EMPTY + s); };
    const uint32_t DONE = BAR(BAR_DONE), RECV = BAR(BAR_RECV), PEER_FREE = BAR(BAR_PEER_FREE);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    uint32_t* tmem_slot = misc;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    volatile uint32_t* granted = misc + 2;   // copies this CTA allowed its partner to send (= RECV phases armed)
    volatile uint32_t* consumed = misc + 3;  // RECV phases this CTA's MMA warp waited for
    auto WAIT = [&](uint32_t bar, uint32_t parity, int code) {
        return wait_bar(bar, parity, abort_flag, prm.err, code, prm.wait_ns);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlotsMax; ++s) {
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
        mbar_init(DONE, 2);
        mbar_init(RECV, 1);
        mbar_init(PEER_FREE, 1);
        misc[1] = misc[2] = misc[3] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {  // whole TMEM: S^T [0,128), dP^T [128,256), staging [256,384) and [384,512)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_slot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the partner's barriers are initialized before any copy or arrive reaches them
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t T_S = tmem, T_DP = tmem + 128;
    auto T_STG = [&](int s) { return tmem + 256u + 128u * s; };

    const int npairs = *prm.npairs;
    const int bs = prm.bs;
    const float scale = prm.scale;
    const int nblocks = num_blocks(rank);  // gradient blocks per tile: the dQ~ and key-side ones
    const int nkey = rank ? 5 : 4;
    // two rings: slots [0, g_slots) carry the gradient blocks' chunks, the next two slots the S / dP
    // items' chunks (rank 1's fifth slot is its P buffer, which it never uses)
    const int s_slots = rank ? kSRing1 : kSRing0;
    const int g_slots = (rank ? kSlotsMax : kSlots) - s_slots;

    if (warp == 12 || warp == 14) {
        // =================== TMA producers: 12 the gradient ring, 14 the S / dP ring ===================
        const bool srole = warp == 14;  // also stages each tile's key row ids and masks
        const int ring0 = srole ? g_slots : 0, ring_n = srole ? s_slots : g_slots;
        int slot = 0;  // position in this producer's ring
        uint32_t sphase = 0;
        int tile_ctr = 0;
        bool ok = true;
        uint32_t issued_mask = 0;
        struct Tile {
            int t0, tile;
            bool contig;
            int32_t my[4];  // this lane's four key rows for gather4 (clamped into the key tensor)
            int32_t run0;   // row of slot 0 (the 2-D tile's first row when contiguous)
        };
        // The pair's tile count and spans are read once per pair, and the block ids of the
        // pair's next tile are fetched one tile ahead: under the reduction traffic a dependent
        // global read costs about a microsecond, and this warp's reads sit between its loads.
        int w_next = cid, tile_next = 0;
        int pw = -1, pt0 = 0, pnslots = 0;  // the pair the cached fields describe
        TokInfo ti0{}, ti1{};
        int32_t pre[4] = {0, 0, 0, 0};  // block ids of this lane's slots in tile pre_tile of pair pw
        int pre_tile = -1;
        auto fetch_blocks = [&](int tile, int32_t (&blk)[4]) {
            const int32_t* bl = prm.blocks + (int64_t)pt0 * prm.topk;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int g = tile * kKeys + 4 * lane + e;
                blk[e] = g < pnslots ? bl[g / bs] : 0;
            }
        };
        auto next_tile = [&](Tile& x) -> bool {
            while (w_next < npairs) {
                if (pw != w_next) {
                    pw = w_next;
                    pt0 = prm.pairs[w_next];
                    pnslots = prm.nblk[pt0] * bs;
                    ti0 = tok_info(prm.sd, pt0);
                    ti1 = tok_info(prm.sd, (int64_t)pt0 + 1);
                    pre_tile = -1;
                }
                const int t0 = pt0;
                const int nslots = pnslots;
                if (tile_next * kKeys >= nslots) {
                    w_next += ncl;
                    tile_next = 0;
                    continue;
                }
                x.t0 = t0;
                x.tile = tile_next++;
                int32_t blkv[4];
                if (pre_tile == x.tile) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) blkv[e] = pre[e];
                } else {
                    fetch_blocks(x.tile, blkv);
                }
                if (tile_next * kKeys < nslots) {  // the pair's next tile: its reads are issued now
                    fetch_blocks(tile_next, pre);
                    pre_tile = tile_next;
                }
                const int rb = tile_ctr & 1;
                if (srole && lane == 0) ok = WAIT(ROWS_EMPTY(rb), ((tile_ctr >> 1) & 1) ^ 1, 101);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) return false;
                // lane L owns slots 4L..4L+3 of the tile; a slot is block i = g / bs, row o = g % bs of it
                bool contig = true;
                uint32_t ownbits = 0;
                int32_t rowv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int g = x.tile * kKeys + 4 * lane + e;
                    int64_t row = -1;
                    bool own = false, any = false;
                    if (g < nslots) {
                        const int i = g / bs, o = g - i * bs;
                        const int64_t blk = blkv[e];
                        row = ti0.kv_start + blk * bs + o;
                        const int k0 = block_rows(blk, bs, ti0, prm.mode), k1 = block_rows(blk, bs, ti1, prm.mode);
                        own = o < (rank ? k1 : k0);
                        any = o < (k0 > k1 ? k0 : k1);
                    }
                    rowv[e] = (int32_t)row;
                    if (srole) rowids[rb * kKeys + 4 * lane + e] = any ? (int32_t)row : (int32_t)0x80000000;
                    if (own) ownbits |= 1u << e;
                }
                // slot 0's row, then a contiguity vote (slots past the list's end do not count)
                const int32_t run0 = __shfl_sync(0xffffffffu, rowv[0], 0);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int g = x.tile * kKeys + 4 * lane + e;
                    if (g < nslots && rowv[e] != run0 + 4 * lane + e) contig = false;
                    int32_t r = rowv[e] < 0 ? run0 : rowv[e];
                    if (r >= prm.T2) r = (int32_t)(prm.T2 - 1);
                    if (r < 0) r = 0;
                    x.my[e] = r;
                }
                x.run0 = run0;
                x.contig = __all_sync(0xffffffffu, contig);
                if (srole) {
                    // own-row validity bits: word w covers slots 32w..32w+31 (lanes 8w..8w+7)
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t part = (lane >> 3) == w ? ownbits << (4 * (lane & 7)) : 0u;
                        const uint32_t word = __reduce_or_sync(0xffffffffu, part);
                        if (lane == 0) masks[rb * 4 + w] = word;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ROWS_FULL(rb));
                }
                ++tile_ctr;
                return true;
            }
            return false;
        };
        // one chunk into the next ring slot: kind 0 key chunk c of tile x, 1 / 2 q / dO chunk c of row t
        auto load = [&](const Tile& x, int kind, int c, int t) -> bool {
            const int gs = ring0 + slot;  // the slot's index in shared memory
            if (lane == 0) ok = WAIT(EMPTY(gs), sphase ^ 1, 102);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) return false;
            const uint32_t dst = sbase + gs * kSlotBytes;
            const int halves = c < 4 ? 2 : 1;
            if (lane == 0) mbar_expect_tx(FULL(gs), halves * 128u * 128u);
            __syncwarp();
            if (kind == 0 && x.contig) {
                if (lane == 0) {
                    const CUtensorMap* map = c < 4 ? &prm.mapK128 : &prm.mapKr128;
                    for (int h = 0; h < halves; ++h)
                        tma_load_2d(dst + h * kHalf, map, c < 4 ? c * 128 + h * 64 : 0, x.run0, FULL(gs));
                }
            } else if (kind == 0) {
                const CUtensorMap* map = c < 4 ? &prm.mapK : &prm.mapKr;
                for (int h = 0; h < halves; ++h)
                    tma_gather4(dst + h * kHalf + lane * 512, map, c < 4 ? c * 128 + h * 64 : 0, x.my[0], x.my[1],
                                x.my[2], x.my[3], FULL(gs));
            } else if (lane == 0) {
                const CUtensorMap* map = kind == 1 ? (c < 4 ? &prm.mapQ : &prm.mapQr) : &prm.mapO;
                for (int h = 0; h < halves; ++h)
                    tma_load_2d(dst + h * kHalf, map, c < 4 ? c * 128 + h * 64 : 0, t * kN1, FULL(gs));
            }
            if (lane == 0) issued_mask |= 1u << gs;
            if (++slot == ring_n) { slot = 0; sphase ^= 1; }
            return true;
        };
        Tile cur;
        if (srole) {
            // every tile's S / dP items: S item c (K_c, q_c), then dP item c (c < 4: dO_c with K_c,
            // which a ring of three or more slots keeps from the S item and a smaller one reloads)
            const bool holdK = ring_n >= 3;
            while (ok && next_tile(cur)) {
                const int t = cur.t0 + (int)rank;
                for (int c = 0; c < 5 && ok; ++c) {
                    ok = load(cur, 0, c, 0);
                    if (ok) ok = load(cur, 1, c, t);
                    if (ok && c < 4 && !holdK) ok = load(cur, 0, c, 0);
                    if (ok && c < 4) ok = load(cur, 2, c, t);
                }
            }
        } else {
            // every tile's gradient blocks: the five key chunks of the dQ~ blocks, then per key-side
            // block the own row's chunk and the partner's (q for dK~, dO for dV)
            const int gkind = rank ? 1 : 2;
            while (ok && next_tile(cur)) {
                for (int c = 0; c < 5 && ok; ++c)
                    if (rank || c != kDqMoved) ok = load(cur, 0, c, 0);
                for (int c = 0; c < nkey && ok; ++c) {
                    ok = load(cur, gkind, c, cur.t0 + (int)rank);
                    if (ok) ok = load(cur, gkind, c, cur.t0 + (int)peer);
                }
            }
        }
        // drain: every issued load must land before the CTA can exit
        if (lane == 0) {
            for (int k = 0; k < ring_n; ++k) {
                const int s = (slot + k) % ring_n;
                const uint32_t ph = s < slot ? sphase : sphase ^ 1;
                if (issued_mask & (1u << (ring0 + s))) {
                    uint64_t t0 = globaltimer();
                    while (!mbar_try(FULL(ring0 + s), ph) && globaltimer() - t0 < 1000000000ull) {
                    }
                }
            }
        }
    } else if (warp == 13 || warp == 15) {
        // =================== MMA issuers: 13 the gradient blocks, 15 the S / dP items ===================
        const bool srole = warp == 15;
        const uint32_t ID_S = idesc(128, kN1, false, false, kF16);  // S^T, dP^T
        const uint32_t ID_G = idesc(128, 128, true, false, kF16);   // dV^T, dK~^T (N = keys)
        const uint32_t ID_Q = idesc(128, kN1, true, true, kF16);    // dQ~^T (N = heads)
        const uint32_t sX = sbase + kOffX, sY = sbase + kOffY, sR = sbase + kOffR;
        const uint32_t bOwn = rank ? sY : sX;  // B of the own row's half: dS (dK~) or P (dV)
        const int ring0 = srole ? g_slots : 0, ring_n = srole ? s_slots : g_slots;
        int slot = 0;
        uint32_t sphase = 0;
        int tile_ctr = 0, blk_ctr = 0;
        uint32_t recv_done = 0;
        bool ok = true;
        auto gslot = [&]() { return ring0 + slot; };  // the current chunk's slot in shared memory
        auto wait_full = [&](int code) -> bool {
            bool r = true;
            if (lane == 0) r = WAIT(FULL(gslot()), sphase, code);
            r = __shfl_sync(0xffffffffu, r, 0);
            if (r) tc_fence_after();
            return r;
        };
        auto advance = [&]() {
            if (++slot == ring_n) { slot = 0; sphase ^= 1; }
        };
        // K = 128 half of a key-side block: A = the chunk in the current slot, B = P or dS in bsrc
        auto grad_half = [&](uint32_t dst, uint32_t bsrc, bool first, int code) -> bool {
            if (!wait_full(code)) return false;
            const uint32_t sa = sbase + gslot() * kSlotBytes;
            if (lane == 0) {
                for (int ks = 0; ks < kN1 / 16; ++ks) {
                    const uint64_t a = sdesc(sa + ks * 2048, kHalf, 1024);
                    const uint64_t bd = sdesc(bsrc + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
                    mma(dst, a, bd, ID_G, (!first || ks > 0) ? 1u : 0u);
                }
                mma_commit(EMPTY(gslot()));
            }
            __syncwarp();
            advance();
            return true;
        };
        int w_next = cid, tile_next = 0;
        int pw = -1, pnslots = 0;  // key slots of pair pw (read once per pair)
        auto next_tile = [&]() -> bool {
            while (w_next < npairs) {
                if (pw != w_next) {
                    pw = w_next;
                    pnslots = prm.nblk[prm.pairs[w_next]] * bs;
                }
                if (tile_next * kKeys >= pnslots) {
                    w_next += ncl;
                    tile_next = 0;
                    continue;
                }
                ++tile_next;
                return true;
            }
            return false;
        };
        if (srole) {
            // ---- every tile's S / dP items: S item c (K_c, q_c) accumulates S^T, dP item c (K_c,
            // dO_c) dP^T; a tile's items start once the softmax has read the previous tile's ----
            while (ok && next_tile()) {
                if (tile_ctr > 0) {
                    if (lane == 0) ok = WAIT(PDS_FULL, (tile_ctr - 1) & 1, 119);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after();
                }
                const bool holdK = ring_n >= 3;  // the key chunk stays from S item c to dP item c
                auto item = [&](uint32_t dst, int sK, int sB, int c) {
                    const int ksteps = c < 4 ? 8 : 4;
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                        mma(dst, sdesc(sbase + sK * kSlotBytes + off, 16, 1024),
                            sdesc(sbase + sB * kSlotBytes + off, 16, 1024), ID_S, (c > 0 || ks > 0) ? 1u : 0u);
                    }
                };
                for (int c = 0; c < 5 && ok; ++c) {
                    if (!(ok = wait_full(103))) break;
                    const int sK = gslot();
                    advance();
                    if (!(ok = wait_full(103))) break;
                    const int sQ = gslot();
                    advance();
                    const bool keepK = holdK && c < 4;
                    if (lane == 0) {
                        item(T_S, sK, sQ, c);
                        mma_commit(EMPTY(sQ));
                        if (!keepK) mma_commit(EMPTY(sK));
                        if (c == 4) mma_commit(SDP_FULL);
                    }
                    __syncwarp();
                    if (c == 4) break;
                    int sK2 = sK;
                    if (!holdK) {
                        if (!(ok = wait_full(103))) break;
                        sK2 = gslot();
                        advance();
                    }
                    if (!(ok = wait_full(103))) break;
                    const int sO = gslot();
                    advance();
                    if (lane == 0) {
                        item(T_DP, sK2, sO, c);
                        mma_commit(EMPTY(sO));
                        mma_commit(EMPTY(sK2));
                    }
                    __syncwarp();
                }
                ++tile_ctr;
            }
        } else {
            while (ok && next_tile()) {
                if (lane == 0) ok = WAIT(PDS_FULL, tile_ctr & 1, 104);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after();
                // ---- dQ~ blocks: A = key chunk [128 dims x 128 keys] (MN), B = dS (MN) of the own row;
                // rank 1 also forms rank 0's block kDqMoved from the received dS, same key chunk ----
                auto dq_block = [&](uint32_t bsrc, bool release) -> bool {
                    const int stg = blk_ctr & 1;
                    bool r = true;
                    if (lane == 0) r = WAIT(STG_EMPTY(stg), ((blk_ctr >> 1) & 1) ^ 1, 105);
                    r = __shfl_sync(0xffffffffu, r, 0);
                    if (!r) return false;
                    tc_fence_after();
                    const uint32_t sa = sbase + gslot() * kSlotBytes;
                    if (lane == 0) {
                        for (int ks = 0; ks < kKeys / 16; ++ks)
                            mma(T_STG(stg), sdesc(sa + ks * 2048, kHalf, 1024), sdesc(bsrc + ks * 2048, kHalf, 1024),
                                ID_Q, ks > 0 ? 1u : 0u);
                        if (release) mma_commit(EMPTY(gslot()));
                        mma_commit(STG_FULL(stg));
                    }
                    __syncwarp();
                    ++blk_ctr;
                    return true;
                };
                for (int c = 0; c < 5 && ok; ++c) {
                    if (!rank && c == kDqMoved) continue;
                    if (!(ok = wait_full(106))) break;
                    const bool moved = rank && c == kDqMoved;
                    if (!(ok = dq_block(sY, !moved))) break;
                    if (moved) {  // rank 0's dS of this tile has landed in R
                        if (lane == 0)
                            ok = wait_cluster(RECV, recv_done & 1, abort_flag, prm.err, 108, prm.wait_ns);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        ++recv_done;
                        tc_fence_after();
                        if (!(ok = dq_block(sR, true))) break;
                    }
                    advance();
                }
                if (!ok) break;
                // ---- key-side block c over both rows: the own row's chunk, then the partner's ----
                for (int c = 0; c < nkey && ok; ++c) {
                    const int stg = blk_ctr & 1;
                    if (lane == 0) ok = WAIT(STG_EMPTY(stg), ((blk_ctr >> 1) & 1) ^ 1, 105);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after();
                    if (!(ok = grad_half(T_STG(stg), bOwn, true, 107))) break;
                    if (c == 0 && !rank) {  // rank 1's P of this tile has landed in R (rank 1 waited above)
                        if (lane == 0)
                            ok = wait_cluster(RECV, recv_done & 1, abort_flag, prm.err, 108, prm.wait_ns);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        ++recv_done;
                        tc_fence_after();
                        if (!rank) fence_view_async_shared();  // R was written by the partner's stores
                    }
                    if (!(ok = grad_half(T_STG(stg), sR, false, 109))) break;
                    if (lane == 0) {
                        mma_commit(STG_FULL(stg));
                        if (c == nkey - 1) mma_commit(PDS_FREE);  // the last reads of P, dS and R
                    }
                    __syncwarp();
                    ++blk_ctr;
                }
                ++tile_ctr;
            }
        }
        if (lane == 0) {
            if (!srole) *consumed = recv_done;
            mma_commit(DONE);  // both MMA warps arrive: every MMA of the CTA has completed
            uint64_t t0 = globaltimer();
            while (!mbar_try(DONE, 0) && globaltimer() - t0 < 1000000000ull) {
            }
        }
    } else if (warp < 4) {
        // =================== softmax / dS of the own row (TMEM lane = key) ===================
        const int j = threadIdx.x;
        const float c1 = scale * 1.4426950408889634f;
        uint8_t* sPp = smem + kOffX;
        uint8_t* sDSp = smem + kOffY;
        const uint32_t peer_free_remote = mapa(PEER_FREE, peer);
        const uint32_t recv_remote = mapa(RECV, peer);
        const uint32_t r_remote = mapa(sbase + kOffR, peer);
        int tile_ctr = 0;
        uint32_t grants = 0;
        bool ok = true;
        for (int w = cid; w < npairs && ok; w += ncl) {
            const int t0 = prm.pairs[w];
            const int t = t0 + (int)rank;
            const int nslots = prm.nblk[t0] * bs;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            {
                const float m = prm.smax[(int64_t)t * kN1 + j];
                const float l = prm.ssum[(int64_t)t * kN1 + j];
                cst[j] = m * 1.4426950408889634f;
                cst[128 + j] = l == 0.f ? 0.f : 1.f / l;
                cst[256 + j] = prm.rowsum[(int64_t)t * kN1 + j];
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            const int ntiles = (nslots + kKeys - 1) / kKeys;
            for (int tile = 0; tile < ntiles && ok; ++tile, ++tile_ctr) {
                ok = WAIT(SDP_FULL, tile_ctr & 1, 110);
                // the own-row mask of this tile (staged with the row ids)
                if (ok) ok = WAIT(ROWS_FULL(tile_ctr & 1), (tile_ctr >> 1) & 1, 115);
                if (ok && tile_ctr > 0) ok = WAIT(PDS_FREE, (tile_ctr - 1) & 1, 111);
                if (ok && threadIdx.x == 0) {
                    // R is free again (this CTA's MMAs of the previous tile completed): grant it to the
                    // partner (rank 1 first arms it for the bulk copy of rank 0's dS; rank 0 receives
                    // rank 1's P as stores and one remote arrive); then wait for the partner's grant,
                    // which also means this CTA's previous tile has been consumed there, before writing
                    if (rank) {
                        mbar_expect_tx(RECV, kTileBytes);
                        ++grants;
                        *granted = grants;
                    }
                    if (tile_ctr > 0) {
                        mbar_arrive_remote(peer_free_remote);
                        ok = wait_cluster(PEER_FREE, (tile_ctr - 1) & 1, abort_flag, prm.err, 112, prm.wait_ns);
                    }
                }
                ok = softmax_all(ok);
                if (!ok) break;
                tc_fence_after();
                const uint32_t mbits = masks[(tile_ctr & 1) * 4 + (j >> 5)];
                const bool kv = (mbits >> (j & 31)) & 1u;  // padding / causally cut keys: P = dS = 0 (selected)
                const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
                for (int cc = 0; cc < kN1 / 32; ++cc) {
                    float s[32], dp[32];
                    tmem_ld32(T_S + lane_base + cc * 32, s);
                    tmem_ld32(T_DP + lane_base + cc * 32, dp);
                    tmem_wait_ld();
                    uint32_t pw[16], dw[16];
                    const float4* cm = reinterpret_cast<const float4*>(cst + cc * 32);
                    const float4* cl = reinterpret_cast<const float4*>(cst + 128 + cc * 32);
                    const float4* cd = reinterpret_cast<const float4*>(cst + 256 + cc * 32);
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
                        if (rank)  // rank 1's P is only read by rank 0: stored straight into its R
                            st_cluster_v4(r_remote + off, pw[4 * u], pw[4 * u + 1], pw[4 * u + 2], pw[4 * u + 3]);
                        else
                            *reinterpret_cast<uint4*>(sPp + off) =
                                make_uint4(pw[4 * u], pw[4 * u + 1], pw[4 * u + 2], pw[4 * u + 3]);
                        *reinterpret_cast<uint4*>(sDSp + off) =
                            make_uint4(dw[4 * u], dw[4 * u + 1], dw[4 * u + 2], dw[4 * u + 3]);
                    }
                }
                fence_view_async_shared();
                if (rank) fence_view_async_cluster();
                tc_fence_before();
                mbar_arrive(PDS_FULL);
                asm volatile("bar.sync 1, 128;" ::: "memory");  // the whole tile is written and fenced
                if (threadIdx.x == 0) {
                    if (rank) mbar_arrive_remote(recv_remote);  // rank 0's R holds this tile's P
                    else bulk_copy_to_peer(r_remote, sbase + kOffY, kTileBytes, recv_remote);  // dS to rank 1
                }
            }
        }
    } else {
        // =================== flush (TMEM lane = output dim) ===================
        const int q = warp & 3;
        const int hsel = (warp - 4) >> 2;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int tile_ctr = 0, blk_ctr = 0;
        bool ok = true;
        float fmul_k = 0.f, fmul_v = 0.f;
        if (DET) {
            const FixExp fe = fix_exponents(*prm.dmax, prm.scale, prm.sd.T1, kN1);
            fmul_k = fix_mul(fe.k);
            fmul_v = fix_mul(fe.v);
        }
        const float fmul = rank ? fmul_k : fmul_v;
        for (int w = cid; w < npairs && ok; w += ncl) {
            const int t0 = prm.pairs[w];
            const int t = t0 + (int)rank;
            const int ntiles = (prm.nblk[t0] * bs + kKeys - 1) / kKeys;
            for (int tile = 0; tile < ntiles && ok; ++tile, ++tile_ctr) {
                const int dqmode = ntiles == 1 ? DQ_SINGLE
                                   : (tile == 0 ? DQ_FIRST : (tile == ntiles - 1 ? DQ_LAST : DQ_MID));
                const int rb = tile_ctr & 1;
                ok = __all_sync(0xffffffffu, WAIT(ROWS_FULL(rb), (tile_ctr >> 1) & 1, 113));
                if (!ok) break;
                const int32_t* rid = rowids + rb * kKeys;
                for (int bi = 0; bi < nblocks && ok; ++bi, ++blk_ctr) {
                    const int stg = blk_ctr & 1;
                    ok = __all_sync(0xffffffffu, WAIT(STG_FULL(stg), (blk_ctr >> 1) & 1, 114));
                    if (!ok) break;
                    tc_fence_after();
                    bool dq, moved;
                    int b;
                    block_of(rank, bi, dq, moved, b);
                    const bool active = b < 4 || q < 2;  // rope blocks: 64 valid dims
                    const int dim = (b < 4 ? b * 128 : kD) + q * 32 + lane;
                    if (active) {
                        for (int cc = 2 * hsel; cc < 2 * hsel + 2; ++cc) {
                            float v[32];
                            tmem_ld32(T_STG(stg) + lane_base + cc * 32, v);
                            tmem_wait_ld();
                            if (dq)  // the moved block: rank 0's row, in rank 0's scratch
                                flush_dq<T>(v, dqmode, cc, moved ? t0 : t, dim, prm,
                                            (int)blockIdx.x - (moved ? (int)rank : 0));
                            else flush_keys<DET>(v, rank ? (size_t)dim : (size_t)(kDK + dim), rid + cc * 32, prm,
                                                 fmul);
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
    // copies this CTA granted its partner may still be landing (only after a timeout): wait for them
    // (bounded) before the cluster barrier lets the partner, whose shared memory they read, exit
    if (threadIdx.x == 0) {
        for (uint32_t ph = *consumed; ph < *granted; ++ph) {
            uint64_t t0 = globaltimer();
            while (!mbar_try_cluster(RECV, ph & 1) && globaltimer() - t0 < 1000000000ull) {
            }
        }
    }
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

// ---------------------------------------------------------------------------
// Pairing of adjacent rows with identical block lists, and the work lists
// ---------------------------------------------------------------------------
// Candidate m = rows (2m, 2m + 1) of the flattened row index, for the candidates that meet
// [row_begin, row_end): a pair when both rows lie in the range and are valid rows of the same
// batch / sequence with the same non-empty list of kept blocks (in the order the kernels read).
// Pairs depend on the row index only, so row ranges whose boundaries are even rows form the
// pairs of the whole call.
__global__ void pair_flags_kernel(const int32_t* __restrict__ blocks, const int32_t* __restrict__ nblk, SeqDesc sd,
                                  int64_t topk, int64_t row_begin, int64_t row_end, int32_t* __restrict__ flags) {
    const int lane = threadIdx.x & 31;
    const int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t t0 = 2 * ((row_begin >> 1) + i);
    if (t0 >= row_end) return;
    bool ok = t0 >= row_begin && t0 + 1 < row_end;
    if (ok) {
        const TokInfo a = tok_info(sd, t0), b = tok_info(sd, t0 + 1);
        ok = a.valid && b.valid && a.kv_start == b.kv_start && a.kv_len == b.kv_len && a.q_len == b.q_len;
    }
    ok = ok && nblk[t0] > 0 && nblk[t0] == nblk[t0 + 1];
    if (ok) {
        const int n0 = nblk[t0];
        bool diff = false;
        const int32_t* x = blocks + t0 * topk;
        const int32_t* y = x + topk;
        for (int k = lane; k < n0; k += 32) diff |= x[k] != y[k];
        ok = !__any_sync(0xffffffffu, diff);
    }
    if (lane == 0) flags[i] = ok ? 1 : 0;
}

// Exclusive block-wide prefix sums of two counters (1024 threads); totals returned in *ta / *tb.
__device__ __forceinline__ void scan2(int a, int b, int& ea, int& eb, int& ta, int& tb) {
    __shared__ int wa[32], wb[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int xa = a, xb = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, xa, o), yb = __shfl_up_sync(0xffffffffu, xb, o);
        if (lane >= o) { xa += ya; xb += yb; }
    }
    if (lane == 31) { wa[w] = xa; wb[w] = xb; }
    __syncthreads();
    if (w == 0) {
        int va = wa[lane], vb = wb[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ya = __shfl_up_sync(0xffffffffu, va, o), yb = __shfl_up_sync(0xffffffffu, vb, o);
            if (lane >= o) { va += ya; vb += yb; }
        }
        wa[lane] = va;
        wb[lane] = vb;
    }
    __syncthreads();
    const int pa = w ? wa[w - 1] : 0, pb = w ? wb[w - 1] : 0;
    ea = pa + xa - a;
    eb = pb + xb - b;
    ta = wa[31];
    tb = wb[31];
    __syncthreads();
}

// One CTA of 1024 threads: the pair list (first rows) and the list of the remaining rows of the
// range, both in descending row order (under the causal masks later rows carry more keys: the
// longest work first).
__global__ void __launch_bounds__(1024) pair_lists_kernel(const int32_t* __restrict__ flags, int64_t row_begin,
                                                          int64_t row_end, int32_t* __restrict__ pairs,
                                                          int32_t* __restrict__ solo, int32_t* __restrict__ counts) {
    const int64_t m0 = row_begin >> 1;
    const int64_t M = ((row_end + 1) >> 1) - m0;  // candidates meeting the range
    int np = 0, ns = 0;
    for (int64_t base = 0; base < M; base += 1024) {
        const int64_t i = M - 1 - (base + threadIdx.x);
        const bool valid = base + threadIdx.x < M;
        const int64_t t0 = 2 * (m0 + i);
        const int f = valid ? flags[i] : 0;
        const bool in0 = valid && t0 >= row_begin, in1 = valid && t0 + 1 < row_end;
        const int a = f, b = f ? 0 : (int)in0 + (int)in1;
        int ea, eb, ta, tb;
        scan2(a, b, ea, eb, ta, tb);
        if (a) pairs[np + ea] = (int32_t)t0;
        if (!f) {
            int o = ns + eb;
            if (in1) solo[o++] = (int32_t)(t0 + 1);
            if (in0) solo[o] = (int32_t)t0;
        }
        np += ta;
        ns += tb;
    }
    if (threadIdx.x == 0) {
        counts[0] = np;
        counts[1] = ns;
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <typename T, bool DET>
cudaError_t launch_pair_t(const PairArgs& a, cudaStream_t st) {
    PairParams p;
    memset(&p, 0, sizeof p);
    const int64_t T1 = a.sd.T1, T2 = a.sd.T2;
    if (!make_map(&p.mapQ, a.q, a.dtype, kD, (uint64_t)T1 * kN1, kD, kN1) ||
        !make_map(&p.mapQr, a.qr, a.dtype, kDr, (uint64_t)T1 * kN1, kDr, kN1) ||
        !make_map(&p.mapO, a.dout, a.dtype, kD, (uint64_t)T1 * kN1, kD, kN1) ||
        !make_map(&p.mapK, a.k, a.dtype, kD, (uint64_t)T2, kD, 1) ||
        !make_map(&p.mapKr, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, 1) ||
        !make_map(&p.mapK128, a.k, a.dtype, kD, (uint64_t)T2, kD, kKeys) ||
        !make_map(&p.mapKr128, a.kr, a.dtype, kDr, (uint64_t)T2, kDr, kKeys))
        return cudaErrorInvalidValue;
    p.blocks = a.blocks;
    p.nblk = a.nblk;
    p.pairs = a.pairs;
    p.npairs = a.npairs;
    p.smax = a.smax;
    p.ssum = a.ssum;
    p.rowsum = a.rowsum;
    p.dkv_acc = a.dkv_acc;
    p.dq_scratch = a.dq_acc;
    p.dq_out = a.dq;
    p.dqr_out = a.dqr;
    p.err = a.err;
    p.dmax = a.dout_absmax;
    p.sd = a.sd;
    p.topk = a.topk;
    p.bs = a.bs;
    p.mode = a.mode;
    p.T2 = T2;
    p.scale = a.scale;
    p.wait_ns = wait_limit_ns();

    auto kern = sfa_bwd_pair_kernel<T, DET>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent: as many clusters as can be resident at once (one CTA per SM), at most the
    // per-CTA dQ~ scratch allows
    int ncl = 0;
    cfg.gridDim = dim3(2, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&ncl, (void*)kern, &cfg) != cudaSuccess || ncl < 1) {
        cudaGetLastError();
        ncl = 64;
    }
    if (ncl > kMaxFusedGrid / 2) ncl = kMaxFusedGrid / 2;
    cfg.gridDim = dim3(2 * ncl, 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pair_lists(const int32_t* blocks, const int32_t* nblk, const SeqDesc& sd, int64_t topk,
                              int64_t row_begin, int64_t row_end, int32_t* flags, int32_t* pairs, int32_t* solo,
                              int32_t* counts, cudaStream_t st) {
    const int64_t M = ((row_end + 1) >> 1) - (row_begin >> 1);
    if (M > 0) {
        const int warps = 8;
        pair_flags_kernel<<<(unsigned)((M + warps - 1) / warps), warps * 32, 0, st>>>(blocks, nblk, sd, topk,
                                                                                      row_begin, row_end, flags);
    }
    pair_lists_kernel<<<1, 1024, 0, st>>>(flags, row_begin, row_end, pairs, solo, counts);
    return cudaGetLastError();
}

cudaError_t launch_bwd_pair(int dtype, const PairArgs& a, cudaStream_t st) {
    if (dtype == SFA_DTYPE_BF16)
        return a.det ? launch_pair_t<__nv_bfloat16, true>(a, st) : launch_pair_t<__nv_bfloat16, false>(a, st);
    return a.det ? launch_pair_t<__half, true>(a, st) : launch_pair_t<__half, false>(a, st);
}

}  // namespace sfa
