// Persistent grouped tensor-core GEMM for sm_100a with a fused epilogue,
// run by CTA pairs (cluster of 2, tcgen05 cta_group::2).
//
// Every product of the Newton-Schulz chain (X X^T, the polynomial-in-R
// products, the final Q X / B X) is one TcProblem; a launch walks a list of
// 256 x 256 output tiles drawn from many problems (matrices of different
// shapes).  A CTA pair owns one tile at a time: CTA r holds rows
// [128 r, 128 r + 128) of A and of B (B split along N), the leader CTA (r = 0)
// issues M=256 N=256 K=16 MMAs that read both CTAs' shared memory, and each
// CTA's TMEM receives its 128 rows of the fp32 accumulator.  Per CTA and
// 64-wide K slice this moves 32 KB of operands for 4.2 MFLOP, a third less
// than a single-CTA 128 x 256 tile.  Persistent launches of long products use
// 256 x 512 tiles instead (the NT = 2 instance): two N=256 MMAs on the same A
// slice into one 512-column accumulator, 48 KB per CTA and K slice for
// 8.4 MFLOP.
//
//   warp 10     tile scheduler (leader CTA): claims tiles, publishes records
//   warp 0      TMA producer (both CTAs): 64-wide K slices of its halves of A
//               and B into a 5-stage ring (128-byte swizzle, no multicast);
//               the transaction bytes of both CTAs land on the leader's barrier
//   warp 1      TMEM owner (both CTAs) and MMA issuer (leader only):
//               two 256-column fp32 accumulators (double-buffered), or one of
//               512 columns for 256 x 512 tiles
//   warps 2..9  epilogue: tcgen05.ld of 32-column slices of the warp's TMEM
//               lane quarter (32 rows), fused combine
//               sigma*(alpha*acc + beta*C1) + gamma*C2 + delta*I; each warp
//               stages its 32 x 32 result in a 64-byte-swizzled box in shared
//               memory and one lane stores it with a TMA bulk store (outputs
//               with an unaligned row pitch: direct stores).  Persistent
//               launches run them as one group: all eight warps take every
//               tile (two per lane quarter, 128 columns each).  Chained
//               launches (short K, one chain counter per tile) run them as
//               two groups of four, one per accumulator: group g takes the
//               pair's tiles g, g + 2, g + 4, ... (all 256 columns), so the
//               fixed per-tile latencies of one group (tile record, problem,
//               dependency, store completion, chain counter) overlap the
//               other group's work.
//
// Symmetric outputs (X X^T and every product of polynomials in R) are only
// computed and stored for the upper 256 x 256 tiles; consumers read a lower
// block through the transposed tensor map of the mirrored upper tile, so no
// transposed (mirror) store is ever issued.
//
// The whole Newton-Schulz chain of a step can run as ONE launch: tiles of all
// chain slots are listed slot by slot and a tile first waits (bounded) until
// every tile of the earlier slots of its matrix has been stored, counted in a
// per-matrix completion counter; matrices progress independently, so the
// dependency waits of one matrix are filled with other matrices' tiles.
//
// Tiles are claimed, in list order, from a global ticket by a scheduler warp
// of the leader CTA, which publishes each claimed tile's 32-byte record to
// every role of both CTAs through a short ring in shared memory.  The ring's
// depth bounds how far the scheduler runs ahead of the slowest role, so a
// pair holds only the next few tiles; the claims and record fetches never
// stall the producers, which only read the ring.  A tile that waits on
// earlier tiles only ever waits on tiles that running pairs have claimed:
// the launch makes progress however many of its pairs are resident (other
// kernels may hold SMs), and the dynamic order also balances tiles of
// unequal K across pairs.
//
// Every wait is bounded: on expiry the kernel records a timeout in the device
// status word, drains its own copies and MMAs, frees TMEM and exits.
#include <algorithm>

#include <cuda.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int BM = 128;        // rows of A (and of the output) per CTA
constexpr int BMP = 2 * BM;    // rows per CTA pair
constexpr int BN = 256;        // output columns per tile
constexpr int BNH = BN / 2;    // B rows (N) loaded per CTA
constexpr int BK = 64;
constexpr int STAGES = 5;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BNH * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
// Tile width: NT halves of 256 columns.  NT = 2 (persistent launches of long-K
// products): a CTA pair computes a 256 x 512 tile, both N halves from the
// same A slice, so a quarter fewer operand bytes per FLOP; the one 512-column
// accumulator takes all of TMEM (the epilogue no longer overlaps the next
// tile's main loop) and 4 stages of 48 KB fit.
template <int NT>
__host__ __device__ constexpr int stages_of() { return NT == 1 ? STAGES : 4; }
template <int NT>
__host__ __device__ constexpr int stage_bytes_of() { return A_BYTES + NT * B_BYTES; }
template <int NT>
__host__ __device__ constexpr int num_acc_of() { return NT == 1 ? 2 : 1; }  // TMEM accumulators (512 columns in all)

constexpr int EPI_WARPS = 8;
constexpr int SCHED_WARP = 2 + EPI_WARPS;       // the tile scheduler (after the epilogue warps)
constexpr int NUM_THREADS = 96 + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;  // 2 accumulators x 256 fp32 columns
constexpr int MN_BLOCK_BYTES = 64 * BK * 2;  // one 64 (MN) x 64 (K) box
constexpr int STORE_BOX_BYTES = 64 * 32;  // one TMA store box: 32 rows of 64 bytes
constexpr int STORE_BYTES = EPI_WARPS * 2 * STORE_BOX_BYTES;  // two boxes per epilogue warp
constexpr int SCHED = 4;  // depth of the tile-record ring: the scheduler's lookahead
// The epilogue warps as GROUPS groups (1 or 2), each taking every GROUPS-th
// tile of the pair.
template <int GROUPS, int NT = 1>
struct EpiShape {
    static constexpr int group_warps = EPI_WARPS / GROUPS;
    static constexpr int cols = BN * NT / (group_warps / 4);  // tile columns per epilogue warp
    // readers of every ring slot: in the leader its producer, its MMA thread
    // and the epilogue warps of the group that takes the tile; in the peer
    // its producer and that group's epilogue warps
    static constexpr uint32_t readers_leader = 2 + group_warps;
    static constexpr uint32_t readers_peer = 1 + group_warps;
    static_assert(group_warps % 4 == 0, "a group covers the four TMEM lane quarters");
    static_assert(num_acc_of<NT>() % GROUPS == 0 && SCHED % GROUPS == 0,
                  "a group owns whole accumulators and ring slots");
};
constexpr int kChainGroups = 2;  // epilogue groups of a chained launch (persistent launches: 1)
static_assert(kTileArrivals == 2 * EpiShape<kChainGroups>::group_warps,
              "chain completions are counted per tile: one group's warps in each CTA");
constexpr size_t SMEM_BYTES = STAGES * STAGE_BYTES + STORE_BYTES + 1024 /*align slack*/ + 1024 /*barriers, ring*/;
static_assert(SMEM_BYTES <= 232448, "over the 227 KB of shared memory a CTA may use");
template <int NT>
constexpr size_t smem_bytes() {
    return static_cast<size_t>(stages_of<NT>()) * stage_bytes_of<NT>() + STORE_BYTES + 1024 + 1024;
}
static_assert(smem_bytes<2>() <= 232448, "over the 227 KB of shared memory a CTA may use");
static_assert(stages_of<2>() <= STAGES, "barrier arrays");

// A ring slot: the raw 32-byte tile record (TcTile), or kRingEnd in its
// first word once the launch's tiles are exhausted.
struct RingRec {
    uint4 a, b;
};
constexpr unsigned kRingEnd = 0xFFFFFFFFu;

struct Shared {
    RingRec ring[SCHED];     // claimed tiles' records (the scheduler writes both CTAs')
    uint64_t full[STAGES];   // leader: both CTAs' operand bytes landed
    uint64_t empty[STAGES];  // each CTA: its slot may be refilled (leader's MMA commit)
    uint64_t tfull[2];       // each CTA: accumulator ready (leader's MMA commit)
    uint64_t tempty[2];      // leader: the owning group's warps of both CTAs drained the accumulator
    uint64_t sfull[SCHED];     // each CTA: ring slot holds a record (leader's producer)
    uint64_t sempty_l[SCHED];  // leader: the leader's readers have read the slot (CTA scope)
    uint64_t sempty_p[SCHED];  // leader: the peer's readers have read the slot (cluster scope)
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Shared) <= 1024, "barrier area");

// Symmetric operands are stored as upper 256 x 256 tiles: the 64-wide K slice
// kb of the 256-row block `blk` lies in a lower (unstored) tile when blk > kb/4.
__device__ __forceinline__ bool slice_is_lower(int blk, int kb) { return blk > (kb * BK) / BN; }

// Tile records never change during a launch: read-only path, two 16-byte loads.
__device__ __forceinline__ RingRec load_tile_raw(const TcTile* tiles, int t) {
    const uint4* p = reinterpret_cast<const uint4*>(tiles + t);
    return RingRec{__ldg(p), __ldg(p + 1)};
}

__device__ __forceinline__ TcTile decode_tile(const RingRec& r) {
    TcTile x;
    x.problem = r.a.x;
    x.bibj = r.a.y;
    x.mat = r.a.z;
    x.need = r.a.w;
    x.kf = r.b.x;
    x.a_map = static_cast<unsigned short>(r.b.y & 0xFFFFu);
    x.b_map = static_cast<unsigned short>(r.b.y >> 16);
    x.a_map_t = static_cast<unsigned short>(r.b.z & 0xFFFFu);
    x.b_map_t = static_cast<unsigned short>(r.b.z >> 16);
    x.a_z = static_cast<unsigned short>(r.b.w & 0xFFFFu);
    x.b_z = static_cast<unsigned short>(r.b.w >> 16);
    return x;
}

__device__ __forceinline__ void record_timeout(Shared* sh, DeviceStatus* st) {
    atomicOr(&st->bits, ST_TIMEOUT);
    *reinterpret_cast<volatile int*>(&sh->abort) = 1;
}

// Writer side of the tile ring (the leader's scheduler warp): publish a record in
// the same slot of both CTAs' rings once every reader has read that slot's
// previous record.  The leader CTA's own readers synchronise with it at CTA
// scope (plain shared-memory stores, CTA-scope release and acquire); only
// the link to the peer CTA uses cluster scope.  False when a wait ran out.
struct RingWriter {
    int slot = 0;
    uint32_t phase = 0;
    __device__ bool push(Shared* sh, const RingRec& rec, volatile int* abort_flag, unsigned long long limit) {
        if (!mbar_wait(&sh->sempty_l[slot], phase ^ 1u, abort_flag, limit)) return false;
        if (!mbar_wait_cluster(&sh->sempty_p[slot], phase ^ 1u, abort_flag, limit)) return false;
        st_shared_v4(smem_u32(&sh->ring[slot]), rec.a);
        st_shared_v4(smem_u32(&sh->ring[slot]) + 16, rec.b);
        mbar_arrive(&sh->sfull[slot]);  // release (CTA scope): the record is visible first
        const uint32_t v = map_to_cta(smem_u32(&sh->ring[slot]), 1);
        st_shared_cluster_v4(v, rec.a);
        st_shared_cluster_v4(v + 16, rec.b);
        mbar_arrive_cluster(map_to_cta(smem_u32(&sh->sfull[slot]), 1));  // release (cluster scope)
        if (++slot == SCHED) {
            slot = 0;
            phase ^= 1u;
        }
        return true;
    }
};

// Reader side: the next published record (false when the wait ran out).
// `leader`: this reader runs in the leader CTA (CTA-scope synchronisation).
// An epilogue group reads every GROUPS-th record, from slot `first` on.
struct RingReader {
    int slot = 0;
    uint32_t phase = 0;
    int stride = 1;
    __device__ RingReader(int first = 0, int step = 1) : slot(first), stride(step) {}
    __device__ bool pop(Shared* sh, RingRec& rec, bool leader, volatile int* abort_flag, unsigned long long limit) {
        const bool got = leader ? mbar_wait(&sh->sfull[slot], phase, abort_flag, limit)
                                : mbar_wait_cluster(&sh->sfull[slot], phase, abort_flag, limit);
        if (!got) return false;
        const volatile uint4* p = reinterpret_cast<const volatile uint4*>(&sh->ring[slot]);
        rec.a = make_uint4(p[0].x, p[0].y, p[0].z, p[0].w);
        rec.b = make_uint4(p[1].x, p[1].y, p[1].z, p[1].w);
        if (leader)
            mbar_arrive(&sh->sempty_l[slot]);  // read: the slot is free (CTA scope)
        else
            mbar_arrive_cluster(map_to_cta(smem_u32(&sh->sempty_p[slot]), 0));
        slot += stride;
        if (slot >= SCHED) {
            slot -= SCHED;
            phase ^= 1u;
        }
        return true;
    }
    // The next record if it is already published, without consuming it (its
    // slot cannot be rewritten before this reader has popped it).
    __device__ bool peek(Shared* sh, RingRec& rec, bool leader) {
        if (!(leader ? mbar_try_wait(&sh->sfull[slot], phase) : mbar_try_wait_cluster(&sh->sfull[slot], phase)))
            return false;
        const volatile uint4* p = reinterpret_cast<const volatile uint4*>(&sh->ring[slot]);
        rec.a = make_uint4(p[0].x, p[0].y, p[0].z, p[0].w);
        rec.b = make_uint4(p[1].x, p[1].y, p[1].z, p[1].w);
        return true;
    }
};

__device__ __forceinline__ RingRec end_rec() { return RingRec{make_uint4(kRingEnd, 0, 0, 0), make_uint4(0, 0, 0, 0)}; }

template <int NT>
__device__ void producer(const TcLaunch& L, uint8_t* tiles_smem, Shared* sh, uint32_t rank) {
    constexpr int kStages = stages_of<NT>(), kStageBytes = stage_bytes_of<NT>();
    volatile int* abort_flag = &sh->abort;
    const unsigned long long lim = L.wait_ns;
    const bool leader = rank == 0;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;
    bool ok = true;
    int last_a = -1, last_b = -1;
    unsigned seen_mat = ~0u, seen_done = 0;  // counters only grow within a launch
    RingReader rd;
    // Both producers read the tile ring (the scheduler warp claims and
    // publishes ahead).  The next tile's dependency and tensor maps are
    // acquired right after the current tile's last fill is issued (the
    // slices still queued hide the wait).
    bool early = false;  // the current tile's dependency was acquired early
    while (ok) {
        RingRec cur;
        if (!rd.pop(sh, cur, leader, abort_flag, lim)) {
            ok = false;
            break;
        }
        if (cur.a.x == kRingEnd) break;
        const TcTile tile = decode_tile(cur);
        RingRec nxt_rec;
        // operands produced by earlier chain slots of the same matrix
        if (tile.need && !(tile.mat == seen_mat && tile.need <= seen_done)) {
            if (!early && !wait_counter(L.done + tile.mat, tile.need, abort_flag, lim)) {
                ok = false;
                break;
            }
            seen_mat = tile.mat;
            seen_done = tile.need;
            fence_proxy_async_global();  // TMA reads see the producers' stores
        }
        early = false;
        const int K = static_cast<int>(tile.kf & kTileMaxK);
        const unsigned fl = tile.kf >> 24;
        const bool a_mn = fl & TILE_A_MN, b_mn = fl & TILE_B_MN, a_sym = fl & TILE_A_SYM, b_sym = fl & TILE_B_SYM;
        const int a_z = tile.a_z, b_z = tile.b_z;
        const int bi = static_cast<int>(tile.bibj >> 16), bj = static_cast<int>(tile.bibj & 0xFFFFu);
        const int h0 = (NT > 1 && (fl & TILE_LOWER0)) ? 1 : 0;  // first N half skipped (lower block)
        const CUtensorMap* ma = L.maps + tile.a_map;
        const CUtensorMap* mb = L.maps + tile.b_map;
        const CUtensorMap* ma_t = a_sym ? L.maps + tile.a_map_t : ma;
        const CUtensorMap* mb_t = b_sym ? L.maps + tile.b_map_t : mb;
        if (tile.a_map != last_a) {
            tma_map_acquire(ma);
            if (a_sym) tma_map_acquire(ma_t);
            last_a = tile.a_map;
        }
        if (tile.b_map != last_b) {
            tma_map_acquire(mb);
            if (b_sym) tma_map_acquire(mb_t);
            last_b = tile.b_map;
        }
        const int arow = bi * BMP + static_cast<int>(rank) * BM;   // this CTA's A rows
        const int nk = (K + BK - 1) / BK;
        for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(&sh->empty[stage], phase ^ 1u, abort_flag, lim)) {
                ok = false;
                break;
            }
            uint8_t* sa = tiles_smem + stage * kStageBytes;
            const uint32_t full_leader = map_to_cta(smem_u32(&sh->full[stage]), 0);
            // both CTAs' A slice and the B halves this tile computes
            if (leader) mbar_arrive_expect_tx(&sh->full[stage], 2 * (A_BYTES + (NT - h0) * B_BYTES));
            // a K slice of a symmetric operand below its stored upper tiles is
            // read transposed from the mirrored tile (same values)
            const bool a_t = a_mn || (a_sym && slice_is_lower(bi, kb));
            if (!a_t) {
                tma_load_3d_pair(sa, ma, full_leader, kb * BK, arow, a_z);
            } else {
#pragma unroll
                for (int j = 0; j < BM / 64; ++j)
                    tma_load_3d_pair(sa + j * MN_BLOCK_BYTES, ma_t, full_leader, arow + 64 * j, kb * BK, a_z);
            }
#pragma unroll
            for (int h = 0; h < NT; ++h) {
                if (h < h0) continue;
                // N half h: 256-column block bj * NT + h, this CTA's 128 rows of it
                const int blk = bj * NT + h;
                const int brow = blk * BN + static_cast<int>(rank) * BNH;
                uint8_t* sb = sa + A_BYTES + h * B_BYTES;
                const bool b_t = b_mn || (b_sym && slice_is_lower(blk, kb));
                if (!b_t) {
                    tma_load_3d_pair(sb, mb, full_leader, kb * BK, brow, b_z);
                } else {
#pragma unroll
                    for (int j = 0; j < BNH / 64; ++j)
                        tma_load_3d_pair(sb + j * MN_BLOCK_BYTES, mb_t, full_leader, brow + 64 * j, kb * BK, b_z);
                }
            }
            ++issued;
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        // the next tile, if the scheduler has published it already
        if (ok && rd.peek(sh, nxt_rec, leader) && nxt_rec.a.x != kRingEnd) {
            const TcTile nxt = decode_tile(nxt_rec);
            if (nxt.need && !(nxt.mat == seen_mat && nxt.need <= seen_done))
                early = ld_acquire_gpu(L.done + nxt.mat) >= nxt.need;
            const unsigned nfl = nxt.kf >> 24;
            if (nxt.a_map != last_a) {
                tma_map_acquire(L.maps + nxt.a_map);
                if (nfl & TILE_A_SYM) tma_map_acquire(L.maps + nxt.a_map_t);
                last_a = nxt.a_map;
            }
            if (nxt.b_map != last_b) {
                tma_map_acquire(L.maps + nxt.b_map);
                if (nfl & TILE_B_SYM) tma_map_acquire(L.maps + nxt.b_map_t);
                last_b = nxt.b_map;
            }
        }
    }
    if (!ok) record_timeout(sh, L.status);
    // Drain (leader): the last fills of every stage must have landed before
    // the pair exits.  Fill i used stage i % STAGES, phase parity (i / STAGES) & 1.
    if (leader) {
        const uint32_t first = issued > kStages ? issued - kStages : 0;
        int never = 0;
        for (uint32_t i = first; i < issued; ++i) {
            if (!mbar_wait(&sh->full[i % kStages], (i / kStages) & 1u, &never, lim)) {
                atomicOr(&L.status->bits, ST_TIMEOUT);
                break;
            }
        }
    }
}

// The tile scheduler (one thread of the leader CTA): claims tiles in list
// order and publishes their records until the list is exhausted, then one end
// marker per epilogue group (the producers and the MMA thread stop at the
// first).  Its waits are only for free ring slots.
template <int GROUPS>
__device__ void scheduler(const TcLaunch& L, Shared* sh) {
    volatile int* abort_flag = &sh->abort;
    const unsigned long long lim = L.wait_ns;
    RingWriter wr;
    int ends = 0;
    while (ends < GROUPS) {
        unsigned t = static_cast<unsigned>(L.ntiles);
        if (ends == 0) t = atomicAdd(L.ticket, 1u);
        const RingRec rec = t < static_cast<unsigned>(L.ntiles) ? load_tile_raw(L.tiles, static_cast<int>(t)) : end_rec();
        if (!wr.push(sh, rec, abort_flag, lim)) {
            record_timeout(sh, L.status);
            return;
        }
        if (rec.a.x == kRingEnd) ++ends;
    }
}

template <int NT>
__device__ void mma_issuer(const TcLaunch& L, uint8_t* tiles_smem, Shared* sh, uint32_t tmem_base) {
    constexpr int kStages = stages_of<NT>(), kStageBytes = stage_bytes_of<NT>(), kAcc = num_acc_of<NT>();
    volatile int* abort_flag = &sh->abort;
    const unsigned long long lim = L.wait_ns;
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool issued_any = false;
    const uint32_t tiles_base = smem_u32(tiles_smem);
    RingReader rd;
    while (ok) {
        RingRec rec;
        if (!rd.pop(sh, rec, true, abort_flag, lim)) {  // the MMA thread runs in the leader CTA
            ok = false;
            break;
        }
        if (rec.a.x == kRingEnd) break;
        const TcTile tile = decode_tile(rec);
        const int K = static_cast<int>(tile.kf & kTileMaxK);
        const unsigned fl = tile.kf >> 24;
        const int a_mn = (fl & TILE_A_MN) ? 1 : 0, b_mn = (fl & TILE_B_MN) ? 1 : 0;
        const int a_sym = (fl & TILE_A_SYM) ? 1 : 0, b_sym = (fl & TILE_B_SYM) ? 1 : 0;
        const int fmt = (fl & TILE_BF16) ? 1 : 0;
        const int bi = static_cast<int>(tile.bibj >> 16), bj = static_cast<int>(tile.bibj & 0xFFFFu);
        const int h0 = (NT > 1 && (fl & TILE_LOWER0)) ? 1 : 0;  // first N half skipped (lower block)
        const int nk = (K + BK - 1) / BK;
        if (!mbar_wait(&sh->tempty[acc], acc_phase ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN * NT);
        for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(&sh->full[stage], phase, abort_flag, lim)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = tiles_base + stage * kStageBytes;
            const int a_t = (a_mn || (a_sym && slice_is_lower(bi, kb))) ? 1 : 0;  // as loaded by the producer
#pragma unroll
            for (int h = 0; h < NT; ++h) {
                if (h < h0) continue;
                // N half h: its own B slice, accumulator columns [256 h, 256 h + 256)
                const uint32_t b_addr = a_addr + A_BYTES + h * B_BYTES;
                const int b_t = (b_mn || (b_sym && slice_is_lower(bj * NT + h, kb))) ? 1 : 0;
                const uint32_t idesc = make_instr_desc(fmt, a_t, b_t, BMP, BN);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k) {
                    // K-major: advance 16 elements (32 B) inside the swizzled row;
                    // MN-major: advance 16 k-rows (two 8-row groups of 1024 B).
                    const uint64_t ad = a_t ? make_smem_desc(a_addr + k * 2048, MN_BLOCK_BYTES, 1024)
                                            : make_smem_desc(a_addr + k * 32, 16, 1024);
                    const uint64_t bd = b_t ? make_smem_desc(b_addr + k * 2048, MN_BLOCK_BYTES, 1024)
                                            : make_smem_desc(b_addr + k * 32, 16, 1024);
                    umma_f16_pair(d_tmem + static_cast<uint32_t>(h * BN), ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                }
            }
            issued_any = true;
            umma_commit_pair(&sh->empty[stage], 0x3);  // both CTAs may refill this slot
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
        umma_commit_pair(&sh->tfull[acc], 0x3);  // accumulator ready in both CTAs
        if (++acc == kAcc) {
            acc = 0;
            acc_phase ^= 1u;
        }
    }
    if (!ok) {
        record_timeout(sh, L.status);
        if (issued_any) {
            // wait for this thread's MMAs before TMEM is released
            int never = 0;
            umma_commit_pair(&sh->drain, 0x1);
            if (!mbar_wait(&sh->drain, 0, &never, lim)) atomicOr(&L.status->bits, ST_TIMEOUT);
        }
    }
}

template <int GROUPS, int NT>
__device__ void epilogue_warps(const TcLaunch& L, Shared* sh, uint32_t stg, uint32_t tmem_base, int warp, int lane,
                               uint32_t rank) {
    using S = EpiShape<GROUPS, NT>;
    constexpr int kAcc = num_acc_of<NT>();
    volatile int* abort_flag = &sh->abort;
    const unsigned long long lim = L.wait_ns;
    const int q = warp & 3;                       // TMEM lane quarter this warp may access
    const int group = (warp - 2) / S::group_warps;       // takes the pair's tiles group, group + GROUPS, ...
    const int part = ((warp - 2) % S::group_warps) >> 2;  // column part of the tile
    const uint32_t tempty_leader[2] = {map_to_cta(smem_u32(&sh->tempty[0]), 0),
                                       map_to_cta(smem_u32(&sh->tempty[1]), 0)};
    // tile i of the pair uses accumulator i % kAcc (the MMA thread alternates)
    int acc = group % kAcc;
    uint32_t acc_phase = 0;
    unsigned seen_mat = ~0u, seen_done = 0;
    uint32_t nstored = 0;  // TMA store boxes issued by this warp (alternating buffers)
    int last_map = -1;
    // this lane's 64-byte row of a store box, 16-byte units swizzled (64-byte mode)
    const uint32_t row_off = static_cast<uint32_t>(lane) * 64;
    const uint32_t sw = (static_cast<uint32_t>(lane) >> 1) & 3u;
    // lane 0 reads the tile ring for the warp (one reader per warp) and
    // passes the record's first half (problem, position, matrix, dependency)
    RingReader rd(group, GROUPS);
    bool timed_out = false;
    while (true) {
        RingRec rec;
        int got_rec = 1;
        if (lane == 0) got_rec = rd.pop(sh, rec, rank == 0, abort_flag, lim) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, got_rec, 0)) {
            timed_out = true;
            break;
        }
        TcTile tile;
        tile.problem = __shfl_sync(0xffffffffu, rec.a.x, 0);
        tile.bibj = __shfl_sync(0xffffffffu, rec.a.y, 0);
        tile.mat = __shfl_sync(0xffffffffu, rec.a.z, 0);
        tile.need = __shfl_sync(0xffffffffu, rec.a.w, 0);
        if (tile.problem == kRingEnd) break;
        // Local copies: the epilogue stores to global memory, so fields read
        // through a reference into the problem table would be reloaded after
        // every store (the compiler cannot rule out aliasing).
        Epilogue ep = L.problems[tile.problem].ep;
        const int PM = L.problems[tile.problem].M, PN = L.problems[tile.problem].N;
        const int bi = static_cast<int>(tile.bibj >> 16), bj = static_cast<int>(tile.bibj & 0xFFFFu);
        // the epilogue inputs (C1) come from earlier slots: acquire them too
        if (tile.need && !(tile.mat == seen_mat && tile.need <= seen_done)) {
            if (lane == 0) (void)wait_counter(L.done + tile.mat, tile.need, abort_flag, lim);
            __syncwarp();
            seen_mat = tile.mat;
            seen_done = tile.need;
        }
        // a 512-wide tile of a symmetric output may reach below the diagonal:
        // a part whose 256-column block is a lower block is not stored (only
        // upper blocks are; their consumers read lower blocks transposed)
        const bool lower = NT > 1 && L.problems[tile.problem].pad_ != 0 && bi > bj * NT + part;
        const bool skip = (ep.skip_idx >= 0 && L.bad[ep.skip_idx] != 0) || lower;
        const float sig = ep.sigma ? *ep.sigma : 1.f;
        const long long row0 = static_cast<long long>(bi) * BMP + rank * BM + q * 32;  // this warp's first row
        const long long row = row0 + lane;
        const int cbase = bj * BN * NT + part * S::cols;
        const bool use_tma = ep.o1_map >= 0;
        const CUtensorMap* omap = use_tma ? L.maps + ep.o1_map : nullptr;
        if (use_tma && ep.o1_map != last_map) {
            if (lane == 0) tma_map_acquire(omap);
            last_map = ep.o1_map;
        }
        const int nbox = ep.o1_dt == DT_F32 ? 2 : 1;  // 64-byte boxes per 32-column slice
        bool stored = false;
        // prefetch the C1 row segment of the first slice while the MMAs run
        Raw32 pre;
        prefetch_row32(ep, PM, PN, row, cbase, pre);
        // C2 (the parameters of the fused update, read once from DRAM): pull
        // this lane's row of the warp's columns into L2 now, so the per-slice
        // loads below hit L2
        if (ep.c2 && !skip && row < PM) {
            const int es = ep.c2_dt == DT_F32 ? 4 : 2;
            const char* p = static_cast<const char*>(ep.c2) + (row * ep.ldc2 + cbase) * es;
            const int bytes = min(S::cols, PN - cbase) * es;
            for (int o = 0; o < bytes; o += 128) prefetch_l2(p + o);
        }
        // The fused update of fp32 parameters, W <- W + d in place (C2 = the
        // output, coefficient 1), in chained launches: the warp stages d alone
        // and the TMA store adds it to W at L2, so W is never loaded into
        // registers and the accumulator is released sooner (the epilogue is
        // the limit there).  The sum is the one rounding of W + d that the
        // register path makes.  Persistent launches keep the register path:
        // their limit is the operand feed from L2, which the adds at L2 would
        // compete with.
        const bool radd = GROUPS == kChainGroups && use_tma && ep.c2 != nullptr && ep.c2 == ep.o1 &&
                          ep.ldc2 == ep.ldo1 && ep.c2_dt == DT_F32 && ep.o1_dt == DT_F32 && ep.gamma == 1.f;
        if (radd) ep.c2 = nullptr;
        // every lane waits; the warp leaves together unless all lanes saw the
        // accumulator arrive (a lane's wait may end just before the arrival)
        const bool got = mbar_wait(&sh->tfull[acc], acc_phase, abort_flag, lim);
        if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0) record_timeout(sh, L.status);
            break;
        }
        tc_fence_after();
        // one slice per iteration, not unrolled: the epilogue's code stays small
#pragma unroll 1
        for (int c = 0; c < S::cols; c += 32) {
            const int col0 = cbase + c;
            Raw32 nxt;  // C1 of the next slice, fetched while this one is processed
            nxt.ok = 0;
            if (c + 32 < S::cols) prefetch_row32(ep, PM, PN, row, col0 + 32, nxt);
            if (col0 >= PN) {  // warp-uniform
                pre = nxt;
                continue;
            }
            uint32_t r[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN * NT + part * S::cols + c, r);
            tmem_wait_ld();
            if (skip || row0 >= PM) {  // warp-uniform
                pre = nxt;
                continue;
            }
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            const bool valid = epilogue_values32(ep, sig, PM, PN, row, col0, v, &pre);
            pre = nxt;
            if (!use_tma) {
                if (valid) {
                    Row32 out;
#pragma unroll
                    for (int j = 0; j < 32; ++j) out.v[j] = v[j];
                    store_row32_cold(ep.o1, ep.o1_dt, ep.ldo1, row, col0, min(32, PN - col0), out);
                }
                continue;
            }
            // staged TMA store: rows past M and columns past N are clipped
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h >= nbox) break;
                const uint32_t buf = stg + ((nstored & 1u) * STORE_BOX_BYTES);
                if (lane == 0 && nstored >= 2) bulk_wait_read<1>();  // the box's previous store has read it
                __syncwarp();
                if (ep.o1_dt == DT_F32) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float* f = v + 16 * h + 4 * u;
                        st_shared_v4(buf + row_off + ((static_cast<uint32_t>(u) ^ sw) << 4),
                                     make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                                                __float_as_uint(f[3])));
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        st_shared_v4(buf + row_off + ((static_cast<uint32_t>(u) ^ sw) << 4), pack8(v + 8 * u, ep.o1_dt));
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    if (radd)
                        tma_reduce_add_3d(omap, buf, col0 + 16 * h, static_cast<int>(row0), ep.o1_z);
                    else
                        tma_store_3d(omap, buf, col0 + 16 * h, static_cast<int>(row0), ep.o1_z);
                    bulk_commit();
                }
                ++nstored;
                stored = true;
            }
        }
        // the accumulator is free as soon as it has been read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
        if (L.done) {
            // this warp's stores are complete and visible before the tile counts as done
            if (lane == 0 && stored) {
                bulk_wait_all();
                fence_proxy_async_global();
            }
            __syncwarp();
            if (lane == 0) red_release_add_gpu(L.done + tile.mat, 1u);
        }
        acc += GROUPS;  // this group's next tile
        if (acc >= kAcc) {
            acc -= kAcc;
            acc_phase ^= 1u;
        }
    }
    if (timed_out && lane == 0) record_timeout(sh, L.status);
    // the staging boxes must stay valid until every store has read them
    if (lane == 0) bulk_wait_all();
    __syncwarp();
}

template <int GROUPS, int NT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ TcLaunch L) {
    using S = EpiShape<GROUPS, NT>;
    constexpr int kStages = stages_of<NT>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles_smem =
        reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* store_smem = tiles_smem + kStages * stage_bytes_of<NT>();  // 1024-byte aligned boxes
    Shared* sh = reinterpret_cast<Shared*>(store_smem + STORE_BYTES);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_cta_rank();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh->tfull[a], 1);
            mbar_init(&sh->tempty[a], 2 * S::group_warps);  // the owning group's warps of both CTAs
        }
        for (int r = 0; r < SCHED; ++r) {
            mbar_init(&sh->sfull[r], 1);                       // the scheduler publishes
            mbar_init(&sh->sempty_l[r], S::readers_leader);  // used in the leader only
            mbar_init(&sh->sempty_p[r], S::readers_peer);    // used in the leader only
        }
        mbar_init(&sh->drain, 1);
        sh->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&sh->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the peer's barriers exist before anyone signals them
    tc_fence_after();
    const uint32_t tmem_base = sh->tmem_base;

    if (warp == 0) {
        if (lane == 0) producer<NT>(L, tiles_smem, sh, rank);
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) mma_issuer<NT>(L, tiles_smem, sh, tmem_base);
    } else if (warp == SCHED_WARP) {
        if (lane == 0 && rank == 0) scheduler<GROUPS>(L, sh);
    } else {
        epilogue_warps<GROUPS, NT>(L, sh, smem_u32(store_smem + (warp - 2) * 2 * STORE_BOX_BYTES), tmem_base, warp, lane,
                                   rank);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its peer may still touch its memory or TMEM
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace

size_t gemm_tc_smem_bytes() { return SMEM_BYTES; }
int gemm_tc_tile_m() { return BMP; }
int gemm_tc_tile_n() { return BN; }
int gemm_tc_wide_tile_n() { return 2 * BN; }

namespace {
// CTA pairs of one instance that can be resident at once.
template <int GROUPS, int NT>
int max_pairs_of() {
    cudaFuncSetAttribute(gemm_tc_kernel<GROUPS, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem_bytes<NT>()));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<NT>();
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<GROUPS, NT>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    return n;
}
}  // namespace

// CTA pairs that can be resident at once (either instance): the grid of a
// persistent launch.
int gemm_tc_max_pairs() {
    static int cached = -1;
    if (cached >= 0) return cached;
    cached = std::min(std::min(max_pairs_of<1, 1>(), max_pairs_of<kChainGroups, 1>()), max_pairs_of<1, 2>());
    return cached;
}

cudaError_t launch_gemm_tc(const TcLaunch& L, int grid, cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<1, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem_bytes<1>()));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemm_tc_kernel<kChainGroups, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem_bytes<1>()));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemm_tc_kernel<1, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem_bytes<2>()));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (L.ntiles <= 0) return cudaSuccess;
    // chained launches (chain counters) split the epilogue into two groups;
    // persistent launches of 512-wide tiles take the wide instance
    if (L.done)
        gemm_tc_kernel<kChainGroups, 1><<<grid, NUM_THREADS, smem_bytes<1>(), stream>>>(L);
    else if (L.nt == 2)
        gemm_tc_kernel<1, 2><<<grid, NUM_THREADS, smem_bytes<2>(), stream>>>(L);
    else
        gemm_tc_kernel<1, 1><<<grid, NUM_THREADS, smem_bytes<1>(), stream>>>(L);
    return cudaGetLastError();
}

}  // namespace muon
