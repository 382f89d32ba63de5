// Persistent grouped tensor-core GEMM for sm_100a with a fused epilogue.
//
// Every product of the Newton-Schulz chain (X X^T, polynomial-in-R products,
// the final Q X / B X) is one TcProblem; a launch runs a list of 128 x 256
// output tiles drawn from many problems (matrices of different shapes).
//
//   warp 0      TMA producer: 64-wide K slices of A (128 rows) and B (256 rows)
//               into a 4-stage shared-memory ring (128-byte swizzle, no multicast)
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma kind::f16, M=128 N=256
//               K=16, fp32 accumulators in TMEM, two accumulator slots
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, fused combine
//               sigma*(alpha*acc + beta*C1) + gamma*C2 + delta*I, stores
//               (mirrored for symmetric outputs)
//
// The epilogue of tile i overlaps the main loop of tile i+1 (double-buffered
// TMEM).  Every wait is bounded: on expiry the kernel records a timeout in the
// device status word, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;  // 2 accumulators x 256 fp32 columns
constexpr int MN_BLOCK_BYTES = 64 * BK * 2;  // one 64 (MN) x 64 (K) box
constexpr size_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align slack*/ + 256 /*barriers*/;

struct Shared {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void record_timeout(Shared* sh, DeviceStatus* st) {
    atomicOr(&st->bits, ST_TIMEOUT);
    *reinterpret_cast<volatile int*>(&sh->abort) = 1;
}

__device__ void producer(const TcLaunch& L, uint8_t* tiles_smem, Shared* sh) {
    volatile int* abort_flag = &sh->abort;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;  // number of stage fills issued
    bool ok = true;
    int last_a = -1, last_b = -1;
    for (int t = blockIdx.x; t < L.ntiles && ok; t += gridDim.x) {
        const uint2 tile = L.tiles[t];
        const TcProblem& P = L.problems[tile.x];
        const int bi = static_cast<int>(tile.y >> 16), bj = static_cast<int>(tile.y & 0xFFFFu);
        const CUtensorMap* ma = L.maps + P.a_map;
        const CUtensorMap* mb = L.maps + P.b_map;
        if (P.a_map != last_a) {
            tma_map_acquire(ma);
            last_a = P.a_map;
        }
        if (P.b_map != last_b) {
            tma_map_acquire(mb);
            last_b = P.b_map;
        }
        const int nk = (P.K + BK - 1) / BK;
        for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(&sh->empty[stage], phase ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            uint8_t* sa = tiles_smem + stage * STAGE_BYTES;
            uint8_t* sb = sa + A_BYTES;
            mbar_arrive_expect_tx(&sh->full[stage], STAGE_BYTES);
            if (!P.a_mn) {
                tma_load_3d(sa, ma, &sh->full[stage], kb * BK, bi * BM, P.a_z);
            } else {
#pragma unroll
                for (int j = 0; j < BM / 64; ++j)
                    tma_load_3d(sa + j * MN_BLOCK_BYTES, ma, &sh->full[stage], bi * BM + 64 * j, kb * BK, P.a_z);
            }
            if (!P.b_mn) {
                tma_load_3d(sb, mb, &sh->full[stage], kb * BK, bj * BN, P.b_z);
            } else {
#pragma unroll
                for (int j = 0; j < BN / 64; ++j)
                    tma_load_3d(sb + j * MN_BLOCK_BYTES, mb, &sh->full[stage], bj * BN + 64 * j, kb * BK, P.b_z);
            }
            ++issued;
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }
    if (!ok) record_timeout(sh, L.status);
    // Drain: every issued fill must have landed before the CTA exits.  Fill i
    // used stage i % STAGES with phase parity (i / STAGES) & 1.
    const uint32_t first = issued > STAGES ? issued - STAGES : 0;
    int never = 0;
    for (uint32_t i = first; i < issued; ++i) {
        if (!mbar_wait(&sh->full[i % STAGES], (i / STAGES) & 1u, &never)) {
            atomicOr(&L.status->bits, ST_TIMEOUT);
            break;
        }
    }
}

__device__ void mma_issuer(const TcLaunch& L, uint8_t* tiles_smem, Shared* sh, uint32_t tmem_base) {
    volatile int* abort_flag = &sh->abort;
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool issued_any = false;
    const uint32_t tiles_base = smem_u32(tiles_smem);
    for (int t = blockIdx.x; t < L.ntiles && ok; t += gridDim.x) {
        const uint2 tile = L.tiles[t];
        const TcProblem& P = L.problems[tile.x];
        const int nk = (P.K + BK - 1) / BK;
        if (!mbar_wait(&sh->tempty[acc], acc_phase ^ 1u, abort_flag)) {
            ok = false;
            break;
        }
        tc_fence_after();
        const uint32_t idesc = make_instr_desc(P.fmt, P.a_mn, P.b_mn, BM, BN);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(&sh->full[stage], phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a_addr = tiles_base + stage * STAGE_BYTES;
            const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
                // K-major: advance 16 elements (32 B) inside the swizzled row;
                // MN-major: advance 16 k-rows (two 8-row groups of 1024 B).
                const uint64_t ad = P.a_mn ? make_smem_desc(a_addr + k * 2048, MN_BLOCK_BYTES, 1024)
                                           : make_smem_desc(a_addr + k * 32, 16, 1024);
                const uint64_t bd = P.b_mn ? make_smem_desc(b_addr + k * 2048, MN_BLOCK_BYTES, 1024)
                                           : make_smem_desc(b_addr + k * 32, 16, 1024);
                umma_f16(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
            }
            issued_any = true;
            umma_commit(&sh->empty[stage]);  // frees the smem slot once these MMAs finish
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
        umma_commit(&sh->tfull[acc]);  // accumulator ready for the epilogue
        if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
        }
    }
    if (!ok) {
        record_timeout(sh, L.status);
        if (issued_any) {
            // wait for this thread's MMAs before TMEM is released
            int never = 0;
            umma_commit(&sh->drain);
            if (!mbar_wait(&sh->drain, 0, &never)) atomicOr(&L.status->bits, ST_TIMEOUT);
        }
    }
}

__device__ void epilogue_warps(const TcLaunch& L, Shared* sh, uint32_t tmem_base, int warp, int lane) {
    volatile int* abort_flag = &sh->abort;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < L.ntiles; t += gridDim.x) {
        const uint2 tile = L.tiles[t];
        const TcProblem& P = L.problems[tile.x];
        const int bi = static_cast<int>(tile.y >> 16), bj = static_cast<int>(tile.y & 0xFFFFu);
        if (!mbar_wait(&sh->tfull[acc], acc_phase, abort_flag)) {
            if (lane == 0) record_timeout(sh, L.status);
            break;
        }
        tc_fence_after();
        const Epilogue& ep = P.ep;
        const bool skip = ep.skip_idx >= 0 && L.bad[ep.skip_idx] != 0;
        const float sig = ep.sigma ? *ep.sigma : 1.f;
        const long long row0 = static_cast<long long>(bi) * BM + q * 32;
        const long long row = row0 + lane;
        for (int c = 0; c < BN; c += 32) {
            const int col0 = bj * BN + c;
            if (col0 >= P.N) break;                          // warp-uniform
            if (ep.sym && row0 > col0 + 31) continue;        // warp-uniform: strictly below the diagonal
            uint32_t r[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c, r);
            tmem_wait_ld();
            if (!skip) {
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
                epilogue_row32(ep, sig, P.M, P.N, row, col0, v);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->tempty[acc]);
        if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
        }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_tc_kernel(const __grid_constant__ TcLaunch L) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles_smem =
        reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Shared* sh = reinterpret_cast<Shared*>(tiles_smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sh->tfull[a], 1);
            mbar_init(&sh->tempty[a], 4);  // one arrival per epilogue warp
        }
        mbar_init(&sh->drain, 1);
        sh->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sh->tmem_base;

    if (warp == 0) {
        if (lane == 0) producer(L, tiles_smem, sh);
    } else if (warp == 1) {
        if (lane == 0) mma_issuer(L, tiles_smem, sh, tmem_base);
    } else {
        epilogue_warps(L, sh, tmem_base, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace

size_t gemm_tc_smem_bytes() { return SMEM_BYTES; }
int gemm_tc_tile_m() { return BM; }
int gemm_tc_tile_n() { return BN; }

cudaError_t launch_gemm_tc(const TcLaunch& L, int grid, cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(SMEM_BYTES));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (L.ntiles <= 0) return cudaSuccess;
    gemm_tc_kernel<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(L);
    return cudaGetLastError();
}

}  // namespace muon
