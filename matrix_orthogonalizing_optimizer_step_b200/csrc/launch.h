// Internal launch interface between the planner and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "muon_internal.h"

namespace muon {

// One tile of work.  Tiles of a matrix's later chain slots depend on all of
// its earlier tiles: before fetching operands, a tile waits until
// done[mat] >= need (done counts epilogue-warp completions, 2 CTAs x 8 warps
// per tile).  need = 0 means no dependency (one launch per chain slot).
//
// A tile record also carries everything the TMA producer and the MMA issuer
// read (K, operand layout flags, tensor maps, batch coordinates): 32 bytes,
// fetched one tile ahead, so no dependent load of the problem table sits
// between two tiles of a CTA pair.
struct TcTile {
    unsigned problem;  // index into the problem table (epilogue, M, N)
    unsigned bibj;     // (tile_row << 16) | tile_col
    unsigned mat;      // matrix index (completion counter)
    unsigned need;
    unsigned kf;       // K (low 24 bits) | operand flags (TILE_*) << 24
    unsigned short a_map, b_map, a_map_t, b_map_t;  // tensor-map indices (_t: transposed, symmetric operands)
    unsigned short a_z, b_z;                          // batch coordinates
};
static_assert(sizeof(TcTile) == 32, "tile records are loaded as two 16-byte vectors");
// TILE_LOWER0: a 256 x 512 tile of a symmetric output whose first 256-column
// half is a lower block: that half is neither loaded, computed nor stored.
enum { TILE_A_MN = 1, TILE_B_MN = 2, TILE_A_SYM = 4, TILE_B_SYM = 8, TILE_BF16 = 16, TILE_LOWER0 = 32 };
constexpr unsigned kTileMaxK = (1u << 24) - 1;

// Tiles are claimed in list order from `ticket` (a global counter, zero at
// launch): a CTA pair processes the tiles it claims in the order it claimed
// them.  Every dependency of a tile is on tiles earlier in the list, which
// are therefore already owned by pairs that are running, whichever pairs of
// the grid the hardware has made resident.
struct TcLaunch {
    const TcProblem* problems;
    const TcTile* tiles;
    int ntiles;
    const CUtensorMap* maps;
    const int* bad;       // per-matrix non-finite flags
    unsigned* done;       // per-matrix completion counters (zeroed before the launch), or null
    unsigned* ticket;     // next unclaimed tile (zeroed before the launch)
    unsigned long long wait_ns;  // bound of every wait of the launch
    DeviceStatus* status;
    int nt;               // tile width in 256-column halves (1, or 2 for persistent launches)
};

constexpr unsigned kTileArrivals = 8;  // epilogue warps of a CTA pair that take one tile (one group per CTA)

size_t gemm_tc_smem_bytes();
int gemm_tc_tile_m();
int gemm_tc_tile_n();
int gemm_tc_wide_tile_n();  // 512: the tile width of the wide (NT = 2) instance
int gemm_tc_max_pairs();
cudaError_t launch_gemm_tc(const TcLaunch& L, int grid, cudaStream_t stream);

struct F32Launch {
    const F32Problem* problems;
    int nproblems;
    int max_m, max_n;
    const int* bad;
};
cudaError_t launch_gemm_f32(const F32Launch& L, cudaStream_t stream);

// AdamW lane: one tensor (flat) of the grouped elementwise launch.
struct AdamTensor {
    void* p;          // parameter (fp32 or bf16)
    const void* g;    // gradient (bf16 or fp32)
    float* m;         // first moment (fp32)
    float* v;         // second moment (fp32)
    long long numel;
    long long chunk_begin;
    int vec_ok;       // numel % 8 == 0 and every pointer 16-byte aligned (8-element access)
};

struct AdamLaunch {
    const AdamTensor* tensors;
    int ntensors;
    long long nchunks;
    int p_dt, g_dt;
    float decay, beta1, beta2, lr_c1, c2, eps;
};
struct MomLaunch {
    const MomMatrix* mats;
    int nmats;
    long long nchunks;
    int in_dt;    // dtype of g (bf16 or f32)
    int mom_dt;   // dtype of m (bf16 or f32), ignored without momentum
    int u_dt;     // dtype of the workspace copy (bf16 or f32)
    int has_momentum;
    int nesterov;
    float mu;
    float lr;           // learning rate of a Muon step (0 for orthogonalize)
    float clip;         // > 0: the update is clipped to [-clip, clip] (soft-threshold split)
    double eps;
    float* partials;    // one per chunk
    int* counters;      // one per matrix, zero between launches
    float* scale;       // per matrix i: [4i] = s, [4i+1] = s*s, [4i+2] = -lr*s, [4i+3] = -lr
    int* bad;           // per matrix non-finite flag
    DeviceStatus* status;
    int mat_index_base; // index of mats[0] in the caller's numbering (status reporting)
    unsigned* done;     // GEMM completion counters and tile tickets to zero for the GEMM launches that follow
    int ndone;
    // hybrid step: the AdamW lane's chunks follow the nchunks Muon chunks in
    // the same grid (adam.ntensors == 0: none); its gradients share in_dt
    AdamLaunch adam;
};
cudaError_t launch_momentum_norm(const MomLaunch& L, cudaStream_t stream);

// Debug canary mode: check (and re-arm) the n workspace guards at base + offs[i].
cudaError_t launch_guard_check(void* base, const unsigned long long* offs, int n, DeviceStatus* status,
                               cudaStream_t stream);

struct ScaleLaunch {
    const ScaleMatrix* mats;
    int nmats;
    long long nchunks;
    int u_dt, out_dt;
    int update;  // 0: out = s*U;  1: out -= lr*s*U
    float lr;
    const float* scale;
    const int* bad;
};
cudaError_t launch_scale_apply(const ScaleLaunch& L, cudaStream_t stream);

cudaError_t launch_adamw(const AdamLaunch& L, cudaStream_t stream);

// The stream bound by muon_set_stream, and the message muon_last_error returns.
cudaStream_t bound_stream();
void set_last_error(const char* msg);

}  // namespace muon
