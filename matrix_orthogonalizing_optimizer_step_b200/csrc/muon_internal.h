// Internal host/device structures of the Muon library.  Not part of the ABI.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace muon {

enum DType : int { DT_BF16 = 0, DT_F32 = 1, DT_F16 = 2 };

inline int dtype_size(int dt) { return dt == DT_F32 ? 4 : 2; }

// device status word bits
enum : int { ST_TIMEOUT = 1, ST_NONFINITE = 2, ST_GUARD = 4 };

// Workspace guards of the debug canary mode (MUON_DEBUG_CANARY=1).
constexpr int kGuardBytes = 1024;
constexpr unsigned char kGuardByte = 0xA5;

struct DeviceStatus {
    int bits;       // ST_* flags, sticky until read by the host
    int first_bad;  // first matrix index with a non-finite norm (or -1 after clear)
};

// Fused epilogue of every GEMM:
//   v = sigma * (alpha * acc + beta * C1) + gamma * C2 + delta * [row == col]
// sigma is 1 when sigma_ptr is null.  sigma == 0 forces the first term to 0
// (so a non-finite accumulator of a rejected matrix does not leak through).
// With sym (fp32 check path only), only elements with row <= col are
// produced and each is also written at the mirrored position (col, row); the
// tensor-core path instead stores symmetric outputs as upper tiles.
struct Epilogue {
    float alpha, beta, gamma, delta;
    const float* sigma;  // per-matrix scale (device) or null
    int skip_idx;        // index into the non-finite flags (skip all stores if set), or -1
    int sym;
    const void* c1; long long ldc1; int c1_dt;
    const void* c2; long long ldc2; int c2_dt;
    void* o1; long long ldo1; int o1_dt;
    void* o2; long long ldo2; int o2_dt;
    // tensor-core path: TMA store map of o1 (boxes of 64 bytes x 32 rows,
    // 64-byte swizzle) and the batch coordinate of this problem in it, or
    // o1_map = -1 (o1 not 16-byte aligned: direct stores)
    int o1_map, o1_z;
};

// One tensor-core GEMM problem D[M x N] = A[M x K] * B[K x N] (B given as N x K
// "rows" in tcgen05 terms).  Operands are read by TMA through tensor maps in
// global memory; a_mn / b_mn select the MN-major (transposed) smem layout.
//
// Symmetric n x n matrices are stored as their upper 256 x 256 tiles only
// (diagonal tiles in full).  An operand marked a_sym / b_sym is such a matrix:
// a 64-wide K slice that falls in a lower tile is fetched from the mirrored
// upper tile through the transposed (MN-major) map a_map_t / b_map_t.
struct TcProblem {
    int M, N, K;
    int a_map, b_map;      // indices into the launch's tensor-map array
    int a_map_t, b_map_t;  // MN-major maps of symmetric operands (else -1)
    int a_z, b_z;          // batch coordinate (3rd tensor-map dimension)
    int a_mn, b_mn;        // 1: operand is MN-major in memory
    int a_sym, b_sym;      // 1: operand is an upper-stored symmetric matrix
    int fmt;               // 0 = f16 operands, 1 = bf16 operands
    int pad_;              // 1: the output is symmetric (upper 256-blocks are stored)
    Epilogue ep;
};

// fp32 SIMT problem: element (i, k) of A at A[i*a_si + k*a_sk], (k, j) of B at
// B[k*b_sk + j*b_sj].
struct F32Problem {
    int M, N, K, pad_;
    const float* A; long long a_si, a_sk;
    const float* B; long long b_sk, b_sj;
    Epilogue ep;
};

// One matrix of the fused momentum / normalise / cast kernel.
struct MomMatrix {
    const void* g;   // gradient (bf16) or the matrix to orthogonalise (bf16/f32)
    void* m;         // momentum buffer (bf16/f32) or null
    void* u;         // workspace copy of U (row stride ldu), bf16 or f32
    long long rows, cols, ldu;
    long long chunk_begin;  // first chunk of this matrix in the launch
    int nchunks;
    int vec_ok;      // 16-byte aligned, cols % 8 == 0, ldu == cols
};

// Elementwise "steps = 0" update: out = s * U (orthogonalize) or W -= lr * s * U.
struct ScaleMatrix {
    const void* u; long long ldu;
    void* out; long long rows, cols;  // out has row stride cols
    long long chunk_begin;            // first chunk (kMomChunk elements) of this matrix
    int mat;  // index into scale / flags
};

constexpr int kMomChunk = 8192;  // elements per CTA of the momentum kernel

}  // namespace muon
