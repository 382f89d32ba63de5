// Allocation-free Frobenius normalisation: Y = X / (||X||_F + eps) per matrix.
//
// Some callers cannot call cudaMalloc at all: code whose device memory is
// owned by a framework's allocator or by a fixed budget reserved up front, and
// latency-critical paths where an allocation (which may synchronise the
// device) is not acceptable.  This entry point serves them.  It is a variant
// of the fused momentum/normalise kernel's norm pass: the per-chunk partial
// sums, the per-matrix ticket counters and the per-matrix scales live in one
// file-scope device array (below) instead of the library's workspace, so the
// call allocates nothing.  The caller passes X and Y.
//
// The array is a module global: every GPU that loads this library holds it
// until the process exits, and every call shares it.
#include <cuda_runtime.h>

#include <cmath>

#include "../../include/muon.h"
#include "epilogue.cuh"
#include "launch.h"

namespace muon {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxDevices = 64;

struct NoAllocScratch {
    float partials[MUON_NOALLOC_MAX_CHUNKS];  // one per 8192-element chunk
    int counters[MUON_NOALLOC_MAX_MATRICES];  // ticket per matrix, zero between calls
    float scale[MUON_NOALLOC_MAX_MATRICES];   // 1 / (||X_i|| + eps); NaN if the norm is not finite
};

static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(NoAllocScratch)];

// Device address of g_noalloc_scratch per device (host code cannot use the
// symbol itself as a device pointer).
NoAllocScratch* g_scratch_addr[kMaxDevices] = {};

template <typename T>
__device__ __forceinline__ T block_sum(T v, T* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    T r = 0;
    if (warp == 0) {
        r = lane < kThreads / 32 ? red[lane] : T(0);
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    }
    return r;
}

// Pass 1: per-chunk sum of squares, and the last chunk of each matrix turns
// the partials (fixed order, fp64) into the matrix's scale.
__global__ void __launch_bounds__(kThreads) noalloc_norm_kernel(const void* X, int dt, long long numel,
                                                                int chunks_per_mat, double eps,
                                                                NoAllocScratch* S) {
    __shared__ float red_f[kThreads / 32];
    __shared__ double red_d[kThreads / 32];
    __shared__ int is_last;
    const long long chunk = blockIdx.x;
    const int mat = static_cast<int>(chunk / chunks_per_mat);
    const long long e0 = (chunk % chunks_per_mat) * kMomChunk;
    const long long base = static_cast<long long>(mat) * numel;
    float ss = 0.f;
    for (int i = threadIdx.x; i < kMomChunk; i += kThreads) {
        const long long e = e0 + i;
        if (e >= numel) break;
        const float u = ld_elem(X, dt, base + e);
        ss = fmaf(u, u, ss);
    }
    const float part = block_sum<float>(ss, red_f);
    if (threadIdx.x == 0) {
        S->partials[chunk] = part;
        __threadfence();
        is_last = (atomicAdd(&S->counters[mat], 1) == chunks_per_mat - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    double acc = 0.0;
    for (int i = threadIdx.x; i < chunks_per_mat; i += kThreads)
        acc += static_cast<double>(__ldcg(&S->partials[static_cast<long long>(mat) * chunks_per_mat + i]));
    const double total = block_sum<double>(acc, red_d);
    if (threadIdx.x == 0) {
        // non-finite norm: NaN marks the matrix as left untouched; a zero
        // matrix with eps = 0 gets s = 0 (its output is 0), not 1/0
        const double denom = sqrt(total) + eps;
        S->scale[mat] = !isfinite(total) ? __int_as_float(0x7fc00000)
                                         : (denom > 0.0 ? static_cast<float>(1.0 / denom) : 0.f);
        S->counters[mat] = 0;
    }
}

// Pass 2: Y = s * X; matrices with a non-finite norm are left untouched.
__global__ void __launch_bounds__(kThreads) noalloc_scale_kernel(const void* X, void* Y, int dt, long long numel,
                                                                 int chunks_per_mat, const NoAllocScratch* S) {
    const long long chunk = blockIdx.x;
    const int mat = static_cast<int>(chunk / chunks_per_mat);
    const float s = S->scale[mat];
    if (s != s) return;  // non-finite norm: Y untouched
    const long long e0 = (chunk % chunks_per_mat) * kMomChunk;
    const long long base = static_cast<long long>(mat) * numel;
    for (int i = threadIdx.x; i < kMomChunk; i += kThreads) {
        const long long e = e0 + i;
        if (e >= numel) break;
        st_elem(Y, dt, base + e, s * ld_elem(X, dt, base + e));
    }
}

int noalloc_fail(int code, const char* msg) {
    set_last_error(msg);
    return code;
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" int muon_normalize_noalloc(int batch, int m, int n, const void* X, void* Y, int dtype, float eps) {
    if (batch < 1 || m < 1 || n < 1) return noalloc_fail(MUON_ERR_INVALID_ARG, "batch, m and n must be >= 1");
    if (!X || !Y) return noalloc_fail(MUON_ERR_INVALID_ARG, "X and Y must not be NULL");
    if (dtype != MUON_DTYPE_BF16 && dtype != MUON_DTYPE_F32)
        return noalloc_fail(MUON_ERR_UNSUPPORTED, "dtype must be MUON_DTYPE_BF16 or MUON_DTYPE_F32");
    if (!(eps >= 0.f) || !std::isfinite(eps)) return noalloc_fail(MUON_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (batch > MUON_NOALLOC_MAX_MATRICES)
        return noalloc_fail(MUON_ERR_INVALID_ARG, "batch exceeds MUON_NOALLOC_MAX_MATRICES");
    const long long numel = static_cast<long long>(m) * n;
    const long long chunks_per_mat = (numel + kMomChunk - 1) / kMomChunk;
    if (chunks_per_mat * batch > MUON_NOALLOC_MAX_CHUNKS)
        return noalloc_fail(MUON_ERR_INVALID_ARG,
                            "batch*ceil(m*n/8192) exceeds MUON_NOALLOC_MAX_CHUNKS (the static scratch size)");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return noalloc_fail(MUON_ERR_CUDA, "no usable CUDA device");
    }
    // One-time set-up per device, with that device current: the device
    // address of the static scratch array.
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return noalloc_fail(MUON_ERR_CUDA, "cudaGetSymbolAddress of the scratch array failed");
        }
        g_scratch_addr[dev] = static_cast<NoAllocScratch*>(p);
    }
    NoAllocScratch* S = g_scratch_addr[dev];
    cudaStream_t st = bound_stream();
    const int dt = dtype == MUON_DTYPE_F32 ? DT_F32 : DT_BF16;
    // the ticket counters must start at zero (a previous call may have been cut short)
    cudaError_t e = cudaMemsetAsync(S->counters, 0, sizeof(int) * batch, st);
    if (e != cudaSuccess) return noalloc_fail(MUON_ERR_CUDA, cudaGetErrorString(e));
    const unsigned grid = static_cast<unsigned>(chunks_per_mat * batch);
    noalloc_norm_kernel<<<grid, kThreads, 0, st>>>(X, dt, numel, static_cast<int>(chunks_per_mat), eps, S);
    noalloc_scale_kernel<<<grid, kThreads, 0, st>>>(X, Y, dt, numel, static_cast<int>(chunks_per_mat), S);
    e = cudaGetLastError();
    if (e != cudaSuccess) return noalloc_fail(MUON_ERR_CUDA, cudaGetErrorString(e));
    return MUON_OK;
}
