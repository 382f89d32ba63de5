// Fused momentum / Nesterov / Frobenius-norm / cast kernel, and the
// elementwise "steps = 0" update.
//
// Momentum step ([NanoGPT-Muon] "工程复现清单": momentum 0.95, nesterov=True;
// [Gram-NS] "ข้อได้เปรียบของอัลกอริทึม": mu is the momentum coefficient):
//     M <- mu*M + G ;  U = G + mu*M (Nesterov) or U = M
// then ||U||_F^2 is reduced per matrix and U is written (bf16) into the
// workspace, where the Newton-Schulz chain reads it.  The normalisation
// X0 = U / (||U||_F + eps) is never materialised: the scale s and s^2 are
// folded into the first GEMM epilogues.
//
// One CTA handles one chunk of kMomChunk elements of one matrix (chunks never
// straddle matrices).  The per-matrix sum of squares is deterministic: each
// chunk writes its fp32 partial (fixed warp-shuffle + shared-memory tree),
// and the last chunk to finish (ticket counter) sums the partials of its
// matrix in fixed order in fp64, writes s = 1 / (sqrt(sum) + eps), s^2 and
// the update factors -lr*s and -lr,
// flags non-finite norms, and resets the ticket for the next launch.
#include <cuda_bf16.h>

#include "adamw.cuh"
#include "epilogue.cuh"
#include "launch.h"

namespace muon {
namespace {

constexpr int kThreads = 256;
// Eight resident CTAs per SM (every warp slot): at most 32 registers a
// thread.  The momentum pass needs no more; the hybrid instance's AdamW body
// would take 47-48 without the bound, and since registers are allocated per
// kernel that would cost the momentum chunks of the same launch a third of
// their occupancy (the bound costs the AdamW body a few spilled words instead).
constexpr int kMinBlocks = 8;
constexpr int kVecPerThread = kMomChunk / 8 / kThreads;  // 8-element vectors per thread
static_assert(kVecPerThread * 8 * kThreads == kMomChunk, "chunk layout");

enum { MOM_NONE = 0, MOM_BF16 = 1, MOM_F32 = 2 };

__device__ __forceinline__ int find_matrix(int n, long long chunk, const MomMatrix* mats) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mats[mid].chunk_begin <= chunk)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void load8(const void* p, bool f32, long long i, float* v) {
    if (f32) {
        const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
        const float4 a = q[0], b = q[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        unpack8(*reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p) + i), DT_BF16, v);
    }
}

__device__ __forceinline__ void store8(void* p, bool f32, long long i, const float* v) {
    if (f32) {
        float4* q = reinterpret_cast<float4*>(static_cast<float*>(p) + i);
        q[0] = make_float4(v[0], v[1], v[2], v[3]);
        q[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p) + i) = pack8(v, DT_BF16);
    }
}

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
    return r;  // valid in thread 0
}

// HYBRID: the grid also carries the AdamW lane's chunks (after the Muon
// chunks).  A separate instance, so that the plain Muon step's code stays
// that of the momentum pass alone.
template <bool G_F32, int MOM, bool U_F32, bool CLIP, bool HYBRID>
__global__ void __launch_bounds__(kThreads, kMinBlocks) momentum_norm_kernel(const MomLaunch L) {
    __shared__ float red_f[kThreads / 32];
    __shared__ double red_d[kThreads / 32];
    __shared__ int is_last;
    const long long chunk = blockIdx.x;
    if (HYBRID && chunk >= L.nchunks) {
        // hybrid step: the AdamW lane's chunks follow the Muon chunks
        if (L.adam.p_dt == DT_F32)
            adamw_chunk<true, G_F32, 4>(L.adam, chunk - L.nchunks);
        else
            adamw_chunk<false, G_F32, 4>(L.adam, chunk - L.nchunks);
        return;
    }
    if (chunk == 0 && L.done)  // the GEMM launches that follow count completions and tickets from zero
        for (int i = threadIdx.x; i < L.ndone; i += kThreads) L.done[i] = 0u;
    const int mi = find_matrix(L.nmats, chunk, L.mats);
    const MomMatrix Mx = L.mats[mi];  // local copy: no reloads after global stores
    const long long numel = Mx.rows * Mx.cols;
    const long long e0 = (chunk - Mx.chunk_begin) * kMomChunk;
    const float mu = L.mu;
    const float clip = L.clip;
    float ss = 0.f;

    auto step = [&](float g, float& m_io) -> float {
        if (MOM == MOM_NONE) return g;
        const float mn = fmaf(mu, m_io, g);
        m_io = mn;
        return L.nesterov ? fmaf(mu, mn, g) : mn;
    };
    // Soft-threshold split (CLIP): the update is clipped to [-clip, clip] (the
    // outlier part is dropped) and the sum of squares is taken of the clipped
    // values.  u - u is 0 for finite u and NaN for +-Inf or NaN, so a
    // non-finite update still flags the matrix.
    auto split = [&](float u, float& acc) -> float {
        if (!CLIP) return u;
        acc += __fsub_rn(u, u);
        return fminf(fmaxf(u, -clip), clip);
    };

    if (Mx.vec_ok) {
#pragma unroll
        for (int v = 0; v < kVecPerThread; ++v) {
            const long long e = e0 + (static_cast<long long>(v) * kThreads + threadIdx.x) * 8;
            if (e < numel && e < e0 + kMomChunk) {
                float g[8], m[8], u[8];
                load8(Mx.g, G_F32, e, g);
                if (MOM != MOM_NONE) load8(Mx.m, MOM == MOM_F32, e, m);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    u[j] = split(step(g[j], m[j]), ss);
                    ss = fmaf(u[j], u[j], ss);
                }
                if (MOM != MOM_NONE) store8(Mx.m, MOM == MOM_F32, e, m);
                store8(Mx.u, U_F32, e, u);
            }
        }
    } else {
        for (int i = threadIdx.x; i < kMomChunk; i += kThreads) {
            const long long e = e0 + i;
            if (e >= numel) break;
            const long long r = e / Mx.cols, c = e - r * Mx.cols;
            const float g = ld_elem(Mx.g, G_F32 ? DT_F32 : DT_BF16, e);
            float m = 0.f;
            if (MOM != MOM_NONE) m = ld_elem(Mx.m, MOM == MOM_F32 ? DT_F32 : DT_BF16, e);
            const float u = split(step(g, m), ss);
            ss = fmaf(u, u, ss);
            if (MOM != MOM_NONE) st_elem(Mx.m, MOM == MOM_F32 ? DT_F32 : DT_BF16, e, m);
            st_elem(Mx.u, U_F32 ? DT_F32 : DT_BF16, r * Mx.ldu + c, u);
        }
    }

    const float part = block_sum<float>(ss, red_f);
    if (threadIdx.x == 0) {
        L.partials[chunk] = part;
        __threadfence();
        const int ticket = atomicAdd(&L.counters[mi], 1);
        is_last = (ticket == Mx.nchunks - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    double acc = 0.0;
    for (long long i = threadIdx.x; i < Mx.nchunks; i += kThreads)
        acc += static_cast<double>(__ldcg(&L.partials[Mx.chunk_begin + i]));
    const double total = block_sum<double>(acc, red_d);
    if (threadIdx.x == 0) {
        const bool finite = isfinite(total);
        // a zero matrix with eps = 0 has no scale: s = 0 (its outputs are 0
        // and its parameter does not move), not 1/0
        const double denom = sqrt(total) + L.eps;
        const double s = (finite && denom > 0.0) ? 1.0 / denom : 0.0;
        L.scale[4 * mi] = static_cast<float>(s);
        L.scale[4 * mi + 1] = static_cast<float>(s * s);
        L.scale[4 * mi + 2] = static_cast<float>(-static_cast<double>(L.lr) * s);
        L.scale[4 * mi + 3] = finite ? -L.lr : 0.f;
        L.bad[mi] = finite ? 0 : 1;
        if (!finite) {
            atomicOr(&L.status->bits, ST_NONFINITE);
            atomicMin(&L.status->first_bad, L.mat_index_base + mi);
        }
        L.counters[mi] = 0;
    }
}

template <bool U_F32, bool OUT_F32>
__global__ void __launch_bounds__(kThreads) scale_apply_kernel(const ScaleLaunch L) {
    const long long chunk = blockIdx.x;
    int lo = 0, hi = L.nmats - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (L.mats[mid].chunk_begin <= chunk)
            lo = mid;
        else
            hi = mid - 1;
    }
    const ScaleMatrix S = L.mats[lo];
    if (L.bad[S.mat]) return;
    const float s = L.scale[4 * S.mat];
    const long long numel = S.rows * S.cols;
    const long long e0 = (chunk - S.chunk_begin) * kMomChunk;
    for (int i = threadIdx.x; i < kMomChunk; i += kThreads) {
        const long long e = e0 + i;
        if (e >= numel) break;
        const long long r = e / S.cols, c = e - r * S.cols;
        const float u = ld_elem(S.u, U_F32 ? DT_F32 : DT_BF16, r * S.ldu + c);
        const int odt = OUT_F32 ? DT_F32 : DT_BF16;
        if (L.update)
            st_elem(S.out, odt, e, ld_elem(S.out, odt, e) - L.lr * (s * u));
        else
            st_elem(S.out, odt, e, s * u);
    }
}

}  // namespace

template <bool CLIP, bool HYBRID>
static cudaError_t launch_step(const MomLaunch& L, dim3 grid, bool gf, cudaStream_t stream) {
    if (gf) {
        if (L.mom_dt == DT_F32)
            momentum_norm_kernel<true, MOM_F32, false, CLIP, HYBRID><<<grid, kThreads, 0, stream>>>(L);
        else
            momentum_norm_kernel<true, MOM_BF16, false, CLIP, HYBRID><<<grid, kThreads, 0, stream>>>(L);
    } else {
        if (L.mom_dt == DT_F32)
            momentum_norm_kernel<false, MOM_F32, false, CLIP, HYBRID><<<grid, kThreads, 0, stream>>>(L);
        else
            momentum_norm_kernel<false, MOM_BF16, false, CLIP, HYBRID><<<grid, kThreads, 0, stream>>>(L);
    }
    return cudaGetLastError();
}

cudaError_t launch_momentum_norm(const MomLaunch& L, cudaStream_t stream) {
    if (L.nchunks <= 0) return cudaSuccess;
    const bool hybrid = L.adam.ntensors > 0;
    if (hybrid && (!L.has_momentum || L.adam.g_dt != L.in_dt)) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(L.nchunks + (hybrid ? L.adam.nchunks : 0)));
    const bool gf = L.in_dt == DT_F32, uf = L.u_dt == DT_F32;
    if (!L.has_momentum) {
        if (gf && uf)
            momentum_norm_kernel<true, MOM_NONE, true, false, false><<<grid, kThreads, 0, stream>>>(L);
        else if (!gf && !uf)
            momentum_norm_kernel<false, MOM_NONE, false, false, false><<<grid, kThreads, 0, stream>>>(L);
        else
            return cudaErrorInvalidValue;
        return cudaGetLastError();
    }
    if (uf) return cudaErrorInvalidValue;
    if (hybrid) {
        if (L.clip > 0.f) return launch_step<true, true>(L, grid, gf, stream);
        return launch_step<false, true>(L, grid, gf, stream);
    }
    if (L.clip > 0.f) return launch_step<true, false>(L, grid, gf, stream);
    return launch_step<false, false>(L, grid, gf, stream);
}

cudaError_t launch_scale_apply(const ScaleLaunch& L, cudaStream_t stream) {
    if (L.nchunks <= 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(L.nchunks));
    const bool uf = L.u_dt == DT_F32, of = L.out_dt == DT_F32;
    if (uf && of)
        scale_apply_kernel<true, true><<<grid, kThreads, 0, stream>>>(L);
    else if (!uf && of)
        scale_apply_kernel<false, true><<<grid, kThreads, 0, stream>>>(L);
    else if (!uf && !of)
        scale_apply_kernel<false, false><<<grid, kThreads, 0, stream>>>(L);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace muon
