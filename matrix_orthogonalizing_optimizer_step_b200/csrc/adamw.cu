// AdamW lane of the hybrid optimizer: the parameters Muon does not handle
// (embeddings, output head, 1-D parameters) take an AdamW step
// ([NanoGPT-Muon] "从 SGD 到 Muon", "工程复现清单": lr 6e-4, betas (0.9, 0.95),
// weight decay 0.1).  Decoupled weight decay, then the bias-corrected update:
//     p <- p (1 - lr wd)
//     m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
//     p <- p - lr (m c1) / (sqrt(v c2) + eps),  c1 = 1/(1 - b1^t), c2 = 1/(1 - b2^t)
// One grouped launch over all tensors: one CTA per chunk of 8192 elements of
// one tensor, 4-element vector access when aligned.  HBM-bound: 26 bytes per
// element with fp32 parameters and bf16 gradients (p, m, v read and written, g read).
#include <cuda_bf16.h>

#include "epilogue.cuh"
#include "launch.h"

namespace muon {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int find_tensor(const AdamTensor* t, int n, long long chunk) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t[mid].chunk_begin <= chunk)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

struct AdamCoef {
    float decay;  // 1 - lr wd
    float b1, omb1, b2, omb2;
    float lr_c1;  // lr / (1 - b1^t)
    float c2;     // 1 / (1 - b2^t)
    float eps;
};

__device__ __forceinline__ float adam_elem(float p, float g, float& m, float& v, const AdamCoef& k) {
    p *= k.decay;
    m = fmaf(k.b1, m, k.omb1 * g);
    v = fmaf(k.b2, v, k.omb2 * g * g);
    return p - k.lr_c1 * m / (sqrtf(v * k.c2) + k.eps);
}

template <bool P_F32, bool G_F32>
__global__ void __launch_bounds__(kThreads) adamw_kernel(const AdamLaunch L) {
    const long long chunk = blockIdx.x;
    const AdamTensor T = L.tensors[find_tensor(L.tensors, L.ntensors, chunk)];
    const long long e0 = (chunk - T.chunk_begin) * kMomChunk;
    const AdamCoef k{L.decay, L.beta1, 1.f - L.beta1, L.beta2, 1.f - L.beta2, L.lr_c1, L.c2, L.eps};
    const int pdt = P_F32 ? DT_F32 : DT_BF16;
    if (T.vec_ok) {
        for (int i = threadIdx.x; i < kMomChunk / 4; i += kThreads) {
            const long long e = e0 + 4LL * i;
            if (e >= T.numel) break;
            float p[4], g[4];
            if (P_F32) {
                const float4 q = *reinterpret_cast<const float4*>(static_cast<const float*>(T.p) + e);
                p[0] = q.x, p[1] = q.y, p[2] = q.z, p[3] = q.w;
            } else {
                const uint2 q = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(T.p) + e);
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
                const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
                p[0] = a.x, p[1] = a.y, p[2] = b.x, p[3] = b.y;
            }
            if (G_F32) {
                const float4 q = *reinterpret_cast<const float4*>(static_cast<const float*>(T.g) + e);
                g[0] = q.x, g[1] = q.y, g[2] = q.z, g[3] = q.w;
            } else {
                const uint2 q = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(T.g) + e);
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
                const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
                g[0] = a.x, g[1] = a.y, g[2] = b.x, g[3] = b.y;
            }
            float4 m = *reinterpret_cast<const float4*>(T.m + e);
            float4 v = *reinterpret_cast<const float4*>(T.v + e);
            p[0] = adam_elem(p[0], g[0], m.x, v.x, k);
            p[1] = adam_elem(p[1], g[1], m.y, v.y, k);
            p[2] = adam_elem(p[2], g[2], m.z, v.z, k);
            p[3] = adam_elem(p[3], g[3], m.w, v.w, k);
            *reinterpret_cast<float4*>(T.m + e) = m;
            *reinterpret_cast<float4*>(T.v + e) = v;
            if (P_F32) {
                *reinterpret_cast<float4*>(static_cast<float*>(T.p) + e) = make_float4(p[0], p[1], p[2], p[3]);
            } else {
                __nv_bfloat162 a = __floats2bfloat162_rn(p[0], p[1]), b = __floats2bfloat162_rn(p[2], p[3]);
                uint2 q;
                q.x = *reinterpret_cast<uint32_t*>(&a);
                q.y = *reinterpret_cast<uint32_t*>(&b);
                *reinterpret_cast<uint2*>(static_cast<uint16_t*>(T.p) + e) = q;
            }
        }
    } else {
        for (int i = threadIdx.x; i < kMomChunk; i += kThreads) {
            const long long e = e0 + i;
            if (e >= T.numel) break;
            float m = T.m[e], v = T.v[e];
            const float p = adam_elem(ld_elem(T.p, pdt, e), ld_elem(T.g, G_F32 ? DT_F32 : DT_BF16, e), m, v, k);
            T.m[e] = m;
            T.v[e] = v;
            st_elem(T.p, pdt, e, p);
        }
    }
}

}  // namespace

cudaError_t launch_adamw(const AdamLaunch& L, cudaStream_t stream) {
    if (L.nchunks <= 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(L.nchunks));
    const bool pf = L.p_dt == DT_F32, gf = L.g_dt == DT_F32;
    if (pf && gf)
        adamw_kernel<true, true><<<grid, kThreads, 0, stream>>>(L);
    else if (pf)
        adamw_kernel<true, false><<<grid, kThreads, 0, stream>>>(L);
    else if (gf)
        adamw_kernel<false, true><<<grid, kThreads, 0, stream>>>(L);
    else
        adamw_kernel<false, false><<<grid, kThreads, 0, stream>>>(L);
    return cudaGetLastError();
}

}  // namespace muon
