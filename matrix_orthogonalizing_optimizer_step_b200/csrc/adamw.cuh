// AdamW lane of the hybrid optimizer (per-chunk body), used by the grouped
// AdamW launch and by the hybrid launch, whose grid appends the AdamW chunks
// to the Muon momentum chunks.
//
// [NanoGPT-Muon] "从 SGD 到 Muon", "工程复现清单" (lr 6e-4, betas (0.9, 0.95),
// weight decay 0.1).  Decoupled weight decay, then the bias-corrected update:
//     p <- p (1 - lr wd)
//     m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
//     p <- p - lr (m c1) / (sqrt(v c2) + eps),  c1 = 1/(1 - b1^t), c2 = 1/(1 - b2^t)
// One CTA (256 threads) per chunk of kMomChunk elements of one tensor, 8-element
// vector access when aligned.
#pragma once
#include <cuda_bf16.h>

#include "epilogue.cuh"
#include "launch.h"

namespace muon {

__device__ __forceinline__ int adam_find_tensor(const AdamTensor* t, int n, long long chunk) {
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

// AdamW on chunk `chunk` of the launch's tensors, by the whole CTA (blockDim.x threads).
template <bool P_F32, bool G_F32>
__device__ __forceinline__ void adamw_chunk(const AdamLaunch& L, long long chunk) {
    const AdamTensor T = L.tensors[adam_find_tensor(L.tensors, L.ntensors, chunk)];
    const long long e0 = (chunk - T.chunk_begin) * kMomChunk;
    const AdamCoef k{L.decay, L.beta1, 1.f - L.beta1, L.beta2, 1.f - L.beta2, L.lr_c1, L.c2, L.eps};
    const int pdt = P_F32 ? DT_F32 : DT_BF16;
    const int nthr = static_cast<int>(blockDim.x);
    if (T.vec_ok) {
        // 8 elements per thread and iteration: two 16-byte accesses per fp32
        // array, one per 16-bit array
        for (int i = threadIdx.x; i < kMomChunk / 8; i += nthr) {
            const long long e = e0 + 8LL * i;
            if (e >= T.numel) break;
            float p[8], g[8], m[8], v[8];
            auto ld8f = [](const float* src, float* dst) {
                const float4 a = *reinterpret_cast<const float4*>(src);
                const float4 b = *reinterpret_cast<const float4*>(src + 4);
                dst[0] = a.x, dst[1] = a.y, dst[2] = a.z, dst[3] = a.w;
                dst[4] = b.x, dst[5] = b.y, dst[6] = b.z, dst[7] = b.w;
            };
            auto st8f = [](float* dst, const float* src) {
                *reinterpret_cast<float4*>(dst) = make_float4(src[0], src[1], src[2], src[3]);
                *reinterpret_cast<float4*>(dst + 4) = make_float4(src[4], src[5], src[6], src[7]);
            };
            if (P_F32)
                ld8f(static_cast<const float*>(T.p) + e, p);
            else
                unpack8(*reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(T.p) + e), DT_BF16, p);
            if (G_F32)
                ld8f(static_cast<const float*>(T.g) + e, g);
            else
                unpack8(*reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(T.g) + e), DT_BF16, g);
            ld8f(T.m + e, m);
            ld8f(T.v + e, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) p[j] = adam_elem(p[j], g[j], m[j], v[j], k);
            st8f(T.m + e, m);
            st8f(T.v + e, v);
            if (P_F32)
                st8f(static_cast<float*>(T.p) + e, p);
            else
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(T.p) + e) = pack8(p, DT_BF16);
        }
    } else {
        for (int i = threadIdx.x; i < kMomChunk; i += nthr) {
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

}  // namespace muon
