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

// AdamW on chunk `chunk` of the launch's tensors, by the whole CTA (blockDim.x
// threads).  VEC elements per thread and iteration when the tensor is aligned:
// 8 (two 16-byte accesses per fp32 array, one per 16-bit array) in the AdamW
// launch; 4 in the hybrid launch, where the AdamW body shares a kernel with
// the momentum pass and must not raise its register count (and lower its
// occupancy) much.
template <bool P_F32, bool G_F32, int VEC>
__device__ __forceinline__ void adamw_chunk(const AdamLaunch& L, long long chunk) {
    static_assert(VEC == 4 || VEC == 8, "vector width");
    const AdamTensor T = L.tensors[adam_find_tensor(L.tensors, L.ntensors, chunk)];
    const long long e0 = (chunk - T.chunk_begin) * kMomChunk;
    const AdamCoef k{L.decay, L.beta1, 1.f - L.beta1, L.beta2, 1.f - L.beta2, L.lr_c1, L.c2, L.eps};
    const int pdt = P_F32 ? DT_F32 : DT_BF16;
    const int nthr = static_cast<int>(blockDim.x);
    if (T.vec_ok) {  // numel % 8 == 0, every pointer 16-byte aligned
        for (int i = threadIdx.x; i < kMomChunk / VEC; i += nthr) {
            const long long e = e0 + static_cast<long long>(VEC) * i;
            if (e >= T.numel) break;
            float p[VEC], g[VEC], m[VEC], v[VEC];
            auto ldf = [](const float* src, float* dst) {
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q) {
                    const float4 a = *reinterpret_cast<const float4*>(src + 4 * q);
                    dst[4 * q] = a.x, dst[4 * q + 1] = a.y, dst[4 * q + 2] = a.z, dst[4 * q + 3] = a.w;
                }
            };
            auto stf = [](float* dst, const float* src) {
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q)
                    *reinterpret_cast<float4*>(dst + 4 * q) =
                        make_float4(src[4 * q], src[4 * q + 1], src[4 * q + 2], src[4 * q + 3]);
            };
            // VEC bf16 values: one 16-byte access (8) or one 8-byte access (4)
            auto ld16 = [](const void* base, long long off, float* dst) {
                const uint16_t* q = static_cast<const uint16_t*>(base) + off;
                if (VEC == 8) {
                    unpack8(*reinterpret_cast<const uint4*>(q), DT_BF16, dst);
                } else {
                    const uint2 w = *reinterpret_cast<const uint2*>(q);
                    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
                    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
                    dst[0] = a.x, dst[1] = a.y, dst[2] = b.x, dst[3] = b.y;
                }
            };
            if (P_F32)
                ldf(static_cast<const float*>(T.p) + e, p);
            else
                ld16(T.p, e, p);
            if (G_F32)
                ldf(static_cast<const float*>(T.g) + e, g);
            else
                ld16(T.g, e, g);
            ldf(T.m + e, m);
            ldf(T.v + e, v);
#pragma unroll
            for (int j = 0; j < VEC; ++j) p[j] = adam_elem(p[j], g[j], m[j], v[j], k);
            stf(T.m + e, m);
            stf(T.v + e, v);
            if (P_F32) {
                stf(static_cast<float*>(T.p) + e, p);
            } else if (VEC == 8) {
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(T.p) + e) = pack8(p, DT_BF16);
            } else {
                __nv_bfloat162 a = __floats2bfloat162_rn(p[0], p[1]), b = __floats2bfloat162_rn(p[2], p[3]);
                *reinterpret_cast<uint2*>(static_cast<uint16_t*>(T.p) + e) =
                    make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
            }
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
