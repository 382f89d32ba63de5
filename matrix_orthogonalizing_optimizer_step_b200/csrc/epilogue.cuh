// Element access and the fused GEMM epilogue shared by the tensor-core and
// the fp32 SIMT kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "muon_internal.h"

namespace muon {

__device__ __forceinline__ float ld_elem(const void* p, int dt, long long i) {
    if (dt == DT_F32) return static_cast<const float*>(p)[i];
    if (dt == DT_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    return __half2float(static_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ void st_elem(void* p, int dt, long long i, float v) {
    if (dt == DT_F32) {
        static_cast<float*>(p)[i] = v;
    } else if (dt == DT_BF16) {
        static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    } else {
        static_cast<__half*>(p)[i] = __float2half_rn(v);
    }
}

// Unpack 8 16-bit values held in a uint4.
__device__ __forceinline__ void unpack8(const uint4& q, int dt, float* out) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (dt == DT_BF16) {
            __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
            float2 f = __bfloat1622float2(h);
            out[2 * i] = f.x;
            out[2 * i + 1] = f.y;
        } else {
            __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
            float2 f = __half22float2(h);
            out[2 * i] = f.x;
            out[2 * i + 1] = f.y;
        }
    }
}

__device__ __forceinline__ uint4 pack8(const float* v, int dt) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (dt == DT_BF16) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        } else {
            __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// 32 values passed by value to the out-of-line (cold) element-wise paths, so
// that the hot paths' register arrays never need an address.
struct Row32 {
    float v[32];
};

// Element-wise load of a ragged or unaligned row segment (cold path).
static __device__ __noinline__ Row32 load_row32_elems(const void* base, int dt, long long off, int nvalid) {
    Row32 r;
#pragma unroll 4
    for (int j = 0; j < 32; ++j) r.v[j] = (j < nvalid) ? ld_elem(base, dt, off + j) : 0.f;
    return r;
}

// Load 32 consecutive elements of one row (columns col0 .. col0+31); columns
// at or beyond col0 + nvalid read as 0.
__device__ __forceinline__ void load_row32(const void* base, int dt, long long ld, long long row, int col0,
                                           int nvalid, float* out) {
    const long long off = row * ld + col0;
    if (dt != DT_F32 && nvalid == 32 && ((reinterpret_cast<uintptr_t>(base) + off * 2) & 15) == 0) {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off);
#pragma unroll
        for (int q = 0; q < 4; ++q) unpack8(p[q], dt, out + 8 * q);
        return;
    }
    if (dt == DT_F32 && nvalid == 32 && ((reinterpret_cast<uintptr_t>(base) + off * 4) & 15) == 0) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float4 f = p[q];
            out[4 * q] = f.x;
            out[4 * q + 1] = f.y;
            out[4 * q + 2] = f.z;
            out[4 * q + 3] = f.w;
        }
        return;
    }
    const Row32 r = load_row32_elems(base, dt, off, nvalid);
#pragma unroll
    for (int j = 0; j < 32; ++j) out[j] = r.v[j];
}

// Store columns [jmin, nvalid) of a 32-wide row segment (one lane's row).
__device__ __forceinline__ void store_row32(void* base, int dt, long long ld, long long row, int col0, int jmin,
                                            int nvalid, const float* v) {
    const long long off = row * ld + col0;
    if (jmin == 0 && nvalid == 32) {
        if (dt != DT_F32 && ((reinterpret_cast<uintptr_t>(base) + off * 2) & 15) == 0) {
            uint4* p = reinterpret_cast<uint4*>(static_cast<uint16_t*>(base) + off);
#pragma unroll
            for (int q = 0; q < 4; ++q) p[q] = pack8(v + 8 * q, dt);
            return;
        }
        if (dt == DT_F32 && ((reinterpret_cast<uintptr_t>(base) + off * 4) & 15) == 0) {
            float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + off);
#pragma unroll
            for (int q = 0; q < 8; ++q) p[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j)
        if (j >= jmin && j < nvalid) st_elem(base, dt, off + j, v[j]);
}

// store_row32 for outputs that TMA cannot store (unaligned row pitch): a cold
// path, kept out of line.
static __device__ __noinline__ void store_row32_cold(void* base, int dt, long long ld, long long row, int col0, int nvalid,
                                              Row32 v) {
    store_row32(base, dt, ld, row, col0, 0, nvalid, v.v);
}

// C1 row segment fetched ahead of its use (16-bit C1, aligned, fully in range).
struct Raw32 {
    uint4 q[4];
    int ok;
};

__device__ __forceinline__ void prefetch_row32(const Epilogue& ep, int M, int N, long long row, int col0, Raw32& r) {
    r.ok = 0;
    if (!ep.c1 || ep.c1_dt == DT_F32 || row >= M || col0 + 32 > N) return;
    const uint16_t* p = static_cast<const uint16_t*>(ep.c1) + row * ep.ldc1 + col0;
    if (reinterpret_cast<uintptr_t>(p) & 15) return;
    const uint4* v = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) r.q[i] = v[i];
    r.ok = 1;
}

// The fused epilogue of a 32-column row segment of the accumulator, in place:
// row `row`, columns col0 .. col0 + 31 of an M x N output become
// sigma * (alpha * acc + beta * C1) + gamma * C2 + delta * I.  `sig` is the
// problem's sigma (already loaded).  Rows at or past M are left untouched
// (returns false); columns past N are computed from zero inputs.
__device__ __forceinline__ bool epilogue_values32(const Epilogue& ep, float sig, int M, int N, long long row, int col0,
                                                  float* acc, const Raw32* pre) {
    if (row >= M) return false;
    const int nvalid = min(32, N - col0);
    if (nvalid <= 0) return false;
    float t1[32];
    if (ep.c1) {
        if (pre && pre->ok) {
#pragma unroll
            for (int i = 0; i < 4; ++i) unpack8(pre->q[i], ep.c1_dt, t1 + 8 * i);
        } else {
            load_row32(ep.c1, ep.c1_dt, ep.ldc1, row, col0, nvalid, t1);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = fmaf(ep.beta, t1[j], ep.alpha * acc[j]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = ep.alpha * acc[j];
    }
    if (sig == 0.f) {
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
    } else if (sig != 1.f) {
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] *= sig;
    }
    if (ep.c2) {
        load_row32(ep.c2, ep.c2_dt, ep.ldc2, row, col0, nvalid, t1);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = fmaf(ep.gamma, t1[j], acc[j]);
    }
    if (ep.delta != 0.f) {
        const long long d = row - col0;
        if (d >= 0 && d < 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j == d) acc[j] += ep.delta;
        }
    }
    return true;
}

}  // namespace muon
