// fp32 check path: a plain shared-memory-tiled SIMT GEMM (true fp32 FMA, no
// TF32) with the same fused epilogue as the tensor-core kernel.  It exists to
// compare the Newton-Schulz chain against the fp64 oracle at 1e-5, not for
// speed.  Grid: (column tiles, row tiles, problems); 64 x 64 tile per CTA,
// 4 x 4 outputs per thread, K slices of 16.
#include "epilogue.cuh"
#include "launch.h"

namespace muon {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(const F32Launch L) {
    const F32Problem& P = L.problems[blockIdx.z];
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    if (m0 >= P.M || n0 >= P.N) return;
    if (P.ep.sym && m0 > n0 + TN - 1) return;  // strictly below the diagonal
    __shared__ float As[TK][TM + 1];
    __shared__ float Bs[TK][TN + 1];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < P.K; k0 += TK) {
        for (int e = threadIdx.x; e < TM * TK; e += 256) {
            const int i = e / TK, kk = e % TK;
            const int gi = m0 + i, gk = k0 + kk;
            As[kk][i] = (gi < P.M && gk < P.K) ? P.A[gi * P.a_si + gk * P.a_sk] : 0.f;
        }
        for (int e = threadIdx.x; e < TN * TK; e += 256) {
            const int j = e % TN, kk = e / TN;
            const int gj = n0 + j, gk = k0 + kk;
            Bs[kk][j] = (gj < P.N && gk < P.K) ? P.B[gk * P.b_sk + gj * P.b_sj] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = As[kk][ty * 4 + r];
#pragma unroll
            for (int c = 0; c < 4; ++c) b[c] = Bs[kk][tx * 4 + c];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
        }
        __syncthreads();
    }
    const Epilogue ep = P.ep;  // local copy: no reloads after global stores
    if (ep.skip_idx >= 0 && L.bad[ep.skip_idx]) return;
    const float sig = ep.sigma ? *ep.sigma : 1.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const long long row = m0 + ty * 4 + r;
        if (row >= P.M) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const long long col = n0 + tx * 4 + c;
            if (col >= P.N) continue;
            if (ep.sym && col < row) continue;
            float v = ep.alpha * acc[r][c];
            if (ep.c1) v = fmaf(ep.beta, ld_elem(ep.c1, ep.c1_dt, row * ep.ldc1 + col), v);
            v = (sig == 0.f) ? 0.f : v * sig;
            if (ep.c2) v = fmaf(ep.gamma, ld_elem(ep.c2, ep.c2_dt, row * ep.ldc2 + col), v);
            if (row == col) v += ep.delta;
            st_elem(ep.o1, ep.o1_dt, row * ep.ldo1 + col, v);
            if (ep.o2) st_elem(ep.o2, ep.o2_dt, row * ep.ldo2 + col, v);
            if (ep.sym && col > row) {
                st_elem(ep.o1, ep.o1_dt, col * ep.ldo1 + row, v);
                if (ep.o2) st_elem(ep.o2, ep.o2_dt, col * ep.ldo2 + row, v);
            }
        }
    }
}

}  // namespace

cudaError_t launch_gemm_f32(const F32Launch& L, cudaStream_t stream) {
    if (L.nproblems <= 0) return cudaSuccess;
    dim3 grid((L.max_n + TN - 1) / TN, (L.max_m + TM - 1) / TM, L.nproblems);
    gemm_f32_kernel<<<grid, 256, 0, stream>>>(L);
    return cudaGetLastError();
}

}  // namespace muon
