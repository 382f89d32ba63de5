// AdamW lane of the hybrid optimizer: the parameters Muon does not handle
// (embeddings, output head, 1-D parameters) take an AdamW step in one grouped
// launch over all tensors (per-chunk body in adamw.cuh).  HBM-bound: 26 bytes
// per element with fp32 parameters and bf16 gradients (p, m, v read and
// written, g read).
#include "adamw.cuh"

namespace muon {
namespace {

constexpr int kThreads = 256;

template <bool P_F32, bool G_F32>
__global__ void __launch_bounds__(kThreads) adamw_kernel(const AdamLaunch L) {
    adamw_chunk<P_F32, G_F32, 8>(L, blockIdx.x);
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
