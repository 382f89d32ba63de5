// Workspace guards of the debug canary mode (MUON_DEBUG_CANARY=1 when a plan
// is built): every region of the workspace arena is followed by a guard of
// kGuardBytes filled with kGuardByte.  After each call's launches one CTA per
// guard compares its guard with the pattern; a difference means some kernel
// wrote past the end of a region.  The CTA records it in the device status
// word (MUON_ERR_GUARD through muon_device_status) and restores the pattern,
// so each call is checked on its own.  A stand-in for a memory checker where
// none can run: it finds out-of-bounds writes into the library's own buffers.
#include <cuda_runtime.h>

#include <cstdint>

#include "launch.h"
#include "muon_internal.h"

namespace muon {
namespace {

constexpr int kGuardThreads = 128;

__global__ void __launch_bounds__(kGuardThreads) guard_check_kernel(unsigned char* base,
                                                                   const unsigned long long* offs,
                                                                   DeviceStatus* status) {
    // a guard starts at the end of its region (any alignment): byte access
    unsigned char* g = base + offs[blockIdx.x];
    int bad = 0;
    for (int i = threadIdx.x; i < kGuardBytes; i += kGuardThreads) {
        if (g[i] != kGuardByte) {
            bad = 1;
            g[i] = kGuardByte;  // re-armed for the next call
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&status->bits, ST_GUARD);
}

}  // namespace

cudaError_t launch_guard_check(void* base, const unsigned long long* offs, int n, DeviceStatus* status,
                               cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    guard_check_kernel<<<n, kGuardThreads, 0, stream>>>(static_cast<unsigned char*>(base), offs, status);
    return cudaGetLastError();
}

}  // namespace muon
