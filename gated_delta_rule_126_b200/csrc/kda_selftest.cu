// kda_wait_timeout_selftest: shows that a bounded wait which runs out leaves the
// device usable and is reported through the workspace status word.
//
// The prefill kernels wait on two kinds of events: an mbarrier phase (a TMA copy or
// a tensor-core commit arriving) and a release/acquire progress counter in shared
// memory (one warp group handing a tile to another).  Each wait gives up after a
// fixed number of SM cycles, sets the status flag and returns.  This kernel runs the
// same two waits on events that nothing ever produces -- an mbarrier that no thread
// arrives at and a counter that no thread writes -- so both limits run out; it then
// exits normally.  Nothing is issued to the copy or tensor engines, so nothing is in
// flight when it returns.
#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace {

constexpr long long kMaxSelftestCycles = 4000000000LL;  // the prefill kernels' limit

// detail bits: which wait ran out
constexpr unsigned kDetailMbarrier = 1u;
constexpr unsigned kDetailCounter = 2u;

__global__ void __launch_bounds__(64, 1) wait_timeout_kernel(kda::DeviceStatus *status, long long max_cycles) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t counter;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        kda::ptx::mbar_init(&bar, 1);
        kda::ptx::fence_mbar_init();
        counter = 0;
    }
    __syncthreads();
    if (lane == 0) {
        bool ok = true;
        if (warp == 0) {
            // phase 0 completes only when one thread arrives; none does
            ok = kda::ptx::mbar_wait_bounded(&bar, 0u, max_cycles);
            if (!ok) atomicOr(&status->detail, kDetailMbarrier);
        } else {
            // the counter stays 0; the wait wants 1
            const long long t0 = clock64();
            while (kda::ptx::ld_acquire(&counter) < 1u) {
                if (clock64() - t0 > max_cycles) {
                    ok = false;
                    break;
                }
                __nanosleep(64);
            }
            if (!ok) atomicOr(&status->detail, kDetailCounter);
        }
        if (!ok) atomicExch(&status->flag, 1u);
    }
    __syncthreads();
}

}  // namespace

extern "C" {

kda_status_t kda_wait_timeout_selftest(void *workspace, size_t workspace_bytes, long long max_cycles,
                                       kda_stream_t stream) {
    if (!workspace || workspace_bytes < kda::WorkspaceLayout::kStatusBytes ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return KDA_ERR_WORKSPACE;
    if (max_cycles < 1 || max_cycles > kMaxSelftestCycles) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto *status = static_cast<kda::DeviceStatus *>(workspace);
    if (cudaMemsetAsync(status, 0, sizeof(kda::DeviceStatus), st) != cudaSuccess) return KDA_ERR_CUDA;
    wait_timeout_kernel<<<1, 64, 0, st>>>(status, max_cycles);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
