// Sequence split of the tensor-core prefill: the chain of start states between
// passes.  The KDA recurrence (state-update equation, section "Kimi Delta Attention
// (KDA)" of the wiki page "Kimi Linear 高效注意力架构") is affine in the state: over
// a segment, S_end = M S_start + L, with M the d_k x d_k transition (the segment run
// from the identity with v = 0) and L the end state from a zero start.  This kernel
// forms S_start(p) = M(p-1) S_start(p-1) + L(p-1) for every split sequence and head.
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int D = 128;

// One block per (split sequence, head), 256 threads: thread t computes row t / 2 and
// 64 columns of the 128 x 128 product, with the input state staged in shared memory.
__global__ void __launch_bounds__(256) split_combine_kernel(const SplitPlan plan, int H, int p) {
    extern __shared__ float s_in[];  // [128][128]
    const int j = blockIdx.x / H, h = blockIdx.x % H;
    const size_t D2 = size_t(D) * D;
    const size_t prev = (size_t(j) * plan.nseg + (p - 1)) * H + h, cur = (size_t(j) * plan.nseg + p) * H + h;
    const float *M = plan.mmat + prev * D2, *L = plan.lmat + prev * D2, *Sin = plan.sstart + prev * D2;
    float *Sout = plan.sstart + cur * D2;
    for (int i = threadIdx.x; i < D * D / 4; i += blockDim.x)
        reinterpret_cast<float4 *>(s_in)[i] = reinterpret_cast<const float4 *>(Sin)[i];
    __syncthreads();
    const int r = threadIdx.x >> 1, c0 = 64 * (threadIdx.x & 1);
    float acc[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) acc[c] = L[size_t(r) * D + c0 + c];
    for (int k = 0; k < D; ++k) {
        const float m = M[size_t(r) * D + k];
        const float4 *srow = reinterpret_cast<const float4 *>(s_in + k * D + c0);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
            const float4 sv = srow[c4];
            acc[4 * c4 + 0] = fmaf(m, sv.x, acc[4 * c4 + 0]);
            acc[4 * c4 + 1] = fmaf(m, sv.y, acc[4 * c4 + 1]);
            acc[4 * c4 + 2] = fmaf(m, sv.z, acc[4 * c4 + 2]);
            acc[4 * c4 + 3] = fmaf(m, sv.w, acc[4 * c4 + 3]);
        }
    }
#pragma unroll
    for (int c4 = 0; c4 < 16; ++c4)
        reinterpret_cast<float4 *>(Sout + size_t(r) * D + c0)[c4] =
            make_float4(acc[4 * c4], acc[4 * c4 + 1], acc[4 * c4 + 2], acc[4 * c4 + 3]);
}

}  // namespace

cudaError_t launch_split_combine(const PrefillArgs &a, int p, cudaStream_t stream) {
    if (a.split.num_seqs == 0) return cudaSuccess;
    const int smem = D * D * sizeof(float);
    cudaError_t err = cudaFuncSetAttribute(split_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    split_combine_kernel<<<unsigned(a.split.num_seqs * a.H), 256, smem, stream>>>(a.split, a.H, p);
    return cudaGetLastError();
}

}  // namespace kda
