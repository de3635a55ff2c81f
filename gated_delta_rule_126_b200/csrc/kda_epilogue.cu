// Output epilogue of the KDA layer applied in place after a prefill that does not
// fuse it (the float32 path): per token and head, y = o / sqrt(mean_j o_j^2 + eps)
// * w * sigmoid(gate) -- the layer's sigmoid output gate and RMSNorm, section
// "模型架构" of the wiki page "Kimi Linear 高效注意力架构".  One warp per (token,
// head) row of d_v <= 128 values.
#include "kda_internal.h"

namespace kda {
namespace {

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

constexpr int kRowsPerBlock = 8;

template <typename T>
__global__ void __launch_bounds__(32 * kRowsPerBlock)
    gated_rmsnorm_kernel(T *y, const T *gate, const float *w, float eps, int64_t rows, int dv) {
    const int64_t r = int64_t(blockIdx.x) * kRowsPerBlock + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    T *yr = y + r * dv;
    const T *gr = gate + r * dv;
    float x[4];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int c = lane + 32 * u;
        x[u] = c < dv ? to_f(yr[c]) : 0.f;
        ss = fmaf(x[u], x[u], ss);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const float rstd = rsqrtf(ss / float(dv) + eps);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int c = lane + 32 * u;
        if (c < dv) {
            const float sg = 1.f / (1.f + expf(-to_f(gr[c])));
            yr[c] = from_f<T>(x[u] * rstd * w[c] * sg);
        }
    }
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const PrefillArgs &a, cudaStream_t stream) {
    const int64_t rows = a.total_tokens * a.H;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = unsigned((rows + kRowsPerBlock - 1) / kRowsPerBlock);
    if (a.dtype == KDA_DTYPE_F32)
        gated_rmsnorm_kernel<float><<<grid, 32 * kRowsPerBlock, 0, stream>>>(
            static_cast<float *>(a.o), static_cast<const float *>(a.gate), a.norm_weight, a.eps, rows, a.dv);
    else
        gated_rmsnorm_kernel<__nv_bfloat16><<<grid, 32 * kRowsPerBlock, 0, stream>>>(
            static_cast<__nv_bfloat16 *>(a.o), static_cast<const __nv_bfloat16 *>(a.gate), a.norm_weight, a.eps,
            rows, a.dv);
    return cudaGetLastError();
}

}  // namespace kda
