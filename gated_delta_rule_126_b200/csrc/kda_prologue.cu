// Input prologue of the KDA layer: short causal depthwise convolution + Swish on the
// q, k, v projections, L2Norm of q and k, and the decay and beta gates -- the parts
// the section "模型架构" of the wiki page "Kimi Linear 高效注意力架构" lists before
// the KDA operator.  Per sequence, head h and channel c:
//   conv(x)[t] = sum_{w < W} weight[h][c][w] x[t - w]   (zero before the sequence start)
//   q = l2norm(swish(conv_q(q_pre))), k likewise, v = swish(conv_v(v_pre))
//   log_alpha = -rate[h] softplus(a),  beta = sigmoid(b)
// Each warp walks 32 consecutive tokens of one head, four channels a lane, keeping
// the convolution's three previous rows in registers and loading rows four tokens
// ahead (bf16 rows stay packed until used, so this fits in 64 registers); HBM-bound.
#include <cmath>

#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kRows = 8;  // warps per block

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float *p) { return *reinterpret_cast<const float4 *>(p); }
    static __device__ __forceinline__ void store(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16 *p) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float4 v) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t *>(&a);
        u.y = *reinterpret_cast<const uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = u;
    }
};

// Four consecutive elements as loaded (bf16 stays packed until used).
template <typename T> struct Raw4;
template <> struct Raw4<float> {
    using type = float4;
    static __device__ __forceinline__ float4 load(const float *p) { return *reinterpret_cast<const float4 *>(p); }
    static __device__ __forceinline__ float4 zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
    static __device__ __forceinline__ float4 widen(float4 v) { return v; }
};
template <> struct Raw4<__nv_bfloat16> {
    using type = uint2;
    static __device__ __forceinline__ uint2 load(const __nv_bfloat16 *p) { return *reinterpret_cast<const uint2 *>(p); }
    static __device__ __forceinline__ uint2 zero() { return make_uint2(0u, 0u); }
    static __device__ __forceinline__ float4 widen(uint2 u) {
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
};

// The CUDA fast intrinsics (a few ulp): the outputs are bf16, or float32 held to 1e-5.
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// max(x, 0) + log(1 + e^{-|x|}): where e^{-|x|} is below fp32's resolution of 1 the
// absolute error stays near 1e-7 (the decay e^{log alpha} then moves by ~1e-7 relative)
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))); }

__device__ __forceinline__ float4 swish4(float4 z) {
    return make_float4(z.x * sigmoid_f(z.x), z.y * sigmoid_f(z.y), z.z * sigmoid_f(z.z), z.w * sigmoid_f(z.w));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// One projection's sliding window for this lane's four channels: the taps' weights and
// the three previous rows as loaded (x[t - 1], x[t - 2], x[t - 3]; zero before the
// sequence start).
template <typename T>
struct Window {
    using Raw = typename Raw4<T>::type;
    float4 w[4];  // w[tap] = weights of channels c0 .. c0 + 3 at that tap (zero past W)
    Raw hist[3];
    __device__ __forceinline__ void load_weights(const float *weight, int W, int h, int d, int c0) {
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
            float v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = (tap < W && c0 < d) ? weight[(size_t(h) * d + c0 + i) * W + tap] : 0.f;
            w[tap] = make_float4(v[0], v[1], v[2], v[3]);
        }
    }
    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int i = 0; i < 3; ++i) hist[i] = Raw4<T>::zero();
    }
    // conv(x)[t] from the current row, then the window moves on by one token
    __device__ __forceinline__ float4 step(Raw xr) {
        const float4 x = Raw4<T>::widen(xr), h0 = Raw4<T>::widen(hist[0]), h1 = Raw4<T>::widen(hist[1]),
                     h2 = Raw4<T>::widen(hist[2]);
        float4 z;
        z.x = w[0].x * x.x + w[1].x * h0.x + w[2].x * h1.x + w[3].x * h2.x;
        z.y = w[0].y * x.y + w[1].y * h0.y + w[2].y * h1.y + w[3].y * h2.y;
        z.z = w[0].z * x.z + w[1].z * h0.z + w[2].z * h1.z + w[3].z * h2.z;
        z.w = w[0].w * x.w + w[1].w * h0.w + w[2].w * h1.w + w[3].w * h2.w;
        hist[2] = hist[1];
        hist[1] = hist[0];
        hist[0] = xr;
        return z;
    }
};

constexpr int kRun = 32;    // consecutive tokens of one head per warp
constexpr int kAhead = 4;   // rows loaded ahead of the one in use

// Walks tokens [t0, t_end) of head h for one projection: swish(conv(x)), L2-normalised
// over the head's d channels when kNorm, stored in out.  seq: the sequence of t0.
// Rows are loaded kAhead tokens ahead into a rotating set of registers.
template <typename T, bool kNorm>
__device__ __forceinline__ void run_projection(const PrologueArgs &a, const T *x, const float *weight, int d, T *out,
                                               int h, int64_t t0, int64_t t_end, int seq, int lane) {
    using Raw = typename Raw4<T>::type;
    const int H = a.H, c0 = 4 * lane;
    const bool on = c0 < d;
    int64_t seq_start = a.cu_seqlens[seq], next = a.cu_seqlens[seq + 1];
    auto ld = [&](int64_t t) { return on ? Raw4<T>::load(x + (size_t(t) * H + h) * d + c0) : Raw4<T>::zero(); };
    Raw ahead[kAhead];
#pragma unroll
    for (int k = 0; k < kAhead; ++k) ahead[k] = t0 + k < t_end ? ld(t0 + k) : Raw4<T>::zero();
    Window<T> win;
    win.load_weights(weight, a.W, h, d, c0);
    win.clear();
    for (int back = 3; back >= 1; --back)  // rows t0 - 3 .. t0 - 1 of the same sequence
        if (t0 - back >= seq_start) win.step(ld(t0 - back));
    for (int64_t tb = t0; tb < t_end; tb += kAhead) {
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
            const int64_t t = tb + k;
            if (t >= t_end) break;
            const Raw cur = ahead[k];
            if (t + kAhead < t_end) ahead[k] = ld(t + kAhead);
            while (t >= next) {  // a new sequence starts at t (empty sequences are skipped)
                ++seq;
                next = a.cu_seqlens[seq + 1];
                win.clear();
            }
            float4 z = swish4(win.step(cur));
            if (kNorm) {
                const float rn = rsqrtf(warp_sum(z.x * z.x + z.y * z.y + z.z * z.z + z.w * z.w) + a.l2_eps);
                z = make_float4(z.x * rn, z.y * rn, z.z * rn, z.w * rn);
            }
            if (on) Vec4<T>::store(out + (size_t(t) * H + h) * d + c0, z);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(32 * kRows, 4) prologue_kernel(const PrologueArgs a) {
    const int H = a.H, lane = threadIdx.x & 31;
    const int64_t wg = int64_t(blockIdx.x) * kRows + (threadIdx.x >> 5);
    const int h = int(wg % H);
    const int64_t t0 = (wg / H) * kRun;
    if (t0 >= a.total_tokens) return;
    const int64_t t_end = min(t0 + int64_t(kRun), a.total_tokens);
    // the sequence holding token t0: the last n with cu_seqlens[n] <= t0
    int lo = 0, hi = a.num_seqs;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (a.cu_seqlens[mid] <= t0) lo = mid; else hi = mid;
    }
    run_projection<T, true>(a, static_cast<const T *>(a.q_pre), a.conv_q, a.dk, static_cast<T *>(a.q), h, t0, t_end, lo, lane);
    run_projection<T, true>(a, static_cast<const T *>(a.k_pre), a.conv_k, a.dk, static_cast<T *>(a.k), h, t0, t_end, lo, lane);
    run_projection<T, false>(a, static_cast<const T *>(a.v_pre), a.conv_v, a.dv, static_cast<T *>(a.v), h, t0, t_end, lo, lane);
    // gates: log alpha = -rate[h] softplus(a_gate), beta = sigmoid(b_gate)
    const float r = -a.rate[h];
    const int c0 = 4 * lane;
    if (c0 < a.dk) {
        for (int64_t tb = t0; tb < t_end; tb += kAhead) {
            float4 g[kAhead];
#pragma unroll
            for (int k = 0; k < kAhead; ++k)
                if (tb + k < t_end) g[k] = *reinterpret_cast<const float4 *>(a.a + (size_t(tb + k) * H + h) * a.dk + c0);
#pragma unroll
            for (int k = 0; k < kAhead; ++k)
                if (tb + k < t_end)
                    *reinterpret_cast<float4 *>(a.log_alpha + (size_t(tb + k) * H + h) * a.dk + c0) =
                        make_float4(r * softplus_f(g[k].x), r * softplus_f(g[k].y), r * softplus_f(g[k].z),
                                    r * softplus_f(g[k].w));
        }
    }
    if (lane < t_end - t0) {
        const size_t row = size_t(t0 + lane) * H + h;
        a.beta[row] = sigmoid_f(a.b[row]);
    }
}

}  // namespace

cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream) {
    if (a.total_tokens == 0) return cudaSuccess;
    const int64_t warps = (a.total_tokens + kRun - 1) / kRun * a.H;
    const unsigned grid = unsigned((warps + kRows - 1) / kRows);
    if (a.dtype == KDA_DTYPE_F32)
        prologue_kernel<float><<<grid, 32 * kRows, 0, stream>>>(a);
    else
        prologue_kernel<__nv_bfloat16><<<grid, 32 * kRows, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace kda
