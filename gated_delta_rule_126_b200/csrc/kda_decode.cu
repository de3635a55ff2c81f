// K4: one-token recurrent decode step of the KDA operator.
//
// State-update equation of the KDA section (wiki page "Kimi Linear 高效注意力架构",
// "Kimi Delta Attention (KDA)"), applied to a single token per sequence:
//   DS = Diag(alpha) S;  y = DS^T k;  z = DS^T q;  e = beta (v - y);
//   S' = DS + k e^T;     o = S'^T q = z + (q . k) e.
// The step is bound by HBM: the 64 KiB fp32 state of every (sequence, head) is
// read once and written once, so the kernel streams it with 128-bit loads and
// stores that bypass L1 (cache-streaming hints) and keeps it in registers between
// the reductions and the write-back.
//
// Launch: one CTA of 256 threads (8 warps) per (sequence, head).  Warp w owns the
// state rows i = w, w + 8, ..., lane l owns the four columns 4l .. 4l + 3, so one
// warp instruction moves one contiguous 512-byte row segment.  Column sums over
// rows are warp-local partials reduced across the 8 warps through shared memory.
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxD = 128;
constexpr int kRows = kMaxD / kWarps;  // state rows per warp at d_k = 128

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float4 fma4(float s, float4 a, float4 b) {
    return make_float4(fmaf(s, a.x, b.x), fmaf(s, a.y, b.y), fmaf(s, a.z, b.z), fmaf(s, a.w, b.w));
}

// kFull: d_k = d_v = 128, no bounds masks.
template <typename T, bool kFull>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(DecodeArgs a) {
    const int bh = blockIdx.x;
    const int dk = kFull ? kMaxD : a.dk;
    const int dv = kFull ? kMaxD : a.dv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    __shared__ float s_k[kMaxD], s_q[kMaxD], s_alpha[kMaxD];
    __shared__ __align__(16) float s_red[2][kWarps][kMaxD];
    __shared__ __align__(16) float s_e[kMaxD];
    __shared__ float s_qk, s_beta;

    // Issue the state loads first: they are the only large transfer.
    const float4 *Sp = reinterpret_cast<const float4 *>(a.S + size_t(bh) * dk * dv);
    const bool col_ok = kFull || (lane * 4 < dv);
    float4 s[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int i = r * kWarps + warp;
        if (kFull || (i < dk && col_ok))
            s[r] = __ldcs(Sp + (size_t(i) * dv) / 4 + lane);
        else
            s[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    const T *qp = static_cast<const T *>(a.q) + size_t(bh) * dk;
    const T *kp = static_cast<const T *>(a.k) + size_t(bh) * dk;
    const float *lap = a.log_alpha + size_t(bh) * dk;
    if (tid < kMaxD) {
        const bool ok = tid < dk;
        s_k[tid] = ok ? to_f(kp[tid]) : 0.f;
        s_q[tid] = ok ? to_f(qp[tid]) : 0.f;
        s_alpha[tid] = ok ? expf(lap[tid]) : 0.f;
    }
    if (tid == 0) s_beta = a.beta[bh];
    __syncthreads();

    // DS = Diag(alpha) S ; partial y = DS^T k and z = DS^T q over this warp's rows.
    float4 py = make_float4(0.f, 0.f, 0.f, 0.f), pz = py;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int i = r * kWarps + warp;
        const float al = s_alpha[i];
        s[r] = make_float4(s[r].x * al, s[r].y * al, s[r].z * al, s[r].w * al);
        py = fma4(s_k[i], s[r], py);
        pz = fma4(s_q[i], s[r], pz);
    }
    if (col_ok) {
        *reinterpret_cast<float4 *>(&s_red[0][warp][lane * 4]) = py;
        *reinterpret_cast<float4 *>(&s_red[1][warp][lane * 4]) = pz;
    }
    if (warp == 0) {
        float t = 0.f;
        for (int i = lane; i < kMaxD; i += 32) t = fmaf(s_q[i], s_k[i], t);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
        if (lane == 0) s_qk = t;
    }
    __syncthreads();

    if (tid < dv) {
        float y = 0.f, z = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            y += s_red[0][w][tid];
            z += s_red[1][w][tid];
        }
        const T *vp = static_cast<const T *>(a.v) + size_t(bh) * dv;
        const float e = s_beta * (to_f(vp[tid]) - y);
        s_e[tid] = e;
        static_cast<T *>(a.o)[size_t(bh) * dv + tid] = from_f<T>(fmaf(s_qk, e, z));
    }
    __syncthreads();

    // S' = DS + k e^T, written back in place.
    float4 *Sw = reinterpret_cast<float4 *>(a.S + size_t(bh) * dk * dv);
    const float4 e4 = col_ok ? *reinterpret_cast<const float4 *>(&s_e[lane * 4])
                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int i = r * kWarps + warp;
        if (kFull || (i < dk && col_ok)) __stcs(Sw + (size_t(i) * dv) / 4 + lane, fma4(s_k[i], e4, s[r]));
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
    const unsigned grid = unsigned(a.B) * unsigned(a.H);
    if (grid == 0) return cudaSuccess;
    const bool full = a.dk == kMaxD && a.dv == kMaxD;
    if (a.dtype == KDA_DTYPE_BF16) {
        if (full) decode_kernel<__nv_bfloat16, true><<<grid, kThreads, 0, stream>>>(a);
        else decode_kernel<__nv_bfloat16, false><<<grid, kThreads, 0, stream>>>(a);
    } else {
        if (full) decode_kernel<float, true><<<grid, kThreads, 0, stream>>>(a);
        else decode_kernel<float, false><<<grid, kThreads, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace kda

// ---------------------------------------------------------------------------
// Multi-token decode through a state-slot table.
//
// The same recurrence, n consecutive tokens per sequence, with the state of
// sequence b taken from (and written back to) slot slot_idx[b] of a state pool.
// The 64 KiB state of each (sequence, head) stays in registers across the n
// tokens, so it crosses HBM once per call instead of once per token; per token
// only q, k, v, log alpha, beta and o move.  Slots outside [0, num_slots) are
// skipped (nothing is read or written for that sequence).
namespace kda {
namespace {

constexpr int kTokBlock = 8;  // tokens whose vectors are staged in shared memory at once

template <typename T, bool kFull>
__global__ void __launch_bounds__(kThreads, 2) decode_tokens_kernel(DecodeTokensArgs a) {
    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh % a.H;
    const int dk = kFull ? kMaxD : a.dk;
    const int dv = kFull ? kMaxD : a.dv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slot = a.slot_idx ? a.slot_idx[b] : b;
    if (slot < 0 || slot >= a.num_slots) return;  // uniform for the whole CTA

    // per staged token: k, q, alpha (= e^{log alpha}), v, and beta
    __shared__ __align__(16) float s_k[kTokBlock][kMaxD], s_q[kTokBlock][kMaxD];
    __shared__ __align__(16) float s_alpha[kTokBlock][kMaxD], s_v[kTokBlock][kMaxD];
    __shared__ float s_beta[kTokBlock], s_qk[kTokBlock];
    __shared__ __align__(16) float s_red[2][kWarps][kMaxD];
    __shared__ __align__(16) float s_e[kMaxD];

    float *Sg = a.S_pool + (size_t(slot) * a.H + h) * dk * dv;
    const bool col_ok = kFull || (lane * 4 < dv);
    float4 s[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int i = r * kWarps + warp;
        if (kFull || (i < dk && col_ok))
            s[r] = __ldcs(reinterpret_cast<const float4 *>(Sg + size_t(i) * dv) + lane);
        else
            s[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    for (int t0 = 0; t0 < a.n; t0 += kTokBlock) {
        const int nt = min(kTokBlock, a.n - t0);
        // stage the vectors of tokens t0 .. t0 + nt - 1 (all loads issued together)
        for (int e = tid; e < nt * kMaxD; e += kThreads) {
            const int j = e / kMaxD, c = e % kMaxD;
            const size_t tok = (size_t(b) * a.n + t0 + j) * a.H + h;  // [B, n, H, .] row
            const bool okk = c < dk, okv = c < dv;
            s_k[j][c] = okk ? to_f(static_cast<const T *>(a.k)[tok * dk + c]) : 0.f;
            s_q[j][c] = okk ? to_f(static_cast<const T *>(a.q)[tok * dk + c]) : 0.f;
            s_alpha[j][c] = okk ? expf(a.log_alpha[tok * dk + c]) : 0.f;
            s_v[j][c] = okv ? to_f(static_cast<const T *>(a.v)[tok * dv + c]) : 0.f;
        }
        if (tid < nt) s_beta[tid] = a.beta[(size_t(b) * a.n + t0 + tid) * a.H + h];
        __syncthreads();
        if (warp < nt) {  // q . k of each staged token, one warp per token
            float x = 0.f;
            for (int i = lane; i < kMaxD; i += 32) x = fmaf(s_q[warp][i], s_k[warp][i], x);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (lane == 0) s_qk[warp] = x;
        }

        for (int j = 0; j < nt; ++j) {
            float4 py = make_float4(0.f, 0.f, 0.f, 0.f), pz = py;
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                const int i = r * kWarps + warp;
                const float al = s_alpha[j][i];
                s[r] = make_float4(s[r].x * al, s[r].y * al, s[r].z * al, s[r].w * al);
                py = fma4(s_k[j][i], s[r], py);
                pz = fma4(s_q[j][i], s[r], pz);
            }
            if (col_ok) {
                *reinterpret_cast<float4 *>(&s_red[0][warp][lane * 4]) = py;
                *reinterpret_cast<float4 *>(&s_red[1][warp][lane * 4]) = pz;
            }
            __syncthreads();
            if (tid < dv) {
                float y = 0.f, z = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    y += s_red[0][w][tid];
                    z += s_red[1][w][tid];
                }
                const float e = s_beta[j] * (s_v[j][tid] - y);
                s_e[tid] = e;
                const size_t tok = (size_t(b) * a.n + t0 + j) * a.H + h;
                static_cast<T *>(a.o)[tok * dv + tid] = from_f<T>(fmaf(s_qk[j], e, z));
            }
            __syncthreads();
            const float4 e4 = col_ok ? *reinterpret_cast<const float4 *>(&s_e[lane * 4])
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                const int i = r * kWarps + warp;
                s[r] = fma4(s_k[j][i], e4, s[r]);
            }
            // s_red and s_e are rewritten by the next token only after its first barrier
        }
        __syncthreads();  // the staged vectors are rewritten by the next block
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        const int i = r * kWarps + warp;
        if (kFull || (i < dk && col_ok)) __stcs(reinterpret_cast<float4 *>(Sg + size_t(i) * dv) + lane, s[r]);
    }
}

}  // namespace

cudaError_t launch_decode_tokens(const DecodeTokensArgs &a, cudaStream_t stream) {
    const unsigned grid = unsigned(a.B) * unsigned(a.H);
    if (grid == 0 || a.n == 0) return cudaSuccess;
    const bool full = a.dk == kMaxD && a.dv == kMaxD;
    if (a.dtype == KDA_DTYPE_BF16) {
        if (full) decode_tokens_kernel<__nv_bfloat16, true><<<grid, kThreads, 0, stream>>>(a);
        else decode_tokens_kernel<__nv_bfloat16, false><<<grid, kThreads, 0, stream>>>(a);
    } else {
        if (full) decode_tokens_kernel<float, true><<<grid, kThreads, 0, stream>>>(a);
        else decode_tokens_kernel<float, false><<<grid, kThreads, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace kda
