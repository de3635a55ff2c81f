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
#include "sm100_ptx.cuh"

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

// d_k = d_v = 128 form of the same call as a persistent kernel that streams states:
// while a CTA runs the tokens of one (sequence, head) from registers, the next unit's
// 64 KiB state arrives in shared memory by bulk copy and its first eight tokens'
// vectors by cp.async, so HBM keeps moving through the compute phase instead of
// idling between a CTA's load and its store.
constexpr int kStreamCtasPerSm = 2;
constexpr uint32_t kStateBytes = kMaxD * kMaxD * 4;
constexpr long long kStreamWait = 4000000000LL;  // about two seconds

template <typename T> constexpr uint32_t stream_raw_bytes() {  // raw vectors of one token block
    return 3 * kTokBlock * kMaxD * sizeof(T) + kTokBlock * kMaxD * 4 + kTokBlock * 4;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm) decode_tokens_stream_kernel(DecodeTokensArgs a) {
    extern __shared__ __align__(128) uint8_t dyn[];
    float *s_next = reinterpret_cast<float *>(dyn);  // the next unit's state, [128][128]
    // the next unit's first token block as stored in HBM: k, q, v [8][128] (T), log alpha [8][128], beta [8]
    T *r_k = reinterpret_cast<T *>(dyn + kStateBytes);
    T *r_q = r_k + kTokBlock * kMaxD, *r_v = r_q + kTokBlock * kMaxD;
    float *r_la = reinterpret_cast<float *>(r_v + kTokBlock * kMaxD);
    float *r_beta = r_la + kTokBlock * kMaxD;
    __shared__ __align__(16) float s_k[kTokBlock][kMaxD], s_q[kTokBlock][kMaxD];
    __shared__ __align__(16) float s_alpha[kTokBlock][kMaxD], s_v[kTokBlock][kMaxD];
    __shared__ float s_beta[kTokBlock], s_qk[kTokBlock];
    __shared__ __align__(16) float s_red[2][kWarps][kMaxD];
    __shared__ __align__(16) float s_e[kMaxD];
    __shared__ __align__(8) uint64_t bar;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, units = a.B * a.H;
    auto slot_of = [&](int u) { const int b = u / H; return a.slot_idx ? a.slot_idx[b] : b; };
    auto next_valid = [&](int u) {  // the first unit >= u of this CTA's stride whose slot is in the pool
        for (; u < units; u += gridDim.x) {
            const int sl = slot_of(u);
            if (sl >= 0 && sl < a.num_slots) return u;
        }
        return units;
    };
    auto state_of = [&](int u) { return a.S_pool + (size_t(slot_of(u)) * H + u % H) * kMaxD * kMaxD; };
    auto fetch = [&](int u) {  // one thread: the state of unit u into s_next
        ptx::mbar_arrive_expect_tx(&bar, kStateBytes);
        const char *src = reinterpret_cast<const char *>(state_of(u));
        for (int part = 0; part < 4; ++part)
            ptx::bulk_load(reinterpret_cast<char *>(s_next) + part * (kStateBytes / 4), src + part * (kStateBytes / 4),
                           kStateBytes / 4, &bar);
    };
    const int nt0 = min(kTokBlock, a.n);
    auto prefetch_tokens = [&](int u) {  // all threads: the first token block of unit u, by cp.async
        const int b = u / H, h = u % H;
        constexpr int kc = kMaxD * int(sizeof(T)) / 16;  // 16-byte chunks in a q/k/v row
        for (int e = tid; e < nt0 * (3 * kc + kMaxD / 4); e += kThreads) {
            const int j = e / (3 * kc + kMaxD / 4), w = e % (3 * kc + kMaxD / 4);
            const size_t tok = (size_t(b) * a.n + j) * H + h;
            if (w < 3 * kc) {
                const int which = w / kc, c = w % kc;
                const T *src = static_cast<const T *>(which == 0 ? a.k : which == 1 ? a.q : a.v) + tok * kMaxD;
                T *dst = (which == 0 ? r_k : which == 1 ? r_q : r_v) + j * kMaxD;
                ptx::cp_async16(reinterpret_cast<char *>(dst) + 16 * c, reinterpret_cast<const char *>(src) + 16 * c);
            } else {
                const int c = w - 3 * kc;
                ptx::cp_async16(r_la + j * kMaxD + 4 * c, a.log_alpha + tok * kMaxD + 4 * c);
            }
        }
        if (tid < nt0) ptx::cp_async4(r_beta + tid, a.beta + (size_t(b) * a.n + tid) * H + h);
        ptx::cp_async_commit();
    };
    if (tid == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int u = next_valid(blockIdx.x);
    if (u < units) {
        if (tid == 0) fetch(u);
        prefetch_tokens(u);
    }
    uint32_t phase = 0;
    while (u < units) {
        const int b = u / H, h = u % H;
        // a wait that ran out ends the kernel for the whole block (decided together, so no
        // thread is left at a barrier)
        const bool ok = ptx::mbar_wait_bounded(&bar, phase & 1u, kStreamWait);
        if (__syncthreads_or(!ok)) return;
        ++phase;
        float4 s[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) s[r] = *reinterpret_cast<const float4 *>(s_next + (r * kWarps + warp) * kMaxD + lane * 4);
        ptx::fence_proxy_async_smem();
        ptx::cp_async_wait_all();  // this unit's first token block
        __syncthreads();  // every thread holds its part: the buffer takes the next unit
        const int un = next_valid(u + gridDim.x);
        if (un < units && tid == 0) fetch(un);
        for (int e = tid; e < nt0 * kMaxD; e += kThreads) {  // first block: from the prefetched copy
            const int j = e / kMaxD, c = e % kMaxD;
            s_k[j][c] = to_f(r_k[j * kMaxD + c]);
            s_q[j][c] = to_f(r_q[j * kMaxD + c]);
            s_alpha[j][c] = expf(r_la[j * kMaxD + c]);
            s_v[j][c] = to_f(r_v[j * kMaxD + c]);
        }
        if (tid < nt0) s_beta[tid] = r_beta[tid];
        __syncthreads();  // the raw copy is free again
        if (un < units) prefetch_tokens(un);

        for (int t0 = 0; t0 < a.n; t0 += kTokBlock) {
            const int nt = min(kTokBlock, a.n - t0);
            for (int e = tid; t0 > 0 && e < nt * kMaxD; e += kThreads) {  // later blocks: direct loads
                const int j = e / kMaxD, c = e % kMaxD;
                const size_t tok = (size_t(b) * a.n + t0 + j) * H + h;
                s_k[j][c] = to_f(static_cast<const T *>(a.k)[tok * kMaxD + c]);
                s_q[j][c] = to_f(static_cast<const T *>(a.q)[tok * kMaxD + c]);
                s_alpha[j][c] = expf(a.log_alpha[tok * kMaxD + c]);
                s_v[j][c] = to_f(static_cast<const T *>(a.v)[tok * kMaxD + c]);
            }
            if (t0 > 0 && tid < nt) s_beta[tid] = a.beta[(size_t(b) * a.n + t0 + tid) * H + h];
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
                *reinterpret_cast<float4 *>(&s_red[0][warp][lane * 4]) = py;
                *reinterpret_cast<float4 *>(&s_red[1][warp][lane * 4]) = pz;
                __syncthreads();
                if (tid < kMaxD) {
                    float y = 0.f, z = 0.f;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) {
                        y += s_red[0][w][tid];
                        z += s_red[1][w][tid];
                    }
                    const float e = s_beta[j] * (s_v[j][tid] - y);
                    s_e[tid] = e;
                    const size_t tok = (size_t(b) * a.n + t0 + j) * H + h;
                    static_cast<T *>(a.o)[tok * kMaxD + tid] = from_f<T>(fmaf(s_qk[j], e, z));
                }
                __syncthreads();
                const float4 e4 = *reinterpret_cast<const float4 *>(&s_e[lane * 4]);
#pragma unroll
                for (int r = 0; r < kRows; ++r) s[r] = fma4(s_k[j][r * kWarps + warp], e4, s[r]);
            }
            __syncthreads();  // the staged vectors are rewritten by the next block
        }
        float *Sg = state_of(u);
#pragma unroll
        for (int r = 0; r < kRows; ++r)
            __stcs(reinterpret_cast<float4 *>(Sg + size_t(r * kWarps + warp) * kMaxD) + lane, s[r]);
        u = un;
    }
}

}  // namespace

cudaError_t launch_decode_tokens(const DecodeTokensArgs &a, cudaStream_t stream) {
    const unsigned grid = unsigned(a.B) * unsigned(a.H);
    if (grid == 0 || a.n == 0) return cudaSuccess;
    const bool full = a.dk == kMaxD && a.dv == kMaxD;
    const uintptr_t rows = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                           reinterpret_cast<uintptr_t>(a.v) | reinterpret_cast<uintptr_t>(a.log_alpha);
    if (full && (rows & 15u) == 0) {  // persistent, state-streaming form (its cp.async copies need 16-byte rows)
        const unsigned pgrid = min(grid, unsigned(device_sm_count() * kStreamCtasPerSm));
        cudaError_t err;
        if (a.dtype == KDA_DTYPE_BF16) {
            constexpr uint32_t smem = kStateBytes + stream_raw_bytes<__nv_bfloat16>();
            err = cudaFuncSetAttribute(decode_tokens_stream_kernel<__nv_bfloat16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (err != cudaSuccess) return err;
            decode_tokens_stream_kernel<__nv_bfloat16><<<pgrid, kThreads, smem, stream>>>(a);
        } else {
            constexpr uint32_t smem = kStateBytes + stream_raw_bytes<float>();
            err = cudaFuncSetAttribute(decode_tokens_stream_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
            if (err != cudaSuccess) return err;
            decode_tokens_stream_kernel<float><<<pgrid, kThreads, smem, stream>>>(a);
        }
        return cudaGetLastError();
    }
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
