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

// d_k = d_v = 128 form of the same call, one warp per column slice: the state of a
// (sequence, head) is cut into eight slices of 16 value columns, and a warp carries one
// slice (128 rows x 16 columns, 8 KiB) through the n tokens.  Every column's sums over
// the key rows (y = DS^T k, z = DS^T q) then stay inside the warp (shuffles over the
// lanes that share the column), so no token waits at a block-wide barrier.  A block's
// four warps take four slices of the same (sequence, head) and share the token vectors,
// staged once per group of up to 4 tokens (alpha = e^{log alpha}, k, q, v in fp32,
// q . k and beta).  Lane (rs, cq) holds columns 4 cq .. 4 cq + 3 of rows
// 32 g + 4 rs + u (g, u = 0..3) of its slice (64 registers), so that the 8 row groups
// read consecutive 16-byte pieces of a staged vector (no bank conflicts).  While a
// block computes one (sequence, head), the next one's four slices and its first token
// group arrive in shared memory by cp.async.
constexpr int kSliceCols = 16;
constexpr int kSlices = kMaxD / kSliceCols;
constexpr int kWarpsPerBlock = 4;                      // slices of one unit per block
constexpr int kSliceBlocksPerSm = 4;
constexpr uint32_t kSliceBytes = kMaxD * kSliceCols * 4;
constexpr int kGroup = 4;                              // tokens staged at once (one warp each)
constexpr uint32_t kStageBytes = kGroup * 4 * kMaxD * 4 + 2 * kGroup * 4;  // alpha, k, q, v; q . k, beta
template <typename T> constexpr uint32_t raw_token_bytes() { return 3 * kMaxD * sizeof(T) + kMaxD * 4; }
template <typename T> constexpr uint32_t slice_smem() {
    return kWarpsPerBlock * kSliceBytes + kStageBytes + kGroup * raw_token_bytes<T>() + kGroup * 4;
}

// byte offset of (row, 16-byte quad q) in a slice buffer: 64-byte rows, with the two
// 64-byte halves of each 128-byte line swapped for rows 4..7 of every 8, so that the
// two rows a quarter-warp reads at once (r and r + 4) fall in different banks
__device__ __forceinline__ uint32_t slice_off(int row, int q) {
    return ((uint32_t(row) * 64u) ^ (uint32_t((row >> 2) & 1) << 6)) + uint32_t(q) * 16u;
}

// four consecutive elements as floats
__device__ __forceinline__ void ld4(const __nv_bfloat16 *p, float (&x)[4]) {
    const uint2 w = *reinterpret_cast<const uint2 *>(p);
    x[0] = __uint_as_float(w.x << 16);
    x[1] = __uint_as_float(w.x & 0xffff0000u);
    x[2] = __uint_as_float(w.y << 16);
    x[3] = __uint_as_float(w.y & 0xffff0000u);
}
__device__ __forceinline__ void ld4(const float *p, float (&x)[4]) {
    const float4 f = *reinterpret_cast<const float4 *>(p);
    x[0] = f.x;
    x[1] = f.y;
    x[2] = f.z;
    x[3] = f.w;
}

__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float (&x)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
    *reinterpret_cast<uint2 *>(p) =
        make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
}
__device__ __forceinline__ void store4(float *p, const float (&x)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}

template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, kSliceBlocksPerSm) decode_tokens_slice_kernel(DecodeTokensArgs a) {
    extern __shared__ __align__(128) uint8_t dyn[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rs = lane >> 2, cq = lane & 3;
    uint8_t *buf = dyn + warp * kSliceBytes;
    float *st_a = reinterpret_cast<float *>(dyn + kWarpsPerBlock * kSliceBytes);  // [kGroup][128] each
    float *st_k = st_a + kGroup * kMaxD, *st_q = st_k + kGroup * kMaxD, *st_v = st_q + kGroup * kMaxD;
    float *st_qk = st_v + kGroup * kMaxD, *st_beta = st_qk + kGroup;
    // the next unit's first token group as stored in HBM: k, q, v [kGroup][128] (T), log alpha, beta
    T *raw_k = reinterpret_cast<T *>(st_beta + kGroup);
    T *raw_q = raw_k + kGroup * kMaxD, *raw_v = raw_q + kGroup * kMaxD;
    float *raw_la = reinterpret_cast<float *>(raw_v + kGroup * kMaxD);
    float *raw_beta = raw_la + kGroup * kMaxD;
    const int H = a.H, n = a.n;
    const int nt0 = min(kGroup, n);
    constexpr int kParts = kSlices / kWarpsPerBlock;          // blocks per (sequence, head)
    const int bitems = a.B * H * kParts;  // (sequence, head, part): one per block step
    auto slot_of = [&](int bi) { const int b = bi / (H * kParts); return a.slot_idx ? a.slot_idx[b] : b; };
    auto next_valid = [&](int bi) {  // the first block item >= bi of this block's stride whose slot is in the pool
        for (; bi < bitems; bi += gridDim.x) {
            const int sl = slot_of(bi);
            if (sl >= 0 && sl < a.num_slots) return bi;
        }
        return bitems;
    };
    auto token = [&](int bi, int t) { return (size_t(bi / (H * kParts)) * n + t) * H + (bi / kParts) % H; };  // [B, n, H, .] row
    auto fetch = [&](int bi) {  // this warp's slice (16 quads a lane) and a quarter of the first token group
        const int h = (bi / kParts) % H, cs = (bi % kParts) * kWarpsPerBlock + warp;
        const float *src = a.S_pool + (size_t(slot_of(bi)) * H + h) * kMaxD * kMaxD + cs * kSliceCols;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int c = lane + 32 * k, row = c >> 2, q = c & 3;
            ptx::cp_async16(buf + slice_off(row, q), src + row * kMaxD + 4 * q);
        }
        constexpr int kc = kMaxD * int(sizeof(T)) / 16;  // 16-byte chunks in a q/k/v row
        constexpr int per_tok = 3 * kc + kMaxD / 4;
        for (int e = tid; e < nt0 * per_tok; e += kWarpsPerBlock * 32) {
            const int j = e / per_tok, w = e % per_tok;
            const size_t tok = token(bi, j);
            if (w < 3 * kc) {
                const int which = w / kc, c = w % kc;
                const T *gs = static_cast<const T *>(which == 0 ? a.k : which == 1 ? a.q : a.v) + tok * kMaxD;
                T *ds = (which == 0 ? raw_k : which == 1 ? raw_q : raw_v) + j * kMaxD;
                ptx::cp_async16(reinterpret_cast<char *>(ds) + 16 * c, reinterpret_cast<const char *>(gs) + 16 * c);
            } else {
                const int c = w - 3 * kc;
                ptx::cp_async16(raw_la + j * kMaxD + 4 * c, a.log_alpha + tok * kMaxD + 4 * c);
            }
        }
        if (tid < nt0) ptx::cp_async4(raw_beta + tid, a.beta + token(bi, tid));
        ptx::cp_async_commit();
    };
    // one token per warp: alpha, k, q, v of token j (from kp, qp, vp, lap) into the staged
    // arrays, four channels a lane, and q . k
    auto stage = [&](int j, const T *kp, const T *qp, const T *vp, const float *lap, float beta) {
        float kx[4], qx[4], vx[4], lx[4];
        ld4(kp + 4 * lane, kx);
        ld4(qp + 4 * lane, qx);
        ld4(vp + 4 * lane, vx);
        ld4(lap + 4 * lane, lx);
        float qk = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            lx[i] = expf(lx[i]);
            qk = fmaf(qx[i], kx[i], qk);
        }
        *reinterpret_cast<float4 *>(st_a + j * kMaxD + 4 * lane) = make_float4(lx[0], lx[1], lx[2], lx[3]);
        *reinterpret_cast<float4 *>(st_k + j * kMaxD + 4 * lane) = make_float4(kx[0], kx[1], kx[2], kx[3]);
        *reinterpret_cast<float4 *>(st_q + j * kMaxD + 4 * lane) = make_float4(qx[0], qx[1], qx[2], qx[3]);
        *reinterpret_cast<float4 *>(st_v + j * kMaxD + 4 * lane) = make_float4(vx[0], vx[1], vx[2], vx[3]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
        if (lane == 0) {
            st_qk[j] = qk;
            st_beta[j] = beta;
        }
    };
    int bi = next_valid(blockIdx.x);
    if (bi < bitems) fetch(bi);
    while (bi < bitems) {
        const int h = (bi / kParts) % H;
        const int cbase = ((bi % kParts) * kWarpsPerBlock + warp) * kSliceCols;  // this warp's first value column
        ptx::cp_async_wait_all();
        __syncthreads();  // this unit's slices and first token group have landed
        // s[m] is row 32 (m / 4) + 4 rs + m % 4: the 8 row groups of a warp read consecutive
        // 16-byte pieces of a staged token vector
        float s[16][4];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float4 f = *reinterpret_cast<const float4 *>(buf + slice_off(32 * (m >> 2) + 4 * rs + (m & 3), cq));
            s[m][0] = f.x;
            s[m][1] = f.y;
            s[m][2] = f.z;
            s[m][3] = f.w;
        }
        if (warp < nt0)
            stage(warp, raw_k + warp * kMaxD, raw_q + warp * kMaxD, raw_v + warp * kMaxD, raw_la + warp * kMaxD,
                  raw_beta[warp]);
        __syncthreads();  // the buffers take the next unit; the staged group is complete
        const int nbi = next_valid(bi + gridDim.x);
        if (nbi < bitems) fetch(nbi);
        for (int t0 = 0; t0 < n; t0 += kGroup) {
            const int nt = min(kGroup, n - t0);
            if (t0 > 0) {  // later groups: loaded directly
                __syncthreads();  // the previous group's vectors have been read
                if (warp < nt) {
                    const size_t tok = token(bi, t0 + warp);
                    stage(warp, static_cast<const T *>(a.k) + tok * kMaxD, static_cast<const T *>(a.q) + tok * kMaxD,
                          static_cast<const T *>(a.v) + tok * kMaxD, a.log_alpha + tok * kMaxD, a.beta[tok]);
                }
                __syncthreads();
            }
            for (int j = 0; j < nt; ++j) {
                const float4 *a4 = reinterpret_cast<const float4 *>(st_a + j * kMaxD + 4 * rs);
                const float4 *k4 = reinterpret_cast<const float4 *>(st_k + j * kMaxD + 4 * rs);
                const float4 *q4 = reinterpret_cast<const float4 *>(st_q + j * kMaxD + 4 * rs);
                // DS = Diag(alpha) S; partial y = DS^T k, z = DS^T q over this lane's rows
                float y[4] = {0.f, 0.f, 0.f, 0.f}, z[4] = {0.f, 0.f, 0.f, 0.f}, kv[16];
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
                    const float4 al = a4[8 * m4], kk = k4[8 * m4], qq = q4[8 * m4];
                    const float alv[4] = {al.x, al.y, al.z, al.w}, qv[4] = {qq.x, qq.y, qq.z, qq.w};
                    kv[4 * m4] = kk.x;
                    kv[4 * m4 + 1] = kk.y;
                    kv[4 * m4 + 2] = kk.z;
                    kv[4 * m4 + 3] = kk.w;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int m = 4 * m4 + u;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            s[m][c] *= alv[u];
                            y[c] = fmaf(kv[m], s[m][c], y[c]);
                            z[c] = fmaf(qv[u], s[m][c], z[c]);
                        }
                    }
                }
                // sums over the 8 row groups: the lanes with the same cq (lane bits 2-4)
#pragma unroll
                for (int off = 4; off < 32; off <<= 1)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        y[c] += __shfl_xor_sync(0xffffffffu, y[c], off);
                        z[c] += __shfl_xor_sync(0xffffffffu, z[c], off);
                    }
                const float4 vv = *reinterpret_cast<const float4 *>(st_v + j * kMaxD + cbase + 4 * cq);
                const float vvv[4] = {vv.x, vv.y, vv.z, vv.w};
                const float beta = st_beta[j], qk = st_qk[j];
                float e[4], o[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    e[c] = beta * (vvv[c] - y[c]);
                    o[c] = fmaf(qk, e[c], z[c]);
                }
                if (rs == 0) store4(static_cast<T *>(a.o) + token(bi, t0 + j) * kMaxD + cbase + 4 * cq, o);
#pragma unroll
                for (int m = 0; m < 16; ++m)
#pragma unroll
                    for (int c = 0; c < 4; ++c) s[m][c] = fmaf(kv[m], e[c], s[m][c]);
            }
        }
        float *dst = a.S_pool + (size_t(slot_of(bi)) * H + h) * kMaxD * kMaxD + cbase;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            __stcs(reinterpret_cast<float4 *>(dst + (32 * (m >> 2) + 4 * rs + (m & 3)) * kMaxD + 4 * cq),
                   make_float4(s[m][0], s[m][1], s[m][2], s[m][3]));
        bi = nbi;
    }
}

}  // namespace

cudaError_t launch_decode_tokens(const DecodeTokensArgs &a, cudaStream_t stream) {
    const unsigned grid = unsigned(a.B) * unsigned(a.H);
    if (grid == 0 || a.n == 0) return cudaSuccess;
    const bool full = a.dk == kMaxD && a.dv == kMaxD;
    const uintptr_t rows = reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k) |
                           reinterpret_cast<uintptr_t>(a.v) | reinterpret_cast<uintptr_t>(a.log_alpha) |
                           reinterpret_cast<uintptr_t>(a.o) | reinterpret_cast<uintptr_t>(a.S_pool);
    if (full && (rows & 15u) == 0) {  // the column-slice form (its row loads are 16-byte vectors)
        const int bitems = a.B * a.H * (kSlices / kWarpsPerBlock);
        const unsigned pgrid = unsigned(min(bitems, device_sm_count() * kSliceBlocksPerSm));
        cudaError_t err;
        if (a.dtype == KDA_DTYPE_BF16) {
            err = cudaFuncSetAttribute(decode_tokens_slice_kernel<__nv_bfloat16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(slice_smem<__nv_bfloat16>()));
            if (err != cudaSuccess) return err;
            decode_tokens_slice_kernel<__nv_bfloat16>
                <<<pgrid, kWarpsPerBlock * 32, slice_smem<__nv_bfloat16>(), stream>>>(a);
        } else {
            err = cudaFuncSetAttribute(decode_tokens_slice_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(slice_smem<float>()));
            if (err != cudaSuccess) return err;
            decode_tokens_slice_kernel<float><<<pgrid, kWarpsPerBlock * 32, slice_smem<float>(), stream>>>(a);
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
