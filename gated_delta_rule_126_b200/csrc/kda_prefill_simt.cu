// Chunked KDA prefill on CUDA cores in fp32 (any d_k, d_v <= 128; chunk 16/32/64).
//
// This is the float32 path (its inputs and outputs may be fp32 or bf16; every
// operation is an fp32 FFMA).  It evaluates the chunkwise (WY/UT) form of the
// state-update equation of the KDA section of the wiki page "Kimi Linear
// 高效注意力架构" ("Kimi Delta Attention (KDA)"): within a chunk of L tokens that
// starts from state S, with g_r the inclusive running sum of log alpha,
//   A_ri = beta_r <k_r e^{g_r - g_i}, k_i>  (i < r)     T = (I + A)^{-1} Diag(beta)
//   P_ri = <q_r e^{g_r - g_i}, k_i>          (i <= r)
//   U = T V - T (K e^{g}) S                 O = (Q e^{g}) S + P U
//   S <- Diag(e^{g_L}) S + (K e^{g_L - g})^T U
// The decay alpha may be anywhere in [0, 1] (the same section's channel-wise decay
// bullet), alpha = 0 included (log alpha = -inf), so no exponent is ever formed as a
// difference of running sums (-inf - -inf) and no factor exceeds 1:
// * the chunk is cut into 16-token blocks; within block R, h_r is the running sum of
//   log alpha from the block's first token to r and s_r the sum over the tokens after r
//   to the block's end;
// * pairs in different blocks (block I < block R) factor through the boundary before
//   block R: e^{g_r - g_i} = e^{h_r} e^{s_i} e^{(totals of the blocks between)}, every
//   factor <= 1;
// * pairs in the same block take the exact product of the alphas between them, a
//   running product per channel, summed over channels by a transposed warp butterfly;
// * the state products use K e^{g}, Q e^{g} = (K, Q) e^{h} e^{(totals before)} and
//   K e^{g_L - g} = K e^{s} e^{(totals after)}.
//
// Launch: one CTA (256 threads) per (sequence, head, 32-column slice of d_v).
// The columns of the state evolve independently, so slices never communicate;
// each CTA recomputes the slice-independent chunk quantities (A, T, P and the
// decayed q/k rows) in shared memory and walks its sequence chunk by chunk.
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kNV = 32;     // state columns per CTA
constexpr int kMaxD = 128;
constexpr int kBlk = 16;    // tokens per decay block
constexpr int kMaxBlk = 4;  // blocks per chunk (chunk <= 64)
constexpr int kDiagVals = 256;  // per block: P_ri (i <= r, 136) and A_ri (i < r, 120)

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__host__ __device__ __forceinline__ int padded_dk(int dk) { return ((dk + 3) & ~3) + 4; }

// Shared-memory footprint in floats for chunk C and key width dk.
__host__ __device__ __forceinline__ size_t simt_smem_floats(int C, int dk) {
    const int LDK = padded_dk(dk);
    return size_t(3) * C * LDK      // Kr, Qr, Kc
         + 12 * kMaxD               // e^{totals before}, e^{totals after}, block-pair factors, e^{g_L}
         + 64                       // beta
         + size_t(kMaxBlk) * 4 * kDiagVals  // diagonal-block partial sums, per block and channel warp
         + size_t(3) * C * C        // A, T, P
         + size_t(dk) * kNV         // state slice
         + size_t(2) * C * kNV;     // V slice, U slice
}

// Position of a diagonal-block value (row r, column i <= r of a 16-token block) in the
// order the running products emit them.  Column i's run is P_ii, A_{i+1,i}, P_{i+1,i},
// A_{i+2,i}, P_{i+2,i}, ... (31 - 2i values); group g (32 values) holds column g's run
// followed by column 15 - g's.
__device__ __forceinline__ int diag_run_start(int i) { return i < 8 ? 32 * i : 32 * (15 - i) + 2 * i + 1; }
__device__ __forceinline__ int diag_index_p(int r, int i) { return diag_run_start(i) + 2 * (r - i); }
__device__ __forceinline__ int diag_index_a(int r, int i) { return diag_run_start(i) + 2 * (r - i) - 1; }

// x[0..31] per lane -> the return value of lane j is the sum over the warp's lanes of
// x[j] (a transposed butterfly: 31 shuffles).
__device__ __forceinline__ float warp_transpose_sum32(float (&x)[32], int lane) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        const bool hi = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = hi ? x[i] : x[m + i];
            const float keep = hi ? x[m + i] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return x[0];
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1) prefill_simt_kernel(PrefillArgs a) {
    const int ntiles = (a.dv + kNV - 1) / kNV;
    const int tile = blockIdx.x % ntiles;
    const int h = (blockIdx.x / ntiles) % a.H;
    const int nidx = blockIdx.x / (ntiles * a.H);
    const int seq = a.order ? a.order[nidx] : nidx;
    const int bos = a.cu_seqlens[seq], eos = a.cu_seqlens[seq + 1];
    const int dk = a.dk, dv = a.dv, C = a.chunk, H = a.H;
    const int nb = C / kBlk;  // blocks per chunk
    const int j0 = tile * kNV;
    const int nv = min(kNV, dv - j0);
    const int LDK = padded_dk(dk);
    const int dk4 = (dk + 3) & ~3;
    const int dk32 = (dk + 31) & ~31;  // threads of the per-channel phase (whole warps)
    const int tid = threadIdx.x, lane = tid & 31;

    extern __shared__ float4 smem_f4[];
    float *Kr = reinterpret_cast<float *>(smem_f4);  // k e^{h}, later W = T K e^{g}
    float *Qr = Kr + C * LDK;                         // q e^{h}, later q e^{g}
    float *Kc = Qr + C * LDK;                         // k e^{s}, later k e^{g_L - g}
    float *ebefore = Kc + C * LDK;                    // [block][c] e^{totals of the blocks before}
    float *eafter = ebefore + kMaxBlk * kMaxD;        // [block][c] e^{totals of the blocks after}
    float *epair = eafter + kMaxBlk * kMaxD;          // [pair][c] e^{totals strictly between}: (0,2) (1,3) (0,3)
    float *gam = epair + 3 * kMaxD;                   // e^{g_L}
    float *bet = gam + kMaxD;
    float *part = bet + 64;                           // [block][channel warp][256]
    float *A = part + kMaxBlk * 4 * kDiagVals;
    float *Tm = A + C * C;
    float *P = Tm + C * C;
    float *S = P + C * C;       // [dk][kNV]
    float *V = S + dk * kNV;    // [C][kNV]
    float *U = V + C * kNV;     // [C][kNV]

    const T *qp = static_cast<const T *>(a.q);
    const T *kp = static_cast<const T *>(a.k);
    const T *vp = static_cast<const T *>(a.v);
    T *op = static_cast<T *>(a.o);

    // Channel padding columns are read by the float4 loops; keep them zero.
    for (int e = tid; e < C * (LDK - dk); e += kThreads) {
        const int r = e / (LDK - dk), c = dk + e % (LDK - dk);
        Kr[r * LDK + c] = 0.f;
        Qr[r * LDK + c] = 0.f;
        Kc[r * LDK + c] = 0.f;
    }
    for (int e = tid; e < dk * kNV; e += kThreads) {
        const int c = e / kNV, j = e % kNV;
        S[e] = (a.S0 && j < nv) ? a.S0[(size_t(seq) * H + h) * dk * dv + size_t(c) * dv + j0 + j] : 0.f;
    }

    for (int s = bos; s < eos; s += C) {
        const int L = min(C, eos - s);
        __syncthreads();  // the previous chunk is done with every buffer

        // Stage 1: per channel (one thread each, whole warps): the block sums h, s and
        // totals, the decayed rows, the factor tables and the diagonal blocks' partial
        // sums over the warp's 32 channels.
        if (tid < dk32) {
            const int c = tid;
            const bool cv = c < dk;
            float tot[kMaxBlk] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int R = 0; R < kMaxBlk; ++R) {
                if (R >= nb) break;
                float la[kBlk], kv[kBlk], qv[kBlk];
#pragma unroll
                for (int j = 0; j < kBlk; ++j) {
                    const int r = R * kBlk + j;
                    const bool ok = cv && r < L;
                    const size_t off = (size_t(s + r) * H + h) * dk + c;
                    la[j] = ok ? a.log_alpha[off] : 0.f;
                    kv[j] = ok ? to_f(kp[off]) : 0.f;
                    qv[j] = ok ? to_f(qp[off]) : 0.f;
                }
                float hs = 0.f;  // running sum from the block's first token (inclusive)
#pragma unroll
                for (int j = 0; j < kBlk; ++j) {
                    hs += la[j];
                    const float e = expf(hs);
                    if (cv) {
                        Kr[(R * kBlk + j) * LDK + c] = kv[j] * e;
                        Qr[(R * kBlk + j) * LDK + c] = qv[j] * e;
                    }
                }
                tot[R] = hs;
                float ss = 0.f;  // sum over the tokens after j to the block's end
#pragma unroll
                for (int j = kBlk - 1; j >= 0; --j) {
                    if (cv) Kc[(R * kBlk + j) * LDK + c] = kv[j] * expf(ss);
                    ss += la[j];
                }
                // the block's own pairs: P_ri = <q_r, k_i * prod_{i<t<=r} alpha_t> and
                // A_ri = <k_r, same> (beta applied later).  Columns i and 15 - i emit
                // 32 values together (diag_index order), summed over the warp's channels.
                float al[kBlk];
#pragma unroll
                for (int j = 0; j < kBlk; ++j) al[j] = expf(la[j]);
                float *pw = part + (R * 4 + (c >> 5)) * kDiagVals;
#pragma unroll
                for (int g = 0; g < kBlk / 2; ++g) {
                    float x[32];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int i = half ? kBlk - 1 - g : g;
                        const int o = half ? 31 - 2 * g : 0;
                        float w = kv[i];
                        x[o] = qv[i] * w;
#pragma unroll
                        for (int r = i + 1; r < kBlk; ++r) {
                            w *= al[r];
                            x[o + 2 * (r - i) - 1] = kv[r] * w;
                            x[o + 2 * (r - i)] = qv[r] * w;
                        }
                    }
                    pw[32 * g + lane] = warp_transpose_sum32(x, lane);
                }
            }
            // factor tables from the block totals (sums of log alpha only)
            if (cv) {
                float before = 0.f;
#pragma unroll
                for (int R = 0; R < kMaxBlk; ++R) {
                    if (R < nb) {
                        ebefore[R * kMaxD + c] = expf(before);
                        before += tot[R];
                    }
                }
                gam[c] = expf(before);
                float after = 0.f;
#pragma unroll
                for (int R = kMaxBlk - 1; R >= 0; --R) {
                    if (R < nb) {
                        eafter[R * kMaxD + c] = expf(after);
                        after += tot[R];
                    }
                }
                if (nb == kMaxBlk) {
                    epair[0 * kMaxD + c] = expf(tot[1]);
                    epair[1 * kMaxD + c] = expf(tot[2]);
                    epair[2 * kMaxD + c] = expf(tot[1] + tot[2]);
                }
            }
        }
        if (tid < C) bet[tid] = tid < L ? a.beta[size_t(s + tid) * H + h] : 0.f;
        for (int e = tid; e < C * kNV; e += kThreads) {
            const int r = e / kNV, j = e % kNV;
            V[e] = (r < L && j < nv) ? to_f(vp[(size_t(s + r) * H + h) * dv + j0 + j]) : 0.f;
        }
        __syncthreads();

        // Stage 2: A (strictly lower, scaled by beta_r) and P (lower, with diagonal):
        // pairs across blocks from the decayed rows, pairs within a block from the
        // partial sums of stage 1.
        const int nwk = (dk + 31) >> 5;  // channel warps
        for (int e = tid; e < C * C; e += kThreads) {
            const int r = e / C, i = e % C;
            const int R = r / kBlk, I = i / kBlk;
            float acc_a = 0.f, acc_p = 0.f;
            if (i <= r && I < R) {
                const float *m = R - I == 1 ? nullptr : epair + (R - I == 3 ? 2 : I) * kMaxD;
                for (int c = 0; c < dk4; c += 4) {
                    float4 kc = *reinterpret_cast<const float4 *>(&Kc[i * LDK + c]);
                    if (m) {
                        const float4 mm = *reinterpret_cast<const float4 *>(&m[c]);
                        kc = make_float4(kc.x * mm.x, kc.y * mm.y, kc.z * mm.z, kc.w * mm.w);
                    }
                    const float4 kr = *reinterpret_cast<const float4 *>(&Kr[r * LDK + c]);
                    const float4 qr = *reinterpret_cast<const float4 *>(&Qr[r * LDK + c]);
                    acc_a = fmaf(kr.x, kc.x, fmaf(kr.y, kc.y, fmaf(kr.z, kc.z, fmaf(kr.w, kc.w, acc_a))));
                    acc_p = fmaf(qr.x, kc.x, fmaf(qr.y, kc.y, fmaf(qr.z, kc.z, fmaf(qr.w, kc.w, acc_p))));
                }
            } else if (i <= r) {
                const int rl = r - R * kBlk, il = i - I * kBlk;
                const float *pr = part + R * 4 * kDiagVals;
                for (int w = 0; w < nwk; ++w) {
                    acc_p += pr[w * kDiagVals + diag_index_p(rl, il)];
                    if (il < rl) acc_a += pr[w * kDiagVals + diag_index_a(rl, il)];
                }
            }
            A[e] = (i < r) ? bet[r] * acc_a : 0.f;
            P[e] = (i <= r) ? acc_p : 0.f;
        }
        __syncthreads();

        // Stage 3: T = (I + A)^{-1} Diag(beta) by forward substitution; thread j
        // owns column j, whose entries above the diagonal are zero.
        if (tid < C) {
            const int j = tid;
            for (int r = 0; r < C; ++r) {
                float x = 0.f;
                if (r >= j) {
                    x = (r == j) ? bet[r] : 0.f;
                    for (int i = j; i < r; ++i) x = fmaf(-A[r * C + i], Tm[i * C + j], x);
                }
                Tm[r * C + j] = x;
            }
        }
        __syncthreads();

        // Stage 4: K e^{g} = K e^{h} e^{totals before} and Q e^{g} likewise; W = T (K e^{g})
        // in place (rows bottom-up, thread owns a channel); K e^{g_L - g} = K e^{s}
        // e^{totals after}.
        if (tid < dk) {
            const int c = tid;
            for (int r = 0; r < C; ++r) {
                const int R = r / kBlk;
                Kr[r * LDK + c] *= ebefore[R * kMaxD + c];
                Qr[r * LDK + c] *= ebefore[R * kMaxD + c];
                Kc[r * LDK + c] *= eafter[R * kMaxD + c];
            }
            for (int r = C - 1; r >= 0; --r) {
                float acc = 0.f;
                for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * C + i], Kr[i * LDK + c], acc);
                Kr[r * LDK + c] = acc;
            }
        }
        __syncthreads();

        // Stage 5: U = T V - W S for this column slice.
        for (int e = tid; e < C * kNV; e += kThreads) {
            const int r = e / kNV, j = e % kNV;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * C + i], V[i * kNV + j], acc);
            for (int c = 0; c < dk; ++c) acc = fmaf(-Kr[r * LDK + c], S[c * kNV + j], acc);
            U[e] = acc;
        }
        __syncthreads();

        // Stage 6: O = (Q e^{g}) S + P U.
        for (int e = tid; e < C * kNV; e += kThreads) {
            const int r = e / kNV, j = e % kNV;
            if (r < L && j < nv) {
                float acc = 0.f;
                for (int c = 0; c < dk; ++c) acc = fmaf(Qr[r * LDK + c], S[c * kNV + j], acc);
                for (int i = 0; i <= r; ++i) acc = fmaf(P[r * C + i], U[i * kNV + j], acc);
                op[(size_t(s + r) * H + h) * dv + j0 + j] = from_f<T>(acc);
            }
        }
        __syncthreads();

        // Stage 7: S <- Diag(e^{g_L}) S + (K e^{g_L - g})^T U.
        for (int e = tid; e < dk * kNV; e += kThreads) {
            const int c = e / kNV, j = e % kNV;
            float acc = gam[c] * S[e];
            for (int i = 0; i < L; ++i) acc = fmaf(Kc[i * LDK + c], U[i * kNV + j], acc);
            S[e] = acc;
        }
    }
    __syncthreads();
    for (int e = tid; e < dk * kNV; e += kThreads) {
        const int c = e / kNV, j = e % kNV;
        if (j < nv) a.S_final[(size_t(seq) * H + h) * dk * dv + size_t(c) * dv + j0 + j] = S[e];
    }
}

// Sequence order for the grid: longest first, ties by index (a stable rank).
__global__ void order_by_length_kernel(const int32_t *cu, int N, int32_t *order) {
    for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < N; n += gridDim.x * blockDim.x) {
        const int ln = cu[n + 1] - cu[n];
        int rank = 0;
        for (int m = 0; m < N; ++m) {
            const int lm = cu[m + 1] - cu[m];
            rank += (lm > ln) || (lm == ln && m < n);
        }
        order[rank] = n;
    }
}

}  // namespace

size_t prefill_simt_smem_bytes(int chunk, int dk) { return simt_smem_floats(chunk, dk) * sizeof(float); }

cudaError_t launch_order_by_length(const PrefillArgs &a, cudaStream_t stream) {
    if (a.num_seqs <= 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (a.num_seqs + threads - 1) / threads;
    order_by_length_kernel<<<blocks, threads, 0, stream>>>(a.cu_seqlens, a.num_seqs, a.order);
    return cudaGetLastError();
}

cudaError_t launch_prefill_simt(const PrefillArgs &a, cudaStream_t stream) {
    const int ntiles = (a.dv + kNV - 1) / kNV;
    const size_t grid = size_t(a.num_seqs) * a.H * ntiles;
    if (grid == 0) return cudaSuccess;
    const size_t smem = prefill_simt_smem_bytes(a.chunk, a.dk);
    cudaError_t err;
    if (a.dtype == KDA_DTYPE_BF16) {
        err = cudaFuncSetAttribute(prefill_simt_kernel<__nv_bfloat16>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (err != cudaSuccess) return err;
        prefill_simt_kernel<__nv_bfloat16><<<unsigned(grid), kThreads, smem, stream>>>(a);
    } else {
        err = cudaFuncSetAttribute(prefill_simt_kernel<float>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (err != cudaSuccess) return err;
        prefill_simt_kernel<float><<<unsigned(grid), kThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace kda
