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
// The per-pair decay e^{g_r - g_i} is split as e^{g_r - g_m} e^{g_m - g_i} around
// the chunk's middle token m, which keeps both factors within e^{+-|g_L|/2}.
//
// Launch: one CTA (256 threads) per (sequence, head, 32-column slice of d_v).
// The columns of the state evolve independently, so slices never communicate;
// each CTA recomputes the slice-independent chunk quantities (g, A, T, P and the
// decayed q/k rows) in shared memory and walks its sequence chunk by chunk.
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kNV = 32;     // state columns per CTA
constexpr int kMaxD = 128;

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
    return size_t(3) * C * LDK      // Kt, Qt, Kb
         + 3 * kMaxD                // e^{g_m}, e^{g_L - g_m}, e^{g_L}
         + 64                       // beta
         + size_t(3) * C * C        // A, T, P
         + size_t(dk) * kNV         // state slice
         + size_t(2) * C * kNV;     // V slice, U slice
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
    const int j0 = tile * kNV;
    const int nv = min(kNV, dv - j0);
    const int LDK = padded_dk(dk);
    const int dk4 = (dk + 3) & ~3;
    const int tid = threadIdx.x;

    extern __shared__ float4 smem_f4[];
    float *Kt = reinterpret_cast<float *>(smem_f4);  // k e^{g - g_m}, later W = T Kt e^{g_m}
    float *Qt = Kt + C * LDK;                         // q e^{g - g_m}, later q e^{g}
    float *Kb = Qt + C * LDK;                         // k e^{g_m - g}, later k e^{g_L - g}
    float *eref = Kb + C * LDK;
    float *ecref = eref + kMaxD;
    float *gam = ecref + kMaxD;
    float *bet = gam + kMaxD;
    float *A = bet + 64;
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
        Kt[r * LDK + c] = 0.f;
        Qt[r * LDK + c] = 0.f;
        Kb[r * LDK + c] = 0.f;
    }
    for (int e = tid; e < dk * kNV; e += kThreads) {
        const int c = e / kNV, j = e % kNV;
        S[e] = (a.S0 && j < nv) ? a.S0[(size_t(seq) * H + h) * dk * dv + size_t(c) * dv + j0 + j] : 0.f;
    }

    for (int s = bos; s < eos; s += C) {
        const int L = min(C, eos - s);
        __syncthreads();  // the previous chunk is done with every buffer

        // Stage 1: running decay per channel and the decayed copies of q, k.
        if (tid < dk) {
            const int c = tid;
            float g = 0.f;
            for (int r = 0; r < L; ++r) {
                g += a.log_alpha[(size_t(s + r) * H + h) * dk + c];
                Kb[r * LDK + c] = g;
            }
            const float gm = Kb[((L - 1) / 2) * LDK + c];
            eref[c] = expf(gm);
            ecref[c] = expf(g - gm);
            gam[c] = expf(g);
            for (int r = 0; r < C; ++r) {
                float kt = 0.f, qt = 0.f, kb = 0.f;
                if (r < L) {
                    const size_t off = (size_t(s + r) * H + h) * dk + c;
                    const float kv = to_f(kp[off]), qv = to_f(qp[off]);
                    const float gr = Kb[r * LDK + c];
                    const float up = expf(gr - gm), dn = expf(gm - gr);
                    kt = kv * up;
                    qt = qv * up;
                    kb = kv * dn;
                }
                Kt[r * LDK + c] = kt;
                Qt[r * LDK + c] = qt;
                Kb[r * LDK + c] = kb;
            }
        }
        if (tid < C) bet[tid] = tid < L ? a.beta[size_t(s + tid) * H + h] : 0.f;
        for (int e = tid; e < C * kNV; e += kThreads) {
            const int r = e / kNV, j = e % kNV;
            V[e] = (r < L && j < nv) ? to_f(vp[(size_t(s + r) * H + h) * dv + j0 + j]) : 0.f;
        }
        __syncthreads();

        // Stage 2: A (strictly lower, scaled by beta_r) and P (lower, with diagonal).
        for (int e = tid; e < C * C; e += kThreads) {
            const int r = e / C, i = e % C;
            float acc_a = 0.f, acc_p = 0.f;
            if (i <= r) {
                for (int c = 0; c < dk4; c += 4) {
                    const float4 kb = *reinterpret_cast<const float4 *>(&Kb[i * LDK + c]);
                    const float4 kt = *reinterpret_cast<const float4 *>(&Kt[r * LDK + c]);
                    const float4 qt = *reinterpret_cast<const float4 *>(&Qt[r * LDK + c]);
                    acc_a = fmaf(kt.x, kb.x, fmaf(kt.y, kb.y, fmaf(kt.z, kb.z, fmaf(kt.w, kb.w, acc_a))));
                    acc_p = fmaf(qt.x, kb.x, fmaf(qt.y, kb.y, fmaf(qt.z, kb.z, fmaf(qt.w, kb.w, acc_p))));
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

        // Stage 4: W = (T Kt) e^{g_m} = T (K e^{g}) in place (rows bottom-up, thread
        // owns a channel); Q e^{g} = Qt e^{g_m}; K e^{g_L - g} = Kb e^{g_L - g_m}.
        if (tid < dk) {
            const int c = tid;
            const float er = eref[c], ec = ecref[c];
            for (int r = C - 1; r >= 0; --r) {
                float acc = 0.f;
                for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * C + i], Kt[i * LDK + c], acc);
                Kt[r * LDK + c] = acc * er;
            }
            for (int r = 0; r < C; ++r) {
                Qt[r * LDK + c] *= er;
                Kb[r * LDK + c] *= ec;
            }
        }
        __syncthreads();

        // Stage 5: U = T V - W S for this column slice.
        for (int e = tid; e < C * kNV; e += kThreads) {
            const int r = e / kNV, j = e % kNV;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * C + i], V[i * kNV + j], acc);
            for (int c = 0; c < dk; ++c) acc = fmaf(-Kt[r * LDK + c], S[c * kNV + j], acc);
            U[e] = acc;
        }
        __syncthreads();

        // Stage 6: O = (Q e^{g}) S + P U.
        for (int e = tid; e < C * kNV; e += kThreads) {
            const int r = e / kNV, j = e % kNV;
            if (r < L && j < nv) {
                float acc = 0.f;
                for (int c = 0; c < dk; ++c) acc = fmaf(Qt[r * LDK + c], S[c * kNV + j], acc);
                for (int i = 0; i <= r; ++i) acc = fmaf(P[r * C + i], U[i * kNV + j], acc);
                op[(size_t(s + r) * H + h) * dv + j0 + j] = from_f<T>(acc);
            }
        }
        __syncthreads();

        // Stage 7: S <- Diag(e^{g_L}) S + (K e^{g_L - g})^T U.
        for (int e = tid; e < dk * kNV; e += kThreads) {
            const int c = e / kNV, j = e % kNV;
            float acc = gam[c] * S[e];
            for (int i = 0; i < L; ++i) acc = fmaf(Kb[i * LDK + c], U[i * kNV + j], acc);
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
