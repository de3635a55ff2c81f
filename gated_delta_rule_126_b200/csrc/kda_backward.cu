// Backward pass of the KDA recurrence (training): exact gradients of
// sum <dO, o> + <dS_final, S_final> with respect to q, k, v, log alpha, beta and S0.
//
// The forward map is the state-update equation of the wiki page "Kimi Linear
// 高效注意力架构", section "关键技术方法 > Kimi Delta Attention (KDA)", read out
// from the post-update state, token by token:
//   P_t = Diag(alpha_t) S_{t-1},  w_t = v_t - P_t^T k_t,  S_t = P_t + beta_t k_t w_t^T,
//   o_t = S_t^T q_t,  alpha_t = exp(log alpha_t).
// Its adjoint, with G = dL/dS_t carried from the last token back to the first:
//   G += q_t do_t^T;  dq_t = S_t do_t;  de = G^T k_t (de = dL/d(beta_t w_t));
//   dv_t = beta_t de;  dbeta_t = de . w_t;  du = -beta_t de;
//   dP = G + k_t du^T;  dk_t = G (beta_t w_t) + P_t du;
//   dlog_alpha_t[i] = sum_j dP[i][j] P_t[i][j];  G <- Diag(alpha_t) dP;  dS0 = G at the start.
//
// Every value column j of the state evolves on its own given (k, alpha, beta): the
// key-side operators act on rows only.  So the work is cut into slices of 16 value
// columns.  The reductions over value columns (dq, dk, dlog_alpha, dbeta) are
// per-slice sums, which the slices add into the zeroed outputs with fp32 atomics in
// L2; the order in which the slices arrive is not fixed, so repeated calls can
// differ in the last bits of those four gradients.
//
// Two launches, after the four outputs are zeroed:
//   1. states: the forward sweep, one warp per slice (lane (rs, cq) holding rows
//      32 g + 4 rs + u (g, u = 0..3) and columns 4 cq .. 4 cq + 3), four slices of one
//      (sequence, head) per block; its one reduction over key rows (w_t) is three
//      shuffle rounds.  It stores w_t for every token and the state before every 32nd
//      token of each sequence (checkpoints); each 32-token block's alpha and k rows are
//      staged in shared memory first;
//   2. grads: the backward sweep, one 128-thread block per (sequence, head, slice),
//      thread i owning key row i of the slice; its reduction over key rows (de) is a
//      transposed warp butterfly plus a 4-warp exchange in shared memory.  It walks
//      32-token blocks from the last; each block's alpha and k rows are staged in
//      shared memory first (off the per-token critical path), and its 4-token
//      sub-blocks (last first) are replayed with the stored w (no reduction needed)
//      from the block's checkpoint or, past the middle, from the state before the
//      block's 16th token, their input states kept in shared memory.
// CUDA cores in fp32 throughout; no tensor cores and no waits on other blocks.
#include <cmath>

#include "kda_internal.h"

namespace {

constexpr int kCols = 16;  // value columns per slice
constexpr int kRows = 128; // threads per block = key rows
constexpr int kBlk = 32;   // tokens between checkpoints
constexpr int kSub = 4;    // tokens per replayed sub-block
constexpr int kMid = kBlk / 2;

struct BwdArgs {
    const void *q, *k, *v, *dO;
    const float *log_alpha, *beta, *S0, *dS_final;
    const int32_t *cu_seqlens;
    int num_seqs, H, dk, dv, nsl;
    int64_t T;
    float *dq, *dk_out, *dv_out, *dla, *dbeta, *dS0;
    float4 *ck;            // [blk][H][nsl][4][128] float4: checkpoint slices, row-interleaved
    float *w;              // [T][H][nsl * 16]
};

struct BwdLayout {
    size_t ck_offset = 0, w_offset = 0, total = 0;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Checkpoint slots: sequence n's blocks start at floor(cu[n] / 32) + n, which leaves
// room for ceil(L_n / 32) blocks before sequence n + 1's first slot.
BwdLayout bwd_layout(int num_seqs, int64_t T, int H, int dk, int dv) {
    BwdLayout L;
    const int nsl = (dv + kCols - 1) / kCols;
    const size_t nblk = size_t(T / kBlk) + size_t(num_seqs) + 1;
    L.ck_offset = kda::WorkspaceLayout::kStatusBytes;
    L.w_offset = L.ck_offset + align256(nblk * size_t(H) * nsl * 4 * kRows * sizeof(float4));
    L.total = L.w_offset + align256(size_t(T) * H * nsl * kCols * sizeof(float));
    return L;
}

__device__ __forceinline__ float ldf(const float *p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

// Sums c[j] over the block's 128 threads for each of the 16 columns j; every thread
// gets all 16 sums.  Within a warp a transposed butterfly halves the columns each
// lane carries at every step (16 shuffles), leaving column (lane >> 1) & 15 summed
// over the warp in lanes 2m and 2m + 1; the 4 warps then meet in shared memory.
// `buf` alternates between two halves on consecutive calls, so one barrier a call
// suffices: a thread's reads of a half come before its next call's barrier.
__device__ __forceinline__ void column_sums(const float (&c)[kCols], float4 (*buf)[4], int warp, int lane,
                                            float (&out)[kCols]) {
    constexpr unsigned kAll = 0xffffffffu;
    float x8[8], x4[4], x2[2];
    const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4, u2 = lane & 2;
#pragma unroll
    for (int j = 0; j < 8; ++j) x8[j] = (u16 ? c[j + 8] : c[j]) + __shfl_xor_sync(kAll, u16 ? c[j] : c[j + 8], 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) x4[j] = (u8 ? x8[j + 4] : x8[j]) + __shfl_xor_sync(kAll, u8 ? x8[j] : x8[j + 4], 8);
#pragma unroll
    for (int j = 0; j < 2; ++j) x2[j] = (u4 ? x4[j + 2] : x4[j]) + __shfl_xor_sync(kAll, u4 ? x4[j] : x4[j + 2], 4);
    float x1 = (u2 ? x2[1] : x2[0]) + __shfl_xor_sync(kAll, u2 ? x2[0] : x2[1], 2);
    x1 += __shfl_xor_sync(kAll, x1, 1);
    if ((lane & 1) == 0) reinterpret_cast<float *>(buf[warp])[lane >> 1] = x1;
    __syncthreads();
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        const float4 a = buf[0][q4], b = buf[1][q4], c2 = buf[2][q4], d = buf[3][q4];
        out[4 * q4 + 0] = (a.x + b.x) + (c2.x + d.x);
        out[4 * q4 + 1] = (a.y + b.y) + (c2.y + d.y);
        out[4 * q4 + 2] = (a.z + b.z) + (c2.z + d.z);
        out[4 * q4 + 3] = (a.w + b.w) + (c2.w + d.w);
    }
}

// x[idx] for a thread-dependent idx < 16, without local memory.
__device__ __forceinline__ float pick(const float (&x)[kCols], int idx) {
    float r = 0.f;
#pragma unroll
    for (int j = 0; j < kCols; ++j) r = idx == j ? x[j] : r;
    return r;
}

// (sequence, head, slice) of this block; slices of one head are adjacent in the grid.
struct Unit {
    int s, h, sl, c0;
    int64_t cs, ce, base;
};
__device__ __forceinline__ Unit unit_of(const BwdArgs &a) {
    Unit u;
    u.sl = int(blockIdx.x % unsigned(a.nsl));
    const int64_t sh = blockIdx.x / unsigned(a.nsl);
    u.h = int(sh % a.H);
    u.s = int(sh / a.H);
    u.c0 = u.sl * kCols;
    u.cs = a.cu_seqlens[u.s];
    u.ce = a.cu_seqlens[u.s + 1];
    u.base = u.cs / kBlk + u.s;
    return u;
}

// checkpoint slice of block `blk` (relative to the sequence) of unit u
__device__ __forceinline__ float4 *ck_slice(const BwdArgs &a, const Unit &u, int64_t blk) {
    return a.ck + (((u.base + blk) * a.H + u.h) * a.nsl + u.sl) * (4 * kRows);
}

// The forward sweep, one warp per slice: lane (rs, cq) holds columns 4 cq .. 4 cq + 3 of
// rows 32 g + 4 rs + u (g, u = 0..3) of the slice (64 registers; S[4 g + u]), so the 8
// row groups read consecutive 16-byte pieces of a staged row (no bank conflicts), and
// the one sum over key rows a token needs (P_t^T k_t) is 3 shuffle rounds over the 8
// lanes that share a column quad; no token waits at a barrier.  A block's kSw warps take kSw slices of one (sequence,
// head) and share each 32-token block's alpha and k rows, v and beta, staged in shared
// memory behind one barrier per block.
constexpr int kSw = 4;  // slices (warps) per block of the forward sweep
static_assert(kSw * 32 == kRows, "the staging gives one key row to each thread");

template <typename T>
__global__ void __launch_bounds__(kSw * 32, 4) bwd_states_kernel(const BwdArgs a) {
    __shared__ __align__(16) float vs[kBlk][kSw * kCols];
    __shared__ float bs[kBlk];
    __shared__ __align__(16) float al_s[kBlk][kRows];
    __shared__ __align__(16) float k_s[kBlk][kRows];
    const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
    const int rs = lane >> 2, cq = lane & 3;
    const int nparts = (a.nsl + kSw - 1) / kSw;
    const int part = int(blockIdx.x % unsigned(nparts));
    const int64_t sh = blockIdx.x / unsigned(nparts);
    const int H = a.H, dk = a.dk, dv = a.dv, dvp = a.nsl * kCols;
    const int h = int(sh % H), s = int(sh / H);
    const int sl = part * kSw + warp;  // this warp's slice; past the last one it only joins the barriers
    const bool live = sl < a.nsl;
    const int c0 = sl * kCols;
    const int64_t cs = a.cu_seqlens[s], ce = a.cu_seqlens[s + 1], base = cs / kBlk + s;
    const bool row = i < dk;  // the staging thread's key row
    const T *kp = static_cast<const T *>(a.k);
    const T *vp = static_cast<const T *>(a.v);

    float S[16][4];
#pragma unroll
    for (int m = 0; m < 16; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int r = 32 * (m >> 2) + 4 * rs + (m & 3), col = c0 + 4 * cq + c;
            S[m][c] = (a.S0 && live && r < dk && col < dv) ? a.S0[((int64_t(s) * H + h) * dk + r) * dv + col] : 0.f;
        }
    for (int64_t tb = cs; tb < ce; tb += kBlk) {
        const int n = int(min(int64_t(kBlk), ce - tb));
        if (live) {  // the checkpoint: quad cq of row r at [cq][r]
            float4 *ckp = a.ck + (((base + (tb - cs) / kBlk) * H + h) * a.nsl + sl) * (4 * kRows);
#pragma unroll
            for (int m = 0; m < 16; ++m)
                ckp[cq * kRows + 32 * (m >> 2) + 4 * rs + (m & 3)] = make_float4(S[m][0], S[m][1], S[m][2], S[m][3]);
        }
        __syncthreads();  // the previous block's reads of the staged rows are done
        for (int e = i; e < kBlk * kSw * kCols; e += kRows) {
            const int tt = e / (kSw * kCols), j = e % (kSw * kCols), col = part * kSw * kCols + j;
            vs[tt][j] = (tt < n && col < dv) ? ldf(vp + ((tb + tt) * H + h) * dv + col) : 0.f;
        }
        if (i < kBlk) bs[i] = i < n ? a.beta[(tb + i) * H + h] : 0.f;
        for (int t8 = 0; t8 < kBlk; t8 += 8) {  // this thread's row of alpha and k, eight tokens' loads at a time
            float la[8], kx[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const bool in = row && t8 + j < n;
                const int64_t r = ((tb + t8 + j) * H + h) * dk + i;
                la[j] = in ? a.log_alpha[r] : 0.f;
                kx[j] = in ? ldf(kp + r) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) al_s[t8 + j][i] = expf(la[j]), k_s[t8 + j][i] = kx[j];
        }
        __syncthreads();
        if (!live) continue;
        for (int tt = 0; tt < n; ++tt) {
            const float4 *a4 = reinterpret_cast<const float4 *>(&al_s[tt][4 * rs]);
            const float4 *k4 = reinterpret_cast<const float4 *>(&k_s[tt][4 * rs]);
            float ps[4] = {0.f, 0.f, 0.f, 0.f}, kv[16];
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4) {
                const float4 al = a4[8 * m4], kk = k4[8 * m4];
                const float alv[4] = {al.x, al.y, al.z, al.w};
                kv[4 * m4] = kk.x;
                kv[4 * m4 + 1] = kk.y;
                kv[4 * m4 + 2] = kk.z;
                kv[4 * m4 + 3] = kk.w;
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        S[4 * m4 + u][c] *= alv[u];
                        ps[c] = fmaf(kv[4 * m4 + u], S[4 * m4 + u][c], ps[c]);
                    }
            }
            // P_t^T k_t: the sums over the 8 row groups (lane bits 2-4)
#pragma unroll
            for (int off = 4; off < 32; off <<= 1)
#pragma unroll
                for (int c = 0; c < 4; ++c) ps[c] += __shfl_xor_sync(0xffffffffu, ps[c], off);
            const float b = bs[tt];
            const float4 vv = *reinterpret_cast<const float4 *>(&vs[tt][warp * kCols + 4 * cq]);
            const float wv[4] = {vv.x - ps[0], vv.y - ps[1], vv.z - ps[2], vv.w - ps[3]};
#pragma unroll
            for (int m = 0; m < 16; ++m)
#pragma unroll
                for (int c = 0; c < 4; ++c) S[m][c] = fmaf(kv[m], b * wv[c], S[m][c]);
            if (rs == 0)
                *reinterpret_cast<float4 *>(a.w + ((tb + tt) * H + h) * dvp + c0 + 4 * cq) =
                    make_float4(wv[0], wv[1], wv[2], wv[3]);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(kRows, 3) bwd_grads_kernel(const BwdArgs a) {
    __shared__ float4 hist[kSub][4][kRows];  // input states of the sub-block's tokens (own rows)
    // alpha and k of the block's tokens (each thread its own row), in dynamic shared memory
    extern __shared__ __align__(16) uint8_t bwd_dyn[];
    float(*als)[kRows] = reinterpret_cast<float(*)[kRows]>(bwd_dyn);
    T(*ks)[kRows] = reinterpret_cast<T(*)[kRows]>(bwd_dyn + kBlk * kRows * sizeof(float));
    __shared__ float4 midst[4][kRows];       // state before the block's middle token (own rows)
    __shared__ float4 red[2][4][4];
    __shared__ float ws[kBlk][kCols], dos[kBlk][kCols];
    __shared__ float bs[kBlk];
    const Unit u = unit_of(a);
    const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
    const int H = a.H, dk = a.dk, dv = a.dv, dvp = a.nsl * kCols;
    const bool row = i < dk;
    const T *qp = static_cast<const T *>(a.q);
    const T *kp = static_cast<const T *>(a.k);
    const T *dop = static_cast<const T *>(a.dO);

    float G[kCols];  // dL/dS of the current token's output state, this row and slice
#pragma unroll
    for (int j = 0; j < kCols; ++j)
        G[j] = (a.dS_final && row && u.c0 + j < dv) ? a.dS_final[((int64_t(u.s) * H + u.h) * dk + i) * dv + u.c0 + j]
                                                     : 0.f;
    int rp = 0;
    const int64_t nb = (u.ce - u.cs + kBlk - 1) / kBlk;
    for (int64_t bi = nb - 1; bi >= 0; --bi) {
        const int64_t t0 = u.cs + bi * kBlk;
        const int n = int(min(int64_t(kBlk), u.ce - t0));
        __syncthreads();  // the previous block's reads of ws, dos and bs are done
        {  // w and dO of the block's tokens: every load issued before any is stored
            constexpr int kPer = kBlk * kCols / kRows;
            float xw[kPer], xd[kPer];
#pragma unroll
            for (int c = 0; c < kPer; ++c) {
                const int e = i + c * kRows, tt = e / kCols, j = e % kCols;
                const bool in = tt < n;
                xw[c] = in ? a.w[((t0 + tt) * H + u.h) * dvp + u.c0 + j] : 0.f;
                xd[c] = (in && u.c0 + j < dv) ? ldf(dop + ((t0 + tt) * H + u.h) * dv + u.c0 + j) : 0.f;
            }
#pragma unroll
            for (int c = 0; c < kPer; ++c) {
                const int e = i + c * kRows;
                ws[e / kCols][e % kCols] = xw[c];
                dos[e / kCols][e % kCols] = xd[c];
            }
        }
        if (i < kBlk) bs[i] = i < n ? a.beta[(t0 + i) * H + u.h] : 0.f;
        for (int t8 = 0; t8 < kBlk; t8 += 8) {  // this thread's row, eight tokens' loads at a time (no barrier needed)
            float la[8];
            T kx[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const bool in = row && t8 + j < n;
                const int64_t r = ((t0 + t8 + j) * H + u.h) * dk + i;
                la[j] = in ? a.log_alpha[r] : 0.f;
                kx[j] = in ? kp[r] : T(0.f);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) als[t8 + j][i] = expf(la[j]), ks[t8 + j][i] = kx[j];
        }
        __syncthreads();
        const float4 *ckp = ck_slice(a, u, bi);
        // S <- Diag(alpha_tt) S + beta_tt k_tt w_tt^T, from the stored w
        auto replay = [&](float(&S)[kCols], int tt) {
            const float al = als[tt][i];
            const float kb = ldf(&ks[tt][i]) * bs[tt];
#pragma unroll
            for (int j = 0; j < kCols; ++j) S[j] = fmaf(kb, ws[tt][j], al * S[j]);
        };
        if (n > kMid) {  // the state before the block's middle token, for the later sub-blocks
            float S[kCols];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 x = ckp[q4 * kRows + i];
                S[4 * q4] = x.x, S[4 * q4 + 1] = x.y, S[4 * q4 + 2] = x.z, S[4 * q4 + 3] = x.w;
            }
#pragma unroll 4
            for (int tt = 0; tt < kMid; ++tt) replay(S, tt);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) midst[q4][i] = make_float4(S[4 * q4], S[4 * q4 + 1], S[4 * q4 + 2], S[4 * q4 + 3]);
        }
        const int nsb = (n + kSub - 1) / kSub;
        for (int sb = nsb - 1; sb >= 0; --sb) {
            // replay from the nearest checkpoint to the sub-block's first token, then record
            // the input state of each of its tokens (each thread touches only its own row)
            const int first = sb * kSub, m_n = min(kSub, n - first);
            const int from = first >= kMid ? kMid : 0;
            float qpre[kSub];
#pragma unroll
            for (int m = 0; m < kSub; ++m)
                qpre[m] = (row && m < m_n) ? ldf(qp + ((t0 + first + m) * H + u.h) * dk + i) : 0.f;
            float S[kCols];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 x = from ? midst[q4][i] : ckp[q4 * kRows + i];
                S[4 * q4] = x.x, S[4 * q4 + 1] = x.y, S[4 * q4 + 2] = x.z, S[4 * q4 + 3] = x.w;
            }
#pragma unroll 4
            for (int tt = from; tt < first + m_n - 1; ++tt) {
                if (tt >= first) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        hist[tt - first][q4][i] = make_float4(S[4 * q4], S[4 * q4 + 1], S[4 * q4 + 2], S[4 * q4 + 3]);
                }
                const float al = als[tt][i];
                const float kb = ldf(&ks[tt][i]) * bs[tt];
#pragma unroll
                for (int j = 0; j < kCols; ++j) S[j] = fmaf(kb, ws[tt][j], al * S[j]);
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                hist[m_n - 1][q4][i] = make_float4(S[4 * q4], S[4 * q4 + 1], S[4 * q4 + 2], S[4 * q4 + 3]);

#pragma unroll
            for (int m = kSub - 1; m >= 0; --m) {
                if (m >= m_n) continue;
                const int tt = first + m;
                const int64_t t = t0 + tt;
                const float al = als[tt][i];
                const float kk = ldf(&ks[tt][i]);
                const float qq = qpre[m];
                const float b = bs[tt];
                float P[kCols], c[kCols];
                float pq = 0.f, dka = 0.f;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 x = hist[m][q4][i];
                    P[4 * q4] = al * x.x, P[4 * q4 + 1] = al * x.y, P[4 * q4 + 2] = al * x.z, P[4 * q4 + 3] = al * x.w;
                }
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    const float e = b * ws[tt][j], d = dos[tt][j];
                    G[j] = fmaf(qq, d, G[j]);
                    pq = fmaf(fmaf(kk, e, P[j]), d, pq);  // (S_t do_t)_i
                    dka = fmaf(G[j], e, dka);
                    c[j] = G[j] * kk;
                }
                float de[kCols];
                column_sums(c, red[rp], warp, lane, de);  // de = G^T k_t over this slice
                rp ^= 1;
                float db = 0.f, dkb = 0.f, dg = 0.f;
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    db = fmaf(de[j], ws[tt][j], db);
                    const float du = -b * de[j];
                    const float dP = fmaf(kk, du, G[j]);
                    dkb = fmaf(P[j], du, dkb);
                    dg = fmaf(dP, P[j], dg);
                    G[j] = al * dP;
                }
                if (i < kCols && u.c0 + i < dv) a.dv_out[(t * H + u.h) * dv + u.c0 + i] = b * pick(de, i);
                const int64_t pr = (t * H + u.h) * dk + i;  // the 8 slices' sums meet in L2
                if (row) {
                    atomicAdd(a.dq + pr, pq);
                    atomicAdd(a.dk_out + pr, dka + dkb);
                    atomicAdd(a.dla + pr, dg);
                }
                if (i == 0) atomicAdd(a.dbeta + t * H + u.h, db);
            }
        }
    }
    if (a.dS0 && row) {
#pragma unroll
        for (int j = 0; j < kCols; ++j)
            if (u.c0 + j < dv) a.dS0[((int64_t(u.s) * H + u.h) * dk + i) * dv + u.c0 + j] = G[j];
    }
}

template <typename T>
cudaError_t launch_backward_t(const BwdArgs &a, cudaStream_t st) {
    const unsigned grid = unsigned(int64_t(a.num_seqs) * a.H * a.nsl);
    const unsigned sgrid = unsigned(int64_t(a.num_seqs) * a.H * ((a.nsl + kSw - 1) / kSw));
    bwd_states_kernel<T><<<sgrid, kSw * 32, 0, st>>>(a);
    constexpr int dyn = kBlk * kRows * int(sizeof(float) + sizeof(T));
    cudaError_t err = cudaFuncSetAttribute(bwd_grads_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (err != cudaSuccess) return err;
    if (a.T > 0) {
        const size_t n = size_t(a.T) * a.H * a.dk * sizeof(float);
        for (float *p : {a.dq, a.dk_out, a.dla}) {
            err = cudaMemsetAsync(p, 0, n, st);
            if (err != cudaSuccess) return err;
        }
        err = cudaMemsetAsync(a.dbeta, 0, size_t(a.T) * a.H * sizeof(float), st);
        if (err != cudaSuccess) return err;
    }
    bwd_grads_kernel<T><<<grid, kRows, dyn, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

size_t kda_backward_workspace_size(int num_seqs, int64_t total_tokens, int H, int d_k, int d_v) {
    if (num_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX || H < 1 || d_k < 1 || d_k > 128 || d_v < 1 ||
        d_v > 128)
        return 0;
    return bwd_layout(num_seqs, total_tokens, H, d_k, d_v).total;
}

kda_status_t kda_backward(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype, const float *log_alpha,
                          const float *beta, const float *S0, const int32_t *cu_seqlens_dev,
                          const int32_t *cu_seqlens_host, int num_seqs, int H, int d_k, int d_v, const void *dO,
                          const float *dS_final, float *dq, float *dk, float *dv, float *dlog_alpha, float *dbeta,
                          float *dS0, void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    if (num_seqs < 0 || H < 1 || d_k < 1 || d_v < 1) return KDA_ERR_INVALID_ARG;
    if (qkv_dtype != KDA_DTYPE_F32 && qkv_dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (d_k > 128 || d_v > 128) return KDA_ERR_UNSUPPORTED;
    if (int64_t(num_seqs) * H * ((d_v + kCols - 1) / kCols) > INT32_MAX) return KDA_ERR_UNSUPPORTED;  // grid size
    if (!cu_seqlens_host || !cu_seqlens_dev) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host[0] != 0) return KDA_ERR_INVALID_ARG;
    for (int n = 0; n < num_seqs; ++n)
        if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return KDA_ERR_INVALID_ARG;
    const int64_t T = cu_seqlens_host[num_seqs];
    if (T > 0 && (!q || !k || !v || !log_alpha || !beta || !dO || !dq || !dk || !dv || !dlog_alpha || !dbeta))
        return KDA_ERR_INVALID_ARG;
    const BwdLayout L = bwd_layout(num_seqs, T, H, d_k, d_v);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return KDA_ERR_WORKSPACE;
    if (num_seqs == 0) return KDA_OK;

    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.dO = dO;
    a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.dS_final = dS_final;
    a.cu_seqlens = cu_seqlens_dev;
    a.num_seqs = num_seqs; a.H = H; a.dk = d_k; a.dv = d_v; a.nsl = (d_v + kCols - 1) / kCols;
    a.T = T;
    a.dq = dq; a.dk_out = dk; a.dv_out = dv; a.dla = dlog_alpha; a.dbeta = dbeta; a.dS0 = dS0;
    char *base = static_cast<char *>(workspace);
    a.ck = reinterpret_cast<float4 *>(base + L.ck_offset);
    a.w = reinterpret_cast<float *>(base + L.w_offset);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = qkv_dtype == KDA_DTYPE_F32 ? launch_backward_t<float>(a, st)
                                                     : launch_backward_t<__nv_bfloat16>(a, st);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
