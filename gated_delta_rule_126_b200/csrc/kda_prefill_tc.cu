// Tensor-core (tcgen05) chunked KDA prefill: bf16 q/k/v, d_k = d_v = 128, chunk 64.
//
// Operator: state-update equation of the KDA section of the wiki page "Kimi Linear
// 高效注意力架构" ("Kimi Delta Attention (KDA)"), read-out o_t = S_t^T q_t, evaluated
// chunk by chunk in the WY/UT form (the chunkwise algorithm of the same section's
// "硬件高效分块算法" bullet; its cost terms T d_k d_v + T C d + T C^2 are the
// comparison table's).  Within a chunk of L <= 64 tokens starting from state S,
// with g the inclusive running sum of log alpha per key channel:
//   A_ri = beta_r <k_r e^{g_r - g_i}, k_i> (i < r),   T = (I + A)^{-1} Diag(beta)
//   P_ri = <q_r e^{g_r - g_i}, k_i> (i <= r)
//   U = T (V - (K e^{g}) S),   O = (Q e^{g}) S + P U,   S <- Diag(e^{g_L}) S + (K e^{g_L - g})^T U
//
// Design (one CTA of 384 threads per (sequence, head), walking its chunks):
// * The fp32 state is kept TRANSPOSED in tensor memory (TMEM lane = value column
//   j, 128 lanes) for the whole sequence, so every product of the chunk step is a
//   128-row UMMA with d_v on the M side.  With Kt = K e^{g-g_m}, Qt = Q e^{g-g_m},
//   Kb = K e^{g_m-g} (g_m: the chunk's middle token, so both factors stay within
//   e^{+-|g_L|/2}) and the fp16 state operand Sop = S^T Diag(e^{g_m}):
//     M1  [A; P]^raw = [Kt; Qt] Kb^T                 M=128 N=64  K=128
//     M2  Z          = Sop [Kt; Qt]^T                M=128 N=128 K=128
//           Z[:, :64] = (K e^{g} S)^T,  Z[:, 64:] = (Q e^{g} S)^T
//     Mv  Z[:, :64] += V^T (-I)     (V read MN-major from its TMA tile)   N=64 K=64
//     M3  U^T        = Y^T T^T,  Y^T = -Z[:, :64]    M=128 N=64  K=64
//     M4  R         += U^T Kb      (Kb read as an MN-major operand)  N=128 K=64
//     M5  Z[:, 64:] += U^T P^T  ( = O^T )                   N=64  K=64
//   TMEM holds R = S^T Diag(e^{g_m - g_L}) of the previous chunk rather than S^T:
//   the per-channel factors e^{g_L - g_m} and e^{g_m} then fold into one pass over
//   R at the start of each chunk, which also packs Sop, so no K e^{g}, Q e^{g} or
//   (K e^{g_L - g})^T tile is built.  Y^T and U^T are written back to TMEM as fp16
//   pairs (over Sop, which M2 has read), so M3-M5 take their A operand from TMEM.
// * Two warp groups work on different chunks at once.  The prep group (warps
//   4-11) builds chunk c + 1 -- decayed rows, M1, A and P, and X = (I + A)^{-1} --
//   while the state group (warps 0-3) runs chunk c -- the pass over R, M2, Y,
//   T = X Diag(beta), M3, U, M4/M5 and the outputs -- and, while it waits for X,
//   the running sums of chunk c + 1.  They hand buffers over through
//   release/acquire progress counters in shared memory; the decayed-row (Kb) and P
//   tiles and the per-chunk vectors are double-buffered by chunk parity.
// * Operands are fp16 (fp32 accumulation): the S-dependent chain keeps the
//   relative error near fp16's 2^-11, which the parity bounds need (bf16 operands
//   do not meet them).
// * q, k, v and log alpha tiles arrive by TMA in the 128-byte swizzled layout that
//   the UMMA descriptors use, so the decayed operand rows are built in place.  A
//   full chunk's outputs leave by two TMA tile stores; a shorter last chunk row by
//   row (its later rows belong to the next sequence).
// * X is formed in fp32 in shared memory by block doubling: the four 16x16
//   diagonal blocks by row substitution, then the two 32x32 halves, then the
//   lower-left 32x32 block, every stage on all 256 prep threads.
// * kGated applies the layer's output epilogue (sigmoid gate and RMSNorm) before
//   the output store; kSplit runs the units of a sequence split (kda_internal.h).
// * Every wait is bounded: one that runs out sets the workspace error flag and
//   both groups stop at their next group barrier (decided uniformly by a
//   barrier-or), drain what they have in flight and free TMEM.
#include <cuda.h>

#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

constexpr int C = 64;    // chunk
constexpr int D = 128;   // d_k = d_v
constexpr int NS = 128;  // state group: warps 0-3
constexpr int NP = 256;  // prep group: warps 4-11
constexpr int NT = NS + NP;
constexpr uint32_t BAR_S = 1, BAR_P = 2;  // named barriers of the two groups

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_QK = 0;        // raw k|q boxes -> [Kt; Qt]  (128 x 128 fp16, K-major)
constexpr uint32_t OFF_LA = 32768;    // raw log alpha boxes -> g (fp32, 64 x 128)
constexpr uint32_t OFF_V = 65536;     // raw v boxes (bf16, 64 x 128)
constexpr uint32_t OFF_KB = 81920;    // Kb (64 x 128 fp16), two buffers
constexpr uint32_t OFF_SCR = 114688;  // fp32 scratch of the triangular solve
constexpr int LDF = 68;
constexpr int LDE = 20;
constexpr uint32_t OFF_AF = OFF_SCR;
constexpr uint32_t OFF_XF = OFF_AF + 64 * LDF * 4;
constexpr uint32_t OFF_EB = OFF_XF + 64 * LDF * 4;  // X_11 A_10 and X_33 A_32; then X_H1 A_21
constexpr int LDG = 33;
constexpr uint32_t OFF_P = 157696;    // P (64 x 64 fp16), two buffers
static_assert(OFF_EB + 32 * LDE * 4 <= OFF_P && OFF_EB + 32 * LDG * 4 <= OFF_P, "solve scratch overflows");
constexpr uint32_t OFF_T = OFF_P + 16384;    // T (64 x 64 fp16)
constexpr uint32_t OFF_Y = OFF_T + 8192;     // the bf16 output tile (two 64 x 64 boxes)
constexpr uint32_t OFF_ID = OFF_Y + 16384;   // -I (64 x 64 bf16): loads -V^T into Z with an MMA
constexpr uint32_t OFF_VEC = OFF_ID + 8192;  // per-chunk vectors, two buffers (chunk parity)
constexpr uint32_t VEC_GM = 0;        // g_m                  128 f32
constexpr uint32_t VEC_EGM = 512;     // e^{g_m}
constexpr uint32_t VEC_ECM = 1024;    // e^{g_L - g_m}
constexpr uint32_t VEC_BETA = 1536;   // beta                 64 f32
constexpr uint32_t VEC_FAC = 1792;    // e^{g_L - g_m}(previous chunk) e^{g_m}: the pass over R
constexpr uint32_t VEC_BYTES = 2304;
constexpr uint32_t OFF_BAR = OFF_VEC + 2 * VEC_BYTES;   // mbarriers
constexpr int NBAR = 8;
constexpr int B_QK = 0, B_LA = 1, B_V = 2, B_M1 = 3, B_M2 = 4, B_M3 = 5, B_M45 = 6, B_G = 7;
constexpr uint32_t OFF_CNT = OFF_BAR + 8 * NBAR;        // progress counters
constexpr int CNT_ROWS = 0, CNT_TP = 1, CNT_SCAN = 2, CNT_M45 = 3, CNT_TW = 4;
constexpr uint32_t OFF_ISS = OFF_CNT + 32;              // phases issued / waited per mbarrier
constexpr uint32_t OFF_WT = OFF_ISS + 4 * NBAR;
constexpr uint32_t OFF_MISC = OFF_WT + 4 * NBAR;        // tmem base, abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
// Running-sum totals of the 4 token blocks (2 KB): over the output tile, which is idle
// between the wait for its last TMA store (top of a chunk) and the next E4.
constexpr uint32_t OFF_PART = OFF_Y;
// The gated output epilogue adds the gate tile (bf16, two 64 x 64 boxes) and the
// per-token reduction of o^2 (4 x 64 partial sums, then 64 reciprocal RMS values).
constexpr uint32_t OFF_G = (SMEM_USED + 1023) / 1024 * 1024;
constexpr uint32_t OFF_RED = OFF_G + 16384;
constexpr uint32_t SMEM_USED_G = OFF_RED + 320 * 4;
constexpr uint32_t smem_alloc(bool gated) { return (gated ? SMEM_USED_G : SMEM_USED) + 1024; }  // + alignment slack
static_assert(smem_alloc(true) <= 232448, "shared memory");

// Tensor memory columns.
constexpr uint32_t TS = 0;      // R (fp32)          128 cols   state group
constexpr uint32_t TZ = 128;    // Z fp32            128 cols   state group
constexpr uint32_t TU = 256;    // U^T fp32           64 cols   state group
constexpr uint32_t TAP = 320;   // [A; P] raw fp32    64 cols   prep group
constexpr uint32_t TSOP = 384;  // Sop fp16           64 cols   state group
constexpr uint32_t TY16 = TSOP;       // Y^T fp16, 32 cols, over Sop once M2 has read it
constexpr uint32_t TU16 = TSOP + 32;  // U^T fp16, 32 cols
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_N64 = ptx::idesc_f16_f32(128, 64);
constexpr uint32_t IDESC_N128 = ptx::idesc_f16_f32(128, 128);
constexpr uint32_t IDESC_N128_BMN = ptx::idesc_f16_f32(128, 128) | (1u << 16);  // B MN-major
// bf16 A (MN-major) and B, fp32 D, M = 128, N = 64
constexpr uint32_t IDESC_BF16_AMN_N64 = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (8u << 17) | (8u << 24);
constexpr long long kWaitCycles = 4000000000LL;  // about two seconds
constexpr float kLog2e = 1.4426950408889634f;

// byte offset of 16-byte chunk `ch` of row `r` in a 128-byte-row swizzled tile
__device__ __forceinline__ uint32_t sw(int r, int ch) { return uint32_t(r) * 128u + (uint32_t((ch ^ (r & 7))) << 4); }

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

struct TcMaps {
    CUtensorMap q, k, v, la, o, g;  // g: the output gate (gated epilogue only)
};

// kGated: the output store applies the layer's output epilogue, y = o / sqrt(mean_j o_j^2 + eps)
// * w * sigmoid(gate) per token and head (the KDA layer's sigmoid output gate and RMSNorm,
// section "模型架构" of the same page), instead of storing o.
// kSplit: the launch runs units of a sequence split (kda_internal.h) before the plain
// (sequence, head) units; plain launches compile without the per-unit modes.
template <bool kGated, bool kSplit>
__global__ void __launch_bounds__(NT, 1)
    prefill_tc_kernel(const __grid_constant__ TcMaps maps, const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = ptx::smem_u32(smem_raw);
    const uint32_t pad = ((raw_s + 1023u) & ~1023u) - raw_s;
    uint8_t *sm = smem_raw + pad;
    const uint32_t sb = raw_s + pad;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int h = blockIdx.x % H;
    // The unit: a split segment (the first a.split.num_units) or a plain sequence.
    constexpr size_t D2 = size_t(D) * D;
    const int ui = blockIdx.x / H;
    int seq, bos, eos, mode = 0;
    const float *s0 = nullptr;  // initial state [d_k][d_v] (nullptr: zero, or the identity for UNIT_HOMOG)
    float *sfin = nullptr;      // where the final state goes (nullptr: nowhere)
    if (kSplit && ui < a.split.num_units) {
        const SplitUnit u = a.split.units[ui];
        seq = u.seq;
        bos = u.bos;
        eos = u.eos;
        mode = u.mode;
        const size_t slot = size_t(u.slot) * H + h;
        if (mode == UNIT_FIRST) {
            s0 = a.S0 ? a.S0 + (size_t(seq) * H + h) * D2 : nullptr;
            sfin = a.split.sstart + (slot + H) * D2;  // the next segment's start state
        } else if (mode == UNIT_LOCAL) {
            sfin = a.split.lmat + slot * D2;
        } else if (mode == UNIT_HOMOG) {
            sfin = a.split.mmat + slot * D2;
        } else {  // UNIT_CONT, UNIT_LAST
            s0 = a.split.sstart + slot * D2;
            if (mode == UNIT_LAST) sfin = a.S_final + (size_t(seq) * H + h) * D2;
        }
    } else {
        seq = a.order[ui - (kSplit ? a.split.num_units : 0)];
        if (kSplit)
            for (int j = 0; j < a.split.num_seqs; ++j)
                if (a.split.seqs[j] == seq) return;  // run by the split units (the same for the whole block)
        bos = a.cu_seqlens[seq];
        eos = a.cu_seqlens[seq + 1];
        s0 = a.S0 ? a.S0 + (size_t(seq) * H + h) * D2 : nullptr;
        sfin = a.S_final + (size_t(seq) * H + h) * D2;
    }
    const bool v_zero = kSplit && mode == UNIT_HOMOG;                       // the transition runs with v = 0
    const bool o_skip = kSplit && (mode == UNIT_LOCAL || mode == UNIT_HOMOG);  // only the final state is wanted
    const int nchunks = (eos - bos + C - 1) / C;

    auto vec = [&](int par, uint32_t field) { return reinterpret_cast<float *>(sm + OFF_VEC + par * VEC_BYTES + field); };
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *cnt = reinterpret_cast<uint32_t *>(sm + OFF_CNT);
    uint32_t *iss = reinterpret_cast<uint32_t *>(sm + OFF_ISS);
    uint32_t *wt = reinterpret_cast<uint32_t *>(sm + OFF_WT);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    int *s_abort = reinterpret_cast<int *>(sm + OFF_MISC + 4);

    if (warp == 0) {
        ptx::tmem_alloc(s_tmem, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (tid == 32) {
        for (int b = 0; b < NBAR; ++b) {
            ptx::mbar_init(bars + b, 1);
            iss[b] = 0;
            wt[b] = 0;
        }
        for (int i = 0; i < 8; ++i) cnt[i] = 0;
        ptx::fence_mbar_init();
        *s_abort = 0;
        *reinterpret_cast<float **>(sm + OFF_MISC + 8) = sfin;  // read back at the end (frees registers)
        ptx::prefetch_tmap(&maps.q);
        ptx::prefetch_tmap(&maps.k);
        ptx::prefetch_tmap(&maps.v);
        ptx::prefetch_tmap(&maps.la);
        ptx::prefetch_tmap(&maps.o);
        if (kGated) ptx::prefetch_tmap(&maps.g);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tbase = *s_tmem;

    auto load_qk = [&](int s) {
        ptx::mbar_arrive_expect_tx(bars + B_QK, 4 * 8192);
        ptx::tma_load_3d(sm + OFF_QK, &maps.k, bars + B_QK, 0, h, s);
        ptx::tma_load_3d(sm + OFF_QK + 8192, &maps.q, bars + B_QK, 0, h, s);
        ptx::tma_load_3d(sm + OFF_QK + 16384, &maps.k, bars + B_QK, 64, h, s);
        ptx::tma_load_3d(sm + OFF_QK + 24576, &maps.q, bars + B_QK, 64, h, s);
        ++iss[B_QK];
    };
    auto load_la = [&](int s) {
        ptx::mbar_arrive_expect_tx(bars + B_LA, 4 * 8192);
        for (int b = 0; b < 4; ++b) ptx::tma_load_3d(sm + OFF_LA + b * 8192, &maps.la, bars + B_LA, 32 * b, h, s);
        ++iss[B_LA];
    };
    auto load_v = [&](int s) {
        ptx::mbar_arrive_expect_tx(bars + B_V, 2 * 8192);
        ptx::tma_load_3d(sm + OFF_V, &maps.v, bars + B_V, 0, h, s);
        ptx::tma_load_3d(sm + OFF_V + 8192, &maps.v, bars + B_V, 64, h, s);
        ++iss[B_V];
    };
    auto load_g = [&](int s) {
        ptx::mbar_arrive_expect_tx(bars + B_G, 2 * 8192);
        ptx::tma_load_3d(sm + OFF_G, &maps.g, bars + B_G, 0, h, s);
        ptx::tma_load_3d(sm + OFF_G + 8192, &maps.g, bars + B_G, 64, h, s);
        ++iss[B_G];
    };
    auto commit = [&](int b) {
        ptx::mma_commit(bars + b);
        ++iss[b];
    };
    auto fail = [&]() {
        atomicExch(&a.status->flag, 1u);
        *s_abort = 1;
    };
    // Wait for phase `phase` of mbarrier b (bounded, gives up on an abort).
    // `leader` records the wait for the drain on abort.
    auto mwait = [&](int b, uint32_t phase, bool leader) {
        const long long t0 = clock64();
        while (!ptx::mbar_try_wait(bars + b, phase & 1u)) {
            if (*reinterpret_cast<volatile int *>(s_abort) || clock64() - t0 > kWaitCycles) {
                fail();
                return false;
            }
        }
        if (leader) wt[b] = phase + 1;
        return true;
    };
    // Wait until progress counter i reaches `target` (bounded, gives up on an abort).
    auto cwait = [&](int i, uint32_t target) {
        if (ptx::ld_acquire(cnt + i) >= target) return true;
        const long long t0 = clock64();
        while (ptx::ld_acquire(cnt + i) < target) {
            if (*reinterpret_cast<volatile int *>(s_abort) || clock64() - t0 > kWaitCycles) {
                fail();
                return false;
            }
            __nanosleep(20);
        }
        return true;
    };

    // Launched with 384 x 168 registers: the prep group (8 warps) drops to 128, the
    // state group (4 warps) rises to 240; 4 x 32 x 240 + 8 x 32 x 128 <= 384 x 168.
    if (warp < 4) {
        // =================================================================== state group
        ptx::regs_inc<240>();
        const int row = tid;  // TMEM lane = value column j
        const uint32_t tl = tbase + (uint32_t(warp * 32) << 16);
        const bool leader = tid == 0;
        if (leader && nchunks > 0) {
            if (!v_zero) load_v(bos);
            if (kGated) load_g(bos);
        }
        const float w_row = kGated ? a.norm_weight[row] : 0.f;  // RMSNorm weight of value channel `row`
        {  // -I as a K-major bf16 operand (rows r, K = i), for Z[:, :64] = V^T (-I)
            uint4 *id = reinterpret_cast<uint4 *>(sm + OFF_ID);
            for (int t = tid; t < 512; t += NS) id[t] = make_uint4(0u, 0u, 0u, 0u);
            ptx::named_barrier(BAR_S, NS);
            if (tid < 64) *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_ID + sw(tid, tid >> 3) + (tid & 7) * 2) =
                __float2bfloat16_rn(-1.f);
            ptx::fence_proxy_async_smem();
        }
        {  // R = S0^T
            uint32_t v[32];
            for (int p = 0; p < 4; ++p) {
                for (int e = 0; e < 32; ++e) {
                    const int c = 32 * p + e;
                    if constexpr (kSplit)
                        v[e] = __float_as_uint(s0 ? s0[c * D + row] : (v_zero && c == row ? 1.f : 0.f));
                    else
                        v[e] = __float_as_uint(a.S0 ? a.S0[((size_t(seq) * H + h) * D + c) * D + row] : 0.f);
                }
                ptx::tmem_st32(tl + TS + 32 * p, v);
            }
            ptx::tmem_wait_st();
        }
        // ---- P1 of chunk cj: g = running sum of log alpha per channel, in base 2 (g log2 e)
        // in place over the log alpha tile, and the chunk's vectors (buffer cj & 1): g_m
        // (base 2), e^{g_m}, e^{g_L - g_m}, the factors of the pass over R and beta.  Warp w
        // sums tokens 16w .. 16w + 15 for four channels a lane (float4 rows); the warps'
        // totals meet in shared memory.  beta is read from global memory one chunk ahead.
        auto load_beta = [&](int cj) {
            const int s = bos + cj * C;
            return (tid < C && cj < nchunks && s + tid < eos) ? a.beta[size_t(s + tid) * H + h] : 0.f;
        };
        float beta_reg = load_beta(0);
        auto scan = [&](int cj) {
            const int L = min(C, eos - (bos + cj * C));
            const int par = cj & 1;
            const int wq = warp, c0 = 4 * lane, lch = lane & 7;
            uint8_t *tile = sm + OFF_LA + (lane >> 3) * 8192;  // box holding channels c0 .. c0 + 3
            const int rm = (L - 1) >> 1;
            mwait(B_LA, cj, leader);
            float4 x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * wq + i;
                x[i] = r < L ? *reinterpret_cast<const float4 *>(tile + sw(r, lch)) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            x[0] = make_float4(x[0].x * kLog2e, x[0].y * kLog2e, x[0].z * kLog2e, x[0].w * kLog2e);
#pragma unroll
            for (int i = 1; i < 16; ++i)
                x[i] = make_float4(fmaf(x[i].x, kLog2e, x[i - 1].x), fmaf(x[i].y, kLog2e, x[i - 1].y),
                                   fmaf(x[i].z, kLog2e, x[i - 1].z), fmaf(x[i].w, kLog2e, x[i - 1].w));
            float4 *part = reinterpret_cast<float4 *>(sm + OFF_PART);
            part[wq * 32 + lane] = x[15];
            ptx::named_barrier(BAR_S, NS);
            float4 off = make_float4(0.f, 0.f, 0.f, 0.f), tot = off;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float4 p = part[w * 32 + lane];
                if (w < wq) off = make_float4(off.x + p.x, off.y + p.y, off.z + p.z, off.w + p.w);
                tot = make_float4(tot.x + p.x, tot.y + p.y, tot.z + p.z, tot.w + p.w);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = make_float4(x[i].x + off.x, x[i].y + off.y, x[i].z + off.z, x[i].w + off.w);
                *reinterpret_cast<float4 *>(tile + sw(16 * wq + i, lch)) = x[i];
            }
            if (wq == (rm >> 4)) {  // the warp holding token rm writes the chunk's vectors
                const float4 gm = *reinterpret_cast<const float4 *>(tile + sw(rm, lch));  // stored above by this thread
                const float4 e = make_float4(exp2f(gm.x), exp2f(gm.y), exp2f(gm.z), exp2f(gm.w));
                // g_L = tot: rows >= L add 0
                const float4 ecm = make_float4(exp2f(tot.x - gm.x), exp2f(tot.y - gm.y), exp2f(tot.z - gm.z),
                                               exp2f(tot.w - gm.w));
                const float4 prev = cj > 0 ? *reinterpret_cast<const float4 *>(vec(par ^ 1, VEC_ECM) + c0)
                                           : make_float4(1.f, 1.f, 1.f, 1.f);
                *reinterpret_cast<float4 *>(vec(par, VEC_GM) + c0) = gm;
                *reinterpret_cast<float4 *>(vec(par, VEC_EGM) + c0) = e;
                *reinterpret_cast<float4 *>(vec(par, VEC_ECM) + c0) = ecm;
                *reinterpret_cast<float4 *>(vec(par, VEC_FAC) + c0) =
                    make_float4(prev.x * e.x, prev.y * e.y, prev.z * e.z, prev.w * e.w);
            }
            if (tid < C) vec(par, VEC_BETA)[tid] = beta_reg;
            beta_reg = load_beta(cj + 1);
            ptx::fence_proxy_async_smem();  // the next log alpha tile overwrites g by TMA
        };
        if (nchunks > 0) {
            scan(0);
            ptx::named_barrier(BAR_S, NS);
            if (leader) ptx::st_release(cnt + CNT_SCAN, 1u);
        }
        for (int ci = 0; ci < nchunks; ++ci) {
            const int s = bos + ci * C;
            const int L = min(C, eos - s);
            const bool has_next = ci + 1 < nchunks;
            const int par = ci & 1;

            // ---- E0: R *= e^{g_L - g_m}(previous chunk) e^{g_m}; Sop = fp16(R).
            {
                const float4 *fac = reinterpret_cast<const float4 *>(vec(par, VEC_FAC));
                uint32_t r4[4][32], pk[16];
#pragma unroll
                for (int p = 0; p < 4; ++p) ptx::tmem_ld32(tl + TS + 32 * p, r4[p]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 2; ++p) {  // 64 columns at a time
                    uint32_t(&v)[32] = r4[2 * p];
                    uint32_t(&w)[32] = r4[2 * p + 1];
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 f0 = fac[16 * p + e4], f1 = fac[16 * p + 8 + e4];
                        v[4 * e4 + 0] = __float_as_uint(__uint_as_float(v[4 * e4 + 0]) * f0.x);
                        v[4 * e4 + 1] = __float_as_uint(__uint_as_float(v[4 * e4 + 1]) * f0.y);
                        v[4 * e4 + 2] = __float_as_uint(__uint_as_float(v[4 * e4 + 2]) * f0.z);
                        v[4 * e4 + 3] = __float_as_uint(__uint_as_float(v[4 * e4 + 3]) * f0.w);
                        w[4 * e4 + 0] = __float_as_uint(__uint_as_float(w[4 * e4 + 0]) * f1.x);
                        w[4 * e4 + 1] = __float_as_uint(__uint_as_float(w[4 * e4 + 1]) * f1.y);
                        w[4 * e4 + 2] = __float_as_uint(__uint_as_float(w[4 * e4 + 2]) * f1.z);
                        w[4 * e4 + 3] = __float_as_uint(__uint_as_float(w[4 * e4 + 3]) * f1.w);
                    }
                    ptx::tmem_st32(tl + TS + 64 * p, v);
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_h2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                    ptx::tmem_st16(tl + TSOP + 32 * p, pk);
                    ptx::tmem_st32(tl + TS + 64 * p + 32, w);
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_h2(__uint_as_float(w[2 * e]), __uint_as_float(w[2 * e + 1]));
                    ptx::tmem_st16(tl + TSOP + 32 * p + 16, pk);
                }
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            if (leader) ptx::bulk_wait_read0();
            if (ptx::named_barrier_or(BAR_S, NS, *s_abort != 0)) break;
            if (leader) {
                cwait(CNT_ROWS, ci + 1);  // [Kt; Qt] of this chunk
                ptx::tc_fence_after();
                // Z = Sop [Kt; Qt]^T (the k and q boxes of a channel block are rows 0-63 and
                // 64-127 of one 128-row operand), then Z[:, :64] += V^T (-I), V read MN-major
                // from its TMA tile
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kq = uint32_t(ks >> 2) * 16384u + uint32_t(ks & 3) * 32u;
                    ptx::mma_ts(tbase + TZ, tbase + TSOP + 8 * ks, ptx::sdesc_sw128(sb + OFF_QK + kq), IDESC_N128,
                                ks > 0);
                }
                if (!v_zero) {
                    mwait(B_V, ci, true);
                    ptx::tc_fence_after();
                    for (int ks = 0; ks < 4; ++ks)
                        ptx::mma_ss(tbase + TZ, ptx::sdesc_sw128_mn(sb + OFF_V + 2048 * ks, 8192, 1024),
                                    ptx::sdesc_sw128(sb + OFF_ID + 32 * ks), IDESC_BF16_AMN_N64, 1u);
                }
                commit(B_M2);
            }
            mwait(B_M2, ci, leader);
            ptx::tc_fence_after();
            if (leader) {
                if (has_next && !v_zero) load_v(s + C);  // the V tile has been read by the MMA
                // the [Kt; Qt] tile is free once M1 of this chunk has read it too
                if (has_next && mwait(B_M1, ci, false)) load_qk(s + C);
            }

            // ---- E2: Y^T = -Z[:, :64] = V^T - (K e^{g} S)^T -> fp16 pairs in TMEM, the A
            // operand of M3 (rows i >= L of V are never used: T's columns i >= L are zero).
            {
                uint32_t vz[2][32], pk[16];
                ptx::tmem_ld32(tl + TZ, vz[0]);
                ptx::tmem_ld32(tl + TZ + 32, vz[1]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 2; ++p) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_h2(-__uint_as_float(vz[p][2 * e]), -__uint_as_float(vz[p][2 * e + 1]));
                    ptx::tmem_st16(tl + TY16 + 16 * p, pk);
                }
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            // P1 of the next chunk.  Its vectors go to the buffer of chunk ci - 1, which the
            // prep group last read in E1 of chunk ci - 1, before its rows of chunk ci.
            if (has_next) scan(ci + 1);
            if (ptx::named_barrier_or(BAR_S, NS, *s_abort != 0)) break;
            if (leader && has_next) ptx::st_release(cnt + CNT_SCAN, ci + 2);

            // ---- M3: U^T = Y^T T^T  (T of this chunk from the prep group).
            cwait(CNT_TP, ci + 1);
            {  // T[r][i] = X[r][i] beta_i for i <= r as an fp16 operand (rows r, K = i)
                const float *X = reinterpret_cast<const float *>(sm + OFF_XF);
                const float *beta = vec(par, VEC_BETA);
                const int rt = tid & 63, part = tid >> 6;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int ch = 4 * part + qq;
                    const float4 x0 = *reinterpret_cast<const float4 *>(X + rt * LDF + 8 * ch);
                    const float4 x1 = *reinterpret_cast<const float4 *>(X + rt * LDF + 8 * ch + 4);
                    const float4 b0 = *reinterpret_cast<const float4 *>(beta + 8 * ch);
                    const float4 b1 = *reinterpret_cast<const float4 *>(beta + 8 * ch + 4);
                    const float xs[8] = {x0.x * b0.x, x0.y * b0.y, x0.z * b0.z, x0.w * b0.w,
                                         x1.x * b1.x, x1.y * b1.y, x1.z * b1.z, x1.w * b1.w};
                    uint32_t pk[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const int i = 8 * ch + 2 * e2;
                        pk[e2] = pack_h2(i <= rt ? xs[2 * e2] : 0.f, i + 1 <= rt ? xs[2 * e2 + 1] : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(sm + OFF_T + sw(rt, ch)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            ptx::fence_proxy_async_smem();
            if (ptx::named_barrier_or(BAR_S, NS, *s_abort != 0)) break;
            if (leader) {
                ptx::st_release(cnt + CNT_TW, ci + 1);
                ptx::tc_fence_after();
                for (int ks = 0; ks < 4; ++ks)
                    ptx::mma_ts(tbase + TU, tbase + TY16 + 8 * ks, ptx::sdesc_sw128(sb + OFF_T + 32 * ks), IDESC_N64,
                                ks > 0);
                commit(B_M3);
            }
            mwait(B_M3, ci, leader);
            ptx::tc_fence_after();
            {  // E3: U^T -> fp16 pairs in TMEM, the A operand of M4 and M5
                uint32_t vu[2][32], pk[16];
                ptx::tmem_ld32(tl + TU, vu[0]);
                ptx::tmem_ld32(tl + TU + 32, vu[1]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 2; ++p) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_h2(__uint_as_float(vu[p][2 * e]), __uint_as_float(vu[p][2 * e + 1]));
                    ptx::tmem_st16(tl + TU16 + 16 * p, pk);
                }
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            if (ptx::named_barrier_or(BAR_S, NS, *s_abort != 0)) break;

            // ---- M4: R += U^T Kb;  M5: O^T = Z[:, 64:] + U^T P^T.
            if (leader) {
                ptx::tc_fence_after();
                const uint32_t kb_base = OFF_KB + par * 16384, p_base = OFF_P + par * 8192;
                for (int ks = 0; ks < 4; ++ks)
                    ptx::mma_ts(tbase + TS, tbase + TU16 + 8 * ks, ptx::sdesc_sw128_mn(sb + kb_base + 2048 * ks, 8192, 1024),
                                IDESC_N128_BMN, 1u);
                for (int ks = 0; ks < 4; ++ks)
                    ptx::mma_ts(tbase + TZ + 64, tbase + TU16 + 8 * ks, ptx::sdesc_sw128(sb + p_base + 32 * ks), IDESC_N64,
                                1u);
                commit(B_M45);
            }
            mwait(B_M45, ci, leader);
            ptx::tc_fence_after();
            if (leader) ptx::st_release(cnt + CNT_M45, ci + 1);
            if (!o_skip) {  // E4: outputs of this chunk, staged over the Y^T tile as two 128-byte
                            // swizzled boxes (columns 0-63, 64-127)
                uint32_t vo[2][32];
                uint8_t *stage = sm + OFF_Y + (row >> 6) * 8192 + (row & 7) * 2;
                const int ch = (row & 63) >> 3;
                ptx::tmem_ld32(tl + TZ + 64, vo[0]);
                ptx::tmem_ld32(tl + TZ + 96, vo[1]);
                ptx::tmem_wait_ld();
                if constexpr (kGated) {
                    // this thread's gate column (64 bf16, packed in pairs of tokens), loaded before
                    // the reduction below so that the loads overlap it
                    mwait(B_G, ci, leader);
                    const uint8_t *gt = sm + OFF_G + (row >> 6) * 8192 + (row & 7) * 2;
                    uint32_t gp[C / 2];
#pragma unroll
                    for (int i = 0; i < C / 2; ++i)
                        gp[i] = uint32_t(*reinterpret_cast<const unsigned short *>(gt + sw(2 * i, ch))) |
                                (uint32_t(*reinterpret_cast<const unsigned short *>(gt + sw(2 * i + 1, ch))) << 16);
                    // sum over the 128 value channels (one per thread) of o^2 for each of the 64
                    // tokens: a transposed butterfly leaves lane l holding tokens 2l and 2l + 1 of
                    // its warp's 32 channels; the four warps' partial sums meet in shared memory
                    float sq[C];
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int e = 0; e < 32; ++e) sq[32 * p + e] = __uint_as_float(vo[p][e]) * __uint_as_float(vo[p][e]);
#pragma unroll
                    for (int m = 16; m >= 1; m >>= 1) {  // 4m partial sums -> 2m
                        const bool hi = (lane & m) != 0;
#pragma unroll
                        for (int i = 0; i < 2 * m; ++i) {
                            const float send = hi ? sq[i] : sq[2 * m + i];
                            const float keep = hi ? sq[2 * m + i] : sq[i];
                            sq[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                        }
                    }
                    float *red = reinterpret_cast<float *>(sm + OFF_RED);
                    red[warp * 64 + 2 * lane] = sq[0];
                    red[warp * 64 + 2 * lane + 1] = sq[1];
                    ptx::named_barrier(BAR_S, NS);
                    if (tid < C)
                        red[256 + tid] = rsqrtf((red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid]) * (1.f / D) + a.eps);
                    // o again from TMEM (held there until the next M2): fewer registers live across the reduction
                    ptx::tmem_ld32(tl + TZ + 64, vo[0]);
                    ptx::tmem_ld32(tl + TZ + 96, vo[1]);
                    ptx::named_barrier(BAR_S, NS);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const float4 rs = *reinterpret_cast<const float4 *>(red + 256 + 32 * p + 4 * e4);
                            const float rsv[4] = {rs.x, rs.y, rs.z, rs.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int r = 32 * p + 4 * e4 + u;
                                const float gv = (r & 1) ? bf16_hi(gp[r >> 1]) : bf16_lo(gp[r >> 1]);
                                const float sg = fmaf(0.5f, ptx::tanh_approx(0.5f * gv), 0.5f);  // sigmoid
                                *reinterpret_cast<__nv_bfloat16 *>(stage + sw(r, ch)) =
                                    __float2bfloat16_rn(__uint_as_float(vo[p][4 * e4 + u]) * rsv[u] * w_row * sg);
                            }
                        }
                } else {
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            *reinterpret_cast<__nv_bfloat16 *>(stage + sw(32 * p + e, ch)) =
                                __float2bfloat16_rn(__uint_as_float(vo[p][e]));
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            if (ptx::named_barrier_or(BAR_S, NS, *s_abort != 0)) break;
            if (kGated && leader && has_next) load_g(s + C);  // the gate tile has been read
            if (o_skip) {
            } else if (L == C) {  // a full chunk: two TMA tile stores
                if (leader) {
                    ptx::tma_store_3d(&maps.o, sm + OFF_Y, 0, h, s);
                    ptx::tma_store_3d(&maps.o, sm + OFF_Y + 8192, 64, h, s);
                    ptx::bulk_commit_group();
                }
            } else {  // rows r < L (the later rows belong to the next sequence), 16 bytes per thread
                char *dst = static_cast<char *>(a.o) + (size_t(s) * H + h) * D * 2;
                for (int t = tid; t < L * 16; t += NS) {
                    const int r = t >> 4, q = t & 15;
                    *reinterpret_cast<uint4 *>(dst + size_t(r) * H * D * 2 + q * 16) =
                        *reinterpret_cast<const uint4 *>(sm + OFF_Y + (q >> 3) * 8192 + sw(r, q & 7));
                }
            }
            // the staged tile is rewritten by the next E2 only after the next E0 barrier, before
            // which the leader waits for the tile stores' reads
        }
        // Final state S_final[c][j] = R[j][c] e^{g_L - g_m}[c] of the last chunk.
        if (!*reinterpret_cast<volatile int *>(s_abort)) {
            ptx::tc_fence_after();
            const float *ecm_last = vec((nchunks - 1) & 1, VEC_ECM);
            float *const sf = *reinterpret_cast<float *const *>(sm + OFF_MISC + 8);
            uint32_t v[32];
            for (int p = 0; p < 4; ++p) {
                ptx::tmem_ld32(tl + TS + 32 * p, v);
                ptx::tmem_wait_ld();
                for (int e = 0; e < 32; ++e) {
                    const int c = 32 * p + e;
                    const float f = nchunks > 0 ? ecm_last[c] : 1.f;
                    if constexpr (kSplit) {
                        if (sf) sf[c * D + row] = __uint_as_float(v[e]) * f;
                    } else {
                        a.S_final[((size_t(seq) * H + h) * D + c) * D + row] = __uint_as_float(v[e]) * f;
                    }
                }
            }
        }
        if (leader) ptx::bulk_wait0();
    } else {
        // =================================================================== prep group
        ptx::regs_dec<128>();
        const int pt = tid - NS;  // 0..255
        const int pw = pt >> 5;   // prep warp 0..7
        const bool leader = pt == 0;
        const int qd = warp & 3, half = pw >> 2;
        const int trow = qd * 32 + lane;  // TMEM lane this thread reads in E1
        const uint32_t tl = tbase + (uint32_t(qd * 32) << 16);
        if (leader && nchunks > 0) {
            load_qk(bos);
            load_la(bos);
        }
        for (int ci = 0; ci < nchunks; ++ci) {
            const int s = bos + ci * C;
            const int L = min(C, eos - s);
            const bool has_next = ci + 1 < nchunks;
            const int par = ci & 1;
            const float *gm = vec(par, VEC_GM), *beta = vec(par, VEC_BETA);

            // ---- P2: Kt, Qt (in place over the raw k|q rows) and Kb; one (token row,
            // 32-channel quarter) per thread.  Kb buffer `par` was last read by M4 of
            // chunk ci - 2.  g and g_m come from the state group's P1.
            cwait(CNT_SCAN, ci + 1);
            mwait(B_QK, ci, leader);
            if (ci >= 2) cwait(CNT_M45, ci - 1);
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;
            {
                const int r = pt & 63, part = pt >> 6, kb = part >> 1;
                const bool valid = r < L;
                uint8_t *kbt = sm + OFF_KB + par * 16384;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int ch = (part & 1) * 4 + qq;
                    const uint32_t ph16 = sw(r, ch);
                    const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + OFF_QK + kb * 16384 + ph16);
                    const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + OFF_QK + kb * 16384 + 8192 + ph16);
                    const int c0 = 64 * kb + 8 * ch;
                    const int box = c0 >> 5, lch = (c0 & 31) >> 2;
                    const float4 ga = *reinterpret_cast<const float4 *>(sm + OFF_LA + box * 8192 + sw(r, lch));
                    const float4 gb = *reinterpret_cast<const float4 *>(sm + OFF_LA + box * 8192 + sw(r, lch + 1));
                    const float4 m0 = *reinterpret_cast<const float4 *>(gm + c0);
                    const float4 m1 = *reinterpret_cast<const float4 *>(gm + c0 + 4);
                    uint32_t o_kt[4] = {0u, 0u, 0u, 0u}, o_qt[4] = {0u, 0u, 0u, 0u}, o_kb[4] = {0u, 0u, 0u, 0u};
                    if (valid) {  // rows >= L stay zero
                        const float dg[8] = {ga.x - m0.x, ga.y - m0.y, ga.z - m0.z, ga.w - m0.w,
                                             gb.x - m1.x, gb.y - m1.y, gb.z - m1.z, gb.w - m1.w};  // base 2
                        const uint32_t kw[4] = {kraw.x, kraw.y, kraw.z, kraw.w};
                        const uint32_t qw[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            float kt[2], qt[2], kbv[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int e = 2 * e2 + u;
                                const float kv = u ? bf16_hi(kw[e2]) : bf16_lo(kw[e2]);
                                const float qv = u ? bf16_hi(qw[e2]) : bf16_lo(qw[e2]);
                                const float up = ptx::ex2_approx(dg[e]);
                                const float dn = ptx::ex2_approx(-dg[e]);
                                kt[u] = kv * up;
                                qt[u] = qv * up;
                                kbv[u] = kv * dn;
                            }
                            o_kt[e2] = pack_h2(kt[0], kt[1]);
                            o_qt[e2] = pack_h2(qt[0], qt[1]);
                            o_kb[e2] = pack_h2(kbv[0], kbv[1]);
                        }
                    }
                    *reinterpret_cast<uint4 *>(sm + OFF_QK + kb * 16384 + ph16) = make_uint4(o_kt[0], o_kt[1], o_kt[2], o_kt[3]);
                    *reinterpret_cast<uint4 *>(sm + OFF_QK + kb * 16384 + 8192 + ph16) = make_uint4(o_qt[0], o_qt[1], o_qt[2], o_qt[3]);
                    *reinterpret_cast<uint4 *>(kbt + kb * 8192 + ph16) = make_uint4(o_kb[0], o_kb[1], o_kb[2], o_kb[3]);
                }
            }
            ptx::fence_proxy_async_smem();
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;

            // ---- M1, then hand the rows to the state group; next chunk's log alpha.
            if (leader) {
                ptx::tc_fence_after();
                const uint32_t kb_base = OFF_KB + par * 16384;
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t ka = uint32_t(ks >> 2) * 16384u + uint32_t(ks & 3) * 32u;
                    const uint32_t kbo = uint32_t(ks >> 2) * 8192u + uint32_t(ks & 3) * 32u;
                    ptx::mma_ss(tbase + TAP, ptx::sdesc_sw128(sb + OFF_QK + ka), ptx::sdesc_sw128(sb + kb_base + kbo),
                                IDESC_N64, ks > 0);
                }
                commit(B_M1);
                ptx::st_release(cnt + CNT_ROWS, ci + 1);
                if (has_next) load_la(s + C);  // g of this chunk is no longer read
            }
            mwait(B_M1, ci, leader);
            ptx::tc_fence_after();

            // ---- E1: A rows -> fp32 scratch, P rows -> fp16 operand (buffer `par`,
            // last read by M5 of chunk ci - 2, already waited for above).
            {
                uint32_t v[32];
                ptx::tmem_ld32(tl + TAP + 32 * half, v);
                ptx::tmem_wait_ld();
                if (qd < 2) {
                    const int r = trow;
                    const float br = beta[r];
                    float *af = reinterpret_cast<float *>(sm + OFF_AF) + r * LDF + 32 * half;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        float4 x;
                        const int i = 32 * half + e;
                        x.x = (i + 0 < r) ? br * __uint_as_float(v[e + 0]) : 0.f;
                        x.y = (i + 1 < r) ? br * __uint_as_float(v[e + 1]) : 0.f;
                        x.z = (i + 2 < r) ? br * __uint_as_float(v[e + 2]) : 0.f;
                        x.w = (i + 3 < r) ? br * __uint_as_float(v[e + 3]) : 0.f;
                        *reinterpret_cast<float4 *>(af + e) = x;
                    }
                } else {
                    const int r = trow - 64;
                    uint8_t *pt_tile = sm + OFF_P + par * 8192;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int e = 8 * qq + 2 * e2, i = 32 * half + e;
                            pk[e2] = pack_h2(i <= r ? __uint_as_float(v[e]) : 0.f,
                                             i + 1 <= r ? __uint_as_float(v[e + 1]) : 0.f);
                        }
                        *reinterpret_cast<uint4 *>(pt_tile + sw(r, 4 * half + qq)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
            }
            ptx::tc_fence_before();
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;

            // ---- T = (I + A)^{-1} Diag(beta).  X = (I + A)^{-1} by block doubling: the four
            // diagonal 16x16 blocks by column substitution in registers (one warp each); then
            // the two 32x32 diagonal halves, X_10 = -(X_11 A_10) X_00 and X_32 = -(X_33 A_32) X_22;
            // then the lower-left half, X_21 = -(X_H1 A_21) X_H0 over 32x32 halves.  The
            // inverse of a unit lower-triangular block matrix [[L0, 0], [B, L1]] is
            // [[L0^-1, 0], [-L1^-1 B L0^-1, L1^-1]].
            {
                const float *Af = reinterpret_cast<const float *>(sm + OFF_AF);
                float *X = reinterpret_cast<float *>(sm + OFF_XF);
                float *E = reinterpret_cast<float *>(sm + OFF_EB);
                if (ci >= 1) cwait(CNT_TW, ci);  // the state group has read X of chunk ci - 1
                if (pw < 4) {
                    const int b = pw, jj = lane & 15;
                    const float *ab = Af + (16 * b) * LDF + 16 * b;
                    float x[16];
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) {  // x_rr = [rr == jj] - sum_{ss < rr} A_bb[rr][ss] x_ss
                        float acc = (rr == jj) ? 1.f : 0.f;
#pragma unroll
                        for (int s4 = 0; s4 < rr; s4 += 4) {
                            const float4 a4 = *reinterpret_cast<const float4 *>(ab + rr * LDF + s4);
                            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                if (s4 + u < rr) acc = fmaf(-av[u], x[s4 + u], acc);
                        }
                        x[rr] = acc;
                    }
                    if (lane < 16) {
#pragma unroll
                        for (int rr = 0; rr < 16; ++rr) X[(16 * b + rr) * LDF + 16 * b + jj] = x[rr];
                    }
                }
                ptx::named_barrier(BAR_P, NP);
                {  // E_h = X_{b1 b1} A_{b1 b0} (16x16, h = 0: b = 1, 0; h = 1: b = 3, 2); two columns a thread.
                   // Diagonal blocks of X hold zeros above their diagonal.
                    const int hh = pt >> 7, r = (pt >> 3) & 15, c2 = 2 * (pt & 7);
                    const int b1 = 2 * hh + 1, b0 = 2 * hh;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float xv = X[(16 * b1 + r) * LDF + 16 * b1 + m];
                        const float2 av = *reinterpret_cast<const float2 *>(Af + (16 * b1 + m) * LDF + 16 * b0 + c2);
                        a0 = fmaf(xv, av.x, a0);
                        a1 = fmaf(xv, av.y, a1);
                    }
                    *reinterpret_cast<float2 *>(E + (16 * hh + r) * LDE + c2) = make_float2(a0, a1);
                }
                ptx::named_barrier(BAR_P, NP);
                {  // X_{b1 b0} = -E_h X_{b0 b0}
                    const int hh = pt >> 7, r = (pt >> 3) & 15, c2 = 2 * (pt & 7);
                    const int b1 = 2 * hh + 1, b0 = 2 * hh;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float ev = E[(16 * hh + r) * LDE + m];
                        const float2 xv = *reinterpret_cast<const float2 *>(X + (16 * b0 + m) * LDF + 16 * b0 + c2);
                        a0 = fmaf(ev, xv.x, a0);
                        a1 = fmaf(ev, xv.y, a1);
                    }
                    *reinterpret_cast<float2 *>(X + (16 * b1 + r) * LDF + 16 * b0 + c2) = make_float2(-a0, -a1);
                }
                ptx::named_barrier(BAR_P, NP);
                {  // F = X_H1 A_21 (32x32; X_H1 = X[32:64, 32:64] is zero above its diagonal, and
                   // its upper-right 16x16 block is never read); F[r][c] at E[r * LDG + c]
                    const int r = pt >> 3, c4 = 4 * (pt & 7);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    const float *xr = X + (32 + r) * LDF + 32;
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float xv = xr[m];
                        const float4 av = *reinterpret_cast<const float4 *>(Af + (32 + m) * LDF + c4);
                        acc[0] = fmaf(xv, av.x, acc[0]);
                        acc[1] = fmaf(xv, av.y, acc[1]);
                        acc[2] = fmaf(xv, av.z, acc[2]);
                        acc[3] = fmaf(xv, av.w, acc[3]);
                    }
                    if (r >= 16) {  // uniform over a warp
#pragma unroll
                        for (int m = 16; m < 32; ++m) {
                            const float xv = xr[m];
                            const float4 av = *reinterpret_cast<const float4 *>(Af + (32 + m) * LDF + c4);
                            acc[0] = fmaf(xv, av.x, acc[0]);
                            acc[1] = fmaf(xv, av.y, acc[1]);
                            acc[2] = fmaf(xv, av.z, acc[2]);
                            acc[3] = fmaf(xv, av.w, acc[3]);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) E[r * LDG + c4 + q] = acc[q];
                }
                ptx::named_barrier(BAR_P, NP);
                {  // X_21 = -F X_H0 (X_H0 = X[0:32, 0:32]; its upper-right block is never read)
                    const int r = pt & 31, c4 = 4 * (pt >> 5);
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    const float *fr = E + r * LDG;
                    if (c4 < 16) {  // uniform over a warp
#pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            const float fv = fr[m];
                            const float4 xv = *reinterpret_cast<const float4 *>(X + m * LDF + c4);
                            acc[0] = fmaf(fv, xv.x, acc[0]);
                            acc[1] = fmaf(fv, xv.y, acc[1]);
                            acc[2] = fmaf(fv, xv.z, acc[2]);
                            acc[3] = fmaf(fv, xv.w, acc[3]);
                        }
                    }
#pragma unroll
                    for (int m = 16; m < 32; ++m) {
                        const float fv = fr[m];
                        const float4 xv = *reinterpret_cast<const float4 *>(X + m * LDF + c4);
                        acc[0] = fmaf(fv, xv.x, acc[0]);
                        acc[1] = fmaf(fv, xv.y, acc[1]);
                        acc[2] = fmaf(fv, xv.z, acc[2]);
                        acc[3] = fmaf(fv, xv.w, acc[3]);
                    }
                    *reinterpret_cast<float4 *>(X + (32 + r) * LDF + c4) = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
                }
                ptx::named_barrier(BAR_P, NP);
            }
            // X (fp32) is handed to the state group, which forms T = X Diag(beta)
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;
            if (leader) ptx::st_release(cnt + CNT_TP, ci + 1);
        }
    }

    __syncthreads();
    if (tid == 0 && *reinterpret_cast<volatile int *>(s_abort)) {
        // drain what is still in flight (each wait bounded) before TMEM goes away
        for (int b = 0; b < NBAR; ++b)
            for (uint32_t ph = wt[b]; ph < iss[b]; ++ph) ptx::mbar_wait_bounded(bars + b, ph & 1u, kWaitCycles);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, TMEM_COLS);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [T, H, 128] row-major tensor, boxes of 128 bytes x 64 tokens, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes, int H, int64_t T) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T)};
    const cuuint64_t strides[2] = {cuuint64_t(D) * elem_bytes, cuuint64_t(H) * D * elem_bytes};
    const cuuint32_t box[3] = {cuuint32_t(128 / elem_bytes), 1u, cuuint32_t(C)};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kGated, bool kSplit>
cudaError_t launch_tc(const TcMaps &maps, const PrefillArgs &a, cudaStream_t stream) {
    cudaError_t err = cudaFuncSetAttribute(prefill_tc_kernel<kGated, kSplit>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_alloc(kGated)));
    if (err != cudaSuccess) return err;
    const unsigned units = unsigned(a.split.num_units) + (a.split.plain_units ? unsigned(a.num_seqs) : 0u);
    const unsigned grid = units * unsigned(a.H);
    if (grid == 0) return cudaSuccess;
    prefill_tc_kernel<kGated, kSplit><<<grid, NT, smem_alloc(kGated), stream>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supported(const PrefillArgs &a) {
    return a.dtype == KDA_DTYPE_BF16 && a.dk == D && a.dv == D && a.chunk == C && a.total_tokens > 0 &&
           a.num_seqs > 0;
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream) {
    TcMaps maps;
    if (!make_map(&maps.q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, a.total_tokens) ||
        !make_map(&maps.k, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, a.total_tokens) ||
        !make_map(&maps.v, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, a.total_tokens) ||
        !make_map(&maps.la, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.H, a.total_tokens) ||
        !make_map(&maps.o, a.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, a.total_tokens))
        return cudaErrorInvalidValue;
    if (a.gate == nullptr) {
        // a launch that holds split units, or skips split sequences, takes the kSplit form
        if (a.split.num_units > 0 || a.split.num_seqs > 0) return launch_tc<false, true>(maps, a, stream);
        return launch_tc<false, false>(maps, a, stream);
    }
    if (!make_map(&maps.g, a.gate, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, a.total_tokens))
        return cudaErrorInvalidValue;
    return launch_tc<true, false>(maps, a, stream);
}

}  // namespace kda
