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
// Decay range.  The section's channel-wise decay bullet allows any alpha in [0, 1],
// alpha = 0 (log alpha = -inf) included, so every exponent here is a sum of log alpha
// over the tokens it spans (never -inf - -inf) and every tensor-core operand stays in
// fp16 range.  The chunk is cut into four 16-token blocks; H_R is block R's total (base
// 2) per channel.  Each chunk takes one of two forms, chosen by the prep group from the
// block totals (a vote over all channels):
// * Fast form, when every block total is >= -kFastBound (2^-5) in every channel: the
//   decays are factored at g_m, the running sum at the end of block 1 (mid-chunk):
//     Kt = K e^{g - g_m}, Qt = Q e^{g - g_m}, Kb = K e^{g_m - g}   (factors within 2^{+-10})
//     M1  [A; P]^raw = [Kt; Qt] Kb^T   (N = 64),
//   the state's products use Kt, Qt and Kb (M2 = Sop [Kt; Qt]^T, M4 += U^T Kb), and TMEM
//   carries S^T Diag(e^{g_m - g_L}) out of the chunk; the pass over R at the start of the
//   next chunk folds the factor back.
// * Block-reference form otherwise.  In block R, h_r sums log alpha from the block's
//   first token to r, s_r over the tokens after r to the block's end.  Each block takes a
//   reference point mu_R = (end of block R-1) + shift_R with shift_R = H_R / 2 for
//   channels whose block decay stays within 2^{-16} (|H_R| <= kShiftBound), else 0.
//     Rows:     Km = K e^{h - shift}, Qm = Q e^{h - shift}            (<= 2^8 |k|)
//     Columns:  Kc^(R)_i = K_i e^{mu_R - g_i}, i < 16 (R + 1): <= 1 for i in earlier
//               blocks, within 2^{+-8} in block R (zero for channels past the bound).
//   M1 issues one MMA per row block R (N = 16, 32, 48, 64); block R's rows of its output
//   are A and P.  A block whose decay leaves that bound in any channel has its own
//   16 x 16 pairs recomputed exactly on CUDA cores (products of the alphas between the
//   two tokens, with k, q and log alpha reloaded from L2), over the tensor-core values.
//   The state products run from the chunk start: Kg = K e^{g}, Qg = Q e^{g},
//   Kl = K e^{g_L - g}, all <= |k|, and TMEM holds S^T itself.
//
// Design (one CTA of 384 threads per (sequence, head), walking its chunks):
// * The fp32 state is kept TRANSPOSED in tensor memory (lane = value column j) for
//   the whole sequence, so every state product is a 128-row UMMA with d_v on M:
//     M1  [A; P]^raw   (fast: N=64 K=128; block-reference: N=16(R+1) K=128, R = 0..3)
//     M2  Z          = Sop [Kg; Qg]^T          M=128 N=128 K=128 (Sop = fp16 of R scaled)
//           Z[:, :64] = (Kg S)^T,  Z[:, 64:] = (Qg S)^T     (Kt, Qt in the fast form)
//     Mv  Z[:, :64] += V^T (-I)     (V read MN-major from its TMA tile)   N=64 K=64
//     M3  U^T        = Y^T T^T  -> Z[:, :64],  Y^T = -Z[:, :64]    N=64 K=64
//     M4  R         += U^T Kl      (Kl, or Kb, read as an MN-major operand)  N=128 K=64
//     M5  Z[:, 64:] += U^T P^T  ( = O^T )                   N=64  K=64
//   The pass over R at the start of a chunk packs Sop = fp16(R f_s) and sets R <- R f_r,
//   with per-channel factors the prep group derives from the block totals for the pair
//   of chunk forms (previous, current).
// * Two warp groups work on different chunks at once.  The prep group (warps 4-11)
//   builds chunk c + 1 -- the block sums, the form vote, the fp16 operand rows over the
//   raw k|q tile, M1, A and P, the exact blocks, and X = (I + A)^{-1} in place but its
//   lower-left 32 x 32 block -- while the state group (warps 0-3) runs chunk c -- the
//   pass over R, M2, Y, X_21 = -(X_H1 A_21) X_H0 and T = X Diag(beta), M3, U, M4/M5 and
//   the outputs.  X_21 and T are formed while M2 runs.  The groups hand buffers over
//   through thread-arrive mbarriers, one per signal and chunk parity, and the MMAs'
//   completion barriers; Kl/Kb and P are double-buffered by chunk parity.
// * Operands are fp16 (fp32 accumulation): the S-dependent chain keeps the relative
//   error near fp16's 2^-11, which the parity bounds need (bf16 operands do not meet
//   them).
// * q, k and v arrive by TMA in the 128-byte swizzled layout the UMMA descriptors
//   use; log alpha and beta are loaded into registers a chunk ahead; the chunk after
//   next is prefetched into L2.  A full chunk's outputs leave by two TMA tile stores,
//   a shorter last chunk row by row (its later rows belong to the next sequence).
// * kGated applies the layer's output epilogue (sigmoid gate and RMSNorm) before the
//   output store; kSplit runs the units of a sequence split (kda_internal.h).
// * Every wait is bounded: one that runs out sets the workspace error flag and both
//   groups stop at their next group barrier (decided uniformly by a barrier-or),
//   drain what they have in flight and free TMEM.
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
constexpr float kShiftBound = 16.f;       // |H_R| (base 2) up to which a block's own pairs use the tensor cores
constexpr float kFastBound = 5.f;         // |H_R| (base 2) of every block up to which a chunk takes the mid-chunk factoring

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_QK = 0;        // raw k|q boxes [k0 q0 k1 q1] -> [Km; Qm] in place (128 x 128 fp16, K-major)
constexpr uint32_t OFF_KQ = 32768;    // [Kg; Qg], same layout
constexpr uint32_t OFF_KC = 65536;    // Kc^(R), R = 0..3: 16 (R + 1) rows, two channel halves each (40 KB)
constexpr uint32_t OFF_KL = 106496;   // Kl (64 x 128 fp16, two channel boxes), two buffers (chunk parity)
constexpr uint32_t OFF_V = 139264;    // raw v boxes (bf16, 64 x 128)
constexpr uint32_t OFF_AX = 155648;   // A, then X = (I + A)^{-1} in place (fp32, 64 x LDF)
constexpr int LDF = 68;
constexpr uint32_t OFF_EB = OFF_AX + 64 * LDF * 4;  // solve scratch; the block totals while the rows are built
constexpr int LDE = 20;
constexpr int LDG = 33;
constexpr uint32_t OFF_P = 178176;    // P (64 x 64 fp16), two buffers (after the control structures below)
static_assert(OFF_EB + 32 * LDG * 4 <= OFF_P && OFF_EB + 8 * D * 4 <= OFF_P, "solve scratch overflows");
constexpr uint32_t OFF_T = OFF_P + 16384;    // T (64 x 64 fp16); the exact diagonal blocks' partial sums
constexpr uint32_t OFF_Y = OFF_T + 8192;     // the bf16 output tile (two 64 x 64 boxes); the gate tile (gated)
constexpr uint32_t OFF_ID = OFF_Y + 16384;   // -I (64 x 64 bf16): loads -V^T into Z with an MMA
constexpr uint32_t OFF_VEC = OFF_ID + 8192;  // per-chunk vectors, two buffers (chunk parity)
constexpr uint32_t VEC_BETA = 0;      // beta                 64 f32
constexpr uint32_t VEC_FS = 256;      // the pass over R: Sop = fp16(R f_s)      128 f32
constexpr uint32_t VEC_FR = 768;      //                  R <- R f_r             128 f32
constexpr uint32_t VEC_BYTES = 1280;
// Small control structures, in the gap before the 1024-aligned P tiles.
constexpr uint32_t OFF_BAR = OFF_EB + 32 * LDG * 4;     // mbarriers of the TMA loads and MMAs
constexpr int NBAR = 8;
constexpr int B_QK = 0, B_V = 1, B_M1 = 2, B_M2 = 3, B_M3 = 4, B_M45 = 5, B_G = 6;
// Hand-overs between the groups: one thread-arrive mbarrier per signal and chunk parity; the
// signal of chunk c completes phase c >> 1 of barrier 2 * signal + (c & 1).  No producer can
// complete chunk c + 2's phase before the consumer has waited for chunk c's.
constexpr uint32_t OFF_SIG = OFF_BAR + 8 * NBAR;
constexpr int S_P2 = 0, S_TP = 1, S_TW = 2, S_M45 = 3, NSIG = 4;
//   S_P2:  prep -> state: the operand rows, f_s, f_r and beta of chunk c (and M1 issued)
//   S_TP:  prep -> state: X of chunk c
//   S_TW:  state -> prep: T of chunk c formed (X read)
//   S_M45: state -> prep: M4/M5 of chunk c done (Kl, P of its parity and the T tile read)
// The prep group learns that M2 of chunk c has read the K/Q operand tile from M2's own
// completion barrier (B_M2), which the tensor core arrives on.
constexpr uint32_t OFF_ISS = OFF_SIG + 8 * 2 * NSIG;    // phases issued / waited per mbarrier
constexpr uint32_t OFF_WT = OFF_ISS + 4 * NBAR;
constexpr uint32_t OFF_FLAG = OFF_WT + 4 * NBAR;        // per (block, channel box): bit 0 past the exact bound,
                                                        // bit 1 past the fast bound; then the chunk kind by parity
constexpr uint32_t OFF_MISC = OFF_FLAG + 48;            // tmem base, abort flag, S_final pointer
constexpr uint32_t OFF_CTRL_END = OFF_MISC + 16;
constexpr uint32_t SMEM_USED = OFF_VEC + 2 * VEC_BYTES;
// The gated output epilogue's per-token reduction of o^2 (4 x 64 partial sums, then 64
// reciprocal RMS values); its gate tile shares the output tile.
constexpr uint32_t OFF_RED = SMEM_USED;
constexpr uint32_t SMEM_USED_G = OFF_RED + 320 * 4;
constexpr uint32_t smem_alloc(bool gated) { return (gated ? SMEM_USED_G : SMEM_USED) + 1024; }  // + alignment slack
static_assert(smem_alloc(true) <= 232448, "shared memory");
static_assert(OFF_CTRL_END <= OFF_P, "control structures overflow into the P tiles");
static_assert(OFF_KL % 1024 == 0 && OFF_V % 1024 == 0 && OFF_P % 1024 == 0 && OFF_Y % 1024 == 0 &&
              OFF_ID % 1024 == 0, "swizzled tiles need 1024-byte alignment");

// Kc^(R), channel half hb: 16 (R + 1) rows of 128 bytes.
__host__ __device__ constexpr uint32_t kc_off(int R, int hb) {
    return OFF_KC + uint32_t(8 * R * (R + 1)) * 256u + uint32_t(hb) * uint32_t(16 * (R + 1)) * 128u;
}
static_assert(kc_off(3, 1) + 64 * 128 == OFF_KL, "Kc layout");

// Tensor memory columns.
constexpr uint32_t TS = 0;      // R = S^T (fp32)      128 cols   state group
constexpr uint32_t TZ = 128;    // Z fp32; U^T in its first 64 columns    128 cols   state group
constexpr uint32_t TSOP = 256;  // Sop fp16             64 cols   state group
constexpr uint32_t TY16 = TSOP;       // Y^T fp16, 32 cols, over Sop once M2 has read it
constexpr uint32_t TU16 = TSOP + 32;  // U^T fp16, 32 cols
constexpr uint32_t TAP = 320;   // M1 outputs: block R at TAP + 8 R (R + 1), 16 (R + 1) cols (160)   prep group
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_N128 = ptx::idesc_f16_f32(128, 128);
constexpr uint32_t IDESC_N64 = ptx::idesc_f16_f32(128, 64);
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

// Position of a diagonal-block value (row r, column i <= r of a 16-token block) in the
// order the exact recomputation emits them: column i's run is P_ii, A_{i+1,i},
// P_{i+1,i}, A_{i+2,i}, ... (31 - 2i values); group g (32 values) holds column g's run
// followed by column 15 - g's.
__device__ __forceinline__ int diag_run_start(int i) { return i < 8 ? 32 * i : 32 * (15 - i) + 2 * i + 1; }

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

// The exact path's partial sums for one 16-token block R and one 64-channel box bx of a
// chunk that starts at token s (L tokens): for every pair i <= r of the block,
// P_ri = sum_c q_rc k_ic prod_{i<t<=r} alpha_tc and A_ri / beta_r = sum_c k_rc k_ic prod(...),
// over the box's channels, in diag_run_start order (one value per lane, eight groups of 32).
// fp32 arithmetic on the bf16 inputs; the rows come from global memory (L2).
__device__ __forceinline__ void exact_block_partials(float *out, const __nv_bfloat16 *kp, const __nv_bfloat16 *qp,
                                                     const float *lap, int H, int s, int L, int h, int R, int bx,
                                                     int lane) {
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int c = 64 * bx + 32 * pass + lane;
        uint32_t kq[16];  // (k, q) of row j as a bf16 pair
        float al[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int r = 16 * R + j;
            const bool ok = r < L;
            const size_t off = (size_t(s + r) * H + h) * D + c;
            const uint32_t kb = ok ? uint32_t(__bfloat16_as_ushort(kp[off])) : 0u;
            const uint32_t qb = ok ? uint32_t(__bfloat16_as_ushort(qp[off])) : 0u;
            kq[j] = kb | (qb << 16);
            al[j] = ok ? ptx::ex2_approx(lap[off] * kLog2e) : 0.f;
        }
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            float x[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {  // column g's run, then column 15 - g's
                const int i = half ? 15 - g : g;
                const int o = half ? 31 - 2 * g : 0;
                float w = bf16_lo(kq[i]);
                x[o] = bf16_hi(kq[i]) * w;
#pragma unroll
                for (int r = i + 1; r < 16; ++r) {
                    w *= al[r];
                    x[o + 2 * (r - i) - 1] = bf16_lo(kq[r]) * w;
                    x[o + 2 * (r - i)] = bf16_hi(kq[r]) * w;
                }
            }
            const float y = warp_transpose_sum32(x, lane);
            if (pass == 0) out[32 * g + lane] = y;
            else out[32 * g + lane] += y;
        }
    }
}

struct TcMaps {
    CUtensorMap q, k, v, la, o, g;  // la: L2 prefetch only; g: the output gate (gated epilogue only)
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
    uint64_t *sigs = reinterpret_cast<uint64_t *>(sm + OFF_SIG);
    uint32_t *iss = reinterpret_cast<uint32_t *>(sm + OFF_ISS);
    uint32_t *wt = reinterpret_cast<uint32_t *>(sm + OFF_WT);
    int *flags = reinterpret_cast<int *>(sm + OFF_FLAG);
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
        for (int i = 0; i < 2 * NSIG; ++i) ptx::mbar_init(sigs + i, 1);
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
    auto load_v = [&](int s) {
        ptx::mbar_arrive_expect_tx(bars + B_V, 2 * 8192);
        ptx::tma_load_3d(sm + OFF_V, &maps.v, bars + B_V, 0, h, s);
        ptx::tma_load_3d(sm + OFF_V + 8192, &maps.v, bars + B_V, 64, h, s);
        ++iss[B_V];
    };
    auto load_g = [&](int s) {
        ptx::mbar_arrive_expect_tx(bars + B_G, 2 * 8192);
        ptx::tma_load_3d(sm + OFF_Y, &maps.g, bars + B_G, 0, h, s);
        ptx::tma_load_3d(sm + OFF_Y + 8192, &maps.g, bars + B_G, 64, h, s);
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
    // Wait for signal g of chunk c (bounded, gives up on an abort); chunk c < 0 needs no wait.
    auto swait = [&](int g, int c) {
        if (c < 0) return true;
        uint64_t *bar = sigs + 2 * g + (c & 1);
        const uint32_t parity = uint32_t(c >> 1) & 1u;
        if (ptx::mbar_try_wait(bar, parity)) return true;
        const long long t0 = clock64();
        while (!ptx::mbar_try_wait(bar, parity)) {
            if (*reinterpret_cast<volatile int *>(s_abort) || clock64() - t0 > kWaitCycles) {
                fail();
                return false;
            }
        }
        return true;
    };
    // Signal g of chunk c (one thread, after its group's barrier): release at CTA scope.
    auto sarrive = [&](int g, int c) { ptx::mbar_arrive(sigs + 2 * g + (c & 1)); };

    // Launched with 384 x 168 registers: the prep group (8 warps) drops to 160, the
    // state group (4 warps) rises to 184; 4 x 32 x 184 + 8 x 32 x 160 = 384 x 168.
    if (warp < 4) {
        // =================================================================== state group
        ptx::regs_inc<184>();
        const int row = tid;  // TMEM lane = value column j
        const uint32_t tl = tbase + (uint32_t(warp * 32) << 16);
        const bool leader = tid == 0;
        if (leader && nchunks > 0 && !v_zero) load_v(bos);
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
        for (int ci = 0; ci < nchunks; ++ci) {
            const int s = bos + ci * C;
            const int L = min(C, eos - s);
            const bool has_next = ci + 1 < nchunks;
            const int par = ci & 1;

            // ---- E0: Sop = fp16(R f_s), R <- R f_r per key channel.  R holds S^T Diag(e^{g_m - g_L})
            // after a fast chunk and S^T after the other kind; this chunk's kind wants Sop =
            // S^T Diag(e^{g_m}) and R = S^T Diag(e^{g_m}) (fast), or Sop = S^T and R = S^T Diag(e^{g_L}).
            swait(S_P2, ci);  // the operand rows, f_s, f_r and beta of this chunk
            const bool fast = flags[8 + par] != 0;
            {
                const float4 *fsv = reinterpret_cast<const float4 *>(vec(par, VEC_FS));
                const float4 *frv = reinterpret_cast<const float4 *>(vec(par, VEC_FR));
                uint32_t r4[4][32], pk[16];
#pragma unroll
                for (int p = 0; p < 4; ++p) ptx::tmem_ld32(tl + TS + 32 * p, r4[p]);
                ptx::tmem_wait_ld();
                // x *= f (32 columns starting at column c0, factors as float4 from f4)
                auto scale32 = [](uint32_t(&x)[32], const float4 *f4) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 f = f4[e4];
                        x[4 * e4 + 0] = __float_as_uint(__uint_as_float(x[4 * e4 + 0]) * f.x);
                        x[4 * e4 + 1] = __float_as_uint(__uint_as_float(x[4 * e4 + 1]) * f.y);
                        x[4 * e4 + 2] = __float_as_uint(__uint_as_float(x[4 * e4 + 2]) * f.z);
                        x[4 * e4 + 3] = __float_as_uint(__uint_as_float(x[4 * e4 + 3]) * f.w);
                    }
                };
                // fp16 pairs of x (times f, when given) -> 16 words
                auto pack32 = [&](const uint32_t(&x)[32], const float4 *f4) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 f = f4 ? f4[e4] : make_float4(1.f, 1.f, 1.f, 1.f);
                        pk[2 * e4] = pack_h2(__uint_as_float(x[4 * e4 + 0]) * f.x, __uint_as_float(x[4 * e4 + 1]) * f.y);
                        pk[2 * e4 + 1] = pack_h2(__uint_as_float(x[4 * e4 + 2]) * f.z, __uint_as_float(x[4 * e4 + 3]) * f.w);
                    }
                };
                if (fast) {  // f_s = f_r: one product per element, packed and stored back
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        scale32(r4[p], fsv + 8 * p);
                        pack32(r4[p], nullptr);
                        ptx::tmem_st16(tl + TSOP + 16 * p, pk);
                        ptx::tmem_st32(tl + TS + 32 * p, r4[p]);
                    }
                } else {
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        pack32(r4[p], fsv + 8 * p);
                        ptx::tmem_st16(tl + TSOP + 16 * p, pk);
                        scale32(r4[p], frv + 8 * p);
                        ptx::tmem_st32(tl + TS + 32 * p, r4[p]);
                    }
                }
                ptx::tmem_wait_st();
            }
            ptx::tc_fence_before();
            if (leader) ptx::bulk_wait_read0();  // the output tile's last store has read it
            if (ptx::named_barrier_or(BAR_S, NS, *s_abort != 0)) break;
            if (leader) {
                if (kGated && !o_skip) load_g(s);  // over the output tile, read (and waited) by this chunk's E4
                if (ci + 2 < nchunks && !v_zero) {
                    ptx::tma_prefetch_l2_3d(&maps.v, 0, h, s + 2 * C);
                    ptx::tma_prefetch_l2_3d(&maps.v, 64, h, s + 2 * C);
                    if (kGated) {
                        ptx::tma_prefetch_l2_3d(&maps.g, 0, h, s + 2 * C);
                        ptx::tma_prefetch_l2_3d(&maps.g, 64, h, s + 2 * C);
                    }
                }
                ptx::tc_fence_after();
                // Z = Sop [Kg; Qg]^T (the k and q boxes of a channel block are rows 0-63 and
                // 64-127 of one 128-row operand), then Z[:, :64] += V^T (-I), V read MN-major
                // from its TMA tile
                const uint32_t kq_base = OFF_KQ;  // [Kt; Qt] or [Kg; Qg]
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kq = uint32_t(ks >> 2) * 16384u + uint32_t(ks & 3) * 32u;
                    ptx::mma_ts(tbase + TZ, tbase + TSOP + 8 * ks, ptx::sdesc_sw128(sb + kq_base + kq), IDESC_N128,
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
            // ---- X_21 and T of this chunk (from the prep group's X) while M2 runs; then E2 and
            // M3: U^T = Y^T T^T into Z[:, :64].
            swait(S_TP, ci);
            {  // X_21 = -(X_H1 A_21) X_H0 over 32x32 halves (X_H1 = X[32:64, 32:64] and X_H0 =
               // X[0:32, 0:32] are zero above their diagonals); F = X_H1 A_21 in fp32 over the T tile
                const float *Af = reinterpret_cast<const float *>(sm + OFF_AX);
                float *X = reinterpret_cast<float *>(sm + OFF_AX);
                float *F = reinterpret_cast<float *>(sm + OFF_T);
                {  // F[r][c], eight columns a thread: r = tid >> 2, c8 = 8 (tid & 3)
                    const int r = tid >> 2, c8 = 8 * (tid & 3);
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    const float *xr = X + (32 + r) * LDF + 32;
                    const int mend = r < 16 ? 16 : 32;
                    for (int m = 0; m < mend; ++m) {
                        const float xv = xr[m];
                        const float4 a0 = *reinterpret_cast<const float4 *>(Af + (32 + m) * LDF + c8);
                        const float4 a1 = *reinterpret_cast<const float4 *>(Af + (32 + m) * LDF + c8 + 4);
                        acc[0] = fmaf(xv, a0.x, acc[0]);
                        acc[1] = fmaf(xv, a0.y, acc[1]);
                        acc[2] = fmaf(xv, a0.z, acc[2]);
                        acc[3] = fmaf(xv, a0.w, acc[3]);
                        acc[4] = fmaf(xv, a1.x, acc[4]);
                        acc[5] = fmaf(xv, a1.y, acc[5]);
                        acc[6] = fmaf(xv, a1.z, acc[6]);
                        acc[7] = fmaf(xv, a1.w, acc[7]);
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) F[r * LDG + c8 + q] = acc[q];
                }
                ptx::named_barrier(BAR_S, NS);
                {  // X_21[r][c] = -sum_m F[r][m] X_H0[m][c], eight columns a thread: r = tid & 31, c8 = 8 (tid >> 5)
                    const int r = tid & 31, c8 = 8 * (tid >> 5);
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    const float *fr = F + r * LDG;
                    for (int m = c8 < 16 ? 0 : 16; m < 32; ++m) {
                        const float fv = fr[m];
                        const float4 x0 = *reinterpret_cast<const float4 *>(X + m * LDF + c8);
                        const float4 x1 = *reinterpret_cast<const float4 *>(X + m * LDF + c8 + 4);
                        acc[0] = fmaf(fv, x0.x, acc[0]);
                        acc[1] = fmaf(fv, x0.y, acc[1]);
                        acc[2] = fmaf(fv, x0.z, acc[2]);
                        acc[3] = fmaf(fv, x0.w, acc[3]);
                        acc[4] = fmaf(fv, x1.x, acc[4]);
                        acc[5] = fmaf(fv, x1.y, acc[5]);
                        acc[6] = fmaf(fv, x1.z, acc[6]);
                        acc[7] = fmaf(fv, x1.w, acc[7]);
                    }
                    *reinterpret_cast<float4 *>(X + (32 + r) * LDF + c8) = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
                    *reinterpret_cast<float4 *>(X + (32 + r) * LDF + c8 + 4) = make_float4(-acc[4], -acc[5], -acc[6], -acc[7]);
                }
                ptx::named_barrier(BAR_S, NS);
            }
            {  // T[r][i] = X[r][i] beta_i for i <= r as an fp16 operand (rows r, K = i)
                const float *X = reinterpret_cast<const float *>(sm + OFF_AX);
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
            if (leader) sarrive(S_TW, ci);  // T is formed: the prep group may overwrite X
            mwait(B_M2, ci, leader);
            ptx::tc_fence_after();
            if (leader) {
                if (has_next && !v_zero) load_v(s + C);  // the V tile has been read by the MMA
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
            if (ptx::named_barrier_or(BAR_S, NS, *s_abort != 0)) break;

            if (leader) {
                ptx::tc_fence_after();
                for (int ks = 0; ks < 4; ++ks)
                    ptx::mma_ts(tbase + TZ, tbase + TY16 + 8 * ks, ptx::sdesc_sw128(sb + OFF_T + 32 * ks), IDESC_N64,
                                ks > 0);
                commit(B_M3);
            }
            mwait(B_M3, ci, leader);
            ptx::tc_fence_after();
            {  // E3: U^T -> fp16 pairs in TMEM, the A operand of M4 and M5
                uint32_t vu[2][32], pk[16];
                ptx::tmem_ld32(tl + TZ, vu[0]);
                ptx::tmem_ld32(tl + TZ + 32, vu[1]);
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

            // ---- M4: R += U^T Kl;  M5: O^T = Z[:, 64:] + U^T P^T.
            if (leader) {
                ptx::tc_fence_after();
                const uint32_t kl_base = OFF_KL + par * 16384, p_base = OFF_P + par * 8192;
                for (int ks = 0; ks < 4; ++ks)
                    ptx::mma_ts(tbase + TS, tbase + TU16 + 8 * ks, ptx::sdesc_sw128_mn(sb + kl_base + 2048 * ks, 8192, 1024),
                                IDESC_N128_BMN, 1u);
                for (int ks = 0; ks < 4; ++ks)
                    ptx::mma_ts(tbase + TZ + 64, tbase + TU16 + 8 * ks, ptx::sdesc_sw128(sb + p_base + 32 * ks), IDESC_N64,
                                1u);
                commit(B_M45);
            }
            mwait(B_M45, ci, leader);
            ptx::tc_fence_after();
            if (leader) sarrive(S_M45, ci);
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
                    const uint8_t *gt = sm + OFF_Y + (row >> 6) * 8192 + (row & 7) * 2;
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
                    // o again from TMEM (held there until the next M2): fewer registers live across the
                    // reduction; the gate tile has been read into registers before the barrier above,
                    // so the staged outputs below may overwrite it
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
            ptx::fence_proxy_async_smem();  // the row copies' reads precede the next TMA write of the tile
            // the staged tile is rewritten (by the gate load or the next E4) only after the next
            // E0 barrier, before which the leader waits for the tile stores' reads
        }
        // Final state S_final[c][j] = R[j][c] f[c], f = e^{g_L - g_m} after a fast last chunk, else 1.
        if (!*reinterpret_cast<volatile int *>(s_abort) && swait(S_P2, nchunks)) {
            ptx::tc_fence_after();
            float *const sf = *reinterpret_cast<float *const *>(sm + OFF_MISC + 8);
            const float *fin = vec(nchunks & 1, VEC_FR);
            uint32_t v[32];
            for (int p = 0; p < 4; ++p) {
                ptx::tmem_ld32(tl + TS + 32 * p, v);
                ptx::tmem_wait_ld();
                for (int e = 0; e < 32; ++e) {
                    const int c = 32 * p + e;
                    const float x = __uint_as_float(v[e]) * fin[c];
                    if constexpr (kSplit) {
                        if (sf) sf[c * D + row] = x;
                    } else {
                        a.S_final[((size_t(seq) * H + h) * D + c) * D + row] = x;
                    }
                }
            }
        }
        if (leader) ptx::bulk_wait0();
    } else {
        // =================================================================== prep group
        ptx::regs_dec<160>();
        const int pt = tid - NS;  // 0..255
        const int pw = pt >> 5;   // prep warp 0..7
        const bool leader = pt == 0;
        // Operand rows: block Rb of the chunk, channel box bx (64 channels), row half hh
        // (8 rows), four channels c0 .. c0 + 3 (byte offset ob in a 128-byte box row).
        const int Rb = pw >> 1, bx = pw & 1, hh = lane >> 4, g4 = lane & 15;
        const int c0 = 64 * bx + 4 * g4;
        const uint32_t ob = uint32_t(g4 & 1) * 8u;
        float4 lap[8];          // log alpha of rows 16 Rb + 8 hh + j, loaded a chunk ahead
        float beta_reg = 0.f;   // beta of token pt (pt < 64), loaded a chunk ahead
        float ecm_prev[4] = {1.f, 1.f, 1.f, 1.f};  // restores S^T from TMEM after the previous chunk
        auto load_la = [&](int cj) {
            if (cj >= nchunks) return;
            const int sj = bos + cj * C;
            const int Lj = min(C, eos - sj);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = 16 * Rb + 8 * hh + j;
                lap[j] = r < Lj ? __ldg(reinterpret_cast<const float4 *>(a.log_alpha + (size_t(sj + r) * H + h) * D + c0))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            beta_reg = (pt < C && pt < Lj) ? a.beta[size_t(sj + pt) * H + h] : 0.f;
        };
        auto prefetch_l2 = [&](int cj) {  // chunk cj's q, k and log alpha tiles into L2
            const int sj = bos + cj * C;
            for (int b = 0; b < 2; ++b) {
                ptx::tma_prefetch_l2_3d(&maps.k, 64 * b, h, sj);
                ptx::tma_prefetch_l2_3d(&maps.q, 64 * b, h, sj);
            }
            for (int b = 0; b < 4; ++b) ptx::tma_prefetch_l2_3d(&maps.la, 32 * b, h, sj);
        };
        if (leader && nchunks > 0) {
            load_qk(bos);
            if (nchunks > 1) prefetch_l2(1);
        }
        load_la(0);
        for (int ci = 0; ci < nchunks; ++ci) {
            const int s = bos + ci * C;
            const int L = min(C, eos - s);
            const int par = ci & 1;

            // ---- P2a: block sums of log alpha (base 2) for this thread's 4 channels: over its
            // 8 rows, then across the block's two row halves by one shuffle.  Every sum adds
            // terms <= 0; none is formed as a difference (alpha = 0 gives -inf, never NaN).
            float la2[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                la2[j][0] = lap[j].x * kLog2e;
                la2[j][1] = lap[j].y * kLog2e;
                la2[j][2] = lap[j].z * kLog2e;
                la2[j][3] = lap[j].w * kLog2e;
            }
            float pq[4], sq[4], Hb[4], shift[4];
            bool good_all = true, fast_all = true;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float t = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) t += la2[j][e];
                const float to = __shfl_xor_sync(0xffffffffu, t, 16);
                const float t0 = hh ? to : t, t1 = hh ? t : to;  // rows 0-7 and 8-15 of the block
                Hb[e] = t0 + t1;
                pq[e] = hh ? t0 : 0.f;  // before this thread's rows, within the block
                sq[e] = hh ? 0.f : t1;  // after them
                const bool good = Hb[e] >= -kShiftBound;
                shift[e] = good ? 0.5f * Hb[e] : 0.f;
                good_all = good_all && good;
                fast_all = fast_all && Hb[e] >= -kFastBound;
            }
            const bool wbad = __any_sync(0xffffffffu, !good_all);
            const bool wslow = __any_sync(0xffffffffu, !fast_all);
            float *xtot = reinterpret_cast<float *>(sm + OFF_EB);  // [block][channel] totals, then shifts
            if (hh == 0) {
                *reinterpret_cast<float4 *>(xtot + Rb * D + c0) = make_float4(Hb[0], Hb[1], Hb[2], Hb[3]);
                *reinterpret_cast<float4 *>(xtot + 4 * D + Rb * D + c0) = make_float4(shift[0], shift[1], shift[2], shift[3]);
            }
            if (lane == 0) flags[2 * Rb + bx] = (wbad ? 1 : 0) | (wslow ? 2 : 0);
            mwait(B_QK, ci, leader);  // the raw k|q tile of this chunk
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;

            // ---- P2b: the chunk's kind, the per-channel factors from the four blocks' totals,
            // then the operand rows from the raw k|q tile (rows >= L belong to the next
            // sequence: zero).
            //   fast (every block's decay within 2^-kFastBound in every channel): the mid-chunk
            //     factoring, g_m = g at the end of block 1: Kt = K e^{g - g_m} and Qt = Q e^{g - g_m}
            //     over the raw rows, Kb = K e^{g_m - g} (factors within 2^{+-2 kFastBound}); TMEM
            //     then holds S^T e^{g_m - g_L} after the chunk.
            //   otherwise: Kl and Kc^(R) for R >= Rb (backward over the rows), then Km, Qm over the
            //     raw rows, Kg and Qg (forward); TMEM holds S^T.
            bool any_bad = false, fast = true;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                any_bad = any_bad || (flags[b] & 1) != 0;
                fast = fast && (flags[b] & 2) == 0;
            }
            if (ci > 0) mwait(B_M2, ci - 1, false);  // M2 of chunk ci - 1 has read the K/Q operand tile
            swait(S_M45, ci - 2);             // M4/M5 of chunk ci - 2 have read Kl and P (buffer par)
            if (Rb == 0 && hh == 0) {  // the pass over R: f_s, f_r; the factor that restores S^T after this chunk
                float fs[4], fr[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float h0 = xtot[0 * D + c0 + e], h1 = xtot[1 * D + c0 + e];
                    const float h2 = xtot[2 * D + c0 + e], h3 = xtot[3 * D + c0 + e];
                    if (fast) {
                        fs[e] = fr[e] = ecm_prev[e] * ptx::ex2_approx(h0 + h1);
                        ecm_prev[e] = ptx::ex2_approx(h2 + h3);
                    } else {
                        fs[e] = ecm_prev[e];
                        fr[e] = ecm_prev[e] * ptx::ex2_approx(h0 + h1 + h2 + h3);
                        ecm_prev[e] = 1.f;
                    }
                }
                *reinterpret_cast<float4 *>(vec(par, VEC_FS) + c0) = make_float4(fs[0], fs[1], fs[2], fs[3]);
                *reinterpret_cast<float4 *>(vec(par, VEC_FR) + c0) = make_float4(fr[0], fr[1], fr[2], fr[3]);
            }
            if (pt == 0) flags[8 + par] = fast ? 1 : 0;
            auto st4 = [&](uint32_t off, float x0, float x1, float x2, float x3) {
                *reinterpret_cast<uint2 *>(sm + off) = make_uint2(pack_h2(x0, x1), pack_h2(x2, x3));
            };
            auto raw4 = [&](uint32_t off, int r, float (&f)[4]) {
                const uint2 w = r < L ? *reinterpret_cast<const uint2 *>(sm + off) : make_uint2(0u, 0u);
                f[0] = bf16_lo(w.x);
                f[1] = bf16_hi(w.x);
                f[2] = bf16_lo(w.y);
                f[3] = bf16_hi(w.y);
            };
            if (fast) {
                float off[4];  // g_r - g_m = (h_r within the block) + (totals before the block) - g_m
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float before = 0.f;
#pragma unroll
                    for (int R = 0; R < 4; ++R)
                        if (R < Rb) before += xtot[R * D + c0 + e];
                    off[e] = pq[e] + before - (xtot[0 * D + c0 + e] + xtot[1 * D + c0 + e]);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = 16 * Rb + 8 * hh + j;
                    const uint32_t o = sw(r, g4 >> 1) + ob;
                    float kf[4], qf[4];
                    raw4(OFF_QK + bx * 16384 + o, r, kf);
                    raw4(OFF_QK + bx * 16384 + 8192 + o, r, qf);
                    float up[4], dn[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        off[e] += la2[j][e];
                        up[e] = ptx::ex2_approx(off[e]);
                        dn[e] = ptx::ex2_approx(-off[e]);
                    }
                    st4(OFF_KQ + bx * 16384 + o, kf[0] * up[0], kf[1] * up[1], kf[2] * up[2], kf[3] * up[3]);
                    st4(OFF_KQ + bx * 16384 + 8192 + o, qf[0] * up[0], qf[1] * up[1], qf[2] * up[2], qf[3] * up[3]);
                    st4(OFF_KL + par * 16384 + bx * 8192 + o, kf[0] * dn[0], kf[1] * dn[1], kf[2] * dn[2], kf[3] * dn[3]);
                }
            } else {
                {
                    float fKl[4], fKd[4], fKc[3][4];
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float after = 0.f;
    #pragma unroll
                        for (int R = 0; R < 4; ++R)
                            if (R > Rb) after += xtot[R * D + c0 + e];
                        fKl[e] = ptx::ex2_approx(after);
                        // block Rb's own columns, e^{shift - h_i} = e^{s_i} e^{-shift}; zero past the bound
                        // (the exact path recomputes that block)
                        fKd[e] = Hb[e] >= -kShiftBound ? ptx::ex2_approx(-shift[e]) : 0.f;
                        float between = 0.f;  // totals of the blocks strictly between Rb and Rb + 1 + k2
    #pragma unroll
                        for (int k2 = 0; k2 < 3; ++k2) {
                            const int R2 = Rb + 1 + k2;
                            fKc[k2][e] = R2 < 4 ? ptx::ex2_approx(between + xtot[4 * D + (R2 & 3) * D + c0 + e]) : 0.f;
                            if (R2 < 4) between += xtot[(R2 & 3) * D + c0 + e];
                        }
                    }
                    float su[4] = {sq[0], sq[1], sq[2], sq[3]};  // sum after row j, within the block
    #pragma unroll
                    for (int j = 7; j >= 0; --j) {
                        const int r = 16 * Rb + 8 * hh + j;
                        const uint32_t o = sw(r, g4 >> 1) + ob;
                        float kf[4];
                        raw4(OFF_QK + bx * 16384 + o, r, kf);
                        float base[4];
    #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            base[e] = kf[e] * ptx::ex2_approx(su[e]);
                            su[e] += la2[j][e];
                        }
                        st4(OFF_KL + par * 16384 + bx * 8192 + o, base[0] * fKl[0], base[1] * fKl[1], base[2] * fKl[2],
                            base[3] * fKl[3]);
                        st4(kc_off(Rb, bx) + o, base[0] * fKd[0], base[1] * fKd[1], base[2] * fKd[2], base[3] * fKd[3]);
    #pragma unroll
                        for (int k2 = 0; k2 < 3; ++k2)
                            if (Rb + 1 + k2 < 4)
                                st4(kc_off(Rb + 1 + k2, bx) + o, base[0] * fKc[k2][0], base[1] * fKc[k2][1],
                                    base[2] * fKc[k2][2], base[3] * fKc[k2][3]);
                    }
                }
                {
                    float eMu[4];  // Kg = Km e^{mu} with mu = (totals before the block) + shift
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float before = 0.f;
    #pragma unroll
                        for (int R = 0; R < 4; ++R)
                            if (R < Rb) before += xtot[R * D + c0 + e];
                        eMu[e] = ptx::ex2_approx(before + shift[e]);
                    }
                    float hr[4] = {pq[0], pq[1], pq[2], pq[3]};  // sum from the block's first token to row j
    #pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int r = 16 * Rb + 8 * hh + j;
                        const uint32_t o = sw(r, g4 >> 1) + ob;
                        float kf[4], qf[4];
                        raw4(OFF_QK + bx * 16384 + o, r, kf);
                        raw4(OFF_QK + bx * 16384 + 8192 + o, r, qf);
                        float km[4], qm[4];
    #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            hr[e] += la2[j][e];
                            const float u = ptx::ex2_approx(hr[e] - shift[e]);
                            km[e] = kf[e] * u;
                            qm[e] = qf[e] * u;
                        }
                        st4(OFF_QK + bx * 16384 + o, km[0], km[1], km[2], km[3]);
                        st4(OFF_QK + bx * 16384 + 8192 + o, qm[0], qm[1], qm[2], qm[3]);
                        st4(OFF_KQ + bx * 16384 + o, km[0] * eMu[0], km[1] * eMu[1], km[2] * eMu[2], km[3] * eMu[3]);
                        st4(OFF_KQ + bx * 16384 + 8192 + o, qm[0] * eMu[0], qm[1] * eMu[1], qm[2] * eMu[2],
                            qm[3] * eMu[3]);
                    }
                }
            }
            if (pt < C) vec(par, VEC_BETA)[pt] = beta_reg;
            ptx::fence_proxy_async_smem();
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;

            // ---- M1: fast, [A; P]^raw = [Kt; Qt] Kb^T (N = 64); otherwise, block R's rows of
            // [Km; Qm] Kc^(R)T for R = 0..3 (N = 16 (R + 1))
            if (leader) {
                if (fast && ci + 1 < nchunks) load_qk(s + C);  // the raw k|q tile has been read
                ptx::tc_fence_after();
                if (fast) {
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t ka = uint32_t(ks >> 2) * 16384u + uint32_t(ks & 3) * 32u;
                        const uint32_t kb = OFF_KL + par * 16384 + uint32_t(ks >> 2) * 8192u + uint32_t(ks & 3) * 32u;
                        ptx::mma_ss(tbase + TAP, ptx::sdesc_sw128(sb + OFF_KQ + ka), ptx::sdesc_sw128(sb + kb), IDESC_N64,
                                    ks > 0);
                    }
                } else {
                for (int R = 0; R < 4; ++R) {
                    const uint32_t idesc = ptx::idesc_f16_f32(128, 16 * (R + 1));
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t ka = uint32_t(ks >> 2) * 16384u + uint32_t(ks & 3) * 32u;
                        const uint32_t kb = kc_off(R, ks >> 2) + uint32_t(ks & 3) * 32u;
                        ptx::mma_ss(tbase + TAP + 8 * R * (R + 1), ptx::sdesc_sw128(sb + OFF_QK + ka),
                                    ptx::sdesc_sw128(sb + kb), idesc, ks > 0);
                    }
                }
                }
                commit(B_M1);
                // then the state group's M2 may follow on the tensor pipe
                sarrive(S_P2, ci);  // the operand rows, f_s, f_r, beta of chunk ci
                if (ci + 2 < nchunks) prefetch_l2(ci + 2);
            }
            mwait(B_M1, ci, leader);
            ptx::tc_fence_after();
            if (leader && !fast && ci + 1 < nchunks) load_qk(s + C);  // M1 has read [Km; Qm] (over the raw tile)

            // ---- E1: A rows -> fp32 (beta_r, i < r) over the previous chunk's X, P rows -> fp16
            // operand (i <= r, zeros above; buffer par, last read by M5 of chunk ci - 2).
            swait(S_TW, ci - 1);  // the state group has formed T from X of chunk ci - 1
            if (fast) {  // every row's 64 columns: lane quarter qd, columns 32 half .. 32 half + 31
                const int qd = warp & 3, half = pw >> 2;
                const int trow = qd * 32 + lane;
                uint32_t v[32];
                ptx::tmem_ld32(tbase + (uint32_t(qd * 32) << 16) + TAP + 32 * half, v);
                ptx::tmem_wait_ld();
                if (qd < 2) {
                    const int r = trow;
                    const float br = vec(par, VEC_BETA)[r];
                    float *af = reinterpret_cast<float *>(sm + OFF_AX) + r * LDF + 32 * half;
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
                // the warps that wrote the diagonal 16x16 blocks of A (rows and columns 0-31:
                // prep warp 0; 32-63: prep warp 5) invert them at once
                const float *Af = reinterpret_cast<const float *>(sm + OFF_AX);
                float *X = reinterpret_cast<float *>(sm + OFF_AX);
                if (pw == 0 || pw == 5) {  // the warps whose E1 wrote the diagonal blocks: 0, 1 and 2, 3
                    const int b = (pw == 0 ? 0 : 2) + (lane >> 4), jj = lane & 15;
                    const float *ab = Af + (16 * b) * LDF + 16 * b;
                    float x[16];
                    __syncwarp();  // this warp's A rows are written
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
                    __syncwarp();  // every lane has read its A_bb
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) X[(16 * b + rr) * LDF + 16 * b + jj] = x[rr];
                }
            } else {
                float *Af = reinterpret_cast<float *>(sm + OFF_AX);
                uint8_t *pt_tile = sm + OFF_P + par * 8192;
                const int qdt = warp & 3;                 // TMEM lane quarter of this warp
                const int hf = pw >> 2;                   // columns 32 hf .. 32 hf + 31
                const uint32_t tq = tbase + (uint32_t(qdt * 32) << 16);
                const int r = (qdt & 1) * 32 + lane;      // token row within the chunk
                const bool is_p = qdt >= 2;
                const float br = vec(par, VEC_BETA)[r];
                for (int pc = 0; pc < 2; ++pc) {            // the half-warps' blocks, one after the other
                    const int pb = (qdt & 1) * 2 + pc;      // block of this piece (uniform over the warp)
                    const int pn = 16 * (pb + 1) - 32 * hf; // its M1 columns within this half
                    const uint32_t col = tq + TAP + 8 * pb * (pb + 1) + 32 * hf;
                    uint32_t v[32];
                    if (pn >= 32) {
                        ptx::tmem_ld32(col, v);
                        ptx::tmem_wait_ld();
                    } else if (pn == 16) {
                        uint32_t v16[16];
                        ptx::tmem_ld16(col, v16);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = v16[e];
#pragma unroll
                        for (int e = 16; e < 32; ++e) v[e] = 0u;
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = 0u;
                    }
                    if ((lane >> 4) != pc) continue;
                    if (!is_p) {
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const int i0 = 32 * hf + 4 * e4;
                            if (i0 >= r) break;
                            float4 x;
                            x.x = i0 + 0 < r ? br * __uint_as_float(v[4 * e4 + 0]) : 0.f;
                            x.y = i0 + 1 < r ? br * __uint_as_float(v[4 * e4 + 1]) : 0.f;
                            x.z = i0 + 2 < r ? br * __uint_as_float(v[4 * e4 + 2]) : 0.f;
                            x.w = i0 + 3 < r ? br * __uint_as_float(v[4 * e4 + 3]) : 0.f;
                            *reinterpret_cast<float4 *>(Af + r * LDF + i0) = x;
                        }
                    } else {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e2 = 0; e2 < 4; ++e2) {
                                const int e = 8 * qq + 2 * e2, i = 32 * hf + e;
                                pk[e2] = pack_h2(i <= r ? __uint_as_float(v[e]) : 0.f,
                                                 i + 1 <= r ? __uint_as_float(v[e + 1]) : 0.f);
                            }
                            *reinterpret_cast<uint4 *>(pt_tile + sw(r, 4 * hf + qq)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
            }
            ptx::tc_fence_before();

            // ---- The exact path for blocks whose decay leaves the tensor-core bound: their own
            // pairs, P_ri = <q_r, k_i prod_{i<t<=r} alpha_t> and A_ri = beta_r <k_r, ...>, from the
            // rows in L2 (fp32, running products), over the values E1 wrote.  Partial sums per
            // (block, channel box) go to the T tile, free once M3 of chunk ci - 1 has read it.
            if (!fast && any_bad) {
                float *part = reinterpret_cast<float *>(sm + OFF_T);  // [block][box][256]
                swait(S_M45, ci - 1);
                if ((flags[2 * Rb] | flags[2 * Rb + 1]) & 1)  // uniform over the warp
                    exact_block_partials(part + (Rb * 2 + bx) * 256, static_cast<const __nv_bfloat16 *>(a.k),
                                         static_cast<const __nv_bfloat16 *>(a.q), a.log_alpha, H, s, L, h, Rb, bx, lane);
                ptx::named_barrier(BAR_P, NP);
                float *Af = reinterpret_cast<float *>(sm + OFF_AX);
                uint8_t *pt_tile = sm + OFF_P + par * 8192;
                const int rl = pt >> 4, il = pt & 15;
                for (int R = 0; R < 4; ++R) {
                    if (!((flags[2 * R] | flags[2 * R + 1]) & 1) || il > rl) continue;
                    const int r = 16 * R + rl, i = 16 * R + il;
                    const float *p0 = part + (R * 2) * 256, *p1 = p0 + 256;
                    const int vp = diag_run_start(il) + 2 * (rl - il);
                    *reinterpret_cast<__half *>(pt_tile + sw(r, i >> 3) + (i & 7) * 2) = __float2half_rn(p0[vp] + p1[vp]);
                    if (il < rl) Af[r * LDF + i] = vec(par, VEC_BETA)[r] * (p0[vp - 1] + p1[vp - 1]);
                }
            }
            ptx::fence_proxy_async_smem();  // P is an MMA operand
            load_la(ci + 1);  // the next chunk's log alpha and beta (registers)
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;

            // ---- X = (I + A)^{-1} in place, by block doubling: the four diagonal 16x16 blocks by
            // column substitution in registers (one warp each); then the two 32x32 diagonal
            // halves, X_10 = -(X_11 A_10) X_00 and X_32 = -(X_33 A_32) X_22; then the lower-left
            // half, X_21 = -(X_H1 A_21) X_H0 over 32x32 halves.  The inverse of a unit
            // lower-triangular block matrix [[L0, 0], [B, L1]] is [[L0^-1, 0], [-L1^-1 B L0^-1, L1^-1]].
            // Each step reads the A blocks it replaces before any thread writes them.
            {
                const float *Af = reinterpret_cast<const float *>(sm + OFF_AX);
                float *X = reinterpret_cast<float *>(sm + OFF_AX);
                float *E = reinterpret_cast<float *>(sm + OFF_EB);
                if (!fast) {  // after the exact path; fast chunks inverted the blocks right after E1
                    if (pw == 0 || pw == 5) {  // the warps whose E1 wrote the diagonal blocks: 0, 1 and 2, 3
                        const int b = (pw == 0 ? 0 : 2) + (lane >> 4), jj = lane & 15;
                        const float *ab = Af + (16 * b) * LDF + 16 * b;
                        float x[16];
                        __syncwarp();  // this warp's A rows are written
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
                        __syncwarp();  // every lane has read its A_bb
#pragma unroll
                        for (int rr = 0; rr < 16; ++rr) X[(16 * b + rr) * LDF + 16 * b + jj] = x[rr];
                    }
                    ptx::named_barrier(BAR_P, NP);
                }
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
            }
            // X but its lower-left 32x32 block (fp32) is handed to the state group, which completes
            // it (X_21) and forms T = X Diag(beta)
            if (ptx::named_barrier_or(BAR_P, NP, *s_abort != 0)) break;
            if (leader) sarrive(S_TP, ci);
        }
        // the factor that restores S^T from TMEM after the last chunk, in the vector buffer the
        // state group read two chunks ago
        if (!*reinterpret_cast<volatile int *>(s_abort)) {
            if (Rb == 0 && hh == 0)
                *reinterpret_cast<float4 *>(vec(nchunks & 1, VEC_FR) + c0) =
                    make_float4(ecm_prev[0], ecm_prev[1], ecm_prev[2], ecm_prev[3]);
            ptx::named_barrier(BAR_P, NP);
            if (leader) sarrive(S_P2, nchunks);
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
    if (a.split.num_units > 0 || a.split.num_seqs > 0) return launch_tc<true, true>(maps, a, stream);
    return launch_tc<true, false>(maps, a, stream);
}

}  // namespace kda
