// Internal declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// Layout of the prefill workspace (all offsets 256-byte aligned).
//   [0, 256)            device status words (error flag + detail)
//   [256, 256 + 4*N)    sequence order, longest first (int32)
// ---- sequence split (tensor-core prefill).  A sequence much longer than the rest
// would keep H SMs busy long after the others finish; it is cut into nseg segments.
// The recurrence is affine in the state, S_end = M S_start + L with M (d_k x d_k) the
// state's transition through a segment and L its end state from a zero start, so:
// pass A runs segment 0 from S0 and, for each middle segment, L (from zero) and M
// (from the identity, v = 0) in parallel; a small kernel chains
// S_start(p) = M(p-1) S_start(p-1) + L(p-1), p = 2 .. nseg - 1; pass B runs the other
// segments from their true start states.  nseg is as large as pass A's units
// (m H (2 nseg - 3) CTAs for m split sequences) fit on the device's SMs, between 3 and
// kMaxSplitP, with segments of at least kSplitMinSeg tokens.
constexpr int kMaxSplitP = 8;
constexpr int kMaxSplitSeqs = 8;
constexpr int kSplitMinLen = 16384;
constexpr int kSplitMinSeg = 4096;
constexpr int kMaxSplitUnits = kMaxSplitSeqs * (2 * kMaxSplitP - 3);
enum UnitMode : int32_t { UNIT_FIRST = 1, UNIT_LOCAL = 2, UNIT_HOMOG = 3, UNIT_CONT = 4, UNIT_LAST = 5 };
struct SplitUnit {
    int32_t bos, eos, seq, mode;
    int32_t slot;  // (split sequence j) * nseg + segment: the scratch state it reads or writes
};
struct SplitPlan {
    int num_units = 0;  // split units at the front of a launch
    int num_seqs = 0;   // split sequences, skipped where the plain ordering meets them
    int nseg = 3;       // segments per split sequence
    bool plain_units = true;  // the launch also runs every plain (sequence, head) after the split units
    int32_t seqs[kMaxSplitSeqs] = {};
    SplitUnit units[kMaxSplitUnits] = {};
    float *sstart = nullptr, *lmat = nullptr, *mmat = nullptr;  // [slot][H][128][128] float32 each
};

// Streaming multiprocessors of the current device (cudaDevAttrMultiProcessorCount,
// read once per device; 148, the B200's count, if the query fails).
int device_sm_count();

// Most sequences a split can take for these sizes on a device with `sms` SMs (the
// criterion in kda_api.cu: L >= kSplitMinLen and 2 L sms > 3 T H, so fewer than
// 2 sms / (3 H) sequences qualify).
inline int split_max_seqs(int64_t total_tokens, int H, int sms) {
    int64_t m = total_tokens / kSplitMinLen;
    m = m < kMaxSplitSeqs ? m : kMaxSplitSeqs;
    const int64_t by_h = 2 * int64_t(sms) / (3 * int64_t(H > 0 ? H : 1));
    return int(m < by_h ? m : by_h);
}

// Segments per split sequence when m sequences of at least `shortest` tokens are split:
// the most for which pass A's m H (2 nseg - 3) units fit on `sms` SMs, within
// [3, kMaxSplitP], and no shorter than kSplitMinSeg tokens a segment.
inline int split_segments(int m, int H, int sms, int64_t shortest) {
    const int64_t fit = (int64_t(sms) / (int64_t(m > 0 ? m : 1) * (H > 0 ? H : 1)) + 3) / 2;
    const int64_t by_len = shortest / kSplitMinSeg;
    int64_t p = fit < by_len ? fit : by_len;
    p = p < kMaxSplitP ? p : kMaxSplitP;
    return int(p > 3 ? p : 3);
}

struct WorkspaceLayout {
    static constexpr size_t kStatusBytes = 256;
    size_t order_offset = kStatusBytes;
    size_t split_offset = 0;  // three scratch state arrays when a split is possible
    size_t split_array_bytes = 0;
    size_t total = 0;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// split_states: room for a sequence split (tensor-core path only) on the current device.
inline WorkspaceLayout workspace_layout(int num_seqs, int64_t total_tokens = 0, int H = 0, bool split_states = false) {
    WorkspaceLayout L;
    L.order_offset = WorkspaceLayout::kStatusBytes;
    L.total = align256(L.order_offset + sizeof(int32_t) * size_t(num_seqs > 0 ? num_seqs : 1));
    const int m = split_states ? split_max_seqs(total_tokens, H, device_sm_count()) : 0;
    if (m > 0) {
        L.split_offset = L.total;
        // room for the most segments one split sequence can take on this device
        const int pmax = split_segments(1, H, device_sm_count(), int64_t(1) << 40);
        L.split_array_bytes = size_t(m) * pmax * size_t(H) * 128 * 128 * sizeof(float);
        L.total = align256(L.split_offset + 3 * L.split_array_bytes);
    }
    return L;
}

// Device status word: 0 = fine; otherwise an error code written by a kernel.
struct DeviceStatus {
    unsigned int flag;
    unsigned int detail;
};

struct PrefillArgs {
    const void *q, *k, *v;
    kda_dtype_t dtype;
    const float *log_alpha, *beta, *S0;
    const int32_t *cu_seqlens;
    int num_seqs, H, dk, dv, chunk;
    int64_t total_tokens;
    int max_seqlen;
    void *o;
    float *S_final;
    DeviceStatus *status;
    int32_t *order;       // sequence order (longest first), num_seqs entries
    SplitPlan split;  // empty: every unit is a plain (sequence, head)
    // output epilogue (kda_prefill_gated): o is replaced by o / sqrt(mean(o^2) + eps) * w * sigmoid(gate)
    const void *gate = nullptr;          // [T, H, d_v], dtype; nullptr = plain prefill
    const float *norm_weight = nullptr;  // [d_v]
    float eps = 0.f;
};

struct PrologueArgs {
    const void *q_pre, *k_pre, *v_pre;
    kda_dtype_t dtype;
    const float *conv_q, *conv_k, *conv_v;  // [H, d, W]
    int W;
    const float *a, *rate, *b;              // [T, H, d_k], [H], [T, H]
    const int32_t *cu_seqlens;              // device, num_seqs + 1
    int num_seqs, H, dk, dv;
    int64_t total_tokens;
    float l2_eps;
    void *q, *k, *v;
    float *log_alpha, *beta;
};

struct DecodeArgs {
    const void *q, *k, *v;
    kda_dtype_t dtype;
    const float *log_alpha, *beta;
    float *S;
    int B, H, dk, dv;
    void *o;
};

struct DecodeTokensArgs {
    const void *q, *k, *v;
    kda_dtype_t dtype;
    const float *log_alpha, *beta;
    float *S_pool;
    const int32_t *slot_idx;  // [B] or NULL (slot = b)
    int num_slots, B, n, H, dk, dv;
    void *o;
};

cudaError_t launch_order_by_length(const PrefillArgs &a, cudaStream_t stream);
cudaError_t launch_decode_tokens(const DecodeTokensArgs &a, cudaStream_t stream);
cudaError_t launch_prefill_simt(const PrefillArgs &a, cudaStream_t stream);
bool prefill_tc_supported(const PrefillArgs &a);
cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream);  // fuses the epilogue when a.gate is set
// S_start(p) = M(p-1) S_start(p-1) + L(p-1) for segment p of every split sequence.
cudaError_t launch_split_combine(const PrefillArgs &a, int p, cudaStream_t stream);
cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream);
// The output epilogue in place over a.o (after a prefill that does not fuse it).
cudaError_t launch_gated_rmsnorm(const PrefillArgs &a, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

}  // namespace kda

namespace kda {
size_t prefill_simt_smem_bytes(int chunk, int dk);
}  // namespace kda
