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
struct WorkspaceLayout {
    static constexpr size_t kStatusBytes = 256;
    size_t order_offset = kStatusBytes;
    size_t total = 0;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WorkspaceLayout workspace_layout(int num_seqs) {
    WorkspaceLayout L;
    L.order_offset = WorkspaceLayout::kStatusBytes;
    L.total = align256(L.order_offset + sizeof(int32_t) * size_t(num_seqs > 0 ? num_seqs : 1));
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
cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream);
// The output epilogue in place over a.o (after a prefill that does not fuse it).
cudaError_t launch_gated_rmsnorm(const PrefillArgs &a, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

}  // namespace kda

namespace kda {
size_t prefill_simt_smem_bytes(int chunk, int dk);
}  // namespace kda
