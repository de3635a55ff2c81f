// C-ABI entry points of the KDA library: argument checks on the host, then
// kernel launches on the caller's stream.  See include/kda.h for the contract.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "kda_internal.h"

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kda_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

bool dtype_ok(kda_dtype_t t) { return t == KDA_DTYPE_F32 || t == KDA_DTYPE_BF16; }

// The shapes the tensor-core prefill takes (it also needs T > 0 and N > 0 at run time).
bool tc_shape(int d_k, int d_v, int chunk, kda_dtype_t t) {
    return t == KDA_DTYPE_BF16 && d_k == 128 && d_v == 128 && chunk == 64;
}

// Shapes every prefill kernel here accepts.
kda_status_t check_prefill_shape(int num_seqs, int H, int d_k, int d_v, int chunk, kda_dtype_t dt) {
    if (num_seqs < 0 || H < 1 || d_k < 1 || d_v < 1 || !dtype_ok(dt)) return KDA_ERR_INVALID_ARG;
    if (chunk != 16 && chunk != 32 && chunk != 64) return KDA_ERR_UNSUPPORTED;
    if (d_k > 128 || d_v > 128) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// Checks shared by kda_prefill and kda_prefill_gated; fills `a` (o = out).  Sets
// *empty when there is nothing to launch (num_seqs == 0).
kda_status_t prepare_prefill(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                             const float *log_alpha, const float *beta, const float *S0,
                             const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int num_seqs, int H,
                             int d_k, int d_v, int chunk, void *out, float *S_final, void *workspace,
                             size_t workspace_bytes, kda::PrefillArgs &a, bool *empty) {
    const kda_status_t shape = check_prefill_shape(num_seqs, H, d_k, d_v, chunk, qkv_dtype);
    if (shape != KDA_OK) return shape;
    if (!cu_seqlens_host || !cu_seqlens_dev || !S_final) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host[0] != 0) return KDA_ERR_INVALID_ARG;
    int max_len = 0;
    for (int n = 0; n < num_seqs; ++n) {
        const int64_t len = int64_t(cu_seqlens_host[n + 1]) - cu_seqlens_host[n];
        if (len < 0) return KDA_ERR_INVALID_ARG;
        if (len > max_len) max_len = int(len);
    }
    const int64_t T = cu_seqlens_host[num_seqs];
    if (T > 0 && (!q || !k || !v || !log_alpha || !beta || !out)) return KDA_ERR_INVALID_ARG;
    if (!aligned16(S_final) || (S0 && !aligned16(S0))) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
                  !aligned16(log_alpha)))
        return KDA_ERR_INVALID_ARG;
    const kda::WorkspaceLayout wl = kda::workspace_layout(num_seqs);
    if (!workspace || workspace_bytes < wl.total) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_WORKSPACE;

    a.q = q; a.k = k; a.v = v; a.dtype = qkv_dtype;
    a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0;
    a.cu_seqlens = cu_seqlens_dev;
    a.num_seqs = num_seqs; a.H = H; a.dk = d_k; a.dv = d_v; a.chunk = chunk;
    a.total_tokens = T; a.max_seqlen = max_len;
    a.o = out; a.S_final = S_final;
    a.status = static_cast<kda::DeviceStatus *>(workspace);
    a.order = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + wl.order_offset);
    *empty = num_seqs == 0;
    return KDA_OK;
}

// Status reset and the length ordering every prefill launch starts with.
kda_status_t launch_prefill_prologue(const kda::PrefillArgs &a, cudaStream_t st) {
    if (cudaMemsetAsync(a.status, 0, sizeof(kda::DeviceStatus), st) != cudaSuccess) return KDA_ERR_CUDA;
    if (kda::launch_order_by_length(a, st) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}

// Plans the sequence split of the tensor-core prefill (see kda_internal.h) when the
// workspace has room: sequences with L >= kSplitMinLen whose critical path exceeds 1.5x
// the even spread of the whole call over the device's SMs (2 L SMs > 3 T H), longest first.
// Returns false (no split) otherwise.
bool plan_split(kda::PrefillArgs &a, const int32_t *cu_host, void *workspace, size_t workspace_bytes) {
    const kda::WorkspaceLayout wl = kda::workspace_layout(a.num_seqs, a.total_tokens, a.H, true);
    if (wl.split_offset == 0 || workspace_bytes < wl.total) return false;
    const int sms = kda::device_sm_count();
    const int m_max = kda::split_max_seqs(a.total_tokens, a.H, sms);
    int picked[kda::kMaxSplitSeqs];
    int m = 0;
    for (; m < m_max; ++m) {  // the longest qualifying sequences not yet picked
        int best = -1;
        int64_t best_len = 0;
        for (int n = 0; n < a.num_seqs; ++n) {
            const int64_t len = int64_t(cu_host[n + 1]) - cu_host[n];
            bool taken = false;
            for (int i = 0; i < m; ++i) taken |= picked[i] == n;
            if (taken || len < kda::kSplitMinLen || 2 * len * sms <= 3 * a.total_tokens * a.H) continue;
            if (len > best_len) best = n, best_len = len;
        }
        if (best < 0) break;
        picked[m] = best;
    }
    if (m == 0) return false;
    int64_t shortest = INT64_MAX;
    for (int j = 0; j < m; ++j) {
        const int64_t len = int64_t(cu_host[picked[j] + 1]) - cu_host[picked[j]];
        shortest = len < shortest ? len : shortest;
    }
    a.split.nseg = kda::split_segments(m, a.H, sms, shortest);
    char *base = static_cast<char *>(workspace) + wl.split_offset;
    a.split.sstart = reinterpret_cast<float *>(base);
    a.split.lmat = reinterpret_cast<float *>(base + wl.split_array_bytes);
    a.split.mmat = reinterpret_cast<float *>(base + 2 * wl.split_array_bytes);
    a.split.num_seqs = m;
    for (int j = 0; j < m; ++j) a.split.seqs[j] = picked[j];
    return true;
}

// Segment p of nseg of a split sequence: chunk-aligned, equal (the last one takes the rest).
void segment_bounds(const int32_t *cu_host, int seq, int p, int nseg, int32_t *b, int32_t *e) {
    const int32_t bos = cu_host[seq], eos = cu_host[seq + 1];
    const int32_t chunks = (eos - bos + 63) / 64;
    const int32_t seg = (chunks + nseg - 1) / nseg * 64;
    *b = bos + p * seg < eos ? bos + p * seg : eos;
    *e = p == nseg - 1 ? eos : (bos + (p + 1) * seg < eos ? bos + (p + 1) * seg : eos);
}

// A second, high-priority stream and two events per device for the split: it runs the
// split units, the chain of start states and pass B (the critical path), while the
// caller's stream runs the plain sequences, which they do not depend on.  Created
// once, never destroyed.
struct SideStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

// Held across a split's whole fork / launches / join sequence: the side stream and its
// events are shared by every caller on the device.
std::mutex g_side_mu;

bool side_stream(SideStream *out) {  // call with g_side_mu held
    static SideStream per_device[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    SideStream &s = per_device[dev];
    if (!s.stream) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) greatest = 0;
        if (cudaStreamCreateWithPriority(&s.stream, cudaStreamNonBlocking, greatest) != cudaSuccess) return false;
        if (cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) != cudaSuccess) {
            s.stream = nullptr;
            return false;
        }
    }
    *out = s;
    return true;
}

// Pass A, the chain of start states and pass B of the split units (kda_internal.h) on
// a high-priority side stream, issued first; the plain sequences on the caller's
// stream meanwhile; then the caller's stream waits for the side stream.  Without a
// side stream, everything runs in order on the caller's stream.
cudaError_t launch_prefill_tc_split(kda::PrefillArgs a, const int32_t *cu_host, cudaStream_t st) {
    using namespace kda;
    std::lock_guard<std::mutex> lock(g_side_mu);
    SideStream side;
    const bool forked = side_stream(&side);
    cudaStream_t chain = forked ? side.stream : st;
    cudaError_t err = cudaSuccess;
    if (forked) {
        err = cudaEventRecord(side.fork, st);
        if (err == cudaSuccess) err = cudaStreamWaitEvent(side.stream, side.fork, 0);
        if (err != cudaSuccess) return err;
    }
    const int P = a.split.nseg;
    int n = 0;
    for (int j = 0; j < a.split.num_seqs; ++j) {
        const int seq = a.split.seqs[j];
        int32_t b, e;
        segment_bounds(cu_host, seq, 0, P, &b, &e);
        a.split.units[n++] = SplitUnit{b, e, seq, UNIT_FIRST, j * P};
        for (int p = 1; p + 1 < P; ++p) {
            segment_bounds(cu_host, seq, p, P, &b, &e);
            a.split.units[n++] = SplitUnit{b, e, seq, UNIT_LOCAL, j * P + p};
            a.split.units[n++] = SplitUnit{b, e, seq, UNIT_HOMOG, j * P + p};
        }
    }
    a.split.num_units = n;
    a.split.plain_units = !forked;
    err = launch_prefill_tc(a, chain);
    for (int p = 2; p < P && err == cudaSuccess; ++p) err = launch_split_combine(a, p, chain);
    if (err != cudaSuccess) return err;
    PrefillArgs passB = a;
    n = 0;
    for (int j = 0; j < a.split.num_seqs; ++j) {
        const int seq = a.split.seqs[j];
        for (int p = 1; p < P; ++p) {
            int32_t b, e;
            segment_bounds(cu_host, seq, p, P, &b, &e);
            passB.split.units[n++] = SplitUnit{b, e, seq, p + 1 < P ? UNIT_CONT : UNIT_LAST, j * P + p};
        }
    }
    passB.split.num_units = n;
    passB.split.plain_units = false;
    err = launch_prefill_tc(passB, chain);
    if (err != cudaSuccess || !forked) return err;
    PrefillArgs plain = a;  // every plain (sequence, head); split sequences are skipped
    plain.split.num_units = 0;
    plain.split.plain_units = true;
    err = launch_prefill_tc(plain, st);
    if (err == cudaSuccess) err = cudaEventRecord(side.join, side.stream);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(st, side.join, 0);
    return err;
}

}  // namespace

namespace kda {

int device_sm_count() {
    constexpr int kMaxDevices = 64;
    static int per_device[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (per_device[dev] <= 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        per_device[dev] = n;
    }
    return per_device[dev];
}

}  // namespace kda

extern "C" {

const char *kda_status_string(kda_status_t s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_DEVICE_FAULT: return "KDA_ERR_DEVICE_FAULT";
    }
    return "KDA_ERR_UNKNOWN";
}

int kda_version(void) { return kVersion; }

size_t kda_prefill_workspace_size(int num_seqs, int64_t total_tokens, int H, int d_k, int d_v,
                                  int chunk, kda_dtype_t qkv_dtype) {
    if (total_tokens < 0 || total_tokens > INT32_MAX) return 0;
    if (check_prefill_shape(num_seqs, H, d_k, d_v, chunk, qkv_dtype) != KDA_OK) return 0;
    return kda::workspace_layout(num_seqs, total_tokens, H, tc_shape(d_k, d_v, chunk, qkv_dtype)).total;
}

kda_status_t kda_prefill(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                         const float *log_alpha, const float *beta, const float *S0,
                         const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                         int num_seqs, int H, int d_k, int d_v, int chunk, void *o,
                         float *S_final, void *workspace, size_t workspace_bytes,
                         kda_stream_t stream) {
    kda::PrefillArgs a;
    bool empty = false;
    const kda_status_t st0 = prepare_prefill(q, k, v, qkv_dtype, log_alpha, beta, S0, cu_seqlens_dev,
                                             cu_seqlens_host, num_seqs, H, d_k, d_v, chunk, o, S_final,
                                             workspace, workspace_bytes, a, &empty);
    if (st0 != KDA_OK || empty) return st0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const kda_status_t pro = launch_prefill_prologue(a, st);
    if (pro != KDA_OK) return pro;
    if (kda::prefill_tc_supported(a)) {
        if (plan_split(a, cu_seqlens_host, workspace, workspace_bytes))
            return from_cuda(launch_prefill_tc_split(a, cu_seqlens_host, st));
        return from_cuda(kda::launch_prefill_tc(a, st));
    }
    return from_cuda(kda::launch_prefill_simt(a, st));
}

kda_status_t kda_prefill_gated(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                               const float *log_alpha, const float *beta, const float *S0,
                               const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                               int num_seqs, int H, int d_k, int d_v, int chunk, const void *gate,
                               const float *norm_weight, float eps, void *y, float *S_final,
                               void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    kda::PrefillArgs a;
    bool empty = false;
    const kda_status_t st0 = prepare_prefill(q, k, v, qkv_dtype, log_alpha, beta, S0, cu_seqlens_dev,
                                             cu_seqlens_host, num_seqs, H, d_k, d_v, chunk, y, S_final,
                                             workspace, workspace_bytes, a, &empty);
    if (st0 != KDA_OK) return st0;
    if (!(eps > 0.f) || !std::isfinite(eps)) return KDA_ERR_INVALID_ARG;
    if (a.total_tokens > 0 && (!gate || !norm_weight || !aligned16(gate))) return KDA_ERR_INVALID_ARG;
    a.gate = gate;
    a.norm_weight = norm_weight;
    a.eps = eps;
    const bool fused = kda::prefill_tc_supported(a);
    if (!fused && qkv_dtype != KDA_DTYPE_F32 && a.total_tokens > 0) return KDA_ERR_UNSUPPORTED;
    if (empty) return KDA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const kda_status_t pro = launch_prefill_prologue(a, st);
    if (pro != KDA_OK) return pro;
    if (fused) {  // long sequences are split as in kda_prefill; the epilogue is per token
        if (plan_split(a, cu_seqlens_host, workspace, workspace_bytes))
            return from_cuda(launch_prefill_tc_split(a, cu_seqlens_host, st));
        return from_cuda(kda::launch_prefill_tc(a, st));
    }
    const cudaError_t err = kda::launch_prefill_simt(a, st);  // o into y, then the epilogue in place
    if (err != cudaSuccess) return KDA_ERR_CUDA;
    return from_cuda(kda::launch_gated_rmsnorm(a, st));
}

kda_status_t kda_prologue(const void *q_pre, const void *k_pre, const void *v_pre, kda_dtype_t dtype,
                          const float *conv_q, const float *conv_k, const float *conv_v, int conv_width,
                          const float *a_gate, const float *rate, const float *b_gate,
                          const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int num_seqs, int H,
                          int d_k, int d_v, float l2_eps, void *q, void *k, void *v, float *log_alpha,
                          float *beta, kda_stream_t stream) {
    if (num_seqs < 0 || H < 1 || d_k < 1 || d_v < 1 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if (!(l2_eps >= 0.f) || !std::isfinite(l2_eps)) return KDA_ERR_INVALID_ARG;
    if (conv_width < 1 || conv_width > 4) return KDA_ERR_UNSUPPORTED;
    if (d_k > 128 || d_v > 128 || (d_k % 4) != 0 || (d_v % 4) != 0) return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens_host || !cu_seqlens_dev || cu_seqlens_host[0] != 0) return KDA_ERR_INVALID_ARG;
    for (int n = 0; n < num_seqs; ++n)
        if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return KDA_ERR_INVALID_ARG;
    const int64_t T = cu_seqlens_host[num_seqs];
    if (T == 0) return KDA_OK;
    const void *ptrs[] = {q_pre, k_pre, v_pre, conv_q, conv_k, conv_v, a_gate, rate, b_gate, q, k, v,
                          log_alpha, beta};
    for (const void *p : ptrs)
        if (!p) return KDA_ERR_INVALID_ARG;
    const void *rows[] = {q_pre, k_pre, v_pre, a_gate, q, k, v, log_alpha};
    for (const void *p : rows)
        if (!aligned16(p)) return KDA_ERR_INVALID_ARG;
    kda::PrologueArgs a;
    a.q_pre = q_pre; a.k_pre = k_pre; a.v_pre = v_pre; a.dtype = dtype;
    a.conv_q = conv_q; a.conv_k = conv_k; a.conv_v = conv_v; a.W = conv_width;
    a.a = a_gate; a.rate = rate; a.b = b_gate;
    a.cu_seqlens = cu_seqlens_dev;
    a.num_seqs = num_seqs; a.H = H; a.dk = d_k; a.dv = d_v; a.total_tokens = T; a.l2_eps = l2_eps;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    return from_cuda(kda::launch_prologue(a, reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_decode_step(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                             const float *log_alpha, const float *beta, float *S, int B, int H,
                             int d_k, int d_v, void *o, kda_stream_t stream) {
    if (B < 0 || H < 1 || d_k < 1 || d_v < 1 || !dtype_ok(qkv_dtype)) return KDA_ERR_INVALID_ARG;
    if (d_k > 128 || d_v > 128 || (d_v % 4) != 0) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    if (!aligned16(S)) return KDA_ERR_INVALID_ARG;
    kda::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.dtype = qkv_dtype;
    a.log_alpha = log_alpha; a.beta = beta; a.S = S;
    a.B = B; a.H = H; a.dk = d_k; a.dv = d_v; a.o = o;
    return from_cuda(kda::launch_decode(a, reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_decode_tokens(const void *q, const void *k, const void *v, kda_dtype_t qkv_dtype,
                               const float *log_alpha, const float *beta, float *S_pool,
                               const int32_t *slot_idx, int num_slots, int B, int n, int H, int d_k,
                               int d_v, void *o, kda_stream_t stream) {
    if (B < 0 || n < 0 || H < 1 || d_k < 1 || d_v < 1 || num_slots < 0 || !dtype_ok(qkv_dtype))
        return KDA_ERR_INVALID_ARG;
    if (d_k > 128 || d_v > 128 || (d_v % 4) != 0) return KDA_ERR_UNSUPPORTED;
    if (!slot_idx && num_slots < B) return KDA_ERR_INVALID_ARG;
    if (B == 0 || n == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S_pool || !o) return KDA_ERR_INVALID_ARG;
    if (!aligned16(S_pool)) return KDA_ERR_INVALID_ARG;
    kda::DecodeTokensArgs a;
    a.q = q; a.k = k; a.v = v; a.dtype = qkv_dtype;
    a.log_alpha = log_alpha; a.beta = beta; a.S_pool = S_pool; a.slot_idx = slot_idx;
    a.num_slots = num_slots; a.B = B; a.n = n; a.H = H; a.dk = d_k; a.dv = d_v; a.o = o;
    return from_cuda(kda::launch_decode_tokens(a, reinterpret_cast<cudaStream_t>(stream)));
}

kda_status_t kda_workspace_status(const void *workspace, kda_stream_t stream) {
    if (!workspace) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
    kda::DeviceStatus h{};
    if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (h.flag == 0) return KDA_OK;
    if (cudaMemset(const_cast<void *>(workspace), 0, sizeof(h)) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_ERR_DEVICE_FAULT;
}

}  // extern "C"
