// kda_prefill_noalloc: kda_prefill for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the operator:
// code that runs under a custom allocator they do not own, plug-ins invoked with
// only input and output pointers, or paths where an allocation would synchronise
// the device or fail under memory pressure.  This entry point takes no workspace:
// the scratch that kda_prefill keeps in the caller's workspace (a device status
// word and the longest-first sequence order) lives in one file-scope device array
// instead.  Every GPU that loads this library holds that array until the process
// exits.  It never splits a long sequence into segments (the split keeps segment
// start states in the workspace), so each (sequence, head) is one unit; for inputs
// that kda_prefill runs unsplit, the launches and results are the same as its.
#include <mutex>

#include "kda_internal.h"

namespace {

// Scratch layout inside the array: [0, 256) status words, [256, ...) order.
constexpr int kMaxSeqs = KDA_NOALLOC_MAX_SEQS;
constexpr size_t kScratchBytes = kda::WorkspaceLayout::kStatusBytes + sizeof(int32_t) * size_t(kMaxSeqs);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device.  Host code cannot use the array's name as a device address.
cudaError_t scratch_on_current_device(void **out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" KDA_API kda_status_t kda_prefill_noalloc(const void *q, const void *k, const void *v,
                                                    kda_dtype_t qkv_dtype, const float *log_alpha,
                                                    const float *beta, const float *S0,
                                                    const int32_t *cu_seqlens_dev,
                                                    const int32_t *cu_seqlens_host, int num_seqs,
                                                    int H, int d_k, int d_v, int chunk, void *o,
                                                    float *S_final, kda_stream_t stream) {
    if (num_seqs > kMaxSeqs) return KDA_ERR_WORKSPACE;
    // The same host-side checks as kda_prefill; nothing is queued before they pass.
    if (num_seqs < 0 || H < 1 || d_k < 1 || d_v < 1) return KDA_ERR_INVALID_ARG;
    if (qkv_dtype != KDA_DTYPE_F32 && qkv_dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (chunk != 16 && chunk != 32 && chunk != 64) return KDA_ERR_UNSUPPORTED;
    if (d_k > 128 || d_v > 128) return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens_host || !cu_seqlens_dev || !S_final) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host[0] != 0) return KDA_ERR_INVALID_ARG;
    int max_len = 0;
    for (int n = 0; n < num_seqs; ++n) {
        const int64_t len = int64_t(cu_seqlens_host[n + 1]) - cu_seqlens_host[n];
        if (len < 0) return KDA_ERR_INVALID_ARG;
        if (len > max_len) max_len = int(len);
    }
    const int64_t T = cu_seqlens_host[num_seqs];
    if (T > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_INVALID_ARG;
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!al16(S_final) || (S0 && !al16(S0))) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al16(log_alpha))) return KDA_ERR_INVALID_ARG;
    if (num_seqs == 0) return KDA_OK;

    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return KDA_ERR_CUDA;

    kda::PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.dtype = qkv_dtype;
    a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0;
    a.cu_seqlens = cu_seqlens_dev;
    a.num_seqs = num_seqs; a.H = H; a.dk = d_k; a.dv = d_v; a.chunk = chunk;
    a.total_tokens = T; a.max_seqlen = max_len;
    a.o = o; a.S_final = S_final;
    a.status = static_cast<kda::DeviceStatus *>(scratch);
    a.order = reinterpret_cast<int32_t *>(static_cast<char *>(scratch) + kda::WorkspaceLayout::kStatusBytes);

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: the status word must start at
    // zero; the order is rewritten in full by its kernel.
    if (cudaMemsetAsync(a.status, 0, sizeof(kda::DeviceStatus), st) != cudaSuccess) return KDA_ERR_CUDA;
    if (kda::launch_order_by_length(a, st) != cudaSuccess) return KDA_ERR_CUDA;
    const cudaError_t err = kda::prefill_tc_supported(a) ? kda::launch_prefill_tc(a, st)
                                                         : kda::launch_prefill_simt(a, st);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
