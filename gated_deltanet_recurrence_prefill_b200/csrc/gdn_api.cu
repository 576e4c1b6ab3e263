// gdn_api.cu -- the C ABI of libgdn (see include/gdn.h): argument checks on the
// host, then kernel launches on the caller's stream.  Nothing here allocates,
// frees or synchronises, except gdn_prefill_status, which documents that it
// waits for the stream (gdn_check_async is its non-waiting form).
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include "../../include/gdn.h"
#include "kernels.h"

namespace {

thread_local int g_last_cuda_error = 0;

gdn_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return GDN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int32_t kD = 128;

gdn_status check_heads(int32_t Hqk, int32_t Hv, int32_t d) {
    if (Hqk <= 0 || Hv <= 0 || d <= 0) return GDN_ERR_INVALID_ARG;
    if (d != kD) return GDN_ERR_UNSUPPORTED;
    if (Hv % Hqk != 0) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

gdn_status check_seqs(const int32_t* cu_seqlens, int32_t n_seq, int64_t T) {
    if (T < 0 || n_seq <= 0) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && n_seq != 1) return GDN_ERR_INVALID_ARG;
    if (T > (int64_t)0x7fffffff) return GDN_ERR_UNSUPPORTED;   // cu_seqlens are int32
    return GDN_OK;
}

// Which prefill kernel runs: the producer / consumer kernel (two or one
// producer CTAs and one consumer CTA per sequence and value head) when it can
// run on the device and the workspace holds at least one unit's ring, else the
// single-CTA kernel.  GDN_PREFILL_KERNEL=single or =pc in the environment
// forces one of them (for comparisons and tests).
enum class PrefillKernel { ProducerConsumer, Single, Unavailable };

PrefillKernel pick_prefill_kernel(size_t workspace_bytes) {
    const char* env = getenv("GDN_PREFILL_KERNEL");
    if (env && strcmp(env, "single") == 0) return PrefillKernel::Single;
    const bool pc = gdn::prefill_pc_available(workspace_bytes);
    if (env && strcmp(env, "pc") == 0) return pc ? PrefillKernel::ProducerConsumer : PrefillKernel::Unavailable;
    return pc ? PrefillKernel::ProducerConsumer : PrefillKernel::Single;
}

}  // namespace

namespace gdn {
// for the entry points defined in other files
gdn_status set_last_cuda_error(cudaError_t e) { return cuda_fail(e); }
}  // namespace gdn


namespace gdn {

size_t prefill_min_workspace_bytes(int32_t n_seq, int32_t Hv) {
    const size_t n = n_seq > 0 ? (size_t)n_seq : 1;
    const size_t hv = Hv > 0 ? (size_t)Hv : 1;
    // header (error word) + one int32 per (sequence, value head)
    return kWsHeaderBytes + ((n * hv * sizeof(int32_t) + 255) / 256) * 256;
}

}  // namespace gdn

extern "C" {

int gdn_abi_version(void) { return GDN_ABI_VERSION; }

const char* gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported shape";
        case GDN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "bounded device wait timed out";
        case GDN_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int gdn_last_cuda_error(void) { return g_last_cuda_error; }

const char* gdn_last_cuda_error_string(void) {
    return cudaGetErrorName((cudaError_t)g_last_cuda_error);
}

gdn_status gdn_conv1d_silu(const uint16_t* qkv, const float* conv_w, const int32_t* cu_seqlens,
                           int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv, int32_t d,
                           const float* conv_state_in, float* conv_state_out, uint16_t* q,
                           uint16_t* k, uint16_t* v, gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if ((st = check_seqs(cu_seqlens, n_seq, T)) != GDN_OK) return st;
    if (!conv_w || (T > 0 && (!qkv || !q || !k || !v))) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {qkv, conv_w, cu_seqlens, conv_state_in, conv_state_out, q, k, v};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    if (conv_state_in && conv_state_in == conv_state_out) return GDN_ERR_INVALID_ARG;
    cudaError_t e = gdn::launch_conv1d_silu(qkv, conv_w, cu_seqlens, n_seq, T, Hqk, Hv,
                                            conv_state_in, conv_state_out, q, k, v,
                                            (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

size_t gdn_conv1d_silu_backward_workspace_size(int64_t T, int32_t Hqk, int32_t Hv, int32_t d) {
    (void)d;
    if (T <= 0 || Hqk <= 0 || Hv <= 0) return 0;
    return gdn::conv1d_silu_backward_workspace_bytes(T, Hqk, Hv);
}

gdn_status gdn_conv1d_silu_backward(const uint16_t* qkv, const float* conv_w, const int32_t* cu_seqlens,
                                    int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv, int32_t d,
                                    const float* conv_state, const float* dq, const float* dk, const float* dv,
                                    float* d_qkv, float* d_conv_w, float* d_conv_state, void* workspace,
                                    size_t workspace_bytes, gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if ((st = check_seqs(cu_seqlens, n_seq, T)) != GDN_OK) return st;
    if (!conv_w || !d_conv_w || (T > 0 && (!qkv || !dq || !dk || !dv || !d_qkv))) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {qkv, conv_w, cu_seqlens, conv_state, dq, dk, dv, d_qkv, d_conv_w, d_conv_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    const size_t need = T > 0 ? gdn::conv1d_silu_backward_workspace_bytes(T, Hqk, Hv) : 0;
    if (need > 0 && (!workspace || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;
    gdn::ConvBackwardArgs a{qkv, conv_w, cu_seqlens, n_seq, T, Hqk, Hv, conv_state, dq, dk, dv,
                            d_qkv, d_conv_w, d_conv_state, workspace};
    cudaError_t e = gdn::launch_conv1d_silu_backward(a, (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

size_t gdn_prefill_workspace_size(int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv, int32_t d) {
    (void)T; (void)Hqk; (void)d;
    const size_t lo = gdn::prefill_min_workspace_bytes(n_seq, Hv);
    const size_t hi = gdn::prefill_pc_workspace_bytes(n_seq, Hv);
    return hi > lo ? hi : lo;
}

gdn_status gdn_prefill(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                       const float* b, const float* A_log, const float* dt_bias,
                       const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                       int32_t Hv, int32_t d, float scale, const float* initial_state,
                       float* final_state, float* o, void* workspace, size_t workspace_bytes,
                       gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if ((st = check_seqs(cu_seqlens, n_seq, T)) != GDN_OK) return st;
    if (!A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !a || !b || !o)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, final_state,
                          o};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < gdn::prefill_min_workspace_bytes(n_seq, Hv))
        return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;
    gdn::PrefillArgs p{q, k, v, a, b, A_log, dt_bias, cu_seqlens, n_seq, T, Hqk, Hv, scale,
                       initial_state, final_state, o, workspace, workspace_bytes};
    const PrefillKernel which = pick_prefill_kernel(workspace_bytes);
    if (which == PrefillKernel::Unavailable) return GDN_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(workspace, 0, gdn::kWsHeaderBytes, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = which == PrefillKernel::ProducerConsumer ? gdn::launch_prefill_pc(p, s) : gdn::launch_prefill_tc(p, s);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_prefill_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                            const float* b, const float* A_log, const float* dt_bias,
                            const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                            int32_t Hv, int32_t d, float scale, const float* initial_state,
                            float* final_state, uint16_t* o, void* workspace, size_t workspace_bytes,
                            gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if ((st = check_seqs(cu_seqlens, n_seq, T)) != GDN_OK) return st;
    if (!A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !a || !b || !o)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, final_state,
                          o};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < gdn::prefill_min_workspace_bytes(n_seq, Hv))
        return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;
    gdn::PrefillArgs p{q, k, v, a, b, A_log, dt_bias, cu_seqlens, n_seq, T, Hqk, Hv, scale,
                       initial_state, final_state, nullptr, workspace, workspace_bytes};
    p.o16 = o;
    const PrefillKernel which = pick_prefill_kernel(workspace_bytes);
    if (which == PrefillKernel::Unavailable) return GDN_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(workspace, 0, gdn::kWsHeaderBytes, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = which == PrefillKernel::ProducerConsumer ? gdn::launch_prefill_pc(p, s) : gdn::launch_prefill_tc(p, s);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_prefill_gated(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                             const float* b, const float* A_log, const float* dt_bias,
                             const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                             int32_t Hv, int32_t d, float scale, const float* initial_state,
                             float* final_state, float* o, const uint16_t* z, const float* norm_w,
                             float eps, uint16_t* y, void* workspace, size_t workspace_bytes,
                             gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if ((st = check_seqs(cu_seqlens, n_seq, T)) != GDN_OK) return st;
    if (!A_log || !dt_bias || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !a || !b || !z || !norm_w || !y)) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, final_state,
                          o, z, norm_w, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < gdn::prefill_min_workspace_bytes(n_seq, Hv))
        return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;
    gdn::PrefillArgs p{q, k, v, a, b, A_log, dt_bias, cu_seqlens, n_seq, T, Hqk, Hv, scale,
                       initial_state, final_state, o, workspace, workspace_bytes};
    p.z = z;
    p.norm_w = norm_w;
    p.eps = eps;
    p.y = y;
    const PrefillKernel which = pick_prefill_kernel(workspace_bytes);
    if (which == PrefillKernel::Unavailable) return GDN_ERR_UNSUPPORTED;
    // the single-CTA kernel has no fused norm: it needs o, then the norm runs on it
    if (which == PrefillKernel::Single && T > 0 && !o) return GDN_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(workspace, 0, gdn::kWsHeaderBytes, s);
    if (e != cudaSuccess) return cuda_fail(e);
    // Without o the norm runs inside the producer / consumer kernel (o never goes
    // through memory).  With o, the prefill writes o and gdn_gated_norm runs on
    // it: two launches, and the faster of the two on B200, where the fused norm's
    // exponentials on the consumer's SM lengthen the state chain more than the
    // second pass costs.  GDN_PREFILL_NORM=fused forces the fused kernel.
    const char* env = getenv("GDN_PREFILL_NORM");
    const bool fused = which == PrefillKernel::ProducerConsumer &&
                       (!o || (env && strcmp(env, "fused") == 0));
    if (fused) {
        e = gdn::launch_prefill_pc(p, s);
    } else {
        p.z = nullptr;
        p.norm_w = nullptr;
        p.y = nullptr;
        e = which == PrefillKernel::ProducerConsumer ? gdn::launch_prefill_pc(p, s) : gdn::launch_prefill_tc(p, s);
        if (e == cudaSuccess && T > 0) e = gdn::launch_gated_norm(o, z, norm_w, T, Hv, 1, eps, y, s);
    }
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_prefill_status(const void* workspace, gdn_stream_t stream) {
    if (!workspace) workspace = gdn::noalloc_scratch();
    if (!workspace) return GDN_ERR_CUDA;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, (const char*)workspace + gdn::kWsErrorWordOffset,
                                    sizeof word, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return word == 0 ? GDN_OK : GDN_ERR_TIMEOUT;
}

gdn_status gdn_check_async(const void* workspace, uint32_t* status_word, gdn_stream_t stream) {
    if (!status_word) return GDN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(status_word) & 3u) != 0) return GDN_ERR_MISALIGNED;
    if (!workspace) workspace = gdn::noalloc_scratch();
    if (!workspace) return GDN_ERR_CUDA;
    // a 4-byte copy enqueued behind the prefill; the host does not wait
    cudaError_t e = cudaMemcpyAsync(status_word, (const char*)workspace + gdn::kWsErrorWordOffset,
                                    sizeof(uint32_t), cudaMemcpyDefault, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return GDN_OK;
}

gdn_status gdn_decode_step(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const float* a, const float* b, const float* A_log,
                           const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                           int32_t Hv, int32_t d, float scale, float* state, float* o,
                           gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if (n_seq < 0 || layers <= 0) return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !o)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, state, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return GDN_ERR_MISALIGNED;
    cudaError_t e = gdn::launch_decode_step(q, k, v, a, b, A_log, dt_bias, n_seq, layers, Hqk,
                                            Hv, scale, state, o, (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_decode_step_fused(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                 const float* a, const float* b, const float* A_log,
                                 const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                 int32_t layers, int32_t Hqk, int32_t Hv, int32_t d, float scale,
                                 int32_t n_slots, float* state, float* o, gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if (n_seq < 0 || layers <= 0 || n_slots <= 0) return GDN_ERR_INVALID_ARG;
    if (!slot && n_slots < n_seq) return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    if (!qkv || !conv_w || !conv_state || !a || !b || !A_log || !dt_bias || !state || !o)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {qkv, conv_w, conv_state, a, b, A_log, dt_bias, slot, state, o};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    cudaError_t e = gdn::launch_decode_fused(qkv, conv_w, conv_state, a, b, A_log, dt_bias, slot, n_seq,
                                             layers, Hqk, Hv, scale, state, o, (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_decode_step_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const float* a, const float* b, const float* A_log,
                                const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                                int32_t Hv, int32_t d, float scale, uint16_t* state, float* o,
                                gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if (n_seq < 0 || layers <= 0) return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !o)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, state, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return GDN_ERR_MISALIGNED;
    cudaError_t e = gdn::launch_decode_step_bf16(q, k, v, a, b, A_log, dt_bias, n_seq, layers, Hqk, Hv,
                                                 scale, state, o, (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_decode_step_fused_bf16(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                      const float* a, const float* b, const float* A_log,
                                      const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                      int32_t layers, int32_t Hqk, int32_t Hv, int32_t d, float scale,
                                      int32_t n_slots, uint16_t* state, float* o, gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if (n_seq < 0 || layers <= 0 || n_slots <= 0) return GDN_ERR_INVALID_ARG;
    if (!slot && n_slots < n_seq) return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    if (!qkv || !conv_w || !conv_state || !a || !b || !A_log || !dt_bias || !state || !o)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {qkv, conv_w, conv_state, a, b, A_log, dt_bias, slot, state, o};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    cudaError_t e = gdn::launch_decode_fused_bf16(qkv, conv_w, conv_state, a, b, A_log, dt_bias, slot,
                                                  n_seq, layers, Hqk, Hv, scale, state, o,
                                                  (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_decode_step_gated(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const float* a, const float* b, const float* A_log,
                                 const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                                 int32_t Hv, int32_t d, float scale, void* state, int32_t state_bf16,
                                 float* o, const uint16_t* z, const float* norm_w, float eps,
                                 uint16_t* y, gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if (n_seq < 0 || layers <= 0 || !(eps >= 0.f) || (state_bf16 != 0 && state_bf16 != 1))
        return GDN_ERR_INVALID_ARG;
    if (n_seq == 0) return GDN_OK;
    if (!q || !k || !v || !a || !b || !A_log || !dt_bias || !state || !z || !norm_w || !y)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, state, o, z, norm_w, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    gdn::DecodeNorm nrm;
    nrm.z = z;
    nrm.w = norm_w;
    nrm.eps = eps;
    nrm.y = y;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = state_bf16
        ? gdn::launch_decode_step_bf16(q, k, v, a, b, A_log, dt_bias, n_seq, layers, Hqk, Hv, scale,
                                       static_cast<uint16_t*>(state), o, s, nrm)
        : gdn::launch_decode_step(q, k, v, a, b, A_log, dt_bias, n_seq, layers, Hqk, Hv, scale,
                                  static_cast<float*>(state), o, s, nrm);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

size_t gdn_prefill_backward_workspace_size(int32_t n_seq, int64_t T, int32_t Hv, int32_t d) {
    (void)d;
    return gdn::backward_workspace_bytes(n_seq > 0 ? n_seq : 1, T > 0 ? T : 0, Hv > 0 ? Hv : 1);
}

size_t gdn_prefill_backward_chunked_workspace_size(int32_t n_seq, int64_t T, int32_t Hv, int32_t d) {
    (void)d;
    return gdn::backward_chunked_workspace_bytes(n_seq > 0 ? n_seq : 1, T > 0 ? T : 0, Hv > 0 ? Hv : 1);
}

}  // extern "C"

namespace {

// the arguments both backward entry points take, checked; runs the token-by-token
// kernel or the chunked one
gdn_status prefill_backward_common(bool chunked, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                   const float* a, const float* b, const float* A_log, const float* dt_bias,
                                   const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv,
                                   int32_t d, float scale, const float* initial_state, const float* d_o,
                                   const float* d_final_state, float* dq, float* dk, float* dv, float* da,
                                   float* db, float* dA_log, float* ddt_bias, float* d_initial_state,
                                   void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    gdn_status st = check_heads(Hqk, Hv, d);
    if (st != GDN_OK) return st;
    if ((st = check_seqs(cu_seqlens, n_seq, T)) != GDN_OK) return st;
    if (!A_log || !dt_bias || !dA_log || !ddt_bias) return GDN_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !a || !b || !d_o || !dq || !dk || !dv || !da || !db))
        return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, d_o, d_final_state,
                          dq, dk, dv, da, db, dA_log, ddt_bias, d_initial_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    const size_t need = chunked ? gdn::backward_chunked_workspace_bytes(n_seq, T, Hv)
                                : gdn::backward_workspace_bytes(n_seq, T, Hv);
    if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;
    gdn::BackwardArgs ba{q, k, v, a, b, A_log, dt_bias, cu_seqlens, n_seq, T, Hqk, Hv, scale,
                         initial_state, d_o, d_final_state, dq, dk, dv, da, db, dA_log, ddt_bias,
                         d_initial_state, workspace};
    cudaError_t e = chunked ? gdn::launch_backward_chunked(ba, (cudaStream_t)stream)
                            : gdn::launch_backward(ba, (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

gdn_status gdn_prefill_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                                const float* b, const float* A_log, const float* dt_bias,
                                const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                                int32_t Hv, int32_t d, float scale, const float* initial_state,
                                const float* d_o, const float* d_final_state, float* dq, float* dk,
                                float* dv, float* da, float* db, float* dA_log, float* ddt_bias,
                                float* d_initial_state, void* workspace, size_t workspace_bytes,
                                gdn_stream_t stream) {
    return prefill_backward_common(false, q, k, v, a, b, A_log, dt_bias, cu_seqlens, n_seq, T, Hqk, Hv, d, scale,
                                   initial_state, d_o, d_final_state, dq, dk, dv, da, db, dA_log, ddt_bias,
                                   d_initial_state, workspace, workspace_bytes, stream);
}

gdn_status gdn_prefill_backward_chunked(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                                        const float* b, const float* A_log, const float* dt_bias,
                                        const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                                        int32_t Hv, int32_t d, float scale, const float* initial_state,
                                        const float* d_o, const float* d_final_state, float* dq, float* dk,
                                        float* dv, float* da, float* db, float* dA_log, float* ddt_bias,
                                        float* d_initial_state, void* workspace, size_t workspace_bytes,
                                        gdn_stream_t stream) {
    return prefill_backward_common(true, q, k, v, a, b, A_log, dt_bias, cu_seqlens, n_seq, T, Hqk, Hv, d, scale,
                                   initial_state, d_o, d_final_state, dq, dk, dv, da, db, dA_log, ddt_bias,
                                   d_initial_state, workspace, workspace_bytes, stream);
}

gdn_status gdn_selftest_bounded_wait(int32_t which, int64_t limit_us, void* workspace, gdn_stream_t stream) {
    if ((which != 0 && which != 1) || limit_us < 1000 || limit_us > 2000000) return GDN_ERR_INVALID_ARG;
    if (!workspace) workspace = gdn::noalloc_scratch();      // the array of gdn_prefill_noalloc
    if (!workspace) return GDN_ERR_CUDA;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(workspace, 0, gdn::kWsHeaderBytes, s);
    if (e == cudaSuccess) e = gdn::launch_selftest_wait(which, (uint64_t)limit_us * 1000ull, workspace, s);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

size_t gdn_gated_norm_backward_workspace_size(int64_t T, int32_t Hv, int32_t d, int32_t layers) {
    (void)d;
    if (T <= 0 || Hv <= 0 || layers <= 0) return 0;
    return gdn::gated_norm_backward_workspace_bytes(T, Hv, layers);
}

gdn_status gdn_gated_norm_backward(const float* o, const uint16_t* z, const float* norm_w, const float* dy,
                                   int64_t T, int32_t Hv, int32_t d, int32_t layers, float eps, float* d_o,
                                   float* d_z, float* d_norm_w, void* workspace, size_t workspace_bytes,
                                   gdn_stream_t stream) {
    if (T < 0 || Hv <= 0 || d <= 0 || layers <= 0 || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (d != kD) return GDN_ERR_UNSUPPORTED;
    if (T > (int64_t)0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (!norm_w || !d_norm_w || (T > 0 && (!o || !z || !dy || !d_o || !d_z))) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {o, z, norm_w, dy, d_o, d_z, d_norm_w};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    const size_t need = T > 0 ? gdn::gated_norm_backward_workspace_bytes(T, Hv, layers) : 0;
    if (need > 0 && (!workspace || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;
    cudaError_t e = gdn::launch_gated_norm_backward(o, z, norm_w, dy, T, Hv, layers, eps, d_o, d_z, d_norm_w,
                                                    workspace, (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

gdn_status gdn_gated_norm(const float* o, const uint16_t* z, const float* norm_w, int64_t T, int32_t Hv,
                          int32_t d, int32_t layers, float eps, uint16_t* y, gdn_stream_t stream) {
    if (T < 0 || Hv <= 0 || d <= 0 || layers <= 0 || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
    if (d != kD) return GDN_ERR_UNSUPPORTED;
    if (T == 0) return GDN_OK;
    if (!o || !z || !norm_w || !y) return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {o, z, norm_w, y};
    for (const void* p : ptrs)
        if (!aligned16(p)) return GDN_ERR_MISALIGNED;
    cudaError_t e = gdn::launch_gated_norm(o, z, norm_w, T, Hv, layers, eps, y, (cudaStream_t)stream);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

}  // extern "C"
