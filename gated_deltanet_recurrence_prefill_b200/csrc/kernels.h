// kernels.h -- internal launch interface between the C ABI (gdn_api.cu) and
// the kernels.  Not installed; the public interface is include/gdn.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

struct PrefillArgs {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    const float* a;
    const float* b;
    const float* A_log;
    const float* dt_bias;
    const int32_t* cu_seqlens;     // NULL: one sequence of length T
    int32_t n_seq;
    int64_t T;
    int32_t Hqk;
    int32_t Hv;
    float scale;
    const float* initial_state;    // may be NULL
    float* final_state;            // may be NULL
    float* o;                      // may be NULL when y or o16 is given
    void* workspace;
    size_t workspace_bytes;
    // fused gated output norm (producer / consumer kernel only): y = norm_w * o /
    // sqrt(mean_v o^2 + eps) * silu(z), bf16, when y != NULL
    const uint16_t* z = nullptr;
    const float* norm_w = nullptr;
    float eps = 0.f;
    uint16_t* y = nullptr;
    uint16_t* o16 = nullptr;       // o stored as bf16 instead of o (round to nearest even)
};

// the gated output norm fused into a decode step (y == NULL: none); norm_w is
// [layers, d], row u of the batch uses layer u % layers
struct DecodeNorm {
    const uint16_t* z = nullptr;
    const float* w = nullptr;
    float eps = 0.f;
    uint16_t* y = nullptr;
};

cudaError_t launch_decode_step(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const float* a, const float* b, const float* A_log,
                               const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                               int32_t Hv, float scale, float* state, float* o,
                               cudaStream_t stream, const DecodeNorm& nrm = DecodeNorm());

cudaError_t launch_decode_step_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const float* a, const float* b, const float* A_log,
                                    const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                                    int32_t Hv, float scale, uint16_t* state, float* o,
                                    cudaStream_t stream, const DecodeNorm& nrm = DecodeNorm());

cudaError_t launch_decode_fused_bf16(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                     const float* a, const float* b, const float* A_log,
                                     const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                     int32_t layers, int32_t Hqk, int32_t Hv, float scale,
                                     uint16_t* state, float* o, cudaStream_t stream);

cudaError_t launch_decode_fused(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                const float* a, const float* b, const float* A_log,
                                const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                int32_t layers, int32_t Hqk, int32_t Hv, float scale, float* state,
                                float* o, cudaStream_t stream);

cudaError_t launch_conv1d_silu(const uint16_t* qkv, const float* w, const int32_t* cu,
                               int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv,
                               const float* cs_in, float* cs_out, uint16_t* q, uint16_t* k,
                               uint16_t* v, cudaStream_t stream);

struct BackwardArgs {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    const float* a;
    const float* b;
    const float* A_log;
    const float* dt_bias;
    const int32_t* cu_seqlens;     // NULL: one sequence of length T
    int32_t n_seq;
    int64_t T;
    int32_t Hqk;
    int32_t Hv;
    float scale;
    const float* initial_state;    // may be NULL
    const float* d_o;
    const float* d_final_state;    // may be NULL
    float* dq;
    float* dk;
    float* dv;
    float* da;
    float* db;
    float* dA_log;
    float* ddt_bias;
    float* d_initial_state;        // may be NULL
    void* workspace;
};
size_t backward_workspace_bytes(int32_t n_seq, int64_t T, int32_t Hv);
cudaError_t launch_selftest_wait(int which, uint64_t limit_ns, void* workspace, cudaStream_t stream);
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t stream);
// the same gradient through the chunked form (backward_chunked.cu): two chains
// over chunks and chunk-parallel work; workspace of backward_chunked_workspace_bytes
size_t backward_chunked_workspace_bytes(int32_t n_seq, int64_t T, int32_t Hv);

// the front end's gradient (conv1d_silu_backward.cu)
struct ConvBackwardArgs {
    const uint16_t* qkv;
    const float* conv_w;
    const int32_t* cu_seqlens;     // NULL: one sequence of length T
    int32_t n_seq;
    int64_t T;
    int32_t Hqk;
    int32_t Hv;
    const float* conv_state;       // may be NULL
    const float* dq;
    const float* dk;
    const float* dv;
    float* d_qkv;
    float* d_conv_w;
    float* d_conv_state;           // may be NULL
    void* workspace;
};
size_t conv1d_silu_backward_workspace_bytes(int64_t T, int32_t Hqk, int32_t Hv);
// the gated output norm's gradient (gated_norm_backward.cu)
size_t gated_norm_backward_workspace_bytes(int64_t T, int32_t Hv, int32_t layers);
cudaError_t launch_gated_norm_backward(const float* o, const uint16_t* z, const float* w, const float* dy,
                                       int64_t T, int32_t Hv, int32_t layers, float eps, float* d_o, float* d_z,
                                       float* d_w, void* workspace, cudaStream_t stream);
cudaError_t launch_conv1d_silu_backward(const ConvBackwardArgs& a, cudaStream_t stream);
cudaError_t launch_backward_chunked(const BackwardArgs& a, cudaStream_t stream);

cudaError_t launch_gated_norm(const float* o, const uint16_t* z, const float* w, int64_t T, int32_t Hv,
                              int32_t layers, float eps, uint16_t* y, cudaStream_t stream);
cudaError_t launch_prefill_tc(const PrefillArgs& p, cudaStream_t stream);
size_t prefill_tc_smem_bytes();
// producer / consumer prefill: a cooperative grid of one consumer and one or
// two producer CTAs per (sequence, value head), handing chunks over through a
// ring in the workspace; available when at least two of its CTAs can be
// resident and the workspace holds one unit's ring
cudaError_t launch_prefill_pc(const PrefillArgs& p, cudaStream_t stream);
bool prefill_pc_available(size_t workspace_bytes);
size_t prefill_pc_smem_bytes();
// workspace with which the producer / consumer kernel runs every unit of a
// launch that fits on the device (the header, counters and rings)
size_t prefill_pc_workspace_bytes(int32_t n_seq, int32_t Hv);
// workspace the single-CTA kernel needs (and the least gdn_prefill accepts)
size_t prefill_min_workspace_bytes(int32_t n_seq, int32_t Hv);

// workspace layout shared by the prefill kernels
constexpr size_t kWsErrorWordOffset = 0;     // uint32 error word (0 = ok)
constexpr size_t kWsHeaderBytes = 256;

// device address of the library-owned prefill scratch array (the workspace of
// gdn_prefill_noalloc) on the current device, looked up once per device and
// cached; null if the lookup fails.  Allocates nothing.
void* noalloc_scratch();
// records e for gdn_last_cuda_error and returns GDN_ERR_CUDA (gdn_api.cu)
gdn_status set_last_cuda_error(cudaError_t e);
size_t noalloc_scratch_bytes();

}  // namespace gdn
