// layer_host.cu -- gdn_layer_prefill_host: the front end and the prefill of one
// layer from pinned host inputs to pinned host outputs, with the PCIe copies
// overlapped with the compute.
//
// The tokens are cut into ranges of whole 64-token chunks, the first of them a
// quarter as long as the others so that the first download starts early (the
// downloads, 24.6 KB per token against 20.9 KB up, are the longer direction).
// Range r's inputs go
// up on the upload stream into one of two device buffers, its front end and
// prefill run on the caller's stream (the front end continues range r-1's
// conv history, the prefill range r-1's state: gdn_conv1d_silu's
// conv_state_in/out and gdn_prefill's initial/final state), and its output goes
// down on the download stream from one of two output buffers.  So range r+1's
// upload and range r-1's download run while range r computes, and the step
// takes about the longer of the two copy directions instead of their sum.
// Events order the three streams; buffer r & 1 is reused by range r + 2 only
// after range r's compute (inputs) or download (outputs) is complete.
#include <cuda_runtime.h>

#include <vector>

#include "../../include/gdn.h"
#include "kernels.h"

namespace {

struct HostPlan {
    int64_t first;             // tokens of range 0 (a multiple of 64, or T)
    int64_t Tb;                // tokens of each later range (a multiple of 64): the buffers' size
    size_t pws, qkv, ab, qk, v, o, cs, st, bytes;   // byte offsets into the workspace
};

// token range r of the plan: [*t0, *t0 + *len)
void host_range(const HostPlan& p, int64_t T, int64_t r, int64_t* t0, int64_t* len) {
    const int64_t s = r == 0 ? 0 : p.first + (r - 1) * p.Tb;
    const int64_t n = r == 0 ? p.first : p.Tb;
    *t0 = s;
    *len = (T - s) < n ? (T - s) : n;
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

bool make_host_plan(int64_t T, int32_t Hqk, int32_t Hv, int32_t d, int32_t n_blocks, HostPlan& p) {
    if (T <= 0 || n_blocks <= 0) return false;
    const int64_t chunks = (T + 63) / 64;
    if (n_blocks == 1 || chunks < 2) {
        p.first = p.Tb = chunks * 64;
    } else {
        // range 0 takes a quarter share, the other n_blocks - 1 ranges the rest
        const int64_t share = (4 * chunks + 4 * n_blocks - 3 - 1) / (4 * n_blocks - 3);   // ceil(chunks / (n - 3/4))
        int64_t f = (share + 3) / 4;
        if (f < 1) f = 1;
        if (f > chunks - 1) f = chunks - 1;
        const int64_t rest = chunks - f;
        p.first = f * 64;
        p.Tb = ((rest + n_blocks - 2) / (n_blocks - 1)) * 64;
        if (p.Tb < p.first) p.Tb = p.first;
    }
    const size_t C = (size_t)(2 * Hqk + Hv) * d;
    size_t off = 0;
    // the prefill's workspace first: its error word is the first word of this one
    p.pws = off;  off = up256(off + gdn_prefill_workspace_size(1, p.Tb, Hqk, Hv, d));
    p.qkv = off;  off = up256(off + 2 * up256((size_t)p.Tb * C * 2));
    p.ab = off;   off = up256(off + 4 * up256((size_t)p.Tb * Hv * 4));
    p.qk = off;   off = up256(off + 2 * up256((size_t)p.Tb * Hqk * d * 2));
    p.v = off;    off = up256(off + (size_t)p.Tb * Hv * d * 2);
    p.o = off;    off = up256(off + 2 * up256((size_t)p.Tb * Hv * d * 4));
    p.cs = off;   off = up256(off + 2 * up256(C * 3 * 4));
    p.st = off;   off = up256(off + 2 * up256((size_t)Hv * d * d * 4));
    p.bytes = off;
    return true;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

size_t gdn_layer_prefill_host_workspace_size(int64_t T, int32_t Hqk, int32_t Hv, int32_t d, int32_t n_blocks) {
    HostPlan p;
    if (Hqk <= 0 || Hv <= 0 || d != 128 || Hv % Hqk != 0 || !make_host_plan(T, Hqk, Hv, d, n_blocks, p)) return 0;
    return p.bytes;
}

gdn_status gdn_layer_prefill_host(const uint16_t* h_qkv, const float* h_a, const float* h_b, const float* conv_w,
                                  const float* A_log, const float* dt_bias, const float* conv_state_in,
                                  const float* initial_state, int64_t T, int32_t Hqk, int32_t Hv, int32_t d,
                                  float scale, int32_t n_blocks, float* h_o, float* h_final_state,
                                  float* conv_state_out, void* workspace, size_t workspace_bytes,
                                  gdn_stream_t stream, gdn_stream_t upload_stream, gdn_stream_t download_stream) {
    if (Hqk <= 0 || Hv <= 0 || d <= 0 || Hv % Hqk != 0) return GDN_ERR_INVALID_ARG;
    if (d != 128) return GDN_ERR_UNSUPPORTED;
    if (T < 0 || n_blocks <= 0 || n_blocks > 4096) return GDN_ERR_INVALID_ARG;
    if (T == 0) return GDN_OK;
    if (!h_qkv || !h_a || !h_b || !conv_w || !A_log || !dt_bias || !h_o || !h_final_state)
        return GDN_ERR_INVALID_ARG;
    if (upload_stream == stream || download_stream == stream || upload_stream == download_stream)
        return GDN_ERR_INVALID_ARG;
    const void* ptrs[] = {h_qkv, h_a, h_b, conv_w, A_log, dt_bias, conv_state_in, initial_state, h_o,
                          h_final_state, conv_state_out};
    for (const void* ptr : ptrs)
        if (ptr && !al16(ptr)) return GDN_ERR_MISALIGNED;
    HostPlan pl;
    if (!make_host_plan(T, Hqk, Hv, d, n_blocks, pl)) return GDN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < pl.bytes) return GDN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_MISALIGNED;

    cudaStream_t s0 = (cudaStream_t)stream, su = (cudaStream_t)upload_stream, sd = (cudaStream_t)download_stream;
    char* ws = static_cast<char*>(workspace);
    const size_t C = (size_t)(2 * Hqk + Hv) * d;
    const int64_t nb = 1 + (T > pl.first ? (T - pl.first + pl.Tb - 1) / pl.Tb : 0);
    auto qkv_buf = [&](int b) { return reinterpret_cast<uint16_t*>(ws + pl.qkv + b * up256((size_t)pl.Tb * C * 2)); };
    auto ab_buf = [&](int i) { return reinterpret_cast<float*>(ws + pl.ab + i * up256((size_t)pl.Tb * Hv * 4)); };
    uint16_t* qb = reinterpret_cast<uint16_t*>(ws + pl.qk);
    uint16_t* kb = reinterpret_cast<uint16_t*>(ws + pl.qk + up256((size_t)pl.Tb * Hqk * d * 2));
    uint16_t* vb = reinterpret_cast<uint16_t*>(ws + pl.v);
    auto o_buf = [&](int b) { return reinterpret_cast<float*>(ws + pl.o + b * up256((size_t)pl.Tb * Hv * d * 4)); };
    auto cs_buf = [&](int b) { return reinterpret_cast<float*>(ws + pl.cs + b * up256(C * 3 * 4)); };
    auto st_buf = [&](int b) { return reinterpret_cast<float*>(ws + pl.st + b * up256((size_t)Hv * d * d * 4)); };
    void* pws = ws + pl.pws;
    const size_t pws_bytes = gdn_prefill_workspace_size(1, pl.Tb, Hqk, Hv, d);

    // events: the start (the workspace is free of earlier work on `stream`), and
    // per range: uploaded, computed, downloaded.  Released at the end of the call;
    // the driver keeps them until the work they mark is done.
    std::vector<cudaEvent_t> ev;
    ev.reserve((size_t)(3 * nb + 1));
    gdn_status status = GDN_OK;
    cudaError_t e = cudaSuccess;
    for (int64_t i = 0; i < 3 * nb + 1 && e == cudaSuccess; ++i) {
        cudaEvent_t x;
        e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
        if (e == cudaSuccess) ev.push_back(x);
    }
    cudaEvent_t ev_start = e == cudaSuccess ? ev[0] : nullptr;
    auto ev_up = [&](int64_t r) { return ev[1 + 3 * r]; };
    auto ev_comp = [&](int64_t r) { return ev[2 + 3 * r]; };
    auto ev_down = [&](int64_t r) { return ev[3 + 3 * r]; };
    if (e == cudaSuccess) e = cudaEventRecord(ev_start, s0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(su, ev_start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sd, ev_start, 0);
    for (int64_t r = 0; r < nb && e == cudaSuccess && status == GDN_OK; ++r) {
        const int b = (int)(r & 1);
        int64_t t0, L;
        host_range(pl, T, r, &t0, &L);
        // upload: buffer b is free once range r - 2 has been computed
        if (r >= 2) e = cudaStreamWaitEvent(su, ev_comp(r - 2), 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(qkv_buf(b), h_qkv + (size_t)t0 * C, (size_t)L * C * 2, cudaMemcpyHostToDevice, su);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(ab_buf(2 * b), h_a + (size_t)t0 * Hv, (size_t)L * Hv * 4, cudaMemcpyHostToDevice, su);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(ab_buf(2 * b + 1), h_b + (size_t)t0 * Hv, (size_t)L * Hv * 4, cudaMemcpyHostToDevice,
                                su);
        if (e == cudaSuccess) e = cudaEventRecord(ev_up(r), su);
        // compute: after the upload, and once range r - 2's output has gone down
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, ev_up(r), 0);
        if (e == cudaSuccess && r >= 2) e = cudaStreamWaitEvent(s0, ev_down(r - 2), 0);
        if (e != cudaSuccess) break;
        const float* cs_in = r == 0 ? conv_state_in : cs_buf((int)((r + 1) & 1));
        status = gdn_conv1d_silu(qkv_buf(b), conv_w, nullptr, 1, L, Hqk, Hv, d, cs_in, cs_buf(b), qb, kb, vb, stream);
        if (status != GDN_OK) break;
        const float* s_in = r == 0 ? initial_state : st_buf((int)((r + 1) & 1));
        status = gdn_prefill(qb, kb, vb, ab_buf(2 * b), ab_buf(2 * b + 1), A_log, dt_bias, nullptr, 1, L, Hqk, Hv, d,
                             scale, s_in, st_buf(b), o_buf(b), pws, pws_bytes, stream);
        if (status != GDN_OK) break;
        e = cudaEventRecord(ev_comp(r), s0);
        // download
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sd, ev_comp(r), 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(h_o + (size_t)t0 * Hv * d, o_buf(b), (size_t)L * Hv * d * 4, cudaMemcpyDeviceToHost,
                                sd);
        if (e == cudaSuccess && r == nb - 1)
            e = cudaMemcpyAsync(h_final_state, st_buf(b), (size_t)Hv * d * d * 4, cudaMemcpyDeviceToHost, sd);
        if (e == cudaSuccess) e = cudaEventRecord(ev_down(r), sd);
    }
    if (e == cudaSuccess && status == GDN_OK && conv_state_out)
        e = cudaMemcpyAsync(conv_state_out, cs_buf((int)((nb - 1) & 1)), C * 3 * 4, cudaMemcpyDeviceToDevice, s0);
    // everything of the call is ordered before later work on `stream`
    if (e == cudaSuccess && status == GDN_OK) e = cudaStreamWaitEvent(s0, ev_down(nb - 1), 0);
    for (cudaEvent_t x : ev) cudaEventDestroy(x);
    if (status != GDN_OK) return status;
    if (e != cudaSuccess) return gdn::set_last_cuda_error(e);
    return GDN_OK;
}

}  // extern "C"
