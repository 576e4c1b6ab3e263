// backward_chunked.cu -- kernels and launch sequence of the chunked backward
// (the algebra and the block functions are in backward_chunked.cuh).
//
//   1. chunk list: per slot the sequence and first token of its chunk;
//   2. prep, one CTA per (chunk, value head): T, W, U', the decays, Y_c (on the
//      tensor cores, or in float32 with GDN_BACKWARD_GRAD=simt);
//   3. forward chain: S_c;
//   4. backward chain: dS_c and dL/dS_0 -- both on the tensor cores, one CTA per
//      (sequence, value head) (backward_chunked_tc.cu), or with
//      GDN_BACKWARD_GRAD=simt in float32 on the CUDA cores, kRowSplit CTAs per
//      (sequence, value head);
//   5. gradients, one CTA per (chunk, value head): dq, dk (per value head), dv,
//      da, db and per-chunk sums for the gate parameters -- on the tensor cores
//      (backward_chunked_tc.cu), or the float32 block function with
//      GDN_BACKWARD_GRAD=simt;
//   6. sums over each key head's value heads and over chunks.
// Every CTA has 256 threads; 2, 3 and 5 take almost all of an SM's shared
// memory, 4 about half.
#include <stdlib.h>
#include <string.h>

#include "backward_chunked.cuh"
#include "kernels.h"

namespace gdn {
namespace {

using namespace bwc;

__global__ void __launch_bounds__(kThreads) bwc_jobs_kernel(Params p) { fill_jobs(p, blockIdx.x, threadIdx.x); }

__global__ void __launch_bounds__(kThreads) bwc_prep_kernel(Params p) {
    extern __shared__ float4 bwc_smem_prep[];
    prep_block(p, blockIdx.x / p.Hv, blockIdx.x % p.Hv, threadIdx.x, reinterpret_cast<float*>(bwc_smem_prep));
}

__global__ void __launch_bounds__(kThreads) bwc_fwd_chain_kernel(Params p) {
    extern __shared__ float4 bwc_smem_fwd[];
    const int unit = blockIdx.x / kRowSplit, rq = blockIdx.x % kRowSplit;
    fwd_chain_block(p, unit / p.Hv, unit % p.Hv, rq, threadIdx.x, reinterpret_cast<float*>(bwc_smem_fwd));
}

__global__ void __launch_bounds__(kThreads) bwc_bwd_chain_kernel(Params p) {
    extern __shared__ float4 bwc_smem_bwd[];
    const int unit = blockIdx.x / kRowSplit, rq = blockIdx.x % kRowSplit;
    bwd_chain_block(p, unit / p.Hv, unit % p.Hv, rq, threadIdx.x, reinterpret_cast<float*>(bwc_smem_bwd));
}

__global__ void __launch_bounds__(kThreads) bwc_grad_kernel(Params p) {
    extern __shared__ float4 bwc_smem_grad[];
    grad_block(p, blockIdx.x / p.Hv, blockIdx.x % p.Hv, threadIdx.x, reinterpret_cast<float*>(bwc_smem_grad));
}

__global__ void __launch_bounds__(kThreads) bwc_reduce_qk_kernel(Params p) {
    reduce_qk_block(p, blockIdx.x, threadIdx.x);
}

__global__ void __launch_bounds__(kThreads) bwc_reduce_gates_kernel(Params p) { reduce_gates_block(p, threadIdx.x); }

template <class K>
cudaError_t launch_smem(K kernel, int64_t blocks, int floats, const Params& p, cudaStream_t s) {
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    const int bytes = floats * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)blocks, kThreads, bytes, s>>>(p);
    return cudaGetLastError();
}

// GDN_BACKWARD_GRAD=simt: the float32 CUDA-core chains and gradient step
bool grad_on_cuda_cores() {
    const char* env = getenv("GDN_BACKWARD_GRAD");
    return env && strcmp(env, "simt") == 0;
}

}  // namespace

cudaError_t launch_backward_grad_tc(const Params& p, int64_t jobs, cudaStream_t s);
cudaError_t launch_backward_chains_tc(const Params& p, int64_t units, bool backward, cudaStream_t s);
cudaError_t launch_backward_prep_tc(const Params& p, int64_t jobs, cudaStream_t s);

size_t backward_chunked_workspace_bytes(int32_t n_seq, int64_t T, int32_t Hv) {
    return make_plan(n_seq, T, Hv).bytes;
}

cudaError_t launch_backward_chunked(const BackwardArgs& a, cudaStream_t s) {
    if (a.n_seq <= 0) return cudaSuccess;
    const Plan plan = make_plan(a.n_seq, a.T, a.Hv);
    Params p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.a = a.a; p.b = a.b; p.A_log = a.A_log; p.dt_bias = a.dt_bias;
    p.cu = a.cu_seqlens; p.s0 = a.initial_state; p.d_o = a.d_o; p.d_fin = a.d_final_state;
    p.n_seq = a.n_seq; p.Hqk = a.Hqk; p.Hv = a.Hv; p.T = a.T; p.scale = a.scale;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv; p.da = a.da; p.db = a.db; p.dA_log = a.dA_log;
    p.ddt_bias = a.ddt_bias; p.d_init = a.d_initial_state;
    bind_workspace(p, a.workspace, plan);
    const int64_t jobs = plan.n_slots * a.Hv;
    const int64_t chains = (int64_t)a.n_seq * a.Hv * kRowSplit;
    cudaError_t e = cudaMemsetAsync(p.err, 0, plan.jobs - plan.err, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.jobs, 0xFF, (size_t)plan.n_slots * 2 * sizeof(int32_t), s);
    if (e == cudaSuccess) {
        bwc_jobs_kernel<<<(unsigned)a.n_seq, kThreads, 0, s>>>(p);
        e = cudaGetLastError();
    }
    const bool simt = grad_on_cuda_cores();
    const int64_t units = (int64_t)a.n_seq * a.Hv;
    if (simt) {
        if (e == cudaSuccess) e = launch_smem(bwc_prep_kernel, jobs, kPrepFloats, p, s);
        if (e == cudaSuccess) e = launch_smem(bwc_fwd_chain_kernel, chains, kChainFloats, p, s);
        if (e == cudaSuccess) e = launch_smem(bwc_bwd_chain_kernel, chains, kChainFloats, p, s);
        if (e == cudaSuccess) e = launch_smem(bwc_grad_kernel, jobs, kGradFloats, p, s);
    } else {
        if (e == cudaSuccess) e = launch_backward_prep_tc(p, jobs, s);
        if (e == cudaSuccess) e = launch_backward_chains_tc(p, units, false, s);
        if (e == cudaSuccess) e = launch_backward_chains_tc(p, units, true, s);
        if (e == cudaSuccess) e = launch_backward_grad_tc(p, jobs, s);
    }
    const int64_t n = a.T * a.Hqk * kD;
    if (e == cudaSuccess && n > 0) {
        bwc_reduce_qk_kernel<<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, s>>>(p);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        bwc_reduce_gates_kernel<<<1, kThreads, 0, s>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace gdn
