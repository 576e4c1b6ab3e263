// conv1d_silu_backward.cu -- kernels and launch of the front end's gradient
// (the algebra and the block functions are in conv1d_silu_backward.cuh):
// one CTA per (32-token tile, packed head), then the weight gradient summed
// over tiles in order.
#include "conv1d_silu_backward.cuh"
#include "kernels.h"

namespace gdn {
namespace {

using namespace fbw;

__global__ void __launch_bounds__(kThreads) fbw_tile_kernel(Params p, int n_heads) {
    extern __shared__ float4 fbw_smem[];
    tile_block(p, blockIdx.x / n_heads, blockIdx.x % n_heads, threadIdx.x, reinterpret_cast<float*>(fbw_smem));
}

__global__ void __launch_bounds__(kThreads) fbw_reduce_kernel(Params p) { reduce_w_block(p, blockIdx.x, threadIdx.x); }

}  // namespace

size_t conv1d_silu_backward_workspace_bytes(int64_t T, int32_t Hqk, int32_t Hv) {
    const size_t bytes = (size_t)fbw::n_tiles(T) * (size_t)(2 * Hqk + Hv) * fbw::kD * 4 * sizeof(float);
    return (bytes + 255) & ~(size_t)255;
}

cudaError_t launch_conv1d_silu_backward(const ConvBackwardArgs& a, cudaStream_t s) {
    const int n_heads = 2 * a.Hqk + a.Hv;
    const int64_t Ctot = (int64_t)n_heads * fbw::kD;
    Params p;
    p.x = a.qkv; p.w = a.conv_w; p.cu = a.cu_seqlens; p.cs = a.conv_state;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv;
    p.n_seq = a.n_seq; p.Hqk = a.Hqk; p.Hv = a.Hv; p.T = a.T; p.n_tiles = fbw::n_tiles(a.T);
    p.dx = a.d_qkv; p.dwp = static_cast<float*>(a.workspace); p.dw = a.d_conv_w; p.dcs = a.d_conv_state;
    cudaError_t e = cudaSuccess;
    if (p.dcs) e = cudaMemsetAsync(p.dcs, 0, (size_t)a.n_seq * Ctot * 3 * sizeof(float), s);
    const int64_t jobs = p.n_tiles * n_heads;
    if (e == cudaSuccess && jobs > 0) {
        if (jobs > 0x7fffffff) return cudaErrorInvalidValue;
        const int bytes = fbw::kTileFloats * (int)sizeof(float);
        e = cudaFuncSetAttribute(fbw_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e == cudaSuccess) {
            fbw_tile_kernel<<<(unsigned)jobs, fbw::kThreads, bytes, s>>>(p, n_heads);
            e = cudaGetLastError();
        }
    }
    if (e == cudaSuccess) {
        if (jobs > 0) {
            fbw_reduce_kernel<<<(unsigned)((Ctot * 4 + fbw::kThreads - 1) / fbw::kThreads), fbw::kThreads, 0, s>>>(p);
            e = cudaGetLastError();
        } else {
            e = cudaMemsetAsync(a.d_conv_w, 0, (size_t)Ctot * 4 * sizeof(float), s);
        }
    }
    return e;
}

}  // namespace gdn
