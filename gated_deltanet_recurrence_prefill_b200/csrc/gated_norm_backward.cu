// gated_norm_backward.cu -- kernels and launch of the gated output norm's
// gradient (the algebra and the block functions are in gated_norm_backward.cuh).
#include "gated_norm_backward.cuh"
#include "kernels.h"

namespace gdn {
namespace {

using namespace nbw;

__global__ void __launch_bounds__(kRowThreads) nbw_rows_kernel(Params p, int ng) {
    __shared__ float smem[kRowsFloats];
    rows_block(p, blockIdx.x / ng, blockIdx.x % ng, threadIdx.x, smem);
}

__global__ void __launch_bounds__(kThreads) nbw_chunk_kernel(Params p, int64_t nc) {
    sum_chunk_block(p, (int)(blockIdx.x / nc), blockIdx.x % nc, threadIdx.x);
}

__global__ void __launch_bounds__(kThreads) nbw_layer_kernel(Params p) { sum_layer_block(p, blockIdx.x, threadIdx.x); }

}  // namespace

size_t gated_norm_backward_workspace_bytes(int64_t T, int32_t Hv, int32_t layers) {
    const size_t p1 = (size_t)n_tiles(T) * n_groups(Hv) * kTok * kD * sizeof(float);
    const size_t p2 = (size_t)layers * n_chunks(T, layers) * kD * sizeof(float);
    return ((p1 + 255) & ~(size_t)255) + ((p2 + 255) & ~(size_t)255);
}

cudaError_t launch_gated_norm_backward(const float* o, const uint16_t* z, const float* w, const float* dy,
                                       int64_t T, int32_t Hv, int32_t layers, float eps, float* d_o, float* d_z,
                                       float* d_w, void* workspace, cudaStream_t s) {
    if (T == 0) return cudaMemsetAsync(d_w, 0, (size_t)layers * kD * sizeof(float), s);
    Params p;
    p.o = o; p.z = z; p.w = w; p.dy = dy; p.T = T; p.Hv = Hv; p.layers = layers; p.eps = eps;
    p.d_o = d_o; p.d_z = d_z; p.dw = d_w;
    const size_t p1 = (size_t)n_tiles(T) * n_groups(Hv) * kTok * kD * sizeof(float);
    p.part1 = static_cast<float*>(workspace);
    p.part2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((p1 + 255) & ~(size_t)255));
    const int ng = n_groups(Hv);
    const int64_t nc = n_chunks(T, layers);
    const int64_t rows_blocks = n_tiles(T) * ng, chunk_blocks = (int64_t)layers * nc;
    if (rows_blocks > 0x7fffffff || chunk_blocks > 0x7fffffff) return cudaErrorInvalidValue;
    nbw_rows_kernel<<<(unsigned)rows_blocks, kRowThreads, 0, s>>>(p, ng);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) {
        nbw_chunk_kernel<<<(unsigned)chunk_blocks, kThreads, 0, s>>>(p, nc);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        nbw_layer_kernel<<<(unsigned)layers, kThreads, 0, s>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace gdn
