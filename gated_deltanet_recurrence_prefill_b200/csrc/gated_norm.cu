// gated_norm.cu -- the gated output norm of the linear-attention layer:
//     y[t, h, :] = w[l] * o[t, h, :] / sqrt(mean_v o[t, h, v]^2 + eps) * silu(z[t, h, :])
// (Qwen3.8-27B architecture page, 2kiu.com, section 2.1: every linear-attention
// layer carries `norm` and `in_proj_z`; the page prints no formula, and the
// reading is an RMS norm over the d_v channels of each value head with one
// weight vector per layer shared by the heads, gated by SiLU of z).
//
// Bound: HBM.  Per row of d = 128 channels it reads o (512 B, float32) and z
// (256 B, bf16) and writes y (256 B, bf16): 1024 B per (token, value head).
// One warp per two rows, four channels per lane (16-byte loads of o and w,
// 8-byte loads of z; both rows' loads issued before either is used, which keeps
// twice the bytes in flight), the sum of squares by warp shuffles; sixteen rows
// per 256-thread block.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int kD = 128;
constexpr int kWarpsPerBlock = 8;
constexpr int kRowsPerWarp = 2;
constexpr int kRowsPerBlock = kWarpsPerBlock * kRowsPerWarp;

// silu(x) = x / (1 + e^{-x}), as x * rcp(1 + e^{-x}): for x -> -inf the
// reciprocal of +inf is 0 and the result -0, for x -> +inf it is x
__device__ __forceinline__ float silu(float x) { return x * __frcp_rn(1.f + __expf(-x)); }

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
gated_norm_kernel(const float* __restrict__ o, const uint16_t* __restrict__ z, const float* __restrict__ w,
                  int64_t rows, int32_t Hv, int32_t layers, float eps, uint16_t* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t row0 = ((int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5)) * kRowsPerWarp;
    // both rows' loads first, so that they are in flight together
    float4 ov[kRowsPerWarp];
    uint2 zv[kRowsPerWarp];
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
        const int64_t row = row0 + j < rows ? row0 + j : rows - 1;    // clamped: read, not written
        ov[j] = __ldcs(reinterpret_cast<const float4*>(o + row * kD) + lane);
        zv[j] = __ldcs(reinterpret_cast<const uint2*>(z + row * kD) + lane);
    }
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
        const int64_t row = row0 + j;
        // row = t * Hv + h; the layer of token t is t % layers (decode units are
        // sequence-major with the layer fastest; a prefill call has one layer)
        const int64_t t = (row < rows ? row : rows - 1) / Hv;
        const int l = (int)(t % layers);
        const float4 wv = __ldg(reinterpret_cast<const float4*>(w + (int64_t)l * kD) + lane);
        float ss = ov[j].x * ov[j].x + ov[j].y * ov[j].y + ov[j].z * ov[j].z + ov[j].w * ov[j].w;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        const float r = rsqrtf(ss * (1.f / kD) + eps);
        const float2 z01 = bf16x2_to_f32x2(zv[j].x), z23 = bf16x2_to_f32x2(zv[j].y);
        const float g0 = silu(z01.x), g1 = silu(z01.y), g2 = silu(z23.x), g3 = silu(z23.y);
        uint2 out;
        out.x = pack_bf16x2(wv.x * (ov[j].x * r) * g0, wv.y * (ov[j].y * r) * g1);
        out.y = pack_bf16x2(wv.z * (ov[j].z * r) * g2, wv.w * (ov[j].w * r) * g3);
        if (row < rows) __stcs(reinterpret_cast<uint2*>(y + row * kD) + lane, out);
    }
}

}  // namespace

cudaError_t launch_gated_norm(const float* o, const uint16_t* z, const float* w, int64_t T, int32_t Hv,
                              int32_t layers, float eps, uint16_t* y, cudaStream_t stream) {
    const int64_t rows = T * Hv;
    if (rows == 0) return cudaSuccess;
    const int64_t blocks = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    gated_norm_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, 0, stream>>>(o, z, w, rows, Hv, layers, eps, y);
    return cudaGetLastError();
}

}  // namespace gdn
