// gated_norm_backward.cuh -- the gradient of the gated output norm
//     y[t, h, :] = w[l] * o * r * silu(z),  r = 1 / sqrt(mean_v o^2 + eps),
//     l = t % layers
// (the reading of the architecture page's `norm` and `in_proj_z` weights,
// section 2.1, that gdn_gated_norm implements), on CUDA cores in float32.
// With g = silu(z) and u = w g dy:
//     do = r u - (r^3 / d) o <o, u>,
//     dz = dy w r o sigma(z) (1 + z (1 - sigma(z))),
//     dw[l] = sum over the rows of layer l of dy r o g.
// Three block functions: rows (a CTA of 8 warps over 8 tokens x 8 heads: warp
// w takes head h0 + w for the 8 tokens, a lane 4 elements of each row, the
// row sums by warp shuffles; the weight gradient of each token of the tile is
// then summed over the warps in order), a sum over chunks of 64 of each
// layer's tokens, and a sum over those chunks -- every sum in a fixed order.
// As in backward_chunked.cuh, the CUDA kernels and the CPU tests' emulation
// run the same source (shuffles included).
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

#ifndef BWC_FN
#define BWC_FN __device__ __forceinline__
#endif
#ifndef BWC_HD
#define BWC_HD __host__ __device__ __forceinline__
#endif
#ifndef BWC_SYNC
#define BWC_SYNC() __syncthreads()
#endif
#ifndef BWC_SHFL_XOR
#define BWC_SHFL_XOR(v, m) __shfl_xor_sync(0xffffffffu, (v), (m))
#endif

namespace gdn {
namespace nbw {

constexpr int kD = 128;
constexpr int kThreads = 128;            // the sums: one thread per element
constexpr int kRowThreads = 256;         // rows: 8 warps, one head each
constexpr int kTok = 8;                  // tokens per rows job
constexpr int kHeads = kRowThreads / 32; // heads per rows job
constexpr int kChunk = 64;               // tokens of one layer per first-stage sum
constexpr int kRowsFloats = kHeads * kTok * kD;

struct Params {
    const float* o;             // [T, Hv, 128]
    const uint16_t* z;          // [T, Hv, 128] bf16
    const float* w;             // [layers, 128]
    const float* dy;            // [T, Hv, 128]
    int64_t T;
    int32_t Hv, layers;
    float eps;
    float* d_o;                 // [T, Hv, 128]
    float* d_z;                 // [T, Hv, 128]
    float* dw;                  // [layers, 128]
    float* part1;               // [ceil(T / kTok), head groups, kTok, 128]
    float* part2;               // [layers, chunks, 128]
};

BWC_HD int64_t n_tiles(int64_t T) { return (T + kTok - 1) / kTok; }
BWC_HD int n_groups(int32_t Hv) { return (Hv + kHeads - 1) / kHeads; }
// chunks of kChunk tokens in the layer with the most tokens
BWC_HD int64_t n_chunks(int64_t T, int32_t layers) {
    const int64_t per_layer = (T + layers - 1) / layers;
    return (per_layer + kChunk - 1) / kChunk;
}

BWC_FN float bf16f(uint16_t h) {
#ifdef __CUDA_ARCH__
    return __uint_as_float((uint32_t)h << 16);
#else
    const uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
#endif
}

// four consecutive floats / bf16 values of a row (16- / 8-byte aligned): one
// vector access on the GPU
BWC_FN void ld4f(const float* src, float* v) {
#ifdef __CUDA_ARCH__
    const float4 t = *reinterpret_cast<const float4*>(src);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
#else
    memcpy(v, src, 4 * sizeof(float));
#endif
}
BWC_FN void st4f(float* dst, const float* v) {
#ifdef __CUDA_ARCH__
    *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
#else
    memcpy(dst, v, 4 * sizeof(float));
#endif
}
BWC_FN void ld4bf(const uint16_t* src, float* v) {
#ifdef __CUDA_ARCH__
    const uint2 t = *reinterpret_cast<const uint2*>(src);
    v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xFFFF0000u);
    v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xFFFF0000u);
#else
    for (int i = 0; i < 4; ++i) v[i] = bf16f(src[i]);
#endif
}

BWC_FN void rows_block(const Params& p, int64_t tile, int hg, int tid, float* sm) {
    float* red = sm;                  // [warp][token][element]: each warp's weight gradient
    const int warp = tid >> 5, lane = tid & 31;
    const int h = hg * kHeads + warp;
    float acc[kTok][4];
#pragma unroll
    for (int j = 0; j < kTok; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;
    if (h < p.Hv) {                                       // the same for every lane of the warp
        // restrict-qualified copies: the stores of one token do not order the
        // next token's loads behind them
        const float* __restrict__ po = p.o;
        const uint16_t* __restrict__ pz = p.z;
        const float* __restrict__ pdy = p.dy;
        float* __restrict__ pdo = p.d_o;
        float* __restrict__ pdz = p.d_z;
#pragma unroll
        for (int j = 0; j < kTok; ++j) {
            const int64_t t = tile * kTok + j;
            if (t >= p.T) continue;                       // the same for every lane
            const int64_t row = (t * p.Hv + h) * kD + lane * 4;
            const float* wl = p.w + (int64_t)(t % p.layers) * kD + lane * 4;
            float o[4], z[4], dy[4], w[4], sg[4], u[4];
            float ss = 0.f, ou = 0.f;
            ld4f(po + row, o);
            ld4bf(pz + row, z);
            ld4f(pdy + row, dy);
            ld4f(wl, w);
            for (int i = 0; i < 4; ++i) {
                sg[i] = 1.f / (1.f + expf(-z[i]));
                u[i] = w[i] * z[i] * sg[i] * dy[i];
                ss = fmaf(o[i], o[i], ss);
                ou = fmaf(o[i], u[i], ou);
            }
            for (int m = 16; m >= 1; m >>= 1) {
                ss += BWC_SHFL_XOR(ss, m);
                ou += BWC_SHFL_XOR(ou, m);
            }
            const float r = 1.f / sqrtf(ss / kD + p.eps);
            float dov[4], dzv[4];
            for (int i = 0; i < 4; ++i) {
                dov[i] = r * u[i] - r * r * r / kD * o[i] * ou;
                dzv[i] = dy[i] * w[i] * r * o[i] * sg[i] * (1.f + z[i] * (1.f - sg[i]));
                acc[j][i] = dy[i] * r * o[i] * (z[i] * sg[i]);
            }
            st4f(pdo + row, dov);
            st4f(pdz + row, dzv);
        }
    }
#pragma unroll
    for (int j = 0; j < kTok; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[(warp * kTok + j) * kD + lane * 4 + i] = acc[j][i];
    BWC_SYNC();
    const int ng = n_groups(p.Hv);
    for (int x = tid; x < kTok * kD; x += kRowThreads) {
        float s = 0.f;
        for (int w = 0; w < kHeads; ++w) s += red[w * kTok * kD + x];
        p.part1[(tile * ng + hg) * kTok * kD + x] = s;
    }
}

// first stage: tokens l + layers m, m in [kChunk k, kChunk (k + 1)), all head groups
BWC_FN void sum_chunk_block(const Params& p, int l, int64_t k, int tid) {
    const int ng = n_groups(p.Hv);
    float s = 0.f;
    for (int64_t m = k * kChunk; m < (k + 1) * kChunk; ++m) {
        const int64_t t = l + (int64_t)p.layers * m;
        if (t >= p.T) break;
        for (int hg = 0; hg < ng; ++hg) s += p.part1[(((t / kTok) * ng + hg) * kTok + t % kTok) * kD + tid];
    }
    p.part2[((int64_t)l * n_chunks(p.T, p.layers) + k) * kD + tid] = s;
}

// second stage: dw[l] = the chunks of layer l in order
BWC_FN void sum_layer_block(const Params& p, int l, int tid) {
    const int64_t nc = n_chunks(p.T, p.layers);
    float s = 0.f;
    for (int64_t k = 0; k < nc; ++k) s += p.part2[((int64_t)l * nc + k) * kD + tid];
    p.dw[(int64_t)l * kD + tid] = s;
}

}  // namespace nbw
}  // namespace gdn
