// gated_norm_backward.cuh -- the gradient of the gated output norm
//     y[t, h, :] = w[l] * o * r * silu(z),  r = 1 / sqrt(mean_v o^2 + eps),
//     l = t % layers
// (the reading of the architecture page's `norm` and `in_proj_z` weights,
// section 2.1, that gdn_gated_norm implements), on CUDA cores in float32.
// With g = silu(z) and u = w g dy:
//     do = r u - (r^3 / d) o <o, u>,
//     dz = dy w r o sigma(z) (1 + z (1 - sigma(z))),
//     dw[l] = sum over the rows of layer l of dy r o g.
// Three block functions: rows (a CTA of 128 threads, one per element, over 8
// tokens x 8 heads, keeping the weight gradient of each token of its tile), a
// sum over chunks of 64 of each layer's tokens, and a sum over those chunks --
// every sum in a fixed order.  As in backward_chunked.cuh, the CUDA kernels
// and the CPU tests' emulation run the same source.
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

namespace gdn {
namespace nbw {

constexpr int kD = 128;
constexpr int kThreads = 128;            // one thread per element of a row
constexpr int kTok = 8;                  // tokens per rows job
constexpr int kHeads = 8;                // heads per rows job
constexpr int kChunk = 64;               // tokens of one layer per first-stage sum
constexpr int kRowsFloats = 2 * kD + 2 * 8;

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

BWC_FN void rows_block(const Params& p, int64_t tile, int hg, int tid, float* sm) {
    float* red = sm;                  // [2][128]: o^2 and o u of this thread's element
    float* part = red + 2 * kD;       // [2][8]: sums of 16 elements each
    const int e = tid;
    const int h0 = hg * kHeads;
    const int h1 = (h0 + kHeads) < p.Hv ? h0 + kHeads : p.Hv;
    float acc[kTok];
    for (int j = 0; j < kTok; ++j) {
        acc[j] = 0.f;
        const int64_t t = tile * kTok + j;
        if (t >= p.T) continue;                           // the same for every thread
        const float w = p.w[(int64_t)(t % p.layers) * kD + e];
        for (int h = h0; h < h1; ++h) {
            const int64_t row = (t * p.Hv + h) * kD;
            const float o = p.o[row + e], z = bf16f(p.z[row + e]), dy = p.dy[row + e];
            const float sg = 1.f / (1.f + expf(-z));
            const float g = z * sg;
            const float u = w * g * dy;
            red[e] = o * o;
            red[kD + e] = o * u;
            BWC_SYNC();
            if (tid < 8) {
                float s0 = 0.f, s1 = 0.f;
                for (int i = 0; i < 16; ++i) {
                    s0 += red[16 * tid + i];
                    s1 += red[kD + 16 * tid + i];
                }
                part[tid] = s0;
                part[8 + tid] = s1;
            }
            BWC_SYNC();
            float ss = 0.f, ou = 0.f;
            for (int i = 0; i < 8; ++i) {
                ss += part[i];
                ou += part[8 + i];
            }
            const float r = 1.f / sqrtf(ss / kD + p.eps);
            p.d_o[row + e] = r * u - r * r * r / kD * o * ou;
            p.d_z[row + e] = dy * w * r * o * sg * (1.f + z * (1.f - sg));
            acc[j] = fmaf(dy * r, o * g, acc[j]);
            BWC_SYNC();
        }
    }
    const int ng = n_groups(p.Hv);
    for (int j = 0; j < kTok; ++j) p.part1[((tile * ng + hg) * kTok + j) * kD + e] = acc[j];
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
