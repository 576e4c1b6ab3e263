// tile_util.cuh -- shared-memory tile helpers for the tcgen05 prefill kernels:
// UMMA descriptors for 128-byte-swizzled bf16 tiles, bf16 row-chunk loads and
// stores in that layout, and tf32 mma.sync fragments on f32 scratch matrices.
#pragma once

#include "common.cuh"
#include "tc_util.cuh"

namespace gdn {
namespace tile {

using namespace tc;

constexpr uint32_t KQ_PANEL = 16384;           // 128 rows x 64 bf16, 128-byte swizzle

// K-major operand, K extent 128 split in two 16 KB panels of 128 rows
TC_DEVICE uint64_t desc_kmajor_2panel(uint32_t base, int kk) {
    return sdesc_sw128(base + (kk >> 2) * KQ_PANEL + (kk & 3) * 32, 16, 1024);
}
// K-major operand with K extent 64 (one panel)
TC_DEVICE uint64_t desc_kmajor_1panel(uint32_t base, int kk) {
    return sdesc_sw128(base + kk * 32, 16, 1024);
}
// MN-major operand: rows are the K index (128 bytes each), 16 rows per step;
// lbo = distance between 64-element MN atoms
TC_DEVICE uint64_t desc_mnmajor(uint32_t base, int kk, uint32_t lbo) {
    return sdesc_sw128(base + kk * 2048, lbo, 1024);
}

// --- tf32 mma.sync fragments (m16n8k8) on fp32 shared-memory matrices -----------
TC_DEVICE void frag_a(const float* M, int ld, int r0, int k0, uint32_t* a, int lane) {
    const int g = lane >> 2, t = lane & 3;
    a[0] = to_tf32(M[(r0 + g) * ld + k0 + t]);
    a[1] = to_tf32(M[(r0 + g + 8) * ld + k0 + t]);
    a[2] = to_tf32(M[(r0 + g) * ld + k0 + t + 4]);
    a[3] = to_tf32(M[(r0 + g + 8) * ld + k0 + t + 4]);
}
TC_DEVICE void frag_b(const float* M, int ld, int k0, int n0, uint32_t* b, int lane) {
    const int g = lane >> 2, t = lane & 3;
    b[0] = to_tf32(M[(k0 + t) * ld + n0 + g]);
    b[1] = to_tf32(M[(k0 + t + 4) * ld + n0 + g]);
}
TC_DEVICE void frag_c_store(float* M, int ld, int r0, int n0, const float* c, float s, int lane) {
    const int g = lane >> 2, t = lane & 3;
    M[(r0 + g) * ld + n0 + 2 * t] = s * c[0];
    M[(r0 + g) * ld + n0 + 2 * t + 1] = s * c[1];
    M[(r0 + g + 8) * ld + n0 + 2 * t] = s * c[2];
    M[(r0 + g + 8) * ld + n0 + 2 * t + 1] = s * c[3];
}
// c (16 x 8) = A[r0:r0+16, k0 + 8 s0 : k0 + 8 s1] * B[kb0 + 8 s0 : kb0 + 8 s1, n0:n0+8]
TC_DEVICE void mma_tile(float* c, const float* A, int lda, int r0, int k0, const float* B, int ldb,
                        int kb0, int n0, int s0, int s1, int lane) {
    c[0] = c[1] = c[2] = c[3] = 0.f;
    for (int s = s0; s < s1; ++s) {
        uint32_t a[4], b[2];
        frag_a(A, lda, r0, k0 + 8 * s, a, lane);
        frag_b(B, ldb, kb0 + 8 * s, n0, b, lane);
        mma_tf32_16x8x8(c, a, b);
    }
}

// write 8 floats as bf16 into row `row`, 16-byte chunk `chunk` of a swizzled tile
TC_DEVICE void st_bf16x8(uint8_t* tile, int row, int chunk, const float* x) {
    uint4 v;
    v.x = pack_bf16x2(x[0], x[1]);
    v.y = pack_bf16x2(x[2], x[3]);
    v.z = pack_bf16x2(x[4], x[5]);
    v.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(tile + sw128_off(row, chunk)) = v;
}
TC_DEVICE void ld_bf16x8(const uint8_t* tile, int row, int chunk, float* x) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + sw128_off(row, chunk));
    float2 f;
    f = bf16x2_to_f32x2(v.x); x[0] = f.x; x[1] = f.y;
    f = bf16x2_to_f32x2(v.y); x[2] = f.x; x[3] = f.y;
    f = bf16x2_to_f32x2(v.z); x[4] = f.x; x[5] = f.y;
    f = bf16x2_to_f32x2(v.w); x[6] = f.x; x[7] = f.y;
}


}  // namespace tile
}  // namespace gdn
