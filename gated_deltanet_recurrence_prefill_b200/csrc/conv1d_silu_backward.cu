// conv1d_silu_backward.cu -- kernels and launch of the front end's gradient
// (the algebra and the block functions are in conv1d_silu_backward.cuh).
//
// Tiles of 32 tokens that lie inside one sequence with their history and the
// three tokens after them (all but a few tiles of a long sequence) are done by
// a streaming kernel: one warp per (tile, packed head), a lane owns 4 channels
// and walks the tile's 35 tokens in order, recomputing the forward with the
// last three inputs in registers, turning each token's output gradient into
// dy (the q / k norm reduced across the warp), finishing d x[t - 3] from the
// last four dy, and summing the tile's weight gradient in registers.  Its
// inputs (16 bytes of the output gradient and 8 of x per lane and token) are
// requested kRingF tokens ahead by cp.async into a ring in shared memory.  The
// other tiles run the block function, one CTA per (tile, head).  Then the
// weight gradient is summed over tiles in order.
#include "conv1d_silu_backward.cuh"
#include "kernels.h"

namespace gdn {
namespace {

using namespace fbw;

// tiles: blockIdx.x / n_heads = k selects tile k, or with tail0 > 0 the first
// tile (k = 0) and then tiles tail0, tail0 + 1, ... (one sequence: only those
// can hold a sequence edge)
__global__ void __launch_bounds__(kThreads) fbw_tile_kernel(Params p, int n_heads, int64_t tail0) {
    extern __shared__ float4 fbw_smem[];
    const int64_t k = blockIdx.x / n_heads;
    const int64_t tile = (tail0 > 0 && k > 0) ? tail0 + k - 1 : k;
    if (stream_tile(p, tile)) return;            // the streaming kernel's tile
    tile_block(p, tile, blockIdx.x % n_heads, threadIdx.x, reinterpret_cast<float*>(fbw_smem));
}

constexpr int kWarpsF = 8;
constexpr int kRingF = 8;                        // tokens in flight per warp (a power of two)
struct RingF {
    uint2 x[kRingF][32];                         // 4 bf16 inputs per lane
    float4 g[kRingF][32];                        // 4 output-gradient values per lane
};

__device__ __forceinline__ void cp_async8(void* sdst, const void* gsrc) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"((uint32_t)__cvta_generic_to_shared(sdst)),
                 "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_async16g(void* sdst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(sdst)),
                 "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float2 bf2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

__global__ void __launch_bounds__(kWarpsF * 32) fbw_stream_kernel(Params p, int n_heads) {
    extern __shared__ __align__(16) uint8_t fsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t job = (int64_t)blockIdx.x * kWarpsF + warp;
    if (job >= p.n_tiles * n_heads) return;
    const int64_t tile = job / n_heads;
    const int hh = (int)(job - tile * n_heads);
    if (!stream_tile(p, tile)) return;           // the block kernel's tile
    RingF& ring = reinterpret_cast<RingF*>(fsm)[warp];
    const int64_t Ctot = (int64_t)n_heads * kD;
    const int64_t c0 = (int64_t)hh * kD + lane * 4;
    const bool normed = hh < 2 * p.Hqk;
    const float* dsrc = (hh < p.Hqk ? p.dq + (int64_t)hh * kD
                         : normed ? p.dk + (int64_t)(hh - p.Hqk) * kD : p.dv + (int64_t)(hh - 2 * p.Hqk) * kD) +
                        lane * 4;
    const int64_t dstride = (normed ? (int64_t)p.Hqk : (int64_t)p.Hv) * kD;
    const int64_t t0 = tile * kTile;
    const uint16_t* xs = p.x + t0 * Ctot + c0;
    const float* gsrc = dsrc + t0 * dstride;
#pragma unroll
    for (int r = 0; r < kRingF; ++r) {
        cp_async8(&ring.x[r][lane], xs + r * Ctot);
        cp_async16g(&ring.g[r][lane], gsrc + r * dstride);
        cp_commit();
    }
    // weights as channel pairs: wp[cp][j] = (w[c0 + 2 cp][j], w[c0 + 2 cp + 1][j])
    float2 wp[2][4];
#pragma unroll
    for (int cp = 0; cp < 2; ++cp) {
        const float4 a = *reinterpret_cast<const float4*>(p.w + (c0 + 2 * cp) * 4);
        const float4 b = *reinterpret_cast<const float4*>(p.w + (c0 + 2 * cp + 1) * 4);
        wp[cp][0] = make_float2(a.x, b.x); wp[cp][1] = make_float2(a.y, b.y);
        wp[cp][2] = make_float2(a.z, b.z); wp[cp][3] = make_float2(a.w, b.w);
    }
    // inputs of the three tokens before the tile (same sequence)
    float2 xh[3][2];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const uint2 r = *reinterpret_cast<const uint2*>(xs + (int64_t)(j - 3) * Ctot);
        xh[j][0] = bf2(r.x);
        xh[j][1] = bf2(r.y);
    }
    float2 dyh[3][2];                            // dy of the last three tokens
    float2 dwa[2][4];
#pragma unroll
    for (int cp = 0; cp < 2; ++cp) {
#pragma unroll
        for (int j = 0; j < 4; ++j) dwa[cp][j] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 3; ++j) dyh[j][cp] = make_float2(0.f, 0.f);
    }
    float* dxp = p.dx + (t0 - 3) * Ctot + c0;       // d x of token t0 + tau - 3
    const uint16_t* xn = xs + kRingF * Ctot;          // the input kRingF tokens ahead
    const float* gn = gsrc + kRingF * dstride;
    // two tokens per iteration, so that the second token's forward overlaps the
    // first one's reductions
#pragma unroll 2
    for (int tau = 0; tau < kSpan; ++tau) {
        cp_wait<kRingF - 1>();
        const int slot = tau & (kRingF - 1);
        const uint2 xr = ring.x[slot][lane];
        const float4 gr = ring.g[slot][lane];
        if (tau + kRingF < kSpan) {
            cp_async8(&ring.x[slot][lane], xn);
            cp_async16g(&ring.g[slot][lane], gn);
        }
        cp_commit();
        xn += Ctot;
        gn += dstride;
        const float2 xc[2] = {bf2(xr.x), bf2(xr.y)};
        const float2 g[2] = {make_float2(gr.x, gr.y), make_float2(gr.z, gr.w)};
        // forward: y (acc), sigma(y), a = y sigma(y)
        float2 sg[2], a[2];
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {
            float2 acc = __fmul2_rn(wp[cp][0], xh[0][cp]);
            acc = __ffma2_rn(wp[cp][1], xh[1][cp], acc);
            acc = __ffma2_rn(wp[cp][2], xh[2][cp], acc);
            acc = __ffma2_rn(wp[cp][3], xc[cp], acc);
            sg[cp] = make_float2(__frcp_rn(1.f + __expf(-acc.x)), __frcp_rn(1.f + __expf(-acc.y)));
            a[cp] = __fmul2_rn(acc, sg[cp]);
        }
        // da: through the q / k norm (sums over the head's 128 channels)
        float2 da[2];
        if (normed) {
            float ss = a[0].x * a[0].x + a[0].y * a[0].y + a[1].x * a[1].x + a[1].y * a[1].y;
            float gd = g[0].x * a[0].x + g[0].y * a[0].y + g[1].x * a[1].x + g[1].y * a[1].y;
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
                ss += __shfl_xor_sync(0xffffffffu, ss, m);
                gd += __shfl_xor_sync(0xffffffffu, gd, m);
            }
            const float inv = rsqrtf(ss + 1e-6f);         // 1 / n
            const float dot = gd * (inv * inv);           // <dout, out> / n
#pragma unroll
            for (int cp = 0; cp < 2; ++cp)
                da[cp] = make_float2((g[cp].x - a[cp].x * dot) * inv, (g[cp].y - a[cp].y * dot) * inv);
        } else {
            da[0] = g[0];
            da[1] = g[1];
        }
        // dy = da (sigma + a (1 - sigma))
        float2 dy[2];
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {
            const float2 one_m = make_float2(1.f - sg[cp].x, 1.f - sg[cp].y);
            dy[cp] = __fmul2_rn(da[cp], __ffma2_rn(a[cp], one_m, sg[cp]));
        }
        if (tau < kTile) {
#pragma unroll
            for (int cp = 0; cp < 2; ++cp) {
                dwa[cp][0] = __ffma2_rn(dy[cp], xh[0][cp], dwa[cp][0]);
                dwa[cp][1] = __ffma2_rn(dy[cp], xh[1][cp], dwa[cp][1]);
                dwa[cp][2] = __ffma2_rn(dy[cp], xh[2][cp], dwa[cp][2]);
                dwa[cp][3] = __ffma2_rn(dy[cp], xc[cp], dwa[cp][3]);
            }
        }
        if (tau >= 3) {
            // d x[t - 3] = w0 dy[t] + w1 dy[t - 1] + w2 dy[t - 2] + w3 dy[t - 3]
            float2 dx[2];
#pragma unroll
            for (int cp = 0; cp < 2; ++cp) {
                float2 acc = __fmul2_rn(wp[cp][3], dyh[0][cp]);
                acc = __ffma2_rn(wp[cp][2], dyh[1][cp], acc);
                acc = __ffma2_rn(wp[cp][1], dyh[2][cp], acc);
                dx[cp] = __ffma2_rn(wp[cp][0], dy[cp], acc);
            }
            *reinterpret_cast<float4*>(dxp) = make_float4(dx[0].x, dx[0].y, dx[1].x, dx[1].y);
        }
        dxp += Ctot;
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {
            xh[0][cp] = xh[1][cp]; xh[1][cp] = xh[2][cp]; xh[2][cp] = xc[cp];
            dyh[0][cp] = dyh[1][cp]; dyh[1][cp] = dyh[2][cp]; dyh[2][cp] = dy[cp];
        }
    }
    cp_wait<0>();
    // this tile's weight-gradient sums: 4 channels x 4 taps, 64 contiguous bytes
    float4* dst = reinterpret_cast<float4*>(p.dwp + (tile * Ctot + c0) * 4);
#pragma unroll
    for (int cp = 0; cp < 2; ++cp) {
        dst[2 * cp] = make_float4(dwa[cp][0].x, dwa[cp][1].x, dwa[cp][2].x, dwa[cp][3].x);
        dst[2 * cp + 1] = make_float4(dwa[cp][0].y, dwa[cp][1].y, dwa[cp][2].y, dwa[cp][3].y);
    }
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
        // streaming tiles (every tile decides for itself)
        const int sbytes = kWarpsF * (int)sizeof(RingF);
        e = cudaFuncSetAttribute(fbw_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sbytes);
        if (e == cudaSuccess) {
            fbw_stream_kernel<<<(unsigned)((jobs + kWarpsF - 1) / kWarpsF), kWarpsF * 32, sbytes, s>>>(p, n_heads);
            e = cudaGetLastError();
        }
        // the other tiles: with one sequence only the first tile and the last
        // ones (they skip the rest themselves with cu_seqlens)
        const int bytes = fbw::kTileFloats * (int)sizeof(float);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fbw_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e == cudaSuccess) {
            if (p.cu) {
                fbw_tile_kernel<<<(unsigned)jobs, fbw::kThreads, bytes, s>>>(p, n_heads, 0);
            } else {
                // the first tile and the tiles whose span passes the end (t0 + kSpan > T)
                int64_t tail0 = (p.T - fbw::kSpan) / fbw::kTile + 1;
                if (tail0 < 1) tail0 = 1;
                const int64_t n_gen = 1 + (p.n_tiles > tail0 ? p.n_tiles - tail0 : 0);
                fbw_tile_kernel<<<(unsigned)(n_gen * n_heads), fbw::kThreads, bytes, s>>>(p, n_heads, tail0);
            }
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
