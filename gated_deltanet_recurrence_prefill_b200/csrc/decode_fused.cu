// decode_fused.cu -- one decode step with the layer's front end fused in: the
// token's packed projection goes through the causal width-4 convolution
// (carried as a rolling three-input state per channel), SiLU and the q / k L2
// norm, and the result drives one step of the gated delta rule, for many
// (sequence, layer) units; both states are updated in place.
//
// Front end: Qwen3.8-27B architecture page (2kiu.com), section 2.1
// (linear_conv_kernel_dim = 4, conv1d.weight); recurrence: the same page,
// section 2.2, with the decay alpha on the erased state (see decode.cu for the
// row-wise form used here).  Sequences reach their state through a slot
// index, so a batch can be any subset of the slots in any order.
//
// Mapping: one CTA of 128 threads per (unit, key head).  Thread t owns channel
// t of the key head's q and k and of each of its value heads' v, so it is the
// only one to read and rewrite that channel's convolution state: the update
// is in place and race-free.  The q / k norms are block reductions.  Then the
// CTA runs the value heads of the group one after the other, each as in
// decode.cu (a warp per 32 state rows, a float4 of a row per lane, eight rows
// in flight), with q, k and v taken from shared memory in float32 -- no bf16
// rounding between the front end and the recurrence.  The state traffic
// dominates: the kernel is bound by HBM bandwidth.
#include "common.cuh"
#include "decode_state.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace gdn {

namespace {

constexpr int kD = 128;
constexpr int kThreads = 128;
// rows in flight per warp: 8 float32 rows or 16 bf16 rows (4 KB either way)
template <typename StateT> constexpr int rows_per_iter() { return sizeof(StateT) == 4 ? 8 : 16; }

// SiLU(y) = y / (1 + e^-y) with the accurate exponential (decode is checked
// to 1e-4, so no fast approximation here)
__device__ __forceinline__ float silu_accurate(float y) { return y / (1.f + expf(-y)); }

// conv + SiLU of one channel: x the current input, cs the three previous
// inputs (oldest first, updated in place to the last three), w the 4 taps
__device__ __forceinline__ float conv_channel(float x, float* cs, const float* w) {
    const float4 w4 = *reinterpret_cast<const float4*>(w);
    const float c0 = cs[0], c1 = cs[1], c2 = cs[2];
    float acc = w4.x * c0;
    acc = fmaf(w4.y, c1, acc);
    acc = fmaf(w4.z, c2, acc);
    acc = fmaf(w4.w, x, acc);
    cs[0] = c1;
    cs[1] = c2;
    cs[2] = x;
    return silu_accurate(acc);
}

__device__ __forceinline__ float block_sum(float v, float* red) {
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();                       // red may still be read by a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    return red[0] + red[1] + red[2] + red[3];
}

template <typename StateT>
__global__ void __launch_bounds__(kThreads, sizeof(StateT) == 2 ? 1 : 5)
decode_fused_kernel(const uint16_t* __restrict__ qkv, const float* __restrict__ conv_w,
                    float* __restrict__ conv_state, const float* __restrict__ a,
                    const float* __restrict__ b, const float* __restrict__ A_log,
                    const float* __restrict__ dt_bias, const int32_t* __restrict__ slot,
                    int32_t layers, int32_t Hqk, int32_t Hv, float scale, StateT* __restrict__ state,
                    float* __restrict__ o) {
    __shared__ __align__(16) float qs[kD], ks[kD], vs[kD];      // read as float4
    __shared__ float red[4];
    const int64_t ug = blockIdx.x;                 // unit * Hqk + key head
    const int64_t u = ug / Hqk;
    const int g = (int)(ug - u * Hqk);
    const int64_t n = u / layers;
    const int l = (int)(u - n * layers);
    const int64_t su = (int64_t)(slot ? slot[n] : n) * layers + l;      // state unit of (slot, layer)
    const int r = Hv / Hqk;                        // value heads per key head
    const int64_t Ctot = (int64_t)(2 * Hqk + Hv) * kD;
    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;

    const uint16_t* xrow = qkv + u * Ctot;
    const float* wl = conv_w + (int64_t)l * Ctot * 4;
    float* csu = conv_state + su * Ctot * 3;

    // ---- q and k of key head g: channel t of each
    {
        const int64_t cq = (int64_t)g * kD + t, ck = (int64_t)(Hqk + g) * kD + t;
        float csq[3], csk[3];
        for (int j = 0; j < 3; ++j) { csq[j] = csu[cq * 3 + j]; csk[j] = csu[ck * 3 + j]; }
        const float yq = conv_channel(bf16_to_f32(xrow[cq]), csq, wl + cq * 4);
        const float yk = conv_channel(bf16_to_f32(xrow[ck]), csk, wl + ck * 4);
        for (int j = 0; j < 3; ++j) { csu[cq * 3 + j] = csq[j]; csu[ck * 3 + j] = csk[j]; }
        const float nq = block_sum(yq * yq, red);
        const float nk = block_sum(yk * yk, red);
        qs[t] = yq * rsqrtf(nq + 1e-6f);
        ks[t] = yk * rsqrtf(nk + 1e-6f);
    }
    __syncthreads();
    // this lane's 4 elements of k and q, and k . q
    const float4 k4 = *reinterpret_cast<const float4*>(ks + lane * 4);
    const float4 q4 = *reinterpret_cast<const float4*>(qs + lane * 4);
    const float kq = warp_sum(k4.x * q4.x + k4.y * q4.y + k4.z * q4.z + k4.w * q4.w);

    for (int j = 0; j < r; ++j) {
        const int h = g * r + j;
        // ---- v of value head h: channel t
        {
            const int64_t cv = (int64_t)(2 * Hqk + h) * kD + t;
            float csv[3];
            for (int m = 0; m < 3; ++m) csv[m] = csu[cv * 3 + m];
            const float yv = conv_channel(bf16_to_f32(xrow[cv]), csv, wl + cv * 4);
            for (int m = 0; m < 3; ++m) csu[cv * 3 + m] = csv[m];
            __syncthreads();                       // the previous head's rows are done with vs
            vs[t] = yv;
            __syncthreads();
        }
        const int64_t uh = u * Hv + h;
        const float alpha = expf(log_alpha_f32(a[uh], A_log[(int64_t)l * Hv + h], dt_bias[(int64_t)l * Hv + h]));
        const float beta = sigmoid_f32(b[uh]);
        StateT* S = state + (su * Hv + h) * (int64_t)(kD * kD);
        constexpr int kRowsPerIter = rows_per_iter<StateT>();
        float* oh = o + uh * kD;
#pragma unroll 1
        for (int r0 = warp * 32; r0 < warp * 32 + 32; r0 += kRowsPerIter) {
            float4 s[kRowsPerIter];
#pragma unroll
            for (int i = 0; i < kRowsPerIter; ++i)
                s[i] = state_load4(S + (int64_t)(r0 + i) * kD, lane);
            float xk[kRowsPerIter], xq[kRowsPerIter];
#pragma unroll
            for (int i = 0; i < kRowsPerIter; ++i) {
                xk[i] = s[i].x * k4.x + s[i].y * k4.y + s[i].z * k4.z + s[i].w * k4.w;
                xq[i] = s[i].x * q4.x + s[i].y * q4.y + s[i].z * q4.z + s[i].w * q4.w;
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
#pragma unroll
                for (int i = 0; i < kRowsPerIter; ++i) {
                    xk[i] += __shfl_xor_sync(0xffffffffu, xk[i], m);
                    xq[i] += __shfl_xor_sync(0xffffffffu, xq[i], m);
                }
            }
            float orow = 0.f;
#pragma unroll
            for (int i = 0; i < kRowsPerIter; ++i) {
                const float w = beta * (vs[r0 + i] - alpha * xk[i]);
                float4 nv;
                nv.x = fmaf(alpha, s[i].x, w * k4.x);
                nv.y = fmaf(alpha, s[i].y, w * k4.y);
                nv.z = fmaf(alpha, s[i].z, w * k4.z);
                nv.w = fmaf(alpha, s[i].w, w * k4.w);
                state_store4(S + (int64_t)(r0 + i) * kD, lane, nv);
                const float oi = scale * fmaf(alpha, xq[i], w * kq);
                if (lane == i) orow = oi;
            }
            if (lane < kRowsPerIter) oh[r0 + lane] = orow;
        }
    }
}

// bf16 state: the states of the key head's r value heads (r x 32 KiB, contiguous)
// are brought into shared memory by one bulk copy issued first, so the copy
// overlaps the front end's arithmetic and the bytes in flight come from shared
// memory instead of registers; each value head's rows are then read from
// shared memory and written back from registers.
constexpr int kFusedBf16Rows = 8;
constexpr uint64_t kFusedWaitLimitNs = 2000000000ull;      // 2 s

__global__ void __launch_bounds__(kThreads, 2)
decode_fused_bf16_smem_kernel(const uint16_t* __restrict__ qkv, const float* __restrict__ conv_w,
                              float* __restrict__ conv_state, const float* __restrict__ a,
                              const float* __restrict__ b, const float* __restrict__ A_log,
                              const float* __restrict__ dt_bias, const int32_t* __restrict__ slot,
                              int32_t layers, int32_t Hqk, int32_t Hv, float scale, uint16_t* __restrict__ state,
                              float* __restrict__ o) {
    extern __shared__ __align__(128) uint8_t tiles[];          // r states of 128 x 128 bf16
    __shared__ __align__(8) uint64_t bar;
    __shared__ __align__(16) float qs[kD], ks[kD], vs[kD];      // read as float4
    __shared__ float red[4];
    __shared__ int abort_flag;
    const int64_t ug = blockIdx.x;                 // unit * Hqk + key head
    const int64_t u = ug / Hqk;
    const int g = (int)(ug - u * Hqk);
    const int64_t n = u / layers;
    const int l = (int)(u - n * layers);
    const int64_t su = (int64_t)(slot ? slot[n] : n) * layers + l;      // state unit of (slot, layer)
    const int r = Hv / Hqk;                        // value heads per key head
    const int64_t Ctot = (int64_t)(2 * Hqk + Hv) * kD;
    const int t = threadIdx.x;
    const int lane = t & 31, warp = t >> 5;
    uint16_t* S0 = state + (su * Hv + (int64_t)g * r) * (int64_t)(kD * kD);
    const uint32_t tile_bytes = (uint32_t)r * kD * kD * 2;
    const uint32_t bar_a = tc::smem_u32(&bar);
    if (t == 0) {
        abort_flag = 0;
        tc::mbar_init(bar_a, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(bar_a, tile_bytes);
        tc::bulk_load(tc::smem_u32(tiles), S0, tile_bytes, bar_a);
    }

    const uint16_t* xrow = qkv + u * Ctot;
    const float* wl = conv_w + (int64_t)l * Ctot * 4;
    float* csu = conv_state + su * Ctot * 3;

    // ---- q and k of key head g: channel t of each
    {
        const int64_t cq = (int64_t)g * kD + t, ck = (int64_t)(Hqk + g) * kD + t;
        float csq[3], csk[3];
        for (int j = 0; j < 3; ++j) { csq[j] = csu[cq * 3 + j]; csk[j] = csu[ck * 3 + j]; }
        const float yq = conv_channel(bf16_to_f32(xrow[cq]), csq, wl + cq * 4);
        const float yk = conv_channel(bf16_to_f32(xrow[ck]), csk, wl + ck * 4);
        for (int j = 0; j < 3; ++j) { csu[cq * 3 + j] = csq[j]; csu[ck * 3 + j] = csk[j]; }
        const float nq = block_sum(yq * yq, red);
        const float nk = block_sum(yk * yk, red);
        qs[t] = yq * rsqrtf(nq + 1e-6f);
        ks[t] = yk * rsqrtf(nk + 1e-6f);
    }
    __syncthreads();
    const float4 k4 = *reinterpret_cast<const float4*>(ks + lane * 4);
    const float4 q4 = *reinterpret_cast<const float4*>(qs + lane * 4);
    const float kq = warp_sum(k4.x * q4.x + k4.y * q4.y + k4.z * q4.z + k4.w * q4.w);
    // the states have landed (bounded: on expiry the outputs of this key head's
    // value heads become NaN, the states are left as they were, and the copy is
    // waited for again, bounded, before the CTA exits)
    const bool landed = tc::mbar_wait(bar_a, 0, &abort_flag, kFusedWaitLimitNs);

    for (int j = 0; j < r; ++j) {
        const int h = g * r + j;
        // ---- v of value head h: channel t (the conv history advances either way)
        {
            const int64_t cv = (int64_t)(2 * Hqk + h) * kD + t;
            float csv[3];
            for (int m = 0; m < 3; ++m) csv[m] = csu[cv * 3 + m];
            const float yv = conv_channel(bf16_to_f32(xrow[cv]), csv, wl + cv * 4);
            for (int m = 0; m < 3; ++m) csu[cv * 3 + m] = csv[m];
            __syncthreads();                       // the previous head's rows are done with vs
            vs[t] = yv;
            __syncthreads();
        }
        const int64_t uh = u * Hv + h;
        float* oh = o + uh * kD;
        if (!landed) {
            oh[t] = __int_as_float(0x7fc00000);
            continue;
        }
        const float alpha = expf(log_alpha_f32(a[uh], A_log[(int64_t)l * Hv + h], dt_bias[(int64_t)l * Hv + h]));
        const float beta = sigmoid_f32(b[uh]);
        uint16_t* S = S0 + (int64_t)j * (kD * kD);
        const uint2* tile = reinterpret_cast<const uint2*>(tiles + (size_t)j * kD * kD * 2);
#pragma unroll 1
        for (int r0 = warp * 32; r0 < warp * 32 + 32; r0 += kFusedBf16Rows) {
            float4 sr[kFusedBf16Rows];
#pragma unroll
            for (int i = 0; i < kFusedBf16Rows; ++i) {
                const uint2 w2 = tile[(r0 + i) * (kD / 4) + lane];
                const float2 x0 = bf16x2_to_f32x2(w2.x), x1 = bf16x2_to_f32x2(w2.y);
                sr[i] = make_float4(x0.x, x0.y, x1.x, x1.y);
            }
            float xk[kFusedBf16Rows], xq[kFusedBf16Rows];
#pragma unroll
            for (int i = 0; i < kFusedBf16Rows; ++i) {
                xk[i] = sr[i].x * k4.x + sr[i].y * k4.y + sr[i].z * k4.z + sr[i].w * k4.w;
                xq[i] = sr[i].x * q4.x + sr[i].y * q4.y + sr[i].z * q4.z + sr[i].w * q4.w;
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
#pragma unroll
                for (int i = 0; i < kFusedBf16Rows; ++i) {
                    xk[i] += __shfl_xor_sync(0xffffffffu, xk[i], m);
                    xq[i] += __shfl_xor_sync(0xffffffffu, xq[i], m);
                }
            }
            float orow = 0.f;
#pragma unroll
            for (int i = 0; i < kFusedBf16Rows; ++i) {
                const float w = beta * (vs[r0 + i] - alpha * xk[i]);
                float4 nv;
                nv.x = fmaf(alpha, sr[i].x, w * k4.x);
                nv.y = fmaf(alpha, sr[i].y, w * k4.y);
                nv.z = fmaf(alpha, sr[i].z, w * k4.z);
                nv.w = fmaf(alpha, sr[i].w, w * k4.w);
                state_store4(S + (int64_t)(r0 + i) * kD, lane, nv);
                const float oi = scale * fmaf(alpha, xq[i], w * kq);
                if (lane == i) orow = oi;
            }
            if (lane < kFusedBf16Rows) oh[r0 + lane] = orow;
        }
    }
    if (!landed) {
        volatile int no_abort = 0;
        tc::mbar_wait(bar_a, 0, &no_abort, kFusedWaitLimitNs);
    }
}

}  // namespace

cudaError_t launch_decode_fused(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                const float* a, const float* b, const float* A_log,
                                const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                int32_t layers, int32_t Hqk, int32_t Hv, float scale, float* state,
                                float* o, cudaStream_t stream) {
    const int64_t blocks = (int64_t)n_seq * layers * Hqk;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    decode_fused_kernel<float><<<(unsigned)blocks, kThreads, 0, stream>>>(
        qkv, conv_w, conv_state, a, b, A_log, dt_bias, slot, layers, Hqk, Hv, scale, state, o);
    return cudaGetLastError();
}

cudaError_t launch_decode_fused_bf16(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                     const float* a, const float* b, const float* A_log,
                                     const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                     int32_t layers, int32_t Hqk, int32_t Hv, float scale,
                                     uint16_t* state, float* o, cudaStream_t stream) {
    const int64_t blocks = (int64_t)n_seq * layers * Hqk;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const int r = Hv / Hqk;
    const size_t smem = (size_t)r * kD * kD * 2;
    if (smem > 200 * 1024) {
        // more value heads per key head than the staged kernel holds: the register kernel
        decode_fused_kernel<uint16_t><<<(unsigned)blocks, kThreads, 0, stream>>>(
            qkv, conv_w, conv_state, a, b, A_log, dt_bias, slot, layers, Hqk, Hv, scale, state, o);
        return cudaGetLastError();
    }
    cudaError_t e = cudaFuncSetAttribute(decode_fused_bf16_smem_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_fused_bf16_smem_kernel<<<(unsigned)blocks, kThreads, smem, stream>>>(
        qkv, conv_w, conv_state, a, b, A_log, dt_bias, slot, layers, Hqk, Hv, scale, state, o);
    return cudaGetLastError();
}

}  // namespace gdn
