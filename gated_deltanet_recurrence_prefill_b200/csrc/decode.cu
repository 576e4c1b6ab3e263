// decode.cu -- one token of the gated delta rule for many (sequence, layer)
// units, state updated in place.
//
// Per value head the step is S <- alpha S (I - beta k k^T) + beta v k^T and
// o = scale S q (Qwen3.8-27B architecture page, 2kiu.com, section 2.2, with
// the decay alpha on the erased state).  Row i of S (d_k wide) changes as
//     x_i = S_i . k,   S_i <- alpha S_i + beta (v_i - alpha x_i) k,
// and the output needs the updated row only through
//     S_i' . q = alpha (S_i . q) + beta (v_i - alpha x_i) (k . q),
// so both dot products are taken from the row as loaded and every row is read
// once and written once.  The state is float32 and dominates the traffic
// (2 x 64 KiB per value head per token); the kernel is bound by HBM bandwidth.
//
// Mapping: one CTA of 128 threads per (unit, value head).  Each warp owns 32
// rows; a lane holds 4 consecutive d_k elements of a row (a float4, or 8 bytes
// for a bf16 state), so a row is one fully coalesced access.  Eight rows are
// in flight per warp to keep enough bytes outstanding.
//
// The state is stored in float32 (the layer's state, architecture page section
// 2.2) or, in the bf16 variant, as bf16: the arithmetic is float32 either way
// and the updated row is rounded to bf16 (nearest even) when stored, which
// halves the bytes of this bandwidth-bound step.  The bf16 variant has a
// kernel of its own that stages each state in shared memory (below).
#include "common.cuh"
#include "decode_state.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace gdn {

namespace {

constexpr int kD = 128;
constexpr int kThreads = 128;
static_assert(kThreads == kD && kThreads / 32 == 4, "the output norm takes one row per thread");
// rows in flight per warp: 8 float32 rows or 16 bf16 rows (4 KB either way)
template <typename StateT> constexpr int rows_per_iter() { return sizeof(StateT) == 4 ? 8 : 16; }

template <typename StateT>
__global__ void __launch_bounds__(kThreads, sizeof(StateT) == 2 ? 3 : 5)
decode_step_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                   const uint16_t* __restrict__ v, const float* __restrict__ a,
                   const float* __restrict__ b, const float* __restrict__ A_log,
                   const float* __restrict__ dt_bias, int32_t layers, int32_t Hqk, int32_t Hv,
                   float scale, StateT* __restrict__ state, float* __restrict__ o, DecodeNorm nrm) {
    __shared__ float o_sm[kD];
    __shared__ float ss_sm[kThreads / 32];
    const int64_t uh = blockIdx.x;                 // unit * Hv + h
    const int64_t u = uh / Hv;
    const int h = (int)(uh - u * Hv);
    const int g = h / (Hv / Hqk);
    const int l = (int)(u % layers);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    // this lane's 4 elements of k and q
    const uint2 kb = *reinterpret_cast<const uint2*>(k + (u * Hqk + g) * kD + lane * 4);
    const uint2 qb = *reinterpret_cast<const uint2*>(q + (u * Hqk + g) * kD + lane * 4);
    const float2 k01 = bf16x2_to_f32x2(kb.x), k23 = bf16x2_to_f32x2(kb.y);
    const float2 q01 = bf16x2_to_f32x2(qb.x), q23 = bf16x2_to_f32x2(qb.y);
    const float kq = warp_sum(k01.x * q01.x + k01.y * q01.y + k23.x * q23.x + k23.y * q23.y);

    const float alpha = expf(log_alpha_f32(a[uh], A_log[(int64_t)l * Hv + h], dt_bias[(int64_t)l * Hv + h]));
    const float beta = sigmoid_f32(b[uh]);

    StateT* S = state + uh * (int64_t)(kD * kD);
    constexpr int kRowsPerIter = rows_per_iter<StateT>();
    const uint16_t* vh = v + uh * kD;
    float* oh = o ? o + uh * kD : nullptr;

#pragma unroll 1
    for (int r0 = warp * 32; r0 < warp * 32 + 32; r0 += kRowsPerIter) {
        float4 s[kRowsPerIter];
#pragma unroll
        for (int j = 0; j < kRowsPerIter; ++j)
            s[j] = state_load4(S + (int64_t)(r0 + j) * kD, lane);
        // v for these rows: 16-byte broadcast loads of 8 values
        float vr[kRowsPerIter];
#pragma unroll
        for (int j8 = 0; j8 < kRowsPerIter; j8 += 8) {
            const uint4 vb = *reinterpret_cast<const uint4*>(vh + r0 + j8);
            float2 t;
            t = bf16x2_to_f32x2(vb.x); vr[j8 + 0] = t.x; vr[j8 + 1] = t.y;
            t = bf16x2_to_f32x2(vb.y); vr[j8 + 2] = t.x; vr[j8 + 3] = t.y;
            t = bf16x2_to_f32x2(vb.z); vr[j8 + 4] = t.x; vr[j8 + 5] = t.y;
            t = bf16x2_to_f32x2(vb.w); vr[j8 + 6] = t.x; vr[j8 + 7] = t.y;
        }
        float xk[kRowsPerIter], xq[kRowsPerIter];
#pragma unroll
        for (int j = 0; j < kRowsPerIter; ++j) {
            xk[j] = s[j].x * k01.x + s[j].y * k01.y + s[j].z * k23.x + s[j].w * k23.y;
            xq[j] = s[j].x * q01.x + s[j].y * q01.y + s[j].z * q23.x + s[j].w * q23.y;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
#pragma unroll
            for (int j = 0; j < kRowsPerIter; ++j) {
                xk[j] += __shfl_xor_sync(0xffffffffu, xk[j], m);
                xq[j] += __shfl_xor_sync(0xffffffffu, xq[j], m);
            }
        }
        float orow = 0.f;
#pragma unroll
        for (int j = 0; j < kRowsPerIter; ++j) {
            const float w = beta * (vr[j] - alpha * xk[j]);
            float4 t;
            t.x = fmaf(alpha, s[j].x, w * k01.x);
            t.y = fmaf(alpha, s[j].y, w * k01.y);
            t.z = fmaf(alpha, s[j].z, w * k23.x);
            t.w = fmaf(alpha, s[j].w, w * k23.y);
            state_store4(S + (int64_t)(r0 + j) * kD, lane, t);
            const float oj = scale * fmaf(alpha, xq[j], w * kq);
            if (lane == j) orow = oj;
        }
        if (lane < kRowsPerIter) {
            if (o) oh[r0 + lane] = orow;
            if (nrm.y) o_sm[r0 + lane] = orow;
        }
    }
    if (nrm.y) {
        // gated output norm of this (unit, head): y = w * o / sqrt(mean o^2 + eps) * silu(z),
        // thread i takes row i
        __syncthreads();
        const int i = threadIdx.x;
        const float oi = o_sm[i];
        const float ssw = warp_sum(oi * oi);
        if (lane == 0) ss_sm[warp] = ssw;
        __syncthreads();
        const float r = rsqrtf(((ss_sm[0] + ss_sm[1]) + (ss_sm[2] + ss_sm[3])) * (1.f / kD) + nrm.eps);
        const float zf = bf16_to_f32(nrm.z[uh * kD + i]);
        const float g = zf * __frcp_rn(1.f + __expf(-zf));
        nrm.y[uh * kD + i] = (uint16_t)f32_to_bf16_bits(nrm.w[(int64_t)l * kD + i] * (oi * r) * g);
    }
}

// bf16 state: the whole 32 KiB state of the (unit, head) is brought into shared
// memory by one bulk copy, so the bytes in flight come from shared memory
// rather than registers (a 16-row register batch kept too few bytes in flight
// per SM for this half-size state).  Five CTAs share an SM, each with its
// state tile in flight; rows are then read from shared memory (a row is 256
// bytes: 8 per lane, conflict-free) and the updated rows are written to global
// memory from registers with streaming stores.
constexpr int kBf16Rows = 8;               // rows per warp iteration
constexpr uint64_t kDecodeWaitLimitNs = 2000000000ull;      // 2 s
constexpr uint32_t kTileBytes = kD * kD * 2;

__global__ void __launch_bounds__(kThreads, 5)
decode_step_bf16_smem_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                             const uint16_t* __restrict__ v, const float* __restrict__ a,
                             const float* __restrict__ b, const float* __restrict__ A_log,
                             const float* __restrict__ dt_bias, int32_t layers, int32_t Hqk, int32_t Hv,
                             float scale, uint16_t* __restrict__ state, float* __restrict__ o,
                             DecodeNorm nrm, uint64_t wait_limit_ns) {
    extern __shared__ __align__(128) uint8_t tile_raw[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float o_sm[kD];
    __shared__ float ss_sm[kThreads / 32];
    __shared__ int abort_flag;
    const int64_t uh = blockIdx.x;                 // unit * Hv + h
    const int64_t u = uh / Hv;
    const int h = (int)(uh - u * Hv);
    const int g = h / (Hv / Hqk);
    const int l = (int)(u % layers);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    uint16_t* S = state + uh * (int64_t)(kD * kD);
    const uint32_t bar_a = tc::smem_u32(&bar);
    if (threadIdx.x == 0) {
        abort_flag = 0;
        tc::mbar_init(bar_a, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(bar_a, kTileBytes);
        tc::bulk_load(tc::smem_u32(tile_raw), S, kTileBytes, bar_a);
    }
    // while the tile is in flight: this lane's 4 elements of k and q, the gates
    const uint2 kb = *reinterpret_cast<const uint2*>(k + (u * Hqk + g) * kD + lane * 4);
    const uint2 qb = *reinterpret_cast<const uint2*>(q + (u * Hqk + g) * kD + lane * 4);
    const float2 k01 = bf16x2_to_f32x2(kb.x), k23 = bf16x2_to_f32x2(kb.y);
    const float2 q01 = bf16x2_to_f32x2(qb.x), q23 = bf16x2_to_f32x2(qb.y);
    const float kq = warp_sum(k01.x * q01.x + k01.y * q01.y + k23.x * q23.x + k23.y * q23.y);
    const float alpha = expf(log_alpha_f32(a[uh], A_log[(int64_t)l * Hv + h], dt_bias[(int64_t)l * Hv + h]));
    const float beta = sigmoid_f32(b[uh]);
    const uint16_t* vh = v + uh * kD;
    float* oh = o ? o + uh * kD : nullptr;
    __syncthreads();                               // the barrier is initialised
    if (!tc::mbar_wait(bar_a, 0, &abort_flag, wait_limit_ns)) {
        // the copy did not land in time (a bound far beyond any legitimate
        // wait): the outputs of this (unit, head) become NaN, which the caller
        // can test, and the state is left as it was.  The copy may still land
        // in this CTA's shared memory, so it is waited for again, bounded,
        // before the CTA exits.
        const int i = threadIdx.x;
        if (oh) oh[i] = __int_as_float(0x7fc00000);
        if (nrm.y) nrm.y[uh * kD + i] = 0x7fc0;
        volatile int no_abort = 0;
        tc::mbar_wait(bar_a, 0, &no_abort, wait_limit_ns);
        return;
    }
    const uint2* tile = reinterpret_cast<const uint2*>(tile_raw);
#pragma unroll 1
    for (int r0 = warp * 32; r0 < warp * 32 + 32; r0 += kBf16Rows) {
        float4 s[kBf16Rows];
#pragma unroll
        for (int j = 0; j < kBf16Rows; ++j) {
            const uint2 r = tile[(r0 + j) * (kD / 4) + lane];
            const float2 x0 = bf16x2_to_f32x2(r.x), x1 = bf16x2_to_f32x2(r.y);
            s[j] = make_float4(x0.x, x0.y, x1.x, x1.y);
        }
        float vr[kBf16Rows];
        {
            const uint4 vb = *reinterpret_cast<const uint4*>(vh + r0);
            float2 t;
            t = bf16x2_to_f32x2(vb.x); vr[0] = t.x; vr[1] = t.y;
            t = bf16x2_to_f32x2(vb.y); vr[2] = t.x; vr[3] = t.y;
            t = bf16x2_to_f32x2(vb.z); vr[4] = t.x; vr[5] = t.y;
            t = bf16x2_to_f32x2(vb.w); vr[6] = t.x; vr[7] = t.y;
        }
        float xk[kBf16Rows], xq[kBf16Rows];
#pragma unroll
        for (int j = 0; j < kBf16Rows; ++j) {
            xk[j] = s[j].x * k01.x + s[j].y * k01.y + s[j].z * k23.x + s[j].w * k23.y;
            xq[j] = s[j].x * q01.x + s[j].y * q01.y + s[j].z * q23.x + s[j].w * q23.y;
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
#pragma unroll
            for (int j = 0; j < kBf16Rows; ++j) {
                xk[j] += __shfl_xor_sync(0xffffffffu, xk[j], m);
                xq[j] += __shfl_xor_sync(0xffffffffu, xq[j], m);
            }
        }
        float orow = 0.f;
#pragma unroll
        for (int j = 0; j < kBf16Rows; ++j) {
            const float w = beta * (vr[j] - alpha * xk[j]);
            float4 t;
            t.x = fmaf(alpha, s[j].x, w * k01.x);
            t.y = fmaf(alpha, s[j].y, w * k01.y);
            t.z = fmaf(alpha, s[j].z, w * k23.x);
            t.w = fmaf(alpha, s[j].w, w * k23.y);
            state_store4(S + (int64_t)(r0 + j) * kD, lane, t);
            const float oj = scale * fmaf(alpha, xq[j], w * kq);
            if (lane == j) orow = oj;
        }
        if (lane < kBf16Rows) {
            if (o) oh[r0 + lane] = orow;
            if (nrm.y) o_sm[r0 + lane] = orow;
        }
    }
    if (nrm.y) {
        // gated output norm of this (unit, head), thread i takes row i
        __syncthreads();
        const int i = threadIdx.x;
        const float oi = o_sm[i];
        const float ssw = warp_sum(oi * oi);
        if (lane == 0) ss_sm[warp] = ssw;
        __syncthreads();
        const float r = rsqrtf(((ss_sm[0] + ss_sm[1]) + (ss_sm[2] + ss_sm[3])) * (1.f / kD) + nrm.eps);
        const float zf = bf16_to_f32(nrm.z[uh * kD + i]);
        const float gz = zf * __frcp_rn(1.f + __expf(-zf));
        nrm.y[uh * kD + i] = (uint16_t)f32_to_bf16_bits(nrm.w[(int64_t)l * kD + i] * (oi * r) * gz);
    }
}

}  // namespace

cudaError_t launch_decode_step(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const float* a, const float* b, const float* A_log,
                               const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                               int32_t Hv, float scale, float* state, float* o,
                               cudaStream_t stream, const DecodeNorm& nrm) {
    const int64_t blocks = (int64_t)n_seq * layers * Hv;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    decode_step_kernel<float><<<(unsigned)blocks, kThreads, 0, stream>>>(
        q, k, v, a, b, A_log, dt_bias, layers, Hqk, Hv, scale, state, o, nrm);
    return cudaGetLastError();
}

cudaError_t launch_decode_step_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const float* a, const float* b, const float* A_log,
                                    const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                                    int32_t Hv, float scale, uint16_t* state, float* o,
                                    cudaStream_t stream, const DecodeNorm& nrm) {
    const int64_t blocks = (int64_t)n_seq * layers * Hv;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(decode_step_bf16_smem_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTileBytes);
    if (e != cudaSuccess) return e;
    decode_step_bf16_smem_kernel<<<(unsigned)blocks, kThreads, kTileBytes, stream>>>(
        q, k, v, a, b, A_log, dt_bias, layers, Hqk, Hv, scale, state, o, nrm, kDecodeWaitLimitNs);
    return cudaGetLastError();
}

}  // namespace gdn
