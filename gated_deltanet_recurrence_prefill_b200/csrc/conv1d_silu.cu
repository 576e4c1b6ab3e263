// conv1d_silu.cu -- the layer's front end: causal depthwise convolution of
// width 4 over time (Qwen3.8-27B architecture page, 2kiu.com, section 2.1:
// linear_conv_kernel_dim = 4, conv1d.weight), SiLU on every channel, then q
// and k divided per head by sqrt(sum of squares + 1e-6).
//
// The work is elementwise in time apart from a 3-token history, so it is bound
// by HBM bandwidth (read the packed bf16 channels once, write q, k, v once).
//
// Mapping: a half-warp covers one head (16 lanes x 8 channels = 128), a warp
// two heads; each lane moves 16 bytes per token.  A warp walks a run of
// kRun consecutive tokens, keeping the last three inputs of its 8 channels in
// registers, so each input is loaded once plus a 3-token halo per run.  The
// inputs of the next 16 tokens are requested ahead by cp.async into a ring in
// shared memory (each lane reads back only its own 16-byte pieces, so no
// barrier is needed); holding them in registers instead kept fewer bytes in
// flight and measured 14% slower (0.104 against 0.090 ms at T = 8192).  At a
// sequence boundary the history restarts from conv_state_in
// (or zeros).  (A variant that staged 64-token tiles in shared memory by TMA
// measured slower: with one tile's arithmetic per barrier the SMs sat idle.)
//
// The kernel is bound as much by instruction issue as by HBM (about 130
// instructions per lane and token for 16 bytes in and 16 out), so a run that
// lies inside one sequence and is a full kRun tokens long takes a fast path:
// the arithmetic on pairs of channels with the packed f32x2 FMA of sm_100a,
// tokens in unrolled steps of three (the width of the history, so the history
// rotates by register renaming instead of copies), and pointers advanced
// instead of recomputed.  Runs that hold a sequence boundary, and the last
// partial run, take the general per-token path.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

namespace {

constexpr int kD = 128;
constexpr int kRun = 48;              // tokens per warp (a multiple of kStep)
constexpr int kWarps = 8;             // warps per CTA
constexpr int kChan = 8;              // channels per lane
#ifndef GDN_CONV_BATCH
#define GDN_CONV_BATCH 4
#endif
constexpr int kBatch = GDN_CONV_BATCH;  // tokens per batch
// Loads in flight: each lane copies its 16 bytes of the next kDepth tokens into
// a ring in shared memory by cp.async (completion tracked per thread, so a
// lane only ever reads back what it copied itself, and no register holds data
// in flight); kDepth / kBatch batches are outstanding at once.
constexpr int kDepth = 16;
static_assert(kDepth % kBatch == 0 && kRun % kBatch == 0, "ring of whole batches");
// fast path: steps of three tokens, four steps in flight in the first 12 ring slots
constexpr int kStep = 3;
constexpr int kFastSteps = 4;
static_assert(kRun % kStep == 0 && kStep * kFastSteps <= kDepth, "fast path ring");
constexpr int kRingBytesPerWarp = kDepth * 32 * 16;

// index of the sequence containing token t: largest n with cu[n] <= t
__device__ int find_seq(const int32_t* cu, int n_seq, int64_t t) {
    int lo = 0, hi = n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// SiLU(x) = x sigmoid(x) = h + h tanh(h), h = x / 2, since sigmoid(x) =
// (1 + tanh(x / 2)) / 2: one special-function instruction per value (the
// hardware tanh approximation, relative error about 2^-11, well below the
// bf16 rounding of the output).
GDN_DEVICE float silu_f32(float x) {
    const float h = 0.5f * x;
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(h));
    return fmaf(h, th, h);
}

GDN_DEVICE void cp_async16(void* sdst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(sdst)),
                 "l"(gsrc)
                 : "memory");
}
GDN_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> GDN_DEVICE void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
GDN_DEVICE void stg_stream(uint16_t* p, uint4 v) { __stcs(reinterpret_cast<uint4*>(p), v); }

GDN_DEVICE float2 silu2(float2 x) {
    const float2 h = __fmul2_rn(x, make_float2(0.5f, 0.5f));
    float tx, ty;
    asm("tanh.approx.f32 %0, %1;" : "=f"(tx) : "f"(h.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(ty) : "f"(h.y));
    return __ffma2_rn(h, make_float2(tx, ty), h);
}

GDN_DEVICE void unpack4x2(const uint4 r, float2* x) {
    x[0] = bf16x2_to_f32x2(r.x);
    x[1] = bf16x2_to_f32x2(r.y);
    x[2] = bf16x2_to_f32x2(r.z);
    x[3] = bf16x2_to_f32x2(r.w);
}

GDN_DEVICE void unpack8(const uint4 r, float* x) {
    float2 t;
    t = bf16x2_to_f32x2(r.x); x[0] = t.x; x[1] = t.y;
    t = bf16x2_to_f32x2(r.y); x[2] = t.x; x[3] = t.y;
    t = bf16x2_to_f32x2(r.z); x[4] = t.x; x[5] = t.y;
    t = bf16x2_to_f32x2(r.w); x[6] = t.x; x[7] = t.y;
}

GDN_DEVICE void load8(const uint16_t* p, float* x) {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    float2 t;
    t = bf16x2_to_f32x2(r.x); x[0] = t.x; x[1] = t.y;
    t = bf16x2_to_f32x2(r.y); x[2] = t.x; x[3] = t.y;
    t = bf16x2_to_f32x2(r.z); x[4] = t.x; x[5] = t.y;
    t = bf16x2_to_f32x2(r.w); x[6] = t.x; x[7] = t.y;
}

__global__ void __launch_bounds__(kWarps * 32, 2)
conv1d_silu_kernel(const uint16_t* __restrict__ qkv, const float* __restrict__ w,
                   const int32_t* __restrict__ cu, int32_t n_seq, int64_t T, int32_t Hqk,
                   int32_t Hv, const float* __restrict__ cs_in, uint16_t* __restrict__ qo,
                   uint16_t* __restrict__ ko, uint16_t* __restrict__ vo, int64_t n_runs) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int n_heads = 2 * Hqk + Hv;
    const int n_pairs = (n_heads + 1) >> 1;
    const int64_t run = gw / n_pairs;
    if (run >= n_runs) return;
    const int pair = (int)(gw - run * n_pairs);
    const int head = pair * 2 + (lane >> 4);
    const bool active = head < n_heads;
    const int hc = head < n_heads ? head : n_heads - 1;        // clamp for address math
    const int64_t Ctot = (int64_t)n_heads * kD;
    const int64_t c0 = (int64_t)hc * kD + (lane & 15) * kChan;  // first channel of this lane

    float wr[kChan][4];
#pragma unroll
    for (int i = 0; i < kChan; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(w + (c0 + i) * 4);
        wr[i][0] = t.x; wr[i][1] = t.y; wr[i][2] = t.z; wr[i][3] = t.w;
    }

    const int64_t t0 = run * kRun;
    const int64_t t1 = t0 + kRun < T ? t0 + kRun : T;
    int n = cu ? find_seq(cu, n_seq, t0) : 0;
    // a sequence of length 0 shares its start with the next one: skip to the
    // sequence that actually contains t0
    int64_t bos = cu ? cu[n] : 0;
    int64_t eos = cu ? cu[n + 1] : T;

    // history h[j] = x[t - 3 + j] for j = 0..2, relative to the current t
    float hist[3][kChan];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int64_t tau = t0 - 3 + j;
        if (tau >= bos) {
            load8(qkv + tau * Ctot + c0, hist[j]);
        } else if (cs_in) {
            const int64_t m = bos - tau;             // 1..3 tokens before the start
#pragma unroll
            for (int i = 0; i < kChan; ++i) hist[j][i] = cs_in[((int64_t)n * Ctot + c0 + i) * 3 + (3 - m)];
        } else {
#pragma unroll
            for (int i = 0; i < kChan; ++i) hist[j][i] = 0.f;
        }
    }

    const bool is_q = head < Hqk;
    const bool is_k = head >= Hqk && head < 2 * Hqk;
    // does either half-warp hold a q or k head (then both take part in the reduction)
    const bool warp_norm = __any_sync(0xffffffffu, is_q || is_k);
    uint16_t* dst_base;
    int64_t dst_stride;
    if (is_q) { dst_base = qo + (int64_t)head * kD; dst_stride = (int64_t)Hqk * kD; }
    else if (is_k) { dst_base = ko + (int64_t)(head - Hqk) * kD; dst_stride = (int64_t)Hqk * kD; }
    else { dst_base = vo + (int64_t)(hc - 2 * Hqk) * kD; dst_stride = (int64_t)Hv * kD; }
    dst_base += (lane & 15) * kChan;

    extern __shared__ __align__(16) uint8_t ring_all[];
    uint8_t* ring = ring_all + (threadIdx.x >> 5) * kRingBytesPerWarp + lane * 16;

    if (t1 - t0 == kRun && eos >= t1) {
        // ---- fast path: a full run inside one sequence.  Step j covers tokens
        // t0 + 3 j .. + 2, whose inputs sit in ring slots 3 (j % 4) .. + 2,
        // requested four steps ahead (one commit group per step).
        float2 w2[4][4], h[3][4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
#pragma unroll
            for (int j = 0; j < 4; ++j) w2[p][j] = make_float2(wr[2 * p][j], wr[2 * p + 1][j]);
#pragma unroll
            for (int j = 0; j < 3; ++j) h[j][p] = make_float2(hist[j][2 * p], hist[j][2 * p + 1]);
        }
        const uint16_t* src = qkv + t0 * Ctot + c0;
#pragma unroll
        for (int st = 0; st < kFastSteps; ++st) {
#pragma unroll
            for (int u = 0; u < kStep; ++u) cp_async16(ring + (st * kStep + u) * 512, src + (st * kStep + u) * Ctot);
            cp_async_commit();
        }
        uint16_t* dst = dst_base + t0 * dst_stride;
#pragma unroll 1
        for (int st = 0; st < kRun / kStep; ++st) {
            cp_async_wait<kFastSteps - 1>();
            const int slot0 = (st % kFastSteps) * kStep;
            float2 x[kStep][4];
#pragma unroll
            for (int u = 0; u < kStep; ++u) unpack4x2(*reinterpret_cast<const uint4*>(ring + (slot0 + u) * 512), x[u]);
            // the slots just read take the step kFastSteps ahead (its group may be empty)
            if (st + kFastSteps < kRun / kStep) {
#pragma unroll
                for (int u = 0; u < kStep; ++u)
                    cp_async16(ring + (slot0 + u) * 512, src + ((st + kFastSteps) * kStep + u) * Ctot);
            }
            cp_async_commit();
#pragma unroll
            for (int u = 0; u < kStep; ++u) {
                // inputs x[t-3], x[t-2], x[t-1], x[t] of token u of this step
                float2 y[4];
                float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 a0 = u == 0 ? h[0][p] : (u == 1 ? h[1][p] : h[2][p]);
                    const float2 a1 = u == 0 ? h[1][p] : (u == 1 ? h[2][p] : x[0][p]);
                    const float2 a2 = u == 0 ? h[2][p] : (u == 1 ? x[0][p] : x[1][p]);
                    float2 acc = __fmul2_rn(w2[p][0], a0);
                    acc = __ffma2_rn(w2[p][1], a1, acc);
                    acc = __ffma2_rn(w2[p][2], a2, acc);
                    acc = __ffma2_rn(w2[p][3], x[u][p], acc);
                    y[p] = silu2(acc);
                    ss2 = __ffma2_rn(y[p], y[p], ss2);
                }
                if (warp_norm) {       // warp-uniform: the shuffles need all 32 lanes
                    float ss = ss2.x + ss2.y;
#pragma unroll
                    for (int m = 8; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                    const float inv = (is_q || is_k) ? rsqrtf(ss + 1e-6f) : 1.f;
                    const float2 iv = make_float2(inv, inv);
#pragma unroll
                    for (int p = 0; p < 4; ++p) y[p] = __fmul2_rn(y[p], iv);
                }
                uint4 out;
                out.x = pack_bf16x2(y[0].x, y[0].y);
                out.y = pack_bf16x2(y[1].x, y[1].y);
                out.z = pack_bf16x2(y[2].x, y[2].y);
                out.w = pack_bf16x2(y[3].x, y[3].y);
                if (active) stg_stream(dst, out);
                dst += dst_stride;
            }
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                h[0][p] = x[0][p];
                h[1][p] = x[1][p];
                h[2][p] = x[2][p];
            }
        }
        cp_async_wait<0>();
        return;
    }

    // tokens are processed in batches of kBatch; token t's 16 bytes of this lane
    // sit in ring slot (t - t0) % kDepth, requested kDepth tokens ahead, one
    // commit group per batch
#pragma unroll
    for (int bq = 0; bq < kDepth / kBatch; ++bq) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int64_t t = t0 + bq * kBatch + u;
            if (t < t1) cp_async16(ring + (bq * kBatch + u) * 512, qkv + t * Ctot + c0);
        }
        cp_async_commit();
    }
    for (int64_t tb = t0; tb < t1; tb += kBatch) {
        cp_async_wait<kDepth / kBatch - 1>();      // this batch's group has landed
        uint4 raw[kBatch];
        const int slot0 = (int)((tb - t0) % kDepth);
#pragma unroll
        for (int u = 0; u < kBatch; ++u) raw[u] = *reinterpret_cast<const uint4*>(ring + (slot0 + u) * 512);
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int64_t t = tb + u;
            if (t >= t1) break;
            if (t >= eos) {
                // next sequence(s): skip empty ones, restart the history
                while (n + 1 < n_seq && (int64_t)cu[n + 1] <= t) ++n;
                bos = cu[n];
                eos = cu[n + 1];
#pragma unroll
                for (int j = 0; j < 3; ++j)
#pragma unroll
                    for (int i = 0; i < kChan; ++i)
                        hist[j][i] = cs_in ? cs_in[((int64_t)n * Ctot + c0 + i) * 3 + j] : 0.f;
            }
            float x[kChan];
            unpack8(raw[u], x);
            float y[kChan];
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < kChan; ++i) {
                float acc = wr[i][0] * hist[0][i];
                acc = fmaf(wr[i][1], hist[1][i], acc);
                acc = fmaf(wr[i][2], hist[2][i], acc);
                acc = fmaf(wr[i][3], x[i], acc);
                const float s = silu_f32(acc);
                y[i] = s;
                ss = fmaf(s, s, ss);
                hist[0][i] = hist[1][i];
                hist[1][i] = hist[2][i];
                hist[2][i] = x[i];
            }
            // sum of squares over the 16 lanes of this head (value heads need none)
            float inv = 1.f;
            if (warp_norm) {        // warp-uniform: the shuffles need all 32 lanes
#pragma unroll
                for (int m = 8; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                if (is_q || is_k) inv = rsqrtf(ss + 1e-6f);
            }
            uint4 out;
            out.x = pack_bf16x2(y[0] * inv, y[1] * inv);
            out.y = pack_bf16x2(y[2] * inv, y[3] * inv);
            out.z = pack_bf16x2(y[4] * inv, y[5] * inv);
            out.w = pack_bf16x2(y[6] * inv, y[7] * inv);
            if (active) stg_stream(dst_base + t * dst_stride, out);
        }
        // the slots just read take the tokens kDepth ahead
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int64_t t = tb + kDepth + u;
            if (t < t1) cp_async16(ring + (slot0 + u) * 512, qkv + t * Ctot + c0);
        }
        cp_async_commit();
    }
    cp_async_wait<0>();
}

// conv_state_out[n, c, s] = x[eos - 3 + s, c], or the incoming history when
// that position lies before the sequence start.
__global__ void conv_state_out_kernel(const uint16_t* __restrict__ qkv, const int32_t* __restrict__ cu,
                                      int32_t n_seq, int64_t T, int64_t Ctot,
                                      const float* __restrict__ cs_in, float* __restrict__ cs_out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)n_seq * Ctot) return;
    const int n = (int)(i / Ctot);
    const int64_t c = i - (int64_t)n * Ctot;
    const int64_t bos = cu ? cu[n] : 0;
    const int64_t eos = cu ? cu[n + 1] : T;
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        const int64_t tau = eos - 3 + s;
        float xv;
        if (tau >= bos) xv = bf16_to_f32(qkv[tau * Ctot + c]);
        else xv = cs_in ? cs_in[((int64_t)n * Ctot + c) * 3 + (3 - (bos - tau))] : 0.f;
        cs_out[i * 3 + s] = xv;
    }
}

}  // namespace

cudaError_t launch_conv1d_silu(const uint16_t* qkv, const float* w, const int32_t* cu,
                               int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv,
                               const float* cs_in, float* cs_out, uint16_t* q, uint16_t* k,
                               uint16_t* v, cudaStream_t stream) {
    const int n_heads = 2 * Hqk + Hv;
    const int n_pairs = (n_heads + 1) / 2;
    const int64_t Ctot = (int64_t)n_heads * kD;
    if (T > 0) {
        const int64_t n_runs = (T + kRun - 1) / kRun;
        const int64_t warps = n_runs * n_pairs;
        const int64_t blocks = (warps + kWarps - 1) / kWarps;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        const int smem = kWarps * kRingBytesPerWarp;
        cudaError_t e = cudaFuncSetAttribute(conv1d_silu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        conv1d_silu_kernel<<<(unsigned)blocks, kWarps * 32, smem, stream>>>(
            qkv, w, cu, n_seq, T, Hqk, Hv, cs_in, q, k, v, n_runs);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (cs_out) {
        const int64_t total = (int64_t)n_seq * Ctot;
        const int64_t blocks = (total + 255) / 256;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        if (blocks > 0)
            conv_state_out_kernel<<<(unsigned)blocks, 256, 0, stream>>>(qkv, cu, n_seq, T, Ctot,
                                                                        cs_in, cs_out);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace gdn
