// backward.cu -- the gradient of the gated delta-rule recurrence (the step of
// the Qwen3.8-27B architecture page, 2kiu.com, section 2.2, with the decay
// alpha on the erased state):
//     S_t = alpha_t S (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   S = S_{t-1},
//     o_t = scale S_t q_t.
// Given dL/do and dL/dS_T, one step back with G = dL/dS_t (including the
// output's scale d_o_t q_t^T) gives
//     dq_t += scale S_t^T d_o_t,    g = G k,    dv_t = beta g,
//     dk_t += -alpha beta (S^T g + G^T S k) + beta G^T v,
//     dalpha = <G, S> - beta (S k).g,   dbeta = -alpha (S k).g + v.g,
//     dL/dS_{t-1} = alpha (G - beta g k^T),
// then through the gates: log alpha = -exp(A_log) softplus(a + dt_bias),
// beta = sigmoid(b).
//
// First version: CUDA cores, one CTA of 512 threads per (sequence, value head),
// every token in turn.  Thread (warp r, lane c) owns rows 8r .. 8r + 7 and
// columns 4c .. 4c + 3 of the 128 x 128 state and of G, in registers, so the
// row sums (S k, G k) stay inside a warp; the column sums (dq, dk) and the
// scalars go through shared memory, one block barrier per token.  The states
// the backward sweep needs come from a forward pass that stores the state at
// every 64-token chunk start (checkpoints), and from a recomputation of each
// chunk, whose per-token states go to a per-CTA scratch in global memory.
// dq and dk are produced per value head and summed over each key head's group
// by a second kernel (fixed order: deterministic); dA_log and dt_bias are
// summed over tokens per (sequence, head) and then over sequences.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int kD = 128;
constexpr int kC = 64;                 // tokens per checkpointed chunk
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = kD / kWarps;     // 8 rows per thread
constexpr int kCols = kD / 32;         // 4 columns per thread
constexpr size_t kStateFloats = (size_t)kD * kD;

struct BwdParams {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    const float* a;
    const float* b;
    const float* A_log;
    const float* dt_bias;
    const int32_t* cu;
    int64_t T;
    int32_t Hqk, Hv;
    float scale;
    const float* s0;        // [n_seq, Hv, d, d] or NULL
    const float* d_o;       // [T, Hv, d]
    const float* d_fin;     // [n_seq, Hv, d, d] or NULL
    float* dqh;             // [T, Hv, d] per value head (summed later)
    float* dkh;             // [T, Hv, d]
    float* dv;              // [T, Hv, d]
    float* da;              // [T, Hv]
    float* db;              // [T, Hv]
    float* gate_part;       // [n_seq, Hv, 2]: sums over tokens of dA_log, ddt_bias
    float* d_init;          // [n_seq, Hv, d, d] or NULL
    float* ckpt;            // [slot (see slot_of)][Hv] checkpoints, each kD * kD floats
    float* hist;            // [n_seq * Hv, kC, kD * kD] per-chunk states
};

// checkpoint slot of the chunk of sequence n that starts at token t0: unique,
// at most T / 64 + n_seq of them
__device__ __forceinline__ int64_t slot_of(int64_t t0, int n) { return t0 / kC + n; }

__device__ __forceinline__ void load4(const uint16_t* p, float* x) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = bf16x2_to_f32x2(u.x), b = bf16x2_to_f32x2(u.y);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}

// this thread's 8 x 4 block of a state in global memory <-> registers
__device__ __forceinline__ void gload(const float* base, int r, int c, float (&s)[kRows][kCols]) {
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(base + (size_t)(r * kRows + i) * kD + c * kCols);
        s[i][0] = t.x; s[i][1] = t.y; s[i][2] = t.z; s[i][3] = t.w;
    }
}
__device__ __forceinline__ void gstore(float* base, int r, int c, const float (&s)[kRows][kCols]) {
#pragma unroll
    for (int i = 0; i < kRows; ++i)
        *reinterpret_cast<float4*>(base + (size_t)(r * kRows + i) * kD + c * kCols) =
            make_float4(s[i][0], s[i][1], s[i][2], s[i][3]);
}

// one forward step on this thread's block: S = alpha S + beta (v - alpha S k) k^T
__device__ __forceinline__ void fwd_step(float (&s)[kRows][kCols], const float* kv, const float* vv,
                                         float alpha, float beta) {
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
        float x = s[i][0] * kv[0] + s[i][1] * kv[1] + s[i][2] * kv[2] + s[i][3] * kv[3];
        x = warp_sum(x);
        const float u = beta * (vv[i] - alpha * x);
#pragma unroll
        for (int j = 0; j < kCols; ++j) s[i][j] = fmaf(alpha, s[i][j], u * kv[j]);
    }
}

__global__ void __launch_bounds__(kThreads, 1) gdn_backward_kernel(BwdParams p) {
    __shared__ float col_part[2][2][kWarps][kD];     // [step parity][dq | dk][warp][column]
    __shared__ float scal_part[2][kWarps][3];        // [step parity][warp][<G,S>, (Sk).g, v.g]
    const int n = blockIdx.x / p.Hv;
    const int h = blockIdx.x % p.Hv;
    const int g = h / (p.Hv / p.Hqk);
    const int r = threadIdx.x >> 5, c = threadIdx.x & 31;
    const int64_t bos = p.cu ? p.cu[n] : 0;
    const int64_t eos = p.cu ? p.cu[n + 1] : p.T;
    const size_t unit = (size_t)n * p.Hv + h;
    const float eA = expf(p.A_log[h]), dtb = p.dt_bias[h];
    float* hist = p.hist + unit * kC * kStateFloats;

    // ---- forward over the sequence: the state at every chunk start
    float s[kRows][kCols];
    if (p.s0) {
        gload(p.s0 + unit * kStateFloats, r, c, s);
    } else {
#pragma unroll
        for (int i = 0; i < kRows; ++i)
#pragma unroll
            for (int j = 0; j < kCols; ++j) s[i][j] = 0.f;
    }
    for (int64_t t = bos; t < eos; ++t) {
        if ((t - bos) % kC == 0) gstore(p.ckpt + ((size_t)slot_of(t, n) * p.Hv + h) * kStateFloats, r, c, s);
        float kv[kCols], vv[kRows];
        load4(p.k + (t * p.Hqk + g) * kD + c * kCols, kv);
        load4(p.v + (t * p.Hv + h) * kD + r * kRows, vv);
        load4(p.v + (t * p.Hv + h) * kD + r * kRows + 4, vv + 4);
        const float alpha = expf(log_alpha_f32(p.a[t * p.Hv + h], p.A_log[h], dtb));
        const float beta = sigmoid_f32(p.b[t * p.Hv + h]);
        fwd_step(s, kv, vv, alpha, beta);
    }

    // ---- backward, chunk by chunk from the last
    float G[kRows][kCols];
    if (p.d_fin) {
        gload(p.d_fin + unit * kStateFloats, r, c, G);
    } else {
#pragma unroll
        for (int i = 0; i < kRows; ++i)
#pragma unroll
            for (int j = 0; j < kCols; ++j) G[i][j] = 0.f;
    }
    float dA_acc = 0.f, ddt_acc = 0.f;            // thread 0's running sums
    int parity = 0;
    const int64_t len = eos - bos;
    for (int64_t c0 = len > 0 ? ((len - 1) / kC) * kC : -1; c0 >= 0; c0 -= kC) {
        const int64_t t0 = bos + c0;
        const int64_t t1 = (t0 + kC < eos) ? t0 + kC : eos;
        // recompute the chunk: hist[j] = state before token t0 + j; s ends as the
        // state after the chunk
        gload(p.ckpt + ((size_t)slot_of(t0, n) * p.Hv + h) * kStateFloats, r, c, s);
        for (int64_t t = t0; t < t1; ++t) {
            gstore(hist + (size_t)(t - t0) * kStateFloats, r, c, s);
            float kv[kCols], vv[kRows];
            load4(p.k + (t * p.Hqk + g) * kD + c * kCols, kv);
            load4(p.v + (t * p.Hv + h) * kD + r * kRows, vv);
            load4(p.v + (t * p.Hv + h) * kD + r * kRows + 4, vv + 4);
            const float alpha = expf(log_alpha_f32(p.a[t * p.Hv + h], p.A_log[h], dtb));
            const float beta = sigmoid_f32(p.b[t * p.Hv + h]);
            fwd_step(s, kv, vv, alpha, beta);
        }
        // s = S_t for the last token of the chunk; each step takes what it needs
        // of S_t, then loads S_{t-1} into s
        for (int64_t t = t1 - 1; t >= t0; --t) {
            float qv[kCols], kv[kCols], vv[kRows], dov[kRows];
            load4(p.q + (t * p.Hqk + g) * kD + c * kCols, qv);
            load4(p.k + (t * p.Hqk + g) * kD + c * kCols, kv);
            load4(p.v + (t * p.Hv + h) * kD + r * kRows, vv);
            load4(p.v + (t * p.Hv + h) * kD + r * kRows + 4, vv + 4);
            {
                const float4 d0 = *reinterpret_cast<const float4*>(p.d_o + (t * p.Hv + h) * kD + r * kRows);
                const float4 d1 = *reinterpret_cast<const float4*>(p.d_o + (t * p.Hv + h) * kD + r * kRows + 4);
                dov[0] = d0.x; dov[1] = d0.y; dov[2] = d0.z; dov[3] = d0.w;
                dov[4] = d1.x; dov[5] = d1.y; dov[6] = d1.z; dov[7] = d1.w;
            }
            const float la = log_alpha_f32(p.a[t * p.Hv + h], p.A_log[h], dtb);
            const float alpha = expf(la);
            const float beta = sigmoid_f32(p.b[t * p.Hv + h]);
            // dq partials (S_t^T d_o over this thread's rows); G += scale d_o q^T
            float cq[kCols] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < kRows; ++i)
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    cq[j] = fmaf(s[i][j], dov[i], cq[j]);
                    G[i][j] = fmaf(p.scale * dov[i], qv[j], G[i][j]);
                }
            float (&sp)[kRows][kCols] = s;             // from here on s holds S_{t-1}
            gload(hist + (size_t)(t - t0) * kStateFloats, r, c, sp);
            // row sums S k and G k (inside the warp), <G, S>
            float Sk[kRows], gk[kRows];
            float gs = 0.f;
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                float a1 = 0.f, a2 = 0.f;
#pragma unroll
                for (int j = 0; j < kCols; ++j) {
                    a1 = fmaf(sp[i][j], kv[j], a1);
                    a2 = fmaf(G[i][j], kv[j], a2);
                    gs = fmaf(G[i][j], sp[i][j], gs);
                }
                Sk[i] = warp_sum(a1);
                gk[i] = warp_sum(a2);
            }
            gs = warp_sum(gs);
            float skg = 0.f, vg = 0.f;
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                skg = fmaf(Sk[i], gk[i], skg);
                vg = fmaf(vv[i], gk[i], vg);
            }
            // dk partials: -alpha beta (S^T g + G^T S k) + beta G^T v over this thread's rows
            float ck[kCols] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < kRows; ++i)
#pragma unroll
                for (int j = 0; j < kCols; ++j)
                    ck[j] += -alpha * beta * (sp[i][j] * gk[i] + G[i][j] * Sk[i]) + beta * G[i][j] * vv[i];
            // dv = beta g (lane 0 of each warp holds its rows' g)
            if (c == 0) {
                float* dvp = p.dv + (t * p.Hv + h) * kD + r * kRows;
#pragma unroll
                for (int i = 0; i < kRows; ++i) dvp[i] = beta * gk[i];
            }
            float (*cp)[kWarps][kD] = col_part[parity];
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                cp[0][r][c * kCols + j] = cq[j];
                cp[1][r][c * kCols + j] = ck[j];
            }
            if (c == 0) {
                scal_part[parity][r][0] = gs;
                scal_part[parity][r][1] = skg;
                scal_part[parity][r][2] = vg;
            }
            // dL/dS_{t-1} = alpha (G - beta g k^T)
#pragma unroll
            for (int i = 0; i < kRows; ++i)
#pragma unroll
                for (int j = 0; j < kCols; ++j) G[i][j] = alpha * (G[i][j] - beta * gk[i] * kv[j]);
            __syncthreads();
            // column sums: threads 0-127 dq, 128-255 dk (fixed order over warps)
            if (threadIdx.x < 2 * kD) {
                const int which = threadIdx.x / kD, e = threadIdx.x % kD;
                float acc = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) acc += cp[which][w][e];
                if (which == 0) p.dqh[(t * p.Hv + h) * kD + e] = p.scale * acc;
                else p.dkh[(t * p.Hv + h) * kD + e] = acc;
            } else if (threadIdx.x == 2 * kD) {
                float GS = 0.f, SKG = 0.f, VG = 0.f;
                for (int w = 0; w < kWarps; ++w) {
                    GS += scal_part[parity][w][0];
                    SKG += scal_part[parity][w][1];
                    VG += scal_part[parity][w][2];
                }
                const float dalpha = GS - beta * SKG;
                const float dbeta = -alpha * SKG + VG;
                const float dla = dalpha * alpha;
                const float x = p.a[t * p.Hv + h] + dtb;
                const float dat = dla * (-eA * sigmoid_f32(x));
                p.da[t * p.Hv + h] = dat;
                p.db[t * p.Hv + h] = dbeta * beta * (1.f - beta);
                ddt_acc += dat;
                dA_acc += dla * la;
            }
            parity ^= 1;
        }
    }
    if (threadIdx.x == 2 * kD) {
        p.gate_part[unit * 2 + 0] = dA_acc;
        p.gate_part[unit * 2 + 1] = ddt_acc;
    }
    if (p.d_init) gstore(p.d_init + unit * kStateFloats, r, c, G);
}

// dq[t, g] = sum over the value heads h of group g of dqh[t, h] (likewise dk),
// in head order; then dA_log, ddt_bias summed over sequences
__global__ void gdn_backward_reduce_kernel(const float* __restrict__ dqh, const float* __restrict__ dkh,
                                           int64_t T, int32_t Hqk, int32_t Hv, float* __restrict__ dq,
                                           float* __restrict__ dk) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // over T * Hqk * kD
    if (i >= T * Hqk * kD) return;
    const int e = (int)(i % kD);
    const int64_t tg = i / kD;
    const int gk = (int)(tg % Hqk);
    const int64_t t = tg / Hqk;
    const int grp = Hv / Hqk;
    float aq = 0.f, ak = 0.f;
    for (int j = 0; j < grp; ++j) {
        const int64_t src = (t * Hv + gk * grp + j) * kD + e;
        aq += dqh[src];
        ak += dkh[src];
    }
    dq[i] = aq;
    dk[i] = ak;
}

__global__ void gdn_backward_gates_kernel(const float* __restrict__ gate_part, int32_t n_seq, int32_t Hv,
                                          float* __restrict__ dA_log, float* __restrict__ ddt_bias) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= Hv) return;
    float s0 = 0.f, s1 = 0.f;
    for (int n = 0; n < n_seq; ++n) {
        s0 += gate_part[((size_t)n * Hv + h) * 2];
        s1 += gate_part[((size_t)n * Hv + h) * 2 + 1];
    }
    dA_log[h] = s0;
    ddt_bias[h] = s1;
}

}  // namespace

size_t backward_workspace_bytes(int32_t n_seq, int64_t T, int32_t Hv) {
    const size_t units = (size_t)n_seq * Hv;
    const size_t slots = (size_t)(T / kC) + (size_t)n_seq + 1;
    const size_t state = kStateFloats * sizeof(float);
    size_t bytes = 0;
    bytes += slots * Hv * state;                           // checkpoints
    bytes += units * kC * state;                           // per-chunk states
    bytes += 2 * (size_t)T * Hv * kD * sizeof(float);      // dq, dk per value head
    bytes += units * 2 * sizeof(float);                    // gate parameter sums
    return ((bytes + 255) / 256) * 256;
}

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t stream) {
    if (a.n_seq <= 0) return cudaSuccess;
    const size_t units = (size_t)a.n_seq * a.Hv;
    const size_t slots = (size_t)(a.T / kC) + (size_t)a.n_seq + 1;
    const size_t state = kStateFloats;
    float* ws = static_cast<float*>(a.workspace);
    BwdParams p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.a = a.a; p.b = a.b; p.A_log = a.A_log; p.dt_bias = a.dt_bias;
    p.cu = a.cu_seqlens; p.T = a.T; p.Hqk = a.Hqk; p.Hv = a.Hv; p.scale = a.scale;
    p.s0 = a.initial_state; p.d_o = a.d_o; p.d_fin = a.d_final_state;
    p.ckpt = ws;
    p.hist = p.ckpt + slots * a.Hv * state;
    p.dqh = p.hist + units * kC * state;
    p.dkh = p.dqh + (size_t)a.T * a.Hv * kD;
    p.gate_part = p.dkh + (size_t)a.T * a.Hv * kD;
    p.dv = a.dv; p.da = a.da; p.db = a.db; p.d_init = a.d_initial_state;
    if (units > 0x7fffffffULL) return cudaErrorInvalidValue;
    gdn_backward_kernel<<<(unsigned)units, kThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = a.T * a.Hqk * kD;
    if (n > 0) {
        gdn_backward_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(p.dqh, p.dkh, a.T, a.Hqk,
                                                                                    a.Hv, a.dq, a.dk);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    gdn_backward_gates_kernel<<<(unsigned)((a.Hv + 127) / 128), 128, 0, stream>>>(p.gate_part, a.n_seq, a.Hv,
                                                                                  a.dA_log, a.ddt_bias);
    return cudaGetLastError();
}

}  // namespace gdn
