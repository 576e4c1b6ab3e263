// prefill_simt.cu -- chunked gated delta-rule prefill on CUDA cores (float32).
//
// A plain, unpipelined kernel computing the same chunk algebra as the
// tensor-core kernel, used to bring up the host logic (varlen, states,
// partial chunks).  One CTA per (sequence, value head, 32-wide d_v slice)
// walks the sequence's chunks of C = 64 tokens in order.
//
// Per chunk, with G the running sum of log(alpha) inside the chunk, gamma =
// e^G, and masks j < i (A) and j <= i (P):
//   A_ij = beta_i e^{G_i - G_j} k_i.k_j          P_ij = e^{G_i - G_j} q_i.k_j
//   T    = (I + A)^{-1}  (forward substitution)
//   W    = T diag(beta gamma) K                   U'   = T diag(beta) V
//   Qh   = diag(gamma) Q - P W                    O'   = P U'
//   U    = U' - W S^T                             o    = scale (O' + Qh S^T)
//   S   <- gamma_C S + U^T diag(gamma_C / gamma) K
// which is the recurrence S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) +
// beta_t v_t k_t^T, o_t = scale S_t q_t, unrolled over the chunk (delta rule
// of the Qwen3.8-27B architecture page, 2kiu.com, section 2.2, with decay).
// Only differences G_i - G_j with i >= j and G itself (both <= 0) are
// exponentiated, so nothing overflows however strong the decay.
#include "common.cuh"
#include "kernels.h"

namespace gdn {

namespace {

constexpr int kD = 128;
constexpr int kC = 64;
constexpr int kBV = 32;          // d_v columns per CTA
constexpr int kThreads = 256;
constexpr int kLd = kD + 1;      // padded row of a [*, 128] float tile

struct SimtSmem {
    float K[kC][kLd];
    float Q[kC][kLd];            // Q, then Qh
    float W[kC][kLd];
    float S[kBV][kLd];           // state slice: rows = d_v, cols = d_k
    float A[kC][kC + 1];
    float P[kC][kC + 1];
    float Tm[kC][kC + 1];
    float V[kC][kBV + 1];
    float Up[kC][kBV + 1];       // U', then U
    float Op[kC][kBV + 1];       // O'
    float G[kC];
    float beta[kC];
};

__global__ void __launch_bounds__(kThreads)
prefill_simt_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                    const uint16_t* __restrict__ v, const float* __restrict__ a,
                    const float* __restrict__ b, const float* __restrict__ A_log,
                    const float* __restrict__ dt_bias, const int32_t* __restrict__ cu,
                    int64_t T, int32_t Hqk, int32_t Hv, float scale,
                    const float* __restrict__ s_in, float* __restrict__ s_out,
                    float* __restrict__ o) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int slices = kD / kBV;
    const int s = blockIdx.x % slices;
    const int h = (blockIdx.x / slices) % Hv;
    const int n = blockIdx.x / (slices * Hv);
    const int g = h / (Hv / Hqk);
    const int64_t bos = cu ? cu[n] : 0;
    const int64_t eos = cu ? cu[n + 1] : T;
    const float Al = A_log[h], dtb = dt_bias[h];

    // initial state slice
    for (int i = tid; i < kBV * kD; i += kThreads) {
        const int r = i / kD, c = i % kD;
        sm.S[r][c] = s_in ? s_in[(((int64_t)n * Hv + h) * kD + s * kBV + r) * kD + c] : 0.f;
    }

    for (int64_t c0 = bos; c0 < eos; c0 += kC) {
        const int L = (int)((eos - c0) < kC ? (eos - c0) : kC);
        __syncthreads();
        // ---- load the chunk (rows >= L are zero) and the gates
        for (int i = tid; i < kC * kD; i += kThreads) {
            const int t = i / kD, c = i % kD;
            float kv = 0.f, qv = 0.f;
            if (t < L) {
                kv = bf16_to_f32(k[((c0 + t) * Hqk + g) * kD + c]);
                qv = bf16_to_f32(q[((c0 + t) * Hqk + g) * kD + c]);
            }
            sm.K[t][c] = kv;
            sm.Q[t][c] = qv;
        }
        for (int i = tid; i < kC * kBV; i += kThreads) {
            const int t = i / kBV, c = i % kBV;
            sm.V[t][c] = t < L ? bf16_to_f32(v[((c0 + t) * Hv + h) * kD + s * kBV + c]) : 0.f;
        }
        if (tid < kC) {
            float lg = 0.f, be = 0.f;
            if (tid < L) {
                lg = log_alpha_f32(a[(c0 + tid) * Hv + h], Al, dtb);
                be = sigmoid_f32(b[(c0 + tid) * Hv + h]);
            }
            sm.G[tid] = lg;
            sm.beta[tid] = be;
        }
        __syncthreads();
        if (tid == 0) {
            float run = 0.f;
            for (int t = 0; t < kC; ++t) { run += sm.G[t]; sm.G[t] = run; }
        }
        __syncthreads();
        // ---- A and P
        for (int i = tid; i < kC * kC; i += kThreads) {
            const int r = i / kC, c = i % kC;
            float kk = 0.f, qk = 0.f;
            if (c <= r) {
                for (int e = 0; e < kD; ++e) {
                    kk = fmaf(sm.K[r][e], sm.K[c][e], kk);
                    qk = fmaf(sm.Q[r][e], sm.K[c][e], qk);
                }
            }
            const float dec = c <= r ? expf(sm.G[r] - sm.G[c]) : 0.f;
            sm.A[r][c] = c < r ? sm.beta[r] * dec * kk : 0.f;
            sm.P[r][c] = c <= r ? dec * qk : 0.f;
        }
        __syncthreads();
        // ---- T = (I + A)^{-1}, one row at a time
        for (int r = 0; r < kC; ++r) {
            if (tid < kC) {
                const int c = tid;
                float val = 0.f;
                if (c < r) {
                    for (int m = c; m < r; ++m) val = fmaf(-sm.A[r][m], sm.Tm[m][c], val);
                } else if (c == r) {
                    val = 1.f;
                }
                sm.Tm[r][c] = val;
            }
            __syncthreads();
        }
        // ---- W = T diag(beta gamma) K ; U' = T diag(beta) V
        for (int i = tid; i < kC * kD; i += kThreads) {
            const int r = i / kD, c = i % kD;
            float acc = 0.f;
            for (int j = 0; j <= r; ++j)
                acc = fmaf(sm.Tm[r][j] * sm.beta[j] * expf(sm.G[j]), sm.K[j][c], acc);
            sm.W[r][c] = acc;
        }
        for (int i = tid; i < kC * kBV; i += kThreads) {
            const int r = i / kBV, c = i % kBV;
            float acc = 0.f;
            for (int j = 0; j <= r; ++j) acc = fmaf(sm.Tm[r][j] * sm.beta[j], sm.V[j][c], acc);
            sm.Up[r][c] = acc;
        }
        __syncthreads();
        // ---- Qh = diag(gamma) Q - P W  (in place) ; O' = P U'
        for (int i = tid; i < kC * kD; i += kThreads) {
            const int r = i / kD, c = i % kD;
            float acc = expf(sm.G[r]) * sm.Q[r][c];
            for (int j = 0; j <= r; ++j) acc = fmaf(-sm.P[r][j], sm.W[j][c], acc);
            sm.Q[r][c] = acc;
        }
        for (int i = tid; i < kC * kBV; i += kThreads) {
            const int r = i / kBV, c = i % kBV;
            float acc = 0.f;
            for (int j = 0; j <= r; ++j) acc = fmaf(sm.P[r][j], sm.Up[j][c], acc);
            sm.Op[r][c] = acc;
        }
        __syncthreads();
        // ---- U = U' - W S^T ; o = scale (O' + Qh S^T)
        for (int i = tid; i < kC * kBV; i += kThreads) {
            const int r = i / kBV, c = i % kBV;
            float ws = 0.f, qs = 0.f;
            for (int e = 0; e < kD; ++e) {
                ws = fmaf(sm.W[r][e], sm.S[c][e], ws);
                qs = fmaf(sm.Q[r][e], sm.S[c][e], qs);
            }
            sm.Up[r][c] -= ws;
            if (r < L) o[((c0 + r) * Hv + h) * kD + s * kBV + c] = scale * (sm.Op[r][c] + qs);
        }
        __syncthreads();
        // ---- S <- gamma_C S + U^T diag(gamma_C / gamma) K
        const float GC = sm.G[kC - 1];
        for (int i = tid; i < kBV * kD; i += kThreads) {
            const int r = i / kD, c = i % kD;
            float acc = expf(GC) * sm.S[r][c];
            for (int j = 0; j < kC; ++j) acc = fmaf(sm.Up[j][r] * expf(GC - sm.G[j]), sm.K[j][c], acc);
            sm.S[r][c] = acc;
        }
    }
    __syncthreads();
    if (s_out) {
        for (int i = tid; i < kBV * kD; i += kThreads) {
            const int r = i / kD, c = i % kD;
            s_out[(((int64_t)n * Hv + h) * kD + s * kBV + r) * kD + c] = sm.S[r][c];
        }
    }
}

}  // namespace

size_t prefill_simt_smem_bytes() { return sizeof(SimtSmem); }

cudaError_t launch_prefill_simt(const PrefillArgs& p, cudaStream_t stream) {
    const size_t smem = sizeof(SimtSmem);
    cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (int64_t)p.n_seq * p.Hv * (kD / kBV);
    if (blocks == 0) return cudaSuccess;
    prefill_simt_kernel<<<(unsigned)blocks, kThreads, smem, stream>>>(
        p.q, p.k, p.v, p.a, p.b, p.A_log, p.dt_bias, p.cu_seqlens, p.T, p.Hqk, p.Hv, p.scale,
        p.initial_state, p.final_state, p.o);
    return cudaGetLastError();
}

}  // namespace gdn
