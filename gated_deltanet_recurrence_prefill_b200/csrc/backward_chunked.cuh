// backward_chunked.cuh -- the gradient of the gated delta rule taken through its
// chunked (WY / UT) form, on CUDA cores in float32.
//
// The forward recurrence is the one of gdn_prefill (Qwen3.8-27B architecture
// page, 2kiu.com, section 2.2, with the decay alpha on the erased state).  In a
// chunk of L <= 64 tokens with start state S (d_v x d_k), G_i the running sum of
// log alpha in the chunk, gam_i = e^{G_i}, Gam_ij = e^{G_i - G_j},
// kap_j = e^{G_{L-1} - G_j}:
//     A' = strict_lower(Gam o K K^T),  T = (I + diag(beta) A')^{-1},
//     W = T diag(beta gam) K,  U' = T diag(beta) V,  U = U' - W S^T,
//     P = lower(Gam o Q K^T),  O = scale (diag(gam) Q S^T + P U),
//     S_end = gam_{L-1} S + U^T diag(kap) K.
// Reverse mode through these, chunk by chunk, leaves two chains over chunks and
// everything else local to a chunk:
//   * forward chain: the chunk-start states S_c;
//   * backward chain: the gradient at each chunk's end, dS_c, with
//         dS_{c-1} = gam_{L-1} dS_c - (diag(kap) K dS_c^T)^T W + Y_c,
//         Y_c = scale (dO^T diag(gam) Q - (P^T dO)^T W)   (no state in it);
//   * per chunk, given S_c and dS_c: dq, dk, dv, d beta and the decays.
// Both chains act on the rows of the state one at a time (row e of S_end
// depends on row e of S only, and likewise for dS), so each (sequence, value
// head) chain is split over kRowSplit CTAs.
//
// The work is written as block functions: one CTA's part of one job, given its
// thread index and its shared memory.  The CUDA kernels of
// backward_chunked.cu call them with threadIdx.x and dynamic shared memory;
// the CPU tests run the same source with one host thread per CUDA thread.
// Threads exchange data only through shared memory between block-wide
// barriers (BWC_SYNC): no warp shuffles, no atomics, so every sum is taken in
// a fixed order and the result is deterministic.
#pragma once

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
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
#ifndef BWC_MISALIGNED
#define BWC_MISALIGNED(ptr) abort()
#endif

namespace gdn {
namespace bwc {

constexpr int kC = 64;                   // chunk length
constexpr int kD = 128;                  // d_k = d_v
constexpr int kThreads = 256;            // every block function runs on 256 threads
constexpr int kRowSplit = 4;             // chain CTAs per (sequence, value head)
constexpr int kRows = kD / kRowSplit;    // state rows per chain CTA
constexpr int kEB = 16;                  // v columns per step of the gradient kernel
constexpr int kLd = kD + 1;              // padded row strides of shared-memory matrices
constexpr int kLc = kC + 1;               // (scalar access: consecutive rows on different banks)
constexpr int kLe = kEB + 1;
constexpr int kL4 = kD + 4;              // row strides for float4 access (16-byte rows)
constexpr int kLt = kC + 4;
constexpr int kLu = kRows + 4;

// ---- workspace plan ----------------------------------------------------------------
// A 256-byte header holding the error word (uint32 at offset 0, 0 = ok: the
// tensor-core gradient kernel sets it when a bounded wait gives up).
// Per (chunk slot, value head): W, U' [64 x 128], T [64 x 64], Y, S_c, dS_c
// [128 x 128], kap and gam_{L-1} [65]; per token and value head: dq, dk before
// the sum over each key head's value heads; per (slot, head) two gate sums.
// A chunk of sequence n starting at token t0 has slot t0 / 64 + n (unique; at
// most T / 64 + n_seq + 1 slots).
struct Plan {
    int64_t n_slots;
    size_t err, jobs, W, Up, T, Y, S, dS, G, dqh, dkh, gpart, bytes;
};

BWC_HD size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

BWC_HD Plan make_plan(int32_t n_seq, int64_t T, int32_t Hv) {
    Plan p;
    p.n_slots = T / kC + n_seq + 1;
    const size_t sh = (size_t)p.n_slots * Hv;
    size_t off = 0;
    p.err = off;  off = 256;
    p.jobs = off; off = align256(off + (size_t)p.n_slots * 2 * sizeof(int32_t));
    p.W = off;    off = align256(off + sh * kC * kD * sizeof(float));
    p.Up = off;   off = align256(off + sh * kC * kD * sizeof(float));
    p.T = off;    off = align256(off + sh * kC * kC * sizeof(float));
    p.Y = off;    off = align256(off + sh * kD * kD * sizeof(float));
    p.S = off;    off = align256(off + sh * kD * kD * sizeof(float));
    p.dS = off;   off = align256(off + sh * kD * kD * sizeof(float));
    p.G = off;    off = align256(off + sh * (kC + 1) * sizeof(float));
    p.dqh = off;  off = align256(off + (size_t)T * Hv * kD * sizeof(float));
    p.dkh = off;  off = align256(off + (size_t)T * Hv * kD * sizeof(float));
    p.gpart = off; off = align256(off + sh * 2 * sizeof(float));
    p.bytes = off;
    return p;
}

struct Params {
    // inputs (layouts as for gdn_prefill_backward)
    const uint16_t* q;          // [T, Hqk, 128] bf16
    const uint16_t* k;          // [T, Hqk, 128] bf16
    const uint16_t* v;          // [T, Hv, 128] bf16
    const float* a;             // [T, Hv]
    const float* b;             // [T, Hv]
    const float* A_log;         // [Hv]
    const float* dt_bias;       // [Hv]
    const int32_t* cu;          // [n_seq + 1] or null (one sequence)
    const float* s0;            // [n_seq, Hv, 128, 128] or null
    const float* d_o;           // [T, Hv, 128]
    const float* d_fin;         // [n_seq, Hv, 128, 128] or null
    int32_t n_seq, Hqk, Hv;
    int64_t T, n_slots;
    float scale;
    // workspace (see Plan)
    uint32_t* err;              // error word (0 = ok)
    int32_t* jobs;              // per slot: sequence (-1: unused) and first token
    float *W, *Up, *Tm, *Y, *S, *dS, *G, *dqh, *dkh, *gpart;
    // outputs
    float *dq, *dk, *dv, *da, *db, *dA_log, *ddt_bias, *d_init;
};

// Point the workspace fields of p at their regions of ws (laid out by plan).
BWC_HD void bind_workspace(Params& p, void* ws, const Plan& plan) {
    char* base = static_cast<char*>(ws);
    p.n_slots = plan.n_slots;
    p.err = reinterpret_cast<uint32_t*>(base + plan.err);
    p.jobs = reinterpret_cast<int32_t*>(base + plan.jobs);
    p.W = reinterpret_cast<float*>(base + plan.W);
    p.Up = reinterpret_cast<float*>(base + plan.Up);
    p.Tm = reinterpret_cast<float*>(base + plan.T);
    p.Y = reinterpret_cast<float*>(base + plan.Y);
    p.S = reinterpret_cast<float*>(base + plan.S);
    p.dS = reinterpret_cast<float*>(base + plan.dS);
    p.G = reinterpret_cast<float*>(base + plan.G);
    p.dqh = reinterpret_cast<float*>(base + plan.dqh);
    p.dkh = reinterpret_cast<float*>(base + plan.dkh);
    p.gpart = reinterpret_cast<float*>(base + plan.gpart);
}

// Shared-memory floats each block function needs.
constexpr int kPrepFloats = 5 * kC * kLd + 3 * kC * kLc + 5 * kC;
constexpr int kFwdChainFloats = 2 * kC * kL4 + kRows * kLd + kC * kLu + kC + 4;
constexpr int kBwdChainFloats = kC * kL4 + kD * kLt + kRows * kLd + kRows * kLt + kC + 4;
constexpr int kChainFloats = kFwdChainFloats > kBwdChainFloats ? kFwdChainFloats : kBwdChainFloats;
constexpr int kGradFloats = 3 * kC * kLd + 5 * kC * kLc + 2 * kEB * kLd + 6 * kC * kLe + 9 * kC + kThreads;

// ---- small helpers ----------------------------------------------------------------------
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

// four consecutive floats from a 16-byte aligned address (the host build checks
// the alignment, so that the CPU tests catch a misaligned vector access)
struct F4 {
    float v[4];
};
BWC_FN F4 ld4(const float* ptr) {
    F4 r;
#ifdef __CUDA_ARCH__
    const float4 x = *reinterpret_cast<const float4*>(ptr);
    r.v[0] = x.x; r.v[1] = x.y; r.v[2] = x.z; r.v[3] = x.w;
#else
    if (reinterpret_cast<uintptr_t>(ptr) & 15u) BWC_MISALIGNED(ptr);
    memcpy(r.v, ptr, sizeof r.v);
#endif
    return r;
}

// softplus(x) = log(1 + e^x) without overflow; log alpha and beta as in the forward
BWC_FN float softplus(float x) { return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x)); }
BWC_FN float log_alpha(float a, float A_log, float dt_bias) { return -expf(A_log) * softplus(a + dt_bias); }
BWC_FN float sigmoid(float x) { return 1.f / (1.f + expf(-x)); }

BWC_FN void seq_bounds(const Params& p, int n, int64_t& bos, int64_t& eos) {
    bos = p.cu ? p.cu[n] : 0;
    eos = p.cu ? p.cu[n + 1] : p.T;
}

BWC_FN size_t sh_index(const Params& p, int64_t slot, int h) { return (size_t)slot * p.Hv + h; }

// Gates of the chunk at t0 (L tokens) for value head h into lg (log alpha),
// be (beta), G (running sum), gam, kap; rows >= L get lg = be = kap = 0 and
// G = G_{L-1}.  Ends with a barrier.
BWC_FN void chunk_gates(const Params& p, int h, int64_t t0, int L, int tid, float* lg, float* be, float* G,
                        float* gam, float* kap) {
    if (tid < kC) {
        const int i = tid;
        float la = 0.f, bb = 0.f;
        if (i < L) {
            const int64_t t = t0 + i;
            la = log_alpha(p.a[t * p.Hv + h], p.A_log[h], p.dt_bias[h]);
            bb = sigmoid(p.b[t * p.Hv + h]);
        }
        lg[i] = la;
        be[i] = bb;
    }
    BWC_SYNC();
    if (tid == 0) {
        float run = 0.f;
        for (int i = 0; i < kC; ++i) {
            run += lg[i];
            G[i] = run;
        }
    }
    BWC_SYNC();
    if (tid < kC) {
        const int i = tid;
        gam[i] = expf(G[i]);
        kap[i] = i < L ? expf(G[L - 1] - G[i]) : 0.f;
    }
    BWC_SYNC();
}

// Rows t0 .. t0 + 63 of a bf16 [T, H, 128] tensor (head hh) into a [64][ld]
// float matrix; rows >= L are zero.
BWC_FN void load_rows_bf16(const uint16_t* x, int H, int hh, int64_t t0, int L, int tid, float* dst,
                           int ld = kLd) {
    for (int idx = tid; idx < kC * kD; idx += kThreads) {
        const int i = idx >> 7, e = idx & (kD - 1);
        dst[i * ld + e] = i < L ? bf16f(x[((t0 + i) * H + hh) * kD + e]) : 0.f;
    }
}

// A' = strict_lower(Gam o K K^T) and P = lower(Gam o Q K^T), rows and columns
// >= L zero.  K and Q are [64][kLd]; A' and P [64][kLc].  Thread tid takes rows
// tid / 16 + 16 x and columns tid % 16 + 16 y (x, y < 4).
BWC_FN void build_ap(const float* Ks, const float* Qs, const float* G, int L, int tid, float* Ap, float* Pm) {
    const int ib = tid >> 4, jb = tid & 15;
    float kk[4][4], qk[4][4];
    for (int x = 0; x < 4; ++x)
        for (int y = 0; y < 4; ++y) kk[x][y] = qk[x][y] = 0.f;
    for (int f = 0; f < kD; ++f) {
        float ki[4], qi[4], kj[4];
        for (int x = 0; x < 4; ++x) {
            ki[x] = Ks[(ib + 16 * x) * kLd + f];
            qi[x] = Qs[(ib + 16 * x) * kLd + f];
            kj[x] = Ks[(jb + 16 * x) * kLd + f];
        }
        for (int x = 0; x < 4; ++x)
            for (int y = 0; y < 4; ++y) {
                kk[x][y] = fmaf(ki[x], kj[y], kk[x][y]);
                qk[x][y] = fmaf(qi[x], kj[y], qk[x][y]);
            }
    }
    for (int x = 0; x < 4; ++x)
        for (int y = 0; y < 4; ++y) {
            const int i = ib + 16 * x, j = jb + 16 * y;
            const float gm = (j <= i && i < L) ? expf(G[i] - G[j]) : 0.f;
            Ap[i * kLc + j] = j < i ? gm * kk[x][y] : 0.f;
            Pm[i * kLc + j] = j <= i ? gm * qk[x][y] : 0.f;
        }
}

// ---- chunk list --------------------------------------------------------------------------
// For sequence n: jobs[2 slot] = n, jobs[2 slot + 1] = first token of the chunk.
// (The host sets every entry to -1 first.)
BWC_FN void fill_jobs(const Params& p, int n, int tid) {
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int64_t nch = (eos - bos + kC - 1) / kC;
    for (int64_t j = tid; j < nch; j += kThreads) {
        const int64_t t0 = bos + j * kC;
        const int64_t slot = t0 / kC + n;
        p.jobs[2 * slot] = n;
        p.jobs[2 * slot + 1] = (int32_t)t0;
    }
}

// ---- prep: per (chunk, value head) -------------------------------------------------------
// T, W, U', kap, gam_{L-1} and Y_c of one chunk.
BWC_FN void prep_block(const Params& p, int64_t slot, int h, int tid, float* sm) {
    const int n = p.jobs[2 * slot];
    const size_t sh = sh_index(p, slot, h);
    if (n < 0) {
        if (tid < 2) p.gpart[sh * 2 + tid] = 0.f;
        return;
    }
    const int64_t t0 = p.jobs[2 * slot + 1];
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int L = (int)((eos - t0) < kC ? (eos - t0) : kC);
    const int g = h / (p.Hv / p.Hqk);

    float* Ks = sm;
    float* Qs = Ks + kC * kLd;
    float* Vs = Qs + kC * kLd;       // V, then dO
    float* Ws = Vs + kC * kLd;
    float* Zs = Ws + kC * kLd;       // P^T dO
    float* Ap = Zs + kC * kLd;
    float* Tm = Ap + kC * kLc;
    float* Pm = Tm + kC * kLc;
    float* lg = Pm + kC * kLc;
    float* be = lg + kC;
    float* G = be + kC;
    float* gam = G + kC;
    float* kap = gam + kC;

    load_rows_bf16(p.k, p.Hqk, g, t0, L, tid, Ks);
    load_rows_bf16(p.q, p.Hqk, g, t0, L, tid, Qs);
    load_rows_bf16(p.v, p.Hv, h, t0, L, tid, Vs);
    chunk_gates(p, h, t0, L, tid, lg, be, G, gam, kap);
    build_ap(Ks, Qs, G, L, tid, Ap, Pm);
    BWC_SYNC();
    // T = (I + diag(beta) A')^{-1} by forward substitution, one column per thread
    if (tid < kC) {
        const int j = tid;
        for (int i = 0; i < kC; ++i) {
            float val;
            if (i < j) {
                val = 0.f;
            } else if (i == j) {
                val = 1.f;
            } else {
                float acc = 0.f;
                for (int m = j; m < i; ++m) acc = fmaf(Ap[i * kLc + m], Tm[m * kLc + j], acc);
                val = -be[i] * acc;
            }
            Tm[i * kLc + j] = val;
        }
    }
    BWC_SYNC();
    // U' = T diag(beta) V and W = T diag(beta gam) K: thread tid takes rows
    // 4 (tid / 16) .. + 4 and columns tid % 16 + 16 c (c < 8)
    float* Wg = p.W + sh * kC * kD;
    float* Ug = p.Up + sh * kC * kD;
    {
        const int i4 = (tid >> 4) * 4, eb = tid & 15;
        float up[4][8], w[4][8];
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 8; ++c) up[r][c] = w[r][c] = 0.f;
        for (int m = 0; m <= i4 + 3; ++m) {     // T is lower triangular (zeros above)
            float tb[4], vv[8], kv[8];
            for (int r = 0; r < 4; ++r) tb[r] = Tm[(i4 + r) * kLc + m] * be[m];
            for (int c = 0; c < 8; ++c) {
                vv[c] = Vs[m * kLd + eb + 16 * c];
                kv[c] = gam[m] * Ks[m * kLd + eb + 16 * c];
            }
            for (int r = 0; r < 4; ++r)
                for (int c = 0; c < 8; ++c) {
                    up[r][c] = fmaf(tb[r], vv[c], up[r][c]);
                    w[r][c] = fmaf(tb[r], kv[c], w[r][c]);
                }
        }
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 8; ++c) {
                const int i = i4 + r, e = eb + 16 * c;
                Ug[i * kD + e] = up[r][c];
                Wg[i * kD + e] = w[r][c];
                Ws[i * kLd + e] = w[r][c];
            }
    }
    float* Tg = p.Tm + sh * kC * kC;
    for (int idx = tid; idx < kC * kC; idx += kThreads) Tg[idx] = Tm[(idx >> 6) * kLc + (idx & (kC - 1))];
    float* Gg = p.G + sh * (kC + 1);
    if (tid < kC) Gg[tid] = kap[tid];
    if (tid == 0) Gg[kC] = gam[L - 1];
    BWC_SYNC();
    // dO over V
    for (int idx = tid; idx < kC * kD; idx += kThreads) {
        const int i = idx >> 7, e = idx & (kD - 1);
        Vs[i * kLd + e] = i < L ? p.d_o[((t0 + i) * p.Hv + h) * kD + e] : 0.f;
    }
    BWC_SYNC();
    // Z = P^T dO: thread tid takes rows 4 (tid / 16) .. + 4, columns tid % 16 + 16 c
    {
        const int j4 = (tid >> 4) * 4, eb = tid & 15;
        float z[4][8];
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 8; ++c) z[r][c] = 0.f;
        for (int i = j4; i < L; ++i) {          // P is lower triangular (zeros above)
            float pv[4], dv[8];
            for (int r = 0; r < 4; ++r) pv[r] = Pm[i * kLc + j4 + r];
            for (int c = 0; c < 8; ++c) dv[c] = Vs[i * kLd + eb + 16 * c];
            for (int r = 0; r < 4; ++r)
                for (int c = 0; c < 8; ++c) z[r][c] = fmaf(pv[r], dv[c], z[r][c]);
        }
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 8; ++c) Zs[(j4 + r) * kLd + eb + 16 * c] = z[r][c];
    }
    BWC_SYNC();
    // Y = scale (dO^T diag(gam) Q - Z^T W): thread tid takes rows tid / 16 + 16 x
    // and columns tid % 16 + 16 c (x, c < 8)
    float* Yg = p.Y + sh * kD * kD;
    {
        const int eb = tid >> 4, fb = tid & 15;
        float y[8][8];
        for (int x = 0; x < 8; ++x)
            for (int c = 0; c < 8; ++c) y[x][c] = 0.f;
        for (int i = 0; i < L; ++i) {
            float dg[8], zv[8], qv[8], wv[8];
            for (int x = 0; x < 8; ++x) {
                dg[x] = gam[i] * Vs[i * kLd + eb + 16 * x];
                zv[x] = Zs[i * kLd + eb + 16 * x];
            }
            for (int c = 0; c < 8; ++c) {
                qv[c] = Qs[i * kLd + fb + 16 * c];
                wv[c] = Ws[i * kLd + fb + 16 * c];
            }
            for (int x = 0; x < 8; ++x)
                for (int c = 0; c < 8; ++c) y[x][c] = fmaf(dg[x], qv[c], fmaf(-zv[x], wv[c], y[x][c]));
        }
        for (int x = 0; x < 8; ++x)
            for (int c = 0; c < 8; ++c) Yg[(size_t)(eb + 16 * x) * kD + fb + 16 * c] = p.scale * y[x][c];
    }
}

// ---- the chains: per (sequence, value head, quarter of the state rows) -----------------
// Thread tid owns rows 4 (tid / 32) .. + 4 of the CTA's 32 state rows and
// columns 4 (tid % 32) .. + 4.

// Forward: S_c for every chunk of sequence n into the workspace.
BWC_FN void fwd_chain_block(const Params& p, int n, int h, int rq, int tid, float* sm) {
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int g = h / (p.Hv / p.Hqk);
    const int r0 = rq * kRows;
    const int w4 = (tid >> 5) * 4, l4 = (tid & 31) * 4;     // my 4 x 4 block of the state rows
    const int i2 = (tid >> 3) * 2, e4 = (tid & 7) * 4;      // my 2 x 4 block of U [64 x 32]
    float* Ws = sm;                            // W             [kC][kL4]
    float* Ks = Ws + kC * kL4;                 // K             [kC][kL4]
    float* Ss = Ks + kC * kL4;                 // my rows of S  [kRows][kLd]
    float* Us = Ss + kRows * kLd;              // U', then kap U for my rows  [kC][kLu]
    float* kap = Us + kC * kLu;
    float* gl = kap + kC;
    float s[4][4];
    const size_t unit = ((size_t)n * p.Hv + h) * kD * kD + (size_t)(r0 + w4) * kD + l4;
    for (int r = 0; r < 4; ++r)
        for (int c = 0; c < 4; ++c) s[r][c] = p.s0 ? p.s0[unit + (size_t)r * kD + c] : 0.f;
    const int64_t nch = (eos - bos + kC - 1) / kC;
    for (int64_t j = 0; j < nch; ++j) {
        const int64_t t0 = bos + j * kC;
        const int L = (int)((eos - t0) < kC ? (eos - t0) : kC);
        const size_t sh = sh_index(p, t0 / kC + n, h);
        float* Sg = p.S + sh * kD * kD + (size_t)(r0 + w4) * kD + l4;
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 4; ++c) {
                Sg[(size_t)r * kD + c] = s[r][c];
                Ss[(w4 + r) * kLd + l4 + c] = s[r][c];
            }
        const float* Wg = p.W + sh * kC * kD;
        const float* Ug = p.Up + sh * kC * kD;
        for (int idx = tid; idx < kC * kD; idx += kThreads) Ws[(idx >> 7) * kL4 + (idx & (kD - 1))] = Wg[idx];
        load_rows_bf16(p.k, p.Hqk, g, t0, L, tid, Ks, kL4);
        for (int idx = tid; idx < kC * kRows; idx += kThreads) {
            const int i = idx / kRows, e = idx % kRows;
            Us[i * kLu + e] = Ug[(size_t)i * kD + r0 + e];
        }
        if (tid < kC) kap[tid] = p.G[sh * (kC + 1) + tid];
        if (tid == 0) gl[0] = p.G[sh * (kC + 1) + kC];
        BWC_SYNC();
        // kap_i (U'_ie - sum_f W_if S_ef) for rows i2, i2 + 1 and my rows e4 .. e4 + 3
        {
            float u[2][4];
            for (int a = 0; a < 2; ++a)
                for (int x = 0; x < 4; ++x) u[a][x] = Us[(i2 + a) * kLu + e4 + x];
            for (int f = 0; f < kD; ++f) {
                const float w0 = Ws[i2 * kL4 + f], w1 = Ws[(i2 + 1) * kL4 + f];
                for (int x = 0; x < 4; ++x) {
                    const float sv = Ss[(e4 + x) * kLd + f];
                    u[0][x] = fmaf(-w0, sv, u[0][x]);
                    u[1][x] = fmaf(-w1, sv, u[1][x]);
                }
            }
            for (int a = 0; a < 2; ++a)
                for (int x = 0; x < 4; ++x) Us[(i2 + a) * kLu + e4 + x] = kap[i2 + a] * u[a][x];
        }
        BWC_SYNC();
        const float gL = gl[0];
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 4; ++c) s[r][c] *= gL;
        for (int i = 0; i < L; ++i) {
            const F4 u = ld4(Us + i * kLu + w4), kv = ld4(Ks + i * kL4 + l4);
            for (int r = 0; r < 4; ++r)
                for (int c = 0; c < 4; ++c) s[r][c] = fmaf(u.v[r], kv.v[c], s[r][c]);
        }
        BWC_SYNC();
    }
}

// Backward: dS_c (the gradient at each chunk's end) for every chunk of sequence
// n, from the last chunk; the gradient at the sequence start into d_init.
BWC_FN void bwd_chain_block(const Params& p, int n, int h, int rq, int tid, float* sm) {
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int g = h / (p.Hv / p.Hqk);
    const int r0 = rq * kRows;
    const int w4 = (tid >> 5) * 4, l4 = (tid & 31) * 4;     // my 4 x 4 block of the state rows
    const int e2 = (tid >> 4) * 2, i4 = (tid & 15) * 4;     // my 2 x 4 block of X [32 x 64]
    float* Ws = sm;                            // W              [kC][kL4]
    float* KT = Ws + kC * kL4;                 // K transposed   [kD][kLt]
    float* Ss = KT + kD * kLt;                 // my rows of dS  [kRows][kLd]
    float* Xs = Ss + kRows * kLd;              // kap_i (dS K^T)_{e,i}  [kRows][kLt]
    float* kap = Xs + kRows * kLt;
    float* gl = kap + kC;
    float s[4][4];
    const size_t unit = ((size_t)n * p.Hv + h) * kD * kD + (size_t)(r0 + w4) * kD + l4;
    for (int r = 0; r < 4; ++r)
        for (int c = 0; c < 4; ++c) s[r][c] = p.d_fin ? p.d_fin[unit + (size_t)r * kD + c] : 0.f;
    const int64_t nch = (eos - bos + kC - 1) / kC;
    for (int64_t j = nch - 1; j >= 0; --j) {
        const int64_t t0 = bos + j * kC;
        const int L = (int)((eos - t0) < kC ? (eos - t0) : kC);
        const size_t sh = sh_index(p, t0 / kC + n, h);
        float* dSg = p.dS + sh * kD * kD + (size_t)(r0 + w4) * kD + l4;
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 4; ++c) {
                dSg[(size_t)r * kD + c] = s[r][c];
                Ss[(w4 + r) * kLd + l4 + c] = s[r][c];
            }
        const float* Wg = p.W + sh * kC * kD;
        for (int idx = tid; idx < kC * kD; idx += kThreads) Ws[(idx >> 7) * kL4 + (idx & (kD - 1))] = Wg[idx];
        for (int idx = tid; idx < kC * kD; idx += kThreads) {
            const int i = idx >> 7, f = idx & (kD - 1);
            KT[f * kLt + i] = i < L ? bf16f(p.k[((t0 + i) * p.Hqk + g) * kD + f]) : 0.f;
        }
        if (tid < kC) kap[tid] = p.G[sh * (kC + 1) + tid];
        if (tid == 0) gl[0] = p.G[sh * (kC + 1) + kC];
        BWC_SYNC();
        {
            float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            for (int f = 0; f < kD; ++f) {
                const float d0 = Ss[e2 * kLd + f], d1 = Ss[(e2 + 1) * kLd + f];
                const F4 kv = ld4(KT + f * kLt + i4);
                for (int c = 0; c < 4; ++c) {
                    x[0][c] = fmaf(d0, kv.v[c], x[0][c]);
                    x[1][c] = fmaf(d1, kv.v[c], x[1][c]);
                }
            }
            for (int a = 0; a < 2; ++a)
                for (int c = 0; c < 4; ++c) Xs[(e2 + a) * kLt + i4 + c] = kap[i4 + c] * x[a][c];
        }
        BWC_SYNC();
        const float gL = gl[0];
        const float* Yg = p.Y + sh * kD * kD + (size_t)(r0 + w4) * kD + l4;
        for (int r = 0; r < 4; ++r) {
            const F4 y = ld4(Yg + (size_t)r * kD);
            for (int c = 0; c < 4; ++c) s[r][c] = fmaf(gL, s[r][c], y.v[c]);
        }
        for (int i = 0; i < L; ++i) {
            const F4 wv = ld4(Ws + i * kL4 + l4);
            float xv[4];
            for (int r = 0; r < 4; ++r) xv[r] = Xs[(w4 + r) * kLt + i];
            for (int r = 0; r < 4; ++r)
                for (int c = 0; c < 4; ++c) s[r][c] = fmaf(-xv[r], wv.v[c], s[r][c]);
        }
        BWC_SYNC();
    }
    if (p.d_init)
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 4; ++c) p.d_init[unit + (size_t)r * kD + c] = s[r][c];
}

// ---- gradients of one (chunk, value head) -------------------------------------------------
// Thread tid owns rows 8 (tid / 32) .. + 8 and columns 4 (tid % 32) .. + 4 of
// the 64 x 128 accumulators (dq, dk, dW), and rows 4 (tid / 16) .. + 4, columns
// 4 (tid % 16) .. + 4 of the 64 x 64 ones (dP, dT).
BWC_FN void grad_block(const Params& p, int64_t slot, int h, int tid, float* sm) {
    const int n = p.jobs[2 * slot];
    if (n < 0) return;
    const int64_t t0 = p.jobs[2 * slot + 1];
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int L = (int)((eos - t0) < kC ? (eos - t0) : kC);
    const int g = h / (p.Hv / p.Hqk);
    const size_t sh = sh_index(p, slot, h);

    float* Ks = sm;
    float* Qs = Ks + kC * kLd;
    float* Ws = Qs + kC * kLd;      // W; after the v loop dW
    float* Pm = Ws + kC * kLd;
    float* Ap = Pm + kC * kLc;
    float* Tm = Ap + kC * kLc;
    float* M1 = Tm + kC * kLc;
    float* M2 = M1 + kC * kLc;
    float* Sb = M2 + kC * kLc;      // S rows e0 .. e0 + 15     [kEB][kLd]
    float* dSb = Sb + kEB * kLd;    // dS_c rows e0 .. e0 + 15  [kEB][kLd]
    float* Ub = dSb + kEB * kLd;    // U' then U, columns e0 .. [kC][kLe]
    float* dUb = Ub + kC * kLe;
    float* dOb = dUb + kC * kLe;
    float* Vb = dOb + kC * kLe;
    float* R1 = Vb + kC * kLe;
    float* R2 = R1 + kC * kLe;
    float* lg = R2 + kC * kLe;
    float* be = lg + kC;
    float* G = be + kC;
    float* gam = G + kC;
    float* kap = gam + kC;
    float* dgam = kap + kC;
    float* dkap = dgam + kC;
    float* dbe = dkap + kC;
    float* dGv = dbe + kC;
    float* part = dGv + kC;         // [kThreads]
    float* SK = Sb;                 // after the v loop: [kC][33] row-sum partials

    load_rows_bf16(p.k, p.Hqk, g, t0, L, tid, Ks);
    load_rows_bf16(p.q, p.Hqk, g, t0, L, tid, Qs);
    {
        const float* Wg = p.W + sh * kC * kD;
        for (int idx = tid; idx < kC * kD; idx += kThreads) Ws[(idx >> 7) * kLd + (idx & (kD - 1))] = Wg[idx];
        const float* Tg = p.Tm + sh * kC * kC;
        for (int idx = tid; idx < kC * kC; idx += kThreads) Tm[(idx >> 6) * kLc + (idx & (kC - 1))] = Tg[idx];
    }
    if (tid < kC) {
        dgam[tid] = 0.f;
        dkap[tid] = 0.f;
        dbe[tid] = 0.f;
    }
    chunk_gates(p, h, t0, L, tid, lg, be, G, gam, kap);
    build_ap(Ks, Qs, G, L, tid, Ap, Pm);

    const int w8 = (tid >> 5) * 8, l4 = (tid & 31) * 4;     // 64 x 128 block
    const int r4 = (tid >> 4) * 4, c4 = (tid & 15) * 4;     // 64 x 64 block
    float dQa[8][4], dKa[8][4], dWa[8][4], dPa[4][4], dTa[4][4];
    for (int r = 0; r < 8; ++r)
        for (int c = 0; c < 4; ++c) dQa[r][c] = dKa[r][c] = dWa[r][c] = 0.f;
    for (int r = 0; r < 4; ++r)
        for (int c = 0; c < 4; ++c) dPa[r][c] = dTa[r][c] = 0.f;
    float ss = 0.f;                                          // this thread's part of <dS_c, S_c>
    const float* Sg = p.S + sh * kD * kD;
    const float* dSg = p.dS + sh * kD * kD;
    BWC_SYNC();

    for (int e0 = 0; e0 < kD; e0 += kEB) {
        // ---- this block of v columns
        for (int idx = tid; idx < kEB * kD; idx += kThreads) {
            const int e = idx >> 7, f = idx & (kD - 1);
            const float sv = Sg[(size_t)(e0 + e) * kD + f], dsv = dSg[(size_t)(e0 + e) * kD + f];
            Sb[e * kLd + f] = sv;
            dSb[e * kLd + f] = dsv;
            ss = fmaf(sv, dsv, ss);
        }
        for (int idx = tid; idx < kC * kEB; idx += kThreads) {
            const int i = idx / kEB, e = idx % kEB;
            Ub[i * kLe + e] = p.Up[sh * kC * kD + (size_t)i * kD + e0 + e];
            const bool ok = i < L;
            dOb[i * kLe + e] = ok ? p.d_o[((t0 + i) * p.Hv + h) * kD + e0 + e] : 0.f;
            Vb[i * kLe + e] = ok ? bf16f(p.v[((t0 + i) * p.Hv + h) * kD + e0 + e]) : 0.f;
        }
        BWC_SYNC();
        // U = U' - W S^T; K dS^T; Q S^T; P^T dO  (row i, columns eg .. eg + 3 per thread)
        {
            static_assert(kC * kEB == 4 * kThreads, "one row and four v columns per thread");
            const int i = tid >> 2, eg = (tid & 3) * 4;
            float u[4], kds[4] = {0.f, 0.f, 0.f, 0.f}, qs[4] = {0.f, 0.f, 0.f, 0.f}, pdo[4] = {0.f, 0.f, 0.f, 0.f};
            for (int x = 0; x < 4; ++x) u[x] = Ub[i * kLe + eg + x];
            for (int f = 0; f < kD; ++f) {
                const float wv = Ws[i * kLd + f], kv = Ks[i * kLd + f], qv = Qs[i * kLd + f];
                for (int x = 0; x < 4; ++x) {
                    const float sv = Sb[(eg + x) * kLd + f], dsv = dSb[(eg + x) * kLd + f];
                    u[x] = fmaf(-wv, sv, u[x]);
                    kds[x] = fmaf(kv, dsv, kds[x]);
                    qs[x] = fmaf(qv, sv, qs[x]);
                }
            }
            for (int m = i; m < L; ++m) {
                const float pm = Pm[m * kLc + i];
                for (int x = 0; x < 4; ++x) pdo[x] = fmaf(pm, dOb[m * kLe + eg + x], pdo[x]);
            }
            for (int x = 0; x < 4; ++x) {
                const int e = eg + x;
                Ub[i * kLe + e] = u[x];
                dUb[i * kLe + e] = kap[i] * kds[x] + p.scale * pdo[x];
                R1[i * kLe + e] = u[x] * kds[x];
                R2[i * kLe + e] = dOb[i * kLe + e] * qs[x];
            }
        }
        BWC_SYNC();
        if (tid < kC) {
            float s1 = 0.f, s2 = 0.f;
            for (int e = 0; e < kEB; ++e) {
                s1 += R1[tid * kLe + e];
                s2 += R2[tid * kLe + e];
            }
            dkap[tid] += s1;
            dgam[tid] += p.scale * s2;
        }
        BWC_SYNC();
        // dk += kap U dS, dq += scale gam dO S, dW -= dU S; dP += dO U^T, dT += dU (beta V)^T
        for (int e = 0; e < kEB; ++e) {
            float s4[4], ds4[4];
            for (int c = 0; c < 4; ++c) {
                s4[c] = Sb[e * kLd + l4 + c];
                ds4[c] = dSb[e * kLd + l4 + c];
            }
            for (int r = 0; r < 8; ++r) {
                const int i = w8 + r;
                const float ku = kap[i] * Ub[i * kLe + e];
                const float sd = p.scale * gam[i] * dOb[i * kLe + e];
                const float du = dUb[i * kLe + e];
                for (int c = 0; c < 4; ++c) {
                    dKa[r][c] = fmaf(ku, ds4[c], dKa[r][c]);
                    dQa[r][c] = fmaf(sd, s4[c], dQa[r][c]);
                    dWa[r][c] = fmaf(-du, s4[c], dWa[r][c]);
                }
            }
            for (int r = 0; r < 4; ++r) {
                const float dov = dOb[(r4 + r) * kLe + e], duv = dUb[(r4 + r) * kLe + e];
                for (int c = 0; c < 4; ++c) {
                    const int j = c4 + c;
                    dPa[r][c] = fmaf(dov, Ub[j * kLe + e], dPa[r][c]);
                    dTa[r][c] = fmaf(duv, be[j] * Vb[j * kLe + e], dTa[r][c]);
                }
            }
        }
        // dv = beta T^T dU; its part of d beta
        for (int idx = tid; idx < kC * kEB; idx += kThreads) {
            const int j = idx / kEB, e = idx % kEB;
            float x = 0.f;
            for (int i = j; i < L; ++i) x = fmaf(Tm[i * kLc + j], dUb[i * kLe + e], x);
            if (j < L) p.dv[((t0 + j) * p.Hv + h) * kD + e0 + e] = be[j] * x;
            R1[j * kLe + e] = x * Vb[j * kLe + e];
        }
        BWC_SYNC();
        if (tid < kC) {
            float s1 = 0.f;
            for (int e = 0; e < kEB; ++e) s1 += R1[tid * kLe + e];
            dbe[tid] += s1;
        }
        BWC_SYNC();
    }

    // ---- <dS_c, S_c> belongs to gam_{L-1}
    part[tid] = ss;
    // dP = scale lower(dO U^T): M1 = dP o Gam, M2 = dP o P (= Gam o dGam from P)
    for (int r = 0; r < 4; ++r)
        for (int c = 0; c < 4; ++c) {
            const int i = r4 + r, j = c4 + c;
            const bool in = j <= i && i < L;
            const float dp = in ? p.scale * dPa[r][c] : 0.f;
            M1[i * kLc + j] = in ? dp * expf(G[i] - G[j]) : 0.f;
            M2[i * kLc + j] = dp * Pm[i * kLc + j];
        }
    // dW over W
    for (int r = 0; r < 8; ++r)
        for (int c = 0; c < 4; ++c) Ws[(w8 + r) * kLd + l4 + c] = dWa[r][c];
    BWC_SYNC();
    if (tid == 0) {
        float s = 0.f;
        for (int x = 0; x < kThreads; ++x) s += part[x];
        dgam[L - 1] += s;
    }
    if (tid < kC) {
        const int i = tid;
        float rs = 0.f, cs = 0.f;
        for (int j = 0; j < kC; ++j) {
            rs += M2[i * kLc + j];
            cs += M2[j * kLc + i];
        }
        dGv[i] = rs - cs;
    }
    // dq += (dP o Gam) K, dk += (dP o Gam)^T Q
    for (int j = 0; j < kC; ++j) {
        float k4[4], q4[4];
        for (int c = 0; c < 4; ++c) {
            k4[c] = Ks[j * kLd + l4 + c];
        }
        for (int r = 0; r < 8; ++r) {
            const float m = M1[(w8 + r) * kLc + j];
            for (int c = 0; c < 4; ++c) dQa[r][c] = fmaf(m, k4[c], dQa[r][c]);
        }
        for (int c = 0; c < 4; ++c) q4[c] = Qs[j * kLd + l4 + c];
        for (int r = 0; r < 8; ++r) {
            const float m = M1[j * kLc + w8 + r];
            for (int c = 0; c < 4; ++c) dKa[r][c] = fmaf(m, q4[c], dKa[r][c]);
        }
    }
    // dT += dW (beta gam K)^T
    for (int f = 0; f < kD; ++f) {
        float dw4[4], k4[4];
        for (int r = 0; r < 4; ++r) dw4[r] = Ws[(r4 + r) * kLd + f];
        for (int c = 0; c < 4; ++c) {
            const int j = c4 + c;
            k4[c] = be[j] * gam[j] * Ks[j * kLd + f];
        }
        for (int r = 0; r < 4; ++r)
            for (int c = 0; c < 4; ++c) dTa[r][c] = fmaf(dw4[r], k4[c], dTa[r][c]);
    }
    // T^T dW: dk += beta gam (T^T dW); sum_f (T^T dW)_jf K_jf for d beta, d gam
    {
        float sk[8];
        for (int r = 0; r < 8; ++r) {
            const int j = w8 + r;
            float tw[4] = {0.f, 0.f, 0.f, 0.f};
            for (int i = j; i < L; ++i) {
                const float t = Tm[i * kLc + j];
                for (int c = 0; c < 4; ++c) tw[c] = fmaf(t, Ws[i * kLd + l4 + c], tw[c]);
            }
            const float bg = be[j] * gam[j];
            float s = 0.f;
            for (int c = 0; c < 4; ++c) {
                dKa[r][c] = fmaf(bg, tw[c], dKa[r][c]);
                s = fmaf(tw[c], Ks[j * kLd + l4 + c], s);
            }
            sk[r] = s;
        }
        BWC_SYNC();     // the v-column buffers (SK aliases them) are free from here
        for (int r = 0; r < 8; ++r) SK[(w8 + r) * 33 + (tid & 31)] = sk[r];
    }
    BWC_SYNC();
    if (tid < kC) {
        const int j = tid;
        float s = 0.f;
        for (int x = 0; x < 32; ++x) s += SK[j * 33 + x];
        dbe[j] += gam[j] * s;
        dgam[j] += be[j] * s;
    }
    // dT (strictly lower part suffices) into M1
    for (int r = 0; r < 4; ++r)
        for (int c = 0; c < 4; ++c) {
            const int i = r4 + r, j = c4 + c;
            M1[i * kLc + j] = j < i ? dTa[r][c] : 0.f;
        }
    BWC_SYNC();
    // M2 = T^T dT
    for (int idx = tid; idx < kC * kC; idx += kThreads) {
        const int i = idx >> 6, j = idx & (kC - 1);
        float x = 0.f;
        for (int m = i; m < kC; ++m) x = fmaf(Tm[m * kLc + i], M1[m * kLc + j], x);
        M2[i * kLc + j] = x;
    }
    BWC_SYNC();
    // dA = -(T^T dT) T^T on the strictly lower part, into M1
    for (int idx = tid; idx < kC * kC; idx += kThreads) {
        const int i = idx >> 6, j = idx & (kC - 1);
        float x = 0.f;
        if (j < i)
            for (int m = 0; m <= j; ++m) x = fmaf(M2[i * kLc + m], Tm[j * kLc + m], x);
        M1[i * kLc + j] = -x;
    }
    BWC_SYNC();
    // A = diag(beta) A': d beta_i += sum_j dA_ij A'_ij; Gam o dGam += dA o beta A';
    // E = dA o beta Gam into M2
    for (int idx = tid; idx < kC * kC; idx += kThreads) {
        const int i = idx >> 6, j = idx & (kC - 1);
        const bool in = j < i && i < L;
        M2[i * kLc + j] = in ? M1[i * kLc + j] * be[i] * expf(G[i] - G[j]) : 0.f;
    }
    if (tid < kC) {
        const int i = tid;
        float db_ = 0.f, rs = 0.f, cs = 0.f;
        for (int j = 0; j < kC; ++j) {
            const float x = M1[i * kLc + j] * Ap[i * kLc + j];
            db_ += x;
            rs += x;
            cs += M1[j * kLc + i] * be[j] * Ap[j * kLc + i];
        }
        dbe[i] += db_;
        dGv[i] += be[i] * rs - cs;
    }
    BWC_SYNC();
    // dk += (E + E^T) K
    for (int j = 0; j < kC; ++j) {
        float k4[4];
        for (int c = 0; c < 4; ++c) k4[c] = Ks[j * kLd + l4 + c];
        for (int r = 0; r < 8; ++r) {
            const int i = w8 + r;
            const float e = M2[i * kLc + j] + M2[j * kLc + i];
            for (int c = 0; c < 4; ++c) dKa[r][c] = fmaf(e, k4[c], dKa[r][c]);
        }
    }
    // decays: dG_i, then d log alpha_m = sum_{i >= m} dG_i, and the gate inputs
    if (tid < kC) {
        const int i = tid;
        dGv[i] += gam[i] * dgam[i] - kap[i] * dkap[i];
    }
    BWC_SYNC();
    if (tid == 0) {
        float ks = 0.f;
        for (int i = 0; i < L; ++i) ks += kap[i] * dkap[i];
        dGv[L - 1] += ks;
        const float eA = expf(p.A_log[h]), dtb = p.dt_bias[h];
        float suf = 0.f, gA = 0.f, gD = 0.f;
        for (int m = L - 1; m >= 0; --m) {
            suf += dGv[m];
            const int64_t t = t0 + m;
            const float dat = suf * (-eA * sigmoid(p.a[t * p.Hv + h] + dtb));
            p.da[t * p.Hv + h] = dat;
            p.db[t * p.Hv + h] = dbe[m] * be[m] * (1.f - be[m]);
            gA = fmaf(suf, lg[m], gA);
            gD += dat;
        }
        p.gpart[sh * 2 + 0] = gA;
        p.gpart[sh * 2 + 1] = gD;
    }
    // dq, dk of this value head
    for (int r = 0; r < 8; ++r) {
        const int i = w8 + r;
        if (i >= L) continue;
        float* dq = p.dqh + ((t0 + i) * p.Hv + h) * kD + l4;
        float* dk = p.dkh + ((t0 + i) * p.Hv + h) * kD + l4;
        for (int c = 0; c < 4; ++c) {
            dq[c] = dQa[r][c];
            dk[c] = dKa[r][c];
        }
    }
}

// ---- sums ------------------------------------------------------------------------------------
// dq, dk [T, Hqk, 128]: the value heads of each key head, in head order; one
// element per thread of block `blk`.
BWC_FN void reduce_qk_block(const Params& p, int64_t blk, int tid) {
    const int64_t idx = blk * kThreads + tid;
    if (idx >= p.T * p.Hqk * kD) return;
    const int f = (int)(idx % kD);
    const int64_t tg = idx / kD;
    const int64_t t = tg / p.Hqk;
    const int g = (int)(tg % p.Hqk);
    const int grp = p.Hv / p.Hqk;
    float sq = 0.f, sk = 0.f;
    for (int x = 0; x < grp; ++x) {
        const size_t o = ((size_t)t * p.Hv + g * grp + x) * kD + f;
        sq += p.dqh[o];
        sk += p.dkh[o];
    }
    p.dq[idx] = sq;
    p.dk[idx] = sk;
}

// dA_log, ddt_bias [Hv]: the per-chunk sums in slot order; one head per thread.
BWC_FN void reduce_gates_block(const Params& p, int tid) {
    for (int h = tid; h < p.Hv; h += kThreads) {
        float sA = 0.f, sD = 0.f;
        for (int64_t s = 0; s < p.n_slots; ++s) {
            sA += p.gpart[sh_index(p, s, h) * 2 + 0];
            sD += p.gpart[sh_index(p, s, h) * 2 + 1];
        }
        p.dA_log[h] = sA;
        p.ddt_bias[h] = sD;
    }
}

}  // namespace bwc
}  // namespace gdn
