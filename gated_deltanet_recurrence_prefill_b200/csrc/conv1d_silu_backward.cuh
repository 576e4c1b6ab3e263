// conv1d_silu_backward.cuh -- the gradient of the front end (4-tap causal
// depthwise conv1d, SiLU, L2 norm of each q and k head), on CUDA cores in
// float32.  The forward is the one of gdn_conv1d_silu (architecture page
// section 2.1: the conv of width 4 ahead of the recurrence; SiLU and the q / k
// norm as for the forward kernel):
//     y[t, c] = sum_j w[c, j] x~[t - 3 + j, c],   a = y sigma(y),
//     out = a / n,  n = sqrt(sum_head a^2 + 1e-6)   (q and k heads; out = a for v),
// where x~ before a sequence's first token is its conv_state history (or zero).
// Reverse mode:
//     da = (dout - out <dout, out>) / n     (q, k);   da = dout  (v)
//     dy = da sigma(y) (1 + y (1 - sigma(y))) = da (sigma + a (1 - sigma))
//     dx[t] = sum_j w[c, j] dy[t + 3 - j]   (tokens of the same sequence)
//     dw[c, j] = sum_t dy[t] x~[t - 3 + j],  d history = the taps that reach it.
//
// A job is one packed head (q heads, k heads, v heads, as in the qkv layout)
// over a tile of kTile tokens, on 128 threads (one per channel); it recomputes
// the forward for its tokens and the next three (dx[t] needs dy up to t + 3).
// The weight gradient is summed per tile, then over tiles in order; the
// history gradient of a sequence is written by the job whose tile holds the
// sequence's first token.  Block functions as in backward_chunked.cuh: the
// CUDA kernels and the CPU tests' emulation run the same source; threads meet
// at block barriers and in warp shuffles, and every sum has a fixed order.
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
namespace fbw {

constexpr int kD = 128;
constexpr int kThreads = 128;            // one thread per channel of a head
constexpr int kTile = 32;                // tokens per job
constexpr int kSpan = kTile + 3;         // tokens whose dy a job needs
constexpr int kLd = kD + 1;

struct Params {
    const uint16_t* x;          // qkv [T, Ctot] bf16, Ctot = (2 Hqk + Hv) * 128
    const float* w;             // [Ctot, 4]
    const int32_t* cu;          // [n_seq + 1] or null (one sequence)
    const float* cs;            // conv_state [n_seq, Ctot, 3] or null (zero history)
    const float* dq;            // [T, Hqk, 128]
    const float* dk;            // [T, Hqk, 128]
    const float* dv;            // [T, Hv, 128]
    int32_t n_seq, Hqk, Hv;
    int64_t T, n_tiles;
    float* dx;                  // [T, Ctot]
    float* dwp;                 // [n_tiles, Ctot, 4] per-tile sums (workspace)
    float* dw;                  // [Ctot, 4]
    float* dcs;                 // [n_seq, Ctot, 3] or null (set to zero first by the host)
};

BWC_HD int64_t n_tiles(int64_t T) { return (T + kTile - 1) / kTile; }

// shared-memory floats of one job
constexpr int kTileFloats = 3 * kSpan * kLd + 4 * kSpan + (kSpan + 3) * kD;

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

// the sequence of token t: the last n with cu[n] <= t
BWC_FN int seq_of(const Params& p, int64_t t) {
    if (!p.cu) return 0;
    int lo = 0, hi = p.n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}


// A tile whose tokens, their three-token history and the three tokens after it
// all lie in one sequence takes the streaming kernel (conv1d_silu_backward.cu);
// tile_block handles every other tile.  Both kernels decide with this test.
BWC_FN bool stream_tile(const Params& p, int64_t tile) {
    const int64_t t0 = tile * kTile;
    if (t0 < 3 || t0 + kSpan > p.T) return false;
    if (!p.cu) return true;
    const int n = seq_of(p, t0);
    return (int64_t)p.cu[n] + 3 <= t0 && t0 + kSpan <= (int64_t)p.cu[n + 1];
}

// x~ at position pos for a token of sequence n starting at bos, channel c:
// x from the tile's staged copy (xr holds positions t0 - 3 ..), or the
// sequence's conv_state history (or zero) before its first token
BWC_FN float xts(const Params& p, int64_t Ctot, int n, int64_t bos, int64_t pos, int64_t c, const float* xr,
                 int64_t t0, int tid) {
    if (pos >= bos) return xr[(pos - (t0 - 3)) * kD + tid];
    return p.cs ? p.cs[((int64_t)n * Ctot + c) * 3 + (3 - (bos - pos))] : 0.f;
}

BWC_FN void tile_block(const Params& p, int64_t tile, int hh, int tid, float* sm) {
    const int64_t Ctot = (int64_t)(2 * p.Hqk + p.Hv) * kD;
    const int64_t t0 = tile * kTile;
    const int ntok = (int)((p.T - t0) < kSpan ? (p.T - t0) : kSpan);
    const int nmain = ntok < kTile ? ntok : kTile;
    const bool normed = hh < 2 * p.Hqk;
    const int64_t c = (int64_t)hh * kD + tid;

    float* as = sm;                       // a = silu(y)          [kSpan][kLd]
    float* sg = as + kSpan * kLd;         // sigma(y)             [kSpan][kLd]
    float* gs = sg + kSpan * kLd;         // dout, then dy        [kSpan][kLd]
    float* nrm = gs + kSpan * kLd;        // per token: n, <dout, out>
    float* dot = nrm + kSpan;
    int32_t* sq = reinterpret_cast<int32_t*>(dot + kSpan);    // per token: sequence
    int32_t* eo = sq + kSpan;                                 // per token: sequence end
    float* xr = reinterpret_cast<float*>(eo + kSpan);         // x at positions t0 - 3 ..  [kSpan + 3][kD]

    if (tid < ntok) {
        const int n = seq_of(p, t0 + tid);
        sq[tid] = n;
        eo[tid] = p.cu ? p.cu[n + 1] : (int32_t)p.T;
    }
    // this channel's inputs at every position the tile reads, loaded up front so
    // that the loads overlap (positions before 0 are never read from here)
    for (int r = 0; r < ntok + 3; ++r) {
        const int64_t pos = t0 - 3 + r;
        xr[r * kD + tid] = pos >= 0 ? bf16f(p.x[pos * Ctot + c]) : 0.f;
    }
    BWC_SYNC();
    float w[4];
    for (int j = 0; j < 4; ++j) w[j] = p.w[c * 4 + j];
    const float* dsrc = hh < p.Hqk ? p.dq + (int64_t)hh * kD
                      : normed ? p.dk + (int64_t)(hh - p.Hqk) * kD : p.dv + (int64_t)(hh - 2 * p.Hqk) * kD;
    const int64_t dstride = (normed ? (int64_t)p.Hqk : (int64_t)p.Hv) * kD;
    // the output gradient of every token, loaded up front (independent loads)
    for (int tau = 0; tau < ntok; ++tau) gs[tau * kLd + tid] = dsrc[(t0 + tau) * dstride + tid];
    for (int tau = 0; tau < ntok; ++tau) {
        const int64_t t = t0 + tau;
        const int n = sq[tau];
        const int64_t bos = p.cu ? p.cu[n] : 0;
        float y = 0.f;
        for (int j = 0; j < 4; ++j) y = fmaf(w[j], xts(p, Ctot, n, bos, t - 3 + j, c, xr, t0, tid), y);
        const float s = 1.f / (1.f + expf(-y));
        as[tau * kLd + tid] = y * s;
        sg[tau * kLd + tid] = s;
    }
    BWC_SYNC();
    // per token: the norm and <dout, out> / n, one warp per token (a lane sums 4
    // channels, then 5 xor shuffles)
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int tau = warp; tau < ntok; tau += kThreads / 32) {
            float ss = 0.f, gd = 0.f;
            for (int x = 0; x < kD / 32; ++x) {
                const float a = as[tau * kLd + lane + 32 * x];
                ss = fmaf(a, a, ss);
                gd = fmaf(gs[tau * kLd + lane + 32 * x], a, gd);
            }
            for (int m = 16; m >= 1; m >>= 1) {
                ss += BWC_SHFL_XOR(ss, m);
                gd += BWC_SHFL_XOR(gd, m);
            }
            if (lane == 0) {
                const float nv = normed ? sqrtf(ss + 1e-6f) : 1.f;
                nrm[tau] = nv;
                dot[tau] = normed ? gd / (nv * nv) : 0.f;     // <dout, out> / n
            }
        }
    }
    BWC_SYNC();
    // dy in place of dout (each thread its own channel)
    for (int tau = 0; tau < ntok; ++tau) {
        const float a = as[tau * kLd + tid], s = sg[tau * kLd + tid], g = gs[tau * kLd + tid];
        const float da = normed ? (g - a * dot[tau]) / nrm[tau] : g;
        gs[tau * kLd + tid] = da * (s + a * (1.f - s));
    }
    // dx for the tile's tokens; this tile's part of dw
    float dwa[4] = {0.f, 0.f, 0.f, 0.f};
    for (int tau = 0; tau < nmain; ++tau) {
        const int64_t t = t0 + tau;
        const int64_t eos = eo[tau];
        float acc = 0.f;
        for (int j = 0; j < 4; ++j) {
            const int64_t u = t + 3 - j;                    // the token whose tap j reads x[t]
            if (u < eos) acc = fmaf(w[j], gs[(u - t0) * kLd + tid], acc);
        }
        p.dx[t * Ctot + c] = acc;
        const int n = sq[tau];
        const int64_t bos = p.cu ? p.cu[n] : 0;
        const float dy = gs[tau * kLd + tid];
        for (int j = 0; j < 4; ++j) dwa[j] = fmaf(dy, xts(p, Ctot, n, bos, t - 3 + j, c, xr, t0, tid), dwa[j]);
    }
    for (int j = 0; j < 4; ++j) p.dwp[(tile * Ctot + c) * 4 + j] = dwa[j];
    // the history gradient of every sequence that starts in this tile
    if (p.dcs) {
        int n = t0 == 0 ? 0 : p.n_seq;                        // one sequence: it starts in tile 0
        if (p.cu) {
            int lo = 0, hi = p.n_seq;                         // first n with cu[n] >= t0
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (p.cu[mid] >= t0) hi = mid;
                else lo = mid + 1;
            }
            n = lo;
        }
        for (; n < p.n_seq; ++n) {
            const int64_t bos = p.cu ? p.cu[n] : 0, eos = p.cu ? p.cu[n + 1] : p.T;
            if (bos >= t0 + nmain) break;
            // slot s holds position bos - 3 + s; token bos + m reads it through tap s - m
            for (int s = 0; s < 3; ++s) {
                float acc = 0.f;
                for (int m = 0; m <= s; ++m)
                    if (bos + m < eos) acc = fmaf(w[s - m], gs[(bos + m - t0) * kLd + tid], acc);
                p.dcs[((int64_t)n * Ctot + c) * 3 + s] = acc;
            }
        }
    }
}

// dw [Ctot, 4]: the per-tile sums in tile order; element blk * kThreads + tid
BWC_FN void reduce_w_block(const Params& p, int64_t blk, int tid) {
    const int64_t Ctot = (int64_t)(2 * p.Hqk + p.Hv) * kD;
    const int64_t i = blk * kThreads + tid;
    if (i >= Ctot * 4) return;
    // the partial sums are added in tile order; 32 are loaded ahead of their
    // additions so that the loads overlap (the order of the additions, and so
    // the result, is the same)
    float s = 0.f;
    const float* src = p.dwp + i;
    const int64_t stride = Ctot * 4;
    int64_t tl = 0;
    for (; tl + 32 <= p.n_tiles; tl += 32) {
        float v[32];
        for (int r = 0; r < 32; ++r) v[r] = src[(tl + r) * stride];
        for (int r = 0; r < 32; ++r) s += v[r];
    }
    for (; tl < p.n_tiles; ++tl) s += src[tl * stride];
    p.dw[i] = s;
}

}  // namespace fbw
}  // namespace gdn
