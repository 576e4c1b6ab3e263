// backward_chunked_tc.cu -- the per-(chunk, value head) gradient step of the
// chunked backward on the tensor cores.
//
// The algebra is that of grad_block in backward_chunked.cuh (reverse mode
// through the chunked WY / UT form of the gated delta rule; Qwen3.8-27B
// architecture page, 2kiu.com, section 2.2, for the recurrence).  Here every
// product of the step is a tcgen05.mma (kind::f16: bf16 operands staged in
// shared memory with the 128-byte swizzle, float32 accumulators in TMEM), and
// the element-wise parts between the products (causal masks, decays, the row
// and column sums of the gate gradients) run on the CUDA cores.  One CTA of 8
// warps per (chunk, value head); the products come in seven rounds, each issued
// by one thread once the operands it needs are in shared memory:
//
//   1. D0 = [Q; K] K^T, [W; Q] S^T, K dS^T        -> P, U = U' - W S^T, kappa U,
//                                                    the kappa and gamma sums
//   2. P^T dO                                      -> dU = kappa K dS^T + scale P^T dO
//   3. [dO; dU] S, [dO; dU] [U; V]^T, (kappa U) dS -> dW, dP -> M1 = scale dP o Gamma,
//                                                    the dP o P sums; dq's first
//                                                    term rescaled in TMEM
//   4. dq += M1 K, dk += M1^T Q + (T diag(beta gam))^T dW, dW K^T
//                                                  -> dT, the T o (dU V^T), T o (dW K^T) sums
//   5. dv = (T diag(beta))^T dU, T^T dT            -> dv, M2
//   6. M2 T^T                                      -> dA, E = dA o beta Gamma, the dA o A' sums
//   7. dk += (E + E^T) K                           -> dq, dk, and the gates
//
// Every product is issued with M = 128.  Where only 64 rows of the result are
// wanted, the A operand's other 64 rows are whatever follows in shared memory
// and the TMEM lanes they produce are never read; operands are placed so that
// a result lands in the lanes (TMEM lanes 0-63 or 64-127) of the warps that
// combine it with another.  The accumulators use all 512 TMEM columns and the
// tiles ~214 KB of shared memory: one CTA per SM.
#include "backward_chunked.cuh"
#include "kernels.h"
#include "tile_util.cuh"

namespace gdn {
namespace {

using namespace bwc;
using namespace tc;

constexpr int kGThreads = 256;
constexpr uint32_t kPanel64 = 64 * 128;         // 64 rows of 64 bf16
constexpr uint32_t kPanel128 = 128 * 128;
constexpr uint32_t kPanel192 = 192 * 128;

// ---- shared memory (byte offsets from a 1024-aligned base) -----------------------------
// bf16 tiles; a tile of 128 columns is two panels of 64 (one per 128-byte row).
constexpr uint32_t S_T = 0;                         // T                64 x 64
constexpr uint32_t S_P = S_T + kPanel64;            // P                64 x 64; E + E^T later
constexpr uint32_t S_KU = S_P + kPanel64;           // kappa U          64 x 128; T diag(beta), T diag(beta gam) later
constexpr uint32_t S_KQW = S_KU + 2 * kPanel64;     // [W; Q; K]        192 x 128
constexpr uint32_t S_S = S_KQW + 2 * kPanel192;     // S (rows e)       128 x 128; [-; dW] later
constexpr uint32_t S_DS = S_S + 2 * kPanel128;      // dS               128 x 128; M1, dT, [-; M2] later
constexpr uint32_t S_UV = S_DS + 2 * kPanel128;     // [U; V]           128 x 128; f32 scratch later
constexpr uint32_t S_DUO = S_UV + 2 * kPanel128;    // [dO; dU]         128 x 128
constexpr uint32_t S_TILES = S_DUO + 2 * kPanel128;
constexpr uint32_t S_DW = S_S;                      // dW in rows 64-127 of a 128 x 128 tile
constexpr uint32_t S_M1 = S_DS;
constexpr uint32_t S_DT = S_DS + kPanel64;
constexpr uint32_t S_M2 = S_DS + 2 * kPanel64;      // M2 in rows 64-127 of a 128 x 64 tile
constexpr uint32_t S_TB = S_KU;
constexpr uint32_t S_TBG = S_KU + kPanel64;
constexpr uint32_t S_ES = S_P;
constexpr uint32_t S_SCR = S_UV;                    // 64 x 128 floats, columns rotated by the row

// float arrays after the tiles
enum : int {
    F_LG = 0, F_BE = 64, F_G = 128, F_GAM = 192, F_KAP = 256,
    F_DKAP = 320,     // [2][64]  sum_e U K dS^T, per column half
    F_DGAM = 448,     // [2][64]  sum_e dO Q S^T
    F_RSM = 576,      // [2][64]  row sums of dP o P
    F_CSM = 704,      // column sums of dP o P
    F_DBET = 768,     // column sums of T o (dU V^T)
    F_SKT = 832,      // column sums of T o (dW K^T)
    F_RSA = 896,      // [2][64]  row sums of dA o A'
    F_CSA = 1024,     // column sums of dA o beta A'
    F_RED = 1088,     // [256]    block reduction
    F_SS = 1344,      // <dS, S>
    F_SIG = 1352,     // sigmoid(a + dt_bias) per row
    F_XCH = 1416,     // [16] exchange between the two gate warps
    F_END = 1432
};
constexpr uint32_t S_MISC = S_TILES;
constexpr uint32_t S_BAR = S_MISC + F_END * 4;      // mbarrier (8), TMEM base (4), abort flag (4)
constexpr uint32_t SMEM_BYTES = S_BAR + 16;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(S_BAR % 8 == 0, "mbarrier alignment");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget of one CTA");

// ---- TMEM columns (lane = row of the M = 128 product) --------------------------------------
constexpr uint32_t T_D0 = 0;       // [Q K^T; K K^T]                           (kept to the end)
constexpr uint32_t T_C1 = 64;      // [W S^T; Q S^T] -> [dO S; dU S] -> dq (lanes 0-63)
constexpr uint32_t T_C2 = 192;     // K dS^T -> [dO; dU][U; V]^T -> dv (lanes 0-63)
constexpr uint32_t T_C3 = 320;     // P^T dO -> dk (lanes 0-63)
constexpr uint32_t T_C4 = 448;     // dW K^T (lanes 64-127) -> T^T dT (0-63) -> M2 T^T (64-127)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t ID_KK128 = idesc_bf16(128, 128, false, false);
constexpr uint32_t ID_KK64 = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_KM128 = idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_MM128 = idesc_bf16(128, 128, true, true);
constexpr uint32_t ID_MM64 = idesc_bf16(128, 64, true, true);

constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s: far beyond any product's time

// K-major operand: 16-deep K step kk of a tile whose 64-column panels are `panel` bytes apart
TC_DEVICE uint64_t kdesc(uint32_t base, uint32_t panel, int kk) {
    return sdesc_sw128(base + (uint32_t)(kk >> 2) * panel + (uint32_t)(kk & 3) * 32u, 16, 1024);
}
// MN-major operand (rows of the tile = the K index): 16 rows per step; lbo =
// distance between the tile's 64-column panels
TC_DEVICE uint64_t mdesc(uint32_t base, uint32_t lbo, int kk) {
    return sdesc_sw128(base + (uint32_t)kk * 2048u, lbo, 1024);
}

TC_DEVICE void mma_run(uint32_t d, uint32_t a_base, uint32_t a_step, bool a_mn, uint32_t b_base,
                       uint32_t b_step, bool b_mn, uint32_t idesc, int nk, bool accumulate) {
    for (int kk = 0; kk < nk; ++kk) {
        const uint64_t ad = a_mn ? mdesc(a_base, a_step, kk) : kdesc(a_base, a_step, kk);
        const uint64_t bd = b_mn ? mdesc(b_base, b_step, kk) : kdesc(b_base, b_step, kk);
        mma_bf16(d, ad, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

TC_DEVICE uint4 pack8(const float4 a, const float4 b) {
    uint4 r;
    r.x = pack_bf16x2(a.x, a.y);
    r.y = pack_bf16x2(a.z, a.w);
    r.z = pack_bf16x2(b.x, b.y);
    r.w = pack_bf16x2(b.z, b.w);
    return r;
}

// 16 bytes (8 bf16) at (row, 16-byte chunk ch) of a tile with `panel`-byte panels
TC_DEVICE void st16(uint8_t* sm, uint32_t base, uint32_t panel, int row, int ch, uint4 v) {
    *reinterpret_cast<uint4*>(sm + base + (uint32_t)(ch >> 3) * panel + sw128_off(row, ch & 7)) = v;
}
TC_DEVICE void put8(uint8_t* sm, uint32_t base, uint32_t panel, int row, int ch, const float* x) {
    tile::st_bf16x8(sm + base + (uint32_t)(ch >> 3) * panel, row, ch & 7, x);
}

TC_DEVICE float4 ldf4(const float* p) { return *reinterpret_cast<const float4*>(p); }
TC_DEVICE uint4 ldu4(const uint16_t* p) { return *reinterpret_cast<const uint4*>(p); }
TC_DEVICE void stf4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

// scratch: quantity 0 in columns 0-63, quantity 1 in 64-127, rotated by the row
// (conflict-free both for a thread per row and for a thread per column)
TC_DEVICE int scr_ix(int i, int j) { return i * 128 + ((j + i) & 127); }

__global__ void __launch_bounds__(kGThreads, 1) bwc_grad_tc_kernel(Params p) {
    extern __shared__ uint8_t bwt_smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bwt_smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t slot = blockIdx.x / p.Hv;
    const int h = blockIdx.x % p.Hv;
    const int n = p.jobs[2 * slot];
    if (n < 0) return;
    const int64_t t0 = p.jobs[2 * slot + 1];
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int L = (int)((eos - t0) < kC ? (eos - t0) : kC);
    const int g = h / (p.Hv / p.Hqk);
    const size_t sh = sh_index(p, slot, h);

    float* F = reinterpret_cast<float*>(sm + S_MISC);
    float *lg = F + F_LG, *be = F + F_BE, *G = F + F_G, *gam = F + F_GAM, *kap = F + F_KAP;
    float* scr = reinterpret_cast<float*>(sm + S_SCR);
    const uint32_t bar = sb + S_BAR;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S_BAR + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + S_BAR + 12);

    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tc_fence_before();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    // gates (warps 0-1, one row each): log alpha, beta, G = running sum of log
    // alpha (an inclusive scan; rows >= L add 0, so they carry G_{L-1}), gamma,
    // kappa, and sigmoid(a + dt_bias) for d a
    if (tid < kC) {
        const int r = tid;
        float la = 0.f, bb = 0.f, sg = 0.f;
        if (r < L) {
            const int64_t t = t0 + r;
            const float av = p.a[t * p.Hv + h], dtb = p.dt_bias[h];
            la = log_alpha(av, p.A_log[h], dtb);
            bb = sigmoid(p.b[t * p.Hv + h]);
            sg = sigmoid(av + dtb);
        }
        float run = la;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, run, m);
            if (lane >= m) run += o;
        }
        if (r == 31) F[F_XCH] = run;
        named_bar_sync(1, kC);
        if (r >= 32) run += F[F_XCH];
        lg[r] = la;
        be[r] = bb;
        G[r] = run;
        gam[r] = expf(run);
        F[F_SIG + r] = sg;
        named_bar_sync(1, kC);
        kap[r] = r < L ? expf(G[L - 1] - run) : 0.f;
    }
    // (this barrier also publishes the TMEM base and the mbarrier)
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const bool issuer = tid == 0;
    const int q = warp & 3, hf = warp >> 2;          // TMEM lane quarter, column half
    const uint32_t tl = tbase + ((uint32_t)(32 * q) << 16);
    const bool lo = q < 2;                           // TMEM lanes 0-63
    const int i = 32 * (q & 1) + lane;               // chunk row of this thread's TMEM lane
    const float scale = p.scale;

    // ---- stage the operands -------------------------------------------------------------
    {
        uint4 kx[4], qx[4], vx[4];
        float4 wx[4][2];
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            const bool ok = r < L;
            kx[x] = ok ? ldu4(p.k + ((size_t)(t0 + r) * p.Hqk + g) * kD + ch * 8) : z4;
            qx[x] = ok ? ldu4(p.q + ((size_t)(t0 + r) * p.Hqk + g) * kD + ch * 8) : z4;
            vx[x] = ok ? ldu4(p.v + ((size_t)(t0 + r) * p.Hv + h) * kD + ch * 8) : z4;
            const float* wp = p.W + sh * kC * kD + (size_t)r * kD + ch * 8;
            wx[x][0] = ldf4(wp);
            wx[x][1] = ldf4(wp + 4);
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            st16(sm, S_KQW, kPanel192, r, ch, pack8(wx[x][0], wx[x][1]));
            st16(sm, S_KQW, kPanel192, 64 + r, ch, qx[x]);
            st16(sm, S_KQW, kPanel192, 128 + r, ch, kx[x]);
            st16(sm, S_UV, kPanel128, 64 + r, ch, vx[x]);
        }
    }
    float ss = 0.f;
    {
        const float* Sg = p.S + sh * kD * kD;
        const float* dSg = p.dS + sh * kD * kD;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float4 sx[4][2], dx[4][2];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int it = tid + kGThreads * (4 * half + x), r = it >> 4, ch = it & 15;
                sx[x][0] = ldf4(Sg + (size_t)r * kD + ch * 8);
                sx[x][1] = ldf4(Sg + (size_t)r * kD + ch * 8 + 4);
                dx[x][0] = ldf4(dSg + (size_t)r * kD + ch * 8);
                dx[x][1] = ldf4(dSg + (size_t)r * kD + ch * 8 + 4);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int it = tid + kGThreads * (4 * half + x), r = it >> 4, ch = it & 15;
                st16(sm, S_S, kPanel128, r, ch, pack8(sx[x][0], sx[x][1]));
                st16(sm, S_DS, kPanel128, r, ch, pack8(dx[x][0], dx[x][1]));
#pragma unroll
                for (int y = 0; y < 2; ++y) {
                    ss = fmaf(sx[x][y].x, dx[x][y].x, ss);
                    ss = fmaf(sx[x][y].y, dx[x][y].y, ss);
                    ss = fmaf(sx[x][y].z, dx[x][y].z, ss);
                    ss = fmaf(sx[x][y].w, dx[x][y].w, ss);
                }
            }
        }
    }
    {
        float4 ox[4][2], tx[2][2];
        const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            const bool ok = r < L;
            const float* op = p.d_o + ((size_t)(t0 + r) * p.Hv + h) * kD + ch * 8;
            ox[x][0] = ok ? ldf4(op) : zf;
            ox[x][1] = ok ? ldf4(op + 4) : zf;
        }
        const float* Tg = p.Tm + sh * kC * kC;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int it = tid + kGThreads * x, r = it >> 3, ch = it & 7;
            tx[x][0] = ldf4(Tg + r * kC + ch * 8);
            tx[x][1] = ldf4(Tg + r * kC + ch * 8 + 4);
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            st16(sm, S_DUO, kPanel128, r, ch, pack8(ox[x][0], ox[x][1]));
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int it = tid + kGThreads * x, r = it >> 3, ch = it & 7;
            st16(sm, S_T, kPanel64, r, ch, pack8(tx[x][0], tx[x][1]));
        }
    }
    F[F_RED + tid] = ss;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    int phase = 0;
    // all threads wait for the products issued last; false (uniformly) if a
    // wait gave up
    auto products_done = [&]() -> bool {
        mbar_wait(bar, (uint32_t)(phase & 1), abort_flag, kWaitLimitNs);
        ++phase;
        __syncthreads();
        tc_fence_after();
        return *abort_flag == 0;
    };
    // the operands written since the last barrier are visible to the tensor core
    auto publish = [&]() {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
    };

    do {
        // ---- round 1
        if (issuer) {
            tc_fence_after();
            // D0 = [Q; K] K^T: lanes 0-63 Q K^T, 64-127 K K^T
            mma_run(tbase + T_D0, sb + S_KQW + 8192, kPanel192, false, sb + S_KQW + 16384, kPanel192, false,
                    ID_KK64, 8, false);
            // [W; Q] S^T: lanes 0-63 W S^T, 64-127 Q S^T
            mma_run(tbase + T_C1, sb + S_KQW, kPanel192, false, sb + S_S, kPanel128, false, ID_KK128, 8, false);
            // K dS^T (lanes 0-63)
            mma_run(tbase + T_C2, sb + S_KQW + 16384, kPanel192, false, sb + S_DS, kPanel128, false, ID_KK128, 8,
                    false);
            mma_commit(bar);
        }
        if (tid == 0) {
            float s = 0.f;
            for (int x = 0; x < kGThreads; ++x) s += F[F_RED + x];
            F[F_SS] = s;
        }
        if (!products_done()) break;

        // ---- epilogue 1: U, kappa U, P (lanes 0-63); the gamma sums (lanes 64-127)
        if (lo) {
            const float ki = kap[i];
            float r1 = 0.f;
            const float* up = p.Up + sh * kC * kD + (size_t)i * kD;
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float x1[32], kd[32];
                tmem_ld32x2(tl + T_C1 + c0, tl + T_C2 + c0, x1, kd);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) {
                    const float4 a = ldf4(up + c0 + 8 * j8), b = ldf4(up + c0 + 8 * j8 + 4);
                    const float upv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                    float u[8], ku[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        u[e] = upv[e] - x1[8 * j8 + e];
                        r1 = fmaf(u[e], kd[8 * j8 + e], r1);
                        ku[e] = ki * u[e];
                    }
                    put8(sm, S_UV, kPanel128, i, c0 / 8 + j8, u);
                    put8(sm, S_KU, kPanel64, i, c0 / 8 + j8, ku);
                }
            }
            F[F_DKAP + 64 * hf + i] = r1;
            float qk[32];
            tmem_ld32(tl + T_D0 + 32 * hf, qk);
            tmem_ld_wait();
            const float Gi = G[i];
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                const int j = 32 * hf + jj;
                qk[jj] = (j <= i && i < L) ? qk[jj] * expf(Gi - G[j]) : 0.f;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) put8(sm, S_P, kPanel64, i, 4 * hf + c, qk + 8 * c);
        } else {
            float r2 = 0.f;
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float qs[32];
                tmem_ld32(tl + T_C1 + c0, qs);
                tmem_ld_wait();
                if (i < L) {
                    const float* op = p.d_o + ((size_t)(t0 + i) * p.Hv + h) * kD + c0;
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 o4 = ldf4(op + 4 * e4);
                        r2 = fmaf(o4.x, qs[4 * e4], r2);
                        r2 = fmaf(o4.y, qs[4 * e4 + 1], r2);
                        r2 = fmaf(o4.z, qs[4 * e4 + 2], r2);
                        r2 = fmaf(o4.w, qs[4 * e4 + 3], r2);
                    }
                }
            }
            F[F_DGAM + 64 * hf + i] = r2;
        }
        publish();

        // ---- round 2: P^T dO (lanes 0-63)
        if (issuer) {
            tc_fence_after();
            mma_run(tbase + T_C3, sb + S_P, kPanel64, true, sb + S_DUO, kPanel128, true, ID_MM128, 4, false);
            mma_commit(bar);
        }
        if (!products_done()) break;

        // ---- epilogue 2: dU = kappa K dS^T + scale P^T dO into rows 64-127 of [dO; dU]
        if (lo) {
            const float ki = kap[i];
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float kd[32], pd[32];
                tmem_ld32x2(tl + T_C2 + c0, tl + T_C3 + c0, kd, pd);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) {
                    float du[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) du[e] = ki * kd[8 * j8 + e] + scale * pd[8 * j8 + e];
                    put8(sm, S_DUO, kPanel128, 64 + i, c0 / 8 + j8, du);
                }
            }
        }
        publish();

        // ---- round 3
        if (issuer) {
            tc_fence_after();
            // [dO; dU] S: lanes 0-63 dO S, 64-127 dU S (= -dW)
            mma_run(tbase + T_C1, sb + S_DUO, kPanel128, false, sb + S_S, kPanel128, true, ID_KM128, 8, false);
            // [dO; dU] [U; V]^T: lanes 0-63 columns 0-63 dO U^T (dP), lanes 64-127 columns 64-127 dU V^T
            mma_run(tbase + T_C2, sb + S_DUO, kPanel128, false, sb + S_UV, kPanel128, false, ID_KK128, 8, false);
            // dk = (kappa U) dS (lanes 0-63)
            mma_run(tbase + T_C3, sb + S_KU, kPanel64, false, sb + S_DS, kPanel128, true, ID_KM128, 8, false);
            mma_commit(bar);
        }
        if (!products_done()) break;

        // ---- epilogue 3
        if (lo) {
            // dq's first term: scale gamma_i (dO S)_i, rewritten in place
            const float sq = scale * gam[i];
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float v[32];
                tmem_ld32(tl + T_C1 + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= sq;
                tmem_st32(tl + T_C1 + c0, v);
            }
            tmem_st_wait();
            // dP -> M1 = scale lower(dP) o Gamma; dP o P for the decays
            float dpv[32], qk[32];
            tmem_ld32x2(tl + T_C2 + 32 * hf, tl + T_D0 + 32 * hf, dpv, qk);
            const float Gi = G[i];
            float rs = 0.f;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                const int j = 32 * hf + jj;
                const bool in = j <= i && i < L;
                const float gm = in ? expf(Gi - G[j]) : 0.f;
                const float dp = in ? scale * dpv[jj] : 0.f;
                const float m2 = dp * (qk[jj] * gm);
                rs += m2;
                scr[scr_ix(i, j)] = m2;
                dpv[jj] = dp * gm;
            }
            F[F_RSM + 64 * hf + i] = rs;
#pragma unroll
            for (int c = 0; c < 4; ++c) put8(sm, S_M1, kPanel64, i, 4 * hf + c, dpv + 8 * c);
        } else {
            // dW = -(dU S) into rows 64-127 of its tile
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float v[32];
                tmem_ld32(tl + T_C1 + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = -v[e];
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) put8(sm, S_DW, kPanel128, 64 + i, c0 / 8 + j8, v + 8 * j8);
            }
            // T diag(beta) and T diag(beta gam) (over kappa U, read by round 3)
            const int ht = 64 * hf + 32 * (q - 2) + lane;
            const float* Tg = p.Tm + sh * kC * kC;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int it = ht + 128 * x, r = it >> 3, ch = it & 7;
                const float4 a = ldf4(Tg + r * kC + ch * 8), b = ldf4(Tg + r * kC + ch * 8 + 4);
                const float tv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                float tb[8], tbg[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    tb[e] = tv[e] * be[8 * ch + e];
                    tbg[e] = tb[e] * gam[8 * ch + e];
                }
                put8(sm, S_TB, kPanel64, r, ch, tb);
                put8(sm, S_TBG, kPanel64, r, ch, tbg);
            }
        }
        publish();

        // ---- round 4
        if (issuer) {
            tc_fence_after();
            // dq += M1 K (lanes 0-63; lanes 64-127 held dU S, already read)
            mma_run(tbase + T_C1, sb + S_M1, kPanel64, false, sb + S_KQW + 16384, kPanel192, true, ID_KM128, 4,
                    true);
            // dk += M1^T Q + (T diag(beta gam))^T dW
            mma_run(tbase + T_C3, sb + S_M1, kPanel64, true, sb + S_KQW + 8192, kPanel192, true, ID_MM128, 4, true);
            mma_run(tbase + T_C3, sb + S_TBG, kPanel64, true, sb + S_DW + 8192, kPanel128, true, ID_MM128, 4, true);
            // dW K^T (lanes 64-127)
            mma_run(tbase + T_C4, sb + S_DW, kPanel128, false, sb + S_KQW + 16384, kPanel192, false, ID_KK64, 8,
                    false);
            mma_commit(bar);
        }
        if (tid < 64) {
            float s = 0.f;
            for (int r = 0; r < 64; ++r) s += scr[scr_ix(r, tid)];
            F[F_CSM + tid] = s;
        }
        if (!products_done()) break;

        // ---- epilogue 4: dT = lower(beta_j dU V^T + beta_j gam_j dW K^T) (lanes 64-127)
        if (!lo) {
            float duv[32], dwk[32];
            tmem_ld32x2(tl + T_C2 + 64 + 32 * hf, tl + T_C4 + 32 * hf, duv, dwk);
            const float* trow = p.Tm + sh * kC * kC + (size_t)i * kC + 32 * hf;
            float dt[32];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                const float4 t4 = ldf4(trow + 4 * j4);
                const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int jj = 4 * j4 + e, j = 32 * hf + jj;
                    const float bj = be[j];
                    dt[jj] = j < i ? bj * duv[jj] + bj * gam[j] * dwk[jj] : 0.f;
                    const float tij = j <= i ? tv[e] : 0.f;
                    scr[scr_ix(i, j)] = tij * duv[jj];
                    scr[scr_ix(i, j + 64)] = tij * dwk[jj];
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) put8(sm, S_DT, kPanel64, i, 4 * hf + c, dt + 8 * c);
        }
        publish();

        // ---- round 5
        if (issuer) {
            tc_fence_after();
            // dv = (T diag(beta))^T dU (lanes 0-63)
            mma_run(tbase + T_C2, sb + S_TB, kPanel64, true, sb + S_DUO + 8192, kPanel128, true, ID_MM128, 4,
                    false);
            // M2 = T^T dT (lanes 0-63)
            mma_run(tbase + T_C4, sb + S_T, kPanel64, true, sb + S_DT, kPanel64, true, ID_MM64, 4, false);
            mma_commit(bar);
        }
        if (tid < 128) {
            const int j = tid & 63, qn = tid >> 6;
            float s = 0.f;
            for (int r = 0; r < 64; ++r) s += scr[scr_ix(r, j + 64 * qn)];
            F[(qn == 0 ? F_DBET : F_SKT) + j] = s;
        }
        if (!products_done()) break;

        // ---- epilogue 5: dv out; M2 into rows 64-127 of its tile (lanes 0-63)
        if (lo) {
            float* dvp = p.dv + ((size_t)(t0 + i) * p.Hv + h) * kD;
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float v[32];
                tmem_ld32(tl + T_C2 + c0, v);
                tmem_ld_wait();
                if (i < L) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4)
                        stf4(dvp + c0 + 4 * e4, v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
                }
            }
            float m2[32];
            tmem_ld32(tl + T_C4 + 32 * hf, m2);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) put8(sm, S_M2, kPanel64, 64 + i, 4 * hf + c, m2 + 8 * c);
        }
        publish();

        // ---- round 6: M2 T^T (lanes 64-127)
        if (issuer) {
            tc_fence_after();
            mma_run(tbase + T_C4, sb + S_M2, kPanel64, false, sb + S_T, kPanel64, false, ID_KK64, 4, false);
            mma_commit(bar);
        }
        if (!products_done()) break;

        // ---- epilogue 6: dA = -lower(M2 T^T); its sums with A' = lower(Gamma o K K^T); E (lanes 64-127)
        if (!lo) {
            float c4[32], kk[32];
            tmem_ld32x2(tl + T_C4 + 32 * hf, tl + T_D0 + 32 * hf, c4, kk);
            const float Gi = G[i], bi = be[i];
            float rs = 0.f;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                const int j = 32 * hf + jj;
                const bool below = j < i;
                const bool in = below && i < L;
                const float gm = in ? expf(Gi - G[j]) : 0.f;
                const float dA = below ? -c4[jj] : 0.f;
                const float x = dA * (kk[jj] * gm);
                rs += x;
                scr[scr_ix(i, j)] = x * bi;
                scr[scr_ix(i, j + 64)] = dA * bi * gm;
            }
            F[F_RSA + 64 * hf + i] = rs;
        }
        __syncthreads();
        // E + E^T
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int it = tid + kGThreads * x, r = it >> 3, ch = it & 7;
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int j = 8 * ch + e;
                v[e] = scr[scr_ix(r, j + 64)] + scr[scr_ix(j, r + 64)];
            }
            put8(sm, S_ES, kPanel64, r, ch, v);
        }
        publish();

        // ---- round 7: dk += (E + E^T) K
        if (issuer) {
            tc_fence_after();
            mma_run(tbase + T_C3, sb + S_ES, kPanel64, false, sb + S_KQW + 16384, kPanel192, true, ID_KM128, 4,
                    true);
            mma_commit(bar);
        }
        if (tid < 64) {
            float s = 0.f;
            for (int r = 0; r < 64; ++r) s += scr[scr_ix(r, tid)];
            F[F_CSA + tid] = s;
        }
        if (!products_done()) break;

        // ---- epilogue 7: dq, dk of this value head (lanes 0-63)
        if (lo) {
            const size_t o = ((size_t)(t0 + i) * p.Hv + h) * kD;
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float dk[32], dq[32];
                tmem_ld32x2(tl + T_C3 + c0, tl + T_C1 + c0, dk, dq);
                if (i < L) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        stf4(p.dkh + o + c0 + 4 * e4, dk[4 * e4], dk[4 * e4 + 1], dk[4 * e4 + 2], dk[4 * e4 + 3]);
                        stf4(p.dqh + o + c0 + 4 * e4, dq[4 * e4], dq[4 * e4 + 1], dq[4 * e4 + 2], dq[4 * e4 + 3]);
                    }
                }
            }
        }
        // the gates (warps 0-1, one row each): dG per row, then
        // d log alpha_m = sum_{i >= m} dG_i (a suffix scan), d a, d b, and the
        // chunk's sums for dA_log and ddt_bias (fixed reduction order)
        if (tid < kC) {
            const int r = tid;
            const float dkap = F[F_DKAP + r] + F[F_DKAP + 64 + r];
            const float sk = F[F_SKT + r];
            const float dgam = scale * (F[F_DGAM + r] + F[F_DGAM + 64 + r]) + be[r] * sk +
                               (r == L - 1 ? F[F_SS] : 0.f);
            const float rsa = F[F_RSA + r] + F[F_RSA + 64 + r];
            const float dbe = F[F_DBET + r] + gam[r] * sk + rsa;
            float dG = (F[F_RSM + r] + F[F_RSM + 64 + r] - F[F_CSM + r]) + (be[r] * rsa - F[F_CSA + r]) +
                       gam[r] * dgam - kap[r] * dkap;
            // sum over the chunk of kappa dkappa (rows >= L have kappa = 0) joins dG_{L-1}
            float kd = warp_sum(kap[r] * dkap);
            if (lane == 0) F[F_XCH + 2 + (r >> 5)] = kd;
            named_bar_sync(1, kC);
            if (r == L - 1) dG += F[F_XCH + 2] + F[F_XCH + 3];
            if (r >= L) dG = 0.f;
            // suffix scan (rows 63 .. 0): within the warp, then warp 0 adds warp 1's total
            float suf = dG;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const float o = __shfl_down_sync(0xffffffffu, suf, m);
                if (lane + m < 32) suf += o;
            }
            if (r == 32) F[F_XCH + 4] = suf;
            named_bar_sync(1, kC);
            if (r < 32) suf += F[F_XCH + 4];
            const float eA = expf(p.A_log[h]);
            const float dat = r < L ? suf * (-eA * F[F_SIG + r]) : 0.f;
            if (r < L) {
                const int64_t t = t0 + r;
                p.da[t * p.Hv + h] = dat;
                p.db[t * p.Hv + h] = dbe * be[r] * (1.f - be[r]);
            }
            const float gA = warp_sum(r < L ? suf * lg[r] : 0.f);
            const float gD = warp_sum(dat);
            if (lane == 0) {
                F[F_XCH + 5 + (r >> 5)] = gA;
                F[F_XCH + 7 + (r >> 5)] = gD;
            }
            named_bar_sync(1, kC);
            if (r == 0) {
                p.gpart[sh * 2 + 0] = F[F_XCH + 5] + F[F_XCH + 6];
                p.gpart[sh * 2 + 1] = F[F_XCH + 7] + F[F_XCH + 8];
            }
        }
    } while (false);

    // ---- teardown: every product is complete (or the wait for them gave up)
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (tid == 0) {
            *reinterpret_cast<volatile uint32_t*>(p.err) = 1u;
            volatile int no_abort = 0;
            mma_commit(bar);
            mbar_wait(bar, (uint32_t)(phase & 1), &no_abort, kWaitLimitNs);
        }
        __syncthreads();
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_backward_grad_tc(const Params& p, int64_t jobs, cudaStream_t s) {
    if (jobs <= 0) return cudaSuccess;
    if (jobs > 0x7fffffff) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(bwc_grad_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    bwc_grad_tc_kernel<<<(unsigned)jobs, kGThreads, SMEM_ALLOC, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
