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
// warps per (chunk, value head); the products come in seven phases, each issued
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

// 16-byte cp.async (src_bytes < 16 zero-fills the rest), its groups
TC_DEVICE void cp_async16z(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
TC_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
TC_DEVICE void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// scratch: quantity 0 in columns 0-63, quantity 1 in 64-127, rotated by the row
// (conflict-free both for a thread per row and for a thread per column)
TC_DEVICE int scr_ix(int i, int j) { return i * 128 + ((j + i) & 127); }
// column j of the scratch summed over its 64 rows (four partial sums, fixed order)
TC_DEVICE float col_sum(const float* scr, int j) {
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 4
    for (int r = 0; r < 64; r += 4) {
        s0 += scr[scr_ix(r, j)];
        s1 += scr[scr_ix(r + 1, j)];
        s2 += scr[scr_ix(r + 2, j)];
        s3 += scr[scr_ix(r + 3, j)];
    }
    return (s0 + s1) + (s2 + s3);
}

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
    // gate inputs (threads 0-63, one row each), requested before the operands
    float g_a = 0.f, g_b = 0.f;
    if (tid < kC && tid < L) {
        const int64_t t = t0 + tid;
        g_a = p.a[t * p.Hv + h];
        g_b = p.b[t * p.Hv + h];
    }

    // ---- stage the operands -------------------------------------------------------------
    // By cp.async straight into their tiles: K, Q, V (bf16 inputs; rows >= L
    // zero-filled), and S, dS and W, which the chains and the preparation wrote
    // as bf16 tiles in this very layout.  dO and T (float32) through registers.
    {
        const uint8_t* Sg = reinterpret_cast<const uint8_t*>(p.S + sh * kD * kD);
        const uint8_t* dSg = reinterpret_cast<const uint8_t*>(p.dS + sh * kD * kD);
        const uint8_t* Wg = reinterpret_cast<const uint8_t*>(p.W + sh * kC * kD);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            const bool ok = r < L;
            const uint32_t z = ok ? 16u : 0u;
            const size_t kq = ((size_t)(t0 + r) * p.Hqk + g) * kD + ch * 8;
            const uint32_t off = (uint32_t)(ch >> 3) * kPanel192;
            cp_async16z(sb + S_KQW + off + sw128_off(128 + r, ch & 7), ok ? p.k + kq : p.k, z);
            cp_async16z(sb + S_KQW + off + sw128_off(64 + r, ch & 7), ok ? p.q + kq : p.q, z);
            cp_async16z(sb + S_UV + (uint32_t)(ch >> 3) * kPanel128 + sw128_off(64 + r, ch & 7),
                        ok ? p.v + ((size_t)(t0 + r) * p.Hv + h) * kD + ch * 8 : p.v, z);
            // W rows 0-63: the tile's panels are 8 KB apart, the [W; Q; K] tile's 24 KB
            cp_async16z(sb + S_KQW + off + sw128_off(r, ch & 7), Wg + (ch >> 3) * kPanel64 + sw128_off(r, ch & 7), 16u);
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            const uint32_t o = (uint32_t)(tid + kGThreads * x) * 16u;
            cp_async16z(sb + S_S + o, Sg + o, 16u);
            cp_async16z(sb + S_DS + o, dSg + o, 16u);
        }
        cp_async_commit();
    }
    {
        float4 ox[4][2], tx[2][2];
        const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
        const float* Tg = p.Tm + sh * kC * kC;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            const bool ok = r < L;
            const float* op = p.d_o + ((size_t)(t0 + r) * p.Hv + h) * kD + ch * 8;
            ox[x][0] = ok ? ldf4(op) : zf;
            ox[x][1] = ok ? ldf4(op + 4) : zf;
        }
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
    // gates (warps 0-1, one row each): log alpha, beta, G = running sum of log
    // alpha (an inclusive scan; rows >= L add 0, so they carry G_{L-1}), gamma,
    // kappa, and sigmoid(a + dt_bias) for d a
    if (tid < kC) {
        const int r = tid;
        float la = 0.f, bb = 0.f, sg = 0.f;
        if (r < L) {
            const float dtb = p.dt_bias[h];
            la = log_alpha(g_a, p.A_log[h], dtb);
            bb = sigmoid(g_b);
            sg = sigmoid(g_a + dtb);
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
    cp_async_wait<0>();
    // <dS, S> over the state (this thread's own 16-byte pieces of the two tiles)
    {
        float ss = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            const uint32_t o = (uint32_t)(tid + kGThreads * x) * 16u;
            const uint4 a4 = *reinterpret_cast<const uint4*>(sm + S_S + o);
            const uint4 b4 = *reinterpret_cast<const uint4*>(sm + S_DS + o);
            const uint32_t av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const float2 sa = bf16x2_to_f32x2(av[y]), sd = bf16x2_to_f32x2(bv[y]);
                ss = fmaf(sa.x, sd.x, fmaf(sa.y, sd.y, ss));
            }
        }
        ss = warp_sum(ss);
        if (lane == 0) F[F_RED + warp] = ss;
    }
    fence_async_smem();
    tc_fence_before();
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
        // ---- phase 1
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
            for (int x = 0; x < kGThreads / 32; ++x) s += F[F_RED + x];
            F[F_SS] = s;
        }
        // epilogue 1's rows from global memory, requested while the products run:
        // U' (lanes 0-63) or dO (lanes 64-127), columns 64 hf .. + 64
        float4 pre[16];
        {
            const bool ok = lo || i < L;
            const float* src = lo ? p.Up + sh * kC * kD + (size_t)i * kD + 64 * hf
                                  : p.d_o + ((size_t)(t0 + (ok ? i : 0)) * p.Hv + h) * kD + 64 * hf;
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) pre[c4] = ok ? ldf4(src + 4 * c4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (!products_done()) break;

        // ---- epilogue 1: U, kappa U, P (lanes 0-63); the gamma sums (lanes 64-127)
        if (lo) {
            const float ki = kap[i];
            float r1 = 0.f;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float x1[32], kd[32];
                tmem_ld32x2(tl + T_C1 + c0, tl + T_C2 + c0, x1, kd);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) {
                    const float4 a = pre[8 * cb + 2 * j8], b = pre[8 * cb + 2 * j8 + 1];
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
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float qs[32];
                tmem_ld32(tl + T_C1 + c0, qs);
                tmem_ld_wait();
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 o4 = pre[8 * cb + e4];
                    r2 = fmaf(o4.x, qs[4 * e4], r2);
                    r2 = fmaf(o4.y, qs[4 * e4 + 1], r2);
                    r2 = fmaf(o4.z, qs[4 * e4 + 2], r2);
                    r2 = fmaf(o4.w, qs[4 * e4 + 3], r2);
                }
            }
            F[F_DGAM + 64 * hf + i] = r2;
        }
        publish();

        // ---- phase 2: P^T dO (lanes 0-63)
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

        // ---- phase 3
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
            // T diag(beta) and T diag(beta gam) (over kappa U, read by phase 3)
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

        // ---- phase 4
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
        if (tid < 64) F[F_CSM + tid] = col_sum(scr, tid);
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

        // ---- phase 5
        if (issuer) {
            tc_fence_after();
            // dv = (T diag(beta))^T dU (lanes 0-63)
            mma_run(tbase + T_C2, sb + S_TB, kPanel64, true, sb + S_DUO + 8192, kPanel128, true, ID_MM128, 4,
                    false);
            // M2 = T^T dT (lanes 0-63)
            mma_run(tbase + T_C4, sb + S_T, kPanel64, true, sb + S_DT, kPanel64, true, ID_MM64, 4, false);
            mma_commit(bar);
        }
        if (tid < 128) F[(tid < 64 ? F_DBET : F_SKT) + (tid & 63)] = col_sum(scr, tid);
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

        // ---- phase 6: M2 T^T (lanes 64-127)
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

        // ---- phase 7: dk += (E + E^T) K
        if (issuer) {
            tc_fence_after();
            mma_run(tbase + T_C3, sb + S_ES, kPanel64, false, sb + S_KQW + 16384, kPanel192, true, ID_KM128, 4,
                    true);
            mma_commit(bar);
        }
        if (tid < 64) F[F_CSA + tid] = col_sum(scr, tid);
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

// ---- the per-chunk preparation on the tensor cores ---------------------------------------
// One CTA of 8 warps per (chunk, value head): the quantities the chains and the
// gradient step read, as prep_block in backward_chunked.cuh computes them:
//   phase 1  D0 = [Q; K] K^T                 -> P = lower(Gamma o Q K^T) (bf16),
//                                               A = diag(beta) strict_lower(Gamma o K K^T) (f32)
//   solve    T = (I + A)^{-1}: 16 x 16 diagonal blocks by forward substitution,
//            then 32 x 32 and 64 x 64 by T10 = -T11 A10 T00 (float32, CUDA cores)
//   phase 2  W = (T diag(beta)) (diag(gam) K), U' = (T diag(beta)) V, Z = P^T dO
//   phase 3  Y / scale = dO^T (diag(gam) Q) - Z^T W
constexpr uint32_t R_QK = 0;                        // [Q; K]             128 x 128
constexpr uint32_t R_V = R_QK + 2 * kPanel128;      // V                  64 x 128
constexpr uint32_t R_DO = R_V + 2 * kPanel64;       // dO (bf16)          64 x 128
constexpr uint32_t R_GK = R_DO + 2 * kPanel64;      // diag(gam) K        64 x 128
constexpr uint32_t R_GQ = R_GK + 2 * kPanel64;      // diag(gam) Q        64 x 128
constexpr uint32_t R_Z = R_GQ + 2 * kPanel64;       // -Z                 64 x 128
constexpr uint32_t R_W = R_Z + 2 * kPanel64;        // W (also the workspace's copy) 64 x 128
constexpr uint32_t R_P = R_W + 2 * kPanel64;        // P                  64 x 64
constexpr uint32_t R_TB = R_P + kPanel64;           // T diag(beta)       64 x 64
constexpr uint32_t R_PAD = R_TB + kPanel64;         // (rows 64-127 of the M = 128 reads of T diag(beta))
constexpr uint32_t R_AF = R_PAD + kPanel64;         // A, f32             64 x 65
constexpr uint32_t R_TF = R_AF + 64 * 65 * 4;       // T, f32             64 x 65
constexpr uint32_t R_XF = R_TF + 64 * 65 * 4;       // solve scratch, f32 64 x 65
constexpr uint32_t R_MISC = R_XF + 64 * 65 * 4;     // gates, exchange
constexpr uint32_t R_BAR = R_MISC + 400 * 4;
constexpr uint32_t PREP_SMEM_ALLOC = R_BAR + 16 + 1024;
static_assert(R_BAR % 8 == 0, "mbarrier alignment");
static_assert(PREP_SMEM_ALLOC <= 232448, "shared memory budget of one CTA");
constexpr uint32_t PT_D0 = 0, PT_W = 64, PT_U = 192, PT_Z = 320, PT_Y = 64;

__global__ void __launch_bounds__(kGThreads, 1) bwc_prep_tc_kernel(Params p) {
    extern __shared__ uint8_t bwt_prep_smem_raw[];
    uint8_t* sm =
        reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bwt_prep_smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t slot = blockIdx.x / p.Hv;
    const int h = blockIdx.x % p.Hv;
    const size_t sh = sh_index(p, slot, h);
    const int n = p.jobs[2 * slot];
    if (n < 0) {
        if (tid < 2) p.gpart[sh * 2 + tid] = 0.f;
        return;
    }
    const int64_t t0 = p.jobs[2 * slot + 1];
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int L = (int)((eos - t0) < kC ? (eos - t0) : kC);
    const int g = h / (p.Hv / p.Hqk);

    float* F = reinterpret_cast<float*>(sm + R_MISC);
    float *be = F, *G = F + 64, *gam = F + 128, *kap = F + 192, *xch = F + 256;
    float* Af = reinterpret_cast<float*>(sm + R_AF);
    float* Tf = reinterpret_cast<float*>(sm + R_TF);
    float* Xf = reinterpret_cast<float*>(sm + R_XF);
    constexpr int kLf = 65;
    const uint32_t bar = sb + R_BAR;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + R_BAR + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + R_BAR + 12);
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tc_fence_before();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    // gates (warps 0-1): beta, G, gamma, kappa
    if (tid < kC) {
        const int r = tid;
        float la = 0.f, bb = 0.f;
        if (r < L) {
            const int64_t t = t0 + r;
            la = log_alpha(p.a[t * p.Hv + h], p.A_log[h], p.dt_bias[h]);
            bb = sigmoid(p.b[t * p.Hv + h]);
        }
        float run = la;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, run, m);
            if (lane >= m) run += o;
        }
        if (r == 31) xch[0] = run;
        named_bar_sync(1, kC);
        if (r >= 32) run += xch[0];
        be[r] = bb;
        G[r] = run;
        gam[r] = expf(run);
        named_bar_sync(1, kC);
        kap[r] = r < L ? expf(G[L - 1] - run) : 0.f;
    }
    // operands: [Q; K], V, dO (rows >= L zero)
    {
        uint4 kx[4], qx[4], vx[4];
        float4 ox[4][2];
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        const float4 zf = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            const bool ok = r < L;
            kx[x] = ok ? ldu4(p.k + ((size_t)(t0 + r) * p.Hqk + g) * kD + ch * 8) : z4;
            qx[x] = ok ? ldu4(p.q + ((size_t)(t0 + r) * p.Hqk + g) * kD + ch * 8) : z4;
            vx[x] = ok ? ldu4(p.v + ((size_t)(t0 + r) * p.Hv + h) * kD + ch * 8) : z4;
            const float* op = p.d_o + ((size_t)(t0 + r) * p.Hv + h) * kD + ch * 8;
            ox[x][0] = ok ? ldf4(op) : zf;
            ox[x][1] = ok ? ldf4(op + 4) : zf;
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            st16(sm, R_QK, kPanel128, r, ch, qx[x]);
            st16(sm, R_QK, kPanel128, 64 + r, ch, kx[x]);
            st16(sm, R_V, kPanel64, r, ch, vx[x]);
            st16(sm, R_DO, kPanel64, r, ch, pack8(ox[x][0], ox[x][1]));
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const bool issuer = tid == 0;
    const int q = warp & 3, hf = warp >> 2;
    const uint32_t tl = tbase + ((uint32_t)(32 * q) << 16);
    const bool lo = q < 2;
    const int i = 32 * (q & 1) + lane;
    int phase = 0;
    auto products_done = [&]() -> bool {
        mbar_wait(bar, (uint32_t)(phase & 1), abort_flag, kWaitLimitNs);
        ++phase;
        __syncthreads();
        tc_fence_after();
        return *abort_flag == 0;
    };
    auto publish = [&]() {
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
    };

    do {
        // ---- phase 1: D0 = [Q; K] K^T (lanes 0-63 Q K^T, 64-127 K K^T)
        if (issuer) {
            tc_fence_after();
            mma_run(tbase + PT_D0, sb + R_QK, kPanel128, false, sb + R_QK + 8192, kPanel128, false, ID_KK64, 8,
                    false);
            mma_commit(bar);
        }
        // meanwhile: T's scratch cleared (the solve reads its zero upper blocks);
        // diag(gam) K and diag(gam) Q (from the staged tiles)
        for (int x = tid; x < 64 * kLf; x += kGThreads) Tf[x] = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            float kv[8], qv[8];
            tile::ld_bf16x8(sm + R_QK + (ch >> 3) * kPanel128, 64 + r, ch & 7, kv);
            tile::ld_bf16x8(sm + R_QK + (ch >> 3) * kPanel128, r, ch & 7, qv);
            const float gr = gam[r];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                kv[e] *= gr;
                qv[e] *= gr;
            }
            put8(sm, R_GK, kPanel64, r, ch, kv);
            put8(sm, R_GQ, kPanel64, r, ch, qv);
        }
        if (!products_done()) break;
        // ---- epilogue 1: P (lanes 0-63), A (lanes 64-127); each warp 32 columns
        {
            float d[32];
            tmem_ld32(tl + PT_D0 + 32 * hf, d);
            tmem_ld_wait();
            const float Gi = G[i];
            if (lo) {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = 32 * hf + jj;
                    d[jj] = (j <= i && i < L) ? d[jj] * expf(Gi - G[j]) : 0.f;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) put8(sm, R_P, kPanel64, i, 4 * hf + c, d + 8 * c);
            } else {
                const float bi = be[i];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = 32 * hf + jj;
                    Af[i * kLf + j] = (j < i && i < L) ? bi * d[jj] * expf(Gi - G[j]) : 0.f;
                }
            }
        }
        __syncthreads();
        // ---- T = (I + A)^{-1}, unit lower triangular
        // 16 x 16 diagonal blocks: warp b, lane c < 16 holds column c
        if (warp < 4) {
            const int b0 = 16 * warp, c = lane & 15;
            float xv[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m) acc = fmaf(Af[(b0 + r) * kLf + b0 + m], xv[m], acc);
                xv[r] = (r == c ? 1.f : 0.f) - acc;
            }
            if (lane < 16) {
#pragma unroll
                for (int r = 0; r < 16; ++r) Tf[(b0 + r) * kLf + b0 + c] = xv[r];
            }
        }
        __syncthreads();
        // 32 x 32 blocks (rows and columns 0-31, 32-63): T[R1][R0] = -T[R1][R1] A[R1][R0] T[R0][R0]
        {
            const int blk = tid >> 7, e = tid & 127;            // two elements of a 16 x 16 block each
            const int R0 = 32 * blk, R1 = R0 + 16;
            const int r = e >> 3, c0 = (e & 7) * 2;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int c = c0 + x;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) acc = fmaf(Af[(R1 + r) * kLf + R0 + m], Tf[(R0 + m) * kLf + R0 + c], acc);
                Xf[(R1 + r) * kLf + R0 + c] = acc;
            }
            __syncthreads();
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int c = c0 + x;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) acc = fmaf(Tf[(R1 + r) * kLf + R1 + m], Xf[(R1 + m) * kLf + R0 + c], acc);
                Tf[(R1 + r) * kLf + R0 + c] = -acc;
            }
        }
        __syncthreads();
        // 64 x 64: T[32:64][0:32] = -T[32:64][32:64] A[32:64][0:32] T[0:32][0:32]; four elements each
        {
            const int r = tid >> 3, c0 = (tid & 7) * 4;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int m = 0; m < 32; ++m) {
                const float av = Af[(32 + r) * kLf + m];
#pragma unroll
                for (int x = 0; x < 4; ++x) acc[x] = fmaf(av, Tf[m * kLf + c0 + x], acc[x]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) Xf[(32 + r) * kLf + c0 + x] = acc[x];
            __syncthreads();
#pragma unroll
            for (int x = 0; x < 4; ++x) acc[x] = 0.f;
#pragma unroll 8
            for (int m = 0; m < 32; ++m) {
                const float tv = Tf[(32 + r) * kLf + 32 + m];
#pragma unroll
                for (int x = 0; x < 4; ++x) acc[x] = fmaf(tv, Xf[(32 + m) * kLf + c0 + x], acc[x]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) Tf[(32 + r) * kLf + c0 + x] = -acc[x];
        }
        __syncthreads();
        // T out (f32, zeros above the diagonal) and T diag(beta) (bf16)
        {
            float* Tg = p.Tm + sh * kC * kC;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int it = tid + kGThreads * x, r = it >> 3, ch = it & 7;
                float tv[8], tb[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int c = 8 * ch + e;
                    tv[e] = c <= r ? Tf[r * kLf + c] : 0.f;
                    tb[e] = tv[e] * be[c];
                }
                stf4(Tg + r * kC + 8 * ch, tv[0], tv[1], tv[2], tv[3]);
                stf4(Tg + r * kC + 8 * ch + 4, tv[4], tv[5], tv[6], tv[7]);
                put8(sm, R_TB, kPanel64, r, ch, tb);
            }
            if (tid <= kC) p.G[sh * (kC + 1) + tid] = tid < kC ? kap[tid] : gam[L - 1];
        }
        publish();
        // ---- phase 2: W, U' (A = T diag(beta), K-major), Z = P^T dO (lanes 0-63)
        if (issuer) {
            tc_fence_after();
            mma_run(tbase + PT_W, sb + R_TB, kPanel64, false, sb + R_GK, kPanel64, true, ID_KM128, 4, false);
            mma_run(tbase + PT_U, sb + R_TB, kPanel64, false, sb + R_V, kPanel64, true, ID_KM128, 4, false);
            mma_run(tbase + PT_Z, sb + R_P, kPanel64, true, sb + R_DO, kPanel64, true, ID_MM128, 4, false);
            mma_commit(bar);
        }
        if (!products_done()) break;
        // ---- epilogue 2 (lanes 0-63): U' out (f32); W (bf16, the operand
        //      layout the chains and the gradient step copy as is) and -Z
        if (lo) {
            float* Ug = p.Up + sh * kC * kD + (size_t)i * kD;
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float w[32], u[32];
                tmem_ld32x2(tl + PT_W + c0, tl + PT_U + c0, w, u);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4)
                    stf4(Ug + c0 + 4 * e4, u[4 * e4], u[4 * e4 + 1], u[4 * e4 + 2], u[4 * e4 + 3]);
#pragma unroll
                for (int c = 0; c < 4; ++c) put8(sm, R_W, kPanel64, i, c0 / 8 + c, w + 8 * c);
                float z[32];
                tmem_ld32(tl + PT_Z + c0, z);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) z[e] = -z[e];
#pragma unroll
                for (int c = 0; c < 4; ++c) put8(sm, R_Z, kPanel64, i, c0 / 8 + c, z + 8 * c);
            }
        }
        publish();
        // ---- phase 3: Y / scale = dO^T (diag(gam) Q) + (-Z)^T W (all 128 lanes: rows e)
        if (issuer) {
            tc_fence_after();
            mma_run(tbase + PT_Y, sb + R_DO, kPanel64, true, sb + R_GQ, kPanel64, true, ID_MM128, 4, false);
            mma_run(tbase + PT_Y, sb + R_Z, kPanel64, true, sb + R_W, kPanel64, true, ID_MM128, 4, true);
            mma_commit(bar);
            // the W tile to the workspace (16 KB, read by the async proxy after the fence above)
            bulk_store(p.W + sh * kC * kD, sb + R_W, 2 * kPanel64);
            bulk_commit();
        }
        if (!products_done()) break;
        {
            const int e = 32 * q + lane;
            float* Yg = p.Y + sh * kD * kD + (size_t)e * kD;
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hf + 32 * cb;
                float y[32];
                tmem_ld32(tl + PT_Y + c0, y);
                tmem_ld_wait();
#pragma unroll
                for (int f4 = 0; f4 < 8; ++f4)
                    stf4(Yg + c0 + 4 * f4, p.scale * y[4 * f4], p.scale * y[4 * f4 + 1], p.scale * y[4 * f4 + 2],
                         p.scale * y[4 * f4 + 3]);
            }
        }
    } while (false);

    if (tid == 0) bulk_wait();
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

// ---- the two state chains on the tensor cores -------------------------------------------
// One CTA of 8 warps per (sequence, value head).  The state (S forward, dS
// backward; float32) stays in registers: thread (warp w, lane l) holds row
// 32 (w % 4) + l, columns 64 (w / 4) .. + 64.  Per chunk, two products:
//   forward   X = W S^T (rows i = tokens), U = kappa (U' - X) (bf16),
//             dS~ = U^T K;   S <- gamma_L S + dS~
//   backward  X = K dS^T (rows i), X <- kappa X (bf16), dS~ = X^T W;
//             dS <- gamma_L dS + Y - dS~
// Both products take the bf16 state as their operand; the chain itself is
// carried in float32.  The chunk's state checkpoint is that bf16 operand tile,
// written out by one bulk copy (the gradient step copies it back as is).  The
// next chunk's operands are requested a whole chunk ahead: K, W (the
// preparation's bf16 tile) and U' (forward) into the other half of double
// buffers by cp.async, the decays through registers; Y (backward, 64 KB) by
// cp.async at the start of the chunk that reads it at its end.
constexpr uint32_t C_ST = 0;                        // the state, bf16       128 x 128
constexpr uint32_t C_WT = C_ST + 2 * kPanel128;     // W, bf16, 2 buffers    64 x 128
constexpr uint32_t C_KT = C_WT + 4 * kPanel64;      // K, bf16, 2 buffers    64 x 128
constexpr uint32_t C_XT = C_KT + 4 * kPanel64;      // kappa U or kappa X    64 x 128
constexpr uint32_t C_BUF = C_XT + 2 * kPanel64;     // U' (2 buffers of 64 rows) or Y (128 rows), f32
constexpr int kBufLd = 132;                         // floats per row (16-byte rows, conflict-free float4 reads)
constexpr uint32_t kBufHalf = 64 * kBufLd * 4;
constexpr uint32_t C_MISC = C_BUF + 2 * kBufHalf;   // kappa [64] and gamma_L, 2 buffers of 68
constexpr uint32_t C_BAR = C_MISC + 2 * 68 * 4;     // mbarrier (8), TMEM base (4), abort flag (4)
constexpr uint32_t CH_SMEM_ALLOC = C_BAR + 16 + 1024;
static_assert(C_BAR % 8 == 0, "mbarrier alignment");
constexpr uint32_t CT_X = 0, CT_D = 128, kChainTmemCols = 256;


template <bool kBwd>
__global__ void __launch_bounds__(kGThreads, 1) bwc_chain_tc_kernel(Params p) {
    extern __shared__ uint8_t bwt_chain_smem_raw[];
    uint8_t* sm =
        reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bwt_chain_smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x / p.Hv, h = blockIdx.x % p.Hv;
    const int g = h / (p.Hv / p.Hqk);
    int64_t bos, eos;
    seq_bounds(p, n, bos, eos);
    const int64_t nch = (eos - bos + kC - 1) / kC;
    const int q = warp & 3, hf = warp >> 2;
    const int row = 32 * q + lane;                   // state row (TMEM lane) of this thread
    const size_t unit = ((size_t)n * p.Hv + h) * kD * kD + (size_t)row * kD + 64 * hf;
    float st[64];
    {
        const float* init = kBwd ? p.d_fin : p.s0;
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
            const float4 v = init ? ldf4(init + unit + 4 * c4) : make_float4(0.f, 0.f, 0.f, 0.f);
            st[4 * c4] = v.x; st[4 * c4 + 1] = v.y; st[4 * c4 + 2] = v.z; st[4 * c4 + 3] = v.w;
        }
    }
    if (nch == 0) {
        if (kBwd && p.d_init) {
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4)
                stf4(p.d_init + unit + 4 * c4, st[4 * c4], st[4 * c4 + 1], st[4 * c4 + 2], st[4 * c4 + 3]);
        }
        return;
    }
    float* misc = reinterpret_cast<float*>(sm + C_MISC);
    const uint32_t bar = sb + C_BAR;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C_BAR + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C_BAR + 12);
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kChainTmemCols);
        tc_fence_before();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        *abort_flag = 0;
    }

    // chunk jj of the walk (backward: from the last)
    auto chunk_t0 = [&](int64_t jj) -> int64_t { return bos + (kBwd ? nch - 1 - jj : jj) * kC; };
    auto slot_of = [&](int64_t t0) -> size_t { return sh_index(p, t0 / kC + n, h); };
    auto fetch_k = [&](int64_t t0, int b) {
        const int Lc = (int)((eos - t0) < kC ? (eos - t0) : kC);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int it = tid + kGThreads * x, r = it >> 4, ch = it & 15;
            const bool ok = r < Lc;
            const uint16_t* src = ok ? p.k + ((size_t)(t0 + r) * p.Hqk + g) * kD + ch * 8 : p.k;
            cp_async16z(sb + C_KT + (uint32_t)b * 2 * kPanel64 + (uint32_t)(ch >> 3) * kPanel64 + sw128_off(r, ch & 7),
                        src, ok ? 16u : 0u);
        }
    };
    // U' (forward, 64 rows, into buffer b) or Y (backward, 128 rows)
    auto fetch_buf = [&](int64_t t0, int b) {
        const size_t sh = slot_of(t0);
        const float* src = kBwd ? p.Y + sh * kD * kD : p.Up + sh * kC * kD;
        const uint32_t base = sb + C_BUF + (kBwd ? 0u : (uint32_t)b * kBufHalf);
        constexpr int kItems = (kBwd ? 128 : 64) * 32 / kGThreads;
#pragma unroll
        for (int x = 0; x < kItems; ++x) {
            const int it = tid + kGThreads * x, r = it >> 5, pc = it & 31;
            cp_async16z(base + (uint32_t)(r * kBufLd + 4 * pc) * 4u, src + (size_t)r * kD + 4 * pc, 16u);
        }
    };
    // W: the preparation's bf16 tile (16 KB, the shared-memory image) into buffer b
    auto fetch_w = [&](int64_t t0, int b) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(p.W + slot_of(t0) * kC * kD);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const uint32_t off = (uint32_t)(tid + kGThreads * x) * 16u;
            cp_async16z(sb + C_WT + (uint32_t)b * 2 * kPanel64 + off, src + off, 16u);
        }
    };
    // kappa_0..63 and gamma_L of a chunk (threads 0..64)
    auto load_gate = [&](int64_t t0) -> float { return tid <= kC ? p.G[slot_of(t0) * (kC + 1) + tid] : 0.f; };

    // prologue: chunk 0's operands
    {
        const int64_t t0 = chunk_t0(0);
        fetch_k(t0, 0);
        fetch_w(t0, 0);
        if (!kBwd) fetch_buf(t0, 0);
        cp_async_commit();
        const float gv = load_gate(t0);
        if (tid <= kC) misc[tid] = gv;
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(32 * q) << 16);
    int phase = 0;
    auto products_done = [&]() -> bool {
        mbar_wait(bar, (uint32_t)(phase & 1), abort_flag, kWaitLimitNs);
        ++phase;
        __syncthreads();
        tc_fence_after();
        return *abort_flag == 0;
    };

    for (int64_t jj = 0; jj < nch; ++jj) {
        const int b = (int)(jj & 1);
        const int64_t t0 = chunk_t0(jj);
        const size_t sh = slot_of(t0);
        const bool more = jj + 1 < nch;
        const int64_t t0n = more ? chunk_t0(jj + 1) : t0;
        const float* kap = misc + 68 * b;
        // requests for later: Y of this chunk (backward), the next chunk's K (and U')
        if (kBwd) {
            fetch_buf(t0, 0);
            cp_async_commit();
        }
        if (more) {
            fetch_k(t0n, b ^ 1);
            fetch_w(t0n, b ^ 1);
            if (!kBwd) fetch_buf(t0n, b ^ 1);
            cp_async_commit();
        }
        const float gnext = more ? load_gate(t0n) : 0.f;
        // the state at this chunk's start (forward) or end (backward) as the bf16
        // operand (its previous bulk copy out has been read: see the end of the loop)
#pragma unroll
        for (int j = 0; j < 8; ++j) put8(sm, C_ST, kPanel128, row, 8 * hf + j, st + 8 * j);
        // this chunk's K (and U') have landed; the requests just made may be in flight
        if (kBwd) {
            if (more) cp_async_wait<2>();
            else cp_async_wait<1>();
        } else {
            if (more) cp_async_wait<1>();
            else cp_async_wait<0>();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        const uint32_t kt = sb + C_KT + (uint32_t)b * 2 * kPanel64;
        const uint32_t wt = sb + C_WT + (uint32_t)b * 2 * kPanel64;
        if (tid == 0) {
            tc_fence_after();
            // X = W S^T (forward) or K dS^T (backward): rows i in TMEM lanes 0-63
            mma_run(tbase + CT_X, kBwd ? kt : wt, kPanel64, false, sb + C_ST, kPanel128, false, ID_KK128, 8, false);
            mma_commit(bar);
            // the state checkpoint: the bf16 operand tile (32 KB) to the workspace
            bulk_store(kBwd ? p.dS + sh * kD * kD : p.S + sh * kD * kD, sb + C_ST, 2 * kPanel128);
            bulk_commit();
        }
        if (!products_done()) break;
        if (q < 2) {
            const int i = row;
            const float ki = kap[i];
#pragma unroll 1
            for (int hb = 0; hb < 2; ++hb) {
                const int c0 = 64 * hf + 32 * hb;
                float x[32];
                tmem_ld32(tl + CT_X + c0, x);
                tmem_ld_wait();
                if (!kBwd) {
                    const float* up = reinterpret_cast<const float*>(sm + C_BUF + (uint32_t)b * kBufHalf) + i * kBufLd + c0;
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 u4 = ldf4(up + 4 * e4);
                        x[4 * e4] = ki * (u4.x - x[4 * e4]);
                        x[4 * e4 + 1] = ki * (u4.y - x[4 * e4 + 1]);
                        x[4 * e4 + 2] = ki * (u4.z - x[4 * e4 + 2]);
                        x[4 * e4 + 3] = ki * (u4.w - x[4 * e4 + 3]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= ki;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) put8(sm, C_XT, kPanel64, i, c0 / 8 + j, x + 8 * j);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // dS~ = (kappa U)^T K (forward) or (kappa X)^T W (backward): A and B
            // MN-major (rows = tokens)
            mma_run(tbase + CT_D, sb + C_XT, kPanel64, true, kBwd ? wt : kt, kPanel64, true, ID_MM128, 4, false);
            mma_commit(bar);
        }
        if (kBwd) {
            // this chunk's Y (the next chunk's K may still be in flight); the
            // barrier in products_done makes every thread's part visible
            if (more) cp_async_wait<1>();
            else cp_async_wait<0>();
        }
        if (!products_done()) break;
        {
            const float gL = kap[kC];
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                float d[32];
                tmem_ld32(tl + CT_D + 64 * hf + 32 * hb, d);
                tmem_ld_wait();
                float* s32 = st + 32 * hb;
                if (!kBwd) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) s32[e] = fmaf(gL, s32[e], d[e]);
                } else {
                    const float* y = reinterpret_cast<const float*>(sm + C_BUF) + row * kBufLd + 64 * hf + 32 * hb;
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 y4 = ldf4(y + 4 * e4);
                        s32[4 * e4] = fmaf(gL, s32[4 * e4], y4.x) - d[4 * e4];
                        s32[4 * e4 + 1] = fmaf(gL, s32[4 * e4 + 1], y4.y) - d[4 * e4 + 1];
                        s32[4 * e4 + 2] = fmaf(gL, s32[4 * e4 + 2], y4.z) - d[4 * e4 + 2];
                        s32[4 * e4 + 3] = fmaf(gL, s32[4 * e4 + 3], y4.w) - d[4 * e4 + 3];
                    }
                }
            }
        }
        // the state tile's copy out has been read before the next chunk rewrites it
        if (tid == 0) bulk_wait_read();
        tc_fence_before();
        __syncthreads();
        // every read of this chunk's decays is done: the next chunk's take their place
        if (more && tid <= kC) misc[68 * (b ^ 1) + tid] = gnext;
    }
    if (kBwd && p.d_init && *abort_flag == 0) {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4)
            stf4(p.d_init + unit + 4 * c4, st[4 * c4], st[4 * c4 + 1], st[4 * c4 + 2], st[4 * c4 + 3]);
    }
    cp_async_wait<0>();
    if (tid == 0) bulk_wait();
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
        tmem_dealloc(tbase, kChainTmemCols);
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

cudaError_t launch_backward_prep_tc(const Params& p, int64_t jobs, cudaStream_t s) {
    if (jobs <= 0) return cudaSuccess;
    if (jobs > 0x7fffffff) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(bwc_prep_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PREP_SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    bwc_prep_tc_kernel<<<(unsigned)jobs, kGThreads, PREP_SMEM_ALLOC, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_backward_chains_tc(const Params& p, int64_t units, bool backward, cudaStream_t s) {
    if (units <= 0) return cudaSuccess;
    if (units > 0x7fffffff) return cudaErrorInvalidValue;
    auto kernel = backward ? bwc_chain_tc_kernel<true> : bwc_chain_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CH_SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)units, kGThreads, CH_SMEM_ALLOC, s>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
