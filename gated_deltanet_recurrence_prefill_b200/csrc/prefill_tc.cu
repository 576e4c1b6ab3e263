// prefill_tc.cu -- chunked gated delta-rule prefill on the sm_100a tensor cores.
//
// The recurrence (Qwen3.8-27B architecture page, 2kiu.com, section 2.2, with
// the decay alpha on the erased state):
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
//     o_t = scale * S_t q_t,
// is computed in chunks of C = 64 tokens.  With G the running sum of
// log2(alpha) inside the chunk, gamma = 2^G, kappa = 2^{G_C - G} and S the
// state at the chunk start (WY / UT form):
//     A_ij = beta_i 2^{G_i - G_j} k_i.k_j  (j < i)      T = (I + A)^{-1}
//     P_ij = 2^{G_i - G_j} q_i.k_j         (j <= i)     R = P T
//     W  = T diag(beta gamma) K       U' = T diag(beta) V        (U = U' - W S^T)
//     Qh = diag(gamma) Q - P W        O' = R diag(beta) V
//     o  = scale (O' + Qh S^T)
//     S <- gamma_C S + U^T diag(kappa) K
// Everything but the two products with S is independent of the state, so the
// sequential chain per chunk is two tensor-core products and two epilogues:
//     D1 = [Qh; W] S^T  ->  U = U' - (W S^T), o = scale (O' + Qh S^T)
//     S += K^T (kappa U)  ->  bf16 copy of S for the next chunk.
// Only exponents G_i - G_j with i >= j, G and G_C - G appear, all <= 0.
//
// The float32 state lives in TMEM as S~ with S = Gamma S~: the decay gamma_C
// of each chunk is folded into the running scalar Gamma (the update is added
// as kappa U / Gamma), so the state is not rewritten every chunk; it is
// rescaled in place only when Gamma would fall below 2^-80.
//
// Mapping.  One CTA per (sequence, value head, 64-wide slice of d_v); the rows
// of S (d_v) evolve independently once T is known, so both slices of a value
// head compute the chunk's T themselves.  16 warps:
//   warp 0       TMA: [K; Q] tiles (2 stages), the V slice, gate inputs
//   warp 1       MMA issuer, state chain (D1, S update)
//   warp 2       MMA issuer, precompute (D0, R, X1, X2); allocates TMEM
//   warps 4-7    chain epilogues (U, o, state), one TMEM lane quadrant each
//   warps 8-15   precompute: gates, A and P, T by blocked forward substitution
//                (16x16 diagonal blocks on CUDA cores, off-diagonal blocks with
//                tf32 mma.sync), scaled bf16 copies of T and R, Qh and W
// Tensor-core products (tcgen05.mma, bf16 operands from shared memory, f32
// accumulators in TMEM):
//   D0 = [K; Q] K^T                    M128 N64  K128
//   R  = [P; T] T                      M128 N64  K64   (rows 0-63 used)
//   X1 = [R bg; T bg] K                M128 N128 K64   (P W; W)
//   X2 = [R b; T b] V                  M128 N64  K64   (O'; U')
//   D1 = [Qh; W] S^T                   M128 N64  K128  (chain)
//   S~ += K^T (kappa U / Gamma)        M128 N64  K64   (chain, accumulates)
// Every wait on an mbarrier is bounded; on expiry the CTA records an error in
// the workspace, stops waiting and drains.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"
#include "tile_util.cuh"

namespace gdn {

namespace {

using namespace tc;
using namespace tile;

constexpr int kD = 128;
constexpr int kC = 64;
constexpr int kBV = 64;
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kPrepWarps = 8;
constexpr int kLdF = 68;                       // fp32 solve scratch row stride

// shared memory layout (byte offsets from a 1024-aligned base)
constexpr uint32_t KQ_STAGE = 2 * KQ_PANEL;    // [K; Q] over d = 0..127
constexpr uint32_t OFF_KQ = 0;                               // 2 stages
constexpr uint32_t OFF_V = OFF_KQ + 2 * KQ_STAGE;            // 64 x 64 bf16
constexpr uint32_t OFF_PT = OFF_V + 8192;                    // P | T (bf16)
constexpr uint32_t OFF_RT1 = OFF_PT + 16384;                 // [R bg; T bg]
constexpr uint32_t OFF_RT2 = OFF_RT1 + 16384;                // [R b; T b]
constexpr uint32_t OFF_QW = OFF_RT2 + 16384;                 // [Qh; W], 2 panels
constexpr uint32_t OFF_ST = OFF_QW + 2 * KQ_PANEL;           // S^T bf16: 128 x 64
constexpr uint32_t OFF_UK = OFF_ST + 16384;                  // kappa U / Gamma: 64 x 64
constexpr uint32_t OFF_AF = OFF_UK + 8192;                   // A: 64 x 68 f32
constexpr uint32_t OFF_TF = OFF_AF + 64 * kLdF * 4;          // T: 64 x 68 f32
constexpr uint32_t OFF_XF = OFF_TF + 64 * kLdF * 4;          // mma.sync scratch
constexpr uint32_t XF_BYTES = 32 * 36 * 4;
constexpr uint32_t OFF_AB = OFF_XF + XF_BYTES;               // 2 stages: a, b (64 x 4 f32 each)
constexpr uint32_t AB_STAGE = 2048;
constexpr uint32_t OFF_GATES = OFF_AB + 2 * AB_STAGE;        // 4 buffers
constexpr int kGateFloats = 5 * 64 + 4;
constexpr uint32_t OFF_MISC = OFF_GATES + 4 * kGateFloats * 4;
constexpr uint32_t OFF_BARS = (OFF_MISC + 64 + 7) & ~7u;
constexpr int kNumBars = 28;
constexpr uint32_t SMEM_BYTES = OFF_BARS + kNumBars * 8;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;           // room to align the base
static_assert(SMEM_ALLOC <= 232448, "shared memory budget of one CTA");

// barrier indices
enum {
    B_KQ_FULL = 0, B_KQ_EMPTY = 2, B_V_FULL = 4, B_V_EMPTY,
    B_D0_FULL, B_D0_EMPTY, B_TP_FULL, B_R_FULL, B_RT_READY, B_X_FULL, B_X2_EMPTY,
    B_X2_EMPTY1, B_QW_READY, B_QW_EMPTY, B_D1_FULL, B_U_READY, B_S_OK, B_S_FULL, B_ST_READY,
    B_DRAIN1, B_DRAIN2
};

// TMEM columns
constexpr uint32_t COL_D0 = 0, COL_R = 64, COL_X1 = 128, COL_X2 = 256, COL_D1 = 384, COL_S = 448;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_D0 = idesc_bf16(128, 64, false, false);
constexpr uint32_t IDESC_R = idesc_bf16(128, 64, false, true);
constexpr uint32_t IDESC_X1 = idesc_bf16(128, 128, false, true);
constexpr uint32_t IDESC_X2 = idesc_bf16(128, kBV, false, true);
constexpr uint32_t IDESC_D1 = idesc_bf16(128, kBV, false, true);
constexpr uint32_t IDESC_S = idesc_bf16(128, kBV, true, true);

constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s: far beyond any legitimate wait
constexpr float kLog2e = 1.4426950408889634f;
// chunks whose total decay stays above 2^-64 form the decay ratios as products
constexpr float kFastDecayLog2 = 64.f;
// the state scale Gamma is folded into the update until it would drop below this
constexpr float kMinGamma = 8.271806125530277e-25f;          // 2^-80

struct GateBuf {
    float beta[64];
    float gamma[64];
    float kappa[64];
    float G[64];
    float igamma[64];      // 2^{-G}; meaningful when `fast`
    float gC;
    int fast;              // G_C >= -kFastDecayLog2: 2^{G_i - G_j} = gamma_i * igamma_j
    float pad[2];
};
static_assert(sizeof(GateBuf) == kGateFloats * 4, "gate buffer layout");

struct TcParams {
    const float* a;
    const float* b;
    const float* A_log;
    const float* dt_bias;
    const int32_t* cu;
    int64_t T;
    int32_t Hqk, Hv;
    float scale;
    const float* s_in;
    float* s_out;
    float* o;
    uint32_t* err;
    int gate_tma;          // a, b staged by TMA (needs Hv % 4 == 0), else read directly
    uint16_t* o16;         // o as bf16 (instead of o)
};

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                  const __grid_constant__ CUtensorMap tm_b, const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // align to 1024 bytes by pointer arithmetic on the shared array, so that
    // every access below stays in the shared state space (LDS/STS)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC + 4);
    float* xchg = reinterpret_cast<float*>(sm + OFF_MISC + 16);      // scan carry
    GateBuf* gates = reinterpret_cast<GateBuf*>(sm + OFF_GATES);
    float* Af = reinterpret_cast<float*>(sm + OFF_AF);
    float* Tf = reinterpret_cast<float*>(sm + OFF_TF);
    float* Xf = reinterpret_cast<float*>(sm + OFF_XF);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int slices = kD / kBV;
    const int slice = blockIdx.x % slices;
    const int h = (blockIdx.x / slices) % p.Hv;
    const int n = blockIdx.x / (slices * p.Hv);
    const int g = h / (p.Hv / p.Hqk);
    const int v0 = slice * kBV;
    const int64_t bos = p.cu ? p.cu[n] : 0;
    const int64_t eos = p.cu ? p.cu[n + 1] : p.T;
    const int64_t len = eos - bos;
    const int nch = (int)((len + kC - 1) / kC);
    const int64_t state_off = ((int64_t)n * p.Hv + h) * kD * kD + (int64_t)v0 * kD;

    if (nch == 0) {
        // empty sequence: the final state is the initial state
        if (p.s_out && p.s_out != p.s_in) {
            for (int i = threadIdx.x; i < kBV * kD; i += kThreads)
                p.s_out[state_off + i] = p.s_in ? p.s_in[state_off + i] : 0.f;
        }
        return;
    }

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_KQ_FULL + s), 1);
            mbar_init(bar(B_KQ_EMPTY + s), 1);
        }
        mbar_init(bar(B_V_FULL), 1);
        mbar_init(bar(B_V_EMPTY), 1);
        mbar_init(bar(B_D0_FULL), 1);
        mbar_init(bar(B_D0_EMPTY), kPrepWarps);
        mbar_init(bar(B_TP_FULL), kPrepWarps);
        mbar_init(bar(B_R_FULL), 1);
        mbar_init(bar(B_RT_READY), kPrepWarps);
        mbar_init(bar(B_X_FULL), 1);
        mbar_init(bar(B_X2_EMPTY), 4);      // one barrier per X2 buffer
        mbar_init(bar(B_X2_EMPTY1), 4);
        mbar_init(bar(B_QW_READY), kPrepWarps);
        mbar_init(bar(B_QW_EMPTY), 1);
        mbar_init(bar(B_D1_FULL), 1);
        mbar_init(bar(B_U_READY), 2);
        mbar_init(bar(B_S_OK), 4);
        mbar_init(bar(B_S_FULL), 1);
        mbar_init(bar(B_ST_READY), 4);
        mbar_init(bar(B_DRAIN1), 1);
        mbar_init(bar(B_DRAIN2), 1);
        fence_mbar_init();
    }
    if (warp == 2) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    // zero the strictly upper blocks of the T scratch once (never written again)
    for (int i = threadIdx.x; i < 64 * kLdF; i += kThreads) Tf[i] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
            if (p.gate_tma) { prefetch_tmap(&tm_a); prefetch_tmap(&tm_b); }
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1, u = c >> 1;
                const int32_t y = (int32_t)(bos + (int64_t)c * kC);
                if (u >= 1 && !mbar_wait(bar(B_KQ_EMPTY + s), (u - 1) & 1, abort_flag, kWaitLimitNs)) break;
                const uint32_t kq = sbase + OFF_KQ + s * KQ_STAGE;
                mbar_arrive_expect_tx(bar(B_KQ_FULL + s), KQ_STAGE + (p.gate_tma ? AB_STAGE : 0));
                tma_load_2d(kq, &tm_k, g * kD, y, bar(B_KQ_FULL + s));
                tma_load_2d(kq + 8192, &tm_q, g * kD, y, bar(B_KQ_FULL + s));
                tma_load_2d(kq + KQ_PANEL, &tm_k, g * kD + 64, y, bar(B_KQ_FULL + s));
                tma_load_2d(kq + KQ_PANEL + 8192, &tm_q, g * kD + 64, y, bar(B_KQ_FULL + s));
                if (p.gate_tma) {
                    // gate inputs: the 4-column group of a and b that holds column h
                    const uint32_t ab = sbase + OFF_AB + s * AB_STAGE;
                    tma_load_2d(ab, &tm_a, h & ~3, y, bar(B_KQ_FULL + s));
                    tma_load_2d(ab + 1024, &tm_b, h & ~3, y, bar(B_KQ_FULL + s));
                }
                if (c >= 1 && !mbar_wait(bar(B_V_EMPTY), (c - 1) & 1, abort_flag, kWaitLimitNs)) break;
                mbar_arrive_expect_tx(bar(B_V_FULL), 8192);
                tma_load_2d(sbase + OFF_V, &tm_v, h * kD + v0, y, bar(B_V_FULL));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer: state chain
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const uint32_t kq = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
                if (!mbar_wait(bar(B_ST_READY), c & 1, abort_flag, kWaitLimitNs)) break;
                if (!mbar_wait(bar(B_QW_READY), c & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + COL_D1, desc_kmajor_2panel(sbase + OFF_QW, kk),
                             desc_mnmajor(sbase + OFF_ST, kk, 16384), IDESC_D1, kk > 0);
                mma_commit(bar(B_D1_FULL));
                mma_commit(bar(B_QW_EMPTY));
                if (!mbar_wait(bar(B_U_READY), c & 1, abort_flag, kWaitLimitNs)) break;
                if (!mbar_wait(bar(B_S_OK), c & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + COL_S, desc_mnmajor(kq, kk, KQ_PANEL),
                             desc_mnmajor(sbase + OFF_UK, kk, 8192), IDESC_S, 1);
                mma_commit(bar(B_S_FULL));
                mma_commit(bar(B_KQ_EMPTY + (c & 1)));
            }
            // drain: every MMA issued by this thread has completed before TMEM is
            // released (bounded even when the CTA is aborting)
            volatile int no_abort = 0;
            mma_commit(bar(B_DRAIN1));
            mbar_wait(bar(B_DRAIN1), 0, &no_abort, kWaitLimitNs);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ MMA issuer: precompute
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const uint32_t kq = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
                if (!mbar_wait(bar(B_KQ_FULL + (c & 1)), (c >> 1) & 1, abort_flag, kWaitLimitNs)) break;
                if (c > 0 && !mbar_wait(bar(B_D0_EMPTY), (c - 1) & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                // D0 = [K; Q] K^T
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + COL_D0, desc_kmajor_2panel(kq, kk), desc_kmajor_2panel(kq, kk),
                             IDESC_D0, kk > 0);
                mma_commit(bar(B_D0_FULL));
                // R = [P; T] T
                if (!mbar_wait(bar(B_TP_FULL), c & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + COL_R, desc_kmajor_1panel(sbase + OFF_PT, kk),
                             desc_mnmajor(sbase + OFF_PT + 8192, kk, 8192), IDESC_R, kk > 0);
                mma_commit(bar(B_R_FULL));
                // X1 = [R bg; T bg] K,  X2 = [R b; T b] V (X2 double-buffered)
                if (!mbar_wait(bar(B_RT_READY), c & 1, abort_flag, kWaitLimitNs)) break;
                if (!mbar_wait(bar(B_V_FULL), c & 1, abort_flag, kWaitLimitNs)) break;
                // buffer c&1 was last read by the epilogue of chunk c-2: completion
                // number (c >> 1) - 1 of that buffer's own barrier
                if (c >= 2 && !mbar_wait(bar(B_X2_EMPTY + (c & 1)), ((c >> 1) - 1) & 1, abort_flag,
                                         kWaitLimitNs))
                    break;
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + COL_X1, desc_kmajor_1panel(sbase + OFF_RT1, kk),
                             desc_mnmajor(kq, kk, KQ_PANEL), IDESC_X1, kk > 0);
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + COL_X2 + (c & 1) * 64, desc_kmajor_1panel(sbase + OFF_RT2, kk),
                             desc_mnmajor(sbase + OFF_V, kk, 8192), IDESC_X2, kk > 0);
                mma_commit(bar(B_X_FULL));
                mma_commit(bar(B_V_EMPTY));
            }
            volatile int no_abort = 0;
            mma_commit(bar(B_DRAIN2));
            mbar_wait(bar(B_DRAIN2), 0, &no_abort, kWaitLimitNs);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ chain epilogues
        const int q = warp - 4;                    // TMEM lane quadrant
        const int r = q * 32 + lane;               // TMEM lane = row
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        uint8_t* st_tile = sm + OFF_ST;
        // initial state: thread r holds d_k row r of S^T (64 v-columns); Gamma = 1
        {
            float s[32];
            for (int half = 0; half < 2; ++half) {
                for (int j = 0; j < 32; ++j) {
                    const int vcol = half * 32 + j;
                    s[j] = p.s_in ? p.s_in[state_off + (int64_t)vcol * kD + r] : 0.f;
                }
                tmem_st32(tl + COL_S + half * 32, s);
                for (int j = 0; j < 4; ++j) st_bf16x8(st_tile, r, half * 4 + j, s + 8 * j);
            }
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_ST_READY));
        }
        float Gam = 1.f;                           // S = Gam * S~ (same value in every thread)
        for (int c = 0; c < nch; ++c) {
            const GateBuf& gb = gates[c & 3];
            const int64_t tok0 = bos + (int64_t)c * kC;
            const uint32_t x2col = COL_X2 + (c & 1) * 64;
            mbar_wait(bar(B_D1_FULL), c & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            const float Gn = Gam * gb.gC;          // scale of the state after this chunk
            const bool resc = !(Gn >= kMinGamma);
            const float inv = resc ? 1.f : 1.f / Gn;
            if (q >= 2) {
                // U_t = U'_t - (W S^T)_t; write kappa_t U_t / Gamma as the update operand
                const int t = r - 64;
                const float sc = gb.kappa[t] * inv;
                for (int half = 0; half < 2; ++half) {
                    float up[32], ws[32];
                    tmem_ld32(tl + x2col + half * 32, up);
                    tmem_ld32(tl + COL_D1 + half * 32, ws);
                    tmem_ld_wait();
                    for (int j = 0; j < 32; ++j) up[j] = sc * (up[j] - ws[j]);
                    for (int j = 0; j < 4; ++j) st_bf16x8(sm + OFF_UK, t, half * 4 + j, up + 8 * j);
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar(B_U_READY));
                    mbar_arrive(bar(B_X2_EMPTY + (c & 1)));
                }
            } else {
                // o_t = scale (O'_t + (Qh S^T)_t)
                const int t = r;
                const bool valid = tok0 + t < eos;
                const int64_t orow_off = ((tok0 + t) * p.Hv + h) * kD + v0;
                for (int half = 0; half < 2; ++half) {
                    float op[32], qs[32];
                    tmem_ld32(tl + x2col + half * 32, op);
                    tmem_ld32(tl + COL_D1 + half * 32, qs);
                    tmem_ld_wait();
                    if (valid) {
                        for (int j = 0; j < 32; j += 4) {
                            float4 w;
                            w.x = p.scale * (op[j] + qs[j]);
                            w.y = p.scale * (op[j + 1] + qs[j + 1]);
                            w.z = p.scale * (op[j + 2] + qs[j + 2]);
                            w.w = p.scale * (op[j + 3] + qs[j + 3]);
                            if (p.o16)
                                *reinterpret_cast<uint2*>(p.o16 + orow_off + half * 32 + j) =
                                    make_uint2(pack_bf16x2(w.x, w.y), pack_bf16x2(w.z, w.w));
                            else
                                *reinterpret_cast<float4*>(p.o + orow_off + half * 32 + j) = w;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_X2_EMPTY + (c & 1)));
            }
            if (resc) {
                // fold the accumulated scale into the stored state: S~ <- Gn S~
                for (int half = 0; half < 2; ++half) {
                    float s[32];
                    tmem_ld32(tl + COL_S + half * 32, s);
                    tmem_ld_wait();
                    for (int j = 0; j < 32; ++j) s[j] *= Gn;
                    tmem_st32(tl + COL_S + half * 32, s);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_S_OK));
            Gam = resc ? 1.f : Gn;
            // new state -> bf16 operand of the next chunk (and the final state)
            mbar_wait(bar(B_S_FULL), c & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            const bool last = (c == nch - 1);
            for (int half = 0; half < 2; ++half) {
                float s[32];
                tmem_ld32(tl + COL_S + half * 32, s);
                tmem_ld_wait();
                for (int j = 0; j < 32; ++j) s[j] *= Gam;
                if (!last) {
                    for (int j = 0; j < 4; ++j) st_bf16x8(st_tile, r, half * 4 + j, s + 8 * j);
                } else if (p.s_out) {
                    for (int j = 0; j < 32; ++j)
                        p.s_out[state_off + (int64_t)(half * 32 + j) * kD + r] = s[j];
                }
            }
            if (!last) {
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_ST_READY));
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ precompute
        const int pw = warp - 8;                   // 0..7
        const int q = pw & 3;                      // TMEM lane quadrant (= warp % 4)
        const int hh = pw >> 2;                    // column half
        const int pt = pw * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const float Al = p.A_log[h], dtb = p.dt_bias[h];
        for (int c = 0; c < nch; ++c) {
            GateBuf& gb = gates[c & 3];
            const int64_t tok0 = bos + (int64_t)c * kC;
            const uint32_t kqo = OFF_KQ + (c & 1) * KQ_STAGE;
            // ---- gates (warps 14, 15): G = running sum of log2(alpha); beta;
            //      gamma = 2^G; kappa = 2^{G_C - G}
            if (pw >= 6) {
                const int t = pt - 192;
                const int64_t tok = tok0 + t;
                mbar_wait(bar(B_KQ_FULL + (c & 1)), (c >> 1) & 1, abort_flag, kWaitLimitNs);
                const float* abt = reinterpret_cast<const float*>(sm + OFF_AB + (c & 1) * AB_STAGE);
                float lg = 0.f, be = 0.f;
                if (tok < eos) {
                    const float av = p.gate_tma ? abt[t * 4 + (h & 3)] : p.a[tok * p.Hv + h];
                    const float bv = p.gate_tma ? abt[256 + t * 4 + (h & 3)] : p.b[tok * p.Hv + h];
                    lg = kLog2e * log_alpha_f32(av, Al, dtb);
                    be = sigmoid_f32(bv);
                }
                float run = lg;
                for (int m = 1; m < 32; m <<= 1) {
                    const float o = __shfl_up_sync(0xffffffffu, run, m);
                    if (lane >= m) run += o;
                }
                if (pw == 6 && lane == 31) xchg[0] = run;
                named_bar_sync(3, 64);
                if (pw == 7) run += xchg[0];
                gb.G[t] = run;
                gb.beta[t] = be;
                gb.gamma[t] = exp2f(run);
                if (t == 63) {
                    xchg[1] = run;
                    gb.gC = exp2f(run);
                    gb.fast = run >= -kFastDecayLog2 ? 1 : 0;
                }
                named_bar_sync(3, 64);
                gb.kappa[t] = exp2f(xchg[1] - run);
                gb.igamma[t] = xchg[1] >= -kFastDecayLog2 ? exp2f(-run) : 0.f;
            }
            named_bar_sync(1, kPrepWarps * 32);
            // ---- D0 rows -> A (f32 scratch) and P (bf16 operand); each warp 32 columns
            mbar_wait(bar(B_D0_FULL), c & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            {
                const bool fast = gb.fast != 0;
                float dv[32];
                tmem_ld32(tl + COL_D0 + hh * 32, dv);
                tmem_ld_wait();
                const int i = (q & 1) * 32 + lane;       // row within KK^T (q<2) or QK^T (q>=2)
                const float Gi = gb.G[i];
                if (q < 2) {
                    // A_ij = beta_i 2^{G_i - G_j} (k_i . k_j), j < i
                    const float ci = fast ? gb.beta[i] * gb.gamma[i] : gb.beta[i];
                    float* arow = Af + i * kLdF + hh * 32;
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = hh * 32 + j4;
                        float4 w;
                        if (fast) {
                            const float4 ig = *reinterpret_cast<const float4*>(&gb.igamma[j]);
                            w.x = (j + 0 < i) ? ci * dv[j4 + 0] * ig.x : 0.f;
                            w.y = (j + 1 < i) ? ci * dv[j4 + 1] * ig.y : 0.f;
                            w.z = (j + 2 < i) ? ci * dv[j4 + 2] * ig.z : 0.f;
                            w.w = (j + 3 < i) ? ci * dv[j4 + 3] * ig.w : 0.f;
                        } else {
                            const float4 gj = *reinterpret_cast<const float4*>(&gb.G[j]);
                            w.x = (j + 0 < i) ? ci * dv[j4 + 0] * exp2f(Gi - gj.x) : 0.f;
                            w.y = (j + 1 < i) ? ci * dv[j4 + 1] * exp2f(Gi - gj.y) : 0.f;
                            w.z = (j + 2 < i) ? ci * dv[j4 + 2] * exp2f(Gi - gj.z) : 0.f;
                            w.w = (j + 3 < i) ? ci * dv[j4 + 3] * exp2f(Gi - gj.w) : 0.f;
                        }
                        *reinterpret_cast<float4*>(arow + j4) = w;
                    }
                } else {
                    // P_ij = 2^{G_i - G_j} (q_i . k_j), j <= i
                    const float ci = fast ? gb.gamma[i] : 1.f;
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = hh * 32 + j4;
                        if (fast) {
                            const float4 ig = *reinterpret_cast<const float4*>(&gb.igamma[j]);
                            dv[j4 + 0] = (j + 0 <= i) ? ci * dv[j4 + 0] * ig.x : 0.f;
                            dv[j4 + 1] = (j + 1 <= i) ? ci * dv[j4 + 1] * ig.y : 0.f;
                            dv[j4 + 2] = (j + 2 <= i) ? ci * dv[j4 + 2] * ig.z : 0.f;
                            dv[j4 + 3] = (j + 3 <= i) ? ci * dv[j4 + 3] * ig.w : 0.f;
                        } else {
                            const float4 gj = *reinterpret_cast<const float4*>(&gb.G[j]);
                            dv[j4 + 0] = (j + 0 <= i) ? dv[j4 + 0] * exp2f(Gi - gj.x) : 0.f;
                            dv[j4 + 1] = (j + 1 <= i) ? dv[j4 + 1] * exp2f(Gi - gj.y) : 0.f;
                            dv[j4 + 2] = (j + 2 <= i) ? dv[j4 + 2] * exp2f(Gi - gj.z) : 0.f;
                            dv[j4 + 3] = (j + 3 <= i) ? dv[j4 + 3] * exp2f(Gi - gj.w) : 0.f;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_bf16x8(sm + OFF_PT, i, hh * 4 + j, dv + 8 * j);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_D0_EMPTY));
            named_bar_sync(1, kPrepWarps * 32);
            // ---- T = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution
            if (pw < 4) {
                const int blk = pw;
                const int col = lane & 15;
                const float* Ab = Af + (16 * blk) * kLdF + 16 * blk;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    // x_i = delta_{i,col} - sum_{m<i} A_im x_m, with four partial sums;
                    // row i of the block is read as float4 (the same address in every lane)
                    float arow[16];
#pragma unroll
                    for (int m4 = 0; m4 < i; m4 += 4) {
                        const float4 a4 = *reinterpret_cast<const float4*>(Ab + i * kLdF + m4);
                        arow[m4] = a4.x; arow[m4 + 1] = a4.y; arow[m4 + 2] = a4.z; arow[m4 + 3] = a4.w;
                    }
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < i; ++m) acc[m & 3] = fmaf(arow[m], x[m], acc[m & 3]);
                    x[i] = ((i == col) ? 1.f : 0.f) - ((acc[0] + acc[1]) + (acc[2] + acc[3]));
                }
                if (lane < 16) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) Tf[(16 * blk + i) * kLdF + 16 * blk + col] = x[i];
                }
            }
            named_bar_sync(1, kPrepWarps * 32);
            // ---- 32x32 blocks: T10 = -T11 A10 T00 (warp: block pair pw>>1, 8 columns)
            if (pw < 4) {
                const int pr = pw >> 1, nh = pw & 1;
                const int R0 = 32 * pr, R1 = R0 + 16;
                float* Xw = Xf + pw * 128;                 // 16 x 8
                float cfr[4];
                mma_tile(cfr, Af, kLdF, R1, R0, Tf, kLdF, R0, R0 + 8 * nh, 0, 2, lane);
                frag_c_store(Xw, 8, 0, 0, cfr, 1.f, lane);
                __syncwarp();
                mma_tile(cfr, Tf, kLdF, R1, R1, Xw, 8, 0, 0, 0, 2, lane);
                frag_c_store(Tf, kLdF, R1, R0 + 8 * nh, cfr, -1.f, lane);
            }
            named_bar_sync(1, kPrepWarps * 32);
            // ---- 64x64: T[32:64, 0:32] = -T[32:64, 32:64] A[32:64, 0:32] T[0:32, 0:32]
            //      (one 16x8 output tile per warp; all-zero k-steps of the
            //      triangular factors are skipped)
            {
                const int mt = pw >> 2, nt = pw & 3;
                float cfr[4];
                mma_tile(cfr, Af, kLdF, 32 + 16 * mt, 0, Tf, kLdF, 0, 8 * nt, nt, 4, lane);
                frag_c_store(Xf, 36, 16 * mt, 8 * nt, cfr, 1.f, lane);
                named_bar_sync(1, kPrepWarps * 32);
                mma_tile(cfr, Tf, kLdF, 32 + 16 * mt, 32, Xf, 36, 0, 8 * nt, 0, 2 * mt + 2, lane);
                frag_c_store(Tf, kLdF, 32 + 16 * mt, 8 * nt, cfr, -1.f, lane);
            }
            named_bar_sync(1, kPrepWarps * 32);
            // ---- T (bf16) as the B operand of R = P T
            for (int u = pt; u < 64 * 8; u += kPrepWarps * 32) {
                const int row = u >> 3, chunk = u & 7;
                const float4 t0 = *reinterpret_cast<const float4*>(Tf + row * kLdF + chunk * 8);
                const float4 t1 = *reinterpret_cast<const float4*>(Tf + row * kLdF + chunk * 8 + 4);
                const float x[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                st_bf16x8(sm + OFF_PT + 8192, row, chunk, x);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_TP_FULL));
            // ---- [R bg; T bg] and [R b; T b] (bf16): columns scaled by beta gamma / beta
            {
                const int i = (q & 1) * 32 + lane;
                float v[32];
                if (q < 2) {
                    // R rows from TMEM
                    mbar_wait(bar(B_R_FULL), c & 1, abort_flag, kWaitLimitNs);
                    tc_fence_after();
                    tmem_ld32(tl + COL_R + hh * 32, v);
                    tmem_ld_wait();
                } else {
                    // T rows from the f32 scratch
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 t4 = *reinterpret_cast<const float4*>(Tf + i * kLdF + hh * 32 + j);
                        v[j] = t4.x; v[j + 1] = t4.y; v[j + 2] = t4.z; v[j + 3] = t4.w;
                    }
                }
                const uint32_t row_off = (q < 2) ? 0u : 8192u;   // R in rows 0-63, T in rows 64-127
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) {
                    const int j0 = hh * 32 + j8 * 8;
                    const float4 b0 = *reinterpret_cast<const float4*>(&gb.beta[j0]);
                    const float4 b1 = *reinterpret_cast<const float4*>(&gb.beta[j0 + 4]);
                    const float4 g0 = *reinterpret_cast<const float4*>(&gb.gamma[j0]);
                    const float4 g1 = *reinterpret_cast<const float4*>(&gb.gamma[j0 + 4]);
                    const float bj[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    const float gj[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                    float wb[8], wg[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        wb[e] = v[j8 * 8 + e] * bj[e];
                        wg[e] = wb[e] * gj[e];
                    }
                    st_bf16x8(sm + OFF_RT1 + row_off, i, hh * 4 + j8, wg);
                    st_bf16x8(sm + OFF_RT2 + row_off, i, hh * 4 + j8, wb);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_RT_READY));
            // ---- X1 -> Qh = diag(gamma) Q - P W (rows 0-63) and W (rows 64-127), bf16
            mbar_wait(bar(B_X_FULL), c & 1, abort_flag, kWaitLimitNs);
            if (c >= 1) mbar_wait(bar(B_QW_EMPTY), (c - 1) & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            {
                const int i = (q & 1) * 32 + lane;
                const float ga = gb.gamma[i];
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const int dcol = hh * 64 + part * 32;          // 32 of the 128 d columns
                    const int panel = dcol >> 6, ch0 = (dcol & 63) >> 3;
                    float x[32];
                    tmem_ld32(tl + COL_X1 + dcol, x);
                    tmem_ld_wait();
                    if (q < 2) {
                        // Qh_i = gamma_i q_i - (P W)_i
                        const uint8_t* qrow = sm + kqo + panel * KQ_PANEL + 8192;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float qv[8];
                            ld_bf16x8(qrow, i, ch0 + j, qv);
#pragma unroll
                            for (int e = 0; e < 8; ++e) x[8 * j + e] = ga * qv[e] - x[8 * j + e];
                        }
                    }
                    uint8_t* dst = sm + OFF_QW + panel * KQ_PANEL + (q < 2 ? 0 : 8192);
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_bf16x8(dst, i, ch0 + j, x + 8 * j);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_QW_READY));
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, 1u);
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// looked up once per process (a function-local static is initialised once,
// thread-safely); null if the driver does not provide it
EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
                cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(ptr);
        cudaGetLastError();    // a refused query leaves no sticky error behind
        return nullptr;
    }();
    return fn;
}

// 2D bf16 tensor [rows, cols] (cols contiguous), 64 x 64 boxes, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D float tensor [rows, cols], 4-column x 64-row boxes, no swizzle
bool make_map_gates(CUtensorMap* m, const float* base, int64_t rows, int64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    cuuint32_t box[2] = {4, 64};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_tc_smem_bytes() { return SMEM_ALLOC; }

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t stream) {
    if (a.T == 0) {
        // every sequence is empty: final state = initial state
        if (a.final_state && a.final_state != a.initial_state) {
            const size_t bytes = (size_t)a.n_seq * a.Hv * kD * kD * sizeof(float);
            return a.initial_state
                       ? cudaMemcpyAsync(a.final_state, a.initial_state, bytes,
                                         cudaMemcpyDeviceToDevice, stream)
                       : cudaMemsetAsync(a.final_state, 0, bytes, stream);
        }
        return cudaSuccess;
    }
    CUtensorMap mq, mk, mv, ma, mb;
    if (!make_map(&mq, a.q, a.T, (int64_t)a.Hqk * kD) || !make_map(&mk, a.k, a.T, (int64_t)a.Hqk * kD) ||
        !make_map(&mv, a.v, a.T, (int64_t)a.Hv * kD))
        return cudaErrorInvalidValue;
    // a and b rows must be a multiple of 16 bytes for TMA; otherwise they are read directly
    const int gate_tma = (a.Hv % 4 == 0) ? 1 : 0;
    if (gate_tma) {
        if (!make_map_gates(&ma, a.a, a.T, a.Hv) || !make_map_gates(&mb, a.b, a.T, a.Hv))
            return cudaErrorInvalidValue;
    } else {
        ma = mq;
        mb = mq;       // unused
    }
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    TcParams p{a.a, a.b, a.A_log, a.dt_bias, a.cu_seqlens, a.T, a.Hqk, a.Hv, a.scale,
               a.initial_state, a.final_state, a.o,
               reinterpret_cast<uint32_t*>(static_cast<char*>(a.workspace) + kWsErrorWordOffset),
               gate_tma, a.o16};
    const int64_t blocks = (int64_t)a.n_seq * a.Hv * (kD / kBV);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    prefill_tc_kernel<<<(unsigned)blocks, kThreads, SMEM_ALLOC, stream>>>(mq, mk, mv, ma, mb, p);
    return cudaGetLastError();
}

}  // namespace gdn
