// prefill_tc.cu -- chunked gated delta-rule prefill on the sm_100a tensor cores.
//
// The recurrence (Qwen3.8-27B architecture page, 2kiu.com, section 2.2, with
// the decay alpha on the erased state):
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
//     o_t = scale * S_t q_t,
// is computed in chunks of C = 64 tokens.  With G the running sum of
// log(alpha) inside the chunk, gamma = e^G, kappa = e^{G_C - G}, and S the
// state at the chunk start, the chunk is (WY / UT form):
//     A_ij = beta_i e^{G_i - G_j} k_i.k_j  (j < i)      T = (I + A)^{-1}
//     P_ij = e^{G_i - G_j} q_i.k_j         (j <= i)     R = P T
//     Y    = [K; Q] S^T                                  (64 + 64 rows)
//     B    = diag(beta) (V - diag(gamma) Y_K)
//     [U; O_intra] = [T; R] B
//     o    = scale (O_intra + diag(gamma) Y_Q)
//     S   <- gamma_C S + U^T diag(kappa) K
// (U = T (diag(beta) V - diag(beta gamma) K S^T) is the corrected write of
// the delta rule; substituting it reproduces the token-by-token recurrence.)
// Only exponents G_i - G_j with i >= j, G and G_C - G appear, all <= 0.
//
// Mapping.  One CTA per (sequence, value head, 64-wide slice of d_v).  The
// rows of S (d_v) evolve independently once T is known, so two CTAs share a
// value head; both solve the chunk's T themselves.  The CTA walks the
// sequence's chunks in order with 12 warps:
//   warp 0      TMA producer: [K; Q] tiles (2 stages) and the V slice
//   warp 1      MMA issuer for the state chain (one thread; also allocates TMEM)
//   warp 2      MMA issuer for the precompute products (one thread)
//   warps 4-7   chain epilogues (B, U, o, state), one TMEM lane quadrant each
//   warps 8-11  precompute: gates, D0 -> A and P, T by blocked forward
//               substitution (16x16 diagonal blocks on CUDA cores, the
//               off-diagonal blocks with tf32 mma.sync), R from TMEM
// Tensor-core products (tcgen05.mma, bf16 operands from shared memory, f32
// accumulators in TMEM):
//   D0 = [K; Q] K^T      M128 N64  K128   (precompute)
//   R  = [P; T] T        M128 N64  K64    (precompute; rows 0-63 used)
//   Y  = [K; Q] S^T      M128 N64  K128   (chain)
//   Z  = [T; R] B        M128 N64  K64    (chain)
//   S += K^T (kappa U)   M128 N64  K64    (chain; accumulates into the state)
// The float32 state lives in TMEM and is only rounded to bf16 for use as an
// operand.  Every wait on an mbarrier is bounded; on expiry the CTA records an
// error in the workspace, stops waiting and drains.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace gdn {

namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kC = 64;
constexpr int kBV = 64;
constexpr int kThreads = 384;
constexpr int kLdF = 68;                       // fp32 solve scratch row stride

// shared memory layout (byte offsets from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;                 // 2 stages: [K;Q] 128 rows x 128 cols bf16, 2 panels
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t KQ_PANEL = 16384;
constexpr uint32_t OFF_V = OFF_KQ + 2 * KQ_STAGE;   // 2 stages: 64 x 64 bf16
constexpr uint32_t V_STAGE = 8192;
constexpr uint32_t OFF_PTR = OFF_V + 2 * V_STAGE;   // P | T | R, 64 x 64 bf16 each
constexpr uint32_t OFF_BB = OFF_PTR + 3 * 8192;     // B: 64 x 64 bf16
constexpr uint32_t OFF_UB = OFF_BB + 8192;          // kappa U: 64 x 64 bf16
constexpr uint32_t OFF_ST = OFF_UB + 8192;          // S^T: 128 x 64 bf16
constexpr uint32_t OFF_AF = OFF_ST + 16384;         // A: 64 x 68 f32
constexpr uint32_t OFF_TF = OFF_AF + 64 * kLdF * 4; // T: 64 x 68 f32
constexpr uint32_t OFF_XF = OFF_TF + 64 * kLdF * 4; // mma.sync scratch
constexpr uint32_t XF_BYTES = 32 * 36 * 4;
constexpr uint32_t OFF_AB = OFF_XF + XF_BYTES;      // 2 stages: a and b, 64 rows x 4 floats each
constexpr uint32_t AB_STAGE = 2048;
constexpr uint32_t OFF_GATES = OFF_AB + 2 * AB_STAGE; // 4 buffers
constexpr int kGateFloats = 5 * 64 + 4;             // beta, gamma, kappa, G (log2 units), 1/gamma; gC, flag
constexpr uint32_t OFF_MISC = OFF_GATES + 4 * kGateFloats * 4;
constexpr uint32_t OFF_BARS = (OFF_MISC + 64 + 7) & ~7u;
constexpr int kNumBars = 24;
constexpr uint32_t SMEM_BYTES = OFF_BARS + kNumBars * 8;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // room to align the base

// barrier indices
enum {
    B_KQ_FULL = 0, B_KQ_EMPTY = 2, B_V_FULL = 4, B_V_EMPTY = 6,
    B_D0_FULL = 8, B_D0_EMPTY, B_TP_FULL, B_R_FULL, B_TR_FULL, B_TR_EMPTY,
    B_Y_FULL, B_B_READY, B_Z_FULL, B_U_READY, B_S_FULL, B_ST_READY, B_S_SCALED, B_DRAIN, B_DRAIN2
};

// TMEM columns
constexpr uint32_t COL_D0 = 0, COL_R = 64, COL_Y = 128, COL_Z = 192, COL_S = 256;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_D0 = idesc_bf16(128, 64, false, false);
constexpr uint32_t IDESC_R = idesc_bf16(128, 64, false, true);
constexpr uint32_t IDESC_Y = idesc_bf16(128, kBV, false, true);
constexpr uint32_t IDESC_Z = idesc_bf16(128, kBV, false, true);
constexpr uint32_t IDESC_S = idesc_bf16(128, kBV, true, true);

constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
// chunks whose total decay stays above 2^-64 form the decay ratios as products
constexpr float kFastDecayLog2 = 64.f;    // 2 s: far beyond any legitimate wait

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
};

// K-major operand, K extent 128 split in two 16 KB panels of 128 rows
TC_DEVICE uint64_t desc_kmajor_2panel(uint32_t base, int kk) {
    return sdesc_sw128(base + (kk >> 2) * KQ_PANEL + (kk & 3) * 32, 16, 1024);
}
// K-major operand with K extent 64 (one panel)
TC_DEVICE uint64_t desc_kmajor_1panel(uint32_t base, int kk) {
    return sdesc_sw128(base + kk * 32, 16, 1024);
}
// MN-major operand: rows are the K index (128 bytes each), 16 rows per step;
// lbo = distance between 64-element MN atoms
TC_DEVICE uint64_t desc_mnmajor(uint32_t base, int kk, uint32_t lbo) {
    return sdesc_sw128(base + kk * 2048, lbo, 1024);
}

// --- tf32 mma.sync fragments (m16n8k8) on fp32 shared-memory matrices -----------
TC_DEVICE void frag_a(const float* M, int ld, int r0, int k0, uint32_t* a, int lane) {
    const int g = lane >> 2, t = lane & 3;
    a[0] = to_tf32(M[(r0 + g) * ld + k0 + t]);
    a[1] = to_tf32(M[(r0 + g + 8) * ld + k0 + t]);
    a[2] = to_tf32(M[(r0 + g) * ld + k0 + t + 4]);
    a[3] = to_tf32(M[(r0 + g + 8) * ld + k0 + t + 4]);
}
TC_DEVICE void frag_b(const float* M, int ld, int k0, int n0, uint32_t* b, int lane) {
    const int g = lane >> 2, t = lane & 3;
    b[0] = to_tf32(M[(k0 + t) * ld + n0 + g]);
    b[1] = to_tf32(M[(k0 + t + 4) * ld + n0 + g]);
}
TC_DEVICE void frag_c_store(float* M, int ld, int r0, int n0, const float* c, float s, int lane) {
    const int g = lane >> 2, t = lane & 3;
    M[(r0 + g) * ld + n0 + 2 * t] = s * c[0];
    M[(r0 + g) * ld + n0 + 2 * t + 1] = s * c[1];
    M[(r0 + g + 8) * ld + n0 + 2 * t] = s * c[2];
    M[(r0 + g + 8) * ld + n0 + 2 * t + 1] = s * c[3];
}
// c (16 x 8) = A[r0:r0+16, k0:k0+8*nk] * B[kb0:kb0+8*nk, n0:n0+8]
TC_DEVICE void mma_tile(float* c, const float* A, int lda, int r0, int k0, const float* B, int ldb,
                        int kb0, int n0, int nk, int lane) {
    c[0] = c[1] = c[2] = c[3] = 0.f;
    for (int s = 0; s < nk; ++s) {
        uint32_t a[4], b[2];
        frag_a(A, lda, r0, k0 + 8 * s, a, lane);
        frag_b(B, ldb, kb0 + 8 * s, n0, b, lane);
        mma_tf32_16x8x8(c, a, b);
    }
}

// write 8 floats as bf16 into row `row`, 16-byte chunk `chunk` of a swizzled tile
TC_DEVICE void st_bf16x8(uint8_t* tile, int row, int chunk, const float* x) {
    uint4 v;
    v.x = pack_bf16x2(x[0], x[1]);
    v.y = pack_bf16x2(x[2], x[3]);
    v.z = pack_bf16x2(x[4], x[5]);
    v.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(tile + sw128_off(row, chunk)) = v;
}
TC_DEVICE void ld_bf16x8(const uint8_t* tile, int row, int chunk, float* x) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + sw128_off(row, chunk));
    float2 f;
    f = bf16x2_to_f32x2(v.x); x[0] = f.x; x[1] = f.y;
    f = bf16x2_to_f32x2(v.y); x[2] = f.x; x[3] = f.y;
    f = bf16x2_to_f32x2(v.z); x[4] = f.x; x[5] = f.y;
    f = bf16x2_to_f32x2(v.w); x[6] = f.x; x[7] = f.y;
}

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
        mbar_init(bar(B_KQ_FULL), 1); mbar_init(bar(B_KQ_FULL + 1), 1);
        mbar_init(bar(B_KQ_EMPTY), 1); mbar_init(bar(B_KQ_EMPTY + 1), 1);
        mbar_init(bar(B_V_FULL), 1); mbar_init(bar(B_V_FULL + 1), 1);
        mbar_init(bar(B_V_EMPTY), 2); mbar_init(bar(B_V_EMPTY + 1), 2);
        mbar_init(bar(B_D0_FULL), 1);
        mbar_init(bar(B_D0_EMPTY), 4);
        mbar_init(bar(B_TP_FULL), 4);
        mbar_init(bar(B_R_FULL), 1);
        mbar_init(bar(B_TR_FULL), 2);
        mbar_init(bar(B_TR_EMPTY), 1);
        mbar_init(bar(B_Y_FULL), 1);
        mbar_init(bar(B_B_READY), 2);
        mbar_init(bar(B_Z_FULL), 1);
        mbar_init(bar(B_U_READY), 2);
        mbar_init(bar(B_S_FULL), 1);
        mbar_init(bar(B_ST_READY), 4);
        mbar_init(bar(B_S_SCALED), 4);
        mbar_init(bar(B_DRAIN), 1);
        mbar_init(bar(B_DRAIN2), 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
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
            prefetch_tmap(&tm_a); prefetch_tmap(&tm_b);
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1, u = c >> 1;
                const int32_t y = (int32_t)(bos + (int64_t)c * kC);
                if (u >= 1 && !mbar_wait(bar(B_KQ_EMPTY + s), (u - 1) & 1, abort_flag, kWaitLimitNs)) break;
                const uint32_t kq = sbase + OFF_KQ + s * KQ_STAGE;
                mbar_arrive_expect_tx(bar(B_KQ_FULL + s), KQ_STAGE + (p.gate_tma ? AB_STAGE : 0));
                if (p.gate_tma) {
                    // gate inputs: the 4-column group of a and b that holds column h
                    const uint32_t ab = sbase + OFF_AB + s * AB_STAGE;
                    tma_load_2d(ab, &tm_a, h & ~3, y, bar(B_KQ_FULL + s));
                    tma_load_2d(ab + 1024, &tm_b, h & ~3, y, bar(B_KQ_FULL + s));
                }
                tma_load_2d(kq, &tm_k, g * kD, y, bar(B_KQ_FULL + s));
                tma_load_2d(kq + 8192, &tm_q, g * kD, y, bar(B_KQ_FULL + s));
                tma_load_2d(kq + KQ_PANEL, &tm_k, g * kD + 64, y, bar(B_KQ_FULL + s));
                tma_load_2d(kq + KQ_PANEL + 8192, &tm_q, g * kD + 64, y, bar(B_KQ_FULL + s));
                if (u >= 1 && !mbar_wait(bar(B_V_EMPTY + s), (u - 1) & 1, abort_flag, kWaitLimitNs)) break;
                mbar_arrive_expect_tx(bar(B_V_FULL + s), V_STAGE);
                tma_load_2d(sbase + OFF_V + s * V_STAGE, &tm_v, h * kD + v0, y, bar(B_V_FULL + s));
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer: state chain
        // Y = [K;Q] S^T, Z = [T;R] B, S += K^T (kappa U), in order, each as soon
        // as its operands are ready (blocking waits, no polling).
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const uint32_t kq = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
                if (!mbar_wait(bar(B_ST_READY), c & 1, abort_flag, kWaitLimitNs)) break;
                if (!mbar_wait(bar(B_TR_FULL), c & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + COL_Y, desc_kmajor_2panel(kq, kk),
                             desc_mnmajor(sbase + OFF_ST, kk, 16384), IDESC_Y, kk > 0);
                mma_commit(bar(B_Y_FULL));
                if (!mbar_wait(bar(B_B_READY), c & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + COL_Z, desc_kmajor_1panel(sbase + OFF_PTR + 8192, kk),
                             desc_mnmajor(sbase + OFF_BB, kk, 8192), IDESC_Z, kk > 0);
                mma_commit(bar(B_Z_FULL));
                mma_commit(bar(B_TR_EMPTY));
                if (!mbar_wait(bar(B_U_READY), c & 1, abort_flag, kWaitLimitNs)) break;
                if (!mbar_wait(bar(B_S_SCALED), c & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + COL_S, desc_mnmajor(kq, kk, KQ_PANEL),
                             desc_mnmajor(sbase + OFF_UB, kk, 8192), IDESC_S, 1);
                mma_commit(bar(B_S_FULL));
                mma_commit(bar(B_KQ_EMPTY + (c & 1)));
            }
            // drain: every MMA issued by this thread has completed before TMEM is
            // released (bounded even when the CTA is aborting)
            volatile int no_abort = 0;
            mma_commit(bar(B_DRAIN));
            mbar_wait(bar(B_DRAIN), 0, &no_abort, kWaitLimitNs);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ MMA issuer: precompute
        // D0 = [K;Q] K^T and R = [P;T] T for each chunk.
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const uint32_t kq = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
                if (!mbar_wait(bar(B_KQ_FULL + (c & 1)), (c >> 1) & 1, abort_flag, kWaitLimitNs)) break;
                if (c > 0 && !mbar_wait(bar(B_D0_EMPTY), (c - 1) & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + COL_D0, desc_kmajor_2panel(kq, kk), desc_kmajor_2panel(kq, kk),
                             IDESC_D0, kk > 0);
                mma_commit(bar(B_D0_FULL));
                if (!mbar_wait(bar(B_TP_FULL), c & 1, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + COL_R, desc_kmajor_1panel(sbase + OFF_PTR, kk),
                             desc_mnmajor(sbase + OFF_PTR + 8192, kk, 8192), IDESC_R, kk > 0);
                mma_commit(bar(B_R_FULL));
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
        // initial state: thread r holds d_k row r of S^T (64 v-columns)
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
        for (int c = 0; c < nch; ++c) {
            const GateBuf& gb = gates[c & 3];
            const int64_t tok0 = bos + (int64_t)c * kC;
            mbar_wait(bar(B_Y_FULL), c & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            const float gC = gb.gC;
            if (q < 2) {
                // B_t = beta_t (v_t - gamma_t Y_t), t = r
                const int t = r;
                mbar_wait(bar(B_V_FULL + (c & 1)), (c >> 1) & 1, abort_flag, kWaitLimitNs);
                const float be = gb.beta[t], ga = gb.gamma[t];
                const uint8_t* vt = sm + OFF_V + (c & 1) * V_STAGE;
                for (int half = 0; half < 2; ++half) {
                    float y[32];
                    tmem_ld32(tl + COL_Y + half * 32, y);
                    tmem_ld_wait();
                    for (int j = 0; j < 4; ++j) {
                        float vv[8], bb[8];
                        ld_bf16x8(vt, t, half * 4 + j, vv);
                        for (int e = 0; e < 8; ++e) bb[e] = be * (vv[e] - ga * y[8 * j + e]);
                        st_bf16x8(sm + OFF_BB, t, half * 4 + j, bb);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar(B_B_READY));
                    mbar_arrive(bar(B_V_EMPTY + (c & 1)));
                }
            }
            // scale the float32 state in TMEM by gamma_C before this chunk's update
            for (int half = 0; half < 2; ++half) {
                float s[32];
                tmem_ld32(tl + COL_S + half * 32, s);
                tmem_ld_wait();
                for (int j = 0; j < 32; ++j) s[j] *= gC;
                tmem_st32(tl + COL_S + half * 32, s);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_S_SCALED));

            mbar_wait(bar(B_Z_FULL), c & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            if (q < 2) {
                // U rows: write kappa_t U_t as the bf16 operand of the state update
                const int t = r;
                const float ka = gb.kappa[t];
                for (int half = 0; half < 2; ++half) {
                    float z[32];
                    tmem_ld32(tl + COL_Z + half * 32, z);
                    tmem_ld_wait();
                    for (int j = 0; j < 32; ++j) z[j] *= ka;
                    for (int j = 0; j < 4; ++j) st_bf16x8(sm + OFF_UB, t, half * 4 + j, z + 8 * j);
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_U_READY));
            } else {
                // output rows: o_t = scale (O_intra_t + gamma_t Y_Q,t)
                const int t = r - 64;
                const float ga = gb.gamma[t];
                const bool valid = tok0 + t < eos;
                float* orow = p.o + ((tok0 + t) * p.Hv + h) * kD + v0;
                for (int half = 0; half < 2; ++half) {
                    float z[32], y[32];
                    tmem_ld32(tl + COL_Z + half * 32, z);
                    tmem_ld32(tl + COL_Y + half * 32, y);
                    tmem_ld_wait();
                    if (valid) {
                        for (int j = 0; j < 32; j += 4) {
                            float4 w;
                            w.x = p.scale * (z[j] + ga * y[j]);
                            w.y = p.scale * (z[j + 1] + ga * y[j + 1]);
                            w.z = p.scale * (z[j + 2] + ga * y[j + 2]);
                            w.w = p.scale * (z[j + 3] + ga * y[j + 3]);
                            *reinterpret_cast<float4*>(orow + half * 32 + j) = w;
                        }
                    }
                }
            }
            // new state -> bf16 operand of the next chunk (and the final state)
            mbar_wait(bar(B_S_FULL), c & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            const bool last = (c == nch - 1);
            for (int half = 0; half < 2; ++half) {
                float s[32];
                tmem_ld32(tl + COL_S + half * 32, s);
                tmem_ld_wait();
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
        const int pw = warp - 8;
        const int pt = pw * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(pw * 32) << 16);
        const float Al = p.A_log[h], dtb = p.dt_bias[h];
        for (int c = 0; c < nch; ++c) {
            GateBuf& gb = gates[c & 3];
            const int64_t tok0 = bos + (int64_t)c * kC;
            // ---- gates (warps 10, 11): G = running sum of log2(alpha); beta;
            //      gamma = 2^G; kappa = 2^{G_C - G}
            if (pw >= 2) {
                const int t = pt - 64;
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
                if (pw == 2 && lane == 31) xchg[0] = run;
                named_bar_sync(3, 64);
                if (pw == 3) run += xchg[0];
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
            named_bar_sync(1, 128);
            // ---- D0 rows -> A (f32 scratch) and P (bf16 operand)
            mbar_wait(bar(B_D0_FULL), c & 1, abort_flag, kWaitLimitNs);
            tc_fence_after();
            // decay ratio 2^{G_i - G_j} (j <= i): gamma_i * igamma_j when the chunk's
            // decay is moderate, else one exp2 per element (never overflows: G_i <= G_j)
            const bool fast = gb.fast != 0;
            if (pw < 2) {
                // A_ij = beta_i 2^{G_i - G_j} (k_i . k_j), j < i
                const int i = pt;
                const float Gi = gb.G[i];
                const float ci = fast ? gb.beta[i] * gb.gamma[i] : gb.beta[i];
                float* arow = Af + i * kLdF;
                for (int half = 0; half < 2; ++half) {
                    float kk[32];
                    tmem_ld32(tl + COL_D0 + half * 32, kk);
                    tmem_ld_wait();
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = half * 32 + j4;
                        float4 w;
                        if (fast) {
                            const float4 ig = *reinterpret_cast<const float4*>(&gb.igamma[j]);
                            w.x = (j + 0 < i) ? ci * kk[j4 + 0] * ig.x : 0.f;
                            w.y = (j + 1 < i) ? ci * kk[j4 + 1] * ig.y : 0.f;
                            w.z = (j + 2 < i) ? ci * kk[j4 + 2] * ig.z : 0.f;
                            w.w = (j + 3 < i) ? ci * kk[j4 + 3] * ig.w : 0.f;
                        } else {
                            const float4 gj = *reinterpret_cast<const float4*>(&gb.G[j]);
                            w.x = (j + 0 < i) ? ci * kk[j4 + 0] * exp2f(Gi - gj.x) : 0.f;
                            w.y = (j + 1 < i) ? ci * kk[j4 + 1] * exp2f(Gi - gj.y) : 0.f;
                            w.z = (j + 2 < i) ? ci * kk[j4 + 2] * exp2f(Gi - gj.z) : 0.f;
                            w.w = (j + 3 < i) ? ci * kk[j4 + 3] * exp2f(Gi - gj.w) : 0.f;
                        }
                        *reinterpret_cast<float4*>(arow + j) = w;
                    }
                }
            } else {
                // P_ij = 2^{G_i - G_j} (q_i . k_j), j <= i
                const int i = pt - 64;
                const float Gi = gb.G[i];
                const float ci = fast ? gb.gamma[i] : 1.f;
                for (int half = 0; half < 2; ++half) {
                    float qk[32];
                    tmem_ld32(tl + COL_D0 + half * 32, qk);
                    tmem_ld_wait();
#pragma unroll
                    for (int j4 = 0; j4 < 32; j4 += 4) {
                        const int j = half * 32 + j4;
                        if (fast) {
                            const float4 ig = *reinterpret_cast<const float4*>(&gb.igamma[j]);
                            qk[j4 + 0] = (j + 0 <= i) ? ci * qk[j4 + 0] * ig.x : 0.f;
                            qk[j4 + 1] = (j + 1 <= i) ? ci * qk[j4 + 1] * ig.y : 0.f;
                            qk[j4 + 2] = (j + 2 <= i) ? ci * qk[j4 + 2] * ig.z : 0.f;
                            qk[j4 + 3] = (j + 3 <= i) ? ci * qk[j4 + 3] * ig.w : 0.f;
                        } else {
                            const float4 gj = *reinterpret_cast<const float4*>(&gb.G[j]);
                            qk[j4 + 0] = (j + 0 <= i) ? qk[j4 + 0] * exp2f(Gi - gj.x) : 0.f;
                            qk[j4 + 1] = (j + 1 <= i) ? qk[j4 + 1] * exp2f(Gi - gj.y) : 0.f;
                            qk[j4 + 2] = (j + 2 <= i) ? qk[j4 + 2] * exp2f(Gi - gj.z) : 0.f;
                            qk[j4 + 3] = (j + 3 <= i) ? qk[j4 + 3] * exp2f(Gi - gj.w) : 0.f;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_bf16x8(sm + OFF_PTR, i, half * 4 + j, qk + 8 * j);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_D0_EMPTY));
            named_bar_sync(1, 128);
            // ---- T = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution
            {
                const int blk = pw;
                const int col = lane & 15;
                const float* Ab = Af + (16 * blk) * kLdF + 16 * blk;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    // x_i = delta_{i,col} - sum_{m<i} A_im x_m, with four partial sums
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < i; ++m) acc[m & 3] = fmaf(Ab[i * kLdF + m], x[m], acc[m & 3]);
                    x[i] = ((i == col) ? 1.f : 0.f) - ((acc[0] + acc[1]) + (acc[2] + acc[3]));
                }
                if (lane < 16) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) Tf[(16 * blk + i) * kLdF + 16 * blk + col] = x[i];
                }
            }
            named_bar_sync(1, 128);
            // ---- 32x32 blocks: T10 = -T11 A10 T00 (warp: block pair pw>>1, 8 columns)
            {
                const int pr = pw >> 1, nh = pw & 1;
                const int R0 = 32 * pr, R1 = R0 + 16;
                float* Xw = Xf + pw * 128;                 // 16 x 8
                float cfr[4];
                mma_tile(cfr, Af, kLdF, R1, R0, Tf, kLdF, R0, R0 + 8 * nh, 2, lane);
                frag_c_store(Xw, 8, 0, 0, cfr, 1.f, lane);
                __syncwarp();
                mma_tile(cfr, Tf, kLdF, R1, R1, Xw, 8, 0, 0, 2, lane);
                frag_c_store(Tf, kLdF, R1, R0 + 8 * nh, cfr, -1.f, lane);
            }
            named_bar_sync(1, 128);
            // ---- 64x64: T[32:64, 0:32] = -T[32:64, 32:64] A[32:64, 0:32] T[0:32, 0:32]
            {
                const int mt = pw >> 1, nc = 16 * (pw & 1);
                float cfr[4];
                for (int j = 0; j < 2; ++j) {
                    mma_tile(cfr, Af, kLdF, 32 + 16 * mt, 0, Tf, kLdF, 0, nc + 8 * j, 4, lane);
                    frag_c_store(Xf, 36, 16 * mt, nc + 8 * j, cfr, 1.f, lane);
                }
                named_bar_sync(1, 128);
                for (int j = 0; j < 2; ++j) {
                    mma_tile(cfr, Tf, kLdF, 32 + 16 * mt, 32, Xf, 36, 0, nc + 8 * j, 4, lane);
                    frag_c_store(Tf, kLdF, 32 + 16 * mt, nc + 8 * j, cfr, -1.f, lane);
                }
            }
            named_bar_sync(1, 128);
            // ---- T (bf16) into the [P; T; R] operand block, once the previous Z product is done
            if (c >= 1) mbar_wait(bar(B_TR_EMPTY), (c - 1) & 1, abort_flag, kWaitLimitNs);
            for (int u = pt; u < 64 * 8; u += 128) {
                const int row = u >> 3, chunk = u & 7;
                const float4 t0 = *reinterpret_cast<const float4*>(Tf + row * kLdF + chunk * 8);
                const float4 t1 = *reinterpret_cast<const float4*>(Tf + row * kLdF + chunk * 8 + 4);
                const float x[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                st_bf16x8(sm + OFF_PTR + 8192, row, chunk, x);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_TP_FULL));
            // ---- R = P T from TMEM -> bf16 rows 64..127 of [T; R]
            if (pw < 2) {
                const int i = pt;
                mbar_wait(bar(B_R_FULL), c & 1, abort_flag, kWaitLimitNs);
                tc_fence_after();
                for (int half = 0; half < 2; ++half) {
                    float rr[32];
                    tmem_ld32(tl + COL_R + half * 32, rr);
                    tmem_ld_wait();
                    for (int j = 0; j < 4; ++j) st_bf16x8(sm + OFF_PTR + 16384, i, half * 4 + j, rr + 8 * j);
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_TR_FULL));
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, 1u);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
                cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
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
               gate_tma};
    const int64_t blocks = (int64_t)a.n_seq * a.Hv * (kD / kBV);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    prefill_tc_kernel<<<(unsigned)blocks, kThreads, SMEM_ALLOC, stream>>>(mq, mk, mv, ma, mb, p);
    return cudaGetLastError();
}

}  // namespace gdn
