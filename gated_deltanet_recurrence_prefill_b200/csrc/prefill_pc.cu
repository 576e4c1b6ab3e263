// prefill_pc.cu -- chunked gated delta-rule prefill on the sm_100a tensor cores,
// as a co-resident grid of producer and consumer CTAs: per (sequence, value
// head) one consumer CTA runs the state chain and one or two producer CTAs the
// state-independent algebra.
//
// The arithmetic is the chunked WY / UT form of the recurrence (Qwen3.8-27B
// architecture page, 2kiu.com, section 2.2, with the decay alpha on the erased
// state), chunks of C = 64 tokens, G the running sum of log2(alpha) in the
// chunk, gamma = 2^G, kappa = 2^{G_C - G}, S the state at the chunk start:
//     A_ij = beta_i 2^{G_i - G_j} k_i.k_j  (j < i)      T = (I + A)^{-1}
//     P_ij = 2^{G_i - G_j} q_i.k_j         (j <= i)     R = P T
//     W  = T diag(beta gamma) K       U' = T diag(beta) V
//     Qh = diag(gamma) Q - P W        O' = R diag(beta) V
//     [U; o / scale] = [U'; O'] + [-W; Qh] S^T
//     S <- gamma_C S + K^T diag(kappa) U
// Everything up to [-W; Qh] and [T beta; R beta] is independent of the state.
//
// Producers (roles 1..P, P = 1 or 2).  Producer p takes chunks p,
// p + P, ...; inside it two groups of 8 warps take alternate chunks.  A thread
// per group (warps 19, 20) issues D0 = [K; Q] K^T (tcgen05) as soon as the
// chunk's [K; Q] lands and the group has read the previous D0.  A group
// computes the gates, A and P from D0, T by blocked forward
// substitution (16x16 diagonal blocks on CUDA cores, off-diagonal blocks with
// tf32 mma.sync), R = P T (tcgen05), the scaled bf16 copies [R bg; T bg] and
// [T b; R b], X1 = [R bg; T bg] K (tcgen05) and from it -W and Qh.  It stages
// the chunk's outgoing bytes where nothing else needs them any more: -W and Qh
// over the K and Q rows of the chunk's [K; Q] stage, [T b; R b] with kappa and
// gamma_C over the A scratch.  A publisher warp per group bulk-stores them to
// the chunk's slot of a ring in global memory (kRing slots per (sequence,
// value head), normally resident in L2), hands the staging back as soon as the
// store has read it, and tells the consumer once the bytes are in place by
// raising a counter in global memory (release / acquire at GPU scope).
// Warp 16 loads [K; Q] and the gate inputs by TMA into three stages.
//
// Consumer (role 0).  A loader thread bulk-loads each chunk from the ring into
// one of two receive slots and hands ring slots back to the producers (a
// second counter per ring slot).  Every product has d_v as its M dimension
// (TMEM lane = v row) and spans 128 columns (measured on B200: a bf16
// tcgen05.mma with M = 128 and K = 16 takes about 50 cycles at N = 64, 66 at
// N = 128 and 130 at N = 256, and M = 64 costs as much as M = 128, so
// N = 128 is the cheapest width per column that keeps the issue rate up):
//   D^T  = V^T [T b; R b]^T                M128 N128 K64   (in the chain's gaps)
//   D^T += S [-W; Qh]^T                    M128 N128 K128  -> [U^T | o^T / scale]
//   S~  += (kappa U / Gamma)^T K           M128 N128 K64   (accumulates in TMEM)
// The last two are the state chain, issued by one thread; the first by another
// thread, in two halves placed so that they run while the chain's epilogues
// would leave the tensor core idle (a thread that issues a tcgen05.mma is held
// until the tensor core takes it, so each issuer has a thread of its own).  The
// chain's A operands, S and (kappa U / Gamma)^T in bf16, are written by the
// epilogue threads straight into TMEM, so the chain keeps off shared memory;
// S is converted in four column blocks, each reported on its own mbarrier, so
// that the chain's first K steps start while the rest is converted.  The
// float32 state lives in TMEM as S~ with S = Gamma S~ (the decay gamma_C of
// each chunk is folded into the running scalar Gamma and the update is added
// as kappa U / Gamma); S~ is rescaled in place only when Gamma would fall
// below 2^-80.  o^T / scale is read back while the state update runs and
// stored straight to global memory (for each token a warp writes 32
// consecutive floats).  D has two buffers so that the next chunk's [U'; O']
// product can start before this chunk's epilogues are done.  With the fused
// output norm (y requested), the TMA warp also stages the gate z of each
// chunk, and after the second epilogue (while the tensor core works on the
// next chunk) the epilogue warps turn their o rows into
// y = norm_w * o / rms(o) * silu(z), bf16, summing each token's squares over
// the four warps of a column share in shared memory.
// Warp 0 loads V and K by TMA (two buffers each).
//
// Grid.  For nu units, blocks [0, nu) are the consumers and blocks
// [nu, (1 + P) nu) the producers (block b serves unit b % nu).  They wait
// on one another, so the launch is cooperative: the whole grid is resident at
// once (one CTA per SM), and units beyond one grid's worth run in further
// launches.  No thread-block cluster is used, so the CTAs of a unit may sit
// anywhere on the GPU.
//
// Every wait is bounded; on expiry a CTA records an error in the workspace
// (which makes the other CTAs' waits on global counters give up too), stops
// waiting and drains its own tensor-core work and copies.  Producer group warps never leave
// their loop early (their named barriers must always complete): after an abort
// their waits simply fall through.
#include <cuda.h>

#include <stdlib.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"
#include "tile_util.cuh"

namespace gdn {

// Per-chunk timestamps of one (sequence, value head) unit for latency analysis,
// compiled in only with -DGDN_PREFILL_TRACE (off in every normal build):
// TRACE_CLK(ev, c) records clock64() of event ev for chunk c.
#ifdef GDN_PREFILL_TRACE
__device__ long long g_prefill_trace[40][4096];
__device__ int g_prefill_trace_unit = -1;
#define TRACE_CLK(ev, c) \
    do { if (x.traced) g_prefill_trace[ev][(c) & 4095] = clock64(); } while (0)
#else
#define TRACE_CLK(ev, c) do { } while (0)
#endif

namespace {

using namespace tc;
using namespace tile;

constexpr int kD = 128;
constexpr int kC = 64;
constexpr int kWarps = 21;
constexpr int kThreads = kWarps * 32;
constexpr int kGroupThreads = 256;
constexpr int kLdF = 68;                       // fp32 solve scratch row stride

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
static_assert(sizeof(GateBuf) == (5 * 64 + 4) * 4, "gate buffer layout");

// ---- producer shared memory (byte offsets from a 1024-aligned base) ----------
constexpr uint32_t KQ_STAGE = 2 * KQ_PANEL;    // [K; Q], d = 0..63 | 64..127
constexpr int kKqStages = 3;
constexpr uint32_t P_KQ = 0;
constexpr uint32_t AB_STAGE = 2048;            // a, b: 64 rows x 4 f32 each
constexpr uint32_t P_AB = P_KQ + kKqStages * KQ_STAGE;
constexpr uint32_t P_GROUP = P_AB + kKqStages * AB_STAGE;
constexpr uint32_t G_PT = 0;                               // P | T, later [R bg; T bg]
constexpr uint32_t G_AF = G_PT + 16384;                    // A: 64 x 68 f32
constexpr uint32_t G_TF = G_AF + 64 * kLdF * 4;            // T: 64 x 68 f32
constexpr uint32_t G_XF = G_TF + 64 * kLdF * 4;            // mma.sync scratch 32 x 36
constexpr uint32_t G_GATES = G_XF + 32 * 36 * 4;           // 2 gate buffers
constexpr uint32_t G_END = G_GATES + 2 * sizeof(GateBuf);
constexpr uint32_t GROUP_BYTES = (G_END + 1023) & ~1023u;
constexpr uint32_t P_END = P_GROUP + 2 * GROUP_BYTES;
static_assert(P_GROUP % 1024 == 0 && GROUP_BYTES % 1024 == 0, "swizzled tiles need 1024-byte alignment");

// ---- consumer shared memory ----------------------------------------------------
// receive slot: [-W; Qh] (2 panels of 128 rows x 64 d) and [T b; R b]
// (128 x 64) -- the producer's staged tiles, copied verbatim; the chunk's
// kappa[64] and gamma_C go to a small gate buffer per slot
constexpr uint32_t SL_QW = 0;
constexpr uint32_t SL_RT2 = 2 * KQ_PANEL;
constexpr uint32_t SLOT_BYTES = SL_RT2 + 16384;             // a multiple of 1024
constexpr uint32_t GATES_AT = 16384;                        // kappa[64], gamma_C after [T b; R b] when staged
constexpr uint32_t GATE_BYTES = 512;
constexpr uint32_t C_RECV = 0;                              // 2 slots
constexpr uint32_t C_V = C_RECV + 2 * SLOT_BYTES;           // V: 2 buffers of 2 panels of 64 x 64 bf16
constexpr uint32_t C_K = C_V + 2 * 16384;                   // K: 2 buffers of 2 panels of 64 x 64 bf16
constexpr uint32_t C_GATES = C_K + 2 * 16384;               // 2 gate buffers
constexpr uint32_t C_NORM = C_GATES + 2 * GATE_BYTES;      // output norm: 2 x [4 cb][16 t][4 q] f32
constexpr uint32_t C_Z = C_NORM + 2 * 1024;                 // output norm gate z: 2 x [64 t][128 v] bf16
constexpr uint32_t C_END = C_Z + 2 * 16384;
// what one chunk sends: the [-W; Qh] tile (staged in place of [K; Q]) and the
// [T b; R b] tile with the gates (staged in the A scratch)
constexpr uint32_t SEND_QW = 2 * KQ_PANEL;
constexpr uint32_t SEND_RT = GATES_AT + GATE_BYTES;
static_assert(SEND_RT == GATES_AT + GATE_BYTES && SEND_RT <= 64 * kLdF * 4, "staging layout");
// The chunks travel through a ring of kRing slots per unit of a launch in the
// workspace (global memory, normally resident in L2): the producer's bulk store
// frees its staging as soon as the bytes have been read, and the consumer
// bulk-loads a chunk into its shared memory when a receive slot is free.  Two
// counters per ring slot, in their own 128-byte line per unit, hand the slot
// back and forth: ready[rs] = chunks written to slot rs, freed[rs] = chunks
// the consumer has taken out of it (chunk c uses slot c % kRing).
constexpr int kRing = 8;
constexpr uint32_t GSLOT_BYTES = SEND_QW + SEND_RT;
static_assert(GSLOT_BYTES % 128 == 0 && kRing % 2 == 0, "ring layout");
constexpr uint32_t kFlagWords = 32;            // per unit: ready[kRing] at 0, freed[kRing] at 16
constexpr uint32_t kFreedAt = 16;
static_assert(kRing <= (int)kFreedAt, "counter layout");
// units whose rings the workspace is sized for (one launch handles at most
// this many; more run in further launches)
constexpr int kMaxSlots = 64;

constexpr uint32_t OFF_MISC = (P_END > C_END ? P_END : C_END);
constexpr uint32_t OFF_BARS = OFF_MISC + 64;

enum {
    // producer
    PB_KQ_FULL = 0, PB_KQ_TAKEN = 2, PB_KQ_EMPTY = 4, PB_D0_FULL = 7, PB_R_FULL = 9,
    PB_X1_FULL = 11, PB_DRAIN = 13, PB_STAGED = 15, PB_AF_FREE = 17,
    // (producer and consumer CTAs use the slots from 19 on for different barriers)
    PB_D0_FREE = 19, PB_D0_DRAIN = 21,
    // consumer
    CB_RECV_FULL = 19, CB_K_FULL = 21, CB_V_FULL = 23, CB_V_EMPTY = 25, CB_SLOT_FREE = 27,
    CB_D_FULL = 29, CB_S_FULL = 30, CB_DRAIN = 31, CB_REL_DONE = 32, CB_K_EMPTY = 34,
    CB_EPI1_DONE = 36, CB_EPI2_BLK = 37, CB_E_FULL = 41, CB_E_DRAIN, CB_CHAIN_ISSUED, CB_SUPD_ISSUED,
    CB_Z_FULL = 45, CB_Z_EMPTY = 47, kNumBars = 49
};
constexpr uint32_t SMEM_BYTES = OFF_BARS + kNumBars * 8;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;           // room to align the base
static_assert(SMEM_ALLOC <= 232448, "shared memory budget of one CTA");

// TMEM columns.  Producer group g: D0 (64), R (64), X1 (128) at 256 g.
// Consumer (lane = d_v row everywhere): D^T = [U'; O']^T + S [-W; Qh]^T
// (columns U^T | o^T / scale) at 0 and 128 (alternate chunks), S~ (d_v x d_k)
// at 256, the bf16 A operands S (64 columns of pairs) at 384 and
// (kappa U / Gamma)^T (32 columns) at 448.
constexpr uint32_t PCOL_D0 = 0, PCOL_R = 64, PCOL_X1 = 128;
constexpr uint32_t CCOL_D = 0, CCOL_S = 256, CCOL_AS = 384, CCOL_AU = 448;
constexpr uint32_t kDCols = 128;               // D has two buffers: chunk c uses CCOL_D + (c & 1) kDCols
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_D0 = idesc_bf16(128, 64, false, false);
constexpr uint32_t IDESC_R = idesc_bf16(128, 64, false, true);
constexpr uint32_t IDESC_X1 = idesc_bf16(128, 128, false, true);
// consumer products, M = d_v: [U'; O']^T = V^T [T b; R b]^T (A = V^T MN-major,
// B K-major), S [-W; Qh]^T (A in TMEM, B K-major), (kappa U / Gamma)^T K (A in
// TMEM, B = K MN-major)
constexpr uint32_t IDESC_UO = idesc_bf16(128, 128, true, false);
constexpr uint32_t IDESC_CHAIN = idesc_bf16(128, 128, false, false);
constexpr uint32_t IDESC_SUPD = idesc_bf16(128, 128, false, true);
// consumer warps: 0 TMA (V, K), 1 the state chain's products, 2 ring loader and
// TMEM allocation, then sixteen epilogue warps, then the ring slot release and
// the [U'; O'] products
constexpr int kEpiWarp0 = 3;
constexpr int kEpiThreads = 16 * 32;
constexpr int kRelWarp = kEpiWarp0 + kEpiThreads / 32;     // ring slot release
constexpr int kUoWarp = kRelWarp + 1;                      // [U'; O'] products
constexpr int kNormBar0 = 1;                   // named barriers 1-4: the output norm of column share cb
static_assert(kUoWarp < kWarps, "consumer warps");

constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s: far beyond any legitimate wait
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kFastDecayLog2 = 64.f;
constexpr float kMinGamma = 8.271806125530277e-25f;          // 2^-80

struct ClParams {
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
    uint8_t* ring;         // kRing slots of GSLOT_BYTES per unit of this launch
    uint32_t* flags;       // kFlagWords counters per unit of this launch
    int gate_tma;          // a, b staged by TMA (needs Hv % 4 == 0), else read directly
    int n_prod;            // producer CTAs per unit (1 or 2); a unit has n_prod + 1 CTAs
    int unit0;             // first (sequence, value head) unit of this launch
    // fused gated output norm (y = norm_w * o / rms(o) * silu(z) per token and
    // head, written as bf16) when y != NULL; o may then be NULL
    const uint16_t* z;
    const float* norm_w;
    float eps;
    uint16_t* y;
    uint16_t* o16;         // o as bf16 (instead of o)
};

struct Ctx {
    uint8_t* sm;
    uint32_t sbase;
    uint32_t tmem;
    volatile int* abort;
    int warp, lane;
    int h, g;              // value head, key head
    uint8_t* ring;         // this unit's ring slots
    uint32_t* ready;       // this unit's counters: chunks written to each ring slot
    uint32_t* freed;       //   and chunks taken out of each ring slot
    const uint32_t* err;   // the launch's error word
    int64_t bos, eos;
    int nch;
    int64_t state_off;
    uint32_t bar0;         // shared address of barrier 0
    int traced;            // this unit's events are recorded (tracing builds only)
    TC_DEVICE uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
};

// ================================================================ consumer
__device__ __forceinline__ void consumer(const Ctx& x, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                         const CUtensorMap* tm_z, const ClParams& p) {
    const int warp = x.warp, lane = x.lane;
    const int nch = x.nch;
    if (warp == 0) {
        // ------------------------------------------------ TMA: V and K of each chunk
        // V(c) and K(c) go to buffers c & 1; V is free once the [U'; O'] product
        // of chunk c - 2 has read it, K once the state update of chunk c - 2 has,
        // so that both land well before they are needed.
        if (lane == 0) {
            prefetch_tmap(tm_k);
            prefetch_tmap(tm_v);
            if (p.y) prefetch_tmap(tm_z);
            int nv = 0, nk = 0, nz = 0;
            for (int c = 0; c < nch; ++c) {
                const int32_t y = (int32_t)(x.bos + (int64_t)c * kC);
                const int vb = c & 1;
                if (c >= 2 && !mbar_wait(x.bar(CB_V_EMPTY + vb), ((c >> 1) - 1) & 1, x.abort, kWaitLimitNs))
                    break;
                TRACE_CLK(28, c);
                mbar_arrive_expect_tx(x.bar(CB_V_FULL + vb), 16384);
                tma_load_2d(x.sbase + C_V + vb * 16384, tm_v, x.h * kD, y, x.bar(CB_V_FULL + vb));
                tma_load_2d(x.sbase + C_V + vb * 16384 + 8192, tm_v, x.h * kD + 64, y, x.bar(CB_V_FULL + vb));
                nv = c + 1;
                if (c >= 2 && !mbar_wait(x.bar(CB_K_EMPTY + vb), ((c >> 1) - 1) & 1, x.abort, kWaitLimitNs))
                    break;
                TRACE_CLK(29, c);
                mbar_arrive_expect_tx(x.bar(CB_K_FULL + vb), 16384);
                tma_load_2d(x.sbase + C_K + vb * 16384, tm_k, x.g * kD, y, x.bar(CB_K_FULL + vb));
                tma_load_2d(x.sbase + C_K + vb * 16384 + 8192, tm_k, x.g * kD + 64, y, x.bar(CB_K_FULL + vb));
                nk = c + 1;
                if (p.y) {
                    // the output norm's gate z of this chunk (free once the epilogues
                    // of chunk c - 2 have read it)
                    if (c >= 2 && !mbar_wait(x.bar(CB_Z_EMPTY + vb), ((c >> 1) - 1) & 1, x.abort, kWaitLimitNs))
                        break;
                    mbar_arrive_expect_tx(x.bar(CB_Z_FULL + vb), 16384);
                    tma_load_2d(x.sbase + C_Z + vb * 16384, tm_z, x.h * kD, y, x.bar(CB_Z_FULL + vb));
                    nz = c + 1;
                }
            }
            // copies still in flight land before the CTA may exit
            volatile int no_abort = 0;
            for (int c = nv >= 2 ? nv - 2 : 0; c < nv; ++c)
                mbar_wait(x.bar(CB_V_FULL + (c & 1)), (c >> 1) & 1, &no_abort, kWaitLimitNs);
            for (int c = nk >= 2 ? nk - 2 : 0; c < nk; ++c)
                mbar_wait(x.bar(CB_K_FULL + (c & 1)), (c >> 1) & 1, &no_abort, kWaitLimitNs);
            for (int c = nz >= 2 ? nz - 2 : 0; c < nz; ++c)
                mbar_wait(x.bar(CB_Z_FULL + (c & 1)), (c >> 1) & 1, &no_abort, kWaitLimitNs);
        }
    } else if (warp == kRelWarp) {
        // ------------------------------------------------ ring slots back to the producers
        // Chunk c's ring slot is free once its bulk load into the receive slot
        // has completed.  This thread issues no copies of its own, so its
        // release store does not wait for the loader's copies in flight (and a
        // warp of its own keeps its waits from holding up another role).  The
        // loader reuses receive slot c & 1 for chunk c + 2 only after REL_DONE,
        // so this wait never falls two phases behind.
        if (lane == 0) {
            for (int c = 0; c < nch; ++c) {
                const int b = c & 1;
                if (!mbar_wait(x.bar(CB_RECV_FULL + b), (c >> 1) & 1, x.abort, kWaitLimitNs)) break;
                fence_async_global();
                st_release_gpu(x.freed + c % kRing, (uint32_t)(c / kRing + 1));
                mbar_arrive(x.bar(CB_REL_DONE + b));
                TRACE_CLK(13, c);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------ loader: ring slot -> receive slot
        // Chunk c sits in ring slot c % kRing and goes to receive slot c & 1,
        // which is free once the epilogues of chunk c - 2 are done with it and
        // its ring slot has been handed back (warp kRelWarp).  The loader never
        // waits for its own copies.
        if (lane == 0) {
            int loaded = 0;
            for (int c = 0; c < nch; ++c) {
                const int b = c & 1, rs = c % kRing;
                TRACE_CLK(10, c);
                if (!gflag_wait_ge(x.ready + rs, (uint32_t)(c / kRing + 1), x.abort, x.err, kWaitLimitNs))
                    break;
                TRACE_CLK(11, c);
                if (c >= 2 && (!mbar_wait(x.bar(CB_SLOT_FREE + b), ((c >> 1) - 1) & 1, x.abort, kWaitLimitNs) ||
                               !mbar_wait(x.bar(CB_REL_DONE + b), ((c >> 1) - 1) & 1, x.abort, kWaitLimitNs)))
                    break;
                fence_async_global();
                const uint32_t slot = x.sbase + C_RECV + b * SLOT_BYTES;
                const uint8_t* g = x.ring + (size_t)rs * GSLOT_BYTES;
                mbar_arrive_expect_tx(x.bar(CB_RECV_FULL + b), GSLOT_BYTES);
                bulk_load(slot + SL_QW, g, SEND_QW, x.bar(CB_RECV_FULL + b));
                bulk_load(slot + SL_RT2, g + SEND_QW, GATES_AT, x.bar(CB_RECV_FULL + b));
                bulk_load(x.sbase + C_GATES + b * GATE_BYTES, g + SEND_QW + GATES_AT, GATE_BYTES,
                          x.bar(CB_RECV_FULL + b));
                loaded = c + 1;
                TRACE_CLK(12, c);
            }
            // loads still in flight land before the CTA may exit
            volatile int no_abort = 0;
            for (int c = loaded >= 2 ? loaded - 2 : 0; c < loaded; ++c)
                mbar_wait(x.bar(CB_RECV_FULL + (c & 1)), (c >> 1) & 1, &no_abort, kWaitLimitNs);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ the state chain's products
        // Per chunk c: D(c) += S [-W; Qh]^T, its K steps issued block by block as
        // the second epilogue of chunk c - 1 turns S into the bf16 operand (so
        // the tensor core starts on S's first 32 columns while the others are
        // converted); then, once the first epilogue of c is done,
        // S~ += (kappa U / Gamma)^T K.  A thread is held up while the tensor core
        // works through the products it has issued, so the [U'; O'] products
        // have a thread of their own (warp kUoWarp).
        if (lane == 0) {
            const uint64_t dsc_qw0 = sdesc_sw128(x.sbase + C_RECV + SL_QW, 16, 1024);
            const uint64_t dsc_k = sdesc_sw128(x.sbase + C_K, 8192, 1024);
            constexpr uint64_t kSlotStep = SLOT_BYTES >> 4;
            for (int c = 0; c < nch && !*x.abort; ++c) {
                const int b = c & 1;
                if (!mbar_wait(x.bar(CB_RECV_FULL + b), (c >> 1) & 1, x.abort, kWaitLimitNs) ||
                    !mbar_wait(x.bar(CB_E_FULL), c & 1, x.abort, kWaitLimitNs))
                    break;
                const uint64_t bq = dsc_qw0 + b * kSlotStep;
                bool ok = true;
                for (int j = 0; j < 4 && ok; ++j) {
                    // columns 32 j .. 32 j + 31 of the bf16 S: K steps 2 j, 2 j + 1
                    ok = mbar_wait(x.bar(CB_EPI2_BLK + j), c & 1, x.abort, kWaitLimitNs);
                    if (!ok) break;
                    tc_fence_after();
                    for (int kk = 2 * j; kk < 2 * j + 2; ++kk)
                        mma_bf16_ta(x.tmem + CCOL_D + b * kDCols, x.tmem + CCOL_AS + kk * 8,
                                    bq + (((kk >> 2) * KQ_PANEL + (kk & 3) * 32) >> 4), IDESC_CHAIN, 1);
                }
                if (!ok) break;
                mma_commit(x.bar(CB_D_FULL));
                mbar_arrive(x.bar(CB_CHAIN_ISSUED));
                TRACE_CLK(0, c);
                if (!mbar_wait(x.bar(CB_EPI1_DONE), c & 1, x.abort, kWaitLimitNs)) break;
                TRACE_CLK(4, c);
                if (!mbar_wait(x.bar(CB_K_FULL + b), (c >> 1) & 1, x.abort, kWaitLimitNs)) break;
                tc_fence_after();
                const uint64_t bk = dsc_k + b * (16384 >> 4);
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ta(x.tmem + CCOL_S, x.tmem + CCOL_AU + kk * 8, bk + kk * 128, IDESC_SUPD, 1);
                mma_commit(x.bar(CB_S_FULL));
                mma_commit(x.bar(CB_K_EMPTY + b));
                mbar_arrive(x.bar(CB_SUPD_ISSUED));
                TRACE_CLK(5, c);
                // receive slot b has been read: its products are complete (the
                // first epilogue waited for them) and so are the epilogues' reads
                // of its gates
                mbar_arrive(x.bar(CB_SLOT_FREE + b));
            }
            volatile int no_abort = 0;
            mma_commit(x.bar(CB_DRAIN));
            mbar_wait(x.bar(CB_DRAIN), 0, &no_abort, kWaitLimitNs);
        }
    } else if (warp == kUoWarp) {
        // ------------------------------------------------ [U'; O']^T = V^T [T b; R b]^T per chunk
        // State-independent: it starts chunk c's accumulator D (buffer c & 1).
        // Its K steps fill the two gaps the chain leaves on the tensor core:
        // tokens 0-31 once chunk c - 1's chain product is issued (they run during
        // its first epilogue), tokens 32-63 once chunk c - 1's state update is
        // issued (they run during its second epilogue).  By the first point the
        // epilogues of chunk c - 2 are done with buffer c & 1.
        if (lane == 0) {
            const uint64_t dsc_rt0 = sdesc_sw128(x.sbase + C_RECV + SL_RT2, 16, 1024);
            const uint64_t dsc_v = sdesc_sw128(x.sbase + C_V, 8192, 1024);
            for (int c = 0; c < nch; ++c) {
                const int b = c & 1;
                if (!mbar_wait(x.bar(CB_RECV_FULL + b), (c >> 1) & 1, x.abort, kWaitLimitNs) ||
                    !mbar_wait(x.bar(CB_V_FULL + b), (c >> 1) & 1, x.abort, kWaitLimitNs))
                    break;
                const uint64_t bt = dsc_rt0 + b * (uint64_t)(SLOT_BYTES >> 4);
                const uint64_t av = dsc_v + b * (16384 >> 4);
                bool ok = true;
                for (int half = 0; half < 2 && ok; ++half) {
                    if (c >= 1)
                        ok = mbar_wait(x.bar(half == 0 ? CB_CHAIN_ISSUED : CB_SUPD_ISSUED), (c - 1) & 1, x.abort,
                                       kWaitLimitNs);
                    if (!ok) break;
                    tc_fence_after();
                    for (int kk = 2 * half; kk < 2 * half + 2; ++kk)
                        mma_bf16(x.tmem + CCOL_D + b * kDCols, av + kk * 128, bt + kk * 2, IDESC_UO, kk > 0);
                }
                if (!ok) break;
                mma_commit(x.bar(CB_E_FULL));
                mma_commit(x.bar(CB_V_EMPTY + b));
                TRACE_CLK(15, c);
            }
            volatile int no_abort = 0;
            mma_commit(x.bar(CB_E_DRAIN));
            mbar_wait(x.bar(CB_E_DRAIN), 0, &no_abort, kWaitLimitNs);
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiThreads / 32) {
        // ------------------------------------------------ epilogues
        // Every product has d_v as its M dimension, so TMEM lane = v row: warp w
        // reads lane quadrant q = w % 4 (the hardware rule); thread = one v row.
        // The four warps of a quadrant split the columns: warp (q, cb), cb =
        // (w - kEpiWarp0) / 4, takes tokens 16 cb .. 16 cb + 15 of U^T and of
        // o^T, state columns 32 cb .. 32 cb + 31 for the rescale and the final
        // state, and columns 32 j + 8 cb .. + 7 of block j when S is turned
        // into the bf16 operand.  The bf16 operands of the chain, S and
        // (kappa U / Gamma)^T, go straight to TMEM, where the tensor core reads
        // them (A operand):
        //   D^T  = [U'; O']^T + S [-W; Qh]^T      columns U^T (0-63), o^T / scale (64-127)
        //   S~  += (kappa U / Gamma)^T K
        // Each warp reports each finished part to the issuing thread on an
        // mbarrier (one arrival per warp).  After an abort the waits fall
        // through; every warp still makes every arrival.
        const int q = warp & 3;                    // TMEM lane quadrant
        const int cb = (warp - kEpiWarp0) >> 2;    // column share
        const int v = q * 32 + lane;               // d_v row
        const bool tracer = (warp == kEpiWarp0 + 1 && lane == 0);
        const uint32_t tl = x.tmem + ((uint32_t)(q * 32) << 16);
        const int64_t o_stride = (int64_t)p.Hv * kD;
        auto report = [&](int bar) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(x.bar(bar));
        };
        // initial state: S~ = S0 (Gamma = 1) on columns 32 cb .. + 31, and its
        // bf16 copy (all four blocks reported at once)
        {
            float sv[32];
            if (p.s_in) {
                const float4* src = reinterpret_cast<const float4*>(p.s_in + x.state_off + (int64_t)v * kD + cb * 32);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 t4 = src[j];
                    sv[4 * j] = t4.x; sv[4 * j + 1] = t4.y; sv[4 * j + 2] = t4.z; sv[4 * j + 3] = t4.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) sv[j] = 0.f;
            }
            tmem_st32(tl + CCOL_S + cb * 32, sv);
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(sv[2 * j], sv[2 * j + 1]);
            tmem_st16u(tl + CCOL_AS + cb * 16, pk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int j = 0; j < 4; ++j) mbar_arrive(x.bar(CB_EPI2_BLK + j));
        }
        float Gam = 1.f;                           // S = Gam * S~ (same value in every thread)
        for (int c = 0; c < nch; ++c) {
            const int b = c & 1;
            const float* kap = reinterpret_cast<const float*>(x.sm + C_GATES + b * GATE_BYTES);
            const int64_t tok0 = x.bos + (int64_t)c * kC;
            const uint32_t dbuf = CCOL_D + b * kDCols;
            mbar_wait(x.bar(CB_RECV_FULL + b), (c >> 1) & 1, x.abort, kWaitLimitNs);
            const float Gn = Gam * kap[64];        // scale of the state after this chunk
            const bool resc = !(Gn >= kMinGamma);
            const float inv = resc ? 1.f : __frcp_rn(Gn);
            if (tracer) TRACE_CLK(1, c);
            mbar_wait(x.bar(CB_D_FULL), c & 1, x.abort, kWaitLimitNs);
            if (tracer) TRACE_CLK(2, c);
            tc_fence_after();
            {
                // U^T, tokens t = 16 cb .. 16 cb + 15 -> (kappa_t U_t / Gamma)^T in bf16
                float uv[16];
                tmem_ld16(tl + dbuf + cb * 16, uv);
                tmem_ld_wait();
                const float4* k4 = reinterpret_cast<const float4*>(kap + cb * 16);
                uint32_t pk[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 kv = k4[j];
                    pk[2 * j] = pack_bf16x2(uv[4 * j] * (kv.x * inv), uv[4 * j + 1] * (kv.y * inv));
                    pk[2 * j + 1] = pack_bf16x2(uv[4 * j + 2] * (kv.z * inv), uv[4 * j + 3] * (kv.w * inv));
                }
                tmem_st8u(tl + CCOL_AU + cb * 8, pk);
            }
            if (resc) {
                // S~ <- Gn S~ on this thread's 32 columns (Gamma restarts at 1)
                float sv[32];
                tmem_ld32(tl + CCOL_S + cb * 32, sv);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) sv[j] *= Gn;
                tmem_st32(tl + CCOL_S + cb * 32, sv);
            }
            if (tracer) TRACE_CLK(3, c);
            report(CB_EPI1_DONE);
            // o^T / scale, tokens t = 16 cb .. 16 cb + 15, read while the state update
            // runs and kept in registers for the output norm at the end of the chunk
            float ov[16];
            const int64_t t0 = tok0 + cb * 16;
            const int64_t nvalid = x.eos - t0;     // rows past the end belong to the next sequence
            const int64_t col = x.h * kD + v;
            tmem_ld16(tl + dbuf + 64 + cb * 16, ov);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) ov[j] *= p.scale;
            if (p.o) {
                // for each t a warp stores 32 consecutive floats of o
                float* ocol = p.o + t0 * o_stride + col;
                if (nvalid >= 16) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) ocol[j * o_stride] = ov[j];
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (j < nvalid) ocol[j * o_stride] = ov[j];
                }
            } else if (p.o16) {
                // bf16 o: each lane packs its tokens j, j + 1; lanes l and l ^ 1 (rows v and
                // v ^ 1) swap the packed words, and each assembles one 4-byte word of
                // the two rows (even lanes token j, odd lanes token j + 1)
                const bool odd = lane & 1;
                const uint32_t sel = odd ? 0x3276u : 0x5410u;
                uint32_t* orow2 = reinterpret_cast<uint32_t*>(p.o16 + t0 * o_stride + x.h * kD + (v & ~1));
                const int64_t wstride = o_stride / 2;
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const uint32_t own = pack_bf16x2(ov[j], ov[j + 1]);
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, own, 1);
                    const int jt = odd ? j + 1 : j;
                    if (jt < nvalid) orow2[jt * wstride] = __byte_perm(own, other, sel);
                }
            }
            Gam = resc ? 1.f : Gn;
            // ---- new state -> bf16 operand of the next chunk (and the final state)
            if (tracer) TRACE_CLK(6, c);
            mbar_wait(x.bar(CB_S_FULL), c & 1, x.abort, kWaitLimitNs);
            if (tracer) TRACE_CLK(7, c);
            tc_fence_after();
            if (c == nch - 1) {
                if (p.s_out) {
                    float sv[32];
                    tmem_ld32(tl + CCOL_S + cb * 32, sv);
                    tmem_ld_wait();
                    float4* dst = reinterpret_cast<float4*>(p.s_out + x.state_off + (int64_t)v * kD + cb * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_float4(Gam * sv[4 * j], Gam * sv[4 * j + 1], Gam * sv[4 * j + 2],
                                             Gam * sv[4 * j + 3]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float sv[8];
                    tmem_ld8(tl + CCOL_S + 32 * j + 8 * cb, sv);
                    tmem_ld_wait();
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) pk[e] = pack_bf16x2(Gam * sv[2 * e], Gam * sv[2 * e + 1]);
                    tmem_st4u(tl + CCOL_AS + 16 * j + 4 * cb, pk);
                    report(CB_EPI2_BLK + j);
                }
            }
            if (tracer) TRACE_CLK(8, c);
            if (p.y) {
                // gated output norm of chunk c, computed here so that it overlaps
                // the tensor core's work on chunk c + 1.  The mean square of o
                // over the 128 rows v of a token is spread over the four warps of
                // this column share (lane quadrants 0-3): each warp sums its 32
                // rows for its 16 tokens by a reduce-scatter (lanes 2i and 2i + 1
                // end with one token's sum), the four partial sums meet in shared
                // memory (two buffers: no warp gets two chunks ahead of another
                // here), and lane j < 16 turns token j's total into 1 / rms.
                float sq[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) sq[j] = ov[j] * ov[j];
                float a8[8], a4[4], a2[2];
                const unsigned full = 0xffffffffu;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const bool hi = lane & 16;
                    a8[i] = (hi ? sq[i + 8] : sq[i]) + __shfl_xor_sync(full, hi ? sq[i] : sq[i + 8], 16);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool hi = lane & 8;
                    a4[i] = (hi ? a8[i + 4] : a8[i]) + __shfl_xor_sync(full, hi ? a8[i] : a8[i + 4], 8);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const bool hi = lane & 4;
                    a2[i] = (hi ? a4[i + 2] : a4[i]) + __shfl_xor_sync(full, hi ? a4[i] : a4[i + 2], 4);
                }
                const bool hi2 = lane & 2;
                float a1 = (hi2 ? a2[1] : a2[0]) + __shfl_xor_sync(full, hi2 ? a2[0] : a2[1], 2);
                a1 += __shfl_xor_sync(full, a1, 1);
                const int tau = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                                ((lane >> 1) & 1);
                float* part = reinterpret_cast<float*>(x.sm + C_NORM + (c & 1) * 1024 + cb * 256);
                if ((lane & 1) == 0) part[tau * 4 + q] = a1;
                named_bar_sync(kNormBar0 + cb, 128);
                const float4 pp = reinterpret_cast<const float4*>(part)[lane & 15];
                const float rl = rsqrtf(((pp.x + pp.y) + (pp.z + pp.w)) * (1.f / kD) + p.eps);
                const float wv = p.norm_w[v];
                uint16_t* ycol = p.y + t0 * o_stride + col;
                // z of this chunk, loaded by TMA: [64 t][128 v] bf16, row-major
                mbar_wait(x.bar(CB_Z_FULL + b), (c >> 1) & 1, x.abort, kWaitLimitNs);
                const uint16_t* zs = reinterpret_cast<const uint16_t*>(x.sm + C_Z + b * 16384) + cb * 16 * kD + v;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float r = __shfl_sync(full, rl, j);
                    if (j < nvalid) {
                        const float zf = __uint_as_float((uint32_t)zs[j * kD] << 16);
                        const float g = __fdividef(zf, 1.f + __expf(-zf));
                        ycol[j * o_stride] = (uint16_t)f32_to_bf16_bits(wv * (ov[j] * r) * g);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(x.bar(CB_Z_EMPTY + b));
            }
        }
    }
}

// ================================================================ producer
__device__ __forceinline__ void producer(const Ctx& x, int pidx, const CUtensorMap* tm_q,
                                         const CUtensorMap* tm_k, const CUtensorMap* tm_a,
                                         const CUtensorMap* tm_b, const ClParams& p) {
    const int warp = x.warp, lane = x.lane;
    const int nch = x.nch;
    const int h = x.h;
    if (warp == 16) {
        // ------------------------------------------------ TMA: [K; Q] and gate inputs
        if (lane == 0) {
            prefetch_tmap(tm_q);
            prefetch_tmap(tm_k);
            if (p.gate_tma) { prefetch_tmap(tm_a); prefetch_tmap(tm_b); }
            // chunk i of this producer goes to stage i % 3 and to group i & 1.  The
            // group's full barrier is armed for its next chunk only after the group
            // has taken the previous one, so each barrier runs at most one phase
            // ahead of its waiters.
            int issued = 0;
            for (int i = 0;; ++i) {
                const int c = pidx + p.n_prod * i;
                if (c >= nch) break;
                const int s = i % kKqStages, grp = i & 1, jj = i >> 1;
                if (i >= kKqStages &&
                    !mbar_wait(x.bar(PB_KQ_EMPTY + s), (i / kKqStages - 1) & 1, x.abort, kWaitLimitNs))
                    break;
                if (jj >= 1 && !mbar_wait(x.bar(PB_KQ_TAKEN + grp), (jj - 1) & 1, x.abort, kWaitLimitNs))
                    break;
                const uint32_t kq = x.sbase + P_KQ + s * KQ_STAGE;
                const int32_t y = (int32_t)(x.bos + (int64_t)c * kC);
                const uint32_t fb = x.bar(PB_KQ_FULL + grp);
                mbar_arrive_expect_tx(fb, KQ_STAGE + (p.gate_tma ? AB_STAGE : 0));
                tma_load_2d(kq, tm_k, x.g * kD, y, fb);
                tma_load_2d(kq + 8192, tm_q, x.g * kD, y, fb);
                tma_load_2d(kq + KQ_PANEL, tm_k, x.g * kD + 64, y, fb);
                tma_load_2d(kq + KQ_PANEL + 8192, tm_q, x.g * kD + 64, y, fb);
                if (p.gate_tma) {
                    // the 4-column group of a and b that holds column h
                    const uint32_t ab = x.sbase + P_AB + s * AB_STAGE;
                    tma_load_2d(ab, tm_a, h & ~3, y, fb);
                    tma_load_2d(ab + 1024, tm_b, h & ~3, y, fb);
                }
                issued = i + 1;
            }
            // copies still in flight land before the CTA may exit: the last chunk
            // armed on each group's barrier
            volatile int no_abort = 0;
            for (int i = issued >= 2 ? issued - 2 : 0; i < issued; ++i)
                mbar_wait(x.bar(PB_KQ_FULL + (i & 1)), (i >> 1) & 1, &no_abort, kWaitLimitNs);
        }
        return;
    }
    if (warp == 17 || warp == 18) {
        // ------------------------------------------------ publisher of one group
        // Once the group has staged a chunk and its ring slot is free, two bulk
        // stores write it to the ring; the staging (the [K; Q] stage and the
        // group's A scratch) is reusable as soon as they have read it, and the
        // consumer is told once the bytes are in global memory.
        const int grp = warp - 17;
        if (lane == 0) {
            const uint32_t stage_rt = x.sbase + P_GROUP + grp * GROUP_BYTES + G_AF;
            for (int jj = 0;; ++jj) {
                const int i = grp + 2 * jj;
                const int c = pidx + p.n_prod * i;
                if (c >= nch) break;
                const int rs = c % kRing;
                if (!mbar_wait(x.bar(PB_STAGED + grp), jj & 1, x.abort, kWaitLimitNs)) break;
                TRACE_CLK(24, c);
                if (c >= kRing &&
                    !gflag_wait_ge(x.freed + rs, (uint32_t)(c / kRing), x.abort, x.err, kWaitLimitNs))
                    break;
                TRACE_CLK(25, c);
                fence_async_global();
                uint8_t* g = x.ring + (size_t)rs * GSLOT_BYTES;
                bulk_store(g, x.sbase + P_KQ + (i % kKqStages) * KQ_STAGE, SEND_QW);
                bulk_store(g + SEND_QW, stage_rt, SEND_RT);
                bulk_commit();
                bulk_wait_read();
                mbar_arrive(x.bar(PB_KQ_EMPTY + i % kKqStages));
                mbar_arrive(x.bar(PB_AF_FREE + grp));
                bulk_wait();
                fence_async_global();
                st_release_gpu(x.ready + rs, (uint32_t)(c / kRing + 1));
                TRACE_CLK(26, c);
            }
        }
        return;
    }
    if (warp == 19 || warp == 20) {
        // ------------------------------------------------ D0 = [K; Q] K^T of one group
        // Issued as soon as the chunk's [K; Q] has landed and the group has read
        // the previous D0, by a thread of its own (a thread that issues
        // tcgen05.mma is held until the tensor core takes them), so that D0 is
        // ready when the group turns to the chunk.
        const int grp = warp - 19;
        if (lane == 0) {
            const uint64_t dsc_kq0 = sdesc_sw128(x.sbase + P_KQ, 16, 1024);
            constexpr uint64_t kStageStep = KQ_STAGE >> 4;
            const uint32_t tg = x.tmem + 256u * grp;
            for (int jj = 0;; ++jj) {
                const int i = grp + 2 * jj;
                const int c = pidx + p.n_prod * i;
                if (c >= nch) break;
                const int s = i % kKqStages;
                if (!mbar_wait(x.bar(PB_KQ_FULL + grp), jj & 1, x.abort, kWaitLimitNs)) break;
                mbar_arrive(x.bar(PB_KQ_TAKEN + grp));
                if (jj >= 1 && !mbar_wait(x.bar(PB_D0_FREE + grp), (jj - 1) & 1, x.abort, kWaitLimitNs)) break;
                tc_fence_after();
                const uint64_t d = dsc_kq0 + s * kStageStep;
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = ((kk >> 2) * KQ_PANEL + (kk & 3) * 32) >> 4;
                    mma_bf16(tg + PCOL_D0, d + off, d + off, IDESC_D0, kk > 0);
                }
                mma_commit(x.bar(PB_D0_FULL + grp));
            }
            volatile int no_abort = 0;
            mma_commit(x.bar(PB_D0_DRAIN + grp));
            mbar_wait(x.bar(PB_D0_DRAIN + grp), 0, &no_abort, kWaitLimitNs);
        }
        return;
    }
    if (warp >= 16) return;
    // ---------------------------------------------------- precompute group
    const int grp = warp >> 3;                 // 0 or 1
    const int pw = warp & 7;                   // warp within the group
    const int q = warp & 3;                    // TMEM lane quadrant
    const int hh = pw >> 2;                    // column half
    const int pt = pw * 32 + lane;
    const int nb = 1 + grp;                    // group-wide named barrier
    const int nb_gates = 3 + grp;              // the two gate warps
    uint8_t* gbase = x.sm + P_GROUP + grp * GROUP_BYTES;
    const uint32_t gsb = x.sbase + P_GROUP + grp * GROUP_BYTES;
    float* Af = reinterpret_cast<float*>(gbase + G_AF);
    float* Tf = reinterpret_cast<float*>(gbase + G_TF);
    float* Xf = reinterpret_cast<float*>(gbase + G_XF);
    GateBuf* gates = reinterpret_cast<GateBuf*>(gbase + G_GATES);
    float* xchg = reinterpret_cast<float*>(x.sm + OFF_MISC + 16 + 8 * grp);
    const uint32_t tg = x.tmem + 256u * grp;
    const uint32_t tl = tg + ((uint32_t)(q * 32) << 16);
    const bool issuer = (pw == 0 && lane == 0);
    const float Al = p.A_log[h], dtb = p.dt_bias[h];
    uint8_t* stage_rt = gbase + G_AF;          // [T b; R b] and the gates, staged for sending
    // shared-memory descriptors, computed once (a K step or a stage adds a byte
    // offset >> 4 to the start address field): rebuilding them per instruction
    // doubles the cost of issuing a tcgen05.mma
    const uint64_t dsc_kq0 = sdesc_sw128(x.sbase + P_KQ, 16, 1024);             // [K; Q], K-major
    const uint64_t dsc_kq0_mn = sdesc_sw128(x.sbase + P_KQ, KQ_PANEL, 1024);    // K rows, MN-major
    const uint64_t dsc_pt = sdesc_sw128(gsb + G_PT, 16, 1024);                  // [P; T] / [R bg; T bg]
    const uint64_t dsc_t = sdesc_sw128(gsb + G_PT + 8192, 8192, 1024);          // T, MN-major
    constexpr uint64_t kStageStep = KQ_STAGE >> 4;

    int jj = 0;                                // chunks done by this group
    for (int i = grp;; i += 2, ++jj) {
        const int c = pidx + p.n_prod * i;
        if (c >= nch) break;
        const int s = i % kKqStages;
        GateBuf& gb = gates[jj & 1];
        const int64_t tok0 = x.bos + (int64_t)c * kC;
        const uint32_t kqo = P_KQ + s * KQ_STAGE;
        // every warp of the group has seen chunk i land before the TMA warp may
        // arm this group's barrier again
        if (pw == 0 && lane == 0) TRACE_CLK(16, c);
        mbar_wait(x.bar(PB_KQ_FULL + grp), jj & 1, x.abort, kWaitLimitNs);
        if (pw == 0 && lane == 0) TRACE_CLK(17, c);
        __syncwarp();
        if (lane == 0) mbar_arrive(x.bar(PB_KQ_TAKEN + grp));
        // ---- gates (warps 6, 7 of the group): G = running sum of log2(alpha);
        //      beta; gamma = 2^G; kappa = 2^{G_C - G}
        if (pw >= 6) {
            const int t = pt - 192;
            const int64_t tok = tok0 + t;
            const float* abt = reinterpret_cast<const float*>(x.sm + P_AB + s * AB_STAGE);
            float lg = 0.f, be = 0.f;
            if (tok < x.eos) {
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
            named_bar_sync(nb_gates, 64);
            if (pw == 7) run += xchg[0];
            gb.G[t] = run;
            gb.beta[t] = be;
            gb.gamma[t] = exp2f(run);
            if (t == 63) {
                xchg[1] = run;
                gb.gC = exp2f(run);
                gb.fast = run >= -kFastDecayLog2 ? 1 : 0;
            }
            named_bar_sync(nb_gates, 64);
            gb.kappa[t] = exp2f(xchg[1] - run);
            gb.igamma[t] = xchg[1] >= -kFastDecayLog2 ? exp2f(-run) : 0.f;
        }
        named_bar_sync(nb, kGroupThreads);
        // ---- D0 rows -> A (f32 scratch) and P (bf16 operand); each warp 32 columns.
        //      The A scratch last held the previous chunk's staged bytes.
        if (jj >= 1) mbar_wait(x.bar(PB_AF_FREE + grp), (jj - 1) & 1, x.abort, kWaitLimitNs);
        if (pw == 0 && lane == 0) TRACE_CLK(18, c);
        mbar_wait(x.bar(PB_D0_FULL + grp), jj & 1, x.abort, kWaitLimitNs);
        if (pw == 0 && lane == 0) TRACE_CLK(19, c);
        tc_fence_after();
        {
            // eight columns at a time, the loop not unrolled (a smaller hot loop)
            const bool fast = gb.fast != 0;
            const int i_ = (q & 1) * 32 + lane;      // row within KK^T (q<2) or QK^T (q>=2)
            const float Gi = gb.G[i_];
            // (the fast and the slow decay forms in separate loops, so that the loop that
            // runs holds one of them)
            if (q < 2) {
                // A_ij = beta_i 2^{G_i - G_j} (k_i . k_j), j < i
                float* arow = Af + i_ * kLdF + hh * 32;
                if (fast) {
                    const float ci = gb.beta[i_] * gb.gamma[i_];
#pragma unroll 1
                    for (int j8 = 0; j8 < 4; ++j8) {
                        float dv[8];
                        tmem_ld8(tl + PCOL_D0 + hh * 32 + j8 * 8, dv);
                        tmem_ld_wait();
#pragma unroll
                        for (int h4 = 0; h4 < 2; ++h4) {
                            const int j4 = 4 * h4;
                            const int j = hh * 32 + j8 * 8 + j4;
                            const float4 ig = *reinterpret_cast<const float4*>(&gb.igamma[j]);
                            float4 w;
                            w.x = (j + 0 < i_) ? ci * dv[j4 + 0] * ig.x : 0.f;
                            w.y = (j + 1 < i_) ? ci * dv[j4 + 1] * ig.y : 0.f;
                            w.z = (j + 2 < i_) ? ci * dv[j4 + 2] * ig.z : 0.f;
                            w.w = (j + 3 < i_) ? ci * dv[j4 + 3] * ig.w : 0.f;
                            *reinterpret_cast<float4*>(arow + j8 * 8 + j4) = w;
                        }
                    }
                } else {
                    const float ci = gb.beta[i_];
#pragma unroll 1
                    for (int j8 = 0; j8 < 4; ++j8) {
                        float dv[8];
                        tmem_ld8(tl + PCOL_D0 + hh * 32 + j8 * 8, dv);
                        tmem_ld_wait();
#pragma unroll
                        for (int h4 = 0; h4 < 2; ++h4) {
                            const int j4 = 4 * h4;
                            const int j = hh * 32 + j8 * 8 + j4;
                            const float4 gj = *reinterpret_cast<const float4*>(&gb.G[j]);
                            float4 w;
                            w.x = (j + 0 < i_) ? ci * dv[j4 + 0] * exp2f(Gi - gj.x) : 0.f;
                            w.y = (j + 1 < i_) ? ci * dv[j4 + 1] * exp2f(Gi - gj.y) : 0.f;
                            w.z = (j + 2 < i_) ? ci * dv[j4 + 2] * exp2f(Gi - gj.z) : 0.f;
                            w.w = (j + 3 < i_) ? ci * dv[j4 + 3] * exp2f(Gi - gj.w) : 0.f;
                            *reinterpret_cast<float4*>(arow + j8 * 8 + j4) = w;
                        }
                    }
                }
            } else {
                // P_ij = 2^{G_i - G_j} (q_i . k_j), j <= i
                if (fast) {
                    const float ci = gb.gamma[i_];
#pragma unroll 1
                    for (int j8 = 0; j8 < 4; ++j8) {
                        float dv[8];
                        tmem_ld8(tl + PCOL_D0 + hh * 32 + j8 * 8, dv);
                        tmem_ld_wait();
#pragma unroll
                        for (int h4 = 0; h4 < 2; ++h4) {
                            const int j4 = 4 * h4;
                            const int j = hh * 32 + j8 * 8 + j4;
                            const float4 ig = *reinterpret_cast<const float4*>(&gb.igamma[j]);
                            dv[j4 + 0] = (j + 0 <= i_) ? ci * dv[j4 + 0] * ig.x : 0.f;
                            dv[j4 + 1] = (j + 1 <= i_) ? ci * dv[j4 + 1] * ig.y : 0.f;
                            dv[j4 + 2] = (j + 2 <= i_) ? ci * dv[j4 + 2] * ig.z : 0.f;
                            dv[j4 + 3] = (j + 3 <= i_) ? ci * dv[j4 + 3] * ig.w : 0.f;
                        }
                        st_bf16x8(gbase + G_PT, i_, hh * 4 + j8, dv);
                    }
                } else {
#pragma unroll 1
                    for (int j8 = 0; j8 < 4; ++j8) {
                        float dv[8];
                        tmem_ld8(tl + PCOL_D0 + hh * 32 + j8 * 8, dv);
                        tmem_ld_wait();
#pragma unroll
                        for (int h4 = 0; h4 < 2; ++h4) {
                            const int j4 = 4 * h4;
                            const int j = hh * 32 + j8 * 8 + j4;
                            const float4 gj = *reinterpret_cast<const float4*>(&gb.G[j]);
                            dv[j4 + 0] = (j + 0 <= i_) ? dv[j4 + 0] * exp2f(Gi - gj.x) : 0.f;
                            dv[j4 + 1] = (j + 1 <= i_) ? dv[j4 + 1] * exp2f(Gi - gj.y) : 0.f;
                            dv[j4 + 2] = (j + 2 <= i_) ? dv[j4 + 2] * exp2f(Gi - gj.z) : 0.f;
                            dv[j4 + 3] = (j + 3 <= i_) ? dv[j4 + 3] * exp2f(Gi - gj.w) : 0.f;
                        }
                        st_bf16x8(gbase + G_PT, i_, hh * 4 + j8, dv);
                    }
                }
            }
        }
        tc_fence_before();
        named_bar_sync(nb, kGroupThreads);
        // D0 has been read: the next chunk's D0 may be issued into it
        if (pw == 0 && lane == 0) mbar_arrive(x.bar(PB_D0_FREE + grp));
        // ---- T = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution
        if (pw < 4) {
            const int blk = pw;
            const int col = lane & 15;
            const float* Ab = Af + (16 * blk) * kLdF + 16 * blk;
            float xv[16];
#pragma unroll
            for (int ii = 0; ii < 16; ++ii) {
                float arow[16];
#pragma unroll
                for (int m4 = 0; m4 < ii; m4 += 4) {
                    const float4 a4 = *reinterpret_cast<const float4*>(Ab + ii * kLdF + m4);
                    arow[m4] = a4.x; arow[m4 + 1] = a4.y; arow[m4 + 2] = a4.z; arow[m4 + 3] = a4.w;
                }
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < ii; ++m) acc[m & 3] = fmaf(arow[m], xv[m], acc[m & 3]);
                xv[ii] = ((ii == col) ? 1.f : 0.f) - ((acc[0] + acc[1]) + (acc[2] + acc[3]));
            }
            if (lane < 16) {
#pragma unroll
                for (int ii = 0; ii < 16; ++ii) Tf[(16 * blk + ii) * kLdF + 16 * blk + col] = xv[ii];
            }
        }
        named_bar_sync(nb, kGroupThreads);
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
        named_bar_sync(nb, kGroupThreads);
        // ---- 64x64: T[32:64, 0:32] = -T[32:64, 32:64] A[32:64, 0:32] T[0:32, 0:32]
        {
            const int mt = pw >> 2, nt = pw & 3;
            float cfr[4];
            mma_tile(cfr, Af, kLdF, 32 + 16 * mt, 0, Tf, kLdF, 0, 8 * nt, nt, 4, lane);
            frag_c_store(Xf, 36, 16 * mt, 8 * nt, cfr, 1.f, lane);
            named_bar_sync(nb, kGroupThreads);
            mma_tile(cfr, Tf, kLdF, 32 + 16 * mt, 32, Xf, 36, 0, 8 * nt, 0, 2 * mt + 2, lane);
            frag_c_store(Tf, kLdF, 32 + 16 * mt, 8 * nt, cfr, -1.f, lane);
        }
        named_bar_sync(nb, kGroupThreads);
        if (pw == 0 && lane == 0) TRACE_CLK(20, c);
        // ---- T (bf16) as the B operand of R = P T
        for (int u = pt; u < 64 * 8; u += kGroupThreads) {
            const int row = u >> 3, chunk = u & 7;
            const float4 t0 = *reinterpret_cast<const float4*>(Tf + row * kLdF + chunk * 8);
            const float4 t1 = *reinterpret_cast<const float4*>(Tf + row * kLdF + chunk * 8 + 4);
            const float xv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            st_bf16x8(gbase + G_PT + 8192, row, chunk, xv);
        }
        fence_async_smem();
        named_bar_sync(nb, kGroupThreads);
        if (issuer) {
            // R = [P; T] T (rows 0-63 used)
            tc_fence_after();
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tg + PCOL_R, dsc_pt + kk * 2, dsc_t + kk * 128, IDESC_R, kk > 0);
            mma_commit(x.bar(PB_R_FULL + grp));
        }
        __syncwarp();
        // ---- [R bg; T bg] (over P | T once R is done) and, staged for sending,
        //      [T b; R b] with the gates (over A, which the solve no longer needs)
        mbar_wait(x.bar(PB_R_FULL + grp), jj & 1, x.abort, kWaitLimitNs);
        if (pw == 0 && lane == 0) TRACE_CLK(21, c);
        tc_fence_after();
        {
            const int i_ = (q & 1) * 32 + lane;
            const int row = (q < 2 ? 0 : 64) + i_;     // [R bg; T bg]: R in rows 0-63
            const int row2 = (q < 2 ? 64 : 0) + i_;    // [T b; R b]: T in rows 0-63
            // eight columns at a time, the loop not unrolled (a smaller hot loop)
#pragma unroll 1
            for (int j8 = 0; j8 < 4; ++j8) {
                const int j0 = hh * 32 + j8 * 8;
                float v8[8];
                if (q < 2) {
                    tmem_ld8(tl + PCOL_R + j0, v8);
                    tmem_ld_wait();
                } else {
                    const float4 t0 = *reinterpret_cast<const float4*>(Tf + i_ * kLdF + j0);
                    const float4 t1 = *reinterpret_cast<const float4*>(Tf + i_ * kLdF + j0 + 4);
                    v8[0] = t0.x; v8[1] = t0.y; v8[2] = t0.z; v8[3] = t0.w;
                    v8[4] = t1.x; v8[5] = t1.y; v8[6] = t1.z; v8[7] = t1.w;
                }
                const float4 b0 = *reinterpret_cast<const float4*>(&gb.beta[j0]);
                const float4 b1 = *reinterpret_cast<const float4*>(&gb.beta[j0 + 4]);
                const float4 g0 = *reinterpret_cast<const float4*>(&gb.gamma[j0]);
                const float4 g1 = *reinterpret_cast<const float4*>(&gb.gamma[j0 + 4]);
                const float bj[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                const float gj[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                float wb[8], wg[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    wb[e] = v8[e] * bj[e];
                    wg[e] = wb[e] * gj[e];
                }
                st_bf16x8(gbase + G_PT, row, hh * 4 + j8, wg);
                st_bf16x8(stage_rt, row2, hh * 4 + j8, wb);
            }
            if (q < 2 && hh == 0) {
                float* sg = reinterpret_cast<float*>(stage_rt + GATES_AT);
                sg[i_] = gb.kappa[i_];
                if (i_ == 63) sg[64] = gb.gC;
            }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar_sync(nb, kGroupThreads);
        if (issuer) {
            // X1 = [R bg; T bg] K  ->  rows 0-63: P W, rows 64-127: W
            tc_fence_after();
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tg + PCOL_X1, dsc_pt + kk * 2, dsc_kq0_mn + s * kStageStep + kk * 128, IDESC_X1,
                         kk > 0);
            mma_commit(x.bar(PB_X1_FULL + grp));
        }
        __syncwarp();
        mbar_wait(x.bar(PB_X1_FULL + grp), jj & 1, x.abort, kWaitLimitNs);
        if (pw == 0 && lane == 0) TRACE_CLK(22, c);
        tc_fence_after();
        // ---- -W over the K rows and Qh = diag(gamma) Q - P W over the Q rows of the
        //      [K; Q] stage (each thread rewrites the Q chunks it has just read)
        {
            const int i_ = (q & 1) * 32 + lane;
            const float ga = gb.gamma[i_];
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                const int dcol = hh * 64 + part * 32;          // 32 of the 128 d columns
                const int panel = dcol >> 6, ch0 = (dcol & 63) >> 3;
                float xv[32];
                tmem_ld32(tl + PCOL_X1 + dcol, xv);
                tmem_ld_wait();
                if (q < 2) {
                    const uint8_t* qrow = x.sm + kqo + panel * KQ_PANEL + 8192;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float qv[8];
                        ld_bf16x8(qrow, i_, ch0 + j, qv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) xv[8 * j + e] = ga * qv[e] - xv[8 * j + e];
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) xv[e] = -xv[e];
                }
                uint8_t* dst = x.sm + kqo + panel * KQ_PANEL + (q < 2 ? 8192 : 0);
#pragma unroll
                for (int j = 0; j < 4; ++j) st_bf16x8(dst, i_, ch0 + j, xv + 8 * j);
            }
        }
        // staged: the publisher may send the chunk
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(x.bar(PB_STAGED + grp));
        if (pw == 0 && lane == 0) TRACE_CLK(23, c);
    }
    if (issuer) {
        volatile int no_abort = 0;
        mma_commit(x.bar(PB_DRAIN + grp));
        mbar_wait(x.bar(PB_DRAIN + grp), 0, &no_abort, kWaitLimitNs);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_pc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                  const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_z,
                  const ClParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // align to 1024 bytes by pointer arithmetic on the shared array, so that
    // every access below stays in the shared state space
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx x;
    x.sm = sm;
    x.sbase = smem_u32(sm);
    x.bar0 = x.sbase + OFF_BARS;
    x.abort = reinterpret_cast<volatile int*>(sm + OFF_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC + 4);
    x.warp = threadIdx.x >> 5;
    x.lane = threadIdx.x & 31;
    // blocks [0, nu) are the consumers of the launch's nu units, then the first
    // producers of every unit, then the second ones: consecutive blocks tend to
    // land on the two SMs of one TPC, and a consumer next to a producer runs its
    // state chain about half as fast as next to another consumer
    const uint32_t nu = gridDim.x / (uint32_t)(p.n_prod + 1);
    const int slot = (int)(blockIdx.x % nu);                        // unit within this launch
    const uint32_t rank = blockIdx.x / nu;                          // 0 = consumer, 1.. = producers
    const int unit = p.unit0 + slot;
    x.h = unit % p.Hv;
    const int n = unit / p.Hv;
    x.g = x.h / (p.Hv / p.Hqk);
    x.bos = p.cu ? p.cu[n] : 0;
    x.eos = p.cu ? p.cu[n + 1] : p.T;
    x.nch = (int)((x.eos - x.bos + kC - 1) / kC);
    x.state_off = ((int64_t)n * p.Hv + x.h) * kD * kD;
    x.ring = p.ring + (size_t)slot * kRing * GSLOT_BYTES;
#ifdef GDN_PREFILL_TRACE
    x.traced = (unit == g_prefill_trace_unit);
#else
    x.traced = 0;
#endif
    x.ready = p.flags + (size_t)slot * kFlagWords;
    x.freed = x.ready + kFreedAt;
    x.err = p.err;

    if (x.nch == 0) {
        // empty sequence (the same in every CTA of the unit): final state = initial state
        if (rank == 0 && p.s_out && p.s_out != p.s_in) {
            for (int i = threadIdx.x; i < kD * kD; i += kThreads)
                p.s_out[x.state_off + i] = p.s_in ? p.s_in[x.state_off + i] : 0.f;
        }
        return;
    }

    if (threadIdx.x == 0) {
        *x.abort = 0;
        if (rank == 0) {
            for (int b = 0; b < 2; ++b) {
                mbar_init(x.bar(CB_RECV_FULL + b), 1);
                mbar_init(x.bar(CB_SLOT_FREE + b), 1);
                mbar_init(x.bar(CB_REL_DONE + b), 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(x.bar(CB_K_FULL + b), 1);
                mbar_init(x.bar(CB_K_EMPTY + b), 1);
                mbar_init(x.bar(CB_V_FULL + b), 1);
                mbar_init(x.bar(CB_V_EMPTY + b), 1);
            }
            mbar_init(x.bar(CB_D_FULL), 1);
            mbar_init(x.bar(CB_EPI1_DONE), kEpiThreads / 32);
            for (int j = 0; j < 4; ++j) mbar_init(x.bar(CB_EPI2_BLK + j), kEpiThreads / 32);
            mbar_init(x.bar(CB_E_FULL), 1);
            mbar_init(x.bar(CB_E_DRAIN), 1);
            mbar_init(x.bar(CB_CHAIN_ISSUED), 1);
            mbar_init(x.bar(CB_SUPD_ISSUED), 1);
            for (int b = 0; b < 2; ++b) {
                mbar_init(x.bar(CB_Z_FULL + b), 1);
                mbar_init(x.bar(CB_Z_EMPTY + b), kEpiThreads / 32);
            }
            mbar_init(x.bar(CB_S_FULL), 1);
            mbar_init(x.bar(CB_DRAIN), 1);
        } else {
            for (int s = 0; s < kKqStages; ++s) mbar_init(x.bar(PB_KQ_EMPTY + s), 1);
            for (int grp = 0; grp < 2; ++grp) {
                mbar_init(x.bar(PB_KQ_FULL + grp), 1);
                mbar_init(x.bar(PB_KQ_TAKEN + grp), 9);     // the group's 8 warps and its D0 issuer
                mbar_init(x.bar(PB_D0_FULL + grp), 1);
                mbar_init(x.bar(PB_R_FULL + grp), 1);
                mbar_init(x.bar(PB_X1_FULL + grp), 1);
                mbar_init(x.bar(PB_DRAIN + grp), 1);
                mbar_init(x.bar(PB_STAGED + grp), 8);
                mbar_init(x.bar(PB_AF_FREE + grp), 1);
                mbar_init(x.bar(PB_D0_FREE + grp), 1);
                mbar_init(x.bar(PB_D0_DRAIN + grp), 1);
            }
        }
        fence_mbar_init();
    }
    if (x.warp == 2) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    if (rank != 0) {
        // zero the strictly upper blocks of both groups' T scratch (never written again)
        for (int gi = 0; gi < 2; ++gi) {
            float* Tf = reinterpret_cast<float*>(sm + P_GROUP + gi * GROUP_BYTES + G_TF);
            for (int i = threadIdx.x; i < 64 * kLdF; i += kThreads) Tf[i] = 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = *tmem_slot;

    if (rank == 0)
        consumer(x, &tm_k, &tm_v, &tm_z, p);
    else
        producer(x, (int)rank - 1, &tm_q, &tm_k, &tm_a, &tm_b, p);

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    // a CTA that gave up records it; the other CTAs' waits on global counters
    // see the error word and give up too
    if (threadIdx.x == 0 && *x.abort) atomicOr(p.err, 1u);
    if (x.warp == 2) {
        tc_fence_after();
        tmem_dealloc(x.tmem, TMEM_COLS);
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

// 2D bf16 tensor [rows, cols], 128-column x 64-row boxes, no swizzle (a
// row-major [64][128] tile: the output norm's gate z of one value head)
bool make_map_plain(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {128, 64};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
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

cudaError_t setup_kernel() {
    return cudaFuncSetAttribute(prefill_pc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)SMEM_ALLOC);
}

// CTAs of this kernel that can be resident at once on the current device (0 if
// none); cached per device
std::atomic<int> g_resident[64];           // stored + 1 (0 = unknown)

int resident_ctas() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int v = g_resident[dev].load(std::memory_order_relaxed);
    if (v > 0) return v - 1;
    int per_sm = 0, sms = 0, coop = 0;
    if (setup_kernel() != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefill_pc_kernel, kThreads, SMEM_ALLOC) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop)
        per_sm = 0;
    cudaGetLastError();    // a refused query leaves no sticky error behind
    const int total = per_sm * sms;
    g_resident[dev].store(total + 1, std::memory_order_relaxed);
    return total;
}

// Producer CTAs per unit: two keep the consumer's state chain busy; one when
// fewer than three CTAs are resident.  GDN_PREFILL_PRODUCERS=1 or =2 in the
// environment forces the choice.
int pick_producers(int resident) {
    const char* env = getenv("GDN_PREFILL_PRODUCERS");
    if (env && (env[0] == '1' || env[0] == '2') && env[1] == 0) {
        const int want = env[0] - '0';
        return resident >= want + 1 ? want : 0;
    }
    return resident >= 3 ? 2 : (resident >= 2 ? 1 : 0);
}

size_t ring_bytes_per_unit() { return (size_t)kRing * GSLOT_BYTES + kFlagWords * sizeof(uint32_t); }

// units whose ring a workspace of `bytes` holds
int64_t slots_in(size_t bytes) {
    if (bytes < kWsHeaderBytes) return 0;
    return (int64_t)((bytes - kWsHeaderBytes) / ring_bytes_per_unit());
}

}  // namespace

size_t prefill_pc_smem_bytes() { return SMEM_ALLOC; }

size_t prefill_pc_workspace_bytes(int32_t n_seq, int32_t Hv) {
    const int64_t units = (int64_t)(n_seq > 0 ? n_seq : 1) * (Hv > 0 ? Hv : 1);
    const int64_t slots = units < kMaxSlots ? units : kMaxSlots;
    return kWsHeaderBytes + (((size_t)slots * ring_bytes_per_unit() + 255) / 256) * 256;
}

bool prefill_pc_available(size_t workspace_bytes) {
    return slots_in(workspace_bytes) >= 1 && resident_ctas() >= 2;
}

cudaError_t launch_prefill_pc(const PrefillArgs& a, cudaStream_t stream) {
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
    CUtensorMap mq, mk, mv, ma, mb, mz;
    if (!make_map(&mq, a.q, a.T, (int64_t)a.Hqk * kD) || !make_map(&mk, a.k, a.T, (int64_t)a.Hqk * kD) ||
        !make_map(&mv, a.v, a.T, (int64_t)a.Hv * kD))
        return cudaErrorInvalidValue;
    if (a.y) {
        if (!make_map_plain(&mz, a.z, a.T, (int64_t)a.Hv * kD)) return cudaErrorInvalidValue;
    } else {
        mz = mq;       // unused
    }
    // a and b rows must be a multiple of 16 bytes for TMA; otherwise they are read directly
    const int gate_tma = (a.Hv % 4 == 0) ? 1 : 0;
    if (gate_tma) {
        if (!make_map_gates(&ma, a.a, a.T, a.Hv) || !make_map_gates(&mb, a.b, a.T, a.Hv))
            return cudaErrorInvalidValue;
    } else {
        ma = mq;
        mb = mq;       // unused
    }
    cudaError_t e = setup_kernel();
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)a.n_seq * a.Hv;
    const int resident = resident_ctas();
    const int n_prod = pick_producers(resident);
    if (n_prod == 0) return cudaErrorNotSupported;
    const int csize = n_prod + 1;
    int64_t per_launch = resident / csize;
    const int64_t slots = slots_in(a.workspace_bytes);
    if (per_launch > slots) per_launch = slots;
    if (per_launch > kMaxSlots) per_launch = kMaxSlots;
    if (per_launch < 1) return cudaErrorNotSupported;
    // whole sequences per launch where they fit, so that a launch's units end
    // together when the sequences differ in length
    if (per_launch > a.Hv && units > per_launch) per_launch -= per_launch % a.Hv;
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    uint32_t* flags = reinterpret_cast<uint32_t*>(ws + kWsHeaderBytes);
    uint8_t* ring = ws + kWsHeaderBytes + (size_t)per_launch * kFlagWords * sizeof(uint32_t);
    ClParams p{a.a, a.b, a.A_log, a.dt_bias, a.cu_seqlens, a.T, a.Hqk, a.Hv, a.scale,
               a.initial_state, a.final_state, a.o,
               reinterpret_cast<uint32_t*>(ws + kWsErrorWordOffset), ring, flags, gate_tma, n_prod, 0,
               a.z, a.norm_w, a.eps, a.y, a.o16};
    // Units run in launches of at most per_launch units, in order; each launch
    // starts from cleared counters.  A unit's CTAs wait on one another, so each
    // launch is cooperative (all of its CTAs resident together).
    for (int64_t u0 = 0; u0 < units; u0 += per_launch) {
        const int64_t nu = units - u0 < per_launch ? units - u0 : per_launch;
        e = cudaMemsetAsync(flags, 0, (size_t)nu * kFlagWords * sizeof(uint32_t), stream);
        if (e != cudaSuccess) return e;
        p.unit0 = (int)u0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(nu * csize));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = SMEM_ALLOC;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, prefill_pc_kernel, mq, mk, mv, ma, mb, mz, p);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace gdn

#ifdef GDN_PREFILL_TRACE
// tracing builds only: read the recorded events and choose the unit to record
extern "C" int gdn_prefill_trace_read(void* host, int next_unit) {
    int e = (int)cudaMemcpyFromSymbol(host, gdn::g_prefill_trace, sizeof(gdn::g_prefill_trace));
    if (e) return e;
    return (int)cudaMemcpyToSymbol(gdn::g_prefill_trace_unit, &next_unit, sizeof(int));
}
#endif
