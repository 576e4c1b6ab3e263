// Host emulation of the chunked backward's kernels, for the CPU tests.
//
// The block functions of backward_chunked.cuh run here exactly as written, one
// host thread per CUDA thread of a 256-thread block, with a std::barrier for
// the block-wide barrier; blocks run one after another in the launch order of
// backward_chunked.cu.  Shared memory and the workspace start filled with NaN
// (the GPU does not clear them either), so a value read before it is written
// shows in the result.  Built with AddressSanitizer by the test, so that an
// out-of-bounds index aborts the run.
//
// usage: bwc_emu <dir>   reads <dir>/meta.txt and the raw input files the test
// writes, runs the backward, writes the gradients as raw float32 files.
#include "emu_common.h"

#define BWC_FN inline
#define BWC_HD inline
#define BWC_SYNC() ::emu::g_bar->arrive_and_wait()
#include "../../gated_deltanet_recurrence_prefill_b200/csrc/backward_chunked.cuh"

using namespace gdn::bwc;
using emu::load;
using emu::save;

static emu::Pool* g_pool = nullptr;

template <class F>
static void run_block(size_t smem_floats, F f) {
    g_pool->run(smem_floats, f);
}

int main(int argc, char** argv) {
    if (argc != 2) return 2;
    const std::string dir = argv[1];
    int n_seq, Hqk, Hv, has_cu, has_s0, has_fin, has_init;
    long long T;
    float scale;
    FILE* m = fopen((dir + "/meta.txt").c_str(), "r");
    if (!m || fscanf(m, "%d %lld %d %d %f %d %d %d %d", &n_seq, &T, &Hqk, &Hv, &scale, &has_cu, &has_s0, &has_fin,
                     &has_init) != 9)
        return 2;
    fclose(m);
    const size_t st = (size_t)n_seq * Hv * kD * kD;
    auto q = load<uint16_t>(dir + "/q.bin", (size_t)T * Hqk * kD);
    auto k = load<uint16_t>(dir + "/k.bin", (size_t)T * Hqk * kD);
    auto v = load<uint16_t>(dir + "/v.bin", (size_t)T * Hv * kD);
    auto a = load<float>(dir + "/a.bin", (size_t)T * Hv);
    auto b = load<float>(dir + "/b.bin", (size_t)T * Hv);
    auto A_log = load<float>(dir + "/A_log.bin", Hv);
    auto dt_bias = load<float>(dir + "/dt_bias.bin", Hv);
    auto d_o = load<float>(dir + "/do.bin", (size_t)T * Hv * kD);
    std::vector<int32_t> cu;
    std::vector<float> s0, fin;
    if (has_cu) cu = load<int32_t>(dir + "/cu.bin", n_seq + 1);
    if (has_s0) s0 = load<float>(dir + "/s0.bin", st);
    if (has_fin) fin = load<float>(dir + "/fin.bin", st);
    std::vector<float> dq((size_t)T * Hqk * kD, NAN), dk((size_t)T * Hqk * kD, NAN), dv((size_t)T * Hv * kD, NAN),
        da((size_t)T * Hv, NAN), db((size_t)T * Hv, NAN), dA_log(Hv, NAN), ddt(Hv, NAN), dinit(st, NAN);

    emu::Pool pool(kThreads);
    g_pool = &pool;
    const Plan plan = make_plan(n_seq, T, Hv);
    std::vector<float> ws(plan.bytes / sizeof(float), NAN);
    Params p;
    p.q = q.data(); p.k = k.data(); p.v = v.data(); p.a = a.data(); p.b = b.data();
    p.A_log = A_log.data(); p.dt_bias = dt_bias.data(); p.cu = has_cu ? cu.data() : nullptr;
    p.s0 = has_s0 ? s0.data() : nullptr; p.d_o = d_o.data(); p.d_fin = has_fin ? fin.data() : nullptr;
    p.n_seq = n_seq; p.Hqk = Hqk; p.Hv = Hv; p.T = T; p.scale = scale;
    p.dq = dq.data(); p.dk = dk.data(); p.dv = dv.data(); p.da = da.data(); p.db = db.data();
    p.dA_log = dA_log.data(); p.ddt_bias = ddt.data(); p.d_init = has_init ? dinit.data() : nullptr;
    bind_workspace(p, ws.data(), plan);

    // the launch sequence of launch_backward_chunked
    memset(p.jobs, 0xFF, (size_t)plan.n_slots * 2 * sizeof(int32_t));
    for (int n = 0; n < n_seq; ++n) run_block(0, [&](int tid, float*) { fill_jobs(p, n, tid); });
    const int64_t jobs = plan.n_slots * Hv;
    for (int64_t x = 0; x < jobs; ++x)
        run_block(kPrepFloats, [&](int tid, float* sm) { prep_block(p, x / Hv, (int)(x % Hv), tid, sm); });
    const int64_t chains = (int64_t)n_seq * Hv * kRowSplit;
    for (int64_t x = 0; x < chains; ++x) {
        const int64_t unit = x / kRowSplit;
        run_block(kChainFloats, [&](int tid, float* sm) {
            fwd_chain_block(p, (int)(unit / Hv), (int)(unit % Hv), (int)(x % kRowSplit), tid, sm);
        });
    }
    for (int64_t x = 0; x < chains; ++x) {
        const int64_t unit = x / kRowSplit;
        run_block(kChainFloats, [&](int tid, float* sm) {
            bwd_chain_block(p, (int)(unit / Hv), (int)(unit % Hv), (int)(x % kRowSplit), tid, sm);
        });
    }
    for (int64_t x = 0; x < jobs; ++x)
        run_block(kGradFloats, [&](int tid, float* sm) { grad_block(p, x / Hv, (int)(x % Hv), tid, sm); });
    const int64_t nqk = T * Hqk * kD;
    for (int64_t blk = 0; blk < (nqk + kThreads - 1) / kThreads; ++blk)
        run_block(0, [&](int tid, float*) { reduce_qk_block(p, blk, tid); });
    run_block(0, [&](int tid, float*) { reduce_gates_block(p, tid); });

    save(dir + "/dq.out", dq.data(), dq.size());
    save(dir + "/dk.out", dk.data(), dk.size());
    save(dir + "/dv.out", dv.data(), dv.size());
    save(dir + "/da.out", da.data(), da.size());
    save(dir + "/db.out", db.data(), db.size());
    save(dir + "/dA_log.out", dA_log.data(), dA_log.size());
    save(dir + "/ddt_bias.out", ddt.data(), ddt.size());
    if (has_init) save(dir + "/dinit.out", dinit.data(), dinit.size());
    return 0;
}
