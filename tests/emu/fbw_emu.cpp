// Host emulation of the front end's gradient kernels (conv1d_silu_backward.cuh)
// for the CPU tests: the block functions run as written, one host thread per
// CUDA thread (emu_common.h), in the launch order of conv1d_silu_backward.cu.
// Outputs and the workspace start as NaN.
//
// usage: fbw_emu <dir>   reads <dir>/meta.txt and the raw inputs the test
// writes, writes d_qkv, d_conv_w (and d_conv_state) as raw float32 files.
#include <cstring>

#include "emu_common.h"

#define BWC_FN inline
#define BWC_HD inline
#define BWC_SYNC() ::emu::g_bar->arrive_and_wait()
#define BWC_SHFL_XOR(v, m) ::emu::shfl_xor((v), (m))
#include "../../gated_deltanet_recurrence_prefill_b200/csrc/conv1d_silu_backward.cuh"

using namespace gdn::fbw;
using emu::load;
using emu::save;

int main(int argc, char** argv) {
    if (argc != 2) return 2;
    const std::string dir = argv[1];
    int n_seq, Hqk, Hv, has_cu, has_cs, has_dcs;
    long long T;
    FILE* m = fopen((dir + "/meta.txt").c_str(), "r");
    if (!m || fscanf(m, "%d %lld %d %d %d %d %d", &n_seq, &T, &Hqk, &Hv, &has_cu, &has_cs, &has_dcs) != 7) return 2;
    fclose(m);
    const int n_heads = 2 * Hqk + Hv;
    const size_t Ctot = (size_t)n_heads * kD;
    auto x = load<uint16_t>(dir + "/qkv.bin", (size_t)T * Ctot);
    auto w = load<float>(dir + "/w.bin", Ctot * 4);
    auto dq = load<float>(dir + "/dq.bin", (size_t)T * Hqk * kD);
    auto dk = load<float>(dir + "/dk.bin", (size_t)T * Hqk * kD);
    auto dv = load<float>(dir + "/dv.bin", (size_t)T * Hv * kD);
    std::vector<int32_t> cu;
    std::vector<float> cs;
    if (has_cu) cu = load<int32_t>(dir + "/cu.bin", n_seq + 1);
    if (has_cs) cs = load<float>(dir + "/cs.bin", (size_t)n_seq * Ctot * 3);
    std::vector<float> dx((size_t)T * Ctot, NAN), dw(Ctot * 4, NAN), dcs((size_t)n_seq * Ctot * 3, NAN);
    std::vector<float> ws((size_t)n_tiles(T) * Ctot * 4 + 1, NAN);

    Params p;
    p.x = x.data(); p.w = w.data(); p.cu = has_cu ? cu.data() : nullptr; p.cs = has_cs ? cs.data() : nullptr;
    p.dq = dq.data(); p.dk = dk.data(); p.dv = dv.data();
    p.n_seq = n_seq; p.Hqk = Hqk; p.Hv = Hv; p.T = T; p.n_tiles = n_tiles(T);
    p.dx = dx.data(); p.dwp = ws.data(); p.dw = dw.data(); p.dcs = has_dcs ? dcs.data() : nullptr;

    // the launch sequence of launch_conv1d_silu_backward
    emu::Pool pool(kThreads);
    if (p.dcs) std::fill(dcs.begin(), dcs.end(), 0.f);
    const int64_t jobs = p.n_tiles * n_heads;
    for (int64_t j = 0; j < jobs; ++j)
        pool.run(kTileFloats, [&](int tid, float* sm) { tile_block(p, j / n_heads, (int)(j % n_heads), tid, sm); });
    if (jobs > 0) {
        for (int64_t blk = 0; blk < ((int64_t)Ctot * 4 + kThreads - 1) / kThreads; ++blk)
            pool.run(0, [&](int tid, float*) { reduce_w_block(p, blk, tid); });
    } else {
        std::fill(dw.begin(), dw.end(), 0.f);
    }
    save(dir + "/dx.out", dx.data(), dx.size());
    save(dir + "/dw.out", dw.data(), dw.size());
    if (has_dcs) save(dir + "/dcs.out", dcs.data(), dcs.size());
    return 0;
}
