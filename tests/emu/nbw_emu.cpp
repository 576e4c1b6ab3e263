// Host emulation of the gated norm's gradient kernels (gated_norm_backward.cuh)
// for the CPU tests: the block functions run as written, one host thread per
// CUDA thread (emu_common.h), in the launch order of gated_norm_backward.cu.
// Outputs and the workspace start as NaN.
//
// usage: nbw_emu <dir>   reads <dir>/meta.txt and raw inputs, writes d_o, d_z,
// d_norm_w as raw float32 files.
#include <cstring>

#include "emu_common.h"

#define BWC_FN inline
#define BWC_HD inline
#define BWC_SYNC() ::emu::g_bar->arrive_and_wait()
#define BWC_SHFL_XOR(v, m) ::emu::shfl_xor((v), (m))
#include "../../gated_deltanet_recurrence_prefill_b200/csrc/gated_norm_backward.cuh"

using namespace gdn::nbw;
using emu::load;
using emu::save;

int main(int argc, char** argv) {
    if (argc != 2) return 2;
    const std::string dir = argv[1];
    long long T;
    int Hv, layers;
    float eps;
    FILE* m = fopen((dir + "/meta.txt").c_str(), "r");
    if (!m || fscanf(m, "%lld %d %d %f", &T, &Hv, &layers, &eps) != 4) return 2;
    fclose(m);
    const size_t n = (size_t)T * Hv * kD;
    auto o = load<float>(dir + "/o.bin", n);
    auto z = load<uint16_t>(dir + "/z.bin", n);
    auto w = load<float>(dir + "/w.bin", (size_t)layers * kD);
    auto dy = load<float>(dir + "/dy.bin", n);
    std::vector<float> d_o(n, NAN), d_z(n, NAN), dw((size_t)layers * kD, NAN);
    std::vector<float> p1((size_t)n_tiles(T) * n_groups(Hv) * kTok * kD + 1, NAN);
    std::vector<float> p2((size_t)layers * n_chunks(T, layers) * kD + 1, NAN);
    Params p;
    p.o = o.data(); p.z = z.data(); p.w = w.data(); p.dy = dy.data(); p.T = T; p.Hv = Hv; p.layers = layers;
    p.eps = eps; p.d_o = d_o.data(); p.d_z = d_z.data(); p.dw = dw.data(); p.part1 = p1.data(); p.part2 = p2.data();

    emu::Pool rows_pool(kRowThreads);
    if (T > 0) {
        const int ng = n_groups(Hv);
        for (int64_t b = 0; b < n_tiles(T) * ng; ++b)
            rows_pool.run(kRowsFloats, [&](int tid, float* sm) { rows_block(p, b / ng, (int)(b % ng), tid, sm); });
    }
    emu::Pool pool(kThreads);
    if (T == 0) {
        std::fill(dw.begin(), dw.end(), 0.f);
    } else {
        const int64_t nc = n_chunks(T, layers);
        for (int64_t b = 0; b < (int64_t)layers * nc; ++b)
            pool.run(0, [&](int tid, float*) { sum_chunk_block(p, (int)(b / nc), b % nc, tid); });
        for (int l = 0; l < layers; ++l) pool.run(0, [&](int tid, float*) { sum_layer_block(p, l, tid); });
    }
    save(dir + "/d_o.out", d_o.data(), n);
    save(dir + "/d_z.out", d_z.data(), n);
    save(dir + "/d_w.out", dw.data(), dw.size());
    return 0;
}
