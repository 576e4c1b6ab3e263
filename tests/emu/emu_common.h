// Shared pieces of the CPU emulation of the kernels' block functions: a pool of
// host threads, one per CUDA thread of a block, meeting at a std::barrier for
// every block barrier, and raw file input / output for the test drivers.
//
// A source using this header defines BWC_SYNC() as ::emu::g_bar->arrive_and_wait()
// (and BWC_SHFL_XOR(v, m) as ::emu::shfl_xor(v, m)) before including the kernel
// header.  Warps must be whole (a multiple of 32 threads) where shuffles are used.
#pragma once

#include <barrier>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <functional>
#include <memory>
#include <string>
#include <thread>
#include <vector>

namespace emu {

inline std::barrier<>* g_bar = nullptr;

// warp shuffles: every lane of a warp writes its value, the warp meets, each
// lane reads its partner's, the warp meets again (so the slots can be reused)
inline thread_local int t_tid = 0;
inline std::vector<std::barrier<>*> g_warp_bars;
inline float g_shfl[32][32];

inline float shfl_xor(float v, int m) {
    const int w = t_tid >> 5, l = t_tid & 31;
    g_shfl[w][l] = v;
    g_warp_bars[w]->arrive_and_wait();
    const float r = g_shfl[w][l ^ m];
    g_warp_bars[w]->arrive_and_wait();
    return r;
}

// nthreads workers kept for the whole run; each block is handed to all of them
// between two barriers shared with the calling thread.  Shared memory starts as
// NaN (the GPU does not clear it either).
class Pool {
  public:
    explicit Pool(int nthreads) : start_(nthreads + 1), end_(nthreads + 1), sync_(nthreads) {
        g_bar = &sync_;
        for (int w = 0; w < (nthreads + 31) / 32; ++w) warp_bars_.emplace_back(new std::barrier<>(32));
        g_warp_bars.clear();
        for (auto& b : warp_bars_) g_warp_bars.push_back(b.get());
        for (int t = 0; t < nthreads; ++t)
            th_.emplace_back([this, t] {
                t_tid = t;
                for (;;) {
                    start_.arrive_and_wait();
                    if (stop_) return;
                    job_(t, sm_);
                    end_.arrive_and_wait();
                }
            });
    }
    ~Pool() {
        stop_ = true;
        start_.arrive_and_wait();
        for (auto& x : th_) x.join();
    }
    template <class F>
    void run(size_t smem_floats, F f) {
        std::vector<float> sm(smem_floats ? smem_floats : 1, NAN);
        sm_ = sm.data();
        job_ = f;
        start_.arrive_and_wait();
        end_.arrive_and_wait();
    }

  private:
    std::barrier<> start_, end_, sync_;
    std::vector<std::unique_ptr<std::barrier<>>> warp_bars_;
    std::vector<std::thread> th_;
    std::function<void(int, float*)> job_;
    float* sm_ = nullptr;
    bool stop_ = false;
};

template <class T>
std::vector<T> load(const std::string& path, size_t n) {
    std::vector<T> v(n);
    FILE* f = fopen(path.c_str(), "rb");
    if (!f || fread(v.data(), sizeof(T), n, f) != n) {
        fprintf(stderr, "cannot read %s\n", path.c_str());
        exit(2);
    }
    fclose(f);
    return v;
}

inline void save(const std::string& path, const float* x, size_t n) {
    FILE* f = fopen(path.c_str(), "wb");
    if (!f || fwrite(x, sizeof(float), n, f) != n) {
        fprintf(stderr, "cannot write %s\n", path.c_str());
        exit(2);
    }
    fclose(f);
}

}  // namespace emu
