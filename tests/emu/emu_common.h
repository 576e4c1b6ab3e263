// Shared pieces of the CPU emulation of the kernels' block functions: a pool of
// host threads, one per CUDA thread of a block, meeting at a std::barrier for
// every block barrier, and raw file input / output for the test drivers.
//
// A source using this header defines BWC_SYNC() as ::emu::g_bar->arrive_and_wait()
// before including the kernel header.
#pragma once

#include <barrier>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <functional>
#include <string>
#include <thread>
#include <vector>

namespace emu {

inline std::barrier<>* g_bar = nullptr;

// nthreads workers kept for the whole run; each block is handed to all of them
// between two barriers shared with the calling thread.  Shared memory starts as
// NaN (the GPU does not clear it either).
class Pool {
  public:
    explicit Pool(int nthreads) : start_(nthreads + 1), end_(nthreads + 1), sync_(nthreads) {
        g_bar = &sync_;
        for (int t = 0; t < nthreads; ++t)
            th_.emplace_back([this, t] {
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
