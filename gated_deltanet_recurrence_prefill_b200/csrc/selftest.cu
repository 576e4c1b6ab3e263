// selftest.cu -- exercises the bounded waits that every producer / consumer
// wait of the prefill is built on, on purpose with nothing to wait for: a
// counter in global memory that no thread raises (gflag_wait_ge, as on the
// ring's ready / freed counters) or an mbarrier phase that never completes
// (mbar_wait, as on the tensor-core and copy barriers).  The wait gives up after
// the given time, the kernel records the error in the workspace's error word
// exactly as the prefill does, and returns; gdn_prefill_status then reports
// GDN_ERR_TIMEOUT.  Nothing faults, traps or hangs, and the context stays
// usable.
#include <cuda_runtime.h>

#include "kernels.h"
#include "tc_util.cuh"

namespace gdn {
namespace {

using namespace tc;

__global__ void selftest_wait_kernel(int which, uint64_t limit_ns, uint32_t* ws_words) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    uint32_t* err = ws_words + kWsErrorWordOffset / sizeof(uint32_t);
    // a counter nobody raises: the first word after the error word, zero on entry
    uint32_t* never = ws_words + 1;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        *never = 0u;
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bool ok;
        if (which == 0)
            ok = gflag_wait_ge(never, 1u, &abort_flag, err, limit_ns);
        else
            ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);     // no thread arrives
        if (!ok) atomicOr(err, 1u);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_selftest_wait(int which, uint64_t limit_ns, void* workspace, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(which, limit_ns, static_cast<uint32_t*>(workspace));
    return cudaGetLastError();
}

}  // namespace gdn
