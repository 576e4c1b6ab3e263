// prefill_noalloc.cu -- gdn_prefill for callers that cannot allocate device
// memory.
//
// gdn_prefill needs a small device workspace (an error word and per-sequence
// bookkeeping).  Some callers have no way to provide one: code running inside a
// host framework that owns every byte of device memory through its own arena
// and hands out only the tensors of the model, plugins that are given input and
// output pointers but no allocator, and latency-critical loops where a
// cudaMalloc (which may synchronise the device) is not acceptable.  For them,
// gdn_prefill_noalloc runs the same kernel with the workspace placed in a
// fixed-size array that lives in the library's own device image.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  Host code
// cannot pass its name to a kernel (on the host the name is only a stand-in for
// the symbol), so the first call on each device looks up its device address
// with cudaGetSymbolAddress while that device is current, and caches it.  The
// cache is per device number and lives as long as the process: a
// cudaDeviceReset destroys the module and with it the array, so a process that
// resets a device must not call gdn_prefill_noalloc on it again.
//
// The array holds 64 KiB, less than one producer / consumer ring (397,440
// bytes), so this entry point always runs the single-CTA prefill kernel
// (about 2.5x slower than gdn_prefill with a full workspace at T = 8192), and
// GDN_PREFILL_KERNEL=pc makes it return GDN_ERR_UNSUPPORTED.
#include <atomic>

#include <cuda_runtime.h>

#include "../../include/gdn.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64 * 1024;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_prefill_scratch[kNoAllocScratchBytes];

std::atomic<void*> g_scratch_addr[kMaxDevices];

}  // namespace

namespace gdn {

void* noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    void* scratch = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!scratch) {
        // one-time set-up on this device (with the device current)
        if (cudaGetSymbolAddress(&scratch, g_prefill_scratch) != cudaSuccess || !scratch) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev].store(scratch, std::memory_order_release);
    }
    return scratch;
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

}  // namespace gdn

extern "C" {

gdn_status gdn_prefill_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const float* a, const float* b, const float* A_log,
                               const float* dt_bias, const int32_t* cu_seqlens, int32_t n_seq,
                               int64_t T, int32_t Hqk, int32_t Hv, int32_t d, float scale,
                               const float* initial_state, float* final_state, float* o,
                               gdn_stream_t stream) {
    // sizes first: nothing touches the GPU when the scratch array is too small
    (void)T; (void)Hqk; (void)d;
    if (gdn::prefill_min_workspace_bytes(n_seq, Hv) > kNoAllocScratchBytes) return GDN_ERR_WORKSPACE;
    void* scratch = gdn::noalloc_scratch();
    if (!scratch) return GDN_ERR_CUDA;
    // gdn_prefill clears the error word at the start of the scratch on `stream`
    // before its kernel runs; everything else in the scratch is written before
    // it is read within one call.
    return gdn_prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens, n_seq, T, Hqk, Hv, d, scale,
                       initial_state, final_state, o, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
