// pa_decode_static: pa_decode for callers that cannot allocate device memory.
//
// pa_decode needs a workspace for the split-context partials, which the
// caller allocates.  Some callers cannot: code running inside a host runtime
// that owns all device allocations, plug-ins that may not call cudaMalloc
// (its implicit synchronisation would stall other streams), or code paths
// where an allocation failure is not acceptable mid-step.  This entry point
// keeps the partials in a fixed array that lives in the library's own device
// image instead, so it allocates nothing at call time.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits.  Host code
// only ever sees a host-side stand-in for its name, so the device address is
// looked up with cudaGetSymbolAddress, once per device, with that device
// current, on the first call made on that device.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/pagedattn.h"
#include "status.h"

namespace pa {
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB

// Split partials of pa_decode_static (every call shares it).
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_static_scratch on the current device, looked up on the
// first call per device; nullptr (with the error in pa_last_error) on failure.
void *static_scratch_ptr() {
    static std::atomic<void *> ptrs[kMaxDevices];
    static std::mutex mu;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        fail(PA_ERR_CUDA, "pa_decode_static: no current CUDA device");
        return nullptr;
    }
    void *p = ptrs[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> lock(mu);
    p = ptrs[dev].load(std::memory_order_relaxed);
    if (p) return p;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
        fail(PA_ERR_CUDA, "pa_decode_static: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
        return nullptr;
    }
    ptrs[dev].store(p, std::memory_order_release);
    return p;
}

}  // namespace
}  // namespace pa

extern "C" {

int pa_decode_static(float *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                     int num_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                     int dtype, void *stream) {
    pa::clear_error();
    const size_t need =
        pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_seq_len, 0);
    if (need > pa::kStaticScratchBytes)
        return pa::fail(PA_ERR_INVALID_ARG,
                        "pa_decode_static: %d sequences x %d heads up to %d tokens need %zu "
                        "bytes of split scratch, more than the %zu-byte static array; use "
                        "pa_decode with a caller workspace",
                        num_seqs, num_heads, max_seq_len, need, pa::kStaticScratchBytes);
    void *ws = nullptr;
    if (need > 0) {
        ws = pa::static_scratch_ptr();
        if (!ws) return PA_ERR_CUDA;
    }
    // the partials are written by the main kernel before the reduce reads
    // them, so nothing has to start at zero
    return pa_decode_ex(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads,
                        num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                        max_seq_len, scale, dtype, ws, need > 0 ? pa::kStaticScratchBytes : 0,
                        0, 0, stream);
}

}  // extern "C"
