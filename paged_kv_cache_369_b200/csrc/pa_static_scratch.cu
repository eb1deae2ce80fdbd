// Split-KV decode for callers that cannot allocate device memory.
//
// pa_decode_split_reduce needs a workspace for the per-partition partials, and
// its caller normally allocates that once with cudaMalloc (or a framework
// allocator).  Some callers have no way to do so: a plugin or custom-op host
// that hands an operator its tensors but no allocator, a serving engine that
// has already reserved all free HBM for its KV block pool (so any further
// cudaMalloc fails), or a latency-critical loop that must not hit cudaMalloc's
// implicit device synchronisation.  This file gives them one entry point whose
// scratch space is built into the library: a file-scope __device__ array of
// PA_STATIC_SCRATCH_BYTES bytes.  Nothing here calls cudaMalloc, cudaFree or
// any allocating routine.
//
// The array's host-side name is only a stand-in for the device copy, so the
// device address is looked up with cudaGetSymbolAddress, once per device, with
// that device current, on the first call made on it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pa.h"

namespace {

__device__ __align__(256) unsigned char g_split_scratch[PA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_lock;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_split_scratch on the current device (nullptr on error).
void *scratch_on_current_device(int *device_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    *device_out = dev;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_split_scratch) != cudaSuccess || !ptr) {
            (void)cudaGetLastError();
            return nullptr;
        }
        g_scratch_addr[dev] = ptr;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" pa_status pa_decode_split_reduce_static_scratch(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float softmax_scale, pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
    int partition_size, int max_seq_len, int *dev_err, void *stream) {
    const size_t need =
        pa_split_workspace_bytes(num_seqs, num_q_heads, head_dim, max_seq_len, partition_size);
    if (need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_INVALID_ARG;  // does not fit
    int dev = -1;
    void *scratch = scratch_on_current_device(&dev);
    if (!scratch) return PA_ERR_CUDA;
    return pa_decode_split_reduce(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                  seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                                  block_size, num_blocks, softmax_scale, q_dtype, kv_dtype, k_scale,
                                  v_scale, partition_size, max_seq_len, scratch,
                                  (size_t)PA_STATIC_SCRATCH_BYTES, dev_err, stream);
}
