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
// device address is looked up with cudaGetSymbolAddress, with the device
// current, on the first call made in a CUDA context.  The address is kept per
// device together with the context's unique id (cuCtxGetId): a call made in
// another context of the device -- a new primary context after
// cudaDeviceReset, or a context the caller created -- looks it up again
// instead of using an address from a context that no longer holds it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pa.h"
#include "pa_internal.h"

namespace {

__device__ __align__(256) unsigned char g_split_scratch[PA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;

struct ScratchAddr {
    unsigned long long ctx_id;  // id of the context the address belongs to
    void *ptr;                  // nullptr: not looked up yet
};

std::mutex g_lock;
ScratchAddr g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <typename Fn> Fn driver_fn(const char *name) {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<Fn>(f);
    return nullptr;
}

// Unique id of the calling thread's current context; false when there is none
// (the runtime has not made one current on this thread yet) or on error.
bool current_ctx_id(unsigned long long *id) {
    static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_split_scratch in the current context (nullptr on error).
void *scratch_in_current_context() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    std::lock_guard<std::mutex> guard(g_lock);
    ScratchAddr &e = g_scratch[dev];
    if (have_id && e.ptr && e.ctx_id == id) return e.ptr;
    // first call in this context: the lookup also makes the device's primary
    // context current when the runtime had not done so on this thread yet
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_split_scratch) != cudaSuccess || !ptr) {
        (void)cudaGetLastError();
        return nullptr;
    }
    if (current_ctx_id(&id)) {
        e.ctx_id = id;
        e.ptr = ptr;
    }
    return ptr;
}

}  // namespace

extern "C" pa_status pa_decode_split_reduce_static_scratch(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float softmax_scale, pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
    int partition_size, int max_seq_len, int *dev_err, void *stream) {
    // argument errors never depend on the device: check them first
    const int st = pa::check_split_reduce_args(
        out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
        num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, softmax_scale, q_dtype,
        kv_dtype, k_scale, v_scale, partition_size, max_seq_len);
    if (st != PA_OK || num_seqs == 0) return static_cast<pa_status>(st);
    const size_t need =
        pa_split_workspace_bytes(num_seqs, num_q_heads, head_dim, max_seq_len, partition_size);
    if (need == 0 || need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_INVALID_ARG;
    void *scratch = scratch_in_current_context();
    if (!scratch) return PA_ERR_CUDA;
    return pa_decode_split_reduce(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                  seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                                  block_size, num_blocks, softmax_scale, q_dtype, kv_dtype, k_scale,
                                  v_scale, partition_size, max_seq_len, scratch,
                                  (size_t)PA_STATIC_SCRATCH_BYTES, dev_err, stream);
}
