// dsa_sparse_attn_noalloc: the attention stage with its scratch space built
// into the library instead of passed in by the caller.
//
// Some callers cannot hand this library a workspace: for example an
// inference engine's plugin hook that is given a stream but no allocator, or
// a latency-critical serving loop that must never call cudaMalloc (it can
// synchronise the whole device). For them the split-k partial results of the
// tensor-core attention kernel live in one fixed device array declared in
// this file. The array is part of the loaded module: every GPU that loads
// libdsa.so holds kScratchBytes for it until the process exits.
//
// The entry point itself allocates nothing. Its first call on a device looks
// up the array's device address with cudaGetSymbolAddress (with that device
// current) and caches it; make that first call before any stream capture.
// Every call on a device uses the same array and leaves its last contents
// there; the kernels overwrite every partial they later read, so nothing has
// to be cleared between calls. Two calls whose kernels overlap on the GPU
// (for example on two streams without ordering between them) race on the
// array and give wrong results: order them on one stream, or use
// dsa_sparse_attn with separate workspaces.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr size_t kScratchBytes = 4u << 20;  // 4 MiB per device

__device__ __align__(256) unsigned char g_attn_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_attn_scratch on the current device (set-up on first use).
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *ptr = nullptr;
        err = cudaGetSymbolAddress(&ptr, g_attn_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace dsa

extern "C" {

size_t dsa_sparse_attn_noalloc_max_scratch_bytes(void) { return dsa::kScratchBytes; }

dsa_status dsa_sparse_attn_noalloc(const void *q, const void *k_cache, const void *v_cache, const int32_t *idx,
                                   const dsa_attn_shape *sh, dsa_dtype dt, void *out, float *lse,
                                   dsa_stream_t stream) {
    // The argument checks of dsa_sparse_attn come first, so that a malformed
    // or unsupported shape gets its own status, never DSA_ERR_WORKSPACE.
    const dsa_status st = dsa::validate_attn_call(q, k_cache, v_cache, idx, sh, dt, out, lse);
    if (st != DSA_OK) return st;
    const size_t need = dsa_sparse_attn_workspace_bytes(sh, dt);
    if (need > dsa::kScratchBytes) return DSA_ERR_WORKSPACE;  // needs more than the built-in scratch
    void *scratch = nullptr;
    if (dsa::scratch_address(&scratch) != cudaSuccess) return DSA_ERR_CUDA;
    return dsa_sparse_attn(q, k_cache, v_cache, idx, sh, dt, out, lse, scratch, dsa::kScratchBytes, stream);
}

}  // extern "C"
