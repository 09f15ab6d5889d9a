// A measurement aid with no counterpart on the pages: the gather of selected
// rows alone, with the 16-byte cp.async pattern of the attention kernels and
// no arithmetic. Timed on the rows a prefill attention selects, it gives the
// rate at which those rows can be moved into shared memory at all (served
// mostly by L2 there), the ceiling that the attention's gather-bound time is
// compared with.
//
// Each CTA (256 threads) walks a contiguous share of the index list in tiles
// of 8, 16 or 32 rows (smaller tiles: more CTAs per SM) through a three-stage
// ring; thread i always moves the 16-byte
// chunk column i % C of rows i / C, i / C + 256 / C, ... (C = row_bytes / 16),
// like the attention kernels' copies. Negative or out-of-range indices are
// skipped (zero-filled, no memory traffic). One word of every landed tile is
// folded into a checksum so that the copies have a consumer.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 256;
constexpr int kStages = 3;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(kThreads)
diag_gather_kernel(const uint8_t *__restrict__ src, int64_t pitch, int row_bytes, int n_src, const int32_t *__restrict__ idx,
                   int64_t n, int64_t per_cta, int tile_rows, unsigned int *sink) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int64_t r0 = (int64_t)blockIdx.x * per_cta;
    const int64_t r1 = min(n, r0 + per_cta);
    if (r0 >= r1) return;
    const int chunks = row_bytes / 16;
    const int rows_per_pass = kThreads / chunks;
    const int ch = threadIdx.x % chunks, rr = threadIdx.x / chunks;
    const int tile_bytes = tile_rows * row_bytes;
    const int n_tiles = (int)((r1 - r0 + tile_rows - 1) / tile_rows);
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    auto issue = [&](int tile, int stage) {
        if (rr >= rows_per_pass) return;
        for (int r = rr; r < tile_rows; r += rows_per_pass) {
            const int64_t j = r0 + (int64_t)tile * tile_rows + r;
            int s = j < r1 ? idx[j] : -1;
            const bool valid = s >= 0 && s < n_src;
            if (!valid) s = 0;
            cp_async16(base + stage * tile_bytes + r * row_bytes + ch * 16, src + (int64_t)s * pitch + ch * 16, valid);
        }
    };
    unsigned int acc = 0;
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (st < n_tiles) issue(st, st);
        cp_async_commit();
    }
    for (int t = 0; t < n_tiles; ++t) {
        const int next = t + kStages - 1;
        if (next < n_tiles) issue(next, next % kStages);
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncthreads();
        acc ^= reinterpret_cast<const unsigned int *>(smem + (t % kStages) * tile_bytes)[threadIdx.x % (tile_bytes / 4)];
        __syncthreads();
    }
    cp_async_wait<0>();
    if (acc == 0x9e3779b9u) atomicXor(sink, acc);  // practically never taken; keeps the loads live
}

}  // namespace

cudaError_t launch_diag_gather(const void *src, int64_t pitch, int row_bytes, int n_src, const int32_t *idx, int64_t n,
                               int tile_rows, unsigned int *sink, cudaStream_t stream) {
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    const size_t smem = (size_t)kStages * tile_rows * row_bytes;
    err = cudaFuncSetAttribute(diag_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, diag_gather_kernel, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    const int64_t ctas_max = (int64_t)info.sm_count * per_sm;
    const int64_t tiles = (n + tile_rows - 1) / tile_rows;
    const int64_t ctas = tiles < ctas_max ? tiles : ctas_max;
    const int64_t per_cta = ((tiles + ctas - 1) / ctas) * tile_rows;
    diag_gather_kernel<<<(unsigned)ctas, kThreads, smem, stream>>>(static_cast<const uint8_t *>(src), pitch, row_bytes, n_src,
                                                                   idx, n, per_cta, tile_rows, sink);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsa
