// Per-row top-k selection by radix select in shared memory.
//
// S_t = the k positions with the largest I[t,s] over s <= t ("DeepSeek Sparse
// Attention: Learned Token Selection from Scratch" §3.1), ties to the lower
// position, every candidate when t+1 <= k.
//
// Scores are mapped to order-preserving 32-bit keys (flip the sign bit of
// non-negative values, all bits of negative ones; -0.0 is folded onto +0.0 so
// that it ties with +0.0 as the float comparison does). Four 8-bit digit
// passes, most significant first, find the exact key T of the k-th largest
// score and the number r of T-valued positions that still fit. A final pass
// walks the row in position order and keeps every key > T and the first r
// keys == T, writing the kept positions in ascending order through a
// block-wide prefix count. The row lives in shared memory when it fits;
// longer rows are re-read from global memory (L2) on every pass.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / kWarp;
constexpr int kBins = 256;
constexpr int kPerThread = 4;  // consecutive positions per thread in the final pass

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the block; *total receives the block sum.
// Uses scratch[kWarps + 1]; contains two barriers.
__device__ __forceinline__ int block_exclusive_scan(int v, int *scratch, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_inclusive_scan(v);
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wv = lane < kWarps ? scratch[lane] : 0;
        const int wincl = warp_inclusive_scan(wv);
        if (lane < kWarps) scratch[lane] = wincl - wv;
        if (lane == 31) scratch[kWarps] = wincl;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    *total = scratch[kWarps];
    return r;
}

__global__ void __launch_bounds__(kThreads)
topk_radix_kernel(const float *__restrict__ scores, int Tq, int L, int q_pos0, int k,
                  int32_t *__restrict__ idx, int cache_cap) {
    extern __shared__ uint32_t keys_sm[];
    __shared__ int hist[kBins];
    __shared__ int scan_scratch[kWarps + 1];
    __shared__ int s_digit, s_above;

    const int row = blockIdx.x;
    const int t = q_pos0 + row % Tq;
    const int n = t + 1;
    int32_t *out = idx + (size_t)row * k;
    const float *src = scores + (size_t)row * L;

    if (n <= k) {  // every candidate is kept
        for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < n ? j : -1;
        return;
    }

    const bool cached = n <= cache_cap;
    if (cached) {
        for (int s = threadIdx.x; s < n; s += kThreads) keys_sm[s] = order_key(src[s]);
    }
    __syncthreads();

    uint32_t prefix = 0u, mask = 0u;
    int remaining = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = threadIdx.x; b < kBins; b += kThreads) hist[b] = 0;
        __syncthreads();
        for (int s = threadIdx.x; s < n; s += kThreads) {
            const uint32_t key = cached ? keys_sm[s] : order_key(__ldg(src + s));
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (kBins - 1)], 1);
        }
        if (threadIdx.x == 0) {
            s_digit = 0;
            s_above = 0;
        }
        __syncthreads();
        if (threadIdx.x < kWarp) {
            // lane owns 8 bins in descending digit order: 255-8*lane .. 248-8*lane
            const int lane = threadIdx.x;
            int c[8], local = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = hist[kBins - 1 - (lane * 8 + j)];
                local += c[j];
            }
            const int incl = warp_inclusive_scan(local);
            const int excl = incl - local;
            if (excl < remaining && incl >= remaining) {
                int run = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run + c[j] >= remaining) {
                        s_digit = kBins - 1 - (lane * 8 + j);
                        s_above = run;
                        break;
                    }
                    run += c[j];
                }
            }
        }
        __syncthreads();
        prefix |= (uint32_t)s_digit << shift;
        mask |= (uint32_t)(kBins - 1) << shift;
        remaining -= s_above;
        __syncthreads();
    }

    // prefix is now the exact key T of the k-th largest score; keep all keys
    // above it and the first `remaining` keys equal to it, in position order.
    const uint32_t T = prefix;
    const int r = remaining;
    int base = 0, eq_seen = 0;
    for (int c0 = 0; c0 < n; c0 += kThreads * kPerThread) {
        const int s_first = c0 + threadIdx.x * kPerThread;
        uint32_t key[kPerThread];
        int n_eq = 0;
#pragma unroll
        for (int v = 0; v < kPerThread; ++v) {
            const int s = s_first + v;
            key[v] = 0u;  // below every real key, never selected (T >= 0x007fffff)
            if (s < n) key[v] = cached ? keys_sm[s] : order_key(__ldg(src + s));
            n_eq += (s < n && key[v] == T);
        }
        int eq_total;
        int eq_rank = eq_seen + block_exclusive_scan(n_eq, scan_scratch, &eq_total);
        bool sel[kPerThread];
        int n_sel = 0;
#pragma unroll
        for (int v = 0; v < kPerThread; ++v) {
            const int s = s_first + v;
            sel[v] = false;
            if (s < n) {
                if (key[v] > T) {
                    sel[v] = true;
                } else if (key[v] == T) {
                    sel[v] = eq_rank < r;
                    ++eq_rank;
                }
            }
            n_sel += sel[v];
        }
        __syncthreads();  // scan_scratch is reused
        int sel_total;
        int pos = base + block_exclusive_scan(n_sel, scan_scratch, &sel_total);
#pragma unroll
        for (int v = 0; v < kPerThread; ++v)
            if (sel[v] && pos < k) out[pos++] = s_first + v;
        base += sel_total;
        eq_seen += eq_total;
        __syncthreads();
        if (base >= k) break;
    }
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int, int) { return 0; }

cudaError_t launch_topk(const TopkProblem &p, cudaStream_t stream) {
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    const int rows = p.B * p.Tq;
    if (rows == 0) return cudaSuccess;
    // Cache the row in shared memory when it fits next to the static arrays.
    const int t_max = p.q_pos0 + p.Tq - 1;
    const size_t static_bytes = sizeof(int) * (kBins + kWarps + 1 + 2);
    const size_t budget = (size_t)info.max_smem_optin - static_bytes - 1024;
    int cache_cap = (int)(budget / sizeof(uint32_t));
    size_t smem = 0;
    if (t_max + 1 <= cache_cap) {
        cache_cap = t_max + 1;
        smem = sizeof(uint32_t) * (size_t)cache_cap;
    } else {
        cache_cap = 0;
    }
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(topk_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem);
        if (err != cudaSuccess) return err;
    }
    topk_radix_kernel<<<rows, kThreads, smem, stream>>>(p.scores, p.Tq, p.L, p.q_pos0, p.k, p.idx,
                                                        cache_cap);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsa
