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

#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

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

// ---------------------------------------------------------------------------
// Cluster variant: one row is shared by a cluster of P CTAs (P = 1..16). Each
// CTA keeps its slice of the row in shared memory; the digit histograms are
// summed across the cluster through distributed shared memory, so every CTA
// derives the same threshold. Digits of 11, 11 and 10 bits (three passes, the
// first fused with the load). Histogram updates are aggregated per warp
// (__match_any_sync) because integer-valued scores pile into few bins. The
// final pass gives each CTA its output offset from the counts of the CTAs
// before it, so the positions still come out in ascending order.

constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / kWarp;
constexpr int kMaxBins = 2048;

__device__ __forceinline__ void hist_add(int *hist, uint32_t bin, bool valid) {
    const uint32_t tag = valid ? bin : 0xffffffffu;
    const unsigned peers = __match_any_sync(0xffffffffu, tag);
    if (valid && (int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

// Block-wide exclusive scan for kCThreads threads (scratch: kCWarps + 1 ints).
__device__ __forceinline__ int cblock_exclusive_scan(int v, int *scratch, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_inclusive_scan(v);
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wv = lane < kCWarps ? scratch[lane] : 0;
        const int wincl = warp_inclusive_scan(wv);
        if (lane < kCWarps) scratch[lane] = wincl - wv;
        if (lane == 31) scratch[kCWarps] = wincl;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    *total = scratch[kCWarps];
    __syncthreads();  // scratch may be reused right away
    return r;
}

// Sum the cluster's histograms (bins [0, nbins)) and find the digit whose
// bucket holds the remaining-th largest key. Writes s_digit / s_above.
__device__ __forceinline__ void cluster_find_digit(cg::cluster_group &cluster, int *hist, int nbins, int P,
                                                   int remaining, int *scratch, int *s_digit, int *s_above) {
    const int per = nbins / kCThreads;  // 4 or 2 bins per thread, descending digit order
    int c[4] = {0, 0, 0, 0};
    int local = 0;
    for (int j = 0; j < per; ++j) {
        const int bin = nbins - 1 - (threadIdx.x * per + j);
        int sum = 0;
        for (int r = 0; r < P; ++r) sum += cluster.map_shared_rank(hist, r)[bin];
        c[j] = sum;
        local += sum;
    }
    int total;
    const int excl = cblock_exclusive_scan(local, scratch, &total);
    if (excl < remaining && excl + local >= remaining) {
        int run = excl;
        for (int j = 0; j < per; ++j) {
            if (run + c[j] >= remaining) {
                *s_digit = nbins - 1 - (threadIdx.x * per + j);
                *s_above = run;
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kCThreads)
topk_cluster_kernel(const float *__restrict__ scores, int Tq, int L, int q_pos0, int k, int32_t *__restrict__ idx) {
    extern __shared__ uint32_t keys_sm[];
    __shared__ int hist[2][kMaxBins];
    __shared__ int scratch[kCWarps + 1];
    __shared__ int s_digit, s_above;
    __shared__ int s_counts[2];

    cg::cluster_group cluster = cg::this_cluster();
    const int P = (int)cluster.num_blocks();
    const int part = (int)cluster.block_rank();
    const int row = blockIdx.x / P;
    const int t = q_pos0 + row % Tq;
    const int n = t + 1;
    int32_t *out = idx + (size_t)row * k;
    const float *src = scores + (size_t)row * L;

    if (n <= k) {  // every candidate is kept (same branch for the whole cluster)
        if (part == 0)
            for (int j = threadIdx.x; j < k; j += kCThreads) out[j] = j < n ? j : -1;
        return;
    }
    const int per = ((n + P - 1) / P + 3) & ~3;
    const int lo = part * per;
    const int cnt = max(0, min(n, lo + per) - lo);

    // pass 1 (bits 31..21) fused with the load
    for (int b = threadIdx.x; b < kMaxBins; b += kCThreads) hist[0][b] = 0;
    __syncthreads();
    for (int base = 0; base < cnt; base += kCThreads) {
        const int s = base + threadIdx.x;
        const bool valid = s < cnt;
        uint32_t key = 0;
        if (valid) {
            key = order_key(src[lo + s]);
            keys_sm[s] = key;
        }
        hist_add(hist[0], key >> 21, valid);
    }
    __syncthreads();
    cluster.sync();
    int remaining = k;
    cluster_find_digit(cluster, hist[0], 2048, P, remaining, scratch, &s_digit, &s_above);
    const uint32_t d1 = (uint32_t)s_digit;
    remaining -= s_above;

    // pass 2 (bits 20..10) among keys whose top 11 bits equal d1
    for (int b = threadIdx.x; b < kMaxBins; b += kCThreads) hist[1][b] = 0;
    __syncthreads();
    for (int base = 0; base < cnt; base += kCThreads) {
        const int s = base + threadIdx.x;
        const uint32_t key = s < cnt ? keys_sm[s] : 0u;
        hist_add(hist[1], (key >> 10) & 2047u, s < cnt && (key >> 21) == d1);
    }
    __syncthreads();
    cluster.sync();  // also: every CTA has finished reading the pass-1 histograms
    cluster_find_digit(cluster, hist[1], 2048, P, remaining, scratch, &s_digit, &s_above);
    const uint32_t p2 = (d1 << 11) | (uint32_t)s_digit;
    remaining -= s_above;

    // pass 3 (bits 9..0) among keys whose top 22 bits equal p2
    for (int b = threadIdx.x; b < 1024; b += kCThreads) hist[0][b] = 0;
    __syncthreads();
    for (int base = 0; base < cnt; base += kCThreads) {
        const int s = base + threadIdx.x;
        const uint32_t key = s < cnt ? keys_sm[s] : 0u;
        hist_add(hist[0], key & 1023u, s < cnt && (key >> 10) == p2);
    }
    __syncthreads();
    cluster.sync();
    cluster_find_digit(cluster, hist[0], 1024, P, remaining, scratch, &s_digit, &s_above);
    const uint32_t T = (p2 << 10) | (uint32_t)s_digit;
    remaining -= s_above;
    const int r = remaining;  // keys equal to T that still fit, lowest positions first

    // counts of this slice, published for the CTAs after it
    int gt = 0, eq = 0;
    for (int s = threadIdx.x; s < cnt; s += kCThreads) {
        gt += keys_sm[s] > T;
        eq += keys_sm[s] == T;
    }
    int gt_total, eq_total;
    cblock_exclusive_scan(gt, scratch, &gt_total);
    cblock_exclusive_scan(eq, scratch, &eq_total);
    if (threadIdx.x == 0) {
        s_counts[0] = gt_total;
        s_counts[1] = eq_total;
    }
    cluster.sync();
    int gt_before = 0, eq_before = 0;
    for (int c = 0; c < part; ++c) {
        const int *rc = cluster.map_shared_rank(s_counts, c);
        gt_before += rc[0];
        eq_before += rc[1];
    }
    cluster.sync();  // no CTA leaves while another may still read its shared memory

    int base_out = gt_before + min(r, eq_before);
    int eq_seen = eq_before;
    for (int c0 = 0; c0 < cnt; c0 += kCThreads * kPerThread) {
        const int s_first = c0 + threadIdx.x * kPerThread;
        uint32_t key[kPerThread];
        int n_eq = 0;
#pragma unroll
        for (int v = 0; v < kPerThread; ++v) {
            const int s = s_first + v;
            key[v] = s < cnt ? keys_sm[s] : 0u;
            n_eq += (s < cnt && key[v] == T);
        }
        int eq_chunk;
        int eq_rank = eq_seen + cblock_exclusive_scan(n_eq, scratch, &eq_chunk);
        bool sel[kPerThread];
        int n_sel = 0;
#pragma unroll
        for (int v = 0; v < kPerThread; ++v) {
            const int s = s_first + v;
            sel[v] = false;
            if (s < cnt) {
                if (key[v] > T) {
                    sel[v] = true;
                } else if (key[v] == T) {
                    sel[v] = eq_rank < r;
                    ++eq_rank;
                }
            }
            n_sel += sel[v];
        }
        int sel_chunk;
        int pos = base_out + cblock_exclusive_scan(n_sel, scratch, &sel_chunk);
#pragma unroll
        for (int v = 0; v < kPerThread; ++v)
            if (sel[v] && pos < k) out[pos++] = lo + s_first + v;
        base_out += sel_chunk;
        eq_seen += eq_chunk;
    }
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int, int) { return 0; }

// Cluster size for a problem: enough CTAs to cover the GPU about twice, and
// slices that fit in shared memory. 0 when the cluster kernel does not apply.
static int cluster_parts(int rows, int n_max, const DeviceInfo &info, size_t *smem_out) {
    const size_t static_bytes = sizeof(int) * (2 * kMaxBins + kCWarps + 1 + 4) + 1024;
    const size_t cap = ((size_t)info.max_smem_optin - static_bytes) / sizeof(uint32_t);
    int P = 1;
    while (P < 16 && (long long)rows * P < (long long)info.sm_count) P *= 2;
    while (P < 16 && (size_t)(((n_max + P - 1) / P + 3) & ~3) > cap) P *= 2;
    const size_t per = (size_t)(((n_max + P - 1) / P + 3) & ~3);
    if (per > cap) return 0;
    *smem_out = per * sizeof(uint32_t);
    return P;
}

static cudaError_t launch_cluster(const TopkProblem &p, const DeviceInfo &info, int P, size_t smem,
                                  cudaStream_t stream) {
    cudaError_t err = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    if (P > 8) {
        err = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return err;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.B * p.Tq) * P);
    cfg.blockDim = dim3(kCThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (P > 8) {  // a non-portable cluster size: make sure one can be scheduled
        int clusters = 0;
        err = cudaOccupancyMaxActiveClusters(&clusters, topk_cluster_kernel, &cfg);
        if (err != cudaSuccess || clusters == 0) {
            (void)cudaGetLastError();
            return cudaErrorNotSupported;
        }
    }
    err = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, p.scores, p.Tq, p.L, p.q_pos0, p.k, p.idx);
    count_launch();
    return err;
}

cudaError_t launch_topk(const TopkProblem &p, cudaStream_t stream) {
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    const int rows = p.B * p.Tq;
    if (rows == 0) return cudaSuccess;
    {
        size_t smem = 0;
        const int P = cluster_parts(rows, p.q_pos0 + p.Tq, info, &smem);
        if (P > 0 && (long long)rows * P < 0x7fffffffLL) {
            err = launch_cluster(p, info, P, smem, stream);
            if (err != cudaErrorNotSupported) return err;
            if (P > 8) {  // retry with a portable cluster of 8
                const int n_max = p.q_pos0 + p.Tq;
                const size_t per = (size_t)(((n_max + 7) / 8 + 3) & ~3);
                const size_t cap = ((size_t)info.max_smem_optin - sizeof(int) * (2 * kMaxBins + kCWarps + 5) -
                                    1024) / sizeof(uint32_t);
                if (per <= cap) return launch_cluster(p, info, 8, per * sizeof(uint32_t), stream);
            }
        }
    }
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
