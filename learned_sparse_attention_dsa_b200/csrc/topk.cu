// Per-row top-k selection by radix select.
//
// S_t = the k positions with the largest I[t,s] over s <= t ("DeepSeek Sparse
// Attention: Learned Token Selection from Scratch" §3.1), ties to the lower
// position, every candidate when t+1 <= k (§7.6 note).
//
// Scores map to order-preserving 32-bit keys (flip the sign bit of
// non-negative values, every bit of negative ones; -0.0 is folded onto +0.0 so
// that it ties with +0.0 as the float comparison does). Three digit passes
// (11, 11 and 10 bits, most significant first) find the exact key T of the
// k-th largest score and the number r of T-valued positions that still fit.
//
// A row is handled by a cluster of P CTAs (P = 1..16; P > 1 when there are
// fewer rows than SMs, as in decode), each owning a contiguous slice. Digit
// histograms are summed across the cluster through distributed shared memory
// so every CTA derives the same threshold. The row is streamed from global
// memory (L2 after the first read) rather than cached, so several CTAs fit on
// an SM. After the first pass the keys of the threshold bucket -- usually a
// few percent of the row -- are compacted into shared memory with their
// positions, and the later passes and the per-warp counts run on that list
// only (rows with more candidates than the list holds are re-streamed).
// Output: each warp owns a contiguous segment of its CTA's slice; with the
// number of keys > T and = T before the segment (from the list, the warps
// before it and the CTAs before it) every kept position's output slot is
//   #(> T before it) + min(r, #(= T before it)),
// so the positions come out in ascending order without a block-wide scan.
#include <math.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / kWarp;
constexpr int kBins = 2048;
constexpr int kListCap = 6144;  // candidate keys + positions kept in shared memory
constexpr int kMaxCluster = 16;

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive block scan (kThreads threads); scratch holds kWarps + 1 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_inclusive_scan(v);
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wv = lane < kWarps ? scratch[lane] : 0;
        const int wincl = warp_inclusive_scan(wv);
        if (lane < kWarps) scratch[lane] = wincl - wv;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    __syncthreads();
    return r;
}

// Sum the cluster's NBINS-bin histograms and find the digit whose bucket
// holds the remaining-th largest key; all P loads of a bin group are issued
// together. Writes *s_digit and *s_above (keys in higher buckets).
template <int NBINS>
__device__ __forceinline__ void find_digit(const cg::cluster_group &cluster, int *hist, int P, int remaining,
                                           int *scratch, int *s_digit, int *s_above) {
    constexpr int PER = NBINS / kThreads;  // 4 or 2 consecutive bins per thread
    const int first = NBINS - PER * (threadIdx.x + 1);  // thread 0 owns the highest bins
    int c[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) c[j] = 0;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
        if (r < P) {
            const int *h = cluster.map_shared_rank(hist, r) + first;
            if constexpr (PER == 4) {
                const int4 v = *reinterpret_cast<const int4 *>(h);
                c[0] += v.x; c[1] += v.y; c[2] += v.z; c[3] += v.w;
            } else {
                const int2 v = *reinterpret_cast<const int2 *>(h);
                c[0] += v.x; c[1] += v.y;
            }
        }
    }
    int local = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) local += c[j];
    const int excl = block_exclusive_scan(local, scratch);
    if (excl < remaining && excl + local >= remaining) {
        int run = excl;
#pragma unroll
        for (int j = PER - 1; j >= 0; --j) {  // descending digit order
            if (run + c[j] >= remaining) {
                *s_digit = first + j;
                *s_above = run;
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
}

struct Slice {
    const float *src;  // first score of this CTA's slice
    int cnt;           // scores in the slice
    int w_lo, w_hi;    // this warp's segment [w_lo, w_hi) of the slice
};

// Apply fn(pos, key, valid) to the warp's segment, 32 consecutive positions
// per step, four steps' loads in flight.
template <typename F>
__device__ __forceinline__ void sweep(const Slice &sl, F fn) {
    const int lane = threadIdx.x & 31;
    for (int base = sl.w_lo; base < sl.w_hi; base += 4 * kWarp) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = base + u * kWarp + lane;
            v[u] = s < sl.w_hi ? __ldg(sl.src + s) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = base + u * kWarp + lane;
            fn(s, order_key(v[u]), s < sl.w_hi);
        }
    }
}

__global__ void __launch_bounds__(kThreads)
topk_kernel(const float *__restrict__ scores, int Tq, int L, int q_pos0, int k, int32_t *__restrict__ idx) {
    __shared__ __align__(16) int hist[2][kBins];
    extern __shared__ __align__(16) uint8_t dyn_smem[];
    uint32_t *list_key = reinterpret_cast<uint32_t *>(dyn_smem);                // [kListCap]
    int32_t *list_pos = reinterpret_cast<int32_t *>(dyn_smem + 4 * kListCap);   // [kListCap]
    __shared__ int scratch[kWarps + 1];
    __shared__ int w_gt[kWarps], w_eq[kWarps];
    __shared__ int s_digit, s_above, s_nlist;
    __shared__ int s_counts[2];

    cg::cluster_group cluster = cg::this_cluster();
    const int P = (int)cluster.num_blocks();
    const int part = (int)cluster.block_rank();
    const int row = blockIdx.x / P;
    const int t = q_pos0 + row % Tq;
    const int n = t + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t *out = idx + (size_t)row * k;

    if (n <= k) {  // every candidate is kept (same branch for the whole cluster)
        if (part == 0)
            for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < n ? j : -1;
        return;
    }
    const int per = (n + P - 1) / P;
    const int lo = part * per;
    Slice sl;
    sl.src = scores + (size_t)row * L + lo;
    sl.cnt = max(0, min(n, lo + per) - lo);
    const int seg = ((sl.cnt + kWarps - 1) / kWarps + 31) & ~31;
    sl.w_lo = min(sl.cnt, warp * seg);
    sl.w_hi = min(sl.cnt, sl.w_lo + seg);

    // ---- pass 1: bits 31..21 of every key
    for (int b = threadIdx.x; b < kBins; b += kThreads) hist[0][b] = 0;
    if (threadIdx.x == 0) s_nlist = 0;
    __syncthreads();
    sweep(sl, [&](int, uint32_t key, bool ok) {
        if (ok) atomicAdd(&hist[0][key >> 21], 1);
    });
    __syncthreads();
    cluster.sync();
    int remaining = k;
    find_digit<kBins>(cluster, hist[0], P, remaining, scratch, &s_digit, &s_above);
    const uint32_t d1 = (uint32_t)s_digit;
    remaining -= s_above;

    // ---- compact the threshold bucket; count keys in higher buckets per warp
    int gt1 = 0;
    sweep(sl, [&](int s, uint32_t key, bool ok) {
        const bool cand = ok && (key >> 21) == d1;
        gt1 += ok && (key >> 21) > d1;
        const unsigned m = __ballot_sync(0xffffffffu, cand);
        if (m) {
            int slot0 = 0;
            if (lane == 0) slot0 = atomicAdd(&s_nlist, __popc(m));
            slot0 = __shfl_sync(0xffffffffu, slot0, 0);
            const int slot = slot0 + __popc(m & lanemask_lt());
            if (cand && slot < kListCap) {
                list_key[slot] = key;
                list_pos[slot] = s;
            }
        }
    });
    gt1 = warp_sum_int(gt1);
    if (lane == 0) {
        w_gt[warp] = gt1;
        w_eq[warp] = 0;
    }
    for (int b = threadIdx.x; b < kBins; b += kThreads) hist[1][b] = 0;
    __syncthreads();
    const int n_list = s_nlist;
    const bool use_list = n_list <= kListCap;

    // ---- pass 2: bits 20..10 of the keys in bucket d1
    if (use_list) {
        for (int j = threadIdx.x; j < n_list; j += kThreads)
            atomicAdd(&hist[1][(list_key[j] >> 10) & 2047u], 1);
    } else {
        sweep(sl, [&](int, uint32_t key, bool ok) {
            if (ok && (key >> 21) == d1) atomicAdd(&hist[1][(key >> 10) & 2047u], 1);
        });
    }
    __syncthreads();
    cluster.sync();  // also: every CTA is done reading the pass-1 histograms
    find_digit<kBins>(cluster, hist[1], P, remaining, scratch, &s_digit, &s_above);
    const uint32_t p2 = (d1 << 11) | (uint32_t)s_digit;
    remaining -= s_above;

    // ---- pass 3: bits 9..0 of the keys whose top 22 bits are p2
    for (int b = threadIdx.x; b < 1024; b += kThreads) hist[0][b] = 0;
    __syncthreads();
    if (use_list) {
        for (int j = threadIdx.x; j < n_list; j += kThreads) {
            const uint32_t key = list_key[j];
            if ((key >> 10) == p2) atomicAdd(&hist[0][key & 1023u], 1);
        }
    } else {
        sweep(sl, [&](int, uint32_t key, bool ok) {
            if (ok && (key >> 10) == p2) atomicAdd(&hist[0][key & 1023u], 1);
        });
    }
    __syncthreads();
    cluster.sync();
    find_digit<1024>(cluster, hist[0], P, remaining, scratch, &s_digit, &s_above);
    const uint32_t T = (p2 << 10) | (uint32_t)s_digit;
    remaining -= s_above;
    const int r = remaining;  // keys equal to T that still fit, lowest positions first

    // ---- keys > T and = T per warp segment
    if (use_list) {
        for (int j = threadIdx.x; j < n_list; j += kThreads) {
            const uint32_t key = list_key[j];
            const int w = list_pos[j] / seg;
            if (key > T) atomicAdd(&w_gt[w], 1);
            else if (key == T) atomicAdd(&w_eq[w], 1);
        }
    } else {
        int gt = 0, eq = 0;
        sweep(sl, [&](int, uint32_t key, bool ok) {
            gt += ok && key > T;
            eq += ok && key == T;
        });
        gt = warp_sum_int(gt);
        eq = warp_sum_int(eq);
        if (lane == 0) {
            w_gt[warp] = gt;
            w_eq[warp] = eq;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int g = 0, e = 0;
        for (int w = 0; w < kWarps; ++w) {
            const int gw = w_gt[w], ew = w_eq[w];
            w_gt[w] = g;  // becomes the exclusive prefix
            w_eq[w] = e;
            g += gw;
            e += ew;
        }
        s_counts[0] = g;
        s_counts[1] = e;
    }
    __syncthreads();
    cluster.sync();
    int gt_b = 0, eq_b = 0;
    for (int c = 0; c < part; ++c) {
        const int *rc = cluster.map_shared_rank(s_counts, c);
        gt_b += rc[0];
        eq_b += rc[1];
    }
    cluster.sync();  // no CTA leaves while another may still read its shared memory

    // ---- write the kept positions of this warp's segment in order
    gt_b += w_gt[warp];
    eq_b += w_eq[warp];
    const unsigned lt = lanemask_lt();
    sweep(sl, [&](int s, uint32_t key, bool ok) {
        const bool gt = ok && key > T;
        const bool eq = ok && key == T;
        const unsigned gm = __ballot_sync(0xffffffffu, gt);
        const unsigned em = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = eq_b + __popc(em & lt);
        if (gt || (eq && eq_rank < r)) {
            const int pos = gt_b + __popc(gm & lt) + min(r, eq_rank);
            if (pos < k) out[pos] = lo + s;
        }
        gt_b += __popc(gm);
        eq_b += __popc(em);
    });
}

}  // namespace

size_t topk_workspace_bytes(int, int, int, int, int) { return 0; }

// CTAs per row: enough to cover the SMs when rows are few (at most 16).
static int cluster_parts(int rows, int sm_count) {
    int P = 1;
    while (P < kMaxCluster && (long long)rows * P < (long long)sm_count) P *= 2;
    return P;
}

static cudaError_t launch_parts(const TopkProblem &p, int P, cudaStream_t stream) {
    constexpr size_t kDynSmem = 8 * (size_t)kListCap;
    cudaError_t err = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDynSmem);
    if (err != cudaSuccess) return err;
    if (P > 8) {
        err = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return err;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.B * p.Tq) * P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kDynSmem;
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
        err = cudaOccupancyMaxActiveClusters(&clusters, topk_kernel, &cfg);
        if (err != cudaSuccess || clusters == 0) {
            (void)cudaGetLastError();
            return cudaErrorNotSupported;
        }
    }
    err = cudaLaunchKernelEx(&cfg, topk_kernel, p.scores, p.Tq, p.L, p.q_pos0, p.k, p.idx);
    count_launch();
    return err;
}

cudaError_t launch_topk(const TopkProblem &p, cudaStream_t stream) {
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    const long long rows = (long long)p.B * p.Tq;
    if (rows == 0) return cudaSuccess;
    int P = cluster_parts((int)(rows < 0x7fffffffLL ? rows : 0x7fffffffLL), info.sm_count);
    if (rows * P >= 0x7fffffffLL) return cudaErrorInvalidValue;
    err = launch_parts(p, P, stream);
    if (err == cudaErrorNotSupported && P > 8) err = launch_parts(p, 8, stream);
    return err;
}

}  // namespace dsa
