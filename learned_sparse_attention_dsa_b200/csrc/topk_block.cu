// Per-row top-k with one CTA per row and the whole row in registers.
//
//   S_t = positions of the k largest I[t,s], s <= t, ties to the lower s
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §3.1),
// all of 0..t when t+1 <= k.
//
// For rows of at most 1024 * KPT scores. Warp w owns positions
// [w * 32 KPT, (w + 1) * 32 KPT), lane l holds positions w * 32 KPT + 32 j + l
// (coalesced loads), as order-preserving uint32 keys in registers. A radix
// select over the keys finds the k-th largest key T in three passes (bits
// 31-21, 20-10, 9-0) over those registers: each pass builds a shared-memory
// histogram of the keys that match the digits found so far, and a block-wide
// suffix scan of the histogram finds the digit where the count from the top
// reaches the number still wanted. The scores are read from memory once. The
// output slot of a kept position is the number of keys > T before it plus
// min(r, the number of keys == T before it), where r is how many keys equal
// to T are taken: per-warp ballots and one block scan give those counts, so
// the positions come out in ascending order.
#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kBlockThreads = 1024;
constexpr int kBlockWarps = kBlockThreads / 32;
constexpr int kBins = 2048;

__device__ __forceinline__ uint32_t block_order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 ties with +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned lanemask_lt_block() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Over hist[0..kBins) (cleared again on return): the digit d such that the
// keys in bins above d number fewer than `want` and those in bins d and above
// at least `want`. Returns d; *above = count in bins above d.
__device__ __forceinline__ int find_digit(int *hist, int want, int *warp_sum, int *s_digit, int *s_above) {
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // thread tid covers bins b1 = kBins-1-2 tid and b0 = b1-1 (descending)
    const int b1 = kBins - 1 - 2 * tid, b0 = b1 - 1;
    const int c1 = hist[b1], c0 = hist[b0];
    const int mine = c1 + c0;
    const int incl = warp_inclusive_scan(mine);
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = warp_sum[lane];
        const int wincl = warp_inclusive_scan(v);
        warp_sum[lane] = wincl - v;  // exclusive prefix of the warps
    }
    __syncthreads();
    const int before = warp_sum[warp] + incl - mine;  // keys in bins above b1
    if (before < want && before + mine >= want) {
        if (before + c1 >= want) {
            *s_digit = b1;
            *s_above = before;
        } else {
            *s_digit = b0;
            *s_above = before + c1;
        }
    }
    hist[b1] = 0;
    hist[b0] = 0;
    __syncthreads();
    return *s_digit;
}

template <int KPT>
__global__ void __launch_bounds__(kBlockThreads, 1)
topk_block_kernel(const float *__restrict__ scores, int Tq, int L, int q_pos0, int k, int include_self,
                  int32_t *__restrict__ idx) {
    __shared__ int hist[kBins];
    __shared__ int warp_sum[kBlockWarps];
    __shared__ int warp_gt[kBlockWarps], warp_eq[kBlockWarps];
    __shared__ int s_digit, s_above;

    const int row = blockIdx.x;
    const int t = q_pos0 + row % Tq;
    const int n = t + 1;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    int32_t *out = idx + (size_t)row * k;

    if (n <= k) {  // every candidate is kept
        for (int j = tid; j < k; j += kBlockThreads) out[j] = j < n ? j : -1;
        return;
    }
    for (int b = tid; b < kBins; b += kBlockThreads) hist[b] = 0;

    // ---- the row's keys into registers; positions >= n get key 0, below
    // every real key (never selected: n > k real keys exist)
    const float *src = scores + (size_t)row * L;
    const int base = warp * 32 * KPT + lane;
    uint32_t key[KPT];
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int s = base + 32 * j;
        key[j] = s < n ? block_order_key(src[s]) : 0u;
        if (include_self && s == t) key[j] = 0xFFFFFFFFu;  // the row's own position is always kept
    }
    __syncthreads();

    // ---- pass 1: bits 31-21
#pragma unroll
    for (int j = 0; j < KPT; ++j)
        if (base + 32 * j < n) atomicAdd(&hist[key[j] >> 21], 1);
    __syncthreads();
    int want = k;
    const uint32_t d1 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
    want -= s_above;
    // ---- pass 2: bits 20-10 of the keys whose bits 31-21 are d1
#pragma unroll
    for (int j = 0; j < KPT; ++j)
        if (base + 32 * j < n && (key[j] >> 21) == d1) atomicAdd(&hist[(key[j] >> 10) & 2047u], 1);
    __syncthreads();
    const uint32_t d2 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
    want -= s_above;
    const uint32_t hi2 = (d1 << 11) | d2;
    // ---- pass 3: bits 9-0 of the keys whose bits 31-10 are (d1, d2)
#pragma unroll
    for (int j = 0; j < KPT; ++j)
        if (base + 32 * j < n && (key[j] >> 10) == hi2) atomicAdd(&hist[key[j] & 1023u], 1);
    __syncthreads();
    const uint32_t d3 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
    want -= s_above;
    const uint32_t T = (hi2 << 10) | d3;  // the k-th largest key
    const int r = want;                   // keys equal to T that are kept (the first r by position)

    // ---- output: counts of keys > T and == T per warp, then in order
    int gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        gt += __popc(__ballot_sync(0xffffffffu, key[j] > T));
        eq += __popc(__ballot_sync(0xffffffffu, key[j] == T));
    }
    if (lane == 0) {
        warp_gt[warp] = gt;
        warp_eq[warp] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        const int g = warp_gt[lane], e = warp_eq[lane];
        const int gi = warp_inclusive_scan(g), ei = warp_inclusive_scan(e);
        warp_gt[lane] = gi - g;
        warp_eq[lane] = ei - e;
    }
    __syncthreads();
    int gt_b = warp_gt[warp], eq_b = warp_eq[warp];
    const unsigned lt = lanemask_lt_block();
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const bool g = key[j] > T, e = key[j] == T;
        const unsigned gm = __ballot_sync(0xffffffffu, g);
        const unsigned em = __ballot_sync(0xffffffffu, e);
        const int eq_rank = eq_b + __popc(em & lt);
        if (g || (e && eq_rank < r)) out[gt_b + __popc(gm & lt) + min(r, eq_rank)] = base + 32 * j;
        gt_b += __popc(gm);
        eq_b += __popc(em);
    }
}

template <int KPT>
cudaError_t launch_block(const TopkProblem &p, cudaStream_t stream) {
    const long long rows = (long long)p.B * p.Tq;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    topk_block_kernel<KPT><<<(unsigned)rows, kBlockThreads, 0, stream>>>(p.scores, p.Tq, p.L, p.q_pos0, p.k,
                                                                          p.include_self ? 1 : 0, p.idx);
    count_launch();
    return cudaGetLastError();
}

// One CTA per row with the row's keys in shared memory (rows of up to
// kSmemMaxN scores): the scores are read once with 16-byte loads, turned
// into keys in shared memory, and the three radix passes and the output run
// from there, with no cluster synchronisation. Positions are dealt to the
// warps in contiguous segments (lane l of a warp takes every 32nd position of
// its segment: conflict-free shared-memory reads), so that per-warp ballots
// and one block scan give each kept position its slot in ascending order.
constexpr int kSmemMaxN = 49152;

__global__ void __launch_bounds__(kBlockThreads, 1)
topk_smem_kernel(const float *__restrict__ scores, int Tq, int L, int q_pos0, int k, int include_self,
                 int32_t *__restrict__ idx) {
    extern __shared__ uint32_t keys[];
    __shared__ int hist[kBins];
    __shared__ int warp_sum[kBlockWarps];
    __shared__ int warp_gt[kBlockWarps], warp_eq[kBlockWarps];
    __shared__ int s_digit, s_above;

    const int row = blockIdx.x;
    const int t = q_pos0 + row % Tq;
    const int n = t + 1;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    int32_t *out = idx + (size_t)row * k;

    if (n <= k) {  // every candidate is kept
        for (int j = tid; j < k; j += kBlockThreads) out[j] = j < n ? j : -1;
        return;
    }
    for (int b = tid; b < kBins; b += kBlockThreads) hist[b] = 0;

    // ---- keys into shared memory: 16-byte loads from the first aligned element
    const float *src = scores + (size_t)row * L;
    const int head = (int)((4 - (((uintptr_t)src >> 2) & 3)) & 3);  // scalars before 16-byte alignment
    const int h = head < n ? head : n;
    for (int s = tid; s < h; s += kBlockThreads) keys[s] = block_order_key(src[s]);
    const int n4 = (n - h) >> 2;
    const float4 *src4 = reinterpret_cast<const float4 *>(src + h);
#pragma unroll 4
    for (int v = tid; v < n4; v += kBlockThreads) {
        const float4 x = src4[v];
        const int s = h + 4 * v;
        keys[s] = block_order_key(x.x);
        keys[s + 1] = block_order_key(x.y);
        keys[s + 2] = block_order_key(x.z);
        keys[s + 3] = block_order_key(x.w);
    }
    for (int s = h + 4 * n4 + tid; s < n; s += kBlockThreads) keys[s] = block_order_key(src[s]);
    __syncthreads();
    if (include_self && tid == 0) keys[t] = 0xFFFFFFFFu;  // the row's own position is always kept
    __syncthreads();

    // ---- pass 1: bits 31-21
    for (int s = tid; s < n; s += kBlockThreads) atomicAdd(&hist[keys[s] >> 21], 1);
    __syncthreads();
    int want = k;
    const uint32_t d1 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
    want -= s_above;
    // ---- pass 2: bits 20-10 of the keys whose bits 31-21 are d1
    for (int s = tid; s < n; s += kBlockThreads) {
        const uint32_t x = keys[s];
        if ((x >> 21) == d1) atomicAdd(&hist[(x >> 10) & 2047u], 1);
    }
    __syncthreads();
    const uint32_t d2 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
    want -= s_above;
    const uint32_t hi2 = (d1 << 11) | d2;
    // ---- pass 3: bits 9-0 of the keys whose bits 31-10 are (d1, d2)
    for (int s = tid; s < n; s += kBlockThreads) {
        const uint32_t x = keys[s];
        if ((x >> 10) == hi2) atomicAdd(&hist[x & 1023u], 1);
    }
    __syncthreads();
    const uint32_t d3 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
    want -= s_above;
    const uint32_t T = (hi2 << 10) | d3;  // the k-th largest key
    const int r = want;                   // keys equal to T that are kept (the first r by position)

    // ---- output: warp w takes positions [w * seg, (w + 1) * seg)
    const int seg = ((n + kBlockWarps - 1) / kBlockWarps + 31) & ~31;
    const int s0 = warp * seg, s1 = min(n, s0 + seg);
    int gt = 0, eq = 0;
    for (int s = s0 + lane; s < s0 + seg; s += 32) {
        const uint32_t x = s < s1 ? keys[s] : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, x > T));
        eq += __popc(__ballot_sync(0xffffffffu, x == T && s < s1));
    }
    if (lane == 0) {
        warp_gt[warp] = gt;
        warp_eq[warp] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        const int g = warp_gt[lane], e = warp_eq[lane];
        const int gi = warp_inclusive_scan(g), ei = warp_inclusive_scan(e);
        warp_gt[lane] = gi - g;
        warp_eq[lane] = ei - e;
    }
    __syncthreads();
    int gt_b = warp_gt[warp], eq_b = warp_eq[warp];
    const unsigned lt = lanemask_lt_block();
    for (int s = s0 + lane; s < s0 + seg; s += 32) {
        const uint32_t x = s < s1 ? keys[s] : 0u;
        const bool g = x > T, e = x == T && s < s1;
        const unsigned gm = __ballot_sync(0xffffffffu, g);
        const unsigned em = __ballot_sync(0xffffffffu, e);
        const int eq_rank = eq_b + __popc(em & lt);
        if (g || (e && eq_rank < r)) out[gt_b + __popc(gm & lt) + min(r, eq_rank)] = s;
        gt_b += __popc(gm);
        eq_b += __popc(em);
    }
}

// Merge of per-shard selections (context parallelism): row `row` has P * kc
// candidates, candidate c = p * kc + j at cand_*[(p * rows + row) * kc + j],
// ordered by ascending global position (shards in position order, each list
// ascending). The k best valid candidates (cand_idx >= 0) by score, ties to
// the lower position (= the lower candidate number), are written as global
// positions in ascending order, then -1. Same radix select as above, with the
// invalid candidates given key 0, below every score.
template <int KPT>
__global__ void __launch_bounds__(kBlockThreads, 1)
topk_merge_kernel(const float *__restrict__ cand_score, const int32_t *__restrict__ cand_idx, int P, int rows,
                  int kc, int k, int32_t *__restrict__ idx) {
    __shared__ int hist[kBins];
    __shared__ int warp_sum[kBlockWarps];
    __shared__ int warp_gt[kBlockWarps], warp_eq[kBlockWarps];
    __shared__ int s_digit, s_above;

    const int row = blockIdx.x;
    const int n = P * kc;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    int32_t *out = idx + (size_t)row * k;
    for (int b = tid; b < kBins; b += kBlockThreads) hist[b] = 0;

    const int base = warp * 32 * KPT + lane;
    uint32_t key[KPT];
    int nvalid = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int c = base + 32 * j;
        key[j] = 0u;
        if (c < n) {
            const int p = c / kc, jj = c - p * kc;
            const size_t off = ((size_t)p * rows + row) * kc + jj;
            if (cand_idx[off] >= 0) {
                key[j] = block_order_key(cand_score[off]);
                ++nvalid;
            }
        }
    }
    nvalid = warp_sum_int(nvalid);
    if (lane == 0) warp_gt[warp] = nvalid;
    __syncthreads();
    int total = 0;
    for (int w = 0; w < kBlockWarps; ++w) total += warp_gt[w];
    __syncthreads();

    uint32_t T = 0u;  // every valid key is above 0
    int r = 0;
    if (total > k) {
#pragma unroll
        for (int j = 0; j < KPT; ++j)
            if (base + 32 * j < n) atomicAdd(&hist[key[j] >> 21], 1);
        __syncthreads();
        int want = k;
        const uint32_t d1 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
        want -= s_above;
#pragma unroll
        for (int j = 0; j < KPT; ++j)
            if (base + 32 * j < n && (key[j] >> 21) == d1) atomicAdd(&hist[(key[j] >> 10) & 2047u], 1);
        __syncthreads();
        const uint32_t d2 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
        want -= s_above;
        const uint32_t hi2 = (d1 << 11) | d2;
#pragma unroll
        for (int j = 0; j < KPT; ++j)
            if (base + 32 * j < n && (key[j] >> 10) == hi2) atomicAdd(&hist[key[j] & 1023u], 1);
        __syncthreads();
        const uint32_t d3 = (uint32_t)find_digit(hist, want, warp_sum, &s_digit, &s_above);
        want -= s_above;
        T = (hi2 << 10) | d3;
        r = want;
    }

    int gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        gt += __popc(__ballot_sync(0xffffffffu, key[j] > T));
        eq += __popc(__ballot_sync(0xffffffffu, key[j] == T));
    }
    if (lane == 0) {
        warp_gt[warp] = gt;
        warp_eq[warp] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        const int g = warp_gt[lane], e = warp_eq[lane];
        const int gi = warp_inclusive_scan(g), ei = warp_inclusive_scan(e);
        warp_gt[lane] = gi - g;
        warp_eq[lane] = ei - e;
    }
    __syncthreads();
    int gt_b = warp_gt[warp], eq_b = warp_eq[warp];
    const unsigned lt = lanemask_lt_block();
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const bool g = key[j] > T, e = key[j] == T && T != 0u;
        const unsigned gm = __ballot_sync(0xffffffffu, g);
        const unsigned em = __ballot_sync(0xffffffffu, e);
        const int eq_rank = eq_b + __popc(em & lt);
        if (g || (e && eq_rank < r)) {
            const int c = base + 32 * j;
            const int p = c / kc, jj = c - p * kc;
            out[gt_b + __popc(gm & lt) + min(r, eq_rank)] = cand_idx[((size_t)p * rows + row) * kc + jj];
        }
        gt_b += __popc(gm);
        eq_b += __popc(em);
    }
    const int kept = total < k ? total : k;
    for (int j = kept + tid; j < k; j += kBlockThreads) out[j] = -1;
}

}  // namespace

cudaError_t launch_topk_merge(const float *cand_score, const int32_t *cand_idx, int P, int rows, int kc, int k,
                              int32_t *idx, cudaStream_t stream) {
    const long long n = (long long)P * kc;
    if (n > (long long)kBlockThreads * 16 || rows < 1) return cudaErrorInvalidValue;
    if (n <= (long long)kBlockThreads * 8)
        topk_merge_kernel<8><<<rows, kBlockThreads, 0, stream>>>(cand_score, cand_idx, P, rows, kc, k, idx);
    else
        topk_merge_kernel<16><<<rows, kBlockThreads, 0, stream>>>(cand_score, cand_idx, P, rows, kc, k, idx);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_topk_smem(const TopkProblem &p, cudaStream_t stream, bool *taken) {
    *taken = false;
    const long long rows = p.B * (long long)p.Tq;
    const long long n_max = (long long)p.q_pos0 + p.Tq;
    if (rows == 0 || rows > 0x7fffffffLL || n_max > kSmemMaxN) return cudaSuccess;
    // with fewer rows than SMs the row is better split over a cluster (decode32k:
    // 16.5 us with eight CTAs per row, 20.5 us with one)
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    if (rows < info.sm_count) return cudaSuccess;
    const size_t smem = (size_t)n_max * sizeof(uint32_t);
    err = cudaFuncSetAttribute(topk_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    *taken = true;
    topk_smem_kernel<<<(unsigned)rows, kBlockThreads, smem, stream>>>(p.scores, p.Tq, p.L, p.q_pos0, p.k,
                                                                      p.include_self ? 1 : 0, p.idx);
    count_launch();
    return cudaGetLastError();
}

// One CTA per row for many rows of at most 16,384 scores (measured on B200:
// prefill8k 0.41 -> 0.27 ms; with 32 keys per thread the kernel spills and is
// slower than the cluster kernel, and a few long decode rows run faster split
// over a cluster of CTAs).
cudaError_t launch_topk_block(const TopkProblem &p, cudaStream_t stream, bool *taken) {
    *taken = false;
    const long long rows = p.B * (long long)p.Tq;
    const long long n_max = (long long)p.q_pos0 + p.Tq;
    if (rows == 0 || n_max > (long long)kBlockThreads * 16) return cudaSuccess;
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    if (rows < info.sm_count) return cudaSuccess;
    *taken = true;
    if (n_max <= (long long)kBlockThreads * 8) return launch_block<8>(p, stream);
    return launch_block<16>(p, stream);
}

}  // namespace dsa
