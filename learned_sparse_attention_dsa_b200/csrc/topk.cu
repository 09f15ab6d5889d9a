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
// fewer rows than SMs, as in decode), each owning a contiguous slice. A slice
// of at most 512 * KPT keys is held in registers (KPT keys per thread);
// longer slices are streamed from global memory (L2 after the first read), so
// two CTAs fit on an SM. The exchange is built from few cluster barriers,
// each preceded by fire-and-forget writes into the other CTAs' shared memory:
//  1. every CTA adds the non-empty bins of its first-digit histogram into
//     every CTA's copy of the row histogram (distributed shared memory
//     atomics); after one barrier each CTA picks the same first digit d1
//     locally;
//  2. every CTA compacts the keys of bucket d1 -- usually a few percent of
//     the row -- into a list in position order and stores it, 16 bytes at a
//     time, into its own region of every CTA's gather buffer, with its
//     candidate count and its count of keys above d1; after a second barrier
//     each CTA runs passes 2 and 3 alone on the gathered keys (warp c walks
//     the region of CTA c) and touches no other CTA's memory again.
// When some CTA has more candidates than its region holds (heavy ties),
// passes 2 and 3 run cluster-wide instead: each CTA reduces one segment of
// the digit histograms over the cluster and the digit is found from the
// segment totals (the lists, or sweeps when a list overflows, feed them).
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
constexpr int kListCap = 4096;    // candidate keys + positions of this CTA, in shared memory
constexpr int kGatherCap = 8192;  // candidate keys of the whole row gathered by every CTA
// (list + gather buffer + scratch + histograms stay under half the shared
// memory of an SM, so two 512-thread CTAs fit)
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

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct FindScratch {
    int local[kWarps];       // per-warp totals of the digit search
    int red[kBins];          // the cluster-summed first-digit histogram; later (passes 2
                             // and 3 of the slow path) this CTA's segment of a summed one
    int seg_total;           // sum of that segment
    int pad_[3];             // keeps the gather buffer after this struct 16-byte aligned
};

__device__ __forceinline__ void pick_in_segment(const int *seg_bins, int seg, int first_digit, int base_above,
                                                int remaining, FindScratch &fs, int *s_digit, int *s_above);

// Cluster-wide digit search by reduce-scatter: CTA `part` sums bins
// [part*seg, (part+1)*seg) over all P histograms (seg = NBINS / P) into its
// own shared memory; after a cluster barrier every CTA reads the P segment
// totals, picks the segment holding the remaining-th largest key (highest
// bins first) and reads only that segment from its owner. Each CTA moves
// NBINS + P + seg values over distributed shared memory per pass instead of
// P * NBINS. Ends with s_digit / s_above set.
template <int NBINS>
__device__ __forceinline__ void find_digit_rs(const cg::cluster_group &cluster, int *hist, int P, int part,
                                              int remaining, FindScratch &fs, int *s_digit, int *s_above,
                                              int *s_seg) {
    const int seg = NBINS / P;  // >= 64, a multiple of 4
    const int lo = part * seg;
    // 1. reduce this CTA's segment over the cluster (int4 columns x ranks)
    for (int c = threadIdx.x; c < seg / 4; c += kThreads) {
        int4 acc = make_int4(0, 0, 0, 0);
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
            if (r < P) {
                const int4 v = *reinterpret_cast<const int4 *>(cluster.map_shared_rank(hist, r) + lo + 4 * c);
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
        }
        *reinterpret_cast<int4 *>(fs.red + lo + 4 * c) = acc;
    }
    __syncthreads();
    if (threadIdx.x < kWarp) {
        int s = 0;
        for (int b = lo + threadIdx.x; b < lo + seg; b += kWarp) s += fs.red[b];
        s = warp_sum_int(s);
        if (threadIdx.x == 0) fs.seg_total = s;
    }
    cluster.sync();
    // 2. which segment (highest bins first), then which bin inside it
    if (threadIdx.x < kWarp) {
        const int lane = threadIdx.x;
        const int sg = P - 1 - lane;  // lane 0 looks at the highest segment
        const int tot = lane < P ? *cluster.map_shared_rank(&fs.seg_total, sg) : 0;
        const int incl = warp_inclusive_scan(tot);
        const int excl = incl - tot;
        if (lane < P && excl < remaining && incl >= remaining) {
            *s_seg = sg;
            *s_above = excl;
        }
    }
    __syncthreads();
    const int sg = *s_seg;
    const int base_above = *s_above;
    pick_in_segment(cluster.map_shared_rank(fs.red, sg) + sg * seg, seg, sg * seg, base_above, remaining, fs,
                    s_digit, s_above);
}

// Bins seg_bins[0..seg) hold the counts of digits first_digit .. first_digit +
// seg - 1; base_above keys lie in higher digits. Find the digit whose bucket
// holds the remaining-th largest key: thread i sums the per = max(1, seg /
// kThreads) consecutive bins below seg - 1 - i * per (descending digits), a
// block-wide scan of those sums finds the one thread whose range crosses
// `remaining`, and that thread walks its own bins. Sets s_digit / s_above.
// Two block barriers.
__device__ __forceinline__ void pick_in_segment(const int *seg_bins, int seg, int first_digit, int base_above,
                                                int remaining, FindScratch &fs, int *s_digit, int *s_above) {
    const int per = seg >= kThreads ? seg / kThreads : 1;
    const int top = seg - 1 - (int)threadIdx.x * per;  // this thread's highest bin
    int local = 0;
    if (top >= 0)
        for (int j = 0; j < per; ++j) local += seg_bins[top - j];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_inclusive_scan(local);
    if (lane == kWarp - 1) fs.local[warp] = incl;  // warp totals
    __syncthreads();
    const int before = warp_sum_int(lane < warp ? fs.local[lane] : 0);  // kWarps <= 32
    const int upto = base_above + before + incl;  // keys in this thread's bins and above
    int run = upto - local;                       // keys above this thread's bins
    if (run < remaining && upto >= remaining) {
        for (int j = 0; j < per; ++j) {
            const int c = seg_bins[top - j];
            if (run + c >= remaining) {
                *s_digit = first_digit + top - j;
                *s_above = run;
                break;
            }
            run += c;
        }
    }
    __syncthreads();
}

struct Slice {
    const float *src;  // first score of this CTA's slice
    int cnt;           // scores in the slice
    int w_lo, w_hi;    // this warp's segment [w_lo, w_hi) of the slice
    int self_s;        // slice position forced into the selection, or -1
};

// Key of slice position s: the order-preserving key of its score, or (SELF:
// keep the row's own position) the largest key, above every finite score.
template <bool SELF>
__device__ __forceinline__ uint32_t slice_key(const Slice &sl, int s, float v) {
    if constexpr (SELF) return s == sl.self_s ? 0xFFFFFFFFu : order_key(v);
    return order_key(v);
}

template <int KPT>
struct RegKeys {
    uint32_t k[KPT > 0 ? KPT : 1];
};

// Apply fn(pos, key, valid) to the warp's segment in position order: 32
// consecutive positions per step. KPT > 0: the keys are the registers loaded
// by load_keys; KPT == 0: streamed from global memory, four steps' loads in
// flight.
template <int KPT, bool SELF, typename F>
__device__ __forceinline__ void sweep(const Slice &sl, const RegKeys<KPT> &rk, F fn) {
    const int lane = threadIdx.x & 31;
    if constexpr (KPT > 0) {
#pragma unroll
        for (int i = 0; i < KPT; ++i) {
            const int s = sl.w_lo + i * kWarp + lane;
            fn(s, rk.k[i], s < sl.w_hi);
        }
    } else {
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
                fn(s, slice_key<SELF>(sl, s, v[u]), s < sl.w_hi);
            }
        }
    }
}

template <int KPT, bool SELF>
__global__ void __launch_bounds__(kThreads, 2)  // two CTAs per SM: at most 64 registers
topk_kernel(const float *__restrict__ scores, int Tq, int L, int q_pos0, int k, int32_t *__restrict__ idx) {
    __shared__ __align__(16) int hist[3][kBins];
    extern __shared__ __align__(16) uint8_t dyn_smem[];
    uint32_t *list_key = reinterpret_cast<uint32_t *>(dyn_smem);                // [kListCap]
    int32_t *list_pos = reinterpret_cast<int32_t *>(dyn_smem + 4 * kListCap);   // [kListCap]
    FindScratch &fs = *reinterpret_cast<FindScratch *>(dyn_smem + 8 * kListCap);
    uint32_t *gkey = reinterpret_cast<uint32_t *>(dyn_smem + 8 * kListCap + sizeof(FindScratch));  // [kGatherCap]
    // per warp: candidates in bucket d1, keys above it, and (gathered path)
    // candidates > T and = T
    __shared__ int w_cnt[kWarps], w_gt[kWarps], w_eq[kWarps], w_gtT[kWarps];
    __shared__ int s_digit, s_above, s_seg;
    __shared__ int s_counts[2], s_before[2];
    __shared__ int g_n[kMaxCluster], g_gt1[kMaxCluster];  // per CTA of the cluster

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
    const int seg = KPT > 0 ? KPT * kWarp : ((sl.cnt + kWarps - 1) / kWarps + 31) & ~31;
    sl.w_lo = min(sl.cnt, warp * seg);
    sl.w_hi = min(sl.cnt, sl.w_lo + seg);
    // the row's own position t = n - 1 sits at the end of the last slice
    sl.self_s = (SELF && t >= lo && t < lo + sl.cnt) ? t - lo : -1;

    // ---- pass 1: bits 31..21 of every key. The keys' loads (into registers)
    // are issued first, so that their latency overlaps the zeroing below.
    RegKeys<KPT> rk;
    if constexpr (KPT > 0) {
#pragma unroll
        for (int i = 0; i < KPT; ++i) {
            const int s = sl.w_lo + i * kWarp + lane;
            const float v = s < sl.w_hi ? __ldg(sl.src + s) : 0.0f;
            rk.k[i] = slice_key<SELF>(sl, s, v);
        }
    }
    // zero the three local histograms and fs.red, which receives the
    // cluster-wide sum of the first-digit histograms
    {
        int4 *h4 = reinterpret_cast<int4 *>(&hist[0][0]);
        for (int i = threadIdx.x; i < 3 * kBins / 4; i += kThreads) h4[i] = make_int4(0, 0, 0, 0);
        int4 *r4 = reinterpret_cast<int4 *>(fs.red);
        for (int i = threadIdx.x; i < kBins / 4; i += kThreads) r4[i] = make_int4(0, 0, 0, 0);
    }
    if (threadIdx.x == 0) {
        s_seg = 0;  // always a valid cluster rank, even if a search found nothing
        s_digit = 0;
        s_above = 0;
        s_before[0] = 0;
        s_before[1] = 0;
    }
    __syncthreads();
    cluster_arrive();  // (1) this CTA's sum is zeroed; waited on after pass 1

    sweep<KPT, SELF>(sl, rk, [&](int, uint32_t key, bool ok) {
        if (ok) atomicAdd(&hist[0][key >> 21], 1);
    });
    __syncthreads();
    cluster_wait();  // (1) every CTA of the cluster has zeroed its sum
    // add this CTA's non-empty bins into every CTA's sum
    for (int b = threadIdx.x; b < kBins; b += kThreads) {
        const int c = hist[0][b];
        if (c)
            for (int r = 0; r < P; ++r) atomicAdd(cluster.map_shared_rank(fs.red, r) + b, c);
    }
    cluster.sync();  // (2) the row's first-digit histogram is complete everywhere
    pick_in_segment(fs.red, kBins, 0, 0, k, fs, &s_digit, &s_above);
    const uint32_t d1 = (uint32_t)s_digit;
    int remaining = k - s_above;

    // ---- per warp: keys in bucket d1 (candidates) and above it
    {
        int cnt = 0, gt1 = 0;
        sweep<KPT, SELF>(sl, rk, [&](int, uint32_t key, bool ok) {
            cnt += ok && (key >> 21) == d1;
            gt1 += ok && (key >> 21) > d1;
        });
        cnt = warp_sum_int(cnt);
        gt1 = warp_sum_int(gt1);
        if (lane == 0) {
            w_cnt[warp] = cnt;
            w_gt[warp] = gt1;
            w_eq[warp] = 0;
        }
    }
    __syncthreads();
    // first slot of this warp's candidates among the CTA's, and their number (kWarps <= 32)
    const int wbase = warp_sum_int(lane < warp ? w_cnt[lane] : 0);
    const int n_list = warp_sum_int(lane < kWarps ? w_cnt[lane] : 0);
    const bool use_list = n_list <= kListCap;
    // gather-buffer region of each CTA (a multiple of four keys); never more
    // than the list holds, so a gathered CTA always has its list
    const int cap = min(kGatherCap / P, kListCap);

    // ---- this CTA's candidates into its list, in position order
    if (use_list) {
        int slot = wbase;
        sweep<KPT, SELF>(sl, rk, [&](int s, uint32_t key, bool ok) {
            const bool cand = ok && (key >> 21) == d1;
            const unsigned m = __ballot_sync(0xffffffffu, cand);
            if (cand) {
                const int j = slot + __popc(m & lanemask_lt());
                list_key[j] = key;
                list_pos[j] = s;
            }
            slot += __popc(m);
        });
    }
    // the number of candidates and of keys above bucket d1, to every CTA
    if (threadIdx.x < P) {
        int g = 0;
        for (int w = 0; w < kWarps; ++w) g += w_gt[w];
        cluster.map_shared_rank(g_n, threadIdx.x)[part] = n_list;
        cluster.map_shared_rank(g_gt1, threadIdx.x)[part] = g;
    }
    if (n_list <= cap) {
        // the list into this CTA's region of every CTA's gather buffer, 16 bytes at a time
        __syncthreads();
        const int n4 = (n_list + 3) >> 2;
        const uint4 *src = reinterpret_cast<const uint4 *>(list_key);
        for (int i = threadIdx.x; i < P * n4; i += kThreads) {
            const int r = i / n4, q = i - r * n4;
            reinterpret_cast<uint4 *>(cluster.map_shared_rank(gkey, r) + part * cap)[q] = src[q];
        }
    }
    cluster.sync();  // (3) candidates and counts delivered; no remote access after this on the gathered path
    // the gathered path when every CTA's candidates fit its region (the same decision everywhere)
    const bool gather = __syncthreads_and(threadIdx.x >= P || g_n[threadIdx.x] <= cap);

    uint32_t T;
    int r, gt_b = 0, eq_b = 0;
    if (gather) {
        // ---- every CTA holds all candidate keys of the row, CTA c's in
        // region c in position order, and finishes the selection alone;
        // warp c walks region c
        const uint32_t *reg = gkey + warp * cap;
        const int n_reg = warp < P ? g_n[warp] : 0;
        for (int j = lane; j < n_reg; j += kWarp) atomicAdd(&hist[1][(reg[j] >> 10) & 2047u], 1);
        __syncthreads();
        pick_in_segment(hist[1], kBins, 0, 0, remaining, fs, &s_digit, &s_above);
        const uint32_t p2 = (d1 << 11) | (uint32_t)s_digit;
        remaining -= s_above;
        for (int j = lane; j < n_reg; j += kWarp) {
            const uint32_t key = reg[j];
            if ((key >> 10) == p2) atomicAdd(&hist[2][key & 1023u], 1);
        }
        __syncthreads();
        pick_in_segment(hist[2], 1024, 0, 0, remaining, fs, &s_digit, &s_above);
        T = (p2 << 10) | (uint32_t)s_digit;
        remaining -= s_above;
        r = remaining;
        // candidates > T and = T in the CTAs before this one (warp c: region c)
        if (warp < part) {
            int gb = 0, eb = 0;
            for (int j = lane; j < n_reg; j += kWarp) {
                const uint32_t key = reg[j];
                gb += key > T;
                eb += key == T;
            }
            gb = warp_sum_int(gb);
            eb = warp_sum_int(eb);
            if (lane == 0) {
                atomicAdd(&s_before[0], gb);
                atomicAdd(&s_before[1], eb);
            }
        }
        // ... and in this warp's own range of this CTA's region
        int wg = 0, we = 0;
        for (int j = lane; j < w_cnt[warp]; j += kWarp) {
            const uint32_t key = gkey[part * cap + wbase + j];
            wg += key > T;
            we += key == T;
        }
        wg = warp_sum_int(wg);
        we = warp_sum_int(we);
        if (lane == 0) {
            w_gtT[warp] = wg;
            w_eq[warp] = we;
        }
        __syncthreads();
        gt_b = s_before[0] + warp_sum_int(lane < warp ? w_gt[lane] + w_gtT[lane] : 0);
        eq_b = s_before[1] + warp_sum_int(lane < warp ? w_eq[lane] : 0);
        for (int c = 0; c < part; ++c) gt_b += g_gt1[c];
    } else {
        // ---- too many candidates (heavy ties): cluster-wide passes 2 and 3
    // ---- pass 2: bits 20..10 of the keys in bucket d1
    if (use_list) {
        for (int j = threadIdx.x; j < n_list; j += kThreads)
            atomicAdd(&hist[1][(list_key[j] >> 10) & 2047u], 1);
    } else {
        sweep<KPT, SELF>(sl, rk, [&](int, uint32_t key, bool ok) {
            if (ok && (key >> 21) == d1) atomicAdd(&hist[1][(key >> 10) & 2047u], 1);
        });
    }
    __syncthreads();
    cluster.sync();
    find_digit_rs<kBins>(cluster, hist[1], P, part, remaining, fs, &s_digit, &s_above, &s_seg);
    const uint32_t p2 = (d1 << 11) | (uint32_t)s_digit;
    remaining -= s_above;

    // ---- pass 3: bits 9..0 of the keys whose top 22 bits are p2
    if (use_list) {
        for (int j = threadIdx.x; j < n_list; j += kThreads) {
            const uint32_t key = list_key[j];
            if ((key >> 10) == p2) atomicAdd(&hist[2][key & 1023u], 1);
        }
    } else {
        sweep<KPT, SELF>(sl, rk, [&](int, uint32_t key, bool ok) {
            if (ok && (key >> 10) == p2) atomicAdd(&hist[2][key & 1023u], 1);
        });
    }
    __syncthreads();
    cluster.sync();
    find_digit_rs<1024>(cluster, hist[2], P, part, remaining, fs, &s_digit, &s_above, &s_seg);
    T = (p2 << 10) | (uint32_t)s_digit;
    remaining -= s_above;
    r = remaining;  // keys equal to T that still fit, lowest positions first

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
        sweep<KPT, SELF>(sl, rk, [&](int, uint32_t key, bool ok) {
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
    for (int c = 0; c < part; ++c) {
        const int *rc = cluster.map_shared_rank(s_counts, c);
        gt_b += rc[0];
        eq_b += rc[1];
    }
    cluster_arrive();  // done with the other CTAs' shared memory
    gt_b += w_gt[warp];
    eq_b += w_eq[warp];
    }

    // ---- write the kept positions of this warp's segment in order
    const unsigned lt = lanemask_lt();
    sweep<KPT, SELF>(sl, rk, [&](int s, uint32_t key, bool ok) {
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
    if (!gather) cluster_wait();  // no CTA leaves while another may still read its shared memory
}

constexpr size_t kDynSmem = 8 * (size_t)kListCap + sizeof(FindScratch) + 4 * (size_t)kGatherCap;

}  // namespace

size_t topk_workspace_bytes(int, int, int, int, int) { return 0; }

namespace {

__global__ void dense_selection_kernel(int Tq, int q_pos0, int k, int32_t *__restrict__ idx) {
    const int row = blockIdx.x;
    const int t = q_pos0 + row % Tq;
    int32_t *out = idx + (size_t)row * k;
    for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = j <= t ? j : -1;
}

}  // namespace

cudaError_t launch_dense_selection(const TopkProblem &p, cudaStream_t stream) {
    const long long rows = (long long)p.B * p.Tq;
    if (rows == 0) return cudaSuccess;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    dense_selection_kernel<<<(unsigned)rows, 256, 0, stream>>>(p.Tq, p.q_pos0, p.k, p.idx);
    count_launch();
    return cudaGetLastError();
}

// CTAs per row: enough to cover the SMs when rows are few (at most 16).
static int cluster_parts(int rows, int sm_count) {
    int P = 1;
    while (P < kMaxCluster && (long long)rows * P < (long long)sm_count) P *= 2;
    return P;
}

template <int KPT, bool SELF>
static cudaError_t launch_parts(const TopkProblem &p, int P, cudaStream_t stream) {
    auto kern = topk_kernel<KPT, SELF>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDynSmem);
    if (err != cudaSuccess) return err;
    if (P > 8) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
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
        err = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
        if (err != cudaSuccess || clusters == 0) {
            (void)cudaGetLastError();
            return cudaErrorNotSupported;
        }
    }
    err = cudaLaunchKernelEx(&cfg, kern, p.scores, p.Tq, p.L, p.q_pos0, p.k, p.idx);
    count_launch();
    return err;
}

// Keys per thread held in registers for a slice of `per` scores (0: stream).
static cudaError_t launch_with(const TopkProblem &p, int P, cudaStream_t stream) {
    const int n_max = p.q_pos0 + p.Tq;
    const int per = (n_max + P - 1) / P;
    if (p.include_self) {
        if (per <= kThreads * 8) return launch_parts<8, true>(p, P, stream);
        if (per <= kThreads * 16) return launch_parts<16, true>(p, P, stream);
        return launch_parts<0, true>(p, P, stream);
    }
    if (per <= kThreads * 8) return launch_parts<8, false>(p, P, stream);
    if (per <= kThreads * 16) return launch_parts<16, false>(p, P, stream);
    return launch_parts<0, false>(p, P, stream);
}

cudaError_t launch_topk_block(const TopkProblem &p, cudaStream_t stream, bool *taken);
cudaError_t launch_topk_smem(const TopkProblem &p, cudaStream_t stream, bool *taken);

cudaError_t launch_topk(const TopkProblem &p, cudaStream_t stream) {
    // many rows of at most 16,384 scores: one CTA per row, the row in registers
    bool taken = false;
    cudaError_t err = launch_topk_block(p, stream, &taken);
    if (taken || err != cudaSuccess) return err;
    // many rows of at most 49,152 scores: one CTA per row, the row in shared memory
    err = launch_topk_smem(p, stream, &taken);
    if (taken || err != cudaSuccess) return err;
    DeviceInfo info;
    err = device_info(&info);
    if (err != cudaSuccess) return err;
    const long long rows = (long long)p.B * p.Tq;
    if (rows == 0) return cudaSuccess;
    int P = cluster_parts((int)(rows < 0x7fffffffLL ? rows : 0x7fffffffLL), info.sm_count);
    if (rows * P >= 0x7fffffffLL) return cudaErrorInvalidValue;
    err = launch_with(p, P, stream);
    if (err == cudaErrorNotSupported && P > 8) err = launch_with(p, 8, stream);
    return err;
}

}  // namespace dsa
