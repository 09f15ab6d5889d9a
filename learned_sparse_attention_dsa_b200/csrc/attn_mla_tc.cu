// Sparse attention over latent KV rows on the 5th-generation tensor cores.
//
//   u[t,h] = sum_{s in S_t} softmax_s(scale * q[t,h] . c[s]) c[s][:512]
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §3.3 and
// §10.1 for the attention, §4.1-4.2 for MLA's shared latent row and the one
// selected set for every head).
//
// Shape: 128 query heads share one 576-wide latent row per position; the value
// is the first 512 columns of that row. The 128 heads are the M of every MMA,
// so each head owns one TMEM lane.
//
// Work split. The two CTAs of a cluster share one (query row, split of S_t)
// and split the 576 columns: part 0 takes columns [0, 320) of Q and of the
// gathered rows, part 1 columns [320, 576). Each computes a partial
//   S_p[h, j] = sum_{e in part p} Q[h, e] c[s_j, e]       M=128, N=64
// on the tensor cores, the parts swap partials through distributed shared
// memory and both form the same S = S_0 + S_1. Part p then owns value columns
// [256 p, 256 p + 256) (part 1 also gathers columns 256-319 for them):
//   O_p[h, :] += P[h, j] c[s_j, 256 p : 256 p + 256]       M=128, N=256
// so each CTA gathers 5 of the 9 64-column boxes of every selected row, and
// holds its part of Q in TMEM as the A operand of QK^T (two bf16 per column).
// An MMA of M=128, K=16 costs about the same for every N up to 64 (measured
// on B200: ~48 cycles, ~65 for N=128, ~129 for N=256), so a tile is 64 keys.
// TMEM: Q part [0,160), S [160,224), O [256,512). Shared memory: a three-slot
// ring of gathered boxes (3 x 40 KB), P twice (2 x 16 KB), the partial-S send
// and receive buffers (2 x 32 KB); the Q part is staged over P and those
// buffers before the first tile, so the ring gathers from the start.
//
// Per CTA (one per SM):
//   warps 0-7  softmax, two warps per TMEM lane quarter: warp w takes heads
//              32 (w % 4) .. + 31 (one per thread) and keys 32 (w / 4) .. + 31
//              of every tile. Each warp swaps its 32 x 32 block of S_p with
//              the same warp of the other part directly: a 4 KB bulk copy
//              into the other part's receive buffer that completes on a
//              barrier of that warp alone. The next tile's S_p is loaded and
//              sent before this tile's softmax, so the swap of tile t + 1 runs
//              under the softmax of tile t. The two warps of a lane quarter
//              agree on the tile's row max through shared memory; the online
//              softmax keeps a reference max that moves only when the row max
//              grows by more than 2^8 (then O is rescaled in TMEM); P goes to
//              shared memory in bf16 (128-byte swizzle), alternating
//              between two buffers so that the softmax of tile t + 1 does not
//              wait for PV of tile t (only a rescale of O does). At the end O
//              leaves TMEM for the output or for a bf16 partial normalised by
//              its own sum.
//   warps 8-14 gather the 5 boxes of 64 selected rows per tile with 16-byte
//              cp.async (one warp instruction fills 4 rows x 128 bytes); the
//              rate at which cp.async is issued grows with the number of
//              issuing warps (measured on B200: ~22 GB/s per SM with three).
//   warp 15    TMEM allocation, the Q staging by TMA, and one thread issuing
//              the MMAs with descriptors built once.
// With several splits, attn_mla_combine_kernel merges the partials.
// Every mbarrier wait is bounded; on a timeout the CTA records an error word,
// waits for the copies and MMAs it issued and for the swaps sent to it, frees
// TMEM and returns.
#include <math.h>

#include <cooperative_groups.h>
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace dsa {

namespace {

using namespace sm100;

constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int kHalfDv = DV / 2;
constexpr int kHeads = 128;                        // query heads per latent row = MMA M
constexpr int kTileN = 64;                         // selected rows per tile
constexpr int kGBoxes = 5;                         // gathered 64-column boxes per part
constexpr int kMaxTiles = 8;                       // tiles per split
constexpr int kMaxSel = kMaxTiles * kTileN;        // selected entries per split
constexpr int kMaxSplits = 32;
constexpr int kSlots = 3;
constexpr int kSoftWarps = 8;
constexpr int kSoftmaxThreads = kSoftWarps * 32;   // 256
constexpr int kGatherThreads = 224;
constexpr int kMmaWarp = (kSoftmaxThreads + kGatherThreads) / 32;  // 15
constexpr int kThreads = (kMmaWarp + 1) * 32;                      // 512
constexpr uint32_t kQBox = kHeads * 128;           // 16,384
constexpr uint32_t kKBox = kTileN * 128;           // 8,192
constexpr uint32_t kKSlot = kGBoxes * kKBox;       // 40,960
constexpr uint32_t kPBytes = kHeads * kTileN * 2;  // 16,384
constexpr uint32_t kXBytes = kHeads * kTileN * 4;  // 32,768: one partial S tile
constexpr uint32_t kXWarpBytes = kXBytes / kSoftWarps;  // 4,096: one warp's 32 heads x 32 keys
constexpr uint32_t kOffP = kSlots * kKSlot;        // P, two buffers; the Q staging from here on
constexpr uint32_t kOffXs = kOffP + 2 * kPBytes;   // this part's S_p, sent to the other part
constexpr uint32_t kOffXr = kOffXs + kXBytes;      // the other part's S_p, received
constexpr uint32_t kOffSel = kOffXr + kXBytes;
constexpr uint32_t kOffMx = kOffSel + kMaxSel * 4;          // [tile parity][key half][head] row maxima
constexpr uint32_t kOffL = kOffMx + 2 * 2 * kHeads * 4;     // [key half][head] row sums
constexpr uint32_t kOffCnt = kOffL + 2 * kHeads * 4;        // [warp] S_p blocks the other part sent here
constexpr uint32_t kOffBar = kOffCnt + kSoftWarps * 4;
constexpr uint32_t kHalfRowBytes = kHalfDv * 2;             // one head's bf16 partial of a part
constexpr int kNumBars = 19 + 2 * kSoftWarps;
constexpr size_t kSmem = 1024 + kOffBar + kNumBars * 8 + 16;  // + slack to align the base to 1024
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;
constexpr uint32_t kColS = 160;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kIdescMnMajorB = 1u << 16;

static_assert(kOffP % 1024 == 0 && kKSlot % 1024 == 0, "operand tiles must sit on 1024-byte boundaries");
static_assert(5 * kQBox <= kOffSel - kOffP, "the Q staging must fit over P and the S_p buffers");
static_assert(kHeads * kHalfRowBytes <= kOffXs, "the partial staging must fit over the ring and P");
static_assert(kOffBar % 8 == 0, "mbarrier alignment");
static_assert(kColS + kTileN <= kColO, "TMEM columns");
static_assert(kSmem <= 232448, "shared memory budget");

// Columns of part p: Q/K boxes [q_box0, q_box0 + q_boxes) for QK^T, gathered
// boxes [4 p, 4 p + 5), value boxes [4 p, 4 p + 4) (local boxes 0-3).
__host__ __device__ constexpr int q_box0(int p) { return p == 0 ? 0 : 5; }
__host__ __device__ constexpr int q_boxes(int p) { return p == 0 ? 5 : 4; }
__host__ __device__ constexpr int g_box0(int p) { return 4 * p; }

__device__ unsigned int g_attn_mla_tc_error = 0;  // kErrTimeout, kErrBadIndex bits

struct Args {
    const __nv_bfloat16 *kv;  // latent rows: element strides sb (batch), ss (position)
    const int32_t *idx;       // [rows, k]
    int Tq, L, k, splits, tiles;  // tiles: 64-entry tiles of the whole selection
    float scale_log2;
    int64_t sb, ss;
    __nv_bfloat16 *out;       // [rows, 128, 512]
    float *lse;               // [rows, 128] or null
    uint4 *part_o;            // split partials (splits > 1), bf16 [rows, splits, 2, 128, 256]
    float *part_ml;           // [rows, 128, splits, 2]: (max in log2 units, sum)
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Where 16-byte chunk q (0..31) of head h's bf16 half row of partials sits:
// rotated by h, so that a warp's 32 rows spread over the shared-memory banks
// of the staging and the combine kernel's loads stay coalesced. The combine
// kernel undoes the rotation.
__host__ __device__ __forceinline__ int rot_chunk(int h, int q) { return (q + h) & 31; }

// Descriptor field arithmetic: the start address sits in the low bits in
// units of 16 bytes, so moving an operand by b bytes adds b >> 4.
__host__ __device__ constexpr uint64_t desc_step(uint32_t bytes) { return (uint64_t)(bytes >> 4); }

// Bulk copy shared -> global of `bytes` (multiple of 16, both 16-byte aligned).
__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_addr(ssrc)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// QK^T of one tile: the part's Q columns (A, TMEM) against its boxes of the
// gathered rows (B, K-major); QB boxes of 4 K=16 steps each.
template <int QB>
__device__ __forceinline__ void issue_qk(uint32_t d, uint32_t a_tmem, uint64_t kd, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < 4 * QB; ++kk)
        mma_f16_ts(d, a_tmem + (uint32_t)(kk * 8), kd + desc_step((kk >> 2) * kKBox + (kk & 3) * 32), idesc,
                   kk > 0 ? 1u : 0u);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *k_sm = smem;               // ring; slots 0-1 first stage the Q part
    uint8_t *p_sm = smem + kOffP;
    uint8_t *xs_sm = smem + kOffXs;
    uint8_t *xr_sm = smem + kOffXr;
    int32_t *sel = reinterpret_cast<int32_t *>(smem + kOffSel);
    float *mx_sm = reinterpret_cast<float *>(smem + kOffMx);
    float *l_sm = reinterpret_cast<float *>(smem + kOffL);
    uint32_t *cnt_sm = reinterpret_cast<uint32_t *>(smem + kOffCnt);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *q_full = bars;            // TMA bytes of the staged Q part
    uint64_t *q_copied = bars + 1;      // 256 softmax threads: Q part in TMEM, staging free
    uint64_t *kv_full = bars + 2;       // [3] gather threads (cp.async arrivals)
    uint64_t *kv_empty = bars + 5;      // [3] MMA commit after PV
    uint64_t *s_full = bars + 8;        // MMA commit after QK^T
    uint64_t *s_free = bars + 9;        // 256 softmax threads (S_p is in registers)
    uint64_t *p_full = bars + 10;       // [2] 256 softmax threads: P buffer b written
    uint64_t *pv_done = bars + 12;      // [2] MMA commit after PV from P buffer b
    uint64_t *drained = bars + 14;      // MMA commit before teardown
    uint64_t *mx_bar = bars + 15;       // [4] the two warps of a lane quarter posted their row maxima
    uint64_t *x_full = bars + 19;       // [8] the other part's block of S_p for warp w landed
    // [8] the other part's warp w may be sent its next block: phase 0 once
    // its receive buffer no longer holds the Q staging, phase t + 1 once it
    // has read block t
    uint64_t *x_free = bars + 19 + kSoftWarps;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);

    const int row = blockIdx.x;
    const int split = blockIdx.y;
    const int part = blockIdx.z;        // = rank in the cluster of two
    const int b = row / a.Tq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this split's tiles: an even share of the selection's 64-entry tiles
    const int tile0 = (int)((long long)split * a.tiles / a.splits);
    const int tile1 = (int)((long long)(split + 1) * a.tiles / a.splits);
    const int j0 = tile0 * kTileN;
    const int n_split = max(0, min(a.k, tile1 * kTileN) - j0);
    const int n_tiles = (n_split + kTileN - 1) / kTileN;

    // this split's selected positions; entries outside [0, L) become -1 (masked)
    for (int j = threadIdx.x; j < n_tiles * kTileN; j += kThreads) {
        int s = -1;
        if (j < n_split) {
            s = a.idx[(size_t)row * a.k + j0 + j];
            note_bad_index(&g_attn_mla_tc_error, s, a.L);
            if (s < 0 || s >= a.L) s = -1;
        }
        sel[j] = s;
    }
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_copied, kSoftmaxThreads);
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&kv_full[i], kGatherThreads);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, kSoftmaxThreads);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&p_full[i], kSoftmaxThreads);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(drained, 1);
        for (int i = 0; i < 4; ++i) mbar_init(&mx_bar[i], 64);
        for (int w = 0; w < kSoftWarps; ++w) {
            mbar_init(&x_full[w], 1);
            mbar_init(&x_free[w], 1);
        }
        fence_barrier_init();
        // armed for the first tile: 4 KB from the other part's warp w
        for (int w = 0; w < kSoftWarps; ++w) mbar_arrive_expect_tx(&x_full[w], kXWarpBytes);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cg::this_cluster().sync();  // both parts' barriers exist before any remote arrival or copy
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = waits_enabled();  // false: the wait limit is 0 (give-up test)
    float m_ref = -INFINITY, l = 0.0f;  // softmax threads: reference max (log2 units), partial sum
    uint32_t sent = 0, recv = 0;        // softmax threads: S_p blocks sent to / received from the other part

    // Tile t lands in ring slot t % 3 (its (t / 3)-th use) and its P in
    // buffer t % 2.
    if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0 && ok) {
            prefetch_tensor_map(&tm_q);
            mbar_arrive_expect_tx(q_full, (uint32_t)q_boxes(part) * kQBox);
#pragma unroll 1
            for (int c = 0; c < q_boxes(part); ++c)
                tma_load_2d(smem + kOffP + c * kQBox, &tm_q, q_full, (q_box0(part) + c) * 64, row * kHeads);
            ok = mbar_wait(q_copied, 0);
            tc_fence_after();
            const uint32_t idesc_qk = idesc_bf16_f32(kHeads, kTileN);
            const uint32_t idesc_pv = idesc_bf16_f32(kHeads, kHalfDv) | kIdescMnMajorB;
            const uint64_t p_desc0 = smem_desc_k_sw128(smem_addr(p_sm));
            // QK^T reads local boxes [q_box0 - g_box0, +q_boxes); PV local boxes 0-3
            const uint64_t k_desc0 =
                smem_desc_k_sw128(smem_addr(k_sm) + (uint32_t)(q_box0(part) - g_box0(part)) * kKBox);
            const uint64_t v_desc0 = smem_desc_mn_sw128(smem_addr(k_sm), kKBox);
            // Two streams of MMAs, each issued as soon as its inputs are ready:
            // QK^T of the next tile (its rows landed, the previous S_p read
            // out of TMEM) and PV of the oldest tile whose P is written. QK^T
            // of tile t + 1 is needed before the softmax of tile t finishes
            // (its S_p block is sent first), so it must not wait behind PV.
            int nq = 0, np = 0;
            uint32_t idle = 0;
            uint64_t t_idle = 0;
            while (ok && np < n_tiles) {
                bool progress = false;
                if (nq < n_tiles && mbar_test_wait(&kv_full[nq % kSlots], (uint32_t)(nq / kSlots) & 1u) &&
                    mbar_test_wait(s_free, ((uint32_t)nq & 1u) ^ 1u)) {
                    fence_proxy_async_smem();  // the rows were written by cp.async
                    tc_fence_after();
                    const uint64_t kd = k_desc0 + desc_step((uint32_t)(nq % kSlots) * kKSlot);
                    if (part == 0)
                        issue_qk<5>(tmem + kColS, tmem + kColQ, kd, idesc_qk);
                    else
                        issue_qk<4>(tmem + kColS, tmem + kColQ, kd, idesc_qk);
                    mma_commit(s_full);
                    ++nq;
                    progress = true;
                }
                if (np < nq && mbar_test_wait(&p_full[np & 1], (uint32_t)(np >> 1) & 1u)) {
                    tc_fence_after();
                    const int slot = np % kSlots;
                    const uint64_t vd = v_desc0 + desc_step((uint32_t)slot * kKSlot);
                    const uint64_t pd = p_desc0 + desc_step((uint32_t)(np & 1) * kPBytes);
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk)  // 16 keys = two 8-row groups = 2048 bytes
                        mma_f16_ss(tmem + kColO, pd + desc_step(kk * 32), vd + desc_step(kk * 2048), idesc_pv,
                                   (np > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&kv_empty[slot]);   // the slot may be refilled
                    mma_commit(&pv_done[np & 1]);  // P buffer np % 2 may be rewritten; O holds every PV so far
                    ++np;
                    progress = true;
                }
                if (progress) {
                    idle = 0;
                } else {
                    // bounded: give up after the wait limit without progress
                    const unsigned long long limit = __ldg(&g_wait_limit_ns);
                    if (idle == 0) t_idle = global_timer_ns();
                    if ((++idle & 63u) == 0u && global_timer_ns() - t_idle > limit) ok = false;
                    __nanosleep(32);
                }
            }
            // nothing of this CTA may still run on the tensor core at teardown,
            // and the Q load has landed
            mma_commit(drained);
            if (!mbar_drain(drained, 0)) ok = false;
            if (!mbar_drain(q_full, 0)) ok = false;
        }
    } else if (warp >= kSoftWarps) {
        // ------------------------------------------------------------ gather
        const int gt = threadIdx.x - kSoftmaxThreads;
        const __nv_bfloat16 *kvb = a.kv + (int64_t)b * a.sb + g_box0(part) * 64;
        const uint32_t k_base = smem_addr(k_sm);
        for (int t = 0; t < n_tiles; ++t) {
            const int slot = t % kSlots;
            if (!mbar_wait(&kv_empty[slot], ((uint32_t)(t / kSlots) & 1u) ^ 1u)) ok = false;
            if (!ok) break;
            const uint32_t dst0 = k_base + (uint32_t)slot * kKSlot;
            // chunk c: local box c / 512, row (c / 8) % 64, 16-byte chunk c % 8
            // of that box row, so a warp covers 4 whole 128-byte box rows
#pragma unroll 4
            for (int c = gt; c < kTileN * kGBoxes * 8; c += kGatherThreads) {
                const int lb = c >> 9;
                const int r = (c >> 3) & (kTileN - 1);
                const int cb = c & 7;
                const int s = sel[t * kTileN + r];
                const uint32_t dst = dst0 + (uint32_t)lb * kKBox + (uint32_t)r * 128 + ((uint32_t)(cb ^ (r & 7)) << 4);
                cp_async16_zfill(dst, kvb + (int64_t)(s < 0 ? 0 : s) * a.ss + lb * 64 + cb * 8, s >= 0);
            }
            cp_async_arrive_noinc(&kv_full[slot]);
        }
        cp_async_wait_all();
    } else {
        // ------------------------------------------------------------ softmax
        const int quarter = warp & 3;                        // TMEM lane quarter
        const int kh = warp >> 2;                            // key half of every tile
        const int h = quarter * 32 + lane;                   // head = TMEM lane
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t peer = (uint32_t)(part ^ 1);
        // this warp's 4 KB block of S_p in the send and receive buffers:
        // [key half][head][32 floats], the thread's row of 8 chunks rotated by h
        const uint32_t blk = (uint32_t)(kh * kHeads + quarter * 32) * 128;
        float4 *xs_row = reinterpret_cast<float4 *>(xs_sm + blk + lane * 128);
        const float4 *xr_row = reinterpret_cast<const float4 *>(xr_sm + blk + lane * 128);
        const uint32_t peer_xr_blk = cluster_smem_addr(xr_sm + blk, peer);
        const uint32_t peer_x_full = cluster_smem_addr(&x_full[warp], peer);
        const uint32_t peer_x_free = cluster_smem_addr(&x_free[warp], peer);
        if (n_tiles > 0) {
            // the part's Q columns of head h, staged by TMA (row h of each box,
            // 128-byte swizzle), into its TMEM lane as raw bf16 pairs; the two
            // warps of a lane quarter take alternate boxes
            if (!mbar_wait(q_full, 0)) ok = false;
            if (__all_sync(0xffffffffu, ok)) {
                for (int c = kh; c < q_boxes(part); c += 2) {  // warp-uniform trip count
                    const uint8_t *box = smem + kOffP + c * kQBox + h * 128;
                    uint32_t w[32];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 x = *reinterpret_cast<const uint4 *>(box + ((j ^ (h & 7)) << 4));
                        w[4 * j] = x.x; w[4 * j + 1] = x.y; w[4 * j + 2] = x.z; w[4 * j + 3] = x.w;
                    }
                    tmem_st_32x32b_x32(tmem + lane_addr + kColQ + (uint32_t)(c * 32), w);
                }
                tmem_st_wait();
            }
            fence_proxy_async_smem();  // the staging is overwritten by P and the S_p blocks next
            tc_fence_before();
            mbar_arrive(q_copied);
            // every warp has copied its boxes: P and the send buffer may be
            // written, and the other part may send into the receive buffer
            if (ok && !mbar_wait(q_copied, 0)) ok = false;
            if (lane == 0) mbar_arrive_remote(peer_x_free);
        }
        ok = __all_sync(0xffffffffu, ok);

        // S_p of tile t (this warp's 32 keys) out of TMEM into registers
        auto load_sp = [&](int t, uint32_t *v) -> bool {
            if (!mbar_spin(s_full, (uint32_t)t & 1u)) return false;
            tc_fence_after();
            tmem_ld_32x32b_x32(tmem + lane_addr + kColS + (uint32_t)(kh * 32), v);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(s_free);  // the next QK^T may overwrite S_p
            return true;
        };
        // this warp's block of S_p of tile t to the same warp of the other
        // part, once that warp may be sent block t (x_free phase t); the block
        // stays in the send buffer, where this warp reads it back
        auto send_sp = [&](int t, const uint32_t *v) -> bool {
            if (!mbar_spin_cluster(&x_free[warp], (uint32_t)t & 1u)) return false;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                xs_row[(c + lane) & 7] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                                                     __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
            fence_proxy_async_smem();  // read by the bulk copy
            __syncwarp();
            if (lane == 0) bulk_copy_to_cluster(peer_xr_blk, xs_sm + blk, kXWarpBytes, peer_x_full);
            ++sent;
            return true;
        };

        uint32_t x[32];
        if (ok && n_tiles > 0) {
            if (!load_sp(0, x) || !send_sp(0, x)) ok = false;
            ok = __all_sync(0xffffffffu, ok);
        }
        for (int t = 0; ok && t < n_tiles; ++t) {
            // the other part's block of S_p for tile t: S = S_0 + S_1
            if (!mbar_spin_cluster(&x_full[warp], (uint32_t)t & 1u)) ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 u = xs_row[(c + lane) & 7];
                const float4 v = xr_row[(c + lane) & 7];
                x[4 * c] = __float_as_uint(u.x + v.x);
                x[4 * c + 1] = __float_as_uint(u.y + v.y);
                x[4 * c + 2] = __float_as_uint(u.z + v.z);
                x[4 * c + 3] = __float_as_uint(u.w + v.w);
            }
            ++recv;
            __syncwarp();  // every lane has read both blocks
            if (lane == 0 && t + 1 < n_tiles) {
                mbar_arrive_expect_tx(&x_full[warp], kXWarpBytes);  // armed for the next block
                mbar_arrive_remote(peer_x_free);                    // the other part may send it
            }
            // the next tile's S_p goes out now, so that its swap runs under
            // this tile's softmax
            if (t + 1 < n_tiles) {
                uint32_t y[32];
                if (!load_sp(t + 1, y) || !send_sp(t + 1, y)) ok = false;
                if (!__all_sync(0xffffffffu, ok)) break;
            }

            // scale, mask entries that are padding, this half's max
            const unsigned vm = __ballot_sync(0xffffffffu, sel[t * kTileN + kh * 32 + lane] >= 0);
            float mt = -INFINITY;
            if (vm == 0xffffffffu) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float z = __uint_as_float(x[j]) * a.scale_log2;
                    x[j] = __float_as_uint(z);
                    mt = fmaxf(mt, z);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float z = ((vm >> j) & 1u) ? __uint_as_float(x[j]) * a.scale_log2 : -INFINITY;
                    x[j] = __float_as_uint(z);
                    mt = fmaxf(mt, z);
                }
            }
            // the row max over both key halves: each warp of the lane quarter
            // posts its half's max (double-buffered by tile) and waits for the
            // other's on a bounded barrier
            mx_sm[((t & 1) * 2 + kh) * kHeads + h] = mt;
            mbar_arrive(&mx_bar[quarter]);
            if (!mbar_spin(&mx_bar[quarter], (uint32_t)t & 1u)) ok = false;
            // P buffer t % 2 was last read by PV of tile t - 2
            if (t >= 2 && ok && !mbar_wait(&pv_done[t & 1], (uint32_t)((t - 2) >> 1) & 1u)) ok = false;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            mt = fmaxf(mt, mx_sm[((t & 1) * 2 + (kh ^ 1)) * kHeads + h]);
            float m_new = m_ref;
            bool grow = false;
            if (mt > -INFINITY) {
                if (m_ref == -INFINITY) {
                    m_new = mt;  // O holds only zero contributions so far
                } else if (mt > m_ref + kRescaleLog2) {
                    m_new = mt;
                    grow = true;
                }
            }
            if (__any_sync(0xffffffffu, grow)) {  // tcgen05.ld/st are warp-wide
                // O may be rescaled once every PV so far (through tile t - 1) is done
                if (!mbar_wait(&pv_done[(t - 1) & 1], (uint32_t)((t - 1) >> 1) & 1u)) ok = false;
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const float f = grow ? exp2f(m_ref - m_new) : 1.0f;
#pragma unroll 1
                for (int c = kh * (kHalfDv / 2); c < (kh + 1) * (kHalfDv / 2); c += 32) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tmem + lane_addr + kColO + (uint32_t)c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                    tmem_st_32x32b_x32(tmem + lane_addr + kColO + (uint32_t)c, o);
                }
                tmem_st_wait();
                l *= f;
            }
            m_ref = m_new;
            // p = 2^(z - m_ref); masked keys have z = -inf, so p = 0 (also when
            // no key of the row is valid yet: then every z is -inf)
            const float mr = m_ref == -INFINITY ? 0.0f : m_ref;
            uint32_t pk[16];
            float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = ex2_approx(__uint_as_float(x[2 * j]) - mr);
                const float p1 = ex2_approx(__uint_as_float(x[2 * j + 1]) - mr);
                ps0 += p0;
                ps1 += p1;
                pk[j] = pack_bf16x2(p0, p1);
            }
            l += ps0 + ps1;
            // P row h of buffer t % 2: 128 bytes, 16-byte chunk c at chunk
            // c ^ (h % 8); this warp's keys are chunks 4 kh .. 4 kh + 3
            uint8_t *prow = p_sm + (t & 1) * kPBytes + h * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4 *>(prow + (((4 * kh + c) ^ (h & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();  // P is read by the tensor core
            tc_fence_before();
            mbar_arrive(&p_full[t & 1]);
        }
        if (ok && n_tiles > 0 &&
            !mbar_wait(&pv_done[(n_tiles - 1) & 1], (uint32_t)((n_tiles - 1) >> 1) & 1u))
            ok = false;
        ok = __all_sync(0xffffffffu, ok);
        l_sm[kh * kHeads + h] = l;
    }

    // ---------------------------------------------------------------- teardown
    // Every S_p block sent to this CTA must have landed before it exits: each
    // softmax warp tells the same warp of the other part how many blocks it
    // sent, and after a cluster barrier a warp that received fewer waits for
    // the one outstanding block (a warp sends block t + 1 only after the
    // other part has read block t, so at most one can be in flight). The
    // barrier is split around the output stores.
    if (warp < kSoftWarps && lane == 0)
        st_cluster_u32(cluster_smem_addr(&cnt_sm[warp], (uint32_t)(part ^ 1)), sent);
    tc_fence_before();
    const bool cta_ok = __syncthreads_and(ok ? 1 : 0) != 0;
    tc_fence_after();
    cluster_arrive();

    // ---------------------------------------------------------------- outputs
    // Every role is done here: MMAs drained, copies landed, O final in TMEM,
    // so the ring and P may be reused as the output staging.
    if (threadIdx.x < kSoftmaxThreads && cta_ok) {
        const int quarter = warp & 3, kh = warp >> 2;
        const int h = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const size_t pair = (size_t)row * kHeads + h;
        const bool have_o = n_tiles > 0;
        const float l_all = l_sm[h] + l_sm[kHeads + h];
        const float inv = l_all > 0.0f ? 1.0f / l_all : 0.0f;
        // this thread: value columns [128 kh, 128 kh + 128) of the part's 256
        uint4 *stage = reinterpret_cast<uint4 *>(smem + h * kHalfRowBytes);
#pragma unroll 1
        for (int c = 0; c < kHalfDv / 2; c += 64) {  // two loads per wait
            uint32_t o[64];
            const uint32_t col = (uint32_t)(kh * (kHalfDv / 2) + c);
            if (have_o) {
                tmem_ld_32x32b_x32(tmem + lane_addr + kColO + col, o);
                tmem_ld_32x32b_x32(tmem + lane_addr + kColO + col + 32, o + 32);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) o[j] = 0u;
            }
            uint4 w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                w[q] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
            const int q0 = (int)col / 8;  // first 16-byte chunk of these 64 columns in the half row
            if (a.splits == 1) {
                uint4 *dst = reinterpret_cast<uint4 *>(a.out + pair * DV + part * kHalfDv) + q0;
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = w[q];
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) stage[rot_chunk(h, q0 + q)] = w[q];
            }
        }
        if (a.splits == 1) {
            if (part == 0 && kh == 0 && a.lse != nullptr)
                a.lse[pair] = l_all > 0.0f ? (m_ref + log2f(l_all)) / kLog2e : -INFINITY;
        } else {
            if (part == 0 && kh == 0) {
                a.part_ml[(pair * a.splits + split) * 2 + 0] = m_ref;
                a.part_ml[(pair * a.splits + split) * 2 + 1] = l_all;
            }
            // this part's partials of all 128 heads, normalised by their own
            // sums, are one contiguous 64 KB block: one bulk copy once every
            // softmax thread has staged its columns (a bulk copy costs about
            // the same per operation up to several KB, so one large copy
            // instead of one per head; every softmax thread gets here, since
            // cta_ok is the same for the whole CTA)
            fence_proxy_async_smem();
            asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
            if (threadIdx.x == 0) {
                bulk_store(a.part_o + (((size_t)row * a.splits + split) * 2 + part) * (kHeads * kHalfRowBytes / 16),
                           smem, kHeads * kHalfRowBytes);
                bulk_commit();
                bulk_wait_read();  // the staging must outlive the copy's reads
            }
        }
    }

    cluster_wait();
    if (warp < kSoftWarps && lane == 0 && cnt_sm[warp] > recv) {
        if (!mbar_drain_cluster(&x_full[warp], recv & 1u)) ok = false;
    }
    if (!ok) atomicOr(&g_attn_mla_tc_error, kErrTimeout);
    tc_fence_before();
    cg::this_cluster().sync();  // no part leaves while the other may still read or write its memory
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge the split partials of one (row, head): two warps per pair, one per
// part's half row. Lane j of each warp holds the (max, sum) of split j; every
// lane owns 8 output columns (one 16-byte chunk of bf16) and loads every
// split's chunk for them independently (all in flight at once), undoing the
// rotation of the half rows. Each split's partial is normalised by its own
// sum l_s, so it is weighted by l_s 2^(m_s - max).
__global__ void attn_mla_combine_kernel(const uint4 *__restrict__ part_o, const float *__restrict__ part_ml,
                                        int n_pairs, int splits, __nv_bfloat16 *__restrict__ out,
                                        float *__restrict__ lse) {
    const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int pair = gw >> 1, half = gw & 1;
    const int lane = threadIdx.x & 31;
    if (pair >= n_pairs) return;
    const int h = pair % kHeads;
    const float *ml = part_ml + (size_t)pair * splits * 2;
    const float m_s = lane < splits ? ml[2 * lane] : -INFINITY;
    const float l_s = lane < splits ? ml[2 * lane + 1] : 0.0f;
    const float m_all = warp_max(m_s);
    const float f_s = (m_all == -INFINITY || lane >= splits) ? 0.0f : l_s * ex2_approx(m_s - m_all);
    const float l_all = warp_sum(f_s);
    const float inv = l_all > 0.0f ? 1.0f / l_all : 0.0f;
    const int row = pair / kHeads;
    // chunk rot_chunk(h, lane) of head h's half row `half` in split sp:
    // part_o[row][sp][half][h][32 chunks]
    const uint4 *po = part_o + (((size_t)row * splits) * 2 + half) * (kHeads * 32) + h * 32 + rot_chunk(h, lane);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll 8
    for (int sp = 0; sp < splits; ++sp) {
        const float f = __shfl_sync(0xffffffffu, f_s, sp);
        float e8[8];
        bf16x8_to_f32(po[(size_t)sp * 2 * (kHeads * 32)], e8);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(f, e8[e], acc[e]);
    }
    uint4 w;
    w.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    w.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    w.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    w.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    reinterpret_cast<uint4 *>(out + (size_t)pair * DV + half * kHalfDv)[lane] = w;
    if (lse != nullptr && half == 0 && lane == 0)
        lse[pair] = l_all > 0.0f ? (m_all + log2f(l_all)) / kLog2e : -INFINITY;
}

// Splits per row: one CTA per SM over (row, split, part), at most kMaxTiles
// tiles per split, at most kMaxSplits splits (one per combine lane), and no
// more splits than the longest one needs.
int mla_tc_splits(const AttnProblem &p, int sm_count) {
    const long long rows = (long long)p.B * p.Tq;
    const int tiles = (p.k + kTileN - 1) / kTileN;
    const int min_splits = (tiles + kMaxTiles - 1) / kMaxTiles;
    long long s = sm_count / (2 * rows);
    if (s < min_splits) s = min_splits;
    if (s > tiles) s = tiles;
    if (s > kMaxSplits) s = kMaxSplits;
    if (s < 1) s = 1;
    // as few splits as give the same longest split (whole tiles each): the
    // same time, fewer partials to write and combine
    const long long per = (tiles + s - 1) / s;
    s = (tiles + per - 1) / per;
    return (int)s;
}

}  // namespace

cudaError_t attn_mla_tc_set_wait_limit(unsigned long long ns) { return set_wait_limit_ns(ns); }

unsigned int attn_mla_tc_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_mla_tc_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_mla_tc_error, &zero, sizeof(zero));
    return v;
}

bool attn_mla_tc_supported(const AttnProblem &p) {
    if (p.dt != DSA_BF16 || p.Dqk != DQK || p.Dv != DV || p.Hq != kHeads || p.Hkv != 1) return false;
    // the value must be the first DV columns of the same latent row
    if (p.v_cache != p.k_cache || p.v_sb != p.k_sb || p.v_ss != p.k_ss) return false;
    if (((uintptr_t)p.k_cache | (uintptr_t)p.q | (uintptr_t)p.out) % 16 != 0) return false;
    if (p.k_ss % 8 != 0 || p.k_sb % 8 != 0 || p.k_ss < DQK) return false;
    if (p.k < 1 || p.k > kMaxSplits * kMaxSel) return false;
    DeviceInfo info;
    if (device_info(&info) != cudaSuccess) return false;
    return info.cc_major == 10 && (size_t)info.max_smem_optin >= kSmem;
}

// Split partials: bf16 [rows, splits, 2 parts, 128 heads, 256], each head's
// half row with its 16-byte chunks rotated by the head and normalised by the
// split's own sum; then fp32 (max in log2 units, sum) [rows, 128, splits, 2].
size_t attn_mla_tc_workspace_bytes(const AttnProblem &p, int sm_count) {
    const int splits = mla_tc_splits(p, sm_count);
    if (splits <= 1) return 0;
    return (size_t)p.B * p.Tq * kHeads * splits * ((size_t)DV * 2 + 2 * sizeof(float));
}

cudaError_t launch_attn_mla_tc(const AttnProblem &p, const DeviceInfo &info, cudaStream_t stream) {
    const int splits = mla_tc_splits(p, info.sm_count);
    const long long rows = (long long)p.B * p.Tq;
    if (rows > 0x7fffffffLL || rows * kHeads > 0x7fffffffLL) return cudaErrorInvalidValue;
    CUtensorMap tm_q;
    if (!make_map_bf16_sw128(&tm_q, p.q, (uint64_t)rows * kHeads, DQK, (uint64_t)DQK * 2, kHeads))
        return cudaErrorInvalidValue;
    Args a;
    a.kv = static_cast<const __nv_bfloat16 *>(p.k_cache);
    a.idx = p.idx;
    a.Tq = p.Tq; a.L = p.L; a.k = p.k;
    a.splits = splits;
    a.tiles = (p.k + kTileN - 1) / kTileN;
    a.scale_log2 = p.scale * kLog2e;
    a.sb = p.k_sb; a.ss = p.k_ss;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.lse = p.lse;
    const size_t n_pairs = (size_t)rows * kHeads;
    a.part_o = splits > 1 ? static_cast<uint4 *>(p.ws) : nullptr;
    a.part_ml = splits > 1 ? reinterpret_cast<float *>(static_cast<char *>(p.ws) + n_pairs * splits * DV * 2)
                           : nullptr;
    cudaError_t err = cudaFuncSetAttribute(attn_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows, splits, 2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;  // the two column parts of a (row, split)
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 2;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, attn_mla_tc_kernel, tm_q, a);
    count_launch();
    if (err != cudaSuccess) return err;
    if (splits > 1) {
        const int warps_per_block = 8;  // two warps per (row, head) pair
        const int blocks = (int)((2 * n_pairs + warps_per_block - 1) / warps_per_block);
        attn_mla_combine_kernel<<<blocks, warps_per_block * 32, 0, stream>>>(a.part_o, a.part_ml, (int)n_pairs,
                                                                            splits, a.out, a.lse);
        count_launch();
        err = cudaGetLastError();
    }
    return err;
}

}  // namespace dsa
