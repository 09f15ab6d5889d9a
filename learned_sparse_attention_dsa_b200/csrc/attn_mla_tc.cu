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
// ring of gathered boxes (3 x 40 KB), P (16 KB), the partial-S send and
// receive buffers (2 x 32 KB). A partial S crosses to the other part as one
// 32 KB bulk copy between the CTAs' shared memories.
//
// Per CTA (one per SM):
//   warps 0-3  softmax, one head per thread: the Q part into TMEM (staged by
//              TMA, then tcgen05.st); per tile tcgen05.ld of S_p (released at
//              once, so the next QK^T overlaps), S_p to the other part, S =
//              S_0 + S_1, online softmax in fp32 against a reference max that
//              moves only when the row max grows by more than 2^8 (then O is
//              rescaled in TMEM), P in bf16 to shared memory (128-byte
//              swizzle); at the end O leaves TMEM for the output or the split
//              partials (one bulk copy per head row).
//   warps 4-6  gather the 5 boxes of 64 selected rows per tile with 16-byte
//              cp.async (one warp instruction fills 4 rows x 128 bytes).
//   warp 7     one thread moves S_p: bulk copy of the send buffer into the
//              other part's receive buffer, then re-arms this part's receive
//              barrier and frees the other part's sends.
//   warp 8     TMEM allocation, the Q staging by TMA, and one thread issuing
//              the MMAs with descriptors built once.
// With several splits, attn_mla_combine_kernel merges the fp32 partials.
// Every mbarrier wait is bounded; on a timeout the CTA records an error word,
// drains its copies and MMAs, frees TMEM and returns.
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
constexpr uint32_t kQBox = kHeads * 128;           // 16,384
constexpr uint32_t kKBox = kTileN * 128;           // 8,192
constexpr uint32_t kKSlot = kGBoxes * kKBox;       // 40,960
constexpr uint32_t kPBytes = kHeads * kTileN * 2;  // 16,384
constexpr uint32_t kXBytes = kHeads * kTileN * 4;  // 32,768: one partial S tile
constexpr uint32_t kOffP = kSlots * kKSlot;
constexpr uint32_t kOffXs = kOffP + kPBytes;       // this part's S_p, sent to the other part
constexpr uint32_t kOffXr = kOffXs + kXBytes;      // the other part's S_p, received
constexpr uint32_t kOffSel = kOffXr + kXBytes;
constexpr uint32_t kOffBar = kOffSel + kMaxSel * 4;
constexpr uint32_t kStageBytes = kHeads * kHalfDv * 4;  // O staging for the partials
constexpr int kNumBars = 18;
constexpr size_t kSmem = 1024 + kOffBar + kNumBars * 8 + 16;  // + slack to align the base to 1024
constexpr int kSoftmaxThreads = 128;
constexpr int kGatherThreads = 96;
constexpr int kXchgWarp = (kSoftmaxThreads + kGatherThreads) / 32;  // 7
constexpr int kMmaWarp = kXchgWarp + 1;                              // 8
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;
constexpr uint32_t kColS = 160;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kIdescMnMajorB = 1u << 16;

static_assert(kOffP % 1024 == 0 && kKSlot % 1024 == 0, "operand tiles must sit on 1024-byte boundaries");
static_assert(5 * kQBox <= 2 * kKSlot, "the Q staging must fit over ring slots 0 and 1");
static_assert(kStageBytes <= kOffXs, "the O staging must fit over the ring and P");
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
    float *part_o, *part_ml;  // split partials (splits > 1)
};


__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Where float4 q (0..63) of head h's half row sits in the O staging and in
// the partials: rotated by h, so that a warp's 32 rows spread over the
// shared-memory banks. The combine kernel undoes the rotation.
__host__ __device__ __forceinline__ int rot_q(int h, int q) { return (q + h) & (kHalfDv / 4 - 1); }

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
    float4 *xs_sm = reinterpret_cast<float4 *>(smem + kOffXs);
    float4 *xr_sm = reinterpret_cast<float4 *>(smem + kOffXr);
    int32_t *sel = reinterpret_cast<int32_t *>(smem + kOffSel);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *q_full = bars;            // TMA bytes of the staged Q part
    uint64_t *q_copied = bars + 1;      // 128 softmax threads: Q part in TMEM, staging free
    uint64_t *kv_full = bars + 2;       // [3] 128 gather threads (cp.async arrivals)
    uint64_t *kv_empty = bars + 5;      // [3] MMA commit after PV
    uint64_t *s_full = bars + 8;        // MMA commit after QK^T
    uint64_t *s_free = bars + 9;        // 128 softmax threads (S_p is in registers)
    uint64_t *p_full = bars + 10;       // 128 softmax threads
    uint64_t *pv_done = bars + 11;      // MMA commit after PV
    uint64_t *drained = bars + 12;      // MMA commit before teardown
    uint64_t *x_full = bars + 13;       // bytes of the other part's S_p in xr_sm (armed per tile)
    uint64_t *x_free = bars + 14;       // the other part has read what we sent
    uint64_t *xs_full = bars + 15;      // 128 softmax threads: send buffer written
    uint64_t *xr_done = bars + 16;      // 128 softmax threads: receive buffer read
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
        mbar_init(p_full, kSoftmaxThreads);
        mbar_init(pv_done, 1);
        mbar_init(drained, 1);
        mbar_init(x_full, 1);
        mbar_init(x_free, 1);
        mbar_init(xs_full, kSoftmaxThreads);
        mbar_init(xr_done, kSoftmaxThreads);
        fence_barrier_init();
        mbar_arrive_expect_tx(x_full, kXBytes);  // armed for the first tile
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    cg::this_cluster().sync();  // both parts' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    float m_ref = -INFINITY, l = 0.0f;  // softmax threads: reference max (log2 units) and sum

    // Tile t lands in ring slot (t + 2) % 3 (its (t / 3)-th use): slots 0-1
    // first hold the Q staging, so tiles 1 and 2 wait for the copy to TMEM.
    if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            prefetch_tensor_map(&tm_q);
            mbar_arrive_expect_tx(q_full, (uint32_t)q_boxes(part) * kQBox);
#pragma unroll 1
            for (int c = 0; c < q_boxes(part); ++c)
                tma_load_2d(smem + c * kQBox, &tm_q, q_full, (q_box0(part) + c) * 64, row * kHeads);
            ok = mbar_wait(q_copied, 0);
            tc_fence_after();
            const uint32_t idesc_qk = idesc_bf16_f32(kHeads, kTileN);
            const uint32_t idesc_pv = idesc_bf16_f32(kHeads, kHalfDv) | kIdescMnMajorB;
            const uint64_t p_desc = smem_desc_k_sw128(smem_addr(p_sm));
            // QK^T reads local boxes [q_box0 - g_box0, +q_boxes); PV local boxes 0-3
            const uint64_t k_desc0 =
                smem_desc_k_sw128(smem_addr(k_sm) + (uint32_t)(q_box0(part) - g_box0(part)) * kKBox);
            const uint64_t v_desc0 = smem_desc_mn_sw128(smem_addr(k_sm), kKBox);
            auto issue_pv = [&](int u) -> bool {
                if (!mbar_wait(p_full, (uint32_t)(u & 1))) return false;
                tc_fence_after();
                const int slot = (u + 2) % kSlots;
                const uint64_t vd = v_desc0 + desc_step((uint32_t)slot * kKSlot);
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk)  // 16 keys = two 8-row groups = 2048 bytes
                    mma_f16_ss(tmem + kColO, p_desc + desc_step(kk * 32), vd + desc_step(kk * 2048), idesc_pv,
                               (u > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&kv_empty[slot]);  // the slot may be refilled
                mma_commit(pv_done);          // P may be rewritten, O is current
                return true;
            };
            for (int t = 0; ok && t < n_tiles; ++t) {
                const int slot = (t + 2) % kSlots;
                if (!mbar_wait(&kv_full[slot], (uint32_t)(t / kSlots) & 1u) ||
                    !mbar_wait(s_free, ((uint32_t)t & 1u) ^ 1u)) {
                    ok = false;
                    break;
                }
                fence_proxy_async_smem();  // the rows were written by cp.async
                tc_fence_after();
                const uint64_t kd = k_desc0 + desc_step((uint32_t)slot * kKSlot);
                if (part == 0)
                    issue_qk<5>(tmem + kColS, tmem + kColQ, kd, idesc_qk);
                else
                    issue_qk<4>(tmem + kColS, tmem + kColQ, kd, idesc_qk);
                mma_commit(s_full);
                if (t > 0 && !issue_pv(t - 1)) ok = false;
            }
            if (ok) ok = issue_pv(n_tiles - 1);
            // nothing of this CTA may still run on the tensor core at teardown
            mma_commit(drained);
            if (!mbar_wait(drained, 0)) ok = false;
        }
    } else if (warp == kXchgWarp) {
        // ------------------------------------------------------------ S_p exchange
        if (lane == 0) {
            const uint32_t peer = (uint32_t)(part ^ 1);
            const uint32_t peer_xr = cluster_smem_addr(xr_sm, peer);
            const uint32_t peer_x_full = cluster_smem_addr(x_full, peer);
            const uint32_t peer_x_free = cluster_smem_addr(x_free, peer);
            for (int t = 0; t < n_tiles; ++t) {
                // the softmax threads have written S_p (after the other part
                // had read the previous one)
                if (!mbar_wait(xs_full, (uint32_t)t & 1u)) { ok = false; break; }
                bulk_copy_to_cluster(peer_xr, xs_sm, kXBytes, peer_x_full);
                // they have read the other part's S_p: re-arm, let it send again
                if (!mbar_wait(xr_done, (uint32_t)t & 1u)) { ok = false; break; }
                if (t + 1 < n_tiles) mbar_arrive_expect_tx(x_full, kXBytes);
                mbar_arrive_remote(peer_x_free);
            }
        }
    } else if (warp >= kSoftmaxThreads / 32) {
        // ------------------------------------------------------------ gather
        const int gt = threadIdx.x - kSoftmaxThreads;
        const __nv_bfloat16 *kvb = a.kv + (int64_t)b * a.sb + g_box0(part) * 64;
        const uint32_t k_base = smem_addr(k_sm);
        for (int t = 0; t < n_tiles; ++t) {
            const int slot = (t + 2) % kSlots;
            if ((t == 1 || t == 2) && !mbar_wait(q_copied, 0)) ok = false;
            if (ok && !mbar_wait(&kv_empty[slot], ((uint32_t)(t / kSlots) & 1u) ^ 1u)) ok = false;
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
        const int h = warp * 32 + lane;                      // head = TMEM lane
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        if (n_tiles > 0) {
            // the part's Q columns of head h, staged by TMA (row h of each box,
            // 128-byte swizzle), into its TMEM lane as raw bf16 pairs
            if (!mbar_wait(q_full, 0)) ok = false;
            if (__all_sync(0xffffffffu, ok)) {
                for (int c = 0; c < q_boxes(part); ++c) {  // warp-uniform trip count
                    const uint8_t *box = smem + c * kQBox + h * 128;
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
            fence_proxy_async_smem();  // the staging is overwritten by the gathers next
            tc_fence_before();
            mbar_arrive(q_copied);
        }
        for (int t = 0; ok && t < n_tiles; ++t) {
            if (!mbar_wait(s_full, (uint32_t)t & 1u)) ok = false;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t x[64];
            tmem_ld_32x32b_x32(tmem + lane_addr + kColS, x);
            tmem_ld_32x32b_x32(tmem + lane_addr + kColS + 32, x + 32);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(s_free);  // the next QK^T may overwrite S_p

            // S_p to the other part: row h of the send buffer (16-byte chunks
            // rotated by h), then one bulk copy into its receive buffer. The
            // send buffer is free again once the other part has read the
            // previous tile (every wait here is bounded).
            if (t > 0 && !mbar_wait_cluster(x_free, (uint32_t)(t - 1) & 1u)) ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
            float4 *xsr = xs_sm + h * (kTileN / 4);
#pragma unroll
            for (int c = 0; c < kTileN / 4; ++c)
                xsr[(c + h) & (kTileN / 4 - 1)] =
                    make_float4(__uint_as_float(x[4 * c]), __uint_as_float(x[4 * c + 1]),
                                __uint_as_float(x[4 * c + 2]), __uint_as_float(x[4 * c + 3]));
            fence_proxy_async_smem();  // read by the bulk copy
            mbar_arrive(xs_full);
            if (!mbar_wait_cluster(x_full, (uint32_t)t & 1u)) ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
            // S = S_0 + S_1 (the same sum on both parts)
            const float4 *xr = xr_sm + h * (kTileN / 4);
#pragma unroll
            for (int c = 0; c < kTileN / 4; ++c) {
                const float4 v = xr[(c + h) & (kTileN / 4 - 1)];
                x[4 * c] = __float_as_uint(__uint_as_float(x[4 * c]) + v.x);
                x[4 * c + 1] = __float_as_uint(__uint_as_float(x[4 * c + 1]) + v.y);
                x[4 * c + 2] = __float_as_uint(__uint_as_float(x[4 * c + 2]) + v.z);
                x[4 * c + 3] = __float_as_uint(__uint_as_float(x[4 * c + 3]) + v.w);
            }
            mbar_arrive(xr_done);

            const unsigned vm0 = __ballot_sync(0xffffffffu, sel[t * kTileN + lane] >= 0);
            const unsigned vm1 = __ballot_sync(0xffffffffu, sel[t * kTileN + 32 + lane] >= 0);
            float mt = -INFINITY;
            if ((vm0 & vm1) == 0xffffffffu) {  // every entry of the tile is a valid position
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const float z = __uint_as_float(x[j]) * a.scale_log2;
                    x[j] = __float_as_uint(z);
                    mt = fmaxf(mt, z);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const bool valid = ((j < 32 ? vm0 >> j : vm1 >> (j - 32)) & 1u) != 0;
                    const float z = valid ? __uint_as_float(x[j]) * a.scale_log2 : -INFINITY;
                    x[j] = __float_as_uint(z);
                    mt = fmaxf(mt, z);
                }
            }
            // PV of the previous tile must be done before P is rewritten or O rescaled
            if (t > 0 && !mbar_wait(pv_done, (uint32_t)(t - 1) & 1u)) ok = false;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
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
                const float f = grow ? exp2f(m_ref - m_new) : 1.0f;
#pragma unroll 1
                for (int c = 0; c < kHalfDv; c += 32) {
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
            uint32_t pk[32];
            float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float p0 = ex2_approx(__uint_as_float(x[2 * j]) - mr);
                const float p1 = ex2_approx(__uint_as_float(x[2 * j + 1]) - mr);
                ps0 += p0;
                ps1 += p1;
                pk[j] = pack_bf16x2(p0, p1);
            }
            l += ps0 + ps1;
            // P row h: 128 bytes, 16-byte chunk c at chunk c ^ (h % 8)
            uint8_t *prow = p_sm + h * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(prow + ((c ^ (h & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();  // P is read by the tensor core
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok && n_tiles > 0 && !mbar_wait(pv_done, (uint32_t)(n_tiles - 1) & 1u)) ok = false;
        ok = __all_sync(0xffffffffu, ok);
    }

    // ---------------------------------------------------------------- outputs
    // Every role is done here: MMAs drained, copies landed, O final in TMEM,
    // so the ring and P may be reused as the O staging.
    tc_fence_before();
    const bool cta_ok = __syncthreads_and(ok ? 1 : 0) != 0;
    tc_fence_after();
    if (threadIdx.x < kSoftmaxThreads && cta_ok) {
        const int h = threadIdx.x;
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const size_t pair = (size_t)row * kHeads + h;
        const bool have_o = n_tiles > 0;
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;
        float4 *stage = reinterpret_cast<float4 *>(smem + h * (kHalfDv * 4));
#pragma unroll 1
        for (int c = 0; c < kHalfDv; c += 64) {  // two loads per wait
            uint32_t o[64];
            if (have_o) {
                tmem_ld_32x32b_x32(tmem + lane_addr + kColO + (uint32_t)c, o);
                tmem_ld_32x32b_x32(tmem + lane_addr + kColO + (uint32_t)(c + 32), o + 32);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) o[j] = 0u;
            }
            if (a.splits == 1) {
                uint4 *dst = reinterpret_cast<uint4 *>(a.out + pair * DV + part * kHalfDv + c);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(o[8 * q + 2 * e]) * inv,
                                           __uint_as_float(o[8 * q + 2 * e + 1]) * inv);
                    dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
#pragma unroll
                for (int v = 0; v < 16; ++v)
                    stage[rot_q(h, c / 4 + v)] =
                        make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                    __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
            }
        }
        if (a.splits == 1) {
            if (part == 0 && a.lse != nullptr) a.lse[pair] = l > 0.0f ? (m_ref + log2f(l)) / kLog2e : -INFINITY;
        } else {
            // one bulk copy of this head's (rotated) half row of partials
            fence_proxy_async_smem();
            bulk_store(a.part_o + (pair * a.splits + split) * DV + part * kHalfDv, stage, kHalfDv * 4);
            bulk_commit();
            if (part == 0) {
                a.part_ml[(pair * a.splits + split) * 2 + 0] = m_ref;
                a.part_ml[(pair * a.splits + split) * 2 + 1] = l;
            }
            bulk_wait_read();  // the staging must outlive the copy's reads
        }
    }

    if (!ok) atomicOr(&g_attn_mla_tc_error, kErrTimeout);
    tc_fence_before();
    cg::this_cluster().sync();  // no part leaves while the other may still write to it
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge the split partials of one (row, head): lane j of each warp holds the
// (max, sum) of split j; the pair's 128 output float4s are spread over four
// warps, and every lane sums the splits' partials for its float4, undoing the
// rotation of the half rows.
__global__ void attn_mla_combine_kernel(const float4 *__restrict__ part_o, const float *__restrict__ part_ml,
                                        int n_pairs, int splits, __nv_bfloat16 *__restrict__ out,
                                        float *__restrict__ lse) {
    // four warps per (row, head): warp quarter qt owns output float4s
    // [32 qt, 32 qt + 32), one per lane, and loads every split's value for it
    // independently (all in flight at once)
    const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int pair = gw >> 2, qt = gw & 3;
    const int lane = threadIdx.x & 31;
    if (pair >= n_pairs) return;
    const int h = pair % kHeads;
    const float *ml = part_ml + (size_t)pair * splits * 2;
    const float m_s = lane < splits ? ml[2 * lane] : -INFINITY;
    const float l_s = lane < splits ? ml[2 * lane + 1] : 0.0f;
    const float m_all = warp_max(m_s);
    const float f_s = (m_all == -INFINITY || lane >= splits) ? 0.0f : ex2_approx(m_s - m_all);
    const float l_all = warp_sum(f_s * l_s);
    const float inv = l_all > 0.0f ? 1.0f / l_all : 0.0f;
    const float4 *po = part_o + (size_t)pair * splits * (DV / 4);
    const int c4 = qt * 32 + lane;  // output float4 index in [0, 128)
    const int hf = c4 / (kHalfDv / 4), q = c4 % (kHalfDv / 4);
    const int pos = hf * (kHalfDv / 4) + rot_q(h, q);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int sp = 0; sp < splits; ++sp) {
        const float f = __shfl_sync(0xffffffffu, f_s, sp);
        const float4 v = po[(size_t)sp * (DV / 4) + pos];
        acc.x = fmaf(f, v.x, acc.x);
        acc.y = fmaf(f, v.y, acc.y);
        acc.z = fmaf(f, v.z, acc.z);
        acc.w = fmaf(f, v.w, acc.w);
    }
    uint2 w;
    w.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    w.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(out + (size_t)pair * DV + 4 * c4) = w;
    if (lse != nullptr && qt == 0 && lane == 0)
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

size_t attn_mla_tc_workspace_bytes(const AttnProblem &p, int sm_count) {
    const int splits = mla_tc_splits(p, sm_count);
    if (splits <= 1) return 0;
    return (size_t)p.B * p.Tq * kHeads * splits * ((size_t)DV + 2) * sizeof(float);
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
    a.part_o = splits > 1 ? static_cast<float *>(p.ws) : nullptr;
    a.part_ml = splits > 1 ? a.part_o + n_pairs * splits * DV : nullptr;
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
        const int warps_per_block = 8;  // four warps per (row, head) pair
        const int blocks = (int)((4 * n_pairs + warps_per_block - 1) / warps_per_block);
        attn_mla_combine_kernel<<<blocks, warps_per_block * 32, 0, stream>>>(
            reinterpret_cast<const float4 *>(a.part_o), a.part_ml, (int)n_pairs, splits, a.out, a.lse);
        count_launch();
        err = cudaGetLastError();
    }
    return err;
}

}  // namespace dsa
