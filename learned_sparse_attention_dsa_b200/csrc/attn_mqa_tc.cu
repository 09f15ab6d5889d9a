// Sparse attention for groups of query rows on the 5th-generation tensor
// cores: 16 query heads share one KV head of width Dqk in {128, 192} with
// values of width 128 (the MQA mode of MLA, prefill).
//
//   u[t,h] = sum_{s in S_t} softmax_s(scale * q[t,h] . k[s]) v[s]
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §3.3 and
// §10.1; one selected set per query row for all heads, §4.1-4.2).
//
// One CTA owns 8 consecutive query rows of one batch entry (heaviest groups,
// the latest rows, first): 8 rows x 16 heads = 128 = the MMA's M, row r of
// every tile being query r / 16, head r % 16 (one TMEM lane each). Each row's
// selected set is marked in a bitmap and the union of the 8 sets is listed in
// ascending position order, every entry holding the position (16 bits) and
// the mask of the rows that selected it. The K and V rows of every union
// position are gathered once for the group, 64 positions per tile:
//   S[r, j] = q[r] . k[s_j]                      M=128, N=64, K=Dqk (Q in TMEM)
//   a logit is -inf where position s_j is not in row r's own set, then the
//   online softmax of row r (one thread per row, a reference max that moves
//   only when the row max grows by more than 2^8, O then rescaled in TMEM)
//   O[r, :] += P[r, j] v[s_j]                    M=128, N=128, K=64
// so the copies of a position selected by several rows of the group are
// shared, and the tensor cores (not a 16-row mma.sync per row) take the
// 8-fold product.
//
// Per CTA (one per SM; shared memory: a three-slot ring of gathered rows,
// P twice, the union list):
//   warps 0-3   softmax, one thread per row (TMEM lane), the Q rows into TMEM
//               first (staged by TMA over the ring)
//   warps 4-13  gather the K and V boxes (64 columns, 128-byte swizzle) of 64
//               union positions per tile with 16-byte cp.async (the rate at
//               which cp.async is issued grows with the number of issuing
//               warps: ~2,450 cycles per 40 KB tile with eight)
//   warp 14     TMEM allocation, the Q staging by TMA, and one thread issuing
//               QK^T and PV as each becomes ready
// Every mbarrier wait is bounded; on a timeout the CTA records an error word,
// waits for the copies and MMAs it issued, frees TMEM and returns.
#include <math.h>

#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kRowsQ = 8;                    // query rows per CTA
constexpr int kHeads = 16;                   // query heads per KV head
constexpr int kM = kRowsQ * kHeads;          // 128: MMA M, TMEM lanes
constexpr int DV = 128;
constexpr int kTileN = 64;                   // union positions per tile
constexpr int kSlots = 3;
constexpr int kSoftThreads = kM;             // one per row
constexpr int kGatherThreads = 320;
constexpr int kMmaWarp = (kSoftThreads + kGatherThreads) / 32;  // 14
constexpr int kThreads = (kMmaWarp + 1) * 32;                   // 480
constexpr uint32_t kBox = kTileN * 128;      // 8 KB: 64 rows of 64 bf16 columns
constexpr uint32_t kQBox = kM * 128;         // 16 KB: 128 rows of 64 bf16 columns
constexpr uint32_t kPBytes = kM * kTileN * 2;
constexpr int kMaxUnion = 16384;             // union entries (min(L, 8 k), k <= 2048)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;                // Q: Dqk / 2 columns of bf16 pairs
constexpr uint32_t kColS = 128;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kIdescMnMajorB = 1u << 16;
constexpr int kNumBars = 15;

template <int DQK>
struct MqaCfg {
    static constexpr int kQBoxes = DQK / 64;             // 64-column boxes of Q and K
    static constexpr int kBoxes = kQBoxes + DV / 64;     // gathered per tile: K boxes, then V boxes
    static constexpr uint32_t kSlot = kBoxes * kBox;
    static constexpr uint32_t kRing = kSlots * kSlot;
    static constexpr uint32_t kOffP = kRing;
    static constexpr uint32_t kOffList = kOffP + 2 * kPBytes;
    static constexpr uint32_t kOffBar = kOffList + kMaxUnion * 4;
    static constexpr size_t kSmem = 1024 + kOffBar + kNumBars * 8 + 16;
    static_assert(kSmem <= 232448, "shared memory budget");
    static_assert(kQBoxes * kQBox <= kRing, "the Q staging must fit over the ring");
    static_assert(kSlot % 1024 == 0 && kOffP % 1024 == 0, "operand tiles on 1024-byte boundaries");
    static_assert(DQK / 2 <= kColS, "TMEM columns of Q");
};

__device__ unsigned int g_attn_mqa_tc_error = 0;  // kErrTimeout, kErrBadIndex bits

struct MqaArgs {
    const __nv_bfloat16 *k_cache, *v_cache;
    const int32_t *idx;  // [B * Tq, k]
    int B, Tq, L, k, ngroups, W;  // W: 32-bit bitmap words per row
    float scale_log2;
    int64_t k_sb, k_ss, v_sb, v_ss;
    __nv_bfloat16 *out;  // [B * Tq, 16, 128]
    float *lse;          // [B * Tq, 16] or null
};

__host__ __device__ constexpr uint64_t desc_step(uint32_t bytes) { return (uint64_t)(bytes >> 4); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int DQK>
__global__ void __launch_bounds__(kThreads, 1)
attn_mqa_group_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const MqaArgs a) {
    using C = MqaCfg<DQK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem;  // the bitmaps, then the Q staging, then the gathered tiles
    uint8_t *p_sm = smem + C::kOffP;
    uint32_t *ulist = reinterpret_cast<uint32_t *>(smem + C::kOffList);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *q_full = bars;           // TMA bytes of the Q staging
    uint64_t *q_copied = bars + 1;     // 128 softmax threads: Q in TMEM, the ring free
    uint64_t *kv_full = bars + 2;      // [3] gather threads (cp.async arrivals)
    uint64_t *kv_empty = bars + 5;     // [3] MMA commit after PV
    uint64_t *s_full = bars + 8;       // MMA commit after QK^T
    uint64_t *s_free = bars + 9;       // 128 softmax threads: S is in registers
    uint64_t *p_full = bars + 10;      // [2] 128 softmax threads: P buffer written
    uint64_t *pv_done = bars + 12;     // [2] MMA commit after PV from P buffer b
    uint64_t *drained = bars + 14;     // MMA commit before teardown
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
    __shared__ int warp_tot[kThreads / 32];
    __shared__ int s_count;

    const int b = blockIdx.x % a.B;
    const int gi = a.ngroups - 1 - (int)(blockIdx.x / a.B);
    const int i0 = gi * kRowsQ;
    const int qn = min(kRowsQ, a.Tq - i0);
    const size_t row0 = (size_t)b * a.Tq + i0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = a.W;

    // ---- the union of the rows' selected sets (bitmaps over the ring)
    uint32_t *bm = reinterpret_cast<uint32_t *>(ring);  // [kRowsQ][W]
    for (int w = threadIdx.x; w < kRowsQ * W; w += kThreads) bm[w] = 0u;
    __syncthreads();
    for (int q = 0; q < qn; ++q) {
        const int32_t *src = a.idx + (row0 + q) * a.k;
        for (int j = threadIdx.x; j < a.k; j += kThreads) {
            const int s = src[j];
            note_bad_index(&g_attn_mqa_tc_error, s, a.L);
            if (s >= 0 && s < a.L) atomicOr(&bm[q * W + (s >> 5)], 1u << (s & 31));
        }
    }
    __syncthreads();
    {
        // thread i owns words [i * per, (i + 1) * per): its union count, a
        // block-wide exclusive scan, then its entries in position order
        const int per = (W + kThreads - 1) / kThreads;
        const int w0 = min(W, (int)threadIdx.x * per), w1 = min(W, w0 + per);
        int cnt = 0;
        for (int w = w0; w < w1; ++w) {
            uint32_t u = 0u;
#pragma unroll
            for (int q = 0; q < kRowsQ; ++q) u |= bm[q * W + w];
            cnt += __popc(u);
        }
        const int incl = warp_inclusive_scan(cnt);
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int base = incl - cnt;
        for (int w = 0; w < warp; ++w) base += warp_tot[w];
        for (int w = w0; w < w1; ++w) {
            uint32_t wq[kRowsQ], u = 0u;
#pragma unroll
            for (int q = 0; q < kRowsQ; ++q) {
                wq[q] = bm[q * W + w];
                u |= wq[q];
            }
            while (u) {
                const int bit = __ffs(u) - 1;
                uint32_t mask = 0u;
#pragma unroll
                for (int q = 0; q < kRowsQ; ++q) mask |= ((wq[q] >> bit) & 1u) << q;
                ulist[base++] = (uint32_t)(w * 32 + bit) | (mask << 16);
                u &= u - 1u;
            }
        }
        if (threadIdx.x == kThreads - 1) s_count = base;
    }
    fence_proxy_async_smem();  // the ring is written next by TMA
    __syncthreads();
    const int n_sel = s_count;
    const int n_tiles = (n_sel + kTileN - 1) / kTileN;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_copied, kSoftThreads);
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&kv_full[i], kGatherThreads);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, kSoftThreads);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&p_full[i], kSoftThreads);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(drained, 1);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = waits_enabled();  // false: the wait limit is 0 (give-up test)

    // Tile t lands in ring slot t % 3 (its (t / 3)-th use), its P in buffer t % 2.
    if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0 && ok) {
            prefetch_tensor_map(&tm_q);
            mbar_arrive_expect_tx(q_full, (uint32_t)C::kQBoxes * kQBox);
#pragma unroll 1
            for (int c = 0; c < C::kQBoxes; ++c)
                tma_load_2d(ring + c * kQBox, &tm_q, q_full, c * 64, (int)(row0 * kHeads));
            ok = mbar_wait(q_copied, 0);
            tc_fence_after();
            const uint32_t idesc_qk = idesc_bf16_f32(kM, kTileN);
            const uint32_t idesc_pv = idesc_bf16_f32(kM, DV) | kIdescMnMajorB;
            const uint64_t p_desc0 = smem_desc_k_sw128(smem_addr(p_sm));
            const uint64_t k_desc0 = smem_desc_k_sw128(smem_addr(ring));
            const uint64_t v_desc0 = smem_desc_mn_sw128(smem_addr(ring) + (uint32_t)C::kQBoxes * kBox, kBox);
            // QK^T of the next tile (its rows landed, the previous S read out
            // of TMEM) and PV of the oldest tile whose P is written, each
            // issued as soon as its inputs are ready
            int nq = 0, np = 0;
            uint32_t idle = 0;
            uint64_t t_idle = 0;
            while (ok && np < n_tiles) {
                bool progress = false;
                if (nq < n_tiles && mbar_test_wait(&kv_full[nq % kSlots], (uint32_t)(nq / kSlots) & 1u) &&
                    mbar_test_wait(s_free, ((uint32_t)nq & 1u) ^ 1u)) {
                    fence_proxy_async_smem();  // the rows were written by cp.async
                    tc_fence_after();
                    const uint64_t kd = k_desc0 + desc_step((uint32_t)(nq % kSlots) * C::kSlot);
#pragma unroll
                    for (int kk = 0; kk < 4 * C::kQBoxes; ++kk)
                        mma_f16_ts(tmem + kColS, tmem + kColQ + (uint32_t)(kk * 8),
                                   kd + desc_step((uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32), idesc_qk,
                                   kk > 0 ? 1u : 0u);
                    mma_commit(s_full);
                    ++nq;
                    progress = true;
                }
                if (np < nq && mbar_test_wait(&p_full[np & 1], (uint32_t)(np >> 1) & 1u)) {
                    tc_fence_after();
                    const int slot = np % kSlots;
                    const uint64_t vd = v_desc0 + desc_step((uint32_t)slot * C::kSlot);
                    const uint64_t pd = p_desc0 + desc_step((uint32_t)(np & 1) * kPBytes);
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk)  // 16 positions = 2048 bytes of the V boxes
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
            // nothing of this CTA may still run on the tensor core at
            // teardown, and the Q load has landed
            mma_commit(drained);
            if (!mbar_drain(drained, 0)) ok = false;
            if (!mbar_drain(q_full, 0)) ok = false;
        }
    } else if (warp >= kSoftThreads / 32) {
        // ------------------------------------------------------------ gather
        const int gt = threadIdx.x - kSoftThreads;
        const __nv_bfloat16 *kb = a.k_cache + (int64_t)b * a.k_sb;
        const __nv_bfloat16 *vb = a.v_cache + (int64_t)b * a.v_sb;
        // the ring holds the Q staging until the rows are in TMEM
        if (n_tiles > 0 && ok && !mbar_wait(q_copied, 0)) ok = false;
        const uint32_t ring_base = smem_addr(ring);
        for (int t = 0; ok && t < n_tiles; ++t) {
            const int slot = t % kSlots;
            if (!mbar_wait(&kv_empty[slot], ((uint32_t)(t / kSlots) & 1u) ^ 1u)) {
                ok = false;
                break;
            }
            const uint32_t dst0 = ring_base + (uint32_t)slot * C::kSlot;
            // chunk c: box c / 512, row (c / 8) % 64, 16-byte chunk c % 8 of
            // that box row; boxes below kQBoxes are K columns, the rest V
#pragma unroll 2
            for (int c = gt; c < kTileN * C::kBoxes * 8; c += kGatherThreads) {
                const int lb = c >> 9;
                const int r = (c >> 3) & (kTileN - 1);
                const int cb = c & 7;
                const int jj = t * kTileN + r;
                const bool valid = jj < n_sel;
                const int s = valid ? (int)(ulist[jj] & 0xFFFFu) : 0;
                const __nv_bfloat16 *src = lb < C::kQBoxes
                                               ? kb + (int64_t)s * a.k_ss + lb * 64 + cb * 8
                                               : vb + (int64_t)s * a.v_ss + (lb - C::kQBoxes) * 64 + cb * 8;
                cp_async16_zfill(dst0 + (uint32_t)lb * kBox + (uint32_t)r * 128 + ((uint32_t)(cb ^ (r & 7)) << 4),
                                 src, valid);
            }
            cp_async_arrive_noinc(&kv_full[slot]);
        }
        cp_async_wait_all();
    } else {
        // ------------------------------------------------------------ softmax
        const int r = threadIdx.x;         // row = TMEM lane
        const int qq = r >> 4, h = r & 15;  // query of the group, head
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        float m_ref = -INFINITY, l = 0.0f;  // reference max (log2 units), running sum
        if (n_tiles > 0) {
            // row r of the staged Q boxes (128-byte swizzle) into TMEM lane r
            if (!mbar_wait(q_full, 0)) ok = false;
            if (__all_sync(0xffffffffu, ok)) {
#pragma unroll 1
                for (int c = 0; c < C::kQBoxes; ++c) {
                    const uint8_t *box = ring + c * kQBox + r * 128;
                    uint32_t w[32];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 x = *reinterpret_cast<const uint4 *>(box + ((j ^ (r & 7)) << 4));
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
        ok = __all_sync(0xffffffffu, ok);
        // the warp's two queries: rows 32 w .. 32 w + 15 and 32 w + 16 .. 32 w + 31
        const int qa = 2 * warp, qb = 2 * warp + 1;
        for (int t = 0; ok && t < n_tiles; ++t) {
            if (!mbar_spin(s_full, (uint32_t)t & 1u)) ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            uint32_t x[64];
            tmem_ld_32x32b_x32(tmem + lane_addr + kColS, x);
            tmem_ld_32x32b_x32(tmem + lane_addr + kColS + 32, x + 32);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(s_free);  // the next QK^T may overwrite S
            // which of the tile's positions this row's query selected
            const int j0 = t * kTileN;
            const uint32_t e0 = j0 + lane < n_sel ? ulist[j0 + lane] : 0u;
            const uint32_t e1 = j0 + 32 + lane < n_sel ? ulist[j0 + 32 + lane] : 0u;
            const uint32_t ma0 = __ballot_sync(0xffffffffu, (e0 >> (16 + qa)) & 1u);
            const uint32_t ma1 = __ballot_sync(0xffffffffu, (e1 >> (16 + qa)) & 1u);
            const uint32_t mb0 = __ballot_sync(0xffffffffu, (e0 >> (16 + qb)) & 1u);
            const uint32_t mb1 = __ballot_sync(0xffffffffu, (e1 >> (16 + qb)) & 1u);
            const uint32_t mlo = lane < 16 ? ma0 : mb0, mhi = lane < 16 ? ma1 : mb1;
            // positions either of the warp's queries selected (the same in
            // every lane): the others need no exponent below
            const uint32_t any_lo = ma0 | mb0, any_hi = ma1 | mb1;
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float z = ((mlo >> j) & 1u) ? __uint_as_float(x[j]) * a.scale_log2 : -INFINITY;
                x[j] = __float_as_uint(z);
                mq[j & 3] = fmaxf(mq[j & 3], z);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float z = ((mhi >> j) & 1u) ? __uint_as_float(x[32 + j]) * a.scale_log2 : -INFINITY;
                x[32 + j] = __float_as_uint(z);
                mq[j & 3] = fmaxf(mq[j & 3], z);
            }
            const float mt = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            // P buffer t % 2 was last read by PV of tile t - 2
            if (t >= 2 && !mbar_wait(&pv_done[t & 1], (uint32_t)((t - 2) >> 1) & 1u)) ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
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
                // O may be rescaled once every PV so far (through tile t - 1) is
                // done; a row with a finite reference max has seen an earlier tile
                if (!mbar_wait(&pv_done[(t - 1) & 1], (uint32_t)((t - 1) >> 1) & 1u)) ok = false;
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const float f = grow ? exp2f(m_ref - m_new) : 1.0f;
#pragma unroll 1
                for (int c = 0; c < DV; c += 32) {
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
            // p = 2^(z - m_ref); masked positions have z = -inf, so p = 0, and
            // positions neither query of the warp selected skip the exponent
            const float mr = m_ref == -INFINITY ? 0.0f : m_ref;
            uint32_t pk[32];
            float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int e0 = 2 * j, e1 = 2 * j + 1;
                const uint32_t any = e0 < 32 ? any_lo : any_hi;
                float p0 = 0.0f, p1 = 0.0f;
                if ((any >> (e0 & 31)) & 1u) p0 = ex2_approx(__uint_as_float(x[e0]) - mr);
                if ((any >> (e1 & 31)) & 1u) p1 = ex2_approx(__uint_as_float(x[e1]) - mr);
                ps[(2 * j) & 3] += p0;
                ps[(2 * j + 1) & 3] += p1;
                pk[j] = pack_bf16x2(p0, p1);
            }
            l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
            // P row r of buffer t % 2: 128 bytes, 16-byte chunk c at c ^ (r % 8)
            uint8_t *prow = p_sm + (t & 1) * kPBytes + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(prow + ((c ^ (r & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();  // P is read by the tensor core
            tc_fence_before();
            mbar_arrive(&p_full[t & 1]);
        }
        if (ok && n_tiles > 0 &&
            !mbar_wait(&pv_done[(n_tiles - 1) & 1], (uint32_t)((n_tiles - 1) >> 1) & 1u))
            ok = false;
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            // O of row r (every PV done) to the output row of query qq, head h
            tc_fence_after();
            const float inv = l > 0.0f ? 1.0f / l : 0.0f;
            uint4 *dst = reinterpret_cast<uint4 *>(a.out + ((row0 + qq) * kHeads + h) * DV);
#pragma unroll 1
            for (int c = 0; c < DV; c += 64) {  // two loads per wait (warp-wide)
                uint32_t o[64];
                if (n_tiles > 0) {
                    tmem_ld_32x32b_x32(tmem + lane_addr + kColO + (uint32_t)c, o);
                    tmem_ld_32x32b_x32(tmem + lane_addr + kColO + (uint32_t)c + 32, o + 32);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) o[j] = 0u;
                }
                if (qq < qn) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[c / 8 + q] = make_uint4(
                            pack_bf16x2(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
                }
            }
            if (a.lse != nullptr && qq < qn)
                a.lse[(row0 + qq) * kHeads + h] = l > 0.0f ? (m_ref + log2f(l)) / kLog2e : -INFINITY;
        }
    }

    if (!ok) atomicOr(&g_attn_mqa_tc_error, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t attn_mqa_tc_set_wait_limit(unsigned long long ns) { return set_wait_limit_ns(ns); }

unsigned int attn_mqa_tc_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_mqa_tc_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_mqa_tc_error, &zero, sizeof(zero));
    return v;
}

// Groups of 8 query rows (16 heads over one KV head, Dqk 128 or 192, Dv 128):
// enough groups to cover the GPU, positions that fit 16 bits, a union list
// that fits (min(L, 8 k) entries), and a Q tensor of at least one 128-row box.
bool attn_mqa_tc_supported(const AttnProblem &p) {
    if (p.dt != DSA_BF16 || p.Hq != kHeads || p.Hkv != 1 || p.Dv != DV) return false;
    if (p.Dqk != 128 && p.Dqk != 192) return false;
    if (p.Tq < 2 || p.L > 65536 || p.k > kMaxUnion / kRowsQ) return false;
    if ((long long)p.B * p.Tq < kRowsQ) return false;
    if (((uintptr_t)p.k_cache | (uintptr_t)p.v_cache | (uintptr_t)p.q | (uintptr_t)p.out) % 16 != 0) return false;
    if (p.k_ss % 8 || p.k_sb % 8 || p.v_ss % 8 || p.v_sb % 8) return false;
    DeviceInfo info;
    if (device_info(&info) != cudaSuccess || info.cc_major != 10) return false;
    const long long groups = (long long)p.B * ((p.Tq + kRowsQ - 1) / kRowsQ);
    if (groups < info.sm_count || groups > 0x7fffffffLL) return false;
    const size_t smem = p.Dqk == 192 ? MqaCfg<192>::kSmem : MqaCfg<128>::kSmem;
    return (size_t)info.max_smem_optin >= smem;
}

int attn_mqa_tc_row_group() { return kRowsQ; }

template <int DQK>
static cudaError_t launch_mqa(const AttnProblem &p, cudaStream_t stream) {
    using C = MqaCfg<DQK>;
    CUtensorMap tm_q;
    const uint64_t qrows = (uint64_t)p.B * p.Tq * kHeads;
    if (!make_map_bf16_sw128(&tm_q, p.q, qrows, DQK, (uint64_t)DQK * 2, kM)) return cudaErrorInvalidValue;
    MqaArgs a;
    a.k_cache = static_cast<const __nv_bfloat16 *>(p.k_cache);
    a.v_cache = static_cast<const __nv_bfloat16 *>(p.v_cache);
    a.idx = p.idx;
    a.B = p.B; a.Tq = p.Tq; a.L = p.L; a.k = p.k;
    a.ngroups = (p.Tq + kRowsQ - 1) / kRowsQ;
    a.W = (p.L + 31) / 32;
    a.scale_log2 = p.scale * kLog2e;
    a.k_sb = p.k_sb; a.k_ss = p.k_ss; a.v_sb = p.v_sb; a.v_ss = p.v_ss;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.lse = p.lse;
    auto kern = attn_mqa_group_tc_kernel<DQK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (err != cudaSuccess) return err;
    const long long grid = (long long)p.B * a.ngroups;
    kern<<<(unsigned)grid, kThreads, C::kSmem, stream>>>(tm_q, a);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_attn_mqa_tc(const AttnProblem &p, cudaStream_t stream) {
    return p.Dqk == 192 ? launch_mqa<192>(p, stream) : launch_mqa<128>(p, stream);
}

}  // namespace dsa
