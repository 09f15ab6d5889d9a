// Backward pass of the lightning indexer on the 5th-generation tensor cores.
//
// For the incoming gradient g = d loss / d I of the indexer's training loss
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §5.4,
// §6.2; §6.4: it reaches only the indexer) and the score of §2.1,
// I[t,s] = sum_j w[t,j] ReLU(x[t,j,s]), x[t,j,s] = q[t,j] . k[s]:
//   G[t,j,s] = g[t,s] w[t,j] [x[t,j,s] > 0]
//   dq[t,j]  = sum_{s<=t} G[t,j,s] k[s]           dw[t,j] = sum_{s<=t} g[t,s] ReLU(x[t,j,s])
//   dk[s]    = sum_{t>=s} sum_j G[t,j,s] q[t,j]
//
// Both products are GEMMs around an elementwise step, so one kernel serves
// both sides with the roles of the operands swapped:
//   query side (dq, dw): a group of 128 / H queries (128 rows (t, j)) stays
//       resident; 128-key tiles stream past it.
//       MMA 1  X[(t,j), s]  = Q[(t,j), :] . K[s, :]        M=128 N=128 K=128
//       epilogue  M = g [X > 0] in bf16 into TMEM (w[t,j] is constant along
//                 a row, so G = w M is applied to the result)
//       MMA 2  acc[(t,j), :] += M[(t,j), s] K[s, :]          M=128 N=128 K=128
//       dq = w acc, and dw = q . acc, since sum_s g ReLU(x) = sum_s M x and
//       x = q . k[s] (one dot product per row and unit, no per-element work)
//   key side (dk): a 128-key tile stays resident; query groups stream past.
//       MMA 1  X[s, (t,j)]  = K[s, :] . Q[(t,j), :]
//       epilogue  G[s, (t,j)] as above
//       MMA 2  dK[s, :] += G[s, (t,j)] Q[(t,j), :]
// MMA 2 reads G from TMEM (A operand) and the streamed tile a second time, as
// an MN-major B operand: a 128-row tile of 128-byte swizzled rows is K-major
// for MMA 1 (rows along N) and MN-major for MMA 2 (rows along K), so one copy
// in shared memory feeds both. x is exact (integer-valued bf16, fp32 sums);
// G is rounded to bf16 for MMA 2; sums are fp32.
//
// Warp roles (576 threads, one CTA per SM, persistent over work units):
//   warp 0     TMA: the resident tile of each unit (two buffers), streamed
//              tiles through a 4-stage ring.
//   warp 1     TMEM owner; one thread issues two streams of MMAs, each as
//              soon as its inputs are ready: MMA 1 runs up to two tiles ahead
//              of the epilogue, MMA 2 follows it.
//   warps 2-17 epilogue: two groups of eight warps taking alternate tiles
//              (two tiles in flight), two warps per TMEM lane quarter in a
//              group, 64 columns each; at the end of a unit all sixteen read
//              the accumulator, 32 columns each.
// TMEM: X in two buffers [0, 256) and G in two [256, 384) (two bf16 per
// column), one pair per epilogue group; the accumulator [384, 512).
// Work: query side, one unit per query group (longest causal range first);
// key side, one unit per (key tile, chunk of query groups), each chunk's
// partial dK written to a workspace slot and the slots of a key tile summed
// in a fixed order by indexer_bwd_reduce_kernel (the same result every call).
// Every mbarrier wait is bounded; on a timeout the CTA records an error word,
// waits for its own MMAs and copies, frees TMEM and returns.
#include <math.h>

#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kRows = 128;                  // MMA M and rows of every tile
constexpr int kD = 128;                     // d_I
constexpr uint32_t kBox = kRows * 128;      // 128 rows x 64 bf16 columns (128-byte swizzle)
constexpr uint32_t kTile = 2 * kBox;        // 128 rows x 128 columns
constexpr int kStages = 4;
constexpr int kResBufs = 2;
constexpr int kEpiWarps = 16;               // four per TMEM lane quarter
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kParts = kEpiWarps / 4;         // column parts of a tile
constexpr int kCW = 128 / kParts;             // columns per epilogue warp
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColX = 0;               // 2 x 128: X
constexpr uint32_t kColG = 256;             // 2 x 64: G (bf16 pairs), A of MMA 2
constexpr uint32_t kColAcc = 384;           // 128: the accumulator
constexpr uint32_t kIdescMnMajorB = 1u << 16;
// barriers: res_full/empty[2], st_full/empty[4], x_full/empty[2], g_full/empty[2], acc_full, acc_empty,
// drain, dw_bar
constexpr int kNumBars = 2 * kResBufs + 2 * kStages + 4 + 4 + 4;
constexpr uint32_t kDwBytes = 2 * kParts * kRows * 4;  // dw partial sums, two buffers
constexpr uint32_t kGBytes = 4 * kRows * 4;            // per stage: g of up to 4 queries x 128 keys
constexpr uint32_t kWBytes = kRows * 4;                // per stage: w of one query group (key side)
constexpr size_t kSmem = 1024 + (size_t)kResBufs * kTile + (size_t)kStages * (kTile + kGBytes + kWBytes) + kDwBytes +
                         kNumBars * 8 + 16;
static_assert(kSmem <= 232448, "shared memory budget");

__device__ unsigned int g_indexer_bwd_error = 0;  // 1 = a bounded wait gave up

struct Params {
    const float *w, *grad;
    int B, Tq, L, q_pos0, H, QPG;  // QPG = 128 / H queries per group
    int ngroups;                    // query groups per batch entry
    int nkt;                        // key tiles per batch entry
    int nchunks, C;                 // key side: chunks of C groups
    int units;
    float *dq, *dw;                 // query side
    float *part;                    // key side: [B * nchunks * nkt][128][128]
};

struct Unit {
    int b;
    int g0, g1;    // query groups [g0, g1) (query side: one group)
    int kt0, kt1;  // key tiles [kt0, kt1) (key side: one tile)
    int slot;      // key side: partial slot
};

__device__ __forceinline__ int first_group(const Params &p, int kt) {
    // first query group holding a query at t >= kt * 128
    const int i = kt * kRows - p.q_pos0;
    return i <= 0 ? 0 : i / p.QPG;
}

template <bool KEY_SIDE>
__device__ __forceinline__ bool decode_unit(int u, const Params &p, Unit &un) {
    if (!KEY_SIDE) {
        const int b = u % p.B;
        const int g = p.ngroups - 1 - u / p.B;
        const int i0 = g * p.QPG;
        const int qcount = min(p.QPG, p.Tq - i0);
        const int t_last = p.q_pos0 + i0 + qcount - 1;
        un.b = b;
        un.g0 = g;
        un.g1 = g + 1;
        un.kt0 = 0;
        un.kt1 = t_last / kRows + 1;
        un.slot = 0;
        return true;
    }
    const int kt = u % p.nkt;
    const int rest = u / p.nkt;
    const int c = rest % p.nchunks;
    const int b = rest / p.nchunks;
    const int gf = first_group(p, kt);
    const int g0 = max(gf, c * p.C);
    const int g1 = min(p.ngroups, (c + 1) * p.C);
    if (g0 >= g1) return false;
    un.b = b;
    un.g0 = g0;
    un.g1 = g1;
    un.kt0 = kt;
    un.kt1 = kt + 1;
    un.slot = u;
    return true;
}

// (lo, hi) = (a_lo * b_lo, a_hi * b_hi)
__device__ __forceinline__ void mul2(float &lo, float &hi, float a_lo, float a_hi, float b_lo, float b_hi) {
    uint64_t a, b, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a_lo), "f"(a_hi));
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b_lo), "f"(b_hi));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <bool KEY_SIDE, int H>
__global__ void __launch_bounds__(kThreads, 1)
indexer_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_w,
                      const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *res_sm = smem;
    uint8_t *st_sm = res_sm + kResBufs * kTile;
    float *g_sm = reinterpret_cast<float *>(st_sm + kStages * kTile);      // [stage][query][128 keys]
    float *w_sm = g_sm + kStages * (kGBytes / 4);                          // [stage][128 (query, head)]
    float *dw_sm = w_sm + kStages * (kWBytes / 4);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(dw_sm) + kDwBytes);
    uint64_t *res_full = bars;
    uint64_t *res_empty = res_full + kResBufs;
    uint64_t *st_full = res_empty + kResBufs;
    uint64_t *st_empty = st_full + kStages;
    uint64_t *x_full = st_empty + kStages;
    uint64_t *x_empty = x_full + 2;
    uint64_t *g_full = x_empty + 2;
    uint64_t *g_empty = g_full + 2;
    uint64_t *acc_full = g_empty + 2;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *drain = acc_empty + 1;
    uint64_t *dw_bar = drain + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dw_bar + 1);

    constexpr int QPG = kRows / H;  // queries per group
    // bytes each streamed tile brings: the tile, g of the group's queries over
    // the 128 keys, and (key side) w of the group
    constexpr uint32_t kStageTx = kTile + QPG * kRows * 4 + (KEY_SIDE ? kRows * 4 : 0);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // the resident tile comes from K on the key side, from Q on the query side
    const CUtensorMap *tm_res = KEY_SIDE ? &tm_k : &tm_q;
    const CUtensorMap *tm_str = KEY_SIDE ? &tm_q : &tm_k;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kResBufs; ++s) {
            mbar_init(&res_full[s], 1);
            mbar_init(&res_empty[s], 1 + kEpiThreads);  // the MMAs and the epilogue's last reads
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&st_full[s], 1);
            mbar_init(&st_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {  // buffer s serves the tiles of epilogue group s
            mbar_init(&x_full[s], 1);
            mbar_init(&x_empty[s], kEpiThreads / 2);
            mbar_init(&g_full[s], kEpiThreads / 2);
            mbar_init(&g_empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiThreads);
        mbar_init(drain, 1);
        mbar_init(dw_bar, kEpiThreads);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = waits_enabled();  // false: the wait limit is 0 (give-up test)

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            prefetch_tensor_map(&tm_q);
            prefetch_tensor_map(&tm_k);
            prefetch_tensor_map(&tm_g);
            if (KEY_SIDE) prefetch_tensor_map(&tm_w);
            int sb = 0, rb = 0;
            uint32_t sph = 0, rph = 0;
            int st_armed[kStages], res_armed[kResBufs];  // parity of each buffer's last armed phase, or -1
            for (int s = 0; s < kStages; ++s) st_armed[s] = -1;
            for (int s = 0; s < kResBufs; ++s) res_armed[s] = -1;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                Unit un;
                if (!decode_unit<KEY_SIDE>(u, p, un)) continue;
                if (!mbar_wait(&res_empty[rb], rph ^ 1u)) { ok = false; break; }
                mbar_arrive_expect_tx(&res_full[rb], kTile);
                res_armed[rb] = (int)rph;
                const int rrow = KEY_SIDE ? un.b * p.L + un.kt0 * kRows : (un.b * p.Tq + un.g0 * p.QPG) * p.H;
                tma_load_2d(res_sm + rb * kTile, tm_res, &res_full[rb], 0, rrow);
                tma_load_2d(res_sm + rb * kTile + kBox, tm_res, &res_full[rb], 64, rrow);
                if (++rb == kResBufs) { rb = 0; rph ^= 1u; }
                const int n0 = KEY_SIDE ? un.g0 : un.kt0, n1 = KEY_SIDE ? un.g1 : un.kt1;
                for (int n = n0; n < n1; ++n) {
                    if (!mbar_wait(&st_empty[sb], sph ^ 1u)) { ok = false; break; }
                    mbar_arrive_expect_tx(&st_full[sb], kStageTx);
                    st_armed[sb] = (int)sph;
                    const int srow = KEY_SIDE ? (un.b * p.Tq + n * QPG) * H : un.b * p.L + n * kRows;
                    tma_load_2d(st_sm + sb * kTile, tm_str, &st_full[sb], 0, srow);
                    tma_load_2d(st_sm + sb * kTile + kBox, tm_str, &st_full[sb], 64, srow);
                    // g[t, s] for the (group, key tile) pair of this step
                    const int grow = un.b * p.Tq + (KEY_SIDE ? n : un.g0) * QPG;
                    const int gcol = (KEY_SIDE ? un.kt0 : n) * kRows;
                    tma_load_2d(g_sm + sb * (kGBytes / 4), &tm_g, &st_full[sb], gcol, grow);
                    if (KEY_SIDE) tma_load_2d(w_sm + sb * (kWBytes / 4), &tm_w, &st_full[sb], 0, grow);
                    if (++sb == kStages) { sb = 0; sph ^= 1u; }
                }
            }
            // no copy may still be landing when the CTA exits
            for (int s = 0; s < kStages; ++s)
                if (st_armed[s] >= 0 && !mbar_drain(&st_full[s], (uint32_t)st_armed[s])) ok = false;
            for (int s = 0; s < kResBufs; ++s)
                if (res_armed[s] >= 0 && !mbar_drain(&res_full[s], (uint32_t)res_armed[s])) ok = false;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            // Two streams of MMAs, each issued as soon as its inputs are
            // ready: MMA 1 of the next tile (a stage landed, an X buffer
            // free) and MMA 2 of the oldest tile whose G is in TMEM. MMA 1
            // thus runs up to two tiles ahead of the epilogue.
            const uint32_t idesc1 = idesc_bf16_f32(kRows, kRows);
            const uint32_t idesc2 = idesc_bf16_f32(kRows, kD) | kIdescMnMajorB;
            int sb1 = 0, xb1 = 0, sb2 = 0, rb = 0;
            uint32_t sph1 = 0, xph1 = 0, xph2 = 0, rph = 0, aph = 0;
            int xb2 = 0;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                Unit un;
                if (!decode_unit<KEY_SIDE>(u, p, un)) continue;
                if (!mbar_wait(&res_full[rb], rph)) { ok = false; break; }
                tc_fence_after();
                const uint64_t a_desc = smem_desc_k_sw128(smem_addr(res_sm + rb * kTile));
                const int ntiles = KEY_SIDE ? un.g1 - un.g0 : un.kt1 - un.kt0;
                int n1 = 0, n2 = 0;
                uint32_t idle = 0;
                uint64_t t_idle = 0;
                while (n2 < ntiles) {
                    bool progress = false;
                    if (n1 < ntiles && mbar_test_wait(&st_full[sb1], sph1) && mbar_test_wait(&x_empty[xb1], xph1 ^ 1u)) {
                        // MMA 1: X = A . B^T, both K-major
                        tc_fence_after();
                        const uint64_t b_desc = smem_desc_k_sw128(smem_addr(st_sm + sb1 * kTile));
                        const uint32_t d = tmem + kColX + (uint32_t)(xb1 * 128);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t off = (uint64_t)(((kk >> 2) * kBox + (kk & 3) * 32) >> 4);
                            mma_f16_ss(d, a_desc + off, b_desc + off, idesc1, kk != 0);
                        }
                        mma_commit(&x_full[xb1]);
                        ++n1;
                        if (++sb1 == kStages) { sb1 = 0; sph1 ^= 1u; }
                        if (++xb1 == 2) { xb1 = 0; xph1 ^= 1u; }
                        progress = true;
                    }
                    if (n2 < n1 && mbar_test_wait(&g_full[xb2], xph2) &&
                        (n2 > 0 || mbar_test_wait(acc_empty, aph ^ 1u))) {
                        // MMA 2: acc += G (TMEM) . B (the same stage, MN-major)
                        tc_fence_after();
                        const uint64_t b_desc = smem_desc_mn_sw128(smem_addr(st_sm + sb2 * kTile), kBox);
                        const uint32_t a_tm = tmem + kColG + (uint32_t)(xb2 * 64);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_f16_ts(tmem + kColAcc, a_tm + (uint32_t)(kk * 8), b_desc + (uint64_t)((kk * 2048) >> 4),
                                       idesc2, (n2 > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&st_empty[sb2]);  // the streamed tile is no longer read
                        mma_commit(&g_empty[xb2]);
                        ++n2;
                        if (++sb2 == kStages) sb2 = 0;
                        if (++xb2 == 2) { xb2 = 0; xph2 ^= 1u; }
                        progress = true;
                    }
                    if (progress) {
                        idle = 0;
                    } else {
                        // bounded: give up after the wait limit without progress
                        const unsigned long long limit = __ldg(&g_wait_limit_ns);
                        if (limit == 0) { ok = false; break; }
                        if (idle == 0) t_idle = global_timer_ns();
                        if ((++idle & 63u) == 0u && global_timer_ns() - t_idle > limit) { ok = false; break; }
                        __nanosleep(20);
                    }
                }
                if (!ok) break;
                mma_commit(acc_full);
                aph ^= 1u;
                mma_commit(&res_empty[rb]);
                if (++rb == kResBufs) { rb = 0; rph ^= 1u; }
            }
            // every MMA issued here has finished before TMEM is freed
            mma_commit(drain);
            if (!mbar_drain(drain, 0)) ok = false;
        }
    } else {
        // ---------------------------------------------------- epilogue
        // Query side: w[t,j] is constant along a TMEM lane, so MMA 2 takes
        // M = g [X > 0] and the accumulator is multiplied by w once per unit
        // (G = w M; for the power-of-two weights the rounding of M and of G
        // to bf16 is the same). Key side: G = (g w)[X > 0], with g constant
        // per (lane, query) and w per column.
        // Tiles alternate between two groups of eight warps (grp), so that two
        // tiles are in the epilogue at once; within a group, the two warps of
        // a lane quarter (sub) take 64 columns each, in two chunks of kCW.
        // At the end of a unit all sixteen warps read the accumulator, kCW
        // columns each (part).
        const int quarter = warp & 3;
        const int part = (warp - 2) >> 2;          // 0..3
        const int grp = part >> 1, sub = part & 1;
        const int col0 = part * kCW;
        const int r = quarter * 32 + lane;         // TMEM lane: resident row
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int unit_n = 0, rb = 0;
        uint32_t aph = 0, rph = 0;
        uint32_t gt = 0;                           // streamed tiles seen so far (all units)
        for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
            Unit un;
            if (!decode_unit<KEY_SIDE>(u, p, un)) continue;
            const int ntiles = KEY_SIDE ? un.g1 - un.g0 : un.kt1 - un.kt0;
            // query side: this lane's (query, head)
            const int qi = r / H, j = r % H;
            const int i_row = un.g0 * QPG + qi;
            const bool row_ok = !KEY_SIDE && i_row < p.Tq;
            const int row = un.b * p.Tq + i_row;
            const int t_row = row_ok ? p.q_pos0 + i_row : -1;  // no such query: nothing passes
            for (int n = 0; n < ntiles && ok; ++n, ++gt) {
                const int xbuf = (int)(gt & 1u);
                if (xbuf != grp) continue;  // the other group takes this tile
                const uint32_t xphase = (gt >> 1) & 1u;
                const int sbuf = (int)(gt % kStages);
                const uint32_t sphase = (gt / kStages) & 1u;
                if (!mbar_wait(&x_full[xbuf], xphase)) { ok = false; break; }
                // (complete already: MMA 1 read this stage) makes the TMA writes of g and w visible here
                if (!mbar_wait(&st_full[sbuf], sphase)) { ok = false; break; }
                tc_fence_after();
                const float *gs = g_sm + sbuf * (kGBytes / 4);
                const float *wsm = w_sm + sbuf * (kWBytes / 4);
                // G of kCW columns starting at c0 from X in xr
                auto chunk = [&](const uint32_t *xr, int c0, uint32_t *gp) {
                    if (!KEY_SIDE) {
                        // columns = keys s_base + c; g[t, s] is the same for the warp's lanes
                        const int s_base = (un.kt0 + n) * kRows + c0;
                        const float4 *g4 = reinterpret_cast<const float4 *>(gs + qi * kRows + c0);
                        if (t_row < s_base) {  // every key of this part lies after t (or no query)
    #pragma unroll
                            for (int c = 0; c < kCW / 2; ++c) gp[c] = 0u;
                        } else if (s_base + kCW - 1 <= t_row) {  // no key of this part after t
    #pragma unroll
                            for (int c4 = 0; c4 < kCW / 4; ++c4) {
                                const float4 gv = g4[c4];
                                gp[2 * c4] = pack_bf16x2(__uint_as_float(xr[4 * c4]) > 0.f ? gv.x : 0.f,
                                                         __uint_as_float(xr[4 * c4 + 1]) > 0.f ? gv.y : 0.f);
                                gp[2 * c4 + 1] = pack_bf16x2(__uint_as_float(xr[4 * c4 + 2]) > 0.f ? gv.z : 0.f,
                                                             __uint_as_float(xr[4 * c4 + 3]) > 0.f ? gv.w : 0.f);
                            }
                        } else {  // the diagonal: keys after t pass nothing
    #pragma unroll
                            for (int c4 = 0; c4 < kCW / 4; ++c4) {
                                const float4 gv = g4[c4];
                                const int s = s_base + 4 * c4;
                                const float m0 = (__uint_as_float(xr[4 * c4]) > 0.f && s <= t_row) ? gv.x : 0.f;
                                const float m1 = (__uint_as_float(xr[4 * c4 + 1]) > 0.f && s + 1 <= t_row) ? gv.y : 0.f;
                                const float m2 = (__uint_as_float(xr[4 * c4 + 2]) > 0.f && s + 2 <= t_row) ? gv.z : 0.f;
                                const float m3 = (__uint_as_float(xr[4 * c4 + 3]) > 0.f && s + 3 <= t_row) ? gv.w : 0.f;
                                gp[2 * c4] = pack_bf16x2(m0, m1);
                                gp[2 * c4 + 1] = pack_bf16x2(m2, m3);
                            }
                        }
                    } else {
                        // lanes = keys s; columns = (query, head) pairs of group g
                        const int g = un.g0 + n;
                        const int s = un.kt0 * kRows + r;
                        constexpr int QPP = kCW / H > 0 ? kCW / H : 1;  // queries in this part
                        constexpr int C4 = (H < kCW ? H : kCW) / 4;     // float4s of one query in the part
    #pragma unroll
                        for (int z = 0; z < QPP; ++z) {
                            const int qz = c0 / H + z;
                            const int i = g * QPG + qz;
                            float gq = 0.f;
                            if (i < p.Tq && s <= p.q_pos0 + i) gq = gs[qz * kRows + r];
                            const float4 *w4 = reinterpret_cast<const float4 *>(wsm + qz * H + (c0 % H));
    #pragma unroll
                            for (int c4 = 0; c4 < C4; ++c4) {
                                const int cc = z * (C4 * 4) + 4 * c4;  // column within the part
                                const float4 wv = w4[c4];
                                float gw0, gw1, gw2, gw3;
                                mul2(gw0, gw1, gq, gq, wv.x, wv.y);
                                mul2(gw2, gw3, gq, gq, wv.z, wv.w);
                                const float x0 = __uint_as_float(xr[cc]), x1 = __uint_as_float(xr[cc + 1]);
                                const float x2 = __uint_as_float(xr[cc + 2]), x3 = __uint_as_float(xr[cc + 3]);
                                gp[cc / 2] = pack_bf16x2(x0 > 0.f ? gw0 : 0.f, x1 > 0.f ? gw1 : 0.f);
                                gp[cc / 2 + 1] = pack_bf16x2(x2 > 0.f ? gw2 : 0.f, x3 > 0.f ? gw3 : 0.f);
                            }
                        }
                    }
                };
                uint32_t xr[kCW], gpa[kCW / 2], gpb[kCW / 2];
                const int c0a = sub * (2 * kCW), c0b = c0a + kCW;
                tmem_ld_32x32b_x32(tmem + lane_addr + kColX + (uint32_t)(xbuf * 128 + c0a), xr);
                tmem_ld_wait();
                chunk(xr, c0a, gpa);
                tmem_ld_32x32b_x32(tmem + lane_addr + kColX + (uint32_t)(xbuf * 128 + c0b), xr);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&x_empty[xbuf]);
                chunk(xr, c0b, gpb);
                // this group's G buffer: MMA 2 of its previous tile has read it
                if (!mbar_wait(&g_empty[xbuf], xphase ^ 1u)) { ok = false; break; }
                tc_fence_after();
                tmem_st_32x32b_x16(tmem + lane_addr + kColG + (uint32_t)(xbuf * 64 + c0a / 2), gpa);
                tmem_st_32x32b_x16(tmem + lane_addr + kColG + (uint32_t)(xbuf * 64 + c0b / 2), gpb);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&g_full[xbuf]);
            }
            if (!ok) break;
            // ---- the unit's accumulator
            if (!mbar_wait(acc_full, aph)) { ok = false; break; }
            tc_fence_after();
            uint32_t ar[kCW];
            tmem_ld_32x32b_x32(tmem + lane_addr + kColAcc + (uint32_t)col0, ar);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(acc_empty);
            aph ^= 1u;
            float *dst = nullptr;
            float scale = 1.f;
            if (KEY_SIDE) {
                tc_fence_before();
                mbar_arrive(&res_empty[rb]);  // nothing here reads the resident tile
                dst = p.part + ((size_t)un.slot * kRows + r) * kD + col0;
            } else {
                // dw[t,j] = sum_s g ReLU(x) = sum_s M[s] x[s] = q[t,j] . (sum_s M[s] k[s]):
                // this lane's resident q row (bf16, 128-byte swizzle) against the
                // unscaled accumulator, over this part's 32 columns
                // (complete already: MMA 1 read this tile) makes the TMA writes visible here
                if (!mbar_wait(&res_full[rb], rph)) { ok = false; break; }
                const uint8_t *qrow = res_sm + rb * kTile + (col0 >> 6) * kBox + r * 128;
                float dwp = 0.f;
#pragma unroll
                for (int c = 0; c < kCW / 8; ++c) {
                    const int chunk = ((col0 & 63) >> 3) + c;
                    const uint4 v = *reinterpret_cast<const uint4 *>(qrow + ((chunk ^ (r & 7)) << 4));
                    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        dwp = fmaf(__uint_as_float(wv[e] << 16), __uint_as_float(ar[8 * c + 2 * e]), dwp);
                        dwp = fmaf(__uint_as_float(wv[e] & 0xffff0000u), __uint_as_float(ar[8 * c + 2 * e + 1]), dwp);
                    }
                }
                mbar_arrive(&res_empty[rb]);
                // the parts' partial sums meet in shared memory (two buffers, by
                // unit parity) and part 0 adds them in a fixed order
                float *dws = dw_sm + (unit_n & 1) * (kParts * kRows);
                dws[part * kRows + r] = dwp;
                mbar_arrive(dw_bar);
                if (part == 0) {
                    if (!mbar_wait(dw_bar, (uint32_t)(unit_n & 1))) { ok = false; break; }
                    float sum = dws[r];
#pragma unroll
                    for (int q = 1; q < kParts; ++q) sum += dws[q * kRows + r];
                    if (row_ok && p.dw) p.dw[(size_t)row * H + j] = sum;
                }
                if (row_ok) {
                    scale = p.w[(size_t)row * H + j];
                    if (p.dq) dst = p.dq + ((size_t)row * H + j) * kD + col0;
                }
            }
            if (dst) {
                float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
                for (int c4 = 0; c4 < kCW / 4; ++c4)
                    d4[c4] = make_float4(__uint_as_float(ar[4 * c4]) * scale, __uint_as_float(ar[4 * c4 + 1]) * scale,
                                         __uint_as_float(ar[4 * c4 + 2]) * scale,
                                         __uint_as_float(ar[4 * c4 + 3]) * scale);
            }
            if (++rb == kResBufs) { rb = 0; rph ^= 1u; }
            ++unit_n;
        }
    }

    if (!ok) atomicOr(&g_indexer_bwd_error, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// dk[b, kt * 128 + r, :] = sum over the key tile's chunks, in chunk order.
__global__ void __launch_bounds__(256)
indexer_bwd_reduce_kernel(const float *__restrict__ part, const Params p, float *__restrict__ dk) {
    const int kt = blockIdx.x, b = blockIdx.y;
    const int gf = first_group(p, kt);
    const int c0 = gf >= p.ngroups ? p.nchunks : gf / p.C;
    const int rows = min(kRows, p.L - kt * kRows);
    for (int v = threadIdx.x; v < rows * (kD / 4); v += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = c0; c < p.nchunks; ++c) {
            const size_t slot = ((size_t)b * p.nchunks + c) * p.nkt + kt;
            const float4 x = reinterpret_cast<const float4 *>(part + slot * kRows * kD)[v];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        reinterpret_cast<float4 *>(dk + ((size_t)b * p.L + (size_t)kt * kRows) * kD)[v] = acc;
    }
}

// The problem shapes this path takes, and its parameters.
bool plan(const IndexerBwdProblem &pr, const DeviceInfo &info, Params &p) {
    if (pr.dt != DSA_BF16 || pr.d != kD) return false;
    if (!(pr.H == 32 || pr.H == 64 || pr.H == 128)) return false;
    if (info.cc_major != 10 || (size_t)info.max_smem_optin < kSmem) return false;
    if (((uintptr_t)pr.q_idx | (uintptr_t)pr.k_idx | (uintptr_t)pr.w | (uintptr_t)pr.grad) % 16 != 0) return false;
    if ((pr.dq && (uintptr_t)pr.dq % 16) || (pr.dk && (uintptr_t)pr.dk % 16)) return false;
    // 16-byte rows of g, and TMA boxes no larger than the tensors they read
    if (pr.L % 4 != 0 || pr.L < kRows) return false;
    // a TMA box may not be taller than the tensor it reads
    if ((long long)pr.B * pr.Tq * pr.H < kRows || (long long)pr.B * pr.L < kRows) return false;
    p.w = pr.w;
    p.grad = pr.grad;
    p.B = pr.B;
    p.Tq = pr.Tq;
    p.L = pr.L;
    p.q_pos0 = pr.q_pos0;
    p.H = pr.H;
    p.QPG = kRows / pr.H;
    p.ngroups = ceil_div(pr.Tq, p.QPG);
    p.nkt = ceil_div(pr.L, kRows);
    p.dq = pr.dq;
    p.dw = pr.dw;
    p.part = nullptr;
    // key side: chunks of C groups, about three units per SM in total
    long long visits = 0;  // (key tile, group) pairs per batch entry
    for (int kt = 0; kt < p.nkt; ++kt) {
        const int i = kt * kRows - pr.q_pos0;
        const int gf = i <= 0 ? 0 : i / p.QPG;
        if (gf < p.ngroups) visits += p.ngroups - gf;
    }
    long long C = (visits * pr.B + 3LL * info.sm_count - 1) / (3LL * info.sm_count);
    if (C < 8) C = 8;
    if (C > p.ngroups) C = p.ngroups;
    p.C = (int)C;
    p.nchunks = ceil_div(p.ngroups, p.C);
    return true;
}

size_t part_bytes(const Params &p) {
    return (size_t)p.B * p.nchunks * p.nkt * kRows * kD * sizeof(float);
}

}  // namespace

cudaError_t indexer_bwd_set_wait_limit(unsigned long long ns) { return set_wait_limit_ns(ns); }

unsigned int indexer_bwd_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_indexer_bwd_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_indexer_bwd_error, &zero, sizeof(zero));
    return v;
}

size_t indexer_bwd_tc_workspace_bytes(const IndexerBwdProblem &pr) {
    DeviceInfo info;
    if (device_info(&info) != cudaSuccess) return 0;
    Params p;
    if (!plan(pr, info, p)) return 0;
    return part_bytes(p);
}

cudaError_t launch_indexer_bwd_tc(const IndexerBwdProblem &pr, cudaStream_t stream, bool *taken) {
    *taken = false;
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    Params p;
    if (!plan(pr, info, p)) return cudaSuccess;
    if (pr.dk && (pr.ws == nullptr || pr.ws_bytes < part_bytes(p) || (uintptr_t)pr.ws % 16 != 0))
        return cudaSuccess;  // no room for the key side's partials: the CUDA-core path takes the call
    CUtensorMap tm_q, tm_k, tm_g, tm_w;
    const uint64_t rows = (uint64_t)pr.B * pr.Tq;
    if (!make_map_bf16_sw128(&tm_q, pr.q_idx, rows * pr.H, kD, kD * 2, kRows) ||
        !make_map_bf16_sw128(&tm_k, pr.k_idx, (uint64_t)pr.B * pr.L, kD, kD * 2, kRows) ||
        !make_map_f32(&tm_g, pr.grad, rows, (uint64_t)pr.L, (uint64_t)pr.L * 4, (uint32_t)p.QPG, kRows) ||
        !make_map_f32(&tm_w, pr.w, rows, (uint64_t)pr.H, (uint64_t)pr.H * 4, (uint32_t)p.QPG, (uint32_t)pr.H))
        return cudaSuccess;
    *taken = true;
    if (pr.dq || pr.dw) {
        Params q = p;
        q.units = p.B * p.ngroups;
        auto kern = pr.H == 32 ? indexer_bwd_tc_kernel<false, 32>
                               : (pr.H == 64 ? indexer_bwd_tc_kernel<false, 64> : indexer_bwd_tc_kernel<false, 128>);
        if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem)) !=
            cudaSuccess)
            return err;
        const int grid = q.units < info.sm_count ? q.units : info.sm_count;
        kern<<<grid, kThreads, kSmem, stream>>>(tm_q, tm_k, tm_g, tm_w, q);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (pr.dk) {
        Params k = p;
        k.part = static_cast<float *>(pr.ws);
        const long long units = (long long)p.B * p.nchunks * p.nkt;
        if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
        k.units = (int)units;
        auto kern = pr.H == 32 ? indexer_bwd_tc_kernel<true, 32>
                               : (pr.H == 64 ? indexer_bwd_tc_kernel<true, 64> : indexer_bwd_tc_kernel<true, 128>);
        if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem)) !=
            cudaSuccess)
            return err;
        const int grid = k.units < info.sm_count ? k.units : info.sm_count;
        kern<<<grid, kThreads, kSmem, stream>>>(tm_q, tm_k, tm_g, tm_w, k);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        indexer_bwd_reduce_kernel<<<dim3(p.nkt, p.B), 256, 0, stream>>>(k.part, k, pr.dk);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace dsa
