// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05).
//
//   I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]),  s <= t
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §2.1;
// "DeepSeek NSA and DSA" §3.2 for H=64 heads of width 128).
//
// The contraction over d is a GEMM with the KEYS on M and (query, head) pairs
// on N:  X[s, (i,j)] = sum_e K[s,e] * Q[(i,j),e].  One CTA tile is 128 keys by
// N_TILE = QPT * H columns (QPT queries of one batch entry), K = d. Putting
// keys on M gives every epilogue thread one key (one TMEM lane) and all heads
// of a query in its own registers, so the ReLU, the weights and the head sum
// need no cross-thread reduction, and the per-head scores never leave the SM.
//
// Warp roles (64 + 32 EPI threads, one CTA per SM, persistent over work units):
//   warp 0      TMA producer: Q tile of the unit once, then key tiles through
//               a K_STAGES-deep ring (128-byte swizzle, K-major).
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (bf16 in, fp32
//               accumulate) into the TMEM accumulators in turn (four when
//               4 * N_TILE columns fit, else two).
//   warps 2..   epilogue, EPI = 8 or 16 warps, EPI / 4 per TMEM lane quarter (each takes every
//               other query of the tile; with one query per tile, as in
//               decode, the groups take the accumulators in turn):
//               tcgen05.ld of the accumulator, ReLU, weight and head sum
//               with packed fp32x2 FMAs, one fp32 score per (query, key),
//               causal mask.
// The accumulators let the epilogue of tile n overlap the MMAs of the tiles
// after it. A work unit is (batch entry, query group, chunk of at most C key
// tiles); units are spread over the CTAs round-robin. Causal: a query group
// only visits key tiles up to its last query position.
//
// Exactness: integer-valued bf16 inputs give integer dot products far below
// 2^24, and power-of-two weights keep every partial sum exact in fp32, so the
// scores equal the exact result regardless of accumulation order.
#include <math.h>

#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kBlockM = 128;       // keys per tile (TMEM lanes)
// Epilogue warps: EPI = 16 (four per TMEM lane quarter) when a tile holds
// several queries (prefill), 8 (two per quarter, taking alternate tiles) for
// one query per tile (decode, where more warps only cost registers).
template <int EPI>
struct Threads {
    static constexpr int kEpilogue = EPI * 32;
    static constexpr int kAll = 64 + kEpilogue;  // + the TMA and MMA warps
};

// acc(lo, hi) += (a_lo * b_lo, a_hi * b_hi), two independent IEEE fp32 FMAs
__device__ __forceinline__ void fma2(uint64_t &acc, float a_lo, float a_hi, float b_lo, float b_hi) {
    uint64_t a, b;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a_lo), "f"(a_hi));
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b_lo), "f"(b_hi));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ float lo_f32(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f32(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
constexpr uint32_t kSmemBudget = 224 * 1024;

__device__ unsigned int g_indexer_error = 0;  // 1 = a bounded wait gave up

struct Params {
    const float *w;
    float *scores;
    int B, Tq, L, q_pos0, H, QPT, ngroups, G, C, units;
    int fill;
};

struct Unit {
    int b, i0, qcount, kt0, kt1;
};

// Work unit u -> (batch entry, query group, key-tile chunk). Chunk-major
// order; a unit whose chunk lies beyond the group's causal extent is empty.
__device__ __forceinline__ bool decode_unit(int u, const Params &p, Unit &un) {
    const int c_idx = u / p.G;
    const int g = u - c_idx * p.G;
    const int b = g / p.ngroups;
    const int qg = g - b * p.ngroups;
    const int i0 = qg * p.QPT;
    const int qcount = min(p.QPT, p.Tq - i0);
    const int t_max = p.q_pos0 + i0 + qcount - 1;
    const int nkt = t_max / kBlockM + 1;
    const int kt0 = c_idx * p.C;
    if (kt0 >= nkt) return false;
    un.b = b;
    un.i0 = i0;
    un.qcount = qcount;
    un.kt0 = kt0;
    un.kt1 = min(kt0 + p.C, nkt);
    return true;
}

template <int D, int N_TILE, bool FP8>
struct Cfg {
    static constexpr int kBoxElems = FP8 ? 128 : 64;                 // elements per 128-byte K slice
    static constexpr int kHalves = D / kBoxElems;                    // 128-byte K slices per row
    static constexpr uint32_t kQHalf = N_TILE * 128;
    static constexpr uint32_t kQBytes = kQHalf * kHalves;
    static constexpr uint32_t kKHalf = kBlockM * 128;
    static constexpr uint32_t kKBytes = kKHalf * kHalves;
    // query buffers: the producer runs at most kQBufs work units ahead of the
    // MMA (bf16 decode keeps it to a few tiles ahead, which measured fastest)
    static constexpr int kQBufs = 2;
    static constexpr int kStagesRaw = (int)((kSmemBudget - kQBufs * kQBytes) / kKBytes);
    // as many key stages as fit: with 16 KB e4m3 stages, 13 keep ~208 KB in flight
    static constexpr int kStages = kStagesRaw > 16 ? 16 : kStagesRaw;
    // accumulator buffers in TMEM: four when they fit (the MMA runs further
    // ahead of the epilogue), else two
    static constexpr int kAcc = 4 * N_TILE <= 512 ? 4 : 2;
    static constexpr uint32_t kTmemCols = kAcc * N_TILE;
    static constexpr int kBars = 2 * kStages + 2 * kQBufs + 2 * kAcc + 1;
    static constexpr size_t kSmem = 1024 + (size_t)kQBufs * kQBytes + (size_t)kStages * kKBytes + kBars * 8 + 16;
    static_assert(kStages >= 2, "shared memory too small for the pipeline");
    static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "TMEM columns");
};

template <int D, int N_TILE, bool FP8, int EPI>
__global__ void __launch_bounds__(Threads<EPI>::kAll, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const Params p) {
    using C = Cfg<D, N_TILE, FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *q_sm = smem;
    uint8_t *k_sm = q_sm + C::kQBufs * C::kQBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(k_sm + C::kStages * C::kKBytes);
    uint64_t *k_full = bars;
    uint64_t *k_empty = k_full + C::kStages;
    uint64_t *q_full = k_empty + C::kStages;
    uint64_t *q_empty = q_full + C::kQBufs;
    uint64_t *acc_full = q_empty + C::kQBufs;
    uint64_t *acc_empty = acc_full + C::kAcc;
    uint64_t *drained = acc_empty + C::kAcc;  // MMA commit at teardown
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drained + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::kQBufs; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        // one query per tile (decode): each tile is taken by one group of
        // four warps (one per TMEM lane quarter), the groups taking the
        // accumulator buffers in turn; else every epilogue warp works on
        // every tile (its share of the queries)
        const int releasers = p.QPT == 1 ? 128 : Threads<EPI>::kEpilogue;
        for (int s = 0; s < C::kAcc; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], releasers);
        }
        mbar_init(drained, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    bool ok = waits_enabled();  // false: the wait limit is 0 (give-up test)

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            prefetch_tensor_map(&tm_q);
            prefetch_tensor_map(&tm_k);
            int ks = 0, qb = 0;
            uint32_t kph = 0, qph = 0;
            // stages and query buffers armed at least once, and the parity of
            // their last arming (drained before the CTA exits)
            uint32_t k_armed = 0, k_par = 0, q_armed = 0, q_par = 0;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                Unit un;
                if (!decode_unit(u, p, un)) continue;
                if (!mbar_wait(&q_empty[qb], qph ^ 1u)) { ok = false; break; }
                q_armed |= 1u << qb;
                q_par = (q_par & ~(1u << qb)) | (qph << qb);
                mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
                const int qrow = (un.b * p.Tq + un.i0) * p.H;
#pragma unroll
                for (int h = 0; h < C::kHalves; ++h)
                    tma_load_2d(q_sm + qb * C::kQBytes + h * C::kQHalf, &tm_q, &q_full[qb], h * C::kBoxElems, qrow);
                if (++qb == C::kQBufs) { qb = 0; qph ^= 1u; }
                for (int kt = un.kt0; kt < un.kt1; ++kt) {
                    if (!mbar_wait(&k_empty[ks], kph ^ 1u)) { ok = false; break; }
                    k_armed |= 1u << ks;
                    k_par = (k_par & ~(1u << ks)) | (kph << ks);
                    mbar_arrive_expect_tx(&k_full[ks], C::kKBytes);
                    const int krow = un.b * p.L + kt * kBlockM;
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h)
                        tma_load_2d(k_sm + ks * C::kKBytes + h * C::kKHalf, &tm_k, &k_full[ks], h * C::kBoxElems, krow);
                    if (++ks == C::kStages) { ks = 0; kph ^= 1u; }
                }
            }
            // every TMA load this CTA issued has landed before it exits (on
            // the normal path these phases were consumed already)
            for (int s = 0; s < C::kStages; ++s)
                if (((k_armed >> s) & 1u) && !mbar_drain(&k_full[s], (k_par >> s) & 1u)) ok = false;
            for (int s = 0; s < C::kQBufs; ++s)
                if (((q_armed >> s) & 1u) && !mbar_drain(&q_full[s], (q_par >> s) & 1u)) ok = false;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            int ks = 0, qb = 0, ab = 0;
            uint32_t kph = 0, qph = 0, aph = 0;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                Unit un;
                if (!decode_unit(u, p, un)) continue;
                if (!mbar_wait(&q_full[qb], qph)) { ok = false; break; }
                tc_fence_after();
                const uint32_t idesc = FP8 ? idesc_e4m3_f32(kBlockM, un.qcount * p.H)
                                           : idesc_bf16_f32(kBlockM, un.qcount * p.H);
                const uint32_t q_base = smem_addr(q_sm + qb * C::kQBytes);
                for (int kt = un.kt0; kt < un.kt1; ++kt) {
                    if (!mbar_wait(&k_full[ks], kph)) { ok = false; break; }
                    if (!mbar_wait(&acc_empty[ab], aph ^ 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(ab * N_TILE);
                    // descriptors of the stage and query buffer once; each MMA
                    // advances their start-address field (bytes / 16, 14 bits,
                    // no carry below 256 KB of shared memory)
                    const uint64_t a0 = smem_desc_k_sw128(smem_addr(k_sm + ks * C::kKBytes));
                    const uint64_t b0 = smem_desc_k_sw128(q_base);
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {  // 4 MMAs of 32 bytes of K per 128-byte swizzle row
                            const uint64_t a = a0 + (uint64_t)((h * C::kKHalf + kk * 32) >> 4);
                            const uint64_t b = b0 + (uint64_t)((h * C::kQHalf + kk * 32) >> 4);
                            if constexpr (FP8)
                                mma_f8_ss(d_tmem, a, b, idesc, (h | kk) != 0);
                            else
                                mma_f16_ss(d_tmem, a, b, idesc, (h | kk) != 0);
                        }
                    }
                    mma_commit(&k_empty[ks]);   // key stage free once these MMAs finish
                    mma_commit(&acc_full[ab]);  // accumulator ready for the epilogue
                    if (++ks == C::kStages) { ks = 0; kph ^= 1u; }
                    if (++ab == C::kAcc) { ab = 0; aph ^= 1u; }
                }
                if (!ok) break;
                mma_commit(&q_empty[qb]);
                if (++qb == C::kQBufs) { qb = 0; qph ^= 1u; }
            }
            // no MMA of this CTA may still run when TMEM is freed
            mma_commit(drained);
            if (!mbar_drain(drained, 0)) ok = false;
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int quarter = warp & 3;                 // TMEM lanes this warp may read
        const int half = (warp - 2) >> 2;             // the warp's group: its share of the tiles' work
        const bool by_tile = p.QPT == 1;              // decode: accumulator `half` only (groups 0, 1)
        const int q_first = by_tile ? 0 : half;       // else queries half, half + EPI / 4, ...
        const int q_step = by_tile ? 1 : EPI / 4;
        const int key_in_tile = quarter * 32 + lane;  // TMEM lane = key
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        int ab = 0;
        uint32_t aph = 0;
        // the query's score of this thread's key from a tile's 64 head columns
        // (x) and weights (wr), in the same order as the general loop below
        auto head_sum64 = [](const uint32_t *x, const float4 *wr) -> float {
            uint64_t part[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float r0 = fmaxf(__uint_as_float(x[4 * j + 0]), 0.0f);
                const float r1 = fmaxf(__uint_as_float(x[4 * j + 1]), 0.0f);
                const float r2 = fmaxf(__uint_as_float(x[4 * j + 2]), 0.0f);
                const float r3 = fmaxf(__uint_as_float(x[4 * j + 3]), 0.0f);
                fma2(part[(2 * j) & 3], wr[j].x, wr[j].y, r0, r1);
                fma2(part[(2 * j + 1) & 3], wr[j].z, wr[j].w, r2, r3);
            }
            return (lo_f32(part[0]) + hi_f32(part[0]) + (lo_f32(part[1]) + hi_f32(part[1]))) +
                   (lo_f32(part[2]) + hi_f32(part[2]) + (lo_f32(part[3]) + hi_f32(part[3])));
        };
        // Decode with 64 indexer heads (one query per tile): the query's
        // weights stay in registers for the whole work unit, and both halves
        // of the accumulator are loaded before one wait.
        const bool decode64 = EPI == 8 && N_TILE == 64 && p.H == 64;
        for (int u = blockIdx.x; ok && decode64 && u < p.units; u += gridDim.x) {
            Unit un;
            if (!decode_unit(u, p, un)) continue;
            const size_t row0 = (size_t)un.b * p.Tq + un.i0;
            float4 wr[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) wr[j] = __ldg(reinterpret_cast<const float4 *>(p.w + row0 * 64) + j);
            const int t = p.q_pos0 + un.i0;
            float *dst_row = p.scores + row0 * (size_t)p.L;
            for (int kt = un.kt0; kt < un.kt1; ++kt) {
                if (ab % (EPI / 4) != half) {  // another warp of the quarter takes this tile
                    if (++ab == C::kAcc) { ab = 0; aph ^= 1u; }
                    continue;
                }
                if (!mbar_wait(&acc_full[ab], aph)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tbase = tmem_base + lane_addr + (uint32_t)(ab * N_TILE);
                uint32_t x[64];
                tmem_ld_32x32b_x32(tbase, x);
                tmem_ld_32x32b_x32(tbase + 32, x + 32);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&acc_empty[ab]);  // the accumulator is in registers
                if (++ab == C::kAcc) { ab = 0; aph ^= 1u; }
                const float acc = head_sum64(x, wr);
                const int s = kt * kBlockM + key_in_tile;
                if (s < p.L) {
                    if (s <= t) {
                        dst_row[s] = acc;
                    } else if (p.fill) {
                        dst_row[s] = -INFINITY;
                    }
                }
            }
        }
        for (int u = blockIdx.x; ok && !decode64 && u < p.units; u += gridDim.x) {
            Unit un;
            if (!decode_unit(u, p, un)) continue;
            const size_t row0 = (size_t)un.b * p.Tq + un.i0;
            const float4 *w4 = reinterpret_cast<const float4 *>(p.w + row0 * p.H);
            for (int kt = un.kt0; kt < un.kt1; ++kt) {
                if (by_tile && ab % (EPI / 4) != half) {  // another warp of the quarter takes this tile
                    if (++ab == C::kAcc) { ab = 0; aph ^= 1u; }
                    continue;
                }
                if (!mbar_wait(&acc_full[ab], aph)) { ok = false; break; }
                tc_fence_after();
                const int s = kt * kBlockM + key_in_tile;
                const uint32_t tbase = tmem_base + lane_addr + (uint32_t)(ab * N_TILE);
                for (int q = q_first; q < un.qcount; q += q_step) {
                    // four independent packed (f32x2) partial sums
                    uint64_t part[4] = {0ull, 0ull, 0ull, 0ull};
                    for (int c = 0; c < p.H; c += 32) {
                        uint32_t x[32];
                        tmem_ld_32x32b_x32(tbase + (uint32_t)(q * p.H + c), x);
                        tmem_ld_wait();
                        const float4 *wq = w4 + (q * p.H + c) / 4;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float4 wv = __ldg(wq + j);
                            const float r0 = fmaxf(__uint_as_float(x[4 * j + 0]), 0.0f);
                            const float r1 = fmaxf(__uint_as_float(x[4 * j + 1]), 0.0f);
                            const float r2 = fmaxf(__uint_as_float(x[4 * j + 2]), 0.0f);
                            const float r3 = fmaxf(__uint_as_float(x[4 * j + 3]), 0.0f);
                            fma2(part[(2 * j) & 3], wv.x, wv.y, r0, r1);
                            fma2(part[(2 * j + 1) & 3], wv.z, wv.w, r2, r3);
                        }
                    }
                    const float acc = (lo_f32(part[0]) + hi_f32(part[0]) + (lo_f32(part[1]) + hi_f32(part[1]))) +
                                      (lo_f32(part[2]) + hi_f32(part[2]) + (lo_f32(part[3]) + hi_f32(part[3])));
                    const int t = p.q_pos0 + un.i0 + q;
                    if (s < p.L) {
                        float *dst = p.scores + (row0 + q) * (size_t)p.L + s;
                        if (s <= t) {
                            *dst = acc;
                        } else if (p.fill) {
                            *dst = -INFINITY;
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&acc_empty[ab]);
                if (++ab == C::kAcc) { ab = 0; aph ^= 1u; }
            }
        }
    }

    if (!ok) atomicOr(&g_indexer_error, kErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// -inf for the keys of row t beyond the key tiles the GEMM visits.
__global__ void fill_beyond_tiles_kernel(float *__restrict__ scores, int Tq, int L, int q_pos0) {
    const int row = blockIdx.x;
    const int t = q_pos0 + row % Tq;
    const int start = (t / kBlockM + 1) * kBlockM;
    float *out = scores + (size_t)row * L;
    for (int s = start + threadIdx.x; s < L; s += blockDim.x) out[s] = -INFINITY;
}

template <int D, int N_TILE, bool FP8, int EPI>
cudaError_t launch_tc(const IndexerProblem &pr, const DeviceInfo &info, cudaStream_t stream) {
    using C = Cfg<D, N_TILE, FP8>;
    if ((size_t)info.max_smem_optin < C::kSmem) return cudaErrorInvalidValue;
    CUtensorMap tm_q, tm_k;
    auto make = FP8 ? make_map_u8_sw128 : make_map_bf16_sw128;
    const uint64_t pitch = (uint64_t)D * (FP8 ? 1 : 2);
    if (!make(&tm_q, pr.q_idx, (uint64_t)pr.B * pr.Tq * pr.H, (uint64_t)D, pitch, N_TILE) ||
        !make(&tm_k, pr.k_idx, (uint64_t)pr.B * pr.L, (uint64_t)D, pitch, kBlockM))
        return cudaErrorInvalidValue;

    Params p;
    p.w = pr.w;
    p.scores = pr.scores;
    p.B = pr.B; p.Tq = pr.Tq; p.L = pr.L; p.q_pos0 = pr.q_pos0; p.H = pr.H;
    p.QPT = N_TILE / pr.H;
    p.ngroups = ceil_div(pr.Tq, p.QPT);
    p.G = pr.B * p.ngroups;
    p.fill = pr.fill_masked ? 1 : 0;
    // total key tiles over all groups, to size the chunks
    long long tiles = 0;
    int nkt_max = 0;
    for (int g = 0; g < p.ngroups; ++g) {
        const int qcount = pr.Tq - g * p.QPT < p.QPT ? pr.Tq - g * p.QPT : p.QPT;
        const int nkt = (pr.q_pos0 + g * p.QPT + qcount - 1) / kBlockM + 1;
        tiles += nkt;
        nkt_max = nkt > nkt_max ? nkt : nkt_max;
    }
    tiles *= pr.B;
    // Units per CTA: about 8 when the query tile is 64 KB (prefill: each unit
    // reloads its query tile). Decode: about 32 for bf16 keys (2-tile units;
    // the query buffers then hold the producer to a few tiles ahead, and the
    // deeper key ring that longer units allow measured slower), about 8 for
    // e4m3 keys, whose 16 KB tiles arrive twice as often: with 2-tile units
    // the MMA thread's per-unit work (unit decode, query wait and release)
    // set the pace at ~0.5 us per tile.
    const long long units_per_cta = pr.Tq == 1 ? (FP8 ? 8 : 32) : 8;
    long long chunk = (tiles + (long long)info.sm_count * units_per_cta - 1) / ((long long)info.sm_count * units_per_cta);
    p.C = (int)(chunk < 1 ? 1 : (chunk > 64 ? 64 : chunk));
    const long long units = (long long)ceil_div(nkt_max, p.C) * p.G;
    if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.units = (int)units;

    auto kern = indexer_tc_kernel<D, N_TILE, FP8, EPI>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (err != cudaSuccess) return err;
    const int grid = p.units < info.sm_count ? p.units : info.sm_count;
    kern<<<grid, Threads<EPI>::kAll, C::kSmem, stream>>>(tm_q, tm_k, p);
    count_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // the first row (t = q_pos0) has the fewest tiles; when its tiles reach L,
    // no row has keys beyond them (decode) and the fill would write nothing
    if (pr.fill_masked && (long long)(pr.q_pos0 / kBlockM + 1) * kBlockM < pr.L) {
        fill_beyond_tiles_kernel<<<pr.B * pr.Tq, 256, 0, stream>>>(pr.scores, pr.Tq, pr.L, pr.q_pos0);
        count_launch();
        err = cudaGetLastError();
    }
    return err;
}

template <int EPI>
cudaError_t dispatch_tc(const IndexerProblem &p, const DeviceInfo &info, cudaStream_t stream, bool fp8, int n_tile) {
    if (fp8) {
        if (n_tile == 64) return launch_tc<128, 64, true, EPI>(p, info, stream);
        if (n_tile == 128) return launch_tc<128, 128, true, EPI>(p, info, stream);
        return launch_tc<128, 256, true, EPI>(p, info, stream);
    }
    if (p.d == 128) {
        if (n_tile == 64) return launch_tc<128, 64, false, EPI>(p, info, stream);
        if (n_tile == 128) return launch_tc<128, 128, false, EPI>(p, info, stream);
        return launch_tc<128, 256, false, EPI>(p, info, stream);
    }
    if (n_tile == 64) return launch_tc<64, 64, false, EPI>(p, info, stream);
    if (n_tile == 128) return launch_tc<64, 128, false, EPI>(p, info, stream);
    return launch_tc<64, 256, false, EPI>(p, info, stream);
}

}  // namespace

cudaError_t indexer_set_wait_limit(unsigned long long ns) { return set_wait_limit_ns(ns); }

unsigned int indexer_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_indexer_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_indexer_error, &zero, sizeof(zero));
    return v;
}

cudaError_t launch_indexer_tc(const IndexerProblem &p, cudaStream_t stream, bool *taken) {
    *taken = false;
    // bf16 rows of 64 or 128 elements; e4m3 rows of 128 (one 128-byte slice)
    const bool fp8 = p.dt == DSA_E4M3;
    if (p.dt != DSA_BF16 && !fp8) return cudaSuccess;
    if (!(p.d == 128 || (p.d == 64 && !fp8))) return cudaSuccess;
    if (!(p.H == 32 || p.H == 64 || p.H == 128)) return cudaSuccess;
    if (((uintptr_t)p.q_idx | (uintptr_t)p.k_idx | (uintptr_t)p.w) % 16 != 0) return cudaSuccess;
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    if (info.cc_major != 10) return cudaSuccess;
    // queries per tile: as many as fit 256 columns, but no more than the rows
    int qpt = 256 / p.H;
    if (p.Tq < qpt) qpt = p.Tq;
    int n = qpt * p.H;
    const int n_tile = n <= 64 ? 64 : (n <= 128 ? 128 : 256);
    // a TMA box may not be taller than the tensor it reads
    if ((long long)p.B * p.Tq * p.H < n_tile || (long long)p.B * p.L < kBlockM) return cudaSuccess;
    *taken = true;
    // one query per tile (decode): 8 epilogue warps, else 16
    if (qpt == 1) return dispatch_tc<8>(p, info, stream, fp8, n_tile);
    return dispatch_tc<16>(p, info, stream, fp8, n_tile);
}

}  // namespace dsa
