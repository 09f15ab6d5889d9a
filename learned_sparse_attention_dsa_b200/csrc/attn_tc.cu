// Sparse attention on tensor cores for groups of 16 query heads that share
// one KV head (the MQA mode of MLA: "DeepSeek Sparse Attention: Learned
// Token Selection from Scratch" §4.1-4.2; "Sparse Attention LLM Design ...",
// "Implemented on MLA's MQA mode").
//
//   u[t,h] = sum_{s in S_t} softmax_s(scale * q[t,h] . k[s]) v[s]   (§3.3, §10.1)
//
// One CTA owns (query row, group of 16 heads, split of the selected list).
// The selected positions are compacted in shared memory (padding dropped),
// then gathered 64 at a time -- K and V rows -- with 16-byte cp.async into a
// multi-stage ring (16-byte chunks XOR-swizzled by row so that ldmatrix reads
// are conflict-free). Each of the four warps takes 16 of the 64 rows:
// S = Q K^T with mma.sync m16n8k16 (bf16 in, fp32 accumulate; Q stays in
// registers), an online softmax in fp32 (exp2 with the log2(e) prescale, as in
// FlashAttention), and O += P V with P re-packed from the S accumulators as
// the A operand. The four warps' (max, sum, O) are merged at the end. With a
// split selected list, up to eight splits form a thread-block cluster and
// merge through distributed shared memory (each split stores its share of
// every owner's output slice there, then one cluster barrier); more splits
// write fp32 partials that a combine kernel merges. Every selected row is
// loaded once for all 16 heads.
#include <math.h>

#include <cooperative_groups.h>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dsa {

cudaError_t launch_attn_cuda_core(const AttnProblem &p, cudaStream_t stream);

namespace {

__device__ unsigned int g_attn_tc_error = 0;  // kErrBadIndex bits

constexpr int kRowsPerTile = 64;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kHeads = 16;
constexpr float kLog2e = 1.4426950408889634f;

// ROWS selected rows per pipeline stage: 64 (each warp 16 rows), or 32 (each
// warp 8 rows) for wide rows without splits, where three 68 KB CTAs per SM
// keep more copies in flight than two 88 KB ones.
template <int DQK, int DV, int ROWS>
struct Cfg {
    static constexpr int kKChunks = DQK / 8;  // 16-byte chunks per K row
    static constexpr int kVChunks = DV / 8;
    static constexpr int kKBytes = ROWS * DQK * 2;
    static constexpr int kVBytes = ROWS * DV * 2;
    static constexpr int kStageBytes = kKBytes + kVBytes;
    static constexpr int kStages = ROWS == 32 ? 3 : ((DQK + DV) > 256 ? 2 : 3);
    static constexpr int kMaxSel = 2048;  // selected entries one CTA handles
    // four warps' (O, m, l), then the CTA's merged (O, m, l) for the cluster merge
    // (plus one merge weight per split and head)
    static constexpr int kMergeBytes = (kWarps + 1) * kHeads * (DV + 10) * 4 + 8 * kHeads * 4;
    static constexpr int kPipeBytes = kStages * kStageBytes;
    static constexpr size_t kRegion = (size_t)(kPipeBytes > kMergeBytes ? kPipeBytes : kMergeBytes);
    static constexpr size_t kSmem = kRegion + kMaxSel * 4 + 64;
    // with the cluster merge: the selection list of one split, then the
    // receive area of this CTA's output slice from every split (P <= 8)
    static constexpr int kQuads = kHeads * DV / 4;
    static size_t cluster_smem(int splits, int per_split) {
        const int per = (kQuads + splits - 1) / splits;
        return kRegion + (size_t)per_split * 4 + (size_t)splits * per * 16 + (size_t)splits * kHeads * 8 + 64;
    }
    static constexpr size_t kSmemMax = kSmem + (size_t)(kQuads + 8) * 16 + 8 * kHeads * 8;
};

struct Args {
    const __nv_bfloat16 *q, *k_cache, *v_cache;
    const int32_t *idx;
    int Tq, L, k, Hq, Hkv, splits, per_split;
    float scale_log2;
    int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
    __nv_bfloat16 *out;
    float *lse;
    float *part_o;   // [rows, Hq, splits, DV] when splits > 1
    float *part_ml;  // [rows, Hq, splits, 2]
    int cluster_merge;  // splits merged inside their cluster (no workspace)
};

// Up to eight splits (a portable cluster) merge through distributed shared
// memory; more splits go through the workspace and the combine kernel.
inline bool uses_cluster_merge(int splits) { return splits > 1 && splits <= 8; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;  // 0 source bytes: the 16 bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// m16n8k8: A 16 x 8 (two registers), B 8 x 8 (one register)
__device__ __forceinline__ void mma_bf16_k8(float *c, const uint32_t *a, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(b0));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int DQK, int DV, int ROWS>
__global__ void __launch_bounds__(kThreads, ROWS == 32 ? 3 : 1)
attn_mma_kernel(const Args a) {
    using C = Cfg<DQK, DV, ROWS>;
    constexpr int NT = ROWS / 32;  // 8-row n-tiles of S per warp
    constexpr int WR = ROWS / 4;   // rows of a stage per warp
    // cluster merge: this CTA has started (waited on before any other CTA
    // stores into its shared memory)
    if (a.cluster_merge) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    extern __shared__ __align__(128) uint8_t smem[];
    int32_t *sel = reinterpret_cast<int32_t *>(smem + (C::kPipeBytes > C::kMergeBytes ? C::kPipeBytes
                                                                                        : C::kMergeBytes));
    __shared__ int s_count;

    const int row = blockIdx.x;                 // flat query row b*Tq + i
    const int hgroup = blockIdx.y;              // 16-head group
    const int split = blockIdx.z;
    const int b = row / a.Tq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h0 = hgroup * kHeads;
    const int g = h0 / (a.Hq / a.Hkv);

    // ---- this split's selected positions first: the gathers wait for them.
    // When every entry is a position in [0, L) (decode) they are used as
    // they are; otherwise the valid ones are compacted (order kept).
    const int j0 = split * a.per_split;
    const int j1 = min(a.k, j0 + a.per_split);
    {
        __shared__ int warp_base[kWarps];
        // all of this split's entries are loaded up front: one memory latency
        constexpr int kIters = C::kMaxSel / kThreads;
        int sv[kIters];
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            const int j = j0 + it * kThreads + threadIdx.x;
            sv[it] = j < j1 ? __ldg(a.idx + (size_t)row * a.k + j) : -1;
        }
        bool mine_valid = true;
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            if (j0 + it * kThreads + (int)threadIdx.x < j1) {
                note_bad_index(&g_attn_tc_error, sv[it], a.L);
                mine_valid = mine_valid && sv[it] >= 0 && sv[it] < a.L;
            }
        }
        if (__syncthreads_and(mine_valid ? 1 : 0)) {
#pragma unroll
            for (int it = 0; it < kIters; ++it) {
                const int j = it * kThreads + threadIdx.x;
                if (j0 + j < j1) sel[j] = sv[it];
            }
            if (threadIdx.x == 0) s_count = j1 - j0;
        } else {
            int base = 0;
#pragma unroll
            for (int it = 0; it < kIters; ++it) {
                if (j0 + it * kThreads >= j1) break;  // uniform
                const int s = sv[it];
                const bool valid = s >= 0 && s < a.L;
                const unsigned m = __ballot_sync(0xffffffffu, valid);
                if (lane == 0) warp_base[warp] = __popc(m);
                __syncthreads();
                int off = base;
                for (int w = 0; w < warp; ++w) off += warp_base[w];
                if (valid) sel[off + __popc(m & ((1u << lane) - 1u))] = s;
                int tot = 0;
                for (int w = 0; w < kWarps; ++w) tot += warp_base[w];
                base += tot;
                __syncthreads();
            }
            if (threadIdx.x == 0) s_count = base;
        }
    }
    __syncthreads();
    const int n_sel = s_count;
    const int n_tiles = (n_sel + ROWS - 1) / ROWS;

    const __nv_bfloat16 *kbase = a.k_cache + b * a.k_sb + g * a.k_sh;
    const __nv_bfloat16 *vbase = a.v_cache + b * a.v_sb + g * a.v_sh;
    const uint32_t smem_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));

    // Copies: K rows, then V rows; for each, thread i moves the fixed 16-byte
    // chunk column i % C of rows r0, r0 + R, ... (C chunks per row, R =
    // kThreads / C rows per pass; threads beyond R * C idle for that part).
    auto issue_rows = [&](uint32_t dst0, const __nv_bfloat16 *base, int64_t ss, int tile, auto chunks_c) {
        constexpr int CH = decltype(chunks_c)::value;
        constexpr int R = kThreads / CH;
        const int ch = threadIdx.x % CH, r0 = threadIdx.x / CH;
        if (r0 >= R) return;
        const __nv_bfloat16 *src0 = base + ch * 8;
#pragma unroll 4
        for (int r = r0; r < ROWS; r += R) {
            const int jj = tile * ROWS + r;
            const bool valid = jj < n_sel;
            const int s = valid ? sel[jj] : 0;
            cp_async16(dst0 + r * (CH * 16) + ((ch ^ (r & 7)) << 4), src0 + (int64_t)s * ss, valid);
        }
    };
    auto issue_tile = [&](int tile, int stage) {
        const uint32_t kdst = smem_base + stage * C::kStageBytes;
        issue_rows(kdst, kbase, a.k_ss, tile, std::integral_constant<int, C::kKChunks>{});
        issue_rows(kdst + C::kKBytes, vbase, a.v_ss, tile, std::integral_constant<int, C::kVChunks>{});
    };

    float o[DV / 8][4];
#pragma unroll
    for (int n = 0; n < DV / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
    float m_r[2] = {-INFINITY, -INFINITY};  // running max of heads lane/4 and lane/4+8 (log2 units)
    float l_r[2] = {0.0f, 0.0f};            // this thread's partial running sums

    // ---- pipeline prologue
#pragma unroll
    for (int st = 0; st < C::kStages - 1; ++st) {
        if (st < n_tiles) issue_tile(st, st);
        cp_async_commit();
    }

    // ---- Q fragments (A operand, 16 heads x DQK) straight from global
    // memory, while the first tiles are in flight
    uint32_t qf[DQK / 16][4];
    {
        const int hr = lane >> 2, kc = (lane & 3) * 2;
        const __nv_bfloat16 *q0 = a.q + ((size_t)row * a.Hq + h0 + hr) * DQK;
        const __nv_bfloat16 *q8 = q0 + 8 * DQK;
#pragma unroll
        for (int kk = 0; kk < DQK / 16; ++kk) {
            qf[kk][0] = *reinterpret_cast<const uint32_t *>(q0 + kk * 16 + kc);
            qf[kk][1] = *reinterpret_cast<const uint32_t *>(q8 + kk * 16 + kc);
            qf[kk][2] = *reinterpret_cast<const uint32_t *>(q0 + kk * 16 + 8 + kc);
            qf[kk][3] = *reinterpret_cast<const uint32_t *>(q8 + kk * 16 + 8 + kc);
        }
    }

    for (int tile = 0; tile < n_tiles; ++tile) {
        const int stage = tile % C::kStages;
        {
            const int next = tile + C::kStages - 1;
            if (next < n_tiles) issue_tile(next, next % C::kStages);
            cp_async_commit();
        }
        cp_async_wait<C::kStages - 1>();
        __syncthreads();

        const uint32_t kt = smem_base + stage * C::kStageBytes;
        const uint32_t vt = kt + C::kKBytes;

        // S = Q K^T for this warp's WR rows (NT n-tiles of 8 rows)
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
        if constexpr (NT == 2) {
            const int r = warp * 16 + (lane & 7) + ((lane >> 4) << 3);
            const uint32_t rbase = kt + r * (DQK * 2);
            const int rx = r & 7;
#pragma unroll
            for (int kk = 0; kk < DQK / 16; ++kk) {
                const int ch = 2 * kk + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(rbase + ((ch ^ rx) << 4), b0, b1, b2, b3);
                mma_bf16(s[0], qf[kk], b0, b1);
                mma_bf16(s[1], qf[kk], b2, b3);
            }
        } else {
            // 8 rows: one ldmatrix.x4 covers two 16-wide k-steps
            const int r = warp * 8 + (lane & 7);
            const uint32_t rbase = kt + r * (DQK * 2);
            const int rx = r & 7;
#pragma unroll
            for (int kk = 0; kk < DQK / 16; kk += 2) {
                const int ch = 2 * kk + (lane >> 3);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(rbase + ((ch ^ rx) << 4), b0, b1, b2, b3);
                mma_bf16(s[0], qf[kk], b0, b1);
                mma_bf16(s[0], qf[kk + 1], b2, b3);
            }
        }
        // mask rows beyond the selected count, scale into log2 units
        const int valid_rows = n_sel - tile * ROWS;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int rr = warp * WR + nt * 8 + (lane & 3) * 2 + (e & 1);
                s[nt][e] = rr < valid_rows ? s[nt][e] * a.scale_log2 : -INFINITY;
            }
        }
        // online softmax update for heads lane/4 (e = 0,1) and lane/4+8 (e = 2,3)
        float p[NT][4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float mx = fmaxf(s[0][2 * hh], s[0][2 * hh + 1]);
#pragma unroll
            for (int nt = 1; nt < NT; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * hh], s[nt][2 * hh + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_r[hh], mx);
            const float corr = m_new == -INFINITY ? 1.0f : ex2_approx(m_r[hh] - m_new);
            const float mr = m_new == -INFINITY ? 0.0f : m_new;  // masked entries: 2^-inf = 0
            float sum = 0.0f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float v = s[nt][2 * hh + e];
                    const float pv = ex2_approx(v - mr);
                    p[nt][2 * hh + e] = pv;
                    sum += pv;
                }
            }
            l_r[hh] = l_r[hh] * corr + sum;
            m_r[hh] = m_new;
#pragma unroll
            for (int n = 0; n < DV / 8; ++n) {
                o[n][2 * hh] *= corr;
                o[n][2 * hh + 1] *= corr;
            }
        }
        // O += P V: P (16 heads x WR rows) as the A operand
        if constexpr (NT == 2) {
            uint32_t pa[4];
            pa[0] = pack_bf16(p[0][0], p[0][1]);
            pa[1] = pack_bf16(p[0][2], p[0][3]);
            pa[2] = pack_bf16(p[1][0], p[1][1]);
            pa[3] = pack_bf16(p[1][2], p[1][3]);
            const int r = warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
            const uint32_t rbase = vt + r * (DV * 2);
            const int rx = r & 7;
#pragma unroll
            for (int nn = 0; nn < DV / 16; ++nn) {
                const int ch = 2 * nn + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(rbase + ((ch ^ rx) << 4), b0, b1, b2, b3);
                mma_bf16(o[2 * nn], pa, b0, b1);
                mma_bf16(o[2 * nn + 1], pa, b2, b3);
            }
        } else {
            // 8 rows: k = 8 MMAs; one transposed ldmatrix.x4 gives four 8-column n-tiles
            uint32_t pa[2];
            pa[0] = pack_bf16(p[0][0], p[0][1]);
            pa[1] = pack_bf16(p[0][2], p[0][3]);
            const int r = warp * 8 + (lane & 7);
            const uint32_t rbase = vt + r * (DV * 2);
            const int rx = r & 7;
#pragma unroll
            for (int nn = 0; nn < DV / 32; ++nn) {
                const int ch = 4 * nn + (lane >> 3);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(rbase + ((ch ^ rx) << 4), b0, b1, b2, b3);
                mma_bf16_k8(o[4 * nn + 0], pa, b0);
                mma_bf16_k8(o[4 * nn + 1], pa, b1);
                mma_bf16_k8(o[4 * nn + 2], pa, b2);
                mma_bf16_k8(o[4 * nn + 3], pa, b3);
            }
        }
        __syncthreads();  // this stage may be refilled next iteration
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- merge the four warps: full row sums, then (m, l, O) across warps
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l_r[hh] += __shfl_xor_sync(0xffffffffu, l_r[hh], 1);
        l_r[hh] += __shfl_xor_sync(0xffffffffu, l_r[hh], 2);
    }
    // rows of DV + 8 floats: the float2 stores below and the column reads
    // after them hit distinct banks
    constexpr int kRowF = DV + 8;
    float *mrg_o = reinterpret_cast<float *>(smem);                    // [warp][16][kRowF]
    float *mrg_ml = mrg_o + kWarps * kHeads * kRowF;                   // [warp][16][2]
    {
        const int hr = lane >> 2, cc = (lane & 3) * 2;
#pragma unroll
        for (int n = 0; n < DV / 8; ++n) {
            *reinterpret_cast<float2 *>(mrg_o + ((warp * kHeads + hr) * kRowF) + n * 8 + cc) =
                make_float2(o[n][0], o[n][1]);
            *reinterpret_cast<float2 *>(mrg_o + ((warp * kHeads + hr + 8) * kRowF) + n * 8 + cc) =
                make_float2(o[n][2], o[n][3]);
        }
        if ((lane & 3) == 0) {
            mrg_ml[(warp * kHeads + hr) * 2 + 0] = m_r[0];
            mrg_ml[(warp * kHeads + hr) * 2 + 1] = l_r[0];
            mrg_ml[(warp * kHeads + hr + 8) * 2 + 0] = m_r[1];
            mrg_ml[(warp * kHeads + hr + 8) * 2 + 1] = l_r[1];
        }
    }
    __syncthreads();
    // thread t handles head t / 8 and columns (t % 8) + 8 * c
    const int hh = threadIdx.x >> 3;
    const int c0 = threadIdx.x & 7;
    float mw[kWarps], m_all = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        mw[w] = mrg_ml[(w * kHeads + hh) * 2];
        m_all = fmaxf(m_all, mw[w]);
    }
    float fw[kWarps], l_all = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        fw[w] = m_all == -INFINITY ? 0.0f : ex2_approx(mw[w] - m_all);
        l_all += fw[w] * mrg_ml[(w * kHeads + hh) * 2 + 1];
    }
    const int h = h0 + hh;
    if (a.splits == 1) {
        const float inv = l_all > 0.0f ? 1.0f / l_all : 0.0f;
        __nv_bfloat16 *dst = a.out + ((size_t)row * a.Hq + h) * DV;
        for (int c = c0; c < DV; c += 8) {
            float acc = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) acc += fw[w] * mrg_o[(w * kHeads + hh) * kRowF + c];
            dst[c] = __float2bfloat16_rn(acc * inv);
        }
        if (a.lse != nullptr && c0 == 0)
            a.lse[(size_t)row * a.Hq + h] = l_all > 0.0f ? (m_all + log2f(l_all)) / kLog2e : -INFINITY;
    } else if (a.cluster_merge) {
        // The splits of this (row, head group) form one cluster. CTA r owns
        // quads [r * per, (r + 1) * per) of the 16 x DV outputs; every CTA
        // stores its (max, sum) of the 16 heads and its O quads of each
        // owner's slice into that owner's receive area (past the selection
        // list, untouched by the owner before the barrier), so that after
        // one cluster barrier each owner merges from its own shared memory.
        float *cta_o = mrg_ml + kWarps * kHeads * 2;  // [16][DV], this CTA's merged O
        float *cta_ml = cta_o + kHeads * DV;          // [16][2]
        for (int c = c0; c < DV; c += 8) {
            float acc = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) acc += fw[w] * mrg_o[(w * kHeads + hh) * kRowF + c];
            cta_o[hh * DV + c] = acc;
        }
        if (c0 == 0) {
            cta_ml[hh * 2 + 0] = m_all;
            cta_ml[hh * 2 + 1] = l_all;
        }
        __syncthreads();
        // every CTA of the cluster has started: its shared memory may be written
        asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
        cg::cluster_group cluster = cg::this_cluster();
        const int P = a.splits;
        constexpr int kQuads = kHeads * DV / 4;
        const int per = (kQuads + P - 1) / P;
        float4 *recv_o = reinterpret_cast<float4 *>(sel + a.per_split);  // [P][per]
        float2 *recv_ml = reinterpret_cast<float2 *>(recv_o + P * per);   // [P][16]
        for (int q = threadIdx.x; q < kQuads; q += kThreads) {
            const int r = q / per;
            cluster.map_shared_rank(recv_o, r)[split * per + (q - r * per)] =
                reinterpret_cast<const float4 *>(cta_o)[q];
        }
        if (threadIdx.x < P * kHeads) {
            const int r = threadIdx.x / kHeads, he = threadIdx.x % kHeads;
            cluster.map_shared_rank(recv_ml, r)[split * kHeads + he] =
                make_float2(cta_ml[he * 2], cta_ml[he * 2 + 1]);
        }
        cluster.sync();  // every slice delivered; no CTA touches another's memory after this
        // (max, sum) of every split for the 16 heads: one weight per
        // (split, head) with the 1/sum folded in
        float *wts = cta_ml + kHeads * 2;  // [8][16]
        if (threadIdx.x < kHeads) {
            const int he = threadIdx.x;
            float ms[8], ls[8], m_x = -INFINITY;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                ms[r] = -INFINITY;
                ls[r] = 0.0f;
                if (r < P) {
                    const float2 v = recv_ml[r * kHeads + he];
                    ms[r] = v.x;
                    ls[r] = v.y;
                }
                m_x = fmaxf(m_x, ms[r]);
            }
            float l_x = 0.0f;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                ms[r] = (r < P && m_x != -INFINITY) ? ex2_approx(ms[r] - m_x) : 0.0f;
                l_x += ms[r] * ls[r];
            }
            const float inv = l_x > 0.0f ? 1.0f / l_x : 0.0f;
#pragma unroll
            for (int r = 0; r < 8; ++r) wts[r * kHeads + he] = ms[r] * inv;
            if (a.lse != nullptr && split == 0)
                a.lse[(size_t)row * a.Hq + h0 + he] = l_x > 0.0f ? (m_x + log2f(l_x)) / kLog2e : -INFINITY;
        }
        __syncthreads();
        // this CTA's slice of the 16 x DV outputs, four columns per step
        const int e0 = split * per, e1 = min(kQuads, e0 + per);
        for (int e = e0 + threadIdx.x; e < e1; e += kThreads) {
            const int he = (4 * e) / DV, ce = 4 * e - he * DV;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                if (r < P) {
                    const float f = wts[r * kHeads + he];
                    const float4 v = recv_o[r * per + (e - e0)];
                    acc.x = fmaf(f, v.x, acc.x);
                    acc.y = fmaf(f, v.y, acc.y);
                    acc.z = fmaf(f, v.z, acc.z);
                    acc.w = fmaf(f, v.w, acc.w);
                }
            }
            __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x, acc.y);
            __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 packed;
            packed.x = *reinterpret_cast<uint32_t *>(&lo2);
            packed.y = *reinterpret_cast<uint32_t *>(&hi2);
            *reinterpret_cast<uint2 *>(a.out + ((size_t)row * a.Hq + h0 + he) * DV + ce) = packed;
        }
    } else {
        const size_t pidx = ((size_t)row * a.Hq + h) * a.splits + split;
        float *dst = a.part_o + pidx * DV;
        for (int c = c0; c < DV; c += 8) {
            float acc = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) acc += fw[w] * mrg_o[(w * kHeads + hh) * kRowF + c];
            dst[c] = acc;
        }
        if (c0 == 0) {
            a.part_ml[pidx * 2 + 0] = m_all;
            a.part_ml[pidx * 2 + 1] = l_all;
        }
    }
}

// Merge the split partials of one (row, head): one warp; lane j holds the
// (max, sum) of split j, then every lane owns four output columns and reads
// all splits' partials for them with independent 16-byte loads.
template <int DV>
__global__ void attn_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml,
                                    int n_pairs, int splits, __nv_bfloat16 *__restrict__ out,
                                    float *__restrict__ lse) {
    const int pair = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (pair >= n_pairs) return;
    const float *ml = part_ml + (size_t)pair * splits * 2;
    const float m_s = lane < splits ? ml[2 * lane] : -INFINITY;
    const float l_s = lane < splits ? ml[2 * lane + 1] : 0.0f;
    const float m_all = warp_max(m_s);
    const float f_s = (m_all == -INFINITY || lane >= splits) ? 0.0f : exp2f(m_s - m_all);
    const float l_all = warp_sum(f_s * l_s);
    const float inv = l_all > 0.0f ? 1.0f / l_all : 0.0f;
    const float4 *po = reinterpret_cast<const float4 *>(part_o + (size_t)pair * splits * DV);
    constexpr int kCols4 = DV / 4;
    for (int cb = 0; cb < kCols4; cb += 32) {  // uniform trip count: the shuffles see all lanes
        const int c4 = cb + lane;
        const bool active = c4 < kCols4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int sp = 0; sp < splits; ++sp) {
            const float f = __shfl_sync(0xffffffffu, f_s, sp);
            if (active) {
                const float4 v = __ldg(po + (size_t)sp * kCols4 + c4);
                acc.x = fmaf(f, v.x, acc.x);
                acc.y = fmaf(f, v.y, acc.y);
                acc.z = fmaf(f, v.z, acc.z);
                acc.w = fmaf(f, v.w, acc.w);
            }
        }
        if (!active) continue;
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        uint2 packed;
        packed.x = *reinterpret_cast<uint32_t *>(&lo);
        packed.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(out + (size_t)pair * DV + 4 * c4) = packed;
    }
    if (lse != nullptr && lane == 0)
        lse[pair] = l_all > 0.0f ? (m_all + log2f(l_all)) / kLog2e : -INFINITY;
}

// Splits of the selected list: enough CTAs to cover the GPU about twice, and
// at most kMaxSel entries per split.
int choose_splits(const AttnProblem &p, int sm_count) {
    const long long ctas = (long long)p.B * p.Tq * (p.Hq / kHeads);
    const int max_tiles = (p.k + kRowsPerTile - 1) / kRowsPerTile;
    int splits = 1;
    if (ctas < 2LL * sm_count) splits = (int)((2LL * sm_count + ctas - 1) / ctas);
    const int min_splits = (max_tiles * kRowsPerTile + 2047) / 2048;
    if (splits < min_splits) splits = min_splits;
    if (splits > max_tiles) splits = max_tiles;
    if (splits > 32) splits = 32;  // the combine kernel keeps one split per lane
    const int tiles_per = (max_tiles + splits - 1) / splits;  // equal whole tiles per split
    return (max_tiles + tiles_per - 1) / tiles_per;
}

bool shape_supported(const AttnProblem &p, int *dqk_dv) {
    if (p.dt != DSA_BF16) return false;
    if ((p.Hq / p.Hkv) % kHeads != 0) return false;
    const int cfgs[][2] = {{64, 64}, {128, 128}, {192, 128}};
    int which = -1;
    for (int i = 0; i < 3; ++i)
        if (p.Dqk == cfgs[i][0] && p.Dv == cfgs[i][1]) which = i;
    if (which < 0) return false;
    // 16-byte aligned rows for cp.async and 4-byte aligned Q for fragment loads
    if (((uintptr_t)p.k_cache | (uintptr_t)p.v_cache | (uintptr_t)p.out) % 16 != 0 || (uintptr_t)p.q % 4 != 0)
        return false;
    if (p.k > 32 * 2048) return false;  // at most 32 splits of 2048 entries
    if (p.k_ss % 8 || p.k_sb % 8 || p.k_sh % 8 || p.v_ss % 8 || p.v_sb % 8 || p.v_sh % 8) return false;
    *dqk_dv = which;
    return true;
}

template <int DQK, int DV, int ROWS>
cudaError_t launch_rows(const AttnProblem &p, int splits, int per_split, cudaStream_t stream) {
    using C = Cfg<DQK, DV, ROWS>;
    if (per_split > C::kMaxSel) return cudaErrorInvalidValue;
    Args a;
    a.q = static_cast<const __nv_bfloat16 *>(p.q);
    a.k_cache = static_cast<const __nv_bfloat16 *>(p.k_cache);
    a.v_cache = static_cast<const __nv_bfloat16 *>(p.v_cache);
    a.idx = p.idx;
    a.Tq = p.Tq; a.L = p.L; a.k = p.k; a.Hq = p.Hq; a.Hkv = p.Hkv;
    a.splits = splits; a.per_split = per_split;
    a.scale_log2 = p.scale * kLog2e;
    a.k_sb = p.k_sb; a.k_ss = p.k_ss; a.k_sh = p.k_sh;
    a.v_sb = p.v_sb; a.v_ss = p.v_ss; a.v_sh = p.v_sh;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.lse = p.lse;
    const int rows = p.B * p.Tq;
    const size_t n_pairs = (size_t)rows * p.Hq;
    a.part_o = nullptr;
    a.part_ml = nullptr;
    a.cluster_merge = uses_cluster_merge(splits) ? 1 : 0;
    if (splits > 1 && !a.cluster_merge) {
        a.part_o = static_cast<float *>(p.ws);
        a.part_ml = a.part_o + n_pairs * splits * DV;
    }
    auto kern = attn_mma_kernel<DQK, DV, ROWS>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemMax);
    if (err != cudaSuccess) return err;
    dim3 grid(rows, p.Hq / kHeads, splits);
    if (a.cluster_merge) {  // the splits of one (row, head group) form a cluster
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = C::cluster_smem(splits, per_split);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = splits;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        err = cudaLaunchKernelEx(&cfg, kern, a);
        count_launch();
        return err;
    }
    kern<<<grid, kThreads, C::kSmem, stream>>>(a);
    count_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (splits > 1) {
        const int warps_per_block = 8;
        attn_combine_kernel<DV><<<(int)((n_pairs + warps_per_block - 1) / warps_per_block), warps_per_block * 32, 0,
                                  stream>>>(a.part_o, a.part_ml, (int)n_pairs, splits, a.out, a.lse);
        count_launch();
        err = cudaGetLastError();
    }
    return err;
}

// Splits are whole 64-row tiles (a multiple of either stage height).
template <int DQK, int DV>
cudaError_t launch_mma(const AttnProblem &p, const DeviceInfo &info, cudaStream_t stream) {
    const int splits = choose_splits(p, info.sm_count);
    const int max_tiles = (p.k + kRowsPerTile - 1) / kRowsPerTile;
    const int per_split = ((max_tiles + splits - 1) / splits) * kRowsPerTile;
    if constexpr (DQK + DV > 256) {
        if (splits == 1) return launch_rows<DQK, DV, 32>(p, splits, per_split, stream);
    }
    return launch_rows<DQK, DV, 64>(p, splits, per_split, stream);
}

}  // namespace

unsigned int attn_tc_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_tc_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_tc_error, &zero, sizeof(zero));
    return v;
}

bool attn_mla_supported(const AttnProblem &p);
size_t attn_mla_workspace_bytes(const AttnProblem &p, int sm_count);
cudaError_t launch_attn_mla(const AttnProblem &p, const DeviceInfo &info, cudaStream_t stream);
bool attn_mla_tc_supported(const AttnProblem &p);
size_t attn_mla_tc_workspace_bytes(const AttnProblem &p, int sm_count);
cudaError_t launch_attn_mla_tc(const AttnProblem &p, const DeviceInfo &info, cudaStream_t stream);
bool attn_mqa_tc_supported(const AttnProblem &p);
cudaError_t launch_attn_mqa_tc(const AttnProblem &p, cudaStream_t stream);

cudaError_t launch_attn_combine(const float *part_o, const float *part_ml, int n_pairs, int splits, int DV,
                                __nv_bfloat16 *out, float *lse, cudaStream_t stream) {
    const int warps_per_block = 8;
    const int blocks = (n_pairs + warps_per_block - 1) / warps_per_block;
    switch (DV) {
        case 64: attn_combine_kernel<64><<<blocks, warps_per_block * 32, 0, stream>>>(part_o, part_ml, n_pairs, splits, out, lse); break;
        case 128: attn_combine_kernel<128><<<blocks, warps_per_block * 32, 0, stream>>>(part_o, part_ml, n_pairs, splits, out, lse); break;
        case 512: attn_combine_kernel<512><<<blocks, warps_per_block * 32, 0, stream>>>(part_o, part_ml, n_pairs, splits, out, lse); break;
        default: return cudaErrorInvalidValue;
    }
    count_launch();
    return cudaGetLastError();
}

size_t attn_tc_workspace_bytes(const AttnProblem &p) {
    DeviceInfo info;
    if (device_info(&info) != cudaSuccess) return 0;
    if (attn_mla_tc_supported(p)) return attn_mla_tc_workspace_bytes(p, info.sm_count);
    if (attn_mqa_tc_supported(p)) return 0;
    if (attn_mla_supported(p)) return attn_mla_workspace_bytes(p, info.sm_count);
    int which;
    if (!shape_supported(p, &which)) return 0;
    const int splits = choose_splits(p, info.sm_count);
    if (splits <= 1 || uses_cluster_merge(splits)) return 0;
    const size_t n_pairs = (size_t)p.B * p.Tq * p.Hq;
    return n_pairs * splits * ((size_t)p.Dv + 2) * sizeof(float);
}

bool attn_tc_takes(const AttnProblem &p) {
    if (attn_mla_tc_supported(p) || attn_mla_supported(p) || attn_mqa_tc_supported(p)) return true;
    int which;
    return shape_supported(p, &which);
}

cudaError_t launch_attn_tc(const AttnProblem &p, cudaStream_t stream, bool *taken) {
    *taken = false;
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    if (attn_mla_tc_supported(p)) {
        if (attn_tc_workspace_bytes(p) > p.ws_bytes) return cudaSuccess;
        *taken = true;
        return launch_attn_mla_tc(p, info, stream);
    }
    if (attn_mla_supported(p)) {
        if (attn_tc_workspace_bytes(p) > p.ws_bytes) return cudaSuccess;
        *taken = true;
        return launch_attn_mla(p, info, stream);
    }
    // groups of 8 query rows of 16 heads sharing the gathers of their union
    if (attn_mqa_tc_supported(p)) {
        *taken = true;
        return launch_attn_mqa_tc(p, stream);
    }
    int which;
    if (!shape_supported(p, &which)) return cudaSuccess;
    if (attn_tc_workspace_bytes(p) > p.ws_bytes) return cudaSuccess;
    *taken = true;
    switch (which) {
        case 0: return launch_mma<64, 64>(p, info, stream);
        case 1: return launch_mma<128, 128>(p, info, stream);
        default: return launch_mma<192, 128>(p, info, stream);
    }
}

}  // namespace dsa
