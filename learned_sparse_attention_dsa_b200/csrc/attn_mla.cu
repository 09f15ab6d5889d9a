// Sparse attention over a latent KV row shared by all query heads, with the
// value a view of the first Dv columns of the same row (the MQA mode of MLA:
// "DeepSeek Sparse Attention: Learned Token Selection from Scratch" §4.1-4.2;
// "Sparse Attention LLM Design ...", "Implemented on MLA's MQA mode": the
// kernel loads each selected latent entry once for all heads).
//
//   u[t,h] = sum_{s in S_t} softmax_s(scale * q[t,h] . c[s]) c[s][:Dv]   (§3.3, §10.1)
//
// Shapes: DQK = 576, DV = 512 (64-column multiples), bf16. One CTA owns
// (query row, 32 heads, split of the selected list) and runs 8 warps: warp
// (g, d) of head group g (16 heads) and quarter d. Per 64 selected rows,
// gathered once into shared memory with 16-byte cp.async (two stages, chunks
// XOR-swizzled by row):
//   - warp (g, d) computes S for head group g and rows 16d..16d+15
//     (mma.sync m16n8k16, Q fragments from shared memory);
//   - the four warps of a group agree on the running max through shared
//     memory, write P (bf16) to shared memory and rescale their outputs;
//   - warp (g, d) accumulates O[:, 128d .. 128d+127] of its group over all 64
//     rows, the value columns read straight from the gathered rows.
// Outputs of different warps cover disjoint columns, so only the softmax sums
// are merged at the end. With a split list the CTA writes fp32 partials that
// the split-k combine kernel merges.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

cudaError_t launch_attn_combine(const float *part_o, const float *part_ml, int n_pairs, int splits, int DV,
                                __nv_bfloat16 *out, float *lse, cudaStream_t stream);

namespace {

__device__ unsigned int g_attn_mla_error = 0;  // kErrBadIndex bits

constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int kRows = 64;                 // selected rows per stage
constexpr int kGroups = 2;                // 16-head groups per CTA
constexpr int kHeadsCta = 16 * kGroups;   // 32
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowChunks = DQK / 8;       // 72 chunks of 16 bytes per latent row
constexpr int kStageBytes = kRows * DQK * 2;          // 73,728
constexpr int kQBytes = kHeadsCta * DQK * 2;          // 36,864
constexpr int kPBytes = kGroups * 16 * kRows * 2;     // 4,096
constexpr int kMaxSel = 2048;
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t kSmem = 2 * (size_t)kStageBytes + kQBytes + 2 * kPBytes + kMaxSel * 4 + 2 * kWarps * 16 * 4 +
                         kWarps * 16 * 4 + 64;

struct Args {
    const __nv_bfloat16 *q, *kv;
    const int32_t *idx;
    int Tq, L, k, Hq, Hkv, splits, per_split;
    float scale_log2;
    int64_t sb, ss, sh;
    __nv_bfloat16 *out;
    float *lse;
    float *part_o, *part_ml;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of 16-byte chunk `chunk` of row `row` in a swizzled tile whose
// rows are `row_chunks` chunks long
__device__ __forceinline__ uint32_t swz(int row, int chunk, int row_chunks) {
    return (uint32_t)((row * row_chunks + (chunk ^ (row & 7))) * 16);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_mla_kernel(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *kv_sm = smem;                                   // 2 stages x [64 rows][576]
    uint8_t *q_sm = kv_sm + 2 * kStageBytes;                 // [32 heads][576]
    uint8_t *p_sm = q_sm + kQBytes;                          // 2 x [2 groups][16 heads][64 rows]
    int32_t *sel = reinterpret_cast<int32_t *>(p_sm + 2 * kPBytes);
    float *xmax = reinterpret_cast<float *>(sel + kMaxSel);  // 2 x [8 warps][16]
    float *lsum = xmax + 2 * kWarps * 16;                    // [8 warps][16]
    __shared__ int warp_cnt[kWarps];
    __shared__ int s_count;

    const int row = blockIdx.x;
    const int hpair = blockIdx.y;
    const int split = blockIdx.z;
    const int b = row / a.Tq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp >> 2, dq = warp & 3;
    const int h0 = hpair * kHeadsCta;
    const int g = h0 / (a.Hq / a.Hkv);
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t q_base = sbase + 2 * kStageBytes;
    const uint32_t p_base = q_base + kQBytes;

    // ---- compact this split's valid positions
    const int j0 = split * a.per_split;
    const int j1 = min(a.k, j0 + a.per_split);
    {
        int base = 0;
        for (int c0 = j0; c0 < j1; c0 += kThreads) {
            const int j = c0 + threadIdx.x;
            const int s = j < j1 ? a.idx[(size_t)row * a.k + j] : -1;
            note_bad_index(&g_attn_mla_error, s, a.L);
            const bool valid = s >= 0 && s < a.L;
            const unsigned m = __ballot_sync(0xffffffffu, valid);
            if (lane == 0) warp_cnt[warp] = __popc(m);
            __syncthreads();
            int off = base, tot = 0;
            for (int w = 0; w < kWarps; ++w) {
                if (w < warp) off += warp_cnt[w];
                tot += warp_cnt[w];
            }
            if (valid) sel[off + __popc(m & ((1u << lane) - 1u))] = s;
            base += tot;
            __syncthreads();
        }
        if (threadIdx.x == 0) s_count = base;
    }
    // ---- Q of the CTA's 32 heads (swizzled rows of 576)
    {
        const __nv_bfloat16 *qsrc = a.q + ((size_t)row * a.Hq + h0) * DQK;
        for (int c = threadIdx.x; c < kHeadsCta * kRowChunks; c += kThreads) {
            const int hh = c / kRowChunks, ch = c - hh * kRowChunks;
            cp_async16(q_base + swz(hh, ch, kRowChunks), qsrc + (size_t)hh * DQK + ch * 8, true);
        }
        cp_async_commit();
    }
    __syncthreads();
    const int n_sel = s_count;
    const int n_tiles = (n_sel + kRows - 1) / kRows;
    const __nv_bfloat16 *kvb = a.kv + b * a.sb + g * a.sh;

    auto issue = [&](int tile, int stage) {
        const uint32_t dst0 = sbase + stage * kStageBytes;
        for (int c = threadIdx.x; c < kRows * kRowChunks; c += kThreads) {
            const int r = c / kRowChunks, ch = c - r * kRowChunks;
            const int jj = tile * kRows + r;
            const bool valid = jj < n_sel;
            const int s = valid ? sel[jj] : 0;
            cp_async16(dst0 + swz(r, ch, kRowChunks), kvb + (int64_t)s * a.ss + ch * 8, valid);
        }
    };

    float o[16][4];  // this warp's 16 heads x 128 columns (16 n-tiles of 8)
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
    float m_r[2] = {-INFINITY, -INFINITY};  // running max of heads lane/4, lane/4+8 (log2 units)
    float l_r[2] = {0.0f, 0.0f};            // this warp's partial sums over its S rows

    if (n_tiles > 0) issue(0, 0);
    cp_async_commit();
    for (int tile = 0; tile < n_tiles; ++tile) {
        const int stage = tile & 1;
        const int pb = tile & 1;  // P / max buffers alternate between tiles
        cp_async_wait_0();        // this tile's rows (and Q) have landed
        __syncthreads();          // ... for every thread; the previous tile is finished by all warps
        if (tile + 1 < n_tiles) issue(tile + 1, stage ^ 1);  // overlaps the math below
        cp_async_commit();
        const uint32_t kt = sbase + stage * kStageBytes;

        // S for head group grp, rows 16dq..16dq+15
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int qr = grp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);   // A rows (heads)
            const int kr = dq * 16 + (lane & 7) + ((lane >> 4) << 3);          // B rows (positions)
#pragma unroll 4
            for (int kk = 0; kk < DQK / 16; ++kk) {
                uint32_t af[4], bf[4];
                ldsm_x4(q_base + swz(qr, 2 * kk + (lane >> 4), kRowChunks), af);
                ldsm_x4(kt + swz(kr, 2 * kk + ((lane >> 3) & 1), kRowChunks), bf);
                mma_bf16(s[0], af, bf[0], bf[1]);
                mma_bf16(s[1], af, bf[2], bf[3]);
            }
        }
        const int valid_rows = n_sel - tile * kRows;
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int rr = dq * 16 + nt * 8 + (lane & 3) * 2 + (e & 1);
                s[nt][e] = rr < valid_rows ? s[nt][e] * a.scale_log2 : -INFINITY;
                tmax[e >> 1] = fmaxf(tmax[e >> 1], s[nt][e]);
            }
        }
        float *xm = xmax + pb * kWarps * 16;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            tmax[hh] = fmaxf(tmax[hh], __shfl_xor_sync(0xffffffffu, tmax[hh], 1));
            tmax[hh] = fmaxf(tmax[hh], __shfl_xor_sync(0xffffffffu, tmax[hh], 2));
        }
        if ((lane & 3) == 0) {
            xm[warp * 16 + (lane >> 2)] = tmax[0];
            xm[warp * 16 + (lane >> 2) + 8] = tmax[1];
        }
        __syncthreads();
        // group-wide max of this tile, new running max, P and rescale
        uint8_t *pg = p_sm + pb * kPBytes + grp * (16 * kRows * 2);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int hr = (lane >> 2) + hh * 8;
            float gm = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) gm = fmaxf(gm, xm[(grp * 4 + w) * 16 + hr]);
            const float m_new = fmaxf(m_r[hh], gm);
            const float corr = m_new == -INFINITY ? 1.0f : exp2f(m_r[hh] - m_new);
            m_r[hh] = m_new;
            float sum = 0.0f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float p0 = s[nt][2 * hh] == -INFINITY ? 0.0f : exp2f(s[nt][2 * hh] - m_new);
                const float p1 = s[nt][2 * hh + 1] == -INFINITY ? 0.0f : exp2f(s[nt][2 * hh + 1] - m_new);
                sum += p0 + p1;
                const int col = dq * 16 + nt * 8 + (lane & 3) * 2;  // position within the tile
                *reinterpret_cast<__nv_bfloat162 *>(pg + swz(hr, col >> 3, kRows / 8) + (col & 7) * 2) =
                    __floats2bfloat162_rn(p0, p1);
            }
            l_r[hh] = l_r[hh] * corr + sum;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                o[n][2 * hh] *= corr;
                o[n][2 * hh + 1] *= corr;
            }
        }
        __syncthreads();
        // O[:, 128dq ..] += P V over the 64 rows of the tile
        {
            const uint32_t pga = p_base + pb * kPBytes + grp * (16 * kRows * 2);
            const int pr = (lane & 7) + (((lane >> 3) & 1) << 3);                 // A rows (heads)
            const int vr_off = (lane & 7) + (((lane >> 3) & 1) << 3);             // B rows (positions)
#pragma unroll
            for (int kk = 0; kk < kRows / 16; ++kk) {
                uint32_t af[4];
                ldsm_x4(pga + swz(pr, 2 * kk + (lane >> 4), kRows / 8), af);
                const int vr = kk * 16 + vr_off;
#pragma unroll
                for (int nn = 0; nn < 8; ++nn) {
                    uint32_t bf[4];
                    ldsm_x4_t(kt + swz(vr, dq * 16 + 2 * nn + (lane >> 4), kRowChunks), bf);
                    mma_bf16(o[2 * nn], af, bf[0], bf[1]);
                    mma_bf16(o[2 * nn + 1], af, bf[2], bf[3]);
                }
            }
        }
        // the next iteration's first barrier orders this tile's reads before
        // this stage and this P buffer are written again
    }
    cp_async_wait_0();

    // ---- softmax sums: this thread's partial -> warp -> group
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l_r[hh] += __shfl_xor_sync(0xffffffffu, l_r[hh], 1);
        l_r[hh] += __shfl_xor_sync(0xffffffffu, l_r[hh], 2);
    }
    if ((lane & 3) == 0) {
        lsum[warp * 16 + (lane >> 2)] = l_r[0];
        lsum[warp * 16 + (lane >> 2) + 8] = l_r[1];
    }
    __syncthreads();
    float l_tot[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int hr = (lane >> 2) + hh * 8;
        float t = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) t += lsum[(grp * 4 + w) * 16 + hr];
        l_tot[hh] = t;
    }
    const int cc = (lane & 3) * 2;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int h = h0 + grp * 16 + (lane >> 2) + hh * 8;
        if (a.splits == 1) {
            const float inv = l_tot[hh] > 0.0f ? 1.0f / l_tot[hh] : 0.0f;
            __nv_bfloat16 *dst = a.out + ((size_t)row * a.Hq + h) * DV + dq * 128 + cc;
#pragma unroll
            for (int n = 0; n < 16; ++n)
                *reinterpret_cast<__nv_bfloat162 *>(dst + n * 8) =
                    __floats2bfloat162_rn(o[n][2 * hh] * inv, o[n][2 * hh + 1] * inv);
            if (a.lse != nullptr && dq == 0 && (lane & 3) == 0)
                a.lse[(size_t)row * a.Hq + h] =
                    l_tot[hh] > 0.0f ? (m_r[hh] + log2f(l_tot[hh])) / kLog2e : -INFINITY;
        } else {
            const size_t pidx = ((size_t)row * a.Hq + h) * a.splits + split;
            float *dst = a.part_o + pidx * DV + dq * 128 + cc;
#pragma unroll
            for (int n = 0; n < 16; ++n)
                *reinterpret_cast<float2 *>(dst + n * 8) = make_float2(o[n][2 * hh], o[n][2 * hh + 1]);
            if (dq == 0 && (lane & 3) == 0) {
                a.part_ml[pidx * 2 + 0] = m_r[hh];
                a.part_ml[pidx * 2 + 1] = l_tot[hh];
            }
        }
    }
}

int mla_splits(const AttnProblem &p, int sm_count) {
    const long long ctas = (long long)p.B * p.Tq * (p.Hq / kHeadsCta);
    const int max_tiles = (p.k + kRows - 1) / kRows;
    int splits = 1;  // one CTA per SM fits: fill the SMs once, never a partial second wave
    if (ctas < sm_count) splits = (int)(sm_count / ctas);
    const int min_splits = (max_tiles * kRows + kMaxSel - 1) / kMaxSel;
    if (splits < min_splits) splits = min_splits;
    if (splits > max_tiles) splits = max_tiles;
    if (splits > 32) splits = 32;
    const int tiles_per = (max_tiles + splits - 1) / splits;
    return (max_tiles + tiles_per - 1) / tiles_per;
}

}  // namespace

unsigned int attn_mla_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_mla_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_mla_error, &zero, sizeof(zero));
    return v;
}

bool attn_mla_supported(const AttnProblem &p) {
    if (p.dt != DSA_BF16 || p.Dqk != DQK || p.Dv != DV) return false;
    if ((p.Hq / p.Hkv) % kHeadsCta != 0) return false;
    // the value must be the first DV columns of the same latent row
    if (p.v_cache != p.k_cache || p.v_sb != p.k_sb || p.v_ss != p.k_ss || p.v_sh != p.k_sh) return false;
    if (((uintptr_t)p.k_cache | (uintptr_t)p.q | (uintptr_t)p.out) % 16 != 0) return false;
    if (p.k_ss % 8 || p.k_sb % 8 || p.k_sh % 8) return false;
    if (p.k > 32 * kMaxSel) return false;
    return true;
}

size_t attn_mla_workspace_bytes(const AttnProblem &p, int sm_count) {
    const int splits = mla_splits(p, sm_count);
    if (splits <= 1) return 0;
    return (size_t)p.B * p.Tq * p.Hq * splits * ((size_t)DV + 2) * sizeof(float);
}

cudaError_t launch_attn_mla(const AttnProblem &p, const DeviceInfo &info, cudaStream_t stream) {
    if ((size_t)info.max_smem_optin < kSmem) return cudaErrorInvalidValue;
    const int splits = mla_splits(p, info.sm_count);
    const int max_tiles = (p.k + kRows - 1) / kRows;
    Args a;
    a.q = static_cast<const __nv_bfloat16 *>(p.q);
    a.kv = static_cast<const __nv_bfloat16 *>(p.k_cache);
    a.idx = p.idx;
    a.Tq = p.Tq; a.L = p.L; a.k = p.k; a.Hq = p.Hq; a.Hkv = p.Hkv;
    a.splits = splits;
    a.per_split = ((max_tiles + splits - 1) / splits) * kRows;
    a.scale_log2 = p.scale * kLog2e;
    a.sb = p.k_sb; a.ss = p.k_ss; a.sh = p.k_sh;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.lse = p.lse;
    const size_t n_pairs = (size_t)p.B * p.Tq * p.Hq;
    a.part_o = splits > 1 ? static_cast<float *>(p.ws) : nullptr;
    a.part_ml = splits > 1 ? a.part_o + n_pairs * splits * DV : nullptr;
    cudaError_t err = cudaFuncSetAttribute(attn_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (err != cudaSuccess) return err;
    dim3 grid(p.B * p.Tq, p.Hq / kHeadsCta, splits);
    attn_mla_kernel<<<grid, kThreads, kSmem, stream>>>(a);
    count_launch();
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (splits > 1) return launch_attn_combine(a.part_o, a.part_ml, (int)n_pairs, splits, DV, a.out, a.lse, stream);
    return cudaSuccess;
}

}  // namespace dsa
