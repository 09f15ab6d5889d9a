// Sparse attention when every query head has its own KV head (Hq == Hkv),
// bf16, head width 64 or 128.
//
//   u[t,h] = sum_{s in S_t} softmax_s(scale * q[t,h] . k[s,h]) v[s,h]
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §3.3,
// §10.1; S_t is shared by all heads, §4.1-4.2).
//
// Each head is a matrix-vector product against its own rows, so tensor cores
// do not apply; the cost is the gather, whose rate grows with the number of
// threads issuing copies on an SM (measured on B200: ~3.9 TB/s out of L2 with
// one 256-thread CTA per SM, ~7 TB/s with two, more with three). One CTA owns one query row
// and all of its heads (one warp per head). The selected positions are
// compacted in shared memory, then the K and V rows of all heads for 16
// positions at a time are gathered with 16-byte cp.async into a two-stage
// ring (32 KB per stage at 8 heads of width 64, so three CTAs share an SM:
// measured faster than three stages with two CTAs);
// every selected row is fetched once for all heads, as whole contiguous rows.
// 16-byte chunks are XOR-swizzled by row so that the reads below are free of
// bank conflicts. Per 16 positions, lanes r and r + 16 of head h's warp each
// compute half of the logit of position r, the warp updates its running max
// and sum (online softmax in fp32, exp2 with the log2(e) prescale), and the
// lanes, each owning D/32 output columns, accumulate the weighted value rows.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kRows = 16;  // selected positions per stage
constexpr int kMaxHeads = 16;
constexpr float kLog2e = 1.4426950408889634f;

struct Args {
    const __nv_bfloat16 *q, *k_cache, *v_cache;
    const int32_t *idx;
    int Tq, L, k, H;
    int rc_shift;  // log2 of the 16-byte chunks per position row (H * D / 8, a power of two)
    float scale_log2;
    int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
    __nv_bfloat16 *out;
    float *lse;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Stage layout: K then V, each [kRows][H * D] bf16; 16-byte chunk c of row r
// is stored at chunk position c ^ (r & 7).
template <int D, int STAGES>
__global__ void __launch_bounds__(D == 64 ? 512 : 256)
attn_perhead_kernel(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int kChunksPerHead = D / 8;
    const int row_chunks = a.H * kChunksPerHead;  // chunks per position (per K or V)
    const int stage_bytes = 2 * kRows * row_chunks * 16;
    int32_t *sel = reinterpret_cast<int32_t *>(smem + STAGES * stage_bytes);
    __shared__ int warp_cnt[kMaxHeads];
    __shared__ int s_count;

    const int row = blockIdx.x;
    const int b = row / a.Tq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthreads = blockDim.x;
    const int nwarps = nthreads >> 5;

    // ---- compact the valid selected positions (order kept)
    {
        int base = 0;
        for (int c0 = 0; c0 < a.k; c0 += nthreads) {
            const int j = c0 + threadIdx.x;
            const int s = j < a.k ? a.idx[(size_t)row * a.k + j] : -1;
            const bool valid = s >= 0 && s < a.L;
            const unsigned m = __ballot_sync(0xffffffffu, valid);
            if (lane == 0) warp_cnt[warp] = __popc(m);
            __syncthreads();
            int off = base, tot = 0;
            for (int w = 0; w < nwarps; ++w) {
                if (w < warp) off += warp_cnt[w];
                tot += warp_cnt[w];
            }
            if (valid) sel[off + __popc(m & ((1u << lane) - 1u))] = s;
            base += tot;
            __syncthreads();
        }
        if (threadIdx.x == 0) s_count = base;
        __syncthreads();
    }
    const int n_sel = s_count;
    const int n_tiles = (n_sel + kRows - 1) / kRows;
    const uint32_t smem_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const __nv_bfloat16 *kb = a.k_cache + b * a.k_sb;
    const __nv_bfloat16 *vb = a.v_cache + b * a.v_sb;

    auto issue = [&](int tile, int stage) {
        const uint32_t kdst = smem_base + stage * stage_bytes;
        const uint32_t vdst = kdst + kRows * row_chunks * 16;
        const int total = 2 * kRows * row_chunks;
        const int half_total = kRows * row_chunks;
        for (int c = threadIdx.x; c < total; c += nthreads) {
            const bool is_v = c >= half_total;
            const int cc = c & (half_total - 1);
            const int r = cc >> a.rc_shift;
            const int x = cc & (row_chunks - 1);  // chunk within the position's row
            const int h = x / kChunksPerHead, ch = x % kChunksPerHead;
            const int jj = tile * kRows + r;
            const bool valid = jj < n_sel;
            const int s = valid ? sel[jj] : 0;
            const __nv_bfloat16 *src = is_v ? vb + (int64_t)s * a.v_ss + h * a.v_sh + ch * 8
                                            : kb + (int64_t)s * a.k_ss + h * a.k_sh + ch * 8;
            const uint32_t dst = (is_v ? vdst : kdst) + (r * row_chunks + (x ^ (r & 7))) * 16;
            cp_async16(dst, src, valid);
        }
    };

    // this warp's head: lane half hf (= lane / 16) holds query columns
    // [hf * D/2, hf * D/2 + D/2), pre-scaled into log2 units
    const int h = warp;
    const int hf = lane >> 4;
    float qreg[D / 2];
    {
        const __nv_bfloat16 *qh = a.q + ((size_t)row * a.H + h) * D + hf * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
            float f[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(qh + c * 8), f);
#pragma unroll
            for (int u = 0; u < 8; ++u) qreg[c * 8 + u] = f[u] * a.scale_log2;
        }
    }
    constexpr int kCols = D / 32;  // output columns per lane: lane*kCols ...
    float acc[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) acc[c] = 0.0f;
    float m = -INFINITY, l = 0.0f;

#pragma unroll
    for (int st = 0; st < STAGES - 1; ++st) {
        if (st < n_tiles) issue(st, st);
        cp_async_commit();
    }
    for (int tile = 0; tile < n_tiles; ++tile) {
        const int stage = tile % STAGES;
        if (tile + STAGES - 1 < n_tiles) issue(tile + STAGES - 1, (tile + STAGES - 1) % STAGES);
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        __syncthreads();

        const uint8_t *kt = smem + stage * stage_bytes;
        const uint8_t *vt = kt + kRows * row_chunks * 16;
        // half hf of the logit of position r (lanes r and r + 16)
        const int r = lane & (kRows - 1);
        float z = -INFINITY;
        {
            const uint8_t *krow = kt + r * row_chunks * 16;
            float dot[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // independent chains
#pragma unroll
            for (int c = 0; c < kChunksPerHead / 2; ++c) {
                const int x = h * kChunksPerHead + hf * (kChunksPerHead / 2) + c;
                float f[8];
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(krow + (x ^ (r & 7)) * 16), f);
#pragma unroll
                for (int u = 0; u < 8; ++u) dot[u & 3] = fmaf(qreg[c * 8 + u], f[u], dot[u & 3]);
            }
            float zp = (dot[0] + dot[1]) + (dot[2] + dot[3]);
            zp += __shfl_xor_sync(0xffffffffu, zp, 16);  // both halves hold the full logit
            if (tile * kRows + r < n_sel) z = zp;
        }
        const float zmax = warp_max(z);
        const float m_new = fmaxf(m, zmax);
        const float corr = m_new == -INFINITY ? 1.0f : ex2_approx(m - m_new);
        const float p = z == -INFINITY ? 0.0f : ex2_approx(z - m_new);
        l = l * corr + warp_sum(hf == 0 ? p : 0.0f);  // each position counted once
        m = m_new;
#pragma unroll
        for (int c = 0; c < kCols; ++c) acc[c] *= corr;
        // weighted value rows: lane owns columns [lane*kCols, lane*kCols + kCols)
        const int valid_rows = min(kRows, n_sel - tile * kRows);
        for (int rr = 0; rr < valid_rows; ++rr) {
            const float pr = __shfl_sync(0xffffffffu, p, rr);
            const int x = h * kChunksPerHead + (lane * kCols) / 8;
            const uint8_t *vrow = vt + rr * row_chunks * 16 + (x ^ (rr & 7)) * 16 + ((lane * kCols) % 8) * 2;
            if constexpr (kCols == 2) {
                const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162 *>(vrow);
                acc[0] = fmaf(pr, __low2float(v2), acc[0]);
                acc[1] = fmaf(pr, __high2float(v2), acc[1]);
            } else {
                const uint2 v4 = *reinterpret_cast<const uint2 *>(vrow);
                acc[0] = fmaf(pr, __uint_as_float(v4.x << 16), acc[0]);
                acc[1] = fmaf(pr, __uint_as_float(v4.x & 0xffff0000u), acc[1]);
                acc[2] = fmaf(pr, __uint_as_float(v4.y << 16), acc[2]);
                acc[3] = fmaf(pr, __uint_as_float(v4.y & 0xffff0000u), acc[3]);
            }
        }
        __syncthreads();  // the stage is refilled by a later iteration's issue
    }
    cp_async_wait<0>();

    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
    __nv_bfloat16 *dst = a.out + ((size_t)row * a.H + h) * D + lane * kCols;
#pragma unroll
    for (int c = 0; c < kCols; c += 2)
        *reinterpret_cast<__nv_bfloat162 *>(dst + c) = __floats2bfloat162_rn(acc[c] * inv, acc[c + 1] * inv);
    if (a.lse != nullptr && lane == 0)
        a.lse[(size_t)row * a.H + h] = l > 0.0f ? (m + log2f(l)) / kLog2e : -INFINITY;
}

}  // namespace

cudaError_t launch_attn_perhead(const AttnProblem &p, cudaStream_t stream, bool *taken) {
    *taken = false;
    if (p.dt != DSA_BF16 || p.Hq != p.Hkv || p.Hq > (p.Dqk == 64 ? kMaxHeads : 8)) return cudaSuccess;
    if ((p.Hq & (p.Hq - 1)) != 0) return cudaSuccess;  // the row layout uses shifts
    if (!((p.Dqk == 64 && p.Dv == 64) || (p.Dqk == 128 && p.Dv == 128))) return cudaSuccess;
    if (((uintptr_t)p.k_cache | (uintptr_t)p.v_cache | (uintptr_t)p.q) % 16 != 0 || (uintptr_t)p.out % 4 != 0)
        return cudaSuccess;
    if (p.k_ss % 8 || p.k_sb % 8 || p.k_sh % 8 || p.v_ss % 8 || p.v_sb % 8 || p.v_sh % 8) return cudaSuccess;
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    const size_t stage_bytes = 2ull * kRows * p.Hq * p.Dqk * 2;
    const size_t sel_bytes = sizeof(int32_t) * (size_t)p.k;
    // two stages: more CTAs per SM issue copies (three stages only help when
    // the copies are few)
    const int stages = 2;
    const size_t smem = stages * stage_bytes + sel_bytes;
    if (smem > (size_t)info.max_smem_optin) return cudaSuccess;
    Args a;
    a.q = static_cast<const __nv_bfloat16 *>(p.q);
    a.k_cache = static_cast<const __nv_bfloat16 *>(p.k_cache);
    a.v_cache = static_cast<const __nv_bfloat16 *>(p.v_cache);
    a.idx = p.idx;
    a.Tq = p.Tq; a.L = p.L; a.k = p.k; a.H = p.Hq;
    a.rc_shift = 0;
    while ((1 << a.rc_shift) < p.Hq * (p.Dqk / 8)) ++a.rc_shift;
    a.scale_log2 = p.scale * kLog2e;
    a.k_sb = p.k_sb; a.k_ss = p.k_ss; a.k_sh = p.k_sh;
    a.v_sb = p.v_sb; a.v_ss = p.v_ss; a.v_sh = p.v_sh;
    a.out = static_cast<__nv_bfloat16 *>(p.out);
    a.lse = p.lse;
    *taken = true;
    auto kern = p.Dqk == 64 ? attn_perhead_kernel<64, 2> : attn_perhead_kernel<128, 2>;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    kern<<<p.B * p.Tq, p.Hq * 32, smem, stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsa
