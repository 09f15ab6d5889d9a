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
// With several query rows the group kernel below is used instead: rows share
// the copies of the union of their selections.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

__device__ unsigned int g_attn_perhead_error = 0;  // kErrBadIndex bits

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

// ldmatrix of four 8x8 bf16 matrices (rows of 16 bytes, one row address per lane)
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t *r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// d += A (16x16, row) . B (16x8, col), bf16 in, fp32 accumulate
__device__ __forceinline__ void mma_bf16_16816(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Stage layout: K then V, each [kRows][H * D] bf16; 16-byte chunk c of row r
// is stored at chunk position c ^ (r & 7).
template <int D, int STAGES>
__global__ void __launch_bounds__(D == 64 ? 512 : 256, 1)
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
            note_bad_index(&g_attn_perhead_error, s, a.L);
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

    // Copies: thread i always moves 16-byte chunk x = i % row_chunks of a
    // position's row (fixed head and column offsets), for rows r0, r0 + step, ...
    // of the tile, K and V alike (row_chunks divides the thread count).
    const int cstep = nthreads / row_chunks;  // rows per pass: 4 (D = 64) or 2 (D = 128)
    const int cx = threadIdx.x % row_chunks, cr0 = threadIdx.x / row_chunks;
    const int64_t koff = (int64_t)(cx / kChunksPerHead) * a.k_sh + (cx % kChunksPerHead) * 8;
    const int64_t voff = (int64_t)(cx / kChunksPerHead) * a.v_sh + (cx % kChunksPerHead) * 8;
    const uint32_t vstage_off = kRows * row_chunks * 16;
    auto issue = [&](int tile, int stage) {
        const uint32_t kdst = smem_base + stage * stage_bytes;
#pragma unroll 4
        for (int r = cr0; r < kRows; r += cstep) {
            const int jj = tile * kRows + r;
            const bool valid = jj < n_sel;
            const int s = valid ? sel[jj] : 0;
            const uint32_t dst = kdst + (r * row_chunks + (cx ^ (r & 7))) * 16;
            cp_async16(dst, kb + (int64_t)s * a.k_ss + koff, valid);
            cp_async16(dst + vstage_off, vb + (int64_t)s * a.v_ss + voff, valid);
        }
    };

    // ---- this warp's head h: both products on the tensor cores (mma.sync
    // m16n8k16, bf16 in, fp32 accumulate). Every row of the A operand is the
    // same query (logits) or the same probabilities (weighted sum), so every
    // accumulator row holds the same values; lane (g, t) = (lane / 4, lane % 4)
    // holds positions 8 nb + 2t, 8 nb + 2t + 1 of each 8-position block nb.
    const int h = warp;
    const int t4 = lane & 3, g8 = lane >> 2;
    constexpr int kKSteps = D / 16;  // 16-wide slices of the head
    constexpr int kNBlk = D / 8;     // 8-wide output column blocks
    uint32_t qa[kKSteps][2];         // A fragments: q pairs (2t, 2t+1) and (2t+8, 2t+9) of each slice
    {
        const __nv_bfloat16 *qh = a.q + ((size_t)row * a.H + h) * D;
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
            qa[ks][0] = *reinterpret_cast<const uint32_t *>(qh + ks * 16 + 2 * t4);
            qa[ks][1] = *reinterpret_cast<const uint32_t *>(qh + ks * 16 + 8 + 2 * t4);
        }
    }
    float acc[kNBlk][2];
#pragma unroll
    for (int j = 0; j < kNBlk; ++j) acc[j][0] = acc[j][1] = 0.0f;
    float m = -INFINITY, l = 0.0f;
    const int hx = h * kChunksPerHead;  // the head's first 16-byte chunk in a position row
    const int row_bytes = row_chunks * 16;

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

        const uint32_t kt = smem_base + stage * stage_bytes;
        const uint32_t vt = kt + kRows * row_bytes;
        // logits of the 16 positions: S = q . K^T, two 8-position blocks
        float sc[2][2];
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < kChunksPerHead; c += 4) {
                // matrices: positions 8 nb .. 8 nb + 7, chunks c .. c + 3 of the head
                const int p = nb * 8 + (lane & 7);
                const int x = hx + c + (lane >> 3);
                uint32_t b[4];
                ldmatrix_x4(kt + p * row_bytes + ((x ^ (p & 7)) << 4), b);
                mma_bf16_16816(d, qa[c / 2][0], qa[c / 2][0], qa[c / 2][1], qa[c / 2][1], b[0], b[1]);
                mma_bf16_16816(d, qa[c / 2 + 1][0], qa[c / 2 + 1][0], qa[c / 2 + 1][1], qa[c / 2 + 1][1], b[2],
                               b[3]);
            }
            const int p0 = tile * kRows + nb * 8 + 2 * t4;
            sc[nb][0] = p0 < n_sel ? d[0] * a.scale_log2 : -INFINITY;
            sc[nb][1] = p0 + 1 < n_sel ? d[1] * a.scale_log2 : -INFINITY;
        }
        // online softmax over the tile (lanes sharing t hold the same values)
        float zmax = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, 1));
        zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, 2));
        const float m_new = fmaxf(m, zmax);
        const float mr = m_new == -INFINITY ? 0.0f : m_new;  // masked entries: 2^-inf = 0
        float pr[2][2], psum = 0.0f;
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                pr[nb][e] = ex2_approx(sc[nb][e] - mr);
                psum += pr[nb][e];
            }
        psum += __shfl_xor_sync(0xffffffffu, psum, 1);
        psum += __shfl_xor_sync(0xffffffffu, psum, 2);
        if (m_new != m) {  // warp-uniform
            const float corr = ex2_approx(m - mr);
            l *= corr;
#pragma unroll
            for (int j = 0; j < kNBlk; ++j) {
                acc[j][0] *= corr;
                acc[j][1] *= corr;
            }
            m = m_new;
        }
        l += psum;
        // weighted value rows: acc += P . V (P in bf16; positions are the K dimension)
        const uint32_t pa0 = pack_bf16x2(pr[0][0], pr[0][1]), pa2 = pack_bf16x2(pr[1][0], pr[1][1]);
#pragma unroll
        for (int j = 0; j < kNBlk; j += 2) {
            // matrices: positions 0-7 and 8-15 of chunks j and j + 1, transposed
            const int mi = lane >> 3;
            const int p = (mi & 1) * 8 + (lane & 7);
            const int x = hx + j + (mi >> 1);
            uint32_t b[4];
            ldmatrix_x4_trans(vt + p * row_bytes + ((x ^ (p & 7)) << 4), b);
            float d0[4] = {acc[j][0], acc[j][1], acc[j][0], acc[j][1]};
            mma_bf16_16816(d0, pa0, pa0, pa2, pa2, b[0], b[1]);
            acc[j][0] = d0[0];
            acc[j][1] = d0[1];
            float d1[4] = {acc[j + 1][0], acc[j + 1][1], acc[j + 1][0], acc[j + 1][1]};
            mma_bf16_16816(d1, pa0, pa0, pa2, pa2, b[2], b[3]);
            acc[j + 1][0] = d1[0];
            acc[j + 1][1] = d1[1];
        }
        __syncthreads();  // the stage is refilled by a later iteration's issue
    }
    cp_async_wait<0>();

    // lane (g, t) writes output columns 8 j + 2t, 8 j + 2t + 1 for j = g, g + 4, ...
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
    __nv_bfloat16 *dst = a.out + ((size_t)row * a.H + h) * D;
#pragma unroll
    for (int j = 0; j < kNBlk; ++j)
        if ((j & 7) == g8)
            *reinterpret_cast<__nv_bfloat162 *>(dst + j * 8 + 2 * t4) =
                __floats2bfloat162_rn(acc[j][0] * inv, acc[j][1] * inv);
    if (a.lse != nullptr && lane == 0)
        a.lse[(size_t)row * a.H + h] = l > 0.0f ? (m + log2f(l)) / kLog2e : -INFINITY;
}


// Query-row groups. QG consecutive query rows of one batch entry (QG in {2,
// 4, 8, 16}) share one gather: their selected sets are marked in one bitmap
// per row, the union is listed in ascending position order, and the K and V
// rows of every union position are fetched once for the group. The head's
// m16n8k16 logits then hold QG queries at once (A-operand row r is query
// r * QG / 16; a single query would repeat in all 16 rows), each logit is
// masked to -inf where its position is not in that query's own set, and each
// lane keeps the online softmax of its two rows' queries (g and g + 8). The
// result is the per-row attention over each row's own S_t; the union only
// shares the copies. A union entry packs the position (16 bits, L <= 65,536)
// with the mask of the group's rows that selected it.
struct GroupArgs {
    int B, ngroups;  // batch entries; row groups per batch entry
    int W;           // 32-bit bitmap words per row: ceil(L / 32)
};

template <int D, int QG>
__global__ void __launch_bounds__(D == 64 ? 512 : 256, 1)
attn_perhead_group_kernel(const Args a, const GroupArgs ga) {
    constexpr int STAGES = 2;
    constexpr int R = 16 / QG;  // A-operand rows per query
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int kChunksPerHead = D / 8;
    const int row_chunks = a.H * kChunksPerHead;
    const int stage_bytes = 2 * kRows * row_chunks * 16;
    const int W = ga.W;
    uint32_t *bm = reinterpret_cast<uint32_t *>(smem + STAGES * stage_bytes);  // [QG][W]
    uint32_t *ulist = bm + QG * W;  // [union]: position | rows' mask << 16
    __shared__ int warp_tot[kMaxHeads];
    __shared__ int s_count;

    // heavy groups (the latest rows, the largest unions) first
    const int b = blockIdx.x % ga.B;
    const int gi = ga.ngroups - 1 - (int)(blockIdx.x / ga.B);
    const int i0 = gi * QG;
    const int qn = min(QG, a.Tq - i0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthreads = blockDim.x;
    const size_t row0 = (size_t)b * a.Tq + i0;

    // ---- one bitmap per row of the group, then the union in position order
    for (int w = threadIdx.x; w < QG * W; w += nthreads) bm[w] = 0u;
    __syncthreads();
    for (int q = 0; q < qn; ++q) {
        const int32_t *src = a.idx + (row0 + q) * a.k;
        for (int j = threadIdx.x; j < a.k; j += nthreads) {
            const int s = src[j];
            note_bad_index(&g_attn_perhead_error, s, a.L);
            if (s >= 0 && s < a.L) atomicOr(&bm[q * W + (s >> 5)], 1u << (s & 31));
        }
    }
    __syncthreads();
    {
        // thread i owns words [i * per, (i + 1) * per): its union count, a
        // block-wide exclusive scan of the counts, then its positions
        const int per = (W + nthreads - 1) / nthreads;
        const int w0 = min(W, threadIdx.x * per), w1 = min(W, w0 + per);
        int cnt = 0;
        for (int w = w0; w < w1; ++w) {
            uint32_t u = 0u;
            for (int q = 0; q < qn; ++q) u |= bm[q * W + w];
            cnt += __popc(u);
        }
        const int incl = warp_inclusive_scan(cnt);
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int base = incl - cnt;
        for (int w = 0; w < warp; ++w) base += warp_tot[w];
        for (int w = w0; w < w1; ++w) {
            uint32_t wq[QG];
            uint32_t u = 0u;
#pragma unroll
            for (int q = 0; q < QG; ++q) {
                wq[q] = q < qn ? bm[q * W + w] : 0u;
                u |= wq[q];
            }
            while (u) {
                const int bit = __ffs(u) - 1;
                uint32_t mask = 0u;
#pragma unroll
                for (int q = 0; q < QG; ++q) mask |= ((wq[q] >> bit) & 1u) << q;
                ulist[base++] = (uint32_t)(w * 32 + bit) | (mask << 16);
                u &= u - 1u;
            }
        }
        if (threadIdx.x == nthreads - 1) s_count = base;
    }
    __syncthreads();
    const int n_sel = s_count;
    const int n_tiles = (n_sel + kRows - 1) / kRows;
    const uint32_t smem_base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const __nv_bfloat16 *kb = a.k_cache + b * a.k_sb;
    const __nv_bfloat16 *vb = a.v_cache + b * a.v_sb;

    // copies as in attn_perhead_kernel, positions from the union list
    const int cstep = nthreads / row_chunks;
    const int cx = threadIdx.x % row_chunks, cr0 = threadIdx.x / row_chunks;
    const int64_t koff = (int64_t)(cx / kChunksPerHead) * a.k_sh + (cx % kChunksPerHead) * 8;
    const int64_t voff = (int64_t)(cx / kChunksPerHead) * a.v_sh + (cx % kChunksPerHead) * 8;
    const uint32_t vstage_off = kRows * row_chunks * 16;
    auto issue = [&](int tile, int stage) {
        const uint32_t kdst = smem_base + stage * stage_bytes;
#pragma unroll 4
        for (int r = cr0; r < kRows; r += cstep) {
            const int jj = tile * kRows + r;
            const bool valid = jj < n_sel;
            const int s = valid ? (int)(ulist[jj] & 0xFFFFu) : 0;
            const uint32_t dst = kdst + (r * row_chunks + (cx ^ (r & 7))) * 16;
            cp_async16(dst, kb + (int64_t)s * a.k_ss + koff, valid);
            cp_async16(dst + vstage_off, vb + (int64_t)s * a.v_ss + voff, valid);
        }
    };

    // ---- this warp's head h; lane (g, t) holds queries qx[0] = g / R (row g)
    // and qx[1] = (g + 8) / R (row g + 8) of the group
    const int h = warp;
    const int t4 = lane & 3, g8 = lane >> 2;
    const int qx[2] = {g8 / R, (g8 + 8) / R};
    constexpr int kKSteps = D / 16;
    constexpr int kNBlk = D / 8;
    uint32_t qf[2][kKSteps][2];  // per query: k-low and k-high pairs of each 16-wide slice
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const bool live = qx[x] < qn;
        const __nv_bfloat16 *qh = a.q + ((row0 + (live ? qx[x] : 0)) * a.H + h) * D;
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
            qf[x][ks][0] = live ? *reinterpret_cast<const uint32_t *>(qh + ks * 16 + 2 * t4) : 0u;
            qf[x][ks][1] = live ? *reinterpret_cast<const uint32_t *>(qh + ks * 16 + 8 + 2 * t4) : 0u;
        }
    }
    float acc[kNBlk][4];
#pragma unroll
    for (int j = 0; j < kNBlk; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
    const int hx = h * kChunksPerHead;
    const int row_bytes = row_chunks * 16;

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

        const uint32_t kt = smem_base + stage * stage_bytes;
        const uint32_t vt = kt + kRows * row_bytes;
        // logits: rows g (query qx[0]) and g + 8 (query qx[1]) of each 8-position block
        float sc[2][2][2];  // [block][position pair][query]
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < kChunksPerHead; c += 4) {
                const int p = nb * 8 + (lane & 7);
                const int xx = hx + c + (lane >> 3);
                uint32_t bf[4];
                ldmatrix_x4(kt + p * row_bytes + ((xx ^ (p & 7)) << 4), bf);
                mma_bf16_16816(d, qf[0][c / 2][0], qf[1][c / 2][0], qf[0][c / 2][1], qf[1][c / 2][1], bf[0], bf[1]);
                mma_bf16_16816(d, qf[0][c / 2 + 1][0], qf[1][c / 2 + 1][0], qf[0][c / 2 + 1][1],
                               qf[1][c / 2 + 1][1], bf[2], bf[3]);
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int jj = tile * kRows + nb * 8 + 2 * t4 + e;
                const uint32_t rows_in = jj < n_sel ? ulist[jj] >> 16 : 0u;  // rows that selected it
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const bool in = (rows_in >> qx[x]) & 1u;
                    sc[nb][e][x] = in ? d[2 * x + e] * a.scale_log2 : -INFINITY;
                }
            }
        }
        // online softmax per query (the four lanes of a row share it)
        float pr[2][2][2];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            float zmax = fmaxf(fmaxf(sc[0][0][x], sc[0][1][x]), fmaxf(sc[1][0][x], sc[1][1][x]));
            zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, 1));
            zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, 2));
            const float m_new = fmaxf(m[x], zmax);
            const float mr = m_new == -INFINITY ? 0.0f : m_new;
            float psum = 0.0f;
#pragma unroll
            for (int nb = 0; nb < 2; ++nb)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    pr[nb][e][x] = ex2_approx(sc[nb][e][x] - mr);
                    psum += pr[nb][e][x];
                }
            psum += __shfl_xor_sync(0xffffffffu, psum, 1);
            psum += __shfl_xor_sync(0xffffffffu, psum, 2);
            if (m_new != m[x]) {  // uniform over the row's four lanes
                const float corr = ex2_approx(m[x] - mr);
                l[x] *= corr;
#pragma unroll
                for (int j = 0; j < kNBlk; ++j) {
                    acc[j][2 * x] *= corr;
                    acc[j][2 * x + 1] *= corr;
                }
                m[x] = m_new;
            }
            l[x] += psum;
        }
        // weighted value rows: P rows g and g + 8 as the A operand
        const uint32_t pa0 = pack_bf16x2(pr[0][0][0], pr[0][1][0]), pa1 = pack_bf16x2(pr[0][0][1], pr[0][1][1]);
        const uint32_t pa2 = pack_bf16x2(pr[1][0][0], pr[1][1][0]), pa3 = pack_bf16x2(pr[1][0][1], pr[1][1][1]);
#pragma unroll
        for (int j = 0; j < kNBlk; j += 2) {
            const int mi = lane >> 3;
            const int p = (mi & 1) * 8 + (lane & 7);
            const int xx = hx + j + (mi >> 1);
            uint32_t bf[4];
            ldmatrix_x4_trans(vt + p * row_bytes + ((xx ^ (p & 7)) << 4), bf);
            mma_bf16_16816(acc[j], pa0, pa1, pa2, pa3, bf[0], bf[1]);
            mma_bf16_16816(acc[j + 1], pa0, pa1, pa2, pa3, bf[2], bf[3]);
        }
        __syncthreads();  // the stage is refilled by a later iteration's issue
    }
    cp_async_wait<0>();

    // the R rows of a query hold the same values: row g writes the column
    // blocks j with j % R == g % R
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        if (qx[x] >= qn) continue;
        const float inv = l[x] > 0.0f ? 1.0f / l[x] : 0.0f;
        __nv_bfloat16 *dst = a.out + ((row0 + qx[x]) * a.H + h) * D;
#pragma unroll
        for (int j = 0; j < kNBlk; ++j)
            if ((j % R) == (g8 % R))
                *reinterpret_cast<__nv_bfloat162 *>(dst + j * 8 + 2 * t4) =
                    __floats2bfloat162_rn(acc[j][2 * x] * inv, acc[j][2 * x + 1] * inv);
        if (a.lse != nullptr && t4 == 0 && g8 % R == 0)
            a.lse[(row0 + qx[x]) * a.H + h] = l[x] > 0.0f ? (m[x] + log2f(l[x])) / kLog2e : -INFINITY;
    }
}

}  // namespace

unsigned int attn_perhead_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_perhead_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_perhead_error, &zero, sizeof(zero));
    return v;
}

namespace {

// Whether the per-head kernels take a shape, their shared-memory footprint,
// and the query-row group: the largest QG whose bitmaps and union list fit
// next to the stages within the single-row kernel's footprint or two CTAs
// per SM (QG = 1: one row per CTA).
struct PerheadPlan {
    bool ok = false;
    size_t smem = 0, smem_g = 0;
    int qg = 1, W = 0;
};

PerheadPlan plan_perhead(const AttnProblem &p, const DeviceInfo &info) {
    PerheadPlan pl;
    if (p.dt != DSA_BF16 || p.Hq != p.Hkv || p.Hq > (p.Dqk == 64 ? kMaxHeads : 8)) return pl;
    if ((p.Hq & (p.Hq - 1)) != 0) return pl;  // the row layout uses shifts
    if (!((p.Dqk == 64 && p.Dv == 64) || (p.Dqk == 128 && p.Dv == 128))) return pl;
    if (((uintptr_t)p.k_cache | (uintptr_t)p.v_cache | (uintptr_t)p.q) % 16 != 0 || (uintptr_t)p.out % 4 != 0)
        return pl;
    if (p.k_ss % 8 || p.k_sb % 8 || p.k_sh % 8 || p.v_ss % 8 || p.v_sb % 8 || p.v_sh % 8) return pl;
    const size_t stage_bytes = 2ull * kRows * p.Hq * p.Dqk * 2;
    const size_t sel_bytes = sizeof(int32_t) * (size_t)p.k;
    // two stages: more CTAs per SM issue copies (three stages only help when
    // the copies are few)
    pl.smem = 2 * stage_bytes + sel_bytes;
    if (pl.smem > (size_t)info.max_smem_optin) return pl;
    pl.ok = true;
    if (p.Tq >= 2 && p.L <= 65536) {
        pl.W = (p.L + 31) / 32;
        const size_t budget = pl.smem > 112 * 1024 ? pl.smem : 112 * 1024;
        for (int qg = 16; qg >= 2; qg /= 2) {
            const size_t ucap = (size_t)(p.L < qg * p.k ? p.L : qg * p.k);
            const size_t smem_g = 2 * stage_bytes + (size_t)qg * pl.W * 4 + ucap * 4;
            if (smem_g > budget || smem_g > (size_t)info.max_smem_optin) continue;
            pl.qg = qg;
            pl.smem_g = smem_g;
            break;
        }
    }
    return pl;
}

}  // namespace

int perhead_row_group(const AttnProblem &p) {
    DeviceInfo info;
    if (device_info(&info) != cudaSuccess) return 0;
    const PerheadPlan pl = plan_perhead(p, info);
    return pl.ok ? pl.qg : 0;
}

cudaError_t launch_attn_perhead(const AttnProblem &p, cudaStream_t stream, bool *taken) {
    *taken = false;
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    const PerheadPlan pl = plan_perhead(p, info);
    if (!pl.ok) return cudaSuccess;
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
    if (pl.qg > 1) {  // groups of QG query rows share the gathers of their union
        const int qg = pl.qg;
        GroupArgs ga;
        ga.B = p.B;
        ga.ngroups = (p.Tq + qg - 1) / qg;
        ga.W = pl.W;
        void (*gk)(const Args, const GroupArgs) = nullptr;
        if (p.Dqk == 64) {
            gk = qg == 16 ? attn_perhead_group_kernel<64, 16> : qg == 8 ? attn_perhead_group_kernel<64, 8>
               : qg == 4 ? attn_perhead_group_kernel<64, 4> : attn_perhead_group_kernel<64, 2>;
        } else {
            gk = qg == 16 ? attn_perhead_group_kernel<128, 16> : qg == 8 ? attn_perhead_group_kernel<128, 8>
               : qg == 4 ? attn_perhead_group_kernel<128, 4> : attn_perhead_group_kernel<128, 2>;
        }
        err = cudaFuncSetAttribute(gk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem_g);
        if (err != cudaSuccess) return err;
        const long long grid = (long long)p.B * ga.ngroups;
        if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
        gk<<<(unsigned)grid, p.Hq * 32, pl.smem_g, stream>>>(a, ga);
        count_launch();
        return cudaGetLastError();
    }
    auto kern = p.Dqk == 64 ? attn_perhead_kernel<64, 2> : attn_perhead_kernel<128, 2>;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
    if (err != cudaSuccess) return err;
    kern<<<p.B * p.Tq, p.Hq * 32, pl.smem, stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsa
