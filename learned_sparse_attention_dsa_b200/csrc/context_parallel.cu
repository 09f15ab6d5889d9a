// Kernels of the context-parallel decode step: the keys and the KV cache are
// split by position over ranks, every rank holds all the query rows.
//
// The selection is exact: every member of the global top-k set S_t ("DeepSeek
// Sparse Attention: Learned Token Selection from Scratch" §3.1) is among the k
// best of its own shard, so merging the shards' selections (k (score,
// position) pairs per row and rank) gives S_t, with the same tie rule when
// the candidates are ordered by global position. The attention over S_t
// (§3.3) splits into per-shard softmax partials that merge by their
// log-sum-exp: u = sum_r exp(lse_r - LSE) u_r, LSE = log sum_r exp(lse_r).
//
//   select_candidates_kernel  local selection -> (score, global position)
//   localize_kernel           global selection -> this shard's positions
//   combine_parts_kernel      per-shard (u_r, lse_r) -> (u, LSE)
// The merge itself is topk_merge_kernel (topk_block.cu).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

__global__ void select_candidates_kernel(const float *__restrict__ scores, const int32_t *__restrict__ idx,
                                         long long rows, int L, int k, int key_pos0, float *__restrict__ cand_score,
                                         int32_t *__restrict__ cand_idx) {
    const long long n = rows * k;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const long long row = e / k;
        const int s = idx[e];
        const bool ok = s >= 0 && s < L;
        cand_score[e] = ok ? scores[row * L + s] : -INFINITY;
        cand_idx[e] = ok ? s + key_pos0 : -1;
    }
}

__global__ void localize_kernel(const int32_t *__restrict__ idx, long long n, int key_pos0, int L_local,
                                int32_t *__restrict__ out) {
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int s = idx[e];
        out[e] = (s >= key_pos0 && s - key_pos0 < L_local) ? s - key_pos0 : -1;
    }
}

// One warp per (row, head): LSE over the parts, then the weighted sum of the
// parts' outputs (a part with lse = -inf selected nothing and weighs 0).
template <typename T>
__global__ void combine_parts_kernel(const T *__restrict__ parts, const float *__restrict__ parts_lse, int P,
                                     long long pairs, int Dv, T *__restrict__ out, float *__restrict__ lse) {
    const long long pair = blockIdx.x * (long long)(blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (pair >= pairs) return;
    float m = -INFINITY;
    for (int p = 0; p < P; ++p) m = fmaxf(m, parts_lse[(size_t)p * pairs + pair]);
    float l = 0.f;
    if (m != -INFINITY)
        for (int p = 0; p < P; ++p) {
            const float x = parts_lse[(size_t)p * pairs + pair];
            if (x != -INFINITY) l += ex2_approx((x - m) * kLog2e);
        }
    const float total = m == -INFINITY ? -INFINITY : m + logf(l);
    for (int e = lane; e < Dv; e += 32) {
        float acc = 0.f;
        for (int p = 0; p < P; ++p) {
            const float x = parts_lse[(size_t)p * pairs + pair];
            if (x == -INFINITY) continue;
            acc += ex2_approx((x - total) * kLog2e) * Elem<T>::load(parts, ((size_t)p * pairs + pair) * Dv + e);
        }
        Elem<T>::store(out, (size_t)pair * Dv + e, acc);
    }
    if (lse && lane == 0) lse[pair] = total;
}

int grid_for(long long n, int threads) {
    long long b = (n + threads - 1) / threads;
    return (int)(b < 1 ? 1 : (b > 65535LL * 8 ? 65535LL * 8 : b));
}

}  // namespace

cudaError_t launch_select_candidates(const float *scores, const int32_t *idx, long long rows, int L, int k,
                                     int key_pos0, float *cand_score, int32_t *cand_idx, cudaStream_t stream) {
    select_candidates_kernel<<<grid_for(rows * k, 256), 256, 0, stream>>>(scores, idx, rows, L, k, key_pos0,
                                                                          cand_score, cand_idx);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_localize(const int32_t *idx, long long n, int key_pos0, int L_local, int32_t *out,
                            cudaStream_t stream) {
    localize_kernel<<<grid_for(n, 256), 256, 0, stream>>>(idx, n, key_pos0, L_local, out);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_combine_parts(const void *parts, const float *parts_lse, int P, long long pairs, int Dv,
                                 dsa_dtype dt, void *out, float *lse, cudaStream_t stream) {
    const int threads = 256;
    const long long blocks = (pairs + threads / 32 - 1) / (threads / 32);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (dt == DSA_F32)
        combine_parts_kernel<float><<<(unsigned)blocks, threads, 0, stream>>>(
            static_cast<const float *>(parts), parts_lse, P, pairs, Dv, static_cast<float *>(out), lse);
    else
        combine_parts_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(parts), parts_lse, P, pairs, Dv, static_cast<__nv_bfloat16 *>(out),
            lse);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsa
