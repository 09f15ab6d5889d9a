// Softmax attention over the selected rows, CUDA-core version (any shape).
//
//   u[t,h] = sum_{s in S_t} softmax_s(scale * q[t,h] . k[s,g]) v[s,g],  g = h / (Hq/Hkv)
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §3.3,
// §10.1; one S_t for every head, §4.1-4.2).
//
// One warp owns one (query row, head). It walks the selected positions 32 at a
// time: each lane computes one logit q.k_s (the query sits in shared memory,
// pre-multiplied by scale*log2(e) so that exp becomes exp2), the warp updates
// its running max and sum (online softmax, as in FlashAttention), then the
// lanes, each owning Dv/32 output columns, accumulate the 32 weighted value
// rows with coalesced loads. All accumulation is fp32.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

cudaError_t launch_attn_tc(const AttnProblem &p, cudaStream_t stream, bool *taken);

namespace {

__device__ unsigned int g_attn_cc_error = 0;  // kErrBadIndex bits

constexpr int kHeadsPerBlock = 4;
constexpr int kMaxCols = 16;  // Dv <= 32 * 16 = 512

struct AttnArgs {
    const void *q, *k_cache, *v_cache;
    const int32_t *idx;
    int Tq, L, k, Hq, Hkv, Dqk, Dv;
    float scale_log2;
    int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
    void *out;
    float *lse;
};

template <typename T, bool kVec>
__device__ __forceinline__ float dot_row(const float *q_sm, const T *krow, int D) {
    float acc = 0.0f;
    if constexpr (kVec) {
        // bf16 rows, 16-byte aligned, D % 8 == 0
        const uint4 *kv = reinterpret_cast<const uint4 *>(krow);
        for (int c = 0; c < D / 8; ++c) {
            float f[8];
            bf16x8_to_f32(__ldg(kv + c), f);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc = fmaf(q_sm[c * 8 + u], f[u], acc);
        }
    } else {
        for (int e = 0; e < D; ++e) acc = fmaf(q_sm[e], Elem<T>::load(krow, e), acc);
    }
    return acc;
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kHeadsPerBlock * kWarp)
attn_cuda_core_kernel(AttnArgs a) {
    extern __shared__ float smem[];
    float *q_sm_all = smem;                                                   // [4][Dqk]
    int32_t *idx_sm = reinterpret_cast<int32_t *>(smem + kHeadsPerBlock * a.Dqk);  // [k]

    const int row = blockIdx.x;
    const int b = row / a.Tq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y * kHeadsPerBlock + warp;

    const T *q = static_cast<const T *>(a.q);
    for (int x = threadIdx.x; x < a.k; x += blockDim.x) {
        const int s = a.idx[(size_t)row * a.k + x];
        note_bad_index(&g_attn_cc_error, s, a.L);
        idx_sm[x] = (s >= 0 && s < a.L) ? s : -1;  // positions outside [0, L) are skipped
    }
    for (int x = threadIdx.x; x < kHeadsPerBlock * a.Dqk; x += blockDim.x) {
        const int hh = blockIdx.y * kHeadsPerBlock + x / a.Dqk;
        const int e = x % a.Dqk;
        q_sm_all[x] = hh < a.Hq ? Elem<T>::load(q, ((size_t)row * a.Hq + hh) * a.Dqk + e) * a.scale_log2
                                : 0.0f;
    }
    __syncthreads();
    if (h >= a.Hq) return;

    const float *q_sm = q_sm_all + warp * a.Dqk;
    const int g = h / (a.Hq / a.Hkv);
    const T *kbase = static_cast<const T *>(a.k_cache) + b * a.k_sb + g * a.k_sh;
    const T *vbase = static_cast<const T *>(a.v_cache) + b * a.v_sb + g * a.v_sh;

    float m = -INFINITY, l = 0.0f;
    float acc[kMaxCols];
#pragma unroll
    for (int c = 0; c < kMaxCols; ++c) acc[c] = 0.0f;

    for (int j0 = 0; j0 < a.k; j0 += kWarp) {
        const int j = j0 + lane;
        const int s = j < a.k ? idx_sm[j] : -1;
        float z = -INFINITY;
        if (s >= 0) z = dot_row<T, kVec>(q_sm, kbase + s * a.k_ss, a.Dqk);
        const float zmax = warp_max(z);
        if (zmax == -INFINITY) continue;  // no valid position in this group (uniform)
        const float m_new = fmaxf(m, zmax);
        const float corr = exp2f(m - m_new);
        const float p = s >= 0 ? exp2f(z - m_new) : 0.0f;
        l = l * corr + warp_sum(p);
#pragma unroll
        for (int c = 0; c < kMaxCols; ++c) acc[c] *= corr;
        for (int r = 0; r < kWarp; ++r) {
            const int sr = __shfl_sync(0xffffffffu, s, r);
            const float pr = __shfl_sync(0xffffffffu, p, r);
            if (sr < 0) continue;
            const T *vrow = vbase + sr * a.v_ss;
#pragma unroll
            for (int c = 0; c < kMaxCols; ++c) {
                const int e = lane + c * kWarp;
                if (e < a.Dv) acc[c] = fmaf(pr, Elem<T>::load(vrow, e), acc[c]);
            }
        }
        m = m_new;
    }

    T *out = static_cast<T *>(a.out) + ((size_t)row * a.Hq + h) * a.Dv;
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
    for (int c = 0; c < kMaxCols; ++c) {
        const int e = lane + c * kWarp;
        if (e < a.Dv) Elem<T>::store(out, e, acc[c] * inv);
    }
    if (a.lse != nullptr && lane == 0) {
        // m is in log2 units: lse = (m + log2 l) * ln 2
        a.lse[(size_t)row * a.Hq + h] = l > 0.0f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
}

template <typename T, bool kVec>
cudaError_t launch_cuda_core(const AttnProblem &p, cudaStream_t stream) {
    AttnArgs a;
    a.q = p.q; a.k_cache = p.k_cache; a.v_cache = p.v_cache; a.idx = p.idx;
    a.Tq = p.Tq; a.L = p.L; a.k = p.k; a.Hq = p.Hq; a.Hkv = p.Hkv; a.Dqk = p.Dqk; a.Dv = p.Dv;
    a.scale_log2 = p.scale * 1.4426950408889634f;
    a.k_sb = p.k_sb; a.k_ss = p.k_ss; a.k_sh = p.k_sh;
    a.v_sb = p.v_sb; a.v_ss = p.v_ss; a.v_sh = p.v_sh;
    a.out = p.out; a.lse = p.lse;
    const size_t smem = sizeof(float) * kHeadsPerBlock * p.Dqk + sizeof(int32_t) * p.k;
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    if (smem > (size_t)info.max_smem_optin) return cudaErrorInvalidValue;
    auto kern = attn_cuda_core_kernel<T, kVec>;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    dim3 grid(p.B * p.Tq, ceil_div(p.Hq, kHeadsPerBlock));
    kern<<<grid, kHeadsPerBlock * kWarp, smem, stream>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

unsigned int attn_cc_take_device_error() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_cc_error, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_attn_cc_error, &zero, sizeof(zero));
    return v;
}

size_t attn_cuda_core_smem_bytes(int Dqk, int k) {
    return sizeof(float) * kHeadsPerBlock * Dqk + sizeof(int32_t) * k;
}

cudaError_t launch_attn_cuda_core(const AttnProblem &p, cudaStream_t stream) {
    if (p.Dv > kWarp * kMaxCols) return cudaErrorInvalidValue;
    if (p.dt == DSA_F32) return launch_cuda_core<float, false>(p, stream);
    const bool vec = (p.Dqk % 8 == 0) && (p.k_ss % 8 == 0) && (p.k_sb % 8 == 0) &&
                     (p.k_sh % 8 == 0) && ((uintptr_t)p.k_cache % 16 == 0);
    return vec ? launch_cuda_core<__nv_bfloat16, true>(p, stream)
               : launch_cuda_core<__nv_bfloat16, false>(p, stream);
}

cudaError_t launch_attn_perhead(const AttnProblem &p, cudaStream_t stream, bool *taken);

cudaError_t launch_attn(const AttnProblem &p, cudaStream_t stream) {
    bool taken = false;
    cudaError_t err = launch_attn_tc(p, stream, &taken);
    if (taken || err != cudaSuccess) return err;
    err = launch_attn_perhead(p, stream, &taken);
    if (taken || err != cudaSuccess) return err;
    return launch_attn_cuda_core(p, stream);
}

size_t attn_tc_workspace_bytes(const AttnProblem &p);
bool attn_tc_takes(const AttnProblem &p);
int perhead_row_group(const AttnProblem &p);

bool attn_mqa_tc_supported(const AttnProblem &p);
int attn_mqa_tc_row_group();

int attn_row_group(const AttnProblem &p) {
    if (attn_mqa_tc_supported(p)) return attn_mqa_tc_row_group();
    if (attn_tc_takes(p)) return 1;
    const int g = perhead_row_group(p);
    return g > 0 ? g : 1;
}

size_t attn_workspace_bytes(const AttnProblem &p) { return attn_tc_workspace_bytes(p); }

}  // namespace dsa
