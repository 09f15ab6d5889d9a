// Backward pass of the lightning indexer on CUDA cores (any H, d; fp32 or
// bf16 inputs).
//
// The indexer score ("DeepSeek Sparse Attention: Learned Token Selection from
// Scratch" §2.1)
//   I[t,s] = sum_j w[t,j] ReLU(x[t,j,s]),  x[t,j,s] = q[t,j] . k[s],  s <= t
// receives the gradient g[t,s] = d loss / d I[t,s] of the indexer's training
// loss (§5.4, §6.2; by §6.4 that loss reaches only the indexer). With
// G[t,j,s] = g[t,s] w[t,j] [x[t,j,s] > 0] (ReLU'(0) = 0):
//   dw[t,j] = sum_{s<=t} g[t,s] ReLU(x[t,j,s])
//   dq[t,j] = sum_{s<=t} G[t,j,s] k[s]
//   dk[s]   = sum_{t>=s} sum_j G[t,j,s] q[t,j]
//
// Query side: one block per query row walks its keys in chunks of 32; key
// side: one block per chunk of 32 keys walks the query rows at or after it.
// Each recomputes x for its chunk (H x 32 dot products), forms G in shared
// memory, and accumulates its outputs in shared memory in fp32. This path
// serves every shape the tensor-core kernels do not take (small heads, fp32
// inputs) and is exact up to fp32 rounding.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

cudaError_t launch_indexer_bwd_tc(const IndexerBwdProblem &p, cudaStream_t stream, bool *taken);

namespace {

constexpr int kChunk = 32;
constexpr int kThreads = 256;

struct BwdParams {
    const void *q_idx, *k_idx;
    const float *w, *grad;
    int B, Tq, L, q_pos0, H, d;
    float *dq, *dk, *dw;
};

// x = q_s[j] . k_s[c] for every (j, c < nk); writes G[j][c] and, when R is
// not null, R[j][c] = g ReLU(x).
__device__ __forceinline__ void chunk_terms(const float *q_s, const float *k_s, int kpitch, const float *g_s,
                                            const float *w_s, int H, int d, int nk, float *G, float *R) {
    for (int pr = threadIdx.x; pr < H * kChunk; pr += blockDim.x) {
        const int j = pr / kChunk, c = pr - j * kChunk;
        float gx = 0.f, rx = 0.f;
        if (c < nk) {
            float x = 0.f;
            for (int e = 0; e < d; ++e) x = fmaf(q_s[j * d + e], k_s[c * kpitch + e], x);
            gx = x > 0.f ? g_s[c] * w_s[j] : 0.f;
            rx = g_s[c] * fmaxf(x, 0.f);
        }
        G[pr] = gx;
        if (R) R[pr] = rx;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
indexer_bwd_q_kernel(const BwdParams p) {
    extern __shared__ float sm[];
    const int H = p.H, d = p.d, kpitch = d + 1;
    float *q_s = sm;                          // [H * d]
    float *dq_s = q_s + H * d;                // [H * d]
    float *k_s = dq_s + H * d;                // [kChunk][d + 1]
    float *G = k_s + kChunk * kpitch;         // [H][kChunk]
    float *R = G + H * kChunk;                // [H][kChunk]
    float *g_s = R + H * kChunk;              // [kChunk]
    float *w_s = g_s + kChunk;                // [H]
    float *dw_s = w_s + H;                    // [H]

    const int row = blockIdx.x;
    const int b = row / p.Tq, t = p.q_pos0 + row % p.Tq;
    const T *q = static_cast<const T *>(p.q_idx) + (size_t)row * H * d;
    const T *kb = static_cast<const T *>(p.k_idx) + (size_t)b * p.L * d;
    const float *g = p.grad + (size_t)row * p.L;
    for (int x = threadIdx.x; x < H * d; x += blockDim.x) {
        q_s[x] = Elem<T>::load(q, x);
        dq_s[x] = 0.f;
    }
    for (int j = threadIdx.x; j < H; j += blockDim.x) {
        w_s[j] = p.w[(size_t)row * H + j];
        dw_s[j] = 0.f;
    }
    for (int s0 = 0; s0 <= t; s0 += kChunk) {
        const int nk = min(kChunk, t + 1 - s0);
        __syncthreads();  // the previous chunk's readers are done
        for (int x = threadIdx.x; x < kChunk * d; x += blockDim.x) {
            const int c = x / d, e = x - c * d;
            k_s[c * kpitch + e] = c < nk ? Elem<T>::load(kb, (size_t)(s0 + c) * d + e) : 0.f;
        }
        for (int c = threadIdx.x; c < kChunk; c += blockDim.x) g_s[c] = c < nk ? g[s0 + c] : 0.f;
        __syncthreads();
        chunk_terms(q_s, k_s, kpitch, g_s, w_s, H, d, nk, G, R);
        __syncthreads();
        for (int o = threadIdx.x; o < H * d; o += blockDim.x) {
            const int j = o / d, e = o - j * d;
            float acc = 0.f;
            for (int c = 0; c < nk; ++c) acc = fmaf(G[j * kChunk + c], k_s[c * kpitch + e], acc);
            dq_s[o] += acc;
        }
        for (int j = threadIdx.x; j < H; j += blockDim.x) {
            float acc = 0.f;
            for (int c = 0; c < nk; ++c) acc += R[j * kChunk + c];
            dw_s[j] += acc;
        }
    }
    __syncthreads();
    if (p.dq)
        for (int o = threadIdx.x; o < H * d; o += blockDim.x) p.dq[(size_t)row * H * d + o] = dq_s[o];
    if (p.dw)
        for (int j = threadIdx.x; j < H; j += blockDim.x) p.dw[(size_t)row * H + j] = dw_s[j];
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
indexer_bwd_k_kernel(const BwdParams p) {
    extern __shared__ float sm[];
    const int H = p.H, d = p.d, kpitch = d + 1;
    float *q_s = sm;                          // [H * d]
    float *dk_s = q_s + H * d;                // [kChunk * d]
    float *k_s = dk_s + kChunk * d;           // [kChunk][d + 1]
    float *G = k_s + kChunk * kpitch;         // [H][kChunk]
    float *g_s = G + H * kChunk;              // [kChunk]
    float *w_s = g_s + kChunk;                // [H]

    const int nchunks = (p.L + kChunk - 1) / kChunk;
    const int b = blockIdx.x / nchunks;
    const int s0 = (blockIdx.x - b * nchunks) * kChunk;
    const int nk = min(kChunk, p.L - s0);
    const T *kb = static_cast<const T *>(p.k_idx) + (size_t)b * p.L * d;
    for (int x = threadIdx.x; x < kChunk * d; x += blockDim.x) {
        const int c = x / d, e = x - c * d;
        k_s[c * kpitch + e] = c < nk ? Elem<T>::load(kb, (size_t)(s0 + c) * d + e) : 0.f;
        dk_s[x] = 0.f;
    }
    const int i0 = max(0, s0 - p.q_pos0);  // first query row with t >= s0
    for (int i = i0; i < p.Tq; ++i) {
        const int t = p.q_pos0 + i;
        const size_t row = (size_t)b * p.Tq + i;
        __syncthreads();  // the previous row's readers are done
        const T *q = static_cast<const T *>(p.q_idx) + row * H * d;
        for (int x = threadIdx.x; x < H * d; x += blockDim.x) q_s[x] = Elem<T>::load(q, x);
        for (int j = threadIdx.x; j < H; j += blockDim.x) w_s[j] = p.w[row * H + j];
        for (int c = threadIdx.x; c < kChunk; c += blockDim.x)
            g_s[c] = (c < nk && s0 + c <= t) ? p.grad[row * p.L + s0 + c] : 0.f;
        __syncthreads();
        chunk_terms(q_s, k_s, kpitch, g_s, w_s, H, d, nk, G, nullptr);
        __syncthreads();
        for (int o = threadIdx.x; o < kChunk * d; o += blockDim.x) {
            const int c = o / d, e = o - c * d;
            float acc = 0.f;
            for (int j = 0; j < H; ++j) acc = fmaf(G[j * kChunk + c], q_s[j * d + e], acc);
            dk_s[o] += acc;
        }
    }
    __syncthreads();
    for (int o = threadIdx.x; o < nk * d; o += blockDim.x) p.dk[((size_t)b * p.L + s0) * d + o] = dk_s[o];
}

size_t q_smem(int H, int d) {
    return sizeof(float) * (2 * (size_t)H * d + (size_t)kChunk * (d + 1) + 2 * (size_t)H * kChunk + kChunk + 2 * H);
}
size_t k_smem(int H, int d) {
    return sizeof(float) * ((size_t)H * d + (size_t)kChunk * d + (size_t)kChunk * (d + 1) + (size_t)H * kChunk +
                            kChunk + H);
}

template <typename T>
cudaError_t launch_cuda_core(const IndexerBwdProblem &p, cudaStream_t stream) {
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    BwdParams bp{p.q_idx, p.k_idx, p.w, p.grad, p.B, p.Tq, p.L, p.q_pos0, p.H, p.d, p.dq, p.dk, p.dw};
    if (p.dq || p.dw) {
        const size_t smem = q_smem(p.H, p.d);
        if (smem > (size_t)info.max_smem_optin) return cudaErrorInvalidValue;
        auto kern = indexer_bwd_q_kernel<T>;
        if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return err;
        kern<<<(unsigned)(p.B * p.Tq), kThreads, smem, stream>>>(bp);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (p.dk) {
        const size_t smem = k_smem(p.H, p.d);
        if (smem > (size_t)info.max_smem_optin) return cudaErrorInvalidValue;
        auto kern = indexer_bwd_k_kernel<T>;
        if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return err;
        const long long blocks = (long long)p.B * ((p.L + kChunk - 1) / kChunk);
        kern<<<(unsigned)blocks, kThreads, smem, stream>>>(bp);
        count_launch();
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace

size_t indexer_bwd_cuda_core_smem_bytes(int H, int d) {
    const size_t a = q_smem(H, d), b = k_smem(H, d);
    return a > b ? a : b;
}

cudaError_t launch_indexer_bwd(const IndexerBwdProblem &p, cudaStream_t stream) {
    bool taken = false;
    cudaError_t err = launch_indexer_bwd_tc(p, stream, &taken);
    if (taken || err != cudaSuccess) return err;
    if (p.dt == DSA_F32) return launch_cuda_core<float>(p, stream);
    return launch_cuda_core<__nv_bfloat16>(p, stream);
}

}  // namespace dsa
