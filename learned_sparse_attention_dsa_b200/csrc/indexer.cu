// Lightning-indexer scores on CUDA cores (any H, d; fp32, bf16 or e4m3 inputs).
//
//   I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]),  s <= t
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §2.1).
//
// One block scores one query row against 128 consecutive keys; the query's
// H x d block and the key tile (transposed, so that thread s reads column s
// without bank conflicts) are staged in shared memory as fp32. Products and
// the weighted head sum are accumulated in fp32; with integer-valued inputs
// and power-of-two weights every partial sum is exact, so the result equals
// the exact score. This kernel serves the small-head shapes (the worked
// example's H=2, d=2) and any shape the tensor-core kernel does not take.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

cudaError_t launch_indexer_tc(const IndexerProblem &p, cudaStream_t stream, bool *taken);

namespace {

constexpr int kKeysPerBlock = 128;

template <typename T>
__global__ void __launch_bounds__(kKeysPerBlock)
indexer_cuda_core_kernel(const T *__restrict__ q_idx, const T *__restrict__ k_idx,
                         const float *__restrict__ w, int Tq, int L, int q_pos0, int H, int d,
                         float *__restrict__ scores, int fill_masked, int row0) {
    extern __shared__ float smem[];
    float *q_sm = smem;                 // [H * d]
    float *w_sm = q_sm + H * d;         // [H]
    float *k_sm = w_sm + H;             // [d][kKeysPerBlock]

    const int row_id = row0 + blockIdx.y;
    const int i = row_id % Tq;
    const int b = row_id / Tq;
    const int t = q_pos0 + i;
    const int s0 = blockIdx.x * kKeysPerBlock;
    const int s = s0 + threadIdx.x;
    const size_t row = (size_t)b * Tq + i;
    float *out = scores + row * L;

    if (s0 > t) {  // the whole tile is above the diagonal
        if (fill_masked && s < L) out[s] = -INFINITY;
        return;
    }
    for (int x = threadIdx.x; x < H * d; x += blockDim.x)
        q_sm[x] = Elem<T>::load(q_idx, row * H * d + x);
    for (int x = threadIdx.x; x < H; x += blockDim.x) w_sm[x] = w[row * H + x];
    for (int x = threadIdx.x; x < kKeysPerBlock * d; x += blockDim.x) {
        const int key = x / d, e = x - key * d;
        const int ss = s0 + key;
        k_sm[e * kKeysPerBlock + key] =
            (ss < L) ? Elem<T>::load(k_idx, ((size_t)b * L + ss) * d + e) : 0.0f;
    }
    __syncthreads();
    if (s >= L) return;
    if (s > t) {
        if (fill_masked) out[s] = -INFINITY;
        return;
    }
    float I = 0.0f;
    for (int j = 0; j < H; ++j) {
        float dot = 0.0f;
        for (int e = 0; e < d; ++e) dot = fmaf(q_sm[j * d + e], k_sm[e * kKeysPerBlock + threadIdx.x], dot);
        I = fmaf(w_sm[j], fmaxf(dot, 0.0f), I);
    }
    out[s] = I;
}

template <typename T>
cudaError_t launch_cuda_core(const IndexerProblem &p, cudaStream_t stream) {
    const size_t smem = sizeof(float) * ((size_t)p.H * p.d + p.H + (size_t)p.d * kKeysPerBlock);
    DeviceInfo info;
    cudaError_t err = device_info(&info);
    if (err != cudaSuccess) return err;
    if (smem > (size_t)info.max_smem_optin) return cudaErrorInvalidValue;
    auto kern = indexer_cuda_core_kernel<T>;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    const int rows = p.B * p.Tq;
    for (int row0 = 0; row0 < rows; row0 += 65535) {  // grid.y is limited to 65535
        dim3 grid(ceil_div(p.L, kKeysPerBlock), rows - row0 < 65535 ? rows - row0 : 65535);
        kern<<<grid, kKeysPerBlock, smem, stream>>>(static_cast<const T *>(p.q_idx),
                                                    static_cast<const T *>(p.k_idx), p.w, p.Tq, p.L,
                                                    p.q_pos0, p.H, p.d, p.scores, p.fill_masked ? 1 : 0,
                                                    row0);
        count_launch();
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

}  // namespace

size_t indexer_cuda_core_smem_bytes(int H, int d) {
    return sizeof(float) * ((size_t)H * d + H + (size_t)d * kKeysPerBlock);
}

cudaError_t launch_indexer_cuda_core(const IndexerProblem &p, cudaStream_t stream) {
    if (p.dt == DSA_F32) return launch_cuda_core<float>(p, stream);
    if (p.dt == DSA_E4M3) return launch_cuda_core<__nv_fp8_e4m3>(p, stream);
    return launch_cuda_core<__nv_bfloat16>(p, stream);
}

cudaError_t launch_indexer(const IndexerProblem &p, cudaStream_t stream) {
    bool taken = false;
    cudaError_t err = launch_indexer_tc(p, stream, &taken);
    if (taken || err != cudaSuccess) return err;
    return launch_indexer_cuda_core(p, stream);
}

}  // namespace dsa
