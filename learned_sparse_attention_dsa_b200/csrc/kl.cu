// The indexer's training loss and its gradient with respect to the scores.
//
//   loss_t = KL(p_t || Softmax(I_t)) over the row's set, p_t = a_t / sum(a_t)
// ("DeepSeek Sparse Attention: Learned Token Selection from Scratch" §5.4 for
// the dense warm-up, set = {s <= t}; §6.2 for the sparse stage, set = S_t;
// the normalisation of the target weights a is step 2 of §5.2), and
//   d(sum_t loss_t) / d I[t,s] = softmax(I_t)_s - p_t[s] on the set, 0 off it.
//
// One CTA per query row. Pass 1 reads the row once and keeps, per thread, a
// running max m and sum z of exp(I - m) (online softmax) and the sums
// S = sum a, sum a*I and sum a*log a, so that
//   loss = (sum a log a) / S - log S - (sum a I) / S + (m + log z)
// needs no second pass. Pass 2 (only when the gradient is wanted) reads the
// row again, from L2, and writes exp(I - LSE) - a / S. HBM-bound: 8 bytes
// read per causal pair (score and target) plus 4 written for the gradient.
// exp and log use the hardware base-2 approximations: with the library
// functions the kernel was bound by instruction issue, not by memory.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// exp(x) and log(x) through the hardware base-2 approximations (relative
// error below 2^-21 after the scaling); ex2 of -inf is 0.
__device__ __forceinline__ float fast_exp(float x) { return ex2_approx(x * kLog2e); }
__device__ __forceinline__ float fast_log(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y * kLn2;
}

struct Acc {
    float m, z, S, aI, alna;
};

__device__ __forceinline__ void acc_init(Acc &c) {
    c.m = -INFINITY;
    c.z = 0.f;
    c.S = 0.f;
    c.aI = 0.f;
    c.alna = 0.f;
}

__device__ __forceinline__ void acc_add(Acc &c, float I, float a) {
    if (I == -INFINITY) {
        // exp(-inf) adds nothing to z
    } else if (I > c.m) {
        c.z = c.z * fast_exp(c.m - I) + 1.f;  // exp(-inf) = 0 for the first element
        c.m = I;
    } else {
        c.z += fast_exp(I - c.m);
    }
    c.S += a;
    if (a > 0.f) {
        c.aI += a * I;
        c.alna += a * fast_log(a);
    }
}

__device__ __forceinline__ void acc_merge(Acc &c, const Acc &o) {
    const float m = fmaxf(c.m, o.m);
    if (m == -INFINITY) {
        c.z = 0.f;
    } else {
        c.z = c.z * fast_exp(c.m - m) + o.z * fast_exp(o.m - m);
    }
    c.m = m;
    c.S += o.S;
    c.aI += o.aI;
    c.alna += o.alna;
}

__device__ __forceinline__ Acc acc_shfl(const Acc &c, int o) {
    Acc r;
    r.m = __shfl_xor_sync(0xffffffffu, c.m, o);
    r.z = __shfl_xor_sync(0xffffffffu, c.z, o);
    r.S = __shfl_xor_sync(0xffffffffu, c.S, o);
    r.aI = __shfl_xor_sync(0xffffffffu, c.aI, o);
    r.alna = __shfl_xor_sync(0xffffffffu, c.alna, o);
    return r;
}

// Whole-block combine; every thread returns the row's totals.
__device__ __forceinline__ Acc block_reduce(Acc c, Acc *sh) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc_merge(c, acc_shfl(c, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[warp] = c;
    __syncthreads();
    Acc r = sh[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) acc_merge(r, sh[w]);
    return r;
}

struct KlParams {
    const float *scores;   // [rows, L]
    const float *target;   // dense [rows, L]; sparse [rows, k]
    const int32_t *idx;    // sparse only: [rows, k]
    int Tq, L, q_pos0, k;
    float *loss_rows;      // [rows]
    float *grad;           // [rows, L] or null
    bool vec4;             // dense rows may use 16-byte accesses
};

template <bool SPARSE>
__global__ void __launch_bounds__(kThreads)
indexer_kl_kernel(const KlParams p) {
    __shared__ Acc red[kWarps];
    const int row = blockIdx.x;
    const int t = p.q_pos0 + row % p.Tq;
    const int tid = threadIdx.x;
    const float *I = p.scores + (size_t)row * p.L;

    Acc c;
    acc_init(c);
    if (SPARSE) {
        const int32_t *sel = p.idx + (size_t)row * p.k;
        const float *a = p.target + (size_t)row * p.k;
        for (int j = tid; j < p.k; j += kThreads) {
            const int s = sel[j];
            if (s >= 0 && s <= t) acc_add(c, I[s], a[j]);
        }
    } else {
        const float *a = p.target + (size_t)row * p.L;
        const int n = t + 1;
        int s0 = 0;
        if (p.vec4) {
            const int n4 = n & ~3;
            const float4 *I4 = reinterpret_cast<const float4 *>(I);
            const float4 *a4 = reinterpret_cast<const float4 *>(a);
            for (int v = tid; v < (n4 >> 2); v += kThreads) {
                const float4 x = I4[v], y = a4[v];
                acc_add(c, x.x, y.x);
                acc_add(c, x.y, y.y);
                acc_add(c, x.z, y.z);
                acc_add(c, x.w, y.w);
            }
            s0 = n4;
        }
        for (int s = s0 + tid; s < n; s += kThreads) acc_add(c, I[s], a[s]);
    }
    const Acc r = block_reduce(c, red);
    const bool any = r.S > 0.f;
    const float lse = r.m + logf(r.z);
    if (tid == 0) {
        const float loss = any ? (r.alna / r.S - logf(r.S) - r.aI / r.S + lse) : 0.f;
        p.loss_rows[row] = loss;
    }
    if (p.grad == nullptr) return;

    float *g = p.grad + (size_t)row * p.L;
    const float inv_S = any ? 1.f / r.S : 0.f;
    if (SPARSE) {
        // zero the row, then write the set's entries over it
        for (int s = tid; s < p.L; s += kThreads) g[s] = 0.f;
        __syncthreads();
        if (!any) return;
        const int32_t *sel = p.idx + (size_t)row * p.k;
        const float *a = p.target + (size_t)row * p.k;
        for (int j = tid; j < p.k; j += kThreads) {
            const int s = sel[j];
            if (s >= 0 && s <= t) g[s] = fast_exp(I[s] - lse) - a[j] * inv_S;
        }
    } else {
        const float *a = p.target + (size_t)row * p.L;
        const int n = any ? t + 1 : 0;  // entries at s >= n are 0
        int s0 = 0;
        if (p.vec4) {
            const float4 *I4 = reinterpret_cast<const float4 *>(I);
            const float4 *a4 = reinterpret_cast<const float4 *>(a);
            float4 *g4 = reinterpret_cast<float4 *>(g);
            for (int v = tid; v < (p.L >> 2); v += kThreads) {
                const int s = v << 2;
                float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s < n) {
                    const float4 x = I4[v], y = a4[v];
                    o.x = fast_exp(x.x - lse) - y.x * inv_S;
                    if (s + 1 < n) o.y = fast_exp(x.y - lse) - y.y * inv_S;
                    if (s + 2 < n) o.z = fast_exp(x.z - lse) - y.z * inv_S;
                    if (s + 3 < n) o.w = fast_exp(x.w - lse) - y.w * inv_S;
                }
                g4[v] = o;
            }
            s0 = p.L & ~3;
        }
        for (int s = s0 + tid; s < p.L; s += kThreads) g[s] = s < n ? fast_exp(I[s] - lse) - a[s] * inv_S : 0.f;
    }
}

// sum over rows of loss_rows in a fixed order (fp64 partial sums): the same
// total on every call
__global__ void __launch_bounds__(1024) kl_sum_kernel(const float *loss_rows, long long rows, float *out) {
    __shared__ double part[32];
    double s = 0.0;
    for (long long r = threadIdx.x; r < rows; r += blockDim.x) s += (double)loss_rows[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) part[warp] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double total = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += part[w];
        *out = (float)total;
    }
}

}  // namespace

cudaError_t launch_indexer_kl(const KlProblem &p, cudaStream_t stream) {
    const long long rows = (long long)p.B * p.Tq;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    KlParams kp{p.scores, p.target, p.idx, p.Tq, p.L, p.q_pos0, p.k, p.loss_rows, p.grad, false};
    const bool a16 = ((uintptr_t)p.scores % 16 == 0) && ((uintptr_t)p.target % 16 == 0) &&
                     (p.grad == nullptr || (uintptr_t)p.grad % 16 == 0);
    kp.vec4 = p.idx == nullptr && p.L % 4 == 0 && a16;
    if (p.idx != nullptr)
        indexer_kl_kernel<true><<<(unsigned)rows, kThreads, 0, stream>>>(kp);
    else
        indexer_kl_kernel<false><<<(unsigned)rows, kThreads, 0, stream>>>(kp);
    count_launch();
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || p.loss_sum == nullptr) return err;
    kl_sum_kernel<<<1, 1024, 0, stream>>>(p.loss_rows, rows, p.loss_sum);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsa
