// C ABI of the DSA forward path: argument checks, workspace layout, dispatch.
//
// Every entry point validates on the host before enqueuing anything; a failed
// check returns a status and leaves the stream untouched.
#include <math.h>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dsa {

size_t indexer_cuda_core_smem_bytes(int H, int d);
size_t attn_cuda_core_smem_bytes(int Dqk, int k);

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::mutex g_info_mutex;
std::atomic<uint64_t> g_launches{0};
}  // namespace

void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

cudaError_t device_info(DeviceInfo *out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_info_mutex);
    if (g_info[dev].device != dev) {
        DeviceInfo d;
        d.device = dev;
        if ((err = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return err;
        if ((err = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
            cudaSuccess)
            return err;
        if ((err = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return err;
        if ((err = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
            return err;
        g_info[dev] = d;
    }
    *out = g_info[dev];
    return cudaSuccess;
}

}  // namespace dsa

using namespace dsa;

namespace {

constexpr size_t kWsAlign = 256;

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }
size_t dtype_bytes(dsa_dtype dt) { return dt == DSA_F32 ? 4 : (dt == DSA_E4M3 ? 1 : 2); }
bool valid_dtype(dsa_dtype dt) { return dt == DSA_F32 || dt == DSA_BF16; }
bool valid_indexer_dtype(dsa_dtype dt) { return valid_dtype(dt) || dt == DSA_E4M3; }

dsa_status from_cuda(cudaError_t err) { return err == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

// Host-side shared-memory limit of the current device (0 when unknown).
int smem_limit() {
    DeviceInfo info;
    return device_info(&info) == cudaSuccess ? info.max_smem_optin : 0;
}

dsa_status check_rows(int B, int Tq, int L, int q_pos0) {
    if (B < 1 || Tq < 1 || L < 1 || q_pos0 < 0) return DSA_ERR_INVALID_ARG;
    if ((int64_t)q_pos0 + Tq > L) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

dsa_status check_indexer(const void *q_idx, const void *k_idx, const float *w, int B, int Tq, int L,
                         int q_pos0, int H_I, int d_I, dsa_dtype dt, const float *scores) {
    if (!q_idx || !k_idx || !w || !scores) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_rows(B, Tq, L, q_pos0);
    if (st != DSA_OK) return st;
    if (H_I < 1 || d_I < 1) return DSA_ERR_INVALID_ARG;
    if (!valid_indexer_dtype(dt)) return DSA_ERR_UNSUPPORTED;
    const size_t eb = dtype_bytes(dt);
    if (!aligned(q_idx, eb) || !aligned(k_idx, eb) || !aligned(w, 4) || !aligned(scores, 4))
        return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

dsa_status check_indexer_fits(int H_I, int d_I) {
    // The CUDA-core kernel is the fallback for every shape: its staging must fit.
    const int lim = smem_limit();
    if (lim == 0) return DSA_ERR_CUDA;
    if (indexer_cuda_core_smem_bytes(H_I, d_I) > (size_t)lim) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
}

dsa_status check_topk(const float *scores, int B, int Tq, int L, int q_pos0, int k, const int32_t *idx) {
    if (!scores || !idx) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_rows(B, Tq, L, q_pos0);
    if (st != DSA_OK) return st;
    if (k < 1) return DSA_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(idx, 4)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

// The attention shape alone (no pointers): sizes, strides, dtype, and the
// shared-memory staging of the CUDA-core kernel that every shape falls back to.
dsa_status check_attn_shape(const dsa_attn_shape *sh, dsa_dtype dt) {
    if (!sh) return DSA_ERR_INVALID_ARG;
    if (sh->B < 1 || sh->Tq < 1 || sh->L < 1 || sh->k < 1) return DSA_ERR_INVALID_ARG;
    if (sh->Hq < 1 || sh->Hkv < 1 || sh->Hq % sh->Hkv != 0) return DSA_ERR_INVALID_ARG;
    if (sh->Dqk < 1 || sh->Dv < 1) return DSA_ERR_INVALID_ARG;
    if (!(sh->scale == sh->scale) || isinf(sh->scale)) return DSA_ERR_INVALID_ARG;
    if (sh->k_stride_s < 1 || sh->v_stride_s < 1 || sh->k_stride_b < 0 || sh->v_stride_b < 0 ||
        sh->k_stride_h < 0 || sh->v_stride_h < 0)
        return DSA_ERR_INVALID_ARG;
    if (!valid_dtype(dt)) return DSA_ERR_UNSUPPORTED;
    if (sh->Dv > 512) return DSA_ERR_UNSUPPORTED;
    const int lim = smem_limit();
    if (lim == 0) return DSA_ERR_CUDA;
    if (attn_cuda_core_smem_bytes(sh->Dqk, sh->k) > (size_t)lim) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
}

dsa_status check_attn(const void *q, const void *k_cache, const void *v_cache, const int32_t *idx,
                      const dsa_attn_shape *sh, dsa_dtype dt, const void *out, const float *lse) {
    if (!sh || !q || !k_cache || !v_cache || !idx || !out) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_attn_shape(sh, dt);
    if (st != DSA_OK) return st;
    const size_t eb = dtype_bytes(dt);
    if (!aligned(q, eb) || !aligned(k_cache, eb) || !aligned(v_cache, eb) || !aligned(out, eb) ||
        !aligned(idx, 4) || (lse && !aligned(lse, 4)))
        return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

AttnProblem make_attn_problem(const void *q, const void *k_cache, const void *v_cache, const int32_t *idx,
                              const dsa_attn_shape *sh, dsa_dtype dt, void *out, float *lse, void *ws,
                              size_t ws_bytes) {
    AttnProblem p;
    p.q = q; p.k_cache = k_cache; p.v_cache = v_cache; p.idx = idx;
    p.B = sh->B; p.Tq = sh->Tq; p.L = sh->L; p.k = sh->k;
    p.Hq = sh->Hq; p.Hkv = sh->Hkv; p.Dqk = sh->Dqk; p.Dv = sh->Dv; p.scale = sh->scale;
    p.k_sb = sh->k_stride_b; p.k_ss = sh->k_stride_s; p.k_sh = sh->k_stride_h;
    p.v_sb = sh->v_stride_b; p.v_ss = sh->v_stride_s; p.v_sh = sh->v_stride_h;
    p.dt = dt; p.out = out; p.lse = lse; p.ws = ws; p.ws_bytes = ws_bytes;
    return p;
}

dsa_attn_shape forward_attn_shape(const dsa_forward_args *a) {
    dsa_attn_shape sh;
    sh.B = a->B; sh.Tq = a->Tq; sh.L = a->L; sh.k = a->k;
    sh.Hq = a->Hq; sh.Hkv = a->Hkv; sh.Dqk = a->Dqk; sh.Dv = a->Dv; sh.scale = a->scale;
    sh.k_stride_b = a->k_stride_b; sh.k_stride_s = a->k_stride_s; sh.k_stride_h = a->k_stride_h;
    sh.v_stride_b = a->v_stride_b; sh.v_stride_s = a->v_stride_s; sh.v_stride_h = a->v_stride_h;
    return sh;
}

struct ForwardLayout {
    size_t scores = 0, idx = 0, topk = 0, attn = 0, total = 0;
    size_t topk_bytes = 0, attn_bytes = 0;
};

ForwardLayout forward_layout(const dsa_forward_args *a) {
    ForwardLayout lay;
    size_t off = 0;
    if (!a->scores_out) {
        lay.scores = off;
        off += align_up(sizeof(float) * (size_t)a->B * a->Tq * a->L, kWsAlign);
    }
    if (!a->idx_out) {
        lay.idx = off;
        off += align_up(sizeof(int32_t) * (size_t)a->B * a->Tq * a->k, kWsAlign);
    }
    lay.topk = off;
    lay.topk_bytes = topk_workspace_bytes(a->B, a->Tq, a->L, a->q_pos0, a->k);
    off += align_up(lay.topk_bytes, kWsAlign);
    lay.attn = off;
    dsa_attn_shape sh = forward_attn_shape(a);
    AttnProblem p = make_attn_problem(a->q, a->k_cache, a->v_cache, nullptr, &sh, a->attn_dtype, a->out,
                                      a->lse, nullptr, 0);
    lay.attn_bytes = attn_workspace_bytes(p);
    off += align_up(lay.attn_bytes, kWsAlign);
    lay.total = off;
    return lay;
}

dsa_status check_forward(const dsa_forward_args *a) {
    if (!a) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_indexer(a->q_idx, a->k_idx, a->w, a->B, a->Tq, a->L, a->q_pos0, a->H_I, a->d_I,
                                  a->idx_dtype, a->scores_out ? a->scores_out : a->w);
    if (st != DSA_OK) return st;
    if (a->k < 1) return DSA_ERR_INVALID_ARG;
    if (a->flags & ~(unsigned)DSA_FLAG_INCLUDE_SELF) return DSA_ERR_INVALID_ARG;
    if (a->idx_out && !aligned(a->idx_out, 4)) return DSA_ERR_INVALID_ARG;
    dsa_attn_shape sh = forward_attn_shape(a);
    // idx is produced internally: pass a non-null placeholder to the check
    st = check_attn(a->q, a->k_cache, a->v_cache, reinterpret_cast<const int32_t *>(a->w), &sh,
                    a->attn_dtype, a->out, a->lse);
    if (st != DSA_OK) return st;
    return check_indexer_fits(a->H_I, a->d_I);
}

}  // namespace

namespace dsa {
dsa_status validate_attn_call(const void *q, const void *k_cache, const void *v_cache, const int32_t *idx,
                              const dsa_attn_shape *sh, dsa_dtype dt, const void *out, const float *lse) {
    return check_attn(q, k_cache, v_cache, idx, sh, dt, out, lse);
}
}  // namespace dsa

extern "C" {

int dsa_version(void) { return 100; }

uint64_t dsa_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

dsa_status dsa_device_error(dsa_stream_t stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
    unsigned int words = dsa::indexer_take_device_error() | dsa::attn_mla_tc_take_device_error() |
                         dsa::indexer_bwd_take_device_error() | dsa::attn_tc_take_device_error() |
                         dsa::attn_mla_take_device_error() | dsa::attn_perhead_take_device_error() |
                         dsa::attn_cc_take_device_error() | dsa::attn_mqa_tc_take_device_error();
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
    if (words & kErrTimeout) return DSA_ERR_TIMEOUT;
    return (words & kErrBadIndex) ? DSA_ERR_BAD_INDEX : DSA_OK;
}

dsa_status dsa_set_wait_limit_ns(uint64_t ns) {
    if (dsa::indexer_set_wait_limit(ns) != cudaSuccess || dsa::indexer_bwd_set_wait_limit(ns) != cudaSuccess ||
        dsa::attn_mla_tc_set_wait_limit(ns) != cudaSuccess || dsa::attn_mqa_tc_set_wait_limit(ns) != cudaSuccess)
        return DSA_ERR_CUDA;
    return DSA_OK;
}

const char *dsa_status_string(dsa_status status) {
    switch (status) {
        case DSA_OK: return "DSA_OK";
        case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG: invalid argument";
        case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED: unsupported shape or dtype";
        case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE: workspace missing or too small";
        case DSA_ERR_CUDA: return "DSA_ERR_CUDA: CUDA runtime or launch failure";
        case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT: bounded device wait expired";
        case DSA_ERR_BAD_INDEX: return "DSA_ERR_BAD_INDEX: selected position outside [0, L) skipped";
    }
    return "unknown dsa_status";
}

dsa_status dsa_indexer_scores_ex(const void *q_idx, const void *k_idx, const float *w, int B, int Tq, int L,
                                 int q_pos0, int H_I, int d_I, dsa_dtype dt, unsigned flags, float *scores,
                                 dsa_stream_t stream) {
    dsa_status st = check_indexer(q_idx, k_idx, w, B, Tq, L, q_pos0, H_I, d_I, dt, scores);
    if (st != DSA_OK) return st;
    if (flags & ~(unsigned)DSA_INDEXER_CAUSAL_ONLY) return DSA_ERR_INVALID_ARG;
    if ((st = check_indexer_fits(H_I, d_I)) != DSA_OK) return st;
    const bool fill = (flags & DSA_INDEXER_CAUSAL_ONLY) == 0;
    IndexerProblem p{q_idx, k_idx, w, B, Tq, L, q_pos0, H_I, d_I, dt, scores, fill};
    return from_cuda(launch_indexer(p, static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_indexer_scores(const void *q_idx, const void *k_idx, const float *w, int B, int Tq, int L,
                              int q_pos0, int H_I, int d_I, dsa_dtype dt, float *scores,
                              dsa_stream_t stream) {
    return dsa_indexer_scores_ex(q_idx, k_idx, w, B, Tq, L, q_pos0, H_I, d_I, dt, 0u, scores, stream);
}

size_t dsa_topk_workspace_bytes(int B, int Tq, int L, int q_pos0, int k) {
    if (check_rows(B, Tq, L, q_pos0) != DSA_OK || k < 1) return 0;
    return topk_workspace_bytes(B, Tq, L, q_pos0, k);
}

dsa_status dsa_topk_ex(const float *scores, int B, int Tq, int L, int q_pos0, int k, unsigned flags, int32_t *idx,
                       void *ws, size_t ws_bytes, dsa_stream_t stream) {
    dsa_status st = check_topk(scores, B, Tq, L, q_pos0, k, idx);
    if (st != DSA_OK) return st;
    if (flags & ~(unsigned)DSA_FLAG_INCLUDE_SELF) return DSA_ERR_INVALID_ARG;
    const size_t need = topk_workspace_bytes(B, Tq, L, q_pos0, k);
    if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return DSA_ERR_WORKSPACE;
    TopkProblem p{scores, B, Tq, L, q_pos0, k, idx, ws, ws_bytes};
    p.include_self = (flags & DSA_FLAG_INCLUDE_SELF) != 0;
    return from_cuda(launch_topk(p, static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_topk(const float *scores, int B, int Tq, int L, int q_pos0, int k, int32_t *idx, void *ws,
                    size_t ws_bytes, dsa_stream_t stream) {
    return dsa_topk_ex(scores, B, Tq, L, q_pos0, k, 0u, idx, ws, ws_bytes, stream);
}

int dsa_sparse_attn_row_group(const dsa_attn_shape *sh, dsa_dtype dt) {
    if (check_attn_shape(sh, dt) != DSA_OK) return 0;
    AttnProblem p = make_attn_problem(nullptr, nullptr, nullptr, nullptr, sh, dt, nullptr, nullptr, nullptr, 0);
    return attn_row_group(p);
}

size_t dsa_sparse_attn_workspace_bytes(const dsa_attn_shape *sh, dsa_dtype dt) {
    if (check_attn_shape(sh, dt) != DSA_OK) return 0;
    AttnProblem p = make_attn_problem(nullptr, nullptr, nullptr, nullptr, sh, dt, nullptr, nullptr, nullptr, 0);
    return attn_workspace_bytes(p);
}

dsa_status dsa_sparse_attn(const void *q, const void *k_cache, const void *v_cache, const int32_t *idx,
                           const dsa_attn_shape *sh, dsa_dtype dt, void *out, float *lse, void *ws,
                           size_t ws_bytes, dsa_stream_t stream) {
    dsa_status st = check_attn(q, k_cache, v_cache, idx, sh, dt, out, lse);
    if (st != DSA_OK) return st;
    AttnProblem p = make_attn_problem(q, k_cache, v_cache, idx, sh, dt, out, lse, ws, ws_bytes);
    const size_t need = attn_workspace_bytes(p);
    if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return DSA_ERR_WORKSPACE;
    return from_cuda(launch_attn(p, static_cast<cudaStream_t>(stream)));
}

size_t dsa_forward_workspace_bytes(const dsa_forward_args *a) {
    if (check_forward(a) != DSA_OK) return 0;
    return forward_layout(a).total;
}

dsa_status dsa_forward(const dsa_forward_args *a, void *ws, size_t ws_bytes, dsa_stream_t stream) {
    dsa_status st = check_forward(a);
    if (st != DSA_OK) return st;
    const ForwardLayout lay = forward_layout(a);
    if (lay.total > 0 && (!ws || ws_bytes < lay.total || !aligned(ws, kWsAlign))) return DSA_ERR_WORKSPACE;
    char *base = static_cast<char *>(ws);
    float *scores = a->scores_out ? a->scores_out : reinterpret_cast<float *>(base + lay.scores);
    int32_t *idx = a->idx_out ? a->idx_out : reinterpret_cast<int32_t *>(base + lay.idx);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // Every row keeping all of its candidates (t + 1 <= k): the selection is
    // known without scores; the indexer runs only when they are asked for.
    const bool short_context = (long long)a->q_pos0 + a->Tq <= a->k;
    cudaError_t err = cudaSuccess;
    if (!short_context || a->scores_out != nullptr) {
        IndexerProblem ip{a->q_idx, a->k_idx, a->w, a->B, a->Tq, a->L, a->q_pos0, a->H_I, a->d_I,
                          a->idx_dtype, scores, a->scores_out != nullptr};
        if ((err = launch_indexer(ip, s)) != cudaSuccess) return DSA_ERR_CUDA;
    }

    TopkProblem tp{scores, a->B, a->Tq, a->L, a->q_pos0, a->k, idx,
                   lay.topk_bytes ? base + lay.topk : nullptr, lay.topk_bytes};
    tp.include_self = (a->flags & DSA_FLAG_INCLUDE_SELF) != 0;
    err = short_context ? launch_dense_selection(tp, s) : launch_topk(tp, s);
    if (err != cudaSuccess) return DSA_ERR_CUDA;

    dsa_attn_shape sh = forward_attn_shape(a);
    AttnProblem ap = make_attn_problem(a->q, a->k_cache, a->v_cache, idx, &sh, a->attn_dtype, a->out, a->lse,
                                       lay.attn_bytes ? base + lay.attn : nullptr, lay.attn_bytes);
    return from_cuda(launch_attn(ap, s));
}

dsa_status dsa_indexer_kl(const float *scores, const float *target, const int32_t *idx, int B, int Tq, int L,
                          int q_pos0, int k, float *loss_rows, float *loss_sum, float *grad, dsa_stream_t stream) {
    if (!scores || !target || !loss_rows) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_rows(B, Tq, L, q_pos0);
    if (st != DSA_OK) return st;
    if (idx && k < 1) return DSA_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(target, 4) || !aligned(loss_rows, 4) || (idx && !aligned(idx, 4)) ||
        (loss_sum && !aligned(loss_sum, 4)) || (grad && !aligned(grad, 4)))
        return DSA_ERR_INVALID_ARG;
    KlProblem p{scores, target, idx, B, Tq, L, q_pos0, idx ? k : 0, loss_rows, loss_sum, grad};
    return from_cuda(launch_indexer_kl(p, static_cast<cudaStream_t>(stream)));
}

size_t dsa_indexer_backward_workspace_bytes(int B, int Tq, int L, int q_pos0, int H_I, int d_I, dsa_dtype dt) {
    if (check_rows(B, Tq, L, q_pos0) != DSA_OK || H_I < 1 || d_I < 1 || !valid_dtype(dt)) return 0;
    // aligned placeholder pointers: the plan depends only on shapes and alignment
    const void *fake = reinterpret_cast<const void *>(uintptr_t(256));
    IndexerBwdProblem p{fake, fake, static_cast<const float *>(fake), static_cast<const float *>(fake), B, Tq, L,
                        q_pos0, H_I, d_I, dt, nullptr, reinterpret_cast<float *>(uintptr_t(256)), nullptr,
                        nullptr, 0};
    return indexer_bwd_tc_workspace_bytes(p);
}

dsa_status dsa_indexer_backward(const void *q_idx, const void *k_idx, const float *w, const float *grad, int B,
                                int Tq, int L, int q_pos0, int H_I, int d_I, dsa_dtype dt, float *dq, float *dk,
                                float *dw, void *ws, size_t ws_bytes, dsa_stream_t stream) {
    if (!q_idx || !k_idx || !w || !grad) return DSA_ERR_INVALID_ARG;
    dsa_status st = check_rows(B, Tq, L, q_pos0);
    if (st != DSA_OK) return st;
    if (H_I < 1 || d_I < 1) return DSA_ERR_INVALID_ARG;
    if (!valid_dtype(dt)) return DSA_ERR_UNSUPPORTED;
    const size_t eb = dtype_bytes(dt);
    if (!aligned(q_idx, eb) || !aligned(k_idx, eb) || !aligned(w, 4) || !aligned(grad, 4) ||
        (dq && !aligned(dq, 4)) || (dk && !aligned(dk, 4)) || (dw && !aligned(dw, 4)))
        return DSA_ERR_INVALID_ARG;
    const int lim = smem_limit();
    if (lim == 0) return DSA_ERR_CUDA;
    if (indexer_bwd_cuda_core_smem_bytes(H_I, d_I) > (size_t)lim) return DSA_ERR_UNSUPPORTED;
    IndexerBwdProblem p{q_idx, k_idx, w, grad, B, Tq, L, q_pos0, H_I, d_I, dt, dq, dk, dw, ws, ws_bytes};
    if (dk) {
        const size_t need = indexer_bwd_tc_workspace_bytes(p);
        if (need > 0 && (!ws || ws_bytes < need || !aligned(ws, 16))) return DSA_ERR_WORKSPACE;
    }
    if (!dq && !dk && !dw) return DSA_OK;
    return from_cuda(launch_indexer_bwd(p, static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_diag_gather(const void *src, int64_t pitch_bytes, int row_bytes, int n_src_rows, const int32_t *idx,
                           int64_t n, int tile_rows, uint32_t *sink, dsa_stream_t stream) {
    if (!src || !idx || !sink || n < 1 || n_src_rows < 1) return DSA_ERR_INVALID_ARG;
    if (tile_rows != 8 && tile_rows != 16 && tile_rows != 32) return DSA_ERR_INVALID_ARG;
    if (row_bytes < 16 || row_bytes > 1024 || row_bytes % 16 != 0) return DSA_ERR_INVALID_ARG;
    if (pitch_bytes < row_bytes || pitch_bytes % 16 != 0) return DSA_ERR_INVALID_ARG;
    if (!aligned(src, 16) || !aligned(idx, 4) || !aligned(sink, 4)) return DSA_ERR_INVALID_ARG;
    return from_cuda(launch_diag_gather(src, pitch_bytes, row_bytes, n_src_rows, idx, n, tile_rows, sink,
                                        static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_cp_select_candidates(const float *scores, const int32_t *idx, int rows, int L, int k, int key_pos0,
                                    float *cand_scores, int32_t *cand_idx, dsa_stream_t stream) {
    if (!scores || !idx || !cand_scores || !cand_idx) return DSA_ERR_INVALID_ARG;
    if (rows < 1 || L < 1 || k < 1 || key_pos0 < 0) return DSA_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(idx, 4) || !aligned(cand_scores, 4) || !aligned(cand_idx, 4))
        return DSA_ERR_INVALID_ARG;
    return from_cuda(launch_select_candidates(scores, idx, rows, L, k, key_pos0, cand_scores, cand_idx,
                                              static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_cp_merge(const float *cand_scores, const int32_t *cand_idx, int P, int rows, int kc, int k,
                        int32_t *idx, dsa_stream_t stream) {
    if (!cand_scores || !cand_idx || !idx) return DSA_ERR_INVALID_ARG;
    if (P < 1 || rows < 1 || kc < 1 || k < 1) return DSA_ERR_INVALID_ARG;
    if ((long long)P * kc > 16384) return DSA_ERR_UNSUPPORTED;
    if (!aligned(cand_scores, 4) || !aligned(cand_idx, 4) || !aligned(idx, 4)) return DSA_ERR_INVALID_ARG;
    return from_cuda(launch_topk_merge(cand_scores, cand_idx, P, rows, kc, k, idx, static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_cp_localize(const int32_t *idx, int rows, int k, int key_pos0, int L_local, int32_t *idx_local,
                           dsa_stream_t stream) {
    if (!idx || !idx_local || rows < 1 || k < 1 || key_pos0 < 0 || L_local < 1) return DSA_ERR_INVALID_ARG;
    if (!aligned(idx, 4) || !aligned(idx_local, 4)) return DSA_ERR_INVALID_ARG;
    return from_cuda(launch_localize(idx, (long long)rows * k, key_pos0, L_local, idx_local,
                                     static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_cp_combine(const void *parts, const float *parts_lse, int P, int rows, int Hq, int Dv, dsa_dtype dt,
                          void *out, float *lse, dsa_stream_t stream) {
    if (!parts || !parts_lse || !out) return DSA_ERR_INVALID_ARG;
    if (P < 1 || rows < 1 || Hq < 1 || Dv < 1) return DSA_ERR_INVALID_ARG;
    if (!valid_dtype(dt)) return DSA_ERR_UNSUPPORTED;
    const size_t eb = dtype_bytes(dt);
    if (!aligned(parts, eb) || !aligned(out, eb) || !aligned(parts_lse, 4) || (lse && !aligned(lse, 4)))
        return DSA_ERR_INVALID_ARG;
    return from_cuda(launch_combine_parts(parts, parts_lse, P, (long long)rows * Hq, Dv, dt, out, lse,
                                          static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
