// Host-side launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// Cached per-device attributes.
struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int max_smem_optin = 0;
    int cc_major = 0, cc_minor = 0;
};
cudaError_t device_info(DeviceInfo *out);

// Process-wide count of kernels this library has enqueued (diagnostics).
void count_launch(int n = 1);

// TMA tensor map over a row-major bf16 matrix [rows, cols] whose rows are
// pitch_bytes apart (a multiple of 16), read as boxes of box_rows x 64
// columns (128 bytes) with the 128-byte swizzle. False if the driver rejects it.
bool make_map_bf16_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                         uint32_t box_rows);
// The same over 8-bit elements (e4m3 codes): boxes of box_rows x 128 columns.
bool make_map_u8_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                       uint32_t box_rows);

// The same over fp32 elements without swizzle: boxes of box_rows x box_cols
// (box_cols * 4 a multiple of 16), rows of the box consecutive in shared memory.
bool make_map_f32(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                  uint32_t box_rows, uint32_t box_cols);

// ----------------------------------------------------------------- indexer
struct IndexerProblem {
    const void *q_idx;   // [B, Tq, H, d]
    const void *k_idx;   // [B, L, d]
    const float *w;      // [B, Tq, H]
    int B, Tq, L, q_pos0, H, d;
    dsa_dtype dt;
    float *scores;       // [B, Tq, L]
    bool fill_masked;    // write -inf at s > t (else those entries are untouched)
};
cudaError_t launch_indexer(const IndexerProblem &p, cudaStream_t stream);

// ----------------------------------------------------------------- top-k
struct TopkProblem {
    const float *scores;  // [B, Tq, L]
    int B, Tq, L, q_pos0, k;
    int32_t *idx;         // [B, Tq, k]
    void *ws;
    size_t ws_bytes;
    bool include_self = false;  // S_t = {t} and the k-1 best of 0..t-1
};
size_t topk_workspace_bytes(int B, int Tq, int L, int q_pos0, int k);
cudaError_t launch_topk(const TopkProblem &p, cudaStream_t stream);
// The selection when every row keeps all of its candidates (q_pos0 + Tq <= k):
// idx[b, i, :] = 0 .. t, then -1. Reads no scores.
cudaError_t launch_dense_selection(const TopkProblem &p, cudaStream_t stream);

// ----------------------------------------------------------------- attention
struct AttnProblem {
    const void *q;        // [B, Tq, Hq, Dqk]
    const void *k_cache;
    const void *v_cache;
    const int32_t *idx;   // [B, Tq, k]
    int B, Tq, L, k, Hq, Hkv, Dqk, Dv;
    float scale;
    int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
    dsa_dtype dt;
    void *out;            // [B, Tq, Hq, Dv]
    float *lse;           // [B, Tq, Hq] or null
    void *ws;
    size_t ws_bytes;
};
size_t attn_workspace_bytes(const AttnProblem &p);
// Query rows of one batch entry whose attention shares the gathers of their
// selections (1: every row gathers its own).
int attn_row_group(const AttnProblem &p);
cudaError_t launch_attn(const AttnProblem &p, cudaStream_t stream);

// The argument checks of dsa_sparse_attn (everything but the workspace).
dsa_status validate_attn_call(const void *q, const void *k_cache, const void *v_cache, const int32_t *idx,
                              const dsa_attn_shape *sh, dsa_dtype dt, const void *out, const float *lse);

// ----------------------------------------------------------------- indexer loss
struct KlProblem {
    const float *scores;    // [B, Tq, L]
    const float *target;    // dense: [B, Tq, L]; restricted: [B, Tq, k]
    const int32_t *idx;     // null (dense loss) or [B, Tq, k]
    int B, Tq, L, q_pos0, k;
    float *loss_rows;       // [B * Tq]
    float *loss_sum;        // [1] or null
    float *grad;            // [B, Tq, L] or null
};
cudaError_t launch_indexer_kl(const KlProblem &p, cudaStream_t stream);

// ----------------------------------------------------------------- indexer backward
struct IndexerBwdProblem {
    const void *q_idx;      // [B, Tq, H, d]
    const void *k_idx;      // [B, L, d]
    const float *w;         // [B, Tq, H]
    const float *grad;      // [B, Tq, L]: d loss / d I
    int B, Tq, L, q_pos0, H, d;
    dsa_dtype dt;
    float *dq;              // [B, Tq, H, d] or null
    float *dk;              // [B, L, d] or null
    float *dw;              // [B, Tq, H] or null
    void *ws;               // tensor-core path: partial dk sums
    size_t ws_bytes;
};
cudaError_t launch_indexer_bwd(const IndexerBwdProblem &p, cudaStream_t stream);
size_t indexer_bwd_cuda_core_smem_bytes(int H, int d);
// Workspace the tensor-core path needs for this problem (0: it does not take it).
size_t indexer_bwd_tc_workspace_bytes(const IndexerBwdProblem &p);

// ----------------------------------------------------------------- context parallelism
cudaError_t launch_select_candidates(const float *scores, const int32_t *idx, long long rows, int L, int k,
                                     int key_pos0, float *cand_score, int32_t *cand_idx, cudaStream_t stream);
cudaError_t launch_topk_merge(const float *cand_score, const int32_t *cand_idx, int P, int rows, int kc, int k,
                              int32_t *idx, cudaStream_t stream);
cudaError_t launch_localize(const int32_t *idx, long long n, int key_pos0, int L_local, int32_t *out,
                            cudaStream_t stream);
cudaError_t launch_combine_parts(const void *parts, const float *parts_lse, int P, long long pairs, int Dv,
                                 dsa_dtype dt, void *out, float *lse, cudaStream_t stream);

// Measurement aid: gather rows idx[0..n) of src (pitch bytes apart, row_bytes
// each) into shared memory with 16-byte cp.async and discard them.
cudaError_t launch_diag_gather(const void *src, int64_t pitch, int row_bytes, int n_src, const int32_t *idx, int64_t n,
                               int tile_rows, unsigned int *sink, cudaStream_t stream);

// Read and clear the error word of a kernel family (kErrTimeout: some launch
// gave up on a bounded wait; kErrBadIndex: an attention launch skipped a
// selected position outside [0, L) other than -1).
unsigned int indexer_take_device_error();
unsigned int attn_mla_tc_take_device_error();
unsigned int indexer_bwd_take_device_error();
unsigned int attn_tc_take_device_error();
unsigned int attn_mla_take_device_error();
unsigned int attn_perhead_take_device_error();
unsigned int attn_cc_take_device_error();
unsigned int attn_mqa_tc_take_device_error();
// Limit of the bounded waits of the kernel families that have them (0: every
// bounded wait gives up before its role issues anything).
cudaError_t indexer_set_wait_limit(unsigned long long ns);
cudaError_t indexer_bwd_set_wait_limit(unsigned long long ns);
cudaError_t attn_mla_tc_set_wait_limit(unsigned long long ns);
cudaError_t attn_mqa_tc_set_wait_limit(unsigned long long ns);

}  // namespace dsa
