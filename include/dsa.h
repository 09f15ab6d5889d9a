/*
 * dsa.h -- C ABI of the DeepSeek Sparse Attention (DSA) forward path on
 * NVIDIA B200 (sm_100a). Library: libdsa.so.
 *
 * The path, as defined on "DeepSeek Sparse Attention: Learned Token Selection
 * from Scratch" (cited below as "Learned Token Selection") and "DeepSeek NSA
 * and DSA" §3.2:
 *
 *   1. lightning-indexer scores   I[t,s] = sum_j w[t,j] * ReLU(q^I[t,j] . k^I[s])
 *      ("Learned Token Selection" §2.1, boxed equation), for candidates s <= t;
 *   2. top-k selection            S_t = positions of the k largest I[t,s]
 *      ("Learned Token Selection" §3.1, boxed equation);
 *   3. attention over S_t         u[t,h] = sum_{s in S_t} softmax_s(q[t,h].k[s]*scale) v[s]
 *      ("Learned Token Selection" §3.3 and §10.1), one S_t shared by every query head
 *      ("Learned Token Selection" §4.1-4.2: the MQA mode of MLA).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Query row i of batch entry b sits at absolute position t = q_pos0 + i.
 *   Prefill: Tq = L, q_pos0 = 0. Decode: Tq = 1, q_pos0 = L - 1 (the cache of
 *   L entries includes the new token).
 * - Candidates of row t are positions 0..t (the page's running example says
 *   "preceding tokens ... (plus itself)").
 * - Equal scores are ordered by position, lower position first. When t+1 <= k,
 *   every candidate is selected ("Learned Token Selection" §7.6 note: DSA collapses to full
 *   attention when the context is shorter than the budget).
 * - Selected positions are written in ascending order, followed by -1 padding
 *   up to k entries.
 * - All pointers are DEVICE pointers owned by the caller. The library never
 *   allocates or frees device memory; scratch space is passed in as a
 *   workspace. Every call is asynchronous on the given stream: it validates its
 *   arguments on the host, enqueues kernels and returns.
 * - Tensors are dense and row-major unless a stride says otherwise. Strides
 *   are in elements. Every base pointer must be 16-byte aligned and every
 *   stride must be a multiple of 16 bytes (the kernels move 16-byte vectors).
 * - Errors: arguments are checked before any launch; a failed check returns a
 *   status other than DSA_OK and enqueues nothing. A failed launch returns
 *   DSA_ERR_CUDA. Kernels never trap or assert. No exception crosses the ABI.
 * - Thread safety: calls on different streams may run concurrently. The only
 *   global state is a per-device cache of device attributes.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* An opaque CUDA stream (cudaStream_t / CUstream). NULL is the legacy default
 * stream. */
typedef void *dsa_stream_t;

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad alignment or stride */
    DSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (dtype, head width) */
    DSA_ERR_WORKSPACE = 3,    /* workspace pointer null or ws_bytes too small */
    DSA_ERR_CUDA = 4,         /* a CUDA runtime call or a kernel launch failed */
    DSA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (dsa_device_error) */
    DSA_ERR_BAD_INDEX = 6     /* an attention call met a selected position that is
                                 neither -1 nor inside [0, L); it was skipped
                                 (dsa_device_error) */
} dsa_status;

typedef enum {
    DSA_F32 = 0,   /* IEEE fp32 */
    DSA_BF16 = 1,  /* bfloat16 */
    DSA_E4M3 = 2   /* 8-bit e4m3 codes (1 sign, 4 exponent bits with bias 7,
                      3 mantissa bits): indexer inputs only (q_idx, k_idx of
                      dsa_indexer_scores and dsa_forward_args.idx_dtype), the
                      FP8 indexer of "Learned Token Selection" §7.4 */
} dsa_dtype;

/* Library version, e.g. 100 for 0.1.0. */
int dsa_version(void);

/* Number of kernels this library has enqueued in this process, over all
 * devices and streams (a diagnostic counter; it never resets). */
uint64_t dsa_kernel_launch_count(void);

/* Static text for a status code (never NULL). */
const char *dsa_status_string(dsa_status status);

/*
 * dsa_device_error -- report and clear the device-side error words of the
 * current device. The library has no counterpart on the pages: its
 * tensor-core kernels bound every wait on an mbarrier (2 s); a wait that
 * gives up makes the kernel set an error word, release its resources and
 * return without finishing its outputs, instead of hanging the GPU.
 *   stream  cudaStream_t (as void*) that ran the calls to check; it is
 *           synchronised first.
 * The attention kernels also record a selected position that is neither -1
 * nor inside the cache [0, L): they skip it like padding (no memory outside
 * the cache is read) and the call's outputs are those of the remaining
 * positions, but the selection it was given was malformed.
 * Returns DSA_OK if no kernel recorded an error since the last call,
 * DSA_ERR_TIMEOUT if a wait gave up (the outputs of that call are invalid;
 * reported first when both happened), DSA_ERR_BAD_INDEX if an attention call
 * skipped a malformed position, and DSA_ERR_CUDA if synchronising or reading
 * the words failed. Blocking; not for use inside stream capture.
 */
dsa_status dsa_device_error(dsa_stream_t stream);

/*
 * dsa_set_wait_limit_ns -- the time limit of every bounded device-side wait
 * of the library's kernels on the current device (default 2,000,000,000 ns).
 * A diagnostic with no counterpart on the pages, for testing the give-up
 * path: with ns = 0 those kernels start every role as having given up (they
 * read the limit once at their start), so no role issues a copy or an MMA;
 * the kernels release their resources, return without their outputs and
 * record DSA_ERR_TIMEOUT (dsa_device_error). Copies and MMAs a CTA did issue
 * are always waited for before it frees tensor memory or exits.
 * Call it while none of the library's kernels runs on the device (it writes
 * device variables like cudaMemcpyToSymbol). Returns DSA_ERR_CUDA if a write
 * failed.
 */
dsa_status dsa_set_wait_limit_ns(uint64_t ns);

/*
 * dsa_indexer_scores -- stage 1, lightning-indexer scores ("Learned Token Selection" §2.1).
 *
 *   scores[b,i,s] = sum_{j<H_I} w[b,i,j] * max(0, sum_{e<d_I} q_idx[b,i,j,e] * k_idx[b,s,e])
 *                   for s <= q_pos0 + i,   and -inf for s > q_pos0 + i.
 *
 * q_idx  [B, Tq, H_I, d_I]  dtype dt (indexer queries)
 * k_idx  [B, L, d_I]        dtype dt (indexer key cache, one key per position,
 *                           shared by all indexer heads)
 * w      [B, Tq, H_I]       fp32 per-head weights
 * scores [B, Tq, L]         fp32 output; every element is written
 *
 * Products are accumulated in fp32 (tensor cores for bf16 with d_I % 64 == 0;
 * CUDA cores otherwise). With integer-valued inputs and power-of-two weights
 * every partial sum is an exact fp32 value, so the result does not depend on
 * the summation order.
 * Requires B, Tq, L, H_I, d_I >= 1, 0 <= q_pos0, q_pos0 + Tq <= L.
 */
dsa_status dsa_indexer_scores(const void *q_idx, const void *k_idx, const float *w,
                              int B, int Tq, int L, int q_pos0, int H_I, int d_I,
                              dsa_dtype dt, float *scores, dsa_stream_t stream);

/* Indexer options (dsa_indexer_scores_ex flags). */
typedef enum {
    /* Write only the causal entries scores[b,i,s], s <= q_pos0 + i; the
     * entries above the diagonal keep whatever the buffer held. What a
     * consumer that reads only the causal part needs (dsa_topk reads
     * scores[b,i,0..t]; the fused dsa_forward writes its scores this way),
     * without the -inf writes of the upper triangle, about half the buffer
     * in prefill. */
    DSA_INDEXER_CAUSAL_ONLY = 1
} dsa_indexer_flags;

/* dsa_indexer_scores with options: flags is 0 or DSA_INDEXER_CAUSAL_ONLY; any
 * other bit gives DSA_ERR_INVALID_ARG. Otherwise as dsa_indexer_scores. */
dsa_status dsa_indexer_scores_ex(const void *q_idx, const void *k_idx, const float *w,
                                 int B, int Tq, int L, int q_pos0, int H_I, int d_I,
                                 dsa_dtype dt, unsigned flags, float *scores, dsa_stream_t stream);

/*
 * dsa_topk -- stage 2, per-row top-k selection ("Learned Token Selection" §3.1).
 *
 * For each row (b, i), t = q_pos0 + i, reads scores[b,i,0..t] and writes the
 * positions of the k largest values to idx[b,i,:] in ascending order, then -1
 * up to k entries. Ties go to the lower position; -0.0 equals +0.0; -inf is
 * an ordinary (lowest) value. NaN scores are not supported.
 * Entries scores[b,i,s] with s > t are never read.
 *
 * scores [B, Tq, L] fp32;  idx [B, Tq, k] int32 output.
 * ws / ws_bytes: workspace of at least dsa_topk_workspace_bytes(...) bytes
 * (may be NULL when that is 0).
 * Requires k >= 1, 0 <= q_pos0, q_pos0 + Tq <= L.
 */
dsa_status dsa_topk(const float *scores, int B, int Tq, int L, int q_pos0, int k,
                    int32_t *idx, void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Selection options (dsa_topk_ex flags, dsa_forward_args.flags). */
typedef enum {
    /* Keep the query's own position: S_t = {t} and the min(t, k-1) best of
     * positions 0..t-1, same order and tie rule ("Learned Token Selection"
     * §3.4: a token that misses its own top k is kept by always including
     * the current token). Without it S_t is the plain top k of 0..t. */
    DSA_FLAG_INCLUDE_SELF = 1
} dsa_flags;

/* dsa_topk with options: flags is 0 or DSA_FLAG_INCLUDE_SELF; any other bit
 * gives DSA_ERR_INVALID_ARG. Otherwise as dsa_topk (same workspace). */
dsa_status dsa_topk_ex(const float *scores, int B, int Tq, int L, int q_pos0, int k, unsigned flags,
                       int32_t *idx, void *ws, size_t ws_bytes, dsa_stream_t stream);

size_t dsa_topk_workspace_bytes(int B, int Tq, int L, int q_pos0, int k);

/* Shape of the attention stage. */
typedef struct dsa_attn_shape {
    int B, Tq, L, k;          /* batch, query rows, cache length, idx entries per row */
    int Hq, Hkv;              /* query heads, KV heads (Hq % Hkv == 0) */
    int Dqk, Dv;              /* query/key width, value width */
    float scale;              /* logit scale, usually 1/sqrt(Dqk) */
    /* element strides of the caches: element (b, s, g, e) of K is at
     * k_cache[b*k_stride_b + s*k_stride_s + g*k_stride_h + e]; same for V.
     * V may alias K (a latent row whose first Dv columns are the value). */
    int64_t k_stride_b, k_stride_s, k_stride_h;
    int64_t v_stride_b, v_stride_s, v_stride_h;
} dsa_attn_shape;

/*
 * dsa_sparse_attn -- stage 3, attention over the selected rows
 * ("Learned Token Selection" §3.3, §10.1; one selection shared by all heads,
 * §4.1-4.2).
 *
 *   out[b,i,h,:] = sum_{s in S} softmax_s(scale * q[b,i,h,:] . K[b,s,g,:]) * V[b,s,g,:]
 *   with g = h / (Hq / Hkv) and S = { idx[b,i,j] : idx[b,i,j] >= 0 }.
 *
 * q   [B, Tq, Hq, Dqk] dtype dt;  out [B, Tq, Hq, Dv] dtype dt
 * idx [B, Tq, k] int32: positions in [0, L) or -1 (skipped); order is free;
 *     a position must not appear twice in one row. Any other value is
 *     skipped as well and reported by dsa_device_error (DSA_ERR_BAD_INDEX).
 * lse [B, Tq, Hq] fp32 or NULL: log sum_{s in S} exp(scale * q.k_s).
 * A row whose idx holds only -1 gets out = 0 and lse = -inf.
 * Logits, softmax and the weighted sum are accumulated in fp32.
 * ws: at least dsa_sparse_attn_workspace_bytes(sh) bytes.
 */
dsa_status dsa_sparse_attn(const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *idx, const dsa_attn_shape *sh, dsa_dtype dt,
                           void *out, float *lse, void *ws, size_t ws_bytes,
                           dsa_stream_t stream);

/* Workspace dsa_sparse_attn needs for this shape; 0 when the shape is
 * invalid or unsupported (the call itself then reports why). */
size_t dsa_sparse_attn_workspace_bytes(const dsa_attn_shape *sh, dsa_dtype dt);

/* Query rows whose attention shares its copies: dsa_sparse_attn (and the
 * fused forward) gather, for each group of this many consecutive query rows
 * of one batch entry, the K and V rows of the union of the rows' selected
 * sets once, and attend every row to its own set only. 1: every row gathers
 * its own selected rows. The gathered bytes of a group are the union size
 * times the row bytes of every KV head. Depends on the shape and the
 * device's shared memory (the current device); 0 for an invalid shape. */
int dsa_sparse_attn_row_group(const dsa_attn_shape *sh, dsa_dtype dt);

/*
 * dsa_sparse_attn_noalloc -- dsa_sparse_attn for callers that cannot pass a
 * workspace. (The pages have no counterpart: this is a library convenience.)
 *
 * Some callers cannot allocate device memory when they call the library: an
 * engine plugin that is handed a stream but no allocator, or a serving loop
 * that must never call cudaMalloc because it can synchronise the device. This
 * entry point takes the same arguments as dsa_sparse_attn minus the
 * workspace, and keeps the split-k partial results in a fixed array inside
 * the library (dsa_sparse_attn_noalloc_max_scratch_bytes() bytes, 4 MiB, held
 * by every GPU that loads libdsa.so until the process exits). It calls no
 * allocator.
 *
 * - Checks its arguments as dsa_sparse_attn does (same statuses), then
 *   returns DSA_ERR_WORKSPACE without launching anything when the problem
 *   needs more scratch than that (dsa_sparse_attn_workspace_bytes(sh, dt) >
 *   the maximum); use dsa_sparse_attn with a workspace then.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, that device current) and caches it: make that first
 *   call before any stream capture.
 * - All calls on a device share the array. Calls whose kernels may overlap on
 *   the GPU (unordered streams) race on it and produce wrong results.
 * - Results are those of dsa_sparse_attn for the same arguments.
 */
dsa_status dsa_sparse_attn_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *idx, const dsa_attn_shape *sh, dsa_dtype dt,
                                   void *out, float *lse, dsa_stream_t stream);

/* Size of the built-in scratch array used by dsa_sparse_attn_noalloc. */
size_t dsa_sparse_attn_noalloc_max_scratch_bytes(void);

/* Arguments of the fused forward pass. */
typedef struct dsa_forward_args {
    int B, Tq, L, q_pos0, k;
    /* indexer (stage 1) */
    const void *q_idx;        /* [B, Tq, H_I, d_I] */
    const void *k_idx;        /* [B, L, d_I] */
    const float *w;           /* [B, Tq, H_I] */
    int H_I, d_I;
    dsa_dtype idx_dtype;
    /* attention (stage 3) */
    const void *q;            /* [B, Tq, Hq, Dqk] */
    const void *k_cache;      /* strided as in dsa_attn_shape */
    const void *v_cache;
    int Hq, Hkv, Dqk, Dv;
    float scale;
    int64_t k_stride_b, k_stride_s, k_stride_h;
    int64_t v_stride_b, v_stride_s, v_stride_h;
    dsa_dtype attn_dtype;
    /* outputs */
    void *out;                /* [B, Tq, Hq, Dv] attn_dtype */
    float *lse;               /* [B, Tq, Hq] or NULL */
    int32_t *idx_out;         /* [B, Tq, k] or NULL: the selected positions */
    float *scores_out;        /* [B, Tq, L] or NULL: the indexer scores (then
                                 filled with -inf above the diagonal) */
    unsigned flags;           /* 0 or DSA_FLAG_INCLUDE_SELF */
} dsa_forward_args;

/*
 * dsa_forward -- stages 1-3 back to back on one stream.
 * Scores and indices go to caller memory when scores_out / idx_out are set,
 * otherwise to the workspace. Results equal those of the three stage calls
 * (dsa_topk_ex with a->flags).
 * Short context: when every query row has t + 1 <= k (q_pos0 + Tq <= k), the
 * selection is all of 0..t by definition, so the top-k is skipped and the
 * dense selections are written directly; the indexer runs only if
 * scores_out asks for its scores. The attention then covers every causal
 * position ("Learned Token Selection" §9.3: short sequences use plain masked
 * attention). The outputs are the same as those of the full path.
 * a->flags: 0 or DSA_FLAG_INCLUDE_SELF (anything else: DSA_ERR_INVALID_ARG).
 * ws: at least dsa_forward_workspace_bytes(a) bytes.
 */
dsa_status dsa_forward(const dsa_forward_args *a, void *ws, size_t ws_bytes,
                       dsa_stream_t stream);

/* Workspace needed by dsa_forward; 0 when the arguments are invalid. */
size_t dsa_forward_workspace_bytes(const dsa_forward_args *a);

/* ------------------------------------------------------------------------
 * The indexer's training loss and its backward pass ("Learned Token
 * Selection" §5 dense warm-up and §6 sparse training; "DeepSeek NSA and DSA"
 * §3.3). The target is supplied by the caller; the main model's attention
 * that would produce it in training lies outside this library.
 * ------------------------------------------------------------------------ */

/*
 * dsa_indexer_kl -- per query row, loss_t = KL(p_t || Softmax(I_t)) over the
 * row's set, and the gradient of sum_t loss_t with respect to I.
 *   scores   [B, Tq, L] fp32: indexer scores I (dsa_indexer_scores). Only
 *            the entries of each row's set are read.
 *   idx      NULL: the dense warm-up loss ("Learned Token Selection" §5.4);
 *            the set of row t is s = 0..t and target is [B, Tq, L] (entries
 *            s > t are not read).
 *            Otherwise [B, Tq, k] int32, e.g. from dsa_topk: the loss of the
 *            sparse stage, restricted to S_t (§6.2). The set is the entries
 *            with 0 <= s <= t (the -1 padding and anything else outside that
 *            range is skipped); entries must be distinct. target is then
 *            [B, Tq, k], aligned with idx.
 *   target   non-negative fp32 weights a of the target distribution, such as
 *            the head sums of the main attention's weights (§5.2, step 1).
 *            Each row is L1-normalised over its set (§5.2, step 2), so an
 *            already normalised p may be passed too. A row whose weights sum
 *            to 0 has loss 0 and a zero gradient; 0 * log 0 counts as 0.
 *   loss_rows [B * Tq] fp32 (required): loss_t of every row.
 *   loss_sum  [1] fp32 or NULL: the sum of loss_rows, accumulated in fp64 in
 *            a fixed order (the same value on every call).
 *   grad     [B, Tq, L] fp32 or NULL: softmax(I_t)_s - p_t[s] on the set, 0
 *            everywhere else (every entry is written). Must not overlap
 *            scores or target.
 * Arithmetic: fp32, exp and log through the hardware base-2 approximations
 * (relative error below 2^-21); the loss is formed from the row sums sum(a),
 * sum(a I), sum(a log a) and the log-sum-exp of I over the set.
 * Errors: DSA_ERR_INVALID_ARG for a null scores, target or loss_rows, bad
 * sizes (as dsa_topk; k >= 1 when idx is given) or pointers not 4-byte
 * aligned.
 */
dsa_status dsa_indexer_kl(const float *scores, const float *target, const int32_t *idx,
                          int B, int Tq, int L, int q_pos0, int k,
                          float *loss_rows, float *loss_sum, float *grad,
                          dsa_stream_t stream);

/*
 * dsa_indexer_backward -- gradients of the indexer's inputs for an incoming
 * gradient g = d loss / d I (e.g. dsa_indexer_kl's grad). Differentiating
 * I[t,s] = sum_j w[t,j] ReLU(x[t,j,s]), x[t,j,s] = q^I[t,j] . k^I[s]
 * ("Learned Token Selection" §2.1; by §6.4 the loss reaches only the
 * indexer), with ReLU'(0) = 0 and G[t,j,s] = g[t,s] w[t,j] [x[t,j,s] > 0]:
 *   dw[t,j] = sum_{s<=t} g[t,s] ReLU(x[t,j,s])
 *   dq[t,j] = sum_{s<=t} G[t,j,s] k^I[s]
 *   dk[s]   = sum over this call's query rows t >= s of sum_j G[t,j,s] q^I[t,j]
 *   q_idx, k_idx, w, B, Tq, L, q_pos0, H_I, d_I, dt: as dsa_indexer_scores;
 *            dt is DSA_BF16 or DSA_F32 (DSA_E4M3: DSA_ERR_UNSUPPORTED).
 *   grad     [B, Tq, L] fp32; entries s > t are not read.
 *   dq       [B, Tq, H_I, d_I] fp32 or NULL (then not computed).
 *   dk       [B, L, d_I] fp32 or NULL; keys that no query row of the call
 *            reaches (s > q_pos0 + Tq - 1) get 0. Every entry is written.
 *   dw       [B, Tq, H_I] fp32 or NULL.
 *   ws       at least dsa_indexer_backward_workspace_bytes(...) bytes when dk
 *            is requested (may be NULL when that is 0).
 * Paths: bf16 inputs with d_I = 128, H_I in {32, 64, 128}, L a multiple of 4,
 * 16-byte aligned pointers, L >= 128 and at least 128 rows of q_idx run on
 * the tensor cores: x is exact there (bf16 products, fp32 sums); the products
 * with k and q take g [x > 0] (times w on the key side) rounded to bf16, so
 * dq and dk carry a relative error of at most 2^-8 of the sums of absolute
 * terms; dw is formed as q . sum_s g [x > 0] k[s] (the same value, since
 * x = q . k[s]) and carries the same bound against sum_s |g| ReLU(x). Every
 * other shape runs on CUDA cores in fp32.
 * Errors: DSA_ERR_INVALID_ARG as dsa_indexer_scores, or a null grad;
 * DSA_ERR_WORKSPACE when dk is requested and ws is missing or too small;
 * DSA_ERR_UNSUPPORTED when the CUDA-core path's staging does not fit.
 */
dsa_status dsa_indexer_backward(const void *q_idx, const void *k_idx, const float *w,
                                const float *grad, int B, int Tq, int L, int q_pos0,
                                int H_I, int d_I, dsa_dtype dt,
                                float *dq, float *dk, float *dw,
                                void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Workspace dsa_indexer_backward needs when dk is requested (16-byte aligned;
 * 0 when the shape takes the CUDA-core path or the arguments are invalid).
 * It holds fp32 partial sums of dk, 64 KB per (128-key tile, chunk of query
 * rows); the chunks of a tile are summed in a fixed order, so dk is the same
 * on every call. */
size_t dsa_indexer_backward_workspace_bytes(int B, int Tq, int L, int q_pos0, int H_I, int d_I,
                                            dsa_dtype dt);

/*
 * dsa_diag_gather -- a measurement aid with no counterpart on the pages: the
 * gather of selected rows alone, without the attention's arithmetic. It
 * moves rows idx[0..n) of src (row r at src + r * pitch_bytes, row_bytes
 * bytes each) into shared memory with the 16-byte cp.async copies the
 * attention kernels use, and discards them. Timed on the rows an attention
 * call selects, it gives the rate at which those rows can be gathered at all,
 * the ceiling of the attention's gather-bound time.
 *   idx      int32; entries outside [0, n_src_rows) are skipped.
 *   tile_rows  8, 16 or 32: rows per shared-memory tile of a CTA (three
 *            tiles in flight); smaller tiles fit more CTAs on an SM.
 *   sink     one uint32 in device memory; written at most rarely (keeps the
 *            copies live).
 * Requires 16 <= row_bytes <= 1024, row_bytes and pitch_bytes multiples of 16,
 * pitch_bytes >= row_bytes, src 16-byte aligned, n >= 1, tile_rows in {8, 16,
 * 32} (else DSA_ERR_INVALID_ARG).
 */
dsa_status dsa_diag_gather(const void *src, int64_t pitch_bytes, int row_bytes, int n_src_rows,
                           const int32_t *idx, int64_t n, int tile_rows, uint32_t *sink, dsa_stream_t stream);

/* ------------------------------------------------------------------------
 * Context parallelism: the indexer keys and the KV cache split by position
 * over P ranks (rank r holds positions [key_pos0_r, key_pos0_r + L_r)), every
 * rank holding all the query rows. Every member of the global selection S_t
 * ("Learned Token Selection" §3.1) is among the k best of its own shard, so
 * the shards' selections merge into S_t exactly; the attention over S_t
 * (§3.3) is a log-sum-exp merge of the shards' partial attentions. A step:
 * dsa_indexer_scores + dsa_topk on the local keys, dsa_cp_select_candidates,
 * an all-gather of the candidates (k scores and k positions per row and
 * rank), dsa_cp_merge, dsa_cp_localize, dsa_sparse_attn with lse on the local
 * cache, an all-gather of (output, lse), dsa_cp_combine. The collectives are
 * the caller's (NCCL through torch.distributed in the Python package).
 * ------------------------------------------------------------------------ */

/*
 * dsa_cp_select_candidates -- a shard's selection as merge candidates.
 *   scores      [rows, L] fp32 local scores; idx [rows, k] int32 local
 *               positions (dsa_topk), -1 padded.
 *   cand_scores [rows, k] fp32: scores[row, idx], -inf for padding.
 *   cand_idx    [rows, k] int32: idx + key_pos0 (global positions), -1 for
 *               padding (and for any entry outside [0, L)).
 */
dsa_status dsa_cp_select_candidates(const float *scores, const int32_t *idx, int rows, int L, int k,
                                    int key_pos0, float *cand_scores, int32_t *cand_idx,
                                    dsa_stream_t stream);

/*
 * dsa_cp_merge -- the global selection from P shards' candidates.
 *   cand_scores, cand_idx  [P, rows, kc] (rank-major, as an all-gather of the
 *               ranks' [rows, kc] arrays leaves them), ranks in ascending
 *               position order, each rank's list ascending (dsa_topk order),
 *               cand_idx -1 for no candidate.
 *   idx         [rows, k] int32: the k best candidates by score, equal scores
 *               to the lower position, as ascending global positions, then
 *               -1 (all valid candidates when there are at most k).
 * Errors: DSA_ERR_UNSUPPORTED when P * kc > 16384 (one CTA holds a row).
 */
dsa_status dsa_cp_merge(const float *cand_scores, const int32_t *cand_idx, int P, int rows, int kc, int k,
                        int32_t *idx, dsa_stream_t stream);

/* dsa_cp_localize -- idx_local = idx - key_pos0 where key_pos0 <= idx <
 * key_pos0 + L_local, else -1 ([rows, k] int32 both). */
dsa_status dsa_cp_localize(const int32_t *idx, int rows, int k, int key_pos0, int L_local,
                           int32_t *idx_local, dsa_stream_t stream);

/*
 * dsa_cp_combine -- merge P partial attentions over disjoint key sets.
 *   parts     [P, rows, Hq, Dv] in dt (DSA_BF16 or DSA_F32); parts_lse
 *             [P, rows, Hq] fp32, -inf where a part selected nothing (its
 *             output is then ignored).
 *   out       [rows, Hq, Dv] in dt: sum_p exp(lse_p - LSE) parts[p], with
 *             LSE = log sum_p exp(lse_p); lse [rows, Hq] fp32 or NULL: LSE.
 *             A pair with no part: out 0, LSE -inf.
 */
dsa_status dsa_cp_combine(const void *parts, const float *parts_lse, int P, int rows, int Hq, int Dv,
                          dsa_dtype dt, void *out, float *lse, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
