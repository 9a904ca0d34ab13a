/*
 * onetrans.h - C ABI of the B200 (sm_100a) OneTrans block-stack forward.
 *
 * The method: OneTrans ("OneTrans: Unified Feature Interaction and Sequence
 * Modeling with One Transformer in Industrial Recommender", WWW 2026).  The
 * summary page's tokenizer, block, pyramid and KV-cache paragraphs define what
 * is computed; the blog page's "Mixed Parameterization" and "Cross-Request KV
 * Caching" designs restate the private-NS-weights and encode-once rules.
 *
 *   - S-tokens (behaviour rows) come first, N NS-tokens per candidate follow.
 *   - Each block: pre-norm RMSNorm, attention, residual, RMSNorm, GELU FFN,
 *     residual.  All S-tokens share one QKV / O / FFN set; NS position n has
 *     its own private set.
 *   - Mask: S-token t sees S-tokens 0..t; NS-token n sees every S-token of the
 *     layer and NS-tokens 0..n of its own candidate.
 *   - Pyramid: layer l reads L_l S rows (L_0 = L0), computes K/V for all of
 *     them, queries for the last q_l only; its S output is those q_l rows,
 *     so L_{l+1} = q_l.
 *   - Cross-request KV cache: the S-side runs once per user (encode) and
 *     stores every layer's S K/V; each candidate's NS-side runs against it.
 *
 * Conventions for every call below:
 *   - Pointers marked "device" are CUDA device pointers owned by the caller,
 *     contiguous, row-major, 16-byte aligned.  "host" pointers are read only
 *     during the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on it; nothing synchronises except
 *     ot_model_create, ot_model_destroy, ot_set_act_scales and
 *     ot_poll_device_error.
 *   - Arguments are checked on the host before anything is launched; a
 *     failed check returns its status and launches nothing.
 *   - Device-side failures (a bounded wait that expired, a failed index
 *     check) set the model's device error word instead of trapping; read it
 *     with ot_poll_device_error.
 *   - No C++ exception crosses this ABI.  The only allocations are made by
 *     ot_model_create (weights and the error word) and the first
 *     ot_set_act_scales (the scale array); hot calls never allocate.
 *   - A model may be used from several streams at once if every concurrent
 *     call has its own workspace and output buffers.
 *
 * Storage dtypes: OT_DTYPE_F32 = float32 everywhere (SIMT fp32 arithmetic,
 * no TF32); OT_DTYPE_BF16 = bfloat16 activations, weights, cache (fp32
 * accumulation on tcgen05 tensor cores); OT_DTYPE_FP8 = bfloat16 storage with
 * every QKV / O / FFN projection run on e4m3 operands, attention and cache in
 * bf16.  FP8 rule (the V2 podcast page credits kernel fusion and FP8 with
 * its speed but gives no recipe; e4m3 with per-tensor fp32 scales is the
 * library's reading): every
 * projection input tensor -- the input of one layer's QKV, O, W1 or W2
 * projection for one parameter set (S, or NS position n), after its RMSNorm
 * and gain where the block has one -- has one fixed fp32 scale s, set with
 * ot_set_act_scales from a calibration (ot_fp8_calibrate); each value is
 * quantised to e4m3(x / s), round to nearest even, saturating at +-448.
 * Each weight matrix (one layer's Wqkv, Wo, W1 or W2, per NS position for
 * the private sets) has one scale amax(W) / 448; the fp32 product is
 * multiplied by both scales.  Until scales are set, and during calibration,
 * each input row is quantised with its own scale amax(row) / 448 (s = 1 for
 * an all-zero row).  Fixed scales do not depend on the batch, so a
 * candidate's result never depends on the other candidates.  Auto-Split
 * stays bf16.
 */
#ifndef ONETRANS_H
#define ONETRANS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OT_MAX_LAYERS 32
/* Rows of K (and of V) in one page of a paged KV cache. */
#define OT_PAGE_ROWS 128

typedef enum {
    OT_OK = 0,
    OT_ERR_ARG = 1,              /* null pointer, negative or zero count */
    OT_ERR_SHAPE = 2,            /* config or call shape outside what the kernels support */
    OT_ERR_DTYPE = 3,            /* dtype not supported by this call */
    OT_ERR_ALIGN = 4,            /* a pointer is not 16-byte aligned */
    OT_ERR_CACHE_TOO_SMALL = 5,  /* reserved: cache sizing is by ot_kv_cache_bytes */
    OT_ERR_WORKSPACE_TOO_SMALL = 6,
    OT_ERR_CUDA = 7,             /* a CUDA runtime / driver call failed */
    OT_ERR_DEVICE_TIMEOUT = 8,   /* a device wait hit its iteration bound */
    OT_ERR_DEVICE_BOUNDS = 9,    /* a device index check failed (e.g. embedding id) */
    OT_ERR_UNSUPPORTED = 10      /* no kernel for this combination */
} ot_status;

typedef enum { OT_DTYPE_F32 = 0, OT_DTYPE_BF16 = 1, OT_DTYPE_FP8 = 2 } ot_dtype;

/* Model shape.  q[l] is the S query tail of layer l (1 <= q[l] <= L_l,
 * L_0 = L0, L_{l+1} = q[l]).  F is the Auto-Split input width (0: no
 * Auto-Split weights).  heads must divide d; d / heads must be 64 for the
 * bf16 / fp8 kernels (16, 32 or 64 for fp32); bf16 / fp8: d and ffn
 * multiples of 128 and F a multiple of 64; fp8: d, ffn <= 1536.
 * full_attn = 1 selects full (non-causal) attention (summary page,
 * limitations paragraph: full attention matches causal attention offline;
 * causal wins only through the KV cache): every token sees every token of
 * its own candidate's sequence, S and NS alike.  S rows then depend on the
 * candidate, so such a model runs only ot_full_forward with one candidate
 * per user (C = 1; give a user with several candidates one row of the batch
 * per candidate); the cached calls return OT_ERR_UNSUPPORTED.
 * moe_experts = E > 0 makes the shared S-side FFN of every block a sparse
 * mixture of E experts (the OneTrans-V2 summary page names a sparse MoE for
 * capacity without a recipe; this is the library's reading): with z the
 * FFN's normalised input n(h; g2), a linear router gives E logits
 * W_router z; the moe_topk (1 or 2) largest, ties to the lower expert index,
 * are softmax-ed into gates g_j, and y = h + sum_j g_j W2_e GELU(W1_e z),
 * each expert of the dense FFN's shape.  NS tokens keep their private dense
 * FFNs.  E <= 64, d of 64, 128 or 256; bf16 or fp32 (not fp8). */
typedef struct {
    int layers, d, heads, ffn, n_ns, L0;
    int q[OT_MAX_LAYERS];
    int F;
    float eps;
    int dtype; /* ot_dtype */
    int full_attn; /* 0 = the OneTrans causal mask, 1 = full attention */
    int moe_experts, moe_topk; /* 0 = dense S-side FFN */
} ot_config;

/* Weights, device pointers in the storage dtype (float32 for OT_DTYPE_F32,
 * bfloat16 otherwise), "out x in" row-major like a linear layer's weight:
 *   Wqkv_s [layers][3d][d] (rows: Q | K | V), Wo_s [layers][d][d],
 *   W1_s [layers][ffn][d], W2_s [layers][d][ffn], g1_s, g2_s [layers][d];
 *   Wqkv_ns [layers][N][3d][d], Wo_ns [layers][N][d][d],
 *   W1_ns [layers][N][ffn][d], W2_ns [layers][N][d][ffn],
 *   g1_ns, g2_ns [layers][N][d];  W_split [N*d][F] (may be NULL if F == 0).
 * g1 / g2 are the RMSNorm gains before attention and before the FFN.
 * Mixture of experts (moe_experts = E > 0; W1_s / W2_s are then unused and
 * may be NULL): W_router [layers][E][d], W1_moe [layers][E][ffn][d],
 * W2_moe [layers][E][d][ffn]; NULL for a dense model. */
typedef struct {
    const void *Wqkv_s, *Wo_s, *W1_s, *W2_s, *g1_s, *g2_s;
    const void *Wqkv_ns, *Wo_ns, *W1_ns, *W2_ns, *g1_ns, *g2_ns;
    const void *W_split;
    const void *W_router, *W1_moe, *W2_moe;
} ot_weights;

typedef struct ot_model ot_model;

/* Validate the config, copy the weights into library-owned device memory in
 * the layout the kernels read (gains folded into the following projection;
 * e4m3 copies with per-matrix scales for OT_DTYPE_FP8), and allocate the
 * device error word.  Runs on the current device; synchronous.
 * Errors: OT_ERR_ARG / OT_ERR_SHAPE / OT_ERR_DTYPE on a bad config,
 * OT_ERR_CUDA if an allocation or copy fails (nothing is leaked). */
ot_status ot_model_create(const ot_config *cfg, const ot_weights *w, ot_model **out);
void ot_model_destroy(ot_model *m);

/* Bytes of the KV cache for `users` users:
 * users * sum_l 2 * L_l * d * sizeof(storage).  Layout per user: layers in
 * order; layer l = K [L_l][d] then V [L_l][d] (heads side by side along d). */
size_t ot_kv_cache_bytes(const ot_model *m, int users);

/* Workspace bytes a call with `users` users and `cands` candidates per user
 * needs (encode: cands = 0; score / full forward: cands >= 1).  Includes
 * room for the KV cache when ot_full_forward is given kv_cache = NULL. */
size_t ot_workspace_bytes(const ot_model *m, int users, int cands);

/* Auto-Split (summary page, tokenizer paragraph: one projection of the
 * concatenated static features, then sliced): ns[r][n][:] =
 * (x[r][:] . W_split^T)[n*d .. n*d+d-1].  x: device [M][F], ns: device
 * [M][N][d], storage dtype.  Errors: OT_ERR_ARG, OT_ERR_SHAPE (F == 0). */
ot_status ot_auto_split(ot_model *m, const void *x, long M, void *ns, void *stream);

/* Embedding gather for S-token assembly: out[i][:] = table[ids[i]][:].
 * table: device bf16 [rows][d]; ids: device int64 [n]; out: device bf16
 * [n][d].  d must be a multiple of 8.  An id outside [0, rows) writes a zero
 * row and sets OT_ERR_DEVICE_BOUNDS in `err_word` if err_word != NULL
 * (device int32, caller-owned). */
ot_status ot_embed_gather(const void *table, long rows, int d, const int64_t *ids, long n,
                          void *out, int32_t *err_word, void *stream);

/* Encode U users (S-side, once per user; summary page, pyramid / KV-cache
 * paragraph: candidates of one request share the user sequence, so the
 * S-side runs once; blog page, "Cross-Request KV Caching").  Every layer l:
 * RMSNorm + shared QKV over its L_l S rows, K / V stored in the cache, causal
 * attention of the q_l tail rows, O, FFN (summary page, block paragraph).
 * S device [U][L0][d] ->
 * kv_cache device (ot_kv_cache_bytes(m, U) bytes) and, if out_s_tail is not
 * NULL, the last layer's S rows device [U][q_last][d].
 * ws: device workspace of ws_bytes >= ot_workspace_bytes(m, U, 0). */
ot_status ot_encode_user(ot_model *m, const void *S, int U, void *kv_cache, void *out_s_tail,
                         void *ws, size_t ws_bytes, void *stream);

/* Append `delta` new S tokens to each of U encoded users without encoding
 * the old ones again (sequence KV caching across requests; summary page,
 * KV-cache paragraph, which gives no schedule for it).  Reading: the pyramid
 * windows stay anchored at their first row, so appending grows L0 and every
 * query tail q[l] by delta; each old row then keeps exactly the keys it had at
 * every layer (the mask is causal), so its K/V and outputs do not change and
 * only the new rows are computed, against the cached K/V.
 *   m        the model of the GROWN sequences: its L0 and q[l] include the
 *            delta new rows (the old cache was written by a model with
 *            L0 - delta and q[l] - delta and the same weights).
 *   kv_old   device, the old cache (layout of that shorter configuration).
 *   S_new    device [U][delta][d], the new rows in sequence order.
 *   kv_new   device, ot_kv_cache_bytes(m, U) bytes: the grown cache, the old
 *            rows' K/V copied into the grown layout and the new rows' K/V
 *            after them in every layer; what ot_encode_user(m, old ++ new)
 *            writes, up to rounding.
 *   out_new  device [U][delta][d]: the new rows' outputs of the last layer,
 *            i.e. the last delta rows of the grown S output (the rows before
 *            them are the old call's output, unchanged).
 * ws >= ot_append_workspace_bytes(m, U, delta).  kv_old and kv_new must not
 * overlap.  Errors: OT_ERR_ARG (null pointer, delta < 1, overlapping
 * caches), OT_ERR_SHAPE (q[last] <= delta, so the old schedule would be
 * empty; d * sizeof(storage) not a multiple of 16; U > 65535),
 * OT_ERR_ALIGN, OT_ERR_WORKSPACE_TOO_SMALL. */
ot_status ot_encode_append(ot_model *m, const void *kv_old, int U, const void *S_new, int delta,
                           void *kv_new, void *out_new, void *ws, size_t ws_bytes, void *stream);
/* Workspace bytes of ot_encode_append for `users` users and `delta` new rows
 * each: the encode buffers for users * delta rows. */
size_t ot_append_workspace_bytes(const ot_model *m, int users, int delta);

/* Score C candidates per user against the users' cached S K/V (NS-side;
 * summary page, pyramid / KV-cache paragraph: the NS-side runs per
 * candidate; block paragraph: NS token n has private weights and sees every
 * S token of the layer and NS tokens 0..n of its own candidate):
 * ns device [U][C][N][d] -> out_ns device [U][C][N][d].  kv_cache as written
 * by ot_encode_user for the same U users.  ws >= ot_workspace_bytes(m, U, C).
 * A candidate's result does not depend on the other candidates in the call. */
ot_status ot_score_candidates(ot_model *m, const void *kv_cache, int U, const void *ns, int C,
                              void *out_ns, void *ws, size_t ws_bytes, void *stream);

/* Paged KV cache (the blog page's engineering reading list points at
 * PagedAttention and prefix caching for the cross-request KV cache; the
 * layout here is the library's).  Instead of one dense block per user the
 * cache is a caller-owned pool of pages, each OT_PAGE_ROWS rows of K [128][d]
 * followed by the same rows of V, and a page table, device int32
 * [U][ot_kv_pages_per_user(m)]: entry off(l) + b of user u names the page
 * holding rows 128 b .. 128 b + 127 of layer l (off(l) = sum over j < l of
 * ceil(L_j / 128); the last page of a layer may be partly used).  Pages may
 * be listed by several users when their K/V rows are identical: users with
 * the same schedule and the same S rows up to the page's last row (a shared
 * prefix) -- every user's encode writes the page, with identical values.
 * A page id outside [0, n_pages) is never dereferenced: the store is
 * skipped, reads use page 0, and OT_ERR_DEVICE_BOUNDS is raised. */
int ot_kv_pages_per_user(const ot_model *m);
/* Bytes of one page: 2 * OT_PAGE_ROWS * d * sizeof(storage). */
size_t ot_kv_page_bytes(const ot_model *m);
/* ot_encode_user into a paged cache: pool device (n_pages pages), pages
 * device int32 [U][ot_kv_pages_per_user(m)]; otherwise as ot_encode_user
 * (same workspace).  Errors as ot_encode_user, plus OT_ERR_ARG for a null
 * pool or table or n_pages < 1. */
ot_status ot_encode_user_paged(ot_model *m, const void *S, int U, void *pool, long long n_pages,
                               const int32_t *pages, void *out_s_tail, void *ws, size_t ws_bytes,
                               void *stream);
/* ot_score_candidates against a paged cache written by ot_encode_user_paged. */
ot_status ot_score_candidates_paged(ot_model *m, const void *pool, long long n_pages,
                                    const int32_t *pages, int U, const void *ns, int C,
                                    void *out_ns, void *ws, size_t ws_bytes, void *stream);

/* Capacity of the scratch array used by ot_score_candidates_noalloc (bytes). */
#define OT_NOALLOC_SCRATCH_BYTES (16u << 20)

/* ot_score_candidates for callers that cannot allocate device memory (a
 * serving runtime that forbids allocation on its request path, or a host
 * that owns all GPU memory through its own pool and lends none to
 * libraries).  The pages have no counterpart: this is a deployment variant
 * of the NS-side call, computing exactly what ot_score_candidates computes.
 * Same arguments minus the workspace: the scratch is a fixed device array of
 * OT_NOALLOC_SCRATCH_BYTES inside the library's device image, present on
 * every GPU that loads the library until the process exits.  The call makes
 * no cudaMalloc / cudaFree or other allocating call.
 *   - The model's device must be current.  The first call on a device looks
 *     up the array's address there (cudaGetSymbolAddress) and keeps it for
 *     that device's current context; a call in a new context (after a
 *     cudaDeviceReset, say) looks it up again.  Make the first call on a
 *     device before any stream capture.
 *   - All calls on a device share the array; concurrent calls (other
 *     streams or threads) race on it and must be serialised by the caller.
 *     Contents persist between calls; the path never reads scratch it has
 *     not written in the same call.
 * Errors, in this order: OT_ERR_ARG (null pointer, U or C < 1),
 * OT_ERR_ALIGN, OT_ERR_SHAPE (U * C * N >= 2^31 or C * N > 2^30),
 * OT_ERR_UNSUPPORTED while per-launch profiling is enabled,
 * OT_ERR_WORKSPACE_TOO_SMALL when the rows need more scratch than
 * OT_NOALLOC_SCRATCH_BYTES (the bytes ot_score_candidates would need: 7 *
 * rows * d + rows * ffn storage elements, fp8 adds rows * max(d, ffn) + 4 *
 * rows, rows = U * C * N), OT_ERR_ARG if another device is current; then as
 * ot_score_candidates. */
ot_status ot_score_candidates_noalloc(ot_model *m, const void *kv_cache, int U, const void *ns,
                                      int C, void *out_ns, void *stream);

/* Training-style batch (summary page, block and pyramid paragraphs: the
 * whole token sequence of a candidate through the stack): B users with C
 * candidates each, S and NS in one call.  Because S tokens never see NS
 * tokens, this computes what ot_encode_user followed by ot_score_candidates
 * computes.  S device [B][L0][d], ns device [B][C][N][d] -> out_s_tail device
 * [B][q_last][d], out_ns device [B][C][N][d]; the S K/V go to kv_cache if
 * not NULL (ot_kv_cache_bytes(m, B) bytes), else to the workspace.
 * ws >= ot_workspace_bytes(m, B, C). */
ot_status ot_full_forward(ot_model *m, const void *S, const void *ns, int B, int C,
                          void *out_s_tail, void *out_ns, void *kv_cache, void *ws,
                          size_t ws_bytes, void *stream);

/* The same batch from pinned host memory: S_host [B][L0][d], x_host [B][C][F]
 * (the Auto-Split input, F = cfg.F > 0) -> out_s_tail_host [B][q_last][d],
 * out_ns_host [B][C][N][d], all in the storage dtype.  The inputs are copied
 * on the model's own copy stream into one of two staging slots of the
 * workspace (alternating per call; a slot is rewritten only after the
 * forward that read it has run), then Auto-Split, the forward and the output
 * copies run on `stream`.  Calls issued back to back on one stream with the
 * same workspace therefore overlap the next call's input copy with this
 * call's work.  ws >= ot_host_workspace_bytes(m, B, C) bytes, device; the
 * host buffers must stay valid until the call's work on `stream` completes.
 * Returns as ot_full_forward; OT_ERR_SHAPE if the model has no Auto-Split. */
size_t ot_host_workspace_bytes(const ot_model *m, int users, int cands);
ot_status ot_full_forward_host(ot_model *m, const void *S_host, const void *x_host, int B, int C,
                               void *out_s_tail_host, void *out_ns_host, void *kv_cache,
                               void *ws, size_t ws_bytes, void *stream);

/* Per-tensor FP8 activation scales (OT_DTYPE_FP8 models only; see the FP8
 * rule above).  scales: host float [layers][1 + n_ns][4] -- parameter set 0
 * is the S side, set 1 + n NS position n; the four inputs of a set in the
 * order QKV, O (attention output), W1, W2 -- each finite and > 0; copied
 * into library-owned device memory (allocated on the first call; the call
 * synchronises the device first, so calls enqueued earlier finish with the
 * scales they were enqueued with).  scales = NULL returns the model to
 * per-row scales.  Errors: OT_ERR_ARG (null model, a scale <= 0 or not
 * finite), OT_ERR_DTYPE (not an FP8 model), OT_ERR_CUDA. */
ot_status ot_set_act_scales(ot_model *m, const float *scales);

/* Calibration for the per-tensor FP8 scales: encode U users S device
 * [U][L0][d] and score their C candidates ns device [U][C][N][d] through
 * every layer with per-row scales (whatever ot_set_act_scales set), and
 * max-accumulate into amax (device float [layers][1 + n_ns][4], the layout
 * of ot_set_act_scales; zero it before the first batch) the largest |x| of
 * every projection input tensor.  Scales amax / 448 then quantise that
 * sample's largest inputs to +-448 exactly.  The outputs are discarded.
 * ws >= ot_workspace_bytes(m, U, C).  Errors: OT_ERR_ARG, OT_ERR_DTYPE (not
 * an FP8 model), OT_ERR_ALIGN, OT_ERR_SHAPE, OT_ERR_WORKSPACE_TOO_SMALL. */
ot_status ot_fp8_calibrate(ot_model *m, const void *S, const void *ns, int U, int C, float *amax,
                           void *ws, size_t ws_bytes, void *stream);

/* Synchronise `stream`, then read and clear the model's device error word.
 * Returns OT_OK, OT_ERR_DEVICE_TIMEOUT, OT_ERR_DEVICE_BOUNDS or OT_ERR_CUDA. */
ot_status ot_poll_device_error(ot_model *m, void *stream);

/* Iteration bound of every device-side wait (mbarrier / flag spin), default
 * 1 << 26 polls.  A wait that reaches it sets OT_ERR_DEVICE_TIMEOUT and the
 * kernel returns early.  Test hook: values < 1 are rejected. */
ot_status ot_set_wait_limit(ot_model *m, long long polls);

/* Kernel family for the bf16 projections and attention: 0 = tcgen05
 * tensor-core kernels (default; the feed-forward runs as one fused kernel
 * where the width allows), 1 = the CUDA-core kernels the fp32 path uses
 * (slow; a second GPU implementation for cross-checks), 2 = tensor-core
 * kernels with the feed-forward as two separate GEMMs (cross-check of the
 * fused kernel).  fp32 models always use the CUDA-core kernels.  Errors:
 * OT_ERR_ARG; OT_ERR_UNSUPPORTED for path 1 on an fp8 model (the CUDA-core
 * kernels read no e4m3). */
ot_status ot_set_kernel_path(ot_model *m, int path);

/* Per-launch timing for roofline reports.  While enabled, every kernel the
 * model launches is bracketed by two CUDA events on its stream and logged
 * with its kind and its algorithmic work (FLOPs of the computed outputs only;
 * bytes = each operand read once plus each output written once).
 * ot_profile_read synchronises the device, copies up to `max` records
 * (oldest first) into `out`, clears the log and returns the number copied
 * (negative on error).  Records beyond an internal 1 << 16 are dropped. */
typedef enum {
    OT_KIND_GEMM_TC = 0, OT_KIND_GEMM_SIMT = 1, OT_KIND_ATTN_TC = 2, OT_KIND_ATTN_SIMT = 3,
    OT_KIND_GATHER = 4, OT_KIND_QUANT = 5, OT_KIND_FFN_TC = 6 /* fused FFN1 + GELU + FFN2 */,
    OT_KIND_ATTN_NS = 7 /* NS attention, <= 64 query rows per (user, head) */,
    OT_KIND_KV_GROW = 8 /* old K/V rows into a grown cache (ot_encode_append) */,
    OT_KIND_MOE = 9 /* mixture of experts: routing or combining the rows */
} ot_kernel_kind;

typedef struct {
    int kind;      /* ot_kernel_kind */
    int role;      /* 0 S-QKV, 1 S-attn, 2 S-O, 3 S-FFN1, 4 S-FFN2, 5..9 the NS ones, 10 Auto-Split,
                      11 other, 12 S-FFN (fused), 13 NS-FFN (fused); 14 O, 15 FFN, 16 QKV:
                      one launch for both sides of a layer in ot_full_forward.
                      Where the FFN kernel runs (bf16, d of 128 or 256) it also
                      does the output projection, so the S-O / NS-O / O roles
                      appear only on the other paths (FP8, d = 384, kernel
                      path 2, mixture of experts); 17 S-MoE: the experts'
                      routing and combining */
    float ms;      /* device time between the two events */
    double flops;  /* algorithmic floating-point operations */
    double bytes;  /* algorithmic HBM bytes */
} ot_launch_record;

ot_status ot_profile_enable(ot_model *m, int enable);
int ot_profile_read(ot_model *m, ot_launch_record *out, int max);

/* ---- Backward pass (training) ----
 * The summary page lists activation checkpointing among the training
 * optimisations on top of the stack (systems paragraph).  ot_full_backward
 * computes, for an fp32 config with the causal mask or full attention
 * (full_attn = 1: one candidate per user, C = 1, as the forward) and a dense
 * or mixture-of-experts S-side FFN (moe_experts = E: gradients of the router
 * and the experts; the selection carries none), the gradients of
 *     loss = sum(s_tail * G_s) + sum(ns_out * G_ns)
 * (s_tail, ns_out: the outputs of ot_full_forward; G_s, G_ns: the upstream
 * gradients) with respect to every weight and gain and to S and ns.
 * Activation checkpointing: a forward pass keeps each layer's input rows
 * and its attention outputs with their softmax statistics (row max and sum);
 * the backward then recomputes the rest of one layer at a time from them,
 * top layer first, and takes its gradients.  CUDA-core fp32 kernels.
 * All pointers are device pointers to fp32, 16-byte aligned:
 *   w      the tensors of ot_weights, fp32, gains NOT folded: Wqkv_s ..
 *          g2_ns, and with E > 0 W_router, W1_moe, W2_moe (then W1_s / W2_s
 *          are not read and may be NULL); W_split is not read;
 *   S [U][L0][d], ns [U][C][N][d], G_s [U][q_last][d], G_ns [U][C][N][d];
 *   out_s_tail [U][q_last][d], out_ns [U][C][N][d]: the forward's outputs
 *          (NULL: not written);
 *   g      gradients in the weights' shapes, overwritten (not
 *          accumulated): the twelve dense ones non-NULL (W1_s / W2_s may be
 *          NULL with E > 0, else they are zeroed), the three MoE ones
 *          non-NULL with E > 0 (not read otherwise);
 *   dS [U][L0][d], dns [U][C][N][d] (NULL: not written).
 * C = 0 runs the S side alone (ns, G_ns, out_ns and dns are not read or
 * written; the NS gradients are set to zero).  No atomics: the same inputs
 * give the same bits.  Nothing is allocated; ws >=
 * ot_backward_workspace_bytes(cfg, U, C).  Errors, in this order:
 * OT_ERR_ARG (null pointer, U < 1, C < 0, a bad config field),
 * OT_ERR_DTYPE (not OT_DTYPE_F32), OT_ERR_SHAPE (the config rules;
 * full_attn with C != 1; rows beyond the kernels' 32-bit row counts),
 * OT_ERR_ALIGN, OT_ERR_WORKSPACE_TOO_SMALL, OT_ERR_CUDA. */
typedef struct {
    float *Wqkv_s, *Wo_s, *W1_s, *W2_s, *g1_s, *g2_s;
    float *Wqkv_ns, *Wo_ns, *W1_ns, *W2_ns, *g1_ns, *g2_ns;
    float *W_router, *W1_moe, *W2_moe; /* mixture of experts only */
} ot_grads;

size_t ot_backward_workspace_bytes(const ot_config *cfg, int U, int C);
/* Kernel launches one ot_full_backward call issues (0 for a rejected shape). */
long long ot_backward_launches(const ot_config *cfg, int U, int C);
ot_status ot_full_backward(const ot_config *cfg, const ot_weights *w, const float *S, const float *ns,
                           int U, int C, const float *G_s, const float *G_ns, float *out_s_tail,
                           float *out_ns, const ot_grads *g, float *dS, float *dns, void *ws,
                           size_t ws_bytes, void *stream);

/* Static string for a status code. */
const char *ot_status_str(ot_status s);

/* Kernel launches issued by this model since creation (host-side count). */
long long ot_launch_count(const ot_model *m);

#ifdef __cplusplus
}
#endif
#endif /* ONETRANS_H */
