// Internal types shared by the host entry points and the kernels.
#pragma once

#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/onetrans.h"

namespace ot {

// Device bounds checks of the checked build (compiled with OT_DEVICE_CHECKS):
// a plain global access of n bytes at byte offset off from a buffer whose
// extent from that base is cap bytes (0: not known, not checked) is made
// only inside the extent; otherwise the model's error word gets
// OT_ERR_DEVICE_BOUNDS and the access is skipped.  The release build
// compiles every check away.
#ifdef OT_DEVICE_CHECKS
constexpr bool kDeviceChecks = true;
#else
constexpr bool kDeviceChecks = false;
#endif

__device__ __forceinline__ bool ot_dev_ok(long long off, long long n, long long cap, int *err)
{
    if (!kDeviceChecks || cap <= 0) return true;
    if (off >= 0 && off + n <= cap) return true;
    if (err) atomicCAS(err, 0, OT_ERR_DEVICE_BOUNDS);
    return false;
}

// Bounded-wait control passed to every kernel that waits on device state.
struct WaitCtl {
    int *err;         // model error word (device)
    long long limit;  // polls before giving up
};

// Row mapping from a GEMM row r (in group g) to a row of some buffer:
//   row = (r / P) * A + (r % P) + B + g * Gs,   skipped when (r % P) < min_t.
// It expresses every layout the block needs: flat rows, per-user tails of a
// pyramid layer, per-user strides of the KV cache, and NS position-major
// groups over candidate-major storage.
struct RowMap {
    long long P, A, B, Gs, min_t;
};

__host__ __device__ inline RowMap rowmap_identity()
{
    return RowMap{1, 1, 0, 0, 0};
}

__host__ __device__ inline long long rowmap_apply(const RowMap &m, long long r, long long g)
{
    long long t = r % m.P;
    return (r / m.P) * m.A + t + m.B + g * m.Gs;
}

__host__ __device__ inline bool rowmap_keep(const RowMap &m, long long r)
{
    return (r % m.P) >= m.min_t;
}

// One output column segment [c_lo, c_hi) of a GEMM: written to
// out + row(r, g) * ld + (c - c_lo).
// Paged KV cache (pages != null): out is the page pool, each page K rows
// [OT_PAGE_ROWS][d] then V rows; the GEMM row r is user u = r / map.P,
// position t = r % map.P + map.B, and goes to row
//   (page * 2 + pg_kv) * OT_PAGE_ROWS + t % OT_PAGE_ROWS,
//   page = pages[u * pg_ustride + pg_off + t / OT_PAGE_ROWS].
struct EpiSeg {
    void *out;
    long long ld;
    int c_lo, c_hi;
    RowMap map;
    const int *pages;
    long long pg_ustride, n_pages;
    int pg_off, pg_kv;
    long long cap; // bytes from out to the end of its buffer (checked build; 0: unknown)
};

// bf16 pair (lo, hi halves of w) -> two e4m3 bytes of x / s (x * inv),
// round to nearest even, saturating; first value in the low byte
__device__ __forceinline__ uint16_t bf16x2_to_e4m3x2(uint32_t w, float inv)
{
    const float2 f = make_float2(__uint_as_float(w << 16) * inv, __uint_as_float(w & 0xFFFF0000u) * inv);
    return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3));
}

// Row of the page pool for GEMM row r of a paged segment; -1 when the page
// id is outside [0, n_pages) (the caller skips the store and reports it).
__host__ __device__ inline long long paged_row(const EpiSeg &s, long long r)
{
    const long long u = r / s.map.P, t = r % s.map.P + s.map.B;
    const long long page = s.pages[u * s.pg_ustride + s.pg_off + t / OT_PAGE_ROWS];
    if (page < 0 || page >= s.n_pages) return -1;
    return (page * 2 + s.pg_kv) * OT_PAGE_ROWS + t % OT_PAGE_ROWS;
}

// OT_STORE_E4M3: e4m3 of (value / qscale[g * qscale_gstride]), rounded to
// nearest even and saturating (the per-tensor FP8 scale of the tensor the
// output feeds, so the next projection reads it without a quantisation pass)
enum { OT_STORE_F32 = 0, OT_STORE_BF16 = 1, OT_STORE_E4M3 = 2 };

// C[r, c] (group g) = epilogue( sum_k A[row_a(r,g), k] * B[g][c][k] ).
// Epilogue, in order: * rsqrt(mean_k A^2 + eps) if norm; * row_scale[row_a]
// if given; * g_scale[g] if given; GELU if gelu; + residual[row_res] if given.
struct GemmArgs {
    int M, N, K, G;
    const void *A;
    long long lda;
    RowMap a_map;
    const void *B;          // [G][N][K]
    long long b_gstride;    // elements between groups of B
    int in_dtype;           // OT_DTYPE_F32 / BF16 / FP8 (operand dtype)
    int store;              // OT_STORE_F32 / BF16
    int nseg;
    EpiSeg seg[3];
    int norm;
    float eps;
    const float *row_scale; // indexed by row_a(r, g)
    const float *g_scale;   // indexed by g
    const float *xg_scale;  // fp8 A operand with a per-group scale: xg_scale[g * xg_gstride]
    long long xg_gstride;
    const float *qscale;    // e4m3 output (OT_STORE_E4M3): its scale per group
    long long qscale_gstride;
    int gelu;
    const void *res;
    long long res_ld;
    RowMap res_map;
    long long res_cap;  // bytes from res to the end of its buffer (checked build; 0: unknown)
    WaitCtl wait;
};

// Attention over one layer.  Query rows come from Q [U][nq][d] (head h at
// columns h*hd); S keys / values from the per-user cache rows
// [U][L][d] (user stride s_ustride elements); NS keys / values from KN / VN
// [U][nkn][d] (NS mode, and S mode with full attention).
//   S mode  : query i is S row t = L - nq + i; it sees S keys 0..t.
//   NS mode : query i is NS token n = i % N of candidate c = i / N; it sees
//             all L S keys and NS keys m <= n of candidate c.
//   full    : full (non-causal) attention, one candidate per user in S mode:
//             an S row sees all L S keys and all nkn NS keys of its user; an
//             NS row all L S keys and all N NS keys of its candidate.
struct AttnArgs {
    int mode;           // 0 = S, 1 = NS
    int U, H, hd, d;
    int L;              // S keys
    int nq;             // query rows per user
    int N;              // NS tokens per candidate
    int full;           // 1: full attention
    int nkn;            // NS key rows per user in KN / VN (NS mode: nq)
    // paged S keys / values (pages != null): KS = VS = the page pool, key
    // block j / OT_PAGE_ROWS of user u in page pages[u * pg_ustride + pg_off + ...]
    const int *pages;
    long long pg_ustride, n_pages;
    int pg_off;
    const void *Q;
    const void *KS, *VS;
    long long s_ustride; // elements between users in KS / VS
    const void *KN, *VN;
    void *O;            // [U][nq][d]
    long long o_cap;    // bytes from O to the end of its buffer (checked build; 0: unknown)
    // e4m3 output (FP8 models with per-tensor scales): O holds e4m3(o / s),
    // s = o_qscale[0] for S rows, o_qscale[(i % N) * o_qstride] for NS row i
    const float *o_qscale;
    long long o_qstride;
    float scale;        // 1/sqrt(hd)
    int dtype;
    WaitCtl wait;
};

// Fused feed-forward over G groups of M rows:
//   Y[row_y(r, g)] = H[row_h(r, g)] + GELU(n(H) W1[g]^T) W2[g]^T,
// n(H) = H * rsqrt(mean(H^2) + eps) (the RMSNorm gain folded into W1).
// H / Y rows are D wide; W1 is [G][F][D], W2 is [G][D][F] (bf16).
//
// fuse_o: the attention's output projection and residual come first, in the
// same kernel: H = X + A Wo[g]^T, with A (the attention output) read where H
// is otherwise read (`H`, h_map), X the block input rows under x_map, Wo
// [G][D][D]; the residual of the FFN is then H in fp32.
struct FfnArgs {
    int M, G, D, F;
    const void *H;
    RowMap h_map;
    const void *W1;
    long long w1_gstride;   // elements between groups of W1
    const void *W2;
    long long w2_gstride;   // elements between groups of W2
    void *Y;
    RowMap y_map;
    float eps;
    WaitCtl wait;
    int fuse_o;
    const void *Wo;
    long long wo_gstride;   // elements between groups of Wo
    const void *X;
    RowMap x_map;
    // rows of each group actually filled (device, [G]; null: M each): tiles
    // past a group's count are skipped (the experts of a mixture)
    const int *group_rows;
};

// Page of key block b (OT_PAGE_ROWS keys) of user u in a paged cache;
// an id outside [0, n_pages) gives page 0 and sets the device error word,
// so no access ever leaves the pool.
__device__ inline long long attn_page(const AttnArgs &a, long long u, long long b)
{
    long long page = a.pages[u * a.pg_ustride + a.pg_off + b];
    if (page < 0 || page >= a.n_pages) {
        if (a.wait.err) atomicCAS(a.wait.err, 0, OT_ERR_DEVICE_BOUNDS);
        page = 0;
    }
    return page;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes; it must call pdl_wait() before
// touching global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Launchers (return cudaGetLastError() after the launch).
cudaError_t launch_gemm_simt(const GemmArgs &a, cudaStream_t s);
cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s);
// two problems with the same K, operand dtype and norm in one launch (a1 may be null)
cudaError_t launch_gemm_tc_multi(const GemmArgs &a, const GemmArgs *a1, cudaStream_t s);
cudaError_t launch_attn_simt(const AttnArgs &a, cudaStream_t s);
cudaError_t launch_attn_tc(const AttnArgs &a, cudaStream_t s);
// NS attention with all query rows of a (user, head) within 64 (decode-shaped)
bool attn_ns_small_supported(const AttnArgs &a);
cudaError_t launch_attn_ns_small(const AttnArgs &a, cudaStream_t s);
bool ffn_tc_supported(int D, int F);
cudaError_t launch_ffn_tc(const FfnArgs &a, cudaStream_t s);
// two problems with the same D, F and eps in one launch (a1 may be null)
cudaError_t launch_ffn_tc_multi(const FfnArgs &a, const FfnArgs *a1, cudaStream_t s);
cudaError_t launch_fold_gain(const void *W, const void *g, void *out, long long rows, int cols,
                             long long groups, long long g_gstride, int dtype, cudaStream_t s);
// Copy of the old K/V rows of a cache into the layout of longer sequences
// (appending S rows): per layer l, the len_src[l] units of K (then of V)
// starting at off_src[l] of a user's cache go to off_dst[l] (V at
// off_dst[l] + len_dst[l]) of the new one.  Units of 16 bytes.
struct KvGrowArgs {
    const uint4 *src;
    uint4 *dst;
    long long ustride_src, ustride_dst;
    long long off_src[OT_MAX_LAYERS], off_dst[OT_MAX_LAYERS];
    long long len_src[OT_MAX_LAYERS], len_dst[OT_MAX_LAYERS];
};
cudaError_t launch_kv_grow(const KvGrowArgs &a, int users, int layers, cudaStream_t s);
// Zero the unused rows of every layer's last page of a paged cache.
struct PageTailArgs {
    void *pool;
    const int *pages;
    long long pg_ustride, n_pages;
    int layers, d, esz;
    int L[OT_MAX_LAYERS], off[OT_MAX_LAYERS]; // rows and first page-table entry of each layer
    int *err;
};
cudaError_t launch_page_tail_clear(const PageTailArgs &a, int users, cudaStream_t s);
cudaError_t launch_embed_gather(const void *table, long long rows, int d, const int64_t *ids,
                                long long n, void *out, int *err, cudaStream_t s);
// Scale rule of an FP8 projection input (group g reads slot g * gstride):
// xscale = the input tensor's fixed scale (NULL: each row's amax / 448);
// amax = where each row's max |x| is max-accumulated (NULL: not recorded).
struct QuantRule {
    const float *xscale;
    float *amax;
    long long gstride;
};
cudaError_t launch_quant_rows(const void *X, long long lda, RowMap map, long long M, int G, int K,
                              const void *gain, long long gain_gstride, int norm, float eps,
                              QuantRule rule, uint8_t *q_out, float *scale_out, cudaStream_t s);
cudaError_t launch_quant_weights(const void *W, long long per_mat, long long mats, uint8_t *q_out,
                                 float *scale_out, float *amax_scratch, cudaStream_t s);

// Sparse mixture of experts (S-side FFN).  Router: rows of H [rows][d] ->
// for each row its top-k experts; choice j of row r takes slot counts[e]++
// of expert e, its row is copied to Hp[e * cap + slot] and route[2 r + j] =
// e * cap + slot, gate[2 r + j] = its gate.  counts must start at zero.
struct MoeRouteArgs {
    long long rows;
    int d, E, topk, dtype;
    float eps;
    const void *H, *gain, *Wr;   // gain [d] (RMSNorm before the FFN), Wr [E][d]
    void *Hp;                    // [E][cap][d]
    long long cap;
    int *counts;                 // [E]
    long long *route;            // [rows][2]
    float *gate;                 // [rows][2]
};
// Combine: Y[r] = H[r] + sum_j gate[2 r + j] (Yp[route[2 r + j]] - H[r]).
struct MoeCombineArgs {
    long long rows;
    int d, topk, dtype;
    const void *H, *Yp;
    void *Y;
    const long long *route;
    const float *gate;
};
cudaError_t launch_moe_route(const MoeRouteArgs &a, cudaStream_t s);
cudaError_t launch_moe_combine(const MoeCombineArgs &a, cudaStream_t s);

// Backward pass (fp32, CUDA cores).  Row sets of the backward kernels: row
// r of group g is buffer row map(r, g), rows of d floats.
struct BwRows {
    const float *X; // input rows
    RowMap map;
    long long rows;
    int G, d;
};
// C = A B^T (NT), A B (NN) or A^T B (TN), C an M x N block, reduction K:
//   NT: C[cmap(m, g)][n] (+)= sum_k A[amap(m, g)][k] B[g][n][k]
//   NN: C[cmap(m, g)][n] (+)= sum_k A[amap(m, g)][k] B[g][k][n]
//   TN: C[g][m][n]       (+)= sum_k A[amap(k, g)][m] B[bmap(k, g)][n]
// B[g] starts at B + g * b_gstride (NT / NN) with row stride ldb; C[g] of
// TN at C + g * c_gstride.
enum { BW_NT = 0, BW_NN = 1, BW_TN = 2 };
struct BwGemm {
    int form, M, N, K, G;
    const float *A;
    long long lda;
    RowMap a_map;
    const float *B;
    long long ldb, b_gstride;
    RowMap b_map;
    float *C;
    long long ldc, c_gstride;
    RowMap c_map;
    int accumulate;
    // TN only: the reduction split over `splits` CTAs, each writing its
    // partial block to partial[split][G][M][N]; a second kernel sums them in
    // split order into C (splits == 1: straight into C)
    int splits;
    float *partial;
    // segments (the experts of a mixture): group g owns buffer rows
    // g_off[g] .. g_off[g] + g_cnt[g] - 1, in place of the row maps of the
    // M rows (NT / NN: A and C) or of the K rows (TN: A and B); rows past
    // g_cnt[g] are not read or written.  Null: the row maps.
    const int *g_off, *g_cnt;
};
// One attention problem of a layer over QKV rows [.][3d] (Q | K | V):
//   mode 0 (S queries): query i of user u is S row t = L - nq + i of the
//     layer, buffer row u * q_ustride + q_off + i of qkv (= skv); it sees S
//     keys 0..t (full: all L S keys and the user's nkn NS keys).
//   mode 1 (NS queries): query i = c * N + n of user u is row
//     u * q_ustride + i of qkv; it sees the user's L S keys (rows u * L + j
//     of skv) and NS keys c * N + m, m <= n (full: every m of candidate c).
// NS keys of user u are rows u * n_ustride + r of nkv (mode 1: nkv = qkv).
// O / dO are [U * nq][d]; stat_* [U * nq][H] (m: the row's max score in
// base-2 units, s * scale * log2(e); l: the sum of 2^(s' - m); D: dO . O);
// dqkv / dskv take dQ and dK, dV in the layout of qkv / skv.
struct BwAttn {
    int mode, U, H, hd, d, L, nq, N;
    int full, nkn;      // full attention; NS key rows per user
    long long ld, q_ustride, q_off, n_ustride;
    const float *qkv, *skv, *nkv;
    float *dqkv, *dskv;
    float *O;
    const float *dO;
    float *stat_m, *stat_l, *stat_D;
    float scale;
};
cudaError_t bw_rms_fwd(const BwRows &a, const float *g, long long g_gstride, float eps, float *z, float *r,
                       cudaStream_t s);
cudaError_t bw_rms_bwd(const BwRows &a, const float *g, long long g_gstride, const float *r,
                       const float *dz, float *dx, int accumulate, cudaStream_t s);
cudaError_t bw_gain_grad(const BwRows &a, const float *r, const float *dz, float *partial, int splits,
                         float *dg, long long g_gstride, cudaStream_t s);
int bw_gain_splits(const BwRows &a);
cudaError_t bw_gelu_fwd(const float *u, float *a, long long n, cudaStream_t s);
cudaError_t bw_gelu_bwd(const float *u, const float *da, float *du, long long n, cudaStream_t s);
cudaError_t bw_rows_add(float *dst, RowMap dst_map, const float *src, long long rows, int d, cudaStream_t s);
cudaError_t bw_gemm(const BwGemm &p, cudaStream_t s);
// reduction split of a TN GEMM (2 * 148 CTAs as the target) and the partial
// buffer floats it needs (0 when not split)
int bw_tn_splits(int M, int N, int K, int G);
long long bw_tn_partial_floats(int M, int N, int K, int G);
cudaError_t bw_attn_fwd(const BwAttn &a, cudaStream_t s);
cudaError_t bw_attn_bwd_q(const BwAttn &a, cudaStream_t s);
cudaError_t bw_attn_bwd_kv_s(const BwAttn &sq, const BwAttn *nsq, cudaStream_t s);
// NS keys: the NS queries of problem a and, if sq (full attention), the S
// queries of sq
cudaError_t bw_attn_bwd_kv_ns(const BwAttn &a, const BwAttn *sq, cudaStream_t s);

// Mixture-of-experts routing of T rows in the backward pass: top-k of the
// E logits per row (ties to the lower index) and softmax gates; a fixed,
// expert-major slot per choice (experts in order, rows in order within an
// expert, no atomics): segment e = slots seg_off[e] .. + seg_cnt[e].
struct BwMoe {
    int T, d, E, k;
    const float *logits; // [T][E]
    int *sel;            // [T][2] chosen experts
    float *gate;         // [T][2]
    int *lrank;          // [T][2] rank within the choice's 128-row chunk
    int *hist;           // [chunks][E]
    int *seg_off, *seg_cnt; // [E]
    int *slot;           // [T][2]
};
int bw_moe_chunks(int T);
// route + copy z rows to their slots (Zp [T k][d]); 4 launches
cudaError_t bw_moe_route(const BwMoe &m, const float *z, float *Zp, cudaStream_t s);
// y = h + sum_j gate_j Y[slot_j]
cudaError_t bw_moe_combine(const BwMoe &m, const float *h, const float *Y, float *y, cudaStream_t s);
// dY[slot_j] = gate_j dy; dlogits [T][E] from the gates' softmax
cudaError_t bw_moe_combine_bwd(const BwMoe &m, const float *dy, const float *Y, float *dY, float *dlogits,
                               cudaStream_t s);
// dz[r] += sum_j dZp[slot_j]
cudaError_t bw_moe_gather(const BwMoe &m, const float *dZp, float *dz, cudaStream_t s);

// Shape / dtype check of a config (the rules of ot_model_create).
ot_status internal_check_config(const ot_config &c);

// Read-only model queries for entry points defined outside ot_api.cu.
int internal_profiling(const ot_model *m);
int internal_device(const ot_model *m);
int internal_n_ns(const ot_model *m);
size_t internal_score_ws_bytes(const ot_model *m, int users, int cands);

// cuTensorMapEncodeTiled through the runtime's driver entry point.
int encode_tmap_3d(void *map, int dtype_bytes, const void *base, const uint64_t dims[3],
                   const uint64_t strides_bytes[2], const uint32_t box[3]);

} // namespace ot
