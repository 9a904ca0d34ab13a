// Host entry points of the C ABI declared in include/onetrans.h: argument
// checks, weight preparation, workspace layout and the per-layer launch
// sequence of the OneTrans block stack.
//
// Per layer l of the S-side (encode, U users, L = L_l rows per user, q = q_l):
//   1. S QKV GEMM over all U*L rows (RMSNorm row scale in the epilogue, gain
//      folded into W): K, V -> KV cache rows of layer l; Q -> only the tail
//      rows t >= L - q, packed [U][q][d].
//   2. S attention (bottom-right causal over the tail) -> A [U][q][d].
//   3. O GEMM + residual from the tail rows of the layer input -> H.
//   4. FFN1 GEMM (norm, GELU) -> hidden; FFN2 GEMM + residual H -> next X.
// Per layer of the NS-side (score, U users x C candidates x N tokens):
//   the same four steps with grouped GEMMs (group = NS position n, its own
//   weights), and NS attention against layer l of the cache.
// Full forward (both sides): steps 1, 3 and 4 of the two sides share one
// launch each (the NS tiles fill the S launch's last partial wave); the NS
// attention runs on a second stream beside the S attention.
#include <cudaTypedefs.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <cstdlib>
#include <initializer_list>
#include <mutex>
#include <utility>
#include <new>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "ot_internal.h"

struct ot_model {
    ot_config cfg;
    int device;
    int esz;            // storage bytes per element
    int path;           // 0 = tensor-core kernels (bf16 / fp8), 1 = CUDA-core kernels
    // bf16 / fp32: gains folded into Wqkv and W1.  fp8: e4m3 copies (gains
    // kept separately and applied in the quantisation pass) + per-matrix scales.
    void *Wqkv_s, *Wo_s, *W1_s, *W2_s;
    void *Wqkv_ns, *Wo_ns, *W1_ns, *W2_ns;
    void *W_split;
    // mixture of experts: router, experts' W1 (gain g2 folded), W2
    void *W_router = nullptr, *W1_moe = nullptr, *W2_moe = nullptr;
    float *sc_qkv_s, *sc_o_s, *sc_1_s, *sc_2_s, *sc_qkv_ns, *sc_o_ns, *sc_1_ns, *sc_2_ns;
    // fp8: per-tensor activation scales [layers][1 + n_ns][4] (device; null =
    // per-row scales), and while ot_fp8_calibrate enqueues, the caller's amax
    // array (same layout) with per-row scales forced
    float *act_scale = nullptr;
    float *act_scale_mem = nullptr;
    float *calib_amax = nullptr;
    void *g1_s, *g2_s, *g1_ns, *g2_ns;
    int *err;
    long long wait_limit;
    long long launches;
    std::vector<void *> allocs;
    // per-launch profiling
    struct Rec {
        int kind, role;
        double flops, bytes;
        cudaEvent_t e0, e1;
    };
    int profiling = 0;
    std::vector<Rec> recs;
    std::vector<cudaEvent_t> event_pool;
    // full_forward overlap: the NS side runs on `side`, layer l starting once
    // kv_ready[l] (recorded after the S QKV GEMM of layer l) has fired.
    cudaStream_t side = nullptr;
    cudaEvent_t kv_ready[OT_MAX_LAYERS];
    cudaEvent_t ns_attn_done[OT_MAX_LAYERS]; // merged full forward: NS attention of layer l
    cudaEvent_t fork_ev = nullptr, join_ev = nullptr;
    // ot_full_forward_host: inputs travel on their own stream into one of two
    // staging slots; in_ready[s] = slot s holds its inputs, in_free[s] = the
    // forward that read slot s is done with it
    cudaStream_t copy_stream = nullptr;
    cudaEvent_t in_ready[2] = {nullptr, nullptr}, in_free[2] = {nullptr, nullptr};
    unsigned long long host_calls = 0;
    // event re-recording must not interleave between calls (recursive: a host
    // call holds it across the forward it enqueues)
    std::recursive_mutex enqueue_mu;
};

namespace ot {

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int encode_tmap_3d(void *map, int esz, const void *base, const uint64_t dims[3],
                   const uint64_t strides_bytes[2], const uint32_t box[3])
{
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return 1;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (strides_bytes[0] & 15) ||
        (strides_bytes[1] & 15))
        return 1;
    CUtensorMapDataType dt = esz == 2   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                             : esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    cuuint64_t gd[3] = {dims[0], dims[1], dims[2]};
    cuuint64_t gs[2] = {strides_bytes[0], strides_bytes[1]};
    cuuint32_t bx[3] = {box[0], box[1], box[2]};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = g_encode(reinterpret_cast<CUtensorMap *>(map), dt, 3, const_cast<void *>(base),
                          gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r != CUDA_SUCCESS;
}

int internal_profiling(const ot_model *m) { return m->profiling; }

int internal_device(const ot_model *m) { return m->device; }

int internal_n_ns(const ot_model *m) { return m->cfg.n_ns; }

} // namespace ot

using namespace ot;

namespace {

inline int rows_at(const ot_config &c, int l) { return l == 0 ? c.L0 : c.q[l - 1]; }

inline long long kv_layer_off(const ot_config &c, int l)
{
    long long off = 0;
    for (int j = 0; j < l; ++j) off += 2LL * c.d * rows_at(c, j);
    return off;
}

inline long long kv_user_elems(const ot_config &c) { return kv_layer_off(c, c.layers); }

// Paged KV cache: first page-table entry of layer l (one entry per
// OT_PAGE_ROWS rows of each layer) and the entries of one user.
inline int page_off(const ot_config &c, int l)
{
    int off = 0;
    for (int j = 0; j < l; ++j) off += (rows_at(c, j) + OT_PAGE_ROWS - 1) / OT_PAGE_ROWS;
    return off;
}

// A paged cache as the runs address it.
struct PagedKv {
    void *pool;
    const int *pages;
    long long n_pages;
    long long ustride; // page-table entries per user
};

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

inline char *at(const void *base, long long elems, int esz)
{
    return const_cast<char *>(static_cast<const char *>(base)) + elems * esz;
}

ot_status check_config(const ot_config &c)
{
    if (c.layers < 1 || c.layers > OT_MAX_LAYERS || c.d < 1 || c.heads < 1 || c.ffn < 1 ||
        c.n_ns < 1 || c.L0 < 1 || c.F < 0 || !(c.eps >= 0.f))
        return OT_ERR_ARG;
    if (c.dtype != OT_DTYPE_F32 && c.dtype != OT_DTYPE_BF16 && c.dtype != OT_DTYPE_FP8)
        return OT_ERR_DTYPE;
    if (c.full_attn != 0 && c.full_attn != 1) return OT_ERR_ARG;
    if (c.moe_experts < 0 || c.moe_experts > 64) return OT_ERR_SHAPE;
    if (c.moe_experts > 0) {
        if (c.moe_topk < 1 || c.moe_topk > 2 || c.moe_topk > c.moe_experts) return OT_ERR_ARG;
        if (c.dtype == OT_DTYPE_FP8) return OT_ERR_DTYPE;
        if (c.d != 64 && c.d != 128 && c.d != 256) return OT_ERR_SHAPE; // the router's row widths
    }
    if (c.d % c.heads) return OT_ERR_SHAPE;
    int L = c.L0;
    for (int l = 0; l < c.layers; ++l) {
        if (c.q[l] < 1 || c.q[l] > L) return OT_ERR_SHAPE;
        L = c.q[l];
    }
    const int hd = c.d / c.heads;
    if (c.dtype == OT_DTYPE_F32) {
        if (hd != 16 && hd != 32 && hd != 64) return OT_ERR_SHAPE;
    } else {
        if (hd != 64 || c.d % 128 || c.ffn % 128 || c.F % 64) return OT_ERR_SHAPE;
        if (c.dtype == OT_DTYPE_FP8 && (c.d % 128 || c.ffn % 128 || c.d > 1536 || c.ffn > 1536))
            return OT_ERR_SHAPE;
    }
    if (static_cast<long long>(c.n_ns) > 4096) return OT_ERR_SHAPE;
    return OT_OK;
}

struct Ws {
    char *p;
    size_t left;
    int esz;
    void *take(long long elems)
    {
        size_t b = (static_cast<size_t>(elems) * esz + 255) & ~static_cast<size_t>(255);
        if (b > left) return nullptr;
        void *r = p;
        p += b;
        left -= b;
        return r;
    }
};

size_t bytes_of(long long elems, int esz)
{
    return (static_cast<size_t>(elems) * esz + 255) & ~static_cast<size_t>(255);
}

size_t fp8_ws_bytes(const ot_config &c, long long rows)
{
    if (c.dtype != OT_DTYPE_FP8) return 0;
    return bytes_of(rows * (c.d > c.ffn ? c.d : c.ffn), 1) + bytes_of(rows, 4);
}

// mixture of experts: expert-major rows in (Hp) and out (Yp), the experts'
// hidden (two-GEMM paths), routes (int64) and gates of 2 choices per row,
// the experts' row counts
size_t moe_ws_bytes(const ot_config &c, long long rows, int esz)
{
    if (c.moe_experts <= 0) return 0;
    const long long er = rows * c.moe_experts;
    return 2 * bytes_of(er * c.d, esz) + bytes_of(er * c.ffn, esz) + bytes_of(rows * 2, 8) +
           bytes_of(rows * 2, 4) + bytes_of(c.moe_experts, 4);
}

size_t encode_ws_bytes(const ot_config &c, int U, int esz)
{
    long long rows = static_cast<long long>(U) * c.L0;
    return 5 * bytes_of(rows * c.d, esz) + bytes_of(rows * c.ffn, esz) + fp8_ws_bytes(c, rows) +
           moe_ws_bytes(c, rows, esz);
}

size_t score_ws_bytes(const ot_config &c, int U, int C, int esz)
{
    long long rows = static_cast<long long>(U) * C * c.n_ns;
    return 7 * bytes_of(rows * c.d, esz) + bytes_of(rows * c.ffn, esz) + fp8_ws_bytes(c, rows);
}

enum { ROLE_S_QKV = 0, ROLE_S_ATTN, ROLE_S_O, ROLE_S_FFN1, ROLE_S_FFN2, ROLE_NS_QKV, ROLE_NS_ATTN,
       ROLE_NS_O, ROLE_NS_FFN1, ROLE_NS_FFN2, ROLE_AUTO_SPLIT, ROLE_OTHER, ROLE_S_FFN, ROLE_NS_FFN,
       // one launch for the S and NS sides of a layer (full forward)
       ROLE_O, ROLE_FFN, ROLE_QKV,
       ROLE_S_MOE }; // routing / combining the rows of a mixture of experts

cudaEvent_t pooled_event(ot_model *m)
{
    if (!m->event_pool.empty()) {
        cudaEvent_t e = m->event_pool.back();
        m->event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Name of a launch role for NVTX ranges (the same order as ot_launch_record::role).
const char *role_name(int role)
{
    static const char *names[] = {"S-QKV", "S-attn", "S-O", "S-FFN1", "S-FFN2", "NS-QKV", "NS-attn",
                                  "NS-O", "NS-FFN1", "NS-FFN2", "Auto-Split", "other", "S-FFN",
                                  "NS-FFN", "O", "FFN", "QKV", "S-MoE"};
    return role >= 0 && role <= ROLE_S_MOE ? names[role] : "launch";
}

// Launch `fn` bracketed by profiling events when profiling is on, inside an
// NVTX range named for its role (free when no tool is attached; a profiler
// timeline then shows which step of the block each kernel is).
template <typename F>
ot_status profiled(ot_model *m, cudaStream_t s, int kind, int role, double flops, double bytes,
                   F fn)
{
    nvtxRangePushA(role_name(role));
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    const bool prof = m->profiling && m->recs.size() < (1u << 16);
    if (prof) {
        e0 = pooled_event(m);
        e1 = pooled_event(m);
        if (e0) cudaEventRecord(e0, s);
    }
    cudaError_t e = fn();
    m->launches++;
    if (prof && e0 && e1) {
        cudaEventRecord(e1, s);
        m->recs.push_back(ot_model::Rec{kind, role, flops, bytes, e0, e1});
    }
    nvtxRangePop();
    return e == cudaSuccess ? OT_OK : OT_ERR_CUDA;
}

long long kept_rows(const RowMap &mp, long long M)
{
    long long full = (M / mp.P) * (mp.P - mp.min_t);
    long long rem = M % mp.P - mp.min_t;
    return full + (rem > 0 ? rem : 0);
}

// algorithmic flops and bytes of one GEMM problem (per-launch profiling)
void gemm_cost(const ot_model *m, const GemmArgs &a, double &flops, double &bytes)
{
    const double esz = a.in_dtype == OT_DTYPE_FP8 ? 1 : m->esz, G = a.G;
    double out_elems = 0;
    for (int i = 0; i < a.nseg; ++i)
        out_elems += static_cast<double>(kept_rows(a.seg[i].map, a.M)) * (a.seg[i].c_hi - a.seg[i].c_lo);
    flops += 2.0 * a.K * out_elems * G;
    bytes += esz * G * (static_cast<double>(a.M) * a.K + static_cast<double>(a.N) * a.K + out_elems +
                        (a.res ? static_cast<double>(a.M) * a.N : 0.0));
}

long long cap_of(const void *p); // extent of a caller buffer (checked build)

void gemm_prepare(const ot_model *m, GemmArgs &a)
{
    a.wait = WaitCtl{m->err, m->wait_limit};
    // operand dtype: e4m3 only where the caller prepared quantised operands
    a.in_dtype = m->cfg.dtype == OT_DTYPE_F32 ? OT_DTYPE_F32
                 : a.in_dtype == OT_DTYPE_FP8 ? OT_DTYPE_FP8
                                              : OT_DTYPE_BF16;
    a.store = m->cfg.dtype == OT_DTYPE_F32 ? OT_STORE_F32 : a.qscale ? OT_STORE_E4M3 : OT_STORE_BF16;
    a.res_cap = cap_of(a.res);
}

ot_status gemm(ot_model *m, GemmArgs &a, cudaStream_t s, int role)
{
    gemm_prepare(m, a);
    const bool simt = m->cfg.dtype == OT_DTYPE_F32 || m->path == 1;
    if (simt && a.in_dtype == OT_DTYPE_FP8) return OT_ERR_UNSUPPORTED;
    double flops = 0, bytes = 0;
    if (m->profiling) gemm_cost(m, a, flops, bytes);
    return profiled(m, s, simt ? OT_KIND_GEMM_SIMT : OT_KIND_GEMM_TC, role, flops, bytes, [&] {
        return simt ? launch_gemm_simt(a, s) : launch_gemm_tc(a, s);
    });
}

// algorithmic flops (visible query-key pairs) and bytes of one attention problem
void attn_cost(const ot_model *m, const AttnArgs &a, double &flops, double &bytes)
{
    const double L = a.L, nq = a.nq, N = a.N, U = a.U, esz = m->esz;
    double pairs; // visible (query, key) pairs per user and head
    if (a.full)
        pairs = a.mode == 0 ? nq * (L + a.nkn) : nq * (L + N);
    else if (a.mode == 0)
        pairs = nq * (L - nq) + nq * (nq + 1) / 2;
    else
        pairs = (nq / N) * (N * L + N * (N + 1) / 2);
    flops += 4.0 * a.hd * pairs * a.H * U;
    bytes += esz * U * a.d * (2 * nq + 2 * L + ((a.mode == 1 || a.full) ? 2.0 * a.nkn : 0.0));
}

ot_status attn(ot_model *m, AttnArgs &a, cudaStream_t s)
{
    a.wait = WaitCtl{m->err, m->wait_limit};
    a.o_cap = cap_of(a.O);
    if (a.mode == 1) a.nkn = a.nq;
    if (a.mode == 0 && a.full && (!a.KN || !a.VN || a.nkn < 1)) return OT_ERR_ARG;
    a.dtype = m->cfg.dtype;
    const bool simt = m->cfg.dtype == OT_DTYPE_F32 || m->path == 1;
    double flops = 0, bytes = 0;
    if (m->profiling) attn_cost(m, a, flops, bytes);
    // a few NS rows per (user, head): the decode-shaped kernel
    const bool ns_small = !simt && attn_ns_small_supported(a);
    return profiled(m, s, simt ? OT_KIND_ATTN_SIMT : ns_small ? OT_KIND_ATTN_NS : OT_KIND_ATTN_TC,
                    a.mode == 0 ? ROLE_S_ATTN : ROLE_NS_ATTN, flops, bytes, [&] {
                        return simt ? launch_attn_simt(a, s)
                               : ns_small ? launch_attn_ns_small(a, s)
                                          : launch_attn_tc(a, s);
                    });
}

// The fused FFN kernel runs for bf16 models on the tensor-core path (not for
// path 2, which keeps the two FFN GEMMs for cross-checks) at supported widths.
bool use_fused_ffn(const ot_model *m)
{
    return m->cfg.dtype == OT_DTYPE_BF16 && m->path == 0 && ffn_tc_supported(m->cfg.d, m->cfg.ffn);
}

// Y = H + GELU(n(H) W1^T) W2^T over G groups of M rows (gain folded into W1).
FfnArgs ffn_args(const ot_model *m, int M, int G, const void *H, RowMap h_map, const void *W1,
                 const void *W2, void *Y, RowMap y_map)
{
    const ot_config &c = m->cfg;
    FfnArgs a;
    memset(&a, 0, sizeof(a));
    a.M = M;
    a.G = G;
    a.D = c.d;
    a.F = c.ffn;
    a.H = H;
    a.h_map = h_map;
    a.W1 = W1;
    a.w1_gstride = static_cast<long long>(c.ffn) * c.d;
    a.W2 = W2;
    a.w2_gstride = static_cast<long long>(c.d) * c.ffn;
    a.Y = Y;
    a.y_map = y_map;
    a.eps = c.eps;
    a.wait = WaitCtl{m->err, m->wait_limit};
    return a;
}

// rows_override > 0: the rows actually computed (a mixture's routed rows,
// not every slot of every expert)
void ffn_cost(const FfnArgs &a, double &flops, double &bytes, double rows_override = 0)
{
    const double rows = rows_override > 0 ? rows_override : static_cast<double>(a.M) * a.G,
                 d = a.D, f = a.F;
    flops += 4.0 * rows * d * f;
    bytes += 2.0 * (2.0 * rows * d + 2.0 * a.G * d * f); // H in, Y out, W1 + W2 once
    if (a.fuse_o) {
        flops += 2.0 * rows * d * d;
        bytes += 2.0 * (rows * d + a.G * d * d); // X in, Wo once (A in replaces H in)
    }
}

// The FFN with the attention's output projection in front (FfnArgs::fuse_o):
// H = X + A Wo^T, A read as the FFN's H otherwise is (rows under a_map), X
// under x_map; then Y = H + GELU(n(H) W1^T) W2^T.
FfnArgs ffn_o_args(const ot_model *m, int M, int G, const void *A, RowMap a_map, const void *Wo,
                   const void *X, RowMap x_map, const void *W1, const void *W2, void *Y, RowMap y_map)
{
    FfnArgs a = ffn_args(m, M, G, A, a_map, W1, W2, Y, y_map);
    a.fuse_o = 1;
    a.Wo = Wo;
    a.wo_gstride = static_cast<long long>(m->cfg.d) * m->cfg.d;
    a.X = X;
    a.x_map = x_map;
    return a;
}

ot_status ffn_run(ot_model *m, const FfnArgs &a, cudaStream_t s, int role, double routed_rows = 0)
{
    double flops = 0, bytes = 0;
    if (m->profiling) ffn_cost(a, flops, bytes, routed_rows);
    return profiled(m, s, OT_KIND_FFN_TC, role, flops, bytes, [&] { return launch_ffn_tc(a, s); });
}

// One launch for the S and NS problems of a layer step (either may be absent).
ot_status gemm2(ot_model *m, GemmArgs *a, GemmArgs *b, cudaStream_t s, int role)
{
    if (!a) a = b, b = nullptr;
    if (!a) return OT_ERR_ARG;
    double flops = 0, bytes = 0;
    for (GemmArgs *g : {a, b})
        if (g) {
            gemm_prepare(m, *g);
            if (m->profiling) gemm_cost(m, *g, flops, bytes);
        }
    return profiled(m, s, OT_KIND_GEMM_TC, role, flops, bytes,
                    [&] { return launch_gemm_tc_multi(*a, b, s); });
}

ot_status ffn2(ot_model *m, FfnArgs *a, FfnArgs *b, cudaStream_t s)
{
    if (!a) a = b, b = nullptr;
    if (!a) return OT_ERR_ARG;
    double flops = 0, bytes = 0;
    if (m->profiling) {
        ffn_cost(*a, flops, bytes);
        if (b) ffn_cost(*b, flops, bytes);
    }
    return profiled(m, s, OT_KIND_FFN_TC, ROLE_FFN, flops, bytes,
                    [&] { return launch_ffn_tc_multi(*a, b, s); });
}

GemmArgs gemm_base(const ot_config &c, int M, int N, int K, int G)
{
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.M = M;
    a.N = N;
    a.K = K;
    a.G = G;
    a.a_map = rowmap_identity();
    a.res_map = rowmap_identity();
    a.eps = c.eps;
    a.in_dtype = -1; // storage dtype unless a projection is prepared in fp8
    return a;
}

// Scratch for the fp8 operand of one projection (reused by every GEMM).
struct Fp8Scratch {
    uint8_t *q;
    float *s;
};

// Projection inputs in the per-tensor scale layout [layer][set][4].
enum { IN_QKV = 0, IN_O = 1, IN_W1 = 2, IN_W2 = 3 };

// Attach the A operand and weights of a projection GEMM.  src: activation
// rows (lda elements apart, through amap); W: weights of group 0 of this
// layer (gstride elements between groups); norm: the projection follows an
// RMSNorm with gain `gain` (gain_gstride elements between groups).
// bf16 / fp32: the norm runs inside the GEMM and the gain is already folded
// into W.  fp8: one pass quantises every (normalised) row to e4m3 -- with the
// input tensor's per-tensor scale (layer l, parameter set set0 + group, input
// `in`) when the model has them, else with the row's own scale -- and the
// GEMM reads the quantised weights and both scales.
ot_status projection(ot_model *m, GemmArgs &g, const void *src, long long lda, RowMap amap,
                     const void *W, long long w_gstride, const float *wscale, const void *gain,
                     long long gain_gstride, bool norm, const Fp8Scratch &f8, cudaStream_t st,
                     int l = 0, int set0 = 0, int in = 0)
{
    g.a_map = amap;
    g.b_gstride = w_gstride;
    g.B = W;
    if (m->cfg.dtype != OT_DTYPE_FP8) {
        g.A = src;
        g.lda = lda;
        g.norm = norm ? 1 : 0;
        return OT_OK;
    }
    double bytes = 0;
    if (m->profiling)
        bytes = static_cast<double>(g.M) * g.G * g.K * (2 + 1) + static_cast<double>(g.M) * g.G * 4;
    const long long slot = (static_cast<long long>(l) * (1 + m->cfg.n_ns) + set0) * 4 + in;
    QuantRule rule{nullptr, nullptr, 4};
    if (m->calib_amax) rule.amax = m->calib_amax + slot; // calibration: per-row scales
    else if (m->act_scale) rule.xscale = m->act_scale + slot;
    ot_status r = profiled(m, st, OT_KIND_QUANT, ROLE_OTHER, 0.0, bytes, [&] {
        return launch_quant_rows(src, lda, amap, g.M, g.G, g.K, gain, gain_gstride, norm ? 1 : 0,
                                 m->cfg.eps, rule, f8.q, f8.s, st);
    });
    if (r != OT_OK) return r;
    g.A = f8.q;
    g.lda = g.K;
    g.norm = 0;
    g.row_scale = f8.s;
    g.g_scale = wscale;
    g.in_dtype = OT_DTYPE_FP8;
    return OT_OK;
}

// FP8 with per-tensor activation scales (and not calibrating): the first
// FFN projection's epilogue writes the hidden as e4m3 with the second
// projection's input scale, and the second projection reads it as is — no
// quantisation pass over the 4d-wide hidden.
bool fp8_fused_hidden(const ot_model *m)
{
    return m->cfg.dtype == OT_DTYPE_FP8 && m->act_scale && !m->calib_amax;
}

// per-tensor scale of input `in` of layer l, parameter set `set` (sets of
// consecutive groups are 4 slots apart)
const float *act_slot(const ot_model *m, int l, int set, int in)
{
    return m->act_scale + (static_cast<long long>(l) * (1 + m->cfg.n_ns) + set) * 4 + in;
}

// The second FFN projection on the e4m3 hidden the first one wrote.
void fp8_hidden_operand(GemmArgs &g, const void *hid, long long lda, RowMap amap, const void *W, long long w_gstride,
                        const float *wscale, const float *xscale)
{
    g.A = hid;
    g.lda = lda;
    g.a_map = amap;
    g.B = W;
    g.b_gstride = w_gstride;
    g.norm = 0;
    g.row_scale = nullptr;
    g.g_scale = wscale;
    g.xg_scale = xscale;
    g.xg_gstride = 4;
    g.in_dtype = OT_DTYPE_FP8;
}

// Extents of the caller's buffers during one call (used by the checked
// build): a pointer inside one of them gets the bytes to its end as the
// bound of the kernels' plain accesses through it.  Thread-local, set by
// each entry point for the length of the call.
struct Region {
    const char *b, *e;
};
thread_local Region t_regions[8];
thread_local int t_nregions = 0;

struct RegionScope {
    RegionScope(std::initializer_list<std::pair<const void *, size_t>> rs)
    {
        t_nregions = 0;
        for (const auto &r : rs)
            if (r.first && r.second && t_nregions < 8)
                t_regions[t_nregions++] = Region{static_cast<const char *>(r.first),
                                                 static_cast<const char *>(r.first) + r.second};
    }
    ~RegionScope() { t_nregions = 0; }
};

// Checked build test hook: OT_CHECK_SHRINK=1 halves every extent, so that
// the kernels' checks fire (and skip the accesses) on a correct call.
bool check_shrink()
{
    static const bool on = kDeviceChecks && getenv("OT_CHECK_SHRINK") && atoi(getenv("OT_CHECK_SHRINK")) == 1;
    return on;
}

long long cap_of(const void *p)
{
    if (!kDeviceChecks || !p) return 0;
    const char *c = static_cast<const char *>(p);
    for (int i = 0; i < t_nregions; ++i)
        if (c >= t_regions[i].b && c < t_regions[i].e) {
            const long long cap = t_regions[i].e - c;
            return check_shrink() ? (cap + 1) / 2 : cap;
        }
    return 0;
}

size_t kv_bytes(const ot_model *m, int U) { return static_cast<size_t>(U) * kv_user_elems(m->cfg) * m->esz; }
size_t tail_bytes(const ot_model *m, int U)
{
    return static_cast<size_t>(U) * m->cfg.q[m->cfg.layers - 1] * m->cfg.d * m->esz;
}
size_t ns_bytes(const ot_model *m, long long rows) { return static_cast<size_t>(rows) * m->cfg.n_ns * m->cfg.d * m->esz; }

EpiSeg seg_of(void *out, long long ld, int lo, int hi, RowMap map)
{
    EpiSeg s{};
    s.out = out;
    s.cap = cap_of(out);
    s.ld = ld;
    s.c_lo = lo;
    s.c_hi = hi;
    s.map = map;
    return s;
}

// Attention arguments shared by both sides of a layer.
AttnArgs attn_base(const ot_config &c, int mode, int U, int L, int nq, const void *Q,
                   const void *K, const void *V, void *O)
{
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.mode = mode;
    a.U = U;
    a.H = c.heads;
    a.hd = c.d / c.heads;
    a.d = c.d;
    a.L = L;
    a.nq = nq;
    a.N = c.n_ns;
    a.Q = Q;
    a.KS = K;
    a.VS = V;
    a.s_ustride = kv_user_elems(c);
    a.O = O;
    a.scale = 1.0f / sqrtf(static_cast<float>(a.hd));
    a.full = c.full_attn;
    return a;
}

// Read the S keys / values of layer l from a paged cache.
void attn_paged(AttnArgs &a, const ot_config &c, const PagedKv *pg, int l)
{
    if (!pg) return;
    a.KS = a.VS = pg->pool;
    a.pages = pg->pages;
    a.pg_ustride = pg->ustride;
    a.n_pages = pg->n_pages;
    a.pg_off = page_off(c, l);
}

// Write the K (kv = 0) or V (kv = 1) segment of layer l into a paged cache.
void seg_paged(EpiSeg &s, const ot_config &c, const PagedKv *pg, int l, int kv)
{
    s.out = pg->pool;
    s.pages = pg->pages;
    s.pg_ustride = pg->ustride;
    s.n_pages = pg->n_pages;
    s.pg_off = page_off(c, l);
    s.pg_kv = kv;
}

// S-side of every layer for U users, one layer at a time: qkv(l), then
// rest(l) (attention, output projection, FFN).  X0: [U][L0][d]; s_out may
// be null.  delta > 0 appends: X0 holds only the delta new rows per user,
// and only they run through each layer (the last delta of its L_l rows, all
// of them queries), attending to the cached K/V of the old rows, which the
// caller has already placed in `kv`; their own K/V go after the old rows.
// full_last: run the whole last layer even when s_out is null (its output
// goes to a workspace buffer; calibration needs its projections).
// Full attention: ns_K / ns_V / ns_rows name the NS keys and values of the
// layer (one candidate per user) that the S rows also see.
struct EncodeRun {
    ot_model *m;
    int U;
    void *kv, *s_out;
    cudaStream_t st;
    cudaEvent_t *kv_ready;
    int delta;
    bool full_last;
    void *Xb[2], *Qb, *Ab, *Hb, *hid;
    Fp8Scratch f8{nullptr, nullptr};
    // mixture of experts: expert-major rows, hidden, routes, gates, counts
    void *Hp = nullptr, *Yp = nullptr, *ehid = nullptr;
    long long *route = nullptr;
    float *gate = nullptr;
    int *counts = nullptr;
    const void *X;
    bool done = false; // the last layer ran its K/V projection only
    const void *ns_K = nullptr, *ns_V = nullptr;
    int ns_rows = 0;
    const PagedKv *pg = nullptr; // the cache is paged (kv unused)

    ot_status init(const void *X0, Ws ws)
    {
        const ot_config &c = m->cfg;
        const long long rows0 = static_cast<long long>(U) * (delta ? delta : c.L0);
        Xb[0] = ws.take(rows0 * c.d);
        Xb[1] = ws.take(rows0 * c.d);
        Qb = ws.take(rows0 * c.d);
        Ab = ws.take(rows0 * c.d);
        Hb = ws.take(rows0 * c.d);
        hid = ws.take(rows0 * c.ffn);
        if (!Xb[0] || !Xb[1] || !Qb || !Ab || !Hb || !hid) return OT_ERR_WORKSPACE_TOO_SMALL;
        if (c.dtype == OT_DTYPE_FP8) {
            Ws w1{ws.p, ws.left, 1};
            f8.q = static_cast<uint8_t *>(w1.take(rows0 * (c.d > c.ffn ? c.d : c.ffn)));
            Ws w4{w1.p, w1.left, 4};
            f8.s = static_cast<float *>(w4.take(rows0));
            if (!f8.q || !f8.s) return OT_ERR_WORKSPACE_TOO_SMALL;
        }
        if (c.moe_experts > 0) {
            const long long er = rows0 * c.moe_experts;
            Hp = ws.take(er * c.d);
            Yp = ws.take(er * c.d);
            ehid = ws.take(er * c.ffn);
            Ws w8{ws.p, ws.left, 8};
            route = static_cast<long long *>(w8.take(rows0 * 2));
            Ws w4{w8.p, w8.left, 4};
            gate = static_cast<float *>(w4.take(rows0 * 2));
            counts = static_cast<int *>(w4.take(c.moe_experts));
            if (!Hp || !Yp || !ehid || !route || !gate || !counts) return OT_ERR_WORKSPACE_TOO_SMALL;
        }
        X = X0;
        return OT_OK;
    }
    int rows(int l) const { return delta ? delta : rows_at(m->cfg, l); }   // rows run through layer l
    int tail(int l) const { return delta ? delta : m->cfg.q[l]; }          // their query tail
    char *K(int l) const { return at(kv, kv_layer_off(m->cfg, l), m->esz); }
    char *V(int l) const { return K(l) + static_cast<long long>(rows_at(m->cfg, l)) * m->cfg.d * m->esz; }

    // 1. QKV (or KV only): RMSNorm1 + shared projection; K/V into the cache
    ot_status qkv(int l)
    {
        const ot_config &c = m->cfg;
        const int d = c.d, esz = m->esz, L = rows_at(c, l), n = rows(l), q = tail(l);
        const bool fp8 = c.dtype == OT_DTYPE_FP8;
        const int wesz = fp8 ? 1 : esz; // bytes per weight element as the GEMM reads it
        const bool last = l == c.layers - 1;
        // the S tail of the last layer is unused
        const bool kv_only = last && s_out == nullptr && !full_last;
        const RowMap cache_map{n, kv_user_elems(c) / d, L - n, 0, 0};
        const void *g1 = fp8 ? at(m->g1_s, static_cast<long long>(l) * d, esz) : nullptr;
        GemmArgs g = gemm_base(c, U * n, kv_only ? 2 * d : 3 * d, d, 1);
        ot_status r;
        if ((r = projection(m, g, X, d, rowmap_identity(),
                            at(m->Wqkv_s, static_cast<long long>(l) * 3 * d * d + (kv_only ? d * d : 0), wesz),
                            3LL * d * d, fp8 ? m->sc_qkv_s + l : nullptr, g1, d, true, f8, st, l, 0,
                            IN_QKV)) != OT_OK)
            return r;
        if (kv_only) {
            g.nseg = 2;
            g.seg[0] = seg_of(pg ? nullptr : K(l), d, 0, d, cache_map);
            g.seg[1] = seg_of(pg ? nullptr : V(l), d, d, 2 * d, cache_map);
        } else {
            g.nseg = 3;
            g.seg[0] = seg_of(Qb, d, 0, d, RowMap{n, q, -(n - q), 0, n - q});
            g.seg[1] = seg_of(pg ? nullptr : K(l), d, d, 2 * d, cache_map);
            g.seg[2] = seg_of(pg ? nullptr : V(l), d, 2 * d, 3 * d, cache_map);
        }
        if (pg) {
            seg_paged(g.seg[kv_only ? 0 : 1], c, pg, l, 0);
            seg_paged(g.seg[kv_only ? 1 : 2], c, pg, l, 1);
        }
        if ((r = gemm(m, g, st, ROLE_S_QKV)) != OT_OK) return r;
        if (kv_ready && cudaEventRecord(kv_ready[l], st) != cudaSuccess) return OT_ERR_CUDA;
        done = kv_only;
        return OT_OK;
    }

    // 2. attention over the tail, 3. O projection + residual, 4. FFN
    ot_status rest(int l)
    {
        if (done) return OT_OK;
        const ot_config &c = m->cfg;
        const int d = c.d, f = c.ffn, esz = m->esz, n = rows(l), q = tail(l);
        const bool fp8 = c.dtype == OT_DTYPE_FP8;
        const int wesz = fp8 ? 1 : esz;
        const bool last = l == c.layers - 1;
        const void *g2 = fp8 ? at(m->g2_s, static_cast<long long>(l) * d, esz) : nullptr;
        AttnArgs at_ = attn_base(c, 0, U, rows_at(c, l), q, Qb, pg ? nullptr : K(l), pg ? nullptr : V(l), Ab);
        attn_paged(at_, c, pg, l);
        at_.KN = ns_K;
        at_.VN = ns_V;
        at_.nkn = ns_rows;
        // FP8 with per-tensor scales: the attention writes e4m3 for the O
        // projection (not for the fused-FFN or mixture paths, bf16 only)
        const bool oq = fp8_fused_hidden(m) && !use_fused_ffn(m) && c.moe_experts == 0;
        if (oq) {
            at_.o_qscale = act_slot(m, l, 0, IN_O);
            at_.o_qstride = 4;
        }
        ot_status r;
        if ((r = attn(m, at_, st)) != OT_OK) return r;
        void *Xn = (last && s_out) ? s_out : Xb[l & 1];
        if (c.moe_experts > 0) {
            if ((r = moe_ffn(l, Xn)) != OT_OK) return r;
            X = Xn;
            return OT_OK;
        }
        if (use_fused_ffn(m)) {
            // 3 + 4 in one launch: O projection + residual from the tail rows
            // of the layer input, RMSNorm2, W1, GELU, W2, residual
            const FfnArgs fa = ffn_o_args(m, U * q, 1, Ab, rowmap_identity(),
                                          at(m->Wo_s, static_cast<long long>(l) * d * d, esz), X,
                                          RowMap{q, n, n - q, 0, 0},
                                          at(m->W1_s, static_cast<long long>(l) * f * d, esz),
                                          at(m->W2_s, static_cast<long long>(l) * d * f, esz), Xn,
                                          rowmap_identity());
            if ((r = ffn_run(m, fa, st, ROLE_S_FFN)) != OT_OK) return r;
            X = Xn;
            return OT_OK;
        }
        // 3. O projection + residual from the tail rows of the layer input
        GemmArgs g = gemm_base(c, U * q, d, d, 1);
        if (oq)
            fp8_hidden_operand(g, Ab, d, rowmap_identity(), at(m->Wo_s, static_cast<long long>(l) * d * d, wesz),
                               static_cast<long long>(d) * d, m->sc_o_s + l, act_slot(m, l, 0, IN_O));
        else if ((r = projection(m, g, Ab, d, rowmap_identity(),
                                 at(m->Wo_s, static_cast<long long>(l) * d * d, wesz),
                                 static_cast<long long>(d) * d, fp8 ? m->sc_o_s + l : nullptr, nullptr, 0,
                                 false, f8, st, l, 0, IN_O)) != OT_OK)
            return r;
        g.res = X;
        g.res_ld = d;
        g.res_map = RowMap{q, n, n - q, 0, 0};
        g.nseg = 1;
        g.seg[0] = seg_of(Hb, d, 0, d, rowmap_identity());
        if ((r = gemm(m, g, st, ROLE_S_O)) != OT_OK) return r;
        // 4. FFN: RMSNorm2 + W1 + GELU, then W2 + residual
        g = gemm_base(c, U * q, f, d, 1);
        if ((r = projection(m, g, Hb, d, rowmap_identity(),
                            at(m->W1_s, static_cast<long long>(l) * f * d, wesz),
                            static_cast<long long>(f) * d, fp8 ? m->sc_1_s + l : nullptr, g2, d, true,
                            f8, st, l, 0, IN_W1)) != OT_OK)
            return r;
        g.gelu = 1;
        g.nseg = 1;
        g.seg[0] = seg_of(hid, f, 0, f, rowmap_identity());
        const bool fh = fp8_fused_hidden(m);
        if (fh) {
            g.qscale = act_slot(m, l, 0, IN_W2);
            g.qscale_gstride = 4;
        }
        if ((r = gemm(m, g, st, ROLE_S_FFN1)) != OT_OK) return r;
        g = gemm_base(c, U * q, d, f, 1);
        if (fh)
            fp8_hidden_operand(g, hid, f, rowmap_identity(), at(m->W2_s, static_cast<long long>(l) * d * f, wesz),
                               static_cast<long long>(d) * f, m->sc_2_s + l, act_slot(m, l, 0, IN_W2));
        else if ((r = projection(m, g, hid, f, rowmap_identity(),
                                 at(m->W2_s, static_cast<long long>(l) * d * f, wesz),
                                 static_cast<long long>(d) * f, fp8 ? m->sc_2_s + l : nullptr, nullptr, 0,
                                 false, f8, st, l, 0, IN_W2)) != OT_OK)
            return r;
        g.res = Hb;
        g.res_ld = d;
        g.nseg = 1;
        g.seg[0] = seg_of(Xn, d, 0, d, rowmap_identity());
        if ((r = gemm(m, g, st, ROLE_S_FFN2)) != OT_OK) return r;
        X = Xn;
        return OT_OK;
    }

    // 3. O projection + residual into H, then the mixture of experts: route
    // every row to its top-k experts (rows copied expert-major), the experts'
    // FFN (Yp = h + FFN_e(n(h)) per slot), combine into Xn
    ot_status moe_ffn(int l, void *Xn)
    {
        const ot_config &c = m->cfg;
        const int d = c.d, f = c.ffn, esz = m->esz, n = rows(l), q = tail(l), E = c.moe_experts;
        const long long cap = static_cast<long long>(U) * q; // an expert takes at most every row
        GemmArgs g = gemm_base(c, U * q, d, d, 1);
        ot_status r;
        if ((r = projection(m, g, Ab, d, rowmap_identity(), at(m->Wo_s, static_cast<long long>(l) * d * d, esz),
                            static_cast<long long>(d) * d, nullptr, nullptr, 0, false, f8, st, l, 0, IN_O)) !=
            OT_OK)
            return r;
        g.res = X;
        g.res_ld = d;
        g.res_map = RowMap{q, n, n - q, 0, 0};
        g.nseg = 1;
        g.seg[0] = seg_of(Hb, d, 0, d, rowmap_identity());
        if ((r = gemm(m, g, st, ROLE_S_O)) != OT_OK) return r;
        if (cudaMemsetAsync(counts, 0, sizeof(int) * E, st) != cudaSuccess) return OT_ERR_CUDA;
        MoeRouteArgs ra;
        memset(&ra, 0, sizeof(ra));
        ra.rows = cap;
        ra.d = d;
        ra.E = E;
        ra.topk = c.moe_topk;
        ra.dtype = c.dtype;
        ra.eps = c.eps;
        ra.H = Hb;
        ra.gain = at(m->g2_s, static_cast<long long>(l) * d, esz);
        ra.Wr = at(m->W_router, static_cast<long long>(l) * E * d, esz);
        ra.Hp = Hp;
        ra.cap = cap;
        ra.counts = counts;
        ra.route = route;
        ra.gate = gate;
        const double rbytes = static_cast<double>(cap) * d * esz * (1 + c.moe_topk) +
                              static_cast<double>(E) * d * esz;
        if ((r = profiled(m, st, OT_KIND_MOE, ROLE_S_MOE, 2.0 * cap * d * E, rbytes,
                          [&] { return launch_moe_route(ra, st); })) != OT_OK)
            return r;
        const RowMap seg_rows{1, 1, 0, cap, 0}; // expert e, slot s -> row e * cap + s
        const char *W1e = at(m->W1_moe, static_cast<long long>(l) * E * f * d, esz);
        const char *W2e = at(m->W2_moe, static_cast<long long>(l) * E * d * f, esz);
        if (use_fused_ffn(m)) {
            // the experts' FFN in one launch: group = expert, only its filled rows
            FfnArgs fa = ffn_args(m, static_cast<int>(cap), E, Hp, seg_rows, W1e, W2e, Yp, seg_rows);
            fa.group_rows = counts;
            if ((r = ffn_run(m, fa, st, ROLE_S_FFN, static_cast<double>(cap) * c.moe_topk)) != OT_OK) return r;
        } else {
            // two grouped GEMMs over every slot of every expert
            g = gemm_base(c, static_cast<int>(cap), f, d, E);
            if ((r = projection(m, g, Hp, d, seg_rows, W1e, static_cast<long long>(f) * d, nullptr, nullptr, 0,
                                true, f8, st)) != OT_OK)
                return r;
            g.gelu = 1;
            g.nseg = 1;
            g.seg[0] = seg_of(ehid, f, 0, f, seg_rows);
            if ((r = gemm(m, g, st, ROLE_S_FFN1)) != OT_OK) return r;
            g = gemm_base(c, static_cast<int>(cap), d, f, E);
            if ((r = projection(m, g, ehid, f, seg_rows, W2e, static_cast<long long>(d) * f, nullptr, nullptr, 0,
                                false, f8, st)) != OT_OK)
                return r;
            g.res = Hp;
            g.res_ld = d;
            g.res_map = seg_rows;
            g.nseg = 1;
            g.seg[0] = seg_of(Yp, d, 0, d, seg_rows);
            if ((r = gemm(m, g, st, ROLE_S_FFN2)) != OT_OK) return r;
        }
        MoeCombineArgs ca;
        memset(&ca, 0, sizeof(ca));
        ca.rows = cap;
        ca.d = d;
        ca.topk = c.moe_topk;
        ca.dtype = c.dtype;
        ca.H = Hb;
        ca.Yp = Yp;
        ca.Y = Xn;
        ca.route = route;
        ca.gate = gate;
        const double cbytes = static_cast<double>(cap) * d * esz * (2 + c.moe_topk);
        return profiled(m, st, OT_KIND_MOE, ROLE_S_MOE, 0.0, cbytes, [&] { return launch_moe_combine(ca, st); });
    }
};

ot_status run_encode(ot_model *m, const void *X0, int U, void *kv, void *s_out, Ws ws,
                     cudaStream_t st, cudaEvent_t *kv_ready = nullptr, int delta = 0,
                     bool full_last = false, const PagedKv *pg = nullptr)
{
    EncodeRun e{m, U, kv, s_out, st, kv_ready, delta, full_last};
    e.pg = pg;
    ot_status r = e.init(X0, ws);
    for (int l = 0; r == OT_OK && l < m->cfg.layers && !e.done; ++l)
        if ((r = e.qkv(l)) == OT_OK) r = e.rest(l);
    return r;
}

// NS-side of every layer, one layer at a time (qkv(l), then rest(l)): U
// users x C candidates, N tokens each, against the S K/V in kv.  out may be
// null (calibration): the last layer then writes a workspace buffer.
struct ScoreRun {
    ot_model *m;
    const void *kv;
    int U, C;
    void *out;
    cudaStream_t st;
    cudaEvent_t *kv_ready;
    const PagedKv *pg = nullptr; // the cache is paged (kv unused)
    void *Xb[2], *Qn, *Kn, *Vn, *An, *Hn, *hid;
    Fp8Scratch f8{nullptr, nullptr};
    const void *X;

    ot_status init(const void *ns, Ws ws)
    {
        const ot_config &c = m->cfg;
        const long long R = static_cast<long long>(U) * C * c.n_ns;
        Xb[0] = ws.take(R * c.d);
        Xb[1] = ws.take(R * c.d);
        Qn = ws.take(R * c.d);
        Kn = ws.take(R * c.d);
        Vn = ws.take(R * c.d);
        An = ws.take(R * c.d);
        Hn = ws.take(R * c.d);
        hid = ws.take(R * c.ffn);
        if (!Xb[0] || !Xb[1] || !Qn || !Kn || !Vn || !An || !Hn || !hid)
            return OT_ERR_WORKSPACE_TOO_SMALL;
        if (c.dtype == OT_DTYPE_FP8) {
            Ws w1{ws.p, ws.left, 1};
            f8.q = static_cast<uint8_t *>(w1.take(R * (c.d > c.ffn ? c.d : c.ffn)));
            Ws w4{w1.p, w1.left, 4};
            f8.s = static_cast<float *>(w4.take(R));
            if (!f8.q || !f8.s) return OT_ERR_WORKSPACE_TOO_SMALL;
        }
        X = ns;
        return OT_OK;
    }
    RowMap grp() const { return RowMap{1, m->cfg.n_ns, 0, 1, 0}; } // candidate m, position g -> row m*N + g

    ot_status qkv(int l)
    {
        const ot_config &c = m->cfg;
        const int d = c.d, N = c.n_ns, esz = m->esz;
        const bool fp8 = c.dtype == OT_DTYPE_FP8;
        const int wesz = fp8 ? 1 : esz;
        const long long lN = static_cast<long long>(l) * N;
        if (kv_ready && cudaStreamWaitEvent(st, kv_ready[l], 0) != cudaSuccess) return OT_ERR_CUDA;
        const void *g1 = fp8 ? at(m->g1_ns, lN * d, esz) : nullptr;
        GemmArgs g = gemm_base(c, U * C, 3 * d, d, N);
        ot_status r;
        if ((r = projection(m, g, X, d, grp(), at(m->Wqkv_ns, lN * 3 * d * d, wesz), 3LL * d * d,
                            fp8 ? m->sc_qkv_ns + lN : nullptr, g1, d, true, f8, st, l, 1, IN_QKV)) != OT_OK)
            return r;
        g.nseg = 3;
        g.seg[0] = seg_of(Qn, d, 0, d, grp());
        g.seg[1] = seg_of(Kn, d, d, 2 * d, grp());
        g.seg[2] = seg_of(Vn, d, 2 * d, 3 * d, grp());
        return gemm(m, g, st, ROLE_NS_QKV);
    }

    ot_status rest(int l)
    {
        const ot_config &c = m->cfg;
        const int d = c.d, f = c.ffn, N = c.n_ns, esz = m->esz, Mc = U * C, L = rows_at(c, l);
        const bool fp8 = c.dtype == OT_DTYPE_FP8;
        const int wesz = fp8 ? 1 : esz;
        const bool last = l == c.layers - 1;
        const long long lN = static_cast<long long>(l) * N;
        const void *g2 = fp8 ? at(m->g2_ns, lN * d, esz) : nullptr;
        const char *K = pg ? nullptr : at(kv, kv_layer_off(c, l), esz);
        const char *V = pg ? nullptr : K + static_cast<long long>(L) * d * esz;
        AttnArgs at_ = attn_base(c, 1, U, L, C * N, Qn, K, V, An);
        attn_paged(at_, c, pg, l);
        at_.KN = Kn;
        at_.VN = Vn;
        at_.nkn = C * N;
        const bool oq = fp8_fused_hidden(m) && !use_fused_ffn(m); // e4m3 attention output for the O projection
        if (oq) {
            at_.o_qscale = act_slot(m, l, 1, IN_O); // NS position n: parameter set 1 + n
            at_.o_qstride = 4;
        }
        ot_status r;
        if ((r = attn(m, at_, st)) != OT_OK) return r;
        void *Xn = last && out ? out : Xb[l & 1];
        const RowMap gm = grp();
        if (use_fused_ffn(m)) {
            // O projection + residual and the FFN in one grouped launch
            const FfnArgs fa = ffn_o_args(m, Mc, N, An, gm, at(m->Wo_ns, lN * d * d, esz), X, gm,
                                          at(m->W1_ns, lN * f * d, esz), at(m->W2_ns, lN * d * f, esz), Xn, gm);
            if ((r = ffn_run(m, fa, st, ROLE_NS_FFN)) != OT_OK) return r;
            X = Xn;
            return OT_OK;
        }
        GemmArgs g = gemm_base(c, Mc, d, d, N);
        if (oq)
            fp8_hidden_operand(g, An, d, gm, at(m->Wo_ns, lN * d * d, wesz), static_cast<long long>(d) * d,
                               m->sc_o_ns + lN, act_slot(m, l, 1, IN_O));
        else if ((r = projection(m, g, An, d, gm, at(m->Wo_ns, lN * d * d, wesz),
                                 static_cast<long long>(d) * d, fp8 ? m->sc_o_ns + lN : nullptr, nullptr,
                                 0, false, f8, st, l, 1, IN_O)) != OT_OK)
            return r;
        g.res = X;
        g.res_ld = d;
        g.res_map = gm;
        g.nseg = 1;
        g.seg[0] = seg_of(Hn, d, 0, d, gm);
        if ((r = gemm(m, g, st, ROLE_NS_O)) != OT_OK) return r;
        g = gemm_base(c, Mc, f, d, N);
        if ((r = projection(m, g, Hn, d, gm, at(m->W1_ns, lN * f * d, wesz),
                            static_cast<long long>(f) * d, fp8 ? m->sc_1_ns + lN : nullptr, g2, d,
                            true, f8, st, l, 1, IN_W1)) != OT_OK)
            return r;
        g.gelu = 1;
        g.nseg = 1;
        g.seg[0] = seg_of(hid, f, 0, f, gm);
        const bool fh = fp8_fused_hidden(m);
        if (fh) {
            g.qscale = act_slot(m, l, 1, IN_W2); // group g: parameter set 1 + g
            g.qscale_gstride = 4;
        }
        if ((r = gemm(m, g, st, ROLE_NS_FFN1)) != OT_OK) return r;
        g = gemm_base(c, Mc, d, f, N);
        if (fh)
            fp8_hidden_operand(g, hid, f, gm, at(m->W2_ns, lN * d * f, wesz), static_cast<long long>(d) * f,
                               m->sc_2_ns + lN, act_slot(m, l, 1, IN_W2));
        else if ((r = projection(m, g, hid, f, gm, at(m->W2_ns, lN * d * f, wesz),
                                 static_cast<long long>(d) * f, fp8 ? m->sc_2_ns + lN : nullptr, nullptr,
                                 0, false, f8, st, l, 1, IN_W2)) != OT_OK)
            return r;
        g.res = Hn;
        g.res_ld = d;
        g.res_map = gm;
        g.nseg = 1;
        g.seg[0] = seg_of(Xn, d, 0, d, gm);
        if ((r = gemm(m, g, st, ROLE_NS_FFN2)) != OT_OK) return r;
        X = Xn;
        return OT_OK;
    }
};

ot_status run_score(ot_model *m, const void *kv, int U, const void *ns, int C, void *out, Ws ws,
                    cudaStream_t st, cudaEvent_t *kv_ready = nullptr, const PagedKv *pg = nullptr)
{
    ScoreRun sc{m, kv, U, C, out, st, kv_ready};
    sc.pg = pg;
    ot_status r = sc.init(ns, ws);
    for (int l = 0; r == OT_OK && l < m->cfg.layers; ++l)
        if ((r = sc.qkv(l)) == OT_OK) r = sc.rest(l);
    return r;
}

// Full attention (one candidate per user): the S rows of layer l also see
// the layer's NS keys, so both sides' projections run before either side's
// attention, layer by layer, on one stream.
ot_status run_full_joint(ot_model *m, const void *X0, int U, const void *ns, void *kv, void *s_out,
                         void *out, Ws ws_enc, Ws ws_sc, cudaStream_t st)
{
    EncodeRun e{m, U, kv, s_out, st, nullptr, 0, true};
    ScoreRun sc{m, kv, U, 1, out, st, nullptr};
    ot_status r = e.init(X0, ws_enc);
    if (r == OT_OK) r = sc.init(ns, ws_sc);
    e.ns_K = sc.Kn;
    e.ns_V = sc.Vn;
    e.ns_rows = m->cfg.n_ns;
    for (int l = 0; r == OT_OK && l < m->cfg.layers; ++l) {
        if ((r = e.qkv(l)) != OT_OK || (r = sc.qkv(l)) != OT_OK || (r = e.rest(l)) != OT_OK) break;
        r = sc.rest(l);
    }
    return r;
}

// The S and NS sides can share launches: bf16 tensor-core path with the
// fused FFN and head_dim 64 attention.
bool merged_supported(const ot_model *m)
{
    return use_fused_ffn(m) && m->cfg.d / m->cfg.heads == 64 && m->cfg.moe_experts == 0;
}

// Full forward with the S and NS sides sharing the QKV, O-projection and FFN
// launches of each layer: the NS work units come after the S ones and fill
// the S launches' last partial waves (at small C a whole NS step costs
// almost nothing there).  The NS attention of layer l runs on the side
// stream once the layer's QKV launch is done, beside the S attention; the
// merged O launch waits for it.  Same arithmetic, buffers and workspace
// layouts as run_encode + run_score.
ot_status run_full_merged(ot_model *m, const void *X0, int U, const void *ns, int C, void *kv,
                          void *s_out, void *out, Ws ws_enc, Ws ws_sc, cudaStream_t st)
{
    const ot_config &c = m->cfg;
    const int d = c.d, f = c.ffn, N = c.n_ns;
    // S-side buffers (as run_encode)
    const long long rows0 = static_cast<long long>(U) * c.L0;
    void *Xb[2] = {ws_enc.take(rows0 * d), ws_enc.take(rows0 * d)};
    void *Qb = ws_enc.take(rows0 * d), *Ab = ws_enc.take(rows0 * d), *Hb = ws_enc.take(rows0 * d);
    if (!Xb[0] || !Xb[1] || !Qb || !Ab || !Hb) return OT_ERR_WORKSPACE_TOO_SMALL;
    // NS-side buffers (as run_score)
    const int Mc = U * C;
    const long long R = static_cast<long long>(Mc) * N;
    void *Yb[2] = {ws_sc.take(R * d), ws_sc.take(R * d)};
    void *Qn = ws_sc.take(R * d), *Kn = ws_sc.take(R * d), *Vn = ws_sc.take(R * d);
    void *An = ws_sc.take(R * d), *Hn = ws_sc.take(R * d);
    if (!Yb[0] || !Yb[1] || !Qn || !Kn || !Vn || !An || !Hn) return OT_ERR_WORKSPACE_TOO_SMALL;
    const long long ustride = kv_user_elems(c);
    const RowMap grp{1, N, 0, 1, 0}; // candidate m, position g -> row m*N + g
    const Fp8Scratch no_f8{nullptr, nullptr};
    // per-launch profiling times each kernel alone: everything on one stream
    cudaStream_t side = m->profiling ? st : m->side;
    const bool two = side != st;
    const void *X = X0, *Y = ns;
    ot_status r;
    for (int l = 0; l < c.layers; ++l) {
        const int L = rows_at(c, l), q = c.q[l];
        const bool last = l == c.layers - 1;
        char *K = at(kv, kv_layer_off(c, l), m->esz);
        char *V = K + static_cast<long long>(L) * d * m->esz;
        const RowMap cache_map{L, ustride / d, 0, 0, 0};
        const long long lN = static_cast<long long>(l) * N;
        // 1. QKV: S rows (K / V into the cache, Q of the tail rows) and NS rows
        GemmArgs gs = gemm_base(c, U * L, 3 * d, d, 1);
        if ((r = projection(m, gs, X, d, rowmap_identity(),
                            at(m->Wqkv_s, static_cast<long long>(l) * 3 * d * d, m->esz), 3LL * d * d, nullptr,
                            nullptr, d, true, no_f8, st)) != OT_OK)
            return r;
        gs.nseg = 3;
        gs.seg[0] = seg_of(Qb, d, 0, d, RowMap{L, q, -(L - q), 0, L - q});
        gs.seg[1] = seg_of(K, d, d, 2 * d, cache_map);
        gs.seg[2] = seg_of(V, d, 2 * d, 3 * d, cache_map);
        // NS rows of the same layer, in the same launch
        GemmArgs gn = gemm_base(c, Mc, 3 * d, d, N);
        if ((r = projection(m, gn, Y, d, grp, at(m->Wqkv_ns, lN * 3 * d * d, m->esz), 3LL * d * d, nullptr,
                            nullptr, d, true, no_f8, st)) != OT_OK)
            return r;
        gn.nseg = 3;
        gn.seg[0] = seg_of(Qn, d, 0, d, grp);
        gn.seg[1] = seg_of(Kn, d, d, 2 * d, grp);
        gn.seg[2] = seg_of(Vn, d, 2 * d, 3 * d, grp);
        if ((r = gemm2(m, &gs, &gn, st, ROLE_QKV)) != OT_OK) return r;
        // 2. NS attention (side stream) needs this layer's S K/V and NS Q/K/V
        if (two && (cudaEventRecord(m->kv_ready[l], st) != cudaSuccess ||
                    cudaStreamWaitEvent(side, m->kv_ready[l], 0) != cudaSuccess))
            return OT_ERR_CUDA;
        AttnArgs as_ = attn_base(c, 0, U, L, q, Qb, K, V, Ab);
        if (c.full_attn) { // the S rows also see the layer's NS keys (one candidate per user)
            as_.KN = Kn;
            as_.VN = Vn;
            as_.nkn = C * N;
        }
        AttnArgs an_ = attn_base(c, 1, U, L, C * N, Qn, K, V, An);
        an_.KN = Kn;
        an_.VN = Vn;
        if ((r = attn(m, an_, side)) != OT_OK) return r;
        if (two && cudaEventRecord(m->ns_attn_done[l], side) != cudaSuccess) return OT_ERR_CUDA;
        // 3. S attention (main stream)
        if ((r = attn(m, as_, st)) != OT_OK) return r;
        if (two && cudaStreamWaitEvent(st, m->ns_attn_done[l], 0) != cudaSuccess) return OT_ERR_CUDA;
        // 4. O projection + residual, RMSNorm, W1, GELU, W2, residual: both
        // sides in one launch
        void *Xn = (last && s_out) ? s_out : Xb[l & 1];
        void *Yn = last ? out : Yb[l & 1];
        FfnArgs fs = ffn_o_args(m, U * q, 1, Ab, rowmap_identity(),
                                at(m->Wo_s, static_cast<long long>(l) * d * d, m->esz), X, RowMap{q, L, L - q, 0, 0},
                                at(m->W1_s, static_cast<long long>(l) * f * d, m->esz),
                                at(m->W2_s, static_cast<long long>(l) * d * f, m->esz), Xn, rowmap_identity());
        FfnArgs fn = ffn_o_args(m, Mc, N, An, grp, at(m->Wo_ns, lN * d * d, m->esz), Y, grp,
                                at(m->W1_ns, lN * f * d, m->esz), at(m->W2_ns, lN * d * f, m->esz), Yn, grp);
        if ((r = ffn2(m, &fs, &fn, st)) != OT_OK) return r;
        X = Xn;
        Y = Yn;
    }
    return OT_OK;
}

ot_status device_copy(ot_model *m, void **dst, const void *src, size_t bytes)
{
    if (cudaMalloc(dst, bytes) != cudaSuccess) return OT_ERR_CUDA;
    m->allocs.push_back(*dst);
    if (cudaMemcpy(*dst, src, bytes, cudaMemcpyDeviceToDevice) != cudaSuccess) return OT_ERR_CUDA;
    return OT_OK;
}

ot_status device_fold(ot_model *m, void **dst, const void *W, const void *gain, long long rows,
                      int cols, long long groups)
{
    size_t bytes = static_cast<size_t>(groups * rows * cols) * m->esz;
    if (cudaMalloc(dst, bytes) != cudaSuccess) return OT_ERR_CUDA;
    m->allocs.push_back(*dst);
    if (launch_fold_gain(W, gain, *dst, rows, cols, groups, cols, m->cfg.dtype == OT_DTYPE_F32
                                                                      ? OT_DTYPE_F32
                                                                      : OT_DTYPE_BF16,
                         0) != cudaSuccess)
        return OT_ERR_CUDA;
    return OT_OK;
}

ot_status device_quant(ot_model *m, void **dst, float **scales, const void *W, long long per_mat,
                       long long mats)
{
    if (cudaMalloc(dst, static_cast<size_t>(per_mat * mats)) != cudaSuccess) return OT_ERR_CUDA;
    m->allocs.push_back(*dst);
    if (cudaMalloc(reinterpret_cast<void **>(scales), sizeof(float) * mats) != cudaSuccess)
        return OT_ERR_CUDA;
    m->allocs.push_back(*scales);
    if (launch_quant_weights(W, per_mat, mats, static_cast<uint8_t *>(*dst), *scales, nullptr, 0) !=
        cudaSuccess)
        return OT_ERR_CUDA;
    return OT_OK;
}

} // namespace

namespace ot {
ot_status internal_check_config(const ot_config &c) { return check_config(c); }

size_t internal_score_ws_bytes(const ot_model *m, int users, int cands)
{
    if (!m || users < 1 || cands < 1) return 0;
    return score_ws_bytes(m->cfg, users, cands, m->esz);
}
} // namespace ot

extern "C" {

const char *ot_status_str(ot_status s)
{
    switch (s) {
    case OT_OK: return "ok";
    case OT_ERR_ARG: return "invalid argument";
    case OT_ERR_SHAPE: return "unsupported shape";
    case OT_ERR_DTYPE: return "unsupported dtype";
    case OT_ERR_ALIGN: return "pointer not 16-byte aligned";
    case OT_ERR_CACHE_TOO_SMALL: return "kv cache too small";
    case OT_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case OT_ERR_CUDA: return "CUDA error";
    case OT_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case OT_ERR_DEVICE_BOUNDS: return "device index out of bounds";
    case OT_ERR_UNSUPPORTED: return "unsupported";
    }
    return "unknown status";
}

ot_status ot_model_create(const ot_config *cfg, const ot_weights *w, ot_model **out)
{
    if (!cfg || !w || !out) return OT_ERR_ARG;
    *out = nullptr;
    ot_status r = check_config(*cfg);
    if (r != OT_OK) return r;
    const bool moe = cfg->moe_experts > 0;
    // a mixture of experts replaces the dense S-side FFN weights
    const void *need[] = {w->Wqkv_s, w->Wo_s, moe ? w->W_router : w->W1_s, moe ? w->W1_moe : w->W2_s,
                          w->g1_s, w->g2_s, w->Wqkv_ns, w->Wo_ns, w->W1_ns, w->W2_ns, w->g1_ns, w->g2_ns,
                          moe ? w->W2_moe : w->Wqkv_s};
    for (const void *p : need) {
        if (!p) return OT_ERR_ARG;
        if (!aligned16(p)) return OT_ERR_ALIGN;
    }
    if (cfg->F > 0 && !w->W_split) return OT_ERR_ARG;
    ot_model *m = new (std::nothrow) ot_model();
    if (!m) return OT_ERR_CUDA;
    m->cfg = *cfg;
    m->esz = cfg->dtype == OT_DTYPE_F32 ? 4 : 2;
    m->path = 0;
    m->wait_limit = 1LL << 26;
    m->launches = 0;
    cudaGetDevice(&m->device);
    const long long L = cfg->layers, d = cfg->d, f = cfg->ffn, N = cfg->n_ns;
    const int esz = m->esz;
    r = OT_OK;
    do {
        if (cudaMalloc(reinterpret_cast<void **>(&m->err), sizeof(int)) != cudaSuccess) {
            r = OT_ERR_CUDA;
            break;
        }
        m->allocs.push_back(m->err);
        if (cudaMemset(m->err, 0, sizeof(int)) != cudaSuccess) { r = OT_ERR_CUDA; break; }
        if (cudaStreamCreateWithFlags(&m->side, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&m->copy_stream, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&m->fork_ev, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&m->join_ev, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&m->in_ready[0], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&m->in_ready[1], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&m->in_free[0], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&m->in_free[1], cudaEventDisableTiming) != cudaSuccess) {
            r = OT_ERR_CUDA;
            break;
        }
        for (int l = 0; l < cfg->layers && r == OT_OK; ++l)
            if (cudaEventCreateWithFlags(&m->kv_ready[l], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&m->ns_attn_done[l], cudaEventDisableTiming) != cudaSuccess)
                r = OT_ERR_CUDA;
        if (r != OT_OK) break;
        if (cfg->dtype == OT_DTYPE_FP8) {
            // e4m3 weights, one scale per matrix; gains stay separate (bf16)
            if ((r = device_quant(m, &m->Wqkv_s, &m->sc_qkv_s, w->Wqkv_s, 3 * d * d, L)) != OT_OK) break;
            if ((r = device_quant(m, &m->Wo_s, &m->sc_o_s, w->Wo_s, d * d, L)) != OT_OK) break;
            if ((r = device_quant(m, &m->W1_s, &m->sc_1_s, w->W1_s, f * d, L)) != OT_OK) break;
            if ((r = device_quant(m, &m->W2_s, &m->sc_2_s, w->W2_s, d * f, L)) != OT_OK) break;
            if ((r = device_quant(m, &m->Wqkv_ns, &m->sc_qkv_ns, w->Wqkv_ns, 3 * d * d, L * N)) != OT_OK)
                break;
            if ((r = device_quant(m, &m->Wo_ns, &m->sc_o_ns, w->Wo_ns, d * d, L * N)) != OT_OK) break;
            if ((r = device_quant(m, &m->W1_ns, &m->sc_1_ns, w->W1_ns, f * d, L * N)) != OT_OK) break;
            if ((r = device_quant(m, &m->W2_ns, &m->sc_2_ns, w->W2_ns, d * f, L * N)) != OT_OK) break;
            if ((r = device_copy(m, &m->g1_s, w->g1_s, L * d * esz)) != OT_OK) break;
            if ((r = device_copy(m, &m->g2_s, w->g2_s, L * d * esz)) != OT_OK) break;
            if ((r = device_copy(m, &m->g1_ns, w->g1_ns, L * N * d * esz)) != OT_OK) break;
            if ((r = device_copy(m, &m->g2_ns, w->g2_ns, L * N * d * esz)) != OT_OK) break;
            if (cfg->F > 0 &&
                (r = device_copy(m, &m->W_split, w->W_split, N * d * cfg->F * esz)) != OT_OK)
                break;
            if (cudaDeviceSynchronize() != cudaSuccess) { r = OT_ERR_CUDA; break; }
            break;
        }
        // gains folded into the projection that follows each norm
        if ((r = device_fold(m, &m->Wqkv_s, w->Wqkv_s, w->g1_s, 3 * d, d, L)) != OT_OK) break;
        if (moe) {
            // experts: g2 folded into every expert's W1 (one gain per layer);
            // the router reads the gain itself, so g2 is kept as well
            const long long E = cfg->moe_experts;
            const size_t w1b = static_cast<size_t>(L * E * f * d) * esz;
            if (cudaMalloc(&m->W1_moe, w1b) != cudaSuccess) { r = OT_ERR_CUDA; break; }
            m->allocs.push_back(m->W1_moe);
            for (long long l = 0; l < L && r == OT_OK; ++l)
                if (launch_fold_gain(at(w->W1_moe, l * E * f * d, esz), at(w->g2_s, l * d, esz),
                                     at(m->W1_moe, l * E * f * d, esz), f, static_cast<int>(d), E, 0,
                                     cfg->dtype == OT_DTYPE_F32 ? OT_DTYPE_F32 : OT_DTYPE_BF16,
                                     0) != cudaSuccess)
                    r = OT_ERR_CUDA;
            if (r != OT_OK) break;
            if ((r = device_copy(m, &m->W2_moe, w->W2_moe, L * E * d * f * esz)) != OT_OK) break;
            if ((r = device_copy(m, &m->W_router, w->W_router, L * E * d * esz)) != OT_OK) break;
            if ((r = device_copy(m, &m->g2_s, w->g2_s, L * d * esz)) != OT_OK) break;
        } else if ((r = device_fold(m, &m->W1_s, w->W1_s, w->g2_s, f, d, L)) != OT_OK) {
            break;
        }
        if ((r = device_fold(m, &m->Wqkv_ns, w->Wqkv_ns, w->g1_ns, 3 * d, d, L * N)) != OT_OK)
            break;
        if ((r = device_fold(m, &m->W1_ns, w->W1_ns, w->g2_ns, f, d, L * N)) != OT_OK) break;
        if ((r = device_copy(m, &m->Wo_s, w->Wo_s, L * d * d * esz)) != OT_OK) break;
        if (!moe && (r = device_copy(m, &m->W2_s, w->W2_s, L * d * f * esz)) != OT_OK) break;
        if ((r = device_copy(m, &m->Wo_ns, w->Wo_ns, L * N * d * d * esz)) != OT_OK) break;
        if ((r = device_copy(m, &m->W2_ns, w->W2_ns, L * N * d * f * esz)) != OT_OK) break;
        if (cfg->F > 0 &&
            (r = device_copy(m, &m->W_split, w->W_split, N * d * cfg->F * esz)) != OT_OK)
            break;
        if (cudaDeviceSynchronize() != cudaSuccess) { r = OT_ERR_CUDA; break; }
    } while (0);
    if (r != OT_OK) {
        ot_model_destroy(m);
        return r;
    }
    *out = m;
    return OT_OK;
}

void ot_model_destroy(ot_model *m)
{
    if (!m) return;
    cudaDeviceSynchronize();
    for (void *p : m->allocs) cudaFree(p);
    for (auto &r : m->recs) {
        cudaEventDestroy(r.e0);
        cudaEventDestroy(r.e1);
    }
    for (cudaEvent_t e : m->event_pool) cudaEventDestroy(e);
    for (int l = 0; l < m->cfg.layers && l < OT_MAX_LAYERS; ++l) {
        if (m->kv_ready[l]) cudaEventDestroy(m->kv_ready[l]);
        if (m->ns_attn_done[l]) cudaEventDestroy(m->ns_attn_done[l]);
    }
    if (m->fork_ev) cudaEventDestroy(m->fork_ev);
    if (m->join_ev) cudaEventDestroy(m->join_ev);
    for (int i = 0; i < 2; ++i) {
        if (m->in_ready[i]) cudaEventDestroy(m->in_ready[i]);
        if (m->in_free[i]) cudaEventDestroy(m->in_free[i]);
    }
    if (m->copy_stream) cudaStreamDestroy(m->copy_stream);
    if (m->side) cudaStreamDestroy(m->side);
    delete m;
}

ot_status ot_profile_enable(ot_model *m, int enable)
{
    if (!m) return OT_ERR_ARG;
    m->profiling = enable != 0;
    return OT_OK;
}

int ot_profile_read(ot_model *m, ot_launch_record *out, int max)
{
    if (!m || (!out && max > 0) || max < 0) return -OT_ERR_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return -OT_ERR_CUDA;
    int n = 0;
    for (auto &r : m->recs) {
        if (n < max) {
            float ms = 0.f;
            cudaEventElapsedTime(&ms, r.e0, r.e1);
            out[n] = ot_launch_record{r.kind, r.role, ms, r.flops, r.bytes};
            ++n;
        }
        m->event_pool.push_back(r.e0);
        m->event_pool.push_back(r.e1);
    }
    m->recs.clear();
    return n;
}

size_t ot_kv_cache_bytes(const ot_model *m, int users)
{
    if (!m || users < 0) return 0;
    return static_cast<size_t>(users) * kv_user_elems(m->cfg) * m->esz;
}

size_t ot_workspace_bytes(const ot_model *m, int users, int cands)
{
    if (!m || users < 0 || cands < 0) return 0;
    size_t enc = encode_ws_bytes(m->cfg, users, m->esz);
    if (cands == 0) return enc;
    size_t sc = score_ws_bytes(m->cfg, users, cands, m->esz);
    size_t kv = bytes_of(static_cast<long long>(users) * kv_user_elems(m->cfg), m->esz);
    return enc + sc + kv; // S and NS sides run concurrently in ot_full_forward
}

ot_status ot_set_wait_limit(ot_model *m, long long polls)
{
    if (!m || polls < 1) return OT_ERR_ARG;
    m->wait_limit = polls;
    return OT_OK;
}

ot_status ot_set_kernel_path(ot_model *m, int path)
{
    if (!m || path < 0 || path > 2) return OT_ERR_ARG;
    if (path == 1 && m->cfg.dtype == OT_DTYPE_FP8) return OT_ERR_UNSUPPORTED;
    m->path = path;
    return OT_OK;
}

long long ot_launch_count(const ot_model *m) { return m ? m->launches : -1; }

ot_status ot_set_act_scales(ot_model *m, const float *scales)
{
    if (!m) return OT_ERR_ARG;
    if (m->cfg.dtype != OT_DTYPE_FP8) return OT_ERR_DTYPE;
    const long long n = static_cast<long long>(m->cfg.layers) * (1 + m->cfg.n_ns) * 4;
    if (!scales) {
        m->act_scale = nullptr; // back to per-row scales (the array stays allocated)
        return OT_OK;
    }
    for (long long i = 0; i < n; ++i)
        if (!(scales[i] > 0.f) || !(scales[i] < 3.0e38f)) return OT_ERR_ARG;
    std::lock_guard<std::recursive_mutex> lock(m->enqueue_mu);
    if (!m->act_scale_mem) {
        if (cudaMalloc(reinterpret_cast<void **>(&m->act_scale_mem), sizeof(float) * n) != cudaSuccess)
            return OT_ERR_CUDA;
        m->allocs.push_back(m->act_scale_mem);
    }
    // synchronous: no call enqueued before this one still reads the old scales
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(m->act_scale_mem, scales, sizeof(float) * n, cudaMemcpyHostToDevice) != cudaSuccess)
        return OT_ERR_CUDA;
    m->act_scale = m->act_scale_mem;
    return OT_OK;
}

ot_status ot_fp8_calibrate(ot_model *m, const void *S, const void *ns, int U, int C, float *amax,
                           void *ws, size_t ws_bytes, void *stream)
{
    if (!m || !S || !ns || !amax || !ws || U < 1 || C < 1) return OT_ERR_ARG;
    if (m->cfg.dtype != OT_DTYPE_FP8) return OT_ERR_DTYPE;
    if (m->cfg.full_attn) return OT_ERR_UNSUPPORTED;
    if (!aligned16(S) || !aligned16(ns) || !aligned16(ws) || (reinterpret_cast<uintptr_t>(amax) & 3))
        return OT_ERR_ALIGN;
    if (static_cast<long long>(U) * m->cfg.L0 > (1LL << 31) - 1 ||
        static_cast<long long>(U) * C * m->cfg.n_ns > (1LL << 31) - 1)
        return OT_ERR_SHAPE;
    if (ws_bytes < ot_workspace_bytes(m, U, C)) return OT_ERR_WORKSPACE_TOO_SMALL;
    const ot_config &c = m->cfg;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Ws w{static_cast<char *>(ws), ws_bytes, m->esz};
    void *kv = w.take(static_cast<long long>(U) * kv_user_elems(c));
    if (!kv) return OT_ERR_WORKSPACE_TOO_SMALL;
    std::lock_guard<std::recursive_mutex> lock(m->enqueue_mu);
    m->calib_amax = amax;
    // every layer in full, S side then NS side against the cache just written
    ot_status r = run_encode(m, S, U, kv, nullptr, w, st, nullptr, 0, true);
    if (r == OT_OK) r = run_score(m, kv, U, ns, C, nullptr, w, st);
    m->calib_amax = nullptr;
    return r;
}

ot_status ot_poll_device_error(ot_model *m, void *stream)
{
    if (!m) return OT_ERR_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return OT_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, m->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return OT_ERR_CUDA;
    if (h != 0 && cudaMemset(m->err, 0, sizeof(int)) != cudaSuccess) return OT_ERR_CUDA;
    return static_cast<ot_status>(h);
}

ot_status ot_auto_split(ot_model *m, const void *x, long M, void *ns, void *stream)
{
    if (!m || !x || !ns || M < 1) return OT_ERR_ARG;
    if (m->cfg.F <= 0) return OT_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(ns)) return OT_ERR_ALIGN;
    if (M > (1L << 30)) return OT_ERR_SHAPE;
    const ot_config &c = m->cfg;
    const int Nd = c.n_ns * c.d;
    GemmArgs g = gemm_base(c, static_cast<int>(M), Nd, c.F, 1);
    g.A = x;
    g.lda = c.F;
    g.B = m->W_split;
    g.b_gstride = static_cast<long long>(Nd) * c.F;
    g.nseg = 1;
    RegionScope rs{{ns, ns_bytes(m, M)}};
    g.seg[0] = seg_of(ns, Nd, 0, Nd, rowmap_identity());
    return gemm(m, g, static_cast<cudaStream_t>(stream), ROLE_AUTO_SPLIT);
}

ot_status ot_embed_gather(const void *table, long rows, int d, const int64_t *ids, long n,
                          void *out, int32_t *err_word, void *stream)
{
    if (!table || !ids || !out || rows < 1 || d < 8 || n < 0) return OT_ERR_ARG;
    if (d % 8) return OT_ERR_SHAPE;
    if (!aligned16(table) || !aligned16(out) || (reinterpret_cast<uintptr_t>(ids) & 7))
        return OT_ERR_ALIGN;
    cudaError_t e = launch_embed_gather(table, rows, d, ids, n, out, err_word,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? OT_OK : OT_ERR_CUDA;
}

ot_status ot_encode_user(ot_model *m, const void *S, int U, void *kv_cache, void *out_s_tail,
                         void *ws, size_t ws_bytes, void *stream)
{
    if (!m || !S || !kv_cache || !ws || U < 1) return OT_ERR_ARG;
    if (m->cfg.full_attn) return OT_ERR_UNSUPPORTED; // S rows depend on the candidate
    if (!aligned16(S) || !aligned16(kv_cache) || !aligned16(ws) ||
        (out_s_tail && !aligned16(out_s_tail)))
        return OT_ERR_ALIGN;
    if (static_cast<long long>(U) * m->cfg.L0 > (1LL << 31) - 1) return OT_ERR_SHAPE;
    if (ws_bytes < ot_workspace_bytes(m, U, 0)) return OT_ERR_WORKSPACE_TOO_SMALL;
    Ws w{static_cast<char *>(ws), ws_bytes, m->esz};
    RegionScope rs{{ws, ws_bytes}, {kv_cache, kv_bytes(m, U)}, {out_s_tail, tail_bytes(m, U)}};
    return run_encode(m, S, U, kv_cache, out_s_tail, w, static_cast<cudaStream_t>(stream));
}

size_t ot_append_workspace_bytes(const ot_model *m, int users, int delta)
{
    if (!m || users < 0 || delta < 0) return 0;
    const long long rows = static_cast<long long>(users) * delta;
    const ot_config &c = m->cfg;
    return 5 * bytes_of(rows * c.d, m->esz) + bytes_of(rows * c.ffn, m->esz) + fp8_ws_bytes(c, rows) +
           moe_ws_bytes(c, rows, m->esz);
}

ot_status ot_encode_append(ot_model *m, const void *kv_old, int U, const void *S_new, int delta,
                           void *kv_new, void *out_new, void *ws, size_t ws_bytes, void *stream)
{
    if (!m || !kv_old || !S_new || !kv_new || !out_new || !ws || U < 1 || delta < 1) return OT_ERR_ARG;
    if (m->cfg.full_attn) return OT_ERR_UNSUPPORTED;
    if (!aligned16(kv_old) || !aligned16(S_new) || !aligned16(kv_new) || !aligned16(out_new) ||
        !aligned16(ws))
        return OT_ERR_ALIGN;
    const ot_config &c = m->cfg; // the grown sequences
    // the configuration the old cache was written with: every window shorter by delta
    ot_config o = c;
    o.L0 -= delta;
    for (int l = 0; l < c.layers; ++l) o.q[l] -= delta;
    if (o.L0 < 1 || o.q[c.layers - 1] < 1) return OT_ERR_SHAPE;
    if ((static_cast<long long>(c.d) * m->esz) % 16) return OT_ERR_SHAPE;
    if (U > 65535 || static_cast<long long>(U) * c.L0 > (1LL << 31) - 1) return OT_ERR_SHAPE;
    const long long bytes_old = static_cast<long long>(U) * kv_user_elems(o) * m->esz;
    const long long bytes_new = static_cast<long long>(U) * kv_user_elems(c) * m->esz;
    const char *po = static_cast<const char *>(kv_old), *pn = static_cast<const char *>(kv_new);
    if (po < pn + bytes_new && pn < po + bytes_old) return OT_ERR_ARG; // the caches overlap
    if (ws_bytes < ot_append_workspace_bytes(m, U, delta)) return OT_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // 1. the old rows' K/V into the grown layout (16-byte units)
    KvGrowArgs g;
    memset(&g, 0, sizeof(g));
    const long long unit = 16 / m->esz; // elements per unit
    g.src = static_cast<const uint4 *>(kv_old);
    g.dst = static_cast<uint4 *>(kv_new);
    g.ustride_src = kv_user_elems(o) / unit;
    g.ustride_dst = kv_user_elems(c) / unit;
    for (int l = 0; l < c.layers; ++l) {
        g.off_src[l] = kv_layer_off(o, l) / unit;
        g.off_dst[l] = kv_layer_off(c, l) / unit;
        g.len_src[l] = static_cast<long long>(rows_at(o, l)) * c.d / unit;
        g.len_dst[l] = static_cast<long long>(rows_at(c, l)) * c.d / unit;
    }
    ot_status r = profiled(m, st, OT_KIND_KV_GROW, ROLE_OTHER, 0.0,
                           2.0 * static_cast<double>(bytes_old), [&] { return launch_kv_grow(g, U, c.layers, st); });
    if (r != OT_OK) return r;
    // 2. the new rows through every layer, against the grown cache
    Ws w{static_cast<char *>(ws), ws_bytes, m->esz};
    RegionScope rs{{ws, ws_bytes}, {kv_new, static_cast<size_t>(bytes_new)},
                   {out_new, static_cast<size_t>(U) * c.q[c.layers - 1] * c.d * m->esz}};
    return run_encode(m, S_new, U, kv_new, out_new, w, st, nullptr, delta);
}

ot_status ot_score_candidates(ot_model *m, const void *kv_cache, int U, const void *ns, int C,
                              void *out_ns, void *ws, size_t ws_bytes, void *stream)
{
    if (!m || !kv_cache || !ns || !out_ns || !ws || U < 1 || C < 1) return OT_ERR_ARG;
    if (m->cfg.full_attn) return OT_ERR_UNSUPPORTED;
    if (!aligned16(kv_cache) || !aligned16(ns) || !aligned16(out_ns) || !aligned16(ws))
        return OT_ERR_ALIGN;
    if (static_cast<long long>(U) * C * m->cfg.n_ns > (1LL << 31) - 1) return OT_ERR_SHAPE;
    if (static_cast<long long>(C) * m->cfg.n_ns > (1LL << 30)) return OT_ERR_SHAPE;
    if (ws_bytes < score_ws_bytes(m->cfg, U, C, m->esz)) return OT_ERR_WORKSPACE_TOO_SMALL;
    Ws w{static_cast<char *>(ws), ws_bytes, m->esz};
    RegionScope rs{{ws, ws_bytes}, {out_ns, ns_bytes(m, static_cast<long long>(U) * C)}};
    return run_score(m, kv_cache, U, ns, C, out_ns, w, static_cast<cudaStream_t>(stream));
}

int ot_kv_pages_per_user(const ot_model *m) { return m ? page_off(m->cfg, m->cfg.layers) : 0; }

size_t ot_kv_page_bytes(const ot_model *m)
{
    return m ? 2 * static_cast<size_t>(OT_PAGE_ROWS) * m->cfg.d * m->esz : 0;
}

ot_status ot_encode_user_paged(ot_model *m, const void *S, int U, void *pool, long long n_pages,
                               const int32_t *pages, void *out_s_tail, void *ws, size_t ws_bytes,
                               void *stream)
{
    if (!m || !S || !pool || !pages || !ws || U < 1 || n_pages < 1) return OT_ERR_ARG;
    if (m->cfg.full_attn) return OT_ERR_UNSUPPORTED;
    if (!aligned16(S) || !aligned16(pool) || !aligned16(ws) || (reinterpret_cast<uintptr_t>(pages) & 3) ||
        (out_s_tail && !aligned16(out_s_tail)))
        return OT_ERR_ALIGN;
    const ot_config &c = m->cfg;
    if (static_cast<long long>(U) * c.L0 > (1LL << 31) - 1 || 2 * n_pages > (1LL << 31) - 1 ||
        (static_cast<long long>(c.d) * m->esz) % 16)
        return OT_ERR_SHAPE;
    if (ws_bytes < ot_workspace_bytes(m, U, 0)) return OT_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const PagedKv pg{pool, pages, n_pages, page_off(c, c.layers)};
    // the unused rows of every layer's last page hold zeros before any layer
    // reads its keys (the kernels read whole key blocks)
    PageTailArgs pt;
    memset(&pt, 0, sizeof(pt));
    pt.pool = pool;
    pt.pages = pages;
    pt.pg_ustride = pg.ustride;
    pt.n_pages = n_pages;
    pt.layers = c.layers;
    pt.d = c.d;
    pt.esz = m->esz;
    pt.err = m->err;
    for (int l = 0; l < c.layers; ++l) {
        pt.L[l] = rows_at(c, l);
        pt.off[l] = page_off(c, l);
    }
    ot_status r = profiled(m, st, OT_KIND_KV_GROW, ROLE_OTHER, 0.0, 0.0,
                           [&] { return launch_page_tail_clear(pt, U, st); });
    if (r != OT_OK) return r;
    Ws w{static_cast<char *>(ws), ws_bytes, m->esz};
    RegionScope rs{{ws, ws_bytes}, {pool, static_cast<size_t>(n_pages) * ot_kv_page_bytes(m)},
                   {out_s_tail, tail_bytes(m, U)}};
    return run_encode(m, S, U, nullptr, out_s_tail, w, st, nullptr, 0, false, &pg);
}

ot_status ot_score_candidates_paged(ot_model *m, const void *pool, long long n_pages,
                                    const int32_t *pages, int U, const void *ns, int C,
                                    void *out_ns, void *ws, size_t ws_bytes, void *stream)
{
    if (!m || !pool || !pages || !ns || !out_ns || !ws || U < 1 || C < 1 || n_pages < 1) return OT_ERR_ARG;
    if (m->cfg.full_attn) return OT_ERR_UNSUPPORTED;
    if (!aligned16(pool) || !aligned16(ns) || !aligned16(out_ns) || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(pages) & 3))
        return OT_ERR_ALIGN;
    if (static_cast<long long>(U) * C * m->cfg.n_ns > (1LL << 31) - 1 ||
        static_cast<long long>(C) * m->cfg.n_ns > (1LL << 30) || 2 * n_pages > (1LL << 31) - 1)
        return OT_ERR_SHAPE;
    if (ws_bytes < score_ws_bytes(m->cfg, U, C, m->esz)) return OT_ERR_WORKSPACE_TOO_SMALL;
    const PagedKv pg{const_cast<void *>(pool), pages, n_pages, page_off(m->cfg, m->cfg.layers)};
    Ws w{static_cast<char *>(ws), ws_bytes, m->esz};
    RegionScope rs{{ws, ws_bytes}, {out_ns, ns_bytes(m, static_cast<long long>(U) * C)}};
    return run_score(m, nullptr, U, ns, C, out_ns, w, static_cast<cudaStream_t>(stream), nullptr, &pg);
}

ot_status ot_full_forward(ot_model *m, const void *S, const void *ns, int B, int C,
                          void *out_s_tail, void *out_ns, void *kv_cache, void *ws,
                          size_t ws_bytes, void *stream)
{
    if (!m || !S || !ns || !out_s_tail || !out_ns || !ws || B < 1 || C < 1) return OT_ERR_ARG;
    if (!aligned16(S) || !aligned16(ns) || !aligned16(out_s_tail) || !aligned16(out_ns) ||
        !aligned16(ws) || (kv_cache && !aligned16(kv_cache)))
        return OT_ERR_ALIGN;
    if (static_cast<long long>(B) * m->cfg.L0 > (1LL << 31) - 1 ||
        static_cast<long long>(B) * C * m->cfg.n_ns > (1LL << 31) - 1)
        return OT_ERR_SHAPE;
    const ot_config &c = m->cfg;
    const size_t enc = encode_ws_bytes(c, B, m->esz), sc = score_ws_bytes(c, B, C, m->esz);
    const size_t kvb = kv_cache ? 0 : bytes_of(static_cast<long long>(B) * kv_user_elems(c), m->esz);
    const size_t serial_need = (enc > sc ? enc : sc) + kvb;
    if (ws_bytes < serial_need) return OT_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    RegionScope rs{{ws, ws_bytes}, {kv_cache, kv_bytes(m, B)}, {out_s_tail, tail_bytes(m, B)},
                   {out_ns, ns_bytes(m, static_cast<long long>(B) * C)}};
    Ws w{static_cast<char *>(ws), ws_bytes, m->esz};
    void *kv = kv_cache;
    if (!kv) {
        kv = w.take(static_cast<long long>(B) * kv_user_elems(c));
        if (!kv) return OT_ERR_WORKSPACE_TOO_SMALL;
    }
    if (c.full_attn) {
        // full attention: the S rows see their candidate's NS keys, one candidate per user
        if (C != 1) return OT_ERR_SHAPE;
        if (w.left < enc + sc) return OT_ERR_WORKSPACE_TOO_SMALL;
        std::lock_guard<std::recursive_mutex> lock(m->enqueue_mu);
        Ws w_enc = w;
        Ws w_sc{w.p + enc, w.left - enc, m->esz};
        if (merged_supported(m) && m->side)
            return run_full_merged(m, S, B, ns, C, kv, out_s_tail, out_ns, w_enc, w_sc, st);
        return run_full_joint(m, S, B, ns, kv, out_s_tail, out_ns, w_enc, w_sc, st);
    }
    // Shared O / FFN launches for both sides where the kernels allow it
    if (merged_supported(m) && m->side && w.left >= enc + sc) {
        std::lock_guard<std::recursive_mutex> lock(m->enqueue_mu);
        Ws w_enc = w;
        Ws w_sc{w.p + enc, w.left - enc, m->esz};
        return run_full_merged(m, S, B, ns, C, kv, out_s_tail, out_ns, w_enc, w_sc, st);
    }
    // Otherwise overlapped when the workspace holds both sides and per-launch
    // profiling (which times each kernel alone) is off: the NS side of layer
    // l waits only for layer l's cached S K/V, so it runs beside S layers l+1...
    const bool overlap = !m->profiling && m->side && w.left >= enc + sc;
    if (!overlap) {
        ot_status r = run_encode(m, S, B, kv, out_s_tail, w, st);
        if (r != OT_OK) return r;
        return run_score(m, kv, B, ns, C, out_ns, w, st);
    }
    std::lock_guard<std::recursive_mutex> lock(m->enqueue_mu);
    Ws w_enc = w;
    Ws w_sc{w.p + enc, w.left - enc, m->esz};
    if (cudaEventRecord(m->fork_ev, st) != cudaSuccess ||
        cudaStreamWaitEvent(m->side, m->fork_ev, 0) != cudaSuccess)
        return OT_ERR_CUDA;
    ot_status r = run_encode(m, S, B, kv, out_s_tail, w_enc, st, m->kv_ready);
    ot_status r2 = OT_OK;
    if (r == OT_OK) r2 = run_score(m, kv, B, ns, C, out_ns, w_sc, m->side, m->kv_ready);
    // always join the side stream back, so the caller's stream orders after it
    if (cudaEventRecord(m->join_ev, m->side) != cudaSuccess ||
        cudaStreamWaitEvent(st, m->join_ev, 0) != cudaSuccess)
        return OT_ERR_CUDA;
    return r != OT_OK ? r : r2;
}

// Workspace of ot_full_forward_host: two staging slots (S and x), the NS
// tokens, the device outputs, then the forward's own workspace; every region
// starts on a 256-byte boundary.
struct HostWs {
    size_t s_bytes, x_bytes, ns_bytes, tail_bytes, slot, total_fixed;
};

static size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

static HostWs host_ws(const ot_model *m, int B, int C)
{
    const ot_config &c = m->cfg;
    HostWs h;
    h.s_bytes = align256(bytes_of(static_cast<long long>(B) * c.L0 * c.d, m->esz));
    h.x_bytes = align256(bytes_of(static_cast<long long>(B) * C * c.F, m->esz));
    h.ns_bytes = align256(bytes_of(static_cast<long long>(B) * C * c.n_ns * c.d, m->esz));
    h.tail_bytes = align256(bytes_of(static_cast<long long>(B) * c.q[c.layers - 1] * c.d, m->esz));
    h.slot = h.s_bytes + h.x_bytes;
    h.total_fixed = 2 * h.slot + 2 * h.ns_bytes + h.tail_bytes; // ns in, ns out, S tail
    return h;
}

size_t ot_host_workspace_bytes(const ot_model *m, int users, int cands)
{
    if (!m || users < 1 || cands < 1 || m->cfg.F <= 0) return 0;
    return host_ws(m, users, cands).total_fixed + ot_workspace_bytes(m, users, cands);
}

ot_status ot_full_forward_host(ot_model *m, const void *S_host, const void *x_host, int B, int C,
                               void *out_s_tail_host, void *out_ns_host, void *kv_cache, void *ws,
                               size_t ws_bytes, void *stream)
{
    if (!m || !S_host || !x_host || !out_s_tail_host || !out_ns_host || !ws || B < 1 || C < 1)
        return OT_ERR_ARG;
    if (m->cfg.F <= 0) return OT_ERR_SHAPE;
    if (!aligned16(ws) || (kv_cache && !aligned16(kv_cache))) return OT_ERR_ALIGN;
    if (ws_bytes < ot_host_workspace_bytes(m, B, C)) return OT_ERR_WORKSPACE_TOO_SMALL;
    if (!m->copy_stream) return OT_ERR_CUDA;
    const HostWs h = host_ws(m, B, C);
    char *base = static_cast<char *>(ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::recursive_mutex> lock(m->enqueue_mu);
    const int slot = static_cast<int>(m->host_calls & 1);
    char *S_dev = base + slot * h.slot, *x_dev = S_dev + h.s_bytes;
    char *ns_dev = base + 2 * h.slot, *out_ns_dev = ns_dev + h.ns_bytes, *tail_dev = out_ns_dev + h.ns_bytes;
    char *fw = base + h.total_fixed;
    // inputs: once the forward two calls back has finished reading this slot
    if (cudaStreamWaitEvent(m->copy_stream, m->in_free[slot], 0) != cudaSuccess ||
        cudaMemcpyAsync(S_dev, S_host, bytes_of(static_cast<long long>(B) * m->cfg.L0 * m->cfg.d, m->esz),
                        cudaMemcpyHostToDevice, m->copy_stream) != cudaSuccess ||
        cudaMemcpyAsync(x_dev, x_host, bytes_of(static_cast<long long>(B) * C * m->cfg.F, m->esz),
                        cudaMemcpyHostToDevice, m->copy_stream) != cudaSuccess ||
        cudaEventRecord(m->in_ready[slot], m->copy_stream) != cudaSuccess ||
        cudaStreamWaitEvent(st, m->in_ready[slot], 0) != cudaSuccess)
        return OT_ERR_CUDA;
    ++m->host_calls;
    ot_status r = ot_auto_split(m, x_dev, static_cast<long>(B) * C, ns_dev, stream);
    if (r == OT_OK)
        r = ot_full_forward(m, S_dev, ns_dev, B, C, tail_dev, out_ns_dev, kv_cache, fw,
                            ws_bytes - h.total_fixed, stream);
    // the slot is free again once the forward has run (also after an error,
    // so later calls do not wait on a stale record)
    if (cudaEventRecord(m->in_free[slot], st) != cudaSuccess) return OT_ERR_CUDA;
    if (r != OT_OK) return r;
    const ot_config &c = m->cfg;
    if (cudaMemcpyAsync(out_s_tail_host, tail_dev,
                        bytes_of(static_cast<long long>(B) * c.q[c.layers - 1] * c.d, m->esz),
                        cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(out_ns_host, out_ns_dev, bytes_of(static_cast<long long>(B) * C * c.n_ns * c.d, m->esz),
                        cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return OT_ERR_CUDA;
    return OT_OK;
}

} // extern "C"
