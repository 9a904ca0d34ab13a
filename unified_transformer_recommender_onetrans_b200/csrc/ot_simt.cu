// CUDA-core kernels: the fp32 path (fp32 storage, fp32 FMA, no TF32, accurate
// expf / erff / rsqrtf-free sqrt) and the generic helpers (gain folding,
// embedding gather).  The fp32 GEMM and attention here take the same
// GemmArgs / AttnArgs as the tensor-core kernels, so both paths share one
// host orchestration.
#include <cuda_bf16.h>
#include <math.h>

#include "ot_internal.h"

namespace ot {

template <typename T> __device__ __forceinline__ float ld_f(const T *p);
template <> __device__ __forceinline__ float ld_f<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(*p);
}

__device__ __forceinline__ void st_out(void *base, long long idx, int store, float v)
{
    if (store == OT_STORE_F32)
        static_cast<float *>(base)[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(base)[idx] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float ld_res(const void *base, long long idx, int store)
{
    if (store == OT_STORE_F32) return static_cast<const float *>(base)[idx];
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(base)[idx]);
}

__device__ __forceinline__ float gelu_erf(float z)
{
    return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}

// --------------------------------------------------------------------------
// SIMT GEMM: 64 x 64 output tile per CTA, 256 threads, 4 x 4 outputs each.
constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16;

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs a)
{
    __shared__ float As[SG_BK][SG_BM + 1];
    __shared__ float Bs[SG_BK][SG_BN + 1];
    __shared__ float ss[SG_BM];
    const int tid = threadIdx.x;
    const int g = blockIdx.z;
    const long long m0 = static_cast<long long>(blockIdx.y) * SG_BM;
    const int n0 = blockIdx.x * SG_BN;
    const T *A = static_cast<const T *>(a.A);
    const T *B = static_cast<const T *>(a.B) + static_cast<long long>(g) * a.b_gstride;
    if (tid < SG_BM) ss[tid] = 0.f;
    float acc[4][4] = {};
    const int tr = tid / 16, tc = tid % 16; // 16 x 16 thread grid
    for (int k0 = 0; k0 < a.K; k0 += SG_BK) {
        __syncthreads();
        for (int e = tid; e < SG_BM * SG_BK; e += 256) {
            int r = e / SG_BK, k = e % SG_BK;
            long long gr = m0 + r;
            float v = 0.f;
            if (gr < a.M && k0 + k < a.K)
                v = ld_f(A + rowmap_apply(a.a_map, gr, g) * a.lda + k0 + k);
            As[k][r] = v;
            if (a.norm && v != 0.f) atomicAdd(&ss[r], v * v);
        }
        for (int e = tid; e < SG_BN * SG_BK; e += 256) {
            int n = e / SG_BK, k = e % SG_BK;
            float v = 0.f;
            if (n0 + n < a.N && k0 + k < a.K) v = ld_f(B + static_cast<long long>(n0 + n) * a.K + k0 + k);
            Bs[k][n] = v;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < SG_BK; ++k) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[k][tr * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = Bs[k][tc * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        long long r = m0 + tr * 4 + i;
        if (r >= a.M) continue;
        float rs = 1.f;
        if (a.norm) rs = 1.0f / sqrtf(ss[tr * 4 + i] / static_cast<float>(a.K) + a.eps);
        long long arow = rowmap_apply(a.a_map, r, g);
        if (a.row_scale) rs *= a.row_scale[arow];
        if (a.g_scale) rs *= a.g_scale[g];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int c = n0 + tc * 4 + j;
            if (c >= a.N) continue;
            float v = acc[i][j] * rs;
            if (a.gelu) v = gelu_erf(v);
            if (a.res) {
                const long long ri = rowmap_apply(a.res_map, r, g) * a.res_ld + c;
                const long long esz = a.store == OT_STORE_F32 ? 4 : 2;
                if (ot_dev_ok(ri * esz, esz, a.res_cap, a.wait.err)) v += ld_res(a.res, ri, a.store);
            }
            for (int s = 0; s < a.nseg; ++s) {
                const EpiSeg &sg = a.seg[s];
                if (c < sg.c_lo || c >= sg.c_hi || !rowmap_keep(sg.map, r)) continue;
                long long orow;
                if (sg.pages) { // paged KV cache: a bad page id is reported, not written
                    orow = paged_row(sg, r);
                    if (orow < 0) {
                        if (a.wait.err) atomicCAS(a.wait.err, 0, OT_ERR_DEVICE_BOUNDS);
                        continue;
                    }
                } else {
                    orow = rowmap_apply(sg.map, r, g);
                }
                const long long oi = orow * sg.ld + (c - sg.c_lo), esz = a.store == OT_STORE_F32 ? 4 : 2;
                if (ot_dev_ok(oi * esz, esz, sg.cap, a.wait.err)) st_out(sg.out, oi, a.store, v);
            }
        }
    }
}

cudaError_t launch_gemm_simt(const GemmArgs &a, cudaStream_t s)
{
    dim3 grid((a.N + SG_BN - 1) / SG_BN, (a.M + SG_BM - 1) / SG_BM, a.G);
    if (a.in_dtype == OT_DTYPE_F32)
        gemm_simt_kernel<float><<<grid, 256, 0, s>>>(a);
    else
        gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

// --------------------------------------------------------------------------
// SIMT attention: one thread per query row, 64 rows per CTA, keys staged
// through shared memory 64 at a time; streaming softmax with accurate expf.
constexpr int SA_ROWS = 64, SA_KT = 64;

template <typename T, int HD>
__global__ void __launch_bounds__(SA_ROWS) attn_simt_kernel(AttnArgs a)
{
    __shared__ float Ks[SA_KT][HD + 1];
    __shared__ float Vs[SA_KT][HD + 1];
    const int u = blockIdx.z, h = blockIdx.y;
    const int i0 = blockIdx.x * SA_ROWS;
    const int i = i0 + threadIdx.x;
    const bool valid = i < a.nq;
    const T *Q = static_cast<const T *>(a.Q) + (static_cast<long long>(u) * a.nq) * a.d + h * HD;
    float q[HD], o[HD];
#pragma unroll
    for (int e = 0; e < HD; ++e) {
        q[e] = valid ? ld_f(Q + static_cast<long long>(i) * a.d + e) * a.scale : 0.f;
        o[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    const int i_last = min(i0 + SA_ROWS, a.nq) - 1;
    // ---- S keys
    int s_keys;
    if (a.mode == 0 && !a.full)
        s_keys = a.L - a.nq + i_last + 1; // the last query row's S row + 1
    else
        s_keys = a.L;
    const int t_self = a.L - a.nq + i; // S mode: this row's S position
    const T *KS = static_cast<const T *>(a.KS) + static_cast<long long>(u) * a.s_ustride + h * HD;
    const T *VS = static_cast<const T *>(a.VS) + static_cast<long long>(u) * a.s_ustride + h * HD;
    // key row j of this user: dense rows, or its page of a paged cache
    auto key_off = [&](int j, int kv) -> long long {
        if (!a.pages) return static_cast<long long>(j) * a.d;
        const long long pg = attn_page(a, u, j / OT_PAGE_ROWS);
        return ((pg * 2 + kv) * OT_PAGE_ROWS + j % OT_PAGE_ROWS) * a.d;
    };
    const T *KB = a.pages ? static_cast<const T *>(a.KS) + h * HD : KS;
    const T *VB = a.pages ? static_cast<const T *>(a.KS) + h * HD : VS;
    for (int j0 = 0; j0 < s_keys; j0 += SA_KT) {
        __syncthreads();
        for (int e = threadIdx.x; e < SA_KT * HD; e += SA_ROWS) {
            int j = e / HD, c = e % HD;
            bool in = j0 + j < s_keys;
            Ks[j][c] = in ? ld_f(KB + key_off(j0 + j, 0) + c) : 0.f;
            Vs[j][c] = in ? ld_f(VB + key_off(j0 + j, 1) + c) : 0.f;
        }
        __syncthreads();
        if (!valid) continue;
        int jend = min(SA_KT, s_keys - j0);
        if (a.mode == 0 && !a.full) jend = min(jend, t_self - j0 + 1);
        for (int j = 0; j < jend; ++j) {
            float sc = 0.f;
#pragma unroll
            for (int e = 0; e < HD; ++e) sc = fmaf(q[e], Ks[j][e], sc);
            if (sc > m) {
                float corr = expf(m - sc);
                l *= corr;
#pragma unroll
                for (int e = 0; e < HD; ++e) o[e] *= corr;
                m = sc;
            }
            float p = expf(sc - m);
            l += p;
#pragma unroll
            for (int e = 0; e < HD; ++e) o[e] = fmaf(p, Vs[j][e], o[e]);
        }
    }
    // ---- NS keys of the candidates this CTA's rows belong to (NS mode), or
    // with full attention in S mode all nkn NS keys of the user
    if (a.mode == 1 || a.full) {
        const int c_first = a.mode == 1 ? i0 / a.N : 0, c_last = a.mode == 1 ? i_last / a.N : 0;
        const int k_begin = c_first * a.N, k_end = a.mode == 1 ? (c_last + 1) * a.N : a.nkn;
        const T *KN = static_cast<const T *>(a.KN) + static_cast<long long>(u) * a.nkn * a.d + h * HD;
        const T *VN = static_cast<const T *>(a.VN) + static_cast<long long>(u) * a.nkn * a.d + h * HD;
        // the row's candidate and position; in full attention every NS key of
        // the candidate is visible (S mode: the user's only candidate)
        const int my_c = a.mode == 1 ? i / a.N : 0, my_n = a.full ? a.N - 1 : i % a.N;
        for (int j0 = k_begin; j0 < k_end; j0 += SA_KT) {
            __syncthreads();
            for (int e = threadIdx.x; e < SA_KT * HD; e += SA_ROWS) {
                int j = e / HD, c = e % HD;
                bool in = j0 + j < k_end;
                Ks[j][c] = in ? ld_f(KN + static_cast<long long>(j0 + j) * a.d + c) : 0.f;
                Vs[j][c] = in ? ld_f(VN + static_cast<long long>(j0 + j) * a.d + c) : 0.f;
            }
            __syncthreads();
            if (!valid) continue;
            int jend = min(SA_KT, k_end - j0);
            for (int j = 0; j < jend; ++j) {
                int key = j0 + j;
                if (key / a.N != my_c || key % a.N > my_n) continue;
                float sc = 0.f;
#pragma unroll
                for (int e = 0; e < HD; ++e) sc = fmaf(q[e], Ks[j][e], sc);
                if (sc > m) {
                    float corr = expf(m - sc);
                    l *= corr;
#pragma unroll
                    for (int e = 0; e < HD; ++e) o[e] *= corr;
                    m = sc;
                }
                float p = expf(sc - m);
                l += p;
#pragma unroll
                for (int e = 0; e < HD; ++e) o[e] = fmaf(p, Vs[j][e], o[e]);
            }
        }
    }
    if (!valid) return;
    float inv = 1.0f / l;
    long long orow = (static_cast<long long>(u) * a.nq + i) * a.d + h * HD;
    if (!ot_dev_ok(orow * (a.dtype == OT_DTYPE_F32 ? 4 : 2), HD * (a.dtype == OT_DTYPE_F32 ? 4 : 2), a.o_cap,
                   a.wait.err))
        return;
#pragma unroll
    for (int e = 0; e < HD; ++e) {
        if (a.dtype == OT_DTYPE_F32)
            static_cast<float *>(a.O)[orow + e] = o[e] * inv;
        else
            static_cast<__nv_bfloat16 *>(a.O)[orow + e] = __float2bfloat16_rn(o[e] * inv);
    }
}

template <typename T>
static cudaError_t attn_simt_dispatch(const AttnArgs &a, cudaStream_t s)
{
    dim3 grid((a.nq + SA_ROWS - 1) / SA_ROWS, a.H, a.U);
    switch (a.hd) {
    case 16: attn_simt_kernel<T, 16><<<grid, SA_ROWS, 0, s>>>(a); break;
    case 32: attn_simt_kernel<T, 32><<<grid, SA_ROWS, 0, s>>>(a); break;
    case 64: attn_simt_kernel<T, 64><<<grid, SA_ROWS, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_attn_simt(const AttnArgs &a, cudaStream_t s)
{
    if (a.dtype == OT_DTYPE_F32) return attn_simt_dispatch<float>(a, s);
    return attn_simt_dispatch<__nv_bfloat16>(a, s);
}

// --------------------------------------------------------------------------
// out[g][r][c] = W[g][r][c] * gain[g][c]  (RMSNorm gain folded into the
// projection that follows the norm: n(x) W^T = r * x (diag(gain) W^T)).
template <typename T>
__global__ void fold_gain_kernel(const T *W, const T *gain, T *out, long long rows, int cols,
                                 long long groups, long long g_gstride)
{
    long long total = groups * rows * cols;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        long long g = e / (rows * cols);
        int c = static_cast<int>(e % cols);
        float v = ld_f(W + e) * ld_f(gain + g * g_gstride + c);
        if constexpr (sizeof(T) == 4)
            out[e] = v;
        else
            out[e] = __float2bfloat16_rn(v);
    }
}

cudaError_t launch_fold_gain(const void *W, const void *g, void *out, long long rows, int cols,
                             long long groups, long long g_gstride, int dtype, cudaStream_t s)
{
    long long total = groups * rows * cols;
    int blocks = static_cast<int>((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
    if (dtype == OT_DTYPE_F32)
        fold_gain_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float *>(W),
                                                       static_cast<const float *>(g),
                                                       static_cast<float *>(out), rows, cols,
                                                       groups, g_gstride);
    else
        fold_gain_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(W), static_cast<const __nv_bfloat16 *>(g),
            static_cast<__nv_bfloat16 *>(out), rows, cols, groups, g_gstride);
    return cudaGetLastError();
}

// --------------------------------------------------------------------------
// Paged KV cache: zero the unused rows of every layer's last page (rows
// L_l % OT_PAGE_ROWS .. OT_PAGE_ROWS - 1, K and V), so the attention kernels,
// which read whole key blocks, never multiply a masked probability by stale
// values.  One CTA per (user, layer).
__global__ void page_tail_clear_kernel(PageTailArgs a)
{
    const int u = blockIdx.x / a.layers, l = blockIdx.x % a.layers;
    const int used = a.L[l] % OT_PAGE_ROWS;
    if (used == 0) return;
    long long pg = a.pages[static_cast<long long>(u) * a.pg_ustride + a.off[l] + a.L[l] / OT_PAGE_ROWS];
    if (pg < 0 || pg >= a.n_pages) {
        if (threadIdx.x == 0 && a.err) atomicCAS(a.err, 0, OT_ERR_DEVICE_BOUNDS);
        return;
    }
    const long long row16 = static_cast<long long>(a.d) * a.esz / 16; // 16-byte units per row
    uint4 *base = static_cast<uint4 *>(a.pool);
    for (int kv = 0; kv < 2; ++kv) {
        uint4 *p = base + ((pg * 2 + kv) * OT_PAGE_ROWS + used) * row16;
        const long long n = (OT_PAGE_ROWS - used) * row16;
        for (long long i = threadIdx.x; i < n; i += blockDim.x) p[i] = make_uint4(0, 0, 0, 0);
    }
}

cudaError_t launch_page_tail_clear(const PageTailArgs &a, int users, cudaStream_t s)
{
    if ((static_cast<long long>(a.d) * a.esz) % 16) return cudaErrorInvalidValue;
    page_tail_clear_kernel<<<users * a.layers, 256, 0, s>>>(a);
    return cudaGetLastError();
}

// --------------------------------------------------------------------------
// Embedding gather: one warp per output row, 16-byte vector copies.  An id
// outside [0, rows) writes zeros and records OT_ERR_DEVICE_BOUNDS.
__global__ void embed_gather_kernel(const uint4 *table, long long rows, int vec_per_row,
                                    const int64_t *ids, long long n, uint4 *out, int *err)
{
    const int lane = threadIdx.x & 31;
    long long w = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
    const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (; w < n; w += nw) {
        long long id = ids[w];
        bool ok = id >= 0 && id < rows;
        if (!ok && lane == 0 && err) atomicCAS(err, 0, OT_ERR_DEVICE_BOUNDS);
        const uint4 *src = table + (ok ? id : 0) * vec_per_row;
        uint4 *dst = out + w * vec_per_row;
        for (int v = lane; v < vec_per_row; v += 32) dst[v] = ok ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
    }
}

cudaError_t launch_embed_gather(const void *table, long long rows, int d, const int64_t *ids,
                                long long n, void *out, int *err, cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    int vec = d * 2 / 16;
    long long warps = n;
    long long blocks = (warps * 32 + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    embed_gather_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
        static_cast<const uint4 *>(table), rows, vec, ids, n, static_cast<uint4 *>(out), err);
    return cudaGetLastError();
}

// Old K/V rows of every (user, layer) into the layout of a longer sequence:
// block (x, l * 2 + kv, u) copies a slice of user u's layer-l K (kv = 0) or
// V (kv = 1) block, all offsets in 16-byte units.
__global__ void kv_grow_kernel(const __grid_constant__ KvGrowArgs a)
{
    const int l = static_cast<int>(blockIdx.y) >> 1, kv = static_cast<int>(blockIdx.y) & 1;
    const long long u = blockIdx.z;
    const long long n = a.len_src[l];
    const uint4 *src = a.src + u * a.ustride_src + a.off_src[l] + kv * n;
    uint4 *dst = a.dst + u * a.ustride_dst + a.off_dst[l] + kv * a.len_dst[l];
    const long long step = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n; i += step)
        dst[i] = __ldg(src + i);
}

cudaError_t launch_kv_grow(const KvGrowArgs &a, int users, int layers, cudaStream_t s)
{
    if (users < 1 || users > 65535 || layers < 1 || layers > OT_MAX_LAYERS) return cudaErrorInvalidValue;
    long long longest = 0;
    for (int l = 0; l < layers; ++l) longest = a.len_src[l] > longest ? a.len_src[l] : longest;
    // enough blocks per (user, layer, K|V) to cover its longest slice in a
    // few strides, at least one
    long long bx = (longest + 4 * 256 - 1) / (4 * 256);
    if (bx < 1) bx = 1;
    if (bx > 64) bx = 64;
    kv_grow_kernel<<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(2 * layers), static_cast<unsigned>(users)),
                     256, 0, s>>>(a);
    return cudaGetLastError();
}

} // namespace ot
