// Backward pass of the block stack: ot_full_backward (fp32 models, the
// OneTrans causal mask or full attention, dense FFNs).  The summary page puts activation
// checkpointing on top of the stack for training (systems paragraph): a
// forward pass keeps every layer's input rows only, and the backward
// recomputes one layer at a time from them, top layer first, before taking
// its gradients.  CUDA-core fp32 kernels, deterministic (no atomics).
//
// Per layer l (S rows X [U][L][d], query tail q; NS rows Y [U][C][N][d]):
//   recompute  Z1 = n(X; g1), QKV = Z1 Wqkv^T, A = attn(QKV), H = X_tail +
//              A Wo^T, Z2 = n(H; g2), U1 = Z2 W1^T, Act = GELU(U1); the NS
//              side the same with its private weights per position n
//              (grouped GEMMs, group = n) and attention over the layer's S
//              keys and the candidate's NS keys m <= n;
//   gradients  dH = dOut + n'(dOut W2 * GELU'(U1) W1), dW2 = dOut^T Act,
//              dW1 = dU1^T Z2, dA = dH Wo, dWo = dH^T A; attention
//              (ot_backward_attn.cu): dQ per query block, dK / dV per key
//              block (S keys collect the S tail rows at or after them and
//              every NS row of the user);
//              dWqkv = dQKV^T Z1, dX = n'(dQKV Wqkv) + dH on the tail rows.
// n'(.) is the RMSNorm backward: with r = (mean(x^2) + eps)^(-1/2),
//   dx = r g dz - x r^3 mean(x g dz),  dg = sum over rows of dz x r.
#include <math.h>
#include <stdint.h>

#include "ot_internal.h"

namespace ot {

__device__ __forceinline__ float bw_warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// rowmap_apply with the common P == 1 case (flat and NS-group maps) taken
// without a division
__device__ __forceinline__ long long bw_row(const RowMap &m, long long r, long long g)
{
    return m.P == 1 ? r * m.A + m.B + g * m.Gs : rowmap_apply(m, r, g);
}

// row r of group g of a GEMM operand: its segment when the GEMM has
// segments, else the row map
__device__ __forceinline__ long long bw_grow(const BwGemm &p, const RowMap &m, long long r, int g)
{
    return p.g_off ? static_cast<long long>(p.g_off[g]) + r : bw_row(m, r, g);
}

// rows of group g (M for NT / NN, K for TN)
__device__ __forceinline__ int bw_grows(const BwGemm &p, int g, int all)
{
    return p.g_cnt ? min(all, p.g_cnt[g]) : all;
}

__device__ __forceinline__ long long bw_warp_id()
{
    return (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
}

__device__ __forceinline__ long long bw_warp_count()
{
    return (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
}

// ---------------------------------------------------------------- RMSNorm
// One warp per row; rows are taken group-major (row r of group g is warp
// item g * rows + r).
__global__ void rms_fwd_kernel(BwRows a, const float *g, long long g_gstride, float eps, float *z,
                               float *r_out)
{
    const int lane = threadIdx.x & 31;
    for (long long w = bw_warp_id(); w < a.rows * a.G; w += bw_warp_count()) {
        const long long grp = w / a.rows, R = bw_row(a.map, w % a.rows, grp);
        const float *x = a.X + R * a.d;
        const float *gg = g + grp * g_gstride;
        float ss = 0.f;
        for (int k = lane; k < a.d; k += 32) ss = fmaf(x[k], x[k], ss);
        const float rs = 1.0f / sqrtf(bw_warp_sum(ss) / static_cast<float>(a.d) + eps);
        for (int k = lane; k < a.d; k += 32) z[R * a.d + k] = x[k] * rs * gg[k];
        if (lane == 0) r_out[R] = rs;
    }
}

__global__ void rms_bwd_kernel(BwRows a, const float *g, long long g_gstride, const float *r_in,
                               const float *dz, float *dx, int accumulate)
{
    const int lane = threadIdx.x & 31;
    for (long long w = bw_warp_id(); w < a.rows * a.G; w += bw_warp_count()) {
        const long long grp = w / a.rows, R = bw_row(a.map, w % a.rows, grp);
        const float *x = a.X + R * a.d;
        const float *dzr = dz + R * a.d;
        const float *gg = g + grp * g_gstride;
        const float rs = r_in[R];
        float s = 0.f;
        for (int k = lane; k < a.d; k += 32) s = fmaf(x[k] * gg[k], dzr[k], s);
        const float c = bw_warp_sum(s) * rs * rs * rs / static_cast<float>(a.d);
        float *dxr = dx + R * a.d;
        for (int k = lane; k < a.d; k += 32) {
            const float v = rs * gg[k] * dzr[k] - x[k] * c;
            dxr[k] = accumulate ? dxr[k] + v : v;
        }
    }
}

// Gain gradient in two deterministic steps: partial column sums over row
// chunks ([splits][G][d]), then their sum in chunk order.
__global__ void gain_partial_kernel(BwRows a, const float *r_in, const float *dz, float *partial, int splits)
{
    __shared__ float red[8][33];
    const int k = blockIdx.x * 32 + threadIdx.x, grp = blockIdx.y, zc = blockIdx.z;
    const long long chunk = (a.rows + splits - 1) / splits;
    const long long r0 = zc * chunk, r1 = min(a.rows, r0 + chunk);
    float acc = 0.f;
    if (k < a.d)
        for (long long r = r0 + threadIdx.y; r < r1; r += 8) {
            const long long R = bw_row(a.map, r, grp);
            acc = fmaf(dz[R * a.d + k] * a.X[R * a.d + k], r_in[R], acc);
        }
    red[threadIdx.y][threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.y == 0 && k < a.d) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) s += red[i][threadIdx.x];
        partial[(static_cast<long long>(zc) * a.G + grp) * a.d + k] = s;
    }
}

__global__ void gain_reduce_kernel(const float *partial, int splits, int G, int d, float *dg, long long g_gstride)
{
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < static_cast<long long>(G) * d;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long grp = i / d, k = i % d;
        float s = 0.f;
        for (int zc = 0; zc < splits; ++zc) s += partial[(static_cast<long long>(zc) * G + grp) * d + k];
        dg[grp * g_gstride + k] = s;
    }
}

// ---------------------------------------------------------------- elementwise
__global__ void gelu_fwd_kernel(const float *u, float *a, long long n)
{
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        a[i] = 0.5f * u[i] * (1.0f + erff(u[i] * 0.70710678118654752f));
}

// d GELU(u) / du = Phi(u) + u phi(u) (exact-erf GELU); du may alias da.
__global__ void gelu_bwd_kernel(const float *u, const float *da, float *du, long long n)
{
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float x = u[i];
        const float cdf = 0.5f * (1.0f + erff(x * 0.70710678118654752f));
        const float pdf = 0.39894228040143268f * expf(-0.5f * x * x);
        du[i] = da[i] * (cdf + x * pdf);
    }
}

// dst[map(r)] += src[r] over rows of d floats
__global__ void rows_add_kernel(float *dst, RowMap map, const float *src, long long rows, int d)
{
    const long long n = rows * d;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long r = i / d, k = i % d;
        dst[rowmap_apply(map, r, 0) * d + k] += src[i];
    }
}

// ---------------------------------------------------------------- GEMM
// 64 x 64 output tile per CTA, 16-deep k steps staged in shared memory,
// 4 x 4 outputs per thread.
constexpr int GB_M = 64, GB_N = 64, GB_K = 16, GB_T = 256;

template <int FORM>
__global__ void __launch_bounds__(GB_T) bw_gemm_kernel(BwGemm p)
{
    __shared__ __align__(16) float As[GB_K][GB_M + 4];
    __shared__ __align__(16) float Bs[GB_K][GB_N + 4];
    const int tid = threadIdx.x;
    const int g = FORM == BW_TN ? static_cast<int>(blockIdx.z) / p.splits : static_cast<int>(blockIdx.z);
    const int split = FORM == BW_TN ? static_cast<int>(blockIdx.z) % p.splits : 0;
    const int m0 = blockIdx.y * GB_M, n0 = blockIdx.x * GB_N;
    const int Mg = FORM == BW_TN ? p.M : bw_grows(p, g, p.M); // output rows of this group
    // reduction range of this CTA (TN: one of `splits` chunks, GB_K aligned)
    int k_lo = 0, k_hi = FORM == BW_TN ? bw_grows(p, g, p.K) : p.K;
    if (FORM == BW_TN && p.splits > 1) {
        const int chunk = ((p.K + p.splits - 1) / p.splits + GB_K - 1) / GB_K * GB_K;
        k_lo = min(k_hi, split * chunk);
        k_hi = min(k_hi, k_lo + chunk);
    }
    const int tm = (tid >> 4) * 4, tn = (tid & 15) * 4;
    // rows of A (NT, NN) and of B (NT) this thread stages: fixed for the kernel
    const float *arow[4] = {nullptr, nullptr, nullptr, nullptr};
    const float *brow[4] = {nullptr, nullptr, nullptr, nullptr};
    if (FORM != BW_TN) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = m0 + (tid >> 4) + 16 * j;
            if (m < Mg) arow[j] = p.A + bw_grow(p, p.a_map, m, g) * p.lda;
        }
    }
    if (FORM == BW_NT) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + (tid >> 4) + 16 * j;
            if (n < p.N) brow[j] = p.B + g * p.b_gstride + static_cast<long long>(n) * p.ldb;
        }
    }
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = k_lo; k0 < k_hi; k0 += GB_K) {
        if (FORM != BW_TN) {
            const int kk = tid & 15, k = k0 + kk;
#pragma unroll
            for (int j = 0; j < 4; ++j) As[kk][(tid >> 4) + 16 * j] = (arow[j] && k < p.K) ? arow[j][k] : 0.f;
        } else {
            const int mm = tid & 63, m = m0 + mm;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int kk = (tid >> 6) + 4 * j, k = k0 + kk;
                As[kk][mm] = (k < k_hi && m < p.M) ? p.A[bw_grow(p, p.a_map, k, g) * p.lda + m] : 0.f;
            }
        }
        if (FORM == BW_NT) {
            const int kk = tid & 15, k = k0 + kk;
#pragma unroll
            for (int j = 0; j < 4; ++j) Bs[kk][(tid >> 4) + 16 * j] = (brow[j] && k < p.K) ? brow[j][k] : 0.f;
        } else {
            const int nn = tid & 63, n = n0 + nn;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int kk = (tid >> 6) + 4 * j, k = k0 + kk;
                float v = 0.f;
                if (k < k_hi && n < p.N) {
                    const long long row = FORM == BW_NN ? static_cast<long long>(k) : bw_grow(p, p.b_map, k, g);
                    v = p.B[(FORM == BW_NN ? g * p.b_gstride : 0) + row * p.ldb + n];
                }
                Bs[kk][nn] = v;
            }
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < GB_K; ++k) {
            const float4 a = *reinterpret_cast<const float4 *>(&As[k][tm]);
            const float4 b = *reinterpret_cast<const float4 *>(&Bs[k][tn]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + tm + i;
        if (m >= Mg) continue;
        float *crow;
        if (FORM == BW_TN && p.splits > 1)
            crow = p.partial + ((static_cast<long long>(split) * p.G + g) * p.M + m) * p.N;
        else if (FORM == BW_TN)
            crow = p.C + g * p.c_gstride + static_cast<long long>(m) * p.ldc;
        else
            crow = p.C + bw_grow(p, p.c_map, m, g) * p.ldc;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tn + j;
            if (n < p.N) crow[n] = p.accumulate && !(FORM == BW_TN && p.splits > 1) ? crow[n] + acc[i][j] : acc[i][j];
        }
    }
}

// The same three forms on 128 x 128 tiles, 8-deep k steps, 8 x 8 outputs
// per thread (rows ty*4 + i and 64 + ty*4 + i, columns likewise), the next
// k step's operands fetched into registers while the current one computes
// and staged into the other of two shared-memory buffers (one barrier per
// k step).
constexpr int GL_M = 128, GL_N = 128, GL_K = 8;

template <int FORM>
__global__ void __launch_bounds__(GB_T, 2) bw_gemm_big_kernel(BwGemm p)
{
    __shared__ __align__(16) float As[2][GL_K][GL_M + 4];
    __shared__ __align__(16) float Bs[2][GL_K][GL_N + 4];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int g = FORM == BW_TN ? static_cast<int>(blockIdx.z) / p.splits : static_cast<int>(blockIdx.z);
    const int split = FORM == BW_TN ? static_cast<int>(blockIdx.z) % p.splits : 0;
    const int m0 = blockIdx.y * GL_M, n0 = blockIdx.x * GL_N;
    const int Mg = FORM == BW_TN ? p.M : bw_grows(p, g, p.M);
    int k_lo = 0, k_hi = FORM == BW_TN ? bw_grows(p, g, p.K) : p.K;
    if (FORM == BW_TN && p.splits > 1) {
        const int chunk = ((p.K + p.splits - 1) / p.splits + GL_K - 1) / GL_K * GL_K;
        k_lo = min(k_hi, split * chunk);
        k_hi = min(k_hi, k_lo + chunk);
    }
    // staging: NT / NN A and NT B are row-major in k (thread: row t / 2,
    // k quad (t % 2) * 4); TN A and NN / TN B are row-major in m / n
    // (thread: k row t / 32, 4 columns (t % 32) * 4)
    const int rq = tid >> 1, kq = (tid & 1) * 4, kr = tid >> 5, cq = (tid & 31) * 4;
    const float *arow = nullptr, *brow = nullptr;
    if (FORM != BW_TN && m0 + rq < Mg) arow = p.A + bw_grow(p, p.a_map, m0 + rq, g) * p.lda;
    if (FORM == BW_NT && n0 + rq < p.N) brow = p.B + g * p.b_gstride + static_cast<long long>(n0 + rq) * p.ldb;
    float ra[4], rb[4];
    auto fetch = [&](int k0) {
        if (FORM != BW_TN) {
#pragma unroll
            for (int q = 0; q < 4; ++q) ra[q] = (arow && k0 + kq + q < k_hi) ? arow[k0 + kq + q] : 0.f;
        } else {
            const int k = k0 + kr;
            const float *src = k < k_hi ? p.A + bw_grow(p, p.a_map, k, g) * p.lda : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) ra[q] = (src && m0 + cq + q < p.M) ? src[m0 + cq + q] : 0.f;
        }
        if (FORM == BW_NT) {
#pragma unroll
            for (int q = 0; q < 4; ++q) rb[q] = (brow && k0 + kq + q < k_hi) ? brow[k0 + kq + q] : 0.f;
        } else {
            const int k = k0 + kr;
            const float *src = nullptr;
            if (k < k_hi)
                src = FORM == BW_NN ? p.B + g * p.b_gstride + static_cast<long long>(k) * p.ldb
                                    : p.B + bw_grow(p, p.b_map, k, g) * p.ldb;
#pragma unroll
            for (int q = 0; q < 4; ++q) rb[q] = (src && n0 + cq + q < p.N) ? src[n0 + cq + q] : 0.f;
        }
    };
    auto stage = [&](int bf) {
        if (FORM != BW_TN) {
#pragma unroll
            for (int q = 0; q < 4; ++q) As[bf][kq + q][rq] = ra[q];
        } else {
            *reinterpret_cast<float4 *>(&As[bf][kr][cq]) = make_float4(ra[0], ra[1], ra[2], ra[3]);
        }
        if (FORM == BW_NT) {
#pragma unroll
            for (int q = 0; q < 4; ++q) Bs[bf][kq + q][rq] = rb[q];
        } else {
            *reinterpret_cast<float4 *>(&Bs[bf][kr][cq]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
        }
    };
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    if (k_lo < k_hi) {
        fetch(k_lo);
        stage(0);
    }
    __syncthreads();
    int bf = 0;
    for (int k0 = k_lo; k0 < k_hi; k0 += GL_K) {
        const bool more = k0 + GL_K < k_hi;
        if (more) fetch(k0 + GL_K);
#pragma unroll
        for (int k = 0; k < GL_K; ++k) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&As[bf][k][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&As[bf][k][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[bf][k][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[bf][k][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        // the other buffer was last read in the previous step, before the
        // barrier that ended it
        if (more) stage(bf ^ 1);
        __syncthreads();
        bf ^= 1;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
        if (m >= Mg) continue;
        float *crow;
        if (FORM == BW_TN && p.splits > 1)
            crow = p.partial + ((static_cast<long long>(split) * p.G + g) * p.M + m) * p.N;
        else if (FORM == BW_TN)
            crow = p.C + g * p.c_gstride + static_cast<long long>(m) * p.ldc;
        else
            crow = p.C + bw_grow(p, p.c_map, m, g) * p.ldc;
        const bool add = p.accumulate && !(FORM == BW_TN && p.splits > 1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
            if (n < p.N) crow[n] = add ? crow[n] + acc[i][j] : acc[i][j];
        }
    }
}

// C[g][m][n] (+)= sum over splits, in split order, of partial[s][g][m][n]
__global__ void tn_reduce_kernel(BwGemm p)
{
    const long long per = static_cast<long long>(p.M) * p.N, n_all = per * p.G;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_all;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long g = i / per, mn = i % per, m = mn / p.N, n = mn % p.N;
        float v = 0.f;
        for (int sp = 0; sp < p.splits; ++sp) v += p.partial[sp * n_all + i];
        float *c = p.C + g * p.c_gstride + m * p.ldc + n;
        *c = p.accumulate ? *c + v : v;
    }
}

// ---------------------------------------------------------------- launchers
static int bw_blocks(long long threads)
{
    long long b = (threads + 255) / 256;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : static_cast<int>(b);
}

cudaError_t bw_rms_fwd(const BwRows &a, const float *g, long long g_gstride, float eps, float *z, float *r,
                       cudaStream_t s)
{
    rms_fwd_kernel<<<bw_blocks(a.rows * a.G * 32), 256, 0, s>>>(a, g, g_gstride, eps, z, r);
    return cudaGetLastError();
}

cudaError_t bw_rms_bwd(const BwRows &a, const float *g, long long g_gstride, const float *r, const float *dz,
                       float *dx, int accumulate, cudaStream_t s)
{
    rms_bwd_kernel<<<bw_blocks(a.rows * a.G * 32), 256, 0, s>>>(a, g, g_gstride, r, dz, dx, accumulate);
    return cudaGetLastError();
}

int bw_gain_splits(const BwRows &a)
{
    const long long col_blocks = static_cast<long long>((a.d + 31) / 32) * a.G;
    long long sp = (2 * 148 + col_blocks - 1) / col_blocks;
    const long long by_rows = (a.rows + 63) / 64;
    if (sp > by_rows) sp = by_rows;
    if (sp > 64) sp = 64;
    return sp < 1 ? 1 : static_cast<int>(sp);
}

cudaError_t bw_gain_grad(const BwRows &a, const float *r, const float *dz, float *partial, int splits, float *dg,
                         long long g_gstride, cudaStream_t s)
{
    if (a.G > 65535 || splits > 64) return cudaErrorInvalidValue;
    gain_partial_kernel<<<dim3((a.d + 31) / 32, a.G, splits), dim3(32, 8), 0, s>>>(a, r, dz, partial, splits);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    gain_reduce_kernel<<<bw_blocks(static_cast<long long>(a.G) * a.d), 256, 0, s>>>(partial, splits, a.G, a.d, dg,
                                                                                    g_gstride);
    return cudaGetLastError();
}

cudaError_t bw_gelu_fwd(const float *u, float *a, long long n, cudaStream_t s)
{
    gelu_fwd_kernel<<<bw_blocks(n), 256, 0, s>>>(u, a, n);
    return cudaGetLastError();
}

cudaError_t bw_gelu_bwd(const float *u, const float *da, float *du, long long n, cudaStream_t s)
{
    gelu_bwd_kernel<<<bw_blocks(n), 256, 0, s>>>(u, da, du, n);
    return cudaGetLastError();
}

cudaError_t bw_rows_add(float *dst, RowMap dst_map, const float *src, long long rows, int d, cudaStream_t s)
{
    rows_add_kernel<<<bw_blocks(rows * d), 256, 0, s>>>(dst, dst_map, src, rows, d);
    return cudaGetLastError();
}

// 128 x 128 tiles where both output dimensions fill them
static bool bw_big(int M, int N) { return M >= GL_M && N >= GL_N; }

int bw_tn_splits(int M, int N, int K, int G)
{
    const int tm = bw_big(M, N) ? GL_M : GB_M, tn = bw_big(M, N) ? GL_N : GB_N;
    const long long tiles = static_cast<long long>((M + tm - 1) / tm) * ((N + tn - 1) / tn) * G;
    long long sp = (2 * 148 + tiles - 1) / tiles;
    const long long by_k = (K + 255) / 256; // at least 256 reduction rows per split
    if (sp > by_k) sp = by_k;
    if (sp > 64) sp = 64;
    return sp < 1 ? 1 : static_cast<int>(sp);
}

long long bw_tn_partial_floats(int M, int N, int K, int G)
{
    const int sp = bw_tn_splits(M, N, K, G);
    return sp > 1 ? static_cast<long long>(sp) * G * M * N : 0;
}

cudaError_t bw_gemm(const BwGemm &p, cudaStream_t s)
{
    const int splits = p.form == BW_TN ? p.splits : 1;
    const bool big = bw_big(p.M, p.N);
    const int tm = big ? GL_M : GB_M, tn = big ? GL_N : GB_N;
    const dim3 grid((p.N + tn - 1) / tn, (p.M + tm - 1) / tm, p.G * splits);
    if (p.M < 1 || p.N < 1 || p.K < 1 || p.G < 1 || splits < 1 || grid.y > 65535 || grid.z > 65535 ||
        (splits > 1 && !p.partial))
        return cudaErrorInvalidValue;
    switch (p.form * 2 + (big ? 1 : 0)) {
    case BW_NT * 2: bw_gemm_kernel<BW_NT><<<grid, GB_T, 0, s>>>(p); break;
    case BW_NN * 2: bw_gemm_kernel<BW_NN><<<grid, GB_T, 0, s>>>(p); break;
    case BW_TN * 2: bw_gemm_kernel<BW_TN><<<grid, GB_T, 0, s>>>(p); break;
    case BW_NT * 2 + 1: bw_gemm_big_kernel<BW_NT><<<grid, GB_T, 0, s>>>(p); break;
    case BW_NN * 2 + 1: bw_gemm_big_kernel<BW_NN><<<grid, GB_T, 0, s>>>(p); break;
    case BW_TN * 2 + 1: bw_gemm_big_kernel<BW_TN><<<grid, GB_T, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || splits == 1) return e;
    tn_reduce_kernel<<<bw_blocks(static_cast<long long>(p.M) * p.N * p.G), 256, 0, s>>>(p);
    return cudaGetLastError();
}

} // namespace ot

// ==================================================================== host
namespace {

using namespace ot;

constexpr RowMap kIdentity{1, 1, 0, 0, 0};

// Workspace carving.  With a null base it only sums the sizes and hands out
// non-null placeholder addresses (a dry run never dereferences them, but
// takes the same branches as a real one).
struct Carve {
    char *base;
    size_t off;
    float *take(long long n)
    {
        float *p = base ? reinterpret_cast<float *>(base + off)
                        : reinterpret_cast<float *>(static_cast<uintptr_t>(off) + 256);
        off += (static_cast<size_t>(n) * sizeof(float) + 255) & ~static_cast<size_t>(255);
        return p;
    }
};

// Intermediates of one side (S or NS) of one layer.
struct Side {
    float *r1, *Z1, *QKV, *A, *H, *r2, *Z2, *U1, *Act; // recomputed forward
    float *dH, *dAct, *dZ2, *dA, *dQKV, *dZ1;           // gradients
    float *sm, *sl, *sD;                                // softmax statistics
};

struct Backward {
    ot_config c;
    int U, C, N, d, f, H, hd, Lyr;
    int Ls[OT_MAX_LAYERS + 1]; // S rows per user entering layer l
    bool dry;
    cudaStream_t st;
    long long launches;
    cudaError_t err;
    const ot_weights *w;
    const ot_grads *g;
    const float *X[OT_MAX_LAYERS + 1], *Y[OT_MAX_LAYERS + 1];
    float *Xout_last, *Yout_last;
    Side s, n;
    float *partial;
    float *tn_partial; // split TN GEMMs: < 2 * 296 tiles of at most 128 x 128 floats
    // mixture of experts (E > 0): routing and the experts' rows, P = T k slots
    int E, K;
    BwMoe moe;
    float *Zp, *U1e, *Acte, *Ye, *dYe, *dActe, *dZp, *logits, *dlogits;
    static constexpr long long kTnPartialFloats = 2LL * 296 * 128 * 128;
    float *dXbuf[2], *dYbuf[2];
    // attention outputs and softmax statistics of every layer, kept from the
    // checkpointing forward: the per-layer recompute skips the attention
    float *sA[OT_MAX_LAYERS], *sM[OT_MAX_LAYERS], *sL[OT_MAX_LAYERS];
    float *nA[OT_MAX_LAYERS], *nM[OT_MAX_LAYERS], *nL[OT_MAX_LAYERS];
    const float *G_s, *G_ns;
    float *dS, *dns;
    size_t bytes;

    const float *wt(const void *p, long long off) const { return static_cast<const float *>(p) + off; }
    long long T(int l) const { return static_cast<long long>(U) * c.q[l]; }
    long long RS(int l) const { return static_cast<long long>(U) * Ls[l]; }
    long long RN() const { return static_cast<long long>(U) * C * N; }
    RowMap nmap() const { return RowMap{1, N, 0, 1, 0}; }

    // a kernel launch (counted; skipped in a dry run or after an error)
    template <typename F> void k(F &&fn)
    {
        ++launches;
        if (!dry && err == cudaSuccess) err = fn();
    }
    void copy(void *dst, const void *src, size_t nbytes)
    {
        if (!dry && err == cudaSuccess) err = cudaMemcpyAsync(dst, src, nbytes, cudaMemcpyDeviceToDevice, st);
    }
    void zero(void *dst, size_t nbytes)
    {
        if (!dry && err == cudaSuccess) err = cudaMemsetAsync(dst, 0, nbytes, st);
    }

    void plan(char *base, const float *S, const float *ns, float *out_s, float *out_ns)
    {
        Carve cv{base, 0};
        X[0] = S;
        Y[0] = ns;
        for (int l = 1; l < Lyr; ++l) {
            X[l] = cv.take(RS(l) * d);
            Y[l] = C ? cv.take(RN() * d) : nullptr;
        }
        Xout_last = out_s;
        Yout_last = out_ns;
        const long long R = RS(0), Tq = T(0), RN_ = RN();
        auto side = [&](Side &x, long long rows, long long tail) {
            x.r1 = cv.take(rows);
            x.Z1 = cv.take(rows * d);
            x.QKV = cv.take(rows * 3 * d);
            x.H = cv.take(tail * d);
            x.r2 = cv.take(tail);
            x.Z2 = cv.take(tail * d);
            x.U1 = cv.take(tail * f);
            x.Act = cv.take(tail * f);
            x.dH = cv.take(tail * d);
            x.dAct = cv.take(tail * f);
            x.dZ2 = cv.take(tail * d);
            x.dA = cv.take(tail * d);
            x.dQKV = cv.take(rows * 3 * d);
            x.dZ1 = cv.take(rows * d);
            x.sD = cv.take(tail * H);
        };
        side(s, R, Tq);
        if (C) side(n, RN_, RN_);
        for (int l = 0; l < Lyr; ++l) {
            sA[l] = cv.take(T(l) * d);
            sM[l] = cv.take(T(l) * H);
            sL[l] = cv.take(T(l) * H);
            if (C) {
                nA[l] = cv.take(RN_ * d);
                nM[l] = cv.take(RN_ * H);
                nL[l] = cv.take(RN_ * H);
            }
        }
        if (E) {
            const long long P = Tq * K;
            auto ints = [&](long long cnt) { return reinterpret_cast<int *>(cv.take(cnt)); };
            logits = cv.take(Tq * E);
            dlogits = cv.take(Tq * E);
            moe.sel = ints(Tq * 2);
            moe.gate = cv.take(Tq * 2);
            moe.lrank = ints(Tq * 2);
            moe.slot = ints(Tq * 2);
            moe.hist = ints(static_cast<long long>(bw_moe_chunks(static_cast<int>(Tq))) * E);
            moe.seg_off = ints(E);
            moe.seg_cnt = ints(E);
            Zp = cv.take(P * d);
            U1e = cv.take(P * f);
            Acte = cv.take(P * f);
            Ye = cv.take(P * d);
            dYe = cv.take(P * d);
            dActe = cv.take(P * f);
            dZp = cv.take(P * d);
        }
        partial = cv.take(64LL * d * (C ? N : 1)); // gain partials: <= 64 chunks, 1 or N groups
        tn_partial = cv.take(kTnPartialFloats);
        dXbuf[0] = cv.take(R * d);
        dXbuf[1] = cv.take(R * d);
        if (C) {
            dYbuf[0] = cv.take(RN_ * d);
            dYbuf[1] = cv.take(RN_ * d);
        }
        bytes = cv.off;
    }

    BwAttn attn_s(int l) const
    {
        BwAttn a{};
        a.mode = 0;
        a.U = U, a.H = H, a.hd = hd, a.d = d, a.L = Ls[l], a.nq = c.q[l], a.N = N;
        a.ld = 3LL * d, a.q_ustride = Ls[l], a.q_off = Ls[l] - c.q[l];
        a.qkv = a.skv = s.QKV;
        a.dqkv = a.dskv = s.dQKV;
        a.full = c.full_attn;
        a.nkv = C ? n.QKV : nullptr, a.n_ustride = static_cast<long long>(C) * N, a.nkn = C * N;
        a.O = s.A, a.dO = s.dA;
        a.stat_m = s.sm, a.stat_l = s.sl, a.stat_D = s.sD;
        a.scale = 1.0f / sqrtf(static_cast<float>(hd));
        return a;
    }
    BwAttn attn_ns(int l) const
    {
        BwAttn a{};
        a.mode = 1;
        a.U = U, a.H = H, a.hd = hd, a.d = d, a.L = Ls[l], a.nq = C * N, a.N = N;
        a.ld = 3LL * d, a.q_ustride = static_cast<long long>(C) * N, a.q_off = 0;
        a.qkv = n.QKV, a.skv = s.QKV;
        a.dqkv = n.dQKV, a.dskv = s.dQKV;
        a.full = c.full_attn;
        a.nkv = n.QKV, a.n_ustride = static_cast<long long>(C) * N, a.nkn = C * N;
        a.O = n.A, a.dO = n.dA;
        a.stat_m = n.sm, a.stat_l = n.sl, a.stat_D = n.sD;
        a.scale = 1.0f / sqrtf(static_cast<float>(hd));
        return a;
    }

    // segments of the experts (group = expert) for the next GEMM
    const int *seg_off_ = nullptr, *seg_cnt_ = nullptr;
    void segs(bool on)
    {
        seg_off_ = on ? moe.seg_off : nullptr;
        seg_cnt_ = on ? moe.seg_cnt : nullptr;
    }
    void seg_fill(BwGemm &p) const
    {
        p.g_off = seg_off_;
        p.g_cnt = seg_cnt_;
    }

    // C = A B^T with B a weight [G][Nn][K]
    void nt(const float *A, long long lda, RowMap am, const float *B, long long bgs, float *Cp, long long ldc,
            RowMap cm, int M, int Nn, int K, int G, int acc)
    {
        BwGemm p{};
        seg_fill(p);
        p.form = BW_NT, p.M = M, p.N = Nn, p.K = K, p.G = G;
        p.A = A, p.lda = lda, p.a_map = am;
        p.B = B, p.ldb = K, p.b_gstride = bgs;
        p.C = Cp, p.ldc = ldc, p.c_map = cm, p.accumulate = acc;
        k([&] { return bw_gemm(p, st); });
    }
    // C = A B with B a weight [G][K][Nn]
    void nn(const float *A, long long lda, RowMap am, const float *B, long long bgs, float *Cp, long long ldc,
            RowMap cm, int M, int Nn, int K, int G)
    {
        BwGemm p{};
        seg_fill(p);
        p.form = BW_NN, p.M = M, p.N = Nn, p.K = K, p.G = G;
        p.A = A, p.lda = lda, p.a_map = am;
        p.B = B, p.ldb = Nn, p.b_gstride = bgs;
        p.C = Cp, p.ldc = ldc, p.c_map = cm;
        k([&] { return bw_gemm(p, st); });
    }
    // weight gradient: C[g] [M][Nn] = sum over the group's K rows of A[row][m] B[row][n]
    void tn(const float *A, long long lda, RowMap am, const float *B, long long ldb, RowMap bm, float *Cp,
            long long cgs, int M, int Nn, int K, int G)
    {
        BwGemm p{};
        seg_fill(p);
        p.form = BW_TN, p.M = M, p.N = Nn, p.K = K, p.G = G;
        p.A = A, p.lda = lda, p.a_map = am;
        p.B = B, p.ldb = ldb, p.b_map = bm;
        p.C = Cp, p.ldc = Nn, p.c_gstride = cgs;
        p.splits = bw_tn_splits(M, Nn, K, G);
        p.partial = tn_partial;
        if (bw_tn_partial_floats(M, Nn, K, G) > kTnPartialFloats && err == cudaSuccess) err = cudaErrorInvalidValue;
        k([&] { return bw_gemm(p, st); });
        if (p.splits > 1) ++launches; // the split-order reduction
    }

    // Layer l forward (both sides); with s_out / n_out also its output rows.
    // The checkpointing pass runs the attention and keeps its outputs and
    // statistics; the recompute (recompute = true) reuses them.
    void forward(int l, float *s_out, float *n_out, bool recompute = false)
    {
        s.A = sA[l], s.sm = sM[l], s.sl = sL[l];
        if (C) n.A = nA[l], n.sm = nM[l], n.sl = nL[l];
        const int L = Ls[l], q = c.q[l];
        const long long R = RS(l), Tq = T(l);
        const long long d3 = 3LL * d, fd = static_cast<long long>(f) * d, dd = static_cast<long long>(d) * d;
        const RowMap nm = nmap();
        const long long RN_ = RN();
        const int M = U * C;
        const long long ln = static_cast<long long>(l) * N;
        // ---- both sides' QKV first (under full attention the S rows read NS keys)
        const BwRows x1{X[l], kIdentity, R, 1, d};
        k([&] { return bw_rms_fwd(x1, wt(w->g1_s, static_cast<long long>(l) * d), 0, c.eps, s.Z1, s.r1, st); });
        nt(s.Z1, d, kIdentity, wt(w->Wqkv_s, l * d3 * d), 0, s.QKV, d3, kIdentity, static_cast<int>(R), 3 * d, d, 1, 0);
        if (C) {
            // NS side: group = NS position, rows of a group = the U * C candidates
            const BwRows y1{Y[l], nm, M, N, d};
            k([&] { return bw_rms_fwd(y1, wt(w->g1_ns, ln * d), d, c.eps, n.Z1, n.r1, st); });
            nt(n.Z1, d, nm, wt(w->Wqkv_ns, ln * d3 * d), d3 * d, n.QKV, d3, nm, M, 3 * d, d, N, 0);
        }
        // ---- S side
        const BwAttn sa = attn_s(l);
        if (!recompute) k([&] { return bw_attn_fwd(sa, st); });
        if (!dry && err == cudaSuccess)
            err = cudaMemcpy2DAsync(s.H, static_cast<size_t>(q) * d * 4, X[l] + static_cast<long long>(L - q) * d,
                                    static_cast<size_t>(L) * d * 4, static_cast<size_t>(q) * d * 4, U,
                                    cudaMemcpyDeviceToDevice, st);
        nt(s.A, d, kIdentity, wt(w->Wo_s, l * dd), 0, s.H, d, kIdentity, static_cast<int>(Tq), d, d, 1, 1);
        const BwRows h2{s.H, kIdentity, Tq, 1, d};
        k([&] { return bw_rms_fwd(h2, wt(w->g2_s, static_cast<long long>(l) * d), 0, c.eps, s.Z2, s.r2, st); });
        if (E) {
            moe_forward(l, s_out);
        } else {
            nt(s.Z2, d, kIdentity, wt(w->W1_s, l * fd), 0, s.U1, f, kIdentity, static_cast<int>(Tq), f, d, 1, 0);
            k([&] { return bw_gelu_fwd(s.U1, s.Act, Tq * f, st); });
            if (s_out) {
                copy(s_out, s.H, static_cast<size_t>(Tq) * d * 4);
                nt(s.Act, f, kIdentity, wt(w->W2_s, l * fd), 0, s_out, d, kIdentity, static_cast<int>(Tq), d, f, 1,
                   1);
            }
        }
        if (!C) return;
        // ---- NS side
        const BwAttn na = attn_ns(l);
        if (!recompute) k([&] { return bw_attn_fwd(na, st); });
        copy(n.H, Y[l], static_cast<size_t>(RN_) * d * 4);
        nt(n.A, d, nm, wt(w->Wo_ns, ln * dd), dd, n.H, d, nm, M, d, d, N, 1);
        const BwRows h2n{n.H, nm, M, N, d};
        k([&] { return bw_rms_fwd(h2n, wt(w->g2_ns, ln * d), d, c.eps, n.Z2, n.r2, st); });
        nt(n.Z2, d, nm, wt(w->W1_ns, ln * fd), fd, n.U1, f, nm, M, f, d, N, 0);
        k([&] { return bw_gelu_fwd(n.U1, n.Act, RN_ * f, st); });
        if (n_out) {
            copy(n_out, n.H, static_cast<size_t>(RN_) * d * 4);
            nt(n.Act, f, nm, wt(w->W2_ns, ln * fd), fd, n_out, d, nm, M, d, f, N, 1);
        }
    }

    // The S-side mixture of layer l on Z2 = n(H; g2): router logits, routing,
    // the experts' FFNs over their segments; with s_out also y = H + sum g Y.
    void moe_forward(int l, float *s_out)
    {
        const int Tq = static_cast<int>(T(l));
        const long long fd = static_cast<long long>(f) * d, Eed = static_cast<long long>(E) * d;
        moe.T = Tq, moe.d = d, moe.E = E, moe.k = K, moe.logits = logits;
        nt(s.Z2, d, kIdentity, wt(w->W_router, l * Eed), 0, logits, E, kIdentity, Tq, E, d, 1, 0);
        k([&] { return bw_moe_route(moe, s.Z2, Zp, st); });
        launches += 3; // top-k, rank, offsets and dispatch
        segs(true);
        nt(Zp, d, kIdentity, wt(w->W1_moe, l * E * fd), fd, U1e, f, kIdentity, Tq, f, d, E, 0);
        k([&] { return bw_gelu_fwd(U1e, Acte, static_cast<long long>(Tq) * K * f, st); });
        nt(Acte, f, kIdentity, wt(w->W2_moe, l * E * fd), fd, Ye, d, kIdentity, Tq, d, f, E, 0);
        segs(false);
        if (s_out) k([&] { return bw_moe_combine(moe, s.H, Ye, s_out, st); });
    }

    // The S-side mixture's backward: dOut -> x.dZ2 (router and experts) and
    // the gradients of the router and the experts of layer l.
    void moe_back(int l, const float *dOut)
    {
        const int Tq = static_cast<int>(T(l));
        const long long fd = static_cast<long long>(f) * d, Eed = static_cast<long long>(E) * d;
        k([&] { return bw_moe_combine_bwd(moe, dOut, Ye, dYe, dlogits, st); });
        tn(dlogits, E, kIdentity, s.Z2, d, kIdentity, g->W_router + l * Eed, 0, E, d, Tq, 1); // dW_r
        nn(dlogits, E, kIdentity, wt(w->W_router, l * Eed), 0, s.dZ2, d, kIdentity, Tq, d, E, 1); // dZ2 = dlogits W_r
        segs(true);
        nn(dYe, d, kIdentity, wt(w->W2_moe, l * E * fd), fd, dActe, f, kIdentity, Tq, f, d, E);      // dAct = dY W2
        tn(dYe, d, kIdentity, Acte, f, kIdentity, g->W2_moe + l * E * fd, fd, d, f, Tq, E);          // dW2
        k([&] { return bw_gelu_bwd(U1e, dActe, dActe, static_cast<long long>(Tq) * K * f, st); });
        tn(dActe, f, kIdentity, Zp, d, kIdentity, g->W1_moe + l * E * fd, fd, f, d, Tq, E);          // dW1
        nn(dActe, f, kIdentity, wt(w->W1_moe, l * E * fd), fd, dZp, d, kIdentity, Tq, d, f, E);      // dZp = dU1 W1
        segs(false);
        k([&] { return bw_moe_gather(moe, dZp, s.dZ2, st); });
    }

    // FFN and output-projection backward of one side: dOut -> x.dH, x.dA and
    // the gradients of W1, W2, Wo and g2.  M rows in each of G groups under map.
    void ffn_back(Side &x, const float *dOut, RowMap map, int M, int G, const float *W1, const float *W2,
                  const float *Wo, const float *g2, long long ggs, float *dW1, float *dW2, float *dWo, float *dg2,
                  int moe_layer = -1)
    {
        const long long rows = static_cast<long long>(M) * G;
        const long long fd = static_cast<long long>(f) * d, dd = static_cast<long long>(d) * d;
        copy(x.dH, dOut, static_cast<size_t>(rows) * d * 4);
        if (moe_layer >= 0) {
            moe_back(moe_layer, dOut);
        } else {
            nn(dOut, d, map, W2, fd, x.dAct, f, map, M, f, d, G); // dAct = dOut W2
            tn(dOut, d, map, x.Act, f, map, dW2, fd, d, f, M, G);  // dW2 = dOut^T Act
            k([&] { return bw_gelu_bwd(x.U1, x.dAct, x.dAct, rows * f, st); });
            tn(x.dAct, f, map, x.Z2, d, map, dW1, fd, f, d, M, G); // dW1 = dU1^T Z2
            nn(x.dAct, f, map, W1, fd, x.dZ2, d, map, M, d, f, G); // dZ2 = dU1 W1
        }
        const BwRows hr{x.H, map, M, G, d};
        k([&] { return bw_rms_bwd(hr, g2, ggs, x.r2, x.dZ2, x.dH, 1, st); });
        const int sp = bw_gain_splits(hr);
        k([&] { return bw_gain_grad(hr, x.r2, x.dZ2, partial, sp, dg2, ggs, st); });
        ++launches; // bw_gain_grad issues two kernels
        nn(x.dH, d, map, Wo, dd, x.dA, d, map, M, d, d, G); // dA = dH Wo
        tn(x.dH, d, map, x.A, d, map, dWo, dd, d, d, M, G);  // dWo = dH^T A
    }

    // QKV projection and first-norm backward of one side: x.dQKV -> dX
    // (written, or added when accumulate), gradients of Wqkv and g1.
    void qkv_back(Side &x, const float *Xin, RowMap map, int M, int G, const float *Wqkv, const float *g1,
                  long long ggs, float *dWqkv, float *dg1, float *dX, int accumulate)
    {
        const long long d3 = 3LL * d;
        tn(x.dQKV, d3, map, x.Z1, d, map, dWqkv, d3 * d, 3 * d, d, M, G); // dWqkv = dQKV^T Z1
        nn(x.dQKV, d3, map, Wqkv, d3 * d, x.dZ1, d, map, M, d, 3 * d, G); // dZ1 = dQKV Wqkv
        const BwRows xr{Xin, map, M, G, d};
        k([&] { return bw_rms_bwd(xr, g1, ggs, x.r1, x.dZ1, dX, accumulate, st); });
        const int sp = bw_gain_splits(xr);
        k([&] { return bw_gain_grad(xr, x.r1, x.dZ1, partial, sp, dg1, ggs, st); });
        ++launches;
    }

    void backward(int l, const float *dXin, float *dXout, const float *dYin, float *dYout)
    {
        const int L = Ls[l], q = c.q[l];
        const long long R = RS(l), Tq = T(l);
        const long long d3 = 3LL * d, fd = static_cast<long long>(f) * d, dd = static_cast<long long>(d) * d;
        const long long ln = static_cast<long long>(l) * N;
        const RowMap nm = nmap();
        const int M = U * C;
        // FFN + output projection, both sides
        ffn_back(s, dXin, kIdentity, static_cast<int>(Tq), 1, wt(w->W1_s, l * fd), wt(w->W2_s, l * fd),
                 wt(w->Wo_s, l * dd), wt(w->g2_s, static_cast<long long>(l) * d), 0,
                 E ? nullptr : g->W1_s + l * fd, E ? nullptr : g->W2_s + l * fd, g->Wo_s + l * dd,
                 g->g2_s + static_cast<long long>(l) * d, E ? l : -1);
        if (C)
            ffn_back(n, dYin, nm, M, N, wt(w->W1_ns, ln * fd), wt(w->W2_ns, ln * fd), wt(w->Wo_ns, ln * dd),
                     wt(w->g2_ns, ln * d), d, g->W1_ns + ln * fd, g->W2_ns + ln * fd, g->Wo_ns + ln * dd,
                     g->g2_ns + ln * d);
        // attention
        zero(s.dQKV, static_cast<size_t>(R) * d3 * 4); // Q columns of the rows above the tail stay 0
        const BwAttn sa = attn_s(l);
        k([&] { return bw_attn_bwd_q(sa, st); });
        BwAttn na{};
        if (C) {
            na = attn_ns(l);
            k([&] { return bw_attn_bwd_q(na, st); });
        }
        k([&] { return bw_attn_bwd_kv_s(sa, C ? &na : nullptr, st); });
        if (C) k([&] { return bw_attn_bwd_kv_ns(na, c.full_attn ? &sa : nullptr, st); });
        // QKV + first norm; the residual adds dH to the tail rows
        qkv_back(s, X[l], kIdentity, static_cast<int>(R), 1, wt(w->Wqkv_s, l * d3 * d),
                 wt(w->g1_s, static_cast<long long>(l) * d), 0, g->Wqkv_s + l * d3 * d,
                 g->g1_s + static_cast<long long>(l) * d, dXout, 0);
        const RowMap tail{q, L, L - q, 0, 0};
        k([&] { return bw_rows_add(dXout, tail, s.dH, Tq, d, st); });
        if (C) {
            copy(dYout, n.dH, static_cast<size_t>(RN()) * d * 4);
            qkv_back(n, Y[l], nm, M, N, wt(w->Wqkv_ns, ln * d3 * d), wt(w->g1_ns, ln * d), d,
                     g->Wqkv_ns + ln * d3 * d, g->g1_ns + ln * d, dYout, 1);
        }
    }

    void run()
    {
        if (E) {
            // the dense S-side FFN is unused: its gradients are zero
            const long long fdL = static_cast<long long>(Lyr) * f * d * 4;
            if (g->W1_s) zero(g->W1_s, fdL);
            if (g->W2_s) zero(g->W2_s, fdL);
        }
        if (!C) {
            const long long fd = static_cast<long long>(f) * d, dd = static_cast<long long>(d) * d;
            const long long LN = static_cast<long long>(Lyr) * N;
            zero(g->Wqkv_ns, LN * 3 * dd * 4);
            zero(g->Wo_ns, LN * dd * 4);
            zero(g->W1_ns, LN * fd * 4);
            zero(g->W2_ns, LN * fd * 4);
            zero(g->g1_ns, LN * d * 4);
            zero(g->g2_ns, LN * d * 4);
        }
        // checkpointing forward: keep every layer's input rows
        for (int l = 0; l < Lyr; ++l) {
            const bool last = l == Lyr - 1;
            forward(l, last ? Xout_last : const_cast<float *>(X[l + 1]),
                    last ? Yout_last : const_cast<float *>(Y[l + 1]));
        }
        // backward, top layer first (its intermediates are still in place)
        for (int l = Lyr - 1; l >= 0; --l) {
            if (l != Lyr - 1) forward(l, nullptr, nullptr, true);
            const float *dXin = l == Lyr - 1 ? G_s : dXbuf[(l + 1) & 1];
            float *dXout = (l == 0 && dS) ? dS : dXbuf[l & 1];
            const float *dYin = !C ? nullptr : (l == Lyr - 1 ? G_ns : dYbuf[(l + 1) & 1]);
            float *dYout = !C ? nullptr : ((l == 0 && dns) ? dns : dYbuf[l & 1]);
            backward(l, dXin, dXout, dYin, dYout);
        }
    }
};

ot_status bw_validate(const ot_config *cfg, int U, int C)
{
    if (!cfg || U < 1 || C < 0) return OT_ERR_ARG;
    if (cfg->dtype != OT_DTYPE_F32) return OT_ERR_DTYPE;
    if (cfg->full_attn && C != 1) return OT_ERR_SHAPE; // one candidate per user, as the forward
    const ot_status r = internal_check_config(*cfg);
    if (r != OT_OK) return r;
    if (cfg->d / cfg->heads > 64) return OT_ERR_SHAPE;
    // GEMM rows stay below 2^31 / 64 (the grid's 65535 row tiles) and U * C fits an int
    const long long rs = static_cast<long long>(U) * cfg->L0, rn = static_cast<long long>(U) * C;
    if (rs > 65535LL * 64 || rn > 65535LL * 64) return OT_ERR_SHAPE;
    if (static_cast<long long>(C) * cfg->n_ns >= (1LL << 30)) return OT_ERR_SHAPE; // NS rows of a user: int
    return OT_OK;
}

void bw_init(Backward &b, const ot_config *cfg, int U, int C)
{
    b.c = *cfg;
    b.U = U, b.C = C, b.N = cfg->n_ns, b.d = cfg->d, b.f = cfg->ffn, b.H = cfg->heads;
    b.hd = cfg->d / cfg->heads, b.Lyr = cfg->layers;
    b.Ls[0] = cfg->L0;
    for (int l = 0; l < cfg->layers; ++l) b.Ls[l + 1] = cfg->q[l];
    b.E = cfg->moe_experts;
    b.K = cfg->moe_experts ? cfg->moe_topk : 0;
    b.launches = 0;
    b.err = cudaSuccess;
    b.bytes = 0;
}

} // namespace

extern "C" {

size_t ot_backward_workspace_bytes(const ot_config *cfg, int U, int C)
{
    if (bw_validate(cfg, U, C) != OT_OK) return 0;
    Backward b{};
    bw_init(b, cfg, U, C);
    b.dry = true;
    b.plan(nullptr, nullptr, nullptr, nullptr, nullptr);
    return b.bytes;
}

long long ot_backward_launches(const ot_config *cfg, int U, int C)
{
    if (bw_validate(cfg, U, C) != OT_OK) return 0;
    Backward b{};
    bw_init(b, cfg, U, C);
    b.dry = true;
    // the output pointers only decide whether the last layer's output GEMMs run
    static float dummy;
    b.plan(nullptr, nullptr, nullptr, &dummy, C ? &dummy : nullptr);
    const ot_weights w0{};
    const ot_grads g0{};
    b.w = &w0;
    b.g = &g0;
    b.run();
    return b.launches;
}

ot_status ot_full_backward(const ot_config *cfg, const ot_weights *w, const float *S, const float *ns, int U, int C,
                           const float *G_s, const float *G_ns, float *out_s_tail, float *out_ns, const ot_grads *g,
                           float *dS, float *dns, void *ws, size_t ws_bytes, void *stream)
{
    if (!cfg || !w || !g || !S || !G_s || !ws || U < 1 || C < 0) return OT_ERR_ARG;
    if (C && (!ns || !G_ns)) return OT_ERR_ARG;
    const bool moe = cfg->moe_experts > 0;
    const void *wp[] = {w->Wqkv_s,  w->Wo_s,   w->W1_s,  w->W2_s,  w->g1_s,   w->g2_s,
                        w->Wqkv_ns, w->Wo_ns,  w->W1_ns, w->W2_ns, w->g1_ns,  w->g2_ns,
                        w->W_router, w->W1_moe, w->W2_moe};
    const void *gp[] = {g->Wqkv_s,  g->Wo_s,   g->W1_s,  g->W2_s,  g->g1_s,   g->g2_s,
                        g->Wqkv_ns, g->Wo_ns,  g->W1_ns, g->W2_ns, g->g1_ns,  g->g2_ns,
                        g->W_router, g->W1_moe, g->W2_moe};
    // required: the dense twelve (W1_s / W2_s not with a mixture), the MoE three with one
    auto needed = [&](int i) { return i < 12 ? !(moe && (i == 2 || i == 3)) : moe; };
    for (int i = 0; i < 15; ++i)
        if (needed(i) && (!wp[i] || !gp[i])) return OT_ERR_ARG;
    const ot_status v = bw_validate(cfg, U, C);
    if (v != OT_OK) return v;
    auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    for (int i = 0; i < 15; ++i)
        if ((needed(i) || (i < 12 && gp[i])) && (!al(wp[i]) || !al(gp[i]))) return OT_ERR_ALIGN;
    if (!al(S) || !al(G_s) || !al(ws) || (C && (!al(ns) || !al(G_ns))) || (out_s_tail && !al(out_s_tail)) ||
        (C && out_ns && !al(out_ns)) || (dS && !al(dS)) || (C && dns && !al(dns)))
        return OT_ERR_ALIGN;
    Backward b{};
    bw_init(b, cfg, U, C);
    b.dry = false;
    b.plan(static_cast<char *>(ws), S, C ? ns : nullptr, out_s_tail, C ? out_ns : nullptr);
    if (b.bytes > ws_bytes) return OT_ERR_WORKSPACE_TOO_SMALL;
    b.st = static_cast<cudaStream_t>(stream);
    b.w = w;
    b.g = g;
    b.G_s = G_s;
    b.G_ns = C ? G_ns : nullptr;
    b.dS = dS;
    b.dns = C ? dns : nullptr;
    b.run();
    return b.err == cudaSuccess ? OT_OK : OT_ERR_CUDA;
}

} // extern "C"
