// Attention of the backward pass (fp32, CUDA cores), tiled in the order of
// the FlashAttention-2 backward: a forward per 64-row query block that keeps
// each row's softmax statistics (max m of the scores in base-2 units, sum l
// of 2^(s log2(e) - m); exponentials by ex2.approx), dQ per 64-row query block,
// and dK / dV per 64-key block, each CTA summing over the query blocks that
// see its keys — every output is written by exactly one CTA, so there are no
// atomics and the result is the same bit for bit run to run.
//
// Tiles: 64 x 64 scores per step in shared memory, 256 threads as 16 x 16,
// each with a 4 x 4 register block (4 rows x 4 keys) and, for the HD-wide
// products, 4 rows x HD / 16 columns.  Operands that a thread reads as 4
// consecutive rows or keys are stored transposed ([HD][64 + 4]).
//
// The key space of a query block of user u: the S keys 0 .. nks - 1 (rows of
// the layer's S QKV buffer), then, for NS queries, the NS keys of the
// candidates the block spans (rows of the NS QKV buffer).  Visibility: an S
// tail row t = L - nq + i sees S keys j <= t; an NS row sees every S key and
// the NS keys m <= n of its own candidate.  Full attention (one candidate
// per user): an S row sees every S key and every NS key of the user, an NS
// row every NS key of its candidate.
#include <math.h>
#include <stdint.h>

#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

namespace {

constexpr int TB = 64;      // query rows / keys per tile
constexpr int TP = TB + 4;  // pitch of transposed tiles (16-byte rows)
constexpr int NT = 256;     // threads
constexpr float LOG2E = 1.4426950408889634f;

struct KeySpace {
    int nks;      // S keys
    int nkn;      // NS keys
    int k_begin;  // first NS key row (within the user's NS rows, < 2^30)
};

// [64][64] tiles of P / dS, written as 4 x 4 blocks by the 16 x 16 threads
// and read as float4 rows: 16-byte chunk c of row r sits at chunk
// c ^ ((r / 4) % 8), so the 16 threads writing rows 4 tx + j of one column
// hit 8 different chunks (2-way instead of 8-way bank conflicts).
__device__ __forceinline__ int sw(int r, int k)
{
    return r * TB + ((((k >> 2) ^ ((r >> 2) & 7)) << 2) | (k & 3));
}

__device__ __forceinline__ long long q_row(const BwAttn &a, int u, int i)
{
    return static_cast<long long>(u) * a.q_ustride + a.q_off + i;
}

// keys of the query rows [i0, i1)
__device__ __forceinline__ KeySpace key_space(const BwAttn &a, int i0, int i1)
{
    KeySpace ks;
    if (a.mode == 0 && a.full) {
        ks.nks = a.L;
        ks.nkn = a.nkn; // every NS key of the user (its one candidate)
        ks.k_begin = 0;
    } else if (a.mode == 0) {
        ks.nks = min(a.L, a.L - a.nq + i1); // the last row sees keys 0 .. L - nq + i1 - 1
        ks.nkn = 0;
        ks.k_begin = 0;
    } else {
        const int c0 = i0 / a.N, c1 = (i1 - 1) / a.N + 1;
        ks.nks = a.L;
        ks.nkn = (c1 - c0) * a.N;
        ks.k_begin = c0 * a.N;
    }
    return ks;
}

__device__ __forceinline__ const float *key_row(const BwAttn &a, const KeySpace &ks, int u, int j)
{
    return j < ks.nks ? a.skv + (static_cast<long long>(u) * a.L + j) * a.ld
                      : a.nkv + (static_cast<long long>(u) * a.n_ustride + ks.k_begin + (j - ks.nks)) * a.ld;
}

__device__ __forceinline__ bool visible(const BwAttn &a, const KeySpace &ks, int i, int j)
{
    if (j < ks.nks) return a.full || a.mode == 1 || j <= a.L - a.nq + i;
    if (a.mode == 0) return true; // S rows meet NS keys only under full attention
    const int r = ks.k_begin + (j - ks.nks);
    const int c0 = (i / a.N) * a.N;
    return r >= c0 && (a.full ? r < c0 + a.N : r <= i); // same candidate (and m <= n)
}

// every (row, key) of rows [i0, i0 + 64) x keys [j0, j0 + 64) visible and
// every key valid (rows past the problem do not matter to the caller)
__device__ __forceinline__ bool block_full(const BwAttn &a, const KeySpace &ks, int i0, int j0)
{
    if (a.full && a.mode == 0) return j0 + TB <= ks.nks + ks.nkn;
    if (j0 + TB > ks.nks) return false; // reaches NS keys or past the S keys
    return a.full || a.mode == 1 || j0 + TB - 1 <= a.L - a.nq + i0;
}

__device__ __forceinline__ float half_warp_max(float v)
{
#pragma unroll
    for (int o = 8; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float half_warp_sum(float v)
{
#pragma unroll
    for (int o = 8; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

// rows [r0, r1) of a [.][HD] head slice -> T[c][r - r0] (zero past r1)
template <int HD, typename RowFn>
__device__ __forceinline__ void load_rows_t(float *T, int n, RowFn row)
{
    for (int e = threadIdx.x; e < TB * HD; e += NT) {
        const int r = e / HD, c = e % HD;
        T[c * TP + r] = r < n ? row(r)[c] : 0.f;
    }
}

// rows -> S[r][c] with pitch HD + 4
template <int HD, typename RowFn>
__device__ __forceinline__ void load_rows(float *S, int n, RowFn row)
{
    for (int e = threadIdx.x; e < TB * HD; e += NT) {
        const int r = e / HD, c = e % HD;
        S[r * (HD + 4) + c] = r < n ? row(r)[c] : 0.f;
    }
}

// acc[i][j] += sum_c A[c][a0 + i] B[c][b0 + j] over transposed tiles
template <int HD>
__device__ __forceinline__ void tile_dot(const float *A, int a0, const float *B, int b0, float (&acc)[4][4])
{
#pragma unroll 8
    for (int c = 0; c < HD; ++c) {
        const float4 x = ld4(A + c * TP + a0), y = ld4(B + c * TP + b0);
        const float xv[4] = {x.x, x.y, x.z, x.w}, yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xv[i], yv[j], acc[i][j]);
    }
}

template <int HD> constexpr int fwd_smem_floats() { return 2 * HD * TP + TB * (HD + 4) + TB * TB; }
template <int HD> constexpr int dq_smem_floats() { return 4 * HD * TP + TB * (HD + 4) + TB * TB + 3 * TB; }
template <int HD> constexpr int dkv_smem_floats() { return 4 * HD * TP + 2 * TB * (HD + 4) + 2 * TB * TB + 3 * TB; }

// ------------------------------------------------------------ forward
template <int HD>
__global__ void __launch_bounds__(NT) attn_fwd_tiled(BwAttn a, int n_qb)
{
    constexpr int CPT = HD / 16, VP = HD + 4;
    extern __shared__ __align__(16) float sm[];
    float *QT = sm, *KT = QT + HD * TP, *Vs = KT + HD * TP, *PT = Vs + TB * VP; // PT: [key][row], sw()
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const long long items = static_cast<long long>(a.U) * a.H * n_qb;
    for (long long item = blockIdx.x; item < items; item += gridDim.x) {
        const int qb = static_cast<int>(item % n_qb), h = static_cast<int>((item / n_qb) % a.H);
        const int u = static_cast<int>(item / n_qb / a.H);
        const int i0 = qb * TB, i1 = min(i0 + TB, a.nq);
        const KeySpace ks = key_space(a, i0, i1);
        const int nk = ks.nks + ks.nkn;
        __syncthreads(); // the previous item's readers are done
        load_rows_t<HD>(QT, i1 - i0, [&](int r) { return a.qkv + q_row(a, u, i0 + r) * a.ld + h * HD; });
        float m[4], l[4], o[4][CPT];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m[i] = -1e30f; // finite, so that fully masked blocks give corr = 1, p = 0
            l[i] = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) o[i][c] = 0.f;
        }
        const float c2 = a.scale * LOG2E; // scores in base-2 units
        for (int j0 = 0; j0 < nk; j0 += TB) {
            __syncthreads();
            for (int e = tid; e < TB * HD; e += NT) {
                const int kk = e / HD, c = e % HD, j = j0 + kk;
                float kv = 0.f, vv = 0.f;
                if (j < nk) {
                    const float *kr = key_row(a, ks, u, j) + h * HD + c;
                    kv = kr[a.d];
                    vv = kr[2 * a.d];
                }
                KT[c * TP + kk] = kv;
                Vs[kk * VP + c] = vv;
            }
            __syncthreads();
            float s[4][4] = {};
            tile_dot<HD>(QT, ty * 4, KT, tx * 4, s);
            const bool full = block_full(a, ks, i0, j0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int qi = i0 + ty * 4 + i;
                float bmax = -INFINITY;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int kj = j0 + tx * 4 + j;
                    const bool vis = full || (qi < i1 && kj < nk && visible(a, ks, qi, kj));
                    s[i][j] = vis ? s[i][j] * c2 : -INFINITY;
                    bmax = fmaxf(bmax, s[i][j]);
                }
                bmax = half_warp_max(bmax);
                const float mn = fmaxf(m[i], bmax), corr = fast_exp2(m[i] - mn);
                m[i] = mn;
                float ps = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float p = fast_exp2(s[i][j] - mn);
                    PT[sw(tx * 4 + j, ty * 4 + i)] = p;
                    ps += p;
                }
                l[i] = l[i] * corr + half_warp_sum(ps);
#pragma unroll
                for (int c = 0; c < CPT; ++c) o[i][c] *= corr;
            }
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < TB; ++kk) {
                const float4 p4 = ld4(PT + sw(kk, ty * 4));
                const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
                float v[CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c) v[c] = Vs[kk * VP + tx * CPT + c];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int c = 0; c < CPT; ++c) o[i][c] = fmaf(pv[i], v[c], o[i][c]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int qi = i0 + ty * 4 + i;
            if (qi >= i1) continue;
            const long long orow = static_cast<long long>(u) * a.nq + qi;
            float *op = a.O + orow * a.d + h * HD + tx * CPT;
#pragma unroll
            for (int c = 0; c < CPT; ++c) op[c] = o[i][c] / l[i];
            if (tx == 0) {
                a.stat_m[orow * a.H + h] = m[i];
                a.stat_l[orow * a.H + h] = l[i];
            }
        }
    }
}

// ------------------------------------------------------------ dQ
// D = rowsum(dO * O); dS = P (dO V^T - D) * scale; dQ = dS K.
template <int HD>
__global__ void __launch_bounds__(NT) attn_dq_tiled(BwAttn a, int n_qb)
{
    constexpr int CPT = HD / 16, VP = HD + 4;
    extern __shared__ __align__(16) float sm[];
    float *QT = sm, *dOT = QT + HD * TP, *KT = dOT + HD * TP, *VT = KT + HD * TP;
    float *Ks = VT + HD * TP, *dST = Ks + TB * VP, *sM = dST + TB * TB, *sL = sM + TB, *sD = sL + TB;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15, lane = tid & 31, warp = tid >> 5;
    const long long items = static_cast<long long>(a.U) * a.H * n_qb;
    for (long long item = blockIdx.x; item < items; item += gridDim.x) {
        const int qb = static_cast<int>(item % n_qb), h = static_cast<int>((item / n_qb) % a.H);
        const int u = static_cast<int>(item / n_qb / a.H);
        const int i0 = qb * TB, i1 = min(i0 + TB, a.nq), n = i1 - i0;
        const KeySpace ks = key_space(a, i0, i1);
        const int nk = ks.nks + ks.nkn;
        const long long orow0 = static_cast<long long>(u) * a.nq + i0;
        __syncthreads();
        load_rows_t<HD>(QT, n, [&](int r) { return a.qkv + q_row(a, u, i0 + r) * a.ld + h * HD; });
        load_rows_t<HD>(dOT, n, [&](int r) { return a.dO + (orow0 + r) * a.d + h * HD; });
        for (int r = warp; r < TB; r += NT / 32) { // D per row, one warp per row
            float dsum = 0.f;
            if (r < n)
                for (int c = lane; c < HD; c += 32)
                    dsum = fmaf(a.dO[(orow0 + r) * a.d + h * HD + c], a.O[(orow0 + r) * a.d + h * HD + c], dsum);
#pragma unroll
            for (int o = 16; o; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
            if (lane == 0) {
                const long long st = (orow0 + r) * a.H + h;
                sD[r] = dsum;
                sM[r] = r < n ? a.stat_m[st] : 0.f;
                sL[r] = r < n ? 1.0f / a.stat_l[st] : 1.f; // 1 / l
                if (r < n) a.stat_D[st] = dsum;
            }
        }
        float dq[4][CPT];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < CPT; ++c) dq[i][c] = 0.f;
        for (int j0 = 0; j0 < nk; j0 += TB) {
            __syncthreads();
            for (int e = tid; e < TB * HD; e += NT) {
                const int kk = e / HD, c = e % HD, j = j0 + kk;
                float kv = 0.f, vv = 0.f;
                if (j < nk) {
                    const float *kr = key_row(a, ks, u, j) + h * HD + c;
                    kv = kr[a.d];
                    vv = kr[2 * a.d];
                }
                KT[c * TP + kk] = kv;
                VT[c * TP + kk] = vv;
                Ks[kk * VP + c] = kv;
            }
            __syncthreads();
            float s[4][4] = {}, dp[4][4] = {};
            tile_dot<HD>(QT, ty * 4, KT, tx * 4, s);
            tile_dot<HD>(dOT, ty * 4, VT, tx * 4, dp);
            const bool full = block_full(a, ks, i0, j0);
            const float c2 = a.scale * LOG2E;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = ty * 4 + i, qi = i0 + r;
                const float mr = sM[r], il = sL[r], dr = sD[r];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int kj = j0 + tx * 4 + j;
                    float ds = 0.f;
                    if (full || (qi < i1 && kj < nk && visible(a, ks, qi, kj))) {
                        const float p = fast_exp2(s[i][j] * c2 - mr) * il;
                        ds = p * (dp[i][j] - dr) * a.scale;
                    }
                    dST[sw(tx * 4 + j, r)] = ds;
                }
            }
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < TB; ++kk) {
                const float4 d4 = ld4(dST + sw(kk, ty * 4));
                const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
                float kv[CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c) kv[c] = Ks[kk * VP + tx * CPT + c];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int c = 0; c < CPT; ++c) dq[i][c] = fmaf(dv[i], kv[c], dq[i][c]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int qi = i0 + ty * 4 + i;
            if (qi >= i1) continue;
            float *dp = a.dqkv + q_row(a, u, qi) * a.ld + h * HD + tx * CPT;
#pragma unroll
            for (int c = 0; c < CPT; ++c) dp[c] = dq[i][c];
        }
    }
}

// ------------------------------------------------------------ dK, dV
// One CTA per 64-key block (kind 0: the layer's S keys of a user, seen by the
// query problems p0 (S tail) and p1 (NS rows, if n_prob == 2); kind 1: NS
// keys of a user, seen by p0 = the NS rows of the same candidates).
// dV = P^T dO, dK = dS^T Q over every query block that sees the keys.
template <int HD>
__global__ void __launch_bounds__(NT) attn_dkv_tiled(BwAttn p0, BwAttn p1, int n_prob, int kind, int n_kb)
{
    constexpr int CPT = HD / 16, VP = HD + 4;
    extern __shared__ __align__(16) float sm[];
    float *KT = sm, *VT = KT + HD * TP, *QT = VT + HD * TP, *dOT = QT + HD * TP;
    float *Qs = dOT + HD * TP, *dOs = Qs + TB * VP, *PS = dOs + TB * VP, *dSs = PS + TB * TB;
    float *sM = dSs + TB * TB, *sL = sM + TB, *sD = sL + TB;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int nkeys = kind == 0 ? p0.L : p0.nq;
    const KeySpace ks{kind == 0 ? p0.L : 0, kind == 0 ? 0 : p0.nq, 0};
    const long long items = static_cast<long long>(p0.U) * p0.H * n_kb;
    for (long long item = blockIdx.x; item < items; item += gridDim.x) {
        const int kb = static_cast<int>(item % n_kb), h = static_cast<int>((item / n_kb) % p0.H);
        const int u = static_cast<int>(item / n_kb / p0.H);
        const int j0 = kb * TB, j1 = min(j0 + TB, nkeys);
        __syncthreads();
        for (int e = tid; e < TB * HD; e += NT) {
            const int kk = e / HD, c = e % HD, j = j0 + kk;
            float kv = 0.f, vv = 0.f;
            if (j < j1) {
                const float *kr = key_row(p0, ks, u, j) + h * HD + c;
                kv = kr[p0.d];
                vv = kr[2 * p0.d];
            }
            KT[c * TP + kk] = kv;
            VT[c * TP + kk] = vv;
        }
        float dk[4][CPT], dv[4][CPT];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < CPT; ++c) dk[i][c] = dv[i][c] = 0.f;
        for (int pi = 0; pi < n_prob; ++pi) {
            const BwAttn &P = pi == 0 ? p0 : p1;
            // the query rows that can see a key of [j0, j1)
            int qa, qe;
            if (kind == 1 && P.mode == 1) {
                qa = (j0 / P.N) * P.N; // the candidates of the keys
                qe = min(P.nq, ((j1 - 1) / P.N + 1) * P.N);
            } else if (kind == 0 && P.mode == 0 && !P.full) {
                qa = max(0, j0 - (P.L - P.nq)); // tail rows at or after the keys
                qe = P.nq;
            } else {
                qa = 0;
                qe = P.nq;
            }
            for (int i0 = qa; i0 < qe; i0 += TB) {
                const int n = min(TB, qe - i0);
                const long long orow0 = static_cast<long long>(u) * P.nq + i0;
                __syncthreads();
                load_rows_t<HD>(QT, n, [&](int r) { return P.qkv + q_row(P, u, i0 + r) * P.ld + h * HD; });
                load_rows<HD>(Qs, n, [&](int r) { return P.qkv + q_row(P, u, i0 + r) * P.ld + h * HD; });
                load_rows_t<HD>(dOT, n, [&](int r) { return P.dO + (orow0 + r) * P.d + h * HD; });
                load_rows<HD>(dOs, n, [&](int r) { return P.dO + (orow0 + r) * P.d + h * HD; });
                for (int r = tid; r < TB; r += NT) {
                    const long long st = (orow0 + r) * P.H + h;
                    sM[r] = r < n ? P.stat_m[st] : 0.f;
                    sL[r] = r < n ? 1.0f / P.stat_l[st] : 1.f; // 1 / l
                    sD[r] = r < n ? P.stat_D[st] : 0.f;
                }
                __syncthreads();
                // thread: keys ty*4 + i, query rows tx*4 + j.  Rows past n
                // hold Q = dO = 0 and D = 0: their p multiplies dO = 0 and
                // their dS is 0, so only the mask needs them
                float s[4][4] = {}, dp[4][4] = {};
                tile_dot<HD>(KT, ty * 4, QT, tx * 4, s);
                tile_dot<HD>(VT, ty * 4, dOT, tx * 4, dp);
                const bool full =
                    n == TB && (kind == 0 ? (P.mode == 1 || P.full || j0 + TB - 1 <= P.L - P.nq + i0)
                                          : P.mode == 0); // NS keys of S rows: full attention only
                const float c2 = P.scale * LOG2E;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = tx * 4 + j, qi = i0 + r;
                    const float mr = sM[r], il = sL[r], dr = sD[r];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int kj = j0 + ty * 4 + i;
                        float p = 0.f, ds = 0.f;
                        if (full || (r < n && kj < j1 && visible(P, ks, qi, kj))) {
                            p = fast_exp2(s[i][j] * c2 - mr) * il;
                            ds = p * (dp[i][j] - dr) * P.scale;
                        }
                        PS[sw(r, ty * 4 + i)] = p;
                        dSs[sw(r, ty * 4 + i)] = ds;
                    }
                }
                __syncthreads();
#pragma unroll 4
                for (int r = 0; r < TB; ++r) {
                    const float4 p4 = ld4(PS + sw(r, ty * 4)), d4 = ld4(dSs + sw(r, ty * 4));
                    const float pv[4] = {p4.x, p4.y, p4.z, p4.w}, dsv[4] = {d4.x, d4.y, d4.z, d4.w};
                    float qv[CPT], ov[CPT];
#pragma unroll
                    for (int c = 0; c < CPT; ++c) {
                        qv[c] = Qs[r * VP + tx * CPT + c];
                        ov[c] = dOs[r * VP + tx * CPT + c];
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int c = 0; c < CPT; ++c) {
                            dv[i][c] = fmaf(pv[i], ov[c], dv[i][c]);
                            dk[i][c] = fmaf(dsv[i], qv[c], dk[i][c]);
                        }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = j0 + ty * 4 + i;
            if (j >= j1) continue;
            float *dr = kind == 0 ? p0.dskv + (static_cast<long long>(u) * p0.L + j) * p0.ld
                                  : p0.dqkv + (static_cast<long long>(u) * p0.q_ustride + j) * p0.ld;
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                dr[p0.d + h * HD + tx * CPT + c] = dk[i][c];
                dr[2 * p0.d + h * HD + tx * CPT + c] = dv[i][c];
            }
        }
    }
}

int tiled_grid(long long items)
{
    const long long g = items < 148LL * 16 ? items : 148LL * 16;
    return g < 1 ? 1 : static_cast<int>(g);
}

template <typename K> cudaError_t smem_opt_in(K kernel, int floats)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                floats * static_cast<int>(sizeof(float)));
}

template <int HD> cudaError_t fwd_launch(const BwAttn &a, cudaStream_t s)
{
    const int n_qb = (a.nq + TB - 1) / TB;
    cudaError_t e = smem_opt_in(attn_fwd_tiled<HD>, fwd_smem_floats<HD>());
    if (e != cudaSuccess) return e;
    attn_fwd_tiled<HD><<<tiled_grid(static_cast<long long>(a.U) * a.H * n_qb), NT,
                         fwd_smem_floats<HD>() * sizeof(float), s>>>(a, n_qb);
    return cudaGetLastError();
}

template <int HD> cudaError_t dq_launch(const BwAttn &a, cudaStream_t s)
{
    const int n_qb = (a.nq + TB - 1) / TB;
    cudaError_t e = smem_opt_in(attn_dq_tiled<HD>, dq_smem_floats<HD>());
    if (e != cudaSuccess) return e;
    attn_dq_tiled<HD><<<tiled_grid(static_cast<long long>(a.U) * a.H * n_qb), NT,
                        dq_smem_floats<HD>() * sizeof(float), s>>>(a, n_qb);
    return cudaGetLastError();
}

template <int HD> cudaError_t dkv_launch(const BwAttn &p0, const BwAttn &p1, int n_prob, int kind, cudaStream_t s)
{
    const int nkeys = kind == 0 ? p0.L : p0.nq;
    const int n_kb = (nkeys + TB - 1) / TB;
    cudaError_t e = smem_opt_in(attn_dkv_tiled<HD>, dkv_smem_floats<HD>());
    if (e != cudaSuccess) return e;
    attn_dkv_tiled<HD><<<tiled_grid(static_cast<long long>(p0.U) * p0.H * n_kb), NT,
                         dkv_smem_floats<HD>() * sizeof(float), s>>>(p0, p1, n_prob, kind, n_kb);
    return cudaGetLastError();
}

} // namespace

cudaError_t bw_attn_fwd(const BwAttn &a, cudaStream_t s)
{
    switch (a.hd) {
    case 16: return fwd_launch<16>(a, s);
    case 32: return fwd_launch<32>(a, s);
    case 64: return fwd_launch<64>(a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t bw_attn_bwd_q(const BwAttn &a, cudaStream_t s)
{
    switch (a.hd) {
    case 16: return dq_launch<16>(a, s);
    case 32: return dq_launch<32>(a, s);
    case 64: return dq_launch<64>(a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t bw_attn_bwd_kv_s(const BwAttn &sq, const BwAttn *nsq, cudaStream_t s)
{
    const BwAttn &p1 = nsq ? *nsq : sq;
    const int n_prob = nsq ? 2 : 1;
    switch (sq.hd) {
    case 16: return dkv_launch<16>(sq, p1, n_prob, 0, s);
    case 32: return dkv_launch<32>(sq, p1, n_prob, 0, s);
    case 64: return dkv_launch<64>(sq, p1, n_prob, 0, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t bw_attn_bwd_kv_ns(const BwAttn &a, const BwAttn *sq, cudaStream_t s)
{
    const BwAttn &p1 = sq ? *sq : a;
    const int n_prob = sq ? 2 : 1;
    switch (a.hd) {
    case 16: return dkv_launch<16>(a, p1, n_prob, 1, s);
    case 32: return dkv_launch<32>(a, p1, n_prob, 1, s);
    case 64: return dkv_launch<64>(a, p1, n_prob, 1, s);
    }
    return cudaErrorInvalidValue;
}

} // namespace ot
