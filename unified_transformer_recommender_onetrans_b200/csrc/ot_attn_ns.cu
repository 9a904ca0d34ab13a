// NS attention when every NS query row of a user fits in 64 (C N <= 64; the
// dispatcher uses it up to 16, e.g. the full forward at C = 1): query i = NS token i % N
// of candidate i / N sees all L cached S keys of the layer and the NS keys
// m <= i % N of its own candidate (the OneTrans mask; with full attention
// every NS key of its candidate).  head_dim 64, bf16
// operands, fp32 scores, softmax and accumulation.
//
// With a handful of query rows a 128-row tensor-memory tile would hold mostly
// padding and pay the full per-block latency chain of the tiled kernel.  Here
// the work is decode-shaped instead: one CTA per (user, head), four warps.
// A warp owns one 16-row query tile and a share of the 32-key blocks (tile
// w % MT, keys b = w / MT (mod KS) with MT x KS = 4), streams its K / V blocks
// through a private 3-deep TMA ring (two CTAs fit an SM, so every CTA of a
// layer is resident at once and their load latencies overlap) and keeps
// everything else in registers:
//   S = Q K^T       m16n8k16 MMAs, Q and K fragments by ldmatrix from the
//                   128-byte-swizzled tiles
//   softmax         online, per row: the 4 lanes of a row agree on the max by
//                   two shuffles; p = 2^(s log2e / sqrt(hd) - m)
//   O += P V        P re-used in registers as the A fragments, V by
//                   transposing ldmatrix
// At the end the warps of one query tile merge their partial (max, sum, O)
// in shared memory and write O / sum as bf16.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int NA_WARPS = 4;
constexpr int NA_KB = 32;                         // keys per block
constexpr int NA_NT = NA_KB / 8;                  // 8-key column tiles of a block (S = Q K^T)
constexpr int NA_KS = NA_KB / 16;                 // 16-key steps of a block (O += P V)
constexpr int NA_HD = 64;
constexpr int NA_MAXQ = 64;                       // query rows per (user, head) the kernel handles
constexpr int NA_MAXQ_FAST = 16;                  // ... and where it beats the tensor-memory kernel
constexpr int NA_STAGES = 3;                      // K / V ring depth per warp
constexpr uint32_t NA_TILE = NA_KB * 128;         // NA_KB rows x 128 bytes
constexpr uint32_t NA_STAGE = 2 * NA_TILE;        // K and V
constexpr uint32_t NA_Q_BYTES = NA_MAXQ * 128;
constexpr size_t NA_BAR_BYTES = 256;
constexpr size_t NA_SMEM = 1024 + NA_Q_BYTES + NA_WARPS * NA_STAGES * NA_STAGE + NA_BAR_BYTES;
static_assert(2 * NA_SMEM <= 227 * 1024, "two CTAs per SM");
static_assert((1 + NA_WARPS * NA_STAGES) * 8 <= NA_BAR_BYTES, "barrier area");
// merge area (re-uses the rings once every warp is done): O [warp][16][64]
// fp32, then max and sum [warp][16]
static_assert(NA_WARPS * 16 * (NA_HD + 2) * 4 <= NA_WARPS * NA_STAGES * NA_STAGE, "merge area");

struct NsAttnParams {
    AttnArgs a;
    int mt;    // query tiles of 16 rows (1, 2 or 4)
    int ks;    // key splits (4 / mt)
    int nb_s;  // S key blocks
    int nb;    // S + NS key blocks
};

// byte offset of 16-byte chunk c of row r in a [rows][128 B] tile written by
// TMA with the 128-byte swizzle (1024-byte aligned base)
__device__ __forceinline__ uint32_t sw_off(int r, int c)
{
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D (16 x 8, fp32) += A (16 x 16, bf16, row) B (16 x 8, bf16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(NA_WARPS * 32, 2)
    attn_ns_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKS,
                   const __grid_constant__ CUtensorMap tmVS, const __grid_constant__ CUtensorMap tmKN,
                   const __grid_constant__ CUtensorMap tmVN, const __grid_constant__ NsAttnParams P)
{
    const AttnArgs &a = P.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sQ = smem;                                  // [64 rows][128 B]
    uint8_t *sKV = sQ + NA_Q_BYTES;                      // [warp][stage][K | V]
    uint64_t *q_full = reinterpret_cast<uint64_t *>(sKV + NA_WARPS * NA_STAGES * NA_STAGE);
    uint64_t *kv_full = q_full + 1;                      // [warp][stage]
    float *mo = reinterpret_cast<float *>(sKV);          // merge: O [warp][16][64]
    float *mm = mo + NA_WARPS * 16 * NA_HD;              // merge: max [warp][16]
    float *ml = mm + NA_WARPS * 16;                      // merge: sum [warp][16]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = static_cast<int>(blockIdx.x) / a.H, h = static_cast<int>(blockIdx.x) % a.H;
    const int mt = warp % P.mt, ks = warp / P.mt;        // query tile, key split
    const int g = lane >> 2, t = lane & 3;               // fragment row group / column pair
    const int nloc = ks < P.ks && ks < P.nb ? (P.nb - ks + P.ks - 1) / P.ks : 0; // this warp's blocks
    volatile int no_abort = 0, aborted = 0;
    volatile int *abort_flag = &aborted;
    // waits at the end ignore the abort flag and never use a test-lowered limit
    const WaitCtl final_wait{a.wait.err, a.wait.limit > (1LL << 24) ? a.wait.limit : (1LL << 24)};
    int issued = 0; // blocks this warp's lane 0 has issued

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < NA_WARPS * NA_STAGES; ++i) mbar_init(&kv_full[i], 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait(); // Q, K, V come from the previous kernels

    // block i of this warp into ring stage s
    auto issue = [&](int i, int s) {
        const int b = ks + i * P.ks;
        uint8_t *k_dst = sKV + (warp * NA_STAGES + s) * NA_STAGE, *v_dst = k_dst + NA_TILE;
        uint64_t *bar = &kv_full[warp * NA_STAGES + s];
        ++issued;
        mbar_arrive_expect_tx(bar, NA_STAGE);
        if (b < P.nb_s && a.pages) {
            // paged cache: block b lies in page b / (OT_PAGE_ROWS / NA_KB)
            constexpr int per = OT_PAGE_ROWS / NA_KB;
            const int pg = static_cast<int>(attn_page(a, u, b / per));
            tma_load_3d(k_dst, &tmKS, bar, h * NA_HD, (b % per) * NA_KB, 2 * pg);
            tma_load_3d(v_dst, &tmVS, bar, h * NA_HD, (b % per) * NA_KB, 2 * pg + 1);
        } else if (b < P.nb_s) {
            tma_load_3d(k_dst, &tmKS, bar, h * NA_HD, b * NA_KB, u);
            tma_load_3d(v_dst, &tmVS, bar, h * NA_HD, b * NA_KB, u);
        } else {
            tma_load_3d(k_dst, &tmKN, bar, h * NA_HD, (b - P.nb_s) * NA_KB, u);
            tma_load_3d(v_dst, &tmVN, bar, h * NA_HD, (b - P.nb_s) * NA_KB, u);
        }
    };
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(q_full, NA_Q_BYTES);
        tma_load_3d(sQ, &tmQ, q_full, h * NA_HD, 0, u);
    }
    if (lane == 0)
        for (int i = 0; i < nloc && i < NA_STAGES; ++i) issue(i, i);

    float o[8][4];    // O: 8 column tiles of 8 dims, rows g and g + 8
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    const float c2 = a.scale * 1.4426950408889634f;
    const int r_lo = mt * 16 + g, r_hi = r_lo + 8;   // this thread's query rows
    const int cand[2] = {r_lo / a.N, r_hi / a.N}, tok[2] = {r_lo % a.N, r_hi % a.N};
    bool ok = nloc > 0, q_seen = false;
    uint32_t qf[4][4]; // Q fragments, one per 16 dims
    if (ok) {
        ok = q_seen = mbar_wait(q_full, 0, a.wait, abort_flag);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, chunk = 2 * kk + (lane >> 4);
            ldsm_x4(smem_u32(sQ) + sw_off(row, chunk), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
    }
    int waited = 0; // blocks whose data this warp has seen
    for (int i = 0; ok && i < nloc; ++i) {
        const int s = i % NA_STAGES;
        if (!mbar_wait(&kv_full[warp * NA_STAGES + s], static_cast<uint32_t>((i / NA_STAGES) & 1), a.wait,
                       abort_flag)) {
            ok = false;
            break;
        }
        waited = i + 1;
        const int b = ks + i * P.ks;
        const uint32_t k_base = smem_u32(sKV + (warp * NA_STAGES + s) * NA_STAGE), v_base = k_base + NA_TILE;
        // S = Q K^T: NA_NT column tiles of 8 keys
        float sc[NA_NT][4];
#pragma unroll
        for (int n = 0; n < NA_NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int n = 0; n < NA_NT; n += 2) {
                uint32_t b0, b1, b2, b3;
                const int key = (n + (lane >> 4)) * 8 + (lane & 7), chunk = 2 * kk + ((lane >> 3) & 1);
                ldsm_x4(k_base + sw_off(key, chunk), b0, b1, b2, b3);
                mma_16816(sc[n], qf[kk], b0, b1);
                mma_16816(sc[n + 1], qf[kk], b2, b3);
            }
        // mask, scale to base 2, block row max
        const bool s_block = b < P.nb_s;
        const int j0 = s_block ? b * NA_KB : (b - P.nb_s) * NA_KB;
        float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < NA_NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hi = e >> 1, key = j0 + n * 8 + 2 * t + (e & 1);
                const bool vis = s_block ? key < a.L
                                         : (key < a.nq && key / a.N == cand[hi] &&
                                            (a.full || key % a.N <= tok[hi]));
                sc[n][e] = vis ? sc[n][e] * c2 : -INFINITY;
                bm[hi] = fmaxf(bm[hi], sc[n][e]);
            }
        float alpha[2];
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            bm[hi] = fmaxf(bm[hi], __shfl_xor_sync(0xffffffffu, bm[hi], 1));
            bm[hi] = fmaxf(bm[hi], __shfl_xor_sync(0xffffffffu, bm[hi], 2));
            const float mn = fmaxf(mrow[hi], bm[hi]);
            // a row with nothing visible yet keeps O = 0, sum = 0
            alpha[hi] = mn == -INFINITY ? 1.f : fast_exp2(mrow[hi] - mn);
            mrow[hi] = mn;
        }
        // P = 2^(s - m), packed as the A fragments of the PV MMAs
        uint32_t pf[NA_KS][4];
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < NA_NT; ++n) {
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hi = e >> 1;
                p[e] = mrow[hi] == -INFINITY ? 0.f : fast_exp2(sc[n][e] - mrow[hi]);
                rs[hi] += p[e];
            }
            // keys 16 (n/2) ..: tile n even -> a0 (row g), a1 (row g+8); odd -> a2, a3
            pf[n >> 1][(n & 1) * 2] = pack_bf16x2(p[0], p[1]);
            pf[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(p[2], p[3]);
        }
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) lrow[hi] = lrow[hi] * alpha[hi] + rs[hi];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            o[n][0] *= alpha[0];
            o[n][1] *= alpha[0];
            o[n][2] *= alpha[1];
            o[n][3] *= alpha[1];
        }
        // O += P V: NA_KS steps of 16 keys, 8 column tiles of 8 dims
#pragma unroll
        for (int kk = 0; kk < NA_KS; ++kk)
#pragma unroll
            for (int n = 0; n < 8; n += 2) {
                uint32_t b0, b1, b2, b3;
                const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, chunk = n + (lane >> 4);
                ldsm_x4_t(v_base + sw_off(key, chunk), b0, b1, b2, b3);
                mma_16816(o[n], pf[kk], b0, b1);
                mma_16816(o[n + 1], pf[kk], b2, b3);
            }
        // the stage is refilled by TMA (async proxy) once every lane has read it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && i + NA_STAGES < nloc) issue(i + NA_STAGES, s);
    }
    // sums: the 4 lanes of a row hold partial sums
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        lrow[hi] += __shfl_xor_sync(0xffffffffu, lrow[hi], 1);
        lrow[hi] += __shfl_xor_sync(0xffffffffu, lrow[hi], 2);
    }
    // never leave a load in flight (only after a timed-out wait is anything left)
    if (lane == 0)
        for (int j = waited; j < issued; ++j)
            mbar_wait(&kv_full[warp * NA_STAGES + j % NA_STAGES], static_cast<uint32_t>((j / NA_STAGES) & 1),
                      final_wait, &no_abort);
    if (threadIdx.x == 0 && !q_seen) mbar_wait(q_full, 0, final_wait, &no_abort);
    // every warp is done with its ring before the merge area overwrites it
    __syncthreads();
    if (nloc > 0) {
        float *ow = mo + warp * 16 * NA_HD;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            *reinterpret_cast<float2 *>(ow + g * NA_HD + n * 8 + 2 * t) = make_float2(o[n][0], o[n][1]);
            *reinterpret_cast<float2 *>(ow + (g + 8) * NA_HD + n * 8 + 2 * t) = make_float2(o[n][2], o[n][3]);
        }
        if (t == 0) {
            mm[warp * 16 + g] = ok ? mrow[0] : -INFINITY;
            mm[warp * 16 + g + 8] = ok ? mrow[1] : -INFINITY;
            ml[warp * 16 + g] = lrow[0];
            ml[warp * 16 + g + 8] = lrow[1];
        }
    } else if (lane < 16) {
        mm[warp * 16 + lane] = -INFINITY; // no keys: contributes nothing
        ml[warp * 16 + lane] = 0.f;
    }
    __syncthreads();
    // merge the key splits of each query row; 8 output columns per thread
    for (int idx = threadIdx.x; idx < a.nq * (NA_HD / 8); idx += NA_WARPS * 32) {
        const int row = idx >> 3, c8 = idx & 7, tile = row >> 4, r = row & 15;
        float mx = -INFINITY;
        for (int k = 0; k < P.ks; ++k) mx = fmaxf(mx, mm[(k * P.mt + tile) * 16 + r]);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, sum = 0.f;
        for (int k = 0; k < P.ks; ++k) {
            const int w = k * P.mt + tile;
            const float mk = mm[w * 16 + r];
            if (mk == -INFINITY) continue;
            const float f = fast_exp2(mk - mx);
            sum += ml[w * 16 + r] * f;
            const float4 *src = reinterpret_cast<const float4 *>(mo + (w * 16 + r) * NA_HD + c8 * 8);
            const float4 x0 = src[0], x1 = src[1];
            acc[0] += x0.x * f;
            acc[1] += x0.y * f;
            acc[2] += x0.z * f;
            acc[3] += x0.w * f;
            acc[4] += x1.x * f;
            acc[5] += x1.y * f;
            acc[6] += x1.z * f;
            acc[7] += x1.w * f;
        }
        const float inv = 1.f / sum;
        uint4 out;
        out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        out.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
        out.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
        const long long o_off = (static_cast<long long>(u) * a.nq + row) * a.d + h * NA_HD + c8 * 8;
        if (a.o_qscale) {
            // e4m3 output: the bf16 values quantised with the O projection's input scale
            const float qi = __frcp_rn(a.o_qscale[static_cast<long long>(row % a.N) * a.o_qstride]);
            const uint2 q8 = make_uint2(static_cast<uint32_t>(bf16x2_to_e4m3x2(out.x, qi)) |
                                            (static_cast<uint32_t>(bf16x2_to_e4m3x2(out.y, qi)) << 16),
                                        static_cast<uint32_t>(bf16x2_to_e4m3x2(out.z, qi)) |
                                            (static_cast<uint32_t>(bf16x2_to_e4m3x2(out.w, qi)) << 16));
            if (ot_dev_ok(o_off, 8, a.o_cap, a.wait.err))
                *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(a.O) + o_off) = q8;
        } else if (ot_dev_ok(o_off * 2, 16, a.o_cap, a.wait.err)) {
            *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.O) + o_off) = out;
        }
    }
}

bool attn_ns_small_supported(const AttnArgs &a)
{
    // bf16 operands (the e4m3 models keep bf16 activations and caches).  Only
    // up to 16 rows, where all four warps split the keys: with 2-4 query
    // tiles each warp walks half or all of the keys alone and the tensor-memory
    // kernel's split-key mode is faster (C sweep: 32 rows 0.368 ms, 64 rows
    // 0.505 ms against 0.319 ms at 128 rows on tcgen05)
    return a.mode == 1 && a.hd == NA_HD && (a.dtype == OT_DTYPE_BF16 || a.dtype == OT_DTYPE_FP8) &&
           a.nq >= 1 && a.nq <= NA_MAXQ_FAST &&
           a.N >= 1 && a.L >= 0 && a.U >= 1 && a.H >= 1;
}

// boxes of 64 columns (one head) x box_rows rows
static int tmap_ns(CUtensorMap *m, const void *base, long long d, long long rows, long long users,
                   long long ustride_elems, uint32_t box_rows)
{
    uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows), static_cast<uint64_t>(users)};
    uint64_t str[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(ustride_elems) * 2};
    uint32_t box[3] = {NA_HD, box_rows, 1};
    return encode_tmap_3d(m, 2, base, dims, str, box);
}

cudaError_t launch_attn_ns_small(const AttnArgs &a, cudaStream_t s)
{
    if (!attn_ns_small_supported(a)) return cudaErrorInvalidValue;
    NsAttnParams p;
    memset(&p, 0, sizeof(p));
    p.a = a;
    p.mt = a.nq <= 16 ? 1 : a.nq <= 32 ? 2 : 4;
    p.ks = NA_WARPS / p.mt;
    p.nb_s = (a.L + NA_KB - 1) / NA_KB;
    p.nb = p.nb_s + (a.nq + NA_KB - 1) / NA_KB;
    alignas(64) CUtensorMap tq, tks, tvs, tkn, tvn;
    const long long nqd = static_cast<long long>(a.nq) * a.d;
    // Q: all (up to 64) rows in one box, NA_Q_BYTES; K / V: one block per box, NA_TILE
    if (tmap_ns(&tq, a.Q, a.d, a.nq, a.U, nqd, NA_MAXQ) || tmap_ns(&tkn, a.KN, a.d, a.nq, a.U, nqd, NA_KB) ||
        tmap_ns(&tvn, a.VN, a.d, a.nq, a.U, nqd, NA_KB))
        return cudaErrorInvalidValue;
    if (a.L > 0 && a.pages) {
        // paged cache: (d, OT_PAGE_ROWS rows, 2 n_pages), K / V of page p at 2 p / 2 p + 1
        if (a.n_pages < 1 || 2 * a.n_pages > (1LL << 31) - 1 ||
            tmap_ns(&tks, a.KS, a.d, OT_PAGE_ROWS, 2 * a.n_pages, static_cast<long long>(OT_PAGE_ROWS) * a.d,
                    NA_KB))
            return cudaErrorInvalidValue;
        tvs = tks;
    } else if (a.L > 0) {
        if (tmap_ns(&tks, a.KS, a.d, a.L, a.U, a.s_ustride, NA_KB) ||
            tmap_ns(&tvs, a.VS, a.d, a.L, a.U, a.s_ustride, NA_KB))
            return cudaErrorInvalidValue;
    } else { // no S keys: the S maps are never read
        tks = tkn;
        tvs = tvn;
    }
    const long long ctas = static_cast<long long>(a.U) * a.H;
    if (ctas > (1LL << 31) - 1) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_ns_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(NA_SMEM));
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_ns_kernel, dim3(static_cast<unsigned>(ctas)), dim3(NA_WARPS * 32), NA_SMEM, s,
                      tq, tks, tvs, tkn, tvn, p);
}

} // namespace ot
