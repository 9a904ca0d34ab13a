// Fused feed-forward of the block: Y = H + GELU(n(H) W1^T) W2^T with the
// RMSNorm gain folded into W1, bf16 operands, fp32 accumulation in TMEM.  The
// hidden activation (4d wide) never leaves the SM: per 128-row tile it is
// produced 128 columns at a time, passed through the norm row scale and GELU
// into shared memory as bf16, and consumed there by the second projection,
// whose accumulator covers the whole output row.
//
// Persistent: one CTA per SM walks 128-row tiles (group-major: a group is an
// NS position with its own weights, or the single shared S-side group).
//   warp 0      TMA: the tile's H rows (D / 64 slabs of [128 rows][128 B],
//               128-byte swizzle), then per hidden chunk c the W1 rows
//               c*128 .. c*128+127 (two slabs per stage).
//   warp 3      TMA: per hidden chunk the W2 columns of the chunk (one
//               [D rows][64 hidden] slab per stage).  Every stage of the ring
//               has one fixed role.
//   warp 1      MMA issuer of FFN1: acc1[c % 2] = H W1_c^T (128 x 128, TMEM
//               columns D + 128 (c % 2)).
//   warp 2      MMA issuer of FFN2: acc2 += G_c W2_c^T (128 x D, TMEM columns
//               0 .. D-1), G_c read from shared memory.  Two issuers: a
//               tcgen05.mma issued from one thread takes ~100 cycles whatever
//               its N up to 128, so one thread could not keep both going.
//   warps 4-19  epilogue, four per TMEM lane quarter (32 of the chunk's 128
//               columns each, so four warps per sub-partition hide the GELU's
//               latencies): the RMSNorm row scale from the H tile in shared
//               memory at the start of a tile (each warp sums a quarter of
//               the row, partials combined in shared memory); per chunk acc1 -> row scale ->
//               GELU -> bf16 into G (the 128-byte-swizzled K-major layout the
//               FFN2 MMA reads); at the end of the tile acc2 + residual H
//               (re-read from global memory, so the H tile can be refilled
//               for the next tile while this one finishes) -> bf16 -> Y.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "ot_gelu_fit.h"
#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int FF_BM = 128;                     // rows per tile
constexpr int FF_BH = 128;                     // hidden columns per chunk
constexpr uint32_t FF_SLAB = 128 * 128;        // [128 rows][128 B]
constexpr int FF_EPI_WARPS = 16;                // four per TMEM lane quarter
constexpr int FF_THREADS = 32 * (4 + FF_EPI_WARPS);

template <int D> struct FfnShape {
    static_assert(D % 128 == 0 && D <= 256, "fused FFN: D in {128, 256}");
    static constexpr int KS = D / 64;                        // K slabs of H and W1
    static constexpr int W1_STAGES = KS / 2;                 // two W1 slabs per stage
    static constexpr uint32_t STAGE = D * 128 > 2 * FF_SLAB ? D * 128 : 2 * FF_SLAB;
    static constexpr int STAGES = W1_STAGES + 2;             // + two W2 slabs per chunk
    static constexpr uint32_t H_BYTES = KS * FF_SLAB;
    static constexpr uint32_t G_BYTES = 2 * FF_SLAB;         // 128 hidden = two K slabs
    static constexpr size_t SMEM = 1024 + H_BYTES + G_BYTES + STAGES * STAGE + 256;
};

struct FfnParams {
    FfnArgs a;
    int grouped;  // H tensor map is (D, G, M) instead of (D, M, 1)
    int m_tiles;
    long long tiles;
};

// exact-erf GELU, z * Phi(z), with Phi(z) ~ 1/2 + 1/2 tanh(z (A + B z^2)):
// the same fitted form as the GEMM epilogue
__device__ __forceinline__ float ffn_gelu(float z)
{
    const float t = tanh_approx(z * fmaf(OT_GELU_B, z * z, OT_GELU_A));
    const float hz = 0.5f * z;
    return fmaf(hz, t, hz);
}

__device__ __forceinline__ long long ffn_row(const RowMap &m, int r, int g)
{
    const unsigned P = static_cast<unsigned>(m.P);
    const unsigned ur = static_cast<unsigned>(r);
    const unsigned qt = ur / P, t = ur - qt * P;
    return static_cast<long long>(qt) * m.A + t + m.B + static_cast<long long>(g) * m.Gs;
}

template <int D>
__global__ void __launch_bounds__(FF_THREADS, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW1,
                  const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ FfnParams P)
{
    using Sh = FfnShape<D>;
    constexpr int KS = Sh::KS;
    constexpr uint32_t IDESC1 = make_idesc(FF_BM, FF_BH, 1, 0, 0);
    constexpr uint32_t IDESC2 = make_idesc(FF_BM, D, 1, 0, 0);
    const FfnArgs &a = P.a;
    const int NC = a.F / FF_BH; // hidden chunks per tile

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sH = smem;
    uint8_t *sG = sH + Sh::H_BYTES;
    uint8_t *sW = sG + Sh::G_BYTES; // [STAGES][STAGE]
    // RMSNorm partial sums [4][FF_BM] at the start of a tile live in G: the
    // previous tile's second projection finished reading G before its output
    // was read out, and this tile's first GELU writes G only after the sums
    float *s_ss = reinterpret_cast<float *>(sG);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sW + Sh::STAGES * Sh::STAGE);
    uint64_t *h_full = bars;
    uint64_t *h_free = h_full + 1;            // FFN1's last MMAs + the epilogue's norm reads
    uint64_t *w_full = h_free + 1;            // [STAGES]
    uint64_t *w_empty = w_full + Sh::STAGES;  // [STAGES]
    uint64_t *a1_full = w_empty + Sh::STAGES; // [2]
    uint64_t *a1_free = a1_full + 2;          // [2]
    uint64_t *g_full = a1_free + 2;
    uint64_t *g_free = g_full + 1;
    uint64_t *a2_full = g_free + 1;
    uint64_t *a2_free = a2_full + 1;
    uint64_t *mma_done = a2_free + 1;         // [2] one per issuer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        mbar_init(h_full, 1);
        mbar_init(h_free, 1 + FF_EPI_WARPS);
        for (int s = 0; s < Sh::STAGES; ++s) {
            mbar_init(&w_full[s], 1);
            mbar_init(&w_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&a1_full[b], 1);
            mbar_init(&a1_free[b], FF_EPI_WARPS);
            mbar_init(&mma_done[b], 1);
        }
        mbar_init(g_full, FF_EPI_WARPS);
        mbar_init(g_free, 1);
        mbar_init(a2_full, 1);
        mbar_init(a2_free, FF_EPI_WARPS);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_acc2 = tmem, t_acc1 = tmem + D;
    const WaitCtl final_wait{a.wait.err, a.wait.limit > (1LL << 24) ? a.wait.limit : (1LL << 24)};
    volatile int no_abort = 0;
    pdl_wait(); // prologue done; from here on the previous kernel's memory is read / written

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------ TMA producers
        // warp 0: H tiles and the W1 stages; warp 3: the W2 stages.  Two
        // threads, so W1 of the next chunk never queues behind W2 stages
        // that wait for the second projection (and through it the GELU).
        const bool w1_side = warp == 0;
        if (lane == 0) {
            if (w1_side) tma_prefetch(&tmH);
            tma_prefetch(w1_side ? &tmW1 : &tmW2);
            const int s_lo = w1_side ? 0 : Sh::W1_STAGES;
            const int s_hi = w1_side ? Sh::W1_STAGES : Sh::STAGES;
            long long gc = 0; // global chunk counter
            int tl = 0, n_h = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++tl) {
                const int g = static_cast<int>(tile / P.m_tiles);
                const int m0 = static_cast<int>(tile % P.m_tiles) * FF_BM;
                if (w1_side) {
                    if (!mbar_wait(h_free, (tl & 1) ^ 1, a.wait, abort_flag)) break;
                    mbar_arrive_expect_tx(h_full, Sh::H_BYTES);
                    for (int k = 0; k < KS; ++k) {
                        if (P.grouped)
                            tma_load_3d(sH + k * FF_SLAB, &tmH, h_full, k * 64, g, m0);
                        else
                            tma_load_3d(sH + k * FF_SLAB, &tmH, h_full, k * 64, m0, 0);
                    }
                    ++n_h;
                }
                for (int c = 0; c < NC; ++c, ++gc) {
                    const uint32_t ph = static_cast<uint32_t>(gc & 1);
                    for (int s = s_lo; s < s_hi && ok; ++s) {
                        if (!mbar_wait(&w_empty[s], ph ^ 1, a.wait, abort_flag)) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = sW + s * Sh::STAGE;
                        if (w1_side) {
                            mbar_arrive_expect_tx(&w_full[s], 2 * FF_SLAB);
                            for (int kk = 0; kk < 2; ++kk)
                                tma_load_3d(dst + kk * FF_SLAB, &tmW1, &w_full[s], (2 * s + kk) * 64,
                                            c * FF_BH, g);
                        } else {
                            mbar_arrive_expect_tx(&w_full[s], D * 128);
                            tma_load_3d(dst, &tmW2, &w_full[s], c * FF_BH + (s - Sh::W1_STAGES) * 64, 0, g);
                        }
                    }
                    if (!ok) break;
                }
            }
            // never leave a load in flight
            if (n_h > 0) mbar_wait(h_full, (n_h - 1) & 1, final_wait, &no_abort);
            if (gc > 0)
                for (int s = s_lo; s < s_hi; ++s)
                    mbar_wait(&w_full[s], static_cast<uint32_t>((gc - 1) & 1), final_wait, &no_abort);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ FFN1 issuer
        if (lane == 0) {
            long long gc = 0;
            int tl = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++tl) {
                if (!mbar_wait(h_full, tl & 1, a.wait, abort_flag)) break;
                tc_fence_after();
                for (int c = 0; c < NC && ok; ++c, ++gc) {
                    const int b = static_cast<int>(gc & 1);
                    const uint32_t ph = static_cast<uint32_t>(gc & 1);
                    if (!mbar_wait(&a1_free[b], static_cast<uint32_t>((gc >> 1) & 1) ^ 1, a.wait,
                                   abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int s = 0; s < Sh::W1_STAGES; ++s) {
                        if (!mbar_wait(&w_full[s], ph, a.wait, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t w_addr = smem_u32(sW + s * Sh::STAGE);
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint32_t h_addr = smem_u32(sH + (2 * s + kk) * FF_SLAB);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                mma_f16(t_acc1 + b * FF_BH, sw128_desc(h_addr + k * 32, 16),
                                        sw128_desc(w_addr + kk * FF_SLAB + k * 32, 16), IDESC1,
                                        (s | kk | k) != 0);
                        }
                        mma_commit(&w_empty[s]);
                    }
                    if (!ok) break;
                    mma_commit(&a1_full[b]);
                }
                // every FFN1 MMA of the tile has read H: the tile may be refilled
                if (ok) mma_commit(h_free);
            }
            mma_commit(&mma_done[0]);
            mbar_wait(&mma_done[0], 0, final_wait, &no_abort);
        }
    } else if (warp == 2) {
        // ------------------------------------------------ FFN2 issuer
        if (lane == 0) {
            long long gc = 0;
            int tl = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++tl) {
                for (int c = 0; c < NC && ok; ++c, ++gc) {
                    const uint32_t ph = static_cast<uint32_t>(gc & 1);
                    if (!mbar_wait(g_full, ph, a.wait, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // the tile's first chunk overwrites acc2: the previous tile's
                    // output must have been read out
                    if (c == 0 && !mbar_wait(a2_free, (tl & 1) ^ 1, a.wait, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < 2; ++j) {
                        const int s = Sh::W1_STAGES + j;
                        if (!mbar_wait(&w_full[s], ph, a.wait, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t g_addr = smem_u32(sG + j * FF_SLAB);
                        const uint32_t w_addr = smem_u32(sW + s * Sh::STAGE);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16(t_acc2, sw128_desc(g_addr + k * 32, 16), sw128_desc(w_addr + k * 32, 16),
                                    IDESC2, (c | j | k) != 0);
                        mma_commit(&w_empty[s]);
                    }
                    if (!ok) break;
                    mma_commit(g_free);
                }
                if (ok) mma_commit(a2_full);
            }
            mma_commit(&mma_done[1]);
            mbar_wait(&mma_done[1], 0, final_wait, &no_abort);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;              // TMEM lane quarter: rows 32q .. 32q+31
        const int sub = (warp - 4) >> 2;     // column quarter of the chunk / of the row
        const int r = 32 * q + lane;         // this thread's row within the tile
        const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
        const __nv_bfloat16 *H = static_cast<const __nv_bfloat16 *>(a.H);
        __nv_bfloat16 *Y = static_cast<__nv_bfloat16 *>(a.Y);
        constexpr int QD = D / 4;            // output columns per warp
        long long gc = 0;
        int tl = 0;
        bool ok = true;
        for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++tl) {
            const int g = static_cast<int>(tile / P.m_tiles);
            const int m0 = static_cast<int>(tile % P.m_tiles) * FF_BM;
            const bool live = m0 + r < a.M;
            if (!mbar_wait(h_full, tl & 1, a.wait, abort_flag)) break;
            // RMSNorm row scale from the tile in shared memory: this warp sums
            // columns sub*QD .. sub*QD+QD-1 of its rows (chunk j of a slab sits
            // at 16-byte position j ^ (r & 7))
            float ss = 0.f;
#pragma unroll
            for (int j8 = 0; j8 < QD / 8; ++j8) {
                const int col = sub * QD + 8 * j8;
                const uint8_t *row = sH + (col / 64) * FF_SLAB + r * 128;
                const uint4 v = *reinterpret_cast<const uint4 *>(row + ((((col % 64) / 8) ^ (r & 7)) << 4));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = __uint_as_float(w4[e] << 16);
                    const float hi = __uint_as_float(w4[e] & 0xFFFF0000u);
                    ss = fmaf(lo, lo, ss);
                    ss = fmaf(hi, hi, ss);
                }
            }
            s_ss[sub * FF_BM + r] = ss;
            named_bar_sync(1, 32 * FF_EPI_WARPS);
            const float rs = rsqrtf(((s_ss[r] + s_ss[FF_BM + r]) + (s_ss[2 * FF_BM + r] + s_ss[3 * FF_BM + r])) /
                                        static_cast<float>(D) +
                                    a.eps);
            named_bar_sync(1, 32 * FF_EPI_WARPS); // partials read before the next tile overwrites them
            // the next TMA write to the tile comes after these generic reads
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(h_free);
            for (int c = 0; c < NC; ++c, ++gc) {
                const int b = static_cast<int>(gc & 1);
                if (!mbar_wait(&a1_full[b], static_cast<uint32_t>((gc >> 1) & 1), a.wait, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[32];
                tmem_ld32(t_acc1 + b * FF_BH + lane_off + sub * 32, v);
                tmem_ld_wait();
                tmem_reg_fence(v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a1_free[b]);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16x2(ffn_gelu(__uint_as_float(v[2 * e]) * rs),
                                        ffn_gelu(__uint_as_float(v[2 * e + 1]) * rs));
                // G is free once FFN2 of the previous chunk has read it
                if (!mbar_wait(g_free, static_cast<uint32_t>(gc & 1) ^ 1, a.wait, abort_flag)) {
                    ok = false;
                    break;
                }
                // columns sub*32 .. sub*32+31: slab sub / 2, 16-byte chunks 4 (sub & 1) ..
                uint8_t *grow = sG + (sub >> 1) * FF_SLAB + r * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4 *>(grow + (((4 * (sub & 1) + j) ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                // generic writes, read next by the tensor core (async proxy)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(g_full);
            }
            if (!ok) break;
            // residual row, columns sub*QD .. sub*QD + QD - 1, prefetched
            uint4 res[QD / 8];
            const long long h_off = live ? ffn_row(a.h_map, m0 + r, g) * D + sub * QD : 0;
#pragma unroll
            for (int i = 0; i < QD / 8; ++i)
                res[i] = live ? __ldg(reinterpret_cast<const uint4 *>(H + h_off) + i) : make_uint4(0, 0, 0, 0);
            if (!mbar_wait(a2_full, tl & 1, a.wait, abort_flag)) break;
            tc_fence_after();
            const long long y_off = live ? ffn_row(a.y_map, m0 + r, g) * D + sub * QD : 0;
#pragma unroll
            for (int c32 = 0; c32 < QD / 32; ++c32) {
                uint32_t v[32];
                tmem_ld32(t_acc2 + lane_off + sub * QD + 32 * c32, v);
                tmem_ld_wait();
                tmem_reg_fence(v);
                uint4 o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 x = res[4 * c32 + i];
                    const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        ow[e] = pack_bf16x2(__uint_as_float(v[8 * i + 2 * e]) + __uint_as_float(w4[e] << 16),
                                            __uint_as_float(v[8 * i + 2 * e + 1]) +
                                                __uint_as_float(w4[e] & 0xFFFF0000u));
                    o[i] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
                if (live) {
                    uint4 *dst = reinterpret_cast<uint4 *>(Y + y_off + 32 * c32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = o[i];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(a2_free);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
static cudaError_t launch_ffn_cfg(const FfnArgs &a, cudaStream_t s)
{
    using Sh = FfnShape<D>;
    alignas(64) CUtensorMap tmH, tmW1, tmW2;
    FfnParams p;
    p.a = a;
    p.grouped = a.G > 1 && a.h_map.Gs != 0;
    p.m_tiles = (a.M + FF_BM - 1) / FF_BM;
    p.tiles = static_cast<long long>(p.m_tiles) * a.G;
    const char *Hbase = static_cast<const char *>(a.H) + a.h_map.B * static_cast<long long>(D) * 2;
    if (p.grouped) {
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.G), static_cast<uint64_t>(a.M)};
        uint64_t str[2] = {static_cast<uint64_t>(a.h_map.Gs) * D * 2, static_cast<uint64_t>(a.h_map.A) * D * 2};
        uint32_t box[3] = {64, 1, FF_BM};
        if (encode_tmap_3d(&tmH, 2, Hbase, dims, str, box)) return cudaErrorInvalidValue;
    } else {
        uint64_t rs = static_cast<uint64_t>(a.h_map.A) * D * 2;
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.M), 1};
        uint64_t str[2] = {rs, rs * static_cast<uint64_t>(a.M)};
        uint32_t box[3] = {64, FF_BM, 1};
        if (encode_tmap_3d(&tmH, 2, Hbase, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.F), static_cast<uint64_t>(a.G)};
        uint64_t str[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(a.w1_gstride) * 2};
        uint32_t box[3] = {64, FF_BH, 1};
        if (encode_tmap_3d(&tmW1, 2, a.W1, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        uint64_t dims[3] = {static_cast<uint64_t>(a.F), static_cast<uint64_t>(D), static_cast<uint64_t>(a.G)};
        uint64_t str[2] = {static_cast<uint64_t>(a.F) * 2, static_cast<uint64_t>(a.w2_gstride) * 2};
        uint32_t box[3] = {64, static_cast<uint32_t>(D), 1};
        if (encode_tmap_3d(&tmW2, 2, a.W2, dims, str, box)) return cudaErrorInvalidValue;
    }
    static int num_sms = 0;
    if (num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            num_sms < 1)
            num_sms = 148;
    }
    auto kern = ffn_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Sh::SMEM));
    if (e != cudaSuccess) return e;
    const long long grid = p.tiles < num_sms ? p.tiles : num_sms;
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(FF_THREADS), Sh::SMEM, s, tmH, tmW1,
                      tmW2, p);
}

bool ffn_tc_supported(int D, int F) { return (D == 128 || D == 256) && F % FF_BH == 0 && F >= FF_BH; }

cudaError_t launch_ffn_tc(const FfnArgs &a, cudaStream_t s)
{
    if (!ffn_tc_supported(a.D, a.F) || a.M < 1 || a.G < 1 || a.h_map.P != 1 || a.y_map.P != 1)
        return cudaErrorInvalidValue;
    if (a.D == 256) return launch_ffn_cfg<256>(a, s);
    return launch_ffn_cfg<128>(a, s);
}

} // namespace ot
