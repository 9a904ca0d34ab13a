// Fused feed-forward of the block: Y = H + GELU(n(H) W1^T) W2^T with the
// RMSNorm gain folded into W1, bf16 operands, fp32 accumulation in TMEM.  The
// hidden activation (4d wide) never leaves the SM: per 128-row tile it is
// produced 64 columns at a time, passed through the norm row scale and GELU
// into shared memory as bf16, and consumed there by the second projection,
// whose accumulator covers the whole output row.  Every hand-off is at least
// double-buffered: W1 and W2 stages (two each), the GELU output G (two), the
// first projection's accumulators (two, 128 TMEM columns each, consumed 64
// columns at a time).
//
// Persistent: one CTA per SM walks 128-row tiles (group-major: a group is an
// NS position with its own weights, or the single shared S-side group).
//   warp 0      TMA: the tile's H rows (D / 64 slabs of [128 rows][128 B],
//               128-byte swizzle) and per FFN1 chunk (128 hidden) the W1 rows
//               of the chunk in two K-half stages.
//   warp 3      TMA: per hidden chunk the W2 columns of the chunk ([D rows]
//               [64 hidden]).  Separate threads, so W1 loads never queue
//               behind W2 stages that wait for the second projection.
//   warp 1      MMA issuer of FFN1, 128 hidden at a time: acc1[j % 2] =
//               H W1_j^T (128 x 128; N = 128 runs at about twice the rate of
//               N = 64 on the tensor core).
//   warp 2      MMA issuer of FFN2: acc2 += G_c W2_c^T (128 x D, TMEM columns
//               0 .. D-1), G_c read from shared memory.
//   warps 4-11  epilogue, two per TMEM lane quarter (32 of the chunk's 64
//               columns each): the RMSNorm row scale from the H tile in shared
//               memory at the start of a tile (each warp sums half the row,
//               partials combined in shared memory); per chunk acc1 -> row
//               scale -> GELU -> bf16 into G (the 128-byte-swizzled K-major
//               layout the FFN2 MMA reads).  The residual is free: at the
//               start of a tile the same pass that sums squares for the norm
//               stores H in fp32 into acc2, and FFN2 accumulates onto it, so
//               the H buffer is released once FFN1 has read it and the next
//               tile's H loads while this tile finishes; at the end acc2 ->
//               bf16, staged in the W2 stages, one TMA store to Y.
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "ot_gelu_fit.h"
#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int FF_BM = 128;                     // rows per tile
constexpr int FF_BH = 64;                      // hidden columns per GELU / FFN2 chunk
constexpr int FF_BH1 = 2 * FF_BH;              // hidden columns per FFN1 chunk (N of its MMAs)
constexpr uint32_t FF_SLAB = 128 * 128;        // [128 rows][128 B]
constexpr int FF_EPI_WARPS = 8;                // two per TMEM lane quarter
constexpr int FF_EPI0 = 4;                     // first epilogue warp
constexpr int FF_THREADS = 32 * (FF_EPI0 + FF_EPI_WARPS);

template <int D> struct FfnShape {
    static_assert(D % 128 == 0 && D <= 256, "fused FFN: D in {128, 256}");
    static constexpr int KS = D / 64;                          // K slabs of H and W1
    static constexpr uint32_t H_BYTES = KS * FF_SLAB;
    static constexpr uint32_t G_BYTES = FF_SLAB;               // one chunk of G
    static constexpr uint32_t W1_BYTES = (KS / 2) * FF_SLAB;   // one K-half of an FFN1 chunk of W1
    static constexpr uint32_t W2_BYTES = D * 128;              // one chunk of W2
    static constexpr size_t SMEM = 1024 + H_BYTES + 2 * G_BYTES + 2 * W1_BYTES + 2 * W2_BYTES + 256;
};

struct FfnParams {
    FfnArgs a;
    int grouped;  // H tensor map is (D, G, M) instead of (D, M, 1)
    int m_tiles;
    long long tiles;
};

// One launch over one or two problems with the same D, F and eps (the S and
// NS feed-forwards of a layer): problem 0's tiles, then problem 1's.
struct FfnMulti {
    FfnParams q[2];
    long long split; // first tile of problem 1
    long long tiles;
};

// problem, group and first row of tile `tile` of the launch
__device__ __forceinline__ int ffn_tile(const FfnMulti &P, long long tile, int &g, int &m0)
{
    const int pi = tile >= P.split ? 1 : 0;
    const long long lt = tile - (pi ? P.split : 0);
    const FfnParams &Q = P.q[pi];
    g = static_cast<int>(lt / Q.m_tiles);
    m0 = static_cast<int>(lt % Q.m_tiles) * FF_BM;
    return pi;
}

// Whether tile `tile` holds a filled row: a group with group_rows set (the
// experts of a mixture) has only its first group_rows[g] rows filled, and
// every role skips the tiles past them alike.
__device__ __forceinline__ bool ffn_tile_live(const FfnMulti &P, long long tile)
{
    int g, m0;
    const int pi = ffn_tile(P, tile, g, m0);
    const int *gr = P.q[pi].a.group_rows;
    return !gr || m0 < gr[g];
}

// exact-erf GELU, z * Phi(z), with Phi(z) ~ 1/2 + 1/2 tanh(z (A + B z^2)):
// the same fitted form as the GEMM epilogue
__device__ __forceinline__ float ffn_gelu(float z)
{
    const float t = tanh_approx(z * fmaf(OT_GELU_B, z * z, OT_GELU_A));
    const float hz = 0.5f * z;
    return fmaf(hz, t, hz);
}

// FO (fused output projection): the tile's TMA load brings the attention
// output A instead of H; the epilogue first seeds acc2 with the block input
// rows X, the FFN1 issuer accumulates A Wo^T onto them (Wo streamed through
// the W1 stages ahead of the tile's W1 chunks), and the epilogue turns
// acc2 = H into the bf16 H tile in shared memory (plus the norm's sums) that
// FFN1 reads; FFN2 then accumulates onto H in fp32.
template <int D, bool FO>
__global__ void __launch_bounds__(FF_THREADS, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmH0, const __grid_constant__ CUtensorMap tmW10,
                  const __grid_constant__ CUtensorMap tmW20, const __grid_constant__ CUtensorMap tmY0,
                  const __grid_constant__ CUtensorMap tmH1, const __grid_constant__ CUtensorMap tmW11,
                  const __grid_constant__ CUtensorMap tmW21, const __grid_constant__ CUtensorMap tmY1,
                  const __grid_constant__ CUtensorMap tmWo0, const __grid_constant__ CUtensorMap tmWo1,
                  const __grid_constant__ FfnMulti P)
{
    using Sh = FfnShape<D>;
    constexpr int KS = Sh::KS;
    constexpr uint32_t IDESC1 = make_idesc(FF_BM, FF_BH1, 1, 0, 0);
    constexpr uint32_t IDESC2 = make_idesc(FF_BM, D, 1, 0, 0);
    const FfnArgs &a = P.q[0].a; // launch-wide: F, eps, wait control
    const int NC = a.F / FF_BH; // hidden chunks per tile
    const bool two = P.tiles > P.split;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sH = smem;
    uint8_t *sG = sH + Sh::H_BYTES;          // [2][G_BYTES]
    uint8_t *sW1 = sG + 2 * Sh::G_BYTES;     // [K-half][W1_BYTES]
    uint8_t *sW2 = sW1 + 2 * Sh::W1_BYTES;   // [2][W2_BYTES]
    // RMSNorm partial sums [2][FF_BM] at the start of a tile live in G: the
    // previous tile's second projection finished reading G before its output
    // was read out, and this tile's first GELU writes G only after the sums
    float *s_ss = reinterpret_cast<float *>(sG);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sW2 + 2 * Sh::W2_BYTES);
    uint64_t *h_full = bars;
    uint64_t *h_free = h_full + 1;     // FFN1's last MMAs and the epilogue's reads of H
    uint64_t *w1_full = h_free + 1;    // [K-half]
    uint64_t *w1_empty = w1_full + 2;  // [K-half]
    uint64_t *w2_full = w1_empty + 2;  // [2]
    uint64_t *w2_empty = w2_full + 2;  // [2]
    uint64_t *a1_full = w2_empty + 2;  // [2] FFN1 accumulators, 128 columns each
    uint64_t *a1_free = a1_full + 2;   // [2]
    uint64_t *g_full = a1_free + 4;    // [2]
    uint64_t *g_free = g_full + 2;     // [2]
    uint64_t *a2_full = g_free + 2;
    uint64_t *a2_init = a2_full + 1;   // acc2 holds the tile's H (the residual) in fp32
    uint64_t *stg_free = a2_init + 1;  // the W2 stages no longer hold the previous output
    uint64_t *mma_done = stg_free + 1; // [2] one per issuer
    uint64_t *o_done = mma_done + 2;   // FO: acc2 = X + A Wo^T complete
    uint64_t *hb_full = o_done + 1;    // FO: the bf16 H tile is in sH
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(hb_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        mbar_init(h_full, 1);
        mbar_init(h_free, 1 + FF_EPI_WARPS);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&w1_full[b], 1);
            mbar_init(&w1_empty[b], 1);
            mbar_init(&w2_full[b], 1);
            mbar_init(&w2_empty[b], 1);
            mbar_init(&g_full[b], FF_EPI_WARPS);
            mbar_init(&g_free[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&a1_full[b], 1);
            mbar_init(&a1_free[b], FF_EPI_WARPS);
            mbar_init(&mma_done[b], 1);
        }
        mbar_init(a2_full, 1);
        mbar_init(a2_init, FF_EPI_WARPS);
        mbar_init(stg_free, 1);
        mbar_init(o_done, 1);
        mbar_init(hb_full, FF_EPI_WARPS);
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
    // prologue done; from here on the previous kernel's memory is read / written
    // (the producers wait after issuing the weight loads that do not depend on it)
    if (warp != 0 && warp != 3) pdl_wait();

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------ TMA producers
        const bool w1_side = warp == 0;
        if (lane == 0) {
            if (w1_side) {
                tma_prefetch(&tmH0);
                tma_prefetch(&tmY0);
                if (two) {
                    tma_prefetch(&tmH1);
                    tma_prefetch(&tmY1);
                }
            }
            tma_prefetch(w1_side ? &tmW10 : &tmW20);
            if (two) tma_prefetch(w1_side ? &tmW11 : &tmW21);
            if (FO && w1_side) {
                tma_prefetch(&tmWo0);
                if (two) tma_prefetch(&tmWo1);
            }
            // W1-side loads per tile: (FO) the KS chunks of Wo, then the NC
            // half-chunks of W1; W2 side: the NC chunks of W2.  Load j of a
            // side goes to stage j % 2 (KS and NC are even, so a W1 chunk's
            // K-half h always lands in stage h)
            constexpr int NWO = FO ? KS : 0;
            const int n_side = (w1_side ? NWO : 0) + NC;
            // The weights are not written by any kernel in flight: the first
            // tile's first two W1 / W2 stages load while the previous kernel
            // finishes (fresh stages, no empty wait); H follows once its
            // outputs are visible.
            // (not with filled-row counts: which tile comes first is known
            // only once the previous kernel's counts are visible)
            const bool counted = P.q[0].a.group_rows || (two && P.q[1].a.group_rows);
            const int n_pre = !counted && static_cast<long long>(blockIdx.x) < P.tiles ? (n_side < 2 ? n_side : 2) : 0;
            // load j of this side for group g into stage st
            auto load = [&](int pi, int g, int j, int st) {
                if (w1_side) {
                    mbar_arrive_expect_tx(&w1_full[st], Sh::W1_BYTES);
                    if (j < NWO) { // Wo columns 64 j .. 64 j + 63, all D rows
                        tma_load_3d(sW1 + st * Sh::W1_BYTES, pi ? &tmWo1 : &tmWo0, &w1_full[st], j * 64, 0, g);
                        return;
                    }
                    const int c = j - NWO;
                    for (int k = 0; k < KS / 2; ++k)
                        tma_load_3d(sW1 + st * Sh::W1_BYTES + k * FF_SLAB, pi ? &tmW11 : &tmW10, &w1_full[st],
                                    (st * (KS / 2) + k) * 64, (c >> 1) * FF_BH1, g);
                } else {
                    mbar_arrive_expect_tx(&w2_full[st], Sh::W2_BYTES);
                    tma_load_3d(sW2 + st * Sh::W2_BYTES, pi ? &tmW21 : &tmW20, &w2_full[st], j * FF_BH, 0, g);
                }
            };
            if (n_pre > 0) {
                int g, m0;
                const int pi = ffn_tile(P, blockIdx.x, g, m0);
                for (int j = 0; j < n_pre; ++j) load(pi, g, j, j);
            }
            pdl_wait();
            long long gc = 0; // global chunk counter
            int tl = 0, n_h = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++tl) {
                if (!ffn_tile_live(P, tile)) { --tl; continue; } // past its group's filled rows
                int g, m0;
                const int pi = ffn_tile(P, tile, g, m0);
                const CUtensorMap *tH = pi ? &tmH1 : &tmH0;
                if (w1_side) {
                    if (!mbar_wait(h_free, (tl & 1) ^ 1, a.wait, abort_flag)) break;
                    mbar_arrive_expect_tx(h_full, Sh::H_BYTES);
                    for (int k = 0; k < KS; ++k) {
                        if (P.q[pi].grouped)
                            tma_load_3d(sH + k * FF_SLAB, tH, h_full, k * 64, g, m0);
                        else
                            tma_load_3d(sH + k * FF_SLAB, tH, h_full, k * 64, m0, 0);
                    }
                    ++n_h;
                } else if (tl > 0 && !mbar_wait(stg_free, (tl - 1) & 1, a.wait, abort_flag)) {
                    break; // the W2 stages staged the previous tile's output
                }
                for (int j = 0; j < n_side; ++j, ++gc) {
                    const int st = static_cast<int>(gc & 1);
                    const uint32_t ph = static_cast<uint32_t>((gc >> 1) & 1);
                    if (gc < n_pre) continue; // issued before the wait
                    if (!mbar_wait(w1_side ? &w1_empty[st] : &w2_empty[st], ph ^ 1, a.wait, abort_flag)) {
                        ok = false;
                        break;
                    }
                    load(pi, g, j, st);
                }
            }
            // never leave a load in flight
            if (n_h > 0) mbar_wait(h_full, (n_h - 1) & 1, final_wait, &no_abort);
            for (long long j = gc > 2 ? gc - 2 : 0; j < gc; ++j)
                mbar_wait(w1_side ? &w1_full[j & 1] : &w2_full[j & 1], static_cast<uint32_t>((j >> 1) & 1),
                          final_wait, &no_abort);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ FFN1 issuer
        if (lane == 0) {
            long long gc1 = 0; // global FFN1 chunk counter (128 hidden each)
            long long gw = 0;  // W1-stage loads consumed (stage gw % 2, use gw / 2 of it)
            int tl = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++tl) {
                if (!ffn_tile_live(P, tile)) { --tl; continue; } // past its group's filled rows
                if (!mbar_wait(h_full, tl & 1, a.wait, abort_flag)) break;
                if (FO) {
                    // acc2 = X (seeded by the epilogue) + A Wo^T, A from the
                    // H buffer, Wo chunk j (K = 64 j .. 64 j + 63) from the W1 stages
                    if (!mbar_wait(a2_init, tl & 1, a.wait, abort_flag)) break;
                    tc_fence_after();
                    for (int j = 0; j < KS; ++j, ++gw) {
                        const int st = static_cast<int>(gw & 1);
                        if (!mbar_wait(&w1_full[st], static_cast<uint32_t>((gw >> 1) & 1), a.wait, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(sH + j * FF_SLAB);
                        const uint32_t w_addr = smem_u32(sW1 + st * Sh::W1_BYTES);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16(t_acc2, sw128_desc(a_addr + k * 32, 16), sw128_desc(w_addr + k * 32, 16),
                                    IDESC2, 1);
                        mma_commit(&w1_empty[st]);
                    }
                    if (!ok) break;
                    mma_commit(o_done);
                    // FFN1 reads the bf16 H the epilogue made of acc2
                    if (!mbar_wait(hb_full, tl & 1, a.wait, abort_flag)) break;
                }
                tc_fence_after();
                for (int c1 = 0; c1 < NC / 2 && ok; ++c1, ++gc1) {
                    const int b = static_cast<int>(gc1 & 1);
                    if (!mbar_wait(&a1_free[b], static_cast<uint32_t>((gc1 >> 1) & 1) ^ 1, a.wait, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int st = 0; st < 2; ++st, ++gw) {
                        // K-half st of this chunk is W1-stage load gw, in stage st
                        if (!mbar_wait(&w1_full[st], static_cast<uint32_t>((gw >> 1) & 1), a.wait, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t w_addr = smem_u32(sW1 + st * Sh::W1_BYTES);
#pragma unroll
                        for (int kk = 0; kk < KS / 2; ++kk) {
                            const uint32_t h_addr = smem_u32(sH + (st * (KS / 2) + kk) * FF_SLAB);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                mma_f16(t_acc1 + b * FF_BH1, sw128_desc(h_addr + k * 32, 16),
                                        sw128_desc(w_addr + kk * FF_SLAB + k * 32, 16), IDESC1,
                                        (st | kk | k) != 0);
                        }
                        mma_commit(&w1_empty[st]);
                    }
                    if (ok) mma_commit(&a1_full[b]);
                }
                // every FFN1 MMA of the tile has read H
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
                if (!ffn_tile_live(P, tile)) { --tl; continue; } // past its group's filled rows
                for (int c = 0; c < NC; ++c, ++gc) {
                    const int st = static_cast<int>(gc & 1);
                    const uint32_t ph = static_cast<uint32_t>((gc >> 1) & 1);
                    if (!mbar_wait(&g_full[st], ph, a.wait, abort_flag) ||
                        !mbar_wait(&w2_full[st], ph, a.wait, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // the tile's first chunk accumulates onto H, which the
                    // epilogue has stored into acc2 (FO: which the output
                    // projection left there and the epilogue has read)
                    if (c == 0 && !mbar_wait(FO ? hb_full : a2_init, tl & 1, a.wait, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t g_addr = smem_u32(sG + st * Sh::G_BYTES);
                    const uint32_t w_addr = smem_u32(sW2 + st * Sh::W2_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16(t_acc2, sw128_desc(g_addr + k * 32, 16), sw128_desc(w_addr + k * 32, 16), IDESC2, 1);
                    mma_commit(&w2_empty[st]);
                    mma_commit(&g_free[st]);
                }
                if (ok) mma_commit(a2_full);
            }
            mma_commit(&mma_done[1]);
            mbar_wait(&mma_done[1], 0, final_wait, &no_abort);
        }
    } else if (warp >= FF_EPI0) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter: rows 32q .. 32q+31
        const int hf = (warp - FF_EPI0) >> 2;   // column half of the chunk / of the row
        const int r = 32 * q + lane;            // this thread's row within the tile
        const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
        constexpr int HALF = D / 2;             // output columns per warp
        long long gc = 0;
        int tl = 0;
        bool ok = true;
        for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++tl) {
            if (!ffn_tile_live(P, tile)) { --tl; continue; } // past its group's filled rows
            int g, m0;
            const int pi = ffn_tile(P, tile, g, m0);
            float ss = 0.f;
            if (FO) {
                // acc2 = X, the block input rows (the output projection's
                // residual); acc2 is free: the previous tile's output was read
                // out of it by these warps
                const FfnArgs &pa = P.q[pi].a;
                const long long gr = static_cast<long long>(m0) + r; // row of the problem in group g
                const bool live = gr < pa.M;
                const __nv_bfloat16 *xrow =
                    static_cast<const __nv_bfloat16 *>(pa.X) + (live ? rowmap_apply(pa.x_map, gr, g) : 0) * D;
#pragma unroll 1
                for (int c32 = 0; c32 < HALF / 32; ++c32) {
                    const int col = hf * HALF + 32 * c32;
                    uint32_t hv[32];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 v = live ? *reinterpret_cast<const uint4 *>(xrow + col + 8 * i) : make_uint4(0, 0, 0, 0);
                        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            hv[8 * i + 2 * e] = w4[e] << 16;
                            hv[8 * i + 2 * e + 1] = w4[e] & 0xFFFF0000u;
                        }
                    }
                    tmem_st32(t_acc2 + lane_off + col, hv);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(a2_init);
                // acc2 = X + A Wo^T = H.  Its bf16 values become the H tile in
                // shared memory (the first projection's operand, laid out as a
                // 128-byte-swizzled TMA load would) and give the norm's sum of
                // squares; acc2 keeps H in fp32 for the second projection
                if (!mbar_wait(o_done, tl & 1, a.wait, abort_flag)) break;
                tc_fence_after();
#pragma unroll 1
                for (int c32 = 0; c32 < HALF / 32; ++c32) {
                    const int col = hf * HALF + 32 * c32;
                    uint32_t v[32];
                    tmem_ld32(t_acc2 + lane_off + col, v);
                    tmem_ld_wait();
                    tmem_reg_fence(v);
                    uint8_t *row = sH + (col / 64) * FF_SLAB + r * 128;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint32_t ow[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            ow[e] = pack_bf16x2(__uint_as_float(v[8 * i + 2 * e]), __uint_as_float(v[8 * i + 2 * e + 1]));
                            const float lo = __uint_as_float(ow[e] << 16);
                            const float hi = __uint_as_float(ow[e] & 0xFFFF0000u);
                            ss = fmaf(lo, lo, ss);
                            ss = fmaf(hi, hi, ss);
                        }
                        *reinterpret_cast<uint4 *>(row + ((((col % 64) / 8 + i) ^ (r & 7)) << 4)) =
                            make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
                // generic writes, read next by the tensor core (async proxy)
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(hb_full);
                    mbar_arrive(h_free);
                }
                // this thread's X half-row of its next tile toward L2: its seed
                // pass then waits for L2, not DRAM
                const long long nt = tile + gridDim.x;
                if (nt < P.tiles) {
                    int g2, m2;
                    const FfnArgs &pb = P.q[ffn_tile(P, nt, g2, m2)].a;
                    const long long r2 = static_cast<long long>(m2) + r;
                    if (r2 < pb.M) {
                        const char *xr = reinterpret_cast<const char *>(
                            static_cast<const __nv_bfloat16 *>(pb.X) + rowmap_apply(pb.x_map, r2, g2) * D + hf * HALF);
                        for (int o = 0; o < HALF * 2; o += 128) prefetch_l2(xr + o);
                    }
                }
            } else {
                if (!mbar_wait(h_full, tl & 1, a.wait, abort_flag)) break;
                // This warp's half of its rows of H (columns hf*HALF ..): the
                // RMSNorm partial sum of squares, and the values in fp32 into
                // acc2, onto which the second projection accumulates (so the
                // residual needs no read at the end).  acc2 is free: the previous
                // tile's output was read out of it by these warps.  Chunk j of a
                // slab row sits at 16-byte position j ^ (r & 7).
#pragma unroll 1
                for (int c32 = 0; c32 < HALF / 32; ++c32) {
                    const int col = hf * HALF + 32 * c32;
                    const uint8_t *row = sH + (col / 64) * FF_SLAB + r * 128;
                    uint32_t hv[32];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(row + ((((col % 64) / 8 + i) ^ (r & 7)) << 4));
                        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo = __uint_as_float(w4[e] << 16);
                            const float hi = __uint_as_float(w4[e] & 0xFFFF0000u);
                            ss = fmaf(lo, lo, ss);
                            ss = fmaf(hi, hi, ss);
                            hv[8 * i + 2 * e] = __float_as_uint(lo);
                            hv[8 * i + 2 * e + 1] = __float_as_uint(hi);
                        }
                    }
                    tmem_st32(t_acc2 + lane_off + col, hv);
                }
                tmem_st_wait();
                // H read (generic proxy) before its buffer is refilled by TMA
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(a2_init);
                    mbar_arrive(h_free);
                }
            }
            s_ss[hf * FF_BM + r] = ss;
            named_bar_sync(1, 32 * FF_EPI_WARPS);
            const float rs = rsqrtf((s_ss[r] + s_ss[FF_BM + r]) / static_cast<float>(D) + a.eps);
            named_bar_sync(1, 32 * FF_EPI_WARPS); // sums read before the first GELU overwrites G
            for (int c = 0; c < NC; ++c, ++gc) {
                // GELU chunk gc is half (gc % 2) of FFN1 chunk gc / 2 in accumulator (gc / 2) % 2
                const long long gc1 = gc >> 1;
                const int b = static_cast<int>(gc1 & 1), st = static_cast<int>(gc & 1);
                if (!mbar_wait(&a1_full[b], static_cast<uint32_t>((gc1 >> 1) & 1), a.wait, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[32];
                tmem_ld32(t_acc1 + b * FF_BH1 + (gc & 1) * FF_BH + lane_off + hf * 32, v);
                tmem_ld_wait();
                tmem_reg_fence(v);
                if (gc & 1) { // both halves of the accumulator read
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&a1_free[b]);
                }
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16x2(ffn_gelu(__uint_as_float(v[2 * e]) * rs),
                                        ffn_gelu(__uint_as_float(v[2 * e + 1]) * rs));
                // G[st] is free once FFN2 of chunk gc - 2 has read it
                if (!mbar_wait(&g_free[st], static_cast<uint32_t>((gc >> 1) & 1) ^ 1, a.wait, abort_flag)) {
                    ok = false;
                    break;
                }
                // columns hf*32 .. hf*32+31 of the chunk: 16-byte chunks 4 hf .. 4 hf + 3
                uint8_t *grow = sG + st * Sh::G_BYTES + r * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4 *>(grow + (((4 * hf + j) ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                // generic writes, read next by the tensor core (async proxy)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&g_full[st]);
            }
            if (!ok) break;
            if (!mbar_wait(a2_full, tl & 1, a.wait, abort_flag)) break;
            tc_fence_after();
            // Y = acc2 (= H + GELU(..) W2^T) as bf16, staged in the W2 stages
            // (the second projection has read its last weights; the next
            // tile's W2 loads wait for stg_free) in the 128-byte-swizzled
            // layout of the Y tensor map, then one TMA store
            uint8_t *stg = sW2;
#pragma unroll 1
            for (int c32 = 0; c32 < HALF / 32; ++c32) {
                const int col = hf * HALF + 32 * c32;
                uint32_t v[32];
                tmem_ld32(t_acc2 + lane_off + col, v);
                tmem_ld_wait();
                tmem_reg_fence(v);
                uint8_t *row = stg + (col / 64) * FF_SLAB + r * 128;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        ow[e] = pack_bf16x2(__uint_as_float(v[8 * i + 2 * e]), __uint_as_float(v[8 * i + 2 * e + 1]));
                    *reinterpret_cast<uint4 *>(row + ((((col % 64) / 8 + i) ^ (r & 7)) << 4)) =
                        make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
            }
            tc_fence_before(); // acc2 read before the next tile's H is stored into it
            // generic writes, read next by the TMA store (async proxy)
            fence_proxy_async_smem();
            named_bar_sync(1, 32 * FF_EPI_WARPS);
            if (warp == FF_EPI0 && lane == 0) {
                const CUtensorMap *tY = pi ? &tmY1 : &tmY0;
                for (int k = 0; k < KS; ++k) {
                    if (P.q[pi].grouped)
                        tma_store_3d(tY, stg + k * FF_SLAB, k * 64, g, m0);
                    else
                        tma_store_3d(tY, stg + k * FF_SLAB, k * 64, m0, 0);
                }
                bulk_commit_group();
                bulk_wait_group_read0();
                mbar_arrive(stg_free); // the W2 stages may take the next tile's weights
            }
        }
        // the output's global writes complete before the kernel ends
        if (warp == FF_EPI0 && lane == 0) bulk_wait_group0();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// tile count and tensor maps of one problem
template <int D>
static cudaError_t prepare_ffn(const FfnArgs &a, FfnParams &p, CUtensorMap *tmH, CUtensorMap *tmW1,
                               CUtensorMap *tmW2, CUtensorMap *tmY, CUtensorMap *tmWo)
{
    p.a = a;
    p.grouped = a.G > 1 && a.h_map.Gs != 0;
    p.m_tiles = (a.M + FF_BM - 1) / FF_BM;
    p.tiles = static_cast<long long>(p.m_tiles) * a.G;
    const char *Hbase = static_cast<const char *>(a.H) + a.h_map.B * static_cast<long long>(D) * 2;
    if (p.grouped) {
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.G), static_cast<uint64_t>(a.M)};
        uint64_t str[2] = {static_cast<uint64_t>(a.h_map.Gs) * D * 2, static_cast<uint64_t>(a.h_map.A) * D * 2};
        uint32_t box[3] = {64, 1, FF_BM};
        if (encode_tmap_3d(tmH, 2, Hbase, dims, str, box)) return cudaErrorInvalidValue;
    } else {
        uint64_t rs = static_cast<uint64_t>(a.h_map.A) * D * 2;
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.M), 1};
        uint64_t str[2] = {rs, rs * static_cast<uint64_t>(a.M)};
        uint32_t box[3] = {64, FF_BM, 1};
        if (encode_tmap_3d(tmH, 2, Hbase, dims, str, box)) return cudaErrorInvalidValue;
    }
    // Y: same row structure as H (rows of a tile are H's rows of the same
    // tile under y_map)
    const char *Ybase = static_cast<const char *>(a.Y) + a.y_map.B * static_cast<long long>(D) * 2;
    if (p.grouped) {
        if (a.y_map.Gs == 0) return cudaErrorInvalidValue;
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.G), static_cast<uint64_t>(a.M)};
        uint64_t str[2] = {static_cast<uint64_t>(a.y_map.Gs) * D * 2, static_cast<uint64_t>(a.y_map.A) * D * 2};
        uint32_t box[3] = {64, 1, FF_BM};
        if (encode_tmap_3d(tmY, 2, Ybase, dims, str, box)) return cudaErrorInvalidValue;
    } else {
        uint64_t rs = static_cast<uint64_t>(a.y_map.A) * D * 2;
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.M), 1};
        uint64_t str[2] = {rs, rs * static_cast<uint64_t>(a.M)};
        uint32_t box[3] = {64, FF_BM, 1};
        if (encode_tmap_3d(tmY, 2, Ybase, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.F), static_cast<uint64_t>(a.G)};
        uint64_t str[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(a.w1_gstride) * 2};
        uint32_t box[3] = {64, FF_BH1, 1};
        if (encode_tmap_3d(tmW1, 2, a.W1, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        uint64_t dims[3] = {static_cast<uint64_t>(a.F), static_cast<uint64_t>(D), static_cast<uint64_t>(a.G)};
        uint64_t str[2] = {static_cast<uint64_t>(a.F) * 2, static_cast<uint64_t>(a.w2_gstride) * 2};
        uint32_t box[3] = {64, static_cast<uint32_t>(D), 1};
        if (encode_tmap_3d(tmW2, 2, a.W2, dims, str, box)) return cudaErrorInvalidValue;
    }
    if (a.fuse_o) {
        // Wo [G][D out][D in]: boxes of 64 input columns x all D output rows
        uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(D), static_cast<uint64_t>(a.G)};
        uint64_t str[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(a.wo_gstride) * 2};
        uint32_t box[3] = {64, static_cast<uint32_t>(D), 1};
        if (encode_tmap_3d(tmWo, 2, a.Wo, dims, str, box)) return cudaErrorInvalidValue;
    } else {
        *tmWo = *tmW2; // unused
    }
    return cudaSuccess;
}

template <int D, bool FO>
static cudaError_t launch_ffn_cfg(const FfnArgs &a, const FfnArgs *a1, cudaStream_t s)
{
    using Sh = FfnShape<D>;
    alignas(64) CUtensorMap tm[2][5];
    FfnMulti P;
    memset(&P, 0, sizeof(P));
    cudaError_t e = prepare_ffn<D>(a, P.q[0], &tm[0][0], &tm[0][1], &tm[0][2], &tm[0][3], &tm[0][4]);
    if (e != cudaSuccess) return e;
    P.split = P.q[0].tiles;
    P.tiles = P.split;
    if (a1) {
        if ((e = prepare_ffn<D>(*a1, P.q[1], &tm[1][0], &tm[1][1], &tm[1][2], &tm[1][3], &tm[1][4])) !=
            cudaSuccess)
            return e;
        P.tiles += P.q[1].tiles;
    } else {
        for (int k = 0; k < 5; ++k) tm[1][k] = tm[0][k];
    }
    static int num_sms = 0;
    if (num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            num_sms < 1)
            num_sms = 148;
    }
    auto kern = ffn_tc_kernel<D, FO>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(Sh::SMEM));
    if (e != cudaSuccess) return e;
    const long long grid = P.tiles < num_sms ? P.tiles : num_sms;
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(FF_THREADS), Sh::SMEM, s, tm[0][0],
                      tm[0][1], tm[0][2], tm[0][3], tm[1][0], tm[1][1], tm[1][2], tm[1][3], tm[0][4], tm[1][4],
                      P);
}

bool ffn_tc_supported(int D, int F) { return (D == 128 || D == 256) && F % FF_BH1 == 0 && F >= FF_BH1; }

static bool ffn_ok(const FfnArgs &a)
{
    return ffn_tc_supported(a.D, a.F) && a.M >= 1 && a.G >= 1 && a.h_map.P == 1 && a.y_map.P == 1 &&
           (!a.fuse_o || (a.Wo && a.X && a.x_map.P >= 1));
}

cudaError_t launch_ffn_tc_multi(const FfnArgs &a, const FfnArgs *a1, cudaStream_t s)
{
    if (!ffn_ok(a)) return cudaErrorInvalidValue;
    if (a1 && (!ffn_ok(*a1) || a1->D != a.D || a1->F != a.F || a1->eps != a.eps || a1->fuse_o != a.fuse_o))
        return cudaErrorInvalidValue;
    if (a.fuse_o) return a.D == 256 ? launch_ffn_cfg<256, true>(a, a1, s) : launch_ffn_cfg<128, true>(a, a1, s);
    return a.D == 256 ? launch_ffn_cfg<256, false>(a, a1, s) : launch_ffn_cfg<128, false>(a, a1, s);
}

cudaError_t launch_ffn_tc(const FfnArgs &a, cudaStream_t s) { return launch_ffn_tc_multi(a, nullptr, s); }

} // namespace ot
