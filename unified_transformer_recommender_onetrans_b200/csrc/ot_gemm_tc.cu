// tcgen05 GEMM for every projection of the block (shared S QKV / O / FFN,
// grouped private NS QKV / O / FFN with one weight matrix per NS position,
// Auto-Split), bf16 or e4m3 operands, fp32 accumulation in TMEM.
//
// Persistent: one CTA per SM walks a static list of 128 x 128 output tiles
// (group-major, then M, then N fastest, so CTAs running together share their
// A tiles in L2).  Warp roles:
//   warp 0      TMA producer: per k-block an A tile [128 rows][128 B] and a
//               B tile [128][128 B], 128-byte swizzle, 6-stage ring.
//   warp 1      TMEM owner (256 columns = two 128-column accumulators); lane 0
//               issues 4 MMAs per k-block (K = 16 bf16 / 32 e4m3 each) into
//               accumulator t % 2, so the MMAs of tile t+1 run while the
//               epilogue drains tile t.
//   warps 2-9   epilogue, two per TMEM lane quarter (32 rows x 64 columns
//               each): residual rows prefetched into a swizzled staging buffer
//               before the accumulator is ready, then per 32 columns: TMEM ->
//               registers, row scale (RMSNorm, fp8 scales), GELU, + residual,
//               bf16 into the staging buffer; finally 128-byte coalesced row
//               stores through the row maps (Q tail, KV cache rows, NS groups),
//               each row's address computed once per tile by its own lane.
//   warps 10-13 RMSNorm warps (projections that follow a norm): read their row
//               of every A stage of the tile in flight and hand
//               sum(x^2) to the epilogue through shared memory; the gain is
//               folded into the weights on the host.
// A stage returns to the producer when its MMAs completed (tcgen05.commit)
// and, for norm GEMMs, the four norm warps read it (their generic-proxy reads
// are ordered before the next TMA write by fence.proxy.async).
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "ot_gelu_fit.h"
#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int G_BM = 128;
constexpr int G_EPI_WARPS = 8, G_NORM_WARPS = 4;
constexpr int G_THREADS = 32 * (2 + G_EPI_WARPS + G_NORM_WARPS);
constexpr uint32_t G_ROWB = 128;                // bytes of K per operand row per stage

// Tile shapes: 128 x BN.  BN = 256 reads 96 B of operands from shared memory
// per MMA clock instead of 128 B for BN = 128 (the A tile is reused across
// twice the columns), leaving bandwidth for the TMA fills and the epilogue.
template <int BN> struct GemmShape {
    static constexpr int STAGES = BN == 256 ? 3 : 6;
    static constexpr uint32_t A_BYTES = G_BM * G_ROWB;
    static constexpr uint32_t B_BYTES = BN * G_ROWB;
    static constexpr int EPI_COLS = BN / 2;                    // per epilogue warp
    static constexpr uint32_t STAGING = 32 * EPI_COLS * 2;     // 32 rows x EPI_COLS bf16
    static constexpr size_t SMEM = 1024 + STAGES * (A_BYTES + B_BYTES) + G_EPI_WARPS * STAGING +
                                   2 * G_BM * sizeof(float) + 256;
};

struct TcGemmParams {
    GemmArgs a;
    int a_grouped; // A tensor map is (K, G, M) instead of (K, M, 1)
    int m_tiles, n_tiles;
    long long tiles;
};

// One launch over one or two problems with the same K, tile shape and norm
// (the S and NS projections of a layer): problem 0's tiles, then problem 1's,
// so the second fills the first's last partial wave.
struct TcGemmMulti {
    TcGemmParams q[2];
    long long split; // first tile of problem 1 (= q[0].tiles)
    long long tiles; // all tiles
};

// the problem a tile of the launch belongs to, and its tile index within it
// (ONE: a single-problem launch; every parameter read then has a constant
// offset, which the epilogue's per-tile reads depend on for speed)
template <bool ONE>
__device__ __forceinline__ int tile_problem(const TcGemmMulti &P, long long tile, long long &local)
{
    if (ONE) {
        local = tile;
        return 0;
    }
    const int pi = tile >= P.split ? 1 : 0;
    local = tile - (pi ? P.split : 0);
    return pi;
}

// exact-erf GELU, z * Phi(z), with Phi(z) ~ 1/2 + 1/2 tanh(z (A + B z^2)):
// fitted A, B (max |Phi error| 1.4e-4) and the hardware tanh, six instructions
__device__ __forceinline__ float gelu_fast(float z)
{
    const float t = tanh_approx(z * fmaf(OT_GELU_B, z * z, OT_GELU_A));
    const float hz = 0.5f * z;
    return fmaf(hz, t, hz);
}

__device__ __forceinline__ void decode_tile(const TcGemmParams &P, long long tile, int bn, int &g,
                                            int &m0, int &n0)
{
    const int nt = static_cast<int>(tile % P.n_tiles);
    const long long rest = tile / P.n_tiles;
    m0 = static_cast<int>(rest % P.m_tiles) * G_BM;
    g = static_cast<int>(rest / P.m_tiles);
    n0 = nt * bn;
}

// four values -> e4m3 bytes (first value in the lowest byte), round to
// nearest even, saturating
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d)
{
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// staging layout: row r (0..31) is ROWB bytes, 16-byte chunk c stored at
// (c & ~7) | ((c ^ r) & 7), so 8 consecutive rows hit 8 different bank groups
template <int ROWB>
__device__ __forceinline__ uint4 *stage_chunk(uint8_t *stage, int r, int c)
{
    return reinterpret_cast<uint4 *>(stage + r * ROWB + (((c & ~7) | ((c ^ r) & 7)) << 4));
}

// Row map with 32-bit quotient / remainder (rows and periods fit in 31 bits).
__device__ __forceinline__ long long rowmap_dev(const RowMap &m, int r, int g)
{
    const unsigned P = static_cast<unsigned>(m.P);
    const unsigned ur = static_cast<unsigned>(r);
    const unsigned qt = ur / P, t = ur - qt * P;
    return static_cast<long long>(qt) * m.A + t + m.B + static_cast<long long>(g) * m.Gs;
}

__device__ __forceinline__ bool rowmap_keep_dev(const RowMap &m, int r)
{
    const unsigned P = static_cast<unsigned>(m.P);
    return static_cast<long long>(static_cast<unsigned>(r) % P) >= m.min_t;
}

// Everything the epilogue needs from a tile's problem, read at constant
// offsets of the parameter block (called once per problem with P.q[0] /
// P.q[1] and the results selected: runtime indexing into the parameters
// turns every read into a dependent global load on the tile's critical path).
struct EpiTile {
    int g, m0, n0;
    int M, gelu;
    long long out_off;          // this lane's row in the output segment (-1: not stored)
    long long res_off;          // this lane's row in the residual
    const __nv_bfloat16 *res;   // null: no residual
    long long res_cap;          // checked build: bytes of the residual buffer from res
    __nv_bfloat16 *obase;       // output segment base
    long long cap;              // checked build: bytes of the output buffer from obase
    const float *row_scale;     // fp8: per-row scale (indexed through the A row map), or null
    long long row_scale_idx;
    float g_scale;              // fp8: per-matrix scale (1 otherwise), times the A operand's per-group scale
    float q_inv;                // e4m3 output: 1 / its scale
    float inv_k, eps;           // RMSNorm
};

// the tile's residual rows first: their loads are the epilogue's longest wait
template <int BN>
__device__ __forceinline__ void epi_res(const TcGemmParams &Q, long long lt, int q, int lane, int half, EpiTile &e)
{
    const GemmArgs &a = Q.a;
    decode_tile(Q, lt, BN, e.g, e.m0, e.n0);
    e.M = a.M;
    const int r = e.m0 + 32 * q + lane;
    e.res = static_cast<const __nv_bfloat16 *>(a.res);
    e.res_cap = a.res_cap;
    e.res_off = 0;
    if (r < a.M && e.res) e.res_off = rowmap_dev(a.res_map, r, e.g) * a.res_ld + e.n0 + half * (BN / 2);
}

template <int BN, bool FP8>
__device__ __forceinline__ void epi_tile(const TcGemmParams &Q, int q, int lane, int half, EpiTile &e)
{
    const GemmArgs &a = Q.a;
    e.gelu = a.gelu;
    e.inv_k = 1.f / static_cast<float>(a.K);
    e.eps = a.eps;
    const int c0 = e.n0 + half * (BN / 2); // first output column of this warp
    const int r = e.m0 + 32 * q + lane;    // this lane's row
    const bool live = r < a.M;
    // column segment of the tile (at most three): constant indices only
    const EpiSeg &s0 = a.seg[0], &s1 = a.seg[1], &s2 = a.seg[2];
    const int sidx = (a.nseg < 2 || (e.n0 >= s0.c_lo && e.n0 < s0.c_hi))   ? 0
                     : (a.nseg < 3 || (e.n0 >= s1.c_lo && e.n0 < s1.c_hi)) ? 1
                                                                            : 2;
#define OT_SEGF(f) (sidx == 0 ? s0.f : sidx == 1 ? s1.f : s2.f)
    const RowMap mp{OT_SEGF(map.P), OT_SEGF(map.A), OT_SEGF(map.B), OT_SEGF(map.Gs), OT_SEGF(map.min_t)};
    e.obase = static_cast<__nv_bfloat16 *>(OT_SEGF(out));
    e.cap = OT_SEGF(cap);
    e.out_off = -1;
    const int *pages = OT_SEGF(pages);
    if (live && rowmap_keep_dev(mp, r)) {
        if (pages) {
            // paged KV cache: the row's page from the table (a bad id: no store)
            EpiSeg sg;
            sg.map = mp;
            sg.pages = pages;
            sg.pg_ustride = OT_SEGF(pg_ustride);
            sg.n_pages = OT_SEGF(n_pages);
            sg.pg_off = OT_SEGF(pg_off);
            sg.pg_kv = OT_SEGF(pg_kv);
            const long long pr = paged_row(sg, r);
            if (pr >= 0)
                e.out_off = pr * OT_SEGF(ld) + (c0 - OT_SEGF(c_lo));
            else if (a.wait.err)
                atomicCAS(a.wait.err, 0, OT_ERR_DEVICE_BOUNDS);
        } else {
            e.out_off = rowmap_dev(mp, r, e.g) * OT_SEGF(ld) + (c0 - OT_SEGF(c_lo));
        }
    }
#undef OT_SEGF
    e.row_scale = live ? a.row_scale : nullptr;
    e.row_scale_idx = e.row_scale ? rowmap_dev(a.a_map, r, e.g) : 0;
    e.g_scale = a.g_scale ? a.g_scale[e.g] : 1.f;
    e.q_inv = 1.f;
    if (FP8) { // per-group activation scale of the A operand; e4m3 output scale
        if (a.xg_scale) e.g_scale *= a.xg_scale[e.g * a.xg_gstride];
        if (a.qscale) e.q_inv = __frcp_rn(a.qscale[e.g * a.qscale_gstride]);
    }
}

template <int BN, bool FP8, bool MULTI>
__global__ void __launch_bounds__(G_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ TcGemmMulti P)
{
    using Sh = GemmShape<BN>;
    constexpr int G_STAGES = Sh::STAGES;
    constexpr int G_BN = BN;
    constexpr int G_EPI_COLS = Sh::EPI_COLS;
    constexpr uint32_t G_STAGING = Sh::STAGING;
    constexpr int ROWB = G_EPI_COLS * 2; // staging row bytes
    constexpr uint32_t IDESC = make_idesc(G_BM, G_BN, FP8 ? 0 : 1, 0, 0);
    const GemmArgs &a0 = P.q[0].a; // launch-wide: K, norm, wait control

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + G_STAGES * Sh::A_BYTES;
    uint8_t *sOut = sB + G_STAGES * Sh::B_BYTES;
    float *ssbuf = reinterpret_cast<float *>(sOut + G_EPI_WARPS * G_STAGING); // [2][128]
    uint64_t *full = reinterpret_cast<uint64_t *>(ssbuf + 2 * G_BM);
    uint64_t *empty = full + G_STAGES;
    uint64_t *tfull = empty + G_STAGES;   // [2]
    uint64_t *tempty = tfull + 2;         // [2]
    uint64_t *nfull = tempty + 2;         // [2]
    uint64_t *nempty = nfull + 2;         // [2]
    uint64_t *mma_done = nempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_kb = a0.K / (FP8 ? 128 : 64);
    const bool norm = a0.norm != 0 && !FP8;
    // e4m3 output: launch-wide, and only with e4m3 operands (the bf16
    // instantiations compile without the branch)
    const bool q8 = FP8 && a0.store == OT_STORE_E4M3;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < G_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], norm ? 1 + G_NORM_WARPS : 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], G_EPI_WARPS);
            mbar_init(&nfull[b], G_NORM_WARPS);
            mbar_init(&nempty[b], G_EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch(&tmA0);
        tma_prefetch(&tmB0);
        if (P.tiles > P.split) {
            tma_prefetch(&tmA1);
            tma_prefetch(&tmB1);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * G_BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // waits at the end ignore the abort flag and never use a test-lowered limit
    const WaitCtl wctl = a0.wait;
    const WaitCtl final_wait{wctl.err, wctl.limit > (1LL << 24) ? wctl.limit : (1LL << 24)};
    volatile int no_abort = 0;
    // prologue done; from here on the previous kernel's memory is read / written
    // (the producer waits after issuing the weight loads that do not depend on it)
    if (warp != 0) pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            // The weights are not written by any kernel in flight: the first
            // tile's B tiles of the first stages load while the previous
            // kernel finishes (the stages are fresh, so no empty wait); their
            // A tiles follow once its outputs are visible.
            int n_pre = 0;
            if (static_cast<long long>(blockIdx.x) < P.tiles) {
                long long lt;
                const int pi = tile_problem<!MULTI>(P, blockIdx.x, lt);
                const CUtensorMap *tB = pi ? &tmB1 : &tmB0;
                int g, m0, n0;
                decode_tile(P.q[pi], lt, G_BN, g, m0, n0);
                n_pre = num_kb < G_STAGES ? num_kb : G_STAGES;
                for (int kb = 0; kb < n_pre; ++kb) {
                    mbar_arrive_expect_tx(&full[kb], Sh::A_BYTES + Sh::B_BYTES);
                    tma_load_3d(sB + kb * Sh::B_BYTES, tB, &full[kb], kb * (FP8 ? 128 : 64), n0, g);
                }
            }
            pdl_wait();
            long long it = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x) {
                long long lt;
                const int pi = tile_problem<!MULTI>(P, tile, lt);
                const CUtensorMap *tA = pi ? &tmA1 : &tmA0, *tB = pi ? &tmB1 : &tmB0;
                int g, m0, n0;
                int a_grouped;
                if (MULTI && pi) {
                    decode_tile(P.q[1], lt, G_BN, g, m0, n0);
                    a_grouped = P.q[1].a_grouped;
                } else {
                    decode_tile(P.q[0], lt, G_BN, g, m0, n0);
                    a_grouped = P.q[0].a_grouped;
                }
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = static_cast<int>(it % G_STAGES);
                    const uint32_t ph = static_cast<uint32_t>((it / G_STAGES) & 1);
                    const bool pre = it < n_pre; // B already issued, transaction bytes armed
                    if (!pre) {
                        if (!mbar_wait(&empty[s], ph ^ 1, wctl, abort_flag)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[s], Sh::A_BYTES + Sh::B_BYTES);
                    }
                    const int kx = kb * (FP8 ? 128 : 64);
                    if (a_grouped)
                        tma_load_3d(sA + s * Sh::A_BYTES, tA, &full[s], kx, g, m0);
                    else
                        tma_load_3d(sA + s * Sh::A_BYTES, tA, &full[s], kx, m0, 0);
                    if (!pre) tma_load_3d(sB + s * Sh::B_BYTES, tB, &full[s], kx, n0, g);
                }
            }
            // never leave a load in flight
            for (long long j = it > G_STAGES ? it - G_STAGES : 0; j < it; ++j)
                mbar_wait(&full[j % G_STAGES], static_cast<uint32_t>((j / G_STAGES) & 1),
                          final_wait, &no_abort);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            long long it = 0;
            int t = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++t) {
                const int b = t & 1;
                if (!mbar_wait(&tempty[b], ((t >> 1) & 1) ^ 1, wctl, abort_flag)) break;
                tc_fence_after();
                const uint32_t acc = tmem + b * G_BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = static_cast<int>(it % G_STAGES);
                    if (!mbar_wait(&full[s], static_cast<uint32_t>((it / G_STAGES) & 1), wctl,
                                   abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + s * Sh::A_BYTES);
                    const uint32_t b_addr = smem_u32(sB + s * Sh::B_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t ad = sw128_desc(a_addr + k * 32, 16);
                        const uint64_t bd = sw128_desc(b_addr + k * 32, 16);
                        if (FP8)
                            mma_f8(acc, ad, bd, IDESC, (kb | k) != 0);
                        else
                            mma_f16(acc, ad, bd, IDESC, (kb | k) != 0);
                    }
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(&tfull[b]);
            }
            // every issued MMA must be complete before TMEM is released
            mma_commit(mma_done);
            mbar_wait(mma_done, 0, final_wait, &no_abort);
        }
    } else if (warp < 2 + G_EPI_WARPS) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;              // TMEM lane quarter = rows 32q .. 32q+31
        const int half = (warp - 2) >> 2;    // columns 64*half .. 64*half+63 of the tile
        uint8_t *stage = sOut + (warp - 2) * G_STAGING;
        int t = 0;
        for (long long tile = blockIdx.x; tile < P.tiles; tile += gridDim.x, ++t) {
            long long lt;
            const int pi = tile_problem<!MULTI>(P, tile, lt);
            // per-row addresses, computed once by the lane that owns the row
            EpiTile et;
            if (MULTI && pi)
                epi_res<G_BN>(P.q[1], lt, q, lane, half, et);
            else
                epi_res<G_BN>(P.q[0], lt, q, lane, half, et);
            const __nv_bfloat16 *res = et.res;
            const int m0 = et.m0;
            const int b = t & 1;
            const long long res_off = et.res_off;
            constexpr int LPR = ROWB / 16;       // lanes per staged row
            constexpr int RPI = 32 / LPR;        // rows per warp instruction
            if (res) {
                // coalesced residual prefetch, RPI rows x ROWB bytes per instruction:
                // every load is issued before the first shared-memory store, so
                // the loads overlap instead of each waiting out the latency
                uint4 rv[32 / RPI];
#pragma unroll
                for (int i = 0; i < 32 / RPI; ++i) {
                    const int rl = RPI * i + lane / LPR, ch = lane % LPR;
                    const long long ro = __shfl_sync(0xffffffffu, res_off, rl);
                    rv[i] = make_uint4(0, 0, 0, 0);
                    if (m0 + 32 * q + rl < et.M && ot_dev_ok((ro + ch * 8) * 2, 16, et.res_cap, wctl.err))
                        rv[i] = __ldg(reinterpret_cast<const uint4 *>(res + ro + ch * 8));
                }
#pragma unroll
                for (int i = 0; i < 32 / RPI; ++i)
                    *stage_chunk<ROWB>(stage, RPI * i + lane / LPR, lane % LPR) = rv[i];
            }
            if (MULTI && pi)
                epi_tile<G_BN, FP8>(P.q[1], q, lane, half, et);
            else
                epi_tile<G_BN, FP8>(P.q[0], q, lane, half, et);
            const long long out_off = et.out_off;
            if (!mbar_wait(&tfull[b], (t >> 1) & 1, wctl, abort_flag)) break;
            tc_fence_after();
            float rs = 1.f;
            if (norm) {
                if (!mbar_wait(&nfull[b], (t >> 1) & 1, wctl, abort_flag)) break;
                rs = rsqrtf(ssbuf[b * G_BM + 32 * q + lane] * et.inv_k + et.eps);
                __syncwarp();
                if (lane == 0) mbar_arrive(&nempty[b]);
            }
            if (et.row_scale) rs *= et.row_scale[et.row_scale_idx];
            rs *= et.g_scale;
            __syncwarp(); // residual staging complete before rows are read back
            if (q8) {
                // e4m3 output (no residual): 32 columns -> two 16-byte chunks
                // of the staging row (its first ROWB / 2 bytes), then
                // coalesced stores
#pragma unroll 1
                for (int c = 0; c < G_EPI_COLS / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tmem + b * G_BN + (static_cast<uint32_t>(q * 32) << 16) +
                                  half * G_EPI_COLS + c * 32,
                              v);
                    tmem_ld_wait();
                    tmem_reg_fence(v);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            f[e] = __uint_as_float(v[8 * j + e]) * rs;
                            if (et.gelu) f[e] = gelu_fast(f[e]);
                            f[e] *= et.q_inv;
                        }
                        uint2 o;
                        o.x = pack_e4m3x4(f[0], f[1], f[2], f[3]);
                        o.y = pack_e4m3x4(f[4], f[5], f[6], f[7]);
                        reinterpret_cast<uint2 *>(stage_chunk<ROWB>(stage, lane, 2 * c + (j >> 1)))[j & 1] = o;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[b]); // accumulator b may be overwritten
                constexpr int LPR8 = ROWB / 32, RPI8 = 32 / LPR8; // e4m3 row: ROWB / 2 bytes
                uint8_t *ob8 = reinterpret_cast<uint8_t *>(et.obase);
#pragma unroll
                for (int i = 0; i < 32 / RPI8; ++i) {
                    const int rl = RPI8 * i + lane / LPR8, ch = lane % LPR8;
                    const long long oo = __shfl_sync(0xffffffffu, out_off, rl);
                    if (oo < 0 || !ot_dev_ok(oo + ch * 16, 16, et.cap, wctl.err)) continue;
                    *reinterpret_cast<uint4 *>(ob8 + oo + ch * 16) = *stage_chunk<ROWB>(stage, rl, ch);
                }
                __syncwarp(); // staging free for the next tile
                continue;
            }
#pragma unroll 1
            for (int c = 0; c < G_EPI_COLS / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + b * G_BN + (static_cast<uint32_t>(q * 32) << 16) +
                              half * G_EPI_COLS + c * 32,
                          v);
                tmem_ld_wait();
                tmem_reg_fence(v);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 *p = stage_chunk<ROWB>(stage, lane, 4 * c + j);
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        f[e] = __uint_as_float(v[8 * j + e]) * rs;
                        if (et.gelu) f[e] = gelu_fast(f[e]);
                    }
                    if (res) {
                        const uint4 x = *p;
                        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            f[2 * e] += __uint_as_float(w[e] << 16);
                            f[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
                        }
                    }
                    uint4 o;
                    o.x = pack_bf16x2(f[0], f[1]);
                    o.y = pack_bf16x2(f[2], f[3]);
                    o.z = pack_bf16x2(f[4], f[5]);
                    o.w = pack_bf16x2(f[6], f[7]);
                    *p = o;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]); // accumulator b may be overwritten
            // coalesced stores: LPR lanes per row, ROWB contiguous bytes
            __nv_bfloat16 *obase = et.obase;
#pragma unroll
            for (int i = 0; i < 32 / RPI; ++i) {
                const int rl = RPI * i + lane / LPR, ch = lane % LPR;
                const long long oo = __shfl_sync(0xffffffffu, out_off, rl);
                if (oo < 0 || !ot_dev_ok((oo + ch * 8) * 2, 16, et.cap, wctl.err)) continue;
                *reinterpret_cast<uint4 *>(obase + oo + ch * 8) = *stage_chunk<ROWB>(stage, rl, ch);
            }
            __syncwarp(); // staging free for the next tile
        }
    } else if (norm) {
        // ------------------------------------------------ RMSNorm row sums
        const int row = 32 * (warp - 2 - G_EPI_WARPS) + lane; // warps 10-13: rows 0..127
        long long it = 0;
        int t = 0;
        bool ok = true;
        for (long long tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++t) {
            const int b = t & 1;
            if (!mbar_wait(&nempty[b], ((t >> 1) & 1) ^ 1, wctl, abort_flag)) break;
            float ss = 0.f;
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = static_cast<int>(it % G_STAGES);
                if (!mbar_wait(&full[s], static_cast<uint32_t>((it / G_STAGES) & 1), wctl,
                               abort_flag)) {
                    ok = false;
                    break;
                }
                const uint4 *src = reinterpret_cast<const uint4 *>(sA + s * Sh::A_BYTES + row * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    // rotate the chunk order by lane: 8 neighbouring rows then read
                    // 8 different bank groups (the row sum ignores the order)
                    const uint4 v = src[(c + lane) & 7];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(w[e] << 16);
                        const float hi = __uint_as_float(w[e] & 0xFFFF0000u);
                        ss = fmaf(lo, lo, ss);
                        ss = fmaf(hi, hi, ss);
                    }
                }
                // the stage is refilled by TMA (async proxy) once released: order
                // these generic-proxy reads before that write
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;
            ssbuf[b * G_BM + row] = ss;
            __syncwarp();
            if (lane == 0) mbar_arrive(&nfull[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * G_BN);
    }
}

static int g_num_sms = 0;

// tile counts and the operand tensor maps of one problem
template <int BN, bool FP8>
static cudaError_t prepare_problem(const GemmArgs &a, TcGemmParams &p, CUtensorMap *tmA, CUtensorMap *tmB)
{
    constexpr int G_BN = BN;
    const int esz = FP8 ? 1 : 2;
    const int kbox = FP8 ? 128 : 64;
    p.a = a;
    p.a_grouped = a.G > 1 && a.a_map.Gs != 0;
    p.m_tiles = (a.M + G_BM - 1) / G_BM;
    p.n_tiles = a.N / G_BN;
    p.tiles = static_cast<long long>(p.m_tiles) * p.n_tiles * a.G;
    const char *Abase = static_cast<const char *>(a.A) + a.a_map.B * a.lda * esz;
    if (p.a_grouped) {
        uint64_t dims[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.G),
                            static_cast<uint64_t>(a.M)};
        uint64_t str[2] = {static_cast<uint64_t>(a.a_map.Gs * a.lda * esz),
                           static_cast<uint64_t>(a.a_map.A * a.lda * esz)};
        uint32_t box[3] = {static_cast<uint32_t>(kbox), 1, G_BM};
        if (encode_tmap_3d(tmA, esz, Abase, dims, str, box)) return cudaErrorInvalidValue;
    } else {
        uint64_t dims[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), 1};
        uint64_t rs = static_cast<uint64_t>(a.a_map.A * a.lda * esz);
        uint64_t str[2] = {rs, rs * static_cast<uint64_t>(a.M)};
        uint32_t box[3] = {static_cast<uint32_t>(kbox), G_BM, 1};
        if (encode_tmap_3d(tmA, esz, Abase, dims, str, box)) return cudaErrorInvalidValue;
    }
    uint64_t dims[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.N),
                        static_cast<uint64_t>(a.G)};
    uint64_t str[2] = {static_cast<uint64_t>(a.K) * esz,
                       static_cast<uint64_t>(a.b_gstride > 0 ? a.b_gstride
                                                             : static_cast<long long>(a.N) * a.K) *
                           esz};
    uint32_t box[3] = {static_cast<uint32_t>(kbox), G_BN, 1};
    if (encode_tmap_3d(tmB, esz, a.B, dims, str, box)) return cudaErrorInvalidValue;
    return cudaSuccess;
}

template <int BN, bool FP8, bool MULTI>
static cudaError_t launch_tc_cfg(const GemmArgs &a, const GemmArgs *a1, cudaStream_t s)
{
    using Sh = GemmShape<BN>;
    alignas(64) CUtensorMap tmA0, tmB0, tmA1, tmB1;
    TcGemmMulti P;
    memset(&P, 0, sizeof(P));
    cudaError_t e = prepare_problem<BN, FP8>(a, P.q[0], &tmA0, &tmB0);
    if (e != cudaSuccess) return e;
    P.split = P.q[0].tiles;
    P.tiles = P.split;
    if (a1) {
        if ((e = prepare_problem<BN, FP8>(*a1, P.q[1], &tmA1, &tmB1)) != cudaSuccess) return e;
        P.tiles += P.q[1].tiles;
    } else {
        tmA1 = tmA0;
        tmB1 = tmB0;
    }
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            g_num_sms < 1)
            g_num_sms = 148;
    }
    auto kern = gemm_tc_kernel<BN, FP8, MULTI>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(Sh::SMEM));
    if (e != cudaSuccess) return e;
    const long long grid = P.tiles < g_num_sms ? P.tiles : g_num_sms;
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(G_THREADS), Sh::SMEM, s, tmA0,
                      tmB0, tmA1, tmB1, P);
}

// shape checks of one problem; wide: 128 x 256 tiles fit its column segments
static bool gemm_ok(const GemmArgs &a, bool &wide)
{
    const bool fp8 = a.in_dtype == OT_DTYPE_FP8;
    if (a.store != OT_STORE_BF16 && a.store != OT_STORE_E4M3) return false;
    if (a.store == OT_STORE_E4M3 && (a.res || !a.qscale || !fp8)) return false;
    if (a.K % (fp8 ? 128 : 64) != 0 || a.a_map.P != 1 || a.N % 128 != 0 || a.M < 1 || a.G < 1)
        return false;
    wide = a.N % 256 == 0;
    for (int i = 0; i < a.nseg; ++i) {
        if (a.seg[i].c_lo % 128 || a.seg[i].c_hi % 128) return false;
        if (a.seg[i].c_lo % 256 || a.seg[i].c_hi % 256) wide = false;
    }
    return true;
}

cudaError_t launch_gemm_tc_multi(const GemmArgs &a, const GemmArgs *a1, cudaStream_t s)
{
    bool wide = false, wide1 = true;
    if (!gemm_ok(a, wide)) return cudaErrorInvalidValue;
    const bool fp8 = a.in_dtype == OT_DTYPE_FP8;
    if (a1) {
        // one launch-wide K and norm, bf16 / fp32 operands
        if (fp8 || !gemm_ok(*a1, wide1) || a1->K != a.K || a1->in_dtype == OT_DTYPE_FP8 ||
            (a1->norm != 0) != (a.norm != 0) || a1->store != a.store)
            return cudaErrorInvalidValue;
    }
    // a single problem whose 128 x 256 tiles would leave SMs idle (the grouped
    // NS projections at small C) gets twice as many 128 x 128 tiles instead
    if (!a1 && wide) {
        if (g_num_sms == 0) {
            int dev = 0;
            cudaGetDevice(&dev);
            if (cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
                g_num_sms < 1)
                g_num_sms = 148;
        }
        const long long tiles256 = static_cast<long long>((a.M + G_BM - 1) / G_BM) * (a.N / 256) * a.G;
        if (tiles256 < g_num_sms) wide = false;
    }
    if (a1) {
        if (wide && wide1) return launch_tc_cfg<256, false, true>(a, a1, s);
        return launch_tc_cfg<128, false, true>(a, a1, s);
    }
    if (wide) return fp8 ? launch_tc_cfg<256, true, false>(a, a1, s) : launch_tc_cfg<256, false, false>(a, a1, s);
    return fp8 ? launch_tc_cfg<128, true, false>(a, a1, s) : launch_tc_cfg<128, false, false>(a, a1, s);
}

cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s)
{
    return launch_gemm_tc_multi(a, nullptr, s);
}

} // namespace ot
