// tcgen05 attention for one layer of the block (head_dim 64, bf16 operands,
// fp32 scores and softmax).  One CTA = one (user, head) and two 128-query
// tiles (256 consecutive query rows), one CTA per SM.
//
// Key blocks of 128 rows are visited in order: first the user's S keys (from
// the KV cache), then, in NS mode, the NS keys of the candidates the CTA's
// rows belong to.  Visibility (the OneTrans mask):
//   S mode  : query i is S row t = L - nq + i (the pyramid tail, bottom-right
//             aligned); it sees S keys 0..t.  Blocks past the CTA's last row
//             are never loaded.
//   NS mode : query i is NS token n = i % N of candidate c = i / N; it sees
//             every S key 0..L-1 and NS keys m <= n of candidate c.  Each
//             cached S K/V tile is read once per CTA and shared by all the
//             CTA's candidates (256 / N of them).
//
//   warp 0      TMA: both Q tiles once, K/V blocks through a 6-deep ring
//               (shared memory holds only Q and K/V, so most of a CTA's keys
//               are in flight at once).
//   warp 1      TMEM (512 cols: S_0, S_1 at 0 / 128, O_0, O_1 at 256 / 320,
//               P_0, P_1 at 384 / 448); lane 0 issues S_w = Q_w K^T (4 MMAs,
//               both operands in shared memory) and O_w += P_w V (8 MMAs, P
//               read from TMEM, V MN-major from its row-major tile).  After
//               P_w(b) is ready it issues S_w(b+1) and then O_w(b), so the
//               tensor core works for one warpgroup while the other runs its
//               softmax.
//   warps 2-5   softmax warpgroup of tile 0, warps 6-9 of tile 1: one query
//               row per thread; scores from TMEM, running max / sum (base-2
//               exponent with 1/sqrt(hd) folded in), P as packed bf16 into
//               TMEM (tcgen05.st).  O accumulates in TMEM across key
//               blocks.  Each block is one pass against the current running
//               max, which is raised (O and l rescaled in place, the pass
//               redone) only when a row's max grows by more than 2^8 -- after
//               the first block that is rare, so most blocks read their scores
//               once and touch no O.  Every fourth exponential is a
//               polynomial on the FMA pipe, the rest use the special-function
//               unit.  Warp-uniform fast paths: no mask arithmetic on blocks
//               every row of the warp fully sees, no exponentials on blocks no
//               row of the warp sees.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "ot_exp2_poly.h"
#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int AT_BM = 128;  // query rows per tile
constexpr int AT_TILES = 2; // tiles per CTA
constexpr int AT_BK = 128;  // keys per block
constexpr int AT_HD = 64;
constexpr uint32_t AT_TILE = AT_BM * 128; // 16 KB: 128 rows x 128 bytes
constexpr int AT_STAGES = 6;              // K/V ring depth
// Q[2], then per stage K and V, then barriers
constexpr size_t AT_SMEM = (2 + 2 * AT_STAGES) * AT_TILE + 256;
constexpr int AT_THREADS = 32 * (2 + 4 * AT_TILES);

// 2^x on the FMA pipe: x = n + f with n the nearest integer (found by adding
// and subtracting 1.5 * 2^23, which leaves n in the low mantissa bits), a
// fitted cubic for 2^f on [-1/2, 1/2] (relative error < 7.5e-5), and n added
// to the exponent field.  Arguments below -126 are clamped (the result is then
// ~1e-38 instead of smaller); the softmax never passes more than 2^8.
__device__ __forceinline__ float poly_exp2(float x)
{
    x = fmaxf(x, -126.0f);
    const float t = x + 12582912.0f;
    const float f = x - (t - 12582912.0f);
    float p = fmaf(f, OT_EXP2_C3, OT_EXP2_C2);
    p = fmaf(f, p, OT_EXP2_C1);
    p = fmaf(f, p, OT_EXP2_C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Lazy rescale threshold (base-2): the running max moves only when it would
// grow by more than 2^8; until then p <= 2^8, well inside fp32 / bf16 range.
constexpr float AT_RESCALE_LOG2 = 8.0f;

// One pass over a row's 128 scores of a key block: p = 2^(s * c2 - m) for
// visible keys (0 elsewhere), bf16 P into the row's 128-byte-swizzled slot,
// sum of p and the max raw score seen.  FULL: every key of the block is
// visible, so no mask arithmetic.  Every fourth exponential is the FMA-pipe
// polynomial, the rest use the special-function unit.
template <bool FULL, typename BeforeStore>
__device__ __forceinline__ void softmax_pass(uint32_t tS_row, uint32_t tP_row, float c2, float m,
                                             int klo, int khi, float &rsum, float &mraw,
                                             BeforeStore &&before_store)
{
#pragma unroll 1
    for (int c = 0; c < AT_BK; c += 64) {
        uint32_t v[2][32];
        tmem_ld32(tS_row + c, v[0]);
        tmem_ld32(tS_row + c + 32, v[1]);
        tmem_ld_wait();
        tmem_reg_fence(v[0]);
        tmem_reg_fence(v[1]);
        uint32_t pk[32]; // 64 keys as bf16 pairs: column c/2 + j holds keys c + 2j, c + 2j + 1
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int cc = c + 32 * hh;
            float p[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float sc = __uint_as_float(v[hh][e]);
                const float x = fmaf(sc, c2, -m);
                const float ex = (e & 3) == 3 ? poly_exp2(x) : fast_exp2(x);
                if (FULL) {
                    p[e] = ex;
                    mraw = fmaxf(mraw, sc);
                } else {
                    const bool vis = cc + e >= klo && cc + e <= khi;
                    p[e] = vis ? ex : 0.f;
                    mraw = vis ? fmaxf(mraw, sc) : mraw;
                }
                rsum += p[e];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[16 * hh + j] = pack_bf16x2(p[2 * j], p[2 * j + 1]);
        }
        if (c == 0) before_store(); // P may be overwritten once the previous PV is done
        tmem_st32(tP_row + c / 2, pk);
    }
    tmem_st_wait();
}

template <bool NS>
__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKS,
                   const __grid_constant__ CUtensorMap tmVS, const __grid_constant__ CUtensorMap tmKN,
                   const __grid_constant__ CUtensorMap tmVN, const __grid_constant__ AttnArgs a)
{
    constexpr uint32_t IDESC_S = make_idesc(128, 128, 1, 0, 0);
    constexpr uint32_t IDESC_O = make_idesc(128, 64, 1, 0, 1);

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *sQ = smem;                    // [2 tiles]
    uint8_t *sKV = smem + 2 * AT_TILE;     // [stage][K | V]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (2 + 2 * AT_STAGES) * AT_TILE);
    uint64_t *q_full = bars + 0;
    uint64_t *kv_full = bars + 1;                  // [AT_STAGES]
    uint64_t *kv_empty = kv_full + AT_STAGES;      // [AT_STAGES]
    uint64_t *s_full = kv_empty + AT_STAGES;       // [2 tiles]
    uint64_t *p_full = s_full + 2;                 // [2 tiles]
    uint64_t *o_full = p_full + 2;                 // [2 tiles]
    uint64_t *mma_done = o_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * (AT_BM * AT_TILES), h = blockIdx.y, u = blockIdx.z;
    pdl_launch_dependents();
    const int i_last = min(i0 + AT_BM * AT_TILES, a.nq) - 1;

    // key-block schedule, shared by both tiles
    int n_s_blocks, k_begin = 0, n_blocks;
    if (!NS) {
        const int t_last = a.L - a.nq + i_last;
        n_s_blocks = (t_last + AT_BK) / AT_BK;
        n_blocks = n_s_blocks;
    } else {
        n_s_blocks = (a.L + AT_BK - 1) / AT_BK;
        k_begin = (i0 / a.N) * a.N;
        const int k_end = (i_last / a.N + 1) * a.N;
        n_blocks = n_s_blocks + (k_end - k_begin + AT_BK - 1) / AT_BK;
    }

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < AT_STAGES; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&o_full[i], 1);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        if (smem_u32(smem) & 1023) { // swizzle atoms need a 1024-byte aligned base
            *abort_flag = 1;
            if (a.wait.err) atomicCAS(a.wait.err, 0, OT_ERR_CUDA);
        }
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
    // waits at the end ignore the abort flag and never use a test-lowered limit
    const WaitCtl final_wait{a.wait.err, a.wait.limit > (1LL << 24) ? a.wait.limit : (1LL << 24)};
    volatile int no_abort = 0;
    const bool aborted_at_start = *abort_flag != 0;
    pdl_wait(); // prologue done; from here on the previous kernel's memory is read / written

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && !aborted_at_start) {
            tma_prefetch(&tmQ);
            mbar_arrive_expect_tx(q_full, AT_TILES * AT_TILE);
            for (int w = 0; w < AT_TILES; ++w)
                tma_load_3d(sQ + w * AT_TILE, &tmQ, q_full, h * AT_HD, i0 + w * AT_BM, u);
            int issued = 0;
            for (int b = 0; b < n_blocks; ++b) {
                const int st = b % AT_STAGES;
                if (!mbar_wait(&kv_empty[st], ((b / AT_STAGES) & 1) ^ 1, a.wait, abort_flag)) break;
                mbar_arrive_expect_tx(&kv_full[st], 2 * AT_TILE);
                uint8_t *k_dst = sKV + 2 * st * AT_TILE, *v_dst = k_dst + AT_TILE;
                if (b < n_s_blocks) {
                    tma_load_3d(k_dst, &tmKS, &kv_full[st], h * AT_HD, b * AT_BK, u);
                    tma_load_3d(v_dst, &tmVS, &kv_full[st], h * AT_HD, b * AT_BK, u);
                } else {
                    const int j0 = k_begin + (b - n_s_blocks) * AT_BK;
                    tma_load_3d(k_dst, &tmKN, &kv_full[st], h * AT_HD, j0, u);
                    tma_load_3d(v_dst, &tmVN, &kv_full[st], h * AT_HD, j0, u);
                }
                issued = b + 1;
            }
            mbar_wait(q_full, 0, final_wait, &no_abort);
            for (int b = issued > AT_STAGES ? issued - AT_STAGES : 0; b < issued; ++b)
                mbar_wait(&kv_full[b % AT_STAGES], (b / AT_STAGES) & 1, final_wait, &no_abort);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (ping-pong)
        if (lane == 0 && !aborted_at_start) {
            const uint32_t q_addr = smem_u32(sQ);
            auto issue_s = [&](int w, int b) {
                const uint32_t k_addr = smem_u32(sKV + 2 * (b % AT_STAGES) * AT_TILE);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16(tmem + w * 128, sw128_desc(q_addr + w * AT_TILE + k * 32, 16),
                            sw128_desc(k_addr + k * 32, 16), IDESC_S, k != 0);
                mma_commit(&s_full[w]);
            };
            bool run = mbar_wait(q_full, 0, a.wait, abort_flag) &&
                       mbar_wait(&kv_full[0], 0, a.wait, abort_flag);
            if (run) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
            }
            for (int b = 0; run && b < n_blocks; ++b) {
                const int st = b % AT_STAGES;
                const uint32_t v_addr = smem_u32(sKV + (2 * st + 1) * AT_TILE);
                for (int w = 0; run && w < AT_TILES; ++w) {
                    if (!mbar_wait(&p_full[w], b & 1, a.wait, abort_flag)) { run = false; break; }
                    tc_fence_after();
                    // the next scores first: the warpgroup can start block b+1
                    // while O(b) is being accumulated
                    if (b + 1 < n_blocks) {
                        if (w == 0 && !mbar_wait(&kv_full[(b + 1) % AT_STAGES],
                                                 ((b + 1) / AT_STAGES) & 1, a.wait, abort_flag)) {
                            run = false;
                            break;
                        }
                        tc_fence_after();
                        issue_s(w, b + 1);
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) // P from TMEM: 8 columns per 16 keys
                        mma_f16_ts(tmem + 256 + w * 64, tmem + 384 + w * 64 + kk * 8,
                                   sw128_desc(v_addr + kk * 2048, AT_TILE), IDESC_O, (b | kk) != 0);
                    mma_commit(&o_full[w]);
                    if (w == AT_TILES - 1) mma_commit(&kv_empty[st]);
                }
            }
            // every issued MMA must be complete before TMEM is released
            mma_commit(mma_done);
            mbar_wait(mma_done, 0, final_wait, &no_abort);
        }
    } else {
        // ------------------------------------------------ softmax warpgroups
        const int w = (warp - 2) >> 2;         // tile of this warpgroup
        const int quarter = warp & 3;          // TMEM lane quarter
        const int row = quarter * 32 + lane;   // row within the tile
        const int i = i0 + w * AT_BM + row;    // query row within the user
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + w * 128, tO = tmem + 256 + w * 64, tP = tmem + 384 + w * 64;
        const float c2 = a.scale * 1.4426950408889634f; // scores -> base-2 exponent
        const int t_self = a.L - a.nq + i;              // S mode
        const int my_c = NS ? i / a.N : 0, my_n = NS ? i % a.N : 0;
        float m = -INFINITY, l = 0.f;
        bool ok = !aborted_at_start;
        // wait for the PV of block j (completion j of this tile's o_full);
        // PV(j + 1) cannot be issued before this warpgroup releases P(j + 1),
        // so the wait never falls two phases behind
        auto wait_o = [&](int j) {
            if (ok && !mbar_wait(&o_full[w], j & 1, a.wait, abort_flag)) ok = false;
            tc_fence_after();
        };
        for (int b = 0; ok && b < n_blocks; ++b) {
            const bool s_block = b < n_s_blocks;
            const int j0 = s_block ? b * AT_BK : k_begin + (b - n_s_blocks) * AT_BK;
            // visible key range [klo, khi] of this row inside the block
            int klo = 0, khi;
            if (s_block) {
                khi = NS ? min(a.L - 1 - j0, AT_BK - 1) : min(t_self - j0, AT_BK - 1);
            } else {
                const int first = my_c * a.N - j0; // key index of (my_c, 0)
                klo = max(first, 0);
                khi = min(first + my_n, AT_BK - 1);
            }
            const bool warp_full = __all_sync(0xffffffffu, klo <= 0 && khi >= AT_BK - 1);
            const bool warp_none = __all_sync(0xffffffffu, khi < klo);
            // P in TMEM was last read by O(b-1): wait for it just before overwriting
            auto before_store = [&] {
                if (b >= 1) wait_o(b - 1);
            };
            if (!mbar_wait(&s_full[w], b & 1, a.wait, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (warp_none) {
                // no row of this warp sees the block: P = 0, state unchanged
                uint32_t z[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) z[j] = 0u;
                before_store();
                tmem_st32(tP + lane_off, z);
                tmem_st32(tP + lane_off + 32, z);
                tmem_st_wait();
            } else {
                // a row with no max yet (its first visible block) needs one first
                if (__any_sync(0xffffffffu, m == -INFINITY)) {
                    float mraw = -INFINITY;
#pragma unroll 1
                    for (int c = 0; c < AT_BK; c += 32) {
                        uint32_t v[32];
                        tmem_ld32(tS + lane_off + c, v);
                        tmem_ld_wait();
                        tmem_reg_fence(v);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (c + e >= klo && c + e <= khi) mraw = fmaxf(mraw, __uint_as_float(v[e]));
                    }
                    if (m == -INFINITY) m = mraw * c2; // l is 0 and O holds nothing for this row
                }
                // one pass against the current max; also track the raw max
                float rsum = 0.f, mraw = -INFINITY;
                if (warp_full)
                    softmax_pass<true>(tS + lane_off, tP + lane_off, c2, m, 0, AT_BK - 1, rsum, mraw, before_store);
                else
                    softmax_pass<false>(tS + lane_off, tP + lane_off, c2, m, klo, khi, rsum, mraw, before_store);
                const float m_cand = fmaxf(m, mraw * c2);
                const bool raise = m_cand > m + AT_RESCALE_LOG2;
                if (__any_sync(0xffffffffu, raise)) {
                    // some row's max grew by more than 2^8: rescale O and l, redo P
                    const float alpha = raise ? fast_exp2(m - m_cand) : 1.f;
                    if (raise) m = m_cand;
                    if (b > 0) { // O holds the blocks before b: the pass above waited for them
#pragma unroll
                        for (int c = 0; c < AT_HD; c += 32) {
                            uint32_t v[32];
                            tmem_ld32(tO + lane_off + c, v);
                            tmem_ld_wait();
                            tmem_reg_fence(v);
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                            tmem_st32(tO + lane_off + c, v);
                        }
                        tmem_st_wait();
                    }
                    l *= alpha;
                    rsum = 0.f;
                    if (warp_full)
                        softmax_pass<true>(tS + lane_off, tP + lane_off, c2, m, 0, AT_BK - 1, rsum, mraw, before_store);
                    else
                        softmax_pass<false>(tS + lane_off, tP + lane_off, c2, m, klo, khi, rsum, mraw, before_store);
                }
                l += rsum;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[w]);
        }
        wait_o(n_blocks - 1); // the last PV
        float o[AT_HD];
#pragma unroll
        for (int c = 0; c < AT_HD; c += 32) {
            uint32_t v[32];
            tmem_ld32(tO + lane_off + c, v);
            tmem_ld_wait();
            tmem_reg_fence(v);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[c + e] = __uint_as_float(v[e]);
        }
        if (ok && i < a.nq) {
            const float inv = 1.f / l;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.O) +
                                 (static_cast<long long>(u) * a.nq + i) * a.d + h * AT_HD;
            uint4 *dp = reinterpret_cast<uint4 *>(dst);
#pragma unroll
            for (int qd = 0; qd < 8; ++qd) {
                uint4 wv;
                wv.x = pack_bf16x2(o[qd * 8 + 0] * inv, o[qd * 8 + 1] * inv);
                wv.y = pack_bf16x2(o[qd * 8 + 2] * inv, o[qd * 8 + 3] * inv);
                wv.z = pack_bf16x2(o[qd * 8 + 4] * inv, o[qd * 8 + 5] * inv);
                wv.w = pack_bf16x2(o[qd * 8 + 6] * inv, o[qd * 8 + 7] * inv);
                dp[qd] = wv;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

static int tmap_rows(CUtensorMap *m, const void *base, long long d, long long rows, long long users,
                     long long ustride_elems)
{
    uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows),
                        static_cast<uint64_t>(users)};
    uint64_t str[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(ustride_elems) * 2};
    uint32_t box[3] = {AT_HD, AT_BK, 1};
    return encode_tmap_3d(m, 2, base, dims, str, box);
}

cudaError_t launch_attn_tc(const AttnArgs &a, cudaStream_t s)
{
    if (a.hd != AT_HD || a.dtype == OT_DTYPE_F32) return cudaErrorInvalidValue;
    alignas(64) CUtensorMap tq, tks, tvs, tkn, tvn;
    if (tmap_rows(&tq, a.Q, a.d, a.nq, a.U, static_cast<long long>(a.nq) * a.d) ||
        tmap_rows(&tks, a.KS, a.d, a.L, a.U, a.s_ustride) ||
        tmap_rows(&tvs, a.VS, a.d, a.L, a.U, a.s_ustride))
        return cudaErrorInvalidValue;
    if (a.mode == 1) {
        if (tmap_rows(&tkn, a.KN, a.d, a.nq, a.U, static_cast<long long>(a.nq) * a.d) ||
            tmap_rows(&tvn, a.VN, a.d, a.nq, a.U, static_cast<long long>(a.nq) * a.d))
            return cudaErrorInvalidValue;
    } else {
        tkn = tks;
        tvn = tvs;
    }
    dim3 grid((a.nq + AT_BM * AT_TILES - 1) / (AT_BM * AT_TILES), a.H, a.U);
    cudaError_t e;
    if (a.mode == 1) {
        e = cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(AT_SMEM));
        if (e != cudaSuccess) return e;
        return launch_pdl(attn_tc_kernel<true>, grid, dim3(AT_THREADS), AT_SMEM, s, tq, tks, tvs,
                          tkn, tvn, a);
    }
    e = cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(AT_SMEM));
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_tc_kernel<false>, grid, dim3(AT_THREADS), AT_SMEM, s, tq, tks, tvs, tkn,
                      tvn, a);
}

} // namespace ot
