// tcgen05 attention for one layer of the block (head_dim 64, bf16 operands,
// fp32 scores and softmax).  One CTA = one (user, head, 128-query tile).
//
// Key blocks of 128 rows are visited in order: first the user's S keys (from
// the KV cache), then, in NS mode, the NS keys of the candidates the tile's
// rows belong to.  Visibility (the OneTrans mask):
//   S mode  : query i is S row t = L - nq + i (the pyramid tail, bottom-right
//             aligned); it sees S keys 0..t.  Blocks past the tile's last row
//             are skipped entirely.
//   NS mode : query i is NS token n = i % N of candidate c = i / N; it sees
//             every S key 0..L-1 and NS keys m <= n of candidate c.  Each
//             cached S K/V tile is read once per CTA and shared by all the
//             tile's candidates (128 / N candidates per tile).
//
//   warp 0      TMA: Q tile once, K/V blocks through a 2-deep ring.
//   warp 1      TMEM (256 cols: S at 0..127, O block at 128..191); lane 0
//               issues S = Q K^T (4 MMAs) and O_b = P V (8 MMAs, V read
//               MN-major straight from its row-major tile).
//   warps 2-5   one query row per thread: scores from TMEM, mask, running
//               max / sum (base-2 exponent with the 1/sqrt(hd) scale folded),
//               P as bf16 into 128-byte-swizzled shared memory for the second
//               MMA, and O = O * alpha + O_b in registers.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int AT_BM = 128;   // query rows per CTA
constexpr int AT_BK = 128;   // keys per block
constexpr int AT_HD = 64;
constexpr uint32_t AT_TILE = AT_BM * 128; // 16 KB: 128 rows x 128 bytes
constexpr size_t AT_SMEM = 7 * AT_TILE + 128; // Q, K[2], V[2], P (2 tiles), barriers

template <bool NS>
__global__ void __launch_bounds__(192, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKS,
                   const __grid_constant__ CUtensorMap tmVS, const __grid_constant__ CUtensorMap tmKN,
                   const __grid_constant__ CUtensorMap tmVN, const __grid_constant__ AttnArgs a)
{
    constexpr uint32_t IDESC_S = make_idesc(128, 128, 1, 0, 0);
    constexpr uint32_t IDESC_O = make_idesc(128, 64, 1, 0, 1);

    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *sQ = smem;
    uint8_t *sK = smem + AT_TILE;          // 2 stages
    uint8_t *sV = smem + 3 * AT_TILE;      // 2 stages
    uint8_t *sP = smem + 5 * AT_TILE;      // keys 0..63 | keys 64..127
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 7 * AT_TILE);
    uint64_t *q_full = bars + 0;
    uint64_t *kv_full = bars + 1;  // [2]
    uint64_t *kv_empty = bars + 3; // [2]
    uint64_t *s_full = bars + 5;
    uint64_t *p_full = bars + 6;
    uint64_t *o_full = bars + 7;
    uint64_t *mma_done = bars + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 9);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * AT_BM, h = blockIdx.y, u = blockIdx.z;
    const int i_last = min(i0 + AT_BM, a.nq) - 1;

    // key-block schedule
    int n_s_blocks, k_begin = 0, k_end = 0, n_blocks;
    if (!NS) {
        const int t_last = a.L - a.nq + i_last;
        n_s_blocks = (t_last + AT_BK) / AT_BK;
        n_blocks = n_s_blocks;
    } else {
        n_s_blocks = (a.L + AT_BK - 1) / AT_BK;
        k_begin = (i0 / a.N) * a.N;
        k_end = (i_last / a.N + 1) * a.N;
        n_blocks = n_s_blocks + (k_end - k_begin + AT_BK - 1) / AT_BK;
    }

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(&kv_full[0], 1);
        mbar_init(&kv_full[1], 1);
        mbar_init(&kv_empty[0], 1);
        mbar_init(&kv_empty[1], 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, 4);
        mbar_init(o_full, 1);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        if (smem_u32(smem) & 1023) { // swizzle atoms need a 1024-byte aligned base
            *abort_flag = 1;
            if (a.wait.err) atomicCAS(a.wait.err, 0, OT_ERR_CUDA);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 128;
    // waits at the end ignore the abort flag and never use a test-lowered limit
    const WaitCtl final_wait{a.wait.err, a.wait.limit > (1LL << 24) ? a.wait.limit : (1LL << 24)};
    volatile int no_abort = 0;
    const bool aborted_at_start = *abort_flag != 0;

    if (warp == 0) {
        if (lane == 0 && !aborted_at_start) {
            tma_prefetch(&tmQ);
            mbar_arrive_expect_tx(q_full, AT_TILE);
            tma_load_3d(sQ, &tmQ, q_full, h * AT_HD, i0, u);
            int issued = 0;
            for (int b = 0; b < n_blocks; ++b) {
                const int st = b & 1;
                if (!mbar_wait(&kv_empty[st], ((b >> 1) & 1) ^ 1, a.wait, abort_flag)) break;
                mbar_arrive_expect_tx(&kv_full[st], 2 * AT_TILE);
                if (b < n_s_blocks) {
                    tma_load_3d(sK + st * AT_TILE, &tmKS, &kv_full[st], h * AT_HD, b * AT_BK, u);
                    tma_load_3d(sV + st * AT_TILE, &tmVS, &kv_full[st], h * AT_HD, b * AT_BK, u);
                } else {
                    const int j0 = k_begin + (b - n_s_blocks) * AT_BK;
                    tma_load_3d(sK + st * AT_TILE, &tmKN, &kv_full[st], h * AT_HD, j0, u);
                    tma_load_3d(sV + st * AT_TILE, &tmVN, &kv_full[st], h * AT_HD, j0, u);
                }
                issued = b + 1;
            }
            mbar_wait(q_full, 0, final_wait, &no_abort);
            for (int b = issued > 2 ? issued - 2 : 0; b < issued; ++b)
                mbar_wait(&kv_full[b & 1], (b >> 1) & 1, final_wait, &no_abort);
        }
    } else if (warp == 1) {
        if (lane == 0 && !aborted_at_start) {
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t p_addr = smem_u32(sP);
            bool run = mbar_wait(q_full, 0, a.wait, abort_flag) &&
                       mbar_wait(&kv_full[0], 0, a.wait, abort_flag);
            if (run) {
                tc_fence_after();
                const uint32_t k_addr = smem_u32(sK);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16(tS, sw128_desc(q_addr + k * 32, 16), sw128_desc(k_addr + k * 32, 16),
                            IDESC_S, k != 0);
                mma_commit(s_full);
            }
            for (int b = 0; run && b < n_blocks; ++b) {
                const int st = b & 1;
                if (!mbar_wait(p_full, b & 1, a.wait, abort_flag)) break;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(sV + st * AT_TILE);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = sw128_desc(p_addr + (kk >> 2) * AT_TILE + (kk & 3) * 32, 16);
                    const uint64_t bd = sw128_desc(v_addr + kk * 2048, AT_TILE);
                    mma_f16(tO, ad, bd, IDESC_O, kk != 0);
                }
                mma_commit(o_full);
                mma_commit(&kv_empty[st]);
                if (b + 1 < n_blocks) {
                    const int st1 = (b + 1) & 1;
                    if (!mbar_wait(&kv_full[st1], ((b + 1) >> 1) & 1, a.wait, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(sK + st1 * AT_TILE);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16(tS, sw128_desc(q_addr + k * 32, 16),
                                sw128_desc(k_addr + k * 32, 16), IDESC_S, k != 0);
                    mma_commit(s_full);
                }
            }
            // every issued MMA must be complete before TMEM is released
            mma_commit(mma_done);
            mbar_wait(mma_done, 0, final_wait, &no_abort);
        }
    } else {
        // ---------------- softmax warps: one query row per thread
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int i = i0 + row;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const float c2 = a.scale * 1.4426950408889634f; // scores -> base-2 exponent
        const int t_self = a.L - a.nq + i;              // S mode
        const int my_c = NS ? i / a.N : 0, my_n = NS ? i % a.N : 0;
        float m = -INFINITY, l = 0.f;
        float o[AT_HD];
#pragma unroll
        for (int e = 0; e < AT_HD; ++e) o[e] = 0.f;
        bool ok = !aborted_at_start;
        for (int b = 0; ok && b < n_blocks; ++b) {
            if (!mbar_wait(s_full, b & 1, a.wait, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const bool s_block = b < n_s_blocks;
            const int j0 = s_block ? b * AT_BK : k_begin + (b - n_s_blocks) * AT_BK;
            // visible key range [klo, khi] for this row inside this block
            // (S blocks: keys <= t_self (S mode) or < L (NS mode); NS blocks:
            // same candidate, m <= n)
            int khi;
            int klo = 0;
            if (s_block) {
                khi = NS ? min(a.L - 1 - j0, AT_BK - 1) : min(t_self - j0, AT_BK - 1);
            } else {
                const int first = my_c * a.N - j0;      // key index of (my_c, 0)
                klo = max(first, 0);
                khi = min(first + my_n, AT_BK - 1);
            }
            float mb = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < AT_BK; c += 32) {
                uint32_t v[32];
                tmem_ld32(tS + lane_off + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int kx = c + e;
                    if (kx >= klo && kx <= khi) mb = fmaxf(mb, __uint_as_float(v[e]) * c2);
                }
            }
            const float m_new = fmaxf(m, mb);
            const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m - m_new);
            float rsum = 0.f;
#pragma unroll 1
            for (int c = 0; c < AT_BK; c += 32) {
                uint32_t v[32];
                tmem_ld32(tS + lane_off + c, v);
                tmem_ld_wait();
                float p[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int kx = c + e;
                    const bool vis = kx >= klo && kx <= khi;
                    p[e] = vis ? fast_exp2(__uint_as_float(v[e]) * c2 - m_new) : 0.f;
                    rsum += p[e];
                }
                // 4 chunks of 8 keys -> swizzled 16-byte slots of this row
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int kc = (c >> 3) + q;          // 8-key chunk index 0..15
                    const int sub = kc >> 3, ch = kc & 7;
                    uint4 w;
                    w.x = pack_bf16x2(p[q * 8 + 0], p[q * 8 + 1]);
                    w.y = pack_bf16x2(p[q * 8 + 2], p[q * 8 + 3]);
                    w.z = pack_bf16x2(p[q * 8 + 4], p[q * 8 + 5]);
                    w.w = pack_bf16x2(p[q * 8 + 6], p[q * 8 + 7]);
                    *reinterpret_cast<uint4 *>(sP + sub * AT_TILE + row * 128 +
                                               ((ch ^ (row & 7)) << 4)) = w;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            l = l * alpha + rsum;
            m = m_new;
            if (!mbar_wait(o_full, b & 1, a.wait, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < AT_HD; c += 32) {
                uint32_t v[32];
                tmem_ld32(tO + lane_off + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[c + e] = fmaf(o[c + e], alpha, __uint_as_float(v[e]));
            }
        }
        if (ok && i < a.nq) {
            const float inv = 1.f / l;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.O) +
                                 (static_cast<long long>(u) * a.nq + i) * a.d + h * AT_HD;
            uint4 *dp = reinterpret_cast<uint4 *>(dst);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint4 w;
                w.x = pack_bf16x2(o[q * 8 + 0] * inv, o[q * 8 + 1] * inv);
                w.y = pack_bf16x2(o[q * 8 + 2] * inv, o[q * 8 + 3] * inv);
                w.z = pack_bf16x2(o[q * 8 + 4] * inv, o[q * 8 + 5] * inv);
                w.w = pack_bf16x2(o[q * 8 + 6] * inv, o[q * 8 + 7] * inv);
                dp[q] = w;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
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
    dim3 grid((a.nq + AT_BM - 1) / AT_BM, a.H, a.U);
    cudaError_t e;
    if (a.mode == 1) {
        e = cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(AT_SMEM));
        if (e != cudaSuccess) return e;
        attn_tc_kernel<true><<<grid, 192, AT_SMEM, s>>>(tq, tks, tvs, tkn, tvn, a);
    } else {
        e = cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(AT_SMEM));
        if (e != cudaSuccess) return e;
        attn_tc_kernel<false><<<grid, 192, AT_SMEM, s>>>(tq, tks, tvs, tkn, tvn, a);
    }
    return cudaGetLastError();
}

} // namespace ot
