// tcgen05 GEMM for every projection of the block (shared S QKV / O / FFN,
// grouped private NS QKV / O / FFN with one weight matrix per NS position,
// Auto-Split), bf16 or e4m3 operands, fp32 accumulation in TMEM.
//
// One CTA computes a 128 x BN tile of one group:
//   warp 0      TMA producer: A tile [128 rows][128 B] and B tile [BN][128 B]
//               per stage, 128-byte swizzle, STAGES-deep ring.
//   warp 1      allocates TMEM (BN columns); lane 0 issues 4 MMAs per stage
//               (K = 16 bf16 / 32 e4m3 each) and commits stage releases.
//   warps 2-5   epilogue.  While the main loop runs they also read their row
//               of every A stage from shared memory and accumulate sum(x^2),
//               which gives the RMSNorm row scale rsqrt(mean(x^2) + eps) for
//               the projections that follow a norm (the gain is folded into
//               the weights on the host).  After the last MMA they load the
//               accumulator from TMEM (thread = row), apply row scale /
//               per-row and per-group fp8 scales / GELU / residual, and store
//               bf16 rows through the row maps.
//
// A stage is released when both the MMAs that read it have completed
// (tcgen05.commit) and, for norm GEMMs, the four epilogue warps have read it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int TC_BM = 128;
constexpr int TC_ROW_BYTES = 128; // one swizzle row of K per stage

struct TcGemmParams {
    GemmArgs a;
    int a_grouped; // A tensor map is (K, G, M) instead of (K, M, 1)
};

__device__ __forceinline__ float gelu_erf_tc(float z)
{
    return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}

template <int BN, int STAGES, bool FP8>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ TcGemmParams P)
{
    constexpr uint32_t A_BYTES = TC_BM * TC_ROW_BYTES;
    constexpr uint32_t B_BYTES = BN * TC_ROW_BYTES;
    constexpr uint32_t IDESC = make_idesc(TC_BM, BN, FP8 ? 0 : 1, 0, 0);
    const GemmArgs &a = P.a;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + STAGES * B_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int m0 = blockIdx.y * TC_BM;
    const int g = blockIdx.z;
    const int num_kb = a.K / (FP8 ? 128 : 64);
    const bool norm = a.norm != 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], norm ? 5 : 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch(&tmA);
        tma_prefetch(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, BN < 32 ? 32 : BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // waits at the end ignore the abort flag and never use a test-lowered limit
    const WaitCtl final_wait{a.wait.err, a.wait.limit > (1LL << 24) ? a.wait.limit : (1LL << 24)};
    volatile int no_abort = 0;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % STAGES;
                const uint32_t ph = (kb / STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, a.wait, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
                const int kx = kb * (FP8 ? 128 : 64);
                if (P.a_grouped)
                    tma_load_3d(sA + s * A_BYTES, &tmA, &full[s], kx, g, m0);
                else
                    tma_load_3d(sA + s * A_BYTES, &tmA, &full[s], kx, m0, 0);
                tma_load_3d(sB + s * B_BYTES, &tmB, &full[s], kx, n0, g);
                issued = kb + 1;
            }
            // never leave a load in flight: wait for the last STAGES issued
            for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
                mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, final_wait, &no_abort);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % STAGES;
                if (!mbar_wait(&full[s], (kb / STAGES) & 1, a.wait, abort_flag)) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(sA + s * A_BYTES);
                const uint32_t b_addr = smem_u32(sB + s * B_BYTES);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t ad = sw128_desc(a_addr + k * 32, 16);
                    const uint64_t bd = sw128_desc(b_addr + k * 32, 16);
                    if (FP8)
                        mma_f8(tmem, ad, bd, IDESC, (kb | k) != 0);
                    else
                        mma_f16(tmem, ad, bd, IDESC, (kb | k) != 0);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(acc_full); // always: completes once every issued MMA is done
        }
    } else {
        // ---------------- epilogue warps
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        float ss = 0.f;
        if (norm) {
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % STAGES;
                if (!mbar_wait(&full[s], (kb / STAGES) & 1, a.wait, abort_flag)) break;
                const uint4 *src = reinterpret_cast<const uint4 *>(sA + s * A_BYTES + row * TC_ROW_BYTES);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 v = src[c];
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float lo = __uint_as_float(w[e] << 16);
                        float hi = __uint_as_float(w[e] & 0xFFFF0000u);
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
        }
        const bool ok = mbar_wait(acc_full, 0, final_wait, &no_abort) && !*abort_flag;
        tc_fence_after();
        const long long r = static_cast<long long>(m0) + row;
        const bool live = ok && r < a.M;
        float rs = 1.f;
        long long arow = 0;
        if (live) {
            arow = rowmap_apply(a.a_map, r, g);
            if (norm) rs = rsqrtf(ss / static_cast<float>(a.K) + a.eps);
            if (a.row_scale) rs *= a.row_scale[arow];
            if (a.g_scale) rs *= a.g_scale[g];
        }
        const __nv_bfloat16 *res = static_cast<const __nv_bfloat16 *>(a.res);
        const long long res_row = (live && res) ? rowmap_apply(a.res_map, r, g) : 0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + c, v);
            tmem_ld_wait();
            if (!live) continue;
            const int col = n0 + c;
            float f[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                f[e] = __uint_as_float(v[e]) * rs;
                if (a.gelu) f[e] = gelu_erf_tc(f[e]);
            }
            if (res) {
                const uint4 *rp = reinterpret_cast<const uint4 *>(res + res_row * a.res_ld + col);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 x = rp[q];
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        f[q * 8 + 2 * e] += __uint_as_float(w[e] << 16);
                        f[q * 8 + 2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
                    }
                }
            }
            for (int sidx = 0; sidx < a.nseg; ++sidx) {
                const EpiSeg &sg = a.seg[sidx];
                if (col < sg.c_lo || col >= sg.c_hi || !rowmap_keep(sg.map, r)) continue;
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(sg.out) +
                                     rowmap_apply(sg.map, r, g) * sg.ld + (col - sg.c_lo);
                uint4 *dp = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 o;
                    o.x = pack_bf16x2(f[q * 8 + 0], f[q * 8 + 1]);
                    o.y = pack_bf16x2(f[q * 8 + 2], f[q * 8 + 3]);
                    o.z = pack_bf16x2(f[q * 8 + 4], f[q * 8 + 5]);
                    o.w = pack_bf16x2(f[q * 8 + 6], f[q * 8 + 7]);
                    dp[q] = o;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, BN < 32 ? 32 : BN);
    }
}

template <int BN, int STAGES, bool FP8>
static cudaError_t launch_tc_cfg(const GemmArgs &a, cudaStream_t s)
{
    const int esz = FP8 ? 1 : 2;
    const int kbox = FP8 ? 128 : 64;
    alignas(64) CUtensorMap tmA, tmB;
    TcGemmParams p;
    p.a = a;
    p.a_grouped = a.G > 1 && a.a_map.Gs != 0;
    const char *Abase = static_cast<const char *>(a.A) + a.a_map.B * a.lda * esz;
    if (p.a_grouped) {
        uint64_t dims[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.G),
                            static_cast<uint64_t>(a.M)};
        uint64_t str[2] = {static_cast<uint64_t>(a.a_map.Gs * a.lda * esz),
                           static_cast<uint64_t>(a.a_map.A * a.lda * esz)};
        uint32_t box[3] = {static_cast<uint32_t>(kbox), 1, TC_BM};
        if (encode_tmap_3d(&tmA, esz, Abase, dims, str, box)) return cudaErrorInvalidValue;
    } else {
        uint64_t dims[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M), 1};
        uint64_t rs = static_cast<uint64_t>(a.a_map.A * a.lda * esz);
        uint64_t str[2] = {rs, rs * static_cast<uint64_t>(a.M)};
        uint32_t box[3] = {static_cast<uint32_t>(kbox), TC_BM, 1};
        if (encode_tmap_3d(&tmA, esz, Abase, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        uint64_t dims[3] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.N),
                            static_cast<uint64_t>(a.G)};
        uint64_t str[2] = {static_cast<uint64_t>(a.K) * esz,
                           static_cast<uint64_t>(a.b_gstride > 0 ? a.b_gstride
                                                                 : static_cast<long long>(a.N) * a.K) *
                               esz};
        uint32_t box[3] = {static_cast<uint32_t>(kbox), static_cast<uint32_t>(BN), 1};
        if (encode_tmap_3d(&tmB, esz, a.B, dims, str, box)) return cudaErrorInvalidValue;
    }
    const size_t smem = 1024 + STAGES * (TC_BM + BN) * TC_ROW_BYTES + 256;
    auto kern = gemm_tc_kernel<BN, STAGES, FP8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(a.N / BN, (a.M + TC_BM - 1) / TC_BM, a.G);
    kern<<<grid, 192, smem, s>>>(tmA, tmB, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s)
{
    const bool fp8 = a.in_dtype == OT_DTYPE_FP8;
    if (a.store != OT_STORE_BF16) return cudaErrorInvalidValue;
    if (a.K % (fp8 ? 128 : 64) != 0 || a.a_map.P != 1) return cudaErrorInvalidValue;
    if (a.N % 128 == 0) {
        return fp8 ? launch_tc_cfg<128, 4, true>(a, s) : launch_tc_cfg<128, 3, false>(a, s);
    }
    if (a.N % 64 == 0) {
        return fp8 ? launch_tc_cfg<64, 4, true>(a, s) : launch_tc_cfg<64, 4, false>(a, s);
    }
    return cudaErrorInvalidValue;
}

} // namespace ot
