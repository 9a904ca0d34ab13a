// FP8 (e4m3) operand preparation for the projections of the block.
//
// Activations: one warp per projection input row (several rows at a time
// for narrow rows), launched as a programmatic dependent of the producer of
// its input.  The row is read once
// (bf16), optionally RMSNorm-ed with its gain (y = x * rsqrt(mean(x^2) + eps)
// * gain) and converted to e4m3(y / s), round to nearest even, saturating.
// The scale s is the input tensor's fixed per-tensor scale when one is given
// (one fp32 value per projection input of a layer and parameter set, found
// by calibration), else the row's own amax / 448 (1 for an all-zero row):
// the calibration pass.  The quotient is taken as y * (1 / s), the
// reciprocal rounded to fp32 once per row: it differs from the correctly
// rounded y / s by at most an ulp of fp32, which moves an e4m3 code only
// when y / s lies that close to a rounding midpoint (about one element in
// 2^20), and keeps the pass bound by memory rather than by divisions.  Either way s does not depend on the other rows of
// the call, so a candidate's result does not depend on which other
// candidates share the batch.  The row's scale is written beside it and the
// GEMM epilogue multiplies the fp32 accumulator by it and by the weight
// matrix's own scale.  Optionally the row's amax is max-accumulated into its
// tensor's slot (calibration).
//
// Weights: one CTA per matrix computes its amax, then writes e4m3(w / s_w).
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int QR_MAX_CHUNKS = 6; // per lane: 6 x 8 elements -> rows up to 1536

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 u, float *v)
{
    const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(wd[e] << 16);
        v[2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u);
    }
}

// CH chunks of 8 elements per lane (rows up to 256 CH wide); RPW rows per
// warp at a time, all their loads issued before any arithmetic, so narrow
// rows keep as many bytes in flight as wide ones.
template <int CH, int RPW>
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16 *X, long long lda,
                                                         RowMap map, long long M, int G, int K,
                                                         const __nv_bfloat16 *gain,
                                                         long long gain_gstride, int norm,
                                                         float eps, QuantRule rule, uint8_t *q,
                                                         float *scale)
{
    pdl_launch_dependents();
    pdl_wait(); // X comes from the previous kernel; q may still be read by it
    const int lane = threadIdx.x & 31;
    const long long warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int chunks = K >> 3;
    const long long items = (M * G + RPW - 1) / RPW;
    for (long long w = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; w < items;
         w += warps) {
        long long arow[RPW];
        int grp[RPW];
        bool live[RPW];
        float v[RPW][CH][8];
#pragma unroll
        for (int t = 0; t < RPW; ++t) {
            const long long rr = w * RPW + t;
            live[t] = rr < M * G;
            const long long r = rr / G;
            grp[t] = static_cast<int>(rr % G);
            arow[t] = live[t] ? rowmap_apply(map, r, grp[t]) : 0;
            const uint4 *src = reinterpret_cast<const uint4 *>(X + arow[t] * lda);
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int c = lane + 32 * i;
                uint4 u = make_uint4(0, 0, 0, 0);
                if (live[t] && c < chunks) u = src[c];
                bf16x8_to_f32(u, v[t][i]);
            }
        }
#pragma unroll
        for (int t = 0; t < RPW; ++t) {
            if (!live[t]) continue; // warp-uniform
            const int g = grp[t];
            if (norm) {
                float ss = 0.f;
#pragma unroll
                for (int i = 0; i < CH; ++i)
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(v[t][i][e], v[t][i][e], ss);
                const float rs = 1.0f / sqrtf(warp_sum(ss) / static_cast<float>(K) + eps);
                const uint4 *gp = reinterpret_cast<const uint4 *>(gain + g * gain_gstride);
#pragma unroll
                for (int i = 0; i < CH; ++i) {
                    const int c = lane + 32 * i;
                    if (c >= chunks) continue;
                    float gv[8];
                    bf16x8_to_f32(gp[c], gv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[t][i][e] *= rs * gv[e];
                }
            }
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < CH; ++i)
#pragma unroll
                for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[t][i][e]));
            amax = warp_max(amax);
            // non-negative floats order like their bit patterns as signed ints
            if (rule.amax && lane == 0)
                atomicMax(reinterpret_cast<int *>(rule.amax + g * rule.gstride), __float_as_int(amax));
            const float s = rule.xscale ? rule.xscale[g * rule.gstride]
                            : amax > 0.f ? __fdiv_rn(amax, 448.0f)
                                         : 1.0f;
            const float inv = __frcp_rn(s);
            uint2 *dst = reinterpret_cast<uint2 *>(q + arow[t] * K);
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int c = lane + 32 * i;
                if (c >= chunks) continue;
                uint32_t packed[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float *x = v[t][i] + 4 * h;
                    __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[0] * inv, x[1] * inv),
                                                                       __NV_SATFINITE, __NV_E4M3);
                    __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(x[2] * inv, x[3] * inv),
                                                                       __NV_SATFINITE, __NV_E4M3);
                    packed[h] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
                }
                dst[c] = make_uint2(packed[0], packed[1]);
            }
            if (lane == 0) scale[arow[t]] = s;
        }
    }
}

template <int CH, int RPW>
static cudaError_t quant_launch(const void *X, long long lda, RowMap map, long long M, int G, int K,
                                const void *gain, long long gain_gstride, int norm, float eps, QuantRule rule,
                                uint8_t *q_out, float *scale_out, cudaStream_t s)
{
    const long long items = (M * G + RPW - 1) / RPW;
    long long blocks = (items * 32 + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    return launch_pdl(quant_rows_kernel<CH, RPW>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                      static_cast<const __nv_bfloat16 *>(X), lda, map, M, G, K,
                      static_cast<const __nv_bfloat16 *>(gain), gain_gstride, norm, eps, rule, q_out, scale_out);
}

cudaError_t launch_quant_rows(const void *X, long long lda, RowMap map, long long M, int G, int K,
                              const void *gain, long long gain_gstride, int norm, float eps,
                              QuantRule rule, uint8_t *q_out, float *scale_out, cudaStream_t s)
{
    if (K % 8 || K > QR_MAX_CHUNKS * 8 * 32) return cudaErrorInvalidValue;
    switch ((K + 255) / 256) {
    case 1: return quant_launch<1, 6>(X, lda, map, M, G, K, gain, gain_gstride, norm, eps, rule, q_out, scale_out, s);
    case 2: return quant_launch<2, 3>(X, lda, map, M, G, K, gain, gain_gstride, norm, eps, rule, q_out, scale_out, s);
    case 3: return quant_launch<3, 2>(X, lda, map, M, G, K, gain, gain_gstride, norm, eps, rule, q_out, scale_out, s);
    case 4: return quant_launch<4, 1>(X, lda, map, M, G, K, gain, gain_gstride, norm, eps, rule, q_out, scale_out, s);
    case 5: return quant_launch<5, 1>(X, lda, map, M, G, K, gain, gain_gstride, norm, eps, rule, q_out, scale_out, s);
    default: return quant_launch<6, 1>(X, lda, map, M, G, K, gain, gain_gstride, norm, eps, rule, q_out, scale_out, s);
    }
}

__global__ void __launch_bounds__(1024) quant_weights_kernel(const __nv_bfloat16 *W,
                                                             long long per_mat, uint8_t *q,
                                                             float *scale)
{
    __shared__ float red[32];
    const long long base = static_cast<long long>(blockIdx.x) * per_mat;
    float amax = 0.f;
    for (long long e = threadIdx.x; e < per_mat; e += blockDim.x)
        amax = fmaxf(amax, fabsf(__bfloat162float(W[base + e])));
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        v = warp_max(v);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float s = red[0] > 0.f ? __fdiv_rn(red[0], 448.0f) : 1.0f;
    for (long long e = threadIdx.x; e < per_mat; e += blockDim.x)
        q[base + e] = static_cast<uint8_t>(
            __nv_cvt_float_to_fp8(__fdiv_rn(__bfloat162float(W[base + e]), s), __NV_SATFINITE,
                                  __NV_E4M3));
    if (threadIdx.x == 0) scale[blockIdx.x] = s;
}

cudaError_t launch_quant_weights(const void *W, long long per_mat, long long mats, uint8_t *q_out,
                                 float *scale_out, float *, cudaStream_t s)
{
    quant_weights_kernel<<<static_cast<int>(mats), 1024, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(W), per_mat, q_out, scale_out);
    return cudaGetLastError();
}

} // namespace ot
