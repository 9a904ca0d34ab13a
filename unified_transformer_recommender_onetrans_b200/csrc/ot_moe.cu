// Sparse mixture of experts as the S-side FFN of a block (the OneTrans-V2
// summary page names a sparse MoE for capacity and gives no recipe; the
// library's reading: the shared S-side FFN becomes E expert FFNs of the
// dense shape, a linear router on the FFN's normalised input picks the top-k
// experts, ties to the lower index, softmax over the chosen logits gives the
// gates, y = h + sum_j g_j FFN_e(j)(n(h)); NS tokens keep their dense FFNs).
//
// Three steps around the experts' FFN:
//   route   one warp per S row h: the RMSNorm row scale, z = h r g2, the E
//           router logits z . W_r[e] (fp32), the top-k (k <= 2) and their
//           softmax gates; each choice takes a slot in its expert's segment
//           (atomic counter) and the row is copied there, so the experts'
//           FFN reads contiguous expert-major rows [E][cap][d];
//   experts the FFN kernels over the E segments (only the counted rows of a
//           segment are computed on the fused path);
//   combine one warp per row: y = h + sum_j g_j (Y[slot_j] - h), where
//           Y = h + FFN_e(n(h)) is what the experts' FFN wrote for the slot.
#include <cuda_bf16.h>
#include <math.h>

#include "ot_internal.h"

namespace ot {

template <typename T> __device__ __forceinline__ float ld_elem(const T *p);
template <> __device__ __forceinline__ float ld_elem<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ld_elem<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ T st_elem(float v);
template <> __device__ __forceinline__ float st_elem<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 st_elem<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float moe_warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

constexpr int MOE_MAX_PER_LANE = 8; // rows up to 256 wide

template <typename T>
__global__ void __launch_bounds__(256) moe_route_kernel(MoeRouteArgs a)
{
    const int lane = threadIdx.x & 31;
    const long long warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int per = a.d / 32;
    for (long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; r < a.rows;
         r += warps) {
        const T *h = static_cast<const T *>(a.H) + r * a.d;
        const T *g = static_cast<const T *>(a.gain);
        float x[MOE_MAX_PER_LANE], z[MOE_MAX_PER_LANE];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < MOE_MAX_PER_LANE; ++i) {
            x[i] = i < per ? ld_elem<T>(h + lane + 32 * i) : 0.f;
            ss = fmaf(x[i], x[i], ss);
        }
        const float rs = 1.0f / sqrtf(moe_warp_sum(ss) / static_cast<float>(a.d) + a.eps);
#pragma unroll
        for (int i = 0; i < MOE_MAX_PER_LANE; ++i)
            z[i] = i < per ? x[i] * rs * ld_elem<T>(g + lane + 32 * i) : 0.f;
        // top-2 of the router logits; a later expert replaces an earlier one
        // only with a strictly larger logit (ties to the lower index)
        float l1 = -INFINITY, l2 = -INFINITY;
        int e1 = 0, e2 = 0;
        for (int e = 0; e < a.E; ++e) {
            const T *wr = static_cast<const T *>(a.Wr) + static_cast<long long>(e) * a.d;
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < MOE_MAX_PER_LANE; ++i)
                if (i < per) acc = fmaf(z[i], ld_elem<T>(wr + lane + 32 * i), acc);
            const float lg = moe_warp_sum(acc);
            if (lg > l1) {
                l2 = l1;
                e2 = e1;
                l1 = lg;
                e1 = e;
            } else if (lg > l2) {
                l2 = lg;
                e2 = e;
            }
        }
        // gates: softmax over the chosen logits
        float g1 = 1.f, g2 = 0.f;
        if (a.topk == 2) {
            const float t = __expf(l2 - l1);
            g1 = 1.f / (1.f + t);
            g2 = t * g1;
        }
        for (int j = 0; j < a.topk; ++j) {
            const int e = j == 0 ? e1 : e2;
            int slot = 0;
            if (lane == 0) slot = atomicAdd(a.counts + e, 1);
            slot = __shfl_sync(0xffffffffu, slot, 0);
            const long long dst = static_cast<long long>(e) * a.cap + slot;
            T *hp = static_cast<T *>(a.Hp) + dst * a.d;
#pragma unroll
            for (int i = 0; i < MOE_MAX_PER_LANE; ++i)
                if (i < per) hp[lane + 32 * i] = h[lane + 32 * i];
            if (lane == 0) {
                a.route[r * 2 + j] = dst;
                a.gate[r * 2 + j] = j == 0 ? g1 : g2;
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(256) moe_combine_kernel(MoeCombineArgs a)
{
    const int lane = threadIdx.x & 31;
    const long long warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int per = a.d / 32;
    for (long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; r < a.rows;
         r += warps) {
        const T *h = static_cast<const T *>(a.H) + r * a.d;
        float y[MOE_MAX_PER_LANE], hv[MOE_MAX_PER_LANE];
#pragma unroll
        for (int i = 0; i < MOE_MAX_PER_LANE; ++i) {
            hv[i] = i < per ? ld_elem<T>(h + lane + 32 * i) : 0.f;
            y[i] = hv[i];
        }
        for (int j = 0; j < a.topk; ++j) {
            const long long src = a.route[r * 2 + j];
            const float gj = a.gate[r * 2 + j];
            const T *yp = static_cast<const T *>(a.Yp) + src * a.d;
#pragma unroll
            for (int i = 0; i < MOE_MAX_PER_LANE; ++i)
                if (i < per) y[i] = fmaf(gj, ld_elem<T>(yp + lane + 32 * i) - hv[i], y[i]);
        }
        T *out = static_cast<T *>(a.Y) + r * a.d;
#pragma unroll
        for (int i = 0; i < MOE_MAX_PER_LANE; ++i)
            if (i < per) out[lane + 32 * i] = st_elem<T>(y[i]);
    }
}

static int moe_blocks(long long rows)
{
    long long b = (rows * 32 + 255) / 256;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : static_cast<int>(b);
}

cudaError_t launch_moe_route(const MoeRouteArgs &a, cudaStream_t s)
{
    if (a.d % 32 || a.d / 32 > MOE_MAX_PER_LANE || a.E < 1 || a.E > 64 || a.topk < 1 || a.topk > 2 ||
        a.topk > a.E)
        return cudaErrorInvalidValue;
    if (a.dtype == OT_DTYPE_F32)
        moe_route_kernel<float><<<moe_blocks(a.rows), 256, 0, s>>>(a);
    else
        moe_route_kernel<__nv_bfloat16><<<moe_blocks(a.rows), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_moe_combine(const MoeCombineArgs &a, cudaStream_t s)
{
    if (a.d % 32 || a.d / 32 > MOE_MAX_PER_LANE || a.topk < 1 || a.topk > 2) return cudaErrorInvalidValue;
    if (a.dtype == OT_DTYPE_F32)
        moe_combine_kernel<float><<<moe_blocks(a.rows), 256, 0, s>>>(a);
    else
        moe_combine_kernel<__nv_bfloat16><<<moe_blocks(a.rows), 256, 0, s>>>(a);
    return cudaGetLastError();
}

} // namespace ot
