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
#include <stdint.h>

#include "ot_internal.h"

namespace ot {

// VPL consecutive elements of a row per lane (VPL = d / 32), moved as one
// vector: 4, 8 or 16 bytes of bf16, 8, 16 or 32 bytes of fp32.
template <typename T, int VPL> struct RowVec {
    static_assert(VPL == 2 || VPL == 4 || VPL == 8, "2, 4 or 8 elements per lane");
    static constexpr int WORDS = VPL * static_cast<int>(sizeof(T)) / 4; // 32-bit words
    uint32_t w[WORDS];
    __device__ __forceinline__ void load(const T *p)
    {
        const uint32_t *q = reinterpret_cast<const uint32_t *>(p);
        if constexpr (WORDS % 4 == 0) {
#pragma unroll
            for (int i = 0; i < WORDS; i += 4) {
                const uint4 v = reinterpret_cast<const uint4 *>(q)[i / 4];
                w[i] = v.x, w[i + 1] = v.y, w[i + 2] = v.z, w[i + 3] = v.w;
            }
        } else if constexpr (WORDS == 2) {
            const uint2 v = *reinterpret_cast<const uint2 *>(q);
            w[0] = v.x, w[1] = v.y;
        } else {
            w[0] = q[0];
        }
    }
    __device__ __forceinline__ void store(T *p) const
    {
        uint32_t *q = reinterpret_cast<uint32_t *>(p);
        if constexpr (WORDS % 4 == 0) {
#pragma unroll
            for (int i = 0; i < WORDS; i += 4)
                reinterpret_cast<uint4 *>(q)[i / 4] = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
        } else if constexpr (WORDS == 2) {
            *reinterpret_cast<uint2 *>(q) = make_uint2(w[0], w[1]);
        } else {
            q[0] = w[0];
        }
    }
    __device__ __forceinline__ float get(int i) const
    {
        if constexpr (sizeof(T) == 4)
            return __uint_as_float(w[i]);
        else
            return __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
    }
    __device__ __forceinline__ void set(int i, float v)
    {
        if constexpr (sizeof(T) == 4) {
            w[i] = __float_as_uint(v);
        } else {
            const uint32_t b = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
            w[i >> 1] = (i & 1) ? ((w[i >> 1] & 0xFFFFu) | (b << 16)) : ((w[i >> 1] & 0xFFFF0000u) | b);
        }
    }
};

__device__ __forceinline__ float moe_warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

constexpr int MOE_THREADS = 256;
constexpr int MOE_WARPS = MOE_THREADS / 32;
constexpr int MOE_RPW = 4;                      // rows per warp per chunk
constexpr int MOE_CHUNK = MOE_WARPS * MOE_RPW;  // rows per CTA per chunk

// Router: the CTA stages the layer's router weights [E][d] in shared memory
// once, then takes chunks of MOE_CHUNK rows.  Slots are reserved per chunk:
// each choice takes a local slot from a shared-memory counter of its
// expert, then one global atomic per expert and chunk reserves the chunk's
// range of the expert's segment (the order of rows inside a segment is
// free: every row's FFN is computed on its own).
template <typename T, int VPL>
__global__ void __launch_bounds__(MOE_THREADS) moe_route_kernel(MoeRouteArgs a)
{
    extern __shared__ __align__(16) uint8_t moe_smem[];
    T *sWr = reinterpret_cast<T *>(moe_smem); // [E][d]
    __shared__ int s_cnt[64], s_base[64];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long wr_vec = static_cast<long long>(a.E) * a.d * sizeof(T) / 16;
    for (long long i = threadIdx.x; i < wr_vec; i += blockDim.x)
        reinterpret_cast<uint4 *>(sWr)[i] = reinterpret_cast<const uint4 *>(a.Wr)[i];
    RowVec<T, VPL> gv;
    gv.load(static_cast<const T *>(a.gain) + lane * VPL);
    for (long long c0 = static_cast<long long>(blockIdx.x) * MOE_CHUNK; c0 < a.rows;
         c0 += static_cast<long long>(gridDim.x) * MOE_CHUNK) {
        if (threadIdx.x < a.E) s_cnt[threadIdx.x] = 0;
        __syncthreads(); // also orders the router weights' staging before first use
        RowVec<T, VPL> hv[MOE_RPW];
        int ex[MOE_RPW][2], ls[MOE_RPW][2];
        float gt[MOE_RPW][2];
#pragma unroll
        for (int t = 0; t < MOE_RPW; ++t) {
            const long long r = c0 + warp * MOE_RPW + t;
            ex[t][0] = ex[t][1] = -1;
            if (r >= a.rows) continue; // warp-uniform
            hv[t].load(static_cast<const T *>(a.H) + r * a.d + lane * VPL);
            float z[VPL], ss = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                z[i] = hv[t].get(i);
                ss = fmaf(z[i], z[i], ss);
            }
            const float rs = 1.0f / sqrtf(moe_warp_sum(ss) / static_cast<float>(a.d) + a.eps);
#pragma unroll
            for (int i = 0; i < VPL; ++i) z[i] *= rs * gv.get(i);
            // top-2 of the router logits; a later expert replaces an earlier
            // one only with a strictly larger logit (ties to the lower index)
            float l1 = -INFINITY, l2 = -INFINITY;
            int e1 = 0, e2 = 0;
            for (int e = 0; e < a.E; ++e) {
                RowVec<T, VPL> wv;
                wv.load(sWr + static_cast<long long>(e) * a.d + lane * VPL);
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < VPL; ++i) acc = fmaf(z[i], wv.get(i), acc);
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
            gt[t][0] = 1.f;
            gt[t][1] = 0.f;
            if (a.topk == 2) {
                const float x = __expf(l2 - l1);
                gt[t][0] = 1.f / (1.f + x);
                gt[t][1] = x * gt[t][0];
            }
            ex[t][0] = e1;
            ex[t][1] = a.topk == 2 ? e2 : -1;
            int l0 = 0, l1s = 0;
            if (lane == 0) {
                l0 = atomicAdd(&s_cnt[e1], 1);
                if (a.topk == 2) l1s = atomicAdd(&s_cnt[e2], 1);
            }
            ls[t][0] = __shfl_sync(0xffffffffu, l0, 0);
            ls[t][1] = __shfl_sync(0xffffffffu, l1s, 0);
        }
        __syncthreads();
        if (threadIdx.x < a.E) s_base[threadIdx.x] = s_cnt[threadIdx.x] ? atomicAdd(a.counts + threadIdx.x, s_cnt[threadIdx.x]) : 0;
        __syncthreads();
#pragma unroll
        for (int t = 0; t < MOE_RPW; ++t) {
            const long long r = c0 + warp * MOE_RPW + t;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int e = ex[t][j];
                if (e < 0) continue; // warp-uniform
                const long long dst = static_cast<long long>(e) * a.cap + s_base[e] + ls[t][j];
                hv[t].store(static_cast<T *>(a.Hp) + dst * a.d + lane * VPL);
                if (lane == 0) {
                    a.route[r * 2 + j] = dst;
                    a.gate[r * 2 + j] = gt[t][j];
                }
            }
        }
        __syncthreads(); // s_cnt / s_base are rewritten by the next chunk
    }
}

template <typename T, int VPL>
__global__ void __launch_bounds__(MOE_THREADS) moe_combine_kernel(MoeCombineArgs a)
{
    const int lane = threadIdx.x & 31;
    const long long warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long r = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; r < a.rows;
         r += warps) {
        const bool two = a.topk == 2;
        RowVec<T, VPL> hv, y0, y1;
        hv.load(static_cast<const T *>(a.H) + r * a.d + lane * VPL);
        const float g0 = a.gate[r * 2], g1 = two ? a.gate[r * 2 + 1] : 0.f;
        y0.load(static_cast<const T *>(a.Yp) + a.route[r * 2] * a.d + lane * VPL);
        if (two) y1.load(static_cast<const T *>(a.Yp) + a.route[r * 2 + 1] * a.d + lane * VPL);
        RowVec<T, VPL> out;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const float h = hv.get(i);
            float y = fmaf(g0, y0.get(i) - h, h);
            if (two) y = fmaf(g1, y1.get(i) - h, y);
            out.set(i, y);
        }
        out.store(static_cast<T *>(a.Y) + r * a.d + lane * VPL);
    }
}

static int moe_blocks(long long rows)
{
    long long b = (rows * 32 + MOE_THREADS - 1) / MOE_THREADS;
    if (b > 148 * 8) b = 148 * 8;
    return b < 1 ? 1 : static_cast<int>(b);
}

static int moe_route_blocks(long long rows)
{
    long long b = (rows + MOE_CHUNK - 1) / MOE_CHUNK;
    if (b > 148 * 4) b = 148 * 4;
    return b < 1 ? 1 : static_cast<int>(b);
}

template <typename T, int VPL>
static cudaError_t route_launch(const MoeRouteArgs &a, cudaStream_t s)
{
    const size_t smem = static_cast<size_t>(a.E) * a.d * sizeof(T);
    auto k = moe_route_kernel<T, VPL>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    k<<<moe_route_blocks(a.rows), MOE_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t route_dispatch(const MoeRouteArgs &a, cudaStream_t s)
{
    switch (a.d / 32) {
    case 2: return route_launch<T, 2>(a, s);
    case 4: return route_launch<T, 4>(a, s);
    case 8: return route_launch<T, 8>(a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t combine_dispatch(const MoeCombineArgs &a, cudaStream_t s)
{
    const int blocks = moe_blocks(a.rows);
    switch (a.d / 32) {
    case 2: moe_combine_kernel<T, 2><<<blocks, MOE_THREADS, 0, s>>>(a); break;
    case 4: moe_combine_kernel<T, 4><<<blocks, MOE_THREADS, 0, s>>>(a); break;
    case 8: moe_combine_kernel<T, 8><<<blocks, MOE_THREADS, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// rows of 64, 128 or 256 elements (2, 4 or 8 per lane), 16-byte aligned
static bool moe_width_ok(int d) { return d == 64 || d == 128 || d == 256; }

cudaError_t launch_moe_route(const MoeRouteArgs &a, cudaStream_t s)
{
    if (!moe_width_ok(a.d) || a.E < 1 || a.E > 64 || a.topk < 1 || a.topk > 2 || a.topk > a.E)
        return cudaErrorInvalidValue;
    return a.dtype == OT_DTYPE_F32 ? route_dispatch<float>(a, s) : route_dispatch<__nv_bfloat16>(a, s);
}

cudaError_t launch_moe_combine(const MoeCombineArgs &a, cudaStream_t s)
{
    if (!moe_width_ok(a.d) || a.topk < 1 || a.topk > 2) return cudaErrorInvalidValue;
    return a.dtype == OT_DTYPE_F32 ? combine_dispatch<float>(a, s) : combine_dispatch<__nv_bfloat16>(a, s);
}

} // namespace ot
