// Sparse mixture of experts in the backward pass (fp32, CUDA cores): the
// S-side FFN of a block as E expert FFNs behind a linear router on the FFN's
// normalised input z (the top-k logits, ties to the lower expert index,
// softmax-ed into gates; y = h + sum_j g_j FFN_e(j)(z)).
//
// Forward pieces (recomputed per layer like the rest of the block):
//   topk      one warp per row: the k largest of the E logits and the gates
//   rank      one thread per 128-row chunk: per expert, how many of the
//             chunk's choices come before each choice (a serial count, so
//             the order is fixed: no atomics)
//   offsets   one thread per expert: the expert's segment start and the
//             start of every chunk's share in it
//   dispatch  the slot of every choice (segment start + chunk share + rank)
//             and z copied there: expert-major rows, chunks in row order
//   combine   y = h + sum_j g_j Y[slot_j]
// Backward pieces:
//   combine'  one warp per row: dg_j = dy . Y[slot_j], dY[slot_j] = g_j dy,
//             the gate softmax backward into the row's E logit gradients
//   gather    dz[row] += sum_j dZ[slot_j]
// The experts' FFNs and their gradients are the grouped GEMMs with segments
// (group = expert).
#include <math.h>
#include <stdint.h>

#include "ot_internal.h"

namespace ot {

namespace {

constexpr int MB_CH = 128; // rows per ranking chunk

__device__ __forceinline__ long long mb_warp_id()
{
    return (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
}

__device__ __forceinline__ long long mb_warps() { return (static_cast<long long>(gridDim.x) * blockDim.x) >> 5; }

__device__ __forceinline__ float mb_warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// the larger of (v, e) and (ov, oe); equal values: the lower expert index
__device__ __forceinline__ void mb_better(float &v, int &e, float ov, int oe)
{
    if (ov > v || (ov == v && oe < e)) {
        v = ov;
        e = oe;
    }
}

// warp arg-max over the lanes' (v, e), ties to the lower index
__device__ __forceinline__ void mb_warp_argmax(float &v, int &e)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oe = __shfl_xor_sync(0xffffffffu, e, o);
        mb_better(v, e, ov, oe);
    }
}

__global__ void moe_topk_kernel(const float *logits, int T, int E, int k, int *sel, float *gate)
{
    const int lane = threadIdx.x & 31;
    for (long long r = mb_warp_id(); r < T; r += mb_warps()) {
        const float *lg = logits + r * E;
        // lane holds experts lane and lane + 32; a NaN logit counts as -inf,
        // so every comparison below is ordered and the chosen indices stay
        // below E (an unordered one could leave the out-of-range marker)
        float v0 = lane < E ? lg[lane] : -INFINITY, v1 = lane + 32 < E ? lg[lane + 32] : -INFINITY;
        if (v0 != v0) v0 = -INFINITY;
        if (v1 != v1) v1 = -INFINITY;
        float bv = v0;
        int be = lane < E ? lane : 1 << 20;
        mb_better(bv, be, v1, lane + 32 < E ? lane + 32 : 1 << 20);
        mb_warp_argmax(bv, be);
        const float l1 = bv;
        const int e1 = be;
        float l2 = -INFINITY;
        int e2 = e1;
        if (k == 2) {
            float cv = lane == e1 ? -INFINITY : v0;
            int ce = lane < E && lane != e1 ? lane : 1 << 20;
            if (lane + 32 < E && lane + 32 != e1) mb_better(cv, ce, v1, lane + 32);
            mb_warp_argmax(cv, ce);
            l2 = cv;
            e2 = ce;
        }
        if (lane == 0) {
            sel[r * 2] = e1;
            sel[r * 2 + 1] = e2;
            if (k == 2) {
                const float t = expf(l2 - l1);
                gate[r * 2] = 1.0f / (1.0f + t);
                gate[r * 2 + 1] = t / (1.0f + t);
            } else {
                gate[r * 2] = 1.0f;
                gate[r * 2 + 1] = 0.0f;
            }
        }
    }
}

// chunk c: rows [c * MB_CH, ...): hist[c][e] = choices of expert e in it,
// lrank[r][j] = choices of the same expert before (r, j) in the chunk
__global__ void moe_rank_kernel(const int *sel, int T, int E, int k, int *hist, int *lrank)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int r0 = c * MB_CH;
    if (r0 >= T) return;
    int cnt[64];
    for (int e = 0; e < E; ++e) cnt[e] = 0;
    const int r1 = min(T, r0 + MB_CH);
    for (int r = r0; r < r1; ++r)
        for (int j = 0; j < k; ++j) {
            const int e = sel[r * 2 + j];
            lrank[r * 2 + j] = cnt[e]++;
        }
    for (int e = 0; e < E; ++e) hist[static_cast<long long>(c) * E + e] = cnt[e];
}

// expert e: seg_off[e] = choices of the experts before e, seg_cnt[e] its
// own; hist[c][e] becomes the start of chunk c's share of the segment
__global__ void moe_offsets_kernel(int *hist, int chunks, int E, int *seg_off, int *seg_cnt)
{
    __shared__ int tot[64];
    const int e = threadIdx.x;
    if (e < E) {
        int s = 0;
        for (int c = 0; c < chunks; ++c) s += hist[static_cast<long long>(c) * E + e];
        tot[e] = s;
    }
    __syncthreads();
    if (e < E) {
        int off = 0;
        for (int i = 0; i < e; ++i) off += tot[i];
        seg_off[e] = off;
        seg_cnt[e] = tot[e];
        for (int c = 0; c < chunks; ++c) {
            const long long at = static_cast<long long>(c) * E + e;
            const int h = hist[at];
            hist[at] = off;
            off += h;
        }
    }
}

// slot[r][j] and the expert-major copy Zp[slot] = z[r]
__global__ void moe_dispatch_kernel(const float *z, int T, int d, int E, int k, const int *sel, const int *lrank,
                                    const int *base, int *slot, float *Zp)
{
    const long long n = static_cast<long long>(T) * k * d;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long rj = i / d;
        const int c = static_cast<int>(i % d);
        const int r = static_cast<int>(rj / k), j = static_cast<int>(rj % k);
        const int e = sel[r * 2 + j];
        const int s = base[static_cast<long long>(r / MB_CH) * E + e] + lrank[r * 2 + j];
        if (c == 0) slot[r * 2 + j] = s;
        Zp[static_cast<long long>(s) * d + c] = z[static_cast<long long>(r) * d + c];
    }
}

__global__ void moe_combine_fwd_kernel(const float *h, const float *Y, const int *slot, const float *gate, int T,
                                       int d, int k, float *y)
{
    const long long n = static_cast<long long>(T) * d;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long r = i / d;
        const int c = static_cast<int>(i % d);
        float v = h[i];
        for (int j = 0; j < k; ++j) v = fmaf(gate[r * 2 + j], Y[static_cast<long long>(slot[r * 2 + j]) * d + c], v);
        y[i] = v;
    }
}

__global__ void moe_combine_bwd_kernel(const float *dy, const float *Y, const int *slot, const int *sel,
                                       const float *gate, int T, int d, int E, int k, float *dY, float *dlogits)
{
    const int lane = threadIdx.x & 31;
    for (long long r = mb_warp_id(); r < T; r += mb_warps()) {
        const float *dyr = dy + r * d;
        float dg[2] = {0.f, 0.f};
        for (int j = 0; j < k; ++j) {
            const long long s = slot[r * 2 + j];
            const float g = gate[r * 2 + j];
            float acc = 0.f;
            for (int c = lane; c < d; c += 32) {
                acc = fmaf(dyr[c], Y[s * d + c], acc);
                dY[s * d + c] = g * dyr[c];
            }
            dg[j] = mb_warp_sum(acc);
        }
        // gates = softmax(chosen logits): dlogit_j = g_j (dg_j - sum_i g_i dg_i)
        float gd = 0.f;
        for (int j = 0; j < k; ++j) gd = fmaf(gate[r * 2 + j], dg[j], gd);
        for (int e = lane; e < E; e += 32) {
            float v = 0.f;
            for (int j = 0; j < k; ++j)
                if (sel[r * 2 + j] == e) v = gate[r * 2 + j] * (dg[j] - gd);
            dlogits[r * E + e] = v;
        }
    }
}

__global__ void moe_gather_kernel(const float *dZp, const int *slot, int T, int d, int k, float *dz)
{
    const long long n = static_cast<long long>(T) * d;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long r = i / d;
        const int c = static_cast<int>(i % d);
        float v = dz[i];
        for (int j = 0; j < k; ++j) v += dZp[static_cast<long long>(slot[r * 2 + j]) * d + c];
        dz[i] = v;
    }
}

int mb_blocks(long long threads)
{
    long long b = (threads + 255) / 256;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : static_cast<int>(b);
}

} // namespace

int bw_moe_chunks(int T) { return (T + MB_CH - 1) / MB_CH; }

cudaError_t bw_moe_route(const BwMoe &m, const float *z, float *Zp, cudaStream_t s)
{
    if (m.E < 1 || m.E > 64 || m.k < 1 || m.k > 2 || m.k > m.E) return cudaErrorInvalidValue;
    moe_topk_kernel<<<mb_blocks(static_cast<long long>(m.T) * 32), 256, 0, s>>>(m.logits, m.T, m.E, m.k, m.sel,
                                                                                m.gate);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int chunks = bw_moe_chunks(m.T);
    moe_rank_kernel<<<(chunks + 127) / 128, 128, 0, s>>>(m.sel, m.T, m.E, m.k, m.hist, m.lrank);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    moe_offsets_kernel<<<1, 64, 0, s>>>(m.hist, chunks, m.E, m.seg_off, m.seg_cnt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    moe_dispatch_kernel<<<mb_blocks(static_cast<long long>(m.T) * m.k * m.d), 256, 0, s>>>(
        z, m.T, m.d, m.E, m.k, m.sel, m.lrank, m.hist, m.slot, Zp);
    return cudaGetLastError();
}

cudaError_t bw_moe_combine(const BwMoe &m, const float *h, const float *Y, float *y, cudaStream_t s)
{
    moe_combine_fwd_kernel<<<mb_blocks(static_cast<long long>(m.T) * m.d), 256, 0, s>>>(h, Y, m.slot, m.gate, m.T,
                                                                                       m.d, m.k, y);
    return cudaGetLastError();
}

cudaError_t bw_moe_combine_bwd(const BwMoe &m, const float *dy, const float *Y, float *dY, float *dlogits,
                               cudaStream_t s)
{
    moe_combine_bwd_kernel<<<mb_blocks(static_cast<long long>(m.T) * 32), 256, 0, s>>>(dy, Y, m.slot, m.sel, m.gate,
                                                                                       m.T, m.d, m.E, m.k, dY, dlogits);
    return cudaGetLastError();
}

cudaError_t bw_moe_gather(const BwMoe &m, const float *dZp, float *dz, cudaStream_t s)
{
    moe_gather_kernel<<<mb_blocks(static_cast<long long>(m.T) * m.d), 256, 0, s>>>(dZp, m.slot, m.T, m.d, m.k, dz);
    return cudaGetLastError();
}

} // namespace ot
