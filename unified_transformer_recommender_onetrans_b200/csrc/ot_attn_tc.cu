// tcgen05 attention for one layer of the block (head_dim 64, bf16 operands,
// fp32 scores and softmax).  Persistent: one CTA per SM walks a list of work
// items, each a (user, head) and two 128-query tiles (256 consecutive query
// rows), or, in NS mode's split-key form, one 128-query tile whose key blocks
// the two tiles of the CTA share out; the next item's Q and K/V loads and its
// first scores overlap the current item's last blocks and output read-out.
//
// Key blocks of 128 rows are visited in order: first the user's S keys (from
// the KV cache), then, in NS mode, the NS keys of the candidates the item's
// rows belong to.  Visibility (the OneTrans mask):
//   S mode  : query i is S row t = L - nq + i (the pyramid tail, bottom-right
//             aligned); it sees S keys 0..t.  Blocks past the item's last row
//             are never loaded.
//   NS mode : query i is NS token n = i % N of candidate c = i / N; it sees
//             every S key 0..L-1 and NS keys m <= n of candidate c.  Each
//             cached S K/V tile is read once per item and shared by all the
//             item's candidates (256 / N of them).
//   full attention (AttnArgs::full, one candidate per user): an S row sees
//             every S key and then the user's nkn NS keys, which follow the S
//             blocks in its item; an NS row every NS key of its candidate.
//
// A tcgen05.mma issued from one thread takes about 100-130 cycles whatever
// its N up to 128, so at head_dim 64 (12 MMAs per tile and key block) the
// kernel is bound by MMA issue unless both tiles have their own issuer.
//   warp 0      TMA: Q of both tiles into one of two Q buffers (item parity),
//               K/V blocks through a 5-deep ring that runs on across items.
//   warps 1, 2  MMA issuers of tiles 0 and 1 (warp 1 also owns the 512 TMEM
//               columns: tile w uses S at 256 w, P at 256 w + 128, O at
//               256 w + 192).  Per key block b: once the softmax holds S(b) in
//               registers, S(b+1) = Q K^T (4 MMAs, operands in shared memory)
//               goes into the S columns, overlapping the exponentials; once
//               P(b) is stored, O += P(b) V (8 MMAs, P from TMEM, V MN-major
//               from its row-major tile).  A tile with no live query row gets
//               no MMAs, only the signals.  In S mode (one tile per CTA,
//               two CTAs per SM, see AtCfg) warp 1 issues the S MMAs and
//               warp 2 the PV MMAs.
//   warp 3      idle (it completes the producer warpgroup, whose registers
//               go to the softmax warpgroups through setmaxnreg).
//   warps 4-7   softmax warpgroup of tile 0, warps 8-11 of tile 1: one query
//               row per thread, its 128 scores read from TMEM in one round
//               trip; block max, lazy running max (O and l rescaled only when
//               the max grows by more than 2^8), p = 2^(s c2 - m) on the
//               special-function unit, P packed to bf16 into TMEM.  Warp-
//               uniform fast paths: no mask arithmetic on blocks every row of
//               the warp fully sees, no exponentials on blocks no row of the
//               warp sees (or whose rows are all past nq).  At the end of an
//               item the warpgroup reads O out of TMEM, frees it for the next
//               item's first PV, and stores O / l.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "ot_internal.h"
#include "ot_ptx.cuh"

namespace ot {

constexpr int AT_BM = 128;  // query rows per tile
constexpr int AT_BK = 128;  // keys per block
constexpr int AT_HD = 64;
constexpr uint32_t AT_TILE = AT_BM * 128; // 16 KB: 128 rows x 128 bytes
constexpr int AT_QBUF = 2;                // Q buffers (items in flight)
// Q[AT_QBUF][TILES], then per stage K and V, then barriers, then the
// split-key exchange (tile 1's running max and sum per row)
constexpr size_t AT_BAR_BYTES = 256;
constexpr size_t AT_XCH_BYTES = AT_BM * 2 * sizeof(float);

// Two shapes of the persistent kernel:
//   TILES = 2  one CTA per SM with two 128-row query tiles (all 512 TMEM
//              columns), a 5-deep K/V ring shared by both tiles; split-key
//              NS items (their two tiles share the key blocks of one row
//              tile);
//   TILES = 1  two CTAs per SM, one tile each (256 TMEM columns, a 2-deep
//              ring per CTA): S items and the other NS items.  The two
//              tiles of an SM run independent pipelines and drift out of
//              step, so one softmax warpgroup's exponentials overlap the
//              other's waits (OneTransS layer-0 S attention 0.140 -> 0.132
//              ms, NS attention of 16 x 512 candidates 1.755 -> 1.714 ms
//              against TILES = 2).
// Register split (setmaxnreg): the producer warpgroup (TMA warp, MMA warps,
// idle warps) drops to REG_PRODUCER per thread and the softmax warpgroups
// rise to REG_SOFTMAX, which holds a row's 128 scores at once.  The sum must
// stay within what the launch allocated (registers per thread x THREADS);
// the launcher checks it against the compiled kernel.
template <int TILES> struct AtCfg {
    static_assert(TILES == 1 || TILES == 2, "one or two tiles per CTA");
    static constexpr int STAGES = TILES == 1 ? 2 : 5;       // K/V ring depth
    static constexpr int CTAS = TILES == 1 ? 2 : 1;         // CTAs per SM
    static constexpr int THREADS = 128 * (1 + TILES);       // producer warpgroup + a softmax warpgroup per tile
    static constexpr int REG_PRODUCER = TILES == 1 ? 40 : 64;
    static constexpr int REG_SOFTMAX = 216;
    static constexpr size_t SMEM = (AT_QBUF * TILES + 2 * STAGES) * AT_TILE + AT_BAR_BYTES + AT_XCH_BYTES;
    static_assert((2 * AT_QBUF + 2 * STAGES + 6 * TILES + 2) * 8 + 8 <= AT_BAR_BYTES, "barrier area");
    static_assert(CTAS * (SMEM + 1024) <= 228 * 1024, "shared memory per SM");
    static_assert(128 * REG_PRODUCER + 128 * TILES * REG_SOFTMAX <= 65536 / CTAS, "register split");
};

// Lazy rescale threshold (base-2): the running max moves only when it would
// grow by more than 2^8; until then p <= 2^8, well inside fp32 / bf16 range.
constexpr float AT_RESCALE_LOG2 = 8.0f;

// Softmax of one row of one key block against the running max m (base-2
// units).  The row's 128 scores are read from TMEM in one round trip, after
// which released() lets the MMA warp reuse the S columns; then
//   1. the block's max over all 128 scores (keys the row cannot see included:
//      a larger reference max leaves the softmax unchanged); m takes it on
//      the row's first block and is raised later only when the block's max
//      exceeds it by more than 2^8 (so p <= 2^8); alpha is the factor O and
//      l must then be rescaled by, 1 otherwise;
//   2. p = 2^(s c2 - m) for the visible keys [klo, khi], 0 elsewhere, packed
//      to bf16 pairs (pk[q][j] holds keys 32 q + 2j, 32 q + 2j + 1) and
//      summed into rsum.  FULL: every key of the block is visible (no mask).
template <bool FULL, typename Released>
__device__ __forceinline__ void softmax_unit(uint32_t tS_row, float c2, int klo, int khi, float &m,
                                             uint32_t (&pk)[4][16], float &alpha, float &rsum,
                                             Released &&released)
{
    uint32_t v[4][32];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld32(tS_row + 32 * q, v[q]);
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_reg_fence(v[q]);
    released();
    // four independent chains of three-input maxima: 64 instructions for 128 scores
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 32; e += 2)
            mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1]));
    const float mb = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * c2;
    alpha = 1.f;
    if (m == -INFINITY) {
        m = mb; // the row's first block: l is 0 and O holds nothing for it
    } else if (mb > m + AT_RESCALE_LOG2) {
        alpha = fast_exp2(m - mb);
        m = mb;
    }
    // per pair of scores: one packed FMA for the exponents, two exponentials,
    // one packed add into the row sum (two independent pair accumulators)
    const uint64_t c2x2 = f32x2(c2, c2), mnx2 = f32x2(-m, -m);
    uint64_t rs2[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float x0, x1;
            f32x2_split(fma_f32x2(f32x2(__uint_as_float(v[q][2 * j]), __uint_as_float(v[q][2 * j + 1])), c2x2,
                                  mnx2),
                        x0, x1);
            float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            if (!FULL) {
                const int k = 32 * q + 2 * j;
                p0 = (k >= klo && k <= khi) ? p0 : 0.f;
                p1 = (k + 1 >= klo && k + 1 <= khi) ? p1 : 0.f;
            }
            rs2[j & 1] = add_f32x2(rs2[j & 1], f32x2(p0, p1));
            pk[q][j] = pack_bf16x2(p0, p1);
        }
    float a0, a1, b0, b1;
    f32x2_split(rs2[0], a0, a1);
    f32x2_split(rs2[1], b0, b1);
    rsum = (a0 + b0) + (a1 + b1);
}

// One work item of the persistent kernel (FA: full attention, AttnArgs::full): a (user, head, query pair) and its
// key-block schedule, shared by every role of the CTA.
struct AtItem {
    int u, h, i0;     // user, head, first query row of the pair
    int n_s_blocks;   // S key blocks
    int k_begin;      // NS mode: first NS key row of the pair's candidates
    int n_blocks;     // S blocks + NS blocks
};

// Query rows per item: two tiles of 128, or one in split-key mode, where
// both tiles of the CTA work on the same rows.
template <bool SPLIT, int TILES> __host__ __device__ constexpr int at_item_rows()
{
    return SPLIT ? AT_BM : AT_BM * TILES;
}

// Item k.  S mode orders the pairs longest first (pairs later in the tail see
// more keys), so the snake assignment below balances the CTAs; NS mode keeps
// the pairs (row tiles in split-key mode) of one (user, head) together so
// they share K/V tiles in L2.
template <bool NS, bool SPLIT, bool FA, int TILES>
__device__ __forceinline__ AtItem at_item(const AttnArgs &a, int n_pairs, int k)
{
    AtItem it;
    int pair, uh;
    if (!NS) {
        const int UH = a.U * a.H;
        pair = n_pairs - 1 - k / UH;
        uh = k % UH;
    } else {
        pair = k % n_pairs;
        uh = k / n_pairs;
    }
    it.u = uh / a.H;
    it.h = uh % a.H;
    it.i0 = pair * at_item_rows<SPLIT, TILES>();
    const int i_last = min(it.i0 + at_item_rows<SPLIT, TILES>(), a.nq) - 1;
    it.k_begin = 0;
    if (!NS) {
        // causal: the keys up to the item's last row; full attention: every
        // S key, then the user's NS keys
        const int t_last = a.L - a.nq + i_last;
        it.n_s_blocks = FA ? (a.L + AT_BK - 1) / AT_BK : (t_last + AT_BK) / AT_BK;
        it.n_blocks = it.n_s_blocks + (FA ? (a.nkn + AT_BK - 1) / AT_BK : 0);
    } else {
        it.n_s_blocks = (a.L + AT_BK - 1) / AT_BK;
        it.k_begin = (it.i0 / a.N) * a.N;
        const int k_end = (i_last / a.N + 1) * a.N;
        it.n_blocks = it.n_s_blocks + (k_end - it.k_begin + AT_BK - 1) / AT_BK;
    }
    return it;
}

// The r-th item of this CTA, or -1: rounds of gridDim.x items, walked
// forwards in even rounds and backwards in odd ones (with longest-first items
// every CTA then gets a similar total).
__device__ __forceinline__ int at_item_of(int r, int n_items)
{
    const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    const long long k = static_cast<long long>(r) * G + ((r & 1) ? G - 1 - c : c);
    return k < n_items ? static_cast<int>(k) : -1;
}

// The key blocks tile w works on, in order, across this CTA's items.  Every
// tile takes every block, except in split-key mode (SPLIT: NS mode with
// items of one 128-row tile), where tile w takes the blocks b = w (mod 2) of
// an item and the two tiles' partial softmax states are merged at its end.
// gb counts all blocks of the CTA (the K/V ring position), lb this tile's.
template <bool NS, bool SPLIT, bool FA, int TILES>
struct BlockCursor {
    int r, k;      // item ordinal within the CTA, item index (k < 0: past the end)
    AtItem it;
    int b;         // block within the item
    int w;         // tile
    long long gb;  // global block counter of the CTA
    long long lb;  // blocks of this tile before this one
    __device__ __forceinline__ bool owned() const { return !SPLIT || (b & 1) == w; }
    __device__ __forceinline__ void step(const AttnArgs &a, int n_pairs, int n_items)
    {
        ++gb;
        if (++b < it.n_blocks) return;
        b = 0;
        k = at_item_of(++r, n_items);
        if (k >= 0) it = at_item<NS, SPLIT, FA, TILES>(a, n_pairs, k);
    }
    __device__ __forceinline__ void init(const AttnArgs &a, int n_pairs, int n_items, int tile)
    {
        w = tile;
        r = 0;
        b = 0;
        gb = 0;
        lb = 0;
        k = at_item_of(0, n_items);
        if (k >= 0) it = at_item<NS, SPLIT, FA, TILES>(a, n_pairs, k);
        while (valid() && !owned()) step(a, n_pairs, n_items);
    }
    __device__ __forceinline__ void next(const AttnArgs &a, int n_pairs, int n_items)
    {
        ++lb;
        do step(a, n_pairs, n_items);
        while (valid() && !owned());
    }
    __device__ __forceinline__ bool valid() const { return k >= 0; }
    __device__ __forceinline__ bool first_in_item() const { return b == (SPLIT ? w : 0); }
    __device__ __forceinline__ bool last_in_item() const
    {
        return SPLIT ? b + 2 >= it.n_blocks : b == it.n_blocks - 1;
    }
};

template <bool NS, bool SPLIT, bool FA, int TILES>
__global__ void __launch_bounds__(AtCfg<TILES>::THREADS, AtCfg<TILES>::CTAS)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKS,
                   const __grid_constant__ CUtensorMap tmVS, const __grid_constant__ CUtensorMap tmKN,
                   const __grid_constant__ CUtensorMap tmVN, const __grid_constant__ AttnArgs a)
{
    constexpr uint32_t IDESC_S = make_idesc(128, 128, 1, 0, 0);
    constexpr uint32_t IDESC_O = make_idesc(128, 64, 1, 0, 1);

    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr int AT_TILES = TILES, AT_STAGES = AtCfg<TILES>::STAGES;
    // S mode: separate S and PV issuing warps (see the MMA issuers below)
    constexpr bool TWO_ISSUERS = TILES == 1 && !NS;
    uint8_t *sQ = smem;                                  // [AT_QBUF][AT_TILES]
    uint8_t *sKV = smem + AT_QBUF * AT_TILES * AT_TILE;  // [stage][K | V]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + 2 * AT_STAGES * AT_TILE);
    uint64_t *q_full = bars;                       // [AT_QBUF]
    uint64_t *q_empty = q_full + AT_QBUF;          // [AT_QBUF]   both MMA warps release
    uint64_t *kv_full = q_empty + AT_QBUF;         // [AT_STAGES]
    uint64_t *kv_empty = kv_full + AT_STAGES;      // [AT_STAGES] both MMA warps release
    uint64_t *s_full = kv_empty + AT_STAGES;       // [tile] S computed
    uint64_t *s_free = s_full + AT_TILES;          // [tile] S read into registers
    uint64_t *p_full = s_free + AT_TILES;          // [tile] P stored
    uint64_t *o_full = p_full + AT_TILES;          // [tile] PV completed
    uint64_t *o_free = o_full + AT_TILES;          // [tile] O read out (end of an item)
    uint64_t *mma_done = o_free + AT_TILES;        // [tile + 1] per issuing thread
    uint64_t *x_full = mma_done + AT_TILES + 1;    // split-key: tile 1's state is in xch
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(x_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *xch = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + AT_BAR_BYTES); // [2][AT_BM]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_pairs = (a.nq + at_item_rows<SPLIT, TILES>() - 1) / at_item_rows<SPLIT, TILES>();
    const int n_items = n_pairs * a.U * a.H;
    pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int i = 0; i < AT_QBUF; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], AT_TILES);
        }
        for (int i = 0; i < AT_STAGES; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], AT_TILES);
        }
        for (int i = 0; i < AT_TILES; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 4);
            mbar_init(&p_full[i], 4);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_free[i], 4);
            mbar_init(&mma_done[i], 1);
        }
        mbar_init(&mma_done[AT_TILES], 1);
        mbar_init(x_full, AT_BM);
        *abort_flag = 0;
        if (smem_u32(smem) & 1023) { // swizzle atoms need a 1024-byte aligned base
            *abort_flag = 1;
            if (a.wait.err) atomicCAS(a.wait.err, 0, OT_ERR_CUDA);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256 * AT_TILES);
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

    if (warp < 4) {
        // producer warpgroup: hand registers to the softmax warpgroups
        setmaxnreg_dec<AtCfg<TILES>::REG_PRODUCER>();
    }
    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && !aborted_at_start) {
            tma_prefetch(&tmQ);
            tma_prefetch(&tmKS);
            tma_prefetch(&tmVS);
            if (NS) {
                tma_prefetch(&tmKN);
                tma_prefetch(&tmVN);
            }
            long long gb = 0; // global key-block counter of this CTA
            int r = 0;        // items whose Q load was issued
            bool ok = true;
            for (; ok; ++r) {
                const int k = at_item_of(r, n_items);
                if (k < 0) break;
                const AtItem it = at_item<NS, SPLIT, FA, TILES>(a, n_pairs, k);
                const int qb = r & 1;
                // the Q buffer of item r - 2 is free once all its S MMAs completed
                if (!mbar_wait(&q_empty[qb], ((r >> 1) & 1) ^ 1, a.wait, abort_flag)) break;
                // split-key: both tiles read the one Q tile of the item
                constexpr int q_tiles = SPLIT ? 1 : AT_TILES;
                mbar_arrive_expect_tx(&q_full[qb], q_tiles * AT_TILE);
                for (int w = 0; w < q_tiles; ++w)
                    tma_load_3d(sQ + (qb * AT_TILES + w) * AT_TILE, &tmQ, &q_full[qb],
                                it.h * AT_HD, it.i0 + w * AT_BM, it.u);
                for (int b = 0; b < it.n_blocks; ++b, ++gb) {
                    const int st = static_cast<int>(gb % AT_STAGES);
                    if (!mbar_wait(&kv_empty[st], static_cast<uint32_t>((gb / AT_STAGES) & 1) ^ 1,
                                   a.wait, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&kv_full[st], 2 * AT_TILE);
                    uint8_t *k_dst = sKV + 2 * st * AT_TILE, *v_dst = k_dst + AT_TILE;
                    if (b < it.n_s_blocks && a.pages) {
                        // paged cache: one page per key block (K rows, then V rows)
                        const int pg = static_cast<int>(attn_page(a, it.u, b));
                        tma_load_3d(k_dst, &tmKS, &kv_full[st], it.h * AT_HD, 0, 2 * pg);
                        tma_load_3d(v_dst, &tmVS, &kv_full[st], it.h * AT_HD, 0, 2 * pg + 1);
                    } else if (b < it.n_s_blocks) {
                        tma_load_3d(k_dst, &tmKS, &kv_full[st], it.h * AT_HD, b * AT_BK, it.u);
                        tma_load_3d(v_dst, &tmVS, &kv_full[st], it.h * AT_HD, b * AT_BK, it.u);
                    } else {
                        const int j0 = it.k_begin + (b - it.n_s_blocks) * AT_BK;
                        tma_load_3d(k_dst, &tmKN, &kv_full[st], it.h * AT_HD, j0, it.u);
                        tma_load_3d(v_dst, &tmVN, &kv_full[st], it.h * AT_HD, j0, it.u);
                    }
                }
                if (!ok) {
                    ++r; // its Q load was issued
                    break;
                }
            }
            // never leave a load in flight: the last two Q loads, the last ring's K/V
            for (int rr = r > AT_QBUF ? r - AT_QBUF : 0; rr < r; ++rr)
                mbar_wait(&q_full[rr & 1], (rr >> 1) & 1, final_wait, &no_abort);
            for (long long j = gb > AT_STAGES ? gb - AT_STAGES : 0; j < gb; ++j)
                mbar_wait(&kv_full[j % AT_STAGES], static_cast<uint32_t>((j / AT_STAGES) & 1),
                          final_wait, &no_abort);
        }
    } else if (warp >= 1 && warp <= (TWO_ISSUERS ? 2 : AT_TILES)) {
        // ------------------------------------------------ MMA issuers
        // Issued from one thread, a short tcgen05.mma takes about 100 cycles.
        // Per key block: once the softmax has S(b) in registers (s_free),
        // S(b+1) = Q K^T goes into the S columns, so it runs while P(b) is
        // being computed; once P(b) is stored (p_full), O += P(b) V.
        //   in general warp 1 + w issues both for tile w (one issuer per tile
        //              keeps both tiles' MMAs flowing);
        //   S mode (one tile per CTA): warp 1 issues the S MMAs, warp 2 the PV
        //              MMAs, so PV(b) goes out as soon as P(b) is stored
        //              instead of queueing behind S(b+1), which waits for its
        //              K/V tile (whose load in turn waits for PV(b-1) to free
        //              the stage).  NS items measured slower that way (their
        //              K/V tiles mostly come from L2), so they keep one issuer.
        const int w = TWO_ISSUERS ? 0 : warp - 1;
        const bool issue_s_side = !TWO_ISSUERS || warp == 1;
        const bool issue_pv_side = !TWO_ISSUERS || warp == 2;
        if (lane == 0 && !aborted_at_start) {
            const uint32_t tS = tmem + w * 256, tP = tS + 128, tO = tS + 192;
            auto live = [&](const AtItem &it) { return SPLIT || it.i0 + w * AT_BM < a.nq; };
            auto issue_s = [&](const BlockCursor<NS, SPLIT, FA, TILES> &c) {
                if (live(c.it)) {
                    const uint32_t q_addr = smem_u32(sQ + ((c.r & 1) * AT_TILES + (SPLIT ? 0 : w)) * AT_TILE);
                    const uint32_t k_addr = smem_u32(sKV + 2 * (c.gb % AT_STAGES) * AT_TILE);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16(tS, sw128_desc(q_addr + k * 32, 16), sw128_desc(k_addr + k * 32, 16),
                                IDESC_S, k != 0);
                }
                mma_commit(&s_full[w]);
                // the item's last S of this tile: its Q buffer is free once they completed
                if (c.last_in_item()) mma_commit(&q_empty[c.r & 1]);
            };
            auto ready_s = [&](const BlockCursor<NS, SPLIT, FA, TILES> &c) {
                return mbar_wait(&kv_full[c.gb % AT_STAGES], static_cast<uint32_t>((c.gb / AT_STAGES) & 1),
                                 a.wait, abort_flag) &&
                       mbar_wait(&q_full[c.r & 1], (c.r >> 1) & 1, a.wait, abort_flag);
            };
            // O += P(b) V once P(b) is stored; false if a wait gave up
            auto issue_pv = [&](const BlockCursor<NS, SPLIT, FA, TILES> &c) {
                if (!mbar_wait(&p_full[w], static_cast<uint32_t>(c.lb & 1), a.wait, abort_flag)) return false;
                tc_fence_after();
                // the first PV of an item overwrites O: the previous item's
                // output has been read out by then (the warpgroup did that
                // before computing P of this block; in split-key mode tile 0
                // reads both tiles' O)
                const bool first = c.first_in_item();
                if (first && c.r > 0) {
                    if (!mbar_wait(&o_free[w], (c.r - 1) & 1, a.wait, abort_flag)) return false;
                    tc_fence_after();
                }
                if (live(c.it)) {
                    const uint32_t v_addr = smem_u32(sKV + (2 * (c.gb % AT_STAGES) + 1) * AT_TILE);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) // P from TMEM: 8 columns per 16 keys
                        mma_f16_ts(tO, tP + kk * 8, sw128_desc(v_addr + kk * 2048, AT_TILE), IDESC_O,
                                   !first || kk != 0);
                }
                mma_commit(&o_full[w]);
                // the arrivals the stage waits for (its S MMAs completed before
                // P(b) existed): split-key stages have one reader
                mma_commit(&kv_empty[c.gb % AT_STAGES]);
                if (SPLIT) mma_commit(&kv_empty[c.gb % AT_STAGES]);
                return true;
            };
            BlockCursor<NS, SPLIT, FA, TILES> cur;
            cur.init(a, n_pairs, n_items, w);
            if (issue_s_side) {
                bool run = cur.valid() && ready_s(cur);
                if (run) {
                    tc_fence_after();
                    issue_s(cur);
                }
                while (run) {
                    BlockCursor<NS, SPLIT, FA, TILES> nxt = cur;
                    nxt.next(a, n_pairs, n_items);
                    if (nxt.valid()) {
                        if (!mbar_wait(&s_free[w], static_cast<uint32_t>(cur.lb & 1), a.wait, abort_flag) ||
                            !ready_s(nxt))
                            break;
                        tc_fence_after();
                        issue_s(nxt);
                    }
                    if (issue_pv_side && !issue_pv(cur)) break;
                    if (!nxt.valid()) break;
                    cur = nxt;
                }
            } else {
                for (; cur.valid(); cur.next(a, n_pairs, n_items))
                    if (!issue_pv(cur)) break;
            }
            // every issued MMA must be complete before TMEM is released
            uint64_t *done = &mma_done[TWO_ISSUERS ? warp - 1 : w];
            mma_commit(done);
            mbar_wait(done, 0, final_wait, &no_abort);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax warpgroups
        setmaxnreg_inc<AtCfg<TILES>::REG_SOFTMAX>();
        const int w = (warp - 4) >> 2;         // tile of this warpgroup
        const int quarter = warp & 3;          // TMEM lane quarter
        const int row = quarter * 32 + lane;   // row within the tile
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = tmem + w * 256 + lane_off, tP = tS + 128, tO = tS + 192;
        const float c2 = a.scale * 1.4426950408889634f; // scores -> base-2 exponent
        bool ok = !aborted_at_start;
        long long lb = 0; // blocks of this tile so far
        int xr = 0;       // split-key hand-overs so far
        // wait for the PV of this tile's block jb (completion jb of
        // o_full[w]).  Waiting twice for the same block is harmless: PV(jb + 1)
        // is not issued before this warpgroup releases P(jb + 1), which it
        // does only after observing PV(jb), so o_full is at most one phase
        // ahead of every wait
        auto wait_o = [&](long long jb) {
            if (ok && !mbar_wait(&o_full[w], static_cast<uint32_t>(jb & 1), a.wait, abort_flag)) ok = false;
            tc_fence_after();
        };
        auto release = [&](uint64_t *bar) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        for (int r = 0; ok; ++r) {
            const int k = at_item_of(r, n_items);
            if (k < 0) break;
            const AtItem it = at_item<NS, SPLIT, FA, TILES>(a, n_pairs, k);
            const int i = it.i0 + (SPLIT ? 0 : w * AT_BM) + row; // query row within the user
            const bool warp_dead = __all_sync(0xffffffffu, i >= a.nq);
            const int t_self = a.L - a.nq + i;      // S mode
            // the row's candidate and the last NS key of it the row sees (S
            // rows meet NS keys only with full attention: all nkn of the user)
            const int my_c = NS ? i / a.N : 0;
            const int my_n = !NS ? (FA ? a.nkn - 1 : 0) : FA ? a.N - 1 : i % a.N;
            float m = -INFINITY, l = 0.f;
            const int b0 = SPLIT ? w : 0; // this tile's first block of the item
            for (int b = b0; ok && b < it.n_blocks; b += SPLIT ? 2 : 1, ++lb) {
                const bool s_block = b < it.n_s_blocks;
                const int j0 = s_block ? b * AT_BK : it.k_begin + (b - it.n_s_blocks) * AT_BK;
                // visible key range [klo, khi] of this row inside the block
                int klo = 0, khi;
                if (s_block) {
                    khi = (NS || FA) ? min(a.L - 1 - j0, AT_BK - 1) : min(t_self - j0, AT_BK - 1);
                } else {
                    const int first = my_c * a.N - j0; // key index of (my_c, 0)
                    klo = max(first, 0);
                    khi = min(first + my_n, AT_BK - 1);
                }
                const bool warp_full = __all_sync(0xffffffffu, klo <= 0 && khi >= AT_BK - 1);
                const bool warp_none = __all_sync(0xffffffffu, khi < klo);
                if (!mbar_wait(&s_full[w], static_cast<uint32_t>(lb & 1), a.wait, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (warp_dead || warp_none) {
                    // nothing of this warp's rows is visible (or no live row):
                    // the scores are not read; a live warp stores P = 0
                    release(&s_free[w]);
                    if (b > b0) wait_o(lb - 1);
                    if (!warp_dead) {
                        uint32_t z[32];
#pragma unroll
                        for (int q = 0; q < 32; ++q) z[q] = 0u;
                        tmem_st32(tP, z);
                        tmem_st32(tP + 32, z);
                        tmem_st_wait();
                    }
                } else {
                    uint32_t pk[4][16];
                    float alpha, rsum;
                    if (warp_full)
                        softmax_unit<true>(tS, c2, 0, AT_BK - 1, m, pk, alpha, rsum, [&] { release(&s_free[w]); });
                    else
                        softmax_unit<false>(tS, c2, klo, khi, m, pk, alpha, rsum, [&] { release(&s_free[w]); });
                    // P(b) goes where the previous PV read its P from
                    if (b > b0) wait_o(lb - 1);
                    if (__any_sync(0xffffffffu, alpha != 1.f)) {
                        // some row raised its max: O holds this item's blocks before
                        // b relative to the old max (their PV has completed)
#pragma unroll
                        for (int c = 0; c < AT_HD; c += 32) {
                            uint32_t v[32];
                            tmem_ld32(tO + c, v);
                            tmem_ld_wait();
                            tmem_reg_fence(v);
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                            tmem_st32(tO + c, v);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) tmem_st16(tP + 16 * q, pk[q]);
                    tmem_st_wait();
                    l = l * alpha + rsum;
                }
                release(&p_full[w]);
            }
            if (!ok) break;
            wait_o(lb - 1); // the item's last PV
            if (!ok) break;
            if (SPLIT && w == 1) {
                // hand the row's state to tile 0, which merges it with its own
                // and reads this tile's O straight from TMEM (its lanes are the
                // same rows); tile 0 also frees this O for the next item
                xch[row] = m;
                xch[AT_BM + row] = l;
                tc_fence_before();
                mbar_arrive(x_full);
                ++xr;
                continue;
            }
            // O / l as bf16 pairs, read 32 columns at a time
            uint32_t ob[AT_HD / 2];
            float a0 = 1.f, a1 = 0.f, inv = 0.f;
            if (SPLIT) {
                // merge with tile 1: O = O0 2^(m0 - m) + O1 2^(m1 - m), same for l
                if (!mbar_wait(x_full, static_cast<uint32_t>(xr & 1), a.wait, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                ++xr;
                const float m1 = xch[row], l1 = xch[AT_BM + row];
                const float mm = fmaxf(m, m1);
                a0 = fast_exp2(m - mm);
                a1 = fast_exp2(m1 - mm);
                l = l * a0 + l1 * a1;
            }
            if (!warp_dead) {
                inv = 1.f / l;
#pragma unroll
                for (int c = 0; c < AT_HD; c += 32) {
                    uint32_t v[32];
                    tmem_ld32(tO + c, v);
                    if (SPLIT) {
                        uint32_t v1[32];
                        tmem_ld32(tO + 256 + c, v1); // tile 1's O, same lanes
                        tmem_ld_wait();
                        tmem_reg_fence(v);
                        tmem_reg_fence(v1);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            v[e] = __float_as_uint(fmaf(__uint_as_float(v[e]), a0, __uint_as_float(v1[e]) * a1));
                    } else {
                        tmem_ld_wait();
                        tmem_reg_fence(v);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        ob[c / 2 + e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv,
                                                    __uint_as_float(v[2 * e + 1]) * inv);
                }
            }
            // O may now be overwritten by the next item's first PV
            release(&o_free[w]);
            if (SPLIT) release(&o_free[1]);
            const long long o_off = (static_cast<long long>(it.u) * a.nq + i) * a.d + it.h * AT_HD;
            if (a.o_qscale && i < a.nq && ot_dev_ok(o_off, AT_HD, a.o_cap, a.wait.err)) {
                // e4m3 output: the bf16 row quantised with the O projection's input scale
                const float qi = __frcp_rn(a.o_qscale[NS ? static_cast<long long>(i % a.N) * a.o_qstride : 0]);
                uint32_t q8[AT_HD / 4];
#pragma unroll
                for (int e = 0; e < AT_HD / 4; ++e)
                    q8[e] = static_cast<uint32_t>(bf16x2_to_e4m3x2(ob[2 * e], qi)) |
                            (static_cast<uint32_t>(bf16x2_to_e4m3x2(ob[2 * e + 1], qi)) << 16);
                uint4 *dp = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(a.O) + o_off);
#pragma unroll
                for (int qd = 0; qd < AT_HD / 16; ++qd)
                    dp[qd] = make_uint4(q8[4 * qd], q8[4 * qd + 1], q8[4 * qd + 2], q8[4 * qd + 3]);
            } else if (!a.o_qscale && i < a.nq && ot_dev_ok(o_off * 2, AT_HD * 2, a.o_cap, a.wait.err)) {
                uint4 *dp = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.O) + o_off);
#pragma unroll
                for (int qd = 0; qd < 8; ++qd)
                    dp[qd] = make_uint4(ob[4 * qd], ob[4 * qd + 1], ob[4 * qd + 2], ob[4 * qd + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256 * AT_TILES);
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
    if (tmap_rows(&tq, a.Q, a.d, a.nq, a.U, static_cast<long long>(a.nq) * a.d))
        return cudaErrorInvalidValue;
    if (a.pages) {
        // paged cache: the pool as (d, OT_PAGE_ROWS rows, 2 n_pages) -- K and V
        // of page p are slices 2 p and 2 p + 1
        static_assert(OT_PAGE_ROWS == AT_BK, "one page per key block");
        if (a.n_pages < 1 || 2 * a.n_pages > (1LL << 31) - 1 ||
            tmap_rows(&tks, a.KS, a.d, OT_PAGE_ROWS, 2 * a.n_pages, static_cast<long long>(OT_PAGE_ROWS) * a.d))
            return cudaErrorInvalidValue;
        tvs = tks;
    } else if (tmap_rows(&tks, a.KS, a.d, a.L, a.U, a.s_ustride) ||
               tmap_rows(&tvs, a.VS, a.d, a.L, a.U, a.s_ustride)) {
        return cudaErrorInvalidValue;
    }
    if (a.mode == 1 || a.full) {
        // NS keys / values: nkn rows per user (NS mode: the query rows themselves)
        const int nk = a.mode == 1 ? a.nq : a.nkn;
        if (nk < 1 || tmap_rows(&tkn, a.KN, a.d, nk, a.U, static_cast<long long>(nk) * a.d) ||
            tmap_rows(&tvn, a.VN, a.d, nk, a.U, static_cast<long long>(nk) * a.d))
            return cudaErrorInvalidValue;
    } else {
        tkn = tks;
        tvn = tvs;
    }
    static int num_sms = 0;
    if (num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            num_sms < 1)
            num_sms = 148;
    }
    // Split-key mode (NS mode with at least one S block, so every item has
    // two or more key blocks and each tile gets one): items of one 128-row
    // tile whose key blocks the CTA's two tiles take alternately, instead of
    // items of two row tiles that both walk every block.  Always with at most
    // 128 rows; above that where the estimated time is lower by a tenth, the
    // estimate being waves of items x (key blocks a tile walks + one for the
    // item's read-out), taken on the first item.  Split-key items read each
    // K/V tile once per row tile rather than once per pair of them (the row
    // tiles of a (user, head) run side by side, so mostly from L2).
    auto key_blocks = [&](int rows) {
        const int k_end = ((min(rows, a.nq) - 1) / a.N + 1) * a.N; // NS keys of the first item
        return static_cast<long long>((a.L + AT_BK - 1) / AT_BK + (k_end + AT_BK - 1) / AT_BK);
    };
    bool split = false;
    if (a.mode == 1 && a.L >= 1 && a.N >= 1) {
        const long long uh = static_cast<long long>(a.U) * a.H;
        const long long items2 = uh * ((a.nq + AT_BM * 2 - 1) / (AT_BM * 2));
        const long long items1 = uh * ((a.nq + AT_BM - 1) / AT_BM);
        const long long t2 = (items2 + num_sms - 1) / num_sms * (key_blocks(AT_BM * 2) + 1);
        const long long t1 = (items1 + num_sms - 1) / num_sms * ((key_blocks(AT_BM) + 1) / 2 + 1);
        split = a.nq <= AT_BM || t1 * 10 < t2 * 9;
    }
    // split-key NS items: two tiles per CTA; everything else one tile per
    // CTA, two CTAs per SM
    const int tiles = (a.mode == 1 && split) ? 2 : 1;
    const int rows = split ? AT_BM : AT_BM * tiles;
    const long long items = static_cast<long long>((a.nq + rows - 1) / rows) * a.H * a.U;
    if (items < 1 || items > (1LL << 30)) return cudaErrorInvalidValue;
    auto run = [&](auto kernel, auto cfg) -> cudaError_t {
        using Cfg = decltype(cfg);
        const long long slots = static_cast<long long>(num_sms) * Cfg::CTAS;
        const dim3 grid(static_cast<unsigned>(items < slots ? items : slots));
        // the setmaxnreg split must fit the registers the launch allocates,
        // or the softmax warpgroups' increase would wait forever
        cudaFuncAttributes fa;
        cudaError_t err = cudaFuncGetAttributes(&fa, kernel);
        if (err != cudaSuccess) return err;
        if (128 * Cfg::REG_PRODUCER + 128 * (Cfg::THREADS / 128 - 1) * Cfg::REG_SOFTMAX > fa.numRegs * Cfg::THREADS)
            return cudaErrorInvalidConfiguration;
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(Cfg::SMEM));
        if (err != cudaSuccess) return err;
        return launch_pdl(kernel, grid, dim3(Cfg::THREADS), Cfg::SMEM, s, tq, tks, tvs, tkn, tvn, a);
    };
    if (a.full) {
        if (a.mode != 1) return run(attn_tc_kernel<false, false, true, 1>, AtCfg<1>{});
        return split ? run(attn_tc_kernel<true, true, true, 2>, AtCfg<2>{})
                     : run(attn_tc_kernel<true, false, true, 1>, AtCfg<1>{});
    }
    if (a.mode != 1) return run(attn_tc_kernel<false, false, false, 1>, AtCfg<1>{});
    return split ? run(attn_tc_kernel<true, true, false, 2>, AtCfg<2>{})
                 : run(attn_tc_kernel<true, false, false, 1>, AtCfg<1>{});
}

} // namespace ot
