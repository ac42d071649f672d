// subblock.cu -- the SubBlock block-sparse attention router.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração somadas chega-se a 6 vezes":
// a block-sparse router cuts, from the 10th denoising step on, the KV blocks
// that take part in attention, at sparsity 0.75 or 0.80.  The pages give no
// rule; this is the plainest reading: tokens are cut into blocks of `block`
// consecutive tokens (the last may be shorter); per head a block is summed
// up by the mean of its rows; query block i scores key block j by the dot
// product of the two means and keeps the n_keep = ceil((1 - s) n_blocks)
// best key blocks (ties to the lower index), listed in increasing order.
//
// Kernels (the router on q and k pools, then scores and selects; the router
// from means, fed by the QK operator, starts at the scores):
//   subblock_pool_kernel    one pass over q and k (HBM bound): CTA (j, b, t,
//                           column chunk) sums the rows of block j of sample
//                           b of tensor t (q or k), a 16-byte column vector
//                           per thread, fp32, and writes the means
//                           [B, 2, n_blocks, H*hd] at the workspace's start.
//   tf32_split_kernel       for hd a multiple of 32: each mean split into a
//                           tf32 high part (low 13 mantissa bits cleared)
//                           and the remainder.
//   subblock_scores_tc_kernel  per (sample, head) the n_blocks x n_blocks
//                           scores on the tensor cores: per 128 query x 256
//                           key block tile, the hi and lo parts brought by
//                           TMA (128-byte swizzle) 32 head-dimension values
//                           at a time through a two-slot ring, hi.hi +
//                           hi.lo + lo.hi accumulated in TMEM by kind::tf32
//                           products.
//   subblock_scores_kernel  the same scores for other head sizes, as a tiled
//                           fp32 GEMM of the L2-resident means (128 x 128
//                           tiles, 8 x 8 per thread).
//   subblock_select_kernel  one warp per query block: the n_keep-th largest
//                           score of its row found bit by bit with warp-wide
//                           counts (the row in registers up to 2048 key
//                           blocks; the last candidates gathered one per
//                           lane) and an ordered ballot compaction that
//                           writes the kept indices in increasing order,
//                           ties at the threshold to the lower index.
#include <cmath>

#include "tcgen05.cuh"

namespace dit {
namespace {

constexpr int kPoolThreads = 128;
constexpr int kSelThreads = 256;
constexpr int kScoreTile = 128;          // query x key blocks per score tile
constexpr int kScoreDK = 32;             // d per staged slice of the score GEMM
constexpr int kMaxBlocks = 8192;           // key blocks per sample

// Means of the rows of one block: CTA (j, b, 2 c + t) takes column vectors
// 128 c .. 128 c + 127 of block j, sample b, tensor t (q or k), one per
// thread; fp32 sums over at most `block` rows in row order (8 rows in
// flight), one divide.
__global__ void __launch_bounds__(kPoolThreads)
subblock_pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, int64_t stride_v,
                     int64_t N, int block, int nb, int Dv, float* __restrict__ pooled) {
    const int j = blockIdx.x, b = blockIdx.y, t = blockIdx.z & 1;
    const int v = (blockIdx.z >> 1) * kPoolThreads + threadIdx.x;
    if (v >= Dv) return;
    const uint4* src = t == 0 ? q : k;
    const int64_t r0 = static_cast<int64_t>(j) * block;
    const int64_t r1 = r0 + block < N ? r0 + block : N;
    const float count = static_cast<float>(r1 - r0);
    float* out = pooled + ((static_cast<int64_t>(b) * 2 + t) * nb + j) * (static_cast<int64_t>(Dv) * 8);
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint4* p = src + (static_cast<int64_t>(b) * N + r0) * stride_v + v;
    int64_t r = r0;
    for (; r + 8 <= r1; r += 8, p += 8 * stride_v) {
        uint4 a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) a[u] = ld_stream(p + u * stride_v);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float f[8];
            unpack8(a[u], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) s[i] += f[i];
        }
    }
    for (; r < r1; ++r, p += stride_v) {
        float f[8];
        unpack8(ld_stream(p), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] += f[i];
    }
    float4* o = reinterpret_cast<float4*>(out + 8 * v);
    o[0] = make_float4(s[0] / count, s[1] / count, s[2] / count, s[3] / count);
    o[1] = make_float4(s[4] / count, s[5] / count, s[6] / count, s[7] / count);
}

// Order-preserving map of a float to uint32 (larger float -> larger code).
__device__ __forceinline__ uint32_t ordered(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp picks one query block's kept key blocks from its fp32 scores
// sc[0..nb) in shared memory.  The n_keep-th largest order-preserving code T
// is the largest T with at least n_keep codes >= T, fixed one bit at a time
// from the top (32 warp-wide counts; no shared-memory atomics, which the
// clustered top bytes of the codes would serialise); then the kept indices --
// every code above T and the lowest-index ties at T -- are written in
// increasing order with ballots.  Same order as sorting (score descending,
// index ascending) and taking the first n_keep.  This form: nb <= 32 * KPL,
// the lane's codes in registers; warp_select_smem below: any nb, the codes
// re-read from shared memory in every count.
template <int KPL>
__device__ void warp_select_reg(const float* sc, int nb, int n_keep, int32_t* out, int lane,
                                uint32_t* stage) {
    uint32_t c[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
        const int j = k * 32 + lane;
        c[k] = j < nb ? ordered(sc[j]) : 0u;
    }
    // a candidate is never 0, so the padding codes (0) are never counted.
    // T: the bits of the threshold found so far (bits >= `bit` + 1); n_ge_t,
    // n_ge_u: the codes >= T and >= U = T + 2^(bit+1).  Once the bucket
    // [T, U) holds at most 32 codes they are gathered one per lane and the
    // remaining bits are found on those alone.
    uint32_t T = 0;
    unsigned n_ge_t = static_cast<unsigned>(nb), n_ge_u = 0;
    int bit = 31;
    for (; bit >= 0 && n_ge_t - n_ge_u > 32u; --bit) {
        const uint32_t cand = T | (1u << bit);
        unsigned cnt = 0;
#pragma unroll
        for (int k = 0; k < KPL; ++k) cnt += c[k] >= cand ? 1u : 0u;
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (cnt >= static_cast<unsigned>(n_keep)) {
            T = cand;
            n_ge_t = cnt;
        } else {
            n_ge_u = cnt;
        }
    }
    if (bit >= 0) {
        // the bucket: nonzero codes whose bits above `bit` are T's
        const int sh = bit + 1;
        unsigned mine = 0;
#pragma unroll
        for (int k = 0; k < KPL; ++k)
            mine += (c[k] != 0u && (sh == 32 || (c[k] >> sh) == (T >> sh))) ? 1u : 0u;
        unsigned off = mine;                        // inclusive scan over the lanes
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const unsigned o = __shfl_up_sync(0xffffffffu, off, d);
            if (lane >= d) off += o;
        }
        off -= mine;
#pragma unroll
        for (int k = 0; k < KPL; ++k)
            if (c[k] != 0u && (sh == 32 || (c[k] >> sh) == (T >> sh))) stage[off++] = c[k];
        __syncwarp();
        const uint32_t e = lane < static_cast<int>(n_ge_t - n_ge_u) ? stage[lane] : 0u;
        __syncwarp();
        const unsigned above = n_ge_u;              // codes above the bucket
        for (; bit >= 0; --bit) {
            const uint32_t cand = T | (1u << bit);
            const unsigned cnt = above + __reduce_add_sync(0xffffffffu, e >= cand ? 1u : 0u);
            if (cnt >= static_cast<unsigned>(n_keep)) {
                T = cand;
                n_ge_t = cnt;
            } else {
                n_ge_u = cnt;
            }
        }
    }
    // now U = T + 1: n_ge_u codes lie above T and n_ge_t - n_ge_u equal it;
    // `need` ties at T are taken, lowest indices first
    const int need = n_keep - static_cast<int>(n_ge_u);
    int written = 0, eq_seen = 0;
    const unsigned below = (1u << lane) - 1u;
    if (static_cast<unsigned>(need) == n_ge_t - n_ge_u) {      // every tie is taken
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            if (k * 32 >= nb) break;
            const bool take = c[k] >= T;                      // padding (0) is below T
            const unsigned tm = __ballot_sync(0xffffffffu, take);
            if (take) out[written + __popc(tm & below)] = k * 32 + lane;
            written += __popc(tm);
        }
        return;
    }
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
        if (k * 32 >= nb) break;
        const int j = k * 32 + lane;
        const bool live = j < nb;
        const bool g = live && c[k] > T;
        const bool eq = live && c[k] == T;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const bool take = g || (eq && eq_seen + __popc(eqm & below) < need);
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        if (take) out[written + __popc(tm & below)] = j;
        written += __popc(tm);
        eq_seen += __popc(eqm);
    }
}

__device__ void warp_select_smem(const float* sc, int nb, int n_keep, int32_t* out, int lane) {
    uint32_t T = 0;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        unsigned cnt = 0;
        for (int j = lane; j < nb; j += 32) cnt += ordered(sc[j]) >= cand ? 1u : 0u;
        if (__reduce_add_sync(0xffffffffu, cnt) >= static_cast<unsigned>(n_keep)) T = cand;
    }
    unsigned gt = 0;
    for (int j = lane; j < nb; j += 32) gt += ordered(sc[j]) > T ? 1u : 0u;
    const int need = n_keep - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
    int written = 0, eq_seen = 0;
    const unsigned below = (1u << lane) - 1u;
    for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t c = j < nb ? ordered(sc[j]) : 0u;
        const bool g = j < nb && c > T;
        const bool eq = j < nb && c == T;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const bool take = g || (eq && eq_seen + __popc(eqm & below) < need);
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        if (take) out[written + __popc(tm & below)] = j;
        written += __popc(tm);
        eq_seen += __popc(eqm);
    }
}

// One d step of a thread's 8 x 8 score tile (see subblock_scores_kernel).
__device__ __forceinline__ void score_step(const float* qrow, const float* krow, int tx, int ty,
                                           float (&acc)[8][8]) {
    constexpr int kHalf = kScoreTile / 2;
    const float4 q0 = *reinterpret_cast<const float4*>(qrow + 4 * ty);
    const float4 q1 = *reinterpret_cast<const float4*>(qrow + kHalf + 4 * ty);
    const float4 k0 = *reinterpret_cast<const float4*>(krow + 4 * tx);
    const float4 k1 = *reinterpret_cast<const float4*>(krow + kHalf + 4 * tx);
    const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const float kv[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = __fmaf_rn(qv[r], kv[c], acc[r][c]);
}

// Scores of one (sample, head) as a tiled fp32 GEMM: CTA (t, h, b) forms
// the 128 x 128 tile t of scores[b, h, i, j] = sum_d qm[i, d] km[j, d] from
// the block means, staging 32-wide d slices of both operands transposed in
// shared memory.  Thread (ty, tx) keeps an 8 x 8 tile: query rows 4ty.. and
// 64 + 4ty.., key columns 4tx.. and 64 + 4tx.., so that each 16-byte read of
// a warp covers contiguous words.  Every score is the fp32 fmaf chain over
// d = 0, 1, ..., hd - 1 from +0 (no padded terms: a zero product could turn
// a -0 score into +0 and reorder an exact tie).
__global__ void __launch_bounds__(kSelThreads)
subblock_scores_kernel(const float* __restrict__ pooled, int nb, int D, int hd,
                       float* __restrict__ scores) {
    __shared__ __align__(16) float qs[kScoreDK][kScoreTile + 4];
    __shared__ __align__(16) float ks[kScoreDK][kScoreTile + 4];
    const int tiles = (nb + kScoreTile - 1) / kScoreTile;
    const int i0 = (blockIdx.x / tiles) * kScoreTile, j0 = (blockIdx.x % tiles) * kScoreTile;
    const int h = blockIdx.y, b = blockIdx.z;
    const float* qsrc = pooled + (static_cast<int64_t>(b) * 2 + 0) * nb * D + h * hd;
    const float* ksrc = pooled + (static_cast<int64_t>(b) * 2 + 1) * nb * D + h * hd;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    constexpr int kHalf = kScoreTile / 2;
    float acc[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.0f;
    for (int d0 = 0; d0 < hd; d0 += kScoreDK) {
        const int dn = min(kScoreDK, hd - d0);          // a multiple of 8
        for (int e = threadIdx.x; e < kScoreTile * (kScoreDK / 4); e += kSelThreads) {
            const int r = e / (kScoreDK / 4), c4 = e % (kScoreDK / 4);
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bk = a;
            if (4 * c4 < dn) {
                if (i0 + r < nb)
                    a = *reinterpret_cast<const float4*>(qsrc + static_cast<int64_t>(i0 + r) * D +
                                                         d0 + 4 * c4);
                if (j0 + r < nb)
                    bk = *reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(j0 + r) * D +
                                                          d0 + 4 * c4);
            }
            qs[4 * c4 + 0][r] = a.x; qs[4 * c4 + 1][r] = a.y;
            qs[4 * c4 + 2][r] = a.z; qs[4 * c4 + 3][r] = a.w;
            ks[4 * c4 + 0][r] = bk.x; ks[4 * c4 + 1][r] = bk.y;
            ks[4 * c4 + 2][r] = bk.z; ks[4 * c4 + 3][r] = bk.w;
        }
        __syncthreads();
        // a full slice runs without a per-step test (a branch in the unrolled
        // loop would keep the shared-memory reads from being issued ahead)
        if (dn == kScoreDK) {
#pragma unroll
            for (int d = 0; d < kScoreDK; ++d) score_step(qs[d], ks[d], tx, ty, acc);
        } else {
#pragma unroll
            for (int d = 0; d < kScoreDK; ++d)
                if (d < dn) score_step(qs[d], ks[d], tx, ty, acc);
        }
        __syncthreads();
    }
    float* out = scores + (static_cast<int64_t>(b) * gridDim.y + h) * nb * nb;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int i = i0 + (r < 4 ? 4 * ty + r : kHalf + 4 * ty + r - 4);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int j = j0 + (c < 4 ? 4 * tx + c : kHalf + 4 * tx + c - 4);
            if (i < nb && j < nb) out[static_cast<int64_t>(i) * nb + j] = acc[r][c];
        }
    }
}

// CTA (g, h, b): warp w selects query block i = 8 g + w of head h, sample b
// from its score row; KPL > 0: nb <= 32 KPL, the row in registers.
template <int KPL>
__global__ void __launch_bounds__(kSelThreads)
subblock_select_kernel(const float* __restrict__ scores, int nb, int n_keep,
                       int32_t* __restrict__ kept) {
    const int h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * (kSelThreads / 32) + warp;
    if (i >= nb) return;
    const int64_t row = (static_cast<int64_t>(b) * gridDim.y + h) * nb + i;
    const float* sc = scores + row * nb;
    int32_t* out = kept + row * n_keep;
    __shared__ uint32_t stage[kSelThreads];
    if constexpr (KPL > 0)
        warp_select_reg<KPL>(sc, nb, n_keep, out, lane, stage + 32 * warp);
    else
        warp_select_smem(sc, nb, n_keep, out, lane);
}

// ---------------------------------------------------------------------------
// Scores on the tensor cores for the router from precomputed means.  The
// scores are a dense contraction (query-block means x key-block means over
// the head dimension), but a selection threshold must be resolved to about
// 2^-14 of the largest score, finer than one TF32 product (11 significant
// bits).  Each mean is therefore split as a = hi + lo, hi = a with its low 13
// mantissa bits cleared (exactly a TF32 value) and lo = a - hi (exact), and
// the products hi*hi + hi*lo + lo*hi are accumulated in fp32 (the three-pass
// split-TF32 method; the dropped lo*lo term and lo's own rounding to TF32 are
// each below 2^-22 of the product).
constexpr int kTcM = 128;        // query blocks per tile (TMEM lanes)
constexpr int kTcN = 256;        // key blocks per tile (TMEM columns)
constexpr int kTcChunk = 32;     // head-dimension values per 128-byte swizzle row
constexpr int kTcSlots = 2;      // chunks in flight
constexpr uint32_t kTcSlotBytes = 2 * (kTcM + kTcN) * kTcChunk * 4;   // hi and lo: 96 KB
constexpr int kTcSmem = kTcSlots * kTcSlotBytes + 1024;

// hi / lo of n fp32 values (n multiple of 4).
__global__ void __launch_bounds__(256)
tf32_split_kernel(const float4* __restrict__ src, float4* __restrict__ hi, float4* __restrict__ lo,
                  int64_t n4) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 a = src[i];
        float4 h, l;
        h.x = __uint_as_float(__float_as_uint(a.x) & 0xFFFFE000u); l.x = a.x - h.x;
        h.y = __uint_as_float(__float_as_uint(a.y) & 0xFFFFE000u); l.y = a.y - h.y;
        h.z = __uint_as_float(__float_as_uint(a.z) & 0xFFFFE000u); l.z = a.z - h.z;
        h.w = __uint_as_float(__float_as_uint(a.w) & 0xFFFFE000u); l.w = a.w - h.w;
        hi[i] = h;
        lo[i] = l;
    }
}

// kind::tf32: fp32 accumulator, TF32 A and B, both K-major.
constexpr uint32_t idesc_tf32(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((static_cast<uint32_t>(N) >> 3) << 17) |
           ((static_cast<uint32_t>(M) >> 4) << 24);
}
constexpr uint32_t kIdescTf32 = idesc_tf32(kTcM, kTcN);

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t da, uint64_t db,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(kIdescTf32), "r"(accumulate)
        : "memory");
}

// CTA (tile, h, b): scores[b, h, i0 .. i0+127, j0 .. j0+255].  Warp 0
// brings the hi and lo tiles of both operands 32 head-dimension values (one
// chunk) at a time into a two-slot ring (96 KB a slot, one CTA per SM); one
// thread of warp 1 issues each chunk's 3 x 4 products (N = 256) as soon as
// it lands and frees its slot with a commit; the four warps read the
// accumulator 64 columns at a time (thread = query block), pass their 32
// rows through shared memory (the ring, free once the products are done)
// and store them row by row, a warp per 64-score row segment.  (128 x 64
// tiles with two CTAs per SM read the query means four times as often and
// measured 7 % slower for the whole call.)  Rows past n_blocks are computed
// on whatever the copy brought (the next group's rows, or zeros past the
// array) and never stored.
__global__ void __launch_bounds__(128, 1)
subblock_scores_tc_kernel(const __grid_constant__ CUtensorMap map_hi_a,
                          const __grid_constant__ CUtensorMap map_lo_a,
                          const __grid_constant__ CUtensorMap map_hi_b,
                          const __grid_constant__ CUtensorMap map_lo_b, int nb, int hd,
                          float* __restrict__ scores, int* status, int stall) {
    extern __shared__ uint8_t tc_smem_raw[];
    __shared__ uint64_t s_bar[2 * kTcSlots + 1];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const uint32_t raw = tc::smem_u32(tc_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const int chunks = hd / kTcChunk;
    constexpr uint32_t a_bytes = kTcM * kTcChunk * 4;      // 16 KB
    constexpr uint32_t b_bytes = kTcN * kTcChunk * 4;      // 32 KB
    // slot layout: A hi, A lo, B hi, B lo
    const uint32_t bar_full = tc::smem_u32(&s_bar[0]);
    const uint32_t bar_empty = tc::smem_u32(&s_bar[kTcSlots]);
    const uint32_t bar_done = tc::smem_u32(&s_bar[2 * kTcSlots]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_j = (nb + kTcN - 1) / kTcN;
    const int i0 = (blockIdx.x / tiles_j) * kTcM, j0 = (blockIdx.x % tiles_j) * kTcN;
    const int h = blockIdx.y, b = blockIdx.z;
    const int H = gridDim.y;
    if (threadIdx.x == 0) {
        for (int c = 0; c <= 2 * kTcSlots; ++c) tc::mbar_init(tc::smem_u32(&s_bar[c]), 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(&s_tmem), kTcN);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s_tmem;
    if (warp == 0) {
        if (lane == 0) {
            const int qrow = (b * 2 + 0) * nb + i0, krow = (b * 2 + 1) * nb + j0;
            int issued = 0;
            // stall (a test hook): no copy is issued, so every wait runs out
            for (int c = 0; c < chunks && !stall; ++c) {
                const int slot = c % kTcSlots;
                if (c >= kTcSlots &&
                    !tc::mbar_wait(bar_empty + 8 * slot, ((c / kTcSlots) - 1) & 1, &s_abort)) {
                    s_abort = 1;
                    break;
                }
                const uint32_t sa = base + slot * kTcSlotBytes, bar = bar_full + 8 * slot;
                const int col = h * hd + c * kTcChunk;
                tc::mbar_expect_tx(bar, kTcSlotBytes);
                tc::tma_load_2d(sa, &map_hi_a, bar, col, qrow);
                tc::tma_load_2d(sa + 2 * a_bytes, &map_hi_b, bar, col, krow);
                tc::tma_load_2d(sa + a_bytes, &map_lo_a, bar, col, qrow);
                tc::tma_load_2d(sa + 2 * a_bytes + b_bytes, &map_lo_b, bar, col, krow);
                issued = c + 1;
            }
            // the copies land before the CTA exits: the last chunk of each
            // slot (earlier ones were consumed before their slot was reused)
            for (int c = issued > kTcSlots ? issued - kTcSlots : 0; c < issued; ++c)
                tc::mbar_wait_drain(bar_full + 8 * (c % kTcSlots), (c / kTcSlots) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t acc = 0;
            for (int c = 0; c < chunks; ++c) {
                const int slot = c % kTcSlots;
                if (!tc::mbar_wait(bar_full + 8 * slot, (c / kTcSlots) & 1, &s_abort)) {
                    s_abort = 1;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t sa = base + slot * kTcSlotBytes;
#pragma unroll
                for (int kk = 0; kk < kTcChunk / 8; ++kk) {
                    const uint32_t o = kk * 32;
                    const uint64_t ah = tc::sw128_desc(sa + o);
                    const uint64_t al = tc::sw128_desc(sa + a_bytes + o);
                    const uint64_t bh = tc::sw128_desc(sa + 2 * a_bytes + o);
                    const uint64_t bl = tc::sw128_desc(sa + 2 * a_bytes + b_bytes + o);
                    mma_tf32(tmem, ah, bh, acc);
                    mma_tf32(tmem, ah, bl, 1u);
                    mma_tf32(tmem, al, bh, 1u);
                    acc = 1u;
                }
                tc::mma_commit(bar_empty + 8 * slot);
            }
            // also after a failed wait: the commit then tracks the products
            // already issued, on chunks that had landed
            tc::mma_commit(bar_done);
        }
        __syncwarp();
    }
    // epilogue: thread = query block i0 + 32 * warp + lane (TMEM lane); the
    // commit is issued in every case, so the drain wait ends; the loads are
    // skipped warp-uniformly after a failure.
    __syncthreads();
    bool failed = s_abort != 0;
    if (!__all_sync(0xffffffffu, tc::mbar_wait_drain(bar_done, 0))) failed = true;
    if (!failed) {
        tc::fence_after_sync();
        constexpr int kCh = 64;             // columns per epilogue chunk
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        // the warp's 32 x 64 scores of a chunk through shared memory, rows
        // kCh + 1 apart (no bank conflicts either way)
        float* st = reinterpret_cast<float*>(tc_smem_raw + (base - raw)) + warp * 32 * (kCh + 1);
        const int rows = nb - (i0 + 32 * warp) < 32 ? nb - (i0 + 32 * warp) : 32;
        float* out = scores + ((static_cast<int64_t>(b) * H + h) * nb + i0 + 32 * warp) * nb + j0;
        for (int c = 0; c < kTcN / kCh && j0 + c * kCh < nb; ++c) {
            float v[kCh];
            tc::tmem_ld32(lane_addr + c * kCh, *reinterpret_cast<float(*)[32]>(v));
            tc::tmem_ld32(lane_addr + c * kCh + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            tc::tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < kCh; ++jj) st[lane * (kCh + 1) + jj] = v[jj];
            __syncwarp();
            const int jc = j0 + c * kCh;
            const bool c0 = jc + lane < nb, c1 = jc + 32 + lane < nb;
            for (int r = 0; r < rows; ++r) {
                if (c0) out[static_cast<int64_t>(r) * nb + c * kCh + lane] = st[r * (kCh + 1) + lane];
                if (c1)
                    out[static_cast<int64_t>(r) * nb + c * kCh + 32 + lane] =
                        st[r * (kCh + 1) + 32 + lane];
            }
            __syncwarp();
        }
    }
    if (failed && lane == 0 && status) atomicExch(status, 1);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, kTcN);
}

int keep_count(int64_t n_blocks, double sparsity) {
    if (n_blocks <= 0 || !(sparsity >= 0.0) || !(sparsity < 1.0)) return DIT_ERR_VALUE;
    const double want = std::ceil((1.0 - sparsity) * static_cast<double>(n_blocks) - 1e-9);
    int64_t keep = static_cast<int64_t>(want);
    if (keep < 1) keep = 1;
    if (keep > n_blocks) keep = n_blocks;
    return static_cast<int>(keep);
}

}  // namespace
}  // namespace dit

extern "C" int dit_subblock_keep_count(int64_t n_blocks, double sparsity) {
    return dit::keep_count(n_blocks, sparsity);
}

extern "C" size_t dit_subblock_workspace_bytes(int B, int64_t N, int H, int hd, int block) {
    if (B < 0 || N < 0 || H < 1 || hd < 1 || block < 1) return 0;
    const int64_t nb = (N + block - 1) / block;
    // the block means [B, 2, nb, H*hd] fp32 (256-byte rounded), then what
    // the router from means needs
    const size_t means = static_cast<size_t>(B) * 2 * nb * H * hd * sizeof(float);
    return ((means + 255) & ~static_cast<size_t>(255)) +
           dit_subblock_means_workspace_bytes(B, N, H, hd, block);
}

namespace dit {
namespace {

// The n_keep largest scores of each row of scores [B, H, nb, nb] into kept.
int select_kept(const float* scores, int B, int nb, int H, int n_keep, int32_t* kept,
                cudaStream_t st) {
    const dim3 sel((nb + 7) / 8, H, B);
    if (nb <= 256)
        subblock_select_kernel<8><<<sel, kSelThreads, 0, st>>>(scores, nb, n_keep, kept);
    else if (nb <= 512)
        subblock_select_kernel<16><<<sel, kSelThreads, 0, st>>>(scores, nb, n_keep, kept);
    else if (nb <= 1024)
        subblock_select_kernel<32><<<sel, kSelThreads, 0, st>>>(scores, nb, n_keep, kept);
    else if (nb <= 2048)
        subblock_select_kernel<64><<<sel, kSelThreads, 0, st>>>(scores, nb, n_keep, kept);
    else
        subblock_select_kernel<0><<<sel, kSelThreads, 0, st>>>(scores, nb, n_keep, kept);
    return launch_status();
}

// Scores and selection from the block means [B, 2, nb, H*hd] (fp32) into
// the scores buffer [B, H, nb, nb].
int route_from_means(const float* pooled, int B, int nb, int H, int hd, int n_keep,
                     int32_t* kept, float* scores, cudaStream_t st) {
    const int64_t D = static_cast<int64_t>(H) * hd;
    const int64_t tiles = (nb + kScoreTile - 1) / kScoreTile;
    subblock_scores_kernel<<<dim3(static_cast<unsigned>(tiles * tiles), H, B), kSelThreads, 0,
                             st>>>(pooled, nb, static_cast<int>(D), hd, scores);
    int rc = launch_status();
    if (rc) return rc;
    return select_kept(scores, B, nb, H, n_keep, kept, st);
}

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// Whether the router from means takes the tensor-core scores (whole
// 32-value chunks of the head dimension).
bool tc_scores(int hd) { return hd % kTcChunk == 0; }

// Tensor-core scores: split the means into hi / lo in the workspace, then one
// CTA per 128 x 256 tile.
int scores_tc(const float* means, int B, int nb, int H, int hd, float* scores, float* hi,
              float* lo, int* status, cudaStream_t st, int stall = 0) {
    const int64_t D = static_cast<int64_t>(H) * hd;
    const int64_t rows = static_cast<int64_t>(B) * 2 * nb;
    const int64_t n4 = rows * D / 4;
    const int sms = device_sm_count();
    if (sms <= 0) return DIT_ERR_LAUNCH;
    int64_t g = (n4 + 255) / 256;
    if (g > static_cast<int64_t>(sms) * 8) g = static_cast<int64_t>(sms) * 8;
    tf32_split_kernel<<<static_cast<unsigned>(g), 256, 0, st>>>(
        reinterpret_cast<const float4*>(means), reinterpret_cast<float4*>(hi),
        reinterpret_cast<float4*>(lo), n4);
    int rc = launch_status();
    if (rc) return rc;
    CUtensorMap mha, mla, mhb, mlb;
    if (!tc::make_map_f32(&mha, hi, rows, D, D, kTcM) || !tc::make_map_f32(&mla, lo, rows, D, D, kTcM) ||
        !tc::make_map_f32(&mhb, hi, rows, D, D, kTcN) || !tc::make_map_f32(&mlb, lo, rows, D, D, kTcN))
        return DIT_ERR_LAUNCH;
    const size_t smem = kTcSmem;
    if (cudaFuncSetAttribute(subblock_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kTcSmem) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    const int64_t tiles = static_cast<int64_t>((nb + kTcM - 1) / kTcM) * ((nb + kTcN - 1) / kTcN);
    subblock_scores_tc_kernel<<<dim3(static_cast<unsigned>(tiles), H, B), 128, smem, st>>>(
        mha, mla, mhb, mlb, nb, hd, scores, status, stall);
    return launch_status();
}
// Scores and selection from block means, in a workspace laid out as
// dit_subblock_means_workspace_bytes describes.
int route_means_ws(const float* means, int B, int nb, int H, int hd, int n_keep, int32_t* kept,
                   void* workspace, int* status, cudaStream_t st) {
    float* scores = static_cast<float*>(workspace);
    if (!tc_scores(hd)) return route_from_means(means, B, nb, H, hd, n_keep, kept, scores, st);
    const size_t sb = round256(static_cast<size_t>(B) * H * nb * nb * sizeof(float));
    const size_t mb = round256(static_cast<size_t>(B) * 2 * nb * H * hd * sizeof(float));
    uint8_t* w = static_cast<uint8_t*>(workspace);
    const int rc = scores_tc(means, B, nb, H, hd, scores, reinterpret_cast<float*>(w + sb),
                             reinterpret_cast<float*>(w + sb + mb), status, st);
    if (rc) return rc;
    return select_kept(scores, B, nb, H, n_keep, kept, st);
}

}  // namespace
}  // namespace dit

extern "C" size_t dit_subblock_means_workspace_bytes(int B, int64_t N, int H, int hd, int block) {
    if (B < 0 || N < 0 || H < 1 || hd < 1 || block < 1) return 0;
    const int64_t nb = (N + block - 1) / block;
    const size_t scores = static_cast<size_t>(B) * H * nb * nb * sizeof(float);
    if (!dit::tc_scores(hd)) return scores;
    // the scores, then the hi and lo parts of the means
    const size_t means = static_cast<size_t>(B) * 2 * nb * H * hd * sizeof(float);
    return dit::round256(scores) + 2 * dit::round256(means);
}

extern "C" int dit_subblock_router_means(const float* block_means, int B, int64_t N, int H,
                                         int hd, int block, double sparsity, int32_t* kept,
                                         void* workspace, size_t workspace_bytes, int* status,
                                         void* stream) {
    using namespace dit;
    if (B < 0 || N < 0 || H < 1 || block < 1) return DIT_ERR_SHAPE;
    if (hd < 8 || hd > 256 || hd % 8) return DIT_ERR_SHAPE;
    if (static_cast<int64_t>(H) * hd > DIT_MAX_D) return DIT_ERR_SHAPE;
    if (!(sparsity >= 0.0) || !(sparsity < 1.0)) return DIT_ERR_VALUE;
    if (B == 0 || N == 0) return DIT_OK;
    const int64_t nb64 = (N + block - 1) / block;
    if (nb64 > kMaxBlocks || B > 65535) return DIT_ERR_SHAPE;
    const int nb = static_cast<int>(nb64);
    if (!block_means || !kept) return DIT_ERR_NULL;
    if (!aligned16(block_means) || reinterpret_cast<uintptr_t>(kept) % 4) return DIT_ERR_ALIGN;
    if (status && reinterpret_cast<uintptr_t>(status) % 4) return DIT_ERR_ALIGN;
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < dit_subblock_means_workspace_bytes(B, N, H, hd, block))
        return DIT_ERR_WORKSPACE;
    return route_means_ws(block_means, B, nb, H, hd, keep_count(nb, sparsity), kept, workspace,
                          status, as_stream(stream));
}

extern "C" int dit_subblock_scores_stall_test(const float* block_means, int B, int64_t N, int H,
                                              int hd, int block, void* workspace,
                                              size_t workspace_bytes, int* status, void* stream) {
    using namespace dit;
    if (B < 1 || N < 1 || H < 1 || block < 1 || !tc_scores(hd)) return DIT_ERR_SHAPE;
    if (static_cast<int64_t>(H) * hd > DIT_MAX_D) return DIT_ERR_SHAPE;
    const int64_t nb64 = (N + block - 1) / block;
    if (nb64 > 512 || B > 4) return DIT_ERR_SHAPE;        // small shapes only
    const int nb = static_cast<int>(nb64);
    if (!block_means || !status) return DIT_ERR_NULL;
    if (!aligned16(block_means) || reinterpret_cast<uintptr_t>(status) % 4) return DIT_ERR_ALIGN;
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < dit_subblock_means_workspace_bytes(B, N, H, hd, block))
        return DIT_ERR_WORKSPACE;
    const size_t sb = round256(static_cast<size_t>(B) * H * nb * nb * sizeof(float));
    const size_t mb = round256(static_cast<size_t>(B) * 2 * nb * H * hd * sizeof(float));
    uint8_t* w = static_cast<uint8_t*>(workspace);
    return scores_tc(block_means, B, nb, H, hd, reinterpret_cast<float*>(w),
                     reinterpret_cast<float*>(w + sb), reinterpret_cast<float*>(w + sb + mb),
                     status, as_stream(stream), 1);
}

extern "C" int dit_subblock_router(const uint16_t* q, const uint16_t* k, int64_t row_stride,
                                   int B, int64_t N, int H, int hd, int block, double sparsity,
                                   int32_t* kept, void* workspace, size_t workspace_bytes,
                                   int* status, void* stream) {
    using namespace dit;
    if (B < 0 || N < 0 || H < 1 || block < 1) return DIT_ERR_SHAPE;
    if (hd < 8 || hd > 256 || hd % 8) return DIT_ERR_SHAPE;
    const int64_t D = static_cast<int64_t>(H) * hd;
    if (D > DIT_MAX_D || row_stride < D) return DIT_ERR_SHAPE;
    if (row_stride % 8) return DIT_ERR_ALIGN;
    if (!(sparsity >= 0.0) || !(sparsity < 1.0)) return DIT_ERR_VALUE;
    if (B == 0 || N == 0) return DIT_OK;
    const int64_t nb64 = (N + block - 1) / block;
    if (nb64 > kMaxBlocks || B > 65535) return DIT_ERR_SHAPE;
    const int nb = static_cast<int>(nb64);
    const int n_keep = keep_count(nb, sparsity);
    if (!q || !k || !kept) return DIT_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || reinterpret_cast<uintptr_t>(kept) % 4)
        return DIT_ERR_ALIGN;
    if (status && reinterpret_cast<uintptr_t>(status) % 4) return DIT_ERR_ALIGN;
    const size_t need = dit_subblock_workspace_bytes(B, N, H, hd, block);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return DIT_ERR_WORKSPACE;
    float* pooled = static_cast<float*>(workspace);
    cudaStream_t st = as_stream(stream);
    const int chunks = static_cast<int>((D / 8 + kPoolThreads - 1) / kPoolThreads);
    subblock_pool_kernel<<<dim3(nb, B, 2 * chunks), kPoolThreads, 0, st>>>(
        reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), row_stride / 8, N,
        block, nb, static_cast<int>(D / 8), pooled);
    int rc = launch_status();
    if (rc) return rc;
    const size_t mb = round256(static_cast<size_t>(B) * 2 * nb * D * sizeof(float));
    return route_means_ws(pooled, B, nb, H, hd, n_keep, kept,
                          static_cast<uint8_t*>(workspace) + mb, status, st);
}
