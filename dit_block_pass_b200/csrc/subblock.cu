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
// Three kernels:
//   subblock_pool_kernel    one pass over q and k (HBM bound): CTA (j, b, t,
//                           column chunk) sums the rows of block j of sample
//                           b of tensor t (q or k), a 16-byte column vector
//                           per thread, fp32, and writes the means
//                           [B, 2, n_blocks, H*hd].
//   subblock_scores_kernel  per (sample, head) the n_blocks x n_blocks fp32
//                           scores as a tiled GEMM of the L2-resident means
//                           (128 x 128 tiles, 8 x 8 per thread), into the
//                           workspace after the means.
//   subblock_select_kernel  one warp per query block: the n_keep-th largest
//                           score of its row found bit by bit with warp-wide
//                           counts (the row in registers up to 2048 key
//                           blocks) and an ordered ballot compaction that
//                           writes the kept indices in increasing order,
//                           ties at the threshold to the lower index.
#include <cmath>

#include "common.cuh"

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
__device__ void warp_select_reg(const float* sc, int nb, int n_keep, int32_t* out, int lane) {
    uint32_t c[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
        const int j = k * 32 + lane;
        c[k] = j < nb ? ordered(sc[j]) : 0u;
    }
    // a candidate is never 0, so the padding codes (0) are never counted
    uint32_t T = 0;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        unsigned cnt = 0;
#pragma unroll
        for (int k = 0; k < KPL; ++k) cnt += c[k] >= cand ? 1u : 0u;
        if (__reduce_add_sync(0xffffffffu, cnt) >= static_cast<unsigned>(n_keep)) T = cand;
    }
    unsigned gt = 0;
#pragma unroll
    for (int k = 0; k < KPL; ++k) gt += c[k] > T ? 1u : 0u;
    // `need` ties at T are taken, lowest indices first
    const int need = n_keep - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
    int written = 0, eq_seen = 0;
    const unsigned below = (1u << lane) - 1u;
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
    if constexpr (KPL > 0)
        warp_select_reg<KPL>(sc, nb, n_keep, out, lane);
    else
        warp_select_smem(sc, nb, n_keep, out, lane);
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
    // the block means [B, 2, nb, H*hd], then the scores [B, H, nb, nb], fp32
    return (static_cast<size_t>(B) * 2 * nb * H * hd + static_cast<size_t>(B) * H * nb * nb) *
           sizeof(float);
}

namespace dit {
namespace {

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

}  // namespace
}  // namespace dit

extern "C" size_t dit_subblock_means_workspace_bytes(int B, int64_t N, int H, int block) {
    if (B < 0 || N < 0 || H < 1 || block < 1) return 0;
    const int64_t nb = (N + block - 1) / block;
    return static_cast<size_t>(B) * H * nb * nb * sizeof(float);
}

extern "C" int dit_subblock_router_means(const float* block_means, int B, int64_t N, int H,
                                         int hd, int block, double sparsity, int32_t* kept,
                                         void* workspace, size_t workspace_bytes, void* stream) {
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
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < dit_subblock_means_workspace_bytes(B, N, H, block))
        return DIT_ERR_WORKSPACE;
    return route_from_means(block_means, B, nb, H, hd, keep_count(nb, sparsity), kept,
                            static_cast<float*>(workspace), as_stream(stream));
}

extern "C" int dit_subblock_router(const uint16_t* q, const uint16_t* k, int64_t row_stride,
                                   int B, int64_t N, int H, int hd, int block, double sparsity,
                                   int32_t* kept, void* workspace, size_t workspace_bytes,
                                   void* stream) {
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
    float* scores = pooled + static_cast<int64_t>(B) * 2 * nb * D;
    return route_from_means(pooled, B, nb, H, hd, n_keep, kept, scores, st);
}
