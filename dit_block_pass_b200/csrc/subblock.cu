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
// Two kernels:
//   subblock_pool_kernel    one pass over q and k (HBM bound): CTA (j, b, t)
//                           sums the rows of block j of sample b of tensor t
//                           (q or k) for every column, 16-byte loads, fp32,
//                           and writes the means [B, 2, n_blocks, H*hd].
//   subblock_select_kernel  CTA (up to 8 query blocks, h, b): the query means
//                           in shared memory, one pass over the key means of
//                           head h (L2 resident) for all scores, then one
//                           warp per query block: the n_keep-th largest
//                           score found bit by bit with warp-wide counts
//                           (the scores in registers up to 1024 key
//                           blocks) and an ordered ballot compaction that
//                           writes the kept indices in increasing order,
//                           ties at the threshold to the lower index.
#include <cmath>

#include "common.cuh"

namespace dit {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kSelThreads = 256;
constexpr int kKeysPerThread = 4;       // key blocks per thread and pass of the score loop
constexpr int kMaxBlocks = 8192;           // key blocks per sample

// Means of the rows of one block, every column: thread t takes column
// vectors t, t + 256, ...; fp32 sums over at most `block` rows, one divide.
__global__ void __launch_bounds__(kPoolThreads)
subblock_pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, int64_t stride_v,
                     int64_t N, int block, int nb, int Dv, float* __restrict__ pooled) {
    const int j = blockIdx.x, b = blockIdx.y, t = blockIdx.z;
    const uint4* src = t == 0 ? q : k;
    const int64_t r0 = static_cast<int64_t>(j) * block;
    const int64_t r1 = r0 + block < N ? r0 + block : N;
    const float count = static_cast<float>(r1 - r0);
    float* out = pooled + ((static_cast<int64_t>(b) * 2 + t) * nb + j) * (static_cast<int64_t>(Dv) * 8);
    for (int v = threadIdx.x; v < Dv; v += kPoolThreads) {
        float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const uint4* p = src + (static_cast<int64_t>(b) * N + r0) * stride_v + v;
        int64_t r = r0;
        // four rows in flight at a time
        for (; r + 4 <= r1; r += 4, p += 4 * stride_v) {
            uint4 a[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) a[u] = ld_stream(p + u * stride_v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
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

// CTA (g, h, b): query blocks i = g*QB .. g*QB + QB - 1 of head h, sample b;
// all 8 warps compute the scores, then warp r selects query block r.
// Shared memory: qmean [8][hd] fp32, scores [QB][nb] fp32.
__global__ void __launch_bounds__(kSelThreads)
subblock_select_kernel(const float* __restrict__ pooled, int nb, int D, int hd, int QB,
                       int n_keep, int32_t* __restrict__ kept) {
    extern __shared__ __align__(16) unsigned char sm[];
    const int h = blockIdx.y, b = blockIdx.z;
    const int i0 = blockIdx.x * QB;
    const int nq = min(QB, nb - i0);
    float* qmean = reinterpret_cast<float*>(sm);                       // 8 * hd
    float* scores = qmean + 8 * hd;                                    // QB * nb
    const float* qsrc = pooled + (static_cast<int64_t>(b) * 2 + 0) * nb * D + h * hd;
    const float* ksrc = pooled + (static_cast<int64_t>(b) * 2 + 1) * nb * D + h * hd;
    // rows past the last query block are zeros (their scores are not kept),
    // so the score loop below has no per-row test
    for (int e = threadIdx.x; e < 8 * hd; e += kSelThreads) {
        const int r = e / hd, d = e - r * hd;
        qmean[r * hd + d] = r < nq ? qsrc[static_cast<int64_t>(i0 + r) * D + d] : 0.0f;
    }
    __syncthreads();
    // scores: thread t takes key blocks t + 256 u (u < kKeysPerThread) per
    // pass; each 16-byte query read feeds 16 FMAs.  Dot products in fp32,
    // d in increasing order.  hd % 8 == 0, so every float4 is aligned.
    const float4* q4 = reinterpret_cast<const float4*>(qmean);
    const int hd4 = hd / 4;
    for (int jb = 0; jb < nb; jb += kKeysPerThread * kSelThreads) {
        const float4* kv[kKeysPerThread];
        bool live[kKeysPerThread];
#pragma unroll
        for (int u = 0; u < kKeysPerThread; ++u) {
            const int j = jb + u * kSelThreads + threadIdx.x;
            live[u] = j < nb;
            kv[u] = reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(live[u] ? j : 0) * D);
        }
        float acc[kKeysPerThread][8];
#pragma unroll
        for (int u = 0; u < kKeysPerThread; ++u)
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[u][r] = 0.0f;
        for (int d4 = 0; d4 < hd4; ++d4) {
            float4 kk[kKeysPerThread];
#pragma unroll
            for (int u = 0; u < kKeysPerThread; ++u) kk[u] = __ldg(kv[u] + d4);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float4 qq = q4[r * hd4 + d4];
#pragma unroll
                for (int u = 0; u < kKeysPerThread; ++u) {
                    acc[u][r] = __fmaf_rn(qq.x, kk[u].x, acc[u][r]);
                    acc[u][r] = __fmaf_rn(qq.y, kk[u].y, acc[u][r]);
                    acc[u][r] = __fmaf_rn(qq.z, kk[u].z, acc[u][r]);
                    acc[u][r] = __fmaf_rn(qq.w, kk[u].w, acc[u][r]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kKeysPerThread; ++u) {
            const int j = jb + u * kSelThreads + threadIdx.x;
#pragma unroll
            for (int r = 0; r < 8; ++r)
                if (live[u] && r < nq) scores[static_cast<int64_t>(r) * nb + j] = acc[u][r];
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < nq) {
        int32_t* out =
            kept + ((static_cast<int64_t>(b) * gridDim.y + h) * nb + i0 + warp) * n_keep;
        const float* sc = scores + static_cast<int64_t>(warp) * nb;
        if (nb <= 256)
            warp_select_reg<8>(sc, nb, n_keep, out, lane);
        else if (nb <= 512)
            warp_select_reg<16>(sc, nb, n_keep, out, lane);
        else if (nb <= 1024)
            warp_select_reg<32>(sc, nb, n_keep, out, lane);
        else
            warp_select_smem(sc, nb, n_keep, out, lane);
    }
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
    return static_cast<size_t>(B) * 2 * nb * H * hd * sizeof(float);
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
    subblock_pool_kernel<<<dim3(nb, B, 2), kPoolThreads, 0, st>>>(
        reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k), row_stride / 8, N,
        block, nb, static_cast<int>(D / 8), pooled);
    int rc = launch_status();
    if (rc) return rc;
    // query blocks per CTA (one per warp): as many as fit in about 96 KB of scores
    int QB = 8;
    while (QB > 1 && static_cast<size_t>(QB) * nb * 4 > 96 * 1024) QB >>= 1;
    const size_t smem = static_cast<size_t>(8) * hd * 4 + static_cast<size_t>(QB) * nb * 4;
    if (cudaFuncSetAttribute(subblock_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    subblock_select_kernel<<<dim3((nb + QB - 1) / QB, H, B), kSelThreads, smem, st>>>(
        pooled, nb, static_cast<int>(D), hd, QB, n_keep, kept);
    return launch_status();
}
