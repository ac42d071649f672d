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
//                           warp per query block: a radix select of the
//                           n_keep-th largest score (four 8-bit histogram
//                           passes) and an ordered ballot compaction that
//                           writes the kept indices in increasing order,
//                           ties at the threshold to the lower index.
#include <cmath>

#include "common.cuh"

namespace dit {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kSelThreads = 256;
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
// sc[0..nb) in shared memory: four 8-bit histogram passes over the
// order-preserving score codes find the n_keep-th largest code T, then the
// kept indices -- every code above T and the lowest-index ties at T -- are
// written in increasing order with ballots.  Same order as sorting (score
// descending, index ascending) and taking the first n_keep.
__device__ void warp_select(const float* sc, int nb, int n_keep, unsigned* hist, int32_t* out,
                            int lane) {
    uint32_t prefix = 0, mask = 0;
    int need = n_keep;              // keys still wanted among those matching the prefix
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int e = lane; e < 256; e += 32) hist[e] = 0;
        __syncwarp();
        for (int j = lane; j < nb; j += 32) {
            const uint32_t c = ordered(sc[j]);
            if ((c & mask) == prefix) atomicAdd(&hist[(c >> shift) & 255u], 1u);
        }
        __syncwarp();
        int digit = 0, above = 0;
        if (lane == 0) {
            // from the top digit down, the first bin that reaches `need`
            int acc = 0, d = 255;
            for (; d > 0; --d) {
                const int cnt = static_cast<int>(hist[d]);
                if (acc + cnt >= need) break;
                acc += cnt;
            }
            digit = d;
            above = acc;
        }
        digit = __shfl_sync(0xffffffffu, digit, 0);
        above = __shfl_sync(0xffffffffu, above, 0);
        need -= above;
        prefix |= static_cast<uint32_t>(digit) << shift;
        mask |= 255u << shift;
        __syncwarp();
    }
    // prefix is T; `need` ties at T are taken, lowest indices first
    int written = 0, eq_seen = 0;
    const unsigned below = (1u << lane) - 1u;
    for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t c = j < nb ? ordered(sc[j]) : 0u;
        const bool gt = j < nb && c > prefix;
        const bool eq = j < nb && c == prefix;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(eqm & below) < need);
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        if (take) out[written + __popc(tm & below)] = j;
        written += __popc(tm);
        eq_seen += __popc(eqm);
    }
}

// CTA (g, h, b): query blocks i = g*QB .. g*QB + QB - 1 of head h, sample b;
// all 8 warps compute the scores, then warp r selects query block r.
// Shared memory: qmean [QB][hd] fp32, scores [QB][nb] fp32, 256-bin
// histograms [8].
__global__ void __launch_bounds__(kSelThreads)
subblock_select_kernel(const float* __restrict__ pooled, int nb, int D, int hd, int QB,
                       int n_keep, int32_t* __restrict__ kept) {
    extern __shared__ __align__(16) unsigned char sm[];
    const int h = blockIdx.y, b = blockIdx.z;
    const int i0 = blockIdx.x * QB;
    const int nq = min(QB, nb - i0);
    float* qmean = reinterpret_cast<float*>(sm);                       // QB * hd
    float* scores = qmean + QB * hd;                                   // QB * nb
    unsigned* hist = reinterpret_cast<unsigned*>(scores + static_cast<int64_t>(QB) * nb);
    const float* qsrc = pooled + (static_cast<int64_t>(b) * 2 + 0) * nb * D + h * hd;
    const float* ksrc = pooled + (static_cast<int64_t>(b) * 2 + 1) * nb * D + h * hd;
    for (int e = threadIdx.x; e < nq * hd; e += kSelThreads) {
        const int r = e / hd, d = e - r * hd;
        qmean[r * hd + d] = qsrc[static_cast<int64_t>(i0 + r) * D + d];
    }
    __syncthreads();
    // scores: thread t takes key blocks t, t + 256, ...; dot products in
    // fp32, d in increasing order
    for (int j = threadIdx.x; j < nb; j += kSelThreads) {
        const float4* kv = reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(j) * D);
        float acc[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r] = 0.0f;
        for (int d4 = 0; d4 < hd / 4; ++d4) {
            const float4 kk = __ldg(kv + d4);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                if (r < nq) {
                    const float* qm = qmean + r * hd + 4 * d4;
                    acc[r] = __fmaf_rn(qm[0], kk.x, acc[r]);
                    acc[r] = __fmaf_rn(qm[1], kk.y, acc[r]);
                    acc[r] = __fmaf_rn(qm[2], kk.z, acc[r]);
                    acc[r] = __fmaf_rn(qm[3], kk.w, acc[r]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r)
            if (r < nq) scores[static_cast<int64_t>(r) * nb + j] = acc[r];
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < nq) {
        int32_t* out =
            kept + ((static_cast<int64_t>(b) * gridDim.y + h) * nb + i0 + warp) * n_keep;
        warp_select(scores + static_cast<int64_t>(warp) * nb, nb, n_keep, hist + 256 * warp, out,
                    lane);
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
    const size_t smem = static_cast<size_t>(QB) * hd * 4 + static_cast<size_t>(QB) * nb * 4 +
                        8 * 256 * sizeof(unsigned);
    if (cudaFuncSetAttribute(subblock_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    subblock_select_kernel<<<dim3((nb + QB - 1) / QB, H, B), kSelThreads, smem, st>>>(
        pooled, nb, static_cast<int>(D), hd, QB, n_keep, kept);
    return launch_status();
}
