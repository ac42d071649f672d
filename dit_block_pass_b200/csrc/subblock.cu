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
//   subblock_select_kernel  CTA (query-block group, h, b): the group's query
//                           means in shared memory, one pass over the key
//                           means of head h (L2 resident) for all scores,
//                           then per query block a bitonic sort of 64-bit
//                           keys (order-preserving score bits, then the
//                           inverted block index) and a second, ascending
//                           sort of the n_keep winners' indices.
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

// Bitonic sort of n (a power of two) 64-bit keys in shared memory by the
// whole CTA, descending or ascending.
__device__ __forceinline__ void bitonic(unsigned long long* keys, int n, bool descending) {
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int e = threadIdx.x; e < n / 2; e += kSelThreads) {
                const int lo = 2 * e - (e & (stride - 1));
                const int hi = lo + stride;
                // sub-sequences alternate direction; the last merge goes the
                // requested way
                const bool first = ((lo & size) == 0) == descending;
                const unsigned long long a = keys[lo], c = keys[hi];
                if (first ? (a < c) : (a > c)) {
                    keys[lo] = c;
                    keys[hi] = a;
                }
            }
            __syncthreads();
        }
    }
}

// CTA (g, h, b): query blocks i = g*QB .. g*QB + QB - 1 of head h, sample b.
// Shared memory: qmean [QB][hd] fp32, scores [QB][nb_pad] fp32, keys
// [nb_pad] u64.
__global__ void __launch_bounds__(kSelThreads)
subblock_select_kernel(const float* __restrict__ pooled, int nb, int nb_pad, int D, int hd,
                       int QB, int n_keep, int keep_pad, int32_t* __restrict__ kept) {
    extern __shared__ __align__(16) unsigned char sm[];
    const int h = blockIdx.y, b = blockIdx.z;
    const int i0 = blockIdx.x * QB;
    const int nq = min(QB, nb - i0);
    float* qmean = reinterpret_cast<float*>(sm);                       // QB * hd
    float* scores = qmean + QB * hd;                                   // QB * nb_pad
    unsigned long long* keys =
        reinterpret_cast<unsigned long long*>(scores + static_cast<int64_t>(QB) * nb_pad);
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
        float acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = 0.0f;
        for (int d4 = 0; d4 < hd / 4; ++d4) {
            const float4 kk = __ldg(kv + d4);
#pragma unroll
            for (int r = 0; r < 16; ++r) {
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
        for (int r = 0; r < 16; ++r)
            if (r < nq) scores[static_cast<int64_t>(r) * nb_pad + j] = acc[r];
    }
    __syncthreads();
    for (int r = 0; r < nq; ++r) {
        // keys: score bits, then the inverted index, so that a descending
        // sort puts equal scores in increasing index order; padding sorts last
        for (int j = threadIdx.x; j < nb_pad; j += kSelThreads) {
            keys[j] = j < nb ? (static_cast<unsigned long long>(
                                    ordered(scores[static_cast<int64_t>(r) * nb_pad + j]))
                                << 32) |
                                   (0xFFFFFFFFu - static_cast<uint32_t>(j))
                             : 0ull;
        }
        __syncthreads();
        bitonic(keys, nb_pad, true);
        // the kept block indices, then sorted ascending (padding last)
        unsigned long long idx[kMaxBlocks / kSelThreads];
        int c = 0;
        for (int e = threadIdx.x; e < keep_pad; e += kSelThreads, ++c)
            idx[c] = e < n_keep ? static_cast<unsigned long long>(
                                      0xFFFFFFFFu - static_cast<uint32_t>(keys[e] & 0xFFFFFFFFull))
                                : ~0ull;
        __syncthreads();
        c = 0;
        for (int e = threadIdx.x; e < keep_pad; e += kSelThreads, ++c) keys[e] = idx[c];
        __syncthreads();
        bitonic(keys, keep_pad, false);
        int32_t* out = kept + ((static_cast<int64_t>(b) * gridDim.y + h) * nb + i0 + r) * n_keep;
        for (int e = threadIdx.x; e < n_keep; e += kSelThreads)
            out[e] = static_cast<int32_t>(keys[e]);
        __syncthreads();
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

int pad_pow2(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
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
    const int nb_pad = pad_pow2(nb);
    const int keep_pad = pad_pow2(n_keep);
    // query blocks per CTA: as many as fit in about 96 KB of scores (<= 16)
    int QB = 16;
    while (QB > 1 && static_cast<size_t>(QB) * nb_pad * 4 > 96 * 1024) QB >>= 1;
    const size_t smem = static_cast<size_t>(QB) * hd * 4 + static_cast<size_t>(QB) * nb_pad * 4 +
                        static_cast<size_t>(nb_pad) * 8;
    if (cudaFuncSetAttribute(subblock_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    subblock_select_kernel<<<dim3((nb + QB - 1) / QB, H, B), kSelThreads, smem, st>>>(
        pooled, nb, nb_pad, static_cast<int>(D), hd, QB, n_keep, keep_pad, kept);
    return launch_status();
}
