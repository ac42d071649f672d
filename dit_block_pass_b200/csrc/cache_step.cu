// cache_step.cu -- the Cache-DiT step cache: the residual the skipped blocks
// add, stored on a computing step and added back on a reusing one, and the
// reuse rule over a denoising run.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração somadas chega-se a 6 vezes":
// Cache-DiT reuses results cached between neighbouring denoising steps, and
// a residual-difference threshold (0.04 conservative, 0.08 in the more
// aggressive stride mode) decides whether a step reuses them.  The pages
// give no more; the cached result is read here as the residual of the
// skipped blocks, stored in bf16 like the hidden state.
//
// Rounding: the exact sum or difference of two bf16 values either fits the
// 24-bit fp32 significand (exponents at most 15 apart) or has its smaller
// operand below 2^-15 of the larger, far under half a bf16 ulp.  So one
// fp32 add followed by one round-to-nearest-even to bf16 gives the nearest
// bf16 of the exact value, with no double rounding.
//
// Design: elementwise and HBM bound (6 bytes per element: two reads, one
// write).  One-shot grid: each thread loads U vectors of both inputs, then
// adds and stores them, and its CTA exits.  32-byte vectors when the count
// and the pointers allow, else 16-byte.  An output may be one of its inputs
// (in place); loads are then coherent.
#include "common.cuh"

namespace dit {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// Two bf16 pairs -> bf16(a + s*b) for each half, s = +1 or -1.
template <bool SUB>
__device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
    const float lo = SUB ? bf16_lo(a) - bf16_lo(b) : bf16_lo(a) + bf16_lo(b);
    const float hi = SUB ? bf16_hi(a) - bf16_hi(b) : bf16_hi(a) + bf16_hi(b);
    return pack2(lo, hi);
}

template <int E, bool INPLACE>
struct RVec;
template <bool INPLACE>
struct RVec<8, INPLACE> {
    using T = uint4;
    static __device__ __forceinline__ T load(const T* p) {
        return INPLACE ? ld_inplace(p) : ld_stream(p);
    }
    static __device__ __forceinline__ void store(T* p, const T& v) { st_stream(p, v); }
    template <bool SUB>
    static __device__ __forceinline__ T add(const T& a, const T& b) {
        return make_uint4(add2<SUB>(a.x, b.x), add2<SUB>(a.y, b.y), add2<SUB>(a.z, b.z),
                          add2<SUB>(a.w, b.w));
    }
};
template <bool INPLACE>
struct RVec<16, INPLACE> {
    using T = u32x8;
    static __device__ __forceinline__ T load(const T* p) {
        return INPLACE ? ld_inplace256(p) : ld_stream256(p);
    }
    static __device__ __forceinline__ void store(T* p, const T& v) { st_stream256(p, v); }
    template <bool SUB>
    static __device__ __forceinline__ T add(const T& a, const T& b) {
        T o;
#pragma unroll
        for (int i = 0; i < 8; ++i) o.w[i] = add2<SUB>(a.w[i], b.w[i]);
        return o;
    }
};

// out = bf16(a + b) (SUB false) or bf16(a - b) (SUB true) over nv vectors.
// CTA c covers vectors [c*T*U, (c+1)*T*U); thread t the U vectors
// c*T*U + u*T + t.
template <int E, bool SUB, bool INPLACE>
__global__ void __launch_bounds__(kThreads)
residual_kernel(const void* a_, const void* b_, void* out_, int64_t nv) {
    using V = RVec<E, INPLACE>;
    using T = typename V::T;
    const T* a = static_cast<const T*>(a_);
    const T* b = static_cast<const T*>(b_);
    T* out = static_cast<T*>(out_);
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kUnroll + threadIdx.x;
    T va[kUnroll], vb[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + static_cast<int64_t>(u) * kThreads;
        if (i < nv) {
            va[u] = V::load(a + i);
            vb[u] = V::load(b + i);
        }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + static_cast<int64_t>(u) * kThreads;
        if (i < nv) V::store(out + i, V::template add<SUB>(va[u], vb[u]));
    }
}

template <bool SUB>
int launch_residual(const uint16_t* a, const uint16_t* b, uint16_t* out, int64_t n,
                    void* stream) {
    if (n < 0) return DIT_ERR_SHAPE;
    if (n == 0) return DIT_OK;
    if (!a || !b || !out) return DIT_ERR_NULL;
    if (n % 8) return DIT_ERR_ALIGN;
    if (!aligned16(a) || !aligned16(b) || !aligned16(out)) return DIT_ERR_ALIGN;
    const size_t bytes = static_cast<size_t>(n) * 2;
    // an output is either one of the inputs exactly or disjoint from both
    if ((out != a && overlaps(out, bytes, a, bytes)) ||
        (out != b && overlaps(out, bytes, b, bytes)))
        return DIT_ERR_OVERLAP;
    const bool inplace = out == a || out == b;
    const bool wide = n % 16 == 0 && aligned32(a) && aligned32(b) && aligned32(out);
    const int64_t nv = wide ? n / 16 : n / 8;
    const int64_t per_cta = static_cast<int64_t>(kThreads) * kUnroll;
    const int64_t ctas = (nv + per_cta - 1) / per_cta;
    if (ctas > 0x7FFFFFFF) return DIT_ERR_SHAPE;
    const dim3 grid(static_cast<unsigned>(ctas));
    cudaStream_t st = as_stream(stream);
    if (wide) {
        if (inplace) residual_kernel<16, SUB, true><<<grid, kThreads, 0, st>>>(a, b, out, nv);
        else residual_kernel<16, SUB, false><<<grid, kThreads, 0, st>>>(a, b, out, nv);
    } else {
        if (inplace) residual_kernel<8, SUB, true><<<grid, kThreads, 0, st>>>(a, b, out, nv);
        else residual_kernel<8, SUB, false><<<grid, kThreads, 0, st>>>(a, b, out, nv);
    }
    return launch_status();
}

}  // namespace
}  // namespace dit

extern "C" int cachedit_residual_store(const uint16_t* before, const uint16_t* after,
                                       uint16_t* residual, int64_t n, void* stream) {
    return dit::launch_residual<true>(after, before, residual, n, stream);
}

extern "C" int cachedit_residual_apply(const uint16_t* h, const uint16_t* residual, uint16_t* out,
                                       int64_t n, void* stream) {
    return dit::launch_residual<false>(h, residual, out, n, stream);
}

extern "C" int dit_cache_policy_init(dit_cache_policy* p, double threshold, int warmup_steps,
                                     int max_cached_steps) {
    if (!p) return DIT_ERR_NULL;
    if (threshold != threshold || warmup_steps < 0 || max_cached_steps < 0) return DIT_ERR_VALUE;
    p->threshold = threshold;
    p->warmup_steps = warmup_steps;
    p->max_cached_steps = max_cached_steps;
    p->step = 0;
    p->run = 0;
    p->computed = 0;
    p->reused = 0;
    return DIT_OK;
}

extern "C" int dit_cache_policy_decide(dit_cache_policy* p, double rel) {
    if (!p) return DIT_ERR_NULL;
    const int t = p->step;
    const bool reuse = t >= 1 && t >= p->warmup_steps && rel < p->threshold &&
                       (p->max_cached_steps == 0 || p->run < p->max_cached_steps);
    p->run = reuse ? p->run + 1 : 0;
    p->step = t + 1;
    if (reuse) ++p->reused;
    else ++p->computed;
    return reuse ? 1 : 0;
}
