// swiglu.cu -- SwiGLU activation, one streaming pass over HBM.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração
// somadas chega-se a 6 vezes": the SwiGLU activation is one of the fused
// operators.  out[m, j] = silu(in[m, j]) * in[m, F + j].
//
// Design: a one-shot grid over the output vectors (each thread loads U = 4
// vectors of both halves, then computes and stores them, and its CTA exits;
// on B200 this sustained ~7% more HBM bandwidth than a persistent grid-stride
// loop, above the measured copy bandwidth, since 2/3 of the traffic is
// reads).  32-byte vectors (16 values, the 256-bit loads and stores of
// sm_100) when F is a multiple of 16 and the pointers are 32-byte aligned,
// else 16-byte vectors.  Reads bypass L1, are evict-first in L2 with a
// 256-byte fetch hint; writes are streaming stores.  Arithmetic intensity is
// ~0.8 flop/byte: the kernel is HBM bound.
#include "common.cuh"

namespace dit {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;   // vectors per thread (measured best on B200)

// silu(a) * b = a * b / (1 + e^-a).  __expf and the fast divide carry a few
// fp32 ulp of relative error, far below half a bf16 ulp.  For a < -87 the
// denominator exceeds 2^126 and the fast divide returns 0, where the exact
// value is below 1e-36 in magnitude.
__device__ __forceinline__ float silu_mul(float a, float b) {
    return __fdividef(a, 1.0f + __expf(-a)) * b;
}

__device__ __forceinline__ uint4 swiglu8(const uint4& a, const uint4& b) {
    float fa[8], fb[8], o[8];
    unpack8(a, fa);
    unpack8(b, fb);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = silu_mul(fa[i], fb[i]);
    return pack8(o);
}

// Vector of E bf16 values: E = 8 (16-byte accesses) or E = 16 (32-byte).
template <int E>
struct Vec;
template <>
struct Vec<8> {
    using T = uint4;
    static __device__ __forceinline__ T load(const T* p) { return ld_stream(p); }
    static __device__ __forceinline__ void store(T* p, const T& v) { st_stream(p, v); }
    static __device__ __forceinline__ T apply(const T& a, const T& b) { return swiglu8(a, b); }
};
template <>
struct Vec<16> {
    using T = u32x8;
    static __device__ __forceinline__ T load(const T* p) { return ld_stream256(p); }
    static __device__ __forceinline__ void store(T* p, const T& v) { st_stream256(p, v); }
    static __device__ __forceinline__ T apply(const T& a, const T& b) {
        const uint4 a0 = make_uint4(a.w[0], a.w[1], a.w[2], a.w[3]);
        const uint4 a1 = make_uint4(a.w[4], a.w[5], a.w[6], a.w[7]);
        const uint4 b0 = make_uint4(b.w[0], b.w[1], b.w[2], b.w[3]);
        const uint4 b1 = make_uint4(b.w[4], b.w[5], b.w[6], b.w[7]);
        const uint4 o0 = swiglu8(a0, b0), o1 = swiglu8(a1, b1);
        T o;
        o.w[0] = o0.x; o.w[1] = o0.y; o.w[2] = o0.z; o.w[3] = o0.w;
        o.w[4] = o1.x; o.w[5] = o1.y; o.w[6] = o1.z; o.w[7] = o1.w;
        return o;
    }
};

// Fv = vectors per output row (F / E); total = M * Fv.  One-shot grid: CTA
// b covers output vectors [b*T*U, (b+1)*T*U), thread t the U vectors
// b*T*U + u*T + t, loads first, then the U results.
template <int E, int U>
__global__ void __launch_bounds__(kThreads)
swiglu_kernel(const void* __restrict__ in_, void* __restrict__ out_, int64_t Fv, int64_t total,
              int64_t step_r, int64_t step_c) {
    using V = Vec<E>;
    using T = typename V::T;
    const T* in = static_cast<const T*>(in_);
    T* out = static_cast<T*>(out_);
    const int64_t v0 = static_cast<int64_t>(blockIdx.x) * (kThreads * U) + threadIdx.x;
    // (row, col) of v0 + u*kThreads, advanced by (step_r, step_c) = divmod(kThreads, Fv)
    int64_t row = v0 / Fv, col = v0 - row * Fv;
    T a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (v0 + u * kThreads < total) {
            const T* src = in + row * 2 * Fv + col;
            a[u] = V::load(src);
            b[u] = V::load(src + Fv);
        }
        row += step_r;
        col += step_c;
        if (col >= Fv) {
            col -= Fv;
            ++row;
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t v = v0 + u * kThreads;
        if (v < total) V::store(out + v, V::apply(a[u], b[u]));
    }
}

}  // namespace
}  // namespace dit

extern "C" int dit_swiglu(const uint16_t* in, uint16_t* out, int64_t M, int F, void* stream) {
    using namespace dit;
    if (M < 0 || F <= 0) return DIT_ERR_SHAPE;
    if (F % 8) return DIT_ERR_ALIGN;
    if (M > (INT64_MAX / 8) / F) return DIT_ERR_SHAPE;
    if (M == 0) return DIT_OK;
    if (!in || !out) return DIT_ERR_NULL;
    if (!aligned16(in) || !aligned16(out)) return DIT_ERR_ALIGN;
    const size_t in_bytes = static_cast<size_t>(M) * 2 * F * 2;
    const size_t out_bytes = static_cast<size_t>(M) * F * 2;
    if (overlaps(in, in_bytes, out, out_bytes)) return DIT_ERR_OVERLAP;

    // 32-byte vectors when the rows allow them, else 16-byte vectors
    const bool wide = (F % 16 == 0) && aligned32(in) && aligned32(out);
    const int E = wide ? 16 : 8;
    const int64_t Fv = F / E;
    const int64_t total = M * Fv;
    auto kernel = wide ? swiglu_kernel<16, kUnroll> : swiglu_kernel<8, kUnroll>;
    const int64_t blocks = (total + kThreads * kUnroll - 1) / (kThreads * kUnroll);
    if (blocks > 0x7FFFFFFF) return DIT_ERR_SHAPE;
    kernel<<<static_cast<unsigned>(blocks), kThreads, 0, as_stream(stream)>>>(
        in, out, Fv, total, kThreads / Fv, kThreads % Fv);
    return launch_status();
}
