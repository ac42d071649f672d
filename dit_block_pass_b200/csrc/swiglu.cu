// swiglu.cu -- SwiGLU activation, one streaming pass over HBM.
//
// "MiniMax-H3 no SGLang em H200", section "Só com três camadas de aceleração
// somadas chega-se a 6 vezes": the SwiGLU activation is one of the fused
// operators.  out[m, j] = silu(in[m, j]) * in[m, F + j].
//
// Design: a persistent grid (SM count x resident CTAs) walks the M*F/8
// output vectors with a grid stride.  Each thread keeps its (row, column)
// position and advances it by a precomputed (rows, columns) step, so the
// loop has no integer division.  U independent vectors are in flight per
// thread (2U 16-byte loads), which covers HBM latency at full occupancy.
// Reads bypass L1 and are evict-first in L2; writes are streaming stores.
// Arithmetic intensity is ~0.8 flop/byte: the kernel is HBM bound.
#include "common.cuh"

namespace dit {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 2;

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

template <int U>
__global__ void __launch_bounds__(kThreads)
swiglu_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t Fv, int64_t total,
              int64_t step_r, int64_t step_c) {
    const int64_t T = static_cast<int64_t>(gridDim.x) * kThreads;
    int64_t v = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    int64_t row = v / Fv;
    int64_t col = v - row * Fv;
    for (; v < total; v += U * T) {
        uint4 a[U], b[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (v + u * T < total) {
                const uint4* src = in + row * 2 * Fv + col;
                a[u] = ld_stream(src);
                b[u] = ld_stream(src + Fv);
            }
            row += step_r;
            col += step_c;
            if (col >= Fv) {
                col -= Fv;
                ++row;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (v + u * T < total) st_stream(out + v + u * T, swiglu8(a[u], b[u]));
    }
}

}  // namespace
}  // namespace dit

extern "C" int dit_swiglu(const uint16_t* in, uint16_t* out, int64_t M, int F, void* stream) {
    using namespace dit;
    if (!in || !out) return DIT_ERR_NULL;
    if (M < 0 || F <= 0) return DIT_ERR_SHAPE;
    if (F % 8 || !aligned16(in) || !aligned16(out)) return DIT_ERR_ALIGN;
    if (M > (INT64_MAX / 8) / F) return DIT_ERR_SHAPE;
    const size_t in_bytes = static_cast<size_t>(M) * 2 * F * 2;
    const size_t out_bytes = static_cast<size_t>(M) * F * 2;
    if (overlaps(in, in_bytes, out, out_bytes)) return DIT_ERR_OVERLAP;
    if (M == 0) return DIT_OK;

    const int64_t Fv = F / 8;
    const int64_t total = M * Fv;
    const int sms = device_sm_count();
    if (sms <= 0) return DIT_ERR_LAUNCH;
    auto kernel = swiglu_kernel<kUnroll>;
    const int occ = occupancy(reinterpret_cast<const void*>(kernel), kThreads, 0);
    int64_t blocks = static_cast<int64_t>(sms) * occ;
    const int64_t need = (total + kThreads - 1) / kThreads;
    if (blocks > need) blocks = need;
    const int64_t T = blocks * kThreads;
    kernel<<<static_cast<unsigned>(blocks), kThreads, 0, as_stream(stream)>>>(
        reinterpret_cast<const uint4*>(in), reinterpret_cast<uint4*>(out), Fv, total, T / Fv,
        T % Fv);
    return launch_status();
}
