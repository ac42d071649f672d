// adaln.cu -- AdaLN modulation, and the gated residual fused with the next
// AdaLN, each in one pass over HBM.
//
// "MiniMax-H3 no SGLang em H200", section "Só com três camadas de aceleração
// somadas chega-se a 6 vezes": the fused AdaLN update and the gated residual
// ("residual com gate"); the fused layer changes no result, so the gated
// variant normalises the residual exactly as stored in bf16.  "MiniMax H3 mở
// trọng số", section "Kiến trúc: tạo hình và tiếng trong cùng một luồng": the
// AdaLN-branch outputs are precomputed, so shift/scale/gate arrive as inputs.
//
// Design: one warp owns one token row at a time and holds the whole row in
// registers (VPL 16-byte vectors per lane; D = 5120 -> 20), so x is read
// once.  Row statistics are two warp-shuffle reductions (a mean of values
// shifted by the row's first element, then the centred sum of squares).
// The modulation vectors of the CTA's sample are staged once in shared
// memory as fp32, split into low and high float4 halves so that a warp's
// 16-byte reads hit 32 distinct banks.  The grid is (CTAs per sample, B)
// with CTAs persistent over rows.  HBM bound: 4 bytes per element moved
// (8 for the gated form) against ~10 flops.
#include "common.cuh"

namespace dit {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

struct RowParams {
    const uint4* x;
    const uint4* r;
    uint4* x_out;
    uint4* y;
    const void* shift;
    const void* scale;
    const void* gate;
    int mod_dtype;
    int64_t mod_stride;
    int64_t N;
    int Dv;
    float inv_D;
    float eps;
};

__device__ __forceinline__ float mod_at(const void* p, int dtype, int64_t i) {
    if (dtype == DIT_F32) return static_cast<const float*>(p)[i];
    return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16);
}

// bf16(x + g*r) with ONE rounding of the exact value.  The fp32 fma rounds
// once to 24 bits; rounding that to bf16 can differ from rounding the exact
// value only when the fp32 result sits exactly on a bf16 tie (low 16 bits
// 0x8000).  Then the sum is redone in fp64, where g*r (<= 32 significant
// bits) is exact, and rounded straight to bf16.
__device__ __forceinline__ float gated_add(float x, float g, float r) {
    const float s = __fmaf_rn(g, r, x);
    if ((__float_as_uint(s) & 0xFFFFu) == 0x8000u) {
        const double e = fma(static_cast<double>(g), static_cast<double>(r),
                             static_cast<double>(x));
        return __bfloat162float(__double2bfloat16(e));
    }
    return __bfloat162float(__float2bfloat16_rn(s));
}

__device__ __forceinline__ void lds8(const float4* lo, const float4* hi, int v, float (&f)[8]) {
    const float4 a = lo[v], b = hi[v];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <int VPL, bool GATED>
__global__ void __launch_bounds__(kThreads)
adaln_rows_kernel(RowParams p) {
    extern __shared__ float4 smem[];
    const int Dv = p.Dv;
    float4* s_sh = smem;            // shift:     [lo Dv][hi Dv]
    float4* s_sc = smem + 2 * Dv;   // 1 + scale: [lo Dv][hi Dv]
    float4* s_g = smem + 4 * Dv;    // gate:      [lo Dv][hi Dv] (GATED)
    const int b = blockIdx.y;
    const int64_t mb = static_cast<int64_t>(b) * p.mod_stride;
    for (int v = threadIdx.x; v < Dv; v += kThreads) {
        float sh[8], sc[8], g[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            sh[i] = mod_at(p.shift, p.mod_dtype, mb + 8 * v + i);
            sc[i] = 1.0f + mod_at(p.scale, p.mod_dtype, mb + 8 * v + i);
            if (GATED) g[i] = mod_at(p.gate, p.mod_dtype, mb + 8 * v + i);
        }
        s_sh[v] = make_float4(sh[0], sh[1], sh[2], sh[3]);
        s_sh[Dv + v] = make_float4(sh[4], sh[5], sh[6], sh[7]);
        s_sc[v] = make_float4(sc[0], sc[1], sc[2], sc[3]);
        s_sc[Dv + v] = make_float4(sc[4], sc[5], sc[6], sc[7]);
        if (GATED) {
            s_g[v] = make_float4(g[0], g[1], g[2], g[3]);
            s_g[Dv + v] = make_float4(g[4], g[5], g[6], g[7]);
        }
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t row0 = static_cast<int64_t>(b) * p.N;
    const int64_t wstep = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * kWarps + warp; n < p.N; n += wstep) {
        const int64_t base = (row0 + n) * Dv;
        uint4 xv[VPL];
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int v = j * 32 + lane;
            xv[j] = (v < Dv) ? ld_inplace(p.x + base + v) : make_uint4(0, 0, 0, 0);
        }
        if constexpr (GATED) {
            uint4 rv[VPL];
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int v = j * 32 + lane;
                rv[j] = (v < Dv) ? ld_stream(p.r + base + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int v = j * 32 + lane;
                if (v < Dv) {
                    float fx[8], fr[8], fg[8];
                    unpack8(xv[j], fx);
                    unpack8(rv[j], fr);
                    lds8(s_g, s_g + Dv, v, fg);
#pragma unroll
                    for (int i = 0; i < 8; ++i) fx[i] = gated_add(fx[i], fg[i], fr[i]);
                    xv[j] = pack8(fx);  // exact: every fx[i] is a bf16 value
                    st_stream(p.x_out + base + v, xv[j]);
                }
            }
        }
        // mean, accumulated relative to the row's first element
        const float x0 = __shfl_sync(0xffffffffu, bf16_lo(xv[0].x), 0);
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            if (j * 32 + lane < Dv) {
                float f[8];
                unpack8(xv[j], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) s += f[i] - x0;
            }
        }
        s = warp_sum(s);
        const float mu = x0 + s * p.inv_D;
        float q = 0.0f;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            if (j * 32 + lane < Dv) {
                float f[8];
                unpack8(xv[j], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float d = f[i] - mu;
                    q = __fmaf_rn(d, d, q);
                }
            }
        }
        q = warp_sum(q);
        const float rstd = rsqrtf(__fmaf_rn(q, p.inv_D, p.eps));
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int v = j * 32 + lane;
            if (v < Dv) {
                float f[8], sh[8], sc[8];
                unpack8(xv[j], f);
                lds8(s_sh, s_sh + Dv, v, sh);
                lds8(s_sc, s_sc + Dv, v, sc);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fmaf_rn((f[i] - mu) * rstd, sc[i], sh[i]);
                st_stream(p.y + base + v, pack8(f));
            }
        }
    }
}

template <bool GATED>
using RowKernel = void (*)(RowParams);

template <bool GATED>
RowKernel<GATED> pick_kernel(int vpl_needed, int* vpl) {
#define DIT_VPL_CASE(V)                              \
    if (vpl_needed <= V) {                           \
        *vpl = V;                                    \
        return adaln_rows_kernel<V, GATED>;          \
    }
    DIT_VPL_CASE(1) DIT_VPL_CASE(2) DIT_VPL_CASE(3) DIT_VPL_CASE(4) DIT_VPL_CASE(6)
    DIT_VPL_CASE(8) DIT_VPL_CASE(10) DIT_VPL_CASE(12) DIT_VPL_CASE(16) DIT_VPL_CASE(20)
    DIT_VPL_CASE(24) DIT_VPL_CASE(32)
#undef DIT_VPL_CASE
    return nullptr;
}

int check_mod(const void* p, int dtype) {
    if (!p) return DIT_ERR_NULL;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if (a % (dtype == DIT_F32 ? 4 : 2)) return DIT_ERR_ALIGN;
    return DIT_OK;
}

template <bool GATED>
int launch_rows(const RowParams& p, int B, cudaStream_t stream) {
    int vpl = 0;
    RowKernel<GATED> kernel = pick_kernel<GATED>((p.Dv + 31) / 32, &vpl);
    if (!kernel) return DIT_ERR_SHAPE;
    const size_t smem = static_cast<size_t>(GATED ? 6 : 4) * p.Dv * sizeof(float4);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    const int sms = device_sm_count();
    if (sms <= 0) return DIT_ERR_LAUNCH;
    const int occ = occupancy(reinterpret_cast<const void*>(kernel), kThreads, smem);
    int64_t per_sample = (static_cast<int64_t>(sms) * occ) / B;
    if (per_sample < 1) per_sample = 1;
    const int64_t need = (p.N + kWarps - 1) / kWarps;
    if (per_sample > need) per_sample = need;
    dim3 grid(static_cast<unsigned>(per_sample), static_cast<unsigned>(B));
    kernel<<<grid, kThreads, smem, stream>>>(p);
    return launch_status();
}

int common_checks(int B, int64_t N, int D, int mod_dtype, int64_t mod_stride, double eps) {
    if (B < 0 || N < 0 || D <= 0 || mod_stride < 0) return DIT_ERR_SHAPE;
    if (D % 8) return DIT_ERR_ALIGN;
    if (D > DIT_MAX_D || B > 65535) return DIT_ERR_SHAPE;
    if (N > (INT64_MAX / 8) / D / (B > 0 ? B : 1)) return DIT_ERR_SHAPE;
    if (mod_dtype != DIT_F32 && mod_dtype != DIT_BF16) return DIT_ERR_DTYPE;
    if (!(eps >= 0.0) || eps > 1e30) return DIT_ERR_VALUE;
    return DIT_OK;
}

}  // namespace
}  // namespace dit

extern "C" int dit_adaln_modulate(const uint16_t* x, uint16_t* y, const void* shift,
                                  const void* scale, int mod_dtype, int64_t mod_batch_stride,
                                  int B, int64_t N, int D, double eps, void* stream) {
    using namespace dit;
    if (!x || !y) return DIT_ERR_NULL;
    int st = common_checks(B, N, D, mod_dtype, mod_batch_stride, eps);
    if (st) return st;
    if ((st = check_mod(shift, mod_dtype)) || (st = check_mod(scale, mod_dtype))) return st;
    if (!aligned16(x) || !aligned16(y)) return DIT_ERR_ALIGN;
    const size_t bytes = static_cast<size_t>(B) * N * D * 2;
    if (x != y && overlaps(x, bytes, y, bytes)) return DIT_ERR_OVERLAP;
    if (B == 0 || N == 0) return DIT_OK;
    RowParams p{};
    p.x = reinterpret_cast<const uint4*>(x);
    p.y = reinterpret_cast<uint4*>(y);
    p.shift = shift;
    p.scale = scale;
    p.mod_dtype = mod_dtype;
    p.mod_stride = mod_batch_stride;
    p.N = N;
    p.Dv = D / 8;
    p.inv_D = 1.0f / static_cast<float>(D);
    p.eps = static_cast<float>(eps);
    return launch_rows<false>(p, B, as_stream(stream));
}

extern "C" int dit_gated_residual_adaln(const uint16_t* x, const uint16_t* r, uint16_t* x_out,
                                        uint16_t* y, const void* gate, const void* shift,
                                        const void* scale, int mod_dtype,
                                        int64_t mod_batch_stride, int B, int64_t N, int D,
                                        double eps, void* stream) {
    using namespace dit;
    if (!x || !r || !x_out || !y) return DIT_ERR_NULL;
    int st = common_checks(B, N, D, mod_dtype, mod_batch_stride, eps);
    if (st) return st;
    if ((st = check_mod(gate, mod_dtype)) || (st = check_mod(shift, mod_dtype)) ||
        (st = check_mod(scale, mod_dtype)))
        return st;
    if (!aligned16(x) || !aligned16(r) || !aligned16(x_out) || !aligned16(y))
        return DIT_ERR_ALIGN;
    const size_t bytes = static_cast<size_t>(B) * N * D * 2;
    if ((x != x_out && overlaps(x, bytes, x_out, bytes)) || overlaps(x, bytes, r, bytes) ||
        overlaps(x, bytes, y, bytes) || overlaps(r, bytes, x_out, bytes) ||
        overlaps(r, bytes, y, bytes) || overlaps(x_out, bytes, y, bytes))
        return DIT_ERR_OVERLAP;
    if (B == 0 || N == 0) return DIT_OK;
    RowParams p{};
    p.x = reinterpret_cast<const uint4*>(x);
    p.r = reinterpret_cast<const uint4*>(r);
    p.x_out = reinterpret_cast<uint4*>(x_out);
    p.y = reinterpret_cast<uint4*>(y);
    p.shift = shift;
    p.scale = scale;
    p.gate = gate;
    p.mod_dtype = mod_dtype;
    p.mod_stride = mod_batch_stride;
    p.N = N;
    p.Dv = D / 8;
    p.inv_D = 1.0f / static_cast<float>(D);
    p.eps = static_cast<float>(eps);
    return launch_rows<true>(p, B, as_stream(stream));
}
