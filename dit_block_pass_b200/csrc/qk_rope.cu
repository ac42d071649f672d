// qk_rope.cu -- per-head QK RMSNorm fused with 3D (t, h, w) rotary position
// embedding, in place, in one pass over HBM.
//
// "MiniMax-H3 no SGLang em H200", section "Só com três camadas de aceleração
// somadas chega-se a 6 vezes": "QK RMSNorm com 3D RoPE" is one fused operator;
// "SGLang acelera MiniMax-H3 em GPUs H200", first paragraph, lists QK RMSNorm
// and 3D RoPE among the fused low-level operations.
//
// Design: one warp per token.  A token row of H heads x hd is H*hd/8
// consecutive 16-byte vectors; warp pass i reads vectors 32*i + lane, so each
// load instruction covers 512 contiguous bytes and a head occupies hd/8
// adjacent lanes.  The head's sum of squares is a shuffle reduction inside
// that lane group.  A lane always holds the same 4 rotation pairs of a head
// (pairs 4*(lane mod hd/8) .. +3), so it computes their 4 angles once per
// token and reuses them for every head of q and k.  Frequencies are fp64
// (computed once per thread), angles pos*omega are formed and reduced modulo
// 2*pi in fp64, and sin/cos are taken in fp32 on the reduced angle, which
// keeps the rotation accurate to a few fp32 ulp for positions in the hundreds.
// q and k are loaded CH vectors per lane at a time (both tensors in one
// stream of vectors) to keep enough bytes in flight.  HBM bound.
#include "common.cuh"

namespace dit {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 8;

struct QKParams {
    uint4* t0;              // first tensor processed (q, or k when q is NULL)
    uint4* t1;              // second tensor or NULL
    const void* w0;
    const void* w1;
    int w_dtype;
    int64_t stride_v;       // row stride in 16-byte vectors
    int64_t rows;           // B * N
    int64_t N;
    int nvr;                // vectors per tensor row = H * hd / 8
    int Hg, Wg;
    const int32_t* pos;
    int64_t pos_offset;
    int pt, ph, pw;
    double theta;
    float eps;
};

__device__ __forceinline__ float w_at(const void* p, int dtype, int i) {
    if (dtype == DIT_F32) return static_cast<const float*>(p)[i];
    return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16);
}

template <int HD>
__global__ void __launch_bounds__(kThreads)
qk_rmsnorm_rope3d_kernel(QKParams p) {
    constexpr int LPH = HD / 8;             // lanes per head
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPH;             // this lane's vector within a head

    // this lane's rotation pairs: p = 4*sub + j
    int axis[4];
    double omega[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int pr = 4 * sub + j;
        int i, P;
        if (pr < p.pt) {
            axis[j] = 0; i = pr; P = p.pt;
        } else if (pr < p.pt + p.ph) {
            axis[j] = 1; i = pr - p.pt; P = p.ph;
        } else {
            axis[j] = 2; i = pr - p.pt - p.ph; P = p.pw;
        }
        omega[j] = pow(p.theta, -2.0 * static_cast<double>(i) / (2.0 * static_cast<double>(P)));
    }
    float w0[8], w1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        w0[i] = w_at(p.w0, p.w_dtype, 8 * sub + i);
        w1[i] = p.t1 ? w_at(p.w1, p.w_dtype, 8 * sub + i) : 0.0f;
    }
    const float inv_hd = 1.0f / static_cast<float>(HD);
    const int nvl = (p.nvr + 31) / 32;      // vectors per lane per tensor row
    const int lanes_total = (p.t1 ? 2 : 1) * nvl;
    const double kTwoPi = 6.283185307179586;
    const double kInvTwoPi = 0.15915494309189535;

    const int64_t wstep = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t tok = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
         tok < p.rows; tok += wstep) {
        int pos3[3];
        if (p.pos) {
            pos3[0] = p.pos[3 * tok + 0];
            pos3[1] = p.pos[3 * tok + 1];
            pos3[2] = p.pos[3 * tok + 2];
        } else {
            const int64_t g = p.pos_offset + tok % p.N;
            const int64_t hw = static_cast<int64_t>(p.Hg) * p.Wg;
            const int64_t t = g / hw;
            const int64_t rem = g - t * hw;
            const int64_t h = rem / p.Wg;
            pos3[0] = static_cast<int>(t);
            pos3[1] = static_cast<int>(h);
            pos3[2] = static_cast<int>(rem - h * p.Wg);
        }
        float cs[4], sn[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int pa = axis[j] == 0 ? pos3[0] : (axis[j] == 1 ? pos3[1] : pos3[2]);
            const double phi = static_cast<double>(pa) * omega[j];
            const double k = rint(phi * kInvTwoPi);
            const float red = static_cast<float>(fma(-k, kTwoPi, phi));
            sincosf(red, &sn[j], &cs[j]);
        }

        for (int c0 = 0; c0 < lanes_total; c0 += kChunk) {
            uint4 v[kChunk];
            uint4* addr[kChunk];
            bool act[kChunk];
#pragma unroll
            for (int u = 0; u < kChunk; ++u) {
                const int jl = c0 + u;
                const int tsel = jl >= nvl ? 1 : 0;
                const int idx = (jl - tsel * nvl) * 32 + lane;
                act[u] = jl < lanes_total && idx < p.nvr;
                addr[u] = (tsel ? p.t1 : p.t0) + tok * p.stride_v + idx;
                v[u] = act[u] ? ld_inplace(addr[u]) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kChunk; ++u) {
                const bool second = (c0 + u) >= nvl;
                float f[8];
                unpack8(v[u], f);
                float ss = 0.0f;
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = __fmaf_rn(f[i], f[i], ss);
#pragma unroll
                for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float inv = rsqrtf(__fmaf_rn(ss, inv_hd, p.eps));
                float o8[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float u0 = f[2 * j] * inv * (second ? w1[2 * j] : w0[2 * j]);
                    const float u1 = f[2 * j + 1] * inv * (second ? w1[2 * j + 1] : w0[2 * j + 1]);
                    o8[2 * j] = __fmaf_rn(u0, cs[j], -u1 * sn[j]);
                    o8[2 * j + 1] = __fmaf_rn(u0, sn[j], u1 * cs[j]);
                }
                if (act[u]) st_stream(addr[u], pack8(o8));
            }
        }
    }
}

using QKKernel = void (*)(QKParams);

QKKernel pick(int hd) {
    switch (hd) {
        case 32: return qk_rmsnorm_rope3d_kernel<32>;
        case 64: return qk_rmsnorm_rope3d_kernel<64>;
        case 128: return qk_rmsnorm_rope3d_kernel<128>;
        case 256: return qk_rmsnorm_rope3d_kernel<256>;
        default: return nullptr;
    }
}

int check_w(const void* p, int dtype) {
    if (!p) return DIT_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(p) % (dtype == DIT_F32 ? 4 : 2)) return DIT_ERR_ALIGN;
    return DIT_OK;
}

}  // namespace
}  // namespace dit

extern "C" int dit_qk_rmsnorm_rope3d(uint16_t* q, uint16_t* k, int64_t row_stride,
                                     const void* w_q, const void* w_k, int w_dtype, int B,
                                     int64_t N, int H, int hd, int T, int Hg, int Wg,
                                     const int32_t* pos, int64_t pos_offset, int pairs_t,
                                     int pairs_h, int pairs_w, double theta, double eps,
                                     void* stream) {
    using namespace dit;
    if (!q && !k) return DIT_ERR_NULL;
    if (w_dtype != DIT_F32 && w_dtype != DIT_BF16) return DIT_ERR_DTYPE;
    int st;
    if (q && (st = check_w(w_q, w_dtype))) return st;
    if (k && (st = check_w(w_k, w_dtype))) return st;
    if (B < 0 || N < 0 || H < 1) return DIT_ERR_SHAPE;
    QKKernel kernel = pick(hd);
    if (!kernel) return DIT_ERR_SHAPE;
    if (pairs_t < 1 || pairs_h < 1 || pairs_w < 1 || pairs_t + pairs_h + pairs_w != hd / 2)
        return DIT_ERR_SHAPE;
    const int64_t width = static_cast<int64_t>(H) * hd;
    if (width > (int64_t(1) << 30) || row_stride < width) return DIT_ERR_SHAPE;
    if (row_stride % 8) return DIT_ERR_ALIGN;
    if ((q && !aligned16(q)) || (k && !aligned16(k))) return DIT_ERR_ALIGN;
    if (!(theta > 0.0) || theta > 1e300 || !(eps >= 0.0) || eps > 1e30) return DIT_ERR_VALUE;
    const int64_t rows = static_cast<int64_t>(B) * N;
    if (B > 0 && N > (INT64_MAX / 4) / row_stride / B) return DIT_ERR_SHAPE;
    if (!pos) {
        if (T < 1 || Hg < 1 || Wg < 1 || pos_offset < 0) return DIT_ERR_SHAPE;
        const int64_t cells = static_cast<int64_t>(T) * Hg * Wg;
        if (cells > INT32_MAX || pos_offset + N > cells) return DIT_ERR_SHAPE;
    } else if (reinterpret_cast<uintptr_t>(pos) % 4) {
        return DIT_ERR_ALIGN;
    }
    if (q && k) {
        // q and k rows share the stride; they must not overlap in any row
        const int64_t d = (reinterpret_cast<intptr_t>(k) - reinterpret_cast<intptr_t>(q)) / 2;
        int64_t m = d % row_stride;
        if (m < 0) m += row_stride;
        if (m < width || row_stride - m < width) return DIT_ERR_OVERLAP;
    }
    if (rows == 0) return DIT_OK;

    QKParams p{};
    p.t0 = reinterpret_cast<uint4*>(q ? q : k);
    p.t1 = q ? reinterpret_cast<uint4*>(k) : nullptr;
    p.w0 = q ? w_q : w_k;
    p.w1 = q ? w_k : nullptr;
    p.w_dtype = w_dtype;
    p.stride_v = row_stride / 8;
    p.rows = rows;
    p.N = N;
    p.nvr = static_cast<int>(width / 8);
    p.Hg = Hg;
    p.Wg = Wg;
    p.pos = pos;
    p.pos_offset = pos_offset;
    p.pt = pairs_t;
    p.ph = pairs_h;
    p.pw = pairs_w;
    p.theta = theta;
    p.eps = static_cast<float>(eps);

    const int sms = device_sm_count();
    if (sms <= 0) return DIT_ERR_LAUNCH;
    const int occ = occupancy(reinterpret_cast<const void*>(kernel), kThreads, 0);
    int64_t blocks = static_cast<int64_t>(sms) * occ;
    const int64_t need = (rows + kWarps - 1) / kWarps;
    if (blocks > need) blocks = need;
    kernel<<<static_cast<unsigned>(blocks), kThreads, 0, as_stream(stream)>>>(p);
    return launch_status();
}
