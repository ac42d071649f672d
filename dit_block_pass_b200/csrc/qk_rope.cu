// qk_rope.cu -- per-head QK RMSNorm fused with 3D (t, h, w) rotary position
// embedding, in place, in one pass over HBM.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração
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
// q and k stream through a per-warp, kStages-deep cp.async pipeline of
// kChunk lane-vectors per stage (each lane copies and later reads back only
// its own vectors, so no barrier is needed): the next chunks are in flight
// while the current one is normalised and rotated.  HBM bound.
#include "common.cuh"

namespace dit {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 10;   // lane-vectors per pipeline stage
constexpr int kStages = 2;   // cp.async stages per warp
constexpr size_t kSmem = static_cast<size_t>(kWarps) * kStages * kChunk * 32 * sizeof(uint4);

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

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}

// Work of one warp is a sequence of jobs: chunk c (0 .. cpt-1) of each of
// the warp's tokens in turn.  Chunks 0 .. cq-1 cover the q row and chunks
// cq .. 2cq-1 the k row, kChunk lane-vectors each (lane-vector i of a row is
// its vector i * 32 + lane), so the tensor, its weights and its row pointer
// are uniform inside a chunk.
template <int HD>
__global__ void __launch_bounds__(kThreads, 2)
qk_rmsnorm_rope3d_kernel(QKParams p) {
    constexpr int LPH = HD / 8;             // lanes per head
    extern __shared__ uint4 qk_stage[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane % LPH;             // this lane's vector within a head
    uint4* stage = qk_stage + warp * (kStages * kChunk * 32) + lane;

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
    const int nvl = (p.nvr + 31) / 32;              // lane-vectors per row
    const int cq = (nvl + kChunk - 1) / kChunk;     // chunks per row
    const int cpt = (p.t1 ? 2 : 1) * cq;            // chunks per token
    const int hw = p.Hg * p.Wg;
    const double kTwoPi = 6.283185307179586;
    const double kInvTwoPi = 0.15915494309189535;
    const int64_t wstep = static_cast<int64_t>(gridDim.x) * kWarps;

    // copy chunk `chunk` of token `tok` into stage slot `slot` (one commit group)
    auto issue = [&](int64_t tok, int chunk, int slot) {
        if (tok < p.rows) {
            const int tensor = chunk >= cq ? 1 : 0;
            const int first = (chunk - tensor * cq) * kChunk;
            const uint4* row = (tensor ? p.t1 : p.t0) + tok * p.stride_v;
            uint4* dst = stage + slot * (kChunk * 32);
#pragma unroll
            for (int u = 0; u < kChunk; ++u) {
                const int idx = (first + u) * 32 + lane;
                if (first + u < nvl && idx < p.nvr) cp_async16(dst + u * 32, row + idx);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    int64_t itok = static_cast<int64_t>(blockIdx.x) * kWarps + warp, ctok = itok;
    int ichunk = 0, cchunk = 0, islot = 0, cslot = 0;
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        issue(itok, ichunk, islot);
        if (++ichunk == cpt) { ichunk = 0; itok += wstep; }
        islot = islot + 1 == kStages ? 0 : islot + 1;
    }
    float cs[4], sn[4];
    while (ctok < p.rows) {
        issue(itok, ichunk, islot);
        if (++ichunk == cpt) { ichunk = 0; itok += wstep; }
        islot = islot + 1 == kStages ? 0 : islot + 1;
        // groups complete in order: all but the newest kStages-1 are done
        asm volatile("cp.async.wait_group %0;" ::"n"(kStages - 1) : "memory");
        if (cchunk == 0) {
            int pos3[3];
            if (p.pos) {
                pos3[0] = p.pos[3 * ctok + 0];
                pos3[1] = p.pos[3 * ctok + 1];
                pos3[2] = p.pos[3 * ctok + 2];
            } else {
                // grid index < 2^31 (checked on the host)
                const int g = static_cast<int>(p.pos_offset + ctok % p.N);
                const int t = g / hw;
                const int rem = g - t * hw;
                const int h = rem / p.Wg;
                pos3[0] = t;
                pos3[1] = h;
                pos3[2] = rem - h * p.Wg;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int pa = axis[j] == 0 ? pos3[0] : (axis[j] == 1 ? pos3[1] : pos3[2]);
                const double phi = static_cast<double>(pa) * omega[j];
                const double kk = rint(phi * kInvTwoPi);
                const float red = static_cast<float>(fma(-kk, kTwoPi, phi));
                sincosf(red, &sn[j], &cs[j]);
            }
        }
        const int tensor = cchunk >= cq ? 1 : 0;
        const int first = (cchunk - tensor * cq) * kChunk;
        uint4* row = (tensor ? p.t1 : p.t0) + ctok * p.stride_v;
        // rotation with the weight folded in: (u0, u1) = inv * (f0 w0, f1 w1)
        //   out0 = inv * (f0 * w0 cos - f1 * w1 sin), out1 = inv * (f0 * w0 sin + f1 * w1 cos)
        float A[4], Bn[4], C[4], Dd[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float wa = tensor ? w1[2 * j] : w0[2 * j];
            const float wb = tensor ? w1[2 * j + 1] : w0[2 * j + 1];
            A[j] = wa * cs[j];
            Bn[j] = -(wb * sn[j]);
            C[j] = wa * sn[j];
            Dd[j] = wb * cs[j];
        }
        const uint4* src = stage + cslot * (kChunk * 32);
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
            const int idx = (first + u) * 32 + lane;
            const bool valid = first + u < nvl && idx < p.nvr;
            float f[8];
            unpack8(valid ? src[u * 32] : make_uint4(0, 0, 0, 0), f);
            float ss = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) ss = __fmaf_rn(f[i], f[i], ss);
#pragma unroll
            for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float inv = rsqrtf(__fmaf_rn(ss, inv_hd, p.eps));
            float o8[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                o8[2 * j] = inv * __fmaf_rn(f[2 * j], A[j], f[2 * j + 1] * Bn[j]);
                o8[2 * j + 1] = inv * __fmaf_rn(f[2 * j], C[j], f[2 * j + 1] * Dd[j]);
            }
            if (valid) st_stream(row + idx, pack8(o8));
        }
        if (++cchunk == cpt) { cchunk = 0; ctok += wstep; }
        cslot = cslot + 1 == kStages ? 0 : cslot + 1;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
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

// Rows i of q ([q + i*rs, q + i*rs + w), elements) and rows j of k overlap
// for some 0 <= i, j < rows iff |d - m*rs| < w for an integer
// m = i - j in (-rows, rows), d = k - q; the distance is smallest for m next
// to d/rs, so the two integers around it (clamped to the range) decide.
bool rows_overlap(const void* q, const void* k, int64_t rows, int64_t rs, int64_t w) {
    const intptr_t bq = reinterpret_cast<intptr_t>(q), bk = reinterpret_cast<intptr_t>(k);
    const intptr_t db = bk - bq;
    if (db % 2) return true;  // not on the same element grid: be conservative
    const int64_t d = static_cast<int64_t>(db / 2);
    int64_t m0 = d >= 0 ? d / rs : -((-d + rs - 1) / rs);  // floor(d / rs)
    for (int64_t m = m0; m <= m0 + 1; ++m) {
        int64_t mc = m;
        if (mc > rows - 1) mc = rows - 1;
        if (mc < -(rows - 1)) mc = -(rows - 1);
        int64_t dist = d - mc * rs;
        if (dist < 0) dist = -dist;
        if (dist < w) return true;
    }
    return false;
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
    if (w_dtype != DIT_F32 && w_dtype != DIT_BF16) return DIT_ERR_DTYPE;
    if (B < 0 || N < 0 || H < 1) return DIT_ERR_SHAPE;
    QKKernel kernel = pick(hd);
    if (!kernel) return DIT_ERR_SHAPE;
    if (pairs_t < 1 || pairs_h < 1 || pairs_w < 1 || pairs_t + pairs_h + pairs_w != hd / 2)
        return DIT_ERR_SHAPE;
    const int64_t width = static_cast<int64_t>(H) * hd;
    if (width > (int64_t(1) << 30) || row_stride < width) return DIT_ERR_SHAPE;
    if (row_stride % 8) return DIT_ERR_ALIGN;
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
    if (rows == 0) return DIT_OK;
    if (!q && !k) return DIT_ERR_NULL;
    int st;
    if (q && (st = check_w(w_q, w_dtype))) return st;
    if (k && (st = check_w(w_k, w_dtype))) return st;
    if ((q && !aligned16(q)) || (k && !aligned16(k))) return DIT_ERR_ALIGN;
    if (q && k && rows_overlap(q, k, rows, row_stride, width)) return DIT_ERR_OVERLAP;

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
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    const int occ = occupancy(reinterpret_cast<const void*>(kernel), kThreads, kSmem);
    int64_t blocks = static_cast<int64_t>(sms) * occ;
    const int64_t need = (rows + kWarps - 1) / kWarps;
    if (blocks > need) blocks = need;
    kernel<<<static_cast<unsigned>(blocks), kThreads, kSmem, as_stream(stream)>>>(p);
    return launch_status();
}
