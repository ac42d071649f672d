// qk_rope.cu -- QK RMSNorm fused with 3D (t, h, w) rotary position
// embedding, in one pass over HBM.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração somadas chega-se a 6 vezes":
// "QK RMSNorm com 3D RoPE" is one fused operator; "SGLang acelera MiniMax-H3
// em GPUs H200", first paragraph, lists QK RMSNorm and 3D RoPE among the
// fused low-level operations.  The pages name the operator only: the pair
// layout and the width of the norm are options here (interleaved pairs and
// a per-head norm by default), and so is where the result goes (in place,
// or into separate q/k buffers with any head-major or token-major layout,
// e.g. the [B, H, N, hd] an attention kernel reads).
//
// Design: one warp per token, one-shot grid (a CTA takes one token per warp
// and exits; on B200 this sustained more HBM bandwidth than persistent
// CTAs).  A token row of H heads x hd is H*hd/8 consecutive 16-byte
// vectors; warp pass j reads vectors 32*j + lane, so each load instruction
// covers 512 contiguous bytes and a head occupies hd/8 adjacent lanes.
//
// The q row is loaded into registers while the k row is copied into the
// warp's shared-memory stage with cp.async, so both are in flight before any
// arithmetic.  Per-head norm: the head's sum of squares is a shuffle
// reduction inside its lane group, and the RMSNorm weight is folded into
// per-lane rotation coefficients once per token and tensor.  Whole-row norm:
// the row's sum of squares is a warp reduction over every vector the lane
// holds; rows up to 5,120 wide take a persistent kernel that stages the
// per-element weights in shared memory once per CTA and streams each warp's
// rows through one stage, wider rows the one-shot kernel with the weights
// read through L1.
//
// Rotation: a lane always holds the same rotation pairs of a head (4 pairs
// inside its vector when pairs are interleaved; 8 pairs (p, p + hd/2) when
// they are rotate-half, the partner elements fetched from the lane hd/16 away
// with a shuffle, or, for the whole-row norm, held by the lane itself in a
// paired layout), so it computes their angles once per token and reuses them
// for every head of q and k.  The hd/2
// frequencies are computed in fp64 once per CTA into shared memory while the
// rows load; the angles pos*omega are formed and reduced modulo 2*pi in
// fp64, and sin/cos are taken in fp32 on the reduced angle, which keeps the
// rotation accurate to a few fp32 ulp for positions in the hundreds.  HBM
// bound.
#include "tcgen05.cuh"

namespace dit {
namespace {

constexpr int kWarps = 8;                    // tokens per CTA
constexpr int kThreads = kWarps * 32;

struct QKParams {
    const uint4* t0;        // first tensor processed (q, or k when q is NULL)
    const uint4* t1;        // second tensor or NULL
    uint4* o0;              // where t0's result goes (t0 itself when in place)
    uint4* o1;
    const void* w0;
    const void* w1;
    int w_dtype;
    int64_t stride_v;       // input row stride in 16-byte vectors
    int64_t osb, osn, osh;  // output strides of sample, token, head (vectors)
    bool o_rows;            // output token rows are evenly spaced: osb == N * osn
    int64_t rows;           // B * N
    int64_t N;
    bool rows32;            // B * N < 2^31: token indices fit 32 bits
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

// Eight weights of elements e .. e+7 (fp32 when WF32, else bf16; 16-byte
// aligned rows).  The dtype is a template argument so that an unrolled loop
// of these loads has no branch between them.
template <bool WF32>
__device__ __forceinline__ void w8_of(const void* w, int e, float (&f)[8]) {
    if (WF32) {
        const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(w) + e);
        const float4 a = __ldg(q), b = __ldg(q + 1);
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
        unpack8(__ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(w) + e)), f);
    }
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}

// First vector of token tok's output row: sample b = tok / N, token n.
__device__ __forceinline__ uint4* out_row(uint4* o, const QKParams& p, int64_t tok) {
    if (p.o_rows) return o + tok * p.osn;
    const int64_t b = tok / p.N;
    return o + b * p.osb + (tok - b * p.N) * p.osn;
}

// Output address of row vector idx: head idx / (hd/8), vector idx mod hd/8.
// CONTIG: the heads of a token row are adjacent (in place, or a token-major
// output), so the address is the row's plus idx.
template <int HD, bool CONTIG>
__device__ __forceinline__ uint4* out_vec(uint4* orow, int64_t osh, int idx) {
    constexpr int LPH = HD / 8;
    if (CONTIG) return orow + idx;
    return orow + (idx / LPH) * osh + (idx % LPH);
}

// Pair pr of an axis with P pairs, local index i: omega = theta^(-2i/(2P)).
// Computed once per CTA, while the rows are in flight.
template <int HD>
__device__ __forceinline__ void omega_table(const QKParams& p, double* s_omega) {
    for (int pr = threadIdx.x; pr < HD / 2; pr += blockDim.x) {
        int i, P;
        if (pr < p.pt) {
            i = pr; P = p.pt;
        } else if (pr < p.pt + p.ph) {
            i = pr - p.pt; P = p.ph;
        } else {
            i = pr - p.pt - p.ph; P = p.pw;
        }
        s_omega[pr] = pow(p.theta, -2.0 * static_cast<double>(i) / (2.0 * static_cast<double>(P)));
    }
}

// The token's (t, h, w) position and this lane's rotation angles:
// LAYOUT 0 pairs 4*sub + k (k < 4), LAYOUT 1 pairs 8*(sub mod hd/16) + k
// (k < 8), sub = the lane's vector within its head.
template <int HD, int LAYOUT>
__device__ __forceinline__ void token_angles(const QKParams& p, const double* s_omega,
                                             int64_t tok, int sub,
                                             float (&cs)[LAYOUT == 0 ? 4 : 8],
                                             float (&sn)[LAYOUT == 0 ? 4 : 8]) {
    constexpr int NP = LAYOUT == 0 ? 4 : 8;
    constexpr int LPH = HD / 8;
    int pos3[3];
    if (p.pos) {
        pos3[0] = p.pos[3 * tok + 0];
        pos3[1] = p.pos[3 * tok + 1];
        pos3[2] = p.pos[3 * tok + 2];
    } else {
        // grid index < 2^31 (checked on the host); a 32-bit modulo when the
        // token indices allow it (a 64-bit one costs several times more)
        const int hw = p.Hg * p.Wg;
        const int64_t n = p.rows32 ? static_cast<int64_t>(static_cast<uint32_t>(tok) %
                                                          static_cast<uint32_t>(p.N))
                                   : tok % p.N;
        const int g = static_cast<int>(p.pos_offset + n);
        const int t = g / hw;
        const int rem = g - t * hw;
        const int h = rem / p.Wg;
        pos3[0] = t;
        pos3[1] = h;
        pos3[2] = rem - h * p.Wg;
    }
    const double kTwoPi = 6.283185307179586;
    const double kInvTwoPi = 0.15915494309189535;
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int pr = LAYOUT == 0 ? 4 * sub + k : 8 * (sub % (LPH / 2)) + k;
        const int pa = pr < p.pt ? pos3[0] : (pr < p.pt + p.ph ? pos3[1] : pos3[2]);
        const double phi = static_cast<double>(pa) * s_omega[pr];
        const double kk = rint(phi * kInvTwoPi);
        sincosf(static_cast<float>(fma(-kk, kTwoPi, phi)), &sn[k], &cs[k]);
    }
}

// Per-head norm of one tensor row held as NVL lane-vectors v (vector
// j * 32 + lane of the row), rotated and stored.
//   LAYOUT 0: pairs (2p, 2p+1) inside a lane's vector.
//   LAYOUT 1: pairs (p, p + hd/2): a lane's 8 elements pair with the same
//             slots of lane ^ (hd/16), fetched with one shuffle of the
//             packed vector.
template <int HD, int NVL, int LAYOUT, bool CONTIG>
__device__ __forceinline__ void qk_head_tensor(const uint4 (&v)[NVL], uint4* orow, int64_t osh,
                                               int nvr, int lane, const void* w, int w_dtype,
                                               const float* cs, const float* sn, float eps) {
    constexpr int LPH = HD / 8;
    constexpr int HALF = LPH / 2;           // partner lane distance for rotate-half
    const int sub = lane % LPH;
    const bool first = (sub & HALF) == 0;   // rotate-half: lane holds the first half
    // per-lane coefficients with the weight folded in
    float A[8], Bc[8], C[4], Dd[4];
    if (LAYOUT == 0) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float wa = w_at(w, w_dtype, 8 * sub + 2 * k);
            const float wb = w_at(w, w_dtype, 8 * sub + 2 * k + 1);
            A[k] = wa * cs[k]; Bc[k] = -(wb * sn[k]); C[k] = wa * sn[k]; Dd[k] = wb * cs[k];
        }
    } else {
        // out_e = inv * (f_e w_e cos -/+ f_partner w_partner sin)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float wo = w_at(w, w_dtype, 8 * sub + i);
            const float wp = w_at(w, w_dtype, 8 * (sub ^ HALF) + i);
            A[i] = wo * cs[i];
            Bc[i] = (first ? -wp : wp) * sn[i];
        }
    }
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        const int idx = j * 32 + lane;
        float f[8];
        unpack8(v[j], f);
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = __fmaf_rn(f[i], f[i], ss);
#pragma unroll
        for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = rsqrtf(__fmaf_rn(ss, 1.0f / static_cast<float>(HD), eps));
        float o8[8];
        if (LAYOUT == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                o8[2 * k] = inv * __fmaf_rn(f[2 * k], A[k], f[2 * k + 1] * Bc[k]);
                o8[2 * k + 1] = inv * __fmaf_rn(f[2 * k], C[k], f[2 * k + 1] * Dd[k]);
            }
        } else {
            uint4 pv;
            pv.x = __shfl_xor_sync(0xffffffffu, v[j].x, HALF);
            pv.y = __shfl_xor_sync(0xffffffffu, v[j].y, HALF);
            pv.z = __shfl_xor_sync(0xffffffffu, v[j].z, HALF);
            pv.w = __shfl_xor_sync(0xffffffffu, v[j].w, HALF);
            float fp[8];
            unpack8(pv, fp);
#pragma unroll
            for (int i = 0; i < 8; ++i) o8[i] = inv * __fmaf_rn(f[i], A[i], fp[i] * Bc[i]);
        }
        if (idx < nvr) st_stream(out_vec<HD, CONTIG>(orow, osh, idx), pack8(o8));
    }
}

// Whole-row norm of one tensor row held as NVL lane-vectors v: the row's
// sum of squares first (a warp reduction), then the weighted, rotated
// values.  The weight has one entry per element of the row.
template <int HD, int NVL, int LAYOUT, bool WF32>
__device__ __forceinline__ void qk_row_tensor(uint4 (&v)[NVL], uint4* orow, int64_t osh, int nvr,
                                              int lane, const void* w, const float* cs,
                                              const float* sn, float eps) {
    constexpr int LPH = HD / 8;
    constexpr int HALF = LPH / 2;
    const bool first = ((lane % LPH) & HALF) == 0;
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        float f[8];
        unpack8(v[j], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = __fmaf_rn(f[i], f[i], ss);
    }
    ss = warp_sum(ss);
    const float inv = rsqrtf(__fmaf_rn(ss, 1.0f / static_cast<float>(nvr * 8), eps));
    // unpack again below rather than keep every unpacked float alive across
    // the reduction (the packed row needs half the registers)
#pragma unroll
    for (int j = 0; j < NVL; ++j)
        asm volatile("" : "+r"(v[j].x), "+r"(v[j].y), "+r"(v[j].z), "+r"(v[j].w));
    // the weights of vector j + PD are requested before vector j is stored
    // (a store is a compiler barrier for loads), so the weight loads run PD
    // vectors ahead of their use
    constexpr int PD = NVL < 2 ? NVL : 2;
    float wr[PD][8];
#pragma unroll
    for (int d = 0; d < PD; ++d) {
        const int idx = d * 32 + lane;
        w8_of<WF32>(w, (idx < nvr ? idx : 0) * 8, wr[d]);
    }
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        const int idx = j * 32 + lane;
        float f[8], wv[8], o8[8];
        unpack8(v[j], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) wv[i] = wr[j % PD][i];
        if (j + PD < NVL) {
            const int nidx = (j + PD) * 32 + lane;
            w8_of<WF32>(w, (nidx < nvr ? nidx : 0) * 8, wr[j % PD]);
        }
        if (LAYOUT == 0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float u0 = f[2 * k] * inv * wv[2 * k];
                const float u1 = f[2 * k + 1] * inv * wv[2 * k + 1];
                o8[2 * k] = __fmaf_rn(u0, cs[k], -u1 * sn[k]);
                o8[2 * k + 1] = __fmaf_rn(u0, sn[k], u1 * cs[k]);
            }
        } else {
            // weight each element on its own lane, then swap the weighted
            // values with the partner lane
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float u = f[i] * inv * wv[i];
                const float up = __shfl_xor_sync(0xffffffffu, u, HALF);
                o8[i] = __fmaf_rn(u, cs[i], (first ? -up : up) * sn[i]);
            }
        }
        if (idx < nvr) st_stream(out_vec<HD, false>(orow, osh, idx), pack8(o8));
    }
}

// Rotate-half pairs with the whole-row norm: a lane holds both members of
// its pairs.  Lane-vector j of a lane is row vector paired_idx(j, lane):
// each 64-vector span of the row holds 64 / (hd/8) whole heads, lane group
// g = lane / (hd/16) takes head g of the span, and the lane takes vector
// lane mod (hd/16) of that head's first half (j even) and the same vector
// of its second half (j odd).  The hd/16 lanes of a group read consecutive
// vectors, so every load and store still covers whole 32-byte sectors.
template <int HD>
__device__ __forceinline__ int paired_idx(int j, int lane) {
    constexpr int LPH = HD / 8, HALF = LPH / 2;
    return (j >> 1) * 64 + (lane / HALF) * LPH + (j & 1) * HALF + lane % HALF;
}

// Whole-row norm and rotate-half rotation of a row held in the paired
// layout (NVL even): the same arithmetic per element as qk_row_tensor,
// with each pair's partner in the lane's own registers.
template <int HD, int NVL, bool WF32>
__device__ __forceinline__ void qk_row_tensor_paired(uint4 (&v)[NVL], uint4* orow, int64_t osh,
                                                     int nvr, int lane, const void* w,
                                                     const float* cs, const float* sn,
                                                     float eps) {
    static_assert(NVL % 2 == 0, "paired rows hold whole pairs");
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        float f[8];
        unpack8(v[j], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = __fmaf_rn(f[i], f[i], ss);
    }
    ss = warp_sum(ss);
    const float inv = rsqrtf(__fmaf_rn(ss, 1.0f / static_cast<float>(nvr * 8), eps));
#pragma unroll
    for (int j = 0; j < NVL; ++j)
        asm volatile("" : "+r"(v[j].x), "+r"(v[j].y), "+r"(v[j].z), "+r"(v[j].w));
    // the pair's weights are loaded as it is processed: loading them a pair
    // ahead spills at 128 registers and measured slower
#pragma unroll
    for (int j = 0; j < NVL; j += 2) {
        const int i0 = paired_idx<HD>(j, lane), i1 = paired_idx<HD>(j + 1, lane);
        const bool ok = i0 < nvr;
        float wa[8], wb[8], u0[8], u1[8], o0[8], o1[8];
        w8_of<WF32>(w, (ok ? i0 : 0) * 8, wa);
        w8_of<WF32>(w, (ok ? i1 : 0) * 8, wb);
        unpack8(v[j], u0);
        unpack8(v[j + 1], u1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            u0[i] = u0[i] * inv * wa[i];
            u1[i] = u1[i] * inv * wb[i];
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            o0[i] = __fmaf_rn(u0[i], cs[i], -u1[i] * sn[i]);
            o1[i] = __fmaf_rn(u1[i], cs[i], u0[i] * sn[i]);
        }
        if (ok) {
            st_stream(out_vec<HD, false>(orow, osh, i0), pack8(o0));
            st_stream(out_vec<HD, false>(orow, osh, i1), pack8(o1));
        }
    }
}

// MODE 0: per-head norm, heads adjacent in the output; 1: per-head norm,
// strided heads (e.g. a head-major output); 2: whole-row norm (with
// rotate-half pairs in the paired layout, NVL being even there).
template <int HD, int NVL, int LAYOUT, int MODE>
__global__ void __launch_bounds__(kThreads, (NVL <= 20 ? 2 : 1))
qk_rmsnorm_rope3d_kernel(QKParams p) {
    constexpr int LPH = HD / 8;             // lanes per head
    constexpr int NP = LAYOUT == 0 ? 4 : 8; // rotation pairs per lane
    constexpr bool PAIRED = LAYOUT == 1 && MODE == 2 && NVL % 2 == 0;
    extern __shared__ uint4 qk_stage[];
    __shared__ double s_omega[HD / 2];      // frequency of each rotation pair
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t tok = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
    const bool live = tok < p.rows;
    const uint4* row0 = p.t0 + tok * p.stride_v;
    const uint4* row1 = p.t1 ? p.t1 + tok * p.stride_v : nullptr;
    uint4* stage = qk_stage + warp * (NVL * 32) + lane;
    uint4 v[NVL];
    if (live) {
        if (row1) {
#pragma unroll
            for (int j = 0; j < NVL; ++j) {
                const int idx = PAIRED ? paired_idx<HD>(j, lane) : j * 32 + lane;
                if (idx < p.nvr) cp_async16(stage + j * 32, row1 + idx);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
#pragma unroll
        for (int j = 0; j < NVL; ++j) {
            const int idx = PAIRED ? paired_idx<HD>(j, lane) : j * 32 + lane;
            v[j] = idx < p.nvr ? ld_inplace(row0 + idx) : make_uint4(0, 0, 0, 0);
        }
    }
    omega_table<HD>(p, s_omega);
    __syncthreads();
    if (!live) return;

    float cs[NP], sn[NP];
    token_angles<HD, LAYOUT>(p, s_omega, tok, lane % LPH, cs, sn);
    if constexpr (PAIRED) {
        if (p.w_dtype == DIT_F32)
            qk_row_tensor_paired<HD, NVL, true>(v, out_row(p.o0, p, tok), p.osh, p.nvr, lane,
                                                p.w0, cs, sn, p.eps);
        else
            qk_row_tensor_paired<HD, NVL, false>(v, out_row(p.o0, p, tok), p.osh, p.nvr, lane,
                                                 p.w0, cs, sn, p.eps);
    } else if (MODE == 2) {
        if (p.w_dtype == DIT_F32)
            qk_row_tensor<HD, NVL, LAYOUT, true>(v, out_row(p.o0, p, tok), p.osh, p.nvr, lane,
                                                 p.w0, cs, sn, p.eps);
        else
            qk_row_tensor<HD, NVL, LAYOUT, false>(v, out_row(p.o0, p, tok), p.osh, p.nvr, lane,
                                                  p.w0, cs, sn, p.eps);
    } else
        qk_head_tensor<HD, NVL, LAYOUT, MODE == 0>(v, out_row(p.o0, p, tok), p.osh, p.nvr, lane,
                                                   p.w0, p.w_dtype, cs, sn, p.eps);
    if (row1) {
        // each lane reads back only the vectors it copied itself
        asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
        for (int j = 0; j < NVL; ++j) {
            const int idx = PAIRED ? paired_idx<HD>(j, lane) : j * 32 + lane;
            v[j] = idx < p.nvr ? stage[j * 32] : make_uint4(0, 0, 0, 0);
        }
        if constexpr (PAIRED) {
            if (p.w_dtype == DIT_F32)
                qk_row_tensor_paired<HD, NVL, true>(v, out_row(p.o1, p, tok), p.osh, p.nvr,
                                                    lane, p.w1, cs, sn, p.eps);
            else
                qk_row_tensor_paired<HD, NVL, false>(v, out_row(p.o1, p, tok), p.osh, p.nvr,
                                                     lane, p.w1, cs, sn, p.eps);
        } else if (MODE == 2) {
            if (p.w_dtype == DIT_F32)
                qk_row_tensor<HD, NVL, LAYOUT, true>(v, out_row(p.o1, p, tok), p.osh, p.nvr,
                                                     lane, p.w1, cs, sn, p.eps);
            else
                qk_row_tensor<HD, NVL, LAYOUT, false>(v, out_row(p.o1, p, tok), p.osh, p.nvr,
                                                      lane, p.w1, cs, sn, p.eps);
        } else
            qk_head_tensor<HD, NVL, LAYOUT, MODE == 0>(v, out_row(p.o1, p, tok), p.osh, p.nvr,
                                                       lane, p.w1, p.w_dtype, cs, sn, p.eps);
    }
}

// ---------------------------------------------------------------------------
// Whole-row norm, persistent (rows of up to 20 lane-vectors, H*hd <= 5120):
// one CTA of kRowWarps warps per SM.  The per-element weights of q and k are
// staged once per CTA in shared memory (fp32, lo/hi float4 halves, so a warp
// reads them without bank conflicts) instead of passing through L1 for every
// token, and each warp streams its rows (q then k of each of its tokens)
// through one shared-memory stage: as soon as a row's values are in
// registers and summed, the next row's copy is issued into the stage, so
// one row per warp is always in flight.  The arithmetic per element is the
// one-shot whole-row kernel's (same lane-vectors, same order of the sums).
constexpr int kRowWarps = 16;
constexpr int kRowMaxNVL = 20;

template <int HD, int NVL, int LAYOUT>
__device__ __forceinline__ void row_copy(const uint4* row, uint4* stage, int nvr, int lane) {
#pragma unroll
    for (int j = 0; j < NVL; ++j) {
        const int idx = LAYOUT == 1 ? paired_idx<HD>(j, lane) : j * 32 + lane;
        if (idx < nvr) cp_async16(stage + j * 32, row + idx);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Weighted rotation and store of a row normalised by inv, the weights read
// from the shared-memory copy s_w (s_w[idx]: elements 8 idx .. 8 idx + 3,
// s_w[nvr + idx]: the next four).
template <int HD, int NVL, int LAYOUT>
__device__ __forceinline__ void qk_row_rotate_smem(const uint4 (&v)[NVL], uint4* orow, int64_t osh,
                                                   int nvr, int lane, const float4* s_w,
                                                   float inv, const float* cs, const float* sn) {
    if constexpr (LAYOUT == 0) {
#pragma unroll
        for (int j = 0; j < NVL; ++j) {
            const int idx = j * 32 + lane;
            if (idx < nvr) {
                float f[8], o8[8];
                unpack8(v[j], f);
                const float4 a = s_w[idx], b = s_w[nvr + idx];
                const float wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float u0 = f[2 * k] * inv * wv[2 * k];
                    const float u1 = f[2 * k + 1] * inv * wv[2 * k + 1];
                    o8[2 * k] = __fmaf_rn(u0, cs[k], -u1 * sn[k]);
                    o8[2 * k + 1] = __fmaf_rn(u0, sn[k], u1 * cs[k]);
                }
                st_stream(out_vec<HD, false>(orow, osh, idx), pack8(o8));
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < NVL; j += 2) {
            const int i0 = paired_idx<HD>(j, lane), i1 = paired_idx<HD>(j + 1, lane);
            if (i0 < nvr) {
                float u0[8], u1[8], o0[8], o1[8];
                unpack8(v[j], u0);
                unpack8(v[j + 1], u1);
                const float4 a0 = s_w[i0], b0 = s_w[nvr + i0];
                const float4 a1 = s_w[i1], b1 = s_w[nvr + i1];
                const float wa[8] = {a0.x, a0.y, a0.z, a0.w, b0.x, b0.y, b0.z, b0.w};
                const float wb[8] = {a1.x, a1.y, a1.z, a1.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    u0[i] = u0[i] * inv * wa[i];
                    u1[i] = u1[i] * inv * wb[i];
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    o0[i] = __fmaf_rn(u0[i], cs[i], -u1[i] * sn[i]);
                    o1[i] = __fmaf_rn(u1[i], cs[i], u0[i] * sn[i]);
                }
                st_stream(out_vec<HD, false>(orow, osh, i0), pack8(o0));
                st_stream(out_vec<HD, false>(orow, osh, i1), pack8(o1));
            }
        }
    }
}

template <int HD, int NVL, int LAYOUT>
__global__ void __launch_bounds__(kRowWarps * 32, 1)
qk_row_persistent_kernel(QKParams p) {
    static_assert(LAYOUT == 0 || NVL % 2 == 0, "paired rows hold whole pairs");
    constexpr int LPH = HD / 8;
    constexpr int NP = LAYOUT == 0 ? 4 : 8;
    extern __shared__ float4 qk_rows_smem[];
    __shared__ double s_omega[HD / 2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvr = p.nvr;
    const int ntens = p.t1 ? 2 : 1;
    uint4* stage = reinterpret_cast<uint4*>(qk_rows_smem + 2 * nvr * ntens) + warp * (NVL * 32) + lane;
    const int64_t tstep = static_cast<int64_t>(gridDim.x) * kRowWarps;
    int64_t tok = static_cast<int64_t>(blockIdx.x) * kRowWarps + warp;
    if (tok < p.rows) row_copy<HD, NVL, LAYOUT>(p.t0 + tok * p.stride_v, stage, nvr, lane);
    // the weights, while the first rows travel
    for (int t = 0; t < ntens; ++t) {
        const void* w = t ? p.w1 : p.w0;
        float4* sw = qk_rows_smem + 2 * nvr * t;
        for (int v = threadIdx.x; v < nvr; v += blockDim.x) {
            float f[8];
            if (p.w_dtype == DIT_F32)
                w8_of<true>(w, 8 * v, f);
            else
                w8_of<false>(w, 8 * v, f);
            sw[v] = make_float4(f[0], f[1], f[2], f[3]);
            sw[nvr + v] = make_float4(f[4], f[5], f[6], f[7]);
        }
    }
    omega_table<HD>(p, s_omega);
    __syncthreads();
    for (; tok < p.rows; tok += tstep) {
        float cs[NP], sn[NP];
        token_angles<HD, LAYOUT>(p, s_omega, tok, lane % LPH, cs, sn);
        for (int t = 0; t < ntens; ++t) {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            uint4 v[NVL];
            float ss = 0.0f;
#pragma unroll
            for (int j = 0; j < NVL; ++j) {
                const int idx = LAYOUT == 1 ? paired_idx<HD>(j, lane) : j * 32 + lane;
                v[j] = idx < nvr ? stage[j * 32] : make_uint4(0, 0, 0, 0);
                float f[8];
                unpack8(v[j], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = __fmaf_rn(f[i], f[i], ss);
            }
            ss = warp_sum(ss);
            const float inv = rsqrtf(__fmaf_rn(ss, 1.0f / static_cast<float>(nvr * 8), p.eps));
            // every lane's stage values are in the sum: the next row's copy
            const bool same = t + 1 < ntens;
            const int64_t ntok = same ? tok : tok + tstep;
            if (ntok < p.rows)
                row_copy<HD, NVL, LAYOUT>((same ? p.t1 : p.t0) + ntok * p.stride_v, stage, nvr,
                                          lane);
#pragma unroll
            for (int j = 0; j < NVL; ++j)
                asm volatile("" : "+r"(v[j].x), "+r"(v[j].y), "+r"(v[j].z), "+r"(v[j].w));
            qk_row_rotate_smem<HD, NVL, LAYOUT>(v, out_row(t ? p.o1 : p.o0, p, tok), p.osh, nvr,
                                                lane, qk_rows_smem + 2 * nvr * t, inv, cs, sn);
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// QK RMSNorm + 3D RoPE in place that also writes the mean of each block of
// `block` consecutive tokens of the rotated q and k (the SubBlock router's
// block summaries), so the router does not read q and k again.
//
// Work split: CTA (g, j, b) takes head group g (32*V row vectors: V vectors
// per lane, whole heads since hd/8 divides 32) of token block j of sample b;
// its 4 warps take consecutive quarters of the block's tokens.  The group's
// slice of a token row is contiguous, so one lane of each warp brings a
// token's q and k slices into a private ring of kPoolStages stages with two
// bulk copies (completion counted on the stage's mbarrier); the warp then
// normalises and rotates the token from shared memory, stores it in place,
// and adds the bf16-rounded results to fp32 sums in token order.  The four
// warps' sums are added in warp order and divided by the block's token count
// once: the summation order is fixed, so the means repeat bit for bit.
//
// Angles: a lane always holds the same rotation pairs.  When a token sits one
// step further along w than the warp's previous token (same t and h), the
// w-axis pairs advance by one rotation by their frequency (t and h pairs
// stay); otherwise, and at least every kRecur tokens, every angle is formed
// afresh (fp64 reduction, fp32 sin/cos).  The recurrence adds at most a few
// fp32 ulp per step, far below a bf16 ulp of the result.
constexpr int kPoolWarps = 4;
constexpr int kPoolStages = 6;
constexpr int kPoolV = 2;            // vectors per lane per tensor
constexpr int kRecur = 128;          // longest run of recurrence steps

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The token's (t, h, w) position (grid index or explicit table).
__device__ __forceinline__ void token_pos(const QKParams& p, int64_t tok, int& t, int& h,
                                          int& w) {
    if (p.pos) {
        t = p.pos[3 * tok + 0];
        h = p.pos[3 * tok + 1];
        w = p.pos[3 * tok + 2];
    } else {
        const int hw = p.Hg * p.Wg;
        const int g = static_cast<int>(p.pos_offset + tok % p.N);
        t = g / hw;
        const int rem = g - t * hw;
        h = rem / p.Wg;
        w = rem - h * p.Wg;
    }
}

template <int HD, int LAYOUT, int V>
__global__ void __launch_bounds__(kPoolWarps * 32, 4)
qk_rope_pool_kernel(QKParams p, int block, int nb, float* __restrict__ means, int* status,
                    int stall) {
    constexpr int LPH = HD / 8;             // lanes per head
    constexpr int HALF = LPH / 2;
    constexpr int NP = LAYOUT == 0 ? 4 : 8; // rotation pairs per lane
    constexpr int SV = 2 * V;               // vectors per lane per token: q, then k
    constexpr uint32_t kStage = SV * 32 * 16;
    extern __shared__ __align__(128) uint8_t pool_smem[];
    __shared__ double s_omega[HD / 2];
    __shared__ __align__(16) float s_w[2][HD];
    __shared__ int s_abort;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
    const int vbase = g * 32 * V;
    const int v0 = vbase + lane;            // this lane's first row vector
    const int nvec = p.nvr - vbase < 32 * V ? p.nvr - vbase : 32 * V;
    const uint32_t chunk = static_cast<uint32_t>(nvec) * 16;   // bytes per tensor and token
    const int sub = lane % LPH;
    const bool first = (sub & HALF) == 0;
    bool valid[V];
#pragma unroll
    for (int u = 0; u < V; ++u) valid[u] = 32 * u + lane < nvec;
    const int64_t n0 = static_cast<int64_t>(j) * block;
    const int count = static_cast<int>((n0 + block < p.N ? n0 + block : p.N) - n0);
    const int per = (block + kPoolWarps - 1) / kPoolWarps;
    const int lo = warp * per < count ? warp * per : count;
    const int hi = lo + per < count ? lo + per : count;
    const int64_t row0 = static_cast<int64_t>(b) * p.N + n0;   // global row of token 0
    const uint32_t ring = tc::smem_u32(pool_smem) + warp * kPoolStages * kStage;
    const uint32_t bars = tc::smem_u32(pool_smem) + kPoolWarps * kPoolStages * kStage +
                          warp * kPoolStages * 8;

    if (threadIdx.x == 0) s_abort = 0;
    if (lane == 0) {
        for (int s = 0; s < kPoolStages; ++s) tc::mbar_init(bars + 8 * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    // token t's q and k slices into stage s (lane 0)
    auto issue = [&](int t, int s) {
        if (lane == 0 && t < hi && !stall) {       // stall: a test hook, no copy goes out
            const int64_t row = row0 + t;
            tc::mbar_expect_tx(bars + 8 * s, 2 * chunk);
            bulk_g2s(ring + s * kStage, p.t0 + row * p.stride_v + vbase, chunk, bars + 8 * s);
            bulk_g2s(ring + s * kStage + V * 32 * 16, p.t1 + row * p.stride_v + vbase, chunk,
                     bars + 8 * s);
        }
    };
#pragma unroll
    for (int s = 0; s < kPoolStages; ++s) issue(lo + s, s);

    omega_table<HD>(p, s_omega);
    for (int e = threadIdx.x; e < 2 * HD; e += blockDim.x)
        s_w[e / HD][e % HD] = w_at(e < HD ? p.w0 : p.w1, p.w_dtype, e % HD);
    __syncthreads();

    // interleaved pairs: this lane's 8 weights of q and of k stay in registers
    float wl[2][8];
#pragma unroll
    for (int ten = 0; ten < 2; ++ten)
#pragma unroll
        for (int i = 0; i < 8; ++i) wl[ten][i] = LAYOUT == 0 ? s_w[ten][8 * sub + i] : 0.0f;
    // this lane's pairs: index, and the per-token step of w-axis pairs
    float stc[NP], sts[NP], cs[NP], sn[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const int pr = LAYOUT == 0 ? 4 * sub + k : 8 * (sub % HALF) + k;
        if (pr >= p.pt + p.ph) {
            double sd, cd;
            sincos(s_omega[pr], &sd, &cd);
            stc[k] = static_cast<float>(cd);
            sts[k] = static_cast<float>(sd);
        } else {
            stc[k] = 1.0f;
            sts[k] = 0.0f;
        }
        cs[k] = 1.0f;
        sn[k] = 0.0f;
    }
    int pt_ = -1, ph_ = -1, pw_ = -1, run = kRecur;
    // grid positions advance token by token (w, then h, then t carry): one
    // division for the warp's first token, none after
    int gt = 0, gh = 0, gw = 0;
    if (!p.pos && lo < hi) token_pos(p, row0 + lo, gt, gh, gw);

    uint64_t acc[2][V][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int u = 0; u < V; ++u)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[t][u][i] = 0ull;

    bool failed = false;
    int done = lo;                          // tokens whose stage was consumed
    for (int t = lo; t < hi; ++t) {
        const int k = t - lo;
        const int s = k % kPoolStages;
        if (!__all_sync(0xffffffffu, tc::mbar_wait(bars + 8 * s, (k / kPoolStages) & 1,
                                                     &s_abort))) {
            failed = true;
            break;
        }
        const uint4* st = reinterpret_cast<const uint4*>(pool_smem + (ring - tc::smem_u32(pool_smem)) +
                                                         s * kStage);
        uint4 v[SV];
#pragma unroll
        for (int x = 0; x < SV; ++x) v[x] = st[x * 32 + lane];
        __syncwarp();
        issue(t + kPoolStages, s);          // every lane has read the stage
        done = t + 1;
        const int64_t row = row0 + t;
        int tt, th, tw;
        if (p.pos) {
            token_pos(p, row, tt, th, tw);
        } else {
            tt = gt;
            th = gh;
            tw = gw;
            if (++gw == p.Wg) {
                gw = 0;
                if (++gh == p.Hg) {
                    gh = 0;
                    ++gt;
                }
            }
        }
        if (tt == pt_ && th == ph_ && tw == pw_ + 1 && run < kRecur) {
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const float c = cs[q], d = sn[q];
                cs[q] = __fmaf_rn(c, stc[q], -(d * sts[q]));
                sn[q] = __fmaf_rn(d, stc[q], c * sts[q]);
            }
            ++run;
        } else {
            token_angles<HD, LAYOUT>(p, s_omega, row, sub, cs, sn);
            run = 0;
        }
        pt_ = tt;
        ph_ = th;
        pw_ = tw;
#pragma unroll
        for (int ten = 0; ten < 2; ++ten) {
            const float* w = s_w[ten];
            uint4* orow = (ten == 0 ? p.o0 : p.o1) + row * p.stride_v + v0;
            float A[8], Bc[8], C[4], Dd[4];
            if (LAYOUT == 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    A[q] = wl[ten][2 * q] * cs[q];
                    Bc[q] = -(wl[ten][2 * q + 1] * sn[q]);
                    C[q] = wl[ten][2 * q] * sn[q];
                    Dd[q] = wl[ten][2 * q + 1] * cs[q];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float wo = w[8 * sub + i], wp = w[8 * (sub ^ HALF) + i];
                    A[i] = wo * cs[i];
                    Bc[i] = (first ? -wp : wp) * sn[i];
                }
            }
#pragma unroll
            for (int u = 0; u < V; ++u) {
                const uint4 x = v[ten * V + u];
                float f[8];
                unpack8(x, f);
                float ss = 0.0f;
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = __fmaf_rn(f[i], f[i], ss);
#pragma unroll
                for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float inv = rsqrtf(__fmaf_rn(ss, 1.0f / static_cast<float>(HD), p.eps));
                float o8[8];
                if (LAYOUT == 0) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        o8[2 * q] = inv * __fmaf_rn(f[2 * q], A[q], f[2 * q + 1] * Bc[q]);
                        o8[2 * q + 1] = inv * __fmaf_rn(f[2 * q], C[q], f[2 * q + 1] * Dd[q]);
                    }
                } else {
                    uint4 pv;
                    pv.x = __shfl_xor_sync(0xffffffffu, x.x, HALF);
                    pv.y = __shfl_xor_sync(0xffffffffu, x.y, HALF);
                    pv.z = __shfl_xor_sync(0xffffffffu, x.z, HALF);
                    pv.w = __shfl_xor_sync(0xffffffffu, x.w, HALF);
                    float fp[8];
                    unpack8(pv, fp);
#pragma unroll
                    for (int i = 0; i < 8; ++i) o8[i] = inv * __fmaf_rn(f[i], A[i], fp[i] * Bc[i]);
                }
                const uint4 packed = pack8(o8);
                if (valid[u]) st_stream(orow + 32 * u, packed);
                float r8[8];
                unpack8(packed, r8);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    acc[ten][u][i] = f2_add(acc[ten][u][i], f2_pack(r8[2 * i], r8[2 * i + 1]));
            }
        }
    }
    if (failed) {
        s_abort = 1;
        if (status) atomicExch(status, 1);
        // the copies this warp issued land before the CTA exits (none when
        // stalled)
        if (lane == 0 && !stall) {
            for (int t = done; t < hi && t < done + kPoolStages; ++t) {
                const int k = t - lo;
                tc::mbar_wait_drain(bars + 8 * (k % kPoolStages), (k / kPoolStages) & 1);
            }
        }
        __syncwarp();
    }
    __syncthreads();
    // warp sums -> shared memory [warp][tensor][u][lane][8], then warp order
    float* cmb = reinterpret_cast<float*>(pool_smem);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int u = 0; u < V; ++u) {
            float a[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) f2_unpack(acc[t][u][i], a[2 * i], a[2 * i + 1]);
            float4* d = reinterpret_cast<float4*>(cmb + (((warp * 2 + t) * V + u) * 32 + lane) * 8);
            d[0] = make_float4(a[0], a[1], a[2], a[3]);
            d[1] = make_float4(a[4], a[5], a[6], a[7]);
        }
    __syncthreads();
    if (s_abort) return;
    const float cnt = static_cast<float>(count);
    const int64_t D = static_cast<int64_t>(p.nvr) * 8;
    for (int c = warp; c < 2 * V; c += kPoolWarps) {
        const int t = c / V, u = c % V;
        float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int w = 0; w < kPoolWarps; ++w) {
            const float* src = cmb + (((w * 2 + t) * V + u) * 32 + lane) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) sum[i] += src[i];
        }
        if (valid[u]) {
            float4* dst = reinterpret_cast<float4*>(
                means + ((static_cast<int64_t>(b) * 2 + t) * nb + j) * D +
                static_cast<int64_t>(v0 + 32 * u) * 8);
            dst[0] = make_float4(sum[0] / cnt, sum[1] / cnt, sum[2] / cnt, sum[3] / cnt);
            dst[1] = make_float4(sum[4] / cnt, sum[5] / cnt, sum[6] / cnt, sum[7] / cnt);
        }
    }
}

using PoolKernel = void (*)(QKParams, int, int, float*, int*, int);

template <int LAYOUT>
PoolKernel pick_pool(int hd) {
    switch (hd) {
        case 32: return qk_rope_pool_kernel<32, LAYOUT, kPoolV>;
        case 64: return qk_rope_pool_kernel<64, LAYOUT, kPoolV>;
        case 128: return qk_rope_pool_kernel<128, LAYOUT, kPoolV>;
        case 256: return qk_rope_pool_kernel<256, LAYOUT, kPoolV>;
        default: return nullptr;
    }
}

using QKKernel = void (*)(QKParams);

struct Pick {
    QKKernel kernel = nullptr;
    int nvl = 0;            // vectors per lane the kernel holds
};

template <int HD, int LAYOUT, int MODE>
Pick pick_nvl(int nvl) {
#define DIT_NVL_CASE(V) \
    if (nvl <= V) return Pick{qk_rmsnorm_rope3d_kernel<HD, V, LAYOUT, MODE>, V};
    DIT_NVL_CASE(1) DIT_NVL_CASE(2) DIT_NVL_CASE(3) DIT_NVL_CASE(4) DIT_NVL_CASE(6)
    DIT_NVL_CASE(8) DIT_NVL_CASE(10) DIT_NVL_CASE(12) DIT_NVL_CASE(16) DIT_NVL_CASE(20)
    DIT_NVL_CASE(24) DIT_NVL_CASE(32)
#undef DIT_NVL_CASE
    return Pick{};
}

template <int LAYOUT, int MODE>
Pick pick_hd(int hd, int nvl) {
    switch (hd) {
        case 32: return pick_nvl<32, LAYOUT, MODE>(nvl);
        case 64: return pick_nvl<64, LAYOUT, MODE>(nvl);
        case 128: return pick_nvl<128, LAYOUT, MODE>(nvl);
        case 256: return pick_nvl<256, LAYOUT, MODE>(nvl);
        default: return Pick{};
    }
}

Pick pick(int hd, int layout, int mode, int nvl) {
    const bool half = layout == DIT_ROPE_HALF;
    switch (mode) {
        case 0: return half ? pick_hd<DIT_ROPE_HALF, 0>(hd, nvl)
                            : pick_hd<DIT_ROPE_INTERLEAVED, 0>(hd, nvl);
        case 1: return half ? pick_hd<DIT_ROPE_HALF, 1>(hd, nvl)
                            : pick_hd<DIT_ROPE_INTERLEAVED, 1>(hd, nvl);
        case 2: return half ? pick_hd<DIT_ROPE_HALF, 2>(hd, nvl)
                            : pick_hd<DIT_ROPE_INTERLEAVED, 2>(hd, nvl);
        default: return Pick{};
    }
}

template <int HD, int LAYOUT>
Pick pick_row_nvl(int nvl) {
#define DIT_ROW_CASE(V)                                                              \
    if (nvl <= V) return Pick{qk_row_persistent_kernel<HD, V, LAYOUT>, V};
    if constexpr (LAYOUT == 0) {
        DIT_ROW_CASE(1) DIT_ROW_CASE(2) DIT_ROW_CASE(3) DIT_ROW_CASE(4) DIT_ROW_CASE(6)
        DIT_ROW_CASE(8) DIT_ROW_CASE(10) DIT_ROW_CASE(12) DIT_ROW_CASE(16) DIT_ROW_CASE(20)
    } else {
        DIT_ROW_CASE(2) DIT_ROW_CASE(4) DIT_ROW_CASE(6) DIT_ROW_CASE(8) DIT_ROW_CASE(10)
        DIT_ROW_CASE(12) DIT_ROW_CASE(16) DIT_ROW_CASE(20)
    }
#undef DIT_ROW_CASE
    return Pick{};
}

// The persistent whole-row kernel for rows of up to kRowMaxNVL lane-vectors.
Pick pick_row(int hd, int layout, int nvl) {
    if (nvl > kRowMaxNVL) return Pick{};
    const bool half = layout == DIT_ROPE_HALF;
    switch (hd) {
        case 32: return half ? pick_row_nvl<32, 1>(nvl) : pick_row_nvl<32, 0>(nvl);
        case 64: return half ? pick_row_nvl<64, 1>(nvl) : pick_row_nvl<64, 0>(nvl);
        case 128: return half ? pick_row_nvl<128, 1>(nvl) : pick_row_nvl<128, 0>(nvl);
        case 256: return half ? pick_row_nvl<256, 1>(nvl) : pick_row_nvl<256, 0>(nvl);
        default: return Pick{};
    }
}

// Rows i of q and k (i < rows, `rs` elements apart, `w` wide) overlap iff
// some row difference m in (-rows, rows) puts k within w elements of q.
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

// Byte range [lo, hi) a buffer touches.
struct Span {
    uintptr_t lo = 0, hi = 0;
    bool meets(const Span& o) const { return lo < o.hi && o.lo < hi; }
};

// The output layout [B, N, H, hd] with strides (sb, sn, sh, 1) must give
// every element its own address: sorted by stride, each dimension of
// extent > 1 must step over everything the smaller ones span.  Returns
// the element span of one tensor, or -1.
int64_t out_extent(int B, int64_t N, int H, int hd, int64_t sb, int64_t sn, int64_t sh) {
    int64_t ext[3] = {B, N, H}, st[3] = {sb, sn, sh};
    for (int a = 0; a < 3; ++a)
        for (int b = a + 1; b < 3; ++b)
            if (st[b] < st[a]) {
                const int64_t e = ext[a], s = st[a];
                ext[a] = ext[b]; st[a] = st[b];
                ext[b] = e; st[b] = s;
            }
    int64_t span = hd;                     // elements covered so far
    for (int a = 0; a < 3; ++a) {
        if (ext[a] <= 1) continue;
        if (st[a] < span) return -1;
        if (st[a] > (INT64_MAX / 4) / ext[a]) return -1;
        span = st[a] * (ext[a] - 1) + span;
        if (span > INT64_MAX / 4) return -1;
    }
    return span;
}

}  // namespace
}  // namespace dit

extern "C" int dit_qk_rmsnorm_rope3d_ex(uint16_t* q, uint16_t* k, int64_t row_stride,
                                        const void* w_q, const void* w_k, int w_dtype, int B,
                                        int64_t N, int H, int hd, int T, int Hg, int Wg,
                                        const int32_t* pos, int64_t pos_offset, int pairs_t,
                                        int pairs_h, int pairs_w, double theta, double eps,
                                        int rope_layout, int norm_width, const dit_qk_out* out,
                                        void* stream) {
    using namespace dit;
    if (w_dtype != DIT_F32 && w_dtype != DIT_BF16) return DIT_ERR_DTYPE;
    if (B < 0 || N < 0 || H < 1) return DIT_ERR_SHAPE;
    if (hd != 32 && hd != 64 && hd != 128 && hd != 256) return DIT_ERR_SHAPE;
    if (rope_layout != DIT_ROPE_INTERLEAVED && rope_layout != DIT_ROPE_HALF) return DIT_ERR_VALUE;
    if (norm_width != DIT_NORM_HEAD && norm_width != DIT_NORM_ROW) return DIT_ERR_VALUE;
    if (pairs_t < 1 || pairs_h < 1 || pairs_w < 1 || pairs_t + pairs_h + pairs_w != hd / 2)
        return DIT_ERR_SHAPE;
    const int64_t width = static_cast<int64_t>(H) * hd;
    if (width > DIT_MAX_D || row_stride < width) return DIT_ERR_SHAPE;
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
    int64_t osb = N * row_stride, osn = row_stride, osh = hd, oext = 0;
    if (out) {
        osb = out->stride_b;
        osn = out->stride_n;
        osh = out->stride_h;
        if (osb < 0 || osn < 0 || osh < 0) return DIT_ERR_SHAPE;
        if (osb % 8 || osn % 8 || osh % 8) return DIT_ERR_ALIGN;
        oext = out_extent(B, N, H, hd, osb, osn, osh);
        if (oext < 0) return DIT_ERR_SHAPE;
    }
    if (rows == 0) return DIT_OK;
    if (!q && !k) return DIT_ERR_NULL;
    int st;
    if (q && (st = check_w(w_q, w_dtype))) return st;
    if (k && (st = check_w(w_k, w_dtype))) return st;
    // whole-row weights are read 16 bytes at a time
    if (norm_width == DIT_NORM_ROW && ((q && !aligned16(w_q)) || (k && !aligned16(w_k))))
        return DIT_ERR_ALIGN;
    if ((q && !aligned16(q)) || (k && !aligned16(k))) return DIT_ERR_ALIGN;
    uint16_t* q_dst = q;
    uint16_t* k_dst = k;
    if (out) {
        if ((q && !out->q) || (k && !out->k)) return DIT_ERR_NULL;
        q_dst = q ? out->q : nullptr;
        k_dst = k ? out->k : nullptr;
        if ((q_dst && !aligned16(q_dst)) || (k_dst && !aligned16(k_dst))) return DIT_ERR_ALIGN;
        // no output may overlap an input or the other output
        const uintptr_t in_bytes = 2 * static_cast<uintptr_t>((rows - 1) * row_stride + width);
        const uintptr_t out_bytes = 2 * static_cast<uintptr_t>(oext);
        auto span = [](const void* p, uintptr_t n) {
            Span s;
            s.lo = reinterpret_cast<uintptr_t>(p);
            s.hi = s.lo + n;
            return s;
        };
        Span outs[2], ins[2];
        int no = 0, ni = 0;
        if (q) { outs[no++] = span(q_dst, out_bytes); ins[ni++] = span(q, in_bytes); }
        if (k) { outs[no++] = span(k_dst, out_bytes); ins[ni++] = span(k, in_bytes); }
        for (int a = 0; a < no; ++a) {
            for (int b = 0; b < ni; ++b)
                if (outs[a].meets(ins[b])) return DIT_ERR_OVERLAP;
            for (int b = a + 1; b < no; ++b)
                if (outs[a].meets(outs[b])) return DIT_ERR_OVERLAP;
        }
    } else if (q && k && rows_overlap(q, k, rows, row_stride, width)) {
        return DIT_ERR_OVERLAP;
    }

    QKParams p{};
    p.t0 = reinterpret_cast<const uint4*>(q ? q : k);
    p.t1 = q ? reinterpret_cast<const uint4*>(k) : nullptr;
    p.o0 = reinterpret_cast<uint4*>(q ? q_dst : k_dst);
    p.o1 = q ? reinterpret_cast<uint4*>(k_dst) : nullptr;
    p.w0 = q ? w_q : w_k;
    p.w1 = q ? w_k : nullptr;
    p.w_dtype = w_dtype;
    p.stride_v = row_stride / 8;
    p.osb = osb / 8;
    p.osn = osn / 8;
    p.osh = osh / 8;
    p.o_rows = osb == N * osn;
    p.rows = rows;
    p.N = N;
    p.rows32 = rows < (int64_t(1) << 31);
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

    const int mode = norm_width == DIT_NORM_ROW ? 2 : (osh == hd ? 0 : 1);
    // rotate-half with the whole-row norm holds the row in whole 64-vector
    // spans (an even count of lane-vectors)
    const int nvl = mode == 2 && rope_layout == DIT_ROPE_HALF ? 2 * ((p.nvr + 63) / 64)
                                                              : (p.nvr + 31) / 32;
    if (mode == 2) {
        const Pick rk = pick_row(hd, rope_layout, nvl);
        if (rk.kernel) {
            const int ntens = p.t1 ? 2 : 1;
            const size_t rsmem = static_cast<size_t>(2 * p.nvr * ntens) * sizeof(float4) +
                                 static_cast<size_t>(kRowWarps) * rk.nvl * 32 * sizeof(uint4);
            if (cudaFuncSetAttribute(rk.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(rsmem)) != cudaSuccess)
                return DIT_ERR_LAUNCH;
            const int sms = device_sm_count();
            const int occ = occupancy(reinterpret_cast<const void*>(rk.kernel), kRowWarps * 32, rsmem);
            if (sms <= 0 || occ <= 0) return DIT_ERR_LAUNCH;
            int64_t ctas = (rows + kRowWarps - 1) / kRowWarps;
            if (ctas > static_cast<int64_t>(sms) * occ) ctas = static_cast<int64_t>(sms) * occ;
            rk.kernel<<<static_cast<unsigned>(ctas), kRowWarps * 32, rsmem, as_stream(stream)>>>(p);
            return launch_status();
        }
    }
    const Pick pk = pick(hd, rope_layout, mode, nvl);
    if (!pk.kernel) return DIT_ERR_SHAPE;
    // the second tensor's stage
    const size_t smem =
        p.t1 ? static_cast<size_t>(kWarps) * pk.nvl * 32 * sizeof(uint4) : 0;
    // opt in whenever dynamic shared memory is used: with the static
    // frequency table the total can pass the 48 KB default
    if (smem > 0 &&
        cudaFuncSetAttribute(pk.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    const int64_t ctas = (rows + kWarps - 1) / kWarps;
    if (ctas > 0x7FFFFFFF) return DIT_ERR_SHAPE;
    pk.kernel<<<static_cast<unsigned>(ctas), kThreads, smem, as_stream(stream)>>>(p);
    return launch_status();
}

extern "C" int dit_qk_rmsnorm_rope3d(uint16_t* q, uint16_t* k, int64_t row_stride,
                                     const void* w_q, const void* w_k, int w_dtype, int B,
                                     int64_t N, int H, int hd, int T, int Hg, int Wg,
                                     const int32_t* pos, int64_t pos_offset, int pairs_t,
                                     int pairs_h, int pairs_w, double theta, double eps,
                                     void* stream) {
    return dit_qk_rmsnorm_rope3d_ex(q, k, row_stride, w_q, w_k, w_dtype, B, N, H, hd, T, Hg, Wg,
                                    pos, pos_offset, pairs_t, pairs_h, pairs_w, theta, eps,
                                    DIT_ROPE_INTERLEAVED, DIT_NORM_HEAD, nullptr, stream);
}

namespace dit {
namespace {

int qk_pooled(uint16_t* q, uint16_t* k, int64_t row_stride, const void* w_q, const void* w_k,
              int w_dtype, int B, int64_t N, int H, int hd, int T, int Hg, int Wg,
              const int32_t* pos, int64_t pos_offset, int pairs_t, int pairs_h, int pairs_w,
              double theta, double eps, int rope_layout, int block, float* block_means,
              int* status, void* stream, int stall) {
    if (w_dtype != DIT_F32 && w_dtype != DIT_BF16) return DIT_ERR_DTYPE;
    if (B < 0 || N < 0 || H < 1 || block < 1) return DIT_ERR_SHAPE;
    if (hd != 32 && hd != 64 && hd != 128 && hd != 256) return DIT_ERR_SHAPE;
    if (rope_layout != DIT_ROPE_INTERLEAVED && rope_layout != DIT_ROPE_HALF) return DIT_ERR_VALUE;
    if (pairs_t < 1 || pairs_h < 1 || pairs_w < 1 || pairs_t + pairs_h + pairs_w != hd / 2)
        return DIT_ERR_SHAPE;
    const int64_t width = static_cast<int64_t>(H) * hd;
    if (width > DIT_MAX_D || row_stride < width) return DIT_ERR_SHAPE;
    if (row_stride % 8) return DIT_ERR_ALIGN;
    if (!(theta > 0.0) || theta > 1e300 || !(eps >= 0.0) || eps > 1e30) return DIT_ERR_VALUE;
    if (B > 65535 || (B > 0 && N > (INT64_MAX / 4) / row_stride / B)) return DIT_ERR_SHAPE;
    if (!pos) {
        if (T < 1 || Hg < 1 || Wg < 1 || pos_offset < 0) return DIT_ERR_SHAPE;
        const int64_t cells = static_cast<int64_t>(T) * Hg * Wg;
        if (cells > INT32_MAX || pos_offset + N > cells) return DIT_ERR_SHAPE;
    } else if (reinterpret_cast<uintptr_t>(pos) % 4) {
        return DIT_ERR_ALIGN;
    }
    const int64_t nb = (N + block - 1) / block;
    if (nb > 65535) return DIT_ERR_SHAPE;
    if (B == 0 || N == 0) return DIT_OK;
    if (!q || !k || !block_means) return DIT_ERR_NULL;
    int st;
    if ((st = check_w(w_q, w_dtype)) || (st = check_w(w_k, w_dtype))) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(block_means)) return DIT_ERR_ALIGN;
    const int64_t rows = static_cast<int64_t>(B) * N;
    if (rows_overlap(q, k, rows, row_stride, width)) return DIT_ERR_OVERLAP;
    const size_t mbytes = static_cast<size_t>(B) * 2 * nb * width * sizeof(float);
    const size_t qbytes = 2 * static_cast<size_t>((rows - 1) * row_stride + width);
    if (overlaps(block_means, mbytes, q, qbytes) || overlaps(block_means, mbytes, k, qbytes))
        return DIT_ERR_OVERLAP;

    QKParams p{};
    p.t0 = reinterpret_cast<const uint4*>(q);
    p.t1 = reinterpret_cast<const uint4*>(k);
    p.o0 = reinterpret_cast<uint4*>(q);
    p.o1 = reinterpret_cast<uint4*>(k);
    p.w0 = w_q;
    p.w1 = w_k;
    p.w_dtype = w_dtype;
    p.stride_v = row_stride / 8;
    p.rows = rows;
    p.N = N;
    p.rows32 = rows < (int64_t(1) << 31);
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
    const PoolKernel kern = rope_layout == DIT_ROPE_HALF ? pick_pool<DIT_ROPE_HALF>(hd)
                                                         : pick_pool<DIT_ROPE_INTERLEAVED>(hd);
    if (!kern) return DIT_ERR_SHAPE;
    const int groups = (p.nvr + 32 * kPoolV - 1) / (32 * kPoolV);
    if (status && reinterpret_cast<uintptr_t>(status) % 4) return DIT_ERR_ALIGN;
    // the rings, then one mbarrier per stage and warp
    const size_t smem = static_cast<size_t>(kPoolWarps) * kPoolStages * (2 * kPoolV * 32 * 16 + 8);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    kern<<<dim3(groups, static_cast<unsigned>(nb), B), kPoolWarps * 32, smem,
           as_stream(stream)>>>(p, block, static_cast<int>(nb), block_means, status, stall);
    return launch_status();
}

}  // namespace
}  // namespace dit

extern "C" int dit_qk_rmsnorm_rope3d_pooled(uint16_t* q, uint16_t* k, int64_t row_stride,
                                            const void* w_q, const void* w_k, int w_dtype, int B,
                                            int64_t N, int H, int hd, int T, int Hg, int Wg,
                                            const int32_t* pos, int64_t pos_offset, int pairs_t,
                                            int pairs_h, int pairs_w, double theta, double eps,
                                            int rope_layout, int block, float* block_means,
                                            int* status, void* stream) {
    return dit::qk_pooled(q, k, row_stride, w_q, w_k, w_dtype, B, N, H, hd, T, Hg, Wg, pos,
                          pos_offset, pairs_t, pairs_h, pairs_w, theta, eps, rope_layout, block,
                          block_means, status, stream, 0);
}

extern "C" int dit_qk_rmsnorm_rope3d_pooled_stall_test(
    uint16_t* q, uint16_t* k, int64_t row_stride, const void* w_q, const void* w_k, int w_dtype,
    int B, int64_t N, int H, int hd, int T, int Hg, int Wg, const int32_t* pos,
    int64_t pos_offset, int pairs_t, int pairs_h, int pairs_w, double theta, double eps,
    int rope_layout, int block, float* block_means, int* status, void* stream) {
    if (!status) return DIT_ERR_NULL;
    if (B < 1 || N < 1 || static_cast<int64_t>(B) * N > 4096) return DIT_ERR_SHAPE;
    return dit::qk_pooled(q, k, row_stride, w_q, w_k, w_dtype, B, N, H, hd, T, Hg, Wg, pos,
                          pos_offset, pairs_t, pairs_h, pairs_w, theta, eps, rope_layout, block,
                          block_means, status, stream, 1);
}
