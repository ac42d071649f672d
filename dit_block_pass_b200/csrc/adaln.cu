// adaln.cu -- AdaLN modulation, and the gated residual fused with the next
// AdaLN, each in one pass over HBM.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração
// somadas chega-se a 6 vezes": the fused AdaLN update and the gated residual
// ("residual com gate"); the fused layer changes no result, so the gated
// variant normalises the residual exactly as stored in bf16.  "MiniMax H3 mở
// trọng số", section "Kiến trúc: tạo hình và tiếng trong cùng một luồng": the
// AdaLN-branch outputs are precomputed, so shift/scale/gate arrive as inputs.
//
// Design: one warp owns one token row at a time and holds the whole row in
// registers (VPL 16-byte vectors per lane; D = 5120 -> 20), so x is read
// once.  The gated variant splits each row across a warp pair and brings the
// branch row r through a per-warp shared-memory stage with cp.async.  Row statistics are two warp-shuffle reductions (a mean of values
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
    const uint8_t* set_index;   // per-token modulation set, or NULL (set 0 everywhere)
    int64_t set_stride;         // elements between the sets of one sample
    int n_sets;
    bool mod_vec;               // every set's vectors can be read 16 bytes at a time
    int staged_sets;            // sets staged in shared memory (1, or 2 for AdaLN)
};

__device__ __forceinline__ float mod_at(const void* p, int dtype, int64_t i) {
    if (dtype == DIT_F32) return static_cast<const float*>(p)[i];
    return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16);
}

// bf16(x + g*r) for two elements with ONE rounding of each exact value.
// The fp32 fma rounds once to 24 bits; rounding that to bf16 can differ
// from rounding the exact value only when the fp32 result sits exactly on a
// bf16 tie (low 16 bits 0x8000).  The pair is then redone in fp64, where
// g*r (<= 32 significant bits) is exact, and rounded straight to bf16.  The
// packed fp32 -> bf16x2 conversion runs on the ALU, not the conversion unit.
__device__ __noinline__ uint32_t gated_pair_fp64(float x0, float g0, float r0, float x1, float g1,
                                                 float r1) {
    const __nv_bfloat16 lo = __double2bfloat16(
        fma(static_cast<double>(g0), static_cast<double>(r0), static_cast<double>(x0)));
    const __nv_bfloat16 hi = __double2bfloat16(
        fma(static_cast<double>(g1), static_cast<double>(r1), static_cast<double>(x1)));
    return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

__device__ __forceinline__ uint32_t gated_pair(uint32_t xw, uint32_t rw, float g0, float g1) {
    const float x0 = bf16_lo(xw), x1 = bf16_hi(xw);
    const float r0 = bf16_lo(rw), r1 = bf16_hi(rw);
    const float s0 = __fmaf_rn(g0, r0, x0);
    const float s1 = __fmaf_rn(g1, r1, x1);
    const bool tie = ((__float_as_uint(s0) & 0xFFFFu) == 0x8000u) |
                     ((__float_as_uint(s1) & 0xFFFFu) == 0x8000u);
    if (tie) return gated_pair_fp64(x0, g0, r0, x1, g1, r1);
    return pack2(s0, s1);
}

__device__ __forceinline__ void lds8(const float4* lo, const float4* hi, int v, float (&f)[8]) {
    const float4 a = lo[v], b = hi[v];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Eight modulation values at element offset off, from global memory (L1/L2
// resident: a set is shared by many rows).  Vector loads when the host
// found every set 16-byte aligned.
__device__ __forceinline__ void mod8(const RowParams& p, const void* m, int64_t off,
                                     float (&f)[8]) {
    if (p.mod_vec) {
        if (p.mod_dtype == DIT_F32) {
            const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(m) + off);
            const float4 a = __ldg(q), b = __ldg(q + 1);
            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
            f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        } else {
            unpack8(__ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(m) + off)),
                    f);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = mod_at(m, p.mod_dtype, off + i);
    }
}

// Modulation set of token n of sample blockIdx.y (0 without an index).  An
// index past the last set returns -1: the row's outputs are then NaN, since
// a kernel cannot return an error to the caller.
template <bool TOK>
__device__ __forceinline__ int token_set(const RowParams& p, int64_t row) {
    if (!TOK) return 0;
    const int s = __ldg(p.set_index + row);
    return s < p.n_sets ? s : -1;
}

// shift and 1 + scale (and gate) of vector v for a row of set `set`: set 0
// from the shared-memory stage, other sets from global memory.
template <bool TOK>
__device__ __forceinline__ void modulation8(const RowParams& p, const float4* s_lo, int Dv,
                                            int v, const void* m, int set, bool one_plus,
                                            float (&f)[8]) {
    if (TOK && set > 0 && set < p.staged_sets) {
        // a second staged set follows the first (4 * Dv float4s apart)
        lds8(s_lo + 4 * Dv, s_lo + 5 * Dv, v, f);
        return;
    }
    if (TOK && set != 0) {
        if (set < 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __int_as_float(0x7fc00000);
            return;
        }
        mod8(p, m, static_cast<int64_t>(blockIdx.y) * p.mod_stride + set * p.set_stride + 8 * v,
             f);
        if (one_plus) {
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = 1.0f + f[i];
        }
        return;
    }
    lds8(s_lo, s_lo + Dv, v, f);
}

// Stage the modulation vectors of sample blockIdx.y in shared memory:
// shift and (1 + scale) (and gate), each as [lo Dv][hi Dv] float4 halves.
template <bool GATED>
__device__ __forceinline__ void stage_one_set(const RowParams& p, float4* smem, int nthreads,
                                              int64_t mb);

template <bool GATED>
__device__ __forceinline__ void stage_modulation(const RowParams& p, float4* smem, int nthreads) {
    const int64_t mb = static_cast<int64_t>(blockIdx.y) * p.mod_stride;
    stage_one_set<GATED>(p, smem, nthreads, mb);
    // AdaLN with per-token sets: set 1 too, 4 * Dv float4s after set 0
    if (!GATED && p.staged_sets > 1)
        stage_one_set<GATED>(p, smem + 4 * p.Dv, nthreads, mb + p.set_stride);
}

template <bool GATED>
__device__ __forceinline__ void stage_one_set(const RowParams& p, float4* smem, int nthreads,
                                              int64_t mb) {
    const int Dv = p.Dv;
    float4* s_sh = smem;
    float4* s_sc = smem + 2 * Dv;
    float4* s_g = smem + 4 * Dv;
    for (int v = threadIdx.x; v < Dv; v += nthreads) {
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
}

// Second half of the LayerNorm of the warp's register-resident row, given
// the shift x0 and the warp's sum of (x - x0): the centred sum of squares,
// then y = (x - mu) * rstd * (1 + scale) + shift.
template <int VPL, bool TOK>
__device__ __forceinline__ void ln_finish_store(const RowParams& p, const float4* smem,
                                                const uint4 (&xv)[VPL], int64_t base, int lane,
                                                float x0, float s, int set) {
    const int Dv = p.Dv;
    const float4* s_sh = smem;
    const float4* s_sc = smem + 2 * Dv;
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
    // the set is decided once per row, outside the unrolled loops, so that a
    // staged row's shared-memory loads can be issued ahead as without sets
    if (!TOK || (set >= 0 && set < p.staged_sets)) {
        const int so = TOK ? 4 * Dv * set : 0;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int v = j * 32 + lane;
            if (v < Dv) {
                float f[8], sh[8], sc[8];
                unpack8(xv[j], f);
                lds8(s_sh + so, s_sh + so + Dv, v, sh);
                lds8(s_sc + so, s_sc + so + Dv, v, sc);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fmaf_rn((f[i] - mu) * rstd, sc[i], sh[i]);
                st_stream(p.y + base + v, pack8(f));
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int v = j * 32 + lane;
            if (v < Dv) {
                float f[8], sh[8], sc[8];
                unpack8(xv[j], f);
                modulation8<TOK>(p, s_sh, Dv, v, p.shift, set, false, sh);
                modulation8<TOK>(p, s_sc, Dv, v, p.scale, set, true, sc);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fmaf_rn((f[i] - mu) * rstd, sc[i], sh[i]);
                st_stream(p.y + base + v, pack8(f));
            }
        }
    }
}

// The LayerNorm of the row with the mean accumulated relative to the row's
// first element (a shift that keeps the fp32 sum small when |mean| >> std).
template <int VPL, bool TOK>
__device__ __forceinline__ void ln_modulate_store(const RowParams& p, const float4* smem,
                                                  const uint4 (&xv)[VPL], int64_t base,
                                                  int lane, int set) {
    const float x0 = __shfl_sync(0xffffffffu, bf16_lo(xv[0].x), 0);
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        if (j * 32 + lane < p.Dv) {
            float f[8];
            unpack8(xv[j], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) s += f[i] - x0;
        }
    }
    ln_finish_store<VPL, TOK>(p, smem, xv, base, lane, x0, s, set);
}

// AdaLN: one warp per row, the row in registers (VPL vectors per lane).
// TOK: modulation sets chosen per token (set 0 staged, others from L1/L2).
template <int VPL, bool TOK>
__global__ void __launch_bounds__(kThreads, (TOK && VPL <= 20) ? 2 : 0)
adaln_rows_kernel(RowParams p) {
    extern __shared__ float4 smem[];
    stage_modulation<false>(p, smem, kThreads);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t row0 = static_cast<int64_t>(blockIdx.y) * p.N;
    const int64_t wstep = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); n < p.N;
         n += wstep) {
        const int64_t base = (row0 + n) * p.Dv;
        uint4 xv[VPL];
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int v = j * 32 + lane;
            xv[j] = (v < p.Dv) ? ld_inplace(p.x + base + v) : make_uint4(0, 0, 0, 0);
        }
        ln_modulate_store<VPL, TOK>(p, smem, xv, base, lane, token_set<TOK>(p, row0 + n));
    }
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}

// First pass of a gated row (the lane's vectors of one half): x + gate * r
// to x_out, kept in xv, and the sum of (x_out - x0).  STAGED reads the gate
// from the shared-memory stage (set 0), otherwise from the row's set.
template <int VPL, bool TOK, bool STAGED>
__device__ __forceinline__ float gated_first_pass(const RowParams& p, const float4* s_g,
                                                  const uint4* stage, uint4 (&xv)[VPL],
                                                  int64_t base, int lane, int half, int set,
                                                  float x0) {
    const int Dv = p.Dv;
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int v = 64 * j + 32 * half + lane;
        if (v < Dv) {
            const uint4 rv = stage[j * 32 + lane];
            float g[8];
            if (STAGED) lds8(s_g, s_g + Dv, v, g);
            else modulation8<TOK>(p, s_g, Dv, v, p.gate, set, false, g);
            uint4 o;
            o.x = gated_pair(xv[j].x, rv.x, g[0], g[1]);
            o.y = gated_pair(xv[j].y, rv.y, g[2], g[3]);
            o.z = gated_pair(xv[j].z, rv.z, g[4], g[5]);
            o.w = gated_pair(xv[j].w, rv.w, g[6], g[7]);
            xv[j] = o;
            st_stream(p.x_out + base + v, o);
            float f[8];
            unpack8(o, f);
            float t = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) t += f[i];
            s += __fmaf_rn(-8.0f, x0, t);
        }
    }
    return s;
}

// Last pass of a gated row: y = (x_out - mu) * rstd * (1 + scale) + shift.
template <int VPL, bool TOK, bool STAGED>
__device__ __forceinline__ void gated_last_pass(const RowParams& p, const float4* s_sh,
                                                const float4* s_sc, const uint4 (&xv)[VPL],
                                                int64_t base, int lane, int half, int set,
                                                float mu, float rstd) {
    const int Dv = p.Dv;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int v = 64 * j + 32 * half + lane;
        if (v < Dv) {
            float f[8], sh[8], sc[8];
            unpack8(xv[j], f);
            if (STAGED) {
                lds8(s_sh, s_sh + Dv, v, sh);
                lds8(s_sc, s_sc + Dv, v, sc);
            } else {
                modulation8<TOK>(p, s_sh, Dv, v, p.shift, set, false, sh);
                modulation8<TOK>(p, s_sc, Dv, v, p.scale, set, true, sc);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __fmaf_rn((f[i] - mu) * rstd, sc[i], sh[i]);
            st_stream(p.y + base + v, pack8(f));
        }
    }
}

// Gated residual + AdaLN: one warp PAIR per row.  Warp h (0, 1) of a pair
// holds vectors v = 64*j + 32*h + lane of the row (each warp instruction
// still covers 512 contiguous bytes), so a lane keeps VPL = ceil(D/512)
// vectors in registers and twice as many warps fit on an SM as with one
// warp per row.  The branch row r goes to a per-warp shared-memory stage
// with cp.async, issued together with the x loads.  The two row statistics
// are exchanged through shared memory with one named barrier per pair each;
// both warps add the two halves in the same order, so they agree exactly.
template <int VPL, int WARPS, bool TOK>
__global__ void __launch_bounds__(WARPS * 32, 1)
gated_rows_kernel(RowParams p) {
    constexpr int PAIRS = WARPS / 2;
    extern __shared__ float4 smem[];
    __shared__ float red[PAIRS][2][2];          // [pair][statistic][half]
    __shared__ float shift[PAIRS][2];           // [pair][half]: each half's shift
    stage_modulation<true>(p, smem, WARPS * 32);
    __syncthreads();
    const int Dv = p.Dv;
    const float4* s_g = smem + 4 * Dv;
    const float4* s_sh = smem;
    const float4* s_sc = smem + 2 * Dv;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int half = warp & 1, pair = warp >> 1;
    const int bar = 1 + pair;                   // named barrier of the pair (0 = __syncthreads)
    uint4* stage = reinterpret_cast<uint4*>(smem + 6 * Dv) + warp * (VPL * 32);
    // elements held by half 1: vectors 64j + 32 + lane < Dv
    const int rem = Dv % 64;
    const float n1 = 8.0f * static_cast<float>((Dv / 64) * 32 + (rem > 32 ? rem - 32 : 0));
    const int64_t row0 = static_cast<int64_t>(blockIdx.y) * p.N;
    const int64_t rstep = static_cast<int64_t>(gridDim.x) * PAIRS;
    bool r_issued = false;                      // this row's r copies went out last row
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * PAIRS + pair; n < p.N; n += rstep) {
        const int64_t base = (row0 + n) * Dv;
        if (!r_issued) {
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int v = 64 * j + 32 * half + lane;
                if (v < Dv) cp_async16(stage + j * 32 + lane, p.r + base + v);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        uint4 xv[VPL];
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int v = 64 * j + 32 * half + lane;
            xv[j] = (v < Dv) ? ld_inplace(p.x + base + v) : make_uint4(0, 0, 0, 0);
        }
        const int set = token_set<TOK>(p, row0 + n);
        // shift for this half's sum: the first element the warp holds (x may be
        // overwritten in place by the other warp, so each warp uses its own)
        const float x0 = __shfl_sync(0xffffffffu, bf16_lo(xv[0].x), 0);
        // each lane reads back only the vectors it copied itself
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        // the set is decided once per row, outside the unrolled loops
        const bool staged = !TOK || set == 0;
        float s = 0.0f;
        if (!TOK) {
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int v = 64 * j + 32 * half + lane;
                if (v < Dv) {
                    const uint4 rv = stage[j * 32 + lane];
                    float g[8];
                    lds8(s_g, s_g + Dv, v, g);
                    uint4 o;
                    o.x = gated_pair(xv[j].x, rv.x, g[0], g[1]);
                    o.y = gated_pair(xv[j].y, rv.y, g[2], g[3]);
                    o.z = gated_pair(xv[j].z, rv.z, g[4], g[5]);
                    o.w = gated_pair(xv[j].w, rv.w, g[6], g[7]);
                    xv[j] = o;
                    st_stream(p.x_out + base + v, o);
                    float f[8];
                    unpack8(o, f);
                    float t = 0.0f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) t += f[i];
                    s += __fmaf_rn(-8.0f, x0, t);
                }
            }
        } else if (staged) {
            s = gated_first_pass<VPL, TOK, true>(p, s_g, stage, xv, base, lane, half, set, x0);
        } else {
            s = gated_first_pass<VPL, TOK, false>(p, s_g, stage, xv, base, lane, half, set, x0);
        }
        // the stage is free (each lane read back its own vectors): the next
        // row's r copies go out now and travel while this row's statistics
        // and y are computed
        const int64_t nn = n + rstep;
        r_issued = nn < p.N;
        if (r_issued) {
            const uint4* rn = p.r + (row0 + nn) * Dv;
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int v = 64 * j + 32 * half + lane;
                if (v < Dv) cp_async16(stage + j * 32 + lane, rn + v);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        s = warp_sum(s);
        if (lane == 0) {
            red[pair][0][half] = s;
            shift[pair][half] = x0;
        }
        asm volatile("bar.sync %0, 64;" ::"r"(bar) : "memory");
        // sum = s0 + n0*x00 + s1 + n1*x01; both warps evaluate the same expression
        const float x00 = shift[pair][0];
        const float mu =
            x00 + __fmaf_rn(n1, shift[pair][1] - x00, red[pair][0][0] + red[pair][0][1]) * p.inv_D;
        float q = 0.0f;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            if (64 * j + 32 * half + lane < Dv) {
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
        if (lane == 0) red[pair][1][half] = q;
        asm volatile("bar.sync %0, 64;" ::"r"(bar) : "memory");
        const float rstd =
            rsqrtf(__fmaf_rn(red[pair][1][0] + red[pair][1][1], p.inv_D, p.eps));
        if (!TOK) {
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int v = 64 * j + 32 * half + lane;
                if (v < Dv) {
                    float f[8], sh[8], sc[8];
                    unpack8(xv[j], f);
                    lds8(s_sh, s_sh + Dv, v, sh);
                    lds8(s_sc, s_sc + Dv, v, sc);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        f[i] = __fmaf_rn((f[i] - mu) * rstd, sc[i], sh[i]);
                    st_stream(p.y + base + v, pack8(f));
                }
            }
        } else if (staged) {
            gated_last_pass<VPL, TOK, true>(p, s_sh, s_sc, xv, base, lane, half, set, mu, rstd);
        } else {
            gated_last_pass<VPL, TOK, false>(p, s_sh, s_sc, xv, base, lane, half, set, mu, rstd);
        }
    }
}

using RowKernel = void (*)(RowParams);

struct RowLaunch {
    RowKernel kernel;
    int threads;
    size_t smem;
};

template <bool TOK>
RowLaunch pick_kernel(bool gated, int Dv) {
    const size_t mod = static_cast<size_t>(gated ? 6 : 4) * Dv * sizeof(float4);
    if (!gated) {
        const int need = (Dv + 31) / 32;
#define DIT_VPL_CASE(V) \
    if (need <= V) return {adaln_rows_kernel<V, TOK>, kThreads, mod};
        DIT_VPL_CASE(1) DIT_VPL_CASE(2) DIT_VPL_CASE(3) DIT_VPL_CASE(4) DIT_VPL_CASE(6)
        DIT_VPL_CASE(8) DIT_VPL_CASE(10) DIT_VPL_CASE(12) DIT_VPL_CASE(16) DIT_VPL_CASE(20)
        DIT_VPL_CASE(24) DIT_VPL_CASE(32)
#undef DIT_VPL_CASE
        return {nullptr, 0, 0};
    }
    const int need = (Dv + 63) / 64;   // a warp pair shares a row
    // 24 warps (80 registers each) for short rows; the per-token form keeps
    // 16, since its second code path spills at 80 registers
#define DIT_VPL_CASE(V)                                                                   \
    if (need <= V) {                                                                      \
        constexpr int WG = (V <= 10 && !TOK) ? 24 : 16;                                   \
        return {gated_rows_kernel<V, WG, TOK>, WG * 32,                                   \
                mod + static_cast<size_t>(WG) * V * 32 * sizeof(uint4)};                  \
    }
    DIT_VPL_CASE(1) DIT_VPL_CASE(2) DIT_VPL_CASE(3) DIT_VPL_CASE(4) DIT_VPL_CASE(5)
    DIT_VPL_CASE(6) DIT_VPL_CASE(8) DIT_VPL_CASE(10) DIT_VPL_CASE(12) DIT_VPL_CASE(16)
#undef DIT_VPL_CASE
    return {nullptr, 0, 0};
}

int launch_rows(const RowParams& p, bool gated, int B, cudaStream_t stream) {
    RowLaunch L = p.set_index ? pick_kernel<true>(gated, p.Dv)
                              : pick_kernel<false>(gated, p.Dv);
    if (L.kernel && !gated && p.staged_sets > 1) L.smem *= 2;     // the second staged set
    if (!L.kernel) return DIT_ERR_SHAPE;
    // opt in whenever dynamic shared memory is used (static arrays count
    // toward the 48 KB default too)
    if (L.smem > 0 &&
        cudaFuncSetAttribute(L.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(L.smem)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    const int sms = device_sm_count();
    if (sms <= 0) return DIT_ERR_LAUNCH;
    const int occ = occupancy(reinterpret_cast<const void*>(L.kernel), L.threads, L.smem);
    int64_t per_sample = (static_cast<int64_t>(sms) * occ) / B;
    if (per_sample < 1) per_sample = 1;
    const int rows_per_cta = gated ? L.threads / 64 : L.threads / 32;
    const int64_t need = (p.N + rows_per_cta - 1) / rows_per_cta;
    if (per_sample > need) per_sample = need;
    dim3 grid(static_cast<unsigned>(per_sample), static_cast<unsigned>(B));
    L.kernel<<<grid, L.threads, L.smem, stream>>>(p);
    return launch_status();
}

int check_mod(const void* p, int dtype) {
    if (!p) return DIT_ERR_NULL;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if (a % (dtype == DIT_F32 ? 4 : 2)) return DIT_ERR_ALIGN;
    return DIT_OK;
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

// Per-token sets: the index and its set stride; whether every set's
// vectors are 16-byte aligned for vector reads.
int set_checks(RowParams& p, const uint8_t* set_index, int n_sets, int64_t set_stride,
               const void* const* mods, int n_mods) {
    if (!set_index) return DIT_ERR_NULL;
    if (n_sets < 1 || n_sets > 255 || set_stride < 0) return DIT_ERR_SHAPE;
    p.set_index = set_index;
    p.n_sets = n_sets;
    p.set_stride = set_stride;
    const int per16 = p.mod_dtype == DIT_F32 ? 4 : 8;     // elements per 16 bytes
    bool vec = p.mod_stride % per16 == 0 && set_stride % per16 == 0;
    for (int i = 0; i < n_mods; ++i) vec = vec && aligned16(mods[i]);
    p.mod_vec = vec;
    // AdaLN stages set 1 beside set 0 when both fit in about 100 KB
    // (2 CTAs per SM); the gated form keeps its shared memory for the stage
    p.staged_sets = (n_mods == 2 && n_sets >= 2 &&
                     2 * static_cast<size_t>(p.Dv) * 4 * sizeof(float4) <= 100 * 1024)
                        ? 2
                        : 1;
    return DIT_OK;
}

}  // namespace
}  // namespace dit

extern "C" int dit_adaln_modulate_tok(const uint16_t* x, uint16_t* y, const void* shift,
                                      const void* scale, int mod_dtype, int64_t mod_batch_stride,
                                      int64_t mod_set_stride, const uint8_t* set_index,
                                      int n_sets, int B, int64_t N, int D, double eps,
                                      void* stream) {
    using namespace dit;
    int st = common_checks(B, N, D, mod_dtype, mod_batch_stride, eps);
    if (st) return st;
    if (set_index && (n_sets < 1 || n_sets > 255 || mod_set_stride < 0)) return DIT_ERR_SHAPE;
    if (B == 0 || N == 0) return DIT_OK;
    if (!x || !y) return DIT_ERR_NULL;
    if ((st = check_mod(shift, mod_dtype)) || (st = check_mod(scale, mod_dtype))) return st;
    if (!aligned16(x) || !aligned16(y)) return DIT_ERR_ALIGN;
    const size_t bytes = static_cast<size_t>(B) * N * D * 2;
    if (x != y && overlaps(x, bytes, y, bytes)) return DIT_ERR_OVERLAP;
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
    if (set_index) {
        const void* mods[2] = {shift, scale};
        if ((st = set_checks(p, set_index, n_sets, mod_set_stride, mods, 2))) return st;
    }
    return launch_rows(p, false, B, as_stream(stream));
}

extern "C" int dit_adaln_modulate(const uint16_t* x, uint16_t* y, const void* shift,
                                  const void* scale, int mod_dtype, int64_t mod_batch_stride,
                                  int B, int64_t N, int D, double eps, void* stream) {
    return dit_adaln_modulate_tok(x, y, shift, scale, mod_dtype, mod_batch_stride, 0, nullptr,
                                  1, B, N, D, eps, stream);
}

extern "C" int dit_gated_residual_adaln_tok(const uint16_t* x, const uint16_t* r,
                                            uint16_t* x_out, uint16_t* y, const void* gate,
                                            const void* shift, const void* scale, int mod_dtype,
                                            int64_t mod_batch_stride, int64_t mod_set_stride,
                                            const uint8_t* set_index, int n_sets, int B,
                                            int64_t N, int D, double eps, void* stream) {
    using namespace dit;
    int st = common_checks(B, N, D, mod_dtype, mod_batch_stride, eps);
    if (st) return st;
    if (set_index && (n_sets < 1 || n_sets > 255 || mod_set_stride < 0)) return DIT_ERR_SHAPE;
    if (B == 0 || N == 0) return DIT_OK;
    if (!x || !r || !x_out || !y) return DIT_ERR_NULL;
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
    if (set_index) {
        const void* mods[3] = {gate, shift, scale};
        if ((st = set_checks(p, set_index, n_sets, mod_set_stride, mods, 3))) return st;
    }
    return launch_rows(p, true, B, as_stream(stream));
}

extern "C" int dit_gated_residual_adaln(const uint16_t* x, const uint16_t* r, uint16_t* x_out,
                                        uint16_t* y, const void* gate, const void* shift,
                                        const void* scale, int mod_dtype,
                                        int64_t mod_batch_stride, int B, int64_t N, int D,
                                        double eps, void* stream) {
    return dit_gated_residual_adaln_tok(x, r, x_out, y, gate, shift, scale, mod_dtype,
                                        mod_batch_stride, 0, nullptr, 1, B, N, D, eps, stream);
}
