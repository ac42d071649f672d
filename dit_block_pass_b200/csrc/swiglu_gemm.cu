// swiglu_gemm.cu -- SwiGLU fused into the up-projection GEMM on the sm_100
// tensor cores: out[m, j] = silu(x W_gate^T)[m, j] * (x W_lin^T)[m, j],
// written once in bf16; the [M, 2F] product never reaches HBM.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração somadas chega-se a 6 vezes",
// names SwiGLU among the fused operators; "SGLang acelera MiniMax-H3 em GPUs
// H200", first paragraph, says the fusion cuts memory traffic and launches.
// Fusing the activation into the GEMM that produces its input is the step
// beyond the one-pass SwiGLU kernel: the 2F-wide product is consumed in the
// accumulator.
//
// Design: persistent, one CTA of 10 warps per SM, output tiles of 256 rows x
// 128 (SwiGLU) or 256 (gated residual) columns taken in a static round robin:
//   warp 0   TMA producer: per 64-wide K step, two 128 x 64 tiles of x (rows
//            m0.. and m0 + 128..) and two 128 x 64 tiles of W (the gate rows
//            n0.. and the linear rows F + n0..) land in a 3-stage ring of
//            64 KB stages (128-byte swizzle), completing a transaction-count
//            mbarrier.  The ring runs on across tiles.
//   warp 1   allocates all 512 TMEM columns and issues tcgen05.mma from one
//            thread: kind::f16, M = 128, N = 256 (gate and linear tiles side
//            by side), K = 16, two MMAs per K slice (one per 128-row half,
//            both reading the same W tile: 131 flop per staged byte), four
//            slices per stage.  tcgen05.commit frees each stage when its
//            MMAs have read it and hands the finished accumulators to the
//            epilogue.
//   warps 2-9 epilogue: two warps per TMEM lane quarter, each taking half
//            of the column chunks; tcgen05.ld pulls 32 accumulators per
//            thread (thread = output row): gate and the matching linear
//            columns -> silu(g) * u, or output columns -> x + gate * acc
//            (gate rows read 16 bytes at a time when aligned); one rounding
//            to bf16, 64-byte row segments to HBM.  Each 128-row half goes
//            back to the MMA warp once its last columns are in registers
//            (half 0 first), so the next tile's first K steps run on half 0
//            while half 1 drains; the producer has meanwhile filled the ring.
// Tiles are numbered in groups of row tiles (column tiles outer within a
// group) so that the tiles in flight share their x and W tiles in L2.  x, W
// tiles beyond M, K or F are zero-filled by TMA; stores past M or F are
// skipped.  The SwiGLU form runs at the sustained tensor peak of B200 (raster
// groups, streaming stores and the epilogue width measured within noise
// there); the heavier residual epilogue gained 8 % from the second epilogue
// warp per lane quarter and vector gate loads.
//
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the CTA
// records an error in the caller's status word, drains what it issued
// (bounded as well), frees its TMEM and exits.  No cluster launch: every TMA
// load fills this CTA's own shared memory.
#include "tcgen05.cuh"

namespace dit {
namespace {

constexpr int kHalves = 2;                  // 128-row MMAs per tile (sharing the W tile)
constexpr int kBM = 128 * kHalves;          // output rows per tile
constexpr int kBN = 128;                    // output columns per tile (each W half)
constexpr int kBK = 64;                     // K per stage: one 128-byte swizzle row
constexpr int kStages = kHalves == 2 ? 3 : 4;
constexpr int kEpiWarps = 8;
constexpr int kThreadsG = 64 + 32 * kEpiWarps;
// Raster groups (row tiles whose column tiles run together so that the tiles
// in flight share their x and W tiles in L2), measured at the H3 shapes:
// SwiGLU [124992, 5120] x [27648, 5120]^T best at 8-12 (16 and more thrash L2:
// 32 cost 12 %, 64 cost 24 %), the down-projection [124992, 13824] x
// [5120, 13824]^T best at 4 (3, 5, 6, 7: +1-2 %; 8: +2-4 %, 16: +8 %).
// Outputs do not depend on it.
#ifndef GEMM_GROUP_SWIGLU
#define GEMM_GROUP_SWIGLU 12
#endif
#ifndef GEMM_GROUP_RESID
#define GEMM_GROUP_RESID 4
#endif
constexpr uint32_t kTileA = kBM * kBK * 2;            // 16 KB per 128 rows
constexpr uint32_t kTileB = 2 * kBN * kBK * 2;        // 32 KB (gate + linear)
constexpr uint32_t kStageBytes = kTileA + kTileB;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256 * kHalves;          // accumulator columns per tile
constexpr uint32_t kAccBufs = kTmemCols / kAccCols;   // tiles in TMEM at once
constexpr size_t kSmemBytes = kStages * kStageBytes + 1024 /*alignment*/ + 256 /*barriers*/;

using namespace tc;

// Instruction descriptor: fp32 accumulator, bf16 K-major A and B, M = 128,
// N = 256.
constexpr uint32_t kIdesc = idesc_f16(128, 256, false, false);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db,
                                         uint32_t accumulate) {
    mma_f16(tmem_d, da, db, kIdesc, accumulate);
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// Epilogues of the one main loop.
enum Epilogue {
    kSwiGLU = 0,            // out[m, j] = silu(acc[m, j]) * acc[m, 128 + j]: 128 outputs per tile
    kGatedResidual = 1,     // out[m, n] = x[m, n] + gate_b[n] * acc[m, n]: 256 outputs per tile
};

struct GemmParams {
    uint16_t* out;
    int* status;            // device word, set to 1 when a wait expires (may be NULL)
    int M, K;
    int cols;               // output columns (F, or D)
    int tiles_m, tiles_n, tiles;
    int group_m;            // raster group: row tiles whose column tiles run together
    int b1_offset;          // row of the second W box relative to the first (0: own map)
    int stall;              // test hook: the producer issues nothing, every wait runs out
    // gated residual
    const uint16_t* x;      // [M, cols] residual stream (may be out)
    const void* gate;       // [B, cols] per-sample gate, fp32 or bf16
    int gate_dtype;
    int64_t gate_stride;
    int64_t tokens;         // token rows per sample
    bool gate_vec;          // every gate row is 16-byte aligned
};

// Output tile of linear tile id t: groups of kGroupM row tiles, the column
// tiles outer within a group, so that the tiles in flight at one time share
// their x and W tiles in L2.
template <int EPI>
__device__ __forceinline__ void tile_coords(const GemmParams& p, int t, int& m0, int& n0) {
    const int per_group = p.group_m * p.tiles_n;
    const int group = t / per_group;
    const int first_m = group * p.group_m;
    const int gsize = min(p.tiles_m - first_m, p.group_m);
    const int in_group = t - group * per_group;
    m0 = (first_m + in_group % gsize) * kBM;
    n0 = (in_group / gsize) * (EPI == kSwiGLU ? kBN : 2 * kBN);
}

__device__ __forceinline__ float gate_at(const GemmParams& p, int64_t off) {
    if (p.gate_dtype == DIT_F32) return __ldg(static_cast<const float*>(p.gate) + off);
    return __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const uint16_t*>(p.gate) + off))
                           << 16);
}

// bf16(x + g * a) for two elements with one rounding of each fp32-exact
// value: the fp32 fma rounds once, and rounding that to bf16 can differ from
// rounding the fma's exact value only on an exact bf16 tie (low half
// 0x8000); that pair is redone in fp64, where g * a (fp32 x fp32) is exact.
__device__ __noinline__ uint32_t resid_pair_fp64(float x0, float g0, float a0, float x1, float g1,
                                                 float a1) {
    const __nv_bfloat16 lo = __double2bfloat16(
        fma(static_cast<double>(g0), static_cast<double>(a0), static_cast<double>(x0)));
    const __nv_bfloat16 hi = __double2bfloat16(
        fma(static_cast<double>(g1), static_cast<double>(a1), static_cast<double>(x1)));
    return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

__device__ __forceinline__ uint32_t resid_pair(uint32_t xw, float g0, float a0, float g1,
                                               float a1) {
    const float x0 = bf16_lo(xw), x1 = bf16_hi(xw);
    const float s0 = __fmaf_rn(g0, a0, x0);
    const float s1 = __fmaf_rn(g1, a1, x1);
    if (((__float_as_uint(s0) & 0xFFFFu) == 0x8000u) | ((__float_as_uint(s1) & 0xFFFFu) == 0x8000u))
        return resid_pair_fp64(x0, g0, a0, x1, g1, a1);
    return pack2(s0, s1);
}

// Persistent: CTA b takes tiles b, b + gridDim.x, ...  The K-step ring runs
// across tiles, and the two accumulator halves (TMEM columns [0, 256) and
// [256, 512)) are released separately, so the epilogue of one tile overlaps
// the first K steps of the next.
template <int EPI>
__global__ void __launch_bounds__(kThreadsG, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_x,
            const __grid_constant__ CUtensorMap map_wg,
            const __grid_constant__ CUtensorMap map_wu, GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned stages (the swizzle atom), barriers after them
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gen_base = smem_raw + (base - raw);
    const uint32_t bar_full = base + kStages * kStageBytes;      // kStages x 8 bytes
    const uint32_t bar_empty = bar_full + 8 * kStages;           // kStages x 8 bytes
    const uint32_t bar_tfull = bar_empty + 8 * kStages;          // 2 x 8: accumulator ready
    const uint32_t bar_tempty = bar_tfull + 16;                  // 2 x 8: half h drained
    const uint32_t bar_drain = bar_tempty + 16;
    uint8_t* tail = gen_base + kStages * kStageBytes + 16 * kStages + 40;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(tail);
    volatile int* abort = reinterpret_cast<volatile int*>(tail + 4);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nk = (p.K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (uint32_t a = 0; a < kAccBufs; ++a) mbar_init(bar_tfull + 8 * a, 1);
        for (int h = 0; h < kHalves; ++h)
            mbar_init(bar_tempty + 8 * h, kEpiWarps);   // one arrival per epilogue warp
        mbar_init(bar_drain, 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(const_cast<uint32_t*>(tmem_slot))),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool failed = false;

    if (warp == 0) {
        if (lane == 0) {
            // producer: K steps of every tile, through the ring
            uint32_t it = 0;
            for (int t = blockIdx.x; t < p.tiles && !failed && !p.stall; t += gridDim.x) {
                int m0, n0;
                tile_coords<EPI>(p, t, m0, n0);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const uint32_t s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, abort)) {
                        failed = true;
                        break;
                    }
                    const uint32_t sa = base + s * kStageBytes;
                    mbar_expect_tx(bar_full + 8 * s, kStageBytes);
#pragma unroll
                    for (int h = 0; h < kHalves; ++h)
                        tma_load_2d(sa + h * (kTileA / kHalves), &map_x, bar_full + 8 * s,
                                    kb * kBK, m0 + 128 * h);
                    tma_load_2d(sa + kTileA, &map_wg, bar_full + 8 * s, kb * kBK, n0);
                    tma_load_2d(sa + kTileA + kTileB / 2, &map_wu, bar_full + 8 * s, kb * kBK,
                                n0 + p.b1_offset);
                }
            }
            if (failed) {
                // let the copies already issued land before the CTA exits
                for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
                    mbar_wait_drain(bar_full + 8 * (j % kStages), (j / kStages) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer.  The accumulator holds both 128-row halves of a tile
            // (all 512 columns); the epilogue releases each half on its own
            // barrier, half 0 first.  A tile starts once half 0 is free: its
            // first K steps issue half 0's products only and keep their ring
            // stages until half 1 is free too (at most kStages of them), then
            // half 1 catches up in K order, so the epilogue of the previous
            // tile overlaps the start of this one.
            uint32_t it = 0, local = 0;
            for (int t = blockIdx.x; t < p.tiles && !failed; t += gridDim.x, ++local) {
                const uint32_t free_ph = (local & 1u) ^ 1u;    // the first tile passes
                if (!mbar_wait(bar_tempty, free_ph, abort)) {
                    failed = true;
                    break;
                }
                fence_after_sync();
                bool h1 = mbar_test(bar_tempty + 8, free_ph);
                if (h1) fence_after_sync();
                const uint32_t it0 = it;
                int pend = 0;                   // first K step whose half-1 products are not issued
                auto issue_half = [&](int kb, int h) {
                    const uint32_t sa = base + ((it0 + kb) % kStages) * kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_bf16(tmem + 256u * h, sw128_desc(sa + h * (kTileA / kHalves) + kk * 32),
                                 sw128_desc(sa + kTileA + kk * 32), (kb | kk) != 0 ? 1u : 0u);
                };
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const uint32_t s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(bar_full + 8 * s, ph, abort)) {
                        failed = true;
                        break;
                    }
                    fence_after_sync();
                    issue_half(kb, 0);
                    if (!h1) {
                        h1 = mbar_test(bar_tempty + 8, free_ph);
                        // every ring stage is held: half 1 must be free before the next step
                        if (!h1 && kb + 1 - pend >= kStages) {
                            if (!mbar_wait(bar_tempty + 8, free_ph, abort)) {
                                failed = true;
                                break;
                            }
                            h1 = true;
                        }
                        if (h1) fence_after_sync();
                    }
                    if (h1) {
                        for (; pend <= kb; ++pend) {
                            issue_half(pend, 1);
                            // stage free once both halves' products have read it
                            mma_commit(bar_empty + 8 * ((it0 + pend) % kStages));
                        }
                    }
                }
                if (!failed && pend < nk) {
                    if (!mbar_wait(bar_tempty + 8, free_ph, abort)) {
                        failed = true;
                    } else {
                        fence_after_sync();
                        for (; pend < nk; ++pend) {
                            issue_half(pend, 1);
                            mma_commit(bar_empty + 8 * ((it0 + pend) % kStages));
                        }
                    }
                }
                if (!failed) mma_commit(bar_tfull);
            }
            if (failed) {
                // every MMA issued has finished when this commit arrives
                mma_commit(bar_drain);
                mbar_wait_drain(bar_drain, 0);
            }
        }
        __syncwarp();
    } else {
        // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31
        const int q = warp & 3;
        const int cg = (warp - 2) / 4;          // which share of the column chunks
        uint32_t local = 0;
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++local) {
            int m0, n0;
            tile_coords<EPI>(p, t, m0, n0);
            const uint32_t acc = local % kAccBufs;
            if (!mbar_wait(bar_tfull + 8 * acc, (local / kAccBufs) & 1u, abort)) {
                failed = true;
                break;
            }
            fence_after_sync();
            // SwiGLU: per half, 4 chunks of 32 gate + 32 linear columns;
            // gated residual: per half, 8 chunks of 32 output columns
            constexpr int kAll = EPI == kSwiGLU ? kBN / 32 : 2 * kBN / 32;
            constexpr int kPer = kAll / (kEpiWarps / 4);
#pragma unroll 1
            for (int hc = 0; hc < kHalves * kPer; ++hc) {
                const int h = hc / kPer, c = kPer * cg + hc % kPer;
                const int row = m0 + 128 * h + 32 * q + lane;
                const uint32_t lane_addr =
                    tmem + acc * kAccCols + 256u * h + (static_cast<uint32_t>(32 * q) << 16);
                float g[32], u[32];
                tmem_ld32(lane_addr + 32 * c, g);
                if (EPI == kSwiGLU) tmem_ld32(lane_addr + kBN + 32 * c, u);
                tmem_wait_ld();
                if (hc % kPer == kPer - 1) {
                    // this half's columns are all in registers: hand it back
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0)
                        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                                         bar_tempty + 8 * h)
                                     : "memory");
                }
                if (row < p.M) {
                    const int col0 = n0 + 32 * c;
                    uint16_t* dst = p.out + static_cast<int64_t>(row) * p.cols + col0;
                    if (EPI == kSwiGLU) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            if (col0 + 8 * v < p.cols) {
                                float o[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    o[i] = silu_mul(g[8 * v + i], u[8 * v + i]);
                                *reinterpret_cast<uint4*>(dst + 8 * v) = pack8(o);
                            }
                        }
                    } else {
                        const uint16_t* xs = p.x + static_cast<int64_t>(row) * p.cols + col0;
                        const int64_t goff = (row / p.tokens) * p.gate_stride + col0;
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            if (col0 + 8 * v < p.cols) {
                                const uint4 xv = *reinterpret_cast<const uint4*>(xs + 8 * v);
                                float gv[8];
                                if (p.gate_vec) {
                                    if (p.gate_dtype == DIT_F32) {
                                        const float4* gp = reinterpret_cast<const float4*>(
                                            static_cast<const float*>(p.gate) + goff + 8 * v);
                                        const float4 ga = __ldg(gp), gb = __ldg(gp + 1);
                                        gv[0] = ga.x; gv[1] = ga.y; gv[2] = ga.z; gv[3] = ga.w;
                                        gv[4] = gb.x; gv[5] = gb.y; gv[6] = gb.z; gv[7] = gb.w;
                                    } else {
                                        unpack8(__ldg(reinterpret_cast<const uint4*>(
                                                    static_cast<const uint16_t*>(p.gate) + goff +
                                                    8 * v)),
                                                gv);
                                    }
                                } else {
#pragma unroll
                                    for (int i = 0; i < 8; ++i) gv[i] = gate_at(p, goff + 8 * v + i);
                                }
                                const float* a = g + 8 * v;
                                uint4 o;
                                o.x = resid_pair(xv.x, gv[0], a[0], gv[1], a[1]);
                                o.y = resid_pair(xv.y, gv[2], a[2], gv[3], a[3]);
                                o.z = resid_pair(xv.z, gv[4], a[4], gv[5], a[5]);
                                o.w = resid_pair(xv.w, gv[6], a[6], gv[7], a[7]);
                                *reinterpret_cast<uint4*>(dst + 8 * v) = o;
                            }
                        }
                    }
                }
            }
        }
    }
    if (failed) {
        *abort = 1;
        if (p.status) atomicExch(p.status, 1);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
}

// ------------------------------------------------------------------ host

}  // namespace
}  // namespace dit

namespace dit {
namespace {

// Shared launch: x [M, K], two W views for the B tile's halves, epilogue EPI.
template <int EPI>
int launch_gemm(const uint16_t* x, const uint16_t* w0, int64_t w0_rows, const uint16_t* w1,
                int64_t w1_rows, GemmParams& p, int64_t M, int K, int cols, void* stream) {
    CUtensorMap mx, m0, m1;
    if (!make_map(&mx, x, M, K, K) || !make_map(&m0, w0, w0_rows, K, K) ||
        !make_map(&m1, w1, w1_rows, K, K))
        return DIT_ERR_LAUNCH;
    p.M = static_cast<int>(M);
    p.K = K;
    p.cols = cols;
    p.tiles_m = static_cast<int>((M + kBM - 1) / kBM);
    const int tile_cols = EPI == kSwiGLU ? kBN : 2 * kBN;
    p.tiles_n = (cols + tile_cols - 1) / tile_cols;
    const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
    if (tiles > 0x7FFFFFFF) return DIT_ERR_SHAPE;
    p.tiles = static_cast<int>(tiles);
    p.group_m = EPI == kSwiGLU ? GEMM_GROUP_SWIGLU : GEMM_GROUP_RESID;
    const int sms = device_sm_count();
    if (sms <= 0) return DIT_ERR_LAUNCH;
    const int64_t ctas = tiles < sms ? tiles : sms;     // one persistent CTA per SM
    if (cudaFuncSetAttribute(gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    gemm_kernel<EPI><<<static_cast<unsigned>(ctas), kThreadsG, kSmemBytes, as_stream(stream)>>>(
        mx, m0, m1, p);
    return launch_status();
}

}  // namespace
}  // namespace dit

extern "C" int dit_swiglu_gemm(const uint16_t* x, const uint16_t* w, uint16_t* out, int64_t M,
                               int K, int F, int* status, void* stream) {
    using namespace dit;
    if (M < 0 || K <= 0 || F <= 0) return DIT_ERR_SHAPE;
    if (K % 8 || F % 8) return DIT_ERR_ALIGN;
    if (M > 0x7FFFFFFFLL - kBM || F > (1 << 30) / 2) return DIT_ERR_SHAPE;
    if (M == 0) return DIT_OK;
    if (!x || !w || !out) return DIT_ERR_NULL;
    if (!aligned16(x) || !aligned16(w) || !aligned16(out)) return DIT_ERR_ALIGN;
    if (status && reinterpret_cast<uintptr_t>(status) % 4) return DIT_ERR_ALIGN;
    const size_t out_bytes = static_cast<size_t>(M) * F * 2;
    if (overlaps(out, out_bytes, x, static_cast<size_t>(M) * K * 2) ||
        overlaps(out, out_bytes, w, static_cast<size_t>(2) * F * K * 2))
        return DIT_ERR_OVERLAP;
    GemmParams p{};
    p.out = out;
    p.status = status;
    p.b1_offset = 0;
    return launch_gemm<kSwiGLU>(x, w, F, w + static_cast<int64_t>(F) * K, F, p, M, K, F, stream);
}

extern "C" int dit_swiglu_gemm_stall_test(const uint16_t* x, const uint16_t* w, uint16_t* out,
                                          int64_t M, int K, int F, int* status, void* stream) {
    using namespace dit;
    if (M <= 0 || M > 4096 || K <= 0 || K > 4096 || F <= 0 || F > 4096) return DIT_ERR_SHAPE;
    if (K % 8 || F % 8) return DIT_ERR_ALIGN;
    if (!x || !w || !out || !status) return DIT_ERR_NULL;
    if (!aligned16(x) || !aligned16(w) || !aligned16(out) ||
        reinterpret_cast<uintptr_t>(status) % 4)
        return DIT_ERR_ALIGN;
    GemmParams p{};
    p.out = out;
    p.status = status;
    p.stall = 1;
    return launch_gemm<kSwiGLU>(x, w, F, w + static_cast<int64_t>(F) * K, F, p, M, K, F, stream);
}

extern "C" int dit_gemm_gated_residual(const uint16_t* h, const uint16_t* w, const uint16_t* x,
                                       uint16_t* x_out, const void* gate, int gate_dtype,
                                       int64_t gate_batch_stride, int B, int64_t N, int K, int D,
                                       int* status, void* stream) {
    using namespace dit;
    if (B < 0 || N < 0 || K <= 0 || D <= 0 || gate_batch_stride < 0) return DIT_ERR_SHAPE;
    if (gate_dtype != DIT_F32 && gate_dtype != DIT_BF16) return DIT_ERR_DTYPE;
    if (K % 8 || D % 8) return DIT_ERR_ALIGN;
    const int64_t M = static_cast<int64_t>(B) * N;
    if (M > 0x7FFFFFFFLL - kBM || D > (1 << 30)) return DIT_ERR_SHAPE;
    if (M == 0) return DIT_OK;
    if (!h || !w || !x || !x_out || !gate) return DIT_ERR_NULL;
    if (!aligned16(h) || !aligned16(w) || !aligned16(x) || !aligned16(x_out)) return DIT_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(gate) % (gate_dtype == DIT_F32 ? 4 : 2)) return DIT_ERR_ALIGN;
    if (status && reinterpret_cast<uintptr_t>(status) % 4) return DIT_ERR_ALIGN;
    const size_t xb = static_cast<size_t>(M) * D * 2;
    // x_out may be x itself (each element is read, then written, by one thread)
    if ((x_out != x && overlaps(x_out, xb, x, xb)) ||
        overlaps(x_out, xb, h, static_cast<size_t>(M) * K * 2) ||
        overlaps(x_out, xb, w, static_cast<size_t>(D) * K * 2))
        return DIT_ERR_OVERLAP;
    GemmParams p{};
    p.out = x_out;
    p.status = status;
    p.b1_offset = kBN;                 // the tile's second 128 rows of the same W
    p.x = x;
    p.gate = gate;
    p.gate_dtype = gate_dtype;
    p.gate_stride = gate_batch_stride;
    p.tokens = N;
    p.gate_vec = aligned16(gate) && gate_batch_stride % (gate_dtype == DIT_F32 ? 4 : 8) == 0;
    return launch_gemm<kGatedResidual>(h, w, D, w, D, p, M, K, D, stream);
}
