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
//            to bf16, 64-byte row segments to HBM.  Once the last columns
//            are in registers the accumulators go back to the MMA warp; the
//            producer has meanwhile filled the ring for the next tile.
// Tiles are numbered in groups of 8 row tiles (column tiles outer within a
// group) so that the tiles in flight share their x and W tiles in L2.  x, W
// tiles beyond M, K or F are zero-filled by TMA; stores past M or F are
// skipped.  The SwiGLU form runs at the sustained tensor peak of B200 (raster
// groups, streaming stores and the epilogue width measured within noise
// there); the heavier residual epilogue gained 8 % from the second epilogue
// warp per lane quarter and vector gate loads.
//
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the CTA
// records an error in the caller's status word, drains what it issued
// (bounded as well), frees its TMEM and exits.  No cluster, no multicast.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace dit {
namespace {

constexpr int kHalves = 2;                  // 128-row MMAs per tile (sharing the W tile)
constexpr int kBM = 128 * kHalves;          // output rows per tile
constexpr int kBN = 128;                    // output columns per tile (each W half)
constexpr int kBK = 64;                     // K per stage: one 128-byte swizzle row
constexpr int kStages = kHalves == 2 ? 3 : 4;
constexpr int kEpiWarps = 8;
constexpr int kThreadsG = 64 + 32 * kEpiWarps;
constexpr int kGroupM = 16 / kHalves;       // raster group (row tiles)
constexpr uint32_t kTileA = kBM * kBK * 2;            // 16 KB per 128 rows
constexpr uint32_t kTileB = 2 * kBN * kBK * 2;        // 32 KB (gate + linear)
constexpr uint32_t kStageBytes = kTileA + kTileB;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256 * kHalves;          // accumulator columns per tile
constexpr uint32_t kAccBufs = kTmemCols / kAccCols;   // tiles in TMEM at once
constexpr size_t kSmemBytes = kStages * kStageBytes + 1024 /*alignment*/ + 256 /*barriers*/;
constexpr unsigned long long kWaitNs = 2000000000ull;

// ----------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete, for at most
// kWaitNs, or until another role of the CTA has given up (*abort != 0).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
    const unsigned long long t0 = now_ns();
    for (uint32_t i = 0;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 255u) == 255u) {
            if (*abort) return false;
            if (now_ns() - t0 > kWaitNs) return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows
// of 128 bytes in groups of 8 (1024 bytes apart).  Fields: start address,
// leading offset (16 bytes), stride offset (1024 bytes), all >> 4; version
// 1; layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(16u >> 4) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) |
                            ((128u >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                     "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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
    int b1_offset;          // row of the second W box relative to the first (0: own map)
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
    const int per_group = kGroupM * p.tiles_n;
    const int group = t / per_group;
    const int first_m = group * kGroupM;
    const int gsize = min(p.tiles_m - first_m, kGroupM);
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

// Persistent: CTA b takes tiles b, b + gridDim.x, ...  The K-step ring and
// the two accumulators (TMEM columns [0, 256) and [256, 512)) run across
// tiles, so the epilogue of one tile overlaps the main loop of the next.
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
    const uint32_t bar_tempty = bar_tfull + 16;                  // 2 x 8: accumulator drained
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
        for (uint32_t a = 0; a < kAccBufs; ++a) {
            mbar_init(bar_tfull + 8 * a, 1);
            mbar_init(bar_tempty + 8 * a, kEpiWarps);   // one arrival per epilogue warp
        }
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
            for (int t = blockIdx.x; t < p.tiles && !failed; t += gridDim.x) {
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
                    mbar_wait(bar_full + 8 * (j % kStages), (j / kStages) & 1u, abort);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer
            uint32_t it = 0, local = 0;
            for (int t = blockIdx.x; t < p.tiles && !failed; t += gridDim.x, ++local) {
                const uint32_t acc = local % kAccBufs;
                const uint32_t aph = (local / kAccBufs) & 1u;
                // the epilogue has drained this accumulator (the first use passes)
                if (!mbar_wait(bar_tempty + 8 * acc, aph ^ 1u, abort)) {
                    failed = true;
                    break;
                }
                fence_after_sync();
                const uint32_t d = tmem + acc * kAccCols;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const uint32_t s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(bar_full + 8 * s, ph, abort)) {
                        failed = true;
                        break;
                    }
                    fence_after_sync();
                    const uint32_t sa = base + s * kStageBytes;
                    const uint32_t sb = sa + kTileA;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
                        for (int h = 0; h < kHalves; ++h)
                            mma_bf16(d + 256u * h, sw128_desc(sa + h * (kTileA / kHalves) + kk * 32),
                                     sw128_desc(sb + kk * 32), (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(bar_empty + 8 * s);  // stage free once these MMAs read it
                }
                if (!failed) mma_commit(bar_tfull + 8 * acc);
            }
            if (failed) {
                // every MMA issued has finished when this commit arrives
                mma_commit(bar_drain);
                mbar_wait(bar_drain, 0, abort);
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
                if (hc == kHalves * kPer - 1) {
                    // every column of this accumulator is in registers: hand it back
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0)
                        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                                         bar_tempty + 8 * acc)
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

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
    static std::once_flag once;
    static EncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

// A [rows, K] bf16 row-major operand read in 64 x 128 boxes, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int K) {
    const EncodeTiled enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {kBK, 128};
    const cuuint32_t elem[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace dit

namespace dit {
namespace {

// Shared launch: x [M, K], two W views for the B tile's halves, epilogue EPI.
template <int EPI>
int launch_gemm(const uint16_t* x, const uint16_t* w0, int64_t w0_rows, const uint16_t* w1,
                int64_t w1_rows, GemmParams& p, int64_t M, int K, int cols, void* stream) {
    CUtensorMap mx, m0, m1;
    if (!make_map(&mx, x, M, K) || !make_map(&m0, w0, w0_rows, K) ||
        !make_map(&m1, w1, w1_rows, K))
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
