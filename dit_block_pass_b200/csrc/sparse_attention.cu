// sparse_attention.cu -- block-sparse attention over the SubBlock router's
// kept key blocks, on the sm_100 tensor cores.
//
// The LMSYS report summary at news.cocoloop.cn ("minimax-h3-sglang-h200"),
// section "Só com três camadas de aceleração somadas chega-se a 6 vezes":
// SubBlock attention lets a block-sparse router cut the KV blocks that take
// part in attention.  For token t of query block i and head h:
//     out[t, h] = sum_u softmax_u(scale * q[t, h] . k[u, h]) v[u, h]
// over the tokens u of the kept key blocks of (b, h, i); non-causal; blocks
// of 128 tokens, head size 128.
//
// Design: one CTA of 6 warps per (query block, head, sample), two CTAs per SM
// (96 KB of shared memory and 256 of the 512 TMEM columns each), so that one
// CTA's softmax runs while the other's products use the tensor cores:
//   warp 0    TMA: the 128 x 128 Q tile once, then K and V of each kept
//             block, one buffer each (128-byte swizzle): K_{n+1} lands while
//             block n's softmax runs, V_{n+1} while S_{n+1} and its softmax run.
//   warp 1    one thread issues tcgen05.mma: S_n = Q K_n^T (shared-memory
//             operands, fp32 into TMEM columns [0, 128)) as two N = 64 halves,
//             and, once the softmax has written P_n, O += P_n V_n with P read
//             from TMEM (the A operand in tensor memory, two bf16 per column
//             over S_n's first 64 columns) and V as an MN-major shared-memory
//             operand (no transpose).  Keys 64..127 of S_{n+1} go into the
//             columns P_n does not use as soon as the softmax has read S_n
//             (so they run during softmax n and P_n V_n); keys 0..63 follow
//             once P_n V_n has read P_n.
//   warps 2-5 softmax, thread = query row (TMEM lane): keys past the
//             sample's last token are set to -inf in TMEM (only a partial
//             block needs it), tcgen05.ld the S row (then report S_n read),
//             the row max of the raw scores in four chains of three-input
//             maxima, weights 2^(s * scale * log2 e - m) with one paired fma
//             per two weights and ex2.approx, row sums in paired adds, with
//             lazy rescaling (the reference max m moves, and O and
//             the row sum are rescaled in TMEM, only when a row's block max
//             exceeds m by more than 8, so weights stay below 2^8), and P
//             written back into TMEM as bf16 pairs.  At the end O / l is
//             written as bf16.
// Every mbarrier wait is bounded (tcgen05.cuh); on expiry the CTA records an
// error in the caller's status word and exits after freeing its TMEM.
#include "tcgen05.cuh"

namespace dit {
namespace {

using namespace tc;

constexpr int kBlk = 128;                       // tokens per block (rows of every tile)
constexpr int kHd = 128;                        // head size
constexpr int kThreadsA = 256;                  // two warpgroups
// Register split (setmaxnreg): the kernel is launched with 128 registers per
// thread (two CTAs of 256 threads fill the SM's 65,536); the copy/MMA
// warpgroup gives up to 40 and the softmax warpgroup takes 216, which adds up
// to the launch total: 128 * (40 + 216) = 256 * 128.
constexpr int kRegsLaunch = 128;
constexpr int kRegsLow = 56;
constexpr int kRegsHigh = 2 * kRegsLaunch - kRegsLow;
constexpr uint32_t kTile = kBlk * kHd * 2;      // 32 KB: one 128 x 128 bf16 tile
constexpr uint32_t kHalfTile = kTile / 2;       // 16 KB: 64 columns (one swizzle atom wide)
constexpr uint32_t kTmemColsA = 256;           // two CTAs share an SM's 512 columns
constexpr uint32_t kColO = 128;                 // S (and P over it) in [0, 128), O in [128, 256)
// Q, K, V, then barriers
constexpr size_t kSmemA = 3 * kTile + 1024 + 256;
constexpr uint32_t kIdescS64 = idesc_f16(128, 64, false, false);   // half of S = Q K^T
constexpr uint32_t kIdescO = idesc_f16(128, 128, false, true);     // O += P V (V MN-major)

// D (TMEM) += A (TMEM, K-major: row m in lane m, two bf16 per column) * B
// (shared-memory descriptor).
__device__ __forceinline__ void mma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

// fp32 pairs in one 64-bit register (sm_100 paired arithmetic).
__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack_f2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add_f2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// max of three (sm_100)
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// 2^x on the special-function unit, subnormal results flushed to zero (a
// weight below 2^-126 of the row's reference is lost in bf16 P anyway).
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// -inf into columns valid .. 127 of this warp's 32 rows of S (tensor
// memory address `row_base`): whole 32-column chunks at once, the chunk
// holding the boundary one column at a time.
__device__ __forceinline__ void mask_tail(uint32_t row_base, int valid) {
    float ninf[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) ninf[e] = -INFINITY;
    for (int c = 0; c < kBlk / 32; ++c) {
        const int c0 = 32 * c;
        if (c0 >= valid) {
            tmem_st32(row_base + c0, ninf);
        } else if (c0 + 32 > valid) {
            for (int col = valid; col < c0 + 32; ++col)
                asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(
                                 row_base + static_cast<uint32_t>(col)),
                             "r"(__float_as_uint(-INFINITY))
                             : "memory");
        }
    }
    tmem_wait_st();
}

// Keys k0 .. k0 + 63 of S = Q K^T (k0 = 0 or 64) into TMEM columns k0 ..
// k0 + 63: eight M = 128, N = 64, K = 16 products; rows k0.. of each 64-wide
// K half start k0 * 128 bytes in (a multiple of the 1024-byte swizzle atom).
__device__ __forceinline__ void issue_s(uint32_t tmem, uint32_t sQ, uint32_t sK, int k0) {
#pragma unroll
    for (int kk = 0; kk < kHd / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kHalfTile + (kk & 3) * 32;
        mma_f16(tmem + k0, sw128_desc(sQ + off), sw128_desc(sK + off + k0 * 128), kIdescS64,
                kk != 0 ? 1u : 0u);
    }
}

struct AttnParams {
    const int32_t* kept;        // [B, H, nb, n_keep]
    uint16_t* out;
    int64_t out_stride;         // elements between output rows
    int* status;
    int64_t N;
    int H, nb, n_keep;
    float scale_log2;           // scale * log2(e)
};

__global__ void __launch_bounds__(kThreadsA, 2)
block_sparse_attention_kernel(const __grid_constant__ CUtensorMap map_q,
                              const __grid_constant__ CUtensorMap map_k,
                              const __grid_constant__ CUtensorMap map_v, AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gen_base = smem_raw + (base - raw);
    const uint32_t sQ = base, sK = base + kTile, sV = base + 2 * kTile;
    const uint32_t bar = base + 3 * kTile;
    const uint32_t bar_q = bar;
    const uint32_t bar_k_full = bar + 8, bar_k_empty = bar + 16;
    const uint32_t bar_v_full = bar + 24, bar_v_empty = bar + 32;
    const uint32_t bar_s_full = bar + 40;           // S_n in TMEM
    const uint32_t bar_p_full = bar + 48;           // P_n in TMEM, O rescaled (4 arrivals)
    const uint32_t bar_o_done = bar + 56;           // P_n V_n done: S/P columns and O free
    const uint32_t bar_drain = bar + 64;
    const uint32_t bar_s_free = bar + 72;           // S_n read into registers (4 arrivals)
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gen_base + 3 * kTile + 80);
    volatile int* abort = reinterpret_cast<volatile int*>(gen_base + 3 * kTile + 84);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int nk = p.n_keep;
    const int32_t* kept = p.kept + ((static_cast<int64_t>(b) * p.H + h) * p.nb + i) * nk;
    const int row0 = static_cast<int>(static_cast<int64_t>(b) * p.N);   // first row of the sample

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_k_full, 1);
        mbar_init(bar_k_empty, 1);
        mbar_init(bar_v_full, 1);
        mbar_init(bar_v_empty, 1);
        mbar_init(bar_s_full, 1);
        mbar_init(bar_p_full, 4);
        mbar_init(bar_o_done, 1);
        mbar_init(bar_drain, 1);
        mbar_init(bar_s_free, 4);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), kTmemColsA);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool failed = false;

    if (warp < 4) {
    // copy and MMA warpgroup (warps 2 and 3 only wait at the end)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
        if (lane == 0) {
            // the Q tile, then K and V of every kept block (one buffer each:
            // K_{n+1} lands while the softmax of block n runs, V_{n+1} while
            // S_{n+1} and its softmax run)
            const int col = h * kHd;
            mbar_expect_tx(bar_q, kTile);
            tma_load_2d(sQ, &map_q, bar_q, col, row0 + i * kBlk);
            tma_load_2d(sQ + kHalfTile, &map_q, bar_q, col + 64, row0 + i * kBlk);
            int issued_k = 0, issued_v = 0;
            for (int n = 0; n < nk; ++n) {
                const int row = row0 + __ldg(kept + n) * kBlk;
                if (!mbar_wait(bar_k_empty, (n & 1) ^ 1, abort)) {
                    failed = true;
                    break;
                }
                mbar_expect_tx(bar_k_full, kTile);
                tma_load_2d(sK, &map_k, bar_k_full, col, row);
                tma_load_2d(sK + kHalfTile, &map_k, bar_k_full, col + 64, row);
                issued_k = n + 1;
                if (!mbar_wait(bar_v_empty, (n & 1) ^ 1, abort)) {
                    failed = true;
                    break;
                }
                mbar_expect_tx(bar_v_full, kTile);
                tma_load_2d(sV, &map_v, bar_v_full, col, row);
                tma_load_2d(sV + kHalfTile, &map_v, bar_v_full, col + 64, row);
                issued_v = n + 1;
            }
            mbar_wait_drain(bar_q, 0);           // the Q copy lands before the CTA exits
            if (failed) {
                if (issued_k) mbar_wait_drain(bar_k_full, (issued_k - 1) & 1);
                if (issued_v) mbar_wait_drain(bar_v_full, (issued_v - 1) & 1);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            if (!mbar_wait(bar_q, 0, abort)) failed = true;
            // S_0, both key halves
            if (!failed && nk > 0) {
                if (!mbar_wait(bar_k_full, 0, abort)) {
                    failed = true;
                } else {
                    fence_after_sync();
                    issue_s(tmem, sQ, sK, 64);
                    issue_s(tmem, sQ, sK, 0);
                    mma_commit(bar_s_full);
                    mma_commit(bar_k_empty);
                }
            }
            for (int n = 0; n < nk && !failed; ++n) {
                const bool more = n + 1 < nk;
                // keys 64..127 of S_{n+1} (columns P_n does not use) once the
                // softmax has read S_n and K_{n+1} is in, and P_n V_n once P_n
                // is written: whichever is ready first
                bool b_done = !more, pv_done = false;
                const unsigned long long t0 = now_ns();
                for (uint32_t it = 0; !(b_done && pv_done); ++it) {
                    if (!b_done && mbar_try(bar_s_free, n & 1) &&
                        mbar_try(bar_k_full, (n + 1) & 1)) {
                        fence_after_sync();
                        issue_s(tmem, sQ, sK, 64);
                        b_done = true;
                    }
                    if (!pv_done && mbar_try(bar_p_full, n & 1) && mbar_try(bar_v_full, n & 1)) {
                        fence_after_sync();
#pragma unroll
                        for (int kk = 0; kk < kBlk / 16; ++kk)
                            mma_f16_ts(tmem + kColO, tmem + 8 * kk,
                                       sw128_desc_mn(sV + kk * 2048, kHalfTile), kIdescO,
                                       (n | kk) != 0 ? 1u : 0u);
                        mma_commit(bar_o_done);
                        mma_commit(bar_v_empty);
                        pv_done = true;
                    }
                    if ((it & 255u) == 255u && (*abort || now_ns() - t0 > kWaitNs)) {
                        failed = true;
                        break;
                    }
                }
                if (failed || !more) continue;
                // keys 0..63 of S_{n+1} overwrite P_n: after P_n V_n has read it
                if (!mbar_wait(bar_o_done, n & 1, abort)) {
                    failed = true;
                    break;
                }
                fence_after_sync();
                issue_s(tmem, sQ, sK, 0);
                mma_commit(bar_s_full);
                mma_commit(bar_k_empty);
            }
            if (failed) {
                mma_commit(bar_drain);
                mbar_wait_drain(bar_drain, 0);
            }
        }
        __syncwarp();
    }
    } else {
        // softmax warpgroup: thread = query row r (TMEM lane)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
        float m_run = -INFINITY, l_run = 0.0f;
        for (int n = 0; n < nk; ++n) {
            // keys past the sample's last token do not take part
            const int64_t j = __ldg(kept + n);
            const int64_t left = p.N - j * kBlk;
            const int valid = left >= kBlk ? kBlk : (left > 0 ? static_cast<int>(left) : 0);
            if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full, n & 1, abort))) {
                failed = true;
                break;
            }
            fence_after_sync();
            // a sample's last block may be partial: its missing keys' scores
            // become -inf in tensor memory (the same block for every row, so
            // the branch is uniform), and full blocks need no mask at all
            if (valid < kBlk) mask_tail(tmem + lane_off, valid);
            float sc[kBlk];
#pragma unroll
            for (int c = 0; c < kBlk / 32; ++c)
                tmem_ld32(tmem + lane_off + 32 * c, *reinterpret_cast<float(*)[32]>(sc + 32 * c));
            tmem_wait_ld();
            // S_n is in registers: its columns 64..127 may take S_{n+1}
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_s_free);
            // the row max of the raw scores (scale > 0 and rounding is monotonic,
            // so scaling the max equals the max of the scaled scores), in four
            // independent chains of three-input maxima
            float mq[4] = {fmaxf(sc[0], sc[4]), fmaxf(sc[1], sc[5]), fmaxf(sc[2], sc[6]),
                           fmaxf(sc[3], sc[7])};
#pragma unroll
            for (int c = 8; c < kBlk; c += 8) {
#pragma unroll
                for (int e = 0; e < 4; ++e) mq[e] = max3(mq[e], sc[c + e], sc[c + 4 + e]);
            }
            const float mr = max3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * p.scale_log2;
            // lazy rescaling: the reference max moves (and O and l are
            // rescaled) only when some row's block max exceeds it by more than
            // 8, so the weights stay below 2^8 and most blocks skip the O
            // round trip through TMEM
            const bool move = __any_sync(0xffffffffu, mr > m_run + 8.0f);
            const float mx = move ? fmaxf(m_run, mr) : m_run;
            const float alpha = move ? ex2_ftz(m_run - mx) : 1.0f;   // 0 on the first block
            const uint64_t sc2 = pack_f2(p.scale_log2, p.scale_log2);
            const uint64_t nm2 = pack_f2(-mx, -mx);
            // weights 2^(s * scale * log2 e - m): one paired fma per two
            // weights, the exponential on the special-function unit, and the
            // row sum in four paired chains
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c = 0; c < kBlk; c += 2) {
                float a, b;
                unpack_f2(fma_f2(pack_f2(sc[c], sc[c + 1]), sc2, nm2), a, b);
                sc[c] = ex2_ftz(a);
                sc[c + 1] = ex2_ftz(b);
                acc[(c >> 1) & 3] = add_f2(acc[(c >> 1) & 3], pack_f2(sc[c], sc[c + 1]));
            }
            float s0, s1, s2, s3;
            unpack_f2(add_f2(acc[0], acc[1]), s0, s1);
            unpack_f2(add_f2(acc[2], acc[3]), s2, s3);
            const float sum = (s0 + s2) + (s1 + s3);
            l_run = l_run * alpha + sum;
            m_run = mx;
            if (n >= 1 && move) {
                // P_{n-1} V_{n-1} is done (S_n was issued after it), so O holds
                // the sum so far
#pragma unroll 1
                for (int c = 0; c < kHd / 32; ++c) {
                    float o[32];
                    tmem_ld32(tmem + lane_off + kColO + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    tmem_st32(tmem + lane_off + kColO + 32 * c, o);
                }
            }
            // P_n as bf16 pairs over S_n's first 64 columns (row r in lane r)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    w[e] = __uint_as_float(pack2(sc[64 * c + 2 * e], sc[64 * c + 2 * e + 1]));
                tmem_st32(tmem + lane_off + 32 * c, w);
            }
            tmem_wait_st();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p_full);
        }
        if (!failed && nk > 0) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done, (nk - 1) & 1, abort))) {
                failed = true;
            } else {
                fence_after_sync();
                const int64_t tok = static_cast<int64_t>(i) * kBlk + r;
                const float inv_l = 1.0f / l_run;
#pragma unroll 1
                for (int c = 0; c < kHd / 32; ++c) {
                    float o[32];
                    tmem_ld32(tmem + lane_off + kColO + 32 * c, o);
                    tmem_wait_ld();
                    if (tok < p.N) {
                        uint16_t* dst = p.out + (row0 + tok) * p.out_stride + h * kHd + 32 * c;
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = o[8 * v + e] * inv_l;
                            *reinterpret_cast<uint4*>(dst + 8 * v) = pack8(f);
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
    if (warp == 1) tmem_dealloc(tmem, kTmemColsA);
}

}  // namespace
}  // namespace dit

extern "C" int dit_block_sparse_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                          int64_t row_stride, uint16_t* out, int64_t out_stride,
                                          int B, int64_t N, int H, int hd, int block,
                                          const int32_t* kept, int n_keep, double scale,
                                          int* status, void* stream) {
    using namespace dit;
    if (B < 0 || N < 0 || H < 1 || n_keep < 1) return DIT_ERR_SHAPE;
    if (hd != kHd || block != kBlk) return DIT_ERR_SHAPE;
    const int64_t D = static_cast<int64_t>(H) * hd;
    if (row_stride < D || out_stride < D) return DIT_ERR_SHAPE;
    if (row_stride % 8 || out_stride % 8) return DIT_ERR_ALIGN;
    if (!(scale > 0.0) || scale > 1e30) return DIT_ERR_VALUE;
    if (B == 0 || N == 0) return DIT_OK;
    const int64_t nb = (N + kBlk - 1) / kBlk;
    if (n_keep > nb || B > 65535 || H > 65535) return DIT_ERR_SHAPE;
    const int64_t rows = static_cast<int64_t>(B) * N;
    if (rows + kBlk > 0x7FFFFFFF) return DIT_ERR_SHAPE;
    if (!q || !k || !v || !out || !kept) return DIT_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        reinterpret_cast<uintptr_t>(kept) % 4)
        return DIT_ERR_ALIGN;
    if (status && reinterpret_cast<uintptr_t>(status) % 4) return DIT_ERR_ALIGN;
    const size_t ob = static_cast<size_t>(rows - 1) * out_stride * 2 + D * 2;
    const size_t ib = static_cast<size_t>(rows - 1) * row_stride * 2 + D * 2;
    if (overlaps(out, ob, q, ib) || overlaps(out, ob, k, ib) || overlaps(out, ob, v, ib))
        return DIT_ERR_OVERLAP;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, rows, D, row_stride) || !make_map(&mk, k, rows, D, row_stride) ||
        !make_map(&mv, v, rows, D, row_stride))
        return DIT_ERR_LAUNCH;
    AttnParams p{};
    p.kept = kept;
    p.out = out;
    p.out_stride = out_stride;
    p.status = status;
    p.N = N;
    p.H = H;
    p.nb = static_cast<int>(nb);
    p.n_keep = n_keep;
    p.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
    // the register split inside the kernel assumes the launch count it was
    // sized for; any other count could make setmaxnreg.inc wait forever
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, block_sparse_attention_kernel) != cudaSuccess ||
        fa.numRegs != kRegsLaunch)
        return DIT_ERR_LAUNCH;
    if (cudaFuncSetAttribute(block_sparse_attention_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemA)) != cudaSuccess)
        return DIT_ERR_LAUNCH;
    block_sparse_attention_kernel<<<dim3(static_cast<unsigned>(nb), H, B), kThreadsA, kSmemA,
                                    as_stream(stream)>>>(mq, mk, mv, p);
    return launch_status();
}
