/*
 * dit_block.h -- C ABI of libdit_block.so: the per-block memory-bound
 * operators of a dense single-stream video+audio diffusion transformer
 * (MiniMax-H3 shaped), as hand-written CUDA kernels for B200 (sm_100a).
 *
 * Sources.  The operators are the ones the SGLang-Diffusion H200 report fuses
 * and the Cache-DiT check it uses:
 *   the LMSYS report summary at news.cocoloop.cn (page "minimax-h3-sglang-h200",
 *   untitled in the text), section "Só com três camadas de aceleração somadas chega-se a 6
 *   vezes": the fused AdaLN update, gated residual, SwiGLU activation and
 *   QK RMSNorm with 3D RoPE ("changes no calculation result"), and Cache-DiT
 *   reuse decided by a residual-difference threshold (0.04 conservative,
 *   0.08 stride mode);
 *   "SGLang acelera MiniMax-H3 em GPUs H200 e redefine geração de vídeo por
 *   IA" (ceviu.com.br), first paragraph: fused kernels for AdaLN, SwiGLU,
 *   QK RMSNorm and 3D RoPE cut memory traffic and kernel launches;
 *   "MiniMax H3 mở trọng số: H3-Base có gì và còn thiếu gì?"
 *   (studioglobal.ai), section "Kiến trúc: tạo hình và tiếng trong cùng một
 *   luồng": a dense single-stream transformer whose AdaLN-branch outputs can
 *   be precomputed and cached (so modulation vectors are inputs here).
 * The pages give names, not formulas; each function states the definition it
 * computes.
 *
 * Conventions for every entry point.
 *  - bf16 tensors are passed as uint16_t* (raw bf16 bit patterns) in DEVICE
 *    memory, token-major and contiguous in the feature dimension.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call is asynchronous on that stream; outputs are valid once the stream
 *    has reached the call.
 *  - The caller owns every buffer and the stream.  The library allocates no
 *    memory and keeps no state between calls except a per-device cache of
 *    device attributes, so calls are thread-safe.
 *  - Arguments are checked on the host before anything is launched.  A bad
 *    argument returns a negative dit_status and launches nothing; nothing
 *    aborts, nothing throws.  DIT_ERR_LAUNCH carries a CUDA launch error
 *    (cudaGetLastError after the launch); it may also report an earlier
 *    asynchronous error already pending on the device.
 *  - An empty problem (B == 0 or N == 0 / M == 0) returns DIT_OK and launches
 *    nothing, except where a function says otherwise; its tensor pointers
 *    are not read and may be NULL.
 *  - Pointer alignment: every bf16 tensor pointer must be 16-byte aligned,
 *    and row lengths must be multiples of 8 elements, because each kernel
 *    moves rows as 128-bit vectors.  There is no scalar or CPU fallback.
 */
#ifndef DIT_BLOCK_H
#define DIT_BLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DIT_OK = 0,
    DIT_ERR_NULL = -1,      /* a required pointer is NULL */
    DIT_ERR_SHAPE = -2,     /* a size is negative, zero where it may not be, or too large */
    DIT_ERR_ALIGN = -3,     /* a pointer or row length breaks the 16-byte rule */
    DIT_ERR_DTYPE = -4,     /* unknown dit_dtype */
    DIT_ERR_LAUNCH = -5,    /* CUDA reported an error at launch */
    DIT_ERR_WORKSPACE = -6, /* workspace NULL or smaller than required */
    DIT_ERR_OVERLAP = -7,   /* buffers overlap where they may not */
    DIT_ERR_VALUE = -8      /* a scalar argument (eps, theta) is out of range */
} dit_status;

/* Element type of modulation vectors and norm weights. */
typedef enum { DIT_F32 = 0, DIT_BF16 = 1 } dit_dtype;

/* Largest model width the row kernels accept (a row is held in registers). */
#define DIT_MAX_D 8192

/* ABI version, bumped on any signature change. */
int dit_abi_version(void);

/* Human-readable name of a dit_status value (static string). */
const char* dit_status_string(int status);

/*
 * AdaLN modulation (the fused "AdaLN update").
 *   For every token row x (D values) of sample b:
 *     mu  = mean(x),  var = mean((x - mu)^2)            (biased variance)
 *     y_d = (x_d - mu) / sqrt(var + eps) * (1 + scale_b[d]) + shift_b[d]
 *   Non-affine LayerNorm; the (1 + scale) form makes zero modulation a plain
 *   LayerNorm.  Statistics in fp32, one rounding to bf16 per output.
 * x, y        [B, N, D] bf16, 16-byte aligned.  y may equal x (in place) but
 *             must not partially overlap it.
 * shift,scale modulation of dtype mod_dtype; sample b's D values start at
 *             element b * mod_batch_stride (>= 0; 0 broadcasts one vector;
 *             6*D walks a [B, 6, D] AdaLN-branch output).  Naturally aligned.
 * D           multiple of 8, 8 <= D <= DIT_MAX_D.  eps >= 0.
 */
int dit_adaln_modulate(const uint16_t* x, uint16_t* y,
                       const void* shift, const void* scale, int mod_dtype,
                       int64_t mod_batch_stride,
                       int B, int64_t N, int D, double eps, void* stream);

/*
 * Gated residual fused with the next AdaLN.
 *   x'_d = bf16(x_d + gate_b[d] * r_d)          (one rounding; the new residual)
 *   y    = AdaLN(x'; shift_b, scale_b, eps)     (as dit_adaln_modulate, on the
 *                                                ROUNDED x', so the fused op
 *                                                equals the unfused chain)
 * x'  is computed so that it is bit-identical to a single round-to-nearest-
 * even of the exact x + gate*r.
 * x, r, x_out, y  [B, N, D] bf16, 16-byte aligned.  x_out may equal x (in
 *                 place); otherwise no two of x, r, x_out, y may overlap.
 * gate, shift, scale  as in dit_adaln_modulate (same dtype and batch stride).
 */
int dit_gated_residual_adaln(const uint16_t* x, const uint16_t* r,
                             uint16_t* x_out, uint16_t* y,
                             const void* gate, const void* shift, const void* scale,
                             int mod_dtype, int64_t mod_batch_stride,
                             int B, int64_t N, int D, double eps, void* stream);

/*
 * The two operators above with modulation chosen per token instead of per
 * sample.  The pages name first/last-frame conditioned generation (FL2VA,
 * H3-Base page, section "Phần nào đã được phát hành?") without saying how
 * the conditioning frames are modulated; these entry points let a caller give
 * such tokens modulation of their own.
 *   set_index       device [B*N] uint8: token (b, n) uses set set_index[b*N+n].
 *   n_sets          1..255.  A token whose index is >= n_sets gets NaN outputs
 *                   (y, and x_out of the gated form); nothing is read for it.
 *   mod_set_stride  elements between consecutive sets of one sample: the
 *                   vectors of set s of sample b start at
 *                   b*mod_batch_stride + s*mod_set_stride (e.g. [B, S, 6, D]
 *                   modulation: mod_batch_stride = 6*S*D, mod_set_stride = 6*D).
 * Set 0 is staged in shared memory as in the per-sample operators; other sets
 * are read through the L1/L2 caches, so rows of set 0 run at full speed and
 * the others somewhat slower.  set_index == NULL is the per-sample operator.
 * Other arguments, aliasing rules and errors as above.
 */
int dit_adaln_modulate_tok(const uint16_t* x, uint16_t* y,
                           const void* shift, const void* scale, int mod_dtype,
                           int64_t mod_batch_stride, int64_t mod_set_stride,
                           const uint8_t* set_index, int n_sets,
                           int B, int64_t N, int D, double eps, void* stream);
int dit_gated_residual_adaln_tok(const uint16_t* x, const uint16_t* r,
                                 uint16_t* x_out, uint16_t* y,
                                 const void* gate, const void* shift, const void* scale,
                                 int mod_dtype, int64_t mod_batch_stride, int64_t mod_set_stride,
                                 const uint8_t* set_index, int n_sets,
                                 int B, int64_t N, int D, double eps, void* stream);

/*
 * SwiGLU activation between the MLP up-projection and down-projection.
 *   out[m, j] = silu(in[m, j]) * in[m, F + j],   silu(a) = a / (1 + exp(-a))
 * (first half of each row is the gate, second half the linear branch).
 * in   [M, 2F] bf16, 16-byte aligned.    out [M, F] bf16, 16-byte aligned,
 *      disjoint from in.                 F multiple of 8, F > 0, M >= 0.
 */
int dit_swiglu(const uint16_t* in, uint16_t* out, int64_t M, int F, void* stream);

/*
 * Per-head QK RMSNorm fused with 3D (t, h, w) rotary position embedding,
 * in place on q and k.
 *   For each token and head (hd values x, weight w of the tensor):
 *     u_j = x_j / sqrt(mean_j(x_j^2) + eps) * w_j
 *   The hd/2 rotation pairs are (u_{2p}, u_{2p+1}).  Pairs [0, pairs_t) use
 *   the token's t position, the next pairs_h its h position, the last pairs_w
 *   its w position.  Pair i of an axis with P pairs turns by
 *     phi = pos_axis * theta^(-2i / (2P))
 *   as (u0, u1) -> (u0 cos phi - u1 sin phi, u0 sin phi + u1 cos phi).
 *   Angles are formed and reduced in fp64, sin/cos taken in fp32.
 * q, k        token rows: token i (i = b*N + n) of q starts at q + i*row_stride
 *             elements and holds H*hd values; same for k.  Either may be NULL
 *             (then only the other is processed), not both.  16-byte
 *             aligned; q and k rows must not overlap.
 * row_stride  elements between tokens, multiple of 8, >= H*hd (3*H*hd for a
 *             fused qkv buffer).
 * w_q, w_k    [hd] weights of dtype w_dtype (needed for each non-NULL tensor).
 * hd          one of 32, 64, 128, 256; pairs_t + pairs_h + pairs_w == hd/2,
 *             each >= 1.  H >= 1, H*hd <= DIT_MAX_D.
 * pos         device [B*N, 3] int32 (t, h, w) per token, or NULL: then token
 *             n of every sample sits at global grid index g = pos_offset + n
 *             of a row-major (T, Hg, Wg) grid, t = g/(Hg*Wg), h = (g/Wg)%Hg,
 *             w = g%Wg, and pos_offset + N <= T*Hg*Wg is required (a sequence
 *             shard passes its first token's global index as pos_offset).
 * theta > 0, eps >= 0.
 */
int dit_qk_rmsnorm_rope3d(uint16_t* q, uint16_t* k, int64_t row_stride,
                          const void* w_q, const void* w_k, int w_dtype,
                          int B, int64_t N, int H, int hd,
                          int T, int Hg, int Wg, const int32_t* pos, int64_t pos_offset,
                          int pairs_t, int pairs_h, int pairs_w,
                          double theta, double eps, void* stream);

/* Options of dit_qk_rmsnorm_rope3d_ex. */
enum { DIT_ROPE_INTERLEAVED = 0, DIT_ROPE_HALF = 1 };
enum { DIT_NORM_HEAD = 0, DIT_NORM_ROW = 1 };

/*
 * Where dit_qk_rmsnorm_rope3d_ex writes its result instead of in place: q
 * and k outputs laid out as [B, N, H, hd] with element strides stride_b,
 * stride_n, stride_h and hd contiguous.  Token-major separate buffers are
 * (N*H*hd, H*hd, hd); the head-major [B, H, N, hd] that attention kernels
 * read is (H*N*hd, hd, N*hd).  Strides are multiples of 8, the pointers
 * 16-byte aligned, and the layout must give every element its own address
 * (else DIT_ERR_SHAPE).  Host memory, read during the call only.
 */
typedef struct dit_qk_out {
    uint16_t* q;        /* device; needed when the q input is given */
    uint16_t* k;        /* device; needed when the k input is given */
    int64_t stride_b, stride_n, stride_h;
} dit_qk_out;

/*
 * dit_qk_rmsnorm_rope3d with the choices the pages leave open (the "QK
 * RMSNorm com 3D RoPE" the report names says neither which pairs rotate
 * nor over how many values the RMS is taken) and an output placement:
 *   rope_layout  DIT_ROPE_INTERLEAVED: rotation pairs (u_{2p}, u_{2p+1});
 *                DIT_ROPE_HALF: rotation pairs (u_p, u_{p + hd/2}).  Pair p's
 *                axis, frequency and angle are the same in both layouts.
 *   norm_width   DIT_NORM_HEAD: RMS over each head's hd values, weights [hd];
 *                DIT_NORM_ROW: RMS over the token's whole H*hd row, weights
 *                [H*hd] (then w_q and w_k must be 16-byte aligned).
 *   out          NULL: in place, as dit_qk_rmsnorm_rope3d.  Else q and k are
 *                only read, and the results go to out->q / out->k, which
 *                must overlap neither input nor each other (DIT_ERR_OVERLAP);
 *                a missing output pointer is DIT_ERR_NULL.
 * Other arguments, errors and limits as dit_qk_rmsnorm_rope3d; an unknown
 * option returns DIT_ERR_VALUE.  dit_qk_rmsnorm_rope3d is this function with
 * (DIT_ROPE_INTERLEAVED, DIT_NORM_HEAD, NULL).
 */
int dit_qk_rmsnorm_rope3d_ex(uint16_t* q, uint16_t* k, int64_t row_stride,
                             const void* w_q, const void* w_k, int w_dtype,
                             int B, int64_t N, int H, int hd,
                             int T, int Hg, int Wg, const int32_t* pos, int64_t pos_offset,
                             int pairs_t, int pairs_h, int pairs_w,
                             double theta, double eps, int rope_layout, int norm_width,
                             const dit_qk_out* out, void* stream);

/*
 * dit_qk_rmsnorm_rope3d_ex in place with per-head norm (DIT_NORM_HEAD), that
 * also writes the SubBlock router's block summaries of its results, so the
 * router need not read q and k again (the LMSYS report, news.cocoloop.cn,
 * "minimax-h3-sglang-h200", section "Só com três camadas de aceleração
 * somadas chega-se a 6 vezes": fused operators cut memory traffic; SubBlock
 * attention routes over KV blocks).
 *   block        tokens per router block, >= 1; n_blocks = ceil(N / block),
 *                counted from the first token of each sample in this call,
 *                <= 65535.
 *   block_means  device fp32 [B, 2, n_blocks, H*hd], 16-byte aligned, not
 *                overlapping q or k: [b][0][j] is the mean over block j's
 *                tokens of the rotated q rows as stored (bf16), [b][1][j] the
 *                same for k (the last block may hold fewer tokens).  Each
 *                mean is an fp32 sum in a fixed order divided once by the
 *                token count, so results repeat run to run.  It is the input
 *                of dit_subblock_router_means.
 *   status       optional device int: set to 1 if a wait of the kernel's
 *                copy pipeline ran out (bounded at 2 s; the means of the
 *                affected blocks are then left unwritten).  NULL: not reported.
 * q and k are both required (DIT_ERR_NULL); other arguments, errors and
 * limits as dit_qk_rmsnorm_rope3d_ex (rope_layout as there; B <= 65535).
 */
int dit_qk_rmsnorm_rope3d_pooled(uint16_t* q, uint16_t* k, int64_t row_stride,
                                 const void* w_q, const void* w_k, int w_dtype,
                                 int B, int64_t N, int H, int hd,
                                 int T, int Hg, int Wg, const int32_t* pos, int64_t pos_offset,
                                 int pairs_t, int pairs_h, int pairs_w,
                                 double theta, double eps, int rope_layout, int block,
                                 float* block_means, int* status, void* stream);

/*
 * Test hook for the failure path of dit_qk_rmsnorm_rope3d_pooled: the same
 * launch with no copy issued, so that every wait of the copy ring runs out
 * (after about 2 s) and the kernel writes 1 to *status and returns, leaving
 * the context usable; q, k and the means are left unwritten.  B*N <= 4096;
 * status is required.  Not for production use.
 */
int dit_qk_rmsnorm_rope3d_pooled_stall_test(uint16_t* q, uint16_t* k, int64_t row_stride,
                                            const void* w_q, const void* w_k, int w_dtype,
                                            int B, int64_t N, int H, int hd,
                                            int T, int Hg, int Wg, const int32_t* pos,
                                            int64_t pos_offset, int pairs_t, int pairs_h,
                                            int pairs_w, double theta, double eps,
                                            int rope_layout, int block, float* block_means,
                                            int* status, void* stream);

/*
 * Cache-DiT residual-difference check between neighbouring denoising steps.
 *   Per sample b:  rel_b   = sum_{n,d} |cur - prev| / sum_{n,d} |prev|
 *                  reuse_b = rel_b < threshold       (strict)
 *   0/0 reads as rel = 0 (identical residuals are reusable); x/0 as +inf.
 *   |cur - prev| and |prev| are summed in fp32 per 8- or 16-element vector
 *   and in fp64 above that, in a fixed order: the result is deterministic run
 *   to run on a given device.
 * prev, cur   [B, N, D] bf16, 16-byte aligned.  D multiple of 8.
 * rel_out     device [B] double;  reuse_out device [B] uint8 (0 or 1).
 * workspace   device scratch of at least cachedit_workspace_bytes(B, N, D)
 *             bytes, 16-byte aligned; its contents on entry do not matter.
 *             Calls that share a workspace must be ordered on the device.
 * N == 0 is allowed (prev and cur may then be NULL) and yields rel = 0,
 * reuse = (threshold > 0); the kernels still run to write rel and reuse.
 */
size_t cachedit_workspace_bytes(int B, int64_t N, int D);
int cachedit_residual_diff(const uint16_t* prev, const uint16_t* cur,
                           int B, int64_t N, int D, double threshold,
                           double* rel_out, uint8_t* reuse_out,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * The two sums of the Cache-DiT check without the decision, for a sequence
 * shard: sums_out[b][0] = sum |cur - prev|, sums_out[b][1] = sum |prev| over
 * this call's N*D elements of sample b (device [B][2] double).  Ranks that
 * each hold a shard exchange these 2*B doubles (an all-gather) and call
 * cachedit_decide on the gathered [R][B][2] array, so every rank reaches the
 * same decision.  Arguments otherwise as cachedit_residual_diff.
 */
int cachedit_residual_sums(const uint16_t* prev, const uint16_t* cur,
                           int B, int64_t N, int D, double* sums_out,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decision from R sets of partial sums: sums is device [R][B][2] double;
 * per sample the R partials are added in a fixed order that depends only on
 * R (so ranks that hold the same gathered array reach bit-identical results),
 * then rel and reuse follow as in cachedit_residual_diff.  R >= 1, B >= 1.
 * sums must be 8-byte aligned.
 */
int cachedit_decide(const double* sums, int R, int B, double threshold,
                    double* rel_out, uint8_t* reuse_out, void* stream);

/*
 * SwiGLU fused into the up-projection GEMM (tensor cores, sm_100):
 *     out[m, j] = silu(g) * u,  g = sum_k x[m, k] w[j, k],
 *                               u = sum_k x[m, k] w[F + j, k]
 * The LMSYS report (news.cocoloop.cn, "minimax-h3-sglang-h200", section "Só
 * com três camadas de aceleração somadas chega-se a 6 vezes") names SwiGLU
 * among the fused operators; here it is fused into the GEMM that produces
 * its input, so the [M, 2F] product is never written.
 *   x    device [M, K] bf16, row-major (token-major activations).
 *   w    device [2F, K] bf16, one row per output feature (the usual linear
 *        weight layout): rows [0, F) the gate half, [F, 2F) the linear half.
 *   out  device [M, F] bf16; must not overlap x or w.
 * K and F multiples of 8; pointers 16-byte aligned.  Products accumulate in
 * fp32 in the tensor memory; silu(g) * u is formed in fp32 and rounded once
 * to bf16.  status (optional device int, 4-byte aligned) is set to 1 if a
 * pipeline wait inside the kernel ran out (a defect, never expected): the
 * output is then incomplete.  The caller clears it.
 */
int dit_swiglu_gemm(const uint16_t* x, const uint16_t* w, uint16_t* out, int64_t M, int K, int F,
                    int* status, void* stream);

/*
 * Test hook for the failure path of the tensor-core kernels: the same launch
 * as dit_swiglu_gemm with its copy warp disabled, so that every pipeline wait
 * runs out (after about 2 s) and the kernel writes 1 to *status, frees its
 * tensor memory and returns, leaving the context usable.  Small shapes only
 * (M, K, F <= 4096); status is required.  Not for production use.
 */
int dit_swiglu_gemm_stall_test(const uint16_t* x, const uint16_t* w, uint16_t* out, int64_t M,
                               int K, int F, int* status, void* stream);

/*
 * The gated residual fused into the down-projection GEMM (tensor cores):
 *     x_out[m, n] = bf16(x[m, n] + gate_b[n] * sum_k h[m, k] w[n, k])
 * a2's residual update with its branch taken straight from the product, so
 * the [M, D] branch is never written.  Same main loop as dit_swiglu_gemm.
 *   h      device [B*N, K] bf16 (the MLP activations, token-major).
 *   w      device [D, K] bf16, one row per output feature.
 *   x      device [B*N, D] bf16 residual stream; x_out may be x (in place) or
 *          must overlap neither x, h nor w.
 *   gate   device [B, D] of gate_dtype (DIT_F32 or DIT_BF16), gate_batch_stride
 *          elements between samples (0 broadcasts); token row m uses sample
 *          m / N.
 * K and D multiples of 8; h, w, x, x_out 16-byte aligned.  The sum runs in
 * fp32 in the tensor memory; x + gate * sum is one fp32 fma rounded once to
 * bf16 (redone in fp64 when the fma lands on a bf16 tie).  status as for
 * dit_swiglu_gemm.
 */
int dit_gemm_gated_residual(const uint16_t* h, const uint16_t* w, const uint16_t* x,
                            uint16_t* x_out, const void* gate, int gate_dtype,
                            int64_t gate_batch_stride, int B, int64_t N, int K, int D,
                            int* status, void* stream);

/*
 * SubBlock block-sparse attention router.  The LMSYS report (news.cocoloop.cn,
 * "minimax-h3-sglang-h200", section "Só com três camadas de aceleração
 * somadas chega-se a 6 vezes") cuts, from the 10th denoising step on, the KV
 * blocks that take part in attention, at sparsity 0.75 or 0.80, and gives no
 * rule.  Reading: the N tokens of a sample are cut into blocks of `block`
 * consecutive tokens (the last may be shorter), n_blocks = ceil(N / block);
 * per head, a block's summary is the mean of its rows; query block i scores
 * key block j by the dot product of the summaries (fp32) and keeps the
 * n_keep = dit_subblock_keep_count(n_blocks, sparsity) = max(1,
 * ceil((1 - sparsity) n_blocks)) best key blocks, ties to the lower index.
 *   q, k       device rows of B*N tokens, row_stride elements apart (a fused
 *              qkv buffer works), H heads of hd values each (hd multiple of
 *              8, <= 256; H*hd <= DIT_MAX_D); 16-byte aligned.
 *   kept       device int32 [B, H, n_blocks, n_keep]: the kept key blocks of
 *              each query block, in increasing order.
 *   workspace  device, >= dit_subblock_workspace_bytes(...) bytes (the block
 *              means [B, 2, n_blocks, H*hd] fp32, then the workspace of
 *              dit_subblock_router_means), 16-byte aligned.
 *   status     optional device int, as dit_subblock_router_means.
 * The scores are taken as dit_subblock_router_means takes them (tensor cores
 * for hd a multiple of 32).
 * 0 <= sparsity < 1 (else DIT_ERR_VALUE); n_blocks <= 8192.  Which steps use
 * the router (the report: from the 10th) is the caller's choice.
 */
int dit_subblock_keep_count(int64_t n_blocks, double sparsity);
size_t dit_subblock_workspace_bytes(int B, int64_t N, int H, int hd, int block);
int dit_subblock_router(const uint16_t* q, const uint16_t* k, int64_t row_stride, int B,
                        int64_t N, int H, int hd, int block, double sparsity, int32_t* kept,
                        void* workspace, size_t workspace_bytes, int* status, void* stream);

/*
 * The SubBlock router from block means already computed (for example by
 * dit_qk_rmsnorm_rope3d_pooled): the scores and the selection of
 * dit_subblock_router, without reading q and k.
 *   block_means  device fp32 [B, 2, n_blocks, H*hd] (q means, then k means),
 *                16-byte aligned; n_blocks = ceil(N / block) <= 8192.
 *   workspace    device, >= dit_subblock_means_workspace_bytes(B, N, H, hd,
 *                block) bytes (the scores [B, H, n_blocks, n_blocks] fp32;
 *                for hd a multiple of 32, also the high and low tf32 parts
 *                of the means), 16-byte aligned.
 *   status       optional device int: set to 1 if a wait of the tensor-core
 *                score kernel ran out (bounded at 2 s; the scores of the
 *                affected tiles are then left unwritten).  NULL: not reported.
 * For hd a multiple of 32 the scores are taken on the tensor cores
 * as three tf32 products (hi.hi + hi.lo + lo.hi, the means split into a tf32
 * high part and the remainder), which keeps them within a few fp32 rounding
 * steps of the fp32 sum; other hd use fp32 FMAs.
 * kept, sparsity, hd limits and errors as dit_subblock_router.
 */
size_t dit_subblock_means_workspace_bytes(int B, int64_t N, int H, int hd, int block);
int dit_subblock_router_means(const float* block_means, int B, int64_t N, int H, int hd,
                              int block, double sparsity, int32_t* kept, void* workspace,
                              size_t workspace_bytes, int* status, void* stream);

/*
 * Test hook for the failure path of the tensor-core score kernel: the split
 * and the score launch of dit_subblock_router_means with the kernel's copy
 * thread issuing nothing, so that every wait runs out (after about 2 s) and
 * the kernel writes 1 to *status, frees its tensor memory and returns,
 * leaving the context usable; the scores are left unwritten and nothing is
 * selected.  hd a multiple of 32, B <= 4, n_blocks <= 512; status is
 * required.  Not for production use.
 */
int dit_subblock_scores_stall_test(const float* block_means, int B, int64_t N, int H, int hd,
                                   int block, void* workspace, size_t workspace_bytes,
                                   int* status, void* stream);

/*
 * Block-sparse attention over the router's kept key blocks (tensor cores):
 * for token t of query block i, head h,
 *     out[t, h] = sum_u softmax_u(scale * q[t, h] . k[u, h]) v[u, h]
 * over the tokens u of the key blocks kept[b, h, i, 0..n_keep) of the same
 * sample (as returned by dit_subblock_router); non-causal.
 *   q, k, v     device rows of B*N tokens, row_stride elements apart (a fused
 *               qkv buffer works), H heads of hd = 128; 16-byte aligned.
 *   out         device rows, out_stride elements apart, H*128 wide; must not
 *               overlap q, k or v.
 *   block       128 (the tile height); n_keep <= n_blocks.
 *   kept        device int32 [B, H, n_blocks, n_keep]; an index outside
 *               [0, n_blocks) contributes no keys (its rows may come out NaN).
 *   scale       the softmax scale, e.g. 1/sqrt(128).
 * S = Q K^T and O = P V run on tcgen05 with fp32 accumulators; the softmax
 * is fp32 in the exp2 domain and P enters the second product as bf16.
 * status as for dit_swiglu_gemm.
 */
int dit_block_sparse_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               int64_t row_stride, uint16_t* out, int64_t out_stride,
                               int B, int64_t N, int H, int hd, int block,
                               const int32_t* kept, int n_keep, double scale,
                               int* status, void* stream);

/*
 * Test hook for the failure path of the block-sparse attention kernel: the
 * same launch as dit_block_sparse_attention with its copy warps issuing
 * nothing, so that every wait runs out (after about 2 s) and the kernel
 * writes 1 to *status, frees its tensor memory and returns, leaving the
 * context usable; out is left unwritten.  B*N <= 1024, H <= 4; status is
 * required.  Not for production use.
 */
int dit_block_sparse_attention_stall_test(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                          int64_t row_stride, uint16_t* out, int64_t out_stride,
                                          int B, int64_t N, int H, int hd, int block,
                                          const int32_t* kept, int n_keep, double scale,
                                          int* status, void* stream);

/*
 * Cache-DiT step cache.  The LMSYS report (news.cocoloop.cn,
 * "minimax-h3-sglang-h200", section "Só com três camadas de aceleração
 * somadas chega-se a 6 vezes") reuses results cached between neighbouring
 * denoising steps when a residual-difference threshold allows (0.04
 * conservative, 0.08 stride mode).  Reading: the cached result is the
 * residual the skipped blocks add to the hidden state.  A run:
 *   step t: h1 = first blocks(h); r1 = cachedit_residual_store(h, h1);
 *           rel = max over samples of the relative L1 difference of r1
 *                 against the previous step's r1 (cachedit_residual_diff);
 *           if dit_cache_policy_decide(&policy, rel):
 *               out = cachedit_residual_apply(h1, R)
 *           else:
 *               out = remaining blocks(h1); R = cachedit_residual_store(h1, out)
 * (at step 0 rel is ignored and the step computes).
 *
 * cachedit_residual_store: residual[i] = bf16(after[i] - before[i]).
 * cachedit_residual_apply: out[i] = bf16(h[i] + residual[i]).
 * Each is the exact value rounded once to nearest-even.  Device pointers,
 * n elements (multiple of 8, >= 0), 16-byte aligned.  The output may be one
 * of the inputs (in place) or disjoint from both (else DIT_ERR_OVERLAP).
 * Asynchronous on `stream`.
 */
int cachedit_residual_store(const uint16_t* before, const uint16_t* after, uint16_t* residual,
                            int64_t n, void* stream);
int cachedit_residual_apply(const uint16_t* h, const uint16_t* residual, uint16_t* out,
                            int64_t n, void* stream);

/*
 * The reuse rule, host only.  Step t (counted by the struct) reuses iff
 *   t >= 1, t >= warmup_steps, rel < threshold (strict; NaN never reuses),
 *   and max_cached_steps == 0 or fewer than max_cached_steps steps in a row
 *   reused before it.
 * warmup_steps and max_cached_steps are guards the pages do not mention
 * (0 = off).  Every rank that passes the same rel sequence takes the same
 * decisions (rel from the all-gathered sums is bit-identical on all ranks).
 * dit_cache_policy_decide returns 1 (reuse) or 0 (compute) and advances
 * the step; a NULL struct returns DIT_ERR_NULL.  init rejects a NaN
 * threshold or negative counts with DIT_ERR_VALUE.  Not thread-safe per
 * struct; the caller owns the struct.
 */
typedef struct dit_cache_policy {
    double threshold;
    int warmup_steps;
    int max_cached_steps;
    int step;           /* next step's index */
    int run;            /* consecutive reuses just before it */
    int computed;       /* steps that computed so far */
    int reused;         /* steps that reused so far */
} dit_cache_policy;

int dit_cache_policy_init(dit_cache_policy* policy, double threshold, int warmup_steps,
                          int max_cached_steps);
int dit_cache_policy_decide(dit_cache_policy* policy, double rel);

/*
 * The Cache-DiT check of cachedit_residual_diff for callers that cannot
 * allocate device memory or pass a workspace (the pages have no counterpart
 * to this entry point; it exists for such callers).  Some callers cannot
 * call cudaMalloc: a plugin inside a serving engine that owns all device
 * memory through its own pool and forbids raw allocations, or a caller on a
 * latency-critical path that cannot accept the device-wide synchronisation a
 * fresh allocation can cause.
 * The partial sums go to a fixed 64 KB array inside the library (4096 pairs
 * of doubles per device, held by every GPU that loads the library until the
 * process exits).  This entry point allocates nothing and calls no
 * allocating routine.
 * Limits: B <= 64 samples, and (partial-sum slots per sample) x B <= 4096
 * (always true for B <= 64 on current GPUs); beyond them it returns
 * DIT_ERR_SHAPE (B) or DIT_ERR_WORKSPACE (slots) and launches nothing.
 * Set-up: a call whose stream is not capturing looks up the array's device
 * address (cudaGetSymbolAddress) with the current device and caches it, so
 * the address stays right after a cudaDeviceReset; a call made while its
 * stream is capturing uses the cached address.  Make the first call on each
 * device before any stream capture on it (else DIT_ERR_LAUNCH).
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents; each call writes every slot it reads before reading it,
 * so nothing needs clearing, but calls that overlap on the GPU (different
 * streams, or host threads without ordering) race on the array: order them.
 * Arguments and results otherwise as cachedit_residual_diff.
 */
int cachedit_residual_diff_noalloc(const uint16_t* prev, const uint16_t* cur,
                                   int B, int64_t N, int D, double threshold,
                                   double* rel_out, uint8_t* reuse_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DIT_BLOCK_H */
