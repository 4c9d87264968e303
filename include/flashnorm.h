/*
 * flashnorm.h — C ABI of the FlashNorm RMSNorm -> linear library for NVIDIA B200 (sm_100a).
 *
 * FlashNorm ("FlashNorm: Fast Normalization for Transformers", Abstract) is an exact reformulation of
 * RMSNorm followed by a linear layer:
 *   (i)  the norm gain g is folded into the weights offline:   W* = diag(g) . W
 *   (ii) the scalar RMS normalisation is deferred to the matmul output:
 *            y = (x . W*) * 1 / sqrt(mean(x^2) + eps)
 *        so the row sum of squares and the contraction run at the same time (here: in one kernel,
 *        on different warps, joined by shared-memory barriers).
 * It extends to GLU feed-forward layers (the deferred scale goes onto the gate and the up outputs
 * before SiLU) and to RMSNorm -> linear -> RMSNorm, where the first norm is dropped by the scale
 * invariance of RMS (same abstract). The abstract also names LayerNorm, RoPE-based attention and
 * quantized models among the cases the technique carries over to; this library covers LayerNorm ->
 * linear, RoPE on the normalised heads of the post-norm path, and FP8 E4M3 weights for decode.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are caller-owned DEVICE memory on the current device; the library never
 *     allocates, frees or keeps them. Pointers must be 16-byte aligned.
 *   - Element types: activations, weights, gains and the unfused intermediate are bf16 (stored as
 *     uint16 bit patterns); outputs are bf16 or fp32 as `out_dtype` says. All arithmetic is fp32
 *     with one round-to-nearest-even conversion per bf16 result.
 *   - Layouts are row-major. x is [M, d]; y is [M, N] (linear, post-norm) or [M, F] (GLU).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every call only
 *     enqueues work on it and returns; nothing synchronises except flashnorm_check_device_error.
 *   - Arguments are validated before anything is launched; a rejected call launches nothing and
 *     returns FN_ERR_INVALID_ARG / FN_ERR_ALIGN / FN_ERR_UNSUPPORTED with a message available from
 *     flashnorm_last_error(). A failed launch returns FN_ERR_CUDA.
 *   - M == 0 is a valid empty call: nothing is launched and FN_OK is returned.
 *   - Outputs must not overlap inputs. Results are deterministic (no atomics on results; the decode
 *     kernel's split-K partial sums are combined in a fixed order), so identical calls give bitwise
 *     identical outputs.
 *   - Every wait inside a kernel is bounded in time; a wait that runs out records FN_ERR_TIMEOUT in a
 *     device-side status word (read and cleared by flashnorm_check_device_error) and the kernel
 *     returns early instead of hanging. The outputs of such a call are not valid; the tensor-core
 *     decode kernel writes the outputs that a failed wait affects as NaN (its K-split partial sums
 *     from the CTA that gave up are NaN), the prefill kernels leave the tiles they did not finish
 *     unwritten.
 *   - Host threads: entry points may be called from several threads. flashnorm_last_error is kept per
 *     thread. The one-time per-device setup of the first calls on a device (kernel shared-memory
 *     attributes, the SM count) sets the same values whoever performs it, so concurrent first calls
 *     only repeat it.
 */
#ifndef FLASHNORM_H
#define FLASHNORM_H

#include <stdint.h>

#if defined(__GNUC__)
#define FN_API __attribute__((visibility("default")))
#else
#define FN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FN_OK = 0,
  FN_ERR_INVALID_ARG = 1, /* a size, pointer or flag is out of range */
  FN_ERR_UNSUPPORTED = 2, /* a legal request the library has no kernel for (e.g. head_dim > 512) */
  FN_ERR_ALIGN = 3,       /* a pointer or a leading dimension is not 16-byte aligned */
  FN_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (message has the CUDA error) */
  FN_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out (see flashnorm_check_device_error) */
} fn_status;

typedef enum { FN_BF16 = 0, FN_F32 = 1 } fn_dtype;

/* Which kernel family a projection runs on.
 *   FN_PATH_TENSOR  the persistent prefill kernel, one CTA per 128-row tile (any M)
 *   FN_PATH_PAIR    the persistent prefill kernel on CTA pairs: one 2-SM MMA per 256-row tile
 *   FN_PATH_GEMV    the CUDA-core GEMV (M <= FN_DECODE_MAX_M)
 *   FN_PATH_DECODE  the tensor-core decode kernel: W* rows on the MMA's M side, the tokens on its
 *                   N side, W* streamed once by TMA (M <= FN_DECODE_MAX_M)
 *   FN_PATH_AUTO    DECODE for M <= FN_DECODE_MAX_M, PAIR for M > 128, TENSOR otherwise */
typedef enum {
  FN_PATH_AUTO = 0,
  FN_PATH_TENSOR = 1,
  FN_PATH_GEMV = 2,
  FN_PATH_DECODE = 3,
  FN_PATH_PAIR = 4
} fn_path;

#define FN_DECODE_MAX_M 16
/* GLU weights are stored gate/up interleaved in blocks of this many output columns (see fold). */
#define FN_GLU_BLOCK 16

/*
 * flashnorm_fold_weights — step (i), weight folding (FlashNorm Abstract, item i: the norm gain is
 * multiplied into the projection that follows, so the norm keeps no weights of its own).
 *   W      bf16 [d, N] row-major, the unfolded projection (y = x . W).
 *   g      bf16 [d], the RMSNorm gain.
 *   Wstar  bf16 [N, d] output: Wstar[n][k] = RNE_bf16(g[k] * W[k][n]), i.e. W* stored K-major (its
 *          transpose, row-major), the operand layout every projection kernel reads. g[k]*W[k][n] is
 *          exact in fp32, so each element is rounded exactly once.
 *   glu    0: N output columns in order. 1: N = 2F columns, gate = W[:, 0:F), up = W[:, F:2F); the
 *          output rows are interleaved in blocks of FN_GLU_BLOCK: rows [32b, 32b+16) hold gate
 *          columns [16b, 16b+16) and rows [32b+16, 32b+32) the matching up columns. Needs F % 16 == 0.
 * Folding with g = 1 is an exact transpose; that is how the unfused path gets its K-major W.
 * Constraints: d >= 8, d % 8 == 0, N >= 8, N % 8 == 0.
 */
FN_API fn_status flashnorm_fold_weights(const void* W, const void* g, void* Wstar, int64_t d, int64_t N,
                                 int glu, void* stream);

/*
 * flashnorm_linear — steps (i)+(ii): y = (x . W*) * 1/sqrt(mean(x^2) + eps) (FlashNorm Abstract).
 *   x      bf16 [M, d]; Wstar bf16 [N, d] from flashnorm_fold_weights(glu = 0); y [M, N] of out_dtype.
 *   For M > 16 one persistent tcgen05 kernel computes x . W* into tensor memory while a separate
 *   warpgroup sums x^2 per row from the same shared-memory x tiles; the epilogue waits for both and
 *   scales each row (CTA pairs sharing 2-SM MMAs for M > 128). For M <= 16 the tensor-core decode
 *   kernel streams W* once, with W* rows on the MMA's M side and the tokens on its N side.
 * Constraints: M >= 0, d % 8 == 0, N % 8 == 0, eps >= 0 and finite.
 */
FN_API fn_status flashnorm_linear(const void* x, const void* Wstar, void* y, int64_t M, int64_t d, int64_t N,
                           float eps, int out_dtype, void* stream);

/* Same as flashnorm_linear with the kernel family chosen explicitly (fn_path). */
FN_API fn_status flashnorm_linear_ex(const void* x, const void* Wstar, void* y, int64_t M, int64_t d, int64_t N,
                              float eps, int out_dtype, int path, void* stream);

/*
 * flashnorm_glu — the GLU feed-forward variant (FlashNorm Abstract: the techniques carry over to
 * gated feed-forward layers): with r = 1/sqrt(mean(x^2) + eps), z = x . W*,
 *     y[m, j] = silu(r * z[m, gate j]) * (r * z[m, up j]),   silu(t) = t / (1 + exp(-t)).
 *   x bf16 [M, d]; Wstar_gu bf16 [2F, d] from flashnorm_fold_weights(glu = 1); y [M, F] of out_dtype.
 * Constraints: as flashnorm_linear, and F % 16 == 0.
 */
FN_API fn_status flashnorm_glu(const void* x, const void* Wstar_gu, void* y, int64_t M, int64_t d, int64_t F,
                        float eps, int out_dtype, void* stream);

FN_API fn_status flashnorm_glu_ex(const void* x, const void* Wstar_gu, void* y, int64_t M, int64_t d, int64_t F,
                           float eps, int out_dtype, int path, void* stream);

/*
 * flashnorm_linear_postnorm — redundant-norm removal (FlashNorm Abstract: when a linear layer sits
 * between two RMSNorms, RMS scale invariance makes the first one unnecessary):
 *     u = x . W*   (the first norm's gain folded into W*, its 1/rms dropped),
 *     y[m, h*hd + j] = u[m, h*hd + j] / sqrt(mean_j u[m, h*hd + j]^2 + eps2) * g2[j]
 *   for each head h of width hd = head_dim.
 *   x bf16 [M, d]; Wstar bf16 [N, d] (fold with glu = 0); g2 bf16 [head_dim]; y [M, N] of out_dtype.
 * Constraints: d % 8 == 0, head_dim % 16 == 0, 16 <= head_dim <= 512, N % head_dim == 0, eps2 >= 0.
 */
FN_API fn_status flashnorm_linear_postnorm(const void* x, const void* Wstar, const void* g2, void* y, int64_t M,
                                    int64_t d, int64_t N, int64_t head_dim, float eps2, int out_dtype,
                                    void* stream);

/*
 * flashnorm_linear_postnorm_ws — flashnorm_linear_postnorm with a caller-provided workspace. The same
 * result (same definition, same tolerances); what changes is how a wide head (256 < head_dim <= 512)
 * is scheduled when it has few 256-row tiles. Without a workspace, each tile's whole contraction runs in
 * one thread-block cluster that keeps its partial sums on chip (few such clusters are resident, so
 * 2048 rows of one 512-wide head occupy 64 SMs). With one, the contraction dimension d is split over
 * independent CTA pairs that fill the device, each writing an fp32 partial product to the workspace,
 * and a second kernel adds the partials in a fixed order (deterministic) and applies the norm.
 *   workspace        device memory, 16-byte aligned, caller-owned, or NULL (no split). Its contents
 *                    are scratch: overwritten by the call and read by its second kernel, so calls whose
 *                    kernels overlap on the GPU (different streams, host threads) must not share one.
 *   workspace_bytes  its size. A non-NULL workspace smaller than flashnorm_postnorm_workspace_bytes
 *                    reports for this shape returns FN_ERR_INVALID_ARG and launches nothing.
 * Shapes for which the split does not apply (head_dim <= 256, or enough row tiles to fill the device
 * without it: the size query returns 0) ignore the workspace.
 */
FN_API fn_status flashnorm_linear_postnorm_ws(const void* x, const void* Wstar, const void* g2, void* y, int64_t M,
                                              int64_t d, int64_t N, int64_t head_dim, float eps2, int out_dtype,
                                              void* workspace, int64_t workspace_bytes, void* stream);

/*
 * flashnorm_postnorm_workspace_bytes — the workspace flashnorm_linear_postnorm_ws uses for this shape on
 * the current device, written to *bytes: K ranges x M x N x 4 (fp32 partial products), or 0 where the
 * split does not apply. FN_ERR_INVALID_ARG for a shape flashnorm_linear_postnorm rejects as invalid.
 */
FN_API fn_status flashnorm_postnorm_workspace_bytes(int64_t M, int64_t d, int64_t N, int64_t head_dim,
                                                    int64_t* bytes);

/*
 * flashnorm_linear_postnorm_rope — flashnorm_linear_postnorm followed, in the same epilogue, by rotary
 * position embedding of the normalised query/key heads. The FlashNorm Abstract lists RoPE-based
 * attention among the cases the technique extends to, and the paper builds on RoFormer; the rotation is
 * RoFormer's: features (2i, 2i+1) of a head of the row at position p are rotated by the angle
 * p * base^(-2i/head_dim):
 *     y[2i]   = v[2i] cos - v[2i+1] sin,     y[2i+1] = v[2i] sin + v[2i+1] cos,
 *   where v is the post-norm output of that head. Only the first n_rope_heads heads of a row are rotated
 *   (in a fused q/k/v projection: the query and key heads); the others are only normalised.
 *   rope_cs   fp32 [max_pos][head_dim / 2][2], (cos, sin) of pair i at position p, e.g. from
 *             flashnorm_rope_table; 16-byte aligned; caller-owned device memory.
 *   positions int32 [M], device memory, 4-byte aligned: the position of each row. A position outside
 *             [0, max_pos) is not read from the table: the row's rotated heads are written as NaN and
 *             the next flashnorm_check_device_error returns FN_ERR_INVALID_ARG.
 * Other arguments and constraints as for flashnorm_linear_postnorm; head_dim of 384 or 512 (the
 * cluster kernel) returns FN_ERR_UNSUPPORTED; 0 <= n_rope_heads <= N / head_dim; max_pos >= 1.
 */
FN_API fn_status flashnorm_linear_postnorm_rope(const void* x, const void* Wstar, const void* g2, const void* rope_cs,
                                                const void* positions, void* y, int64_t M, int64_t d, int64_t N,
                                                int64_t head_dim, int64_t n_rope_heads, int64_t max_pos, float eps2,
                                                int out_dtype, void* stream);

/*
 * LayerNorm -> linear (FlashNorm Abstract: the same techniques extend to LayerNorm). With
 *   LN(x) = (x - mu) / sqrt(var + eps) * gamma + beta,  mu = mean(x), var = mean((x - mu)^2) over the d features,
 * y = LN(x) . W is computed as y = r (x . W*) - (r mu) colsum + bias with r = 1/sqrt(var + eps):
 * gamma is folded into W* = diag(gamma) W as for RMSNorm, the mean subtraction becomes a rank-1 correction
 * with the column sums of W*, and beta becomes a bias vector. mu and var are summed by the same warps
 * that sum x^2 for RMSNorm, from the same staged x tiles, concurrently with the contraction; the correction
 * and the bias are applied in the epilogue.
 *
 * flashnorm_fold_layernorm: W bf16 [d, N] row-major, gamma bf16 [d], beta bf16 [d] or NULL (no bias) ->
 *   Wstar bf16 [N, d] (exactly flashnorm_fold_weights(W, gamma, glu = 0)), colsum fp32 [N] = sum over k of the
 *   bf16 W*[n][k], bias fp32 [N] = sum over k of beta[k] W[k][n] (fp32). All caller-owned device memory.
 * flashnorm_layernorm_linear: x bf16 [M, d] -> y [M, N] of out_dtype: M <= FN_DECODE_MAX_M on the
 *   tensor-core decode kernel (the weights stream once), larger M on the CTA-pair tensor-core kernel.
 *   Constraints: d % 8 == 0, N % 8 == 0, eps >= 0. The variance is taken as
 *   E[x^2] - mu^2 in fp32 (clamped at 0), accurate while |mu| is not large against the spread of x.
 */
FN_API fn_status flashnorm_fold_layernorm(const void* W, const void* gamma, const void* beta, void* Wstar,
                                          void* colsum, void* bias, int64_t d, int64_t N, void* stream);
FN_API fn_status flashnorm_layernorm_linear(const void* x, const void* Wstar, const void* colsum, const void* bias,
                                            void* y, int64_t M, int64_t d, int64_t N, float eps, int out_dtype,
                                            void* stream);

/*
 * Quantized W* (FlashNorm Abstract: folded checkpoints stay compatible with quantized models). The gain
 * is folded first, then each output channel is quantized to FP8 E4M3 with its own scale; the deferred
 * 1/rms and the channel scale multiply the output together:
 *     W*[n][k] = g[k] W[k][n] (exact in fp32),   s[n] = max_k |W*[n][k]| / 448 (1 for a zero channel),
 *     Q[n][k] = E4M3(W*[n][k] / s[n]) (fp32 division, round to nearest even, saturating),
 *     y[m][n] = (sum_k x[m][k] Q[n][k]) * s[n] / sqrt(mean_k x[m][k]^2 + eps).
 * flashnorm_fold_weights_fp8: W bf16 [d, N] row-major, g bf16 [d] -> Q uint8 [N, d] (K-major E4M3 codes)
 *   and scales fp32 [N]; caller-owned device memory. d % 16 == 0, N % 8 == 0.
 * flashnorm_linear_fp8: the decode path (M <= FN_DECODE_MAX_M), streaming Q, one byte per weight, half
 *   the bytes of bf16 W*: y = (x . dec(Q)^T) * scales * 1/sqrt(mean(x^2) + eps). x bf16 [M, d];
 *   y [M, N] of out_dtype. Larger M returns FN_ERR_UNSUPPORTED. Runs flashnorm_linear_fp8_ex with
 *   FN_PATH_AUTO.
 * flashnorm_linear_fp8_ex: the same with a kernel choice. FN_PATH_DECODE: the tensor-core kernel (Q widened
 *   on chip, exactly, to bf16 in tensor memory; x as it is; fp32 accumulation). FN_PATH_GEMV: the
 *   CUDA-core GEMV (x staged in shared memory, each 16-byte load carries 16 weights). FN_PATH_AUTO: the
 *   GEMV for one token, the tensor-core kernel for more. Other paths return FN_ERR_INVALID_ARG.
 */
FN_API fn_status flashnorm_fold_weights_fp8(const void* W, const void* g, void* Q, void* scales, int64_t d, int64_t N,
                                            void* stream);
FN_API fn_status flashnorm_linear_fp8(const void* x, const void* Q, const void* scales, void* y, int64_t M, int64_t d,
                                      int64_t N, float eps, int out_dtype, void* stream);
FN_API fn_status flashnorm_linear_fp8_ex(const void* x, const void* Q, const void* scales, void* y, int64_t M,
                                         int64_t d, int64_t N, float eps, int out_dtype, int path, void* stream);

/*
 * flashnorm_linear_fp8_ws — flashnorm_linear_fp8_ex with a caller-provided workspace. The same result
 * (same definition, same tolerances); what changes is how the tensor-core kernel splits the contraction
 * d. Without a workspace, the CTAs that share one 128-row slab of Q form a thread-block cluster and add
 * their partial sums on chip. With one, they are independent CTAs, enough for two on every SM, that write
 * fp32 partials to the workspace; the last of a slab's CTAs to finish adds them in a fixed order
 * (deterministic, whichever CTA comes last) and writes the output. FN_PATH_AUTO then takes the
 * tensor-core kernel for one token as well.
 *   workspace        device memory, 16-byte aligned, caller-owned, or NULL (no workspace). Its first
 *                    1024 bytes are arrival counters: zero them (cudaMemset) before the workspace's
 *                    first use; every call leaves them zero again. The rest is scratch. Calls whose
 *                    kernels may overlap on the GPU (different streams, host threads) must not share
 *                    one; successive calls on one stream may, whatever their shapes.
 *   workspace_bytes  its size. A non-NULL workspace smaller than flashnorm_fp8_workspace_bytes reports
 *                    for this shape returns FN_ERR_INVALID_ARG and launches nothing.
 * Shapes for which the split does not apply (more 128-row slabs than SMs: the size query returns 0),
 * and FN_PATH_GEMV, ignore the workspace.
 */
FN_API fn_status flashnorm_linear_fp8_ws(const void* x, const void* Q, const void* scales, void* y, int64_t M,
                                         int64_t d, int64_t N, float eps, int out_dtype, int path, void* workspace,
                                         int64_t workspace_bytes, void* stream);

/*
 * flashnorm_fp8_workspace_bytes — the workspace flashnorm_linear_fp8_ws uses for this shape on the current
 * device, written to *bytes: 1024 + slabs x K ranges x (128 x 16 + 16) x 4, or 0 where the split does not
 * apply (M == 0 or M > FN_DECODE_MAX_M included). FN_ERR_INVALID_ARG for a shape flashnorm_linear_fp8
 * rejects as invalid (d % 16 != 0, N % 8 != 0, out-of-range sizes).
 */
FN_API fn_status flashnorm_fp8_workspace_bytes(int64_t M, int64_t d, int64_t N, int64_t* bytes);
FN_API fn_status flashnorm_fp8_workspace_bytes(int64_t M, int64_t d, int64_t N, int64_t* bytes);

/*
 * NVFP4 (4-bit) W* (the same Abstract item: folded checkpoints stay compatible with quantized models).
 * Reading: weight-only; the NVFP4 element and micro-block encoding (E2M1 codes, one E4M3 scale per 16
 * consecutive k of an output channel) with one fp32 scale per output channel in place of the format's
 * per-tensor scale, quantized after the fold:
 *     W*[n][k] = g[k] W[k][n],   s2[n] = max_k |W*[n][k]| / (448 * 6)   (1 for an all-zero channel),
 *     sb[n][b] = E4M3(max_{k in block b} |W*[n][k]| / (6 s2[n])),
 *     Q[n][k]  = E2M1(W*[n][k] / (sb[n][k / 16] s2[n]))   (0 where sb is 0),
 *     y[m][n]  = (sum_k x[m][k] Q[n][k] sb[n][k / 16]) * s2[n] / sqrt(mean_k x[m][k]^2 + eps),
 * products and divisions in fp32, each rounding to nearest even and saturating (E4M3 at 448, E2M1 at 6).
 * Storage of Q and sb (caller-owned, N rows of ceil(d / 256) * 144 bytes): per output channel, groups of
 * 256 k of 144 bytes. Bytes 0..127 of a group are 32 little-endian uint32 words; word j holds the codes of
 * k = 8 j + 2 i in bits 4 i .. 4 i + 3 and of k = 8 j + 2 i + 1 in bits 16 + 4 i .. 16 + 4 i + 3 (i = 0..3,
 * k counted within the group). Byte 128 + b is the E4M3 scale of the group's block b (k = 16 b .. + 15).
 * Past d: zero codes and zero scales.
 * flashnorm_fold_weights_nvfp4: W bf16 [d, N] row-major, g bf16 [d] -> Q4 as above and s2 fp32 [N].
 *   d % 16 == 0, N % 8 == 0.
 * flashnorm_linear_nvfp4: decode (M <= FN_DECODE_MAX_M) on the tensor cores: each code is widened on chip,
 *   exactly, to the bf16 value Q * sb, x is used as it is, fp32 accumulation. x bf16 [M, d], y [M, N] of
 *   out_dtype. workspace / workspace_bytes as for flashnorm_linear_fp8_ws (the first 1024 bytes zero before
 *   first use and left zero by every call; NULL: one CTA per 128-row slab over all of d, slower). Larger M
 *   returns FN_ERR_UNSUPPORTED.
 * flashnorm_nvfp4_workspace_bytes: the workspace flashnorm_linear_nvfp4 uses for this shape on the current
 *   device, 0 where the split does not apply (more 128-row slabs than SMs, M == 0, M > FN_DECODE_MAX_M).
 */
FN_API fn_status flashnorm_fold_weights_nvfp4(const void* W, const void* g, void* Q4, void* s2, int64_t d, int64_t N,
                                              void* stream);
FN_API fn_status flashnorm_linear_nvfp4(const void* x, const void* Q4, const void* s2, void* y, int64_t M, int64_t d,
                                        int64_t N, float eps, int out_dtype, void* workspace, int64_t workspace_bytes,
                                        void* stream);
FN_API fn_status flashnorm_nvfp4_workspace_bytes(int64_t M, int64_t d, int64_t N, int64_t* bytes);

/*
 * flashnorm_rope_table — fills rope_cs (fp32 [max_pos][head_dim / 2][2], caller-owned device memory,
 * 16-byte aligned) with cos and sin of p * base^(-2i/head_dim), computed in double precision and
 * rounded once to fp32. head_dim even, max_pos >= 1, base > 1 (RoFormer uses 10000). Asynchronous on
 * `stream`.
 */
FN_API fn_status flashnorm_rope_table(void* rope_cs, int64_t max_pos, int64_t head_dim, double base, void* stream);

/*
 * The unfused baseline the pages compare against (FlashNorm Abstract: its speedups are stated against a
 * plain norm-then-project pipeline): kernel 1 writes xn = RNE_bf16(x * 1/sqrt(mean(x^2)+eps) * g), kernel 2 runs the
 * same tensor-core GEMM on xn with no scale. Kept for measuring what folding + deferral buy.
 *
 * flashnorm_rmsnorm: x bf16 [M, d], g bf16 [d] -> xn bf16 [M, d] (caller-owned).
 * flashnorm_linear_unfused: W_kmajor bf16 [N, d] is the UNFOLDED weight transposed (fold with g = 1);
 *   xn_ws bf16 [M, d] is caller-owned scratch that receives the normalised activations.
 * flashnorm_glu_unfused: the same for GLU; W_kmajor_gu from fold(glu = 1, g = 1); y [M, F].
 */
FN_API fn_status flashnorm_rmsnorm(const void* x, const void* g, void* xn, int64_t M, int64_t d, float eps,
                            void* stream);
FN_API fn_status flashnorm_linear_unfused(const void* x, const void* g, const void* W_kmajor, void* xn_ws, void* y,
                                   int64_t M, int64_t d, int64_t N, float eps, int out_dtype, void* stream);
FN_API fn_status flashnorm_glu_unfused(const void* x, const void* g, const void* W_kmajor_gu, void* xn_ws, void* y,
                                int64_t M, int64_t d, int64_t F, float eps, int out_dtype, void* stream);

/*
 * flashnorm_linear_unfused_noalloc — flashnorm_linear_unfused without a caller-supplied workspace.
 * The paper has no counterpart to this entry point; it exists for callers that cannot provide one:
 * a drop-in norm+projection op whose interface carries only inputs and outputs, or a caller whose
 * device memory is all handed out by its own pool allocator, so an extra cudaMalloc would fail (and
 * cudaMalloc may synchronise the device, which a latency-bound loop cannot afford).
 * The normalised activations go to a scratch array that is part of the library's device image
 * (16 MiB of bf16, FN_NOALLOC_MAX_ELEMS elements), which every GPU that loads the library keeps until
 * the process exits. This call allocates nothing: no cudaMalloc, cudaFree or allocating routine.
 *   Arguments and results as flashnorm_linear_unfused; M * d must not exceed FN_NOALLOC_MAX_ELEMS
 *   (larger requests return FN_ERR_UNSUPPORTED and launch nothing).
 *   The first call on a device looks up the scratch array's device address on that device (with
 *   that device current) and keeps it for the life of the process; make that first call before any
 *   stream capture. A device reset (cudaDeviceReset, or the primary context torn down and created
 *   again) invalidates the kept address: do not call this entry point on a device after resetting it.
 *   All calls share the one array and it keeps the previous call's contents (every call overwrites
 *   the rows it uses before reading them). Calls whose kernels overlap on the GPU -- on different
 *   streams, or from different host threads -- race on it; serialise them.
 */
#define FN_NOALLOC_MAX_ELEMS (1LL << 23)
FN_API fn_status flashnorm_linear_unfused_noalloc(const void* x, const void* g, const void* W_kmajor, void* y,
                                                  int64_t M, int64_t d, int64_t N, float eps, int out_dtype,
                                                  void* stream);

/*
 * flashnorm_check_device_error — synchronises `stream`, then reads and clears the device-side status
 * word of the current device. Returns FN_ERR_TIMEOUT if any kernel of this library gave up on a bounded
 * wait since the last check, FN_ERR_INVALID_ARG if a RoPE position fell outside its table (see
 * flashnorm_linear_postnorm_rope), FN_ERR_CUDA if the synchronisation itself failed, FN_OK otherwise.
 */
FN_API fn_status flashnorm_check_device_error(void* stream);

/*
 * flashnorm_selftest_timeout — exercises the failure path without faulting anything: launches one
 * thread that waits on a device barrier nothing will complete, bounded by `limit_us` microseconds
 * (and as many thousand SM cycles), then synchronises `stream` and reads the status word like
 * flashnorm_check_device_error. A working library returns FN_ERR_TIMEOUT here and leaves the word
 * cleared and the CUDA context usable for the next call. limit_us must be in [1, 1e7]. (The pages
 * have no counterpart: this checks the library's own bounded waits.)
 */
FN_API fn_status flashnorm_selftest_timeout(int64_t limit_us, void* stream);

/* Static description of a status code. */
FN_API const char* flashnorm_status_string(int status);
/* Detail of the most recent failed call on this host thread ("" if none). */
FN_API const char* flashnorm_last_error(void);
/* ABI version of this library: major * 10000 + minor * 100 + patch. */
FN_API int flashnorm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLASHNORM_H */
