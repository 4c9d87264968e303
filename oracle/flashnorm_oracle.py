"""Plain fp64 CPU oracle for FlashNorm (RMSNorm followed by a linear layer).

TEST INFRASTRUCTURE ONLY. This module is imported by the tests, by
__graft_entry__.smoke() and by the CPU-baseline leg of bench.py. The library itself
never imports it, calls it or falls back to it; it shares no code with the
CUDA kernels (only the seeded input generator feeds both).

Sources. The method is stated in prose in the abstract of "FlashNorm: Fast
Normalization for Transformers" (arXiv 2407.09577; mlsanity paper page and
arxivdaily page, section "Abstract"). The pages print no equation, so each
function below states the plainest reading of that prose:

* RMSNorm (the paper builds on "Root Mean Square Layer Normalization", listed
  under "Builds on"): RMSNorm(x) = x / sqrt(mean(x^2) + eps) * g, the mean
  taken over the d features of one row, eps inside the square root.
* (i) weight folding: the gain g is folded into the next linear layer,
  W* = diag(g) . W.
* (ii) deferred normalization: the scalar 1/rms is applied to the output of
  the matrix multiplication, y = (x . W*) * 1/sqrt(mean(x^2) + eps).
* GLU feed-forward variant (the abstract lists gated feed-forward layers among
  the cases the techniques extend to): the deferred scale is applied to the
  gate and the up outputs before SiLU, y = silu(z_gate) * z_up,
  silu(t) = t / (1 + exp(-t)).
* Redundant-norm removal (with a linear layer between two RMSNorms, the abstract
  drops the first norm by the scale invariance of RMS): linear -> RMSNorm
  replaces RMSNorm -> linear -> RMSNorm.
* LayerNorm (the abstract says the techniques extend to it): gamma folded,
  1/sqrt(var + eps) deferred, the mean removed by a rank-1 term with the column
  sums of W*, beta turned into a bias vector.
* RoPE on the normalised query/key heads (the abstract names RoPE-based
  attention; the paper builds on RoFormer): pairs (2i, 2i+1) of a head rotated
  by pos * base^(-2i/head_dim), RoFormer's own pairing.
* Quantized W* (the abstract: folded checkpoints stay compatible with quantized
  models): weight-only FP8 E4M3 with one scale per output channel, and NVFP4
  (E2M1 elements, an E4M3 scale per 16 k, a per-channel fp32 scale), both
  quantized after the fold, the channel scale applied with the deferred 1/rms.

Everything is computed in float64 from inputs given as bf16 bit patterns; the
only library primitive is numpy's float64 matrix product. No blocking, fusion
or reordering beyond the formulas above.

Every function here is pinned by the CPU tests (hand-worked golden cases,
closed forms, invariants, brute force in exact arithmetic, and torch's own
CPU RMSNorm / SiLU / bf16 conversion on the special cases they cover). None is
"parity unpinned".
"""

from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------------------
# bf16 encoding (IEEE-754 binary32 truncated to 16 bits: 1 sign, 8 exponent,
# 7 stored mantissa bits; 8 significant bits with the implicit one).
# ---------------------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    """Decode bf16 bit patterns exactly to float64.

    Source: the bf16 format itself (the top 16 bits of an IEEE-754 binary32), not the pages.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    """Round float64 values to bf16 with round-to-nearest, ties to even.

    Written from the definition: a finite value is rounded to a multiple of
    its quantum, 2^(e-8) for |v| in [2^(e-1), 2^e) (8 significant bits), with
    the quantum floored at 2^-133 (bf16 subnormals). np.rint rounds halfway
    cases to the even integer, which is ties-to-even on the significand.
    Magnitudes that round to 2^128 or beyond become infinities.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    finite = np.isfinite(v)
    vf = np.where(finite, v, 0.0)
    _, e = np.frexp(vf)
    quantum = np.ldexp(1.0, np.maximum(e - 8, -133))
    r = np.rint(vf / quantum) * quantum
    with np.errstate(over="ignore"):
        r32 = r.astype(np.float32)  # exact: r has at most 8 significant bits
    bits = (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    out[...] = bits
    nan = np.isnan(v)
    out[nan] = np.uint16(0x7FC0)
    posinf = np.isposinf(v)
    neginf = np.isneginf(v)
    out[posinf] = np.uint16(0x7F80)
    out[neginf] = np.uint16(0xFF80)
    return out


# ---------------------------------------------------------------------------
# RMSNorm and the unfolded, undeferred chain (the plain definition).
# ---------------------------------------------------------------------------

def inv_rms(x: np.ndarray, eps: float) -> np.ndarray:
    """Per-row 1 / sqrt(mean_i x_i^2 + eps), mean over the feature axis.

    Source: the RMSNorm definition ("Root Mean Square Layer Normalization", the paper it builds on); the
    scalar the "FlashNorm: Fast Normalization for Transformers", Abstract item (ii) defers.
    """
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1)
    return 1.0 / np.sqrt(ms + eps)


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm(x) = x / sqrt(mean(x^2) + eps) * g, row-wise.

    Source: "Root Mean Square Layer Normalization", the RMSNorm definition the FlashNorm paper builds
    on.
    """
    x = np.asarray(x, dtype=np.float64)
    return x * inv_rms(x, eps)[..., None] * np.asarray(g, dtype=np.float64)


def norm_then_project(x, g, W, eps):
    """The operation FlashNorm reformulates: RMSNorm(x) . W, W of shape [d, N].

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, the RMSNorm -> linear pair the
    method starts from.
    """
    return rmsnorm(x, g, eps) @ np.asarray(W, dtype=np.float64)


# ---------------------------------------------------------------------------
# (i) Weight folding and (ii) deferred normalization.
# ---------------------------------------------------------------------------

def fold(W, g) -> np.ndarray:
    """W* = diag(g) . W in float64 (row i of W scaled by g_i).

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, item (i), weight folding.
    """
    return np.asarray(g, dtype=np.float64)[:, None] * np.asarray(W, dtype=np.float64)


def fold_bf16(w_bits, g_bits) -> np.ndarray:
    """W* rounded once to bf16: bits of RNE(g_i * W_ij), same [d, N] shape as W.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, item (i); the single RNE
    rounding to bf16 is the reading that makes the fold exact to check.
    """
    return f64_to_bf16(fold(bf16_to_f64(w_bits), bf16_to_f64(g_bits)))


def deferred(x, Wstar, eps):
    """(x . W*) scaled per row by 1/sqrt(mean(x^2) + eps): the reformulated form.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, item (ii), deferred
    normalization.
    """
    x = np.asarray(x, dtype=np.float64)
    return (x @ np.asarray(Wstar, dtype=np.float64)) * inv_rms(x, eps)[:, None]


# ---------------------------------------------------------------------------
# GLU (SwiGLU) feed-forward variant. W has 2F columns: gate = [0, F), up = [F, 2F).
# ---------------------------------------------------------------------------

def silu(t):
    """SiLU(t) = t / (1 + exp(-t)).

    Source: the SiLU of the gated feed-forward layers that "FlashNorm: Fast Normalization for
    Transformers", Abstract names among the extensions.
    """
    t = np.asarray(t, dtype=np.float64)
    with np.errstate(over="ignore"):
        return t / (1.0 + np.exp(-t))


def glu_norm_then_project(x, g, W_gu, eps):
    """silu(z_gate) * z_up with z = RMSNorm(x) . W (unfolded, undeferred)."""
    z = norm_then_project(x, g, W_gu, eps)
    F = z.shape[1] // 2
    return silu(z[:, :F]) * z[:, F:]


def glu_deferred(x, Wstar_gu, eps):
    """silu(r * (x . W*_gate)) * (r * (x . W*_up)), r = 1/rms(x): scale before SiLU.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, the GLU variants: the deferred
    scale goes on gate and up before SiLU.
    """
    x = np.asarray(x, dtype=np.float64)
    r = inv_rms(x, eps)[:, None]
    z = x @ np.asarray(Wstar_gu, dtype=np.float64)
    F = z.shape[1] // 2
    return silu(r * z[:, :F]) * (r * z[:, F:])


# ---------------------------------------------------------------------------
# Redundant-norm removal: RMSNorm -> linear -> RMSNorm becomes linear -> RMSNorm.
# The second norm acts per head of width head_dim with a shared gain g2.
# ---------------------------------------------------------------------------

def _per_head_rmsnorm(v, g2, eps2, head_dim):
    """RMSNorm over each head of head_dim consecutive features of a row, one gain g2 [head_dim] for all
    heads.

    Source: the per-head (query/key) norm of the redundant-norm case in "FlashNorm: Fast Normalization
    for Transformers", Abstract; a head as the unit is the reading for QK-norm models.
    """
    M, N = v.shape
    vh = v.reshape(M, N // head_dim, head_dim)
    return rmsnorm(vh, g2, eps2).reshape(M, N)


def postnorm_full(x, g1, W, g2, eps1, eps2, head_dim):
    """The full chain: per-head RMSNorm(RMSNorm(x; g1) . W; g2). Keeps the first norm."""
    v = norm_then_project(x, g1, W, eps1)
    return _per_head_rmsnorm(v, g2, eps2, head_dim)


def postnorm_elided(x, Wstar1, g2, eps2, head_dim):
    """The first norm dropped: per-head RMSNorm(x . W*1; g2), with g1 folded into W*1."""
    u = np.asarray(x, dtype=np.float64) @ np.asarray(Wstar1, dtype=np.float64)
    return _per_head_rmsnorm(u, g2, eps2, head_dim)


def postnorm_elided_exact_eps(x, Wstar1, g2, eps1, eps2, head_dim):
    """What the full chain equals when eps1, eps2 > 0, written through u = x . W*1.

    With v = u * r1 and r1 = 1/sqrt(ms_x + eps1), mean(v^2) = r1^2 mean(u^2), so
    v / sqrt(mean(v^2) + eps2) = u / sqrt(mean(u^2) + eps2 (ms_x + eps1)).
    The elided form drops the eps2 (ms_x + eps1) correction; it is exact at eps = 0.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, redundant-norm removal by scale
    invariance; this is that identity with eps kept.
    """
    x = np.asarray(x, dtype=np.float64)
    u = x @ np.asarray(Wstar1, dtype=np.float64)
    M, N = u.shape
    uh = u.reshape(M, N // head_dim, head_dim)
    ms_x = np.mean(x * x, axis=-1)
    denom = np.sqrt(np.mean(uh * uh, axis=-1) + eps2 * (ms_x + eps1)[:, None])
    return (uh / denom[..., None] * np.asarray(g2, dtype=np.float64)).reshape(M, N)


# ---------------------------------------------------------------------------
# Quantized W* (the abstract: the folded checkpoints stay compatible with
# quantized models). Reading: weight-only fp8 E4M3 with one
# scale per output channel, quantized AFTER the fold, so the gain is folded into
# the quantized weight and the deferred 1/rms is applied with the channel scale:
#   W*[n, k] = g[k] W[k, n] (exact: a bf16 x bf16 product fits fp32),
#   s[n] = max_k |W*[n, k]| / 448 (fp32; 1 if the channel is all zero),
#   Q[n, k] = E4M3_rne(W*[n, k] / s[n]) (fp32 division),
#   y[m, n] = (sum_k x[m, k] dec(Q[n, k])) * s[n] * 1/sqrt(mean(x^2) + eps).
# The scale and the codes are integer decisions taken in fp32, the kernel's
# precision, so the oracle takes them in np.float32 too and the codes match bit
# for bit. E4M3 ("fn" variant): 1 sign bit, 4 exponent bits with bias 7, 3
# mantissa bits; normals 2^-6 .. 448, subnormals in steps of 2^-9, no infinity.
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def f64_to_e4m3(v) -> np.ndarray:
    """Round to E4M3 with round-to-nearest, ties to even, saturating at +-448; return the codes (uint8).

    Written from the format: a value in [2^e, 2^(e+1)) with e >= -6 is a multiple of 2^(e-3) (4
    significant bits); below 2^-6 the quantum is 2^-9. np.rint rounds halfway cases to the even integer.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    _, e = np.frexp(a)                       # a = f * 2^e, f in [0.5, 1): a in [2^(e-1), 2^e)
    q = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    r = np.minimum(np.rint(a / q) * q, E4M3_MAX)
    # encode r (now exactly representable)
    _, er = np.frexp(r)
    ex = er - 1                              # r in [2^ex, 2^(ex+1))
    normal = r >= 2.0 ** -6
    mant_n = np.where(normal, np.rint((np.ldexp(r, -np.where(normal, ex, 0)) - 1.0) * 8.0), 0)
    code_n = ((np.where(normal, ex, 0) + 7) << 3) + mant_n.astype(np.int64)
    code_s = np.rint(r / 2.0 ** -9).astype(np.int64)     # subnormals (and zero): m * 2^-9
    code = np.where(normal, code_n, code_s).astype(np.int64)
    code = code | np.where(np.signbit(v), 0x80, 0)  # the sign is kept, also on values that round to zero
    return code.astype(np.uint8)


def e4m3_to_f64(codes) -> np.ndarray:
    """Decode E4M3 codes exactly (0x7F / 0xFF, the NaN codes, never produced by f64_to_e4m3, decode as NaN)."""
    c = np.asarray(codes, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


def fold_fp8(w_bits, g_bits):
    """(codes uint8 [N, d], scales float32 [N]): the fold, then per-channel E4M3 quantization, in fp32."""
    W = (np.asarray(w_bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    g = (np.asarray(g_bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    Ws = (g[:, None] * W).T.astype(np.float32)            # [N, d], exact products
    amax = np.max(np.abs(Ws), axis=1)
    scales = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    v = (Ws / scales[:, None]).astype(np.float32)          # IEEE fp32 division
    return f64_to_e4m3(v.astype(np.float64)), scales


def deferred_fp8(x, codes, scales, eps):
    """y = (x . dec(Q)^T) * s * 1/sqrt(mean(x^2) + eps), in fp64.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, folded weights staying
    compatible with quantized models; the E4M3 per-channel scheme is the reading stated at fold_fp8.
    """
    x = np.asarray(x, dtype=np.float64)
    Wq = e4m3_to_f64(codes) * np.asarray(scales, dtype=np.float64)[:, None]   # [N, d]
    return (x @ Wq.T) * inv_rms(x, eps)[:, None]


# ---------------------------------------------------------------------------
# NVFP4 (4-bit) W*, the second quantized format. Reading: weight-only, the
# NVFP4 element and micro-block encoding (E2M1 elements, one E4M3 scale per 16
# consecutive elements along the contraction dimension k), and, in place of the
# format's per-tensor fp32 scale, one fp32 scale per output channel, so that it
# multiplies the output together with the deferred 1/rms as the fp8 channel
# scale does. Quantized after the fold:
#   W*[n, k] = g[k] W[k, n] (exact in fp32),
#   s2[n] = max_k |W*[n, k]| / (448 * 6) (fp32; 1 if the channel is all zero),
#   sb[n, b] = E4M3_rne(max_{k in block b} |W*[n, k]| / (6 * s2[n])) (the
#              product 6 * s2[n] rounded to fp32, then the fp32 division),
#   Q[n, k] = E2M1_rne(W*[n, k] / (dec(sb[n, b]) * s2[n])) (the product rounded
#             to fp32, then the fp32 division; 0 where dec(sb) is 0),
#   y[m, n] = (sum_k x[m, k] dec(Q[n, k]) dec(sb[n, k // 16])) * s2[n] / rms(x_m).
# E2M1: 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit: magnitudes
# 0, 0.5, 1, 1.5, 2, 3, 4, 6 (0.5 is the one subnormal); no infinity, no NaN.
# The library stores the codes packed (see pack_nvfp4); the oracle keeps them
# one per array element.
# ---------------------------------------------------------------------------

E2M1_MAX = 6.0


def f64_to_e2m1(v) -> np.ndarray:
    """Round to E2M1 with round-to-nearest, ties to even, saturating at +-6; return the 4-bit codes (uint8).

    Written from the format: a magnitude in [2^e, 2^(e+1)) with e >= 0 is a multiple of 2^(e-1) (2
    significant bits); below 1 the quantum is 0.5. np.rint rounds halfway cases to the even integer.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    _, e = np.frexp(a)                       # a in [2^(e-1), 2^e)
    q = np.ldexp(1.0, np.maximum(e - 1, 0) - 1)
    r = np.minimum(np.rint(a / q) * q, E2M1_MAX)
    _, er = np.frexp(r)
    ex = er - 1                              # r in [2^ex, 2^(ex+1))
    normal = r >= 1.0
    mant = np.where(normal, np.rint((np.ldexp(r, -np.where(normal, ex, 0)) - 1.0) * 2.0), 0)
    code_n = ((np.where(normal, ex, 0) + 1) << 1) + mant.astype(np.int64)
    code_s = np.rint(r / 0.5).astype(np.int64)          # 0 or 0.5
    code = np.where(normal, code_n, code_s).astype(np.int64)
    code = code | np.where(np.signbit(v), 0x8, 0)
    return code.astype(np.uint8)


def e2m1_to_f64(codes) -> np.ndarray:
    """Decode E2M1 codes (the low 4 bits) exactly."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    s = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    val = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.ldexp(1.0, e - 1))
    return s * val


NVFP4_BLOCK = 16


def fold_nvfp4(w_bits, g_bits):
    """(codes uint8 [N, d] one E2M1 code each, block scales uint8 [N, ceil(d/16)] E4M3, s2 float32 [N]): the
    fold, then NVFP4 quantization with a per-channel second-level scale, every decision in fp32."""
    W = (np.asarray(w_bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    g = (np.asarray(g_bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    Ws = (g[:, None] * W).T.astype(np.float32)            # [N, d], exact products
    N, d = Ws.shape
    nb = -(-d // NVFP4_BLOCK)
    amax = np.max(np.abs(Ws), axis=1)
    s2 = np.where(amax > 0, amax / np.float32(E4M3_MAX * E2M1_MAX), np.float32(1.0)).astype(np.float32)
    pad = np.zeros((N, nb * NVFP4_BLOCK), dtype=np.float32)
    pad[:, :d] = Ws
    blocks = pad.reshape(N, nb, NVFP4_BLOCK)
    bmax = np.max(np.abs(blocks), axis=2)                   # [N, nb]
    six_s2 = (np.float32(E2M1_MAX) * s2).astype(np.float32)
    bscale = f64_to_e4m3((bmax / six_s2[:, None]).astype(np.float32).astype(np.float64))
    dsb = e4m3_to_f64(bscale).astype(np.float32)            # exact in fp32
    den = (dsb * s2[:, None]).astype(np.float32)             # [N, nb], one fp32 rounding
    safe = np.where(den > 0, den, np.float32(1.0)).astype(np.float32)
    t = (blocks / safe[:, :, None]).astype(np.float32)       # IEEE fp32 division
    t = np.where(den[:, :, None] > 0, t, np.float32(0.0))
    codes = f64_to_e2m1(t.astype(np.float64)).reshape(N, nb * NVFP4_BLOCK)[:, :d]
    return codes, bscale, s2


def dequant_nvfp4(codes, bscales, s2) -> np.ndarray:
    """W*q [N, d] in fp64: dec(Q) * dec(sb) * s2."""
    codes = np.asarray(codes)
    d = codes.shape[1]
    sb = e4m3_to_f64(bscales)[:, np.arange(d) // NVFP4_BLOCK]
    return e2m1_to_f64(codes) * sb * np.asarray(s2, dtype=np.float64)[:, None]


def deferred_nvfp4(x, codes, bscales, s2, eps):
    """y = (x . (dec(Q) dec(sb))^T) * s2 * 1/sqrt(mean(x^2) + eps), in fp64.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, folded weights staying
    compatible with quantized models; the NVFP4 scheme is the reading stated at fold_nvfp4.
    """
    x = np.asarray(x, dtype=np.float64)
    return (x @ dequant_nvfp4(codes, bscales, s2).T) * inv_rms(x, eps)[:, None]


NVFP4_GROUP = 256          # k per packed group
NVFP4_GROUP_BYTES = 144    # 128 bytes of codes + 16 block scales


def pack_nvfp4(codes, bscales) -> np.ndarray:
    """The library's storage of NVFP4 W*: per output channel, groups of 256 k of 144 bytes each. Bytes
    0..127 of group G are 32 little-endian 32-bit words; word j holds the codes of k = 256 G + 8 j + 2 i
    in bits 4 i .. 4 i + 3 and of k = 256 G + 8 j + 2 i + 1 in bits 16 + 4 i .. 16 + 4 i + 3 (i = 0..3):
    the even k in the low half, the odd k in the high half. Byte 128 + b holds the E4M3 scale of block b
    (k = 256 G + 16 b .. + 15). A last partial group is padded with zero codes and zero scales. Returns
    uint8 [N, ceil(d/256) * 144]."""
    codes = np.asarray(codes, dtype=np.uint8)
    bscales = np.asarray(bscales, dtype=np.uint8)
    N, d = codes.shape
    G = -(-d // NVFP4_GROUP)
    c = np.zeros((N, G * NVFP4_GROUP), dtype=np.uint32)
    c[:, :d] = codes & 0xF
    c = c.reshape(N, G, NVFP4_GROUP // 8, 4, 2)             # [n, group, word, i, even/odd]
    shifts = (4 * np.arange(4, dtype=np.uint32))[:, None] + np.array([0, 16], dtype=np.uint32)[None, :]
    words = np.bitwise_or.reduce(c << shifts, axis=(3, 4)).astype(np.uint32)   # [n, group, 32]
    s = np.zeros((N, G * NVFP4_GROUP // NVFP4_BLOCK), dtype=np.uint8)
    s[:, :bscales.shape[1]] = bscales
    packed = np.concatenate([words.astype("<u4").view(np.uint8).reshape(N, G, 128),
                             s.reshape(N, G, NVFP4_GROUP // NVFP4_BLOCK)], axis=2)
    return packed.reshape(N, G * NVFP4_GROUP_BYTES)


# ---------------------------------------------------------------------------
# LayerNorm -> linear. The abstract says the same techniques extend to
# LayerNorm; the pages give no formula. Reading: the standard LayerNorm over the
# d features of a row, biased variance, eps inside the root, gain gamma and bias
# beta:  LN(x) = (x - mu) / sqrt(var + eps) * gamma + beta,
#        mu = mean(x), var = mean((x - mu)^2).
# Folded and deferred the way the abstract does it for RMSNorm: gamma goes into
# W* = diag(gamma) W, the scalar 1/sqrt(var + eps) moves behind the product, and
# the mean subtraction, being x - mu 1, becomes a rank-1 term with the column
# sums c = 1^T W*; beta becomes the bias b = beta^T W:
#        LN(x) . W = r (x . W* - mu c) + b,   r = 1 / sqrt(var + eps).
# ---------------------------------------------------------------------------

def layernorm(x, gamma, beta, eps):
    """LayerNorm over the last axis (biased variance, two passes), float64.

    Source: the standard LayerNorm definition, which "FlashNorm: Fast Normalization for Transformers",
    Abstract says the techniques extend to.
    """
    x = np.asarray(x, dtype=np.float64)
    mu = np.mean(x, axis=-1, keepdims=True)
    var = np.mean((x - mu) ** 2, axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, dtype=np.float64) + np.asarray(beta, dtype=np.float64)


def layernorm_then_project(x, gamma, beta, W, eps):
    """The definition: LN(x; gamma, beta) . W."""
    return layernorm(x, gamma, beta, eps) @ np.asarray(W, dtype=np.float64)


def layernorm_fold(W, gamma, beta):
    """(W* = diag(gamma) W, c = 1^T W*, b = beta^T W), float64.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, item (i) applied to LayerNorm,
    with the mean as a rank-1 term (the extension the abstract names).
    """
    Ws = fold(W, gamma)
    return Ws, np.sum(Ws, axis=0), np.asarray(beta, dtype=np.float64) @ np.asarray(W, dtype=np.float64)


def layernorm_deferred(x, Wstar, colsum, bias, eps):
    """The folded, deferred form: r (x . W* - mu c) + b with r = 1/sqrt(var + eps).

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, item (ii) applied to LayerNorm.
    """
    x = np.asarray(x, dtype=np.float64)
    mu = np.mean(x, axis=-1)
    var = np.mean((x - mu[:, None]) ** 2, axis=-1)
    r = 1.0 / np.sqrt(var + eps)
    acc = x @ np.asarray(Wstar, dtype=np.float64)
    return r[:, None] * (acc - mu[:, None] * np.asarray(colsum, dtype=np.float64)[None, :]) + \
        np.asarray(bias, dtype=np.float64)[None, :]


# ---------------------------------------------------------------------------
# Rotary position embedding on the normalised heads. The abstract lists RoPE-based
# attention among the cases the techniques extend to, and the paper builds on
# "RoFormer: Enhanced Transformer with Rotary Position Embedding" (mlsanity page,
# "Builds on"). The pages give no formula; the reading taken is RoFormer's own:
# the features of a head are paired as (2i, 2i+1), i = 0 .. head_dim/2 - 1, and
# pair i of the token at position p is rotated by the angle p * base^(-2i/head_dim).
# In a fused q/k/v projection with per-head normalisation, the rotation applies
# to the query and key heads (the first n_rope_heads heads of a row); the value
# heads are only normalised.
# ---------------------------------------------------------------------------

def rope_table(max_pos: int, head_dim: int, base: float) -> np.ndarray:
    """(cos, sin) of the rotation angles, float64 [max_pos, head_dim/2, 2].

    Source: RoFormer's rotary embedding (the paper builds on it; "FlashNorm: Fast Normalization for
    Transformers", Abstract names RoPE-based attention).
    """
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = np.power(float(base), -2.0 * i / head_dim)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1)


def apply_rope(v, cs, positions, head_dim: int, n_rope_heads: int) -> np.ndarray:
    """Rotate pairs (2i, 2i+1) of the first n_rope_heads heads of every row of v [M, N].

    cs is a (cos, sin) table [max_pos, head_dim/2, 2] (any float type; widened to
    float64) and positions [M] the position of each row.

    Source: RoFormer's rotary embedding, adjacent-pair form.
    """
    v = np.array(v, dtype=np.float64, copy=True)
    M, N = v.shape
    cs = np.asarray(cs, dtype=np.float64)[np.asarray(positions, dtype=np.int64)]  # [M, hd/2, 2]
    c, s = cs[..., 0], cs[..., 1]
    vh = v.reshape(M, N // head_dim, head_dim)
    for h in range(min(n_rope_heads, N // head_dim)):
        a = vh[:, h, 0::2].copy()
        b = vh[:, h, 1::2].copy()
        vh[:, h, 0::2] = a * c - b * s
        vh[:, h, 1::2] = a * s + b * c
    return vh.reshape(M, N)


def postnorm_rope_full(x, g1, W, g2, eps1, eps2, head_dim, positions, n_rope_heads, base):
    """The full chain with RoPE: rotate(per-head RMSNorm(RMSNorm(x; g1) . W; g2)), exact trig."""
    v = postnorm_full(x, g1, W, g2, eps1, eps2, head_dim)
    table = rope_table(int(np.max(positions)) + 1, head_dim, base)
    return apply_rope(v, table, positions, head_dim, n_rope_heads)


# ---------------------------------------------------------------------------
# The unfused norm-then-project pipeline the pages compare against: the norm
# output is materialised in bf16 (one rounding), then multiplied by W.
# ---------------------------------------------------------------------------

def unfused_norm_then_project(x, g, W, eps):
    """bf16(RMSNorm(x; g)) . W, the two-kernel baseline with its bf16 intermediate."""
    xn = bf16_to_f64(f64_to_bf16(rmsnorm(x, g, eps)))
    return xn @ np.asarray(W, dtype=np.float64)


# ---------------------------------------------------------------------------
# Convenience wrappers on bf16 bit arrays (what the tests and the bench feed).
# ---------------------------------------------------------------------------

def reference_output(kind: str, bits: dict, eps: float, *, eps2: float = 0.0, head_dim: int = 0,
                     rows=None) -> np.ndarray:
    """Oracle output of a workload from its bf16 input bits, optionally for a subset of rows.

    kind "linear": RMSNorm(x; g) . W.   kind "glu": silu(z_gate) * z_up.
    kind "postnorm": the full RMSNorm -> linear -> per-head RMSNorm chain with
    g1 = bits["g"], g2 = bits["g2"], eps1 = eps.
    """
    x = bf16_to_f64(bits["x"])
    if rows is not None:
        x = x[rows]
    g = bf16_to_f64(bits["g"])
    W = bf16_to_f64(bits["w"])
    if kind == "linear":
        return norm_then_project(x, g, W, eps)
    if kind == "glu":
        return glu_norm_then_project(x, g, W, eps)
    if kind == "postnorm":
        return postnorm_full(x, g, W, bf16_to_f64(bits["g2"]), eps, eps2, head_dim)
    raise ValueError(kind)


def exact_operand_output(kind: str, bits: dict, wstar_bits, eps: float, *, eps2: float = 0.0,
                         head_dim: int = 0, rows=None) -> np.ndarray:
    """Oracle of the reformulated form on the bf16 W* (given as [d, N] bits).

    Used for fp32 outputs, where the fold's own bf16 rounding of W* would
    otherwise dominate the comparison.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, items (i) and (ii), evaluated on
    the rounded operands.
    """
    x = bf16_to_f64(bits["x"])
    if rows is not None:
        x = x[rows]
    Ws = bf16_to_f64(wstar_bits)
    if kind == "linear":
        return deferred(x, Ws, eps)
    if kind == "glu":
        return glu_deferred(x, Ws, eps)
    if kind == "postnorm":
        return postnorm_elided(x, Ws, bf16_to_f64(bits["g2"]), eps2, head_dim)
    raise ValueError(kind)


def reference_postnorm_rope(bits: dict, eps: float, eps2: float, head_dim: int, positions, n_rope_heads: int,
                            base: float, rows=None) -> np.ndarray:
    """Oracle of the full RMSNorm -> linear -> per-head RMSNorm -> RoPE chain (first norm kept)."""
    x = bf16_to_f64(bits["x"])
    pos = np.asarray(positions)
    if rows is not None:
        x, pos = x[rows], pos[rows]
    return postnorm_rope_full(x, bf16_to_f64(bits["g"]), bf16_to_f64(bits["w"]), bf16_to_f64(bits["g2"]), eps, eps2,
                              head_dim, pos, n_rope_heads, base)


def exact_operand_postnorm_rope(bits: dict, wstar_bits, eps2: float, head_dim: int, positions, n_rope_heads: int,
                                table, rows=None) -> np.ndarray:
    """The elided post-norm on the bf16 W*, rotated with the given (cos, sin) table: the fp32-output bar.

    Source: "FlashNorm: Fast Normalization for Transformers", Abstract, redundant-norm removal, then
    RoFormer's rotation.
    """
    x = bf16_to_f64(bits["x"])
    pos = np.asarray(positions)
    if rows is not None:
        x, pos = x[rows], pos[rows]
    u = postnorm_elided(x, bf16_to_f64(wstar_bits), bf16_to_f64(bits["g2"]), eps2, head_dim)
    return apply_rope(u, table, pos, head_dim, n_rope_heads)


def exact_operand_fp8(bits: dict, eps: float, rows=None) -> np.ndarray:
    """The quantized path on its own operands: the oracle's fold_fp8 codes and scales (the library's fold
    matches them bit for bit), then y = (x . dec(Q)^T) * s * 1/rms in fp64.

    Source: as deferred_fp8.
    """
    x = bf16_to_f64(bits["x"])
    if rows is not None:
        x = x[rows]
    codes, scales = fold_fp8(bits["w"], bits["g"])
    return deferred_fp8(x, codes, scales, eps)


def exact_operand_nvfp4(bits: dict, eps: float, rows=None) -> np.ndarray:
    """The NVFP4 path on its own operands: the oracle's fold_nvfp4 codes and scales (the library's fold
    matches them bit for bit), then y = (x . Wq^T) * s2 * 1/rms in fp64.

    Source: as deferred_nvfp4.
    """
    x = bf16_to_f64(bits["x"])
    if rows is not None:
        x = x[rows]
    codes, bscales, s2 = fold_nvfp4(bits["w"], bits["g"])
    return deferred_nvfp4(x, codes, bscales, s2, eps)


def reference_layernorm(bits: dict, eps: float, rows=None) -> np.ndarray:
    """Oracle of LN(x; gamma = bits["g"], beta = bits["beta"]) . W from bf16 bits (the definition)."""
    x = bf16_to_f64(bits["x"])
    if rows is not None:
        x = x[rows]
    return layernorm_then_project(x, bf16_to_f64(bits["g"]), bf16_to_f64(bits["beta"]), bf16_to_f64(bits["w"]), eps)


def exact_operand_layernorm(bits: dict, wstar_bits, eps: float, rows=None) -> np.ndarray:
    """The folded, deferred form on the bf16 W* (colsum from its bf16 values, bias from W and beta).

    Source: as layernorm_deferred.
    """
    x = bf16_to_f64(bits["x"])
    if rows is not None:
        x = x[rows]
    Ws = bf16_to_f64(wstar_bits)
    bias = bf16_to_f64(bits["beta"]) @ bf16_to_f64(bits["w"])
    return layernorm_deferred(x, Ws, np.sum(Ws, axis=0), bias, eps)


def rel_err(y, y_ref) -> float:
    """max |y - y_ref| / max |y_ref|, the parity metric.

    Source: not the pages; the parity metric the tests state.
    """
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    denom = np.max(np.abs(y_ref))
    return float(np.max(np.abs(y - y_ref)) / denom) if denom > 0 else float(np.max(np.abs(y - y_ref)))
