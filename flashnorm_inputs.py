"""Seeded synthetic inputs for the FlashNorm RMSNorm -> linear path.

This module only draws random numbers and stores them as bf16 bit patterns.
It holds none of the method's arithmetic (no norm, no fold, no contraction), so
that the fp64 oracle and the CUDA library can both be fed from it without
sharing any computation.

Distributions (the workloads named for SmolLM2-135M, Llama-7B and a
DeepSeek-V2-like MLA latent in the FlashNorm abstract, "FlashNorm: Fast
Normalization for Transformers", Abstract): the pages give no tensor
statistics, so the recipe is synthetic:

* activations x[M, d]: N(0, 1) per element, times a per-row scale drawn
  log-uniformly from [0.1, 10] (so rows span two decades of RMS);
* norm gain g[d]: U(0.5, 1.5);
* projection weight W[d, N]: N(0, 1/d) (row-major, y = x . W).

Every tensor is drawn in float32 from numpy's PCG64 stream keyed by
(seed, tensor tag), then rounded to bf16 with round-to-nearest-even. Values
are returned as ``uint16`` bit patterns; callers decode them as they see fit.
"""

from __future__ import annotations

import dataclasses

import numpy as np

BASE_SEED = 24070957

_TAGS = {"x": 1, "g": 2, "w": 3, "g2": 4, "w2": 5, "beta": 6}


def _rng(seed: int, tag: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), _TAGS[tag]]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    out = r.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def activations(M: int, d: int, seed: int) -> np.ndarray:
    """x[M, d] as bf16 bits: N(0,1) times a per-row log-uniform [0.1, 10] scale."""
    rng = _rng(seed, "x")
    row_scale = np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=(M, 1))).astype(np.float32)
    x = rng.standard_normal(size=(M, d), dtype=np.float32)
    x *= row_scale
    return f32_to_bf16_bits(x)


def activations_offset(M: int, d: int, seed: int) -> np.ndarray:
    """x[M, d] as bf16 bits for the LayerNorm cases: per row, (N(0,1) + a mean offset drawn from U(-1, 1))
    times a log-uniform [0.1, 10] scale, so that the mean subtraction matters."""
    rng = _rng(seed, "x")
    row_scale = np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=(M, 1))).astype(np.float32)
    offset = rng.uniform(-1.0, 1.0, size=(M, 1)).astype(np.float32)
    x = rng.standard_normal(size=(M, d), dtype=np.float32)
    x = (x + offset) * row_scale
    return f32_to_bf16_bits(x)


def bias(d: int, seed: int) -> np.ndarray:
    """beta[d] as bf16 bits: U(-0.5, 0.5)."""
    rng = _rng(seed, "beta")
    return f32_to_bf16_bits(rng.uniform(-0.5, 0.5, size=d).astype(np.float32))


def gain(d: int, seed: int, tag: str = "g") -> np.ndarray:
    """g[d] as bf16 bits: U(0.5, 1.5)."""
    rng = _rng(seed, tag)
    return f32_to_bf16_bits(rng.uniform(0.5, 1.5, size=d).astype(np.float32))


def weight(d: int, N: int, seed: int, tag: str = "w") -> np.ndarray:
    """W[d, N] row-major as bf16 bits: N(0, 1/d)."""
    rng = _rng(seed, tag)
    w = rng.standard_normal(size=(d, N), dtype=np.float32)
    w *= np.float32(1.0 / np.sqrt(d))
    return f32_to_bf16_bits(w)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic problem: shapes, epsilon and the variant it exercises."""

    name: str
    kind: str  # "linear" | "glu" | "postnorm" | "postnorm_rope" | "layernorm" | "linear_fp8" | "linear_nvfp4"
    M: int
    d: int
    N: int  # linear: output columns; glu: F (W has 2F columns); postnorm: latent width
    eps: float
    head_dim: int = 0  # postnorm only
    eps2: float = 0.0  # postnorm only
    seed: int = BASE_SEED
    n_rope_heads: int = 0  # postnorm_rope: heads of a row that are rotated (the q and k heads come first)
    rope_base: float = 10000.0

    @property
    def w_cols(self) -> int:
        return 2 * self.N if self.kind == "glu" else self.N

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of the contraction (2 * M * d * columns of W)."""
        return 2 * self.M * self.d * self.w_cols

    @property
    def bytes(self) -> int:
        """Algorithmic HBM bytes: read x and W* once, write y once (bf16); with RoPE also each row's
        position and its fp32 (cos, sin) table row."""
        b = 2 * (self.M * self.d + self.d * self.w_cols + self.M * self.N)
        if self.kind == "postnorm_rope":
            b += 4 * self.M + 4 * self.M * self.head_dim
        if self.kind == "linear_fp8":  # one byte per weight plus a fp32 scale per output channel
            b = 2 * (self.M * self.d + self.M * self.N) + self.d * self.N + 4 * self.N
        if self.kind == "linear_nvfp4":  # half a byte per weight, a byte per 16 weights, a fp32 scale per channel
            b = 2 * (self.M * self.d + self.M * self.N) + self.N * (self.d // 2 + self.d // 16 + 4)
        return b

    def positions(self) -> np.ndarray:
        """Positions of the rows (postnorm_rope): a prefill of M tokens, 0 .. M-1, int32."""
        return np.arange(self.M, dtype=np.int32)

    def draw(self) -> dict:
        """All inputs of this workload as bf16 bit arrays."""
        out = {
            "x": (activations_offset if self.kind == "layernorm" else activations)(self.M, self.d, self.seed),
            "g": gain(self.d, self.seed),
            "w": weight(self.d, self.w_cols, self.seed),
        }
        if self.kind == "layernorm":
            out["beta"] = bias(self.d, self.seed)
        if self.kind in ("postnorm", "postnorm_rope"):
            out["g2"] = gain(self.head_dim, self.seed, tag="g2")
        return out


# The five problem families, at their full sizes. The small SmolLM2 case is the
# one the oracle finishes in seconds; the others are timed on the GPU.
WORKLOADS = {
    "smollm2_qkv_m64": Workload("smollm2_qkv_m64", "linear", 64, 576, 960, 1e-5, seed=BASE_SEED + 0),
    "smollm2_qkv_m8192": Workload("smollm2_qkv_m8192", "linear", 8192, 576, 960, 1e-5, seed=BASE_SEED + 1),
    "smollm2_ffn_m8192": Workload("smollm2_ffn_m8192", "glu", 8192, 576, 1536, 1e-5, seed=BASE_SEED + 11),
    "llama7b_qkv_m1": Workload("llama7b_qkv_m1", "linear", 1, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_qkv_m4": Workload("llama7b_qkv_m4", "linear", 4, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_qkv_m16": Workload("llama7b_qkv_m16", "linear", 16, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_qkv_m2048": Workload("llama7b_qkv_m2048", "linear", 2048, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_ffn_m2048": Workload("llama7b_ffn_m2048", "glu", 2048, 4096, 11008, 1e-6, seed=BASE_SEED + 3),
    "mla_latent_m2048": Workload("mla_latent_m2048", "postnorm", 2048, 5120, 512, 1e-6,
                                 head_dim=512, eps2=1e-6, seed=BASE_SEED + 4),
    # Per-head QKV normalisation at Gemma-like widths (model dimension 2560, 16 heads of 256 or 32 of
    # 128 over the concatenated q/k/v projections): the pre-attention RMSNorm is elided.
    "gemma_qkvnorm_hd256_m2048": Workload("gemma_qkvnorm_hd256_m2048", "postnorm", 2048, 2560, 4096, 1e-6,
                                          head_dim=256, eps2=1e-6, seed=BASE_SEED + 5),
    "gemma_qkvnorm_hd128_m2048": Workload("gemma_qkvnorm_hd128_m2048", "postnorm", 2048, 2560, 4096, 1e-6,
                                          head_dim=128, eps2=1e-6, seed=BASE_SEED + 6),
    # Llama-7B QKV decode with the folded weight quantized to FP8 E4M3 per output channel
    "llama7b_qkv_fp8_m1": Workload("llama7b_qkv_fp8_m1", "linear_fp8", 1, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_qkv_fp8_m4": Workload("llama7b_qkv_fp8_m4", "linear_fp8", 4, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_qkv_fp8_m16": Workload("llama7b_qkv_fp8_m16", "linear_fp8", 16, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    # the same with NVFP4 (E2M1 codes, E4M3 scales per 16 k, a fp32 scale per output channel)
    "llama7b_qkv_nvfp4_m1": Workload("llama7b_qkv_nvfp4_m1", "linear_nvfp4", 1, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_qkv_nvfp4_m4": Workload("llama7b_qkv_nvfp4_m4", "linear_nvfp4", 4, 4096, 12288, 1e-6, seed=BASE_SEED + 2),
    "llama7b_qkv_nvfp4_m16": Workload("llama7b_qkv_nvfp4_m16", "linear_nvfp4", 16, 4096, 12288, 1e-6,
                                      seed=BASE_SEED + 2),
    # LayerNorm (gain and bias) before the SmolLM2-sized QKV projection, 8192 tokens
    "layernorm_qkv_m8192": Workload("layernorm_qkv_m8192", "layernorm", 8192, 576, 960, 1e-5, seed=BASE_SEED + 7),
    # LayerNorm before the Llama-7B-sized QKV projection at decode, 4 tokens
    "layernorm_llama7b_qkv_m4": Workload("layernorm_llama7b_qkv_m4", "layernorm", 4, 4096, 12288, 1e-5,
                                         seed=BASE_SEED + 8),
    # The same with RoPE fused after the per-head norm on the query and key heads (8 q + 4 k heads of 256,
    # then 4 value heads), positions 0 .. 2047 of a prefill.
    "gemma_qkvnorm_rope_hd256_m2048": Workload("gemma_qkvnorm_rope_hd256_m2048", "postnorm_rope", 2048, 2560, 4096,
                                               1e-6, head_dim=256, eps2=1e-6, seed=BASE_SEED + 5, n_rope_heads=12),
}


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
