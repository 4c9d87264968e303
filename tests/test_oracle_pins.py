"""Pins for the fp64 oracle: it is checked against things other than itself.

* hand-worked golden cases (tests/golden/hand_worked.json), derived from the
  definitions in the FlashNorm abstract by hand;
* torch's own CPU RMSNorm, SiLU and float32 -> bf16 conversion on the special
  cases those library routines cover;
* closed forms (constant rows, d = 1, identity weights, GLU with proportional
  gate and up columns);
* invariants the abstract states: folded == unfolded ("exact reformulation"),
  scale invariance of RMS, and the redundant-norm identity;
* brute force in exact rational arithmetic (50-digit square roots) on tiny inputs;
* for the extensions: hand-worked RoPE and LayerNorm cases (tests/golden/), torch's CPU
  layer_norm and float8_e4m3fn conversion, RoFormer's complex-exponential form of the
  rotation, and the FP8 output within the bound its half-step quantization gives;
* the parity metric itself (rel_err, the comparator every GPU parity test uses) on
  hand-worked cases where a sign, an absolute value or the denominator matters.

The last test plants plausible mistakes in the oracle (on the CPU) and checks
that every one of them is caught by at least one pin.
"""

import json
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import flashnorm_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
GOLDEN_ROPE = os.path.join(os.path.dirname(__file__), "golden", "rope_hand_worked.json")
GOLDEN_LN = os.path.join(os.path.dirname(__file__), "golden", "layernorm_hand_worked.json")


def _arr(v):
    return np.asarray(v, dtype=np.float64)


# ---------------------------------------------------------------------------
# Pin checks. Each returns a list of failure strings (empty = pass), so the
# mutation test can run them against a deliberately broken oracle.
# ---------------------------------------------------------------------------

def check_golden(O):
    fails = []
    with open(GOLDEN) as f:
        data = json.load(f)
    for c in data["cases"]:
        op = c["op"]
        if op == "norm_then_project":
            y = O.norm_then_project(_arr(c["x"]), _arr(c["g"]), _arr(c["W"]), c["eps"])
        elif op == "deferred_of_fold":
            y = O.deferred(_arr(c["x"]), O.fold(_arr(c["W"]), _arr(c["g"])), c["eps"])
        elif op == "unfused_norm_then_project":
            y = O.unfused_norm_then_project(_arr(c["x"]), _arr(c["g"]), _arr(c["W"]), c["eps"])
        elif op == "glu_norm_then_project":
            y = O.glu_norm_then_project(_arr(c["x"]), _arr(c["g"]), _arr(c["W"]), c["eps"])
        elif op == "postnorm_full":
            y = O.postnorm_full(_arr(c["x"]), _arr(c["g"]), _arr(c["W"]), _arr(c["g2"]), c["eps"],
                                c["eps2"], c["head_dim"])
        elif op == "postnorm_elided_exact_eps":
            y = O.postnorm_elided_exact_eps(_arr(c["x"]), _arr(c["Wstar"]), _arr(c["g2"]), c["eps"],
                                            c["eps2"], c["head_dim"])
        elif op == "postnorm_elided":
            y = O.postnorm_elided(_arr(c["x"]), _arr(c["Wstar"]), _arr(c["g2"]), c["eps2"], c["head_dim"])
        else:
            raise AssertionError(op)
        exp = _arr(c["expected"])
        if y.shape != exp.shape or not np.allclose(y, exp, rtol=1e-14, atol=1e-14):
            fails.append(f"golden {c['name']}: got {y.tolist()} expected {exp.tolist()}")
    for c in data["fold_bits"]["cases"]:
        g = np.array([int(c["g"], 16)], dtype=np.uint16)
        w = np.array([[int(c["w"], 16)]], dtype=np.uint16)
        got = int(O.fold_bf16(w, g)[0, 0])
        if got != int(c["wstar"], 16):
            fails.append(f"fold bits g={c['g']} w={c['w']}: got {got:#06x} expected {c['wstar']}")
    return fails


def check_torch_rmsnorm(O):
    rng = np.random.default_rng(1)
    fails = []
    for d, eps in ((1, 1e-5), (7, 0.0), (64, 1e-6), (576, 1e-5)):
        x = rng.standard_normal((5, d)) * np.exp(rng.uniform(-3, 3, (5, 1)))
        g = rng.uniform(0.5, 1.5, d)
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (d,), torch.from_numpy(g), eps).numpy()
        if not np.allclose(O.rmsnorm(x, g, eps), ref, rtol=1e-13, atol=0):
            fails.append(f"rmsnorm vs torch d={d}")
    return fails


def check_torch_silu(O):
    t = np.linspace(-40, 40, 1001)
    ref = torch.nn.functional.silu(torch.from_numpy(t)).numpy()
    return [] if np.allclose(O.silu(t), ref, rtol=1e-14, atol=1e-300) else ["silu vs torch"]


def check_torch_bf16(O):
    """fp32-representable values: RNE to bf16 must equal torch's fp32 -> bf16 cast."""
    rng = np.random.default_rng(2)
    bits32 = rng.integers(0, 2**32, size=200000, dtype=np.uint64).astype(np.uint32)
    # add exact ties and near-ties around a few exponents
    base = rng.integers(0, 2**16, size=4000, dtype=np.uint64).astype(np.uint32) << np.uint32(16)
    ties = np.concatenate([base | np.uint32(0x8000), base | np.uint32(0x7FFF), base | np.uint32(0x8001)])
    bits32 = np.concatenate([bits32, ties])
    f = bits32.view(np.float32)
    f = f[np.isfinite(f) & (np.abs(f) < 3.0e38)]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f64_to_bf16(f.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    return [] if bad.size == 0 else [f"bf16 RNE vs torch: {bad.size} mismatches, e.g. {f[bad[0]]!r}"]


def check_closed_forms(O):
    fails = []
    rng = np.random.default_rng(3)
    # constant row x = c * 1: y_j = c / sqrt(c^2 + eps) * sum_i g_i W_ij
    d, N, c, eps = 16, 5, -0.7, 1e-3
    g = rng.uniform(0.5, 1.5, d)
    W = rng.standard_normal((d, N))
    y = O.norm_then_project(np.full((1, d), c), g, W, eps)
    exp = c / np.sqrt(c * c + eps) * (g @ W)
    if not np.allclose(y[0], exp, rtol=1e-13):
        fails.append("constant row closed form")
    # d = 1: y = x / sqrt(x^2 + eps) * g * W
    x = np.array([[2.5], [-0.25]])
    y = O.norm_then_project(x, np.array([1.25]), np.array([[3.0, -2.0]]), 0.5)
    exp = x / np.sqrt(x * x + 0.5) * 1.25 * np.array([[3.0, -2.0]])
    if not np.allclose(y, exp, rtol=1e-14):
        fails.append("d=1 closed form")
    # W = I, g = 1, eps = 0: mean(y^2) = 1 for every row
    x = rng.standard_normal((4, 32)) * 7.0
    y = O.norm_then_project(x, np.ones(32), np.eye(32), 0.0)
    if not np.allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-14):
        fails.append("identity weights: mean(y^2) != 1")
    # GLU with up = 2 * gate: y = silu(z) * 2z, z = the linear output on the gate columns
    Wg = rng.standard_normal((32, 6))
    x = rng.standard_normal((3, 32))
    gg = rng.uniform(0.5, 1.5, 32)
    z = O.norm_then_project(x, gg, Wg, 1e-5)
    y = O.glu_norm_then_project(x, gg, np.concatenate([Wg, 2 * Wg], axis=1), 1e-5)
    if not np.allclose(y, 2 * z * (z / (1 + np.exp(-z))), rtol=1e-13):
        fails.append("GLU up = 2*gate closed form (gate/up order)")
    return fails


def check_invariants(O):
    fails = []
    rng = np.random.default_rng(4)
    M, d, N = 6, 40, 12
    x = rng.standard_normal((M, d)) * np.exp(rng.uniform(-2, 2, (M, 1)))
    g = rng.uniform(0.5, 1.5, d)
    W = rng.standard_normal((d, N)) / np.sqrt(d)
    eps = 1e-5
    # (i)+(ii): folded, deferred form equals the unfolded chain
    if not np.allclose(O.deferred(x, O.fold(W, g), eps), O.norm_then_project(x, g, W, eps), rtol=1e-12, atol=0):
        fails.append("folded deferred != unfolded")
    Wgu = rng.standard_normal((d, 2 * N)) / np.sqrt(d)
    if not np.allclose(O.glu_deferred(x, O.fold(Wgu, g), eps), O.glu_norm_then_project(x, g, Wgu, eps),
                       rtol=1e-12, atol=1e-300):
        fails.append("GLU folded deferred != unfolded")
    # scale invariance at eps = 0; closed form a x / sqrt(a^2 ms + eps) with eps > 0
    for a in (1e-3, 0.37, 1e3):
        if not np.allclose(O.norm_then_project(a * x, g, W, 0.0), O.norm_then_project(x, g, W, 0.0),
                           rtol=1e-12, atol=0):
            fails.append(f"scale invariance a={a}")
        ms = np.mean(x * x, axis=1, keepdims=True)
        if not np.allclose(O.rmsnorm(a * x, g, eps), a * x / np.sqrt(a * a * ms + eps) * g, rtol=1e-12):
            fails.append(f"eps>0 scaling closed form a={a}")
    # redundant norm: full chain == elided at eps = 0; == eps-corrected form at eps > 0
    hd = 4
    g2 = rng.uniform(0.5, 1.5, hd)
    full0 = O.postnorm_full(x, g, W, g2, 0.0, 0.0, hd)
    if not np.allclose(full0, O.postnorm_elided(x, O.fold(W, g), g2, 0.0, hd), rtol=1e-12, atol=0):
        fails.append("postnorm identity at eps=0")
    full1 = O.postnorm_full(x, g, W, g2, 1e-2, 3e-2, hd)
    if not np.allclose(full1, O.postnorm_elided_exact_eps(x, O.fold(W, g), g2, 1e-2, 3e-2, hd),
                       rtol=1e-12, atol=0):
        fails.append("postnorm identity with eps correction")
    return fails


def _dsqrt(fr: Fraction) -> Decimal:
    return (Decimal(fr.numerator) / Decimal(fr.denominator)).sqrt()


def _brute_linear(x, g, W, eps):
    """RMSNorm -> linear in exact rationals, square root to 50 digits, pure Python loops."""
    out = []
    for row in x:
        d = len(row)
        ms = sum(Fraction(v) * Fraction(v) for v in row) / d + Fraction(eps)
        inv = Decimal(1) / _dsqrt(ms)
        n = [Decimal(Fraction(row[i]).numerator) / Decimal(Fraction(row[i]).denominator) * inv
             * (Decimal(Fraction(g[i]).numerator) / Decimal(Fraction(g[i]).denominator)) for i in range(d)]
        outrow = []
        for j in range(len(W[0])):
            acc = Decimal(0)
            for i in range(d):
                w = Fraction(W[i][j])
                acc += n[i] * (Decimal(w.numerator) / Decimal(w.denominator))
            outrow.append(float(acc))
        out.append(outrow)
    return np.array(out)


def check_brute_force(O):
    getcontext().prec = 50
    rng = np.random.default_rng(5)
    fails = []
    for trial in range(12):
        M, d, N = rng.integers(1, 4), rng.integers(1, 9), rng.integers(1, 5)
        # dyadic values (exact in binary) so Fraction sees the very numbers numpy sees
        x = rng.integers(-64, 65, (M, d)) / 16.0
        x[0, 0] = 1.5  # no all-zero row
        g = rng.integers(8, 25, d) / 16.0
        W = rng.integers(-32, 33, (d, N)) / 32.0
        eps = float(rng.choice([0.0, 1.0 / 1024, 0.5]))
        if eps == 0.0 and np.any(np.all(x == 0, axis=1)):
            continue
        exp = _brute_linear(x.tolist(), g.tolist(), W.tolist(), eps)
        y = O.norm_then_project(x, g, W, eps)
        scale = max(1.0, float(np.max(np.abs(exp))))
        if np.max(np.abs(y - exp)) > 1e-14 * scale:
            fails.append(f"brute force trial {trial}")
    return fails


def check_rope(O):
    """RoPE on the normalised heads: hand-worked cases, the table against scalar math.cos / math.sin,
    and the properties a rotation by position * frequency must have."""
    import math

    fails = []
    with open(GOLDEN_ROPE) as f:
        data = json.load(f)
    for k, c in enumerate(data["cases"]):
        pos = np.asarray(c["positions"])
        table = O.rope_table(int(pos.max()) + 1, c["head_dim"], c["base"])
        y = O.apply_rope(_arr(c["v"]), table, pos, c["head_dim"], c["n_rope_heads"])
        if np.max(np.abs(y - _arr(c["y"]))) > 1e-14:
            fails.append(f"rope golden case {k}")
    # the table, entry by entry, against the scalar definition
    hd, base = 16, 500.0
    t = O.rope_table(40, hd, base)
    for p in (0, 1, 7, 39):
        for i in range(hd // 2):
            a = p * base ** (-2.0 * i / hd)
            if abs(t[p, i, 0] - math.cos(a)) > 1e-15 or abs(t[p, i, 1] - math.sin(a)) > 1e-15:
                fails.append(f"rope table p={p} i={i}")
    rng = np.random.default_rng(12)
    hd, H = 8, 3
    table = O.rope_table(64, hd, 10000.0)
    v = rng.standard_normal((5, hd * H))
    # position 0 is the identity; heads past n_rope_heads are untouched
    if np.max(np.abs(O.apply_rope(v, table, np.zeros(5, dtype=int), hd, H) - v)) > 0:
        fails.append("rope position 0 not identity")
    pos = rng.integers(0, 64, 5)
    y = O.apply_rope(v, table, pos, hd, 2)
    if np.max(np.abs(y[:, 2 * hd:] - v[:, 2 * hd:])) > 0:
        fails.append("rope touched a value head")
    # every pair keeps its length (a rotation)
    pl = lambda a: np.hypot(a[:, 0::2], a[:, 1::2])
    if np.max(np.abs(pl(y[:, :2 * hd]) - pl(v[:, :2 * hd]))) > 1e-12:
        fails.append("rope changed a pair's length")
    # relative position: <R_p q, R_p' k> depends only on p' - p
    q, k = rng.standard_normal((1, hd)), rng.standard_normal((1, hd))
    def dot(p, pp):
        return float(np.sum(O.apply_rope(q, table, [p], hd, 1) * O.apply_rope(k, table, [pp], hd, 1)))
    for p, pp, s in ((3, 10, 5), (0, 20, 11), (30, 2, 7)):
        if abs(dot(p, pp) - dot(p + s, pp + s)) > 1e-12:
            fails.append(f"rope relative position {p},{pp},{s}")
    # RoFormer's complex form: pair (2i, 2i+1) as the number v_2i + j v_2i+1, multiplied by exp(j p theta_i)
    theta = 10000.0 ** (-2.0 * np.arange(hd // 2) / hd)
    z = v[:, :2 * hd].reshape(5, 2, hd // 2, 2)
    zc = (z[..., 0] + 1j * z[..., 1]) * np.exp(1j * pos[:, None, None] * theta[None, None, :])
    yc = np.stack([zc.real, zc.imag], axis=-1).reshape(5, 2 * hd)
    if np.max(np.abs(yc - y[:, :2 * hd])) > 1e-12:
        fails.append("rope vs the complex-exponential form")
    return fails


def check_layernorm(O):
    """LayerNorm -> linear: hand-worked cases, torch's CPU layer_norm, the closed form of a constant row,
    shift invariance, and folded + deferred == the definition."""
    fails = []
    with open(GOLDEN_LN) as f:
        data = json.load(f)
    for k, c in enumerate(data["cases"]):
        y = O.layernorm_then_project(_arr(c["x"]), _arr(c["gamma"]), _arr(c["beta"]), _arr(c["W"]), c["eps"])
        if np.max(np.abs(y - _arr(c["y"]))) > 1e-14:
            fails.append(f"layernorm golden case {k}")
    rng = np.random.default_rng(21)
    for d, eps in ((7, 1e-5), (64, 0.0), (300, 0.1)):
        x = rng.standard_normal((6, d)) * 3 + rng.uniform(-2, 2, (6, 1))
        g, b = rng.uniform(0.5, 1.5, d), rng.uniform(-0.5, 0.5, d)
        ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (d,), torch.from_numpy(g), torch.from_numpy(b),
                                             eps).numpy()
        if np.max(np.abs(O.layernorm(x, g, b, eps) - ref)) > 1e-12:
            fails.append(f"layernorm vs torch d={d}")
        if np.max(np.abs(O.layernorm(x + 5.0, g, b, eps) - O.layernorm(x, g, b, eps))) > 1e-11:
            fails.append(f"layernorm not shift invariant d={d}")
        W = rng.standard_normal((d, 5))
        Ws, cs, bb = O.layernorm_fold(W, g, b)
        if np.max(np.abs(O.layernorm_deferred(x, Ws, cs, bb, eps) - O.layernorm_then_project(x, g, b, W, eps))) > 1e-10:
            fails.append(f"layernorm folded != definition d={d}")
        const = np.full((1, d), 1.75)  # dyadic: the mean is exact and x - mu is exactly 0
        if np.max(np.abs(O.layernorm_then_project(const, g, b, W, max(eps, 1e-6)) - b @ W)) > 1e-12:
            fails.append(f"layernorm constant row d={d}")
    return fails


def check_fp8(O):
    """E4M3 weight quantization: torch's own float8_e4m3fn conversion (encode on values within +-448,
    decode of all 256 codes), hand-worked codes, and the properties of the per-channel fold."""
    fails = []
    rng = np.random.default_rng(31)
    v = np.concatenate([rng.standard_normal(4000) * 60, rng.standard_normal(4000) * 0.02,
                        np.arange(-600, 601) * 2.0 ** -11, [448.0, -448.0, 0.0, -0.0]])
    v = np.clip(v, -448, 448).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    if np.any(O.f64_to_e4m3(v.astype(np.float64)) != ref):
        fails.append("e4m3 encode vs torch")
    codes = np.arange(256, dtype=np.uint8)
    dec = O.e4m3_to_f64(codes)
    tdec = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    if not np.all((dec == tdec) | (np.isnan(dec) & np.isnan(tdec))):
        fails.append("e4m3 decode vs torch")
    # hand-worked: 1 = 2^0 -> exponent field 7, mantissa 0; 448 = 1.75 * 2^8 -> 15, 6; 2^-9 is the smallest
    # subnormal; 0.1 -> 1.625 * 2^-4 = 0.1015625 (3, 5); -0.3 -> -(1.25 * 2^-2) (sign, 5, 2)
    for val, code in ((1.0, 0x38), (448.0, 0x7E), (2.0 ** -9, 0x01), (0.1, 0x1D), (-0.3, 0xAA), (0.0, 0x00)):
        if int(O.f64_to_e4m3(np.array([val]))[0]) != code:
            fails.append(f"e4m3 code of {val}")
    # the fold: every channel's largest weight maps to +-448 and every weight is within half a step
    d, N = 96, 24
    wb = O.f64_to_bf16(rng.standard_normal((d, N)) / np.sqrt(d))
    gb = O.f64_to_bf16(rng.uniform(0.5, 1.5, d))
    Q, s = O.fold_fp8(wb, gb)
    Ws = O.fold(O.bf16_to_f64(wb), O.bf16_to_f64(gb)).T  # [N, d]
    deq = O.e4m3_to_f64(Q) / 1.0
    if np.any(np.max(np.abs(deq), axis=1) != 448.0):
        fails.append("fp8 fold: channel maximum not at 448")
    err = np.abs(deq * s[:, None] - Ws)
    step = np.maximum(np.abs(Ws) * 2.0 ** -4, 2.0 ** -10 * s[:, None])  # half a step: 2^-4 relative, 2^-10 s below 2^-6 s
    if np.any(err > step * (1 + 1e-6)):
        fails.append("fp8 fold: weight off by more than half a step")
    # the quantized deferred output against the definition (RMSNorm, then the unquantized W): within the
    # bound those half steps give, r_m * sum_k |x_mk| * step_nk, and well away from zero error
    x = O.bf16_to_f64(O.f64_to_bf16(rng.standard_normal((6, d)) * np.exp(rng.uniform(-2, 2, (6, 1)))))
    eps = 1e-6
    y8 = O.deferred_fp8(x, Q, s, eps)
    ydef = O.norm_then_project(x, O.bf16_to_f64(gb), O.bf16_to_f64(wb), eps)
    bound = O.inv_rms(x, eps)[:, None] * (np.abs(x) @ step.T)
    if np.any(np.abs(y8 - ydef) > bound * (1 + 1e-9) + 1e-15):
        fails.append("fp8 deferred output outside the quantization bound")
    if not (1e-4 < O.rel_err(y8, ydef) < 0.1):
        fails.append("fp8 deferred output: error not of the size E4M3 gives")
    return fails


E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # the format's eight magnitudes, codes 0..7


def check_nvfp4(O):
    """NVFP4 weight quantization: the E2M1 table, hand-worked roundings (ties to even, saturation), brute
    force over the grid, a hand-worked fold of one channel, the invariants of the fold on random weights,
    the packed layout byte by byte, and the deferred output against the unquantized definition."""
    fails = []
    # decode: the format's table, sign in bit 3
    want = np.array(E2M1_TABLE + [-v for v in E2M1_TABLE])
    got = O.e2m1_to_f64(np.arange(16))
    if not (np.array_equal(got, want) and np.all(np.signbit(got[8:]))):
        fails.append("e2m1 decode table")
    # encode, worked by hand: halfway cases go to the even mantissa, magnitudes above 6 saturate
    for val, code in ((0.25, 0), (0.3, 1), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (2.9, 5), (3.5, 6),
                      (5.0, 6), (5.1, 7), (7.0, 7), (1e9, 7), (-0.25, 8), (-1.75, 12), (-6.0, 15), (0.0, 0)):
        if int(O.f64_to_e2m1(np.array([val]))[0]) != code:
            fails.append(f"e2m1 code of {val}")
    # brute force: the nearest grid value, ties to the even code
    rng = np.random.default_rng(47)
    v = np.concatenate([rng.uniform(-7.5, 7.5, 3000), np.arange(-30, 31) * 0.25])
    grid = np.array(E2M1_TABLE)
    for x in v:
        a = min(abs(x), 6.0)
        dist = np.abs(grid - a)
        best = np.flatnonzero(dist == dist.min())
        mag = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        expect = mag | (8 if np.signbit(x) else 0)
        if int(O.f64_to_e2m1(np.array([x]))[0]) != expect:
            fails.append(f"e2m1 brute force at {x}")
            break
    # a fold worked by hand: one channel, g = 1, d = 32. Block 0 holds grid values times 2^-3 (channel
    # maximum 0.75), block 1 grid values times 2^-4 (block maximum 0.09375).
    #   s2 = 0.75 / 2688; block 0: 0.75 / (6 s2) = 448 -> scale 448 (E4M3 0x7E), step 448 s2 = 1/8;
    #   block 1: 0.09375 / (6 s2) = 56 -> scale 56 = 1.75 * 2^5 (E4M3 0x66), step 56 s2 = 2^-6.
    b0 = [6, 3, -1.5, 0.5, 4, -6, 0, 1, 2, -0.5, 1.5, -3, 0, 4, -2, 1]
    b1 = [1, 0.5, -1, 1.5, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, -0.5]
    col = np.array([t * 2.0 ** -3 for t in b0] + [t * 2.0 ** -4 for t in b1])
    codes, bsc, s2 = O.fold_nvfp4(O.f64_to_bf16(col[:, None]), O.f64_to_bf16(np.ones(32)))
    want0 = [7, 5, 11, 1, 6, 15, 0, 2, 4, 9, 3, 13, 0, 6, 12, 2]
    want1 = [6, 4, 14, 7, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 12]   # b1 * 2^-4 / 2^-6 = 4 * b1
    if list(codes[0]) != want0 + want1:
        fails.append("nvfp4 fold: codes of the hand-worked channel")
    if list(bsc[0]) != [0x7E, 0x66]:
        fails.append("nvfp4 fold: block scales of the hand-worked channel")
    if s2[0] != np.float32(0.75) / np.float32(2688.0):
        fails.append("nvfp4 fold: channel scale")
    if np.max(np.abs(O.dequant_nvfp4(codes, bsc, s2)[0] - col)) > 1e-7 * 0.75:
        fails.append("nvfp4 fold: grid values not reproduced")
    # invariants on random weights: each nonzero block's largest code is +-6, the block holding the channel
    # maximum has scale 448, and every weight is within half a quantum of its block's grid
    d, N = 80, 24
    wb = O.f64_to_bf16(rng.standard_normal((d, N)) / np.sqrt(d) * np.exp(rng.uniform(-3, 3, (1, N))))
    gb = O.f64_to_bf16(rng.uniform(0.5, 1.5, d))
    codes, bsc, s2 = O.fold_nvfp4(wb, gb)
    Ws = O.fold(O.bf16_to_f64(wb), O.bf16_to_f64(gb)).T           # [N, d]
    dec = O.e2m1_to_f64(codes)
    if np.any(np.max(np.abs(dec.reshape(N, d // 16, 16)), axis=2) != 6.0):
        fails.append("nvfp4 fold: a block maximum not at 6")
    if np.any(np.max(O.e4m3_to_f64(bsc), axis=1) != 448.0):
        fails.append("nvfp4 fold: channel maximum block not at scale 448")
    step = O.e4m3_to_f64(bsc)[:, np.arange(d) // 16] * s2[:, None].astype(np.float64)
    t = Ws / step
    half_q = np.where(np.abs(t) < 2, 0.25, np.where(np.abs(t) < 4, 0.5, 1.0))
    if np.any(np.abs(t - dec) > half_q * (1 + 1e-6)):
        fails.append("nvfp4 fold: weight off by more than half a quantum")
    # packed layout, by hand: codes 0..15 repeated along k, scales 0x40, 0x41 for the two blocks of d = 32.
    # Word 0 (k = 0..7) holds even codes 0, 2, 4, 6 in its low half (0x6420) and odd codes 1, 3, 5, 7 in its
    # high half (0x7531): 0x75316420, little endian; word 1 (k = 8..15): 0xFDB9ECA8.
    c = np.tile(np.arange(16, dtype=np.uint8), (2, 2))
    packed = O.pack_nvfp4(c, np.array([[0x40, 0x41], [0x40, 0x41]], dtype=np.uint8))
    w0, w1 = [0x20, 0x64, 0x31, 0x75], [0xA8, 0xEC, 0xB9, 0xFD]
    row = (w0 + w1) * 2 + [0] * 112 + [0x40, 0x41] + [0] * 14
    if packed.shape != (2, 144) or list(packed[1]) != row:
        fails.append("nvfp4 packed layout")
    # the deferred output against the definition: within the bound the half quanta give, not exact
    x = O.bf16_to_f64(O.f64_to_bf16(rng.standard_normal((5, d)) * np.exp(rng.uniform(-2, 2, (5, 1)))))
    eps = 1e-6
    y4 = O.deferred_nvfp4(x, codes, bsc, s2, eps)
    ydef = O.norm_then_project(x, O.bf16_to_f64(gb), O.bf16_to_f64(wb), eps)
    bound = O.inv_rms(x, eps)[:, None] * (np.abs(x) @ (half_q * step).T)
    if np.any(np.abs(y4 - ydef) > bound * (1 + 1e-9) + 1e-15):
        fails.append("nvfp4 deferred output outside the quantization bound")
    if not (1e-3 < O.rel_err(y4, ydef) < 0.3):
        fails.append("nvfp4 deferred output: error not of the size E2M1 gives")
    return fails


def check_rel_err(O):
    """The parity metric max|y - y_ref| / max|y_ref| on hand-worked cases, chosen so that a sign, a
    missing absolute value, the wrong denominator or swapped arguments each change the result."""
    fails = []
    cases = [
        # y, y_ref, expected (worked by hand)
        ([-5.0, 1.0], [-4.0, 1.0], 0.25),            # |dy| = (1, 0); max|y_ref| = 4 (not max y_ref = 1)
        ([[0.0, 3.0], [1.0, 1.0]], [[0.5, 2.0], [1.0, -2.0]], 1.5),  # max|dy| = 3 at a negative reference
        ([2.0, -3.0], [2.0, -3.0], 0.0),
        ([1e-3, -2e-3], [0.0, 0.0], 2e-3),          # zero reference: the absolute difference
    ]
    for y, ref, want in cases:
        got = O.rel_err(_arr(y), _arr(ref))
        if not abs(got - want) <= 1e-15:
            fails.append(f"rel_err({y}, {ref}) = {got}, expected {want}")
    return fails


ALL_CHECKS = [check_golden, check_torch_rmsnorm, check_torch_silu, check_torch_bf16,
              check_closed_forms, check_invariants, check_brute_force, check_rope, check_layernorm, check_fp8,
              check_nvfp4, check_rel_err]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    fails = check(O)
    assert not fails, fails


def test_reference_output_wrappers():
    """The bit-array wrappers route to the pinned functions with the right operands, row subsets
    included: linear, SwiGLU, post-norm, post-norm + RoPE, LayerNorm and FP8."""
    from flashnorm_inputs import Workload

    rows = [1, 3]
    # linear and SwiGLU (gate = the first F columns of W, up = the last F)
    for kind in ("linear", "glu"):
        bits = Workload("t", kind, 5, 24, 8, 1e-5, seed=3).draw()
        x, g, W = (O.bf16_to_f64(bits[k]) for k in ("x", "g", "w"))
        ws = O.fold_bf16(bits["w"], bits["g"])
        Ws = O.bf16_to_f64(ws)
        plain = O.norm_then_project if kind == "linear" else O.glu_norm_then_project
        folded = O.deferred if kind == "linear" else O.glu_deferred
        assert np.allclose(O.reference_output(kind, bits, 1e-5), plain(x, g, W, 1e-5), rtol=1e-15, atol=0)
        assert np.allclose(O.reference_output(kind, bits, 1e-5, rows=rows), plain(x[rows], g, W, 1e-5),
                           rtol=1e-15, atol=0)
        assert np.allclose(O.exact_operand_output(kind, bits, ws, 1e-5, rows=rows), folded(x[rows], Ws, 1e-5),
                           rtol=1e-15, atol=0)
        assert O.reference_output(kind, bits, 1e-5).shape == (5, 8)
    # post-norm: the full chain keeps the first norm, the exact-operand form drops it
    wl = Workload("t", "postnorm", 5, 24, 8, 1e-6, head_dim=4, eps2=1e-6, seed=7)
    bits = wl.draw()
    x, g, W, g2 = (O.bf16_to_f64(bits[k]) for k in ("x", "g", "w", "g2"))
    y = O.reference_output("postnorm", bits, 1e-6, eps2=1e-6, head_dim=4)
    assert np.allclose(y, O.postnorm_full(x, g, W, g2, 1e-6, 1e-6, 4), rtol=1e-15)
    ws = O.fold_bf16(bits["w"], bits["g"])
    y2 = O.exact_operand_output("postnorm", bits, ws, 1e-6, eps2=1e-6, head_dim=4, rows=rows)
    assert np.allclose(y2, O.postnorm_elided(x[rows], O.bf16_to_f64(ws), g2, 1e-6, 4), rtol=1e-15)
    # post-norm + RoPE: positions follow the selected rows
    pos = np.array([4, 0, 2, 9, 1])
    y = O.reference_postnorm_rope(bits, 1e-6, 1e-6, 4, pos, 1, 10000.0, rows=rows)
    assert np.allclose(y, O.postnorm_rope_full(x[rows], g, W, g2, 1e-6, 1e-6, 4, pos[rows], 1, 10000.0),
                       rtol=1e-15)
    table = O.rope_table(10, 4, 10000.0)
    y = O.exact_operand_postnorm_rope(bits, ws, 1e-6, 4, pos, 1, table, rows=rows)
    u = O.postnorm_elided(x[rows], O.bf16_to_f64(ws), g2, 1e-6, 4)
    assert np.allclose(y, O.apply_rope(u, table, pos[rows], 4, 1), rtol=1e-15)
    assert not np.allclose(y, u)  # the rotation did something
    # LayerNorm: gamma = bits["g"], beta = bits["beta"]; colsum of the bf16 W*, bias from the unfolded W
    bits = Workload("t", "layernorm", 5, 24, 8, 1e-5, seed=4).draw()
    x, g, W, beta = (O.bf16_to_f64(bits[k]) for k in ("x", "g", "w", "beta"))
    assert np.allclose(O.reference_layernorm(bits, 1e-5, rows=rows),
                       O.layernorm_then_project(x[rows], g, beta, W, 1e-5), rtol=1e-15)
    ws = O.fold_bf16(bits["w"], bits["g"])
    Ws = O.bf16_to_f64(ws)
    assert np.allclose(O.exact_operand_layernorm(bits, ws, 1e-5, rows=rows),
                       O.layernorm_deferred(x[rows], Ws, Ws.sum(axis=0), beta @ W, 1e-5), rtol=1e-13)
    # FP8: the oracle's own fold, then the deferred form on the decoded codes
    bits = Workload("t", "linear_fp8", 3, 32, 8, 1e-6, seed=5).draw()
    x = O.bf16_to_f64(bits["x"])
    codes, scales = O.fold_fp8(bits["w"], bits["g"])
    assert np.allclose(O.exact_operand_fp8(bits, 1e-6, rows=[0, 2]), O.deferred_fp8(x[[0, 2]], codes, scales, 1e-6),
                       rtol=1e-15)
    # NVFP4: likewise, with the block scales and the channel scale
    codes, bsc, s2 = O.fold_nvfp4(bits["w"], bits["g"])
    assert np.allclose(O.exact_operand_nvfp4(bits, 1e-6, rows=[0, 2]),
                       O.deferred_nvfp4(x[[0, 2]], codes, bsc, s2, 1e-6), rtol=1e-15)


# ---------------------------------------------------------------------------
# Planted mistakes: each must be caught by at least one pin.
# ---------------------------------------------------------------------------

def _mut_mean_d_minus_1(x, eps):
    x = np.asarray(x, dtype=np.float64)
    n = max(x.shape[-1] - 1, 1)
    return 1.0 / np.sqrt(np.sum(x * x, axis=-1) / n + eps)


def _mut_eps_outside(x, eps):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (np.sqrt(np.mean(x * x, axis=-1)) + eps)


def _mut_rms_not_inverted(x, eps):
    x = np.asarray(x, dtype=np.float64)
    return np.sqrt(np.mean(x * x, axis=-1) + eps)


def _mut_drop_gain(x, g, eps):
    x = np.asarray(x, dtype=np.float64)
    return x * O.inv_rms(x, eps)[..., None]


def _mut_fold_columns(W, g):
    W = np.asarray(W, dtype=np.float64)
    return W * np.resize(np.asarray(g, dtype=np.float64), W.shape[1])[None, :]


def _mut_silu_sign(t):
    t = np.asarray(t, dtype=np.float64)
    return t / (1.0 + np.exp(t))


def _mut_glu_swap(x, g, W_gu, eps):
    z = O.norm_then_project(x, g, W_gu, eps)
    F = z.shape[1] // 2
    return O.silu(z[:, F:]) * z[:, :F]


def _mut_glu_scale_after(x, Wstar_gu, eps):
    x = np.asarray(x, dtype=np.float64)
    r = O.inv_rms(x, eps)[:, None]
    z = x @ Wstar_gu
    F = z.shape[1] // 2
    return r * r * O.silu(z[:, :F]) * z[:, F:]


def _mut_rne_truncate(v):
    v = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (v.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _mut_rne_ties_away(v):
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    q = np.ldexp(1.0, np.maximum(e - 8, -133))
    r = np.sign(v) * np.floor(np.abs(v) / q + 0.5) * q
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _mut_transpose_product(x, g, W, eps):
    n = O.rmsnorm(x, g, eps)
    W = np.asarray(W, dtype=np.float64)
    return n @ W if W.shape[0] != W.shape[1] else n @ W.T


def _mut_postnorm_whole_row(v, g2, eps2, head_dim):
    M, N = v.shape
    return O.rmsnorm(v, np.tile(g2, N // head_dim), eps2)


def _mut_rope_half_pairs(v, cs, positions, head_dim, n_rope_heads):
    v = np.array(v, dtype=np.float64, copy=True)
    M, N = v.shape
    cs = np.asarray(cs, dtype=np.float64)[np.asarray(positions, dtype=np.int64)]
    c, s = cs[..., 0], cs[..., 1]
    vh = v.reshape(M, N // head_dim, head_dim)
    h2 = head_dim // 2
    for h in range(min(n_rope_heads, N // head_dim)):
        a, b = vh[:, h, :h2].copy(), vh[:, h, h2:].copy()
        vh[:, h, :h2] = a * c - b * s
        vh[:, h, h2:] = a * s + b * c
    return vh.reshape(M, N)


def _mut_rope_sin_sign(v, cs, positions, head_dim, n_rope_heads):
    cs = np.array(cs, dtype=np.float64, copy=True)
    cs[..., 1] = -cs[..., 1]
    return _ORIG_APPLY_ROPE(v, cs, positions, head_dim, n_rope_heads)


def _mut_rope_freq(max_pos, head_dim, base):
    i = np.arange(head_dim // 2, dtype=np.float64)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * np.power(float(base), -i / head_dim)[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1)


def _mut_rope_all_heads(v, cs, positions, head_dim, n_rope_heads):
    return _ORIG_APPLY_ROPE(v, cs, positions, head_dim, np.asarray(v).shape[1] // head_dim)


_ORIG_APPLY_ROPE = O.apply_rope


def _mut_fp8_truncate(v):
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 448.0)
    _, e = np.frexp(a)
    q = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    return _ORIG_F64_TO_E4M3(np.sign(v) * np.floor(a / q) * q)


def _mut_fp8_bias8(codes):
    c = np.asarray(codes, dtype=np.int64)
    return _ORIG_E4M3_TO_F64(codes) * np.where(((c >> 3) & 0xF) == 0, 1.0, 0.5)


def _mut_fp8_scale_rows(w_bits, g_bits):
    W = O.bf16_to_f64(w_bits).astype(np.float32)
    g = O.bf16_to_f64(g_bits).astype(np.float32)
    Ws = (g[:, None] * W).T.astype(np.float32)
    amax = np.max(np.abs(Ws), axis=0)  # per input feature instead of per output channel
    s = np.float32(np.max(amax) / 448.0)
    scales = np.full(Ws.shape[0], s, dtype=np.float32)
    return _ORIG_F64_TO_E4M3((Ws / scales[:, None]).astype(np.float64)), scales


_ORIG_F64_TO_E4M3 = O.f64_to_e4m3
_ORIG_E4M3_TO_F64 = O.e4m3_to_f64


def _mut_ln_unbiased(x, gamma, beta, eps):
    x = np.asarray(x, dtype=np.float64)
    mu = np.mean(x, axis=-1, keepdims=True)
    var = np.sum((x - mu) ** 2, axis=-1, keepdims=True) / max(x.shape[-1] - 1, 1)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def _mut_ln_no_centering(x, gamma, beta, eps):
    x = np.asarray(x, dtype=np.float64)
    mu = np.mean(x, axis=-1, keepdims=True)
    var = np.mean((x - mu) ** 2, axis=-1, keepdims=True)
    return x / np.sqrt(var + eps) * gamma + beta


def _mut_ln_beta_inside(x, gamma, beta, eps):
    x = np.asarray(x, dtype=np.float64)
    mu = np.mean(x, axis=-1, keepdims=True)
    var = np.mean((x - mu) ** 2, axis=-1, keepdims=True)
    return ((x - mu) / np.sqrt(var + eps) + beta) * gamma


def _mut_ln_fold_colsum_unfolded(W, gamma, beta):
    Ws = O.fold(W, gamma)
    return Ws, np.sum(np.asarray(W, dtype=np.float64), axis=0), np.asarray(beta) @ np.asarray(W, dtype=np.float64)

def _mut_fp8_deferred_no_scale(x, codes, scales, eps):
    x = np.asarray(x, dtype=np.float64)
    return (x @ O.e4m3_to_f64(codes).T) * O.inv_rms(x, eps)[:, None]


def _mut_fp8_deferred_scale_by_row(x, codes, scales, eps):
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(scales, dtype=np.float64)
    return (x @ O.e4m3_to_f64(codes).T) * O.inv_rms(x, eps)[:, None] * s[: x.shape[0], None]


def _mut_e2m1_ties_away(v):
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 6.0)
    _, e = np.frexp(a)
    q = np.ldexp(1.0, np.maximum(e - 1, 0) - 1)
    return _ORIG_F64_TO_E2M1(np.where(np.signbit(v), -1.0, 1.0) * np.floor(a / q + 0.5) * q)


def _mut_e2m1_bias0(codes):
    return _ORIG_E2M1_TO_F64(codes) * np.where((np.asarray(codes, dtype=np.int64) >> 1) & 3, 2.0, 1.0)


def _mut_nvfp4_block32(w_bits, g_bits):
    saved = O.NVFP4_BLOCK
    O.NVFP4_BLOCK = 32
    try:
        codes, bsc, s2 = _ORIG_FOLD_NVFP4(w_bits, g_bits)
    finally:
        O.NVFP4_BLOCK = saved
    return codes, np.repeat(bsc, 2, axis=1)[:, : -(-codes.shape[1] // 16)], s2


def _mut_nvfp4_scale_without_6(w_bits, g_bits):
    saved = O.E2M1_MAX
    O.E2M1_MAX = 1.0  # the block maximum mapped to 1 instead of 6 (codes then saturate)
    try:
        return _ORIG_FOLD_NVFP4(w_bits, g_bits)
    finally:
        O.E2M1_MAX = saved


def _mut_nvfp4_no_s2(codes, bscales, s2):
    d = np.asarray(codes).shape[1]
    return O.e2m1_to_f64(codes) * O.e4m3_to_f64(bscales)[:, np.arange(d) // 16]


def _mut_nvfp4_pack_nibbles_swapped(codes, bscales):
    c = np.asarray(codes, dtype=np.uint8)
    swapped = c.copy()
    swapped[:, 0::2], swapped[:, 1::2] = c[:, 1::2], c[:, 0::2]
    return _ORIG_PACK_NVFP4(swapped, bscales)


_ORIG_F64_TO_E2M1 = O.f64_to_e2m1
_ORIG_E2M1_TO_F64 = O.e2m1_to_f64
_ORIG_FOLD_NVFP4 = O.fold_nvfp4
_ORIG_PACK_NVFP4 = O.pack_nvfp4


def _mut_rel_err_signed(y, y_ref):
    y, y_ref = np.asarray(y, dtype=np.float64), np.asarray(y_ref, dtype=np.float64)
    return float(np.max(y - y_ref) / np.max(np.abs(y_ref)))


def _mut_rel_err_denominator_of_y(y, y_ref):
    y, y_ref = np.asarray(y, dtype=np.float64), np.asarray(y_ref, dtype=np.float64)
    return float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y)))


def _mut_rel_err_max_not_abs(y, y_ref):
    y, y_ref = np.asarray(y, dtype=np.float64), np.asarray(y_ref, dtype=np.float64)
    d = np.max(y_ref)
    return float(np.max(np.abs(y - y_ref)) / d) if d > 0 else float(np.max(np.abs(y - y_ref)))


MUTANTS = {
    "mean over d-1": ("inv_rms", _mut_mean_d_minus_1),
    "eps outside sqrt": ("inv_rms", _mut_eps_outside),
    "rms not inverted": ("inv_rms", _mut_rms_not_inverted),
    "gain dropped": ("rmsnorm", _mut_drop_gain),
    "fold scales columns": ("fold", _mut_fold_columns),
    "silu sign": ("silu", _mut_silu_sign),
    "gate/up swapped": ("glu_norm_then_project", _mut_glu_swap),
    "deferred GLU scale after silu": ("glu_deferred", _mut_glu_scale_after),
    "bf16 truncation": ("f64_to_bf16", _mut_rne_truncate),
    "bf16 ties away": ("f64_to_bf16", _mut_rne_ties_away),
    "W transposed": ("norm_then_project", _mut_transpose_product),
    "post-norm over whole row": ("_per_head_rmsnorm", _mut_postnorm_whole_row),
    "rope pairs (i, i + hd/2)": ("apply_rope", _mut_rope_half_pairs),
    "rope rotates the wrong way": ("apply_rope", _mut_rope_sin_sign),
    "rope frequency base^(-i/hd)": ("rope_table", _mut_rope_freq),
    "rope on the value heads too": ("apply_rope", _mut_rope_all_heads),
    "layernorm unbiased variance": ("layernorm", _mut_ln_unbiased),
    "layernorm without centering": ("layernorm", _mut_ln_no_centering),
    "layernorm bias before gain": ("layernorm", _mut_ln_beta_inside),
    "layernorm colsum of unfolded W": ("layernorm_fold", _mut_ln_fold_colsum_unfolded),
    "fp8 truncation": ("f64_to_e4m3", _mut_fp8_truncate),
    "fp8 exponent bias 8": ("e4m3_to_f64", _mut_fp8_bias8),
    "fp8 one scale for the whole matrix": ("fold_fp8", _mut_fp8_scale_rows),
    "fp8 channel scale dropped": ("deferred_fp8", _mut_fp8_deferred_no_scale),
    "fp8 scale indexed by token": ("deferred_fp8", _mut_fp8_deferred_scale_by_row),
    "e2m1 ties away from zero": ("f64_to_e2m1", _mut_e2m1_ties_away),
    "e2m1 exponent bias 0": ("e2m1_to_f64", _mut_e2m1_bias0),
    "nvfp4 blocks of 32": ("fold_nvfp4", _mut_nvfp4_block32),
    "nvfp4 block maximum mapped to 1": ("fold_nvfp4", _mut_nvfp4_scale_without_6),
    "nvfp4 channel scale dropped": ("dequant_nvfp4", _mut_nvfp4_no_s2),
    "nvfp4 nibbles swapped": ("pack_nvfp4", _mut_nvfp4_pack_nibbles_swapped),
    "rel_err without the absolute value": ("rel_err", _mut_rel_err_signed),
    "rel_err relative to the result": ("rel_err", _mut_rel_err_denominator_of_y),
    "rel_err relative to max(y_ref)": ("rel_err", _mut_rel_err_max_not_abs),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in ALL_CHECKS:
        try:
            if check(O):
                caught.append(check.__name__)
        except Exception as e:  # a crash also counts as caught
            caught.append(f"{check.__name__} raised {type(e).__name__}")
    assert caught, f"planted mistake '{name}' passed every pin"
