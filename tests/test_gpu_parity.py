"""GPU parity: every kernel of the library against the fp64 oracle on the same seeded inputs.

Bars (stated for the FlashNorm path): bf16 outputs within max|y - y_ref| / max|y_ref| <= 5e-3 of the
oracle's unfolded, undeferred chain; fp32 outputs within 1e-5 of the oracle's reformulated form on the
exact bf16 operands (the folded W* the library produced, checked bitwise first). The fold is
bit-exact. All calls go through the C ABI (the thin binding only passes pointers).
"""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import oracle_layout, to_dev, to_host_bits, to_host_f64

pytestmark = pytest.mark.gpu

BF16_TOL = 5e-3
F32_TOL = 1e-5


def _wl(kind, M, d, N, eps=1e-5, seed=11, head_dim=0, eps2=0.0):
    return I.Workload("t", kind, M, d, N, eps, head_dim=head_dim, eps2=eps2, seed=seed)


def _fold(bits, glu):
    W, g = to_dev(bits["w"]), to_dev(bits["g"])
    ws = fn.flashnorm_fold_weights(W, g, glu=glu)
    return ws


@pytest.fixture(autouse=True)
def _clean_status():
    yield
    fn.flashnorm_check_device_error()


# ------------------------------------------------------------------------------------------ fold
@pytest.mark.parametrize("d,N,glu", [(576, 960, False), (576, 3072, True), (4096, 1024, False), (200, 136, False),
                                     (72, 96, True), (8, 8, False)])
def test_fold_bitwise(d, N, glu):
    bits = _wl("glu" if glu else "linear", 1, d, N // 2 if glu else N).draw()
    ws = _fold(bits, glu)
    torch.cuda.synchronize()
    expect = oracle_layout(O.fold_bf16(bits["w"], bits["g"]), glu)
    got = to_host_bits(ws)
    assert got.shape == expect.shape
    assert np.array_equal(got, expect)


def test_fold_unit_gain_is_transpose():
    bits = _wl("linear", 1, 576, 960).draw()
    ones = np.full(576, 0x3F80, dtype=np.uint16)
    ws = fn.flashnorm_fold_weights(to_dev(bits["w"]), to_dev(ones))
    assert np.array_equal(to_host_bits(ws), bits["w"].T)


# ------------------------------------------------------------------------------------------ linear
LINEAR_CASES = [
    # M, d, N, path
    (64, 576, 960, "auto"),      # SmolLM2 QKV, 64 tokens
    (333, 576, 960, "auto"),     # ragged M over three row tiles
    (200, 4096, 512, "tensor"),  # long K (64 k-blocks)
    (130, 72, 200, "tensor"),    # ragged K (one full and one partial k-block), N not a tile multiple
    (17, 576, 960, "tensor"),    # just above the decode threshold
    (16, 576, 960, "tensor"),    # decode-sized M on the tensor path
    (1, 4096, 1024, "gemv"),
    (3, 4096, 1024, "gemv"),
    (4, 4096, 1024, "gemv"),
    (16, 4096, 1024, "gemv"),
    (7, 264, 136, "gemv"),       # odd sizes on the GEMV path
]


@pytest.mark.parametrize("M,d,N,path", LINEAR_CASES)
def test_linear_parity(M, d, N, path):
    bits = _wl("linear", M, d, N, seed=M * 7 + d).draw()
    x = to_dev(bits["x"])
    ws = _fold(bits, False)
    y16 = fn.flashnorm_linear(x, ws, 1e-5, path=path)
    y32 = fn.flashnorm_linear(x, ws, 1e-5, out_dtype=torch.float32, path=path)
    torch.cuda.synchronize()
    ref = O.reference_output("linear", bits, 1e-5)
    assert O.rel_err(to_host_f64(y16), ref) <= BF16_TOL
    wsn = to_host_bits(ws).T  # back to the oracle's [d, N] orientation
    ref_exact = O.exact_operand_output("linear", bits, wsn, 1e-5)
    assert O.rel_err(to_host_f64(y32), ref_exact) <= F32_TOL


# ------------------------------------------------------------------------------------------ GLU
GLU_CASES = [
    (64, 576, 1536, "auto"),
    (257, 576, 256, "tensor"),
    (100, 4096, 1024, "tensor"),
    (130, 72, 48, "tensor"),
    (1, 4096, 512, "gemv"),
    (16, 4096, 512, "gemv"),
    (5, 576, 1536, "auto"),
]


@pytest.mark.parametrize("M,d,F,path", GLU_CASES)
def test_glu_parity(M, d, F, path):
    bits = _wl("glu", M, d, F, seed=M * 5 + F).draw()
    x = to_dev(bits["x"])
    ws = _fold(bits, True)
    y16 = fn.flashnorm_glu(x, ws, 1e-5, path=path)
    y32 = fn.flashnorm_glu(x, ws, 1e-5, out_dtype=torch.float32, path=path)
    torch.cuda.synchronize()
    ref = O.reference_output("glu", bits, 1e-5)
    assert O.rel_err(to_host_f64(y16), ref) <= BF16_TOL
    wsn = O.fold_bf16(bits["w"], bits["g"])  # bitwise equal to the library's (tested above)
    ref_exact = O.exact_operand_output("glu", bits, wsn, 1e-5)
    assert O.rel_err(to_host_f64(y32), ref_exact) <= F32_TOL


# ------------------------------------------------------------------------------------------ post-norm
POSTNORM_CASES = [
    # M, d, N, head_dim
    (300, 512, 512, 128),
    (200, 256, 1024, 256),
    (64, 640, 384, 384),
    (150, 5120, 512, 512),
    (40, 128, 64, 16),
]


@pytest.mark.parametrize("M,d,N,hd", POSTNORM_CASES)
def test_postnorm_parity(M, d, N, hd):
    bits = _wl("postnorm", M, d, N, eps=1e-6, eps2=1e-6, head_dim=hd, seed=M + hd).draw()
    x = to_dev(bits["x"])
    ws = _fold(bits, False)
    g2 = to_dev(bits["g2"])
    y16 = fn.flashnorm_linear_postnorm(x, ws, g2, hd, 1e-6)
    y32 = fn.flashnorm_linear_postnorm(x, ws, g2, hd, 1e-6, out_dtype=torch.float32)
    torch.cuda.synchronize()
    # bf16 against the FULL chain, first RMSNorm included
    ref = O.reference_output("postnorm", bits, 1e-6, eps2=1e-6, head_dim=hd)
    assert O.rel_err(to_host_f64(y16), ref) <= BF16_TOL
    ref_exact = O.exact_operand_output("postnorm", bits, O.fold_bf16(bits["w"], bits["g"]), 1e-6, eps2=1e-6,
                                       head_dim=hd)
    assert O.rel_err(to_host_f64(y32), ref_exact) <= F32_TOL


# ------------------------------------------------------------------------------------------ unfused baseline
@pytest.mark.parametrize("kind,M,d,N", [("linear", 64, 576, 960), ("linear", 333, 576, 960),
                                         ("glu", 200, 576, 1536), ("linear", 150, 4096, 512)])
def test_unfused_parity(kind, M, d, N):
    bits = _wl(kind, M, d, N, seed=3 * M + 1).draw()
    x, g = to_dev(bits["x"]), to_dev(bits["g"])
    ones = to_dev(np.full(d, 0x3F80, dtype=np.uint16))
    wk = fn.flashnorm_fold_weights(to_dev(bits["w"]), ones, glu=(kind == "glu"))
    if kind == "glu":
        y = fn.flashnorm_glu_unfused(x, g, wk, 1e-5)
    else:
        y = fn.flashnorm_linear_unfused(x, g, wk, 1e-5)
    xn = fn.flashnorm_rmsnorm(x, g, 1e-5)
    torch.cuda.synchronize()
    ref = O.reference_output(kind, bits, 1e-5)
    assert O.rel_err(to_host_f64(y), ref) <= BF16_TOL
    # the normalised intermediate itself
    xn_ref = O.rmsnorm(O.bf16_to_f64(bits["x"]), O.bf16_to_f64(bits["g"]), 1e-5)
    assert O.rel_err(to_host_f64(xn), xn_ref) <= BF16_TOL


def test_folded_unfolded_oracle_agree_smollm2_m64():
    """The 64-token SmolLM2 QKV case: folded + deferred, unfused, and the oracle agree."""
    wl = I.WORKLOADS["smollm2_qkv_m64"]
    bits = wl.draw()
    x, g = to_dev(bits["x"]), to_dev(bits["g"])
    ws = _fold(bits, False)
    ones = to_dev(np.full(wl.d, 0x3F80, dtype=np.uint16))
    wk = fn.flashnorm_fold_weights(to_dev(bits["w"]), ones)
    y_fold = to_host_f64(fn.flashnorm_linear(x, ws, wl.eps))
    y_unf = to_host_f64(fn.flashnorm_linear_unfused(x, g, wk, wl.eps))
    ref = O.reference_output("linear", bits, wl.eps)
    assert O.rel_err(y_fold, ref) <= BF16_TOL
    assert O.rel_err(y_unf, ref) <= BF16_TOL
    assert O.rel_err(y_fold, y_unf) <= 2 * BF16_TOL


# ------------------------------------------------------------------------------------------ full sizes, sampled
FULL = ["smollm2_qkv_m8192", "smollm2_ffn_m8192", "llama7b_qkv_m1", "llama7b_qkv_m4", "llama7b_qkv_m16",
        "llama7b_qkv_m2048", "llama7b_ffn_m2048", "mla_latent_m2048"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    """Every workload at its full size, in the launch configuration the benchmark uses; the oracle
    recomputes a seeded sample of rows (always including the first and last row)."""
    wl = I.WORKLOADS[name]
    bits = wl.draw()
    x = to_dev(bits["x"])
    ws = _fold(bits, wl.kind == "glu")
    if wl.kind == "linear":
        y = fn.flashnorm_linear(x, ws, wl.eps)
    elif wl.kind == "glu":
        y = fn.flashnorm_glu(x, ws, wl.eps)
    else:
        y = fn.flashnorm_linear_postnorm(x, ws, to_dev(bits["g2"]), wl.head_dim, wl.eps2)
    torch.cuda.synchronize()
    rng = np.random.default_rng(99)
    rows = np.unique(np.concatenate([[0, wl.M - 1], rng.integers(0, wl.M, size=min(wl.M, 48))]))
    ref = O.reference_output(wl.kind, bits, wl.eps, eps2=wl.eps2, head_dim=wl.head_dim, rows=rows)
    got = to_host_f64(y)[rows]
    assert O.rel_err(got, ref) <= BF16_TOL
    assert np.isfinite(to_host_f64(y)).all()


# ------------------------------------------------------------------------------------------ join / lag / determinism
@pytest.mark.parametrize("path,M", [("tensor", 300), ("gemv", 4)])
def test_no_stale_output_back_to_back(path, M):
    """Many calls back to back on one stream into ONE output buffer, each followed by an async copy
    out; no host sync in between. Every copy must match its own input and not the previous one
    (the failure the talk pages describe: outputs one step behind)."""
    d, N, T = 576, 960, 24
    wl = _wl("linear", M, d, N, seed=5)
    bits = wl.draw()
    ws = _fold(bits, False)
    xs_bits = [I.activations(M, d, 1000 + t) for t in range(T)]
    xs = [to_dev(b) for b in xs_bits]
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    outs = []
    torch.cuda.synchronize()
    for t in range(T):
        fn.flashnorm_linear(xs[t], ws, 1e-5, out=y, path=path)
        outs.append(y.clone())
    torch.cuda.synchronize()
    for t in range(T):
        b = dict(bits, x=xs_bits[t])
        ref = O.reference_output("linear", b, 1e-5)
        got = to_host_f64(outs[t])
        assert O.rel_err(got, ref) <= BF16_TOL, t
        if t > 0:
            prev = O.reference_output("linear", dict(bits, x=xs_bits[t - 1]), 1e-5)
            assert O.rel_err(got, prev) > 0.1


def test_two_streams_and_determinism():
    bits = _wl("glu", 500, 576, 1536, seed=9).draw()
    x = to_dev(bits["x"])
    ws = _fold(bits, True)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        a = fn.flashnorm_glu(x, ws, 1e-5)
    with torch.cuda.stream(s2):
        b = fn.flashnorm_glu(x, ws, 1e-5)
    torch.cuda.synchronize()
    c = fn.flashnorm_glu(x, ws, 1e-5)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


# ------------------------------------------------------------------------------------------ edge cases
def test_empty_and_zero_rows():
    d, N = 576, 960
    bits = _wl("linear", 40, d, N).draw()
    bits["x"][[0, 17, 39]] = 0  # all-zero rows
    x = to_dev(bits["x"])
    ws = _fold(bits, False)
    for path in ("tensor", "gemv"):
        xx = x if path == "tensor" else x[:16].contiguous()
        y = fn.flashnorm_linear(xx, ws, 1e-5, path=path)
        torch.cuda.synchronize()
        yh = to_host_f64(y)
        assert np.all(yh[0] == 0)
        ref = O.reference_output("linear", dict(bits, x=bits["x"][: xx.shape[0]]), 1e-5)
        assert O.rel_err(yh, ref) <= BF16_TOL
    # M = 0 launches nothing and succeeds
    y0 = fn.flashnorm_linear(x[:0], ws, 1e-5)
    assert y0.shape == (0, N)
    # eps = 0: a zero row is 0 * inf = NaN on both sides, other rows stay finite
    y = to_host_f64(fn.flashnorm_linear(x, ws, 0.0))
    ref = O.reference_output("linear", bits, 0.0)
    assert np.array_equal(np.isnan(y), np.isnan(ref))
    ok = ~np.isnan(ref).any(axis=1)
    assert O.rel_err(y[ok], ref[ok]) <= BF16_TOL


def test_invalid_arguments_raise():
    x = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fn.FlashNormError):
        fn.flashnorm_linear(x, w, 1e-5)  # d = 12 is not a multiple of 8
    x = torch.zeros(64, 576, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(960, 576, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fn.FlashNormError):
        fn.flashnorm_linear(x, w, 1e-5, path="gemv")  # GEMV takes M <= 16
