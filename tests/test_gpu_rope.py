"""GPU parity of the post-norm epilogue with RoPE on the query/key heads, and of the library's (cos, sin)
table, against the fp64 oracle (rotation of feature pairs (2i, 2i+1) by position * base^(-2i/head_dim))."""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64
from tests.test_gpu_parity import F32_TOL, _fold, check_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("max_pos,hd,base", [(2048, 256, 10000.0), (8192, 128, 10000.0), (100, 64, 500000.0)])
def test_rope_table_matches_oracle(max_pos, hd, base):
    cs = fn.flashnorm_rope_table(max_pos, hd, base)
    torch.cuda.synchronize()
    ref = O.rope_table(max_pos, hd, base)
    got = cs.cpu().numpy().astype(np.float64)
    # both sides take the angle and its cos / sin in float64 and round once to fp32: within one fp32 rounding
    assert np.max(np.abs(got - ref)) <= 2.0 ** -24 * 1.01


def _run(M, d, H, hd, n_rope, seed, max_pos=None, positions=None):
    wl = I.Workload("t", "postnorm_rope", M, d, H * hd, 1e-6, head_dim=hd, eps2=1e-6, seed=seed, n_rope_heads=n_rope)
    bits = wl.draw()
    if positions is None:
        rng = np.random.default_rng(seed)
        max_pos = max_pos or 4 * M
        positions = rng.integers(0, max_pos, M).astype(np.int32)
    cs = fn.flashnorm_rope_table(max_pos, hd, wl.rope_base)
    x, ws, g2 = to_dev(bits["x"]), _fold(bits, False), to_dev(bits["g2"])
    pos = torch.from_numpy(positions).cuda()
    y16 = fn.flashnorm_linear_postnorm_rope(x, ws, g2, cs, pos, hd, n_rope, 1e-6)
    y32 = fn.flashnorm_linear_postnorm_rope(x, ws, g2, cs, pos, hd, n_rope, 1e-6, out_dtype=torch.float32)
    torch.cuda.synchronize()
    return wl, bits, positions, max_pos, y16, y32


@pytest.mark.parametrize("M,d,H,hd,n_rope", [
    (300, 512, 4, 128, 3),     # three rotated heads, one value head, ragged M
    (130, 256, 8, 64, 8),      # every head rotated, four heads per tile
    (257, 576, 2, 256, 1),     # one 256-wide head per tile
    (64, 320, 6, 64, 0),       # no head rotated: equals flashnorm_linear_postnorm
    (40, 128, 1, 320, 1),      # 320-wide head on the single-CTA 512-column path
])
def test_postnorm_rope_parity(M, d, H, hd, n_rope):
    wl, bits, pos, max_pos, y16, y32 = _run(M, d, H, hd, n_rope, seed=M + hd)
    ref = O.reference_postnorm_rope(bits, 1e-6, 1e-6, hd, pos, n_rope, wl.rope_base)
    table32 = O.rope_table(max_pos, hd, wl.rope_base).astype(np.float32)
    ex = O.exact_operand_postnorm_rope(bits, O.fold_bf16(bits["w"], bits["g"]), 1e-6, hd, pos, n_rope, table32)
    check_bf16(to_host_f64(y16), ref, ex)
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL
    if n_rope == 0:
        plain = fn.flashnorm_linear_postnorm(to_dev(bits["x"]), _fold(bits, False), to_dev(bits["g2"]), hd, 1e-6)
        torch.cuda.synchronize()
        assert torch.equal(plain.view(torch.int16), y16.view(torch.int16))


def test_postnorm_rope_full_size_sampled():
    """The Gemma-width case the benchmark runs (positions 0 .. M-1), a seeded sample of rows."""
    wl = I.WORKLOADS["gemma_qkvnorm_rope_hd256_m2048"]
    bits = wl.draw()
    positions = wl.positions()
    cs = fn.flashnorm_rope_table(wl.M, wl.head_dim, wl.rope_base)
    y = fn.flashnorm_linear_postnorm_rope(to_dev(bits["x"]), _fold(bits, False), to_dev(bits["g2"]), cs,
                                          torch.from_numpy(positions).cuda(), wl.head_dim, wl.n_rope_heads, wl.eps2)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, wl.M - 1], np.random.default_rng(4).integers(0, wl.M, 40)]))
    ref = O.reference_postnorm_rope(bits, wl.eps, wl.eps2, wl.head_dim, positions, wl.n_rope_heads, wl.rope_base,
                                    rows=rows)
    table32 = O.rope_table(wl.M, wl.head_dim, wl.rope_base).astype(np.float32)
    ex = O.exact_operand_postnorm_rope(bits, O.fold_bf16(bits["w"], bits["g"]), wl.eps2, wl.head_dim, positions,
                                       wl.n_rope_heads, table32, rows=rows)
    yh = to_host_f64(y)
    check_bf16(yh[rows], ref, ex)
    assert np.isfinite(yh).all()


def test_position_outside_table_is_reported():
    M, hd, H = 50, 64, 3
    positions = np.arange(M, dtype=np.int32)
    positions[7] = 64   # == max_pos
    positions[11] = -1
    wl, bits, pos, max_pos, y16, y32 = _run(M, 128, H, hd, 2, seed=5, max_pos=64, positions=positions)
    with pytest.raises(fn.FlashNormError) as e:
        fn.flashnorm_check_device_error()
    assert e.value.status == fn.FN_ERR_INVALID_ARG
    yh = to_host_f64(y32)
    bad = [7, 11]
    assert np.all(np.isnan(yh[bad, : 2 * hd]))          # rotated heads of the bad rows
    assert np.all(np.isfinite(yh[bad, 2 * hd:]))        # their value head is still normalised
    good = np.setdiff1d(np.arange(M), bad)
    table32 = O.rope_table(64, hd, wl.rope_base).astype(np.float32)
    ex = O.exact_operand_postnorm_rope(bits, O.fold_bf16(bits["w"], bits["g"]), 1e-6, hd, pos, 2, table32, rows=good)
    assert O.rel_err(yh[good], ex) <= F32_TOL
    fn.flashnorm_check_device_error()  # the word was cleared
