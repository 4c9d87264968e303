"""GPU parity of LayerNorm -> linear (gain folded, 1/sqrt(var + eps) deferred, mean removed by a rank-1
correction with the column sums of W*, beta turned into a bias) against the fp64 oracle."""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64
from tests.test_gpu_parity import F32_TOL, check_bf16

pytestmark = pytest.mark.gpu


def _fold(bits, with_beta=True):
    return fn.flashnorm_fold_layernorm(to_dev(bits["w"]), to_dev(bits["g"]), to_dev(bits["beta"]) if with_beta else None)


def test_fold_outputs():
    """W* is the RMSNorm fold bit for bit; colsum and bias match the oracle's on the same bf16 values."""
    bits = I.Workload("t", "layernorm", 8, 200, 136, 1e-5, seed=3).draw()
    Ws, cs, b = _fold(bits)
    ref_ws = fn.flashnorm_fold_weights(to_dev(bits["w"]), to_dev(bits["g"]))
    torch.cuda.synchronize()
    assert torch.equal(Ws.view(torch.int16), ref_ws.view(torch.int16))
    ws64 = O.bf16_to_f64(O.fold_bf16(bits["w"], bits["g"]))
    assert np.max(np.abs(cs.cpu().numpy() - ws64.sum(axis=0))) <= 1e-5 * np.max(np.abs(ws64.sum(axis=0)))
    b64 = O.bf16_to_f64(bits["beta"]) @ O.bf16_to_f64(bits["w"])
    assert np.max(np.abs(b.cpu().numpy() - b64)) <= 1e-5 * np.max(np.abs(b64))
    _, _, b0 = _fold(bits, with_beta=False)
    torch.cuda.synchronize()
    assert torch.count_nonzero(b0) == 0


@pytest.mark.parametrize("M,d,N", [(300, 576, 960), (17, 576, 960), (130, 72, 200), (600, 4096, 512),
                                   (257, 256, 1536),
                                   # decode-sized: the tensor-core decode kernel (K split in 2 and in 4)
                                   (1, 4096, 1024), (4, 576, 960), (16, 256, 1536), (7, 200, 136),
                                   (16, 4096, 12288)])
def test_layernorm_parity(M, d, N):
    bits = I.Workload("t", "layernorm", M, d, N, 1e-5, seed=M + d).draw()
    Ws, cs, b = _fold(bits)
    x = to_dev(bits["x"])
    y16 = fn.flashnorm_layernorm_linear(x, Ws, cs, b, 1e-5)
    y32 = fn.flashnorm_layernorm_linear(x, Ws, cs, b, 1e-5, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.reference_layernorm(bits, 1e-5)
    ex = O.exact_operand_layernorm(bits, O.fold_bf16(bits["w"], bits["g"]), 1e-5)
    check_bf16(to_host_f64(y16), ref, ex)
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL


def test_layernorm_full_size_sampled():
    wl = I.WORKLOADS["layernorm_qkv_m8192"]
    bits = wl.draw()
    Ws, cs, b = _fold(bits)
    y = fn.flashnorm_layernorm_linear(to_dev(bits["x"]), Ws, cs, b, wl.eps)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, wl.M - 1], np.random.default_rng(6).integers(0, wl.M, 48)]))
    ref = O.reference_layernorm(bits, wl.eps, rows=rows)
    ex = O.exact_operand_layernorm(bits, O.fold_bf16(bits["w"], bits["g"]), wl.eps, rows=rows)
    yh = to_host_f64(y)
    check_bf16(yh[rows], ref, ex)
    assert np.isfinite(yh).all()


def test_layernorm_many_tiles_all_rows():
    """Every row with several tiles per CTA pair (the 1/sigma and mean of a row block are computed once and
    reused across its column tiles)."""
    bits = I.Workload("t", "layernorm", 2048, 576, 6144, 1e-6, seed=9).draw()
    Ws, cs, b = _fold(bits)
    y32 = fn.flashnorm_layernorm_linear(to_dev(bits["x"]), Ws, cs, b, 1e-6, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ex = O.exact_operand_layernorm(bits, O.fold_bf16(bits["w"], bits["g"]), 1e-6)
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL


def test_layernorm_decode_full_size():
    """The benchmark's LayerNorm decode shape (4 tokens, Llama-7B QKV): every output against the oracle."""
    wl = I.WORKLOADS["layernorm_llama7b_qkv_m4"]
    bits = wl.draw()
    Ws, cs, b = _fold(bits)
    x = to_dev(bits["x"])
    y16 = fn.flashnorm_layernorm_linear(x, Ws, cs, b, wl.eps)
    y32 = fn.flashnorm_layernorm_linear(x, Ws, cs, b, wl.eps, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ex = O.exact_operand_layernorm(bits, O.fold_bf16(bits["w"], bits["g"]), wl.eps)
    check_bf16(to_host_f64(y16), O.reference_layernorm(bits, wl.eps), ex)
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL
