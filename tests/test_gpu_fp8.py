"""GPU parity of the FP8 (E4M3, per-output-channel scale) folded weights and of the decode GEMV that
streams them, against the fp64 oracle."""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64
from tests.test_gpu_parity import F32_TOL, check_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,N", [(64, 8), (576, 960), (4096, 1024), (208, 136)])
def test_fold_fp8_bit_exact(d, N):
    """The codes and the scales are integer / fp32 decisions: bit for bit the oracle's."""
    bits = I.Workload("t", "linear_fp8", 1, d, N, 1e-6, seed=d + N).draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    torch.cuda.synchronize()
    codes, scales = O.fold_fp8(bits["w"], bits["g"])
    assert np.array_equal(Q.cpu().numpy(), codes)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), scales.view(np.uint32))


def test_fold_fp8_zero_channel():
    bits = I.Workload("t", "linear_fp8", 1, 64, 16, 1e-6, seed=1).draw()
    bits["w"][:, 5] = 0
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    torch.cuda.synchronize()
    assert s[5].item() == 1.0 and int(Q[5].abs().sum().item()) == 0


@pytest.mark.parametrize("M,d,N", [(1, 4096, 1024), (3, 576, 960), (4, 4096, 2048), (7, 208, 136), (16, 576, 512),
                                   (2, 64, 8)])
def test_linear_fp8_parity(M, d, N):
    bits = I.Workload("t", "linear_fp8", M, d, N, 1e-6, seed=M * 13 + d).draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    x = to_dev(bits["x"])
    y16 = fn.flashnorm_linear_fp8(x, Q, s, 1e-6)
    y32 = fn.flashnorm_linear_fp8(x, Q, s, 1e-6, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ex = O.exact_operand_fp8(bits, 1e-6)
    ref = O.reference_output("linear", bits, 1e-6)  # the unquantized definition
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL
    check_bf16(to_host_f64(y16), ref, ex)
    # what E4M3 itself costs against the unquantized chain (3 mantissa bits per weight)
    assert O.rel_err(ex, ref) <= 5e-2


def test_linear_fp8_full_size():
    wl = I.WORKLOADS["llama7b_qkv_fp8_m4"]
    bits = wl.draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    y32 = fn.flashnorm_linear_fp8(to_dev(bits["x"]), Q, s, wl.eps, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert O.rel_err(to_host_f64(y32), O.exact_operand_fp8(bits, wl.eps)) <= F32_TOL
