"""Failure detection on the GPU without a fault: a bounded device-side wait that nothing completes runs
out, the library reports FN_ERR_TIMEOUT through its status word, and the context keeps working."""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    fn.flashnorm_check_device_error()  # start clean
    assert fn.flashnorm_selftest_timeout(20_000) == fn.FN_ERR_TIMEOUT
    # the word was cleared by the read, so the next check is clean again
    fn.flashnorm_check_device_error()


def test_context_usable_after_a_timeout():
    assert fn.flashnorm_selftest_timeout(5_000) == fn.FN_ERR_TIMEOUT
    wl = I.Workload("t", "linear", 300, 576, 960, 1e-5, seed=77)
    bits = wl.draw()
    ws = fn.flashnorm_fold_weights(to_dev(bits["w"]), to_dev(bits["g"]))
    y32 = fn.flashnorm_linear(to_dev(bits["x"]), ws, 1e-5, out_dtype=torch.float32)
    torch.cuda.synchronize()
    fn.flashnorm_check_device_error()
    ex = O.exact_operand_output("linear", bits, O.fold_bf16(bits["w"], bits["g"]), 1e-5)
    assert O.rel_err(to_host_f64(y32), ex) <= 1e-5
    assert np.isfinite(to_host_f64(y32)).all()
