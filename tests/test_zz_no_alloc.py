"""The no-allocation entry point (flashnorm_linear_unfused_noalloc).

Some callers cannot hand the unfused baseline a workspace: their op signature has only inputs and
outputs, or their device memory is entirely owned by their own pool. This entry point keeps the
normalised activations in a fixed scratch array inside the library instead. It runs the same
deterministic kernels as flashnorm_linear_unfused, so its results must equal that entry point's bit
for bit, call after call; both are also held to the oracle's definition at the flat 5e-3 bar that
test_unfused_parity uses. Collected last so that a failure here never hides another.
"""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64

pytestmark = pytest.mark.gpu

BF16_TOL = 5e-3


def _inputs(M, d, N, seed):
    b = I.Workload("noalloc", "linear", M, d, N, 1e-5, seed=seed).draw()
    ones = to_dev(np.full(d, 0x3F80, dtype=np.uint16))
    wk = fn.flashnorm_fold_weights(to_dev(b["w"]), ones)  # unfolded W, K-major
    return b, to_dev(b["x"]), to_dev(b["g"]), wk


def _same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


@pytest.mark.parametrize("M,d,N", [(64, 576, 960), (333, 576, 960), (2048, 4096, 512)])
def test_noalloc_matches_workspace_entry_point_two_calls(M, d, N):
    b1, x1, g, wk = _inputs(M, d, N, seed=M + 1)
    b2, x2, _, _ = _inputs(M, d, N, seed=M + 2)  # a second, different batch through the same scratch
    b2 = dict(b1, x=b2["x"])  # same g and W as the first batch
    refs = [O.reference_output("linear", b, 1e-5) for b in (b1, b2)]
    for out_dtype in (torch.bfloat16, torch.float32):
        for x, ref in zip((x1, x2), refs):
            want = fn.flashnorm_linear_unfused(x, g, wk, 1e-5, out_dtype=out_dtype)
            y = fn.flashnorm_linear_unfused_noalloc(x, g, wk, 1e-5, out_dtype=out_dtype)
            torch.cuda.synchronize()
            assert _same_bits(y, want)
            assert O.rel_err(to_host_f64(y), ref) <= BF16_TOL
    # two calls in a row with no host sync between them, then one check each
    y1 = fn.flashnorm_linear_unfused_noalloc(x1, g, wk, 1e-5)
    y2 = fn.flashnorm_linear_unfused_noalloc(x2, g, wk, 1e-5)
    r1 = fn.flashnorm_linear_unfused(x1, g, wk, 1e-5)
    r2 = fn.flashnorm_linear_unfused(x2, g, wk, 1e-5)
    torch.cuda.synchronize()
    assert _same_bits(y1, r1) and _same_bits(y2, r2)
    assert O.rel_err(to_host_f64(y1), refs[0]) <= BF16_TOL
    assert O.rel_err(to_host_f64(y2), refs[1]) <= BF16_TOL
    fn.flashnorm_check_device_error()


def test_noalloc_rejects_requests_beyond_the_scratch():
    d = 4096
    M = fn.NOALLOC_MAX_ELEMS // d + 1
    x = torch.zeros(M, d, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(d, dtype=torch.bfloat16, device="cuda")
    wk = torch.zeros(64, d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fn.FlashNormError) as ei:
        fn.flashnorm_linear_unfused_noalloc(x, g, wk, 1e-5)
    assert ei.value.status == fn.FN_ERR_UNSUPPORTED
    # the largest request that fits is accepted
    y = fn.flashnorm_linear_unfused_noalloc(x[: M - 1], g, wk, 1e-5)
    torch.cuda.synchronize()
    assert y.shape == (M - 1, 64)
