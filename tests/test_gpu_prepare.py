"""Prepared calls (plan once, launch many): the same results as the direct calls, bit for bit, on inputs
rewritten in place, with the scratch they chose kept alive by the prepared call itself."""

import gc

import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64

pytestmark = pytest.mark.gpu


def _bits_eq(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def _cases():
    lin = I.Workload("t", "linear", 4, 1024, 1024, 1e-5, seed=61).draw()
    glu = I.Workload("t", "glu", 300, 576, 768, 1e-5, seed=62).draw()
    pn = I.Workload("t", "postnorm", 256, 2048, 1024, 1e-6, head_dim=512, eps2=1e-6, seed=63).draw()
    f8 = I.Workload("t", "linear_fp8", 5, 4096, 12288, 1e-6, seed=64).draw()
    f4 = I.Workload("t", "linear_nvfp4", 4, 4096, 12288, 1e-6, seed=65).draw()
    W_lin = fn.flashnorm_fold_weights(to_dev(lin["w"]), to_dev(lin["g"]))
    W_glu = fn.flashnorm_fold_weights(to_dev(glu["w"]), to_dev(glu["g"]), glu=True)
    W_pn, g2 = fn.flashnorm_fold_weights(to_dev(pn["w"]), to_dev(pn["g"])), to_dev(pn["g2"])
    Q, sc = fn.flashnorm_fold_weights_fp8(to_dev(f8["w"]), to_dev(f8["g"]))
    Q4, s2 = fn.flashnorm_fold_weights_nvfp4(to_dev(f4["w"]), to_dev(f4["g"]))
    xs = {k: to_dev(b["x"]) for k, b in (("lin", lin), ("glu", glu), ("pn", pn), ("f8", f8), ("f4", f4))}
    calls = {
        "lin": (fn.flashnorm_linear, (xs["lin"], W_lin, 1e-5), {}),
        "glu": (fn.flashnorm_glu, (xs["glu"], W_glu, 1e-5), {}),
        "pn": (fn.flashnorm_linear_postnorm, (xs["pn"], W_pn, g2, 512, 1e-6), {"out_dtype": torch.float32}),
        "f8": (fn.flashnorm_linear_fp8, (xs["f8"], Q, sc, 1e-6), {"out_dtype": torch.float32}),
        "f4": (fn.flashnorm_linear_nvfp4, (xs["f4"], Q4, s2, 1e-6), {"out_dtype": torch.float32}),
    }
    return xs, calls, {"pn": pn, "f8": f8, "f4": f4}


def test_prepared_calls_match_direct_calls():
    xs, calls, _ = _cases()
    prepared = {k: fn.prepare(f, *a, **kw) for k, (f, a, kw) in calls.items()}
    for t in range(3):
        for k, x in xs.items():
            x.copy_(to_dev(I.activations(x.shape[0], x.shape[1], 7000 + 10 * t + len(k))))
        for k, (f, a, kw) in calls.items():
            for _ in range(5):
                got = prepared[k]()
            want = f(*a, **kw)
            torch.cuda.synchronize()
            assert got is prepared[k].result
            assert _bits_eq(got, want), (k, t)
    fn.flashnorm_check_device_error()


def test_prepared_call_keeps_its_workspace():
    """The split post-norm and the FP8 decode choose a workspace inside the call ("auto"); the prepared
    call holds it, so dropping every other reference and collecting garbage changes nothing."""
    xs, calls, bits = _cases()
    f, a, kw = calls["pn"]
    p_pn = fn.prepare(f, *a, **kw)
    f, a, kw = calls["f8"]
    p_f8 = fn.prepare(f, *a, **kw)
    f, a, kw = calls["f4"]
    p_f4 = fn.prepare(f, *a, **kw)
    fn._fp8_ws_cache.clear()
    gc.collect()
    torch.cuda.empty_cache()
    filler = torch.full((64 << 20,), 0x7F, dtype=torch.uint8, device="cuda")  # reuse any freed blocks
    y_pn = p_pn()
    y_f8 = p_f8()
    y_f4 = p_f4()
    torch.cuda.synchronize()
    del filler
    pn, f8 = bits["pn"], bits["f8"]
    W = O.fold_bf16(pn["w"], pn["g"])
    ex_pn = O.exact_operand_output("postnorm", pn, W, 1e-6, eps2=1e-6, head_dim=512)
    assert O.rel_err(to_host_f64(y_pn), ex_pn) <= 1e-5
    assert O.rel_err(to_host_f64(y_f8), O.exact_operand_fp8(f8, 1e-6)) <= 1e-5
    assert O.rel_err(to_host_f64(y_f4), O.exact_operand_nvfp4(bits["f4"], 1e-6)) <= 1e-5
