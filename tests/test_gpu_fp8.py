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


# (path, workspace): the tensor-core kernel with its contraction split over independent CTAs through a
# workspace ("auto") or inside thread-block clusters (None); the CUDA-core GEMV
PATHS_WS = [("decode", "auto"), ("decode", None), ("gemv", None)]


@pytest.mark.parametrize("path,workspace", PATHS_WS)
@pytest.mark.parametrize("M,d,N", [(1, 4096, 1024), (3, 576, 960), (4, 4096, 2048), (7, 208, 136), (16, 576, 512),
                                   (2, 64, 8), (16, 4096, 12288), (5, 400, 200), (5, 1008, 6000), (1, 4096, 20480),
                                   (9, 2048, 128), (4, 128, 12288)])
def test_linear_fp8_parity(M, d, N, path, workspace):
    bits = I.Workload("t", "linear_fp8", M, d, N, 1e-6, seed=M * 13 + d).draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    x = to_dev(bits["x"])
    y16 = fn.flashnorm_linear_fp8(x, Q, s, 1e-6, path=path, workspace=workspace)
    y32 = fn.flashnorm_linear_fp8(x, Q, s, 1e-6, out_dtype=torch.float32, path=path, workspace=workspace)
    torch.cuda.synchronize()
    ex = O.exact_operand_fp8(bits, 1e-6)
    ref = O.reference_output("linear", bits, 1e-6)  # the unquantized definition
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL
    # Against the unquantized definition the bar is what E4M3 itself costs (the quantization is the
    # method's approximation, 3 mantissa bits per weight) plus the output's rounding: the derived bar.
    check_bf16(to_host_f64(y16), ref, ex, derived=True)
    assert O.rel_err(ex, ref) <= 5e-2


@pytest.mark.parametrize("path,workspace", PATHS_WS)
@pytest.mark.parametrize("name", ["llama7b_qkv_fp8_m1", "llama7b_qkv_fp8_m4", "llama7b_qkv_fp8_m16"])
def test_linear_fp8_full_size(name, path, workspace):
    """The Llama-7B QKV decode shapes the benchmark runs, every output against the quantized operands."""
    wl = I.WORKLOADS[name]
    bits = wl.draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    y32 = fn.flashnorm_linear_fp8(to_dev(bits["x"]), Q, s, wl.eps, out_dtype=torch.float32, path=path,
                                  workspace=workspace)
    torch.cuda.synchronize()
    assert O.rel_err(to_host_f64(y32), O.exact_operand_fp8(bits, wl.eps)) <= F32_TOL


def test_linear_fp8_token_scales_cover_a_wide_range():
    """Tokens whose magnitudes differ by 2^40 and a token with one huge and many tiny values: the per-token
    power-of-two scale keeps every activation exact in the tensor-core kernel's f16 operand."""
    bits = I.Workload("t", "linear_fp8", 6, 1024, 384, 1e-6, seed=77).draw()
    x = O.bf16_to_f64(bits["x"])
    x[0] *= 2.0 ** -20
    x[1] *= 2.0 ** 20
    x[2, 0] = 3.0e4       # one large value, the rest about 1: the small ones stay exact
    x[3] *= 2.0 ** -60    # far below f16's range without the scale
    x[4] = 0.0            # zero row
    bits = dict(bits, x=O.f64_to_bf16(x))
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    y32 = fn.flashnorm_linear_fp8(to_dev(bits["x"]), Q, s, 1e-6, out_dtype=torch.float32, path="decode")
    torch.cuda.synchronize()
    ex = O.exact_operand_fp8(bits, 1e-6)
    got = to_host_f64(y32)
    for m in range(6):  # row by row: the rows' scales differ by many decades
        assert O.rel_err(got[m], ex[m]) <= F32_TOL, m


@pytest.mark.parametrize("path,workspace", PATHS_WS)
def test_linear_fp8_subnormal_codes(path, workspace):
    """Every channel: one weight at the channel's maximum (code 448) and all others in E4M3's subnormal range
    (|W*| / s below 2^-6). The subnormal codes carry about 1e-3 of each output, so a widening that flushed
    them to zero would miss the fp32 bar by two orders of magnitude."""
    M, d, N = 3, 1024, 256
    bits = I.Workload("t", "linear_fp8", M, d, N, 1e-6, seed=31).draw()
    rng = np.random.default_rng(8)
    g = O.bf16_to_f64(bits["g"])
    mag = rng.uniform(0.2, 0.9, size=(d, N)) * 2.0 ** -6 / 448.0
    w = np.where(rng.random((d, N)) < 0.5, -mag, mag) / g[:, None]
    k0 = rng.integers(0, d, size=N)
    w[k0, np.arange(N)] = 1.0 / g[k0]
    bits = dict(bits, w=I.f32_to_bf16_bits(w.astype(np.float32)))
    codes, _ = O.fold_fp8(bits["w"], bits["g"])
    assert np.mean((codes & 0x78) == 0) > 0.9  # exponent field zero: subnormal (or zero) codes
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    y32 = fn.flashnorm_linear_fp8(to_dev(bits["x"]), Q, s, 1e-6, out_dtype=torch.float32, path=path,
                                  workspace=workspace)
    torch.cuda.synchronize()
    ex = O.exact_operand_fp8(bits, 1e-6)
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL


def _fp8_case(M, d, N, seed):
    bits = I.Workload("t", "linear_fp8", M, d, N, 1e-6, seed=seed).draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    return bits, to_dev(bits["x"]), Q, s


def test_fp8_workspace_applies_where_expected():
    """The split takes a workspace while there are at most as many 128-row slabs as SMs."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert fn.flashnorm_fp8_workspace_bytes(4, 4096, 12288) > 1024
    assert fn.flashnorm_fp8_workspace_bytes(4, 4096, 128 * sms) > 1024
    assert fn.flashnorm_fp8_workspace_bytes(4, 4096, 128 * sms + 128) == 0
    assert fn.flashnorm_fp8_workspace_bytes(0, 4096, 12288) == 0


def test_fp8_workspace_too_small_is_rejected():
    bits, x, Q, s = _fp8_case(4, 4096, 12288, 3)
    need = fn.flashnorm_fp8_workspace_bytes(4, 4096, 12288)
    small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    y = torch.full((4, 12288), float("nan"), dtype=torch.float32, device="cuda")
    with pytest.raises(fn.FlashNormError):
        fn.flashnorm_linear_fp8(x, Q, s, 1e-6, out_dtype=torch.float32, out=y, path="decode", workspace=small)
    torch.cuda.synchronize()
    assert torch.isnan(y).all()  # nothing was launched


def test_fp8_workspace_shared_back_to_back():
    """One workspace serves calls of different shapes on one stream, one after another: each call leaves
    the counters at zero, every repeat is bitwise the first result, and the first is the oracle's."""
    cases = [(4, 4096, 12288, 5), (1, 576, 960, 6), (16, 2048, 1024, 7), (3, 208, 136, 8)]
    need = max(fn.flashnorm_fp8_workspace_bytes(M, d, N) for M, d, N, _ in cases)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    data = [_fp8_case(M, d, N, seed) for M, d, N, seed in cases]
    first = []
    for bits, x, Q, s in data:
        first.append(fn.flashnorm_linear_fp8(x, Q, s, 1e-6, out_dtype=torch.float32, workspace=ws))
    outs = []
    for it in range(60):
        bits, x, Q, s = data[it % len(data)]
        outs.append(fn.flashnorm_linear_fp8(x, Q, s, 1e-6, out_dtype=torch.float32, workspace=ws))
    torch.cuda.synchronize()
    for it, y in enumerate(outs):
        assert torch.equal(y.view(torch.int32), first[it % len(data)].view(torch.int32)), it
    for (bits, x, Q, s), y in zip(data, first):
        assert O.rel_err(to_host_f64(y), O.exact_operand_fp8(bits, 1e-6)) <= F32_TOL
    assert int(ws[:1024].count_nonzero().item()) == 0


def test_fp8_workspace_auto_per_stream():
    """workspace="auto" on two streams: each stream gets its own scratch, and both results are exact."""
    bits, x, Q, s = _fp8_case(4, 4096, 12288, 9)
    ref = fn.flashnorm_linear_fp8(x, Q, s, 1e-6, out_dtype=torch.float32, workspace=None)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    ys = []
    for st in (s1, s2):
        with torch.cuda.stream(st):
            ys.append([fn.flashnorm_linear_fp8(x, Q, s, 1e-6, out_dtype=torch.float32) for _ in range(20)])
    torch.cuda.synchronize()
    ex = O.exact_operand_fp8(bits, 1e-6)
    for lst in ys:
        assert O.rel_err(to_host_f64(lst[-1]), ex) <= F32_TOL
        for y in lst[1:]:
            assert torch.equal(y.view(torch.int32), lst[0].view(torch.int32))
    assert O.rel_err(to_host_f64(ref), ex) <= F32_TOL
