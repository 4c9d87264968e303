"""GPU parity of the NVFP4 folded weights (E2M1 codes, E4M3 scales per 16 k, a fp32 scale per output channel)
and of the tensor-core decode kernel that streams them, against the fp64 oracle."""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64
from tests.test_gpu_parity import F32_TOL, check_bf16

pytestmark = pytest.mark.gpu


def _case(M, d, N, seed):
    bits = I.Workload("t", "linear_nvfp4", M, d, N, 1e-6, seed=seed).draw()
    Q4, s2 = fn.flashnorm_fold_weights_nvfp4(to_dev(bits["w"]), to_dev(bits["g"]))
    return bits, to_dev(bits["x"]), Q4, s2


@pytest.mark.parametrize("d,N", [(64, 8), (576, 960), (4096, 1024), (208, 136), (272, 40), (4096, 12288)])
def test_fold_nvfp4_bit_exact(d, N):
    """Codes, block scales and channel scales are integer / fp32 decisions: bit for bit the oracle's, in the
    stored layout (partial 256-k groups padded with zeros)."""
    bits = I.Workload("t", "linear_nvfp4", 1, d, N, 1e-6, seed=d + N).draw()
    Q4, s2 = fn.flashnorm_fold_weights_nvfp4(to_dev(bits["w"]), to_dev(bits["g"]))
    torch.cuda.synchronize()
    codes, bsc, s2_ref = O.fold_nvfp4(bits["w"], bits["g"])
    assert np.array_equal(Q4.cpu().numpy(), O.pack_nvfp4(codes, bsc))
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_ref.view(np.uint32))


def test_fold_nvfp4_zero_channel_and_tiny_blocks():
    """An all-zero channel (s2 = 1, every code and scale 0), and blocks whose largest weight is so much
    smaller than the channel's that their E4M3 scale is subnormal or zero."""
    bits = I.Workload("t", "linear_nvfp4", 1, 256, 16, 1e-6, seed=2).draw()
    w = O.bf16_to_f64(bits["w"])
    w[:, 5] = 0
    w[32:64, 7] *= 2.0 ** -17   # block scale about 448 * 2^-17 < 2^-6: E4M3 subnormal
    w[64:80, 7] *= 2.0 ** -30   # below E4M3's range: scale 0, codes 0
    bits = dict(bits, w=O.f64_to_bf16(w))
    Q4, s2 = fn.flashnorm_fold_weights_nvfp4(to_dev(bits["w"]), to_dev(bits["g"]))
    torch.cuda.synchronize()
    codes, bsc, s2_ref = O.fold_nvfp4(bits["w"], bits["g"])
    assert np.array_equal(Q4.cpu().numpy(), O.pack_nvfp4(codes, bsc))
    assert s2[5].item() == 1.0 and int(Q4[5].count_nonzero().item()) == 0
    assert (bsc[7, 2:4] < 8).all() and bsc[7, 4] == 0  # exponent field 0: subnormal, and one zero scale


@pytest.mark.parametrize("workspace", ["auto", None])
@pytest.mark.parametrize("M,d,N", [(1, 4096, 1024), (3, 576, 960), (4, 4096, 2048), (7, 208, 136), (16, 576, 512),
                                   (2, 64, 8), (16, 4096, 12288), (5, 400, 200), (1, 4096, 20480), (9, 2048, 128),
                                   (4, 272, 12288)])
def test_linear_nvfp4_parity(M, d, N, workspace):
    bits, x, Q4, s2 = _case(M, d, N, M * 13 + d)
    y16 = fn.flashnorm_linear_nvfp4(x, Q4, s2, 1e-6, workspace=workspace)
    y32 = fn.flashnorm_linear_nvfp4(x, Q4, s2, 1e-6, out_dtype=torch.float32, workspace=workspace)
    torch.cuda.synchronize()
    ex = O.exact_operand_nvfp4(bits, 1e-6)
    ref = O.reference_output("linear", bits, 1e-6)  # the unquantized definition
    assert O.rel_err(to_host_f64(y32), ex) <= F32_TOL
    # Against the unquantized definition the bar is what NVFP4 itself costs (two significant bits per
    # weight, scaled per 16) plus the output's rounding: the derived bar.
    check_bf16(to_host_f64(y16), ref, ex, derived=True)
    assert O.rel_err(ex, ref) <= 0.3


@pytest.mark.parametrize("workspace", ["auto", None])
@pytest.mark.parametrize("name", ["llama7b_qkv_nvfp4_m1", "llama7b_qkv_nvfp4_m4", "llama7b_qkv_nvfp4_m16"])
def test_linear_nvfp4_full_size(name, workspace):
    """The Llama-7B QKV decode shapes the benchmark runs, every output against the quantized operands."""
    wl = I.WORKLOADS[name]
    bits = wl.draw()
    Q4, s2 = fn.flashnorm_fold_weights_nvfp4(to_dev(bits["w"]), to_dev(bits["g"]))
    y32 = fn.flashnorm_linear_nvfp4(to_dev(bits["x"]), Q4, s2, wl.eps, out_dtype=torch.float32, workspace=workspace)
    torch.cuda.synchronize()
    assert O.rel_err(to_host_f64(y32), O.exact_operand_nvfp4(bits, wl.eps)) <= F32_TOL


def test_nvfp4_workspace_applies_where_expected():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert fn.flashnorm_nvfp4_workspace_bytes(4, 4096, 12288) > 1024
    assert fn.flashnorm_nvfp4_workspace_bytes(4, 4096, 128 * sms + 128) == 0
    assert fn.flashnorm_nvfp4_workspace_bytes(0, 4096, 12288) == 0


def test_nvfp4_workspace_too_small_is_rejected():
    bits, x, Q4, s2 = _case(4, 4096, 12288, 3)
    need = fn.flashnorm_nvfp4_workspace_bytes(4, 4096, 12288)
    small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    y = torch.full((4, 12288), float("nan"), dtype=torch.float32, device="cuda")
    with pytest.raises(fn.FlashNormError):
        fn.flashnorm_linear_nvfp4(x, Q4, s2, 1e-6, out_dtype=torch.float32, out=y, workspace=small)
    torch.cuda.synchronize()
    assert torch.isnan(y).all()


def test_nvfp4_and_fp8_share_the_stream_workspace():
    """NVFP4 and FP8 calls of several shapes, interleaved on one stream with workspace="auto" (one scratch
    per stream for both): every repeat is bitwise the first result, the first is the oracle's, and the
    counters are zero at the end."""
    cases = [(4, 4096, 12288, 5), (1, 576, 960, 6), (16, 2048, 1024, 7)]
    data = []
    for M, d, N, seed in cases:
        bits, x, Q4, s2 = _case(M, d, N, seed)
        b8 = I.Workload("t", "linear_fp8", M, d, N, 1e-6, seed=seed).draw()
        Q8, sc8 = fn.flashnorm_fold_weights_fp8(to_dev(b8["w"]), to_dev(b8["g"]))
        data.append((bits, x, Q4, s2, b8, to_dev(b8["x"]), Q8, sc8))
    run4 = lambda t: fn.flashnorm_linear_nvfp4(t[1], t[2], t[3], 1e-6, out_dtype=torch.float32)
    run8 = lambda t: fn.flashnorm_linear_fp8(t[5], t[6], t[7], 1e-6, out_dtype=torch.float32)
    first = [(run4(t), run8(t)) for t in data]
    outs = []
    for it in range(30):
        t = data[it % len(data)]
        outs.append((run4(t), run8(t)))
    torch.cuda.synchronize()
    for it, (a4, a8) in enumerate(outs):
        f4, f8 = first[it % len(data)]
        assert torch.equal(a4.view(torch.int32), f4.view(torch.int32)), it
        assert torch.equal(a8.view(torch.int32), f8.view(torch.int32)), it
    for t, (f4, f8) in zip(data, first):
        assert O.rel_err(to_host_f64(f4), O.exact_operand_nvfp4(t[0], 1e-6)) <= F32_TOL
        assert O.rel_err(to_host_f64(f8), O.exact_operand_fp8(t[4], 1e-6)) <= F32_TOL
    ws = fn._fp8_ws_cache[(0, fn._stream_ptr(data[0][1]))]
    assert int(ws[:1024].count_nonzero().item()) == 0
