"""Guard bands: every kernel family writes exactly its output and nothing past it.

Each output is a contiguous slice at the start of a larger buffer whose remainder holds a sentinel
pattern; after the call the sentinel must be intact, and the output must match the oracle. Shapes are
ragged (M not a multiple of any tile, N not a multiple of the tile width) so that the partial tiles and
the row and column guards in the epilogues are exercised."""

import numpy as np
import pytest
import torch

import flashnorm_inputs as I
import rmsnorm_linear_projection_fold_b200 as fn
from oracle import flashnorm_oracle as O
from tests.gpu_util import to_dev, to_host_f64

pytestmark = pytest.mark.gpu

PAD = 4096          # elements of sentinel after the output
SENTINEL = 0x7BAD   # a bf16 / fp32-half pattern no kernel writes by accident


def _guarded(shape, dtype):
    n = int(np.prod(shape))
    flat = torch.empty(n + PAD, dtype=torch.int16 if dtype == torch.bfloat16 else torch.int32, device="cuda")
    flat.fill_(SENTINEL if dtype == torch.bfloat16 else (SENTINEL << 16) | SENTINEL)
    out = flat[:n].view(dtype).view(*shape)
    return flat, out, n


def _intact(flat, n):
    tail = flat[n:].cpu().numpy()
    ref = SENTINEL if flat.dtype == torch.int16 else (SENTINEL << 16) | SENTINEL
    return bool(np.all(tail == ref))


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("kind,M,d,N,path", [
    ("linear", 333, 576, 968, "pair"), ("linear", 333, 576, 968, "tensor"), ("linear", 7, 576, 968, "decode"),
    ("linear", 5, 576, 968, "gemv"), ("glu", 301, 576, 272, "pair"), ("glu", 301, 576, 272, "tensor"),
    ("glu", 9, 576, 272, "decode"),
])
def test_projection_writes_stay_in_bounds(kind, M, d, N, path, out_dtype):
    bits = I.Workload("t", kind, M, d, N, 1e-5, seed=M + N).draw()
    glu = kind == "glu"
    ws = fn.flashnorm_fold_weights(to_dev(bits["w"]), to_dev(bits["g"]), glu=glu)
    flat, y, n = _guarded((M, N), out_dtype)
    f = fn.flashnorm_glu if glu else fn.flashnorm_linear
    f(to_dev(bits["x"]), ws, 1e-5, out_dtype=out_dtype, out=y, path=path)
    torch.cuda.synchronize()
    assert _intact(flat, n)
    ex = O.exact_operand_output(kind, bits, O.fold_bf16(bits["w"], bits["g"]), 1e-5)
    tol = 1e-5 if out_dtype == torch.float32 else 5e-3
    assert O.rel_err(to_host_f64(y), ex) <= tol


@pytest.mark.parametrize("M,d,N,hd", [(130, 256, 640, 64), (70, 320, 512, 512), (40, 128, 640, 320)])
def test_postnorm_writes_stay_in_bounds(M, d, N, hd):
    bits = I.Workload("t", "postnorm", M, d, N, 1e-6, head_dim=hd, eps2=1e-6, seed=M).draw()
    ws = fn.flashnorm_fold_weights(to_dev(bits["w"]), to_dev(bits["g"]))
    flat, y, n = _guarded((M, N), torch.float32)
    fn.flashnorm_linear_postnorm(to_dev(bits["x"]), ws, to_dev(bits["g2"]), hd, 1e-6, out_dtype=torch.float32, out=y)
    torch.cuda.synchronize()
    assert _intact(flat, n)
    ex = O.exact_operand_output("postnorm", bits, O.fold_bf16(bits["w"], bits["g"]), 1e-6, eps2=1e-6, head_dim=hd)
    assert O.rel_err(to_host_f64(y), ex) <= 1e-5


@pytest.mark.parametrize("M,d,N,hd", [(700, 1000, 320, 320), (150, 5120, 1024, 512)])
def test_postnorm_split_writes_stay_in_bounds(M, d, N, hd):
    """The split wide-head schedule: its partial products stay inside the workspace size the query
    reports, and the finalize kernel writes exactly y."""
    need = fn.flashnorm_postnorm_workspace_bytes(M, d, N, hd)
    assert need > 0
    bits = I.Workload("t", "postnorm", M, d, N, 1e-6, head_dim=hd, eps2=1e-6, seed=M + 1).draw()
    ws = fn.flashnorm_fold_weights(to_dev(bits["w"]), to_dev(bits["g"]))
    flat_ws, wsp, n_ws = _guarded((need // 4,), torch.float32)
    flat, y, n = _guarded((M, N), torch.bfloat16)
    fn.flashnorm_linear_postnorm(to_dev(bits["x"]), ws, to_dev(bits["g2"]), hd, 1e-6, out=y,
                                 workspace=wsp.view(torch.uint8))
    torch.cuda.synchronize()
    assert _intact(flat_ws, n_ws) and _intact(flat, n)
    ex = O.exact_operand_output("postnorm", bits, O.fold_bf16(bits["w"], bits["g"]), 1e-6, eps2=1e-6, head_dim=hd)
    assert O.rel_err(to_host_f64(y), ex) <= 5e-3


@pytest.mark.parametrize("M,d,N", [(5, 1008, 200), (3, 4096, 12288), (16, 208, 136)])
def test_fp8_workspace_writes_stay_in_bounds(M, d, N):
    """FP8 decode with its K split over a workspace: the partials stay inside the size the query reports,
    the counters are zero again afterwards, and y is written exactly."""
    need = fn.flashnorm_fp8_workspace_bytes(M, d, N)
    assert need > 1024
    bits = I.Workload("t", "linear_fp8", M, d, N, 1e-6, seed=M + d).draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    flat_ws, wsp, n_ws = _guarded((need // 4,), torch.float32)
    wsp[:256].view(torch.int32).zero_()  # the counters start at zero
    flat, y, n = _guarded((M, N), torch.bfloat16)
    for _ in range(3):
        fn.flashnorm_linear_fp8(to_dev(bits["x"]), Q, s, 1e-6, out=y, path="decode", workspace=wsp.view(torch.uint8))
    torch.cuda.synchronize()
    assert _intact(flat_ws, n_ws) and _intact(flat, n)
    assert int(wsp[:256].view(torch.int32).count_nonzero().item()) == 0
    assert O.rel_err(to_host_f64(y), O.exact_operand_fp8(bits, 1e-6)) <= 5e-3


@pytest.mark.parametrize("M,d,N,workspace", [(5, 1008, 200, True), (3, 4096, 12288, True), (7, 272, 136, False)])
def test_nvfp4_writes_stay_in_bounds(M, d, N, workspace):
    """NVFP4 decode: the partials stay inside the workspace size the query reports (the counters zero again
    afterwards), the fold writes exactly its two outputs, and y is written exactly."""
    bits = I.Workload("t", "linear_nvfp4", M, d, N, 1e-6, seed=M + d + 1).draw()
    rowb = -(-d // 256) * 144
    flat_q, q4, n_q = _guarded((N * rowb // 2,), torch.bfloat16)   # the codes' bytes, viewed as int16
    flat_s, s2, n_s = _guarded((N,), torch.float32)
    Q4, S2 = q4.view(torch.uint8).view(N, rowb), s2
    W, g = to_dev(bits["w"]), to_dev(bits["g"])
    assert fn.load_library().flashnorm_fold_weights_nvfp4(W.data_ptr(), g.data_ptr(), Q4.data_ptr(), S2.data_ptr(),
                                                          d, N, fn._stream_ptr(W)) == fn.FN_OK
    ws = None
    if workspace:
        need = fn.flashnorm_nvfp4_workspace_bytes(M, d, N)
        assert need > 1024
        flat_ws, wsp, n_ws = _guarded((need // 4,), torch.float32)
        wsp[:256].view(torch.int32).zero_()
        ws = wsp.view(torch.uint8)
    flat, y, n = _guarded((M, N), torch.bfloat16)
    for _ in range(3):
        fn.flashnorm_linear_nvfp4(to_dev(bits["x"]), Q4, S2, 1e-6, out=y, workspace=ws)
    torch.cuda.synchronize()
    assert _intact(flat_q, n_q) and _intact(flat_s, n_s) and _intact(flat, n)
    if workspace:
        assert _intact(flat_ws, n_ws) and int(wsp[:256].view(torch.int32).count_nonzero().item()) == 0
    assert O.rel_err(to_host_f64(y), O.exact_operand_nvfp4(bits, 1e-6)) <= 5e-3


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_layernorm_decode_writes_stay_in_bounds(out_dtype):
    """LayerNorm at decode size (the tensor-core decode kernel, ragged N, K split over a cluster)."""
    bits = I.Workload("t", "layernorm", 5, 576, 200, 1e-5, seed=41).draw()
    Ws, cs, bias = fn.flashnorm_fold_layernorm(to_dev(bits["w"]), to_dev(bits["g"]), to_dev(bits["beta"]))
    flat, y, n = _guarded((5, 200), out_dtype)
    fn.flashnorm_layernorm_linear(to_dev(bits["x"]), Ws, cs, bias, 1e-5, out_dtype=out_dtype, out=y)
    torch.cuda.synchronize()
    assert _intact(flat, n)
    tol = 1e-5 if out_dtype == torch.float32 else 5e-3
    ex = O.exact_operand_layernorm(bits, O.fold_bf16(bits["w"], bits["g"]), 1e-5)
    assert O.rel_err(to_host_f64(y), ex if out_dtype == torch.float32 else O.reference_layernorm(bits, 1e-5)) <= tol


def test_rope_layernorm_fp8_unfused_writes_stay_in_bounds():
    # RoPE on the post-norm path
    M, d, hd, H = 77, 256, 64, 3
    wl = I.Workload("t", "postnorm_rope", M, d, H * hd, 1e-6, head_dim=hd, eps2=1e-6, seed=3, n_rope_heads=2)
    bits = wl.draw()
    cs = fn.flashnorm_rope_table(M, hd)
    pos = torch.from_numpy(wl.positions()).cuda()
    flat, y, n = _guarded((M, H * hd), torch.bfloat16)
    fn.flashnorm_linear_postnorm_rope(to_dev(bits["x"]), fn.flashnorm_fold_weights(to_dev(bits["w"]), to_dev(bits["g"])),
                                      to_dev(bits["g2"]), cs, pos, hd, 2, 1e-6, out=y)
    torch.cuda.synchronize()
    assert _intact(flat, n)
    # LayerNorm
    bits = I.Workload("t", "layernorm", 145, 576, 200, 1e-5, seed=4).draw()
    Ws, csum, bias = fn.flashnorm_fold_layernorm(to_dev(bits["w"]), to_dev(bits["g"]), to_dev(bits["beta"]))
    flat, y, n = _guarded((145, 200), torch.bfloat16)
    fn.flashnorm_layernorm_linear(to_dev(bits["x"]), Ws, csum, bias, 1e-5, out=y)
    torch.cuda.synchronize()
    assert _intact(flat, n)
    assert O.rel_err(to_host_f64(y), O.reference_layernorm(bits, 1e-5)) <= 5e-3
    # FP8 decode
    bits = I.Workload("t", "linear_fp8", 3, 576, 136, 1e-6, seed=5).draw()
    Q, s = fn.flashnorm_fold_weights_fp8(to_dev(bits["w"]), to_dev(bits["g"]))
    flat, y, n = _guarded((3, 136), torch.float32)
    fn.flashnorm_linear_fp8(to_dev(bits["x"]), Q, s, 1e-6, out_dtype=torch.float32, out=y)
    torch.cuda.synchronize()
    assert _intact(flat, n)
    assert O.rel_err(to_host_f64(y), O.exact_operand_fp8(bits, 1e-6)) <= 1e-5
    # unfused baseline: both its intermediate and its output
    bits = I.Workload("t", "linear", 150, 576, 520, 1e-5, seed=6).draw()
    ones = to_dev(np.full(576, 0x3F80, dtype=np.uint16))
    wk = fn.flashnorm_fold_weights(to_dev(bits["w"]), ones)
    flat_xn, xn, n_xn = _guarded((150, 576), torch.bfloat16)
    flat, y, n = _guarded((150, 520), torch.bfloat16)
    fn.flashnorm_linear_unfused(to_dev(bits["x"]), to_dev(bits["g"]), wk, 1e-5, xn_ws=xn, out=y)
    torch.cuda.synchronize()
    assert _intact(flat_xn, n_xn) and _intact(flat, n)
    fn.flashnorm_check_device_error()
