"""The C-ABI library: it loads without a GPU, exports every entry point the header declares, and
rejects bad arguments on the host before it would touch the device."""

import ctypes
import os
import re

import pytest

import rmsnorm_linear_projection_fold_b200 as fn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashnorm.h")


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^FN_API\s+[\w\s\*]+?\b(flashnorm_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from rmsnorm_linear_projection_fold_b200 import build

    build.build()
    return fn.load_library()


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for required in ("flashnorm_fold_weights", "flashnorm_linear", "flashnorm_glu", "flashnorm_linear_postnorm"):
        assert required in names
    # the binding knows every declared entry point, and nothing undeclared
    assert set(names) == set(fn.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.flashnorm_version() >= 100
    for s in range(6):
        assert lib.flashnorm_status_string(s).startswith(b"FN_")


# Fake, aligned, never-dereferenced addresses: every call below must be rejected on the host.
P = ctypes.c_void_p(1 << 20)
P_MISALIGNED = ctypes.c_void_p((1 << 20) + 2)
NULL = ctypes.c_void_p(0)


@pytest.mark.parametrize("args,expected", [
    ((P, P, P, 4, 7, 960, 1e-5, 0, 0, NULL), fn.FN_ERR_INVALID_ARG),      # d % 8 != 0
    ((P, P, P, 4, 576, 964, 1e-5, 0, 0, NULL), fn.FN_ERR_INVALID_ARG),    # N % 8 != 0
    ((P, P, P, -1, 576, 960, 1e-5, 0, 0, NULL), fn.FN_ERR_INVALID_ARG),   # M < 0
    ((P, P, P, 4, 576, 960, -1.0, 0, 0, NULL), fn.FN_ERR_INVALID_ARG),    # eps < 0
    ((P, P, P, 4, 576, 960, float("nan"), 0, 0, NULL), fn.FN_ERR_INVALID_ARG),
    ((P, P, P, 4, 576, 960, 1e-5, 7, 0, NULL), fn.FN_ERR_INVALID_ARG),    # out dtype
    ((P, P, P, 4, 576, 960, 1e-5, 0, 9, NULL), fn.FN_ERR_INVALID_ARG),    # path
    ((NULL, P, P, 4, 576, 960, 1e-5, 0, 0, NULL), fn.FN_ERR_INVALID_ARG),  # x NULL
    ((P_MISALIGNED, P, P, 4, 576, 960, 1e-5, 0, 0, NULL), fn.FN_ERR_ALIGN),
    ((P, P, P, 64, 576, 960, 1e-5, 0, 2, NULL), fn.FN_ERR_UNSUPPORTED),   # GEMV forced with M > 16
    ((P, P, P, 0, 576, 960, 1e-5, 0, 0, NULL), fn.FN_OK),                # empty call: nothing launched
])
def test_linear_validation(lib, args, expected):
    assert lib.flashnorm_linear_ex(*args) == expected
    if expected != fn.FN_OK:
        assert lib.flashnorm_last_error() != b""


def test_glu_postnorm_fold_validation(lib):
    # GLU: F must be a multiple of 16
    assert lib.flashnorm_glu_ex(P, P, P, 4, 576, 24, 1e-5, 0, 0, NULL) == fn.FN_ERR_INVALID_ARG
    # post-norm: head_dim limits and N % head_dim
    assert lib.flashnorm_linear_postnorm(P, P, P, P, 4, 576, 1024, 1024, 1e-6, 0, NULL) == fn.FN_ERR_UNSUPPORTED
    assert lib.flashnorm_linear_postnorm(P, P, P, P, 4, 576, 1000, 8, 1e-6, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_linear_postnorm(P, P, P, P, 4, 576, 960, 128, 1e-6, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_linear_postnorm(P, P, P, NULL, 4, 576, 512, 128, 1e-6, 0, NULL) == fn.FN_ERR_INVALID_ARG
    # fold: sizes, flags, GLU needs N = 2F with F % 16 == 0
    assert lib.flashnorm_fold_weights(P, P, P, 576, 12, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_fold_weights(P, P, P, 576, 960, 2, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_fold_weights(P, P, P, 576, 48, 1, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_fold_weights(P, P, P_MISALIGNED, 576, 960, 0, NULL) == fn.FN_ERR_ALIGN
    # unfused: the workspace pointer is checked
    assert lib.flashnorm_linear_unfused(P, P, P, NULL, P, 4, 576, 960, 1e-5, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_rmsnorm(P, P, P, 4, 12, 1e-5, NULL) == fn.FN_ERR_INVALID_ARG


def test_postnorm_workspace_validation(lib):
    """The workspace entry point validates like flashnorm_linear_postnorm, and its size query rejects
    shapes the call would reject."""
    assert lib.flashnorm_linear_postnorm_ws(P, P, P, P, 4, 576, 1024, 1024, 1e-6, 0, NULL, 0, NULL) == \
        fn.FN_ERR_UNSUPPORTED
    assert lib.flashnorm_linear_postnorm_ws(P, P, P, P, 4, 576, 960, 128, 1e-6, 0, NULL, 0, NULL) == \
        fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_linear_postnorm_ws(P, P, P, P, 4, 576, 512, 512, 1e-6, 0, P, -1, NULL) == \
        fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_linear_postnorm_ws(P, P, P, P, 0, 576, 512, 512, 1e-6, 0, NULL, 0, NULL) == fn.FN_OK
    nbytes = ctypes.c_int64(-7)
    out = ctypes.c_void_p(ctypes.addressof(nbytes))
    assert lib.flashnorm_postnorm_workspace_bytes(2048, 5120, 512, 512, NULL) == fn.FN_ERR_INVALID_ARG
    for shape in [(2048, 5120, 500, 512), (2048, 5120, 512, 24), (2048, 12, 512, 512), (-1, 5120, 512, 512),
                  (2048, 5120, 1024, 1024)]:
        assert lib.flashnorm_postnorm_workspace_bytes(*shape, out) == fn.FN_ERR_INVALID_ARG, shape
    # heads of at most 256 features never split; an empty call needs nothing
    for shape in [(2048, 5120, 1024, 256), (0, 5120, 512, 512)]:
        assert lib.flashnorm_postnorm_workspace_bytes(*shape, out) == fn.FN_OK
        assert nbytes.value == 0


def test_binding_rejects_cpu_tensors():
    import torch

    x = torch.zeros(4, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fn.flashnorm_linear(x, torch.zeros(16, 16, dtype=torch.bfloat16), 1e-5)


def test_binding_rejects_mixed_devices():
    # the C ABI takes bare pointers on one device, so the binding refuses tensors spread over several
    import torch

    a, b = torch.zeros(2), torch.zeros(2, device="meta")
    fn._same_device(a, b=torch.zeros(3), c=None)
    with pytest.raises(ValueError, match="b is on meta"):
        fn._same_device(a, b=b)


@pytest.mark.parametrize("limit_us", [0, -5, 10_000_001])
def test_selftest_timeout_rejects_bad_limits(lib, limit_us):
    assert lib.flashnorm_selftest_timeout(limit_us, NULL) == fn.FN_ERR_INVALID_ARG


# flashnorm_linear_postnorm_rope(x, W*, g2, rope_cs, positions, y, M, d, N, head_dim, n_rope_heads, max_pos, eps2,
#                                out_dtype, stream): rejected on the host
@pytest.mark.parametrize("hd,n_rope,max_pos,pos_ptr,expected", [
    (24, 1, 16, P, fn.FN_ERR_INVALID_ARG),    # head_dim % 16 != 0
    (512, 1, 16, P, fn.FN_ERR_UNSUPPORTED),   # wide heads run on the cluster kernel, which has no RoPE
    (64, -1, 16, P, fn.FN_ERR_INVALID_ARG),   # n_rope_heads < 0
    (64, 5, 16, P, fn.FN_ERR_INVALID_ARG),    # more rotated heads than heads (N = 256)
    (64, 1, 0, P, fn.FN_ERR_INVALID_ARG),     # empty table
    (64, 1, 16, NULL, fn.FN_ERR_INVALID_ARG),  # no positions
    (64, 1, 16, ctypes.c_void_p((1 << 20) + 2), fn.FN_ERR_ALIGN),  # positions not 4-byte aligned
])
def test_postnorm_rope_validation(lib, hd, n_rope, max_pos, pos_ptr, expected):
    st = lib.flashnorm_linear_postnorm_rope(P, P, P, P, pos_ptr, P, 4, 128, 256 if hd != 512 else 512, hd, n_rope,
                                            max_pos, 1e-6, 0, NULL)
    assert st == expected


@pytest.mark.parametrize("max_pos,hd,base", [(0, 64, 1e4), (8, 7, 1e4), (8, 64, 1.0), (8, 64, float("inf"))])
def test_rope_table_validation(lib, max_pos, hd, base):
    assert lib.flashnorm_rope_table(P, max_pos, hd, base, NULL) == fn.FN_ERR_INVALID_ARG


def test_layernorm_validation(lib):
    # d % 8, N % 8, eps < 0, misaligned colsum: all rejected on the host
    assert lib.flashnorm_layernorm_linear(P, P, P, P, P, 4, 12, 64, 1e-5, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_layernorm_linear(P, P, P, P, P, 4, 64, 60, 1e-5, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_layernorm_linear(P, P, P, P, P, 4, 64, 64, -1.0, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_layernorm_linear(P, P, P_MISALIGNED, P, P, 4, 64, 64, 1e-5, 0, NULL) == fn.FN_ERR_ALIGN
    assert lib.flashnorm_fold_layernorm(P, P, P, P, P, NULL, 64, 64, NULL) == fn.FN_ERR_INVALID_ARG


def test_fp8_fold_validation(lib):
    assert lib.flashnorm_fold_weights_fp8(P, P, P, P, 24, 64, NULL) == fn.FN_ERR_INVALID_ARG   # d % 16
    assert lib.flashnorm_fold_weights_fp8(P, P, P, P, 64, 60, NULL) == fn.FN_ERR_INVALID_ARG   # N % 8
    assert lib.flashnorm_linear_fp8(P, P, P, P, 17, 64, 64, 1e-6, 0, NULL) == fn.FN_ERR_UNSUPPORTED  # M > 16
    assert lib.flashnorm_linear_fp8(P, P, P, P, 4, 72, 64, 1e-6, 0, NULL) == fn.FN_ERR_INVALID_ARG  # d % 16


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no fallback: every entry point goes through load_library, which raises when the library is not built
    monkeypatch.setattr(fn, "_LIB_PATH", str(tmp_path / "libflashnorm.so"))
    monkeypatch.setattr(fn, "_lib", None)
    with pytest.raises(fn.FlashNormError, match="is missing"):
        fn.load_library()


def test_header_is_plain_c_and_links(tmp_path):
    # a C99 program that includes the header, takes the address of every declared entry point and is
    # linked against the library: the boundary needs nothing beyond C and the shared object
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    from rmsnorm_linear_projection_fold_b200 import build

    lib_path = build.build()
    names = _declared_symbols()
    src = tmp_path / "consumer.c"
    src.write_text("#include \"flashnorm.h\"\n#include <stdio.h>\n"
                   "typedef void (*fn_ptr)(void);\n"
                   "int main(void) {\n  fn_ptr fns[] = {\n"
                   + "".join(f"    (fn_ptr)&{n},\n" for n in names)
                   + "  };\n  printf(\"%d\\n\", (int)(sizeof(fns) / sizeof(fns[0])));\n  return 0;\n}\n")
    exe = tmp_path / "consumer"
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
           lib_path, "-Wl,--unresolved-symbols=ignore-in-shared-libs", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, LD_LIBRARY_PATH=os.path.dirname(lib_path) + ":" + os.environ.get("LD_LIBRARY_PATH", ""))
    r = subprocess.run([str(exe)], capture_output=True, text=True, env=env, timeout=60)
    assert r.returncode == 0 and int(r.stdout) == len(names), (r.stdout, r.stderr)


def test_noalloc_limit_matches_the_header():
    text = open(HEADER).read()
    m = re.search(r"#define\s+FN_NOALLOC_MAX_ELEMS\s+\(?\s*([^\n/]+?)\)?\s*(?:/[/*].*)?$", text, flags=re.M)
    assert m, "FN_NOALLOC_MAX_ELEMS not found in the header"
    expr = m.group(1).replace("LL", "").replace("ll", "").replace("(int64_t)", "")
    assert eval(expr, {"__builtins__": {}}) == fn.NOALLOC_MAX_ELEMS


# flashnorm_linear_unfused_noalloc(x, g, W_kmajor, y, M, d, N, eps, out_dtype, stream): everything below is
# decided before any CUDA call, so fake pointers never reach the device.
@pytest.mark.parametrize("args,expected", [
    ((P, P, P, P, 4, 576, 964, 1e-5, 0, NULL), fn.FN_ERR_INVALID_ARG),            # N % 8 != 0
    ((NULL, P, P, P, 4, 576, 960, 1e-5, 0, NULL), fn.FN_ERR_INVALID_ARG),         # x NULL
    ((P_MISALIGNED, P, P, P, 4, 576, 960, 1e-5, 0, NULL), fn.FN_ERR_ALIGN),       # x misaligned
    ((P, P, P, P, 4, 576, 960, -1.0, 0, NULL), fn.FN_ERR_INVALID_ARG),            # eps < 0
    ((P, P, P, P, fn.NOALLOC_MAX_ELEMS // 4096 + 1, 4096, 512, 1e-5, 0, NULL), fn.FN_ERR_UNSUPPORTED),
    ((P, P, P, P, 0, 576, 960, 1e-5, 0, NULL), fn.FN_OK),                          # empty call
])
def test_noalloc_validation(lib, args, expected):
    assert lib.flashnorm_linear_unfused_noalloc(*args) == expected
    if expected != fn.FN_OK:
        assert lib.flashnorm_last_error() != b""


# flashnorm_linear_fp8_ex(x, Q, scales, y, M, d, N, eps, out_dtype, path, stream): rejected on the host
@pytest.mark.parametrize("args,expected", [
    ((P, P, P, P, 4, 576, 960, 1e-6, 0, 1, NULL), fn.FN_ERR_INVALID_ARG),    # the 1-CTA prefill path
    ((P, P, P, P, 4, 576, 960, 1e-6, 0, 9, NULL), fn.FN_ERR_INVALID_ARG),    # unknown path
    ((P, P, P, P, 17, 576, 960, 1e-6, 0, 0, NULL), fn.FN_ERR_UNSUPPORTED),   # decode only: M <= 16
    ((P, P, P, P, 4, 584, 960, 1e-6, 0, 3, NULL), fn.FN_ERR_INVALID_ARG),    # d % 16 != 0
    ((P, P, NULL, P, 4, 576, 960, 1e-6, 0, 3, NULL), fn.FN_ERR_INVALID_ARG),  # scales NULL
    ((P, P, P, P, 0, 576, 960, 1e-6, 0, 3, NULL), fn.FN_OK),                  # empty call
])
def test_fp8_validation(lib, args, expected):
    assert lib.flashnorm_linear_fp8_ex(*args) == expected


def test_fp8_workspace_validation(lib):
    """The workspace entry point validates like flashnorm_linear_fp8_ex before it looks at the device,
    and its size query rejects shapes the call would reject (no device needed for either)."""
    ws = fn._SIGNATURES["flashnorm_linear_fp8_ws"]
    assert len(ws) == 13
    assert lib.flashnorm_linear_fp8_ws(P, P, P, P, 4, 576, 960, 1e-6, 0, 9, NULL, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_linear_fp8_ws(P, P, P, P, 17, 576, 960, 1e-6, 0, 0, NULL, 0, NULL) == fn.FN_ERR_UNSUPPORTED
    assert lib.flashnorm_linear_fp8_ws(P, P, P, P, 4, 584, 960, 1e-6, 0, 3, NULL, 0, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_linear_fp8_ws(P, P, P, P, 4, 576, 960, 1e-6, 0, 3, P, -1, NULL) == fn.FN_ERR_INVALID_ARG
    assert lib.flashnorm_linear_fp8_ws(P, P, P, P, 0, 576, 960, 1e-6, 0, 3, P, 16, NULL) == fn.FN_OK
    nbytes = ctypes.c_int64(-7)
    out = ctypes.c_void_p(ctypes.addressof(nbytes))
    assert lib.flashnorm_fp8_workspace_bytes(4, 4096, 12288, NULL) == fn.FN_ERR_INVALID_ARG
    for shape in [(4, 4104, 12288), (4, 4096, 12284), (-1, 4096, 12288), (4, 0, 12288)]:
        assert lib.flashnorm_fp8_workspace_bytes(*shape, out) == fn.FN_ERR_INVALID_ARG, shape
    # an empty call and M above the decode limit need nothing (and no device to say so)
    for shape in [(0, 4096, 12288), (17, 4096, 12288)]:
        nbytes.value = -7
        assert lib.flashnorm_fp8_workspace_bytes(*shape, out) == fn.FN_OK
        assert nbytes.value == 0


def test_binding_names_resolve():
    """Every name the package exports exists (a star import would fail otherwise)."""
    for name in fn.__all__:
        assert hasattr(fn, name), name


def test_prepare_propagates_errors_and_resets():
    """prepare() runs the call's own checks: a rejected call raises as it would directly, and leaves no
    recording state behind (a second prepare is not taken for a nested one)."""
    import torch

    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    for _ in range(2):
        with pytest.raises((ValueError, TypeError, fn.FlashNormError)):
            fn.prepare(fn.flashnorm_linear, x, x, 1e-5)
    assert fn._recording() is None and getattr(fn._rec, "keep", None) is None


def test_prepare_recording_is_per_thread():
    """While one thread records a call for prepare(), library calls of other threads are not captured."""
    import threading

    seen = {}
    fn._rec.calls, fn._rec.keep = [], []
    try:
        t = threading.Thread(target=lambda: seen.setdefault("other", fn._recording()))
        t.start()
        t.join()
        assert seen["other"] is None and fn._recording() == []
    finally:
        fn._rec.calls, fn._rec.keep = None, None


def test_nvfp4_validation(lib):
    """The NVFP4 entry points reject bad shapes on the host; the size query needs no device for them."""
    assert lib.flashnorm_fold_weights_nvfp4(P, P, P, P, 24, 64, NULL) == fn.FN_ERR_INVALID_ARG   # d % 16
    assert lib.flashnorm_fold_weights_nvfp4(P, P, P, P, 64, 60, NULL) == fn.FN_ERR_INVALID_ARG   # N % 8
    assert lib.flashnorm_fold_weights_nvfp4(P, P, NULL, P, 64, 64, NULL) == fn.FN_ERR_INVALID_ARG  # Q4 NULL
    lin = lib.flashnorm_linear_nvfp4
    assert lin(P, P, P, P, 17, 4096, 12288, 1e-6, 0, NULL, 0, NULL) == fn.FN_ERR_UNSUPPORTED     # M > 16
    assert lin(P, P, P, P, 4, 4104, 12288, 1e-6, 0, NULL, 0, NULL) == fn.FN_ERR_INVALID_ARG      # d % 16
    assert lin(P, P, P, P, 4, 4096, 12284, 1e-6, 0, NULL, 0, NULL) == fn.FN_ERR_INVALID_ARG      # N % 8
    assert lin(P, P, NULL, P, 4, 4096, 12288, 1e-6, 0, NULL, 0, NULL) == fn.FN_ERR_INVALID_ARG   # s2 NULL
    assert lin(P, P, P, P, 4, 4096, 12288, 1e-6, 0, P, -1, NULL) == fn.FN_ERR_INVALID_ARG        # bytes < 0
    assert lin(P, P, P, P, 0, 4096, 12288, 1e-6, 0, NULL, 0, NULL) == fn.FN_OK                   # empty call
    nbytes = ctypes.c_int64(-7)
    out = ctypes.c_void_p(ctypes.addressof(nbytes))
    assert lib.flashnorm_nvfp4_workspace_bytes(4, 4096, 12288, NULL) == fn.FN_ERR_INVALID_ARG
    for shape in [(4, 4104, 12288), (4, 4096, 12284), (-1, 4096, 12288)]:
        assert lib.flashnorm_nvfp4_workspace_bytes(*shape, out) == fn.FN_ERR_INVALID_ARG, shape
    for shape in [(0, 4096, 12288), (17, 4096, 12288)]:
        nbytes.value = -7
        assert lib.flashnorm_nvfp4_workspace_bytes(*shape, out) == fn.FN_OK
        assert nbytes.value == 0
