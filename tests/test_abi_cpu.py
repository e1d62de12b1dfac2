"""C-ABI checks that need no GPU: the library builds and loads, it exports
every entry point include/svdq.h declares, and host-side argument validation
answers before any device work."""
import ctypes

import pytest

import bit_quantized_linear_svdq_b200 as S
from bit_quantized_linear_svdq_b200 import build as B


@pytest.fixture(scope="module")
def lib():
    B.build()
    return S.load_library()


def test_exports_every_declared_symbol(lib):
    names = S.exported_names()
    assert set(names) == {
        "svdq_linear_create", "svdq_linear_destroy", "svdq_workspace_bytes", "svdq_quantize_act",
        "svdq_linear_forward", "svdq_linear_forward_host", "svdq_device_status", "svdq_status_string",
        "svdq_last_error", "svdq_version", "svdq_linear_forward_quantize", "svdq_linear_forward_gemm",
        "svdq_linear_forward_noalloc", "svdq_quantize_weight", "svdq_hadamard_transform",
        "svdq_linear_gemm_kernel", "svdq_mxfp4_create", "svdq_mxfp4_destroy", "svdq_mxfp4_workspace_bytes",
        "svdq_mxfp4_quantize", "svdq_mxfp4_forward", "svdq_mxfp4_device_status", "svdq_fp4_mma_loop",
        "svdq_fp4_mma_loop_status"}
    for n in names:
        assert hasattr(lib, n), n


def test_gemm_kernel_query_without_handle(lib):
    # Host-only query: a NULL handle or M <= 0 names no kernel.
    assert S.svdq_linear_gemm_kernel(None, 1) == ""


def test_status_strings_and_version(lib):
    assert S.svdq_version() >> 16 == 1
    for code in range(7):
        assert S.svdq_status_string(code)
    assert S.svdq_status_string(0) == "ok"


def _desc(**kw):
    base = dict(K=256, N=256, R=32, rotate_block=0, act_unsigned=0, qweight=1, wscales=1, proj_down=1,
                proj_up=1, smooth_factor=1, wcscales=None, wtscale=None)
    base.update(kw)
    return S.svdq_linear_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(K=24), 2),                 # K % 16
    (dict(K=0), 2),
    (dict(N=0), 2),
    (dict(R=8), 2),
    (dict(R=40), 2),
    (dict(R=256), 2),
    (dict(rotate_block=64), 2),
    (dict(K=272, rotate_block=128), 2),
    (dict(act_unsigned=1), 3),
    (dict(qweight=None), 1),
    (dict(smooth_factor=None), 1),
])
def test_create_validation_is_host_side(lib, kw, status):
    h = ctypes.c_void_p(123)
    st = lib.svdq_linear_create(ctypes.byref(h), ctypes.byref(_desc(**kw)), None)
    assert st == status
    assert h.value is None


def test_null_handle_calls(lib):
    assert lib.svdq_workspace_bytes(None, 16) == 0
    assert lib.svdq_quantize_act(None, 1, 1, 1, 1, None, None) == 1
    assert lib.svdq_linear_forward(None, 1, 1, 1, 1, None) == 1
    assert lib.svdq_linear_forward_noalloc(None, 1, 1, 1, None) == 1
    assert lib.svdq_linear_create(None, None, None) == 1
    lib.svdq_linear_destroy(None)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(S, "_lib", None)
    monkeypatch.setattr(S, "library_path", lambda: str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="not built"):
        S.load_library()


@pytest.mark.parametrize("args,status", [
    ((0, 16, 256, 0, 16, 16), 1),        # null weight
    ((16, 16, 256, 0, 0, 16), 1),        # null qweight
    ((16, 16, 256, 0, 16, 0), 1),        # null wscales
    ((8, 16, 256, 0, 16, 16), 1),        # weight not 16-byte aligned
    ((16, 16, 256, 0, 12, 16), 1),       # qweight not 8-byte aligned
    ((16, 16, 24, 0, 16, 16), 2),        # K % 16
    ((16, 0, 256, 0, 16, 16), 2),        # N < 1
    ((16, 16, 272, 128, 16, 16), 2),     # rotation block does not divide K
    ((16, 16, 256, 64, 16, 16), 2),      # rotation block other than 128
])
def test_quantize_weight_argument_errors(lib, args, status):
    """Argument errors are answered on the host, before any launch."""
    w, N, K, rot, qw, ws = args
    assert lib.svdq_quantize_weight(w, N, K, rot, qw, ws, None) == status


@pytest.mark.parametrize("args,status", [
    ((16, 4, 3, 0), 2),          # n not a power of two
    ((16, 4, 0, 0), 2),          # n < 1
    ((16, 4, 65536, 0), 2),      # n > 32768
    ((16, 4, 64, 2), 1),         # dtype other than bf16 / fp16
    ((16, -1, 64, 0), 1),        # rows < 0
    ((0, 4, 64, 0), 1),          # null x
    ((17, 4, 64, 0), 1),         # x not 2-byte aligned
    ((0, 0, 64, 0), 0),          # no rows: no-op
])
def test_hadamard_transform_argument_errors(lib, args, status):
    x, rows, n, dt = args
    assert lib.svdq_hadamard_transform(x, rows, n, dt, None) == status


@pytest.mark.parametrize("kw,status", [
    (dict(K=48), 2),                 # K % 32
    (dict(K=0), 2),
    (dict(N=0), 2),
    (dict(hadamard_group=16), 2),
    (dict(qweight=None), 1),
    (dict(wscales=None), 1),
    (dict(alpha=float("inf")), 1),
])
def test_mxfp4_create_rejects_bad_desc_on_host(lib, kw, status):
    base = dict(K=256, N=256, hadamard_group=32, qweight=1, wscales=1, alpha=1.0)
    base.update(kw)
    h = ctypes.c_void_p(123)
    st = lib.svdq_mxfp4_create(ctypes.byref(h), ctypes.byref(S.svdq_mxfp4_desc(**base)), None)
    assert st == status and h.value is None


def test_mxfp4_quantize_rejects_bad_args_on_host(lib):
    assert lib.svdq_mxfp4_quantize(16, 4, 48, 32, 16, 16, None) == 2     # K % 32
    assert lib.svdq_mxfp4_quantize(16, 4, 64, 8, 16, 16, None) == 2      # group
    assert lib.svdq_mxfp4_quantize(None, 4, 64, 32, 16, 16, None) == 1   # null x
    assert lib.svdq_mxfp4_quantize(24, 4, 64, 32, 16, 16, None) == 1     # misaligned x
    assert lib.svdq_mxfp4_quantize(16, 0, 64, 32, 16, 16, None) == 0     # M == 0: no-op
    assert lib.svdq_mxfp4_workspace_bytes(None, 4) == 0
    assert lib.svdq_mxfp4_forward(None, 16, 4, 16, 256, None) == 1


def test_fp4_loop_rejects_bad_iters_on_host(lib):
    ctas = ctypes.c_int(-1)
    assert lib.svdq_fp4_mma_loop(0, ctypes.byref(ctas), None) == 1
    assert lib.svdq_fp4_mma_loop((1 << 20) + 1, ctypes.byref(ctas), None) == 1


def test_build_stamp_is_independent_of_the_tree_location(tmp_path):
    # The stamp beside the library is a digest of the sources and flags; a copy
    # of the tree at another path (with its built library) must not rebuild,
    # and a changed source must.
    import importlib.util
    import shutil

    root = tmp_path / "copy"
    shutil.copytree(B.PKG, root / "bit_quantized_linear_svdq_b200",
                    ignore=shutil.ignore_patterns("_lib", "__pycache__"))
    shutil.copytree(f"{B.ROOT}/include", root / "include")
    spec = importlib.util.spec_from_file_location("build_copy", root / "bit_quantized_linear_svdq_b200" / "build.py")
    Bc = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(Bc)
    assert Bc.ROOT == str(root)
    assert Bc._digest(Bc._sources()[1]) == B._digest(B._sources()[1])
    with open(root / "bit_quantized_linear_svdq_b200" / "csrc" / "kcommon.cuh", "a") as f:
        f.write("\n")
    assert Bc._digest(Bc._sources()[1]) != B._digest(B._sources()[1])
