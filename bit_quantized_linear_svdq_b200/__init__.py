"""B200 (sm_100a) SVDQuant W4A4 linear layer -- Python binding of the C ABI.

The entry points mirror include/svdq.h name for name and only marshal
arguments (pointers, sizes, streams); all arithmetic runs in the CUDA library
``_lib/libsvdq_b200.so`` (build it with ``python -m bit_quantized_linear_svdq_b200.build``).
There is no fallback: if the library is missing or cannot be loaded, every
call raises.

PyTorch supplies device memory and streams only.  ``SVDQLinear`` is a small
convenience wrapper that validates tensor dtypes/shapes and owns a workspace.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

__all__ = [
    "SvdqError", "svdq_linear_desc", "load_library", "library_path", "exported_names",
    "svdq_linear_create", "svdq_linear_destroy", "svdq_workspace_bytes", "svdq_quantize_act",
    "svdq_linear_forward", "svdq_linear_forward_host", "svdq_linear_forward_quantize",
    "svdq_linear_forward_gemm", "svdq_linear_gemm_kernel", "svdq_device_status", "svdq_status_string",
    "svdq_last_error", "svdq_version", "svdq_quantize_weight", "quantize_weight", "svdq_hadamard_transform",
    "hadamard_transform", "SVDQLinear", "STATUS", "svdq_mxfp4_desc", "svdq_mxfp4_create", "svdq_mxfp4_destroy",
    "svdq_mxfp4_workspace_bytes", "svdq_mxfp4_quantize", "svdq_mxfp4_forward", "svdq_mxfp4_device_status",
    "mxfp4_quantize", "MXFP4Linear", "svdq_fp4_mma_loop", "svdq_fp4_mma_loop_status",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_HEADER = os.path.join(os.path.dirname(_PKG), "include", "svdq.h")

STATUS = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_SHAPE", 3: "SVDQ_ERR_UNSUPPORTED",
    4: "SVDQ_ERR_CUDA", 5: "SVDQ_ERR_WORKSPACE", 6: "SVDQ_ERR_DEVICE",
}
SVDQ_ERR_WORKSPACE = 5

# Size of the fixed per-device scratch array of svdq_linear_forward_noalloc
# (SVDQ_NOALLOC_SCRATCH_BYTES in the header).
NOALLOC_SCRATCH_BYTES = 32 << 20


class SvdqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = svdq_last_error() if _lib is not None else ""
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class svdq_linear_desc(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int), ("N", ctypes.c_int), ("R", ctypes.c_int),
        ("rotate_block", ctypes.c_int), ("act_unsigned", ctypes.c_int),
        ("qweight", ctypes.c_void_p), ("wscales", ctypes.c_void_p),
        ("proj_down", ctypes.c_void_p), ("proj_up", ctypes.c_void_p),
        ("smooth_factor", ctypes.c_void_p), ("wcscales", ctypes.c_void_p),
        ("wtscale", ctypes.c_void_p),
    ]


class svdq_mxfp4_desc(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int), ("N", ctypes.c_int), ("hadamard_group", ctypes.c_int),
        ("qweight", ctypes.c_void_p), ("wscales", ctypes.c_void_p), ("alpha", ctypes.c_float),
    ]


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return os.path.join(_PKG, "_lib", "libsvdq_b200.so")


def load_library() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run: python -m bit_quantized_linear_svdq_b200.build)")
    lib = ctypes.CDLL(path)
    vp, ci, cs = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "svdq_linear_create": (ci, [ctypes.POINTER(vp), ctypes.POINTER(svdq_linear_desc), vp]),
        "svdq_linear_destroy": (None, [vp]),
        "svdq_workspace_bytes": (cs, [vp, ci]),
        "svdq_quantize_act": (ci, [vp, vp, ci, vp, vp, vp, vp]),
        "svdq_linear_forward": (ci, [vp, vp, ci, vp, vp, vp]),
        "svdq_linear_forward_host": (ci, [vp, vp, ci, vp, vp, vp, vp, vp]),
        "svdq_linear_forward_quantize": (ci, [vp, vp, ci, vp, vp]),
        "svdq_linear_forward_gemm": (ci, [vp, ci, vp, vp, vp]),
        "svdq_linear_gemm_kernel": (ctypes.c_char_p, [vp, ci]),
        "svdq_linear_forward_noalloc": (ci, [vp, vp, ci, vp, vp]),
        "svdq_device_status": (ci, [vp, ctypes.POINTER(ci)]),
        "svdq_status_string": (ctypes.c_char_p, [ci]),
        "svdq_last_error": (ctypes.c_char_p, []),
        "svdq_version": (ci, []),
        "svdq_quantize_weight": (ci, [vp, ci, ci, ci, vp, vp, vp]),
        "svdq_hadamard_transform": (ci, [vp, ci, ci, ci, vp]),
        "svdq_mxfp4_create": (ci, [ctypes.POINTER(vp), ctypes.POINTER(svdq_mxfp4_desc), vp]),
        "svdq_mxfp4_destroy": (None, [vp]),
        "svdq_mxfp4_workspace_bytes": (cs, [vp, ci]),
        "svdq_mxfp4_quantize": (ci, [vp, ci, ci, ci, vp, vp, vp]),
        "svdq_mxfp4_forward": (ci, [vp, vp, ci, vp, vp, vp]),
        "svdq_mxfp4_device_status": (ci, [vp, ctypes.POINTER(ci)]),
        "svdq_fp4_mma_loop": (ci, [ci, ctypes.POINTER(ci), vp]),
        "svdq_fp4_mma_loop_status": (ci, [ctypes.POINTER(ci)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def exported_names():
    """Function names declared with SVDQ_API in include/svdq.h."""
    with open(_HEADER) as f:
        text = f.read()
    return re.findall(r"SVDQ_API\s+[\w\s\*]+?\b(svdq_\w+)\s*\(", text)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SvdqError(status, where)


# ----------------------------------------------------------------- 1:1 C ABI

def svdq_version() -> int:
    return load_library().svdq_version()


def svdq_status_string(status: int) -> str:
    return load_library().svdq_status_string(status).decode()


def svdq_last_error() -> str:
    return load_library().svdq_last_error().decode()


def svdq_linear_create(desc: svdq_linear_desc, stream=None) -> int:
    h = ctypes.c_void_p()
    _check(load_library().svdq_linear_create(ctypes.byref(h), ctypes.byref(desc), _stream(stream)),
           "svdq_linear_create")
    return h.value


def svdq_linear_destroy(handle: Optional[int]) -> None:
    load_library().svdq_linear_destroy(handle)


def svdq_workspace_bytes(handle: int, M: int) -> int:
    return load_library().svdq_workspace_bytes(handle, M)


def svdq_quantize_act(handle, x_ptr, M, codes_ptr, scales_ptr, lowrank_ptr=None, stream=None) -> None:
    _check(load_library().svdq_quantize_act(handle, x_ptr, M, codes_ptr, scales_ptr, lowrank_ptr,
                                            _stream(stream)), "svdq_quantize_act")


def svdq_linear_forward(handle, x_ptr, M, y_ptr, workspace_ptr, stream=None) -> None:
    _check(load_library().svdq_linear_forward(handle, x_ptr, M, y_ptr, workspace_ptr, _stream(stream)),
           "svdq_linear_forward")


def svdq_linear_forward_quantize(handle, x_ptr, M, workspace_ptr, stream=None) -> None:
    _check(load_library().svdq_linear_forward_quantize(handle, x_ptr, M, workspace_ptr, _stream(stream)),
           "svdq_linear_forward_quantize")


def svdq_linear_forward_gemm(handle, M, y_ptr, workspace_ptr, stream=None) -> None:
    _check(load_library().svdq_linear_forward_gemm(handle, M, y_ptr, workspace_ptr, _stream(stream)),
           "svdq_linear_forward_gemm")


def svdq_linear_gemm_kernel(handle, M) -> str:
    """Name of the kernel svdq_linear_forward_gemm launches for M rows."""
    return (load_library().svdq_linear_gemm_kernel(handle, M) or b"").decode()


def svdq_linear_forward_host(handle, x_host_ptr, M, y_host_ptr, x_dev_ptr, y_dev_ptr, workspace_ptr,
                             stream=None) -> None:
    _check(load_library().svdq_linear_forward_host(handle, x_host_ptr, M, y_host_ptr, x_dev_ptr, y_dev_ptr,
                                                   workspace_ptr, _stream(stream)),
           "svdq_linear_forward_host")


def svdq_linear_forward_noalloc(handle, x_ptr, M, y_ptr, stream=None) -> None:
    """The forward pass with its intermediates in the library's fixed per-device
    scratch array (no workspace argument, nothing allocated): for callers that
    cannot allocate device memory when they run the layer.  M too large for the
    array raises SvdqError(SVDQ_ERR_WORKSPACE); calls that can overlap on the
    GPU share the array and race."""
    st = load_library().svdq_linear_forward_noalloc(handle, x_ptr, M, y_ptr, _stream(stream))
    if st == SVDQ_ERR_WORKSPACE:
        need = svdq_workspace_bytes(handle, M)
        raise SvdqError(st, f"svdq_linear_forward_noalloc: M={M} needs {need} bytes of scratch, "
                            f"the fixed array holds {NOALLOC_SCRATCH_BYTES}")
    _check(st, "svdq_linear_forward_noalloc")


def svdq_quantize_weight(w_ptr, N, K, rotate_block, qweight_ptr, wscales_ptr, stream=None) -> None:
    _check(load_library().svdq_quantize_weight(w_ptr, N, K, rotate_block, qweight_ptr, wscales_ptr,
                                               _stream(stream)), "svdq_quantize_weight")


def svdq_hadamard_transform(x_ptr, rows, n, dtype, stream=None) -> None:
    _check(load_library().svdq_hadamard_transform(x_ptr, rows, n, dtype, _stream(stream)), "svdq_hadamard_transform")


def hadamard_transform(x: torch.Tensor, inplace: bool = True, stream=None) -> torch.Tensor:
    """x <- x H_n / sqrt(n) along the last dimension (n a power of two <= 32768), bf16 or fp16."""
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError("x must be bf16 or fp16")
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    y = x if inplace else x.clone()
    n = y.shape[-1] if y.dim() else 1
    rows = y.numel() // n if n else 0
    svdq_hadamard_transform(y.data_ptr(), rows, n, 0 if y.dtype == torch.bfloat16 else 1, stream)
    return y


def svdq_mxfp4_create(desc: "svdq_mxfp4_desc", stream=None) -> int:
    h = ctypes.c_void_p()
    _check(load_library().svdq_mxfp4_create(ctypes.byref(h), ctypes.byref(desc), _stream(stream)),
           "svdq_mxfp4_create")
    return h.value


def svdq_mxfp4_destroy(handle: Optional[int]) -> None:
    load_library().svdq_mxfp4_destroy(handle)


def svdq_mxfp4_workspace_bytes(handle: int, M: int) -> int:
    return load_library().svdq_mxfp4_workspace_bytes(handle, M)


def svdq_mxfp4_quantize(x_ptr, M, K, hadamard_group, codes_ptr, scales_ptr, stream=None) -> None:
    _check(load_library().svdq_mxfp4_quantize(x_ptr, M, K, hadamard_group, codes_ptr, scales_ptr, _stream(stream)),
           "svdq_mxfp4_quantize")


def svdq_mxfp4_forward(handle, x_ptr, M, y_ptr, workspace_ptr, stream=None) -> None:
    _check(load_library().svdq_mxfp4_forward(handle, x_ptr, M, y_ptr, workspace_ptr, _stream(stream)),
           "svdq_mxfp4_forward")


def svdq_mxfp4_device_status(handle) -> int:
    flags = ctypes.c_int(0)
    st = load_library().svdq_mxfp4_device_status(handle, ctypes.byref(flags))
    if st not in (0, 6):
        raise SvdqError(st, "svdq_mxfp4_device_status")
    return flags.value


def mxfp4_quantize(x: torch.Tensor, hadamard_group: int = 32, stream=None):
    """x (M, K) bf16 -> (codes (M, K/2) uint8, E8M0 scales (M, K/32) uint8): the
    fused grouped-Hadamard + MXFP4 step (also the offline weight quantizer)."""
    if x.dim() != 2:
        raise ValueError("x must be (M, K)")
    M, K = x.shape
    _need(x, "x", torch.bfloat16, (M, K))
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device=x.device)
    svdq_mxfp4_quantize(x.data_ptr(), M, K, hadamard_group, codes.data_ptr(), scales.data_ptr(), stream)
    return codes, scales


class MXFP4Linear:
    """The FP-Quant MXFP4 linear on the current CUDA device: y = alpha * Q(x R^T) Q(W')^T
    with qweight (N, K/2) and wscales (N, K/32) E8M0 bytes of the rotated weight."""

    def __init__(self, qweight, wscales, alpha: float = 1.0, hadamard_group: int = 32, stream=None):
        N, K2 = qweight.shape
        K = 2 * K2
        _need(qweight, "qweight", qweight.dtype, (N, K // 2))
        _need(wscales, "wscales", wscales.dtype, (N, K // 32))
        if qweight.dtype not in (torch.int8, torch.uint8) or wscales.dtype != torch.uint8:
            raise TypeError("qweight int8/uint8, wscales uint8 (E8M0 bytes)")
        self.K, self.N, self.group = K, N, hadamard_group
        d = svdq_mxfp4_desc(K=K, N=N, hadamard_group=hadamard_group, qweight=qweight.data_ptr(),
                            wscales=wscales.data_ptr(), alpha=float(alpha))
        self.handle = svdq_mxfp4_create(d, stream)
        self._ws = None

    def workspace(self, M: int) -> torch.Tensor:
        nbytes = svdq_mxfp4_workspace_bytes(self.handle, M)
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
        return self._ws

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        M = x.shape[0]
        _need(x, "x", torch.bfloat16, (M, self.K))
        y = torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(y, "y", torch.bfloat16, (M, self.N))
        svdq_mxfp4_forward(self.handle, x.data_ptr(), M, y.data_ptr(), self.workspace(M).data_ptr(), stream)
        return y

    __call__ = forward

    def device_status(self) -> int:
        return svdq_mxfp4_device_status(self.handle)

    def close(self) -> None:
        if getattr(self, "handle", None):
            svdq_mxfp4_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def svdq_fp4_mma_loop(iters: int, stream=None) -> int:
    """Launch the FP4 tensor-rate loop (one CTA per SM); returns the CTA count."""
    ctas = ctypes.c_int(0)
    _check(load_library().svdq_fp4_mma_loop(iters, ctypes.byref(ctas), _stream(stream)), "svdq_fp4_mma_loop")
    return ctas.value


def svdq_fp4_mma_loop_status() -> int:
    flags = ctypes.c_int(0)
    st = load_library().svdq_fp4_mma_loop_status(ctypes.byref(flags))
    if st not in (0, 6):
        raise SvdqError(st, "svdq_fp4_mma_loop_status")
    return flags.value


def svdq_device_status(handle) -> int:
    flags = ctypes.c_int(0)
    st = load_library().svdq_device_status(handle, ctypes.byref(flags))
    if st not in (0, 6):
        raise SvdqError(st, "svdq_device_status")
    return flags.value


# ----------------------------------------------------------------- torch convenience

def _need(t: torch.Tensor, name: str, dtype, shape) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: must be a contiguous CUDA tensor")


def quantize_weight(w: torch.Tensor, rotate_block: int = 0, stream=None):
    """Dense bf16 W (N, K) on the GPU -> (qweight (N, K/2) uint8, wscales (K/16, N) uint8),
    the checkpoint's weight tensors (optional 128-block row rotation)."""
    if w.dim() != 2:
        raise ValueError("w must be (N, K)")
    N, K = w.shape
    _need(w, "w", torch.bfloat16, (N, K))
    qweight = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    wscales = torch.empty((K // 16, N), dtype=torch.uint8, device=w.device)
    svdq_quantize_weight(w.data_ptr(), N, K, rotate_block, qweight.data_ptr(), wscales.data_ptr(), stream)
    return qweight, wscales


class SVDQLinear:
    """One quantized linear layer on the current CUDA device.

    Tensors follow the checkpoint contract of "SVDQuant W4A4" (vLLM-Omni
    svdquant.md, section "Checkpoint contract"): qweight (N, K/2) int8/uint8,
    wscales (K/16, N) float8_e4m3fn (or its uint8 bits), proj_down (K, R),
    proj_up (N, R), smooth_factor (K,), wcscales (N,), wtscale (1,) bf16.
    """

    def __init__(self, qweight, wscales, proj_down, proj_up, smooth_factor, wcscales=None, wtscale=None,
                 rotate_block: int = 0, stream=None):
        N, K2 = qweight.shape
        K = 2 * K2
        R = proj_down.shape[1]
        if qweight.dtype not in (torch.int8, torch.uint8):
            raise TypeError("qweight must be int8/uint8")
        if wscales.dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise TypeError("wscales must be float8_e4m3fn or uint8 bits")
        _need(qweight, "qweight", qweight.dtype, (N, K // 2))
        _need(wscales, "wscales", wscales.dtype, (K // 16, N))
        _need(proj_down, "proj_down", torch.bfloat16, (K, R))
        _need(proj_up, "proj_up", torch.bfloat16, (N, R))
        _need(smooth_factor, "smooth_factor", torch.bfloat16, (K,))
        if wcscales is not None:
            _need(wcscales, "wcscales", torch.bfloat16, (N,))
        if wtscale is not None:
            _need(wtscale, "wtscale", torch.bfloat16, (1,))
        self.K, self.N, self.R, self.rotate_block = K, N, R, rotate_block
        d = svdq_linear_desc(
            K=K, N=N, R=R, rotate_block=rotate_block, act_unsigned=0,
            qweight=qweight.data_ptr(), wscales=wscales.data_ptr(), proj_down=proj_down.data_ptr(),
            proj_up=proj_up.data_ptr(), smooth_factor=smooth_factor.data_ptr(),
            wcscales=None if wcscales is None else wcscales.data_ptr(),
            wtscale=None if wtscale is None else wtscale.data_ptr())
        self.handle = svdq_linear_create(d, stream)
        self._ws = None

    def workspace(self, M: int) -> torch.Tensor:
        nbytes = svdq_workspace_bytes(self.handle, M)
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
        return self._ws

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        M = x.shape[0]
        _need(x, "x", torch.bfloat16, (M, self.K))
        y = torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(y, "y", torch.bfloat16, (M, self.N))
        ws = self.workspace(M)
        svdq_linear_forward(self.handle, x.data_ptr(), M, y.data_ptr(), ws.data_ptr(), stream)
        return y

    __call__ = forward

    def quantize_act(self, x: torch.Tensor, with_lowrank: bool = True, stream=None):
        M = x.shape[0]
        _need(x, "x", torch.bfloat16, (M, self.K))
        codes = torch.empty((M, self.K // 2), dtype=torch.uint8, device=x.device)
        scales = torch.empty((M, self.K // 16), dtype=torch.uint8, device=x.device)
        lowrank = torch.empty((M, self.R), dtype=torch.bfloat16, device=x.device) if with_lowrank else None
        svdq_quantize_act(self.handle, x.data_ptr(), M, codes.data_ptr(), scales.data_ptr(),
                          None if lowrank is None else lowrank.data_ptr(), stream)
        return codes, scales, lowrank

    def device_status(self) -> int:
        return svdq_device_status(self.handle)

    def gemm_kernel(self, M: int) -> str:
        """Name of the kernel the GEMM stage launches for M rows."""
        return svdq_linear_gemm_kernel(self.handle, M)

    def close(self) -> None:
        if getattr(self, "handle", None):
            svdq_linear_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
