"""Python binding of libw4a16.so, the B200 W4A16 group-128 linear layer.

Marshalling only: every function below checks tensor metadata, passes raw
device pointers and the current CUDA stream to the C ABI declared in
``include/w4a16.h`` and turns a non-zero status into ``W4A16Error``.  All
arithmetic runs in the library's CUDA kernels; there is no fallback, and
importing this package fails loudly when the shared library has not been
built (``python decode_w4a16_g128_b200/build.py``).

Tensors: ``x`` bf16 [M, K]; ``wq`` int32/uint32 [N, K/8] (eight 4-bit codes
per word, low nibble first); ``scales``/``biases`` bf16 [N, K/128]; the result
``y`` is bf16 [M, N].  All on the same CUDA device, contiguous.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libw4a16.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_MISALIGNED = 3
ERR_CUDA = 4
ERR_NO_MEMORY = 5
ERR_DEVICE = 6
ERR_TIMEOUT = 7

PATH_AUTO = 0
PATH_MATVEC = 1
PATH_GEMM = 2
PATH_MATVEC_ROWS = 3

DTYPE_F32 = 0
DTYPE_BF16 = 1

FLAG_NO_PDL = 1
FLAG_STATIC_WEIGHTS = 2
FLAG_TEST_DROP_COPY = 4


class W4A16Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Options(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("splits", ctypes.c_int32), ("workers", ctypes.c_int32),
                ("sm_count", ctypes.c_int32), ("flags", ctypes.c_int32), ("row_blocks", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("splits", ctypes.c_int32), ("grid_x", ctypes.c_int32),
                ("grid_y", ctypes.c_int32), ("grid_z", ctypes.c_int32), ("block", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("cluster", ctypes.c_int32), ("tiles", ctypes.c_int64),
                ("units", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64), ("row_blocks", ctypes.c_int32),
                ("slices", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIBRARY_PATH):
        raise ImportError(f"{LIBRARY_PATH} is missing: build it with "
                          "`python decode_w4a16_g128_b200/build.py` (needs nvcc)")
    lib = ctypes.CDLL(LIBRARY_PATH)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.w4a16_matmul.argtypes = [p, p, p, p, p, i64, i64, i64, p]
    lib.w4a16_matmul_ex.argtypes = [p, p, p, p, p, i64, i64, i64, p, ctypes.POINTER(Options)]
    lib.w4a16_matmul_last_rows.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p]
    lib.w4a16_plan.argtypes = [i64, i64, i64, ctypes.POINTER(Options), ctypes.POINTER(PlanInfo)]
    lib.w4a16_device_status.argtypes = [p]
    lib.w4a16_release.argtypes = []
    lib.w4a16_release.restype = None
    lib.w4a16_status_string.argtypes = [i32]
    lib.w4a16_status_string.restype = ctypes.c_char_p
    lib.w4a16_last_cuda_error.argtypes = []
    lib.w4a16_version.argtypes = []
    lib.w4a16_streamk_owner.argtypes = [i64, i64, i64]
    lib.w4a16_streamk_owner.restype = i64
    lib.w4a16_matvec_noalloc.argtypes = [p, p, p, p, p, i64, i64, i64, p]
    lib.w4a16_quantize.argtypes = [p, ctypes.c_int32, p, p, p, i64, i64, p]
    lib.w4a16_gate_up.argtypes = [p, p, p, p, p, i64, i64, i64, p]
    lib.w4a16_matmul_bits.argtypes = [p, p, p, p, p, i64, i64, i64, ctypes.c_int32, p]
    for name in ("w4a16_matmul", "w4a16_matmul_ex", "w4a16_matmul_last_rows", "w4a16_plan",
                 "w4a16_device_status", "w4a16_last_cuda_error", "w4a16_version", "w4a16_matvec_noalloc",
                 "w4a16_quantize", "w4a16_gate_up", "w4a16_matmul_bits"):
        getattr(lib, name).restype = i32
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.w4a16_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise W4A16Error(status, where)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check_tensors(x, wq, scales, biases, y):
    import torch
    if x.dtype != torch.bfloat16 or scales.dtype != torch.bfloat16 or biases.dtype != torch.bfloat16:
        raise TypeError("x, scales and biases must be bfloat16")
    if wq.dtype not in (torch.int32, torch.uint32):
        raise TypeError("wq must be int32 or uint32 (packed codes)")
    for name, t in (("x", x), ("wq", wq), ("scales", scales), ("biases", biases)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    M, K = x.shape
    N = wq.shape[0]
    if tuple(wq.shape) != (N, K // 8) or tuple(scales.shape) != (N, K // 128) or \
            tuple(biases.shape) != (N, K // 128):
        raise ValueError(f"shape mismatch: x {tuple(x.shape)}, wq {tuple(wq.shape)}, "
                         f"scales {tuple(scales.shape)}, biases {tuple(biases.shape)}")
    if y is not None and (y.dtype != torch.bfloat16 or not y.is_cuda or not y.is_contiguous()):
        raise ValueError("y must be a contiguous bfloat16 CUDA tensor")
    return M, N, K


def w4a16_matmul(x, wq, scales, biases, y=None, stream=None):
    """y = x . dequant(wq)^T on the current (or given) CUDA stream; returns y."""
    import torch
    M, N, K = _check_tensors(x, wq, scales, biases, y)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif tuple(y.shape) != (M, N):
        raise ValueError("y must be [M, N]")
    _check(lib.w4a16_matmul(_ptr(x), _ptr(wq), _ptr(scales), _ptr(biases), _ptr(y), M, N, K,
                            _stream_handle(stream)), "w4a16_matmul")
    return y


def make_options(path=PATH_AUTO, splits=0, workers=0, sm_count=0, flags=0, row_blocks=0) -> Options:
    return Options(int(path), int(splits), int(workers), int(sm_count), int(flags), int(row_blocks))


def w4a16_matmul_ex(x, wq, scales, biases, y=None, stream=None, path=PATH_AUTO, splits=0, workers=0,
                    flags=0, row_blocks=0):
    """w4a16_matmul with a forced path / split count / worker count / row blocks per CTA."""
    import torch
    M, N, K = _check_tensors(x, wq, scales, biases, y)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif tuple(y.shape) != (M, N):
        raise ValueError("y must be [M, N]")
    opt = make_options(path, splits, workers, 0, flags, row_blocks)
    _check(lib.w4a16_matmul_ex(_ptr(x), _ptr(wq), _ptr(scales), _ptr(biases), _ptr(y), M, N, K,
                               _stream_handle(stream), ctypes.byref(opt)), "w4a16_matmul_ex")
    return y


def w4a16_matmul_last_rows(x, wq, scales, biases, keep: int, y=None, stream=None):
    """Project only the last ``keep`` rows of x (0 = every row); returns y [keep, N]."""
    import torch
    M, N, K = _check_tensors(x, wq, scales, biases, None)
    rows = M if keep == 0 else keep
    if y is None:
        y = torch.empty((rows, N), dtype=torch.bfloat16, device=x.device)
    elif tuple(y.shape) != (rows, N):
        raise ValueError("y must be [keep, N]")
    _check(lib.w4a16_matmul_last_rows(_ptr(x), _ptr(wq), _ptr(scales), _ptr(biases), _ptr(y), M,
                                      int(keep), N, K, _stream_handle(stream)),
           "w4a16_matmul_last_rows")
    return y


NOALLOC_MAX_N = 1048576


def w4a16_matvec_noalloc(x, wq, scales, biases, y, stream=None):
    """The matvec (M <= 8) without any allocation, for callers that cannot allocate
    device memory: its split-row scratch is a fixed array inside the library, so
    calls that can overlap on the GPU must be serialised.  y must be given."""
    M, N, K = _check_tensors(x, wq, scales, biases, y)
    if tuple(y.shape) != (M, N):
        raise ValueError("y must be [M, N]")
    _check(lib.w4a16_matvec_noalloc(_ptr(x), _ptr(wq), _ptr(scales), _ptr(biases), _ptr(y), M, N, K,
                                    _stream_handle(stream)), "w4a16_matvec_noalloc")
    return y


def interleave_gate_up(gate, up):
    """Row-interleave a gate and an up tensor [N2, ...] (codes, scales or biases of the two
    layers) in blocks of 8, the weight layout w4a16_gate_up reads (layout only)."""
    import torch
    if gate.shape != up.shape or gate.shape[0] % 8:
        raise ValueError("gate and up need the same shape and a row count divisible by 8")
    n2 = gate.shape[0]
    return torch.stack([gate.reshape(n2 // 8, 8, -1), up.reshape(n2 // 8, 8, -1)], dim=1).reshape(2 * n2, -1)


def w4a16_gate_up(x, wq, scales, biases, h=None, stream=None):
    """Fused gate/up projection, M <= 8: h [M, N2] = bf16(silu(x . gate^T) * (x . up^T)) with the
    two layers' rows interleaved in blocks of 8 in wq, scales and biases (2 N2 rows)."""
    import torch
    M, N, K = _check_tensors(x, wq, scales, biases, h)
    if N % 16:
        raise ValueError("the interleaved gate/up rows come in blocks of 16")
    N2 = N // 2
    if h is None:
        h = torch.empty((M, N2), dtype=torch.bfloat16, device=x.device)
    elif tuple(h.shape) != (M, N2):
        raise ValueError("h must be [M, N2]")
    _check(lib.w4a16_gate_up(_ptr(x), _ptr(wq), _ptr(scales), _ptr(biases), _ptr(h), M, N2, K,
                             _stream_handle(stream)), "w4a16_gate_up")
    return h


def w4a16_matmul_bits(x, wq, scales, biases, bits: int, y=None, stream=None):
    """y = x . dequant(wq)^T with b-bit codes (b = 2, 4 or 8): wq int32/uint32 [N, K b / 32], 32 / b
    codes per word, the lowest code in the lowest bits.  2 and 8 bits: M <= 32."""
    import torch
    if bits not in (2, 4, 8):
        raise W4A16Error(ERR_UNSUPPORTED, "w4a16_matmul_bits")
    if x.dtype != torch.bfloat16 or scales.dtype != torch.bfloat16 or biases.dtype != torch.bfloat16:
        raise TypeError("x, scales and biases must be bfloat16")
    if wq.dtype not in (torch.int32, torch.uint32):
        raise TypeError("wq must be int32 or uint32 (packed codes)")
    for name, t in (("x", x), ("wq", wq), ("scales", scales), ("biases", biases)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    M, K = x.shape
    N = wq.shape[0]
    if tuple(wq.shape) != (N, K * bits // 32) or tuple(scales.shape) != (N, K // 128) or \
            tuple(biases.shape) != (N, K // 128):
        raise ValueError(f"shape mismatch: x {tuple(x.shape)}, wq {tuple(wq.shape)}, "
                         f"scales {tuple(scales.shape)}, biases {tuple(biases.shape)} for {bits}-bit codes")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    elif tuple(y.shape) != (M, N) or y.dtype != torch.bfloat16 or not y.is_cuda or not y.is_contiguous():
        raise ValueError("y must be a contiguous bfloat16 CUDA tensor [M, N]")
    _check(lib.w4a16_matmul_bits(_ptr(x), _ptr(wq), _ptr(scales), _ptr(biases), _ptr(y), M, N, K, int(bits),
                                 _stream_handle(stream)), "w4a16_matmul_bits")
    return y


def w4a16_quantize(w, wq=None, scales=None, biases=None, stream=None):
    """Quantise weights W [N, K] (float32 or bfloat16, CUDA, contiguous) on the GPU into the
    packed format: returns (wq int32 [N, K/8], scales bf16 [N, K/128], biases bf16 [N, K/128])."""
    import torch
    if w.dim() != 2 or not w.is_cuda or not w.is_contiguous():
        raise ValueError("w must be a contiguous 2-D CUDA tensor")
    if w.dtype == torch.float32:
        dt = DTYPE_F32
    elif w.dtype == torch.bfloat16:
        dt = DTYPE_BF16
    else:
        raise TypeError("w must be float32 or bfloat16")
    N, K = w.shape
    if K % 128:
        raise W4A16Error(ERR_UNSUPPORTED, "w4a16_quantize")
    if wq is None:
        wq = torch.empty((N, K // 8), dtype=torch.int32, device=w.device)
    if scales is None:
        scales = torch.empty((N, K // 128), dtype=torch.bfloat16, device=w.device)
    if biases is None:
        biases = torch.empty((N, K // 128), dtype=torch.bfloat16, device=w.device)
    if tuple(wq.shape) != (N, K // 8) or tuple(scales.shape) != (N, K // 128) or tuple(biases.shape) != (N, K // 128):
        raise ValueError("output shapes must be [N, K/8], [N, K/128], [N, K/128]")
    _check(lib.w4a16_quantize(_ptr(w), dt, _ptr(wq), _ptr(scales), _ptr(biases), N, K, _stream_handle(stream)),
           "w4a16_quantize")
    return wq, scales, biases


def w4a16_plan(M: int, N: int, K: int, path=PATH_AUTO, splits=0, workers=0, sm_count=0, row_blocks=0) -> dict:
    opt = make_options(path, splits, workers, sm_count, 0, row_blocks)
    info = PlanInfo()
    _check(lib.w4a16_plan(M, N, K, ctypes.byref(opt), ctypes.byref(info)), "w4a16_plan")
    return {name: getattr(info, name) for name, _ in PlanInfo._fields_ if name != "reserved"}


def w4a16_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return lib.w4a16_device_status(_stream_handle(stream))


def w4a16_release() -> None:
    lib.w4a16_release()


def w4a16_version() -> int:
    return lib.w4a16_version()


def w4a16_streamk_owner(units: int, workers: int, u: int) -> int:
    return lib.w4a16_streamk_owner(units, workers, u)


__all__ = [
    "w4a16_matmul", "w4a16_matmul_ex", "w4a16_matmul_last_rows", "w4a16_plan", "w4a16_device_status",
    "w4a16_release", "w4a16_version", "w4a16_streamk_owner", "w4a16_matvec_noalloc", "w4a16_quantize",
    "w4a16_gate_up", "interleave_gate_up", "w4a16_matmul_bits",
    "status_string", "W4A16Error", "Options",
    "PlanInfo", "make_options", "lib", "LIBRARY_PATH",
]
