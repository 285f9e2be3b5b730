"""Python binding of libgq (include/gq.h): argument marshalling only.

Every function below passes device pointers, sizes and the current CUDA stream
to the C entry point of the same name and raises ``GQError`` on a non-OK
status.  All arithmetic happens in the CUDA kernels of libgq.so; there is no
Python or CPU fallback, and importing this package fails if the library has
not been built (``python bit_gemv_q4_b200/build.py``).

PyTorch is used only to allocate device memory and to name the stream.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgq.so")

GQ_OK = 0
GQ_F32, GQ_F16, GQ_BF16 = 0, 1, 2
GQ_FMT_Q4_0, GQ_FMT_KSB = 0, 1
GQ_DEV_NONFINITE, GQ_DEV_RANGE, GQ_DEV_TIMEOUT = 1, 2, 4
GQ_GEMV_PDL = 1
GQ_QUANT_REF_RULE = 1

# every symbol include/gq.h declares
EXPORTS = (
    "gq_abi_version", "gq_status_string", "gq_status_from_dev",
    "gq_q4_0_bytes", "gq_ksb_bytes",
    "gq_quantize_q4_0", "gq_quantize_q4_0_ex", "gq_quantize_ksb",
    "gq_dequantize_q4_0", "gq_dequantize_ksb",
    "gq_gemv_workspace_bytes", "gq_gemv_q4_0", "gq_gemv_ksb",
    "gq_gemv_q4_0_grouped", "gq_gemv_ksb_grouped",
    "gq_gemm_workspace_bytes", "gq_gemm_q4_0", "gq_gemm_ksb",
    "gq_selftest_gemv_timeout", "gq_gemv_q4_0_noalloc", "gq_stream_read",
    "gq_tiled_bytes", "gq_repack_q4_0", "gq_repack_ksb", "gq_gemv_q4_0_tiled", "gq_gemv_ksb_tiled",
    "gq_gemv_q4_0_tiled_grouped", "gq_gemv_ksb_tiled_grouped",
)

_DTYPE_CODE = {torch.float32: GQ_F32, torch.float16: GQ_F16, torch.bfloat16: GQ_BF16}


class GQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {gq_status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libgq.so not found at {LIB_PATH}; build it with `python bit_gemv_q4_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    i64, vp, c_int, c_uint = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    L.gq_abi_version.restype = c_int
    L.gq_status_string.argtypes = [c_int]
    L.gq_status_string.restype = ctypes.c_char_p
    L.gq_status_from_dev.argtypes = [c_int]
    L.gq_status_from_dev.restype = c_int
    L.gq_q4_0_bytes.argtypes = [i64]
    L.gq_q4_0_bytes.restype = ctypes.c_size_t
    L.gq_ksb_bytes.argtypes = [i64]
    L.gq_ksb_bytes.restype = ctypes.c_size_t
    for name in ("gq_quantize_q4_0", "gq_quantize_ksb"):
        f = getattr(L, name)
        f.argtypes = [vp, i64, vp, vp, vp]
        f.restype = c_int
    L.gq_quantize_q4_0_ex.argtypes = [vp, i64, vp, ctypes.c_uint, vp, vp]
    L.gq_quantize_q4_0_ex.restype = c_int
    for name in ("gq_dequantize_q4_0", "gq_dequantize_ksb"):
        f = getattr(L, name)
        f.argtypes = [vp, i64, vp, vp]
        f.restype = c_int
    L.gq_gemv_workspace_bytes.argtypes = [c_int, i64, i64, i64, c_int]
    L.gq_gemv_workspace_bytes.restype = ctypes.c_size_t
    for name in ("gq_gemv_q4_0", "gq_gemv_ksb"):
        f = getattr(L, name)
        f.argtypes = [vp, i64, i64, vp, c_int, i64, vp, c_int, vp, ctypes.c_size_t, c_uint, vp,
                      vp]
        f.restype = c_int
    for name in ("gq_gemv_q4_0_grouped", "gq_gemv_ksb_grouped"):
        f = getattr(L, name)
        f.argtypes = [vp, c_int, i64, vp, c_int, i64, c_int, c_uint, vp, vp]
        f.restype = c_int
    L.gq_gemm_workspace_bytes.argtypes = [c_int, i64, i64, i64]
    L.gq_gemm_workspace_bytes.restype = ctypes.c_size_t
    for name in ("gq_gemm_q4_0", "gq_gemm_ksb"):
        f = getattr(L, name)
        f.argtypes = [vp, i64, i64, vp, c_int, i64, vp, c_int, vp, ctypes.c_size_t, vp, vp]
        f.restype = c_int
    L.gq_gemv_q4_0_noalloc.argtypes = [vp, i64, i64, vp, vp, c_int, c_uint, vp, vp]
    L.gq_gemv_q4_0_noalloc.restype = c_int
    L.gq_selftest_gemv_timeout.argtypes = [vp, i64, i64, vp, vp, vp, vp]
    L.gq_selftest_gemv_timeout.restype = c_int
    L.gq_stream_read.argtypes = [vp, ctypes.c_size_t, vp, vp]
    L.gq_stream_read.restype = c_int
    L.gq_tiled_bytes.argtypes = [c_int, i64, i64]
    L.gq_tiled_bytes.restype = ctypes.c_size_t
    for name in ("gq_repack_q4_0", "gq_repack_ksb"):
        f = getattr(L, name)
        f.argtypes = [vp, i64, i64, vp, vp]
        f.restype = c_int
    for name in ("gq_gemv_q4_0_tiled", "gq_gemv_ksb_tiled"):
        f = getattr(L, name)
        f.argtypes = [vp, i64, i64, vp, c_int, vp, c_int, c_uint, vp, vp]
        f.restype = c_int
    for name in ("gq_gemv_q4_0_tiled_grouped", "gq_gemv_ksb_tiled_grouped"):
        f = getattr(L, name)
        f.argtypes = [vp, c_int, i64, vp, c_int, c_int, c_uint, vp, vp]
        f.restype = c_int
    return L


lib = _load()


def gq_abi_version() -> int:
    return int(lib.gq_abi_version())


def gq_status_string(status: int) -> str:
    return lib.gq_status_string(int(status)).decode()


def gq_status_from_dev(flags: int) -> int:
    return int(lib.gq_status_from_dev(int(flags)))


def gq_q4_0_bytes(n: int) -> int:
    return int(lib.gq_q4_0_bytes(int(n)))


def gq_ksb_bytes(n: int) -> int:
    return int(lib.gq_ksb_bytes(int(n)))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libgq must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libgq must be contiguous")
    return t.data_ptr() or None


def _check(status: int, where: str) -> None:
    if status != GQ_OK:
        raise GQError(status, where)


def _quantize(name: str, nbytes, x: torch.Tensor, out, dev_status, stream):
    if x.dtype != torch.float32:
        raise TypeError("quantizer input must be float32")
    n = x.numel()
    if out is None:
        out = torch.empty(max(nbytes(n), 0), dtype=torch.uint8, device=x.device)
    _check(getattr(lib, name)(_ptr(x), n, _ptr(out), _ptr(dev_status), _stream(stream)), name)
    return out


def gq_quantize_q4_0(x: torch.Tensor, out: torch.Tensor | None = None,
                     dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 values (numel % 32 == 0) -> uint8 Q4_0 blocks (18 bytes per 32)."""
    return _quantize("gq_quantize_q4_0", gq_q4_0_bytes, x, out, dev_status, stream)


def gq_quantize_q4_0_ex(x: torch.Tensor, flags: int, out: torch.Tensor | None = None,
                        dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """gq_quantize_q4_0 with a rule flag (0, or GQ_QUANT_REF_RULE for the page's
    reference quantizer: d = signed max / -8, codes min(15, trunc(x/d + 8.5)))."""
    if x.dtype != torch.float32:
        raise TypeError("quantizer input must be float32")
    n = x.numel()
    if out is None:
        out = torch.empty(max(gq_q4_0_bytes(n), 0), dtype=torch.uint8, device=x.device)
    _check(lib.gq_quantize_q4_0_ex(_ptr(x), n, _ptr(out), int(flags), _ptr(dev_status),
                                   _stream(stream)), "gq_quantize_q4_0_ex")
    return out


def gq_quantize_ksb(x: torch.Tensor, out: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 values (numel % 256 == 0) -> uint8 super-blocks (138 bytes per 256)."""
    return _quantize("gq_quantize_ksb", gq_ksb_bytes, x, out, dev_status, stream)


def _dequantize(name: str, q: torch.Tensor, n: int, out, stream):
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=q.device)
    _check(getattr(lib, name)(_ptr(q), int(n), _ptr(out), _stream(stream)), name)
    return out


def gq_dequantize_q4_0(q: torch.Tensor, n: int, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    return _dequantize("gq_dequantize_q4_0", q, n, out, stream)


def gq_dequantize_ksb(q: torch.Tensor, n: int, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    return _dequantize("gq_dequantize_ksb", q, n, out, stream)


def gq_gemv_workspace_bytes(fmt: int, M: int, K: int, B: int, x_dtype) -> int:
    code = _DTYPE_CODE[x_dtype] if isinstance(x_dtype, torch.dtype) else int(x_dtype)
    return int(lib.gq_gemv_workspace_bytes(int(fmt), int(M), int(K), int(B), code))


# Zeroed GEMV workspaces, one per (device, stream): calls on one stream run in
# order, and each successful call leaves the workspace ready for the next.
_gemv_ws: dict = {}


def _gemv_workspace(need: int, device: torch.device, stream) -> torch.Tensor:
    key = (device.index, _stream(stream))
    ws = _gemv_ws.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _gemv_ws[key] = ws
    return ws


def _gemv(name: str, fmt: int, W: torch.Tensor, M: int, K: int, x: torch.Tensor, y_dtype, out,
          workspace, flags: int, dev_status, stream):
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    B = x2.shape[0]
    if x2.shape[1] != K:
        raise ValueError(f"x has {x2.shape[1]} columns, expected K={K}")
    if x2.dtype not in _DTYPE_CODE or y_dtype not in _DTYPE_CODE:
        raise TypeError("activations and outputs must be float32, float16 or bfloat16")
    if out is None:
        out = torch.empty((B, M), dtype=y_dtype, device=x2.device)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a uint8 CUDA tensor")
        need = gq_gemv_workspace_bytes(fmt, M, K, B, x2.dtype)
        workspace = _gemv_workspace(need, x2.device, stream) if need else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(getattr(lib, name)(_ptr(W), int(M), int(K), _ptr(x2), _DTYPE_CODE[x2.dtype], B,
                              _ptr(out), _DTYPE_CODE[out.dtype], _ptr(workspace), ws_bytes,
                              int(flags), _ptr(dev_status), _stream(stream)), name)
    return out


def gq_gemv_q4_0(W: torch.Tensor, M: int, K: int, x: torch.Tensor, y_dtype=torch.float16,
                 out: torch.Tensor | None = None, flags: int = 0,
                 dev_status: torch.Tensor | None = None, stream=None,
                 workspace=None) -> torch.Tensor:
    """y[B, M] = W_hat[M, K] @ x[B, K]^T for Q4_0 weights; B in 1..8.

    workspace: None (the default path), "auto" (a zeroed scratch buffer cached
    per device and stream) or a uint8 CUDA tensor of at least
    gq_gemv_workspace_bytes(...) bytes, zero before its first use; with a
    workspace, batch-1 fp16 calls take the integer tensor-core path."""
    return _gemv("gq_gemv_q4_0", GQ_FMT_Q4_0, W, M, K, x, y_dtype, out, workspace, flags,
                 dev_status, stream)


def gq_gemv_ksb(W: torch.Tensor, M: int, K: int, x: torch.Tensor, y_dtype=torch.float16,
                out: torch.Tensor | None = None, flags: int = 0,
                dev_status: torch.Tensor | None = None, stream=None,
                workspace=None) -> torch.Tensor:
    """y[B, M] = W_hat[M, K] @ x[B, K]^T for super-block weights; B in 1..8."""
    return _gemv("gq_gemv_ksb", GQ_FMT_KSB, W, M, K, x, y_dtype, out, workspace, flags,
                 dev_status, stream)


class GemvDesc(ctypes.Structure):
    """gq_gemv_desc: one matrix of a grouped GEMV."""
    _fields_ = [("W", ctypes.c_void_p), ("M", ctypes.c_int64), ("y", ctypes.c_void_p)]


def _gemv_grouped(name: str, Ws, Ms, K: int, x: torch.Tensor, y_dtype, outs, flags: int,
                  dev_status, stream):
    if len(Ws) != len(Ms):
        raise ValueError("one M per matrix")
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    B = x2.shape[0]
    if x2.shape[1] != K:
        raise ValueError(f"x has {x2.shape[1]} columns, expected K={K}")
    if x2.dtype not in _DTYPE_CODE or y_dtype not in _DTYPE_CODE:
        raise TypeError("activations and outputs must be float32, float16 or bfloat16")
    if outs is None:
        outs = [torch.empty((B, int(M)), dtype=y_dtype, device=x2.device) for M in Ms]
    if len(outs) != len(Ws) or any(o.dtype != outs[0].dtype for o in outs):
        raise ValueError("one output per matrix, all of one dtype")
    descs = (GemvDesc * len(Ws))(*[GemvDesc(_ptr(W), int(M), _ptr(o))
                                   for W, M, o in zip(Ws, Ms, outs)])
    ytype = _DTYPE_CODE[outs[0].dtype] if outs else _DTYPE_CODE[y_dtype]
    _check(getattr(lib, name)(ctypes.cast(descs, ctypes.c_void_p), len(Ws), int(K), _ptr(x2),
                              _DTYPE_CODE[x2.dtype], B, ytype,
                              int(flags), _ptr(dev_status), _stream(stream)), name)
    return outs


def gq_gemv_q4_0_grouped(Ws, Ms, K: int, x: torch.Tensor, y_dtype=torch.float16, outs=None,
                         flags: int = 0, dev_status: torch.Tensor | None = None, stream=None):
    """[y_i = W_hat_i @ x^T for each Q4_0 matrix W_i (M_i x K)], one shared x [B, K]."""
    return _gemv_grouped("gq_gemv_q4_0_grouped", Ws, Ms, K, x, y_dtype, outs, flags,
                         dev_status, stream)


def gq_gemv_ksb_grouped(Ws, Ms, K: int, x: torch.Tensor, y_dtype=torch.float16, outs=None,
                        flags: int = 0, dev_status: torch.Tensor | None = None, stream=None):
    """[y_i = W_hat_i @ x^T for each super-block matrix W_i (M_i x K)], one shared x."""
    return _gemv_grouped("gq_gemv_ksb_grouped", Ws, Ms, K, x, y_dtype, outs, flags,
                         dev_status, stream)


def gq_gemm_workspace_bytes(fmt: int, M: int, K: int, B: int) -> int:
    return int(lib.gq_gemm_workspace_bytes(int(fmt), int(M), int(K), int(B)))


def _gemm(name: str, fmt: int, W: torch.Tensor, M: int, K: int, X: torch.Tensor, y_dtype, out,
          workspace, dev_status, stream):
    X2 = X if X.dim() == 2 else X.reshape(1, -1)
    B = X2.shape[0]
    if X2.shape[1] != K:
        raise ValueError(f"X has {X2.shape[1]} columns, expected K={K}")
    if X2.dtype not in _DTYPE_CODE or y_dtype not in _DTYPE_CODE:
        raise TypeError("X must be bfloat16; Y float32, float16 or bfloat16")
    if out is None:
        out = torch.empty((B, M), dtype=y_dtype, device=X2.device)
    need = gq_gemm_workspace_bytes(fmt, M, K, B)
    if workspace is None and need > 0:
        workspace = torch.zeros(need, dtype=torch.uint8, device=X2.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(getattr(lib, name)(_ptr(W), int(M), int(K), _ptr(X2), _DTYPE_CODE[X2.dtype], B,
                              _ptr(out), _DTYPE_CODE[out.dtype], _ptr(workspace), ws_bytes,
                              _ptr(dev_status), _stream(stream)), name)
    return out


def gq_gemm_q4_0(W: torch.Tensor, M: int, K: int, X: torch.Tensor, y_dtype=torch.float32,
                 out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                 dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y[B, M] = W_hat[M, K] @ X[B, K]^T on the tensor cores (X bfloat16, B <= 256)."""
    return _gemm("gq_gemm_q4_0", GQ_FMT_Q4_0, W, M, K, X, y_dtype, out, workspace, dev_status,
                 stream)


def gq_gemm_ksb(W: torch.Tensor, M: int, K: int, X: torch.Tensor, y_dtype=torch.float32,
                out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y[B, M] = W_hat[M, K] @ X[B, K]^T for super-block weights on the tensor cores."""
    return _gemm("gq_gemm_ksb", GQ_FMT_KSB, W, M, K, X, y_dtype, out, workspace, dev_status,
                 stream)


def gq_gemv_q4_0_noalloc(W: torch.Tensor, M: int, K: int, x: torch.Tensor, y_dtype=torch.float16,
                         out: torch.Tensor | None = None, flags: int = 0,
                         dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Batch-1 Q4_0 GEMV (fp16 x) on the library's static scratch."""
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    if x2.shape != (1, K) or x2.dtype != torch.float16:
        raise ValueError("x must be one fp16 vector of length K")
    if out is None:
        out = torch.empty((1, M), dtype=y_dtype, device=x2.device)
    _check(lib.gq_gemv_q4_0_noalloc(_ptr(W), int(M), int(K), _ptr(x2), _ptr(out),
                                    _DTYPE_CODE[out.dtype], int(flags), _ptr(dev_status),
                                    _stream(stream)), "gq_gemv_q4_0_noalloc")
    return out


def gq_selftest_gemv_timeout(W: torch.Tensor, M: int, K: int, x: torch.Tensor, y: torch.Tensor,
                             dev_status: torch.Tensor, stream=None) -> None:
    """Run the GEMV with a first stage that never fills; the bounded wait must
    report GQ_DEV_TIMEOUT in dev_status (see include/gq.h)."""
    _check(lib.gq_selftest_gemv_timeout(_ptr(W), int(M), int(K), _ptr(x), _ptr(y),
                                        _ptr(dev_status), _stream(stream)),
           "gq_selftest_gemv_timeout")


def gq_stream_read(buf: torch.Tensor, sink: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """Read every byte of `buf` once on the GPU and XOR its 32-bit words into
    `sink` (an int32 tensor of one element, zeroed here when not given): the
    practical read ceiling of one launch of that size."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
    nbytes = buf.numel() * buf.element_size()
    _check(lib.gq_stream_read(_ptr(buf), nbytes, _ptr(sink), _stream(stream)), "gq_stream_read")
    return sink


def gq_tiled_bytes(fmt: int, M: int, K: int) -> int:
    """Bytes of the tiled storage of an M x K matrix (0 for unsupported K)."""
    return int(lib.gq_tiled_bytes(int(fmt), int(M), int(K)))


def gq_repack(fmt: int, W: torch.Tensor, M: int, K: int, out: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """Canonical packed rows (uint8 CUDA tensor) -> tiled storage (uint8)."""
    n = gq_tiled_bytes(fmt, M, K)
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=W.device)
    name = "gq_repack_q4_0" if fmt == GQ_FMT_Q4_0 else "gq_repack_ksb"
    _check(getattr(lib, name)(_ptr(W), int(M), int(K), _ptr(out), _stream(stream)), name)
    return out


def _gemv_tiled(name: str, T: torch.Tensor, M: int, K: int, x: torch.Tensor, y_dtype, out,
                flags: int, dev_status, stream):
    x1 = x.reshape(-1)
    if x1.numel() != K:
        raise ValueError(f"x has {x1.numel()} values, expected K={K}")
    if x1.dtype not in _DTYPE_CODE or y_dtype not in _DTYPE_CODE:
        raise TypeError("activations and outputs must be float32, float16 or bfloat16")
    if out is None:
        out = torch.empty((1, M), dtype=y_dtype, device=x1.device)
    _check(getattr(lib, name)(_ptr(T), int(M), int(K), _ptr(x1), _DTYPE_CODE[x1.dtype],
                              _ptr(out), _DTYPE_CODE[out.dtype], int(flags), _ptr(dev_status),
                              _stream(stream)), name)
    return out


def gq_gemv_q4_0_tiled(T: torch.Tensor, M: int, K: int, x: torch.Tensor, y_dtype=torch.float16,
                       out: torch.Tensor | None = None, flags: int = 0,
                       dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[1, M] = W_hat @ x for Q4_0 weights in tiled storage (x: K fp16 values)."""
    return _gemv_tiled("gq_gemv_q4_0_tiled", T, M, K, x, y_dtype, out, flags, dev_status, stream)


def gq_gemv_ksb_tiled(T: torch.Tensor, M: int, K: int, x: torch.Tensor, y_dtype=torch.float16,
                      out: torch.Tensor | None = None, flags: int = 0,
                      dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[1, M] = W_hat @ x for super-block weights in tiled storage."""
    return _gemv_tiled("gq_gemv_ksb_tiled", T, M, K, x, y_dtype, out, flags, dev_status, stream)


def _gemv_tiled_grouped(name: str, Ts, Ms, K: int, x: torch.Tensor, y_dtype, outs, flags: int,
                        dev_status, stream):
    if len(Ts) != len(Ms):
        raise ValueError("one M per matrix")
    x1 = x.reshape(-1)
    if x1.numel() != K:
        raise ValueError(f"x has {x1.numel()} values, expected K={K}")
    if x1.dtype not in _DTYPE_CODE or y_dtype not in _DTYPE_CODE:
        raise TypeError("activations and outputs must be float32, float16 or bfloat16")
    if outs is None:
        outs = [torch.empty((1, int(M)), dtype=y_dtype, device=x1.device) for M in Ms]
    if len(outs) != len(Ts) or any(o.dtype != outs[0].dtype for o in outs):
        raise ValueError("one output per matrix, all of one dtype")
    descs = (GemvDesc * len(Ts))(*[GemvDesc(_ptr(T), int(M), _ptr(o))
                                   for T, M, o in zip(Ts, Ms, outs)])
    ytype = _DTYPE_CODE[outs[0].dtype] if outs else _DTYPE_CODE[y_dtype]
    _check(getattr(lib, name)(ctypes.cast(descs, ctypes.c_void_p), len(Ts), int(K), _ptr(x1),
                              _DTYPE_CODE[x1.dtype], ytype, int(flags), _ptr(dev_status),
                              _stream(stream)), name)
    return outs


def gq_gemv_q4_0_tiled_grouped(Ts, Ms, K: int, x: torch.Tensor, y_dtype=torch.float16,
                               outs=None, flags: int = 0, dev_status: torch.Tensor | None = None,
                               stream=None):
    """[y_i = W_hat_i @ x for each Q4_0 matrix in tiled storage T_i (M_i x K)], one fp16 x."""
    return _gemv_tiled_grouped("gq_gemv_q4_0_tiled_grouped", Ts, Ms, K, x, y_dtype, outs, flags,
                               dev_status, stream)


def gq_gemv_ksb_tiled_grouped(Ts, Ms, K: int, x: torch.Tensor, y_dtype=torch.float16,
                              outs=None, flags: int = 0, dev_status: torch.Tensor | None = None,
                              stream=None):
    """[y_i = W_hat_i @ x for each super-block matrix in tiled storage T_i], one fp16 x."""
    return _gemv_tiled_grouped("gq_gemv_ksb_tiled_grouped", Ts, Ms, K, x, y_dtype, outs, flags,
                               dev_status, stream)
