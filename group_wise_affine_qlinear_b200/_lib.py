"""ctypes marshalling for libqlinear.so (see include/qlinear.h for the contract)."""
from __future__ import annotations

import ctypes
import os
import threading

import torch

GROUP = 64
PATH_AUTO, PATH_GEMV, PATH_TC_SKINNY, PATH_TC_FUSED = 0, 1, 2, 3
_F32, _BF16 = 0, 1

STATUS = {
    0: "QL_OK",
    1: "QL_ERR_INVALID_ARG",
    2: "QL_ERR_ALIGNMENT",
    3: "QL_ERR_UNSUPPORTED",
    4: "QL_ERR_WORKSPACE",
    5: "QL_ERR_CUDA",
    6: "QL_ERR_DEVICE_TIMEOUT",
    7: "QL_ERR_BOUNDS",
}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libqlinear.so"
_lock = threading.Lock()
_lib = None


class QLinearError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


def library_path() -> str:
    """The in-tree libqlinear.so, or the library QL_LIBRARY names (e.g. the bounds-checked build)."""
    return os.environ.get("QL_LIBRARY") or os.path.join(_HERE, _LIB_NAME)


def lib() -> ctypes.CDLL:
    """Load libqlinear.so (built in-tree by group_wise_affine_qlinear_b200.build)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        _lib = load_library(library_path())
        return _lib


def load_library(path: str) -> ctypes.CDLL:
    """A CDLL of a qlinear library at `path` with every entry point's argument and result types set."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m group_wise_affine_qlinear_b200.build`")
    L = ctypes.CDLL(path)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    L.qlinear_workspace_size.argtypes = [i64, i64, i64, i32]
    L.qlinear_workspace_size.restype = sz
    L.qlinear_workspace_size_config.argtypes = [i64, i64, i64, i32, i32, i32]
    L.qlinear_workspace_size_config.restype = sz
    L.qlinear_forward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp, sz, vp]
    L.qlinear_forward.restype = ctypes.c_int
    L.qlinear_forward_config.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, i64, i64, i64, i32, i32, i32, vp, sz, vp]
    L.qlinear_forward_config.restype = ctypes.c_int
    L.qlinear_dequant.argtypes = [vp, vp, vp, i64, i64, i32, vp, ctypes.c_int, vp]
    L.qlinear_dequant.restype = ctypes.c_int
    L.qlinear_pack.argtypes = [vp, vp, i64, i64, i32, vp, vp, vp, vp]
    L.qlinear_pack.restype = ctypes.c_int
    L.qlinear_get_device_status.argtypes = [vp]
    L.qlinear_get_device_status.restype = ctypes.c_int
    L.qlinear_last_dispatch.argtypes = [ctypes.c_char_p, sz]
    L.qlinear_last_dispatch.restype = ctypes.c_int
    L.qlinear_forward_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp]
    L.qlinear_forward_noalloc.restype = ctypes.c_int
    L.qlinear_set_profile_events.argtypes = [vp, vp]
    L.qlinear_set_profile_events.restype = ctypes.c_int
    L.qlinear_status_string.argtypes = [ctypes.c_int]
    L.qlinear_status_string.restype = ctypes.c_char_p
    L.qlinear_version.argtypes = []
    L.qlinear_version.restype = ctypes.c_int32
    L.qlinear8_workspace_size.argtypes = [i64, i64, i64, i32]
    L.qlinear8_workspace_size.restype = sz
    L.qlinear8_workspace_size_config.argtypes = [i64, i64, i64, i32, i32, i32]
    L.qlinear8_workspace_size_config.restype = sz
    L.qlinear8_forward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp, sz, vp]
    L.qlinear8_forward.restype = ctypes.c_int
    L.qlinear8_forward_config.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, i64, i64, i64, i32, i32, i32, vp, sz,
                                          vp]
    L.qlinear8_forward_config.restype = ctypes.c_int
    L.qlinear8_dequant.argtypes = [vp, vp, vp, i64, i64, i32, vp, ctypes.c_int, vp]
    L.qlinear8_dequant.restype = ctypes.c_int
    L.qlinear8_pack.argtypes = [vp, vp, i64, i64, i32, vp, vp, vp, vp]
    L.qlinear8_pack.restype = ctypes.c_int
    L.qlinear_selftest_bounded_wait.argtypes = [vp]
    L.qlinear_selftest_bounded_wait.restype = ctypes.c_int
    L.qlinear_reduce_partials.argtypes = [vp, i32, i64, vp, ctypes.c_int, vp]
    L.qlinear_reduce_partials.restype = ctypes.c_int
    L.qlinear_swiglu_workspace_size.argtypes = [i64, i64, i64, i32]
    L.qlinear_swiglu_workspace_size.restype = sz
    L.qlinear_swiglu_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, i64, i64, i64, i32, vp, sz, vp]
    L.qlinear_swiglu_forward.restype = ctypes.c_int
    L.qlinear_test_stall.argtypes = [i32, ctypes.c_uint64]
    L.qlinear_test_stall.restype = ctypes.c_int
    L.qlinear_test_ring_depth.argtypes = [i32]
    L.qlinear_test_ring_depth.restype = ctypes.c_int
    L.qlinear_test_delay.argtypes = [i32, ctypes.c_uint64]
    L.qlinear_test_delay.restype = ctypes.c_int
    return L


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status: int, what: str) -> None:
    if status != 0:
        raise QLinearError(status, what)


def _need_cuda(t: torch.Tensor, name: str, dtype, shape=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _weights_shape(codes: torch.Tensor, scales: torch.Tensor, bits: int = 4):
    N, Kw = codes.shape
    K = (32 // bits) * Kw
    return N, K


def workspace_size(M: int, K: int, N: int, path: int = PATH_AUTO, split_k: int = 0, bits: int = 4) -> int:
    fn = lib().qlinear_workspace_size_config if bits == 4 else lib().qlinear8_workspace_size_config
    v = fn(M, K, N, GROUP, path, split_k)
    if v == ctypes.c_size_t(-1).value:
        raise ValueError("shape or path not supported")
    return int(v)


def workspace_size8(M: int, K: int, N: int, path: int = PATH_AUTO, split_k: int = 0) -> int:
    """Workspace bytes of forward8 (qlinear8_workspace_size_config)."""
    return workspace_size(M, K, N, path, split_k, bits=8)


def forward(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
            out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
            path: int = PATH_AUTO, split_k: int = 0, out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """y = x . W^T for the packed W; see include/qlinear.h (qlinear_forward[_config])."""
    return _forward(x, codes, scales, biases, out, workspace, path, split_k, out_dtype, stream, 4)


def forward8(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
             out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
             path: int = PATH_AUTO, split_k: int = 0, out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """forward() for 8-bit codes, int32 [N][K/4] (qlinear8_forward[_config])."""
    return _forward(x, codes, scales, biases, out, workspace, path, split_k, out_dtype, stream, 8)


def _forward(x, codes, scales, biases, out, workspace, path, split_k, out_dtype, stream, bits):
    L = lib()
    N, K = _weights_shape(codes, scales, bits)
    M = x.shape[0]
    _need_cuda(x, "x", torch.bfloat16, (M, K))
    _need_cuda(codes, "codes", torch.int32, (N, K * bits // 32))
    _need_cuda(scales, "scales", torch.float16, (N, K // GROUP))
    _need_cuda(biases, "biases", torch.float16, (N, K // GROUP))
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _need_cuda(out, "out", out_dtype, (M, N))
    need = workspace_size(M, K, N, path, split_k, bits)
    if need > 0 and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _stream_handle(stream)
    name = "qlinear_forward" if bits == 4 else "qlinear8_forward"
    if path == PATH_AUTO and split_k == 0 and out_dtype == torch.bfloat16:
        s = getattr(L, name)(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), biases.data_ptr(), out.data_ptr(),
                             M, K, N, GROUP, ws_ptr, ws_bytes, st)
    else:
        s = getattr(L, name + "_config")(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                                         out.data_ptr(), _BF16 if out_dtype == torch.bfloat16 else _F32,
                                         M, K, N, GROUP, path, split_k, ws_ptr, ws_bytes, st)
    _check(s, name)
    return out


def forward_noalloc(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Small-M forward that allocates nothing on the device (qlinear_forward_noalloc in include/qlinear.h)."""
    L = lib()
    N, K = _weights_shape(codes, scales)
    M = x.shape[0]
    _need_cuda(x, "x", torch.bfloat16, (M, K))
    _need_cuda(codes, "codes", torch.int32, (N, K // 8))
    _need_cuda(scales, "scales", torch.float16, (N, K // GROUP))
    _need_cuda(biases, "biases", torch.float16, (N, K // GROUP))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need_cuda(out, "out", torch.bfloat16, (M, N))
    _check(L.qlinear_forward_noalloc(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                                     out.data_ptr(), M, K, N, GROUP, _stream_handle(stream)), "qlinear_forward_noalloc")
    return out


def dequant(codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, out_dtype=torch.float32,
            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W[n][k] = RN_fp32(scale * q + bias) (optionally rounded again to bf16)."""
    return _dequant(codes, scales, biases, out_dtype, out, stream, 4)


def dequant8(codes: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, out_dtype=torch.float32,
             out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dequant() for 8-bit codes, int32 [N][K/4] (qlinear8_dequant)."""
    return _dequant(codes, scales, biases, out_dtype, out, stream, 8)


def _dequant(codes, scales, biases, out_dtype, out, stream, bits):
    L = lib()
    N, K = _weights_shape(codes, scales, bits)
    _need_cuda(codes, "codes", torch.int32, (N, K * bits // 32))
    _need_cuda(scales, "scales", torch.float16, (N, K // GROUP))
    _need_cuda(biases, "biases", torch.float16, (N, K // GROUP))
    if out is None:
        out = torch.empty((N, K), dtype=out_dtype, device=codes.device)
    _need_cuda(out, "out", out_dtype, (N, K))
    dt = {torch.float32: _F32, torch.bfloat16: _BF16}[out_dtype]
    name = "qlinear_dequant" if bits == 4 else "qlinear8_dequant"
    _check(getattr(L, name)(codes.data_ptr(), scales.data_ptr(), biases.data_ptr(), K, N, GROUP, out.data_ptr(), dt,
                            _stream_handle(stream)), name)
    return out


def pack(w: torch.Tensor, imatrix: torch.Tensor | None = None, stream=None):
    """Quantize fp32 W [N][K] -> (codes, scales, biases): round-to-nearest, or the imatrix-weighted fit."""
    return _pack(w, imatrix, stream, 4)


def pack8(w: torch.Tensor, stream=None):
    """Round-to-nearest quantization of fp32 W [N][K] to 8-bit codes, int32 [N][K/4] (qlinear8_pack)."""
    return _pack(w, None, stream, 8)


def _pack(w, imatrix, stream, bits):
    L = lib()
    N, K = w.shape
    _need_cuda(w, "w", torch.float32, (N, K))
    codes = torch.empty((N, K * bits // 32), dtype=torch.int32, device=w.device)
    scales = torch.empty((N, K // GROUP), dtype=torch.float16, device=w.device)
    biases = torch.empty((N, K // GROUP), dtype=torch.float16, device=w.device)
    imp = None
    if imatrix is not None:
        _need_cuda(imatrix, "imatrix", torch.float32, (K,))
        imp = imatrix.data_ptr()
    name = "qlinear_pack" if bits == 4 else "qlinear8_pack"
    _check(getattr(L, name)(w.data_ptr(), imp, K, N, GROUP, codes.data_ptr(), scales.data_ptr(), biases.data_ptr(),
                            _stream_handle(stream)), name)
    return codes, scales, biases


def swiglu_workspace_size(M: int, K: int, I: int) -> int:
    """Workspace bytes of swiglu() (qlinear_swiglu_workspace_size)."""
    v = lib().qlinear_swiglu_workspace_size(M, K, I, GROUP)
    if v == ctypes.c_size_t(-1).value:
        raise ValueError("shape not supported")
    return int(v)


def swiglu(x: torch.Tensor, gate, up, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
           out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """h = silu(x . W_gate^T) * (x . W_up^T) for two packed [I][K] weights (qlinear_swiglu_forward).

    gate and up are (codes int32 [I][K/8], scales f16 [I][K/64], biases f16 [I][K/64]) triples.
    """
    L = lib()
    gc, gs, gb = gate
    uc, us, ub = up
    I, K = _weights_shape(gc, gs)
    M = x.shape[0]
    _need_cuda(x, "x", torch.bfloat16, (M, K))
    for name, c, s, b in (("gate", gc, gs, gb), ("up", uc, us, ub)):
        _need_cuda(c, name + " codes", torch.int32, (I, K // 8))
        _need_cuda(s, name + " scales", torch.float16, (I, K // GROUP))
        _need_cuda(b, name + " biases", torch.float16, (I, K // GROUP))
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    if out is None:
        out = torch.empty((M, I), dtype=out_dtype, device=x.device)
    _need_cuda(out, "out", out_dtype, (M, I))
    need = swiglu_workspace_size(M, K, I)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(L.qlinear_swiglu_forward(x.data_ptr(), gc.data_ptr(), gs.data_ptr(), gb.data_ptr(), uc.data_ptr(),
                                    us.data_ptr(), ub.data_ptr(), out.data_ptr(),
                                    _BF16 if out_dtype == torch.bfloat16 else _F32, M, K, I, GROUP,
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream_handle(stream)), "qlinear_swiglu_forward")
    return out


def reduce_partials(partials: torch.Tensor, out: torch.Tensor | None = None, out_dtype=torch.bfloat16,
                    stream=None) -> torch.Tensor:
    """Sum fp32 partials [S][...] over S in order, rounded once (qlinear_reduce_partials) -> [...]."""
    L = lib()
    if not isinstance(partials, torch.Tensor) or partials.dim() < 2:
        raise ValueError("partials must be a tensor [S][...]")
    _need_cuda(partials, "partials", torch.float32)
    S = partials.shape[0]
    shape = tuple(partials.shape[1:])
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=partials.device)
    _need_cuda(out, "out", out_dtype, shape)
    _check(L.qlinear_reduce_partials(partials.data_ptr(), S, out.numel(), out.data_ptr(),
                                     _BF16 if out_dtype == torch.bfloat16 else _F32, _stream_handle(stream)),
           "qlinear_reduce_partials")
    return out


def selftest_bounded_wait(stream=None) -> None:
    """Enqueue the bounded-wait self-test (qlinear_selftest_bounded_wait); device_status() then reads 6."""
    _check(lib().qlinear_selftest_bounded_wait(_stream_handle(stream)), "qlinear_selftest_bounded_wait")


def device_status(stream=None) -> int:
    """Synchronize the stream, then read and clear the device status word (0 = no kernel error)."""
    return int(lib().qlinear_get_device_status(_stream_handle(stream)))


def last_dispatch() -> str:
    buf = ctypes.create_string_buffer(256)
    _check(lib().qlinear_last_dispatch(buf, 256), "qlinear_last_dispatch")
    return buf.value.decode()


def set_profile_events(start, stop) -> None:
    """Record torch.cuda.Event `start`/`stop` around the main kernel of each later forward call (None, None: off)."""
    if start is None:
        _check(lib().qlinear_set_profile_events(None, None), "qlinear_set_profile_events")
    else:
        _check(lib().qlinear_set_profile_events(start.cuda_event, stop.cuda_event), "qlinear_set_profile_events")


def version() -> int:
    return int(lib().qlinear_version())
