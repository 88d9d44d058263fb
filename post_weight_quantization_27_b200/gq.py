"""ctypes binding of libgq.so (declared in include/gq.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch supplies device memory and the current CUDA stream.  Loading fails
loudly if libgq.so has not been built; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgq.so")

GQ_F32, GQ_F16, GQ_BF16 = 0, 1, 2
_DTYPES = {torch.float32: GQ_F32, torch.float16: GQ_F16, torch.bfloat16: GQ_BF16}

_c_i64, _c_int, _c_f32, _c_vp, _c_sz = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class GQError(RuntimeError):
    def __init__(self, status: int, name: str, detail: str, where: str):
        super().__init__(f"{where}: {name} ({detail})")
        self.status = status
        self.name = name


class SeqLayer(ctypes.Structure):
    """gq_seq_layer of include/gq.h."""
    _fields_ = [("W", ctypes.c_void_p), ("w_dtype", ctypes.c_int32), ("d_out", ctypes.c_int64),
                ("d_in", ctypes.c_int64), ("act", ctypes.c_int), ("residual_from", ctypes.c_int),
                ("qpacked", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zeros", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgq.so (loaded once)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m post_weight_quantization_27_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.gq_status_string.restype = ctypes.c_char_p
    L.gq_status_string.argtypes = [_c_int]
    L.gq_last_error.restype = ctypes.c_char_p
    L.gq_last_error.argtypes = []
    L.gq_launch_count.restype = ctypes.c_uint64
    L.gq_launch_count.argtypes = []
    L.gq_hessian_workspace_size.restype = _c_sz
    L.gq_hessian_workspace_size.argtypes = [_c_i64, _c_i64]
    L.gq_hessian_accumulate.restype = _c_int
    L.gq_hessian_accumulate.argtypes = [_c_vp, _c_i64, _c_i64, _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_hessian_compute.restype = _c_int
    L.gq_hessian_compute.argtypes = [_c_vp, _c_i64, _c_i64, _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_damp_cholesky_workspace_size.restype = _c_sz
    L.gq_damp_cholesky_workspace_size.argtypes = [_c_i64]
    L.gq_damp_cholesky_inverse.restype = _c_int
    L.gq_damp_cholesky_inverse.argtypes = [_c_vp, _c_i64, _c_f32, _c_int, _c_vp, _c_vp, _c_vp,
                                           _c_vp, _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_damp_cholesky_inverse_noalloc.restype = _c_int
    L.gq_damp_cholesky_inverse_noalloc.argtypes = [_c_vp, _c_i64, _c_f32, _c_int, _c_vp, _c_vp,
                                                   _c_vp, _c_vp, _c_vp, _c_vp]
    L.gq_gptq_workspace_size.restype = _c_sz
    L.gq_gptq_workspace_size.argtypes = [_c_i64, _c_i64, _c_int]
    L.gq_gptq_quantize_layer.restype = _c_int
    L.gq_gptq_quantize_layer.argtypes = [_c_vp, _c_int, _c_i64, _c_i64, _c_vp, _c_int, _c_int,
                                         _c_int, _c_int, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp,
                                         _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_rtn_quantize_pack.restype = _c_int
    L.gq_rtn_quantize_pack.argtypes = [_c_vp, _c_int, _c_i64, _c_i64, _c_int, _c_int, _c_int,
                                       _c_vp, _c_vp, _c_vp, _c_vp]
    L.gq_recon_workspace_size.restype = _c_sz
    L.gq_recon_workspace_size.argtypes = [_c_i64, _c_i64, _c_i64]
    L.gq_recon_error.restype = _c_int
    L.gq_recon_error.argtypes = [_c_vp, _c_int, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64,
                                 _c_int, _c_int, _c_int, _c_vp, _c_i64, _c_vp, _c_vp, _c_vp,
                                 _c_vp, _c_sz, _c_vp]
    L.gq_recon_error_hessian_workspace_size.restype = _c_sz
    L.gq_recon_error_hessian_workspace_size.argtypes = [_c_i64, _c_i64]
    L.gq_recon_error_hessian.restype = _c_int
    L.gq_recon_error_hessian.argtypes = [_c_vp, _c_int, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64,
                                         _c_i64, _c_int, _c_int, _c_int, _c_vp, _c_i64, _c_vp,
                                         _c_vp, _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_w4a16_workspace_size.restype = _c_sz
    L.gq_w4a16_workspace_size.argtypes = [_c_i64, _c_i64, _c_i64]
    L.gq_w4a16_matmul.restype = _c_int
    L.gq_w4a16_matmul.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64, _c_int, _c_int,
                                  _c_int, _c_vp, _c_i64, _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_qlinear_bf16.restype = _c_int
    L.gq_qlinear_bf16.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_i64, _c_i64,
                                  _c_int, _c_int, _c_int, _c_vp, _c_i64, _c_int, _c_vp, _c_vp,
                                  _c_vp, _c_sz, _c_vp]
    L.gq_gptq_sequential_workspace_size.restype = _c_sz
    L.gq_gptq_sequential_workspace_size.argtypes = [_c_vp, _c_int, _c_i64, _c_int]
    L.gq_gptq_sequential.restype = _c_int
    L.gq_gptq_sequential.argtypes = [_c_vp, _c_i64, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _c_f32, _c_vp, _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_awq_workspace_size.restype = _c_sz
    L.gq_awq_workspace_size.argtypes = [_c_i64, _c_i64, _c_i64, _c_int, _c_int, _c_int]
    L.gq_awq_rtn_search.restype = _c_int
    L.gq_awq_rtn_search.argtypes = [_c_vp, _c_int, _c_i64, _c_i64, _c_vp, _c_vp, _c_i64, _c_int,
                                    _c_int, _c_int, _c_int, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp,
                                    _c_vp, _c_vp, _c_sz, _c_vp]
    L.gq_workspace_status.restype = _c_int
    L.gq_workspace_status.argtypes = [_c_vp, _c_vp, _c_vp]
    L.gq_selftest_bounded_wait.restype = _c_int
    L.gq_selftest_bounded_wait.argtypes = [_c_int, ctypes.c_uint64, _c_vp, _c_sz, _c_vp]
    L.gq_kernel_timer_start.restype = _c_int
    L.gq_kernel_timer_start.argtypes = [ctypes.c_uint32, ctypes.c_int32]
    L.gq_kernel_timer_stop.restype = _c_int
    L.gq_kernel_timer_stop.argtypes = []
    L.gq_kernel_timer_read.restype = ctypes.c_int32
    L.gq_kernel_timer_read.argtypes = [_c_vp, _c_vp, _c_vp, ctypes.c_int32]
    L.gq_kernel_timer_release.restype = _c_int
    L.gq_kernel_timer_release.argtypes = []
    _lib = L
    return L


EXPORTS = ("gq_status_string", "gq_last_error", "gq_launch_count", "gq_hessian_workspace_size",
           "gq_hessian_accumulate", "gq_hessian_compute", "gq_damp_cholesky_workspace_size", "gq_damp_cholesky_inverse",
           "gq_damp_cholesky_inverse_noalloc",
           "gq_gptq_workspace_size", "gq_gptq_quantize_layer", "gq_rtn_quantize_pack",
           "gq_recon_workspace_size", "gq_recon_error", "gq_recon_error_hessian_workspace_size",
           "gq_recon_error_hessian", "gq_w4a16_workspace_size",
           "gq_w4a16_matmul", "gq_qlinear_bf16", "gq_gptq_sequential_workspace_size",
           "gq_gptq_sequential", "gq_awq_workspace_size",
           "gq_awq_rtn_search", "gq_workspace_status", "gq_selftest_bounded_wait",
           "gq_kernel_timer_start",
           "gq_kernel_timer_stop", "gq_kernel_timer_read", "gq_kernel_timer_release")


def _check(status: int, where: str) -> None:
    if status != 0:
        L = lib()
        raise GQError(status, L.gq_status_string(status).decode(),
                      L.gq_last_error().decode(), where)


def _p(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def workspace(nbytes: int, device) -> torch.Tensor:
    """A caller-owned workspace buffer (256-byte aligned by the allocator)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def launch_count() -> int:
    return int(lib().gq_launch_count())


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    """Device status word of the last call given ``ws`` (synchronises the
    stream).  Raises GQError(GQ_ERR_TIMEOUT) if a device-side wait of that
    call gave up; returns the word (0) otherwise."""
    word = ctypes.c_int32(-1)
    st = lib().gq_workspace_status(_p(ws), ctypes.byref(word), _stream(stream))
    _check(st, "gq_workspace_status")
    return int(word.value)


def selftest_bounded_wait(arrive: bool, limit_ns: int, stream=None) -> int:
    """Runs the bounded-wait self test and returns its status code (0, or 7
    when the wait gave up) without raising."""
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = workspace(256, dev)
    return int(lib().gq_selftest_bounded_wait(int(bool(arrive)), int(limit_ns), _p(ws),
                                              ws.numel(), _stream(stream)))


# ------------------------------------------------------------------ Hessian

def hessian_workspace_size(n_tok: int, d_in: int) -> int:
    return int(lib().gq_hessian_workspace_size(n_tok, d_in))


def hessian_accumulate(X: torch.Tensor, H: torch.Tensor, ws: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """H := sym(H) + 2 X^T X (in place); X [n_tok, d_in] bf16, H fp32."""
    _dev(X, "X", torch.bfloat16)
    n_tok, d_in = X.shape
    _dev(H, "H", torch.float32, (d_in, d_in))
    need = hessian_workspace_size(n_tok, d_in)
    ws = workspace(need, X.device) if ws is None else ws
    _check(lib().gq_hessian_accumulate(_p(X), n_tok, d_in, _p(H), _p(ws), ws.numel(),
                                       _stream(stream)), "gq_hessian_accumulate")
    return H


def hessian(X: torch.Tensor, H: torch.Tensor | None = None, ws: torch.Tensor | None = None,
            stream=None) -> torch.Tensor:
    """H = 2 X^T X (overwrites H when given; nothing is cleared first)."""
    _dev(X, "X", torch.bfloat16)
    n_tok, d_in = X.shape
    if H is None:
        H = torch.empty((d_in, d_in), dtype=torch.float32, device=X.device)
    _dev(H, "H", torch.float32, (d_in, d_in))
    ws = workspace(hessian_workspace_size(n_tok, d_in), X.device) if ws is None else ws
    _check(lib().gq_hessian_compute(_p(X), n_tok, d_in, _p(H), _p(ws), ws.numel(),
                                    _stream(stream)), "gq_hessian_compute")
    return H


# ------------------------------------------------------------------ damp + Cholesky

def damp_cholesky_workspace_size(d_in: int) -> int:
    return int(lib().gq_damp_cholesky_workspace_size(d_in))


def damp_cholesky_inverse(H: torch.Tensor, damp_percent: float = 0.01, act_order: bool = False,
                          U: torch.Tensor | None = None, check: bool = True,
                          ws: torch.Tensor | None = None, stream=None):
    """Dead columns, damping, optional act-order and U (H^-1 = U^T U).

    H is used as scratch.  Returns (U, perm or None, dead uint8, info int32
    device tensor).  With check=True the call synchronises and raises
    GQError(GQ_ERR_NOT_PD) if the damped H is not positive definite."""
    _dev(H, "H", torch.float32)
    d = H.shape[0]
    dev = H.device
    U = torch.empty((d, d), dtype=torch.float32, device=dev) if U is None else _dev(U, "U", torch.float32, (d, d))
    perm = torch.empty(d, dtype=torch.int32, device=dev) if act_order else None
    dead = torch.empty(d, dtype=torch.uint8, device=dev)
    info = torch.empty(1, dtype=torch.int32, device=dev)
    info_host = ctypes.c_int32(-1)
    ws = workspace(damp_cholesky_workspace_size(d), dev) if ws is None else ws
    st = lib().gq_damp_cholesky_inverse(_p(H), d, float(damp_percent), int(bool(act_order)),
                                        _p(perm), _p(dead), _p(U), _p(info),
                                        ctypes.byref(info_host) if check else None,
                                        _p(ws), ws.numel(), _stream(stream))
    _check(st, "gq_damp_cholesky_inverse")
    return U, perm, dead, info


def damp_cholesky_inverse_noalloc(H: torch.Tensor, damp_percent: float = 0.01,
                                  act_order: bool = False, U: torch.Tensor | None = None,
                                  check: bool = True, stream=None):
    """As damp_cholesky_inverse, through the entry point that takes no
    workspace (for callers that cannot allocate device memory; d_in <= 4096).
    The output tensors here are still allocated by torch for convenience."""
    _dev(H, "H", torch.float32)
    d = H.shape[0]
    dev = H.device
    U = torch.empty((d, d), dtype=torch.float32, device=dev) if U is None else _dev(U, "U", torch.float32, (d, d))
    perm = torch.empty(d, dtype=torch.int32, device=dev) if act_order else None
    dead = torch.empty(d, dtype=torch.uint8, device=dev)
    info = torch.empty(1, dtype=torch.int32, device=dev)
    info_host = ctypes.c_int32(-1)
    st = lib().gq_damp_cholesky_inverse_noalloc(_p(H), d, float(damp_percent),
                                                int(bool(act_order)), _p(perm), _p(dead), _p(U),
                                                _p(info), ctypes.byref(info_host) if check else None,
                                                _stream(stream))
    _check(st, "gq_damp_cholesky_inverse_noalloc")
    return U, perm, dead, info


# ------------------------------------------------------------------ GPTQ

def gptq_workspace_size(d_out: int, d_in: int, block_size: int = 128) -> int:
    return int(lib().gq_gptq_workspace_size(d_out, d_in, block_size))


def _n_groups(d_in: int, group_size: int) -> int:
    return 1 if group_size <= 0 else d_in // group_size


def _outputs(d_out, d_in, group_size, sym, dev, with_g_idx, bits=4):
    """Output tensors of a quantised layer; the dict also records its code
    width (``bits``), which the consumers of the packed format read."""
    ng = _n_groups(d_in, group_size)
    return dict(qpacked=torch.empty((d_out, bits * d_in // 32), dtype=torch.int32, device=dev),
                scales=torch.empty((d_out, ng), dtype=torch.float16, device=dev),
                zeros=None if sym else torch.empty((d_out, ng), dtype=torch.float16, device=dev),
                g_idx=torch.empty(d_in, dtype=torch.int32, device=dev) if with_g_idx else None,
                bits=bits)


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, bits: int = 4, group_size: int = -1,
                        block_size: int = 128, sym: bool = True, perm: torch.Tensor | None = None,
                        dead: torch.Tensor | None = None, out: dict | None = None,
                        ws: torch.Tensor | None = None, stream=None) -> dict:
    """GPTQ on one layer.  Returns dict(qpacked int32 [d_out, d_in/8] (uint32
    bit patterns), scales fp16, zeros fp16 or None, g_idx int32 or None)."""
    _dev(W, "W")
    if W.dtype not in _DTYPES:
        raise ValueError(f"unsupported W dtype {W.dtype}")
    d_out, d_in = W.shape
    _dev(U, "U", torch.float32, (d_in, d_in))
    if perm is not None:
        _dev(perm, "perm", torch.int32, (d_in,))
    if dead is not None:
        _dev(dead, "dead", torch.uint8, (d_in,))
    o = _outputs(d_out, d_in, group_size, sym, W.device, perm is not None, bits) \
        if out is None else out
    ws = workspace(gptq_workspace_size(d_out, d_in, block_size), W.device) if ws is None else ws
    st = lib().gq_gptq_quantize_layer(_p(W), _DTYPES[W.dtype], d_out, d_in, _p(U), bits,
                                      group_size, block_size, int(bool(sym)), _p(perm), _p(dead),
                                      _p(o["qpacked"]), _p(o["scales"]), _p(o["zeros"]),
                                      _p(o["g_idx"]), _p(ws), ws.numel(), _stream(stream))
    _check(st, "gq_gptq_quantize_layer")
    return o


# ------------------------------------------------------------------ RTN

def rtn_quantize_pack(W: torch.Tensor, bits: int = 4, group_size: int = -1, sym: bool = True,
                      out: dict | None = None, stream=None) -> dict:
    """Round-to-nearest with packing.  Same output layout as GPTQ."""
    _dev(W, "W")
    if W.dtype not in _DTYPES:
        raise ValueError(f"unsupported W dtype {W.dtype}")
    d_out, d_in = W.shape
    o = _outputs(d_out, d_in, group_size, sym, W.device, False, bits) if out is None else out
    st = lib().gq_rtn_quantize_pack(_p(W), _DTYPES[W.dtype], d_out, d_in, bits, group_size,
                                    int(bool(sym)), _p(o["qpacked"]), _p(o["scales"]),
                                    _p(o["zeros"]), _stream(stream))
    _check(st, "gq_rtn_quantize_pack")
    return o


# ------------------------------------------------------------------ reconstruction error

def recon_workspace_size(d_out: int, d_in: int, n_tok: int) -> int:
    return int(lib().gq_recon_workspace_size(d_out, d_in, n_tok))


def recon_error(W: torch.Tensor, q: dict, X: torch.Tensor, group_size: int = -1,
                sym: bool = True, sync: bool = True, sse: torch.Tensor | None = None,
                ws: torch.Tensor | None = None, stream=None):
    """SSE = ||(W - W^) X^T||_F^2 of a quantised layer ``q`` (dict as
    returned above).  With sync=True returns (sse, mse) as Python floats;
    otherwise the device fp64 tensor holding the SSE."""
    _dev(W, "W")
    _dev(X, "X", torch.bfloat16)
    d_out, d_in = W.shape
    n_tok = X.shape[0]
    sse = torch.empty(1, dtype=torch.float64, device=W.device) if sse is None else sse
    ws = workspace(recon_workspace_size(d_out, d_in, n_tok), W.device) if ws is None else ws
    sse_h, mse_h = ctypes.c_double(0.0), ctypes.c_double(0.0)
    st = lib().gq_recon_error(_p(W), _DTYPES[W.dtype], _p(q["qpacked"]), _p(q["scales"]),
                              _p(q.get("zeros")), _p(q.get("g_idx")), d_out, d_in,
                              int(q.get("bits", 4)), group_size, int(bool(sym)), _p(X), n_tok,
                              _p(sse),
                              ctypes.byref(sse_h) if sync else None,
                              ctypes.byref(mse_h) if sync else None,
                              _p(ws), ws.numel(), _stream(stream))
    _check(st, "gq_recon_error")
    return (sse_h.value, mse_h.value) if sync else sse


def recon_error_hessian_workspace_size(d_out: int, d_in: int) -> int:
    return int(lib().gq_recon_error_hessian_workspace_size(d_out, d_in))


def recon_error_hessian(W: torch.Tensor, q: dict, H0: torch.Tensor, n_tok: int,
                        group_size: int = -1, sym: bool = True, sync: bool = True,
                        sse: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                        stream=None):
    """The same SSE from the undamped Hessian H0 = 2 X^T X:
    tr((W - W^) H0 (W - W^)^T) / 2.  ``n_tok`` only scales the MSE.  Returns
    like recon_error."""
    _dev(W, "W")
    d_out, d_in = W.shape
    _dev(H0, "H0", torch.float32, (d_in, d_in))
    sse = torch.empty(1, dtype=torch.float64, device=W.device) if sse is None else sse
    ws = workspace(recon_error_hessian_workspace_size(d_out, d_in), W.device) if ws is None else ws
    sse_h, mse_h = ctypes.c_double(0.0), ctypes.c_double(0.0)
    st = lib().gq_recon_error_hessian(_p(W), _DTYPES[W.dtype], _p(q["qpacked"]),
                                      _p(q["scales"]), _p(q.get("zeros")), _p(q.get("g_idx")),
                                      d_out, d_in, int(q.get("bits", 4)), group_size,
                                      int(bool(sym)), _p(H0), n_tok,
                                      _p(sse), ctypes.byref(sse_h) if sync else None,
                                      ctypes.byref(mse_h) if sync else None,
                                      _p(ws), ws.numel(), _stream(stream))
    _check(st, "gq_recon_error_hessian")
    return (sse_h.value, mse_h.value) if sync else sse


# ------------------------------------------------------------------ products with a quantised layer

ACT = {"none": 0, "relu": 1, "gelu": 2}


def w4a16_workspace_size(d_out: int, d_in: int, n_tok: int) -> int:
    return int(lib().gq_w4a16_workspace_size(d_out, d_in, n_tok))


def w4a16_matmul(q: dict, d_in: int, X: torch.Tensor, group_size: int = -1, sym: bool = True,
                 Y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """Y = W^ X^T (fp32 [d_out][n_tok]) from a quantised layer ``q`` (dict as
    returned by the quantisers) and bf16 activations X [n_tok][d_in]."""
    _dev(X, "X", torch.bfloat16)
    d_out = q["qpacked"].shape[0]
    n_tok = X.shape[0]
    Y = torch.empty((d_out, n_tok), dtype=torch.float32, device=X.device) if Y is None else Y
    ws = workspace(w4a16_workspace_size(d_out, d_in, n_tok), X.device) if ws is None else ws
    st = lib().gq_w4a16_matmul(_p(q["qpacked"]), _p(q["scales"]), _p(q.get("zeros")),
                               _p(q.get("g_idx")), d_out, d_in, int(q.get("bits", 4)),
                               group_size, int(bool(sym)), _p(X), n_tok, _p(Y), _p(ws),
                               ws.numel(), _stream(stream))
    _check(st, "gq_w4a16_matmul")
    return Y


def qlinear_bf16(X: torch.Tensor, d_out: int, q: dict | None = None, W: torch.Tensor | None = None,
                 group_size: int = -1, sym: bool = True, act: str = "none",
                 R: torch.Tensor | None = None, Z: torch.Tensor | None = None,
                 ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Z = act(X W^T) (+ R), bf16 [n_tok][d_out]: the layer applied to its
    input, from the packed layer ``q`` or (q None) from dense weights W."""
    _dev(X, "X", torch.bfloat16)
    n_tok, d_in = X.shape
    Z = torch.empty((n_tok, d_out), dtype=torch.bfloat16, device=X.device) if Z is None else Z
    if R is not None:
        _dev(R, "R", torch.bfloat16, (n_tok, d_out))
    ws = workspace(256, X.device) if ws is None else ws
    qq = q or {}
    st = lib().gq_qlinear_bf16(_p(qq.get("qpacked")), _p(qq.get("scales")), _p(qq.get("zeros")),
                               _p(qq.get("g_idx")), _p(W), _DTYPES.get(W.dtype, 0) if W is not None else 0,
                               d_out, d_in, int(qq.get("bits", 4)), group_size, int(bool(sym)),
                               _p(X), n_tok, ACT[act], _p(R), _p(Z), _p(ws), ws.numel(),
                               _stream(stream))
    _check(st, "gq_qlinear_bf16")
    return Z


# ------------------------------------------------------------------ sequential quantisation

def gptq_sequential(X0: torch.Tensor, layers: list, bits: int = 4, group_size: int = -1,
                    block_size: int = 128, sym: bool = True, damp_percent: float = 0.01,
                    stream=None):
    """A chain of layers quantised one after another, each on the input it
    receives from the quantised layers before it.  ``layers``: list of dicts
    with W (device [d_out, d_in]), act ("none", "relu", "gelu") and
    residual_from (None or the index of an earlier input added to the
    output).  Returns (list of quantised-layer dicts, sse numpy [n_layers],
    list of the inputs X_0 .. X_n as bf16 device tensors, X_n the chain's
    output)."""
    import numpy as np
    _dev(X0, "X0", torch.bfloat16)
    n_tok = X0.shape[0]
    dev = X0.device
    arr = (SeqLayer * len(layers))()
    outs = []
    for i, L in enumerate(layers):
        W = _dev(L["W"], "W")
        d_out, d_in = W.shape
        o = _outputs(d_out, d_in, group_size, sym, dev, False, bits)
        outs.append(o)
        r = L.get("residual_from")
        arr[i] = SeqLayer(W.data_ptr(), _DTYPES[W.dtype], d_out, d_in, ACT[L.get("act", "none")],
                          -1 if r is None else int(r), o["qpacked"].data_ptr(),
                          o["scales"].data_ptr(), _p(o["zeros"]))
    lib_ = lib()
    need = int(lib_.gq_gptq_sequential_workspace_size(ctypes.addressof(arr), len(layers), n_tok,
                                                      block_size))
    ws = workspace(need, dev)
    sse = torch.empty(len(layers), dtype=torch.float64, device=dev)
    widths = [L["W"].shape[1] for L in layers] + [layers[-1]["W"].shape[0]]
    X_all = torch.empty(n_tok * sum(widths), dtype=torch.bfloat16, device=dev)
    st = lib_.gq_gptq_sequential(_p(X0), n_tok, ctypes.addressof(arr), len(layers), bits,
                                 group_size, block_size, int(bool(sym)), float(damp_percent),
                                 _p(sse), _p(X_all), _p(ws), ws.numel(), _stream(stream))
    _check(st, "gq_gptq_sequential")
    xs, off = [], 0
    for d in widths:
        xs.append(X_all[off:off + n_tok * d].view(n_tok, d))
        off += n_tok * d
    return outs, sse.cpu().numpy().astype(np.float64), xs


# ------------------------------------------------------------------ activation-aware scaling

def awq_workspace_size(d_out: int, d_in: int, n_tok: int, group_size: int = -1,
                       sym: bool = True, bits: int = 4) -> int:
    return int(lib().gq_awq_workspace_size(d_out, d_in, n_tok, bits, group_size,
                                           int(bool(sym))))


def awq_rtn_search(W: torch.Tensor, H: torch.Tensor, X: torch.Tensor, bits: int = 4,
                   group_size: int = -1, sym: bool = True, n_grid: int = 20,
                   ws: torch.Tensor | None = None, stream=None) -> dict:
    """Per-channel activation-aware scaling before RTN (include/gq.h).
    Returns the RTN outputs for the chosen alpha plus ``col_scale`` (device
    fp32 [d_in]), ``mse`` (list of the error per alpha) and ``best`` (k)."""
    import numpy as np
    _dev(W, "W")
    _dev(H, "H", torch.float32)
    _dev(X, "X", torch.bfloat16)
    d_out, d_in = W.shape
    n_tok = X.shape[0]
    o = _outputs(d_out, d_in, group_size, sym, W.device, False, bits)
    col = torch.empty(d_in, dtype=torch.float32, device=W.device)
    mse = np.zeros(n_grid, dtype=np.float64)
    best = ctypes.c_int32(-1)
    ws = workspace(awq_workspace_size(d_out, d_in, n_tok, group_size, sym, bits), W.device) \
        if ws is None else ws
    st = lib().gq_awq_rtn_search(_p(W), _DTYPES[W.dtype], d_out, d_in, _p(H), _p(X), n_tok, bits,
                                 group_size, int(bool(sym)), n_grid, _p(o["qpacked"]),
                                 _p(o["scales"]), _p(o["zeros"]), _p(col), mse.ctypes.data,
                                 ctypes.byref(best), _p(ws), ws.numel(), _stream(stream))
    _check(st, "gq_awq_rtn_search")
    o.update(col_scale=col, mse=mse, best=int(best.value))
    return o


# ------------------------------------------------------------------ per-launch kernel timing

# gq_kernel values (include/gq.h) and the unit of each kernel's work figure
KERNELS = ("hessian_mma", "potrf_trsm", "block_inverse", "gemm_tf32x3", "gptq_block", "rtn",
           "recon_mma", "qlinear", "syrk_bf16")
KERNEL_UNITS = {"hessian_mma": "flop", "potrf_trsm": "flop", "block_inverse": "flop",
                "gemm_tf32x3": "flop", "gptq_block": "byte", "rtn": "byte", "recon_mma": "flop",
                "qlinear": "flop", "syrk_bf16": "flop"}


def kernel_timer_start(kernels, capacity: int) -> None:
    """Time every launch of the named kernels (up to ``capacity`` launches)."""
    mask = 0
    for k in kernels:
        mask |= 1 << KERNELS.index(k)
    _check(lib().gq_kernel_timer_start(mask, int(capacity)), "gq_kernel_timer_start")


def kernel_timer_stop() -> None:
    _check(lib().gq_kernel_timer_stop(), "gq_kernel_timer_stop")


def kernel_timer_read() -> list:
    """[(kernel name, ms, algorithmic work)] of the recorded launches (their
    last execution); call after the work has finished."""
    import numpy as np
    L = lib()
    n = L.gq_kernel_timer_read(None, None, None, 0)
    if n < 0:
        _check(8, "gq_kernel_timer_read")
    kind = np.zeros(max(n, 1), dtype=np.int32)
    ms = np.zeros(max(n, 1), dtype=np.float32)
    work = np.zeros(max(n, 1), dtype=np.float64)
    m = L.gq_kernel_timer_read(kind.ctypes.data, ms.ctypes.data, work.ctypes.data, n)
    if m < 0:
        _check(8, "gq_kernel_timer_read")
    return [(KERNELS[k], float(t), float(w)) for k, t, w in zip(kind[:n], ms[:n], work[:n])
            if k >= 0]


def kernel_timer_release() -> None:
    _check(lib().gq_kernel_timer_release(), "gq_kernel_timer_release")
