"""Python binding of libstq1.so, the STQ1_0 quantized-matmul library for B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels (or, for ``quantize_ref``, its C++ host encoder).
PyTorch supplies device memory and the current CUDA stream.  There is no CPU
fallback: if the compiled library is missing, importing this package raises.

The functions mirror the C ABI declared in ``include/stq1.h``:
``quantize_ref``, ``dequant``, ``gemv``, ``moe_gateup``, ``status``.
"""

from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# STQ1_DEBUG=1 in the environment at import selects the bounds-checking build
DEBUG_BUILD = os.environ.get("STQ1_DEBUG", "") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libstq1_debug.so" if DEBUG_BUILD else "libstq1.so")

OK = 0
ERRORS = {
    -1: "STQ1_ERR_SHAPE", -2: "STQ1_ERR_NULL", -3: "STQ1_ERR_CUDA", -4: "STQ1_ERR_DEVICE",
    -5: "STQ1_ERR_VALUE", -6: "STQ1_ERR_ALIGN", -7: "STQ1_ERR_WORKSPACE", -8: "STQ1_ERR_ARG",
    -9: "STQ1_ERR_SCRATCH",
}
DEV_BAD_EXPERT = 1
DEV_WAIT_LIMIT = 2
DEV_BAD_VALUE = 4
DEV_BOUNDS = 8
BUILD_DEBUG = 1
ENC_PLAIN = 0
ENC_SHERRY = 1
MOE_WEIGHT_UP = 1
MOE_FP8 = 2
MOE_SKIP_FOREIGN = 4
BLOCK_BYTES = 42
BLOCK_WEIGHTS = 256
FMT_STQ1_0 = 0
FMT_STQ2 = 1
STQ2_BLOCK_BYTES = 66

# Every symbol include/stq1.h declares: name -> (restype, argtypes)
_c = ctypes
SIGNATURES = {
    "stq1_version": (_c.c_int, []),
    "stq1_quantize_ref": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int,
                                     _c.c_int, _c.c_void_p, _c.c_int]),
    "stq1_dequant": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p]),
    "stq1_gemv_workspace": (_c.c_size_t, [_c.c_int64, _c.c_int64, _c.c_int]),
    "stq1_gemv": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int,
                             _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "stq1_gemv_prefetch": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int,
                                      _c.c_void_p, _c.c_size_t, _c.c_void_p, _c.c_int64, _c.c_void_p]),
    "stq1_moe_workspace": (_c.c_size_t, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int]),
    "stq1_moe_gateup": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                   _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                   _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "stq1_status": (_c.c_int, [_c.c_void_p, _c.c_void_p]),
    "stq1_set_path": (_c.c_int, [_c.c_int]),
    "stq1_gemv_noalloc": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int,
                                     _c.c_void_p]),
    "stq1_swiglu": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p]),
    "stq1_moe_combine": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int, _c.c_int64,
                                    _c.c_void_p]),
    "stq1_moe_ffn_workspace": (_c.c_size_t, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int]),
    "stq1_moe_ffn": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64, _c.c_int,
                                _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "stq1_moe_ffn_local_workspace": (_c.c_size_t, [_c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64,
                                                    _c.c_int]),
    "stq1_moe_ffn_local": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                      _c.c_void_p, _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int64,
                                      _c.c_int, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "stq1_quantize": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int, _c.c_int,
                                 _c.c_void_p, _c.c_void_p]),
    "stq1_quantize_x_e4m3": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p,
                                        _c.c_void_p]),
    "stq1_quantize_stq2": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int, _c.c_void_p,
                                      _c.c_void_p]),
    "stq1_hessian_diag": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int64, _c.c_void_p,
                                     _c.c_void_p]),
    "stq1_hessian_error": (_c.c_int, [_c.c_int, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                      _c.c_int64, _c.c_int64, _c.c_int64, _c.c_int64, _c.c_void_p,
                                      _c.c_void_p]),
    "stq1_selftest_wait": (_c.c_int, [_c.c_int, _c.c_void_p]),
    "stq1_selftest_bounds": (_c.c_int, [_c.c_int, _c.c_int, _c.c_void_p]),
    "stq1_build_flags": (_c.c_int, []),
    "stq1_ep_dispatch": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int, _c.c_int, _c.c_int,
                                    _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                    _c.c_void_p, _c.c_void_p]),
    "stq1_ep_combine": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int, _c.c_int64,
                                   _c.c_void_p]),
    "stq1_mix_allocate": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64,
                                     _c.c_double, _c.c_void_p]),
}


class Stq1Error(RuntimeError):
    def __init__(self, func: str, code: int, device_err: int = 0):
        self.code = code
        self.device_err = device_err
        super().__init__(f"{func} returned {ERRORS.get(code, code)}"
                         + (f" (device error bits {device_err:#x})" if device_err else ""))


_lib = None
_lib_lock = threading.Lock()


def _load():
    """Loads libstq1.so once; raises ImportError if it is missing (no CPU fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{os.path.basename(LIB_PATH)} not found at {LIB_PATH}; build it with "
                    "`python -m sub_bit_sparse_b200.build`" + (" --debug" if DEBUG_BUILD else "")
                    + " (needs the CUDA toolkit)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def __getattr__(name):
    # ``sub_bit_sparse_b200.LIB`` loads the library on first access, so the build
    # module can be imported before the library exists.
    if name == "LIB":
        return _load()
    raise AttributeError(name)


def _check(func: str, rc: int):
    if rc != OK:
        raise Stq1Error(func, rc)


def packed_bytes(n: int, k: int) -> int:
    """Size in bytes of an [n, k] STQ1_0 matrix."""
    return n * (k // BLOCK_WEIGHTS) * BLOCK_BYTES


# ---------------------------------------------------------------------------
# Host encoder
# ---------------------------------------------------------------------------


def quantize_ref(w: np.ndarray, h: np.ndarray | None = None, mode: str = "plain", rounds: int = 3,
                 threads: int = 0) -> np.ndarray:
    """Encodes fp32 weights [N, K] with the host encoder; returns N*K/256*42 bytes (uint8)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    if w.ndim != 2:
        raise ValueError("w must be [N, K]")
    n, k = w.shape
    hh = None if h is None else np.ascontiguousarray(h, dtype=np.float32)
    out = np.empty(max(packed_bytes(n, k), 1), dtype=np.uint8)
    m = {"plain": ENC_PLAIN, "sherry": ENC_SHERRY}[mode]
    rc = _load().stq1_quantize_ref(w.ctypes.data, None if hh is None else hh.ctypes.data, n, k, m, rounds,
                               out.ctypes.data, threads)
    _check("stq1_quantize_ref", rc)
    return out[: packed_bytes(n, k)]


# ---------------------------------------------------------------------------
# Device calls
# ---------------------------------------------------------------------------

_ws_lock = threading.Lock()
_ws_cache: dict = {}


_torch_mod = None


def _torch():
    global _torch_mod
    if _torch_mod is None:
        import torch
        _torch_mod = torch
    return _torch_mod


def workspace(nbytes: int, device, kind: str = "gemv") -> "torch.Tensor | None":
    """A cached, zero-filled device workspace of at least ``nbytes`` for one kind of call
    ("gemv" or "moe"); the GEMV kind keeps its counter bytes zero between calls."""
    if nbytes == 0:
        return None
    torch = _torch()
    dev = torch.device(device)
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    key = (idx, kind)
    with _ws_lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=f"cuda:{idx}")
            _ws_cache[key] = buf
        return buf


_raw_stream = None


def _stream(t):
    """The current CUDA stream of t's device, as the handle the C ABI takes."""
    global _raw_stream
    torch = _torch()
    if _raw_stream is None:
        # torch's raw getter skips building a Stream object (about 2 us per call);
        # fall back to the public call if this torch lacks it
        getter = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        _raw_stream = getter if getter is not None else (
            lambda idx: torch.cuda.current_stream(idx).cuda_stream)
    return _raw_stream(t.get_device())


def _require(t, dtype, name):
    if getattr(t, "dtype", None) is dtype and t.is_cuda and t.is_contiguous():
        return
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    raise ValueError(f"{name} must be contiguous")


def dequant(w_packed, n: int, k: int, out=None):
    """Decoded weights [n, k] as bf16."""
    torch = _torch()
    _require(w_packed, torch.uint8, "w_packed")
    if out is None:
        out = torch.empty((n, k), dtype=torch.bfloat16, device=w_packed.device)
    _require(out, torch.bfloat16, "out")
    rc = _load().stq1_dequant(w_packed.data_ptr(), out.data_ptr(), n, k, _stream(w_packed))
    _check("stq1_dequant", rc)
    return out


def gemv(w_packed, x, n: int, k: int, out=None, ws=None, prefetch=None):
    """y [b, n] fp32 = W^ x for x [b, k] bf16.

    prefetch: the packed weights (uint8 CUDA tensor) of a following call, to be
    brought into L2 while this one runs (stq1_gemv_prefetch)."""
    torch = _torch()
    _require(w_packed, torch.uint8, "w_packed")
    _require(x, torch.bfloat16, "x")
    b = x.shape[0] if x.dim() == 2 else 1
    if out is None:
        out = torch.empty((b, n), dtype=torch.float32, device=x.device)
    _require(out, torch.float32, "out")
    lib = _lib if _lib is not None else _load()
    if ws is None:
        ws = workspace(lib.stq1_gemv_workspace(n, k, b), x.device)
    wsp, wsn = (None, 0) if ws is None else (ws.data_ptr(), ws.numel())
    if prefetch is None:
        rc = lib.stq1_gemv(w_packed.data_ptr(), x.data_ptr(), out.data_ptr(), n, k, b, wsp, wsn, _stream(x))
        if rc:
            _check("stq1_gemv", rc)
        return out
    _require(prefetch, torch.uint8, "prefetch")
    rc = lib.stq1_gemv_prefetch(w_packed.data_ptr(), x.data_ptr(), out.data_ptr(), n, k, b, wsp, wsn,
                                prefetch.data_ptr(), prefetch.numel(), _stream(x))
    if rc:
        _check("stq1_gemv_prefetch", rc)
    return out


def gemv_noalloc(w_packed, x, n: int, k: int, out=None):
    """Like ``gemv`` but the library allocates nothing and takes no workspace: for
    callers that cannot allocate device memory.  Its built-in scratch is shared by
    all calls in the process, so calls must not overlap on the GPU."""
    torch = _torch()
    _require(w_packed, torch.uint8, "w_packed")
    _require(x, torch.bfloat16, "x")
    b = x.shape[0] if x.dim() == 2 else 1
    if out is None:
        out = torch.empty((b, n), dtype=torch.float32, device=x.device)
    _require(out, torch.float32, "out")
    rc = _load().stq1_gemv_noalloc(w_packed.data_ptr(), x.data_ptr(), out.data_ptr(), n, k, b, _stream(x))
    _check("stq1_gemv_noalloc", rc)
    return out


def moe_gateup(expert_blocks, x, topk_ids, topk_weights, n: int, k: int, n_experts: int, flags: int = 0,
               out=None, ws=None):
    """y [T, topk, n] fp32: each token's routed experts' fused gate/up projections."""
    torch = _torch()
    _require(expert_blocks, torch.uint8, "expert_blocks")
    _require(x, torch.bfloat16, "x")
    _require(topk_ids, torch.int32, "topk_ids")
    if topk_weights is not None:
        _require(topk_weights, torch.float32, "topk_weights")
    t, topk = topk_ids.shape
    if out is None:
        out = torch.empty((t, topk, n), dtype=torch.float32, device=x.device)
    _require(out, torch.float32, "out")
    need = _load().stq1_moe_workspace(t, topk, n_experts, n, k, flags)
    if ws is None:
        ws = workspace(need, x.device, kind="moe")
    rc = _load().stq1_moe_gateup(expert_blocks.data_ptr(), x.data_ptr(), topk_ids.data_ptr(),
                             None if topk_weights is None else topk_weights.data_ptr(), out.data_ptr(),
                             t, topk, n_experts, n, k, flags,
                             None if ws is None else ws.data_ptr(), 0 if ws is None else ws.numel(),
                             _stream(x))
    _check("stq1_moe_gateup", rc)
    return out


def swiglu(y, n: int, out=None):
    """fp32 [P, n] fused gate/up rows -> bf16 [P, n/2] = SiLU(gate) * up."""
    torch = _torch()
    _require(y, torch.float32, "y")
    p = y.numel() // n
    if out is None:
        out = torch.empty((p, n // 2), dtype=torch.bfloat16, device=y.device)
    _require(out, torch.bfloat16, "out")
    _check("stq1_swiglu", _load().stq1_swiglu(y.data_ptr(), out.data_ptr(), p, n, _stream(y)))
    return out


def moe_combine(y, weights=None, out=None):
    """fp32 [T, topk, H] -> [T, H], routing-weighted sum over slots (plain sum without weights)."""
    torch = _torch()
    _require(y, torch.float32, "y")
    t, topk, h = y.shape
    if weights is not None:
        _require(weights, torch.float32, "weights")
    if out is None:
        out = torch.empty((t, h), dtype=torch.float32, device=y.device)
    _require(out, torch.float32, "out")
    rc = _load().stq1_moe_combine(y.data_ptr(), None if weights is None else weights.data_ptr(), out.data_ptr(),
                                  t, topk, h, _stream(y))
    _check("stq1_moe_combine", rc)
    return out


def moe_ffn(gateup_blocks, down_blocks, x, topk_ids, topk_weights, n: int, hidden: int, n_experts: int,
            flags: int = 0, out=None, ws=None):
    """Routed MoE feed-forward: gate/up -> SwiGLU -> down -> combine; returns fp32 [T, hidden]."""
    torch = _torch()
    _require(gateup_blocks, torch.uint8, "gateup_blocks")
    _require(down_blocks, torch.uint8, "down_blocks")
    _require(x, torch.bfloat16, "x")
    _require(topk_ids, torch.int32, "topk_ids")
    if topk_weights is not None:
        _require(topk_weights, torch.float32, "topk_weights")
    t, topk = topk_ids.shape
    if out is None:
        out = torch.empty((t, hidden), dtype=torch.float32, device=x.device)
    _require(out, torch.float32, "out")
    need = _load().stq1_moe_ffn_workspace(t, topk, n_experts, n, hidden, flags)
    if ws is None:
        ws = workspace(need, x.device, kind="ffn")
    rc = _load().stq1_moe_ffn(gateup_blocks.data_ptr(), down_blocks.data_ptr(), x.data_ptr(), topk_ids.data_ptr(),
                              None if topk_weights is None else topk_weights.data_ptr(), out.data_ptr(), t, topk,
                              n_experts, n, hidden, flags, None if ws is None else ws.data_ptr(),
                              0 if ws is None else ws.numel(), _stream(x))
    _check("stq1_moe_ffn", rc)
    return out


def moe_ffn_local(gateup_local, down_local, x, topk_ids, topk_weights, n: int, hidden: int, n_local: int,
                  expert_begin: int, flags: int = 0, out=None, ws=None):
    """This rank's partial MoE feed-forward output [T, hidden] for experts
    [expert_begin, expert_begin + n_local); pairs routed elsewhere contribute 0."""
    torch = _torch()
    _require(gateup_local, torch.uint8, "gateup_local")
    _require(down_local, torch.uint8, "down_local")
    _require(x, torch.bfloat16, "x")
    _require(topk_ids, torch.int32, "topk_ids")
    if topk_weights is not None:
        _require(topk_weights, torch.float32, "topk_weights")
    t, topk = topk_ids.shape
    if out is None:
        out = torch.empty((t, hidden), dtype=torch.float32, device=x.device)
    _require(out, torch.float32, "out")
    lib = _load()
    if ws is None:
        ws = workspace(lib.stq1_moe_ffn_local_workspace(t, topk, n_local, n, hidden, flags), x.device, kind="ffn")
    rc = lib.stq1_moe_ffn_local(gateup_local.data_ptr(), down_local.data_ptr(), x.data_ptr(), topk_ids.data_ptr(),
                                None if topk_weights is None else topk_weights.data_ptr(), out.data_ptr(), t, topk,
                                n_local, expert_begin, n, hidden, flags, None if ws is None else ws.data_ptr(),
                                0 if ws is None else ws.numel(), _stream(x))
    _check("stq1_moe_ffn_local", rc)
    return out


def quantize_gpu(w, h=None, mode: str = "plain", rounds: int = 3, out=None):
    """fp32 [N, K] CUDA tensor -> packed STQ1_0 bytes (uint8 CUDA tensor), byte-identical to quantize_ref."""
    torch = _torch()
    _require(w, torch.float32, "w")
    n, k = w.shape
    if h is not None:
        _require(h, torch.float32, "h")
    if out is None:
        out = torch.empty((n * (k // BLOCK_WEIGHTS) * BLOCK_BYTES,), dtype=torch.uint8, device=w.device)
    _require(out, torch.uint8, "out")
    m = ENC_SHERRY if mode == "sherry" else ENC_PLAIN
    rc = _load().stq1_quantize(w.data_ptr(), None if h is None else h.data_ptr(), n, k, m, rounds, out.data_ptr(),
                               _stream(w))
    _check("stq1_quantize", rc)
    return out


def stq2_quantize(w, h=None, rounds: int = 0, out=None):
    """fp32 [N, K] CUDA tensor -> packed STQ2 bytes (uint8 CUDA tensor, N*K/256*66).

    rounds = 0 is the amax encoding; rounds > 0 fits the scale to the
    per-column importance h (fp32 [K], or None for h = 1)."""
    torch = _torch()
    _require(w, torch.float32, "w")
    n, k = w.shape
    if h is not None:
        _require(h, torch.float32, "h")
    if out is None:
        out = torch.empty((n * (k // BLOCK_WEIGHTS) * STQ2_BLOCK_BYTES,), dtype=torch.uint8, device=w.device)
    _require(out, torch.uint8, "out")
    rc = _load().stq1_quantize_stq2(w.data_ptr(), None if h is None else h.data_ptr(), n, k, rounds,
                                    out.data_ptr(), _stream(w))
    _check("stq1_quantize_stq2", rc)
    return out


def hessian_diag(x, out=None):
    """bf16 calibration rows [L, rows, K] (or [rows, K]) -> fp32 [L, K]: sum over rows of x^2."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    nl, rows, k = x3.shape
    if out is None:
        out = torch.empty((nl, k), dtype=torch.float32, device=x.device)
    _require(out, torch.float32, "out")
    _check("stq1_hessian_diag", _load().stq1_hessian_diag(x3.data_ptr(), nl, rows, k, out.data_ptr(), _stream(x)))
    return out


def hessian_error(fmt: int, packed, w, x, h, out=None):
    """Per-layer (full, diagonal) Hessian error of a quantised weight set.

    packed: uint8 [L * N * K/256 * block bytes]; w: fp32 [L, N, K]; x: bf16
    [L, n_cal, K]; h: fp32 [L, K].  Returns fp64 [L, 2] on the device.
    """
    torch = _torch()
    _require(packed, torch.uint8, "packed")
    _require(w, torch.float32, "w")
    _require(x, torch.bfloat16, "x")
    _require(h, torch.float32, "h")
    nl, n, k = w.shape
    n_cal = x.shape[1]
    if out is None:
        out = torch.empty((nl, 2), dtype=torch.float64, device=w.device)
    _require(out, torch.float64, "out")
    rc = _load().stq1_hessian_error(fmt, packed.data_ptr(), w.data_ptr(), x.data_ptr(), h.data_ptr(), nl, n, k,
                                    n_cal, out.data_ptr(), _stream(w))
    _check("stq1_hessian_error", rc)
    return out


def mix_allocate(err_low, err_high, bytes_low, bytes_high, budget: float) -> np.ndarray:
    """Greedy per-byte layer allocation (host): bool [L], True = the higher-bit format."""
    arrs = [np.ascontiguousarray(v, dtype=np.float64) for v in (err_low, err_high, bytes_low, bytes_high)]
    n = arrs[0].shape[0]
    if any(a.shape != (n,) for a in arrs):
        raise ValueError("all four inputs must be 1-D of the same length")
    pick = np.zeros(max(n, 1), dtype=np.uint8)
    rc = _load().stq1_mix_allocate(*(a.ctypes.data for a in arrs), n, float(budget), pick.ctypes.data)
    _check("stq1_mix_allocate", rc)
    return pick[:n].astype(bool)


def quantize_x_e4m3(x, out=None, scales=None):
    """bf16 [T, K] -> (E4M3 codes uint8 [T, K], fp32 scales [T]), as the fp8 tile variant does."""
    torch = _torch()
    _require(x, torch.bfloat16, "x")
    t, k = x.shape
    if out is None:
        out = torch.empty((t, k), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((t,), dtype=torch.float32, device=x.device)
    _require(out, torch.uint8, "out")
    _require(scales, torch.float32, "scales")
    rc = _load().stq1_quantize_x_e4m3(x.data_ptr(), t, k, out.data_ptr(), scales.data_ptr(), _stream(x))
    _check("stq1_quantize_x_e4m3", rc)
    return out, scales


def ep_dispatch(topk_ids, x, topk_weights, n_experts: int, world: int):
    """Groups this rank's (token, slot) pairs by the rank owning their expert
    (stq1_ep_dispatch).  Returns (order, inv, counts [world + 1], local_ids,
    x_send [T*topk, K], w_send or None), all CUDA tensors."""
    torch = _torch()
    _require(topk_ids, torch.int32, "topk_ids")
    _require(x, torch.bfloat16, "x")
    t, topk = topk_ids.shape
    k = x.shape[1]
    n = t * topk
    dev = x.device
    order = torch.empty(n, dtype=torch.int32, device=dev)
    inv = torch.empty(n, dtype=torch.int32, device=dev)
    counts = torch.empty(world + 1, dtype=torch.int32, device=dev)
    local_ids = torch.empty(n, dtype=torch.int32, device=dev)
    x_send = torch.empty((n, k), dtype=torch.bfloat16, device=dev)
    w_send = None
    if topk_weights is not None:
        _require(topk_weights, torch.float32, "topk_weights")
        w_send = torch.empty(n, dtype=torch.float32, device=dev)
    rc = _load().stq1_ep_dispatch(topk_ids.data_ptr(), x.data_ptr(),
                                  None if topk_weights is None else topk_weights.data_ptr(), t, topk, n_experts,
                                  world, k, order.data_ptr(), inv.data_ptr(), counts.data_ptr(), local_ids.data_ptr(),
                                  x_send.data_ptr(), None if w_send is None else w_send.data_ptr(), _stream(x))
    _check("stq1_ep_dispatch", rc)
    return order, inv, counts, local_ids, x_send, w_send


def ep_combine(rows, inv, t: int, topk: int, out=None):
    """out [t, H] = per-token sum of the returned rows through inv (stq1_ep_combine)."""
    torch = _torch()
    _require(rows, torch.float32, "rows")
    _require(inv, torch.int32, "inv")
    h = rows.shape[1]
    if out is None:
        out = torch.empty((t, h), dtype=torch.float32, device=rows.device)
    _require(out, torch.float32, "out")
    rc = _load().stq1_ep_combine(rows.data_ptr(), inv.data_ptr(), out.data_ptr(), t, topk, h, _stream(rows))
    _check("stq1_ep_combine", rc)
    return out


PATH_AUTO, PATH_TABLE, PATH_TILES, PATH_MMA = 0, 1, 2, 3


def set_path(path: int) -> None:
    """Selects the matmul kernel process-wide (0 by size, 1 table kernel, 2 tile kernel,
    3 tensor-core decode kernel)."""
    _check("stq1_set_path", _load().stq1_set_path(path))


def selftest_wait(arrive: bool, stream=None) -> int:
    """Runs the bounded-wait self-test (see include/stq1.h) and returns the device error bits."""
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    _check("stq1_selftest_wait", _load().stq1_selftest_wait(1 if arrive else 0, ctypes.c_void_p(s.cuda_stream)))
    return status(s)


def selftest_bounds(index: int, bound: int, stream=None) -> int:
    """Runs the bounds-check self-test (see include/stq1.h) and returns the device error bits."""
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    _check("stq1_selftest_bounds", _load().stq1_selftest_bounds(int(index), int(bound), ctypes.c_void_p(s.cuda_stream)))
    return status(s)


def build_flags() -> int:
    """BUILD_DEBUG if the loaded library is the bounds-checking build, else 0."""
    return int(_load().stq1_build_flags())


def status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error word; raises on errors."""
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    err = ctypes.c_int(0)
    rc = _load().stq1_status(ctypes.c_void_p(s.cuda_stream), ctypes.byref(err))
    if rc not in (OK, -4):
        raise Stq1Error("stq1_status", rc)
    return err.value
