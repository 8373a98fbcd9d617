"""Python binding of the Muon C ABI (``include/muon.h``): argument marshalling only.

Every step of the optimizer runs in ``libmuon_b200.so`` (sm_100a kernels).  There is
no fallback: if the library is missing or the device is not a B200-class GPU, the
calls raise.

    h = muon_init(0)
    muon_step(h, params, grads, moms, lr=0.02, momentum=0.95)   # lists of CUDA tensors
    muon_destroy(h)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmuon_b200.so")

MUON_OK = 0
MUON_ERR_INVALID_ARG = 1
MUON_ERR_UNSUPPORTED = 2
MUON_ERR_OOM = 3
MUON_ERR_CUDA = 4
MUON_ERR_TIMEOUT = 5
MUON_ERR_TOO_LARGE = 6
MUON_ERR_CORRUPT = 7

MUON_F32 = 0
MUON_BF16 = 1
MUON_MODE_BF16 = 0
MUON_MODE_FP32_VALIDATE = 1
MUON_MODE_FP32_SIMT = 2

EXPORTED = ("muon_init", "muon_step", "muon_step_ex", "muon_newton_schulz", "muon_newton_schulz_noalloc",
            "muon_sync",
            "muon_selftest_wait_timeout", "muon_selftest_fail_next_alloc", "muon_selftest_stall_persistent",
            "muon_selftest_corrupt_guard",
            "muon_set_launch_mode",
            "muon_workspace_bytes",
            "muon_last_launch_count", "muon_profile_enable", "muon_profile_read", "muon_destroy",
            "muon_status_string", "muon_last_error")

# muon_kernel_kind
KERNEL_KINDS = ("momentum_norm", "gram", "poly", "update", "apply", "update_apply", "ns_persistent")

# muon_launch_mode
LAUNCH_MODES = {"auto": 0, "phases": 1, "persistent": 2}


class MuonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(msg)
        self.code = code


class muon_matrix(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p), ("momentum", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("param_dtype", ctypes.c_int), ("grad_dtype", ctypes.c_int)]


MUON_MOMENTUM_SGD = 0
MUON_MOMENTUM_LERP = 1


class muon_options(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("momentum", ctypes.c_float), ("nesterov", ctypes.c_int),
                ("momentum_form", ctypes.c_int), ("coeffs", ctypes.POINTER(ctypes.c_float)),
                ("ns_steps", ctypes.c_int), ("eps", ctypes.c_float), ("mode", ctypes.c_int),
                ("weight_decay", ctypes.c_float), ("cautious", ctypes.c_int),
                ("normuon", ctypes.c_int), ("normuon_beta2", ctypes.c_float), ("normuon_eps", ctypes.c_float),
                ("normuon_state", ctypes.POINTER(ctypes.c_void_p))]


_lib_handle = None


def load_library(path: str = LIB_PATH):
    """Loads libmuon_b200.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m muon_newton_schulz_06_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    lib.muon_init.argtypes = [ctypes.POINTER(vp), i32]
    lib.muon_init.restype = i32
    lib.muon_step.argtypes = [vp, ctypes.POINTER(muon_matrix), i32, f32, f32, i32, ctypes.POINTER(f32), i32,
                              f32, i32, vp]
    lib.muon_step.restype = i32
    lib.muon_step_ex.argtypes = [vp, ctypes.POINTER(muon_matrix), i32, ctypes.POINTER(muon_options), vp]
    lib.muon_step_ex.restype = i32
    lib.muon_newton_schulz.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(i64),
                                       ctypes.POINTER(i64), i32, i32, ctypes.POINTER(f32), i32, f32, i32, vp]
    lib.muon_newton_schulz.restype = i32
    lib.muon_newton_schulz_noalloc.argtypes = [vp, vp, i64, i64, i32, ctypes.POINTER(f32), i32, f32, vp, vp]
    lib.muon_newton_schulz_noalloc.restype = i32
    lib.muon_selftest_wait_timeout.argtypes = [vp, i64, vp]
    lib.muon_selftest_wait_timeout.restype = i32
    lib.muon_selftest_corrupt_guard.argtypes = [vp]
    lib.muon_selftest_corrupt_guard.restype = i32
    lib.muon_selftest_stall_persistent.argtypes = [vp, i64]
    lib.muon_selftest_stall_persistent.restype = i32
    lib.muon_set_launch_mode.argtypes = [vp, i32]
    lib.muon_set_launch_mode.restype = i32
    lib.muon_selftest_fail_next_alloc.argtypes = [vp]
    lib.muon_selftest_fail_next_alloc.restype = i32
    lib.muon_sync.argtypes = [vp]
    lib.muon_sync.restype = i32
    lib.muon_workspace_bytes.argtypes = [vp]
    lib.muon_workspace_bytes.restype = i64
    lib.muon_last_launch_count.argtypes = [vp]
    lib.muon_last_launch_count.restype = i32
    lib.muon_profile_enable.argtypes = [vp, i32]
    lib.muon_profile_enable.restype = i32
    lib.muon_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)]
    lib.muon_profile_read.restype = i32
    lib.muon_destroy.argtypes = [vp]
    lib.muon_destroy.restype = i32
    lib.muon_status_string.argtypes = [i32]
    lib.muon_status_string.restype = ctypes.c_char_p
    lib.muon_last_error.argtypes = [vp]
    lib.muon_last_error.restype = ctypes.c_char_p
    _lib_handle = lib
    return lib


def muon_status_string(code: int) -> str:
    return load_library().muon_status_string(int(code)).decode()


def _check(code: int, handle=None):
    if code != MUON_OK:
        lib = load_library()
        detail = lib.muon_last_error(handle).decode() if handle is not None else ""
        raise MuonError(code, f"{muon_status_string(code)}" + (f" ({detail})" if detail else ""))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MUON_BF16
    if t.dtype == torch.float32:
        return MUON_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _check_tensor(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D tensor")


def _coeff_array(coeffs, ns_steps):
    if coeffs is None:
        return None
    flat = [float(v) for row in coeffs for v in row]
    if len(flat) != 3 * ns_steps:
        raise ValueError("coeffs must hold ns_steps rows of (a, b, c)")
    return (ctypes.c_float * len(flat))(*flat)


def _mode_code(mode) -> int:
    if mode in ("bf16", MUON_MODE_BF16):
        return MUON_MODE_BF16
    if mode in ("fp32", "fp32_validate", MUON_MODE_FP32_VALIDATE):
        return MUON_MODE_FP32_VALIDATE
    if mode in ("fp32_simt", MUON_MODE_FP32_SIMT):
        return MUON_MODE_FP32_SIMT
    raise ValueError(f"unknown mode {mode!r}")


def _stream_ptr(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def muon_init(device: int = 0):
    """Returns an opaque handle bound to CUDA device ``device``."""
    h = ctypes.c_void_p()
    _check(load_library().muon_init(ctypes.byref(h), int(device)))
    return h


def _matrix_array(params, grads, moms):
    n = len(params)
    if len(grads) != n or len(moms) != n:
        raise ValueError("params, grads and moms must have the same length")
    arr = (muon_matrix * max(n, 1))()
    for i, (w, g, m) in enumerate(zip(params, grads, moms)):
        _check_tensor(w, "param")
        _check_tensor(g, "grad")
        _check_tensor(m, "momentum")
        if m.dtype != torch.float32:
            raise TypeError("momentum buffers must be float32")
        if g.shape != w.shape or m.shape != w.shape:
            raise ValueError(f"matrix {i}: param, grad and momentum shapes differ")
        arr[i] = muon_matrix(w.data_ptr(), g.data_ptr(), m.data_ptr(), w.shape[0], w.shape[1],
                             _dtype_code(w), _dtype_code(g))
    return arr, n


def muon_step(handle, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor],
              moms: Sequence[torch.Tensor], lr: float, momentum: float = 0.95, nesterov: bool = True,
              coeffs=None, ns_steps: int = 5, eps: float = 1e-7, mode="bf16", stream=None) -> None:
    """One Muon step over matched lists of parameters (bf16/fp32, updated in place),
    gradients (bf16/fp32) and float32 momentum buffers (updated in place)."""
    arr, n = _matrix_array(params, grads, moms)
    dev = params[0].device if n else torch.device("cuda")
    c = _coeff_array(coeffs, ns_steps)
    _check(load_library().muon_step(handle, arr, n, float(lr), float(momentum), 1 if nesterov else 0, c,
                                    int(ns_steps), float(eps), _mode_code(mode), _stream_ptr(stream, dev)),
           handle)


def muon_step_ex(handle, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor],
                 moms: Sequence[torch.Tensor], lr: float, momentum: float = 0.95, nesterov: bool = True,
                 momentum_form: str = "sgd", coeffs=None, ns_steps: int = 5, eps: float = 1e-7, mode="bf16",
                 weight_decay: float = 0.0, cautious: bool = False, normuon_state=None,
                 normuon_beta2: float = 0.95, normuon_eps: float = 1e-8, stream=None) -> None:
    """muon_step with every option: momentum_form "sgd" or "lerp"; weight_decay (0 = off);
    cautious (decay only where the update and the weight agree in sign); normuon_state
    (list of float32 CUDA vectors of min(rows, cols) entries, zero at the start) turns
    on the NorMuon rescaling and is updated in place."""
    forms = {"sgd": MUON_MOMENTUM_SGD, "lerp": MUON_MOMENTUM_LERP}
    if momentum_form not in forms:
        raise ValueError(f"unknown momentum_form {momentum_form!r}")
    arr, n = _matrix_array(params, grads, moms)
    dev = params[0].device if n else torch.device("cuda")
    c = _coeff_array(coeffs, ns_steps)
    ns_arr = None
    if normuon_state is not None:
        if len(normuon_state) != n:
            raise ValueError("normuon_state must hold one vector per matrix")
        ns_arr = (ctypes.c_void_p * max(n, 1))()
        for i, (v, w) in enumerate(zip(normuon_state, params)):
            if not (isinstance(v, torch.Tensor) and v.is_cuda and v.dtype == torch.float32 and v.is_contiguous()):
                raise TypeError("normuon_state entries must be contiguous float32 CUDA tensors")
            if v.numel() != min(w.shape):
                raise ValueError(f"normuon_state[{i}] must have min(rows, cols) = {min(w.shape)} entries")
            ns_arr[i] = v.data_ptr()
    opt = muon_options(float(lr), float(momentum), 1 if nesterov else 0, forms[momentum_form], c, int(ns_steps),
                       float(eps), _mode_code(mode), float(weight_decay), 1 if cautious else 0,
                       1 if normuon_state is not None else 0, float(normuon_beta2), float(normuon_eps),
                       ns_arr)
    _check(load_library().muon_step_ex(handle, arr, n, ctypes.byref(opt), _stream_ptr(stream, dev)), handle)


def muon_newton_schulz(handle, xs: Sequence[torch.Tensor], outs: Sequence[torch.Tensor], coeffs=None,
                       ns_steps: int = 5, eps: float = 1e-7, mode="bf16", stream=None) -> None:
    """outs[i] <- Newton-Schulz of xs[i] / (||xs[i]||_F + eps); xs and outs share a dtype."""
    n = len(xs)
    if len(outs) != n:
        raise ValueError("xs and outs must have the same length")
    if n == 0:
        return
    dt = _dtype_code(xs[0])
    xin = (ctypes.c_void_p * n)()
    xout = (ctypes.c_void_p * n)()
    rows = (ctypes.c_int64 * n)()
    cols = (ctypes.c_int64 * n)()
    for i, (x, o) in enumerate(zip(xs, outs)):
        _check_tensor(x, "x")
        _check_tensor(o, "out")
        if _dtype_code(x) != dt or _dtype_code(o) != dt:
            raise TypeError("all inputs and outputs must share one dtype")
        if o.shape != x.shape:
            raise ValueError(f"matrix {i}: output shape differs from input shape")
        xin[i], xout[i], rows[i], cols[i] = x.data_ptr(), o.data_ptr(), x.shape[0], x.shape[1]
    c = _coeff_array(coeffs, ns_steps)
    _check(load_library().muon_newton_schulz(handle, xin, xout, rows, cols, n, dt, c, int(ns_steps), float(eps),
                                             _mode_code(mode), _stream_ptr(stream, xs[0].device)), handle)


def muon_newton_schulz_noalloc(x: torch.Tensor, out: torch.Tensor, coeffs=None, ns_steps: int = 5,
                               eps: float = 1e-7, status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Allocation-free Newton-Schulz of one matrix on the current device: for callers
    that may not allocate device memory (memory reserved up front by their own pool,
    no allocation after start-up).  Uses a fixed 32 MiB scratch inside the library;
    matrices that do not fit raise MuonError with code MUON_ERR_TOO_LARGE.  Calls that
    overlap on the GPU race on that scratch.  ``status``: optional int32 CUDA tensor
    that receives 1 if a device-side wait times out."""
    _check_tensor(x, "x")
    _check_tensor(out, "out")
    if _dtype_code(x) != _dtype_code(out) or out.shape != x.shape:
        raise ValueError("x and out must share shape and dtype")
    if out.device != x.device:
        raise ValueError("x and out must be on the same device")
    st_ptr = None
    if status is not None:
        if not status.is_cuda or status.dtype != torch.int32:
            raise TypeError("status must be an int32 CUDA tensor")
        if status.device != x.device:
            raise ValueError("status must be on the device of x")
        st_ptr = status.data_ptr()
    c = _coeff_array(coeffs, ns_steps)
    # the library works on the current device: make it x's for the call
    with torch.cuda.device(x.device):
        _check(load_library().muon_newton_schulz_noalloc(x.data_ptr(), out.data_ptr(), x.shape[0], x.shape[1],
                                                         _dtype_code(x), c, int(ns_steps), float(eps), st_ptr,
                                                         _stream_ptr(stream, x.device)))


def muon_selftest_wait_timeout(handle, limit_ns: int, stream=None) -> None:
    """Enqueues the bounded-wait diagnostic (see include/muon.h); the next muon_sync
    raises MuonError with code MUON_ERR_TIMEOUT."""
    _check(load_library().muon_selftest_wait_timeout(handle, int(limit_ns), _stream_ptr(stream, None)), handle)


def muon_set_launch_mode(handle, mode: str = "auto") -> None:
    """How later bf16-mode calls launch the Newton-Schulz steps: "phases" (one grouped
    launch per phase and step), "persistent" (one launch for all steps) or "auto"."""
    if mode not in LAUNCH_MODES:
        raise ValueError(f"unknown launch mode {mode!r}; use one of {sorted(LAUNCH_MODES)}")
    _check(load_library().muon_set_launch_mode(handle, LAUNCH_MODES[mode]), handle)


def muon_selftest_stall_persistent(handle, limit_ns: int) -> None:
    """Arms the abort-path diagnostic of the persistent launch (see include/muon.h): the
    handle's next persistent launch gives up after limit_ns and the next muon_sync raises
    MuonError with code MUON_ERR_TIMEOUT."""
    _check(load_library().muon_selftest_stall_persistent(handle, int(limit_ns)), handle)


def muon_selftest_corrupt_guard(handle) -> None:
    """Overwrites one byte of a guard band of a debug-mode handle (MUON_DEBUG=1 when it was
    created); the next call raises MuonError with code MUON_ERR_CORRUPT."""
    _check(load_library().muon_selftest_corrupt_guard(handle), handle)


def muon_selftest_fail_next_alloc(handle) -> None:
    """Makes the handle's next workspace allocation report failure once (see
    include/muon.h); that call raises MuonError with code MUON_ERR_OOM."""
    _check(load_library().muon_selftest_fail_next_alloc(handle), handle)


def muon_sync(handle) -> None:
    _check(load_library().muon_sync(handle), handle)


def muon_workspace_bytes(handle) -> int:
    return int(load_library().muon_workspace_bytes(handle))


def muon_last_launch_count(handle) -> int:
    return int(load_library().muon_last_launch_count(handle))


def muon_profile_enable(handle, enable: bool = True) -> None:
    _check(load_library().muon_profile_enable(handle, 1 if enable else 0), handle)


def muon_profile_read(handle) -> dict:
    """{kind: (total_ms, launches)} since the last read (waits for the recorded events)."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(load_library().muon_profile_read(handle, ms, cnt), handle)
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}


def muon_destroy(handle) -> None:
    _check(load_library().muon_destroy(handle))


class Muon:
    """Small convenience wrapper owning one handle."""

    def __init__(self, device: int = 0):
        self.handle = muon_init(device)

    def step(self, params, grads, moms, **kw):
        muon_step_ex(self.handle, params, grads, moms, **kw)

    def newton_schulz(self, xs, outs, **kw):
        muon_newton_schulz(self.handle, xs, outs, **kw)

    def close(self):
        if self.handle is not None:
            muon_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
