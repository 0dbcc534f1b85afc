"""ctypes binding of ``libmamba_scan.so`` (C ABI: ``include/mamba_scan.h``).

Argument marshalling only: shapes and dtypes are checked, outputs are
allocated with torch when the caller does not pass them, and raw device
pointers plus the current CUDA stream are handed to the library.  Every step
of the computation runs in the library's CUDA kernels; there is no host or
PyTorch fallback, and a missing library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

from . import build as _build

MAMBA_F32, MAMBA_BF16 = 0, 1
_ACT = {torch.float32: MAMBA_F32, torch.bfloat16: MAMBA_BF16}

MAMBA_OK = 0
STATUS_NAMES = {0: "MAMBA_OK", -1: "MAMBA_ERR_NULL", -2: "MAMBA_ERR_SHAPE",
                -3: "MAMBA_ERR_UNSUPPORTED", -4: "MAMBA_ERR_ALIGN",
                -5: "MAMBA_ERR_CUDA", -6: "MAMBA_ERR_DEVICE", -7: "MAMBA_ERR_OVERLAP",
                -8: "MAMBA_ERR_WORKSPACE", -9: "MAMBA_ERR_TIMEOUT", -10: "MAMBA_ERR_BOUNDS"}
MAMBA_ERR_UNSUPPORTED = -3
MAMBA_ERR_TIMEOUT = -9
MAMBA_ERR_BOUNDS = -10
SCHEDULE_AUTO, SCHEDULE_STATIC, SCHEDULE_PERSISTENT, SCHEDULE_LOCAL = 0, 1, 2, 3

# Every function include/mamba_scan.h declares.
EXPORTED = ("mamba_scan_fwd", "mamba_scan_fwd_tuned", "mamba_scan_fwd_ws",
            "mamba_scan_plan", "mamba_scan_plan_noworkspace", "mamba_scan_workspace_size",
            "mamba_scan_workspace_status",
            "mamba_scan_fwd_noalloc", "mamba_scan_fwd_init", "mamba_scan_state", "mamba_scan_fwd_strided",
            "mamba_scan_fwd_complex", "mamba_delta_sum", "mamba_state_fold", "mamba_scan_fwd_conv",
            "mamba_scan_host_scratch_size", "mamba_scan_fwd_host", "mamba_debug_stall_group",
            "mamba_get_device_status", "mamba_scan_bwd", "mamba_scan_bwd_init",
            "mamba_scan_bwd_workspace_size", "mamba_scan_ckpt_size", "mamba_scan_fwd_ckpt",
            "mamba_scan_bwd_ckpt",
            "mamba_state_update", "mamba_conv1d_fwd",
            "mamba_conv1d_update", "mamba_status_string", "mamba_abi_version",
            "mamba_bounds_checked", "mamba_debug_bounds_status", "mamba_debug_shrink_output_extent")


class MambaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)} ({msg})")
        self.code = code


class Tuning(ctypes.Structure):
    _fields_ = [("lanes_per_channel", ctypes.c_int), ("threads_per_block", ctypes.c_int),
                ("schedule", ctypes.c_int), ("chunk_timesteps", ctypes.c_int)]


class Stride3(ctypes.Structure):
    """Element strides of one sequence tensor (batch, row, time)."""
    _fields_ = [("batch", ctypes.c_int64), ("row", ctypes.c_int64), ("time", ctypes.c_int64)]


class ScanStrides(ctypes.Structure):
    _fields_ = [(k, Stride3) for k in ("u", "delta", "z", "out", "B", "C")]


_lock = threading.Lock()
_lib: Optional[ctypes.CDLL] = None


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    vp, fp, i64, ci = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    scan_args = [vp, vp, fp, vp, vp, fp, vp, fp, ci, vp, fp, i64, i64, i64, i64, ci]
    lib.mamba_scan_fwd.argtypes = scan_args + [vp]
    lib.mamba_scan_fwd.restype = ci
    lib.mamba_scan_fwd_tuned.argtypes = scan_args + [ctypes.POINTER(Tuning), vp]
    lib.mamba_scan_fwd_tuned.restype = ci
    lib.mamba_scan_fwd_ws.argtypes = scan_args + [ctypes.POINTER(Tuning), vp, ctypes.c_size_t, vp]
    lib.mamba_scan_fwd_ws.restype = ci
    lib.mamba_scan_fwd_init.argtypes = scan_args[:9] + [fp] + scan_args[9:] + [
        ctypes.POINTER(Tuning), vp, ctypes.c_size_t, vp]
    lib.mamba_scan_fwd_init.restype = ci
    lib.mamba_scan_state.argtypes = [vp, vp, fp, vp, fp, ci, fp, fp, i64, i64, i64, i64, ci, vp, ctypes.c_size_t,
                                     vp]
    lib.mamba_scan_state.restype = ci
    lib.mamba_scan_fwd_strided.argtypes = scan_args[:9] + [fp] + scan_args[9:] + [
        ctypes.POINTER(ScanStrides), ctypes.POINTER(Tuning), vp]
    lib.mamba_scan_fwd_strided.restype = ci
    lib.mamba_scan_fwd_complex.argtypes = scan_args[:9] + [fp] + scan_args[9:] + [
        ctypes.POINTER(Tuning), vp]
    lib.mamba_scan_fwd_complex.restype = ci
    dp = vp  # double *
    lib.mamba_scan_fwd_conv.argtypes = [vp, fp, fp, i64, i64, vp, fp, vp, vp, fp, vp, i64, fp, fp, vp, fp, vp,
                                        i64, i64, i64, i64, ci, vp, ctypes.c_size_t, vp]
    lib.mamba_scan_fwd_conv.restype = ci
    lib.mamba_get_device_status.argtypes = [vp]
    lib.mamba_get_device_status.restype = ci
    lib.mamba_debug_stall_group.argtypes = [ci]
    lib.mamba_debug_stall_group.restype = ci
    lib.mamba_bounds_checked.argtypes = []
    lib.mamba_bounds_checked.restype = ci
    lib.mamba_debug_bounds_status.argtypes = [vp, vp]
    lib.mamba_debug_bounds_status.restype = ci
    lib.mamba_debug_shrink_output_extent.argtypes = [ci]
    lib.mamba_debug_shrink_output_extent.restype = ci
    lib.mamba_scan_host_scratch_size.argtypes = [i64, i64, i64, i64, ci]
    lib.mamba_scan_host_scratch_size.restype = ctypes.c_size_t
    lib.mamba_scan_fwd_host.argtypes = scan_args[:9] + [fp] + scan_args[9:] + [vp, ctypes.c_size_t, vp]
    lib.mamba_scan_fwd_host.restype = ci
    lib.mamba_delta_sum.argtypes = [vp, fp, ci, dp, i64, i64, i64, ci, vp]
    lib.mamba_delta_sum.restype = ci
    lib.mamba_state_fold.argtypes = [fp, dp, fp, fp, fp, i64, i64, i64, i64, vp]
    lib.mamba_state_fold.restype = ci
    lib.mamba_scan_fwd_noalloc.argtypes = scan_args + [vp]
    lib.mamba_scan_fwd_noalloc.restype = ci
    lib.mamba_scan_plan.argtypes = [i64, i64, i64, i64, ci, ctypes.POINTER(Tuning)]
    lib.mamba_scan_plan.restype = ci
    lib.mamba_scan_plan_noworkspace.argtypes = [i64, i64, i64, i64, ci, ctypes.POINTER(Tuning)]
    lib.mamba_scan_plan_noworkspace.restype = ci
    lib.mamba_scan_workspace_size.argtypes = [i64, i64, i64, i64, ci]
    lib.mamba_scan_workspace_size.restype = ctypes.c_size_t
    lib.mamba_scan_workspace_status.argtypes = [vp, vp]
    lib.mamba_scan_workspace_status.restype = ci
    lib.mamba_state_update.argtypes = [fp, vp, vp, fp, vp, vp, fp, vp, fp, ci, vp,
                                       i64, i64, i64, ci, vp]
    lib.mamba_state_update.restype = ci
    lib.mamba_scan_bwd.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, ci, vp, fp, vp, vp, fp, fp, fp, fp,
                                   vp, fp, i64, i64, i64, i64, ci, vp, ctypes.c_size_t, vp]
    lib.mamba_scan_bwd.restype = ci
    bwd = lib.mamba_scan_bwd.argtypes
    lib.mamba_scan_bwd_init.argtypes = bwd[:9] + [fp] + bwd[9:19] + [fp] + bwd[19:]
    lib.mamba_scan_bwd_init.restype = ci
    lib.mamba_scan_bwd_workspace_size.argtypes = [i64, i64, i64, i64]
    lib.mamba_scan_bwd_workspace_size.restype = ctypes.c_size_t
    lib.mamba_scan_ckpt_size.argtypes = [i64, i64, i64, i64]
    lib.mamba_scan_ckpt_size.restype = ctypes.c_size_t
    lib.mamba_scan_fwd_ckpt.argtypes = scan_args[:9] + [fp, vp, fp, fp, ctypes.c_size_t, i64, i64, i64, i64, ci, vp]
    lib.mamba_scan_fwd_ckpt.restype = ci
    lib.mamba_scan_bwd_ckpt.argtypes = bwd[:9] + [fp, fp] + bwd[9:19] + [fp] + bwd[19:]
    lib.mamba_scan_bwd_ckpt.restype = ci
    lib.mamba_conv1d_fwd.argtypes = [vp, fp, fp, ci, vp, i64, i64, i64, i64, i64, ci, vp]
    lib.mamba_conv1d_fwd.restype = ci
    lib.mamba_conv1d_update.argtypes = [fp, vp, fp, fp, ci, vp, i64, i64, i64, i64, ci, vp]
    lib.mamba_conv1d_update.restype = ci
    lib.mamba_status_string.argtypes = [ci]
    lib.mamba_status_string.restype = ctypes.c_char_p
    lib.mamba_abi_version.argtypes = []
    lib.mamba_abi_version.restype = ci
    return lib


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load the CUDA library, building it with nvcc first if it is missing or
    older than its sources.  Raises if it cannot be built or loaded."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or _build.LIB
        if path is None and not _build.up_to_date():
            _build.build()
        if not os.path.exists(p):
            raise RuntimeError(f"CUDA library {p} is missing and could not be built")
        lib = _declare(ctypes.CDLL(p))
        if path is None:
            _lib = lib
        return lib


def status_string(code: int) -> str:
    return load_library().mamba_status_string(code).decode()


def _check(fn: str, code: int):
    if code != MAMBA_OK:
        raise MambaError(fn, code, status_string(code))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: Optional[torch.Tensor], name: str, device, dtype, shape):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def mamba_scan_fwd(u: torch.Tensor, delta: torch.Tensor, A: torch.Tensor,
                   B: torch.Tensor, C: torch.Tensor, D: Optional[torch.Tensor] = None,
                   z: Optional[torch.Tensor] = None,
                   delta_bias: Optional[torch.Tensor] = None,
                   delta_softplus: bool = True, out: Optional[torch.Tensor] = None,
                   last_state: Optional[torch.Tensor] = None,
                   return_last_state: bool = False, lanes_per_channel: int = 0,
                   threads_per_block: int = 0, schedule: int = SCHEDULE_AUTO,
                   workspace: Optional[torch.Tensor] = None, chunk_timesteps: int = 0,
                   h0: Optional[torch.Tensor] = None):
    """Selective scan forward on the current CUDA stream.

    u, delta, z: (batch, dim, L); B, C: (batch, N, L) -- all one dtype,
    float32 or bfloat16.  A: (dim, N) fp32; D, delta_bias: (dim,) fp32.
    Returns ``out`` (batch, dim, L), or ``(out, last_state)`` when
    ``return_last_state`` is set or ``last_state`` is passed.

    Without a workspace the library picks the local schedule (one block per
    SM splits whole channel groups among its warps, carries in shared memory)
    or the static one.  A device workspace (``mamba_scan_workspace_size``
    bytes; allocated here with torch when ``schedule`` is SCHEDULE_PERSISTENT
    and none is given) enables the device-wide persistent schedule;
    ``schedule`` / ``lanes_per_channel`` / ``threads_per_block`` force a
    launch configuration (0 = automatic).

    ``h0`` (batch, dim, N) fp32 starts every row's recurrence from that
    state instead of zeros (it may be ``last_state`` itself).
    """
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, seqlen)")
    batch, dim, L = u.shape
    if A.dim() != 2:
        raise ValueError("A must be (dim, dstate)")
    N = A.shape[1]
    dev, act = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    _need(u, "u", dev, act, (batch, dim, L))
    _need(delta, "delta", dev, act, (batch, dim, L))
    _need(z, "z", dev, act, (batch, dim, L))
    _need(B, "B", dev, act, (batch, N, L))
    _need(C, "C", dev, act, (batch, N, L))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    if out is None:
        out = torch.empty_like(u)
    _need(out, "out", dev, act, (batch, dim, L))
    want_state = return_last_state or last_state is not None
    if want_state and last_state is None:
        last_state = torch.empty((batch, dim, N), device=dev, dtype=torch.float32)
    _need(last_state, "last_state", dev, torch.float32, (batch, dim, N))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N))
    lib = load_library()
    if workspace is None and schedule == SCHEDULE_PERSISTENT:
        nbytes = lib.mamba_scan_workspace_size(batch, dim, L, N, _ACT[act])
        if nbytes:
            workspace = torch.empty(nbytes, device=dev, dtype=torch.uint8)
    if workspace is not None and (workspace.device != dev or not workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous tensor on the input device")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = [_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
            _ptr(delta_bias), int(bool(delta_softplus)), _ptr(out), _ptr(last_state),
            batch, dim, L, N, _ACT[act]]
    tun = Tuning(int(lanes_per_channel), int(threads_per_block), int(schedule),
                 int(chunk_timesteps))
    with torch.cuda.device(dev):
        if h0 is None:
            fn = "mamba_scan_fwd_ws"
            rc = lib.mamba_scan_fwd_ws(*args, ctypes.byref(tun), _ptr(workspace), ws_bytes,
                                       _stream(dev))
        else:
            fn = "mamba_scan_fwd_init"
            rc = lib.mamba_scan_fwd_init(*args[:9], _ptr(h0), *args[9:], ctypes.byref(tun),
                                         _ptr(workspace), ws_bytes, _stream(dev))
    _check(fn, rc)
    return (out, last_state) if want_state else out


def _need_strided(t: Optional[torch.Tensor], name: str, device, dtype, shape):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _stride3(t: Optional[torch.Tensor]) -> Stride3:
    return Stride3(0, 0, 0) if t is None else Stride3(*t.stride())


def mamba_scan_fwd_strided(u: torch.Tensor, delta: torch.Tensor, A: torch.Tensor,
                           B: torch.Tensor, C: torch.Tensor, D: Optional[torch.Tensor] = None,
                           z: Optional[torch.Tensor] = None,
                           delta_bias: Optional[torch.Tensor] = None,
                           delta_softplus: bool = True, out: Optional[torch.Tensor] = None,
                           last_state: Optional[torch.Tensor] = None,
                           return_last_state: bool = False, h0: Optional[torch.Tensor] = None,
                           lanes_per_channel: int = 0, threads_per_block: int = 0,
                           schedule: int = SCHEDULE_AUTO):
    """:func:`mamba_scan_fwd` on tensors with any strides: u, delta, z (and
    out) of logical shape (batch, dim, L) and B, C of (batch, N, L), each
    laid out however it is -- e.g. ``x.transpose(1, 2)`` of a (batch, L, dim)
    activation, or a slice of a wider projection output.  ``out`` is
    allocated channel-contiguous like u when u is.  Dense (batch, L, dim)
    activations with dense (batch, L, N) B / C run the block-local lane-split
    kernel (SCHEDULE_AUTO or SCHEDULE_LOCAL, lanes 0 / 2 / 4, no block size
    given); every other layout, or SCHEDULE_STATIC, the static kernel."""
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, seqlen)")
    batch, dim, L = u.shape
    if A.dim() != 2:
        raise ValueError("A must be (dim, dstate)")
    N = A.shape[1]
    dev, act = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _need_strided(t, name, dev, act, (batch, dim, L))
    _need_strided(B, "B", dev, act, (batch, N, L))
    _need_strided(C, "C", dev, act, (batch, N, L))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    if out is None:
        if u.stride(1) == 1 and L > 1:
            out = torch.empty((batch, L, dim), device=dev, dtype=act).transpose(1, 2)
        else:
            out = torch.empty((batch, dim, L), device=dev, dtype=act)
    _need_strided(out, "out", dev, act, (batch, dim, L))
    want_state = return_last_state or last_state is not None
    if want_state and last_state is None:
        last_state = torch.empty((batch, dim, N), device=dev, dtype=torch.float32)
    _need(last_state, "last_state", dev, torch.float32, (batch, dim, N))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N))
    st = ScanStrides(_stride3(u), _stride3(delta), _stride3(z), _stride3(out), _stride3(B), _stride3(C))
    tun = Tuning(int(lanes_per_channel), int(threads_per_block), int(schedule), 0)
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_scan_fwd_strided(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(out),
                                        _ptr(last_state), batch, dim, L, N, _ACT[act], ctypes.byref(st),
                                        ctypes.byref(tun), _stream(dev))
    _check("mamba_scan_fwd_strided", rc)
    return (out, last_state) if want_state else out


def mamba_scan_fwd_complex(u: torch.Tensor, delta: torch.Tensor, A: torch.Tensor,
                           B: torch.Tensor, C: torch.Tensor, D: Optional[torch.Tensor] = None,
                           z: Optional[torch.Tensor] = None,
                           delta_bias: Optional[torch.Tensor] = None,
                           delta_softplus: bool = True, out: Optional[torch.Tensor] = None,
                           last_state: Optional[torch.Tensor] = None,
                           return_last_state: bool = False, h0: Optional[torch.Tensor] = None,
                           lanes_per_channel: int = 0):
    """Complex-valued mode.  u, delta, z: (batch, dim, L) in the activation
    dtype; A: (dim, N, 2) fp32 (re, im); B, C: (batch, N, L, 2) in the
    activation dtype; h0 / last_state: (batch, dim, N, 2) fp32.  Returns
    ``out`` or ``(out, last_state)``."""
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, seqlen)")
    batch, dim, L = u.shape
    if A.dim() != 3 or A.shape[2] != 2:
        raise ValueError("A must be (dim, dstate, 2)")
    N = A.shape[1]
    dev, act = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _need(t, name, dev, act, (batch, dim, L))
    _need(B, "B", dev, act, (batch, N, L, 2))
    _need(C, "C", dev, act, (batch, N, L, 2))
    _need(A, "A", dev, torch.float32, (dim, N, 2))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    if out is None:
        out = torch.empty_like(u)
    _need(out, "out", dev, act, (batch, dim, L))
    want_state = return_last_state or last_state is not None
    if want_state and last_state is None:
        last_state = torch.empty((batch, dim, N, 2), device=dev, dtype=torch.float32)
    _need(last_state, "last_state", dev, torch.float32, (batch, dim, N, 2))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N, 2))
    tun = Tuning(int(lanes_per_channel), 0, SCHEDULE_AUTO, 0)
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_scan_fwd_complex(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                        _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(out),
                                        _ptr(last_state), batch, dim, L, N, _ACT[act], ctypes.byref(tun),
                                        _stream(dev))
    _check("mamba_scan_fwd_complex", rc)
    return (out, last_state) if want_state else out


def _rows(t: Optional[torch.Tensor], name: str, device, dtype, batch: int, dim: int, L: int) -> int:
    """Batch stride of a (batch, >= dim, L) tensor whose rows are dense."""
    if t is None:
        return 0
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if t.dim() != 3 or t.shape[0] != batch or t.shape[1] < dim or t.shape[2] != L:
        raise ValueError(f"{name} must be (batch, >= {dim}, {L}), got {tuple(t.shape)}")
    if t.stride(2) != 1 or (t.shape[1] > 1 and t.stride(1) != L):
        raise ValueError(f"{name} rows must be dense (strides (*, L, 1))")
    return int(t.stride(0)) if batch > 1 else int(t.shape[1]) * L


def mamba_scan_fwd_conv(x: torch.Tensor, conv_weight: torch.Tensor, conv_bias: Optional[torch.Tensor],
                        delta: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
                        D: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                        delta_bias: Optional[torch.Tensor] = None, h0: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, last_state: Optional[torch.Tensor] = None,
                        return_last_state: bool = False, return_u: bool = False,
                        workspace: Optional[torch.Tensor] = None):
    """Causal depthwise conv1d + silu fused into the scan (softplus on).

    x: (batch, >= dim, L) -- the first ``dim`` channel rows are the conv
    input (so the in-projection's (batch, 2 dim, L) output can be passed
    whole); z: None or (batch, >= dim, L) likewise (e.g. ``xz[:, dim:]``);
    dim = delta.shape[1].  conv_weight (dim, K <= 4), conv_bias (dim,) fp32.
    Returns out, plus last_state and / or u when asked, in that order."""
    if delta.dim() != 3:
        raise ValueError("delta must be (batch, dim, seqlen)")
    batch, dim, L = delta.shape
    N = A.shape[1]
    dev, act = delta.device, delta.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    xbs = _rows(x, "x", dev, act, batch, dim, L)
    zbs = _rows(z, "z", dev, act, batch, dim, L)
    if conv_weight.dim() != 2 or conv_weight.shape[0] != dim:
        raise ValueError("conv_weight must be (dim, width)")
    K = conv_weight.shape[1]
    _need(conv_weight, "conv_weight", dev, torch.float32, (dim, K))
    _need(conv_bias, "conv_bias", dev, torch.float32, (dim,))
    _need(delta, "delta", dev, act, (batch, dim, L))
    _need(B, "B", dev, act, (batch, N, L))
    _need(C, "C", dev, act, (batch, N, L))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N))
    if out is None:
        out = torch.empty_like(delta)
    _need(out, "out", dev, act, (batch, dim, L))
    want_state = return_last_state or last_state is not None
    if want_state and last_state is None:
        last_state = torch.empty((batch, dim, N), device=dev, dtype=torch.float32)
    _need(last_state, "last_state", dev, torch.float32, (batch, dim, N))
    u = torch.empty_like(delta) if return_u else None
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(max(1, lib.mamba_scan_workspace_size(batch, dim, L, N, _ACT[act])),
                                device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        rc = lib.mamba_scan_fwd_conv(_ptr(x), _ptr(conv_weight), _ptr(conv_bias), K, xbs, _ptr(delta), _ptr(A),
                                     _ptr(B), _ptr(C), _ptr(D), _ptr(z), zbs, _ptr(delta_bias), _ptr(h0),
                                     _ptr(out), _ptr(last_state), _ptr(u), batch, dim, L, N, _ACT[act],
                                     _ptr(workspace), workspace.numel(), _stream(dev))
    _check("mamba_scan_fwd_conv", rc)
    res = (out,) + ((last_state,) if want_state else ()) + ((u,) if return_u else ())
    return res[0] if len(res) == 1 else res


def mamba_scan_fwd_host(u: torch.Tensor, delta: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                        C: torch.Tensor, D: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                        delta_bias: Optional[torch.Tensor] = None, delta_softplus: bool = True,
                        h0: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                        last_state: Optional[torch.Tensor] = None, return_last_state: bool = False,
                        scratch: Optional[torch.Tensor] = None):
    """The scan on sequences in host memory (ideally pinned): u, delta, z, B,
    C on the CPU; A, D, delta_bias (and h0) on the GPU.  Returns host
    ``out`` (and host ``last_state``).  Runs on the current stream of A's
    device; the results are ready once that stream has reached this point."""
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, seqlen)")
    batch, dim, L = u.shape
    N = A.shape[1]
    dev, act = A.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("A, D, delta_bias must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    cpu = torch.device("cpu")
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _need(t, name, cpu, act, (batch, dim, L))
    _need(B, "B", cpu, act, (batch, N, L))
    _need(C, "C", cpu, act, (batch, N, L))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N))
    if out is None:
        out = torch.empty((batch, dim, L), dtype=act, pin_memory=u.is_pinned())
    _need(out, "out", cpu, act, (batch, dim, L))
    want_state = return_last_state or last_state is not None
    if want_state and last_state is None:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, pin_memory=u.is_pinned())
    _need(last_state, "last_state", cpu, torch.float32, (batch, dim, N))
    lib = load_library()
    if scratch is None:
        scratch = torch.empty(lib.mamba_scan_host_scratch_size(batch, dim, L, N, _ACT[act]), device=dev,
                              dtype=torch.uint8)
    with torch.cuda.device(dev):
        rc = lib.mamba_scan_fwd_host(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                     _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(out),
                                     _ptr(last_state), batch, dim, L, N, _ACT[act], _ptr(scratch),
                                     scratch.numel(), _stream(dev))
    _check("mamba_scan_fwd_host", rc)
    return (out, last_state) if want_state else out


def mamba_scan_state(u: torch.Tensor, delta: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                     delta_bias: Optional[torch.Tensor] = None, delta_softplus: bool = True,
                     h0: Optional[torch.Tensor] = None, last_state: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The final state of the scan alone (no readout, gate or outputs):
    u, delta (batch, dim, L), B (batch, N, L) in the activation dtype; A
    (dim, N) fp32; h0 / the returned last_state (batch, dim, N) fp32.  Raises
    MambaError (MAMBA_ERR_UNSUPPORTED) where the lane-split kernel cannot run
    (dstate > 16, rows not whole 16-byte vectors)."""
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, seqlen)")
    batch, dim, L = u.shape
    N = A.shape[1] if A.dim() == 2 else -1
    dev, act = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    _need(delta, "delta", dev, act, (batch, dim, L))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(B, "B", dev, act, (batch, N, L))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N))
    if last_state is None:
        last_state = torch.empty((batch, dim, N), device=dev, dtype=torch.float32)
    _need(last_state, "last_state", dev, torch.float32, (batch, dim, N))
    ws_bytes = 0
    if workspace is not None:
        if workspace.device != dev:
            raise ValueError("workspace must be on the tensors' device")
        ws_bytes = workspace.numel() * workspace.element_size()
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_scan_state(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(delta_bias),
                                  int(bool(delta_softplus)), _ptr(h0), _ptr(last_state), batch, dim, L, N,
                                  _ACT[act], _ptr(workspace), ws_bytes, _stream(dev))
    _check("mamba_scan_state", rc)
    return last_state


def mamba_delta_sum(delta: torch.Tensor, delta_bias: Optional[torch.Tensor] = None,
                    delta_softplus: bool = True) -> torch.Tensor:
    """Per-row sum over time of delta after bias and softplus: (batch, dim)
    fp64."""
    if delta.dim() != 3:
        raise ValueError("delta must be (batch, dim, seqlen)")
    batch, dim, L = delta.shape
    dev, act = delta.device, delta.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    _need(delta, "delta", dev, act, (batch, dim, L))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    out = torch.empty((batch, dim), device=dev, dtype=torch.float64)
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_delta_sum(_ptr(delta), _ptr(delta_bias), int(bool(delta_softplus)), _ptr(out),
                                 batch, dim, L, _ACT[act], _stream(dev))
    _check("mamba_delta_sum", rc)
    return out


def mamba_state_fold(A: torch.Tensor, delta_sums: torch.Tensor, h_local: torch.Tensor,
                     h_init: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The state after ``count`` shards from ``h_init`` (zeros if None):
    delta_sums (count, batch, dim) fp64, h_local (count, batch, dim, N)
    fp32; returns (batch, dim, N) fp32."""
    if h_local.dim() != 4:
        raise ValueError("h_local must be (count, batch, dim, dstate)")
    count, batch, dim, N = h_local.shape
    dev = A.device
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(delta_sums, "delta_sums", dev, torch.float64, (count, batch, dim))
    _need(h_local, "h_local", dev, torch.float32, (count, batch, dim, N))
    _need(h_init, "h_init", dev, torch.float32, (batch, dim, N))
    if out is None:
        out = torch.empty((batch, dim, N), device=dev, dtype=torch.float32)
    _need(out, "out", dev, torch.float32, (batch, dim, N))
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_state_fold(_ptr(h_init), _ptr(delta_sums), _ptr(A), _ptr(h_local), _ptr(out),
                                  batch, dim, N, count, _stream(dev))
    _check("mamba_state_fold", rc)
    return out


def device_status(device=None) -> int:
    """Synchronise the current stream and return the library's device status
    (0 = ok, MAMBA_ERR_TIMEOUT after a bounded wait gave up, MAMBA_ERR_CUDA
    after a CUDA error)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return load_library().mamba_get_device_status(_stream(dev))


def load_checked_library() -> ctypes.CDLL:
    """The bounds-checked build of the library (built with nvcc first if it
    is missing or older than its sources), declared like the normal one.
    The binding keeps using the normal library; a caller that wants the
    checked one for the binding's functions sets it in their place."""
    with _lock:
        if _build.CHECKED_LIB not in _checked:
            if not _build.up_to_date(checked=True):
                _build.build(checked=True)
            _checked[_build.CHECKED_LIB] = _declare(ctypes.CDLL(_build.CHECKED_LIB))
        return _checked[_build.CHECKED_LIB]


_checked = {}


def bounds_status(lib: Optional[ctypes.CDLL] = None):
    """The first access outside its tensor that a bounds-checked launch
    skipped since the previous call, as (site, byte offset), or None; clears
    the record (the normal build always returns None).  Call after the work
    has completed."""
    lib = lib or load_library()
    site, off = ctypes.c_int(0), ctypes.c_longlong(0)
    rc = lib.mamba_debug_bounds_status(ctypes.c_void_p(ctypes.addressof(site)), ctypes.c_void_p(ctypes.addressof(off)))
    if rc < 0:
        _check("mamba_debug_bounds_status", rc)
    return (site.value, off.value) if rc else None


def workspace_status(workspace: torch.Tensor) -> int:
    """Synchronise the current stream and return the status word a persistent
    launch left in ``workspace`` (0 = ok, MAMBA_ERR_TIMEOUT otherwise)."""
    with torch.cuda.device(workspace.device):
        return load_library().mamba_scan_workspace_status(_ptr(workspace), _stream(workspace.device))


def mamba_scan_workspace_size(batch: int, dim: int, seqlen: int, dstate: int,
                              dtype: torch.dtype = torch.bfloat16) -> int:
    return int(load_library().mamba_scan_workspace_size(batch, dim, seqlen, dstate, _ACT[dtype]))


def mamba_scan_plan(batch: int, dim: int, seqlen: int, dstate: int,
                    dtype: torch.dtype = torch.bfloat16, workspace: bool = True) -> Tuple[int, int, int]:
    """(lanes_per_channel, threads_per_block, schedule) the library picks for a
    shape on the current device, with aligned tensors and a workspace
    (``workspace=False``: what the no-workspace call picks)."""
    t = Tuning()
    lib = load_library()
    fn = lib.mamba_scan_plan if workspace else lib.mamba_scan_plan_noworkspace
    _check("mamba_scan_plan", fn(batch, dim, seqlen, dstate, _ACT[dtype], ctypes.byref(t)))
    return t.lanes_per_channel, t.threads_per_block, t.schedule


def mamba_state_update(state: torch.Tensor, u: torch.Tensor, delta: torch.Tensor,
                       A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
                       D: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                       delta_bias: Optional[torch.Tensor] = None,
                       delta_softplus: bool = True,
                       out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One recurrent step, updating ``state`` (batch, dim, N) fp32 in place.

    u, delta, z: (batch, dim); B, C: (batch, N) in one dtype.  Returns out
    (batch, dim)."""
    if state.dim() != 3:
        raise ValueError("state must be (batch, dim, dstate)")
    batch, dim, N = state.shape
    dev, act = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    _need(state, "state", dev, torch.float32, (batch, dim, N))
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _need(t, name, dev, act, (batch, dim))
    _need(B, "B", dev, act, (batch, N))
    _need(C, "C", dev, act, (batch, N))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    if out is None:
        out = torch.empty_like(u)
    _need(out, "out", dev, act, (batch, dim))
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_state_update(_ptr(state), _ptr(u), _ptr(delta), _ptr(A), _ptr(B),
                                    _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                    int(bool(delta_softplus)), _ptr(out), batch, dim, N,
                                    _ACT[act], _stream(dev))
    _check("mamba_state_update", rc)
    return out


def mamba_conv1d_fwd(x: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     apply_silu: bool = True, dim: Optional[int] = None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Causal depthwise conv1d + bias (+ silu) on the current CUDA stream.

    x: contiguous (batch, C, L) with C >= dim; the first ``dim`` channel rows
    are convolved (``dim`` defaults to C), so the x half of a (batch, 2 dim, L)
    projection output can be passed as is.  weight: (dim, K) fp32, K <= 4;
    bias: (dim,) fp32.  Returns out (batch, dim, L) in x's dtype."""
    if x.dim() != 3:
        raise ValueError("x must be (batch, channels, L)")
    batch, C, L = x.shape
    dim = C if dim is None else int(dim)
    dev, act = x.device, x.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    if not x.is_contiguous() or dim > C:
        raise ValueError("x must be contiguous with at least dim channel rows")
    if weight.dim() != 2:
        raise ValueError("weight must be (dim, width)")
    K = weight.shape[1]
    _need(weight, "weight", dev, torch.float32, (dim, K))
    _need(bias, "bias", dev, torch.float32, (dim,))
    if out is None:
        out = torch.empty(batch, dim, L, device=dev, dtype=act)
    _need(out, "out", dev, act, (batch, dim, L))
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_conv1d_fwd(_ptr(x), _ptr(weight), _ptr(bias), int(bool(apply_silu)), _ptr(out),
                                  batch, dim, L, K, C * L, _ACT[act], _stream(dev))
    _check("mamba_conv1d_fwd", rc)
    return out


def mamba_conv1d_update(conv_state: Optional[torch.Tensor], x: torch.Tensor, weight: torch.Tensor,
                        bias: Optional[torch.Tensor] = None, apply_silu: bool = True,
                        out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One token of :func:`mamba_conv1d_fwd`.  conv_state: (batch, dim, K-1)
    fp32, oldest input first, updated in place (None when K is 1); x:
    (batch, dim).  Returns out (batch, dim)."""
    if x.dim() != 2:
        raise ValueError("x must be (batch, dim)")
    batch, dim = x.shape
    dev, act = x.device, x.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    if weight.dim() != 2:
        raise ValueError("weight must be (dim, width)")
    K = weight.shape[1]
    _need(x, "x", dev, act, (batch, dim))
    _need(weight, "weight", dev, torch.float32, (dim, K))
    _need(bias, "bias", dev, torch.float32, (dim,))
    if K > 1 and conv_state is None:
        raise ValueError("conv_state is required for width > 1")
    _need(conv_state, "conv_state", dev, torch.float32, (batch, dim, K - 1))
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", dev, act, (batch, dim))
    lib = load_library()
    with torch.cuda.device(dev):
        rc = lib.mamba_conv1d_update(_ptr(conv_state), _ptr(x), _ptr(weight), _ptr(bias),
                                     int(bool(apply_silu)), _ptr(out), batch, dim, K, dim,
                                     _ACT[act], _stream(dev))
    _check("mamba_conv1d_update", rc)
    return out


def mamba_scan_ckpt_size(batch: int, dim: int, seqlen: int, dstate: int) -> int:
    """Bytes of the checkpoints :func:`mamba_scan_fwd_ckpt` writes."""
    return int(load_library().mamba_scan_ckpt_size(batch, dim, seqlen, dstate))


def mamba_scan_fwd_ckpt(u: torch.Tensor, delta: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                        C: torch.Tensor, D: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                        delta_bias: Optional[torch.Tensor] = None, delta_softplus: bool = True,
                        h0: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                        last_state: Optional[torch.Tensor] = None, ckpt: Optional[torch.Tensor] = None):
    """:func:`mamba_scan_fwd` that also keeps the state every 32 steps for
    the backward pass.  Returns (out, last_state, ckpt); pass ``ckpt`` to
    :func:`mamba_scan_bwd`."""
    batch, dim, L = u.shape
    N = A.shape[1]
    dev, act = u.device, u.dtype
    if dev.type != "cuda" or act not in _ACT:
        raise ValueError("u must be a float32 or bfloat16 CUDA tensor")
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _need(t, name, dev, act, (batch, dim, L))
    _need(B, "B", dev, act, (batch, N, L))
    _need(C, "C", dev, act, (batch, N, L))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N))
    lib = load_library()
    out = torch.empty_like(u) if out is None else out
    last_state = torch.empty(batch, dim, N, device=dev, dtype=torch.float32) if last_state is None else last_state
    _need(out, "out", dev, act, (batch, dim, L))
    _need(last_state, "last_state", dev, torch.float32, (batch, dim, N))
    nbytes = lib.mamba_scan_ckpt_size(batch, dim, L, N)
    if ckpt is None:
        ckpt = torch.empty(max(nbytes // 4, 1), device=dev, dtype=torch.float32)
    with torch.cuda.device(dev):
        rc = lib.mamba_scan_fwd_ckpt(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                     _ptr(delta_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(out),
                                     _ptr(last_state), _ptr(ckpt), ckpt.numel() * ckpt.element_size(),
                                     batch, dim, L, N, _ACT[act], _stream(dev))
    _check("mamba_scan_fwd_ckpt", rc)
    return out, last_state, ckpt


def mamba_scan_bwd(dout: torch.Tensor, u: torch.Tensor, delta: torch.Tensor, A: torch.Tensor,
                   B: torch.Tensor, C: torch.Tensor, D: Optional[torch.Tensor] = None,
                   z: Optional[torch.Tensor] = None, delta_bias: Optional[torch.Tensor] = None,
                   delta_softplus: bool = True, dlast_state: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   h0: Optional[torch.Tensor] = None, ckpt: Optional[torch.Tensor] = None) -> dict:
    """Gradients of :func:`mamba_scan_fwd` for dL/dout = ``dout`` (and
    dL/dlast_state = ``dlast_state``).  Returns a dict: du, ddelta, dz (act
    dtype, like u; dz None without z), dA (dim, N), dB, dC (batch, N, L),
    dD, ddelta_bias (dim,) -- fp32 (dD / ddelta_bias None when D / the bias
    are not given) -- and dh0 (batch, dim, N) fp32 when the forward started
    from the state ``h0`` (else None).  ``ckpt``: the checkpoints
    :func:`mamba_scan_fwd_ckpt` wrote for the same inputs (and h0), which
    spares the backward its own sweep over the inputs."""
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, L)")
    batch, dim, L = u.shape
    N = A.shape[-1]
    dev, act = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if act not in _ACT:
        raise TypeError(f"unsupported activation dtype {act}")
    for name, t in (("u", u), ("delta", delta), ("z", z), ("dout", dout)):
        _need(t, name, dev, act, (batch, dim, L))
    _need(B, "B", dev, act, (batch, N, L))
    _need(C, "C", dev, act, (batch, N, L))
    _need(A, "A", dev, torch.float32, (dim, N))
    _need(D, "D", dev, torch.float32, (dim,))
    _need(delta_bias, "delta_bias", dev, torch.float32, (dim,))
    _need(dlast_state, "dlast_state", dev, torch.float32, (batch, dim, N))
    _need(h0, "h0", dev, torch.float32, (batch, dim, N))
    lib = load_library()
    need = lib.mamba_scan_bwd_workspace_size(batch, dim, L, N)
    if need == 0:
        raise MambaError("mamba_scan_bwd", -3, "unsupported sizes (dstate <= 16)")
    if workspace is None:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    f32 = dict(device=dev, dtype=torch.float32)
    r = {"du": torch.empty_like(u), "ddelta": torch.empty_like(u),
         "dz": torch.empty_like(u) if z is not None else None,
         "dA": torch.empty(dim, N, **f32), "dB": torch.empty(batch, N, L, **f32),
         "dC": torch.empty(batch, N, L, **f32),
         "dD": torch.empty(dim, **f32) if D is not None else None,
         "ddelta_bias": torch.empty(dim, **f32) if delta_bias is not None else None,
         "dh0": torch.empty(batch, dim, N, **f32) if h0 is not None else None}
    head = [_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(delta_softplus))]
    grads = [_ptr(dout), _ptr(dlast_state), _ptr(r["du"]), _ptr(r["ddelta"]), _ptr(r["dA"]),
             _ptr(r["dB"]), _ptr(r["dC"]), _ptr(r["dD"]), _ptr(r["dz"]), _ptr(r["ddelta_bias"])]
    tail = [batch, dim, L, N, _ACT[act], _ptr(workspace), workspace.numel(), _stream(dev)]
    if ckpt is not None:
        need_ck = lib.mamba_scan_ckpt_size(batch, dim, L, N)
        if ckpt.device != dev or not ckpt.is_contiguous() or ckpt.numel() * ckpt.element_size() < need_ck:
            raise ValueError("ckpt must be a contiguous device tensor of mamba_scan_ckpt_size bytes")
    with torch.cuda.device(dev):
        if ckpt is not None:
            fn = "mamba_scan_bwd_ckpt"
            rc = lib.mamba_scan_bwd_ckpt(*head, _ptr(h0), _ptr(ckpt), *grads, _ptr(r["dh0"]), *tail)
        elif h0 is None:
            fn = "mamba_scan_bwd"
            rc = lib.mamba_scan_bwd(*head, *grads, *tail)
        else:
            fn = "mamba_scan_bwd_init"
            rc = lib.mamba_scan_bwd_init(*head, _ptr(h0), *grads, _ptr(r["dh0"]), *tail)
    _check(fn, rc)
    return r
