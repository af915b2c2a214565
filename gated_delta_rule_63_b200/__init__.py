"""Gated delta-rule layer on NVIDIA B200 (sm_100a): Python binding of libgdr.so.

A thin ctypes layer over the C ABI declared in ``include/gdr.h``: each function
checks dtypes and shapes, passes raw device pointers and the current CUDA
stream, and raises ``GdrError`` on a non-zero status.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback path.
PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

__all__ = [
    "GdrError", "lib", "status_string", "prepare_chunks", "causal_conv", "chunk_prefill",
    "chunk_prefill_noalloc", "chunk_prefill_slots", "prefill_schedule", "prefill_workspace", "linear", "prefill_fused_workspace", "prefill_window",
    "decode_step", "decode_step_slots", "gated_rmsnorm", "get_device_error", "debug_wait_timeout",
    "HEAD_DIM", "CHUNK",
]

HEAD_DIM = 128
CHUNK = 64
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdr.so")

_vp = ctypes.c_void_p
_ip = ctypes.POINTER(ctypes.c_int32)


class GdrError(RuntimeError):
    def __init__(self, fn: str, code: int):
        detail = lib().gdr_last_error_string().decode() if code == 7 else ""
        super().__init__(f"{fn}: {status_string(code)} (status {code})" + (f" [{detail}]" if detail else ""))
        self.code = code


class FuseArgs(ctypes.Structure):
    """Mirror of ``gdr_prefill_fuse_t``."""
    _fields_ = [("x", _vp), ("conv_w", _vp), ("conv_state_in", _vp), ("conv_state_out", _vp),
                ("z", _vp), ("norm_w", _vp), ("eps", ctypes.c_float), ("y", _vp)]


_lib = None


def lib(path: Optional[str] = None):
    """Load libgdr.so (built in-tree by ``gated_delta_rule_63_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m gated_delta_rule_63_b200.build`")
    L = ctypes.CDLL(path)
    L.gdr_status_string.restype = ctypes.c_char_p
    L.gdr_status_string.argtypes = [ctypes.c_int]
    L.gdr_abi_version.restype = ctypes.c_int
    L.gdr_last_error_string.restype = ctypes.c_char_p
    L.gdr_last_error_string.argtypes = []
    L.gdr_prepare_chunks.argtypes = [_ip, ctypes.c_int, ctypes.c_int, _ip, _ip, _ip, ctypes.c_int,
                                     ctypes.POINTER(ctypes.c_int)]
    L.gdr_causal_conv.argtypes = [_vp, _vp, _vp, _vp, _vp, _ip, ctypes.c_int, ctypes.c_int, _vp, _vp]
    L.gdr_chunk_prefill.argtypes = [_vp, _vp, _vp, ctypes.c_int64, ctypes.c_int64, _vp, _vp, _vp,
                                    _vp, ctypes.c_float, ctypes.c_int,
                                    ctypes.c_int, _vp, _ip, ctypes.c_int, _vp, _vp, _vp,
                                    ctypes.POINTER(FuseArgs), _vp, ctypes.c_size_t, _vp]
    L.gdr_chunk_prefill_noalloc.argtypes = [_vp, _vp, _vp, ctypes.c_int64, ctypes.c_int64, _vp, _vp,
                                            _vp, _vp, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                            _vp, _ip, ctypes.c_int, _vp, _vp, _vp, _vp]
    L.gdr_chunk_prefill_noalloc.restype = ctypes.c_int
    L.gdr_chunk_prefill_noalloc_scratch_bytes.restype = ctypes.c_size_t
    L.gdr_chunk_prefill_noalloc_scratch_bytes.argtypes = []
    L.gdr_chunk_prefill_fused_workspace_size.restype = ctypes.c_size_t
    L.gdr_chunk_prefill_fused_workspace_size.argtypes = [ctypes.c_int] * 6
    L.gdr_chunk_prefill_workspace_size.restype = ctypes.c_size_t
    L.gdr_chunk_prefill_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int]
    L.gdr_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_int,
                                  ctypes.c_int, _vp, _vp, ctypes.c_int, _vp]
    L.gdr_decode_step_slots.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_int,
                                        ctypes.c_int, _vp, ctypes.c_int, _vp, _vp, ctypes.c_int, _vp]
    L.gdr_gated_rmsnorm.argtypes = [_vp, _vp, _vp, ctypes.c_float, ctypes.c_int64, ctypes.c_int, _vp,
                                    _vp]
    L.gdr_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), _vp]
    L.gdr_debug_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_ulonglong, _vp, _vp]
    L.gdr_chunk_prefill_slots.argtypes = [_vp, _vp, _vp, ctypes.c_int64, ctypes.c_int64, _vp, _vp, _vp, _vp,
                                          ctypes.c_float, ctypes.c_int, ctypes.c_int, _vp, _ip, ctypes.c_int,
                                          _vp, ctypes.c_int, _vp, ctypes.c_int, _vp, _vp, ctypes.c_size_t, _vp]
    L.gdr_linear.argtypes = [_vp, _vp, _vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _vp]
    L.gdr_chunk_prefill_schedule.argtypes = [_ip, ctypes.c_int, ctypes.c_int, ctypes.c_size_t, ctypes.c_int,
                                             ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    for fn in ("gdr_prepare_chunks", "gdr_causal_conv", "gdr_chunk_prefill", "gdr_decode_step",
               "gdr_decode_step_slots", "gdr_gated_rmsnorm", "gdr_get_device_error",
               "gdr_debug_wait_timeout", "gdr_chunk_prefill_slots", "gdr_chunk_prefill_schedule", "gdr_linear"):
        getattr(L, fn).restype = ctypes.c_int
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().gdr_status_string(int(code)).decode()


def _check(fn: str, code: int):
    if code != 0:
        raise GdrError(fn, code)


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t, dtype=None, name="tensor", rows=False):
    """Device pointer of a tensor; with rows=True only the last two dims must be dense."""
    if t is None:
        return None
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if rows:
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must be [T, heads, 128] with dense rows")
    elif not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _tok_stride(t):
    return 0 if t is None else int(t.stride(0))


def _device_of(*tensors):
    """The one device of the given tensors (None skipped); tensors on two devices raise.

    Each call runs on that device with its stream, so no kernel is handed a pointer into
    another GPU's memory."""
    dev = None
    for t in tensors:
        d = getattr(t, "device", None)
        if d is None or d.type != "cuda":
            continue   # not a CUDA tensor: _ptr rejects it by name
        if dev is None:
            dev = d
        elif d != dev:
            raise ValueError(f"tensors on {dev} and {d}: all tensors of a call must be on one device")
    return dev


def _stream(stream=None, device=None):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if device is not None and getattr(stream, "device", device) != device:
        raise ValueError(f"stream on {stream.device}, tensors on {device}")
    return stream.cuda_stream


def _host_cu(cu_host):
    cu = np.ascontiguousarray(np.asarray(cu_host), dtype=np.int32)
    return cu, cu.ctypes.data_as(_ip)


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def prepare_chunks(cu_seqlens_host, chunk: int = CHUNK):
    """Chunk table (chunk_seq, chunk_start, chunk_len) of packed sequences."""
    cu, cup = _host_cu(cu_seqlens_host)
    n = cu.shape[0] - 1
    total = int(cu[-1]) if n > 0 else 0
    cap = max(1, total // max(chunk, 1) + n + 1)
    seq = np.zeros(cap, np.int32); st = np.zeros(cap, np.int32); ln = np.zeros(cap, np.int32)
    m = ctypes.c_int(0)
    _check("gdr_prepare_chunks", lib().gdr_prepare_chunks(
        cup, n, int(chunk), seq.ctypes.data_as(_ip), st.ctypes.data_as(_ip), ln.ctypes.data_as(_ip),
        cap, ctypes.byref(m)))
    k = m.value
    return seq[:k].copy(), st[:k].copy(), ln[:k].copy()


def causal_conv(x, w, cu_seqlens, cu_seqlens_host, conv_state_in=None, conv_state_out=None, y=None,
                stream=None):
    """Depthwise causal conv4 + SiLU.  x [T, C] bf16, w [C, 4] bf16 -> y [T, C] bf16."""
    torch = _torch()
    bf = torch.bfloat16
    cu, cup = _host_cu(cu_seqlens_host)
    if y is None:
        y = torch.empty_like(x)
    C = x.shape[1]
    dev = _device_of(x, w, conv_state_in, conv_state_out, cu_seqlens, y)
    with torch.cuda.device(dev):
        _check("gdr_causal_conv", lib().gdr_causal_conv(
            _ptr(x, bf, "x"), _ptr(w, bf, "w"), _ptr(conv_state_in, bf, "conv_state_in"),
            _ptr(conv_state_out, bf, "conv_state_out"), _ptr(cu_seqlens, torch.int32, "cu_seqlens"), cup,
            cu.shape[0] - 1, C, _ptr(y, bf, "y"), _stream(stream, dev)))
    return y


DEFAULT_WORKSPACE_BYTES = 512 << 20


def prefill_window(cu_seqlens_host, hv: int, max_bytes: int = DEFAULT_WORKSPACE_BYTES,
                   has_final_state: bool = True) -> int:
    """Largest chunk window (<= the longest sequence) whose workspace fits max_bytes."""
    cu = np.asarray(cu_seqlens_host, dtype=np.int64)
    n = len(cu) - 1
    if n <= 0:
        return 1
    max_chunks = int(max(1, ((np.diff(cu) + CHUNK - 1) // CHUNK).max()))
    per_chunk = lib().gdr_chunk_prefill_workspace_size(n, hv, 1, 1)
    carry = lib().gdr_chunk_prefill_workspace_size(n, hv, 1, int(has_final_state)) - per_chunk
    fit = max(1, (max_bytes - carry) // per_chunk)
    return int(min(max_chunks, fit))


def prefill_schedule(cu_seqlens_host, hv: int, workspace_bytes: int, has_final_state: bool = True):
    """(windows, pipelined) of gdr_chunk_prefill for these sequences and workspace size on the
    current CUDA device: the number of windows (one operand launch and one state launch each)
    and whether the next window is built beside the current one's state walk."""
    cu, cup = _host_cu(cu_seqlens_host)
    w, pl = ctypes.c_int(0), ctypes.c_int(0)
    _check("gdr_chunk_prefill_schedule", lib().gdr_chunk_prefill_schedule(
        cup, cu.shape[0] - 1, int(hv), int(workspace_bytes), int(bool(has_final_state)), ctypes.byref(w),
        ctypes.byref(pl)))
    return w.value, bool(pl.value)


def prefill_workspace(cu_seqlens_host, hv: int, device, window: Optional[int] = None,
                      has_final_state: bool = True):
    """A torch uint8 device buffer sized for gdr_chunk_prefill."""
    torch = _torch()
    cu = np.asarray(cu_seqlens_host)
    n = len(cu) - 1
    if window is None:
        window = prefill_window(cu_seqlens_host, hv, has_final_state=has_final_state)
    nbytes = lib().gdr_chunk_prefill_workspace_size(max(n, 1), hv, max(int(window), 1),
                                                    int(has_final_state))
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def prefill_fused_workspace(cu_seqlens_host, hk: int, hv: int, device, window: Optional[int] = None,
                            has_final_state: bool = True):
    """Workspace for gdr_chunk_prefill running the conv in the same call: the conv output, then the records."""
    torch = _torch()
    cu = np.asarray(cu_seqlens_host)
    n = len(cu) - 1
    T = int(cu[-1]) if n > 0 else 0
    if window is None:
        window = prefill_window(cu_seqlens_host, hv, has_final_state=has_final_state)
    nbytes = lib().gdr_chunk_prefill_fused_workspace_size(max(n, 1), int(hk), int(hv), T, max(int(window), 1),
                                                          int(has_final_state))
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def chunk_prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens, cu_seqlens_host, h0=None, hT=None,
                  o=None, scale: float = 1.0, fuse: Optional[dict] = None, workspace=None,
                  window: Optional[int] = None, stream=None):
    """Chunk-64 prefill.  q, k [T, hk, 128], v [T, hv, 128], a, b [T, hv] bf16.

    q, k, v may be token-strided views (e.g. slices of the [T, q|k|v] conv output); with the
    conv run by the same call (``fuse`` holding "x", "conv_w" and "hk") they are None.

    Returns o [T, hv, 128] bf16 (and writes hT [N, hv, 128, 128] fp32 when given).
    ``fuse`` (optional) maps gdr_prefill_fuse_t field names to tensors.
    """
    torch = _torch()
    bf, f32 = torch.bfloat16, torch.float32
    cu, cup = _host_cu(cu_seqlens_host)
    fz = None
    if fuse is not None:
        fz = FuseArgs()
        for name in ("x", "conv_w", "conv_state_in", "conv_state_out", "z", "y"):
            setattr(fz, name, _ptr(fuse.get(name), bf, name))
        fz.norm_w = _ptr(fuse.get("norm_w"), f32, "norm_w")
        fz.eps = float(fuse.get("eps", 1e-6))
    hk = q.shape[1] if q is not None else int(fuse["hk"])
    hv = a.shape[1]
    if q is not None and k.stride(0) != q.stride(0):
        raise ValueError("q and k must share their token stride")
    if o is None and (fuse is None or fuse.get("y") is None or fuse.get("keep_o", False)):
        T = a.shape[0]
        o = torch.empty((T, hv, HEAD_DIM), dtype=bf, device=a.device)
    if workspace is None:
        if fuse is not None and fuse.get("x") is not None:
            workspace = prefill_fused_workspace(cu_seqlens_host, hk, hv, a.device, window, hT is not None)
        else:
            workspace = prefill_workspace(cu_seqlens_host, hv, a.device, window, hT is not None)
    fuse_tensors = [fuse.get(n) for n in ("x", "conv_w", "conv_state_in", "conv_state_out", "z", "y",
                                          "norm_w")] if fuse is not None else []
    dev = _device_of(q, k, v, a, b, A_log, dt_bias, cu_seqlens, h0, hT, o, workspace, *fuse_tensors)
    with torch.cuda.device(dev):
        _check("gdr_chunk_prefill", lib().gdr_chunk_prefill(
            _ptr(q, bf, "q", rows=True), _ptr(k, bf, "k", rows=True), _ptr(v, bf, "v", rows=True),
            _tok_stride(q), _tok_stride(v), _ptr(a, bf, "a"), _ptr(b, bf, "b"),
            _ptr(A_log, f32, "A_log"), _ptr(dt_bias, f32, "dt_bias"), float(scale), int(hk), int(hv),
            _ptr(cu_seqlens, torch.int32, "cu_seqlens"), cup, cu.shape[0] - 1,
            _ptr(h0, f32, "h0"), _ptr(hT, f32, "hT"), _ptr(o, bf, "o"),
            ctypes.byref(fz) if fz is not None else None, _ptr(workspace, torch.uint8, "workspace"),
            int(workspace.numel()), _stream(stream, dev)))
    return o


def chunk_prefill_noalloc(q, k, v, a, b, A_log, dt_bias, cu_seqlens, cu_seqlens_host, h0=None,
                          hT=None, o=None, scale: float = 1.0, stream=None):
    """gdr_chunk_prefill on the library's own scratch array (no workspace argument).

    For callers that cannot allocate device memory; see gdr_chunk_prefill_noalloc
    in include/gdr.h for the size limit and the rule that calls must not overlap.
    """
    torch = _torch()
    bf, f32 = torch.bfloat16, torch.float32
    cu, cup = _host_cu(cu_seqlens_host)
    hv = a.shape[1]
    if o is None:
        o = torch.empty((a.shape[0], hv, HEAD_DIM), dtype=bf, device=a.device)
    dev = _device_of(q, k, v, a, b, A_log, dt_bias, cu_seqlens, h0, hT, o)
    with torch.cuda.device(dev):
        _check("gdr_chunk_prefill_noalloc", lib().gdr_chunk_prefill_noalloc(
            _ptr(q, bf, "q", rows=True), _ptr(k, bf, "k", rows=True), _ptr(v, bf, "v", rows=True),
            _tok_stride(q), _tok_stride(v), _ptr(a, bf, "a"), _ptr(b, bf, "b"),
            _ptr(A_log, f32, "A_log"), _ptr(dt_bias, f32, "dt_bias"), float(scale), int(q.shape[1]),
            int(hv), _ptr(cu_seqlens, torch.int32, "cu_seqlens"), cup, cu.shape[0] - 1,
            _ptr(h0, f32, "h0"), _ptr(hT, f32, "hT"), _ptr(o, bf, "o"), _stream(stream, dev)))
    return o


def chunk_prefill_slots(q, k, v, a, b, A_log, dt_bias, cu_seqlens, cu_seqlens_host, state_pool, slot,
                        init_from_pool: bool = False, o=None, scale: float = 1.0, workspace=None, stream=None):
    """gdr_chunk_prefill on a pool of cached states: sequence n starts from entry slot[n] of
    state_pool (or from zero, init_from_pool=False) and leaves its final state there.  A slot
    outside the pool is a sequence that starts from zero and keeps no state."""
    torch = _torch()
    bf, f32 = torch.bfloat16, torch.float32
    cu, cup = _host_cu(cu_seqlens_host)
    hv = a.shape[1]
    if o is None:
        o = torch.empty((a.shape[0], hv, HEAD_DIM), dtype=bf, device=a.device)
    if workspace is None:
        workspace = prefill_workspace(cu, hv, a.device, has_final_state=False)
    dev = _device_of(q, k, v, a, b, A_log, dt_bias, cu_seqlens, state_pool, slot, o, workspace)
    with torch.cuda.device(dev):
        _check("gdr_chunk_prefill_slots", lib().gdr_chunk_prefill_slots(
            _ptr(q, bf, "q", rows=True), _ptr(k, bf, "k", rows=True), _ptr(v, bf, "v", rows=True),
            _tok_stride(q), _tok_stride(v), _ptr(a, bf, "a"), _ptr(b, bf, "b"),
            _ptr(A_log, f32, "A_log"), _ptr(dt_bias, f32, "dt_bias"), float(scale), int(q.shape[1]),
            int(hv), _ptr(cu_seqlens, torch.int32, "cu_seqlens"), cup, cu.shape[0] - 1,
            _ptr(state_pool, f32, "state_pool"), int(state_pool.shape[0]), _ptr(slot, torch.int32, "slot"),
            int(bool(init_from_pool)), _ptr(o, bf, "o"), _ptr(workspace, torch.uint8, "workspace"),
            workspace.numel(), _stream(stream, dev)))
    return o


def decode_step(x, conv_w, conv_state, a, b, A_log, dt_bias, state, o=None, scale: float = 1.0,
                hk: int = 16, stream=None):
    """One token for each of B sequences; conv_state and state are updated in place."""
    torch = _torch()
    bf, f32 = torch.bfloat16, torch.float32
    B, hv = a.shape
    if o is None:
        o = torch.empty((B, hv, HEAD_DIM), dtype=bf, device=a.device)
    dev = _device_of(x, conv_w, conv_state, a, b, A_log, dt_bias, state, o)
    with torch.cuda.device(dev):
        _check("gdr_decode_step", lib().gdr_decode_step(
            _ptr(x, bf, "x"), _ptr(conv_w, bf, "conv_w"), _ptr(conv_state, bf, "conv_state"),
            _ptr(a, bf, "a"), _ptr(b, bf, "b"), _ptr(A_log, f32, "A_log"), _ptr(dt_bias, f32, "dt_bias"),
            float(scale), int(hk), int(hv), _ptr(state, f32, "state"), _ptr(o, bf, "o"), int(B),
            _stream(stream, dev)))
    return o


def decode_step_slots(x, conv_w, conv_state_pool, a, b, A_log, dt_bias, state_pool, slot, o=None,
                      scale: float = 1.0, hk: int = 16, stream=None):
    """One token for each of B rows; row i updates pool entry slot[i] of both pools in place.

    slot is an int32 CUDA tensor [B]; a slot outside [0, n_slots) is a padding row (zero o).
    """
    torch = _torch()
    bf, f32 = torch.bfloat16, torch.float32
    B, hv = a.shape
    n_slots = int(state_pool.shape[0])
    if tuple(slot.shape) != (B,):
        raise ValueError(f"slot must have shape ({B},), got {tuple(slot.shape)}")
    if int(conv_state_pool.shape[0]) != n_slots:
        raise ValueError("conv_state_pool and state_pool must hold the same number of slots")
    if o is None:
        o = torch.empty((B, hv, HEAD_DIM), dtype=bf, device=a.device)
    dev = _device_of(x, conv_w, conv_state_pool, a, b, A_log, dt_bias, state_pool, slot, o)
    with torch.cuda.device(dev):
        _check("gdr_decode_step_slots", lib().gdr_decode_step_slots(
            _ptr(x, bf, "x"), _ptr(conv_w, bf, "conv_w"), _ptr(conv_state_pool, bf, "conv_state_pool"),
            _ptr(a, bf, "a"), _ptr(b, bf, "b"), _ptr(A_log, f32, "A_log"), _ptr(dt_bias, f32, "dt_bias"),
            float(scale), int(hk), int(hv), _ptr(state_pool, f32, "state_pool"), n_slots,
            _ptr(slot, torch.int32, "slot"), _ptr(o, bf, "o"), int(B), _stream(stream, dev)))
    return o


def linear(x, w, y=None, stream=None):
    """y = x w^T: x [M, K], w [N, K] bf16 CUDA tensors (dense rows) -> y [M, N] bf16."""
    torch = _torch()
    bf = torch.bfloat16
    if x.dim() != 2 or w.dim() != 2 or x.shape[1] != w.shape[1]:
        raise ValueError("linear: x [M, K] and w [N, K] with the same K")
    M, K = x.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=bf, device=x.device)
    if tuple(y.shape) != (M, N):
        raise ValueError("linear: y must be [M, N]")
    dev = _device_of(x, w, y)
    with torch.cuda.device(dev):
        _check("gdr_linear", lib().gdr_linear(_ptr(x, bf, "x"), _ptr(w, bf, "w"), _ptr(y, bf, "y"), int(M), int(N),
                                              int(K), _stream(stream, dev)))
    return y


def gated_rmsnorm(o, z, w=None, eps: float = 1e-6, y=None, stream=None):
    """y = o / sqrt(mean(o^2) + eps) * w * SiLU(z) over rows of 128."""
    torch = _torch()
    bf = torch.bfloat16
    if y is None:
        y = torch.empty_like(o)
    d = o.shape[-1]
    rows = o.numel() // d
    dev = _device_of(o, z, w, y)
    with torch.cuda.device(dev):
        _check("gdr_gated_rmsnorm", lib().gdr_gated_rmsnorm(
            _ptr(o, bf, "o"), _ptr(z, bf, "z"), _ptr(w, torch.float32, "w"), float(eps), int(rows), int(d),
            _ptr(y, bf, "y"), _stream(stream, dev)))
    return y


def get_device_error(stream=None) -> int:
    """Read and clear the library's device error word (synchronises the stream)."""
    v = ctypes.c_int(0)
    _check("gdr_get_device_error", lib().gdr_get_device_error(ctypes.byref(v), _stream(stream)))
    return v.value


def debug_wait_timeout(kind: int, limit: int, device=None, stream=None) -> int:
    """Run the bounded-wait self-test kernel (gdr_debug_wait_timeout): one CTA waits on an
    mbarrier nothing arrives at until `limit` runs out (kind 0: polls, kind 1: SM cycles).
    Returns the kernel's own verdict (0 = the wait gave up); the device error word then holds
    GDR_ERR_TIMEOUT (read it with get_device_error)."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        res = torch.full((1,), -1, dtype=torch.int32, device=dev)
        _check("gdr_debug_wait_timeout", lib().gdr_debug_wait_timeout(int(kind), int(limit), res.data_ptr(),
                                                                      _stream(stream, dev)))
        return int(res.item())
