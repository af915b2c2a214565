"""Python face of the fp64 CPU oracle (``gdr_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
does, and this module never imports the CUDA library.

The C file holds the arithmetic.  This module converts bf16 bit patterns to
fp64 exactly, calls the C functions and composes them into the layer's paths
in the order the pages give (conv -> gates -> recurrence -> gated norm).
Rounding points (bf16, round to nearest even) are the boundary tensors of the
layer: the conv output, the recurrence output o and the norm output.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_ip = ctypes.POINTER(ctypes.c_int32)
_up = ctypes.POINTER(ctypes.c_uint16)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/liboracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.oracle_round_bf16.restype = ctypes.c_uint16
        L.oracle_round_bf16.argtypes = [ctypes.c_double]
        L.oracle_round_bf16_array.argtypes = [_dp, ctypes.c_int64, _up]
        L.oracle_softplus.restype = ctypes.c_double
        L.oracle_softplus.argtypes = [ctypes.c_double]
        L.oracle_sigmoid.restype = ctypes.c_double
        L.oracle_sigmoid.argtypes = [ctypes.c_double]
        L.oracle_gates.argtypes = [_dp, _dp, _fp, _fp, ctypes.c_int64, ctypes.c_int, _dp, _dp]
        core = [ctypes.c_int] * 4 + [_dp] * 5 + [ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                                 _ip, ctypes.c_int, _dp, _dp, _dp, _ip]
        L.oracle_gdr_stepwise.argtypes = core + [ctypes.c_int]
        L.oracle_gdr_stepwise.restype = ctypes.c_int
        L.oracle_gdr_chunked.argtypes = core + [ctypes.c_int, ctypes.c_int]
        L.oracle_gdr_chunked.restype = ctypes.c_int
        L.oracle_causal_conv.argtypes = [_dp, _dp, _dp, _ip, ctypes.c_int, ctypes.c_int, _dp, _dp,
                                         ctypes.c_int]
        L.oracle_conv_step.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int, _dp]
        L.oracle_gated_rmsnorm.argtypes = [_dp, _dp, _dp, ctypes.c_double, ctypes.c_int64,
                                           ctypes.c_int, _dp]
        L.oracle_prepare_chunks.argtypes = [_ip, ctypes.c_int, ctypes.c_int, _ip, _ip, _ip,
                                            ctypes.c_int]
        L.oracle_prepare_chunks.restype = ctypes.c_int
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _d(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns (round to nearest, ties to even)."""
    x = _d(x)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_round_bf16_array(_ptr(x, _dp), x.size, _ptr(out, _up))
    return out


def round_bf16_f64(x: np.ndarray) -> np.ndarray:
    """fp64 rounded to the nearest bf16 value, returned as fp64."""
    return bf16_to_f64(round_bf16(x))


# ---------------------------------------------------------------------------
# pieces
# ---------------------------------------------------------------------------

def softplus(x: float) -> float:
    return lib().oracle_softplus(float(x))


def sigmoid(x: float) -> float:
    return lib().oracle_sigmoid(float(x))


def gates(a: np.ndarray, b: np.ndarray, A_log: np.ndarray, dt_bias: np.ndarray):
    """g, beta from fp64 a, b of shape [T, hv] ("33B 只做 18 层 ..." (yfxerp.com) §1.2:
    g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b))."""
    a = _d(a); b = _d(b)
    T, hv = a.shape
    A_log = np.ascontiguousarray(A_log, dtype=np.float32)
    dt_bias = np.ascontiguousarray(dt_bias, dtype=np.float32)
    g = np.empty_like(a); beta = np.empty_like(a)
    lib().oracle_gates(_ptr(a, _dp), _ptr(b, _dp), _ptr(A_log, _fp), _ptr(dt_bias, _fp),
                       T, hv, _ptr(g, _dp), _ptr(beta, _dp))
    return g, beta


def _core(fn, q, k, v, g, beta, cu, h0, scale, use_l2norm, l2eps, heads, nthreads, extra=()):
    q = _d(q); k = _d(k); v = _d(v); g = _d(g); beta = _d(beta)
    T, hk, dk = q.shape
    _, hv, dv = v.shape
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    n = cu.shape[0] - 1
    h0d = None if h0 is None else _d(h0)
    o = np.zeros((T, hv, dv))
    hT = np.zeros((n, hv, dk, dv))
    mask = None
    if heads is not None:
        mask = np.zeros(hv, dtype=np.int32)
        mask[list(heads)] = 1
    rc = fn(hk, hv, dk, dv, _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(g, _dp),
            _ptr(beta, _dp), float(scale), int(use_l2norm), float(l2eps), _ptr(cu, _ip), n,
            _ptr(h0d, _dp), _ptr(o, _dp), _ptr(hT, _dp), _ptr(mask, _ip), *extra,
            nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o, hT


def gdr_stepwise(q, k, v, g, beta, cu, h0=None, scale=1.0, use_l2norm=True, l2eps=1e-6,
                 heads: Optional[Sequence[int]] = None, nthreads=None):
    """Token-by-token recurrence in fp64 ("Sapiens AI 发布 Agnes-3.0-Flash", delta 规则循环层究竟怎么
    运作, with the forget gate of "33B 只做 18 层 ..." §1.2).  Returns (o [T,hv,dv], hT [N,hv,dk,dv])."""
    return _core(lib().oracle_gdr_stepwise, q, k, v, g, beta, cu, h0, scale, use_l2norm, l2eps,
                 heads, nthreads)


def gdr_chunked(q, k, v, g, beta, cu, h0=None, scale=1.0, use_l2norm=True, l2eps=1e-6,
                chunk=64, heads=None, nthreads=None):
    """Chunked form, a self-check of the stepwise form ("33B 只做 18 层 ..." §1.2 names a
    chunk-64 path interchangeable with the per-token one; the algebra is in gdr_oracle.c)."""
    return _core(lib().oracle_gdr_chunked, q, k, v, g, beta, cu, h0, scale, use_l2norm, l2eps,
                 heads, nthreads, extra=(int(chunk),))


def causal_conv(x, w, cu, conv_state=None, round_y=True):
    """Kernel-4 causal conv + SiLU over packed sequences ("Agnes-3.0-Flash 深度解析",
    注意力层的细节).  Returns (y [T,C], conv_state_out [N,3,C])."""
    x = _d(x); w = _d(w)
    T, C = x.shape
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    n = cu.shape[0] - 1
    cs = None if conv_state is None else _d(conv_state)
    y = np.empty((T, C)); cso = np.empty((n, 3, C))
    lib().oracle_causal_conv(_ptr(x, _dp), _ptr(w, _dp), _ptr(cs, _dp), _ptr(cu, _ip), n, C,
                             _ptr(y, _dp), _ptr(cso, _dp), int(round_y))
    return y, cso


def conv_step(x, w, conv_state):
    """One decode step of the conv ("33B 只做 18 层 ..." (mhpq.cn) §2.1, the single-step
    causal conv); returns (y [B,C] fp64 unrounded, new state)."""
    x = _d(x); w = _d(w)
    st = _d(conv_state).copy()
    B, C = x.shape
    y = np.empty((B, C))
    lib().oracle_conv_step(_ptr(x, _dp), _ptr(w, _dp), _ptr(st, _dp), B, C, _ptr(y, _dp))
    return y, st


def gated_rmsnorm(o, z, w=None, eps=1e-6):
    """y = o / sqrt(mean(o^2) + eps) * w * SiLU(z) per row of d ("Agnes-3.0-Flash 深度解析",
    注意力层的细节: gated RMS-norm; z of width 48 x 128 in the parameter table of "33B 只做 18 层 ..."
    §2), in fp64, unrounded."""
    o = _d(o); z = _d(z)
    d = o.shape[-1]
    rows = o.size // d
    wd = None if w is None else _d(w)
    y = np.empty(o.shape)
    lib().oracle_gated_rmsnorm(_ptr(o, _dp), _ptr(z, _dp), _ptr(wd, _dp), float(eps), rows, d,
                               _ptr(y, _dp))
    return y


def prepare_chunks(cu, chunk=64):
    """Chunk table (chunk_seq, chunk_start, chunk_len) of packed sequences: chunks of `chunk`
    tokens restarting at every sequence start ("33B 只做 18 层 ..." §1.2, the chunk-64 walk)."""
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    n = cu.shape[0] - 1
    total = int(cu[-1]) if n > 0 else 0
    cap = total // chunk + n + 1
    seq = np.zeros(cap, np.int32); st = np.zeros(cap, np.int32); ln = np.zeros(cap, np.int32)
    m = lib().oracle_prepare_chunks(_ptr(cu, _ip), n, int(chunk), _ptr(seq, _ip), _ptr(st, _ip),
                                    _ptr(ln, _ip), cap)
    if m < 0:
        raise ValueError("invalid cu_seqlens")
    return seq[:m].copy(), st[:m].copy(), ln[:m].copy()


# ---------------------------------------------------------------------------
# compositions: the layer's paths
# ---------------------------------------------------------------------------

def core_path(inp, heads=None, nthreads=None, chunked=False):
    """Recurrence alone on ``gdr_inputs.CoreInputs``.

    Returns (o_bf16_bits [T,hv,dv], o_f64, hT_f64 [N,hv,dk,dv]).
    """
    q = bf16_to_f64(inp.q); k = bf16_to_f64(inp.k); v = bf16_to_f64(inp.v)
    g, beta = gates(bf16_to_f64(inp.a), bf16_to_f64(inp.b), inp.A_log, inp.dt_bias)
    fn = gdr_chunked if chunked else gdr_stepwise
    o, hT = fn(q, k, v, g, beta, inp.cu_seqlens, h0=inp.h0, scale=inp.scale, heads=heads,
               nthreads=nthreads)
    return round_bf16(o), o, hT


def linear(x_bits, w_bits):
    """One of the layer's projections ("33B 只做 18 层 ...", §2 parameter table: hidden 5120 to
    q|k|v, z, a, b and 6144 back to 5120): y = x W^T of the bf16 inputs x [M, K] and W [N, K],
    in fp64, rounded to bf16.  Returns bf16 bits [M, N]."""
    return round_bf16(bf16_to_f64(x_bits) @ bf16_to_f64(w_bits).T)


def split_qkv(y, hk, hv, dk, dv):
    T = y.shape[0]
    q = y[:, : hk * dk].reshape(T, hk, dk)
    k = y[:, hk * dk: 2 * hk * dk].reshape(T, hk, dk)
    v = y[:, 2 * hk * dk:].reshape(T, hv, dv)
    return q, k, v


def full_path(inp, heads=None, nthreads=None):
    """conv4+SiLU -> recurrence -> gated RMSNorm on ``gdr_inputs.FullInputs``.

    Returns dict with y (bf16 bits [T,hv,dv]), o (bf16 bits), hT (fp64),
    conv_state_out (bf16 bits [N,3,C]) and the conv output (bf16 bits).
    """
    x = bf16_to_f64(inp.x)
    w = bf16_to_f64(inp.conv_w)
    cs = None if inp.conv_state is None else bf16_to_f64(inp.conv_state)
    yconv, cso = causal_conv(x, w, inp.cu_seqlens, cs, round_y=True)
    q, k, v = split_qkv(yconv, inp.hk, inp.hv, inp.dk, inp.dv)
    g, beta = gates(bf16_to_f64(inp.a), bf16_to_f64(inp.b), inp.A_log, inp.dt_bias)
    o, hT = gdr_stepwise(q, k, v, g, beta, inp.cu_seqlens, h0=inp.h0, scale=inp.scale,
                         heads=heads, nthreads=nthreads)
    o_bits = round_bf16(o)
    y = gated_rmsnorm(bf16_to_f64(o_bits), bf16_to_f64(inp.z), inp.norm_w, inp.eps)
    return {"y": round_bf16(y), "o": o_bits, "hT": hT, "conv_state_out": round_bf16(cso),
            "conv_y": round_bf16(yconv)}


def decode_steps(inp, steps: Optional[int] = None, heads=None, nthreads=None, keep_o=()):
    """Advance ``gdr_inputs.DecodeInputs`` by `steps` single-token steps.

    Each step: conv step on x (output rounded to bf16) -> L2 norm, gates ->
    one step of the recurrence per sequence.  Returns (o_bits per kept step,
    final state fp64, final conv state fp64).
    """
    steps = inp.steps if steps is None else steps
    w = bf16_to_f64(inp.conv_w)
    cs = bf16_to_f64(inp.conv_state)
    H = inp.state.astype(np.float64)
    B = inp.B
    cu = np.arange(B + 1, dtype=np.int32)
    kept = {}
    for s in range(steps):
        y, cs = conv_step(bf16_to_f64(inp.x[s]), w, cs)
        y = round_bf16_f64(y)
        q, k, v = split_qkv(y, inp.hk, inp.hv, inp.dk, inp.dv)
        g, beta = gates(bf16_to_f64(inp.a[s]), bf16_to_f64(inp.b[s]), inp.A_log, inp.dt_bias)
        o, Hn = gdr_stepwise(q, k, v, g, beta, cu, h0=H, scale=inp.scale, heads=heads,
                             nthreads=nthreads)
        if heads is not None:
            # heads outside the sample keep their (unused) old state
            keep = np.zeros(inp.hv, bool); keep[list(heads)] = True
            Hn[:, ~keep] = H[:, ~keep]
        H = Hn
        if s in keep_o or (s - steps) in keep_o:
            kept[s] = round_bf16(o)
    return kept, H, cs


def decode_step_slots(x, a, b, conv_w, A_log, dt_bias, conv_pool, state_pool, slot, hk, hv,
                      scale=1.0, dk=128, dv=128, heads=None, nthreads=None):
    """One decode step on pools of cached states ("33B 只做 18 层 ...", §1.2: each request's
    recurrent and conv states live in a per-layer cache and the next token resumes from them).

    Row i of the batch (x [B,C], a, b [B,hv] bf16 bits) reads and writes entry slot[i] of
    conv_pool [S,3,C] and state_pool [S,hv,dk,dv]; a slot outside [0, S) is a padding row
    whose o row is zero and which touches no entry.  Rows must name distinct slots.  The
    step itself is the decode step above on the gathered rows.  Returns (o bits [B,hv,dv],
    new conv pool fp64, new state pool fp64).
    """
    slot = np.asarray(slot, dtype=np.int64)
    S = state_pool.shape[0]
    live = np.nonzero((slot >= 0) & (slot < S))[0]
    ids = slot[live]
    if len(np.unique(ids)) != len(ids):
        raise ValueError("rows name the same slot twice")
    cpool = _d(conv_pool).copy()
    spool = _d(state_pool).copy()
    B = x.shape[0]
    o_bits = np.zeros((B, hv, dv), dtype=np.uint16)
    if len(live) == 0:
        return o_bits, cpool, spool
    y, cs = conv_step(bf16_to_f64(x[live]), bf16_to_f64(conv_w), cpool[ids])
    y = round_bf16_f64(y)
    q, k, v = split_qkv(y, hk, hv, dk, dv)
    g, beta = gates(bf16_to_f64(a[live]), bf16_to_f64(b[live]), A_log, dt_bias)
    cu = np.arange(len(live) + 1, dtype=np.int32)
    o, Hn = gdr_stepwise(q, k, v, g, beta, cu, h0=spool[ids], scale=scale, heads=heads,
                         nthreads=nthreads)
    if heads is not None:
        keep = np.zeros(hv, bool); keep[list(heads)] = True
        Hn[:, ~keep] = spool[ids][:, ~keep]
    o_bits[live] = round_bf16(o)
    cpool[ids] = cs
    spool[ids] = Hn
    return o_bits, cpool, spool
