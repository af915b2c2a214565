"""The C ABI without a GPU: the library loads, exports what include/gdr.h
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import gated_delta_rule_63_b200 as G
from gated_delta_rule_63_b200 import build as B
from oracle import oracle as O
import gdr_inputs as GI

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return G.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "gdr.h")).read()
    return sorted(set(re.findall(r"GDR_API[^;(]*?\b(gdr_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for fn in ("gdr_causal_conv", "gdr_chunk_prefill", "gdr_decode_step", "gdr_gated_rmsnorm",
               "gdr_prepare_chunks", "gdr_status_string"):
        assert fn in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert G.status_string(0) == "GDR_OK"
    for code in range(1, 10):
        assert G.status_string(code).startswith("GDR_ERR_")
    assert "UNKNOWN" in G.status_string(12345)
    assert L.gdr_abi_version() == 6


@pytest.mark.parametrize("lengths", [[0], [1], [64], [65, 0, 128, 1, 63], [5000, 3, 64 * 7 + 1],
                                     list(GI.varlen8_lengths())])
def test_prepare_chunks_is_bit_exact_with_oracle(L, lengths):
    cu = GI.cu_seqlens_from_lengths(lengths)
    got = G.prepare_chunks(cu, 64)
    ref = O.prepare_chunks(cu, 64)
    for g, r in zip(got, ref):
        assert g.dtype == np.int32 and np.array_equal(g, r)


@settings(max_examples=40, deadline=None)
@given(lengths=st.lists(st.integers(0, 300), min_size=1, max_size=10), chunk=st.integers(1, 100))
def test_prepare_chunks_bit_exact_on_random_offsets(L, lengths, chunk):
    cu = GI.cu_seqlens_from_lengths(lengths)
    got = G.prepare_chunks(cu, chunk)
    ref = O.prepare_chunks(cu, chunk)
    for g, r in zip(got, ref):
        assert g.dtype == np.int32 and np.array_equal(g, r)


def test_prepare_chunks_errors(L):
    with pytest.raises(G.GdrError) as e:
        G.prepare_chunks(np.array([0, 5, 4], np.int32))
    assert e.value.code == 4
    with pytest.raises(G.GdrError) as e:
        G.prepare_chunks(np.array([2, 5], np.int32))
    assert e.value.code == 4
    cu = np.array([0, 200], np.int32)
    seq = np.zeros(2, np.int32)
    m = ctypes.c_int(0)
    ip = ctypes.POINTER(ctypes.c_int32)
    rc = L.gdr_prepare_chunks(cu.ctypes.data_as(ip), 1, 64, seq.ctypes.data_as(ip),
                              seq.ctypes.data_as(ip), seq.ctypes.data_as(ip), 2, ctypes.byref(m))
    assert rc == 2 and m.value == 2   # needs 4 entries, had room for 2


FAKE = 0x10000      # an aligned address that is never dereferenced: checks fail first
ODD = 0x10002


def _cu(lengths):
    cu = GI.cu_seqlens_from_lengths(lengths)
    return cu, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def test_prefill_rejects_bad_arguments_on_host(L):
    cu, cup = _cu([10, 5])
    args = dict(q=FAKE, k=FAKE, v=FAKE, qs=0, vs=0, a=FAKE, b=FAKE, A_log=FAKE, dt_bias=FAKE, scale=1.0, hk=16,
                hv=48, cu_dev=FAKE, cu_host=cup, n=2, h0=None, hT=FAKE, o=FAKE, fuse=None, ws=FAKE,
                wsb=1 << 30, s=None)

    def call(**kw):
        a = dict(args); a.update(kw)
        return L.gdr_chunk_prefill(a["q"], a["k"], a["v"], a["qs"], a["vs"], a["a"], a["b"],
                                   a["A_log"], a["dt_bias"],
                                   a["scale"], a["hk"], a["hv"], a["cu_dev"], a["cu_host"], a["n"],
                                   a["h0"], a["hT"], a["o"], a["fuse"], a["ws"], a["wsb"], a["s"])
    assert call(hk=16, hv=40) == 5          # grouping not integral
    assert call(hk=1, hv=48) == 5           # group of 48 > 8
    assert call(hk=0) == 2
    assert call(q=None) == 1
    assert call(cu_dev=None) == 1
    assert call(cu_host=None) == 1
    assert call(o=ODD) == 3
    bad, badp = _cu([3])
    bad[0] = 1
    assert call(cu_host=badp, n=1) == 4
    assert call(h0=FAKE + 64, hT=FAKE) == 9  # partial overlap of h0 and hT
    assert call(qs=16 * 128 - 8) == 2          # token stride shorter than a row
    assert call(vs=48 * 128 + 4) == 3          # token stride not a multiple of 8
    assert call(ws=None) == 6                  # no workspace
    assert call(wsb=1000) == 6                 # too small for one chunk window
    assert call(ws=FAKE + 8) == 3


def test_prefill_workspace_size(L):
    L.gdr_chunk_prefill_workspace_size.restype = ctypes.c_size_t
    one = L.gdr_chunk_prefill_workspace_size(2, 48, 1, 1)
    assert one == 2 * 48 * 82944
    assert L.gdr_chunk_prefill_workspace_size(2, 48, 5, 1) == 5 * one
    assert L.gdr_chunk_prefill_workspace_size(2, 48, 5, 0) == 5 * one + 2 * 48 * 128 * 128 * 4
    assert L.gdr_chunk_prefill_workspace_size(0, 48, 5, 1) == 0


def test_prefill_with_fused_conv_checks_on_host(L):
    """Conv fused into the prefill (fuse.x): q, k, v must be NULL, conv_w is required, and the
    workspace holds the conv output in front of the chunk records."""
    cu, cup = _cu([10, 5])
    fz = G.FuseArgs()
    fz.x, fz.conv_w = FAKE, FAKE

    def call(q=None, wsb=1 << 30, fuse=fz):
        return L.gdr_chunk_prefill(q, None, None, 0, 0, FAKE, FAKE, FAKE, FAKE, 1.0, 16, 48, FAKE, cup, 2,
                                   None, FAKE, FAKE, ctypes.byref(fuse), FAKE, wsb, None)
    assert call(q=FAKE) == 2                   # q, k, v come from the conv
    no_w = G.FuseArgs()
    no_w.x = FAKE
    assert call(fuse=no_w) == 1                # conv weights required
    need = L.gdr_chunk_prefill_fused_workspace_size(2, 16, 48, 15, 1, 1)
    assert call(wsb=need - 16) == 6            # the conv output does not fit in front of the records
    odd = G.FuseArgs()
    odd.x, odd.conv_w, odd.conv_state_in = FAKE, FAKE, ODD
    assert call(fuse=odd) == 3


def test_fused_workspace_size(L):
    conv = 100 * 10240 * 2                      # already a whole number of KiB
    assert L.gdr_chunk_prefill_fused_workspace_size(2, 16, 48, 100, 1, 1) == conv + 2 * 48 * 82944
    # one key and one value head: 3 tokens x 384 channels x 2 B = 2304 B, rounded up to 3 KiB
    assert L.gdr_chunk_prefill_fused_workspace_size(2, 1, 1, 3, 1, 1) == 3072 + 2 * 82944
    assert L.gdr_chunk_prefill_fused_workspace_size(2, 16, 48, 100, 2, 0) == (
        conv + L.gdr_chunk_prefill_workspace_size(2, 48, 2, 0))
    assert L.gdr_chunk_prefill_fused_workspace_size(0, 16, 48, 100, 1, 1) == 0
    assert L.gdr_chunk_prefill_fused_workspace_size(2, 16, 48, -1, 1, 1) == 0


def test_wait_self_test_rejects_bad_arguments(L):
    L.gdr_debug_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_ulonglong, ctypes.c_void_p, ctypes.c_void_p]
    assert L.gdr_debug_wait_timeout(2, 10, FAKE, None) == 2          # unknown kind
    assert L.gdr_debug_wait_timeout(0, 0, FAKE, None) == 2           # no bound
    assert L.gdr_debug_wait_timeout(0, 1 << 40, FAKE, None) == 2     # bound above 2^31
    assert L.gdr_debug_wait_timeout(0, 10, None, None) == 1          # no result word


def test_linear_rejects_bad_arguments_on_host(L):
    f = L.gdr_linear
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [ctypes.c_void_p]
    Y = FAKE + (1 << 30)
    assert f(FAKE, FAKE, None, 4, 8, 8, None) == 1                  # no output
    assert f(FAKE, FAKE, Y, 4, 12, 8, None) == 2                    # N not a multiple of 8
    assert f(FAKE, FAKE, Y, 4, 8, 12, None) == 2                    # K not a multiple of 8
    assert f(FAKE, FAKE, Y, -1, 8, 8, None) == 2
    assert f(FAKE, FAKE, Y, 4, 0, 8, None) == 2
    assert f(FAKE, FAKE, Y, 0, 8, 8, None) == 0                     # no rows: nothing to do
    assert f(ODD, FAKE, Y, 4, 8, 8, None) == 3
    assert f(FAKE, FAKE, FAKE + 32, 4, 8, 8, None) == 9             # y overlaps x


def test_prefill_schedule_on_host(L):
    """Windows of a call as the workspace shrinks (no pipelining below 33 chunks, so no device
    query), and argument rejection."""
    f = L.gdr_chunk_prefill_schedule
    f.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.c_int, ctypes.c_int, ctypes.c_size_t, ctypes.c_int,
                  ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    cu, cup = _cu([300, 64, 1])                # 5, 1, 1 chunks
    w, pl = ctypes.c_int(-1), ctypes.c_int(-1)
    for chunks, final, want in ((5, 1, 1), (2, 1, 3), (1, 1, 5), (3, 0, 2)):
        ws = L.gdr_chunk_prefill_workspace_size(3, 48, chunks, final)
        assert f(cup, 3, 48, ws, final, ctypes.byref(w), ctypes.byref(pl)) == 0
        assert (w.value, pl.value) == (want, 0), chunks
    assert f(cup, 3, 48, L.gdr_chunk_prefill_workspace_size(3, 48, 1, 1) - 1, 1, ctypes.byref(w),
             ctypes.byref(pl)) == 6
    assert f(cup, 3, 48, 1 << 30, 1, None, ctypes.byref(pl)) == 1
    assert f(cup, 3, 0, 1 << 30, 1, ctypes.byref(w), ctypes.byref(pl)) == 2
    assert f(cup, 3, 48, 1 << 30, 2, ctypes.byref(w), ctypes.byref(pl)) == 2
    bad, badp = _cu([3])
    bad[1] = -1
    assert f(badp, 1, 48, 1 << 30, 1, ctypes.byref(w), ctypes.byref(pl)) == 4
    empty, emptyp = _cu([0, 0])
    assert f(emptyp, 2, 48, 0, 1, ctypes.byref(w), ctypes.byref(pl)) == 0 and w.value == 1


def test_prefill_slots_rejects_bad_arguments_on_host(L):
    f = L.gdr_chunk_prefill_slots
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 2 + [ctypes.c_void_p] * 4 + [
        ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_size_t, ctypes.c_void_p]
    cu, cup = _cu([70, 5])
    ws = L.gdr_chunk_prefill_workspace_size(2, 48, 1, 0)

    def call(slot=FAKE, pool=FAKE, n_slots=4, init=0, hv=48, wsb=ws, q=FAKE):
        return f(q, FAKE, FAKE, 0, 0, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(1.0), 16, hv, FAKE, cup, 2,
                 pool, n_slots, slot, init, FAKE, FAKE, wsb, None)
    assert call(slot=None) == 1                   # no slot array
    assert call(pool=None) == 1                   # entries without a pool
    assert call(q=None) == 1                      # tokens without inputs
    assert call(n_slots=-1) == 2
    assert call(init=2) == 2
    assert call(hv=50) == 5                       # grouping not supported
    assert call(slot=FAKE + 2) == 3               # slot array not 4-byte aligned
    assert call(wsb=ws - 16) == 6                 # workspace below one window plus the carry
    assert ws == L.gdr_chunk_prefill_workspace_size(2, 48, 1, 1) + 2 * 48 * 128 * 128 * 4


def test_other_entry_points_reject_bad_arguments(L):
    cu, cup = _cu([4])
    assert L.gdr_causal_conv(FAKE, FAKE, None, None, FAKE, cup, 1, 10, FAKE, None) == 2   # C % 8
    assert L.gdr_causal_conv(FAKE, FAKE, FAKE, FAKE, FAKE, cup, 1, 16, FAKE, None) == 9   # state alias
    assert L.gdr_causal_conv(ODD, FAKE, None, None, FAKE, cup, 1, 16, FAKE, None) == 3
    assert L.gdr_gated_rmsnorm(FAKE, FAKE, None, ctypes.c_float(1e-6), 10, 64, FAKE, None) == 5
    assert L.gdr_gated_rmsnorm(None, FAKE, None, ctypes.c_float(1e-6), 10, 128, FAKE, None) == 1
    assert L.gdr_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(1.0), 16, 50,
                             FAKE, FAKE, 4, None) == 5
    assert L.gdr_decode_step(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(1.0), 16, 48,
                             FAKE, FAKE, 4, None) == 1
    # zero-sized work is accepted without touching the device
    assert L.gdr_decode_step(None, None, None, None, None, None, None, ctypes.c_float(1.0), 16, 48,
                             None, None, 0, None) == 0
    assert L.gdr_gated_rmsnorm(None, None, None, ctypes.c_float(1e-6), 0, 128, None, None) == 0


def test_decode_slots_rejects_bad_arguments_on_host(L):
    f1 = ctypes.c_float(1.0)
    dec = L.gdr_decode_step_slots
    # heads, null slot array, null pool with slots, negative sizes, misaligned slot array
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f1, 16, 50, FAKE, 4, FAKE, FAKE, 4, None) == 5
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f1, 16, 48, FAKE, 4, None, FAKE, 4, None) == 1
    assert dec(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, f1, 16, 48, FAKE, 4, FAKE, FAKE, 4, None) == 1
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f1, 16, 48, None, 4, FAKE, FAKE, 4, None) == 1
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f1, 16, 48, FAKE, -1, FAKE, FAKE, 4, None) == 2
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f1, 16, 48, FAKE, 4, FAKE, FAKE, -1, None) == 2
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f1, 16, 48, FAKE, 4, FAKE + 2, FAKE, 4, None) == 3
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f1, 16, 48, ODD, 4, FAKE, FAKE, 4, None) == 3
    # an empty batch is accepted without touching the device
    assert dec(None, None, None, None, None, None, None, f1, 16, 48, None, 0, None, None, 0, None) == 0


def test_binding_fails_loudly_without_the_library(tmp_path):
    import gated_delta_rule_63_b200 as mod
    saved = mod._lib
    try:
        mod._lib = None
        with pytest.raises(RuntimeError):
            mod.lib(str(tmp_path / "missing.so"))
    finally:
        mod._lib = saved


def test_binding_refuses_tensors_on_two_devices():
    """A call runs on its tensors' one device; a mix never reaches a kernel (no GPU needed:
    the check reads only the tensors' device attributes)."""
    import types
    import torch
    d0 = types.SimpleNamespace(device=torch.device("cuda", 0))
    d1 = types.SimpleNamespace(device=torch.device("cuda", 1))
    host = types.SimpleNamespace(device=torch.device("cpu"))
    assert G._device_of(None, d0, host, d0) == torch.device("cuda", 0)
    assert G._device_of(None, host) is None
    with pytest.raises(ValueError):
        G._device_of(d0, None, d1)
    with pytest.raises(ValueError):
        G._stream(types.SimpleNamespace(device=torch.device("cuda", 1), cuda_stream=0), torch.device("cuda", 0))
