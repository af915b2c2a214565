"""gdr_chunk_prefill_noalloc: the prefill for callers that cannot allocate.

It runs the prefill kernels on a scratch array that lives inside the library,
so a caller without a way to obtain device memory (a plugin whose framework
owns all allocations, a fixed-budget deployment, code where cudaMalloc is not
allowed) can still call it.  This file is collected last on purpose, and it
also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_63_b200 as G
import gdr_inputs as GI
from oracle import oracle as O
from tests.helpers import TOL_BF16, TOL_STATE, bits_f64, dev_bf16, dev_f32, dev_i32, host_bits, rel_l2

pytestmark = pytest.mark.gpu


def _args(inp):
    return (dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.a), dev_bf16(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_i32(inp.cu_seqlens), inp.cu_seqlens)


def _noalloc_raw(L, args, h0, hT, o):
    """gdr_chunk_prefill_noalloc through the C ABI with plain pointers (hT may be None)."""
    q, k, v, a, b, A_log, dt_bias, cu_d, cu_h = args
    cu_h = np.ascontiguousarray(cu_h, dtype=np.int32)
    return L.gdr_chunk_prefill_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, 0, a.data_ptr(), b.data_ptr(),
        A_log.data_ptr(), dt_bias.data_ptr(), ctypes.c_float(1.0), 16, 48, cu_d.data_ptr(),
        cu_h.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu_h) - 1, h0.data_ptr(),
        hT.data_ptr() if hT is not None else None, o.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_the_oracle_and_the_workspace_entry_point_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = G.lib()
    assert L.gdr_chunk_prefill_noalloc_scratch_bytes() == 32 << 20
    # three sequences, 1000 tokens in all: the scratch holds a window of a few
    # chunks, so the long sequence crosses several windows
    inp = GI.make_core_inputs(90, [700, 65, 235], prenorm_qk=False, h0_std=0.02)
    args = _args(inp)
    h0 = dev_f32(inp.h0)
    ref_hT = torch.empty_like(h0)
    ref_o = G.chunk_prefill(*args, h0=h0, hT=ref_hT)
    torch.cuda.synchronize()
    want_bits, _, want_hT = O.core_path(inp)
    for call in range(2):
        hT = torch.full_like(h0, float("nan"))
        o = torch.full_like(ref_o, float("nan"))
        rc = _noalloc_raw(L, args, h0, hT, o)
        assert rc == 0, G.status_string(rc)
        torch.cuda.synchronize()
        o_bits, hT_np = host_bits(o), hT.cpu().numpy()
        # the same kernels on fp32 state carries: bit for bit the workspace entry point's results
        assert np.array_equal(o_bits, host_bits(ref_o)), call
        assert np.array_equal(hT_np, ref_hT.cpu().numpy()), call
        # and within the layer's tolerances of the oracle, sequence by sequence
        cu = inp.cu_seqlens
        for n in range(inp.n_seqs):
            s, e = int(cu[n]), int(cu[n + 1])
            assert rel_l2(bits_f64(o_bits[s:e]), bits_f64(want_bits[s:e])) <= TOL_BF16, (call, n)
            assert rel_l2(hT_np[n], want_hT[n]) <= TOL_STATE, (call, n)
    assert G.get_device_error() == 0


def test_noalloc_without_final_state_carries_the_state_in_its_scratch():
    """hT = NULL: the state crosses the windows inside the scratch array, one chunk per window
    for these three sequences; o still equals the workspace entry point's bit for bit and the
    oracle's within the tolerance."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = G.lib()
    inp = GI.make_core_inputs(92, [300, 130, 7], prenorm_qk=False, h0_std=0.02)
    args = _args(inp)
    h0 = dev_f32(inp.h0)
    ref_o = G.chunk_prefill(*args, h0=h0)
    want_bits, _, _ = O.core_path(inp)
    for call in range(2):
        o = torch.full_like(ref_o, float("nan"))
        rc = _noalloc_raw(L, args, h0, None, o)
        assert rc == 0, G.status_string(rc)
        torch.cuda.synchronize()
        o_bits = host_bits(o)
        assert np.array_equal(o_bits, host_bits(ref_o)), call
        cu = inp.cu_seqlens
        for n in range(inp.n_seqs):
            s, e = int(cu[n]), int(cu[n + 1])
            assert rel_l2(bits_f64(o_bits[s:e]), bits_f64(want_bits[s:e])) <= TOL_BF16, (call, n)
    assert G.get_device_error() == 0


def test_noalloc_rejects_work_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    inp = GI.make_core_inputs(91, [3] * 10, prenorm_qk=False)   # 10 sequences: one window is > 32 MiB
    with pytest.raises(G.GdrError) as e:
        G.chunk_prefill_noalloc(*_args(inp), hT=torch.empty((10, 48, 128, 128), device="cuda"))
    assert e.value.code == 6
