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
from tests.helpers import TOL_BF16, TOL_STATE, bits_f64, dev_bf16, dev_f32, dev_i32, host_bits, rel_l2

pytestmark = pytest.mark.gpu


def _args(inp):
    return (dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.a), dev_bf16(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_i32(inp.cu_seqlens), inp.cu_seqlens)


def test_noalloc_matches_the_workspace_entry_point_twice_in_a_row():
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
    for call in range(2):
        hT = torch.full_like(h0, float("nan"))
        o = torch.full_like(ref_o, float("nan"))
        q, k, v, a, b, A_log, dt_bias, cu_d, cu_h = args
        cu_h = np.ascontiguousarray(cu_h, dtype=np.int32)
        rc = L.gdr_chunk_prefill_noalloc(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, 0, a.data_ptr(), b.data_ptr(),
            A_log.data_ptr(), dt_bias.data_ptr(), ctypes.c_float(1.0), 16, 48, cu_d.data_ptr(),
            cu_h.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu_h) - 1, h0.data_ptr(),
            hT.data_ptr(), o.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == 0, G.status_string(rc)
        torch.cuda.synchronize()
        assert rel_l2(bits_f64(host_bits(o)), bits_f64(host_bits(ref_o))) <= TOL_BF16, call
        assert rel_l2(hT.cpu().numpy(), ref_hT.cpu().numpy()) <= TOL_STATE, call
    assert G.get_device_error() == 0


def test_noalloc_rejects_work_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    inp = GI.make_core_inputs(91, [3] * 10, prenorm_qk=False)   # 10 sequences: one window is > 32 MiB
    with pytest.raises(G.GdrError) as e:
        G.chunk_prefill_noalloc(*_args(inp), hT=torch.empty((10, 48, 128, 128), device="cuda"))
    assert e.value.code == 6
