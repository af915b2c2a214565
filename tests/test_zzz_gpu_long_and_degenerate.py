"""Parity on a B200 for the decode workload at its measured length and for keys that
repeat within a chunk.  This file sorts after the other GPU test files: its cases are the
longest and the most degenerate ones."""
import numpy as np
import pytest
import torch

import gated_delta_rule_63_b200 as G
import gdr_inputs as GI
from oracle import oracle as O
from tests.helpers import TOL_BF16, TOL_STATE, bits_f64, rel_l2, restrict_decode_heads
from tests.test_gpu_parity import check_core, run_gpu_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    G.lib()
    yield
    assert G.get_device_error() == 0


def test_prefill_repeated_key_full_write():
    """Every token of a key head carries the same key and every write strength is 1: the
    rank-one case of the recurrence (each token overwrites the key direction), where every
    in-chunk entry of A has k.k = 1 and the chunked form cancels the most."""
    inp = GI.make_core_inputs(91, [150, 64], prenorm_qk=False, h0_std=0.02)
    inp.k = np.ascontiguousarray(np.broadcast_to(inp.k[:1], inp.k.shape))
    inp.b = GI.f32_to_bf16_bits(np.full(inp.b.shape, 200.0, np.float32))
    check_core(inp)


def test_decode_workload_1000_steps_sampled_heads():
    """The decode workload as measured: B = 64, 1000 consecutive steps on one state, compared
    with the oracle run over all 1000 steps at the first and the last step's output and the
    final state of three sampled value heads; the conv state, all channels, bit for bit."""
    dec = GI.workload_decode_B64()
    heads = [0, 23, 47]
    S = dec.steps
    outs, st, cs = run_gpu_decode(dec, S, keep=(0, S - 1))
    kept, H, _ = O.decode_steps(restrict_decode_heads(dec, heads), keep_o=(0, -1))
    for s in (0, S - 1):
        assert rel_l2(bits_f64(outs[s][:, heads]), bits_f64(kept[s])) <= TOL_BF16, s
    assert rel_l2(st[:, heads], H) <= TOL_STATE
    # after three or more steps the conv state holds the last three inputs, oldest first
    assert np.array_equal(cs, np.transpose(dec.x[S - 3:], (1, 0, 2)))
