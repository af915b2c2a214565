"""The layer sharded by heads over two ranks (gloo on CPU, the fp64 oracle as each rank's
compute): each rank projects the hidden state to its heads' q, k, v, z, a, b, runs the layer
(conv -> recurrence -> gated norm) on them, and multiplies its slice of the normed output by its
columns of the output projection; one all-reduce of the partial outputs gives the full layer.
This checks the sharding plan (gated_delta_rule_63_b200.shard) and the one exchange, not the
kernels (the GPU test runs those)."""
import datetime
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

HIDDEN, LENGTHS = 64, [13, 11]


def _layer_inputs():
    import gdr_inputs as GI
    r = np.random.default_rng(61)
    h = GI.f32_to_bf16_bits(r.standard_normal((sum(LENGTHS), HIDDEN)).astype(np.float32))
    w_in = GI.f32_to_bf16_bits((r.standard_normal((GI.IN_PROJ_N, HIDDEN)) / 8).astype(np.float32))
    w_out = GI.f32_to_bf16_bits((r.standard_normal((HIDDEN, GI.OUT_PROJ_K)) / 78).astype(np.float32))
    conv_w = GI.f32_to_bf16_bits((r.standard_normal((2 * GI.HK * GI.DK + GI.HV * GI.DV, 4)) * 0.5)
                                 .astype(np.float32))
    A_log = np.log(r.uniform(1, 16, GI.HV)).astype(np.float32)
    dt_bias = np.log(np.expm1(r.uniform(1e-3, 0.1, GI.HV))).astype(np.float32)
    return h, w_in, w_out, conv_w, A_log, dt_bias


def _normed(h, w_in_rows, conv_w, A_log, dt_bias, hk, hv):
    """Oracle: the projection to q|k|v, z, a, b, then conv -> recurrence -> gated norm."""
    import gdr_inputs as GI
    from oracle import oracle as O
    y = O.linear(h, w_in_rows)
    c = 2 * hk * 128 + hv * 128
    T = y.shape[0]
    inp = GI.FullInputs(x=np.ascontiguousarray(y[:, :c]), conv_w=conv_w, conv_state=None,
                        a=np.ascontiguousarray(y[:, c + hv * 128: c + hv * 128 + hv]),
                        b=np.ascontiguousarray(y[:, c + hv * 128 + hv:]),
                        z=np.ascontiguousarray(y[:, c: c + hv * 128]).reshape(T, hv, 128), norm_w=None,
                        A_log=A_log, dt_bias=dt_bias, cu_seqlens=GI.cu_seqlens_from_lengths(LENGTHS), h0=None,
                        hk=hk, hv=hv)
    return O.full_path(inp)["y"].reshape(T, hv * 128)


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from oracle import oracle as O
        from gated_delta_rule_63_b200.shard import head_shard
        h, w_in, w_out, conv_w, A_log, dt_bias = _layer_inputs()
        s = head_shard(rank, world)
        y = _normed(h, w_in[s.in_rows], conv_w[s.conv_channels], A_log[s.heads], dt_bias[s.heads], s.hk, s.hv)
        partial = torch.from_numpy(O.bf16_to_f64(y) @ O.bf16_to_f64(w_out[:, s.out_cols]).T)
        dist.all_reduce(partial)                        # the one exchange: sum of the partial outputs
        out[rank] = (y, partial.numpy())
    finally:
        dist.destroy_process_group()


def test_two_head_shards_and_one_all_reduce_give_the_full_layer():
    from oracle import oracle as O
    from gated_delta_rule_63_b200.shard import head_shard
    world = 2
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    h, w_in, w_out, conv_w, A_log, dt_bias = _layer_inputs()
    y_full = _normed(h, w_in, conv_w, A_log, dt_bias, 16, 48)
    full = O.bf16_to_f64(y_full) @ O.bf16_to_f64(w_out).T
    for r in range(world):
        y, summed = out[r]
        s = head_shard(r, world)
        assert np.array_equal(y, y_full[:, s.out_cols])          # a shard's heads are the full layer's
        assert np.allclose(summed, full, rtol=1e-12, atol=1e-12)  # and the partials sum to its output


def test_head_shard_plan_covers_every_output_once():
    from gated_delta_rule_63_b200.shard import head_shard
    import gdr_inputs as GI
    for n in (1, 2, 4, 8, 16):
        parts = [head_shard(r, n) for r in range(n)]
        rows = np.concatenate([p.in_rows for p in parts])
        cols = np.concatenate([p.out_cols for p in parts])
        assert np.array_equal(np.sort(rows), np.arange(GI.IN_PROJ_N))
        assert np.array_equal(np.sort(cols), np.arange(GI.OUT_PROJ_K))
        for p in parts:   # q, k, v channels of the shard's key and value heads, in [q | k | v] order
            assert p.n_conv == 2 * p.hk * 128 + p.hv * 128 and p.hv == 3 * p.hk
    import pytest
    with pytest.raises(ValueError):
        head_shard(0, 3)
