"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Tolerances of the layer: rel-L2 <= 2e-3 on bf16 outputs and <= 1e-4 on the
fp32 final state; chunk/varlen indexing and copied conv states bit-exact.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_63_b200 as G
import gdr_inputs as GI
from oracle import oracle as O
from tests.helpers import (TOL_BF16, TOL_STATE, bits_f64, dev_bf16, dev_f32, dev_i32, host_bits,
                           rel_l2, ulp_diff_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    G.lib()
    yield
    assert G.get_device_error() == 0


# ---------------------------------------------------------------------------
# helpers running the GPU path
# ---------------------------------------------------------------------------

def gpu_core(inp, h0_inplace=False):
    """Run gdr_chunk_prefill on CoreInputs; returns (o bits, hT f32)."""
    cu_d = dev_i32(inp.cu_seqlens)
    N = inp.n_seqs
    hv = inp.v.shape[1]
    h0 = dev_f32(inp.h0) if inp.h0 is not None else None
    if h0_inplace:
        hT = h0
    else:
        hT = torch.full((N, hv, 128, 128), float("nan"), device="cuda")
    o = G.chunk_prefill(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.a),
                        dev_bf16(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias), cu_d,
                        inp.cu_seqlens, h0=h0, hT=hT, scale=inp.scale)
    torch.cuda.synchronize()
    return host_bits(o), hT.cpu().numpy()


def check_core(inp, heads=None, h0_inplace=False):
    o_bits, hT = gpu_core(inp, h0_inplace)
    ref_bits, _, ref_hT = O.core_path(inp, heads=heads)
    if heads is not None:
        o_bits = o_bits[:, heads]; ref_bits = ref_bits[:, heads]
        hT = hT[:, heads]; ref_hT = ref_hT[:, heads]
    eo = rel_l2(bits_f64(o_bits), bits_f64(ref_bits))
    eh = rel_l2(hT, ref_hT)
    assert np.all(np.isfinite(hT))
    assert eo <= TOL_BF16, f"o rel-L2 {eo:.3e}"
    assert eh <= TOL_STATE, f"state rel-L2 {eh:.3e}"
    # per-sequence attribution: every sequence must be right on its own
    cu = inp.cu_seqlens
    for n in range(inp.n_seqs):
        s, e = int(cu[n]), int(cu[n + 1])
        if e > s:
            assert rel_l2(bits_f64(o_bits[s:e]), bits_f64(ref_bits[s:e])) <= TOL_BF16
        # (a state the oracle leaves exactly zero, e.g. an empty sequence without h0, must be zero)
        assert rel_l2(hT[n], ref_hT[n]) <= TOL_STATE, n
    return eo, eh


# ---------------------------------------------------------------------------
# causal conv
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("with_state", [False, True])
def test_conv_varlen_matches_oracle(with_state):
    lengths = [1, 2, 0, 3, 5, 64, 100, 33]
    inp = GI.make_full_inputs(50, lengths, conv_state_std=1.0 if with_state else None)
    C = inp.channels
    cu_d = dev_i32(inp.cu_seqlens)
    cs_in = dev_bf16(inp.conv_state) if with_state else None
    cs_out = torch.zeros((len(lengths), 3, C), dtype=torch.bfloat16, device="cuda")
    y = G.causal_conv(dev_bf16(inp.x), dev_bf16(inp.conv_w), cu_d, inp.cu_seqlens, cs_in, cs_out)
    torch.cuda.synchronize()
    ref_y, ref_cs = O.causal_conv(bits_f64(inp.x), bits_f64(inp.conv_w), inp.cu_seqlens,
                                  bits_f64(inp.conv_state) if with_state else None, round_y=True)
    got = host_bits(y)
    ref = O.round_bf16(ref_y)
    assert ulp_diff_bf16(got, ref).max() <= 1       # fp32 vs fp64 before the same rounding
    assert (got != ref).mean() < 1e-3
    assert np.array_equal(host_bits(cs_out), O.round_bf16(ref_cs))   # raw copies: exact


# ---------------------------------------------------------------------------
# gated RMSNorm
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("with_w", [False, True])
def test_gated_rmsnorm_matches_oracle(with_w):
    r = np.random.default_rng(51)
    rows = 1000
    o = GI.f32_to_bf16_bits(r.standard_normal((rows, 128)).astype(np.float32) * 3)
    z = GI.f32_to_bf16_bits(r.standard_normal((rows, 128)).astype(np.float32))
    w = (1 + 0.1 * r.standard_normal(128)).astype(np.float32) if with_w else None
    y = G.gated_rmsnorm(dev_bf16(o), dev_bf16(z), dev_f32(w) if with_w else None, eps=1e-6)
    torch.cuda.synchronize()
    ref = O.round_bf16(O.gated_rmsnorm(bits_f64(o), bits_f64(z), w, eps=1e-6))
    got = host_bits(y)
    assert rel_l2(bits_f64(got), bits_f64(ref)) <= TOL_BF16
    assert ulp_diff_bf16(got, ref).max() <= 2


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def run_gpu_decode(dec, steps, keep=()):
    cs = dev_bf16(dec.conv_state)
    st = dev_f32(dec.state)
    cw = dev_bf16(dec.conv_w)
    Al, db = dev_f32(dec.A_log), dev_f32(dec.dt_bias)
    xs, as_, bs = dev_bf16(dec.x), dev_bf16(dec.a), dev_bf16(dec.b)
    outs = {}
    for s in range(steps):
        o = G.decode_step(xs[s], cw, cs, as_[s], bs[s], Al, db, st, scale=dec.scale, hk=dec.hk)
        if s in keep:
            outs[s] = host_bits(o)
    torch.cuda.synchronize()
    return outs, st.cpu().numpy(), host_bits(cs)


def test_decode_small_batch_several_steps():
    dec = GI.make_decode_inputs(52, 3, 6)
    outs, st, cs = run_gpu_decode(dec, 6, keep=range(6))
    kept, H, ref_cs = O.decode_steps(dec, keep_o=tuple(range(6)))
    for s in range(6):
        assert rel_l2(bits_f64(outs[s]), bits_f64(kept[s])) <= TOL_BF16, s
    assert rel_l2(st, H) <= TOL_STATE
    assert np.array_equal(cs, O.round_bf16(ref_cs))


@pytest.mark.parametrize("case", ["no_decay", "instant_decay", "no_write", "full_write"])
def test_decode_degenerate_gates(case):
    """The decode step at the gates' limits (as the prefill test of the same name)."""
    dec = GI.make_decode_inputs(54, 2, 3)
    if case == "no_decay":
        dec.A_log = np.full(dec.hv, -1e30, np.float32)
    elif case == "instant_decay":
        dec.A_log = np.full(dec.hv, np.log(16.0), np.float32)
        dec.a = GI.f32_to_bf16_bits(np.full(dec.a.shape, 20.0, np.float32))
    elif case == "no_write":
        dec.b = GI.f32_to_bf16_bits(np.full(dec.b.shape, -200.0, np.float32))
    else:
        dec.b = GI.f32_to_bf16_bits(np.full(dec.b.shape, 200.0, np.float32))
    outs, st, cs = run_gpu_decode(dec, 3, keep=range(3))
    kept, H, ref_cs = O.decode_steps(dec, keep_o=tuple(range(3)))
    for s in range(3):
        assert rel_l2(bits_f64(outs[s]), bits_f64(kept[s])) <= TOL_BF16, s
    assert rel_l2(st, H) <= TOL_STATE
    assert np.array_equal(cs, O.round_bf16(ref_cs))


def test_decode_full_batch_sampled_heads():
    dec = GI.make_decode_inputs(53, 64, 3)
    heads = [0, 1, 2, 25, 47]
    outs, st, cs = run_gpu_decode(dec, 3, keep=(2,))
    kept, H, ref_cs = O.decode_steps(dec, heads=heads, keep_o=(2,))
    assert rel_l2(bits_f64(outs[2][:, heads]), bits_f64(kept[2][:, heads])) <= TOL_BF16
    assert rel_l2(st[:, heads], H[:, heads]) <= TOL_STATE
    assert np.array_equal(cs, O.round_bf16(ref_cs))


def test_decode_slots_match_oracle_and_plain_decode():
    """Decode on pools of cached states: live rows agree with the oracle's slot step and, bit
    for bit, with the plain decode of the same rows; padding rows are zero; entries no row
    names keep their bits; an empty pool turns every row into padding."""
    steps, S = 3, 9
    dec = GI.make_decode_inputs(55, 5, steps)
    slot = np.array([7, -1, 0, 3, S + 2], np.int32)
    live = [0, 2, 3]
    r = np.random.default_rng(56)
    C = dec.x.shape[2]
    cpool = GI.f32_to_bf16_bits(r.standard_normal((S, 3, C)).astype(np.float32))
    spool = (r.standard_normal((S, dec.hv, 128, 128)) * 0.02).astype(np.float32)
    for row in live:
        cpool[slot[row]] = dec.conv_state[row]
        spool[slot[row]] = dec.state[row]
    cw = dev_bf16(dec.conv_w)
    Al, db = dev_f32(dec.A_log), dev_f32(dec.dt_bias)
    xs, as_, bs = dev_bf16(dec.x), dev_bf16(dec.a), dev_bf16(dec.b)
    cp_d, sp_d, slot_d = dev_bf16(cpool), dev_f32(spool), dev_i32(slot)
    outs = []
    for s in range(steps):
        o = torch.full((5, dec.hv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        G.decode_step_slots(xs[s], cw, cp_d, as_[s], bs[s], Al, db, sp_d, slot_d, o=o, scale=dec.scale)
        outs.append(host_bits(o))
    torch.cuda.synchronize()
    sp_got, cp_got = sp_d.cpu().numpy(), host_bits(cp_d)

    # the oracle's slot step, carried over the steps
    cp_ref, sp_ref = O.bf16_to_f64(cpool), spool.astype(np.float64)
    for s in range(steps):
        o_ref, cp_ref, sp_ref = O.decode_step_slots(dec.x[s], dec.a[s], dec.b[s], dec.conv_w, dec.A_log,
                                                    dec.dt_bias, cp_ref, sp_ref, slot, dec.hk, dec.hv,
                                                    scale=dec.scale)
        assert rel_l2(bits_f64(outs[s][live]), bits_f64(o_ref[live])) <= TOL_BF16, s
        assert not outs[s][[1, 4]].any(), s
    ids = slot[live]
    assert rel_l2(sp_got[ids], sp_ref[ids]) <= TOL_STATE
    assert np.array_equal(cp_got, O.round_bf16(cp_ref))
    untouched = [e for e in range(S) if e not in ids]
    assert np.array_equal(sp_got[untouched], spool[untouched])

    # the plain decode of the live rows gives the same bits
    plain = GI.DecodeInputs(dec.x[:, live], dec.a[:, live], dec.b[:, live], dec.conv_w,
                            dec.conv_state[live], dec.state[live], dec.A_log, dec.dt_bias,
                            dec.hk, dec.hv, scale=dec.scale)
    p_outs, p_st, p_cs = run_gpu_decode(plain, steps, keep=range(steps))
    for s in range(steps):
        assert np.array_equal(outs[s][live], p_outs[s]), s
    assert np.array_equal(sp_got[ids], p_st)
    assert np.array_equal(cp_got[ids], p_cs)

    # an empty pool: every row is padding
    o = torch.full((2, dec.hv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    G.decode_step_slots(xs[0][:2], cw, torch.empty((0, 3, C), dtype=torch.bfloat16, device="cuda"),
                        as_[0][:2], bs[0][:2], Al, db,
                        torch.empty((0, dec.hv, 128, 128), dtype=torch.float32, device="cuda"),
                        dev_i32(np.array([-1, 0], np.int32)), o=o)
    assert not host_bits(o).any()


# ---------------------------------------------------------------------------
# chunked prefill
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("window", [None, 1])
def test_prefill_into_pool_entries_then_decode_from_the_pool(window):
    """Mixed serving batch on one pool of cached states: new requests are prefilled into their
    entries (from zero), a sequence without an entry keeps nothing, a second call continues two
    entries from their states, then one decode step runs rows on prefilled and pre-existing
    entries.  Against the oracle (recurrence from the entries' states, decode on the pool) and
    bit for bit against the plain prefill on the same initial states; entries no call names
    stay unchanged bit for bit.  window=1 makes every sequence cross windows (pool entries in
    place, the entry-less sequence through the workspace carry)."""
    S, hv = 6, 48
    r = np.random.default_rng(57)
    pool0 = (r.standard_normal((S, hv, 128, 128)) * 0.02).astype(np.float32)
    pool = dev_f32(pool0)
    # call 1: lengths 70, 0, 5, 130 into entries 4, 1, none, 2, from zero
    inp = GI.make_core_inputs(94, [70, 0, 5, 130], prenorm_qk=False)
    slot1 = np.array([4, 1, -1, 2], np.int32)
    args = (dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.a), dev_bf16(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_i32(inp.cu_seqlens), inp.cu_seqlens)
    ws = (G.prefill_workspace(inp.cu_seqlens, hv, "cuda", window=window, has_final_state=False)
          if window else None)
    o1 = G.chunk_prefill_slots(*args, pool, dev_i32(slot1), init_from_pool=False, workspace=ws)
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    ref_bits, _, ref_h = O.core_path(inp)                  # from zero states
    got = pool.cpu().numpy()
    cu = inp.cu_seqlens
    o1b = host_bits(o1)
    for n in range(4):
        s_, e_ = int(cu[n]), int(cu[n + 1])
        if e_ > s_:
            assert rel_l2(bits_f64(o1b[s_:e_]), bits_f64(ref_bits[s_:e_])) <= TOL_BF16, n
    for n, e in ((0, 4), (3, 2)):
        assert rel_l2(got[e], ref_h[n]) <= TOL_STATE, n
    assert not got[1].any()                                 # an empty new request: zero state
    for e in (0, 3, 5):                                     # entries no sequence names
        assert np.array_equal(got[e], pool0[e]), e
    # bit for bit the plain prefill from zero states
    hT = torch.empty((4, hv, 128, 128), device="cuda")
    o_plain = G.chunk_prefill(*args, hT=hT)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(o_plain), o1b)
    hTn = hT.cpu().numpy()
    assert np.array_equal(got[4], hTn[0]) and np.array_equal(got[2], hTn[3])

    # call 2: continue entries 4 and 0 from their states (lengths 64, 33)
    inp2 = GI.make_core_inputs(95, [64, 33], prenorm_qk=False)
    slot2 = np.array([4, 0], np.int32)
    before = pool.cpu().numpy()
    inp2.h0 = np.ascontiguousarray(before[slot2])
    args2 = (dev_bf16(inp2.q), dev_bf16(inp2.k), dev_bf16(inp2.v), dev_bf16(inp2.a), dev_bf16(inp2.b),
             dev_f32(inp2.A_log), dev_f32(inp2.dt_bias), dev_i32(inp2.cu_seqlens), inp2.cu_seqlens)
    ws2 = (G.prefill_workspace(inp2.cu_seqlens, hv, "cuda", window=window, has_final_state=False)
           if window else None)
    o2 = G.chunk_prefill_slots(*args2, pool, dev_i32(slot2), init_from_pool=True, workspace=ws2)
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    ref2_bits, _, ref2_h = O.core_path(inp2)
    got2 = pool.cpu().numpy()
    o2b = host_bits(o2)
    for n in range(2):
        s_, e_ = int(inp2.cu_seqlens[n]), int(inp2.cu_seqlens[n + 1])
        assert rel_l2(bits_f64(o2b[s_:e_]), bits_f64(ref2_bits[s_:e_])) <= TOL_BF16, n
        assert rel_l2(got2[slot2[n]], ref2_h[n]) <= TOL_STATE, n
    for e in (1, 2, 3, 5):
        assert np.array_equal(got2[e], before[e]), e

    # one decode step on rows naming a prefilled entry (2), a continued one (4), an untouched
    # one (5) and a padding row, from the same pool
    dec = GI.make_decode_inputs(96, 4, 1)
    slot3 = np.array([2, 4, 5, -1], np.int32)
    C = dec.x.shape[2]
    cpool0 = GI.f32_to_bf16_bits(r.standard_normal((S, 3, C)).astype(np.float32))
    cp_d = dev_bf16(cpool0)
    od = torch.full((4, hv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    G.decode_step_slots(dev_bf16(dec.x[0]), dev_bf16(dec.conv_w), cp_d, dev_bf16(dec.a[0]), dev_bf16(dec.b[0]),
                        dev_f32(dec.A_log), dev_f32(dec.dt_bias), pool, dev_i32(slot3), o=od)
    torch.cuda.synchronize()
    o_ref, _, sp_ref = O.decode_step_slots(dec.x[0], dec.a[0], dec.b[0], dec.conv_w, dec.A_log, dec.dt_bias,
                                           O.bf16_to_f64(cpool0), got2.astype(np.float64), slot3, dec.hk, dec.hv)
    odb = host_bits(od)
    assert rel_l2(bits_f64(odb[:3]), bits_f64(o_ref[:3])) <= TOL_BF16
    assert not odb[3].any()
    got3 = pool.cpu().numpy()
    for e in (2, 4, 5):
        assert rel_l2(got3[e], sp_ref[e]) <= TOL_STATE, e
    for e in (0, 1, 3):
        assert np.array_equal(got3[e], got2[e]), e


@pytest.mark.parametrize("lengths", [[1], [63], [64], [65], [200], [1, 64, 65, 0, 130, 3]])
def test_prefill_lengths_and_varlen(lengths):
    inp = GI.make_core_inputs(60 + len(lengths), lengths, prenorm_qk=False, h0_std=0.02)
    check_core(inp)


@pytest.mark.parametrize("window", [1, 3])
@pytest.mark.parametrize("final_state", [True, False])
def test_prefill_windows_carry_state(window, final_state):
    """Sequences longer than the workspace window: the state crosses windows in hT, or in the
    workspace tail when the caller asks for no final state."""
    inp = GI.make_core_inputs(80 + window, [300, 64, 1, 190], prenorm_qk=False, h0_std=0.02)
    hv = inp.v.shape[1]
    hT = torch.full((inp.n_seqs, hv, 128, 128), float("nan"), device="cuda") if final_state else None
    ws = G.prefill_workspace(inp.cu_seqlens, hv, "cuda", window=window, has_final_state=final_state)
    o = G.chunk_prefill(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.a),
                        dev_bf16(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias),
                        dev_i32(inp.cu_seqlens), inp.cu_seqlens, h0=dev_f32(inp.h0), hT=hT,
                        scale=inp.scale, workspace=ws)
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    ref_bits, _, ref_hT = O.core_path(inp)
    o_bits = host_bits(o)
    cu = inp.cu_seqlens
    for n in range(inp.n_seqs):
        s, e = int(cu[n]), int(cu[n + 1])
        assert rel_l2(bits_f64(o_bits[s:e]), bits_f64(ref_bits[s:e])) <= TOL_BF16
    if final_state:
        assert rel_l2(hT.cpu().numpy(), ref_hT) <= TOL_STATE


@pytest.mark.parametrize("final_state", [True, False])
def test_prefill_pipelined_windows_equal_one_window(final_state):
    """One sequence (96 chain CTAs: SMs left idle) over 41 chunks with a workspace for 32
    chunks: the call runs three windows of 16 chunks on two record buffers, the prep of window
    w + 1 beside the chain of window w on the library's own pair of streams, joined back to the
    caller's stream.  o and the final state equal a one-window call's bit for bit (the state
    crosses windows in fp32), and o matches the oracle on three heads."""
    T = 64 * 40 + 17
    inp = GI.make_core_inputs(97, [T], prenorm_qk=False, h0_std=0.02)
    hv = inp.v.shape[1]
    args = (dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.a), dev_bf16(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_i32(inp.cu_seqlens), inp.cu_seqlens)
    h0 = dev_f32(inp.h0)
    outs = []
    for window in (None, 32):
        hT = torch.full((1, hv, 128, 128), float("nan"), device="cuda") if final_state else None
        ws = G.prefill_workspace(inp.cu_seqlens, hv, "cuda", window=window, has_final_state=final_state)
        assert G.prefill_schedule(inp.cu_seqlens, hv, ws.numel(), final_state) == ((1, False) if window is None
                                                                                     else (3, True))
        o = torch.full((T, hv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        G.chunk_prefill(*args, h0=h0, hT=hT, o=o, scale=inp.scale, workspace=ws)
        torch.cuda.synchronize()
        assert G.get_device_error() == 0
        outs.append((host_bits(o), None if hT is None else hT.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0])
    if final_state:
        assert np.array_equal(outs[0][1], outs[1][1])
    heads = [0, 25, 47]
    ref_bits, _, ref_hT = O.core_path(inp, heads=heads)
    assert rel_l2(bits_f64(outs[1][0][:, heads]), bits_f64(ref_bits[:, heads])) <= TOL_BF16
    if final_state:
        assert rel_l2(outs[1][1][:, heads], ref_hT[:, heads]) <= TOL_STATE
    # the same call captured into a graph keeps to the caller's stream (one buffer at a time)
    # and replays the eager bits
    hT = torch.empty((1, hv, 128, 128), device="cuda") if final_state else None
    ws = G.prefill_workspace(inp.cu_seqlens, hv, "cuda", window=32, has_final_state=final_state)
    o = torch.empty((T, hv, 128), dtype=torch.bfloat16, device="cuda")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        G.chunk_prefill(*args, h0=h0, hT=hT, o=o, scale=inp.scale, workspace=ws)
    o.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    assert np.array_equal(host_bits(o), outs[0][0])
    if final_state:
        assert np.array_equal(hT.cpu().numpy(), outs[0][1])
        # the pooled form on the same schedule: entry 2 of a 3-entry pool holds h0 and receives
        # the final state, in place across the pipelined windows
        pool = torch.zeros((3, hv, 128, 128), device="cuda")
        pool[2] = h0[0]
        ws = G.prefill_workspace(inp.cu_seqlens, hv, "cuda", window=32, has_final_state=False)
        assert G.prefill_schedule(inp.cu_seqlens, hv, ws.numel(), has_final_state=False) == (3, True)
        o = G.chunk_prefill_slots(*args, pool, dev_i32(np.array([2], np.int32)), init_from_pool=True,
                                  scale=inp.scale, workspace=ws)
        torch.cuda.synchronize()
        assert G.get_device_error() == 0
        assert np.array_equal(host_bits(o), outs[0][0])
        assert np.array_equal(pool[2:].cpu().numpy(), outs[0][1])
        assert not pool[:2].cpu().numpy().any()


@pytest.mark.parametrize("case", ["no_decay", "instant_decay", "no_write", "full_write"])
def test_prefill_degenerate_gates(case):
    """Limits of the gates on the GPU path: g = 0 (exp(A_log) = 0), g far below zero (the
    state is forgotten at every token), beta = 0 (nothing is written, the state only decays)
    and beta = 1 (every token overwrites)."""
    inp = GI.make_core_inputs(90, [130, 64], prenorm_qk=False, h0_std=0.02)
    hv = inp.v.shape[1]
    if case == "no_decay":
        inp.A_log = np.full(hv, -1e30, np.float32)
    elif case == "instant_decay":   # g = -16 softplus(20 + dt_bias), about -320 per token
        inp.A_log = np.full(hv, np.log(16.0), np.float32)
        inp.a = GI.f32_to_bf16_bits(np.full(inp.a.shape, 20.0, np.float32))
    elif case == "no_write":
        inp.b = GI.f32_to_bf16_bits(np.full(inp.b.shape, -200.0, np.float32))
    else:
        inp.b = GI.f32_to_bf16_bits(np.full(inp.b.shape, 200.0, np.float32))
    check_core(inp)


def test_prefill_scale_and_zero_initial_state():
    inp = GI.make_core_inputs(70, [150, 7], prenorm_qk=True, scale=128 ** -0.5)
    check_core(inp)


def test_prefill_in_place_state():
    inp = GI.make_core_inputs(71, [90, 40], prenorm_qk=False, h0_std=0.02)
    check_core(inp, h0_inplace=True)


def test_prefill_key_heads_group_contiguously():
    inp = GI.make_core_inputs(72, [70], hk=16, hv=48, prenorm_qk=False)
    o1, _ = gpu_core(inp)
    k2 = inp.k.copy()
    k2[:, 1] = GI.f32_to_bf16_bits(GI.bf16_bits_to_f32(k2[:, 1]) * np.float32(-1.5) + np.float32(0.3))
    inp.k = k2
    o2, _ = gpu_core(inp)
    moved = [h for h in range(48) if not np.array_equal(o1[:, h], o2[:, h])]
    assert moved == [3, 4, 5]


def test_prefill_workload_T128():
    eo, eh = check_core(GI.workload_core_T128())
    print(f"T=128: o rel-L2 {eo:.2e}, state rel-L2 {eh:.2e}")


def test_full_path_T4096_unfused():
    """conv -> prefill -> gated norm as three calls, against the oracle."""
    inp = GI.workload_full_T4096()
    cu_d = dev_i32(inp.cu_seqlens)
    x = dev_bf16(inp.x)
    y = G.causal_conv(x, dev_bf16(inp.conv_w), cu_d, inp.cu_seqlens)
    T = inp.T
    hk, hv = inp.hk, inp.hv
    q = y[:, : hk * 128].view(T, hk, 128)            # strided views of the conv output
    k = y[:, hk * 128: 2 * hk * 128].view(T, hk, 128)
    v = y[:, 2 * hk * 128:].view(T, hv, 128)
    hT = torch.empty((1, hv, 128, 128), device="cuda")
    o = G.chunk_prefill(q, k, v, dev_bf16(inp.a), dev_bf16(inp.b), dev_f32(inp.A_log),
                        dev_f32(inp.dt_bias), cu_d, inp.cu_seqlens, hT=hT, scale=inp.scale)
    out = G.gated_rmsnorm(o, dev_bf16(inp.z).reshape(T, hv, 128), None, eps=inp.eps)
    torch.cuda.synchronize()
    ref = O.full_path(inp)
    assert rel_l2(bits_f64(host_bits(o)), bits_f64(ref["o"])) <= TOL_BF16
    assert rel_l2(bits_f64(host_bits(out)), bits_f64(ref["y"])) <= TOL_BF16
    assert rel_l2(hT.cpu().numpy(), ref["hT"]) <= TOL_STATE


def run_full_gpu(inp, fused_norm, keep_o=False):
    """conv -> prefill (-> gated norm, fused into the prefill or as its own call)."""
    cu_d = dev_i32(inp.cu_seqlens)
    y = G.causal_conv(dev_bf16(inp.x), dev_bf16(inp.conv_w), cu_d, inp.cu_seqlens)
    T, hk, hv = inp.T, inp.hk, inp.hv
    q = y[:, : hk * 128].view(T, hk, 128)
    k = y[:, hk * 128: 2 * hk * 128].view(T, hk, 128)
    v = y[:, 2 * hk * 128:].view(T, hv, 128)
    hT = torch.empty((inp.n_seqs, hv, 128, 128), device="cuda")
    z = dev_bf16(inp.z).reshape(T, hv, 128)
    w = dev_f32(inp.norm_w) if inp.norm_w is not None else None
    h0 = dev_f32(inp.h0) if inp.h0 is not None else None
    args = (q, k, v, dev_bf16(inp.a), dev_bf16(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias), cu_d,
            inp.cu_seqlens)
    if fused_norm:
        out = torch.full((T, hv, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        o = torch.empty((T, hv, 128), dtype=torch.bfloat16, device="cuda") if keep_o else None
        G.chunk_prefill(*args, h0=h0, hT=hT, o=o, scale=inp.scale,
                        fuse={"z": z, "norm_w": w, "eps": inp.eps, "y": out})
    else:
        o = G.chunk_prefill(*args, h0=h0, hT=hT, scale=inp.scale)
        out = G.gated_rmsnorm(o, z, w, eps=inp.eps)
    torch.cuda.synchronize()
    return (host_bits(o) if o is not None else None), host_bits(out), hT.cpu().numpy()


def test_fused_gated_norm_varlen_matches_unfused_and_oracle():
    """The gated RMSNorm fused into the prefill's output equals the separate norm call."""
    inp = GI.make_full_inputs(80, [200, 65, 1, 0, 130], h0_std=0.02, norm_w_std=0.1)
    o_u, y_u, h_u = run_full_gpu(inp, fused_norm=False)
    o_f, y_f, h_f = run_full_gpu(inp, fused_norm=True, keep_o=True)
    assert np.array_equal(o_f, o_u)                 # the recurrence is the same
    assert np.array_equal(h_f, h_u)
    assert ulp_diff_bf16(y_f, y_u).max() <= 1       # only the sum-of-squares order differs
    ref = O.full_path(inp)
    assert rel_l2(bits_f64(y_f), bits_f64(ref["y"])) <= TOL_BF16
    cu = inp.cu_seqlens
    for n in range(inp.n_seqs):                     # every sequence on its own
        s, e = int(cu[n]), int(cu[n + 1])
        if e > s:
            assert rel_l2(bits_f64(y_f[s:e]), bits_f64(ref["y"][s:e])) <= TOL_BF16


def run_fused_conv_gpu(inp, fused_norm):
    """One gdr_chunk_prefill call that runs the conv too (fuse.x), optionally the norm."""
    cu_d = dev_i32(inp.cu_seqlens)
    T, hv = inp.T, inp.hv
    hT = torch.full((inp.n_seqs, hv, 128, 128), float("nan"), device="cuda")
    cs_out = torch.full(inp.conv_state.shape if inp.conv_state is not None else (inp.n_seqs, 3, inp.x.shape[1]),
                        float("nan"), dtype=torch.bfloat16, device="cuda")
    fuse = {"x": dev_bf16(inp.x), "conv_w": dev_bf16(inp.conv_w), "hk": inp.hk, "conv_state_out": cs_out}
    if inp.conv_state is not None:
        fuse["conv_state_in"] = dev_bf16(inp.conv_state)
    y = None
    if fused_norm:
        y = torch.empty((T, hv, 128), dtype=torch.bfloat16, device="cuda")
        fuse.update({"z": dev_bf16(inp.z).reshape(T, hv, 128), "eps": inp.eps, "y": y, "keep_o": True,
                     "norm_w": dev_f32(inp.norm_w) if inp.norm_w is not None else None})
    h0 = dev_f32(inp.h0) if inp.h0 is not None else None
    o = G.chunk_prefill(None, None, None, dev_bf16(inp.a), dev_bf16(inp.b), dev_f32(inp.A_log),
                        dev_f32(inp.dt_bias), cu_d, inp.cu_seqlens, h0=h0, hT=hT, scale=inp.scale, fuse=fuse)
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    return host_bits(o), (host_bits(y) if y is not None else None), hT.cpu().numpy(), host_bits(cs_out)


@pytest.mark.parametrize("fused_norm", [False, True])
def test_fused_conv_equals_separate_calls(fused_norm):
    """The conv fused into the prefill call gives the separate calls' results bit for bit,
    conv state included, on packed sequences with empty ones, conv and recurrent states."""
    inp = GI.make_full_inputs(81, [200, 65, 1, 0, 130], h0_std=0.02, conv_state_std=1.0, norm_w_std=0.1)
    o_f, y_f, h_f, cs_f = run_fused_conv_gpu(inp, fused_norm)
    # the same three kernels called one by one
    cu_d = dev_i32(inp.cu_seqlens)
    T, hk, hv = inp.T, inp.hk, inp.hv
    cs_sep = torch.empty(inp.conv_state.shape, dtype=torch.bfloat16, device="cuda")
    yc = G.causal_conv(dev_bf16(inp.x), dev_bf16(inp.conv_w), cu_d, inp.cu_seqlens,
                       dev_bf16(inp.conv_state), cs_sep)
    q = yc[:, : hk * 128].view(T, hk, 128)
    k = yc[:, hk * 128: 2 * hk * 128].view(T, hk, 128)
    v = yc[:, 2 * hk * 128:].view(T, hv, 128)
    hT = torch.empty((inp.n_seqs, hv, 128, 128), device="cuda")
    o = G.chunk_prefill(q, k, v, dev_bf16(inp.a), dev_bf16(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias),
                        cu_d, inp.cu_seqlens, h0=dev_f32(inp.h0), hT=hT, scale=inp.scale)
    torch.cuda.synchronize()
    assert np.array_equal(o_f, host_bits(o))
    assert np.array_equal(h_f, hT.cpu().numpy())
    assert np.array_equal(cs_f, host_bits(cs_sep))
    ref = O.full_path(inp)
    assert np.array_equal(cs_f, ref["conv_state_out"])
    assert rel_l2(bits_f64(o_f), bits_f64(ref["o"])) <= TOL_BF16
    assert rel_l2(h_f, ref["hT"]) <= TOL_STATE
    if fused_norm:
        assert rel_l2(bits_f64(y_f), bits_f64(ref["y"])) <= TOL_BF16


def test_prefill_step_replays_from_a_cuda_graph():
    """conv -> prefill -> gated norm captured once into a CUDA graph and replayed gives the
    eager results bit for bit: the calls enqueue only kernels on the caller's stream."""
    inp = GI.make_full_inputs(82, [300, 70], h0_std=0.02)
    T, hk, hv = inp.T, inp.hk, inp.hv
    cu_d = dev_i32(inp.cu_seqlens)
    x, w = dev_bf16(inp.x), dev_bf16(inp.conv_w)
    a, b = dev_bf16(inp.a), dev_bf16(inp.b)
    Al, db, h0 = dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_f32(inp.h0)
    z = dev_bf16(inp.z).reshape(T, hv, 128)
    conv_y = torch.empty_like(x)
    o = torch.empty((T, hv, 128), dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(o)
    hT = torch.empty((inp.n_seqs, hv, 128, 128), device="cuda")
    ws = G.prefill_workspace(inp.cu_seqlens, hv, "cuda")

    def step():
        G.causal_conv(x, w, cu_d, inp.cu_seqlens, None, None, conv_y)
        q = conv_y[:, : hk * 128].view(T, hk, 128)
        k = conv_y[:, hk * 128: 2 * hk * 128].view(T, hk, 128)
        v = conv_y[:, 2 * hk * 128:].view(T, hv, 128)
        G.chunk_prefill(q, k, v, a, b, Al, db, cu_d, inp.cu_seqlens, h0=h0, hT=hT, o=o, scale=inp.scale,
                        workspace=ws)
        G.gated_rmsnorm(o, z, None, inp.eps, y)

    step()   # eager (also the library's one-time set-up)
    torch.cuda.synchronize()
    eager = (host_bits(o), host_bits(y), hT.cpu().numpy())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for t in (o, y, hT, conv_y):
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    assert np.array_equal(host_bits(o), eager[0])
    assert np.array_equal(host_bits(y), eager[1])
    assert np.array_equal(hT.cpu().numpy(), eager[2])


def test_full_path_T4096_fused_norm():
    """The bench workload with the gated norm fused, against the oracle."""
    inp = GI.workload_full_T4096()
    _, y_f, h_f = run_full_gpu(inp, fused_norm=True)
    ref = O.full_path(inp)
    assert rel_l2(bits_f64(y_f), bits_f64(ref["y"])) <= TOL_BF16
    assert rel_l2(h_f, ref["hT"]) <= TOL_STATE


def test_prefill_long_context_sampled_heads():
    """B=1, T=262144: every head on the GPU, three heads through the oracle.  The bounds hold
    over the whole sequence, over every 4096-token window (64 chunks) of every sampled head
    and over the last chunk alone, so that an error confined to one stretch of the 4096-chunk
    state carry cannot hide in the total."""
    inp = GI.workload_core_T262144()
    heads = [0, 23, 47]
    o_bits, hT = gpu_core(inp)
    ref_bits, _, ref_hT = O.core_path(inp, heads=heads)
    got = bits_f64(o_bits[:, heads])
    ref = bits_f64(ref_bits[:, heads])
    del o_bits, ref_bits
    assert np.all(np.isfinite(hT))
    eo, eh = rel_l2(got, ref), rel_l2(hT[:, heads], ref_hT[:, heads])
    assert eo <= TOL_BF16, f"o rel-L2 {eo:.3e}"
    assert eh <= TOL_STATE, f"state rel-L2 {eh:.3e}"
    W = 64 * 64
    worst = max((rel_l2(got[s:s + W, j], ref[s:s + W, j]), s, heads[j])
                for s in range(0, inp.T, W) for j in range(len(heads)))
    assert worst[0] <= TOL_BF16, f"window at token {worst[1]}, head {worst[2]}: rel-L2 {worst[0]:.3e}"
    for j, h in enumerate(heads):
        assert rel_l2(got[-64:, j], ref[-64:, j]) <= TOL_BF16, h
        assert rel_l2(hT[0, h], ref_hT[0, h]) <= TOL_STATE, h
    print(f"T=262144: o rel-L2 {eo:.2e} (worst window {worst[0]:.2e}), state rel-L2 {eh:.2e}")


def test_prefill_varlen8_full_path_sampled_heads():
    """8 packed sequences of U{1024..32768} tokens with initial states, the full path; two
    value heads through the oracle.  o, y and the final state are checked over all
    sequences and over each sequence on its own."""
    inp = GI.workload_full_varlen8()
    cu_d = dev_i32(inp.cu_seqlens)
    y = G.causal_conv(dev_bf16(inp.x), dev_bf16(inp.conv_w), cu_d, inp.cu_seqlens)
    T, hk, hv = inp.T, inp.hk, inp.hv
    q = y[:, : hk * 128].view(T, hk, 128)            # strided views of the conv output
    k = y[:, hk * 128: 2 * hk * 128].view(T, hk, 128)
    v = y[:, 2 * hk * 128:].view(T, hv, 128)
    hT = torch.empty((inp.n_seqs, hv, 128, 128), device="cuda")
    o = G.chunk_prefill(q, k, v, dev_bf16(inp.a), dev_bf16(inp.b), dev_f32(inp.A_log),
                        dev_f32(inp.dt_bias), cu_d, inp.cu_seqlens, h0=dev_f32(inp.h0), hT=hT,
                        scale=inp.scale)
    out = G.gated_rmsnorm(o, dev_bf16(inp.z).reshape(T, hv, 128), None, eps=inp.eps)
    torch.cuda.synchronize()
    heads = [5, 40]
    ref = O.full_path(inp, heads=heads)
    got = {"o": bits_f64(host_bits(o)[:, heads]), "y": bits_f64(host_bits(out)[:, heads])}
    want = {"o": bits_f64(ref["o"][:, heads]), "y": bits_f64(ref["y"][:, heads])}
    got_h, want_h = hT.cpu().numpy()[:, heads], ref["hT"][:, heads]
    for key in ("o", "y"):
        assert rel_l2(got[key], want[key]) <= TOL_BF16, key
    assert rel_l2(got_h, want_h) <= TOL_STATE
    cu = inp.cu_seqlens
    for n in range(inp.n_seqs):
        s, e = int(cu[n]), int(cu[n + 1])
        for key in ("o", "y"):
            assert rel_l2(got[key][s:e], want[key][s:e]) <= TOL_BF16, (key, n)
        assert rel_l2(got_h[n], want_h[n]) <= TOL_STATE, n


# ---------------------------------------------------------------------------
# head sharding: the layer split over GPUs by heads needs no exchange
# ---------------------------------------------------------------------------

def _shard_channels(C_hk, C_hv, hk, hv, shard, n_shards):
    """Channel indices of one head shard in the [q | k | v] layout: its key heads' q and k
    channels and its value heads' v channels (contiguous head groups)."""
    ks, vs = hk // n_shards, hv // n_shards
    q = np.arange(shard * ks * 128, (shard + 1) * ks * 128)
    k = C_hk + q
    v = 2 * C_hk + np.arange(shard * vs * 128, (shard + 1) * vs * 128)
    return np.concatenate([q, k, v]), slice(shard * ks, (shard + 1) * ks), slice(shard * vs, (shard + 1) * vs)


def test_head_sharded_layer_equals_the_full_layer():
    """Two head shards (8 key / 24 value heads each, as a 2-GPU split of the layer would hold
    them) run through the same entry points on their slices of the inputs give the full
    layer's o, final states and conv states bit for bit: heads never exchange data inside the
    layer, so sharding by heads is a split of the inputs and nothing else (here both shards run
    on one GPU, one after the other)."""
    hk, hv = GI.HK, GI.HV
    n = 2
    # prefill: several windows, varlen, initial states
    inp = GI.make_core_inputs(98, [300, 64, 129], prenorm_qk=False, h0_std=0.02)
    full_o, full_h = None, None
    def run(q, k, v, a, b, Al, db, h0):
        hT = torch.empty_like(h0)
        o = G.chunk_prefill(q, k, v, a, b, Al, db, dev_i32(inp.cu_seqlens), inp.cu_seqlens, h0=h0, hT=hT)
        torch.cuda.synchronize()
        return host_bits(o), hT.cpu().numpy()
    full_o, full_h = run(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_bf16(inp.a), dev_bf16(inp.b),
                         dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_f32(inp.h0))
    for s in range(n):
        _, ks, vs = _shard_channels(hk * 128, hv * 128, hk, hv, s, n)
        o, h = run(dev_bf16(np.ascontiguousarray(inp.q[:, ks])), dev_bf16(np.ascontiguousarray(inp.k[:, ks])),
                   dev_bf16(np.ascontiguousarray(inp.v[:, vs])), dev_bf16(np.ascontiguousarray(inp.a[:, vs])),
                   dev_bf16(np.ascontiguousarray(inp.b[:, vs])), dev_f32(inp.A_log[vs]), dev_f32(inp.dt_bias[vs]),
                   dev_f32(np.ascontiguousarray(inp.h0[:, vs])))
        assert np.array_equal(o, full_o[:, vs]), s
        assert np.array_equal(h, full_h[:, vs]), s
    assert G.get_device_error() == 0

    # decode: conv step, norms, gates and the state update on the shard's channels and heads
    dec = GI.make_decode_inputs(99, 4, 2)
    f_outs, f_st, f_cs = run_gpu_decode(dec, 2, keep=(0, 1))
    for s in range(n):
        ch, ks, vs = _shard_channels(hk * 128, hv * 128, hk, hv, s, n)
        part = GI.DecodeInputs(np.ascontiguousarray(dec.x[:, :, ch]), np.ascontiguousarray(dec.a[:, :, vs]),
                               np.ascontiguousarray(dec.b[:, :, vs]), np.ascontiguousarray(dec.conv_w[ch]),
                               np.ascontiguousarray(dec.conv_state[:, :, ch]),
                               np.ascontiguousarray(dec.state[:, vs]), dec.A_log[vs], dec.dt_bias[vs],
                               hk // n, hv // n, scale=dec.scale)
        outs, st, cs = run_gpu_decode(part, 2, keep=(0, 1))
        for step in (0, 1):
            assert np.array_equal(outs[step], f_outs[step][:, vs]), (s, step)
        assert np.array_equal(st, f_st[:, vs]), s
        assert np.array_equal(cs, f_cs[:, :, ch]), s


# ---------------------------------------------------------------------------
# the layer's projections
# ---------------------------------------------------------------------------

def _ulp_diff(a_bits, b_bits):
    """Distance in bf16 units in the last place between two arrays of finite bf16 bits."""
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - u, u)   # order-preserving map of the bit patterns
    return np.abs(key(a_bits) - key(b_bits))


def _check_linear(got, ref, x, w):
    """Element by element within the bound of the arithmetic: the GPU sums K products in fp32
    (error at most K 2^-24 sum_k |x_k w_k|, the usual bound for recursive summation) and both
    sides round to bf16 (together at most one ulp of the larger value); and rel-L2 <= 1e-3."""
    g, r = bits_f64(got), bits_f64(ref)
    K = x.shape[1]
    mag = np.abs(O.bf16_to_f64(x)) @ np.abs(O.bf16_to_f64(w)).T
    big = np.maximum(np.abs(g), np.abs(r))
    ulp = np.exp2(np.floor(np.log2(np.maximum(big, 1e-300))) - 7)   # bf16: 8 significant bits
    assert np.all(np.abs(g - r) <= ulp + K * 2.0 ** -24 * mag)
    assert rel_l2(g, r) <= 1e-3


@pytest.mark.parametrize("M,N,K", [(300, 600, 512), (128, 48, 5120), (1, 8, 8), (257, 264, 136), (129, 256, 64)])
def test_linear_matches_oracle(M, N, K):
    """y = x W^T against the fp64 product rounded to bf16, element by element: ragged tiles in M
    (tile 128), N (tile 256) and K (step 64) and the a/b projection's N = 48.  The GPU sums in
    fp32, so an output may round to a neighbouring bf16 value (rarely; further only where the
    sum cancels to far below its terms)."""
    x, w = GI.make_linear_inputs(M + 7 * N + 13 * K, M, N, K)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    G.linear(dev_bf16(x), dev_bf16(w), y)
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    got, ref = host_bits(y), O.linear(x, w)
    _check_linear(got, ref, x, w)
    assert np.mean(_ulp_diff(got, ref) > 0) < 0.02


@pytest.mark.parametrize("which", ["in_proj", "out_proj"])
def test_linear_projections_full_size_sampled_rows(which):
    """The two projections of the T = 4096 prefill at full size (4096 x 5120 -> 16 480 and
    4096 x 6144 -> 5120), 40 rows (including the first and last) against the oracle."""
    x, w = GI.workload_in_proj_T4096() if which == "in_proj" else GI.workload_out_proj_T4096()
    M, N = x.shape[0], w.shape[0]
    y = G.linear(dev_bf16(x), dev_bf16(w))
    torch.cuda.synchronize()
    assert G.get_device_error() == 0
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(8).choice(M, 38, replace=False)]))
    got = y[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    ref = O.linear(x[rows], w)
    _check_linear(got, ref, x[rows], w)


def _layer_ours(h, w_in, conv_w, A_log, dt_bias, w_out, cu, hk, hv):
    """Our kernels end to end: projection -> conv -> recurrence -> gated norm -> projection
    (the normed output and the output projection's result, both bf16 bits)."""
    T = h.shape[0]
    c = 2 * hk * 128 + hv * 128
    yi = G.linear(dev_bf16(h), dev_bf16(w_in))
    x = yi[:, :c].contiguous()
    z = yi[:, c:c + hv * 128].contiguous().view(T, hv, 128)
    a = yi[:, c + hv * 128:c + hv * 128 + hv].contiguous()
    b = yi[:, c + hv * 128 + hv:].contiguous()
    conv_y = torch.empty_like(x)
    G.causal_conv(x, dev_bf16(conv_w), dev_i32(cu), cu, None, None, conv_y)
    q = conv_y[:, :hk * 128].view(T, hk, 128)
    k = conv_y[:, hk * 128:2 * hk * 128].view(T, hk, 128)
    v = conv_y[:, 2 * hk * 128:].view(T, hv, 128)
    o = G.chunk_prefill(q, k, v, a, b, dev_f32(A_log), dev_f32(dt_bias), dev_i32(cu), cu)
    y = G.gated_rmsnorm(o, z, None, 1e-6)
    out = G.linear(y.view(T, hv * 128), dev_bf16(np.ascontiguousarray(w_out)))
    torch.cuda.synchronize()
    return host_bits(y).reshape(T, hv * 128), host_bits(out)


def test_layer_with_projections_sharded_by_heads():
    """The whole layer with its projections through our kernels, unsharded and as two head
    shards (gated_delta_rule_63_b200.shard: 8 key / 24 value heads each, the shards run one
    after the other on this GPU): each shard's normed output equals the unsharded one's columns
    bit for bit; the sum of the shards' out-projection partials (the all-reduce of a two-GPU
    run) matches the unsharded output, and both match the fp64 oracle of the whole layer."""
    from gated_delta_rule_63_b200.shard import head_shard
    import tests.test_head_shard as TH
    h, w_in, w_out, conv_w, A_log, dt_bias = TH._layer_inputs()
    cu = GI.cu_seqlens_from_lengths(TH.LENGTHS)
    y_full, out_full = _layer_ours(h, w_in, conv_w, A_log, dt_bias, w_out, cu, 16, 48)
    assert G.get_device_error() == 0
    summed, bound = np.zeros(out_full.shape), np.zeros(out_full.shape)
    wf = bits_f64(w_out)
    for r in range(2):
        s = head_shard(r, 2)
        y, part = _layer_ours(h, w_in[s.in_rows], conv_w[s.conv_channels], A_log[s.heads], dt_bias[s.heads],
                              w_out[:, s.out_cols], cu, s.hk, s.hv)
        assert np.array_equal(y, y_full[:, s.out_cols]), r
        summed += bits_f64(part)
        # each partial: fp32 sum of 3072 products, rounded to bf16
        mag = np.abs(bits_f64(y)) @ np.abs(wf[:, s.out_cols]).T
        bound += 2.0 ** -8 * np.abs(bits_f64(part)) + 3072 * 2.0 ** -24 * mag
    # the partials sum to the exact product of the (shared) normed output and the weight, within
    # their roundings; so does the unsharded output, rounded once
    exact = bits_f64(y_full) @ wf.T
    assert np.all(np.abs(summed - exact) <= bound + 1e-30)
    full_mag = np.abs(bits_f64(y_full)) @ np.abs(wf).T
    assert np.all(np.abs(bits_f64(out_full) - exact) <= 2.0 ** -8 * np.abs(exact) + 6144 * 2.0 ** -24 * full_mag)
    ref_y = TH._normed(h, w_in, conv_w, A_log, dt_bias, 16, 48)
    assert rel_l2(bits_f64(y_full), bits_f64(ref_y)) <= TOL_BF16
    ref_out = O.linear(ref_y, w_out)
    assert rel_l2(bits_f64(out_full), bits_f64(ref_out)) <= TOL_BF16
