"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test checks the oracle against a hand-worked example, a closed form, an
invariant of the recurrence, a library routine or brute force, chosen so that
a dropped term, a wrong sign, a wrong index or a transposed operand in the
oracle fails at least one of them.
"""
import dataclasses
import json
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

from oracle import oracle as O
import gdr_inputs as GI

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed):
    return np.random.default_rng(seed)


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------

def test_round_bf16_ties_and_specials():
    r = O.lib().oracle_round_bf16
    assert r(1.0) == 0x3F80
    assert r(1.0 + 2 ** -8) == 0x3F80           # tie -> even (mantissa 0)
    assert r(1.0 + 3 * 2 ** -8) == 0x3F82       # tie -> even (mantissa 2)
    assert r(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81  # just above the tie rounds up
    assert r(-2.0) == 0xC000
    assert r(0.0) == 0 and r(-0.0) == 0x8000
    assert r(float("inf")) == 0x7F80


def test_round_bf16_matches_torch_on_fp32_values():
    x = rng(1).standard_normal(20000).astype(np.float32) * np.float32(37.0)
    x[:100] *= np.float32(1e-39)               # subnormals
    ours = O.round_bf16(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(ours, GI.f32_to_bf16_bits(x))


# ---------------------------------------------------------------------------
# gates
# ---------------------------------------------------------------------------

def test_gate_closed_forms():
    assert O.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert O.softplus(25.0) == 25.0                       # above the threshold
    assert O.softplus(-30.0) == pytest.approx(math.exp(-30.0), rel=1e-12)
    assert O.sigmoid(0.0) == 0.5
    g, beta = O.gates(np.zeros((1, 1)), np.zeros((1, 1)), np.zeros(1, np.float32),
                      np.zeros(1, np.float32))
    assert g[0, 0] == pytest.approx(-math.log(2.0), rel=1e-15)
    assert beta[0, 0] == 0.5
    # exp(A_log) scales the gate; dt_bias shifts the softplus argument
    g, _ = O.gates(np.full((1, 1), -1.0), np.zeros((1, 1)), np.full(1, math.log(4.0), np.float32),
                   np.full(1, 1.0, np.float32))
    assert g[0, 0] == pytest.approx(-4.0 * math.log(2.0), rel=1e-6)


def test_gates_match_torch_library():
    r = rng(2)
    a = r.standard_normal((50, 48)) * 5
    b = r.standard_normal((50, 48)) * 5
    A_log, dt_bias = GI._head_params(np.random.default_rng(3), 48)
    g, beta = O.gates(a, b, A_log, dt_bias)
    ta = torch.from_numpy(a)
    gref = -torch.exp(torch.from_numpy(A_log.astype(np.float64))) * torch.nn.functional.softplus(
        ta + torch.from_numpy(dt_bias.astype(np.float64)))
    bref = torch.sigmoid(torch.from_numpy(b))
    np.testing.assert_allclose(g, gref.numpy(), rtol=1e-14, atol=0)
    np.testing.assert_allclose(beta, bref.numpy(), rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------------------
# the recurrence
# ---------------------------------------------------------------------------

def _core_case(seed, lengths, hk=2, hv=6, dk=16, dv=8, h0=True, g_scale=1.0):
    r = rng(seed)
    T = int(sum(lengths))
    q = r.standard_normal((T, hk, dk))
    k = r.standard_normal((T, hk, dk))
    v = r.standard_normal((T, hv, dv))
    g = -np.abs(r.standard_normal((T, hv))) * g_scale
    beta = r.uniform(0, 1, (T, hv))
    cu = GI.cu_seqlens_from_lengths(lengths)
    H0 = r.standard_normal((len(lengths), hv, dk, dv)) if h0 else None
    return q, k, v, g, beta, cu, H0


def test_hand_worked_example():
    with open(os.path.join(GOLDEN, "hand_d2.json")) as f:
        G = json.load(f)
    q = np.array(G["q"])[:, None, :]
    k = np.array(G["k"])[:, None, :]
    v = np.array(G["v"])[:, None, :]
    g = np.array(G["g"])[:, None]
    beta = np.array(G["beta"])[:, None]
    cu = np.array([0, 2], np.int32)
    for fn in (O.gdr_stepwise, O.gdr_chunked):
        o, hT = fn(q, k, v, g, beta, cu, use_l2norm=False)
        np.testing.assert_allclose(o[:, 0, :], np.array(G["o"]), rtol=0, atol=1e-14)
        np.testing.assert_allclose(hT[0, 0], np.array(G["hT"]), rtol=0, atol=1e-14)


def test_beta0_g0_leaves_state_unchanged():
    q, k, v, g, beta, cu, H0 = _core_case(10, [5])
    g[:] = 0.0
    beta[:] = 0.0
    o, hT = O.gdr_stepwise(q, k, v, g, beta, cu, H0, scale=0.7)
    np.testing.assert_array_equal(hT, H0)
    qn = q / np.sqrt(np.sum(q * q, -1, keepdims=True) + 1e-6)
    for h in range(6):
        expect = 0.7 * np.einsum("ij,ti->tj", H0[0, h], qn[:, h // 3])
        np.testing.assert_allclose(o[:, h], expect, rtol=1e-12, atol=1e-12)


def test_beta1_unit_key_overwrites():
    # With beta = 1 and a unit key the new state maps k to v exactly: S k = v,
    # whatever the gate and the old state.
    r = rng(11)
    for trial in range(5):
        q, k, v, g, beta, cu, H0 = _core_case(100 + trial, [1], hk=1, hv=1, dk=32, dv=16)
        beta[:] = 1.0
        g[:] = -r.uniform(0, 3)
        _, hT = O.gdr_stepwise(q, k, v, g, beta, cu, H0)
        kn = k[0, 0] / math.sqrt(np.sum(k[0, 0] ** 2) + 1e-6)
        S = hT[0, 0].T                                      # S = H^T
        # |kn|^2 = 1 - delta with delta ~ 1e-6/|k|^2 from the norm's epsilon
        np.testing.assert_allclose(S @ kn, v[0, 0], rtol=0, atol=1e-5 * np.abs(v).max())
    # exactly unit key (no L2 norm): exact overwrite
    q, k, v, g, beta, cu, H0 = _core_case(7, [1], hk=1, hv=1, dk=32, dv=16)
    beta[:] = 1.0
    k[0, 0] = unit(k[0, 0])
    _, hT = O.gdr_stepwise(q, k, v, g, beta, cu, H0, use_l2norm=False)
    np.testing.assert_allclose(hT[0, 0].T @ k[0, 0], v[0, 0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("form", ["stepwise", "chunked"])
def test_repeated_unit_key_with_full_write_closed_form(form):
    # One exactly unit key repeated for every token, beta = 1: each token overwrites the
    # k direction and decays the rest, so H_t = e^gamma_t (I - k k^T) H0 + k v_t^T and
    # o_t = s (e^gamma_t H0^T (I - k k^T) q_t + v_t (k . q_t)).  In the chunked form every
    # A entry of a chunk then carries k.k = 1, the most correlated keys can be.
    q, k, v, g, beta, cu, H0 = _core_case(17, [150], hk=1, hv=1, dk=32, dv=16)
    kk = unit(rng(18).standard_normal(32))
    k[:, 0] = kk
    beta[:] = 1.0
    g *= 0.05
    scale = 0.7
    fn = O.gdr_stepwise if form == "stepwise" else O.gdr_chunked
    o, hT = fn(q, k, v, g, beta, cu, H0, scale=scale, use_l2norm=False)
    P = np.eye(32) - np.outer(kk, kk)
    gam = np.cumsum(g[:, 0])
    for t in range(150):
        ref = scale * (math.exp(gam[t]) * H0[0, 0].T @ (P @ q[t, 0]) + v[t, 0] * (kk @ q[t, 0]))
        np.testing.assert_allclose(o[t, 0], ref, rtol=1e-9, atol=1e-11)
    Href = math.exp(gam[-1]) * P @ H0[0, 0] + np.outer(kk, v[-1, 0])
    np.testing.assert_allclose(hT[0, 0], Href, rtol=1e-9, atol=1e-11)


def test_large_negative_gate_resets_state():
    q, k, v, g, beta, cu, H0 = _core_case(12, [1], hk=1, hv=1, dk=16, dv=8)
    g[:] = -1e30
    _, hT = O.gdr_stepwise(q, k, v, g, beta, cu, H0)
    kn = k[0, 0] / math.sqrt(np.sum(k[0, 0] ** 2) + 1e-6)
    np.testing.assert_allclose(hT[0, 0], np.outer(kn, beta[0, 0] * v[0, 0]), rtol=1e-14, atol=0)


def test_single_token_from_zero_state_closed_form():
    q, k, v, g, beta, cu, _ = _core_case(13, [1], hk=1, hv=1, dk=16, dv=8, h0=False)
    o, _ = O.gdr_stepwise(q, k, v, g, beta, cu, None, scale=0.3)
    qn = q[0, 0] / math.sqrt(np.sum(q[0, 0] ** 2) + 1e-6)
    kn = k[0, 0] / math.sqrt(np.sum(k[0, 0] ** 2) + 1e-6)
    np.testing.assert_allclose(o[0, 0], 0.3 * beta[0, 0] * np.dot(kn, qn) * v[0, 0], rtol=1e-13)


@pytest.mark.parametrize("fn", ["stepwise", "chunked"])
def test_orthonormal_keys_reduce_to_decayed_linear_attention(fn):
    # Distinct basis vectors as keys make every delta correction vanish, which
    # leaves o_t = s sum_{i<=t} exp(gamma_t - gamma_i) beta_i (q_t.k_i) v_i.
    r = rng(14)
    dk, dv, T = 128, 16, 128
    perm = r.permutation(dk)
    k = np.eye(dk)[perm][:T][:, None, :]
    q = r.standard_normal((T, 1, dk))
    v = r.standard_normal((T, 1, dv))
    g = -r.uniform(0, 0.3, (T, 1))
    beta = r.uniform(0.1, 1, (T, 1))
    cu = np.array([0, T], np.int32)
    f = O.gdr_stepwise if fn == "stepwise" else O.gdr_chunked
    o, hT = f(q, k, v, g, beta, cu, scale=0.5, use_l2norm=False)
    gam = np.cumsum(g[:, 0])
    qk = q[:, 0] @ k[:, 0].T
    M = np.tril(np.exp(gam[:, None] - gam[None, :]))
    expect = 0.5 * (qk * M * beta[None, :, 0]) @ v[:, 0]
    np.testing.assert_allclose(o[:, 0], expect, rtol=1e-11, atol=1e-11)
    Hexp = (k[:, 0] * (np.exp(gam[-1] - gam) * beta[:, 0])[:, None]).T @ v[:, 0]
    np.testing.assert_allclose(hT[0, 0], Hexp, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("lengths", [[1], [63], [64], [65], [129], [1, 64, 65, 2, 130]])
def test_chunked_form_equals_stepwise(lengths):
    q, k, v, g, beta, cu, H0 = _core_case(15, lengths, g_scale=0.5)
    o1, h1 = O.gdr_stepwise(q, k, v, g, beta, cu, H0, scale=128 ** -0.5)
    o2, h2 = O.gdr_chunked(q, k, v, g, beta, cu, H0, scale=128 ** -0.5, chunk=64)
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(h2, h1, rtol=1e-10, atol=1e-12)


@settings(max_examples=12, deadline=None)
@given(lengths=st.lists(st.integers(0, 150), min_size=1, max_size=4), seed=st.integers(0, 1000),
       chunk=st.sampled_from([16, 64]))
def test_chunked_form_equals_stepwise_on_random_packings(lengths, seed, chunk):
    """Property form of the check above: random packings (empty sequences included), seeds and
    chunk sizes."""
    q, k, v, g, beta, cu, H0 = _core_case(seed, lengths, g_scale=0.5)
    o1, h1 = O.gdr_stepwise(q, k, v, g, beta, cu, H0)
    o2, h2 = O.gdr_chunked(q, k, v, g, beta, cu, H0, chunk=chunk)
    np.testing.assert_allclose(o2, o1, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(h2, h1, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("split", [1, 37, 64, 128, 129])
def test_split_and_resume_equals_whole(split):
    q, k, v, g, beta, cu, H0 = _core_case(16, [200])
    o, hT = O.gdr_stepwise(q, k, v, g, beta, cu, H0)
    a = slice(0, split); b = slice(split, 200)
    oa, ha = O.gdr_stepwise(q[a], k[a], v[a], g[a], beta[a], np.array([0, split], np.int32), H0)
    ob, hb = O.gdr_chunked(q[b], k[b], v[b], g[b], beta[b], np.array([0, 200 - split], np.int32), ha)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(hb, hT, rtol=1e-11, atol=1e-12)


def test_packed_sequences_match_separate_runs_and_heads_group_contiguously():
    lengths = [3, 70, 1, 64]
    q, k, v, g, beta, cu, H0 = _core_case(17, lengths)
    o, hT = O.gdr_stepwise(q, k, v, g, beta, cu, H0)
    for n, L in enumerate(lengths):
        s = slice(int(cu[n]), int(cu[n + 1]))
        on, hn = O.gdr_stepwise(q[s], k[s], v[s], g[s], beta[s], np.array([0, L], np.int32),
                                H0[n:n + 1])
        np.testing.assert_array_equal(on, o[s])
        np.testing.assert_array_equal(hn[0], hT[n])
    # perturbing key head 1 must move value heads 3..5 only (contiguous groups of 3)
    k2 = k.copy(); k2[:, 1] += 0.5
    o2, _ = O.gdr_stepwise(q, k2, v, g, beta, cu, H0)
    moved = [h for h in range(6) if not np.array_equal(o2[:, h], o[:, h])]
    assert moved == [3, 4, 5]


def test_state_norm_contraction_bound():
    # (I - beta k k^T) has eigenvalues 1 and 1 - beta, and exp(g) <= 1, so the
    # state norm grows at most by beta |v| per token.
    q, k, v, g, beta, cu, H0 = _core_case(18, [300], hk=1, hv=1, dk=32, dv=32)
    _, hT = O.gdr_stepwise(q, k, v, g * 0.01, beta, cu, H0)
    bound = np.linalg.norm(H0[0, 0]) + np.sum(beta[:, 0] * np.linalg.norm(v[:, 0], axis=1))
    assert np.linalg.norm(hT[0, 0]) <= bound * (1 + 1e-12)


def test_core_path_on_workload_inputs_runs_both_forms():
    inp = GI.make_core_inputs(5, [70, 3], hk=2, hv=6, prenorm_qk=True, h0_std=0.02)
    ob, o1, h1 = O.core_path(inp)
    _, o2, h2 = O.core_path(inp, chunked=True)
    np.testing.assert_allclose(o2, o1, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(h2, h1, rtol=1e-9, atol=1e-12)
    assert ob.dtype == np.uint16 and ob.shape == (73, 6, 128)


# ---------------------------------------------------------------------------
# causal conv
# ---------------------------------------------------------------------------

def test_conv_matches_numpy_convolve():
    r = rng(20)
    T, C = 37, 5
    x = r.standard_normal((T, C)); w = r.standard_normal((C, 4))
    y, _ = O.causal_conv(x, w, np.array([0, T], np.int32), None, round_y=False)
    for c in range(C):
        pre = np.convolve(x[:, c], w[c, ::-1])[:T]
        np.testing.assert_allclose(y[:, c], torch.nn.functional.silu(torch.from_numpy(pre)).numpy(),
                                   rtol=1e-13, atol=1e-15)


def test_conv_identity_tap_is_silu():
    r = rng(21)
    x = r.standard_normal((10, 3)); w = np.tile([0.0, 0.0, 0.0, 1.0], (3, 1))
    y, _ = O.causal_conv(x, w, np.array([0, 10], np.int32), r.standard_normal((1, 3, 3)),
                         round_y=False)
    np.testing.assert_allclose(y, x / (1 + np.exp(-x)), rtol=1e-14)


@pytest.mark.parametrize("L", [1, 2, 3, 9])
def test_conv_step_repeated_equals_sequence_conv(L):
    r = rng(22)
    C = 6
    x = r.standard_normal((L, C)); w = r.standard_normal((C, 4)); cs = r.standard_normal((1, 3, C))
    y, cso = O.causal_conv(x, w, np.array([0, L], np.int32), cs, round_y=False)
    st = cs.copy()
    for t in range(L):
        yt, st = O.conv_step(x[t:t + 1], w, st)
        np.testing.assert_allclose(yt[0], y[t], rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(st, cso)
    full = np.concatenate([cs[0], x])
    np.testing.assert_array_equal(cso[0], full[-3:])


def test_conv_does_not_leak_across_sequences():
    r = rng(23)
    lengths = [2, 5, 1]
    C = 4
    x = r.standard_normal((8, C)); w = r.standard_normal((C, 4)); cs = r.standard_normal((3, 3, C))
    cu = GI.cu_seqlens_from_lengths(lengths)
    y, cso = O.causal_conv(x, w, cu, cs, round_y=True)
    for n in range(3):
        s = slice(int(cu[n]), int(cu[n + 1]))
        yn, csn = O.causal_conv(x[s], w, np.array([0, lengths[n]], np.int32), cs[n:n + 1])
        np.testing.assert_array_equal(yn, y[s])
        np.testing.assert_array_equal(csn[0], cso[n])
    # rounded outputs are bf16 values
    np.testing.assert_array_equal(O.round_bf16_f64(y), y)


# ---------------------------------------------------------------------------
# gated RMSNorm
# ---------------------------------------------------------------------------

def test_gated_rmsnorm_matches_torch_rms_norm():
    r = rng(30)
    o = r.standard_normal((9, 128)) * 3; z = r.standard_normal((9, 128)); w = r.standard_normal(128)
    y = O.gated_rmsnorm(o, z, w, eps=1e-6)
    to = torch.from_numpy(o)
    ref = torch.nn.functional.rms_norm(to, (128,), torch.from_numpy(w), 1e-6) * \
        torch.nn.functional.silu(torch.from_numpy(z))
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_gated_rmsnorm_closed_forms():
    z = np.full((2, 128), 0.7)
    o = np.array([np.full(128, 2.5), np.full(128, -0.1)])
    y = O.gated_rmsnorm(o, z, None, eps=1e-6)
    s = 0.7 / (1 + math.exp(-0.7))
    np.testing.assert_allclose(y[0], 2.5 / math.sqrt(6.25 + 1e-6) * s, rtol=1e-14)
    np.testing.assert_allclose(y[1], -0.1 / math.sqrt(0.01 + 1e-6) * s, rtol=1e-14)
    # scale invariance (eps aside) and a zero gate
    r = rng(31)
    o = r.standard_normal((4, 128)); z = r.standard_normal((4, 128))
    np.testing.assert_allclose(O.gated_rmsnorm(1000 * o, z, eps=0.0), O.gated_rmsnorm(o, z, eps=0.0),
                               rtol=1e-12)
    assert np.all(O.gated_rmsnorm(o, np.zeros_like(z)) == 0)


# ---------------------------------------------------------------------------
# chunk table
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("lengths", [[], [0], [1], [64], [65, 0, 128, 1, 63], [5000, 3]])
def test_prepare_chunks_brute_force(lengths):
    cu = GI.cu_seqlens_from_lengths(lengths) if lengths else np.array([0], np.int32)
    seq, st, ln = O.prepare_chunks(cu, 64)
    # brute force: walk tokens, cut at sequence starts and every 64 tokens
    exp = []
    for n, L in enumerate(lengths):
        for c0 in range(0, L, 64):
            exp.append((n, int(cu[n]) + c0, min(64, L - c0)))
    assert list(zip(seq.tolist(), st.tolist(), ln.tolist())) == exp
    covered = np.zeros(int(cu[-1]), int)
    for s0, l0 in zip(st, ln):
        covered[s0:s0 + l0] += 1
    assert np.all(covered == 1)


@settings(max_examples=40, deadline=None)
@given(lengths=st.lists(st.integers(0, 400), min_size=0, max_size=12), chunk=st.integers(1, 130))
def test_prepare_chunks_brute_force_on_random_offsets(lengths, chunk):
    cu = GI.cu_seqlens_from_lengths(lengths) if lengths else np.array([0], np.int32)
    seq, st_, ln = O.prepare_chunks(cu, chunk)
    exp = [(n, int(cu[n]) + c0, min(chunk, L - c0)) for n, L in enumerate(lengths) for c0 in range(0, L, chunk)]
    assert list(zip(seq.tolist(), st_.tolist(), ln.tolist())) == exp


def test_prepare_chunks_rejects_bad_offsets():
    with pytest.raises(ValueError):
        O.prepare_chunks(np.array([0, 5, 3], np.int32))
    with pytest.raises(ValueError):
        O.prepare_chunks(np.array([1, 5], np.int32))


# ---------------------------------------------------------------------------
# composed paths
# ---------------------------------------------------------------------------

def test_decode_steps_equal_prefill_of_the_same_tokens():
    # Decode (single-step conv + one recurrence step per token) over S steps
    # must equal the sequence conv + recurrence over the same S tokens with the
    # same initial conv and recurrent state.
    hk, hv, dk, dv, B, S = 2, 6, 128, 128, 3, 5
    dec = GI.make_decode_inputs(40, B, S, hk=hk, hv=hv, dk=dk, dv=dv)
    kept, H, cs = O.decode_steps(dec, keep_o=tuple(range(S)))
    C = dec.x.shape[2]
    x = np.transpose(dec.x, (1, 0, 2)).reshape(B * S, C)          # sequence-major packing
    cu = np.arange(0, B * S + 1, S, dtype=np.int32)
    y, cso = O.causal_conv(O.bf16_to_f64(x), O.bf16_to_f64(dec.conv_w), cu,
                           O.bf16_to_f64(dec.conv_state), round_y=True)
    q, k, v = O.split_qkv(y, hk, hv, dk, dv)
    a = np.transpose(dec.a, (1, 0, 2)).reshape(B * S, hv)
    b = np.transpose(dec.b, (1, 0, 2)).reshape(B * S, hv)
    g, beta = O.gates(O.bf16_to_f64(a), O.bf16_to_f64(b), dec.A_log, dec.dt_bias)
    o, hT = O.gdr_stepwise(q, k, v, g, beta, cu, h0=dec.state.astype(np.float64))
    np.testing.assert_allclose(hT, H, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cso, cs)
    ob = O.round_bf16(o).reshape(B, S, hv, dv)
    for s in range(S):
        np.testing.assert_array_equal(kept[s], ob[:, s])


def test_decode_slots_reduce_to_the_plain_step_on_gathered_rows():
    # The slot form is indexing around the decode step: on a pool laid out in any order,
    # each live row must give exactly what the plain step gives on that row's own state,
    # write it back to its own entry, leave every other entry bit for bit as it was and
    # give zeros on padding rows (slot -1 and slot past the pool).
    hk, hv = 2, 6
    dec = GI.make_decode_inputs(44, 4, 1, hk=hk, hv=hv)
    S = 6
    slot = np.array([4, -1, 1, S + 1], dtype=np.int32)
    live = [0, 2]
    r = rng(45)
    cpool = GI.f32_to_bf16_bits(r.standard_normal((S, 3, dec.x.shape[2])).astype(np.float32))
    spool = (r.standard_normal((S, hv, 128, 128)) * 0.02).astype(np.float32)
    for row in live:
        cpool[slot[row]] = dec.conv_state[row]
        spool[slot[row]] = dec.state[row]
    o, cp, sp = O.decode_step_slots(dec.x[0], dec.a[0], dec.b[0], dec.conv_w, dec.A_log, dec.dt_bias,
                                    O.bf16_to_f64(cpool), spool, slot, hk, hv)
    plain = GI.DecodeInputs(dec.x[:, live], dec.a[:, live], dec.b[:, live], dec.conv_w,
                            dec.conv_state[live], dec.state[live], dec.A_log, dec.dt_bias, hk, hv)
    kept, H, cs = O.decode_steps(plain, keep_o=(0,))
    np.testing.assert_array_equal(o[live], kept[0])
    assert not o[[1, 3]].any()
    np.testing.assert_array_equal(sp[slot[live]], H)
    np.testing.assert_array_equal(cp[slot[live]], cs)
    untouched = [e for e in range(S) if e not in slot[live]]
    np.testing.assert_array_equal(sp[untouched], spool[untouched].astype(np.float64))
    np.testing.assert_array_equal(cp[untouched], O.bf16_to_f64(cpool[untouched]))


def test_decode_slots_identity_is_the_plain_step_and_duplicates_are_rejected():
    hk, hv = 2, 6
    dec = GI.make_decode_inputs(46, 3, 1, hk=hk, hv=hv)
    o, cp, sp = O.decode_step_slots(dec.x[0], dec.a[0], dec.b[0], dec.conv_w, dec.A_log, dec.dt_bias,
                                    O.bf16_to_f64(dec.conv_state), dec.state, np.arange(3), hk, hv)
    kept, H, cs = O.decode_steps(dec, keep_o=(0,))
    np.testing.assert_array_equal(o, kept[0])
    np.testing.assert_array_equal(sp, H)
    np.testing.assert_array_equal(cp, cs)
    with pytest.raises(ValueError):
        O.decode_step_slots(dec.x[0], dec.a[0], dec.b[0], dec.conv_w, dec.A_log, dec.dt_bias,
                            O.bf16_to_f64(dec.conv_state), dec.state, np.array([1, 0, 1]), hk, hv)


def test_decode_on_sampled_heads_equals_the_full_layer_on_them():
    # The parity tests run the oracle on a few value heads of a large decode workload by
    # cutting out their channels; that cut must give exactly the full layer's results.
    from tests.helpers import restrict_decode_heads
    dec = GI.make_decode_inputs(47, 2, 4)
    heads = [0, 23, 25, 47]            # 23 and 25 share no key head, 0 and 47 are the ends
    kept, H, cs = O.decode_steps(dec, keep_o=(0, 3))
    sub = restrict_decode_heads(dec, heads)
    kept_s, H_s, _ = O.decode_steps(sub, keep_o=(0, 3))
    for s in (0, 3):
        np.testing.assert_array_equal(kept_s[s], kept[s][:, heads])
    np.testing.assert_array_equal(H_s, H[:, heads])
    # after three or more steps the conv state is the last three inputs, oldest first
    np.testing.assert_array_equal(O.round_bf16(cs), np.transpose(dec.x[1:], (1, 0, 2)))


@settings(max_examples=12, deadline=None)
@given(st.integers(1, 5), st.integers(0, 3), st.integers(0, 2**31 - 1))
def test_decode_slots_on_random_pools_match_the_plain_step(batch, extra_slots, seed):
    # Any slot table (distinct live entries, padding as -1 or past the pool) gives, row by
    # row, the plain step on that row's own state, and leaves every other entry as it was.
    hk, hv = 1, 2
    r = rng(seed)
    n_pad = int(r.integers(0, batch + 1))
    n_slots = batch - n_pad + extra_slots
    slot = GI.make_slot_table(seed, batch, max(n_slots, 1), n_pad) if n_slots > 0 else np.full(batch, -1, np.int32)
    if n_pad:
        slot[batch - n_pad:] = r.choice([-1, n_slots, n_slots + 7], n_pad)
    dec = GI.make_decode_inputs(seed % 1000, batch, 1, hk=hk, hv=hv)
    C = dec.x.shape[2]
    cpool = GI.f32_to_bf16_bits(r.standard_normal((n_slots, 3, C)).astype(np.float32))
    spool = (r.standard_normal((n_slots, hv, 128, 128)) * 0.02).astype(np.float32)
    live = [i for i in range(batch) if 0 <= slot[i] < n_slots]
    for i in live:
        cpool[slot[i]] = dec.conv_state[i]
        spool[slot[i]] = dec.state[i]
    o, cp, sp = O.decode_step_slots(dec.x[0], dec.a[0], dec.b[0], dec.conv_w, dec.A_log, dec.dt_bias,
                                    O.bf16_to_f64(cpool), spool, slot, hk, hv)
    pad = [i for i in range(batch) if i not in live]
    assert not o[pad].any()
    if live:
        plain = GI.DecodeInputs(dec.x[:, live], dec.a[:, live], dec.b[:, live], dec.conv_w,
                                dec.conv_state[live], dec.state[live], dec.A_log, dec.dt_bias, hk, hv)
        kept, H, cs = O.decode_steps(plain, keep_o=(0,))
        np.testing.assert_array_equal(o[live], kept[0])
        np.testing.assert_array_equal(sp[slot[live]], H)
        np.testing.assert_array_equal(cp[slot[live]], cs)
    others = [e for e in range(n_slots) if e not in set(slot[live].tolist())]
    np.testing.assert_array_equal(sp[others], spool[others].astype(np.float64))
    np.testing.assert_array_equal(cp[others], O.bf16_to_f64(cpool[others]))


def test_slot_table_generator():
    slot = GI.make_slot_table(3, 10, 16, n_padding=2)
    assert slot.dtype == np.int32 and slot.shape == (10,)
    assert (slot[-2:] == -1).all()
    live = slot[:-2]
    assert len(set(live.tolist())) == 8 and live.min() >= 0 and live.max() < 16
    np.testing.assert_array_equal(slot, GI.make_slot_table(3, 10, 16, n_padding=2))
    with pytest.raises(ValueError):
        GI.make_slot_table(3, 10, 4)


def test_full_path_shapes_and_rounding():
    inp = GI.make_full_inputs(41, [5, 66], hk=2, hv=6, h0_std=0.02, conv_state_std=1.0,
                              norm_w_std=0.1)
    out = O.full_path(inp)
    assert out["y"].shape == (71, 6, 128) and out["y"].dtype == np.uint16
    assert out["hT"].shape == (2, 6, 128, 128)
    assert out["conv_state_out"].shape == (2, 3, inp.channels)
    # the conv state out is made of the raw inputs: the last 3 tokens of each sequence
    np.testing.assert_array_equal(out["conv_state_out"][1], inp.x[71 - 3:71])
    np.testing.assert_array_equal(out["conv_state_out"][0], inp.x[2:5])


# ---------------------------------------------------------------------------
# composition of the full path: channel order of the conv output and the
# rounding points between the kernels
# ---------------------------------------------------------------------------

def _perturb_channels(inp, lo, hi, seed):
    x = inp.x.copy()
    x[:, lo:hi] = GI.f32_to_bf16_bits(rng(seed).standard_normal((x.shape[0], hi - lo)).astype(np.float32))
    return dataclasses.replace(inp, x=x)


def test_full_path_reads_q_k_v_from_their_channel_blocks():
    """The conv runs over the channels [q | k | v] (hk*128 q channels, hk*128 k channels, then
    hv*128 v channels, value head h in block h).  The conv is depthwise, so a channel of x
    reaches only the same channel of the conv output.  q enters only the output: new values
    in the q channels change o and leave the final state identical bit for bit.  New values
    in the k channels of key head 1 change the state of value heads 3..5 only (heads group
    contiguously, three per key head).  New values in the v channels of value head 4 change
    that head's state and output alone."""
    hk, hv, d = 2, 6, 128
    inp = GI.make_full_inputs(42, [40, 70], hk=hk, hv=hv, h0_std=0.02)
    base = O.full_path(inp)
    heads_changed = lambda out, key: [h for h in range(hv)
                                      if not np.array_equal(out[key][..., h, :] if key == "o" else out[key][:, h],
                                                            base[key][..., h, :] if key == "o" else base[key][:, h])]
    pq = O.full_path(_perturb_channels(inp, 0, hk * d, 1))
    assert np.array_equal(pq["hT"], base["hT"])
    assert heads_changed(pq, "o") == list(range(hv))
    pk = O.full_path(_perturb_channels(inp, hk * d + d, 2 * hk * d, 2))
    assert heads_changed(pk, "hT") == [3, 4, 5]
    pv = O.full_path(_perturb_channels(inp, 2 * hk * d + 4 * d, 2 * hk * d + 5 * d, 3))
    assert heads_changed(pv, "hT") == [4]
    assert heads_changed(pv, "o") == [4]


def test_full_path_is_the_recurrence_on_the_rounded_conv_output():
    """The recurrence of the full path runs on the conv output as the bf16 tensor the conv
    emits, split at the channel offsets of the [q | k | v] layout (written out here), with
    the gates of a and b: the full path's o and final state equal those of the pinned
    stepwise recurrence run on those slices."""
    hk, hv, d = 2, 6, 128
    inp = GI.make_full_inputs(45, [33, 66], hk=hk, hv=hv, h0_std=0.02, conv_state_std=1.0)
    out = O.full_path(inp)
    yc, _ = O.causal_conv(O.bf16_to_f64(inp.x), O.bf16_to_f64(inp.conv_w), inp.cu_seqlens,
                          O.bf16_to_f64(inp.conv_state), round_y=False)
    assert np.array_equal(out["conv_y"], O.round_bf16(yc))
    y = O.bf16_to_f64(out["conv_y"])
    T = y.shape[0]
    q = y[:, 0:256].reshape(T, hk, d)
    k = y[:, 256:512].reshape(T, hk, d)
    v = y[:, 512:1280].reshape(T, hv, d)
    g, beta = O.gates(O.bf16_to_f64(inp.a), O.bf16_to_f64(inp.b), inp.A_log, inp.dt_bias)
    o, hT = O.gdr_stepwise(q, k, v, g, beta, inp.cu_seqlens, h0=inp.h0)
    assert np.array_equal(out["o"], O.round_bf16(o))
    assert np.array_equal(out["hT"], hT)


def test_full_path_norm_reads_the_bf16_output():
    """The gated norm of the full path reads o as the bf16 tensor the recurrence emits: y is
    the pinned gated norm of the returned o bits, rounded to bf16, exactly.  (On this input
    the unrounded o gives a different y in many places, so the rounding point is seen.)"""
    inp = GI.make_full_inputs(44, [50, 30], hk=2, hv=6, h0_std=0.02, norm_w_std=0.1)
    out = O.full_path(inp)
    y = O.round_bf16(O.gated_rmsnorm(O.bf16_to_f64(out["o"]), O.bf16_to_f64(inp.z), inp.norm_w, inp.eps))
    assert np.array_equal(out["y"], y)


def test_linear_is_the_product_written_out():
    """The projection oracle against explicit sums on a tiny case, including a column where the
    bf16 rounding of the sum is decided by the last term (so a dropped term or a transposed
    operand changes bits)."""
    r = np.random.default_rng(3)
    x = GI.f32_to_bf16_bits(r.standard_normal((3, 5)).astype(np.float32))
    w = GI.f32_to_bf16_bits(r.standard_normal((4, 5)).astype(np.float32))
    xf, wf = O.bf16_to_f64(x), O.bf16_to_f64(w)
    want = np.zeros((3, 4))
    for m in range(3):
        for n in range(4):
            acc = 0.0
            for k in range(5):
                acc += xf[m, k] * wf[n, k]
            want[m, n] = acc
    assert np.array_equal(O.linear(x, w), O.round_bf16(want))
    # x = e_0, W = rows of distinct values: y picks column 0 of W, exactly
    e = GI.f32_to_bf16_bits(np.eye(2, 5, dtype=np.float32))
    assert np.array_equal(O.linear(e, w), w[:, :2].T)
