"""Planted mistakes in the oracle: each must fail at least one of its pins.

Every mutant below is one plausible slip in oracle/gdr_oracle.c (a dropped term, a wrong
sign, a swapped index or operand, a misplaced factor).  The test builds that copy of the
source with gcc into a temporary library, points the oracle module at it, runs the pins of
tests/test_oracle.py and requires that at least one of them fails.  The real oracle is
restored afterwards.  Mutants apply to every occurrence of the pattern, so the stepwise and
chunked forms carry the same slip where both have the line.
"""
import inspect
import os
import subprocess

import pytest

from oracle import oracle as O
from tests import test_oracle as P

SRC = O._SRC

# (name, pattern in gdr_oracle.c, replacement)
MUTANTS = [
    ("delta term added instead of subtracted", "u[j] = bt * (vt[j] - acc[j]);", "u[j] = bt * (vt[j] + acc[j]);"),
    ("decay of the state dropped", "for (int e = 0; e < dk * dv; ++e) H[e] *= decay;", ""),
    ("write strength dropped", "u[j] = bt * (vt[j] - acc[j]);", "u[j] = (vt[j] - acc[j]);"),
    ("output reads H q instead of H^T q", "acc[j] += H[i * dv + j] * qn[i];", "acc[j] += H[j * dv + i] * qn[i];"),
    ("state update uses q for k", "H[i * dv + j] += kn[i] * u[j];", "H[i * dv + j] += qn[i] * u[j];"),
    ("output scale dropped", "ot[j] = c->scale * acc[j];", "ot[j] = acc[j];"),
    ("exp of A_log dropped", "g[i] = -exp((double)A_log[h]) *", "g[i] = -((double)A_log[h]) *"),
    ("dt_bias dropped", "oracle_softplus(a[i] + (double)dt_bias[h])", "oracle_softplus(a[i])"),
    ("sigmoid sign", "return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    ("softplus threshold reversed", "if (x > 20.0) return x;", "if (x < 20.0) return x;"),
    ("L2 norm skipped", "double r = use ? 1.0 / sqrt(s + eps) : 1.0;", "double r = 1.0;"),
    ("key heads interleaved", "const int kh = h / (hv / hk);", "const int kh = h % hk;"),
    ("chunked: decay direction in A", "a = bt[i] * exp(gam[i] - gam[j]) * d;", "a = bt[i] * exp(gam[j] - gam[i]) * d;"),
    ("chunked: beta missing in W", "sacc += Tm[i * C + j] * bt[j] * exp(gam[j]) * Kn[j * dk + x];",
     "sacc += Tm[i * C + j] * exp(gam[j]) * Kn[j * dk + x];"),
    ("conv taps reversed", "acc += w[(size_t)c * 4 + j] * xv;", "acc += w[(size_t)c * 4 + (3 - j)] * xv;"),
    ("conv state read newest first", "conv_state[((size_t)n * 3 + (3 - back)) * C + c]",
     "conv_state[((size_t)n * 3 + (back - 1)) * C + c]"),
    ("conv step: state rolled the wrong way", "s[c] = s1; s[C + c] = s2; s[2 * C + c] = xv;",
     "s[c] = xv; s[C + c] = s1; s[2 * C + c] = s2;"),
    ("conv step: current token on the oldest tap", "wc[0] * s0 + wc[1] * s1 + wc[2] * s2 + wc[3] * xv",
     "wc[3] * s0 + wc[1] * s1 + wc[2] * s2 + wc[0] * xv"),
    ("norm mean over d dropped", "double inv = 1.0 / sqrt(ss / d + eps);", "double inv = 1.0 / sqrt(ss + eps);"),
    ("norm gate not SiLU", "* (w ? w[j] : 1.0) * silu(zrow[j]);", "* (w ? w[j] : 1.0) * zrow[j];"),
    ("delta read from the undecayed state", "u[j] = bt * (vt[j] - acc[j]);", "u[j] = bt * (vt[j] - acc[j] / decay);"),
    ("write strength of the key head", "const double bt = c->beta[(size_t)t * hv + h];",
     "const double bt = c->beta[(size_t)t * hv + kh];"),
    ("chunked: diagonal dropped from the output mask", "for (int j = 0; j <= i; ++j) {", "for (int j = 0; j < i; ++j) {"),
    ("chunked: forward substitution sign", "x -= A[i * C + j] * Tm[j * C + col];", "x += A[i * C + j] * Tm[j * C + col];"),
    ("chunked: W H0 added to U", "sacc -= W[i * dk + x] * H[x * dv + y];", "sacc += W[i * dk + x] * H[x * dv + y];"),
    ("chunked: carried state not decayed", "double sacc = eL * H[x * dv + y];", "double sacc = H[x * dv + y];"),
    ("chunked: state update without in-chunk decay", "exp(gam[L - 1] - gam[j]) * U[j * dv + y]", "U[j * dv + y]"),
    ("chunked: output from the carried state undecayed", "double ei = exp(gam[i]);", "double ei = 1.0;"),
    ("chunked: beta missing in Ut", "sacc += Tm[i * C + j] * bt[j] * V[j * dv + y];",
     "sacc += Tm[i * C + j] * V[j * dv + y];"),
    ("chunked: intra-chunk output decay reversed", "intra += qk * exp(gam[i] - gam[j]) * U[j * dv + y];",
     "intra += qk * exp(gam[j] - gam[i]) * U[j * dv + y];"),
]

# the pins, as (name, call)
PINS = [
    ("gate closed forms", P.test_gate_closed_forms),
    ("gates vs torch", P.test_gates_match_torch_library),
    ("hand-worked example", P.test_hand_worked_example),
    ("beta 0, g 0", P.test_beta0_g0_leaves_state_unchanged),
    ("beta 1 overwrite", P.test_beta1_unit_key_overwrites),
    ("reset", P.test_large_negative_gate_resets_state),
    ("one token closed form", P.test_single_token_from_zero_state_closed_form),
    ("orthonormal keys, stepwise", lambda: P.test_orthonormal_keys_reduce_to_decayed_linear_attention("stepwise")),
    ("orthonormal keys, chunked", lambda: P.test_orthonormal_keys_reduce_to_decayed_linear_attention("chunked")),
    ("chunked = stepwise", lambda: P.test_chunked_form_equals_stepwise([1, 64, 65, 2, 130])),
    ("split and resume", lambda: P.test_split_and_resume_equals_whole(37)),
    ("packed and grouped", P.test_packed_sequences_match_separate_runs_and_heads_group_contiguously),
    ("conv vs numpy", P.test_conv_matches_numpy_convolve),
    ("conv identity tap", P.test_conv_identity_tap_is_silu),
    ("conv step x T", lambda: P.test_conv_step_repeated_equals_sequence_conv(3)),
    ("conv no leak", P.test_conv_does_not_leak_across_sequences),
    ("norm vs torch", P.test_gated_rmsnorm_matches_torch_rms_norm),
    ("decode steps = prefill", P.test_decode_steps_equal_prefill_of_the_same_tokens),
    ("norm closed forms", P.test_gated_rmsnorm_closed_forms),
    ("repeated unit key, stepwise", lambda: P.test_repeated_unit_key_with_full_write_closed_form("stepwise")),
    ("repeated unit key, chunked", lambda: P.test_repeated_unit_key_with_full_write_closed_form("chunked")),
]


def _use_library(src, lib):
    O._SRC, O._LIB, O._lib = src, lib, None


@pytest.fixture
def restore_oracle():
    saved = (O._SRC, O._LIB)
    yield
    O._SRC, O._LIB = saved
    O._lib = None


@pytest.mark.parametrize("name,pattern,replacement", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(name, pattern, replacement, tmp_path, restore_oracle):
    text = open(SRC).read()
    assert pattern in text, f"pattern of mutant '{name}' not found"
    src = tmp_path / "gdr_oracle_mutant.c"
    src.write_text(text.replace(pattern, replacement))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-o", str(lib),
                           str(src), "-lm", "-lpthread"])
    _use_library(str(src), str(lib))
    failed = []
    for pin_name, pin in PINS:
        try:
            pin()
        except Exception:   # an assertion, or the oracle rejecting what it computed
            failed.append(pin_name)
    assert failed, f"no pin catches the planted mistake '{name}'"


def test_pins_pass_on_the_real_oracle(restore_oracle):
    """The same pin list passes on the unmodified oracle (so the failures above are the mutants')."""
    assert os.path.exists(O.build())
    O._lib = None
    for _, pin in PINS:
        pin()


# Slips in the Python composition of the oracle (oracle/oracle.py): (name, function, pattern,
# replacement).  The mutated function replaces the real one in the module for the test.
COMPOSITION_MUTANTS = [
    ("q and k channel blocks swapped", "split_qkv",
     "q = y[:, : hk * dk].reshape(T, hk, dk)\n    k = y[:, hk * dk: 2 * hk * dk].reshape(T, hk, dk)",
     "k = y[:, : hk * dk].reshape(T, hk, dk)\n    q = y[:, hk * dk: 2 * hk * dk].reshape(T, hk, dk)"),
    ("v read from the k channels on", "split_qkv", "v = y[:, 2 * hk * dk:].reshape(T, hv, dv)",
     "v = y[:, hk * dk: hk * dk + hv * dv].reshape(T, hv, dv)"),
    ("o not rounded before the gated norm", "full_path", "y = gated_rmsnorm(bf16_to_f64(o_bits),",
     "y = gated_rmsnorm(o,"),
    ("conv output not rounded", "full_path", "causal_conv(x, w, inp.cu_seqlens, cs, round_y=True)",
     "causal_conv(x, w, inp.cu_seqlens, cs, round_y=False)"),
]

COMPOSITION_PINS = PINS + [
    ("channel blocks", P.test_full_path_reads_q_k_v_from_their_channel_blocks),
    ("recurrence on the rounded conv output", P.test_full_path_is_the_recurrence_on_the_rounded_conv_output),
    ("norm reads the bf16 o", P.test_full_path_norm_reads_the_bf16_output),
]


@pytest.mark.parametrize("name,func,pattern,replacement", COMPOSITION_MUTANTS,
                         ids=[m[0] for m in COMPOSITION_MUTANTS])
def test_planted_composition_mistake_fails_a_pin(name, func, pattern, replacement, monkeypatch):
    src = inspect.getsource(getattr(O, func))
    assert pattern in src, f"pattern of mutant '{name}' not found"
    ns = dict(vars(O))
    exec(compile(src.replace(pattern, replacement), O.__file__, "exec"), ns)
    monkeypatch.setattr(O, func, ns[func])
    failed = []
    for pin_name, pin in COMPOSITION_PINS:
        try:
            pin()
        except Exception:
            failed.append(pin_name)
    assert failed, f"no pin catches the planted mistake '{name}'"


def test_composition_pins_pass_on_the_real_oracle():
    for _, pin in COMPOSITION_PINS[len(PINS):]:
        pin()
