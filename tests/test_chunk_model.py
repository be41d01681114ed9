"""The chunkwise algebra (tests/chunk_model.py) equals the token recurrence.

"Every valid C provides exact results" ("Linear Attention, Visualized",
"Chunkwise algorithm" / "Cost"): the chunk model must match the oracle for any
chunk size, including C = 1 (recurrent form), C = T (fully parallel form) and
T not divisible by C (identity-token padding).
"""
import numpy as np
import pytest

import oracle
from chunk_model import chunk_forward_heads
from test_oracle_pins import rand_inputs, rel_err

CASES = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
         ("delta", "none"), ("delta", "scalar"), ("delta", "channel")]


@pytest.mark.parametrize("update,gate", CASES)
@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunk_model_matches_oracle(oracle_mod, update, gate, C):
    T = 150  # not a multiple of 4, 16 or 64
    q, k, v, g, beta, S0 = rand_inputs(31, BH=2, T=T, dk=16, dv=12, gate=gate,
                                       delta=(update == "delta"), s0=True, gmin=-0.5)
    o, ST = oracle.gdn_forward(update, gate, q, k, v, g=g, beta=beta, S0=S0)
    oc, Sc = chunk_forward_heads(update, gate, q, k, v, g=g, beta=beta, S0=S0, C=C)
    assert rel_err(oc, o) < 1e-10
    assert rel_err(Sc, ST) < 1e-10


def test_chunk_equals_full_parallel_form(oracle_mod):
    q, k, v, g, beta, S0 = rand_inputs(32, BH=1, T=40, dk=8, dv=8, gate="channel", delta=True, s0=True)
    o, ST = oracle.gdn_forward("delta", "channel", q, k, v, g=g, beta=beta, S0=S0)
    oc, Sc = chunk_forward_heads("delta", "channel", q, k, v, g=g, beta=beta, S0=S0, C=40)
    assert rel_err(oc, o) < 1e-10 and rel_err(Sc, ST) < 1e-10


def _workload_head(update, gate, T=1024):
    from synth import WORKLOADS, make_prefill_inputs
    name = {"scalar": "gdn_prefill_bf16", "channel": "kda_prefill_bf16", "none": "linear_attn_bf16"}[gate]
    w = WORKLOADS[name].with_(T=T)
    x = make_prefill_inputs(w, heads=[(0, 1)])
    o, ST = oracle.gdn_forward(update, gate, x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    return x, o, ST


@pytest.mark.parametrize("update,gate", [("delta", "scalar"), ("delta", "channel"), ("additive", "none")])
def test_fp16_operands_stay_within_tolerance(oracle_mod, update, gate):
    """fp16 tensor-core operands (11-bit significand) keep a workload-like head
    well inside the 2e-2 bf16-input bound (fp32 output)."""
    x, o, ST = _workload_head(update, gate)
    oc, Sc = chunk_forward_heads(update, gate, x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"],
                                 S0=x["S0"], C=64, emulate_bf16="fp16")
    eo, es = rel_err(oc, o), rel_err(Sc, ST)
    assert eo < 8e-3 and es < 8e-3, (eo, es)


def test_bf16_operands_would_exceed_tolerance(oracle_mod):
    """Why the tensor-core kernel does not feed bf16 intermediates: with every
    operand rounded to bf16 (8-bit significand) the GDN head already exceeds
    2e-2, because max|o| is ~7x rms(o) and each rounding point adds ~1e-2."""
    x, o, ST = _workload_head("delta", "scalar")
    oc, _ = chunk_forward_heads("delta", "scalar", x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"],
                                S0=x["S0"], C=64, emulate_bf16="bf16")
    assert rel_err(oc, o) > 2e-2


# ----------------------------------------------------------------------------
# The chunkwise backward (the passes of the tensor-core backward) equals the
# oracle's reverse mode through the token loop, for every chunk size.
BWD_CASES = [("additive", "none"), ("decay", "scalar"), ("delta", "none"), ("delta", "scalar")]


@pytest.mark.parametrize("update,gate", BWD_CASES)
@pytest.mark.parametrize("C,T", [(64, 150), (16, 40), (64, 1), (4, 64)])
@pytest.mark.parametrize("s0,grads", [(True, (True, True)), (False, (True, False)), (True, (False, True))])
def test_chunk_backward_model_matches_oracle(update, gate, C, T, s0, grads):
    from chunk_model import chunk_backward

    q, k, v, g, beta, S0 = rand_inputs(43, BH=2, T=T, dk=16, dv=12, gate=gate,
                                       delta=(update == "delta"), s0=s0, gmin=-0.5)
    r = np.random.default_rng(44)
    dO = r.standard_normal((2, T, 12)) if grads[0] else None
    dST = r.standard_normal((2, 12, 16)) if grads[1] else None
    ref = oracle.gdn_backward_np(update, gate, q, k, v, g, beta, S0, dO, dST)
    for h in range(2):
        one = lambda a: None if a is None else a[h]
        got = chunk_backward(update, gate, one(q), one(k), one(v), one(g), one(beta), one(S0), one(dO), one(dST),
                             C=C)
        for name, a, b in zip(["dq", "dk", "dv", "dg", "dbeta", "dS0"], got, ref):
            if b is None:
                assert a is None, name
                continue
            assert rel_err(a, b[h]) < 1e-10, (name, rel_err(a, b[h]))


@pytest.mark.parametrize("update", ["decay", "delta"])
@pytest.mark.parametrize("C,T", [(64, 150), (16, 40), (64, 1)])
def test_chunk_backward_channel_gate_model_matches_oracle(update, C, T):
    """The per-channel gate (KDA / GLA) form of the chunkwise backward: every
    decay factor inside the q / k products, the gate gradient per channel."""
    from chunk_model import chunk_backward_channel

    q, k, v, g, beta, S0 = rand_inputs(45, BH=2, T=T, dk=16, dv=12, gate="channel",
                                       delta=(update == "delta"), s0=True, gmin=-0.5)
    r = np.random.default_rng(46)
    dO, dST = r.standard_normal((2, T, 12)), r.standard_normal((2, 12, 16))
    ref = oracle.gdn_backward_np(update, "channel", q, k, v, g, beta, S0, dO, dST)
    for h in range(2):
        one = lambda a: None if a is None else a[h]
        got = chunk_backward_channel(update, one(q), one(k), one(v), one(g), one(beta), one(S0), one(dO),
                                     one(dST), C=C)
        for name, a, b in zip(["dq", "dk", "dv", "dg", "dbeta", "dS0"], got, ref):
            if b is None:
                assert a is None, name
                continue
            assert rel_err(a, b[h]) < 1e-10, (name, rel_err(a, b[h]))
