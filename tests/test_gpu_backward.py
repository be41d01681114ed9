"""GPU parity of the backward pass (gdn_chunk_bwd) against the float64 oracle
``oracle.gdn_backward_np`` (itself pinned to finite differences of the forward
definition): every mode, dk and dv in {64, 128}, fp32 and bf16 inputs, ragged
lengths, with and without S0 and the two upstream gradients."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import dev, np64, rel_err
from synth import round_to_bf16

pytestmark = pytest.mark.gpu

MODES = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
         ("delta", "none"), ("delta", "scalar"), ("delta", "channel")]
# fp32 arithmetic against float64 on the same (rounded) inputs
TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    gdn.device_status(clear=True)


def inputs(seed, update, gate, B=1, H=2, T=130, dk=128, dv=128, bf16=False, s0=True, grads=(True, True)):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, H, T, dk))
    k = r.standard_normal((B, H, T, dk))
    if update == "additive":
        q, k = np.where(q > 0, q + 1, np.exp(q)) / np.sqrt(dk), np.where(k > 0, k + 1, np.exp(k)) / np.sqrt(dk)
    else:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, H, T, dv))
    if bf16:
        q, k, v = (round_to_bf16(np.asarray(x, np.float32)).astype(np.float64) for x in (q, k, v))
    else:
        q, k, v = (np.asarray(x, np.float32).astype(np.float64) for x in (q, k, v))
    g = None
    if gate == "scalar":
        g = -np.log1p(np.exp(r.standard_normal((B, H, T)) - 3.0))
    elif gate == "channel":
        g = -np.log1p(np.exp(r.standard_normal((B, H, T, dk)) - 4.0))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((B, H, T)))) if update == "delta" else None
    S0 = 0.05 * r.standard_normal((B, H, dv, dk)) if s0 else None
    dO = r.standard_normal((B, H, T, dv)) if grads[0] else None
    dST = r.standard_normal((B, H, dv, dk)) if grads[1] else None
    f32 = lambda x: None if x is None else np.asarray(x, np.float32).astype(np.float64)
    return q, k, v, f32(g), f32(beta), f32(S0), f32(dO), f32(dST)


def run(update, gate, x, bf16):
    q, k, v, g, beta, S0, dO, dST = x
    dt = torch.bfloat16 if bf16 else torch.float32
    gdn.device_status(clear=True)
    got = gdn.chunk_bwd(dev(q, dt), dev(k, dt), dev(v, dt), dev(g), dev(beta), dev(S0), dev(dO), dev(dST),
                        update=update, gate=gate)
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    ref = oracle.gdn_backward_np(update, gate, q, k, v, g, beta, S0, dO, dST)
    names = ["dq", "dk", "dv", "dg", "dbeta", "dS0"]
    for name, a, b in zip(names, got, ref):
        if b is None:
            assert a is None, name
            continue
        err = rel_err(np64(a), b)
        assert err <= TOL, (name, err)


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64)])
def test_backward_modes(update, gate, dk, dv):
    run(update, gate, inputs(3, update, gate, T=130, dk=dk, dv=dv), bf16=False)


@pytest.mark.parametrize("update,gate", MODES)
def test_backward_bf16_inputs(update, gate):
    run(update, gate, inputs(4, update, gate, T=100, bf16=True), bf16=True)


@pytest.mark.parametrize("T", [1, 7, 8, 63, 64, 65, 200])
def test_backward_ragged_lengths(T):
    run("delta", "scalar", inputs(5, "delta", "scalar", T=T), bf16=False)


@pytest.mark.parametrize("s0,grads", [(False, (True, False)), (True, (False, True)), (False, (False, False))])
def test_backward_optional_inputs(s0, grads):
    run("delta", "channel", inputs(6, "delta", "channel", T=90, s0=s0, grads=grads), bf16=False)


def test_backward_many_heads_and_value_slices():
    run("delta", "scalar", inputs(7, "delta", "scalar", B=3, H=5, T=70, dv=128, bf16=True), bf16=True)


def test_backward_empty_sequence_copies_state_gradient():
    q = torch.zeros((1, 2, 0, 128), device="cuda")
    dST = torch.randn((1, 2, 128, 128), device="cuda")
    out = gdn.chunk_bwd(q, q, q, None, torch.zeros((1, 2, 0), device="cuda"), None, None, dST,
                        update="delta", gate="none")
    torch.cuda.synchronize()
    assert torch.equal(out[5], dST) and out[0].numel() == 0


# ----------------------------------------------------------------------------
# Saved chunk states: gdn_chunk_fwd_states writes the state entering every chunk
# of 64 tokens (the tensor-core forward, fp16 operands), gdn_chunk_bwd_states
# starts from them.  Their rounding bounds these cases, so the bound is the
# bf16 one of the forward parity tests.
TOL_STATES = 2e-2


def _dev_inputs(x):
    q, k, v, g, beta, S0, dO, dST = x
    dt = torch.bfloat16
    return dev(q, dt), dev(k, dt), dev(v, dt), dev(g), dev(beta), dev(S0), dev(dO), dev(dST)


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dv,T", [(128, 150), (64, 64), (128, 1)])
def test_forward_states_are_the_chunk_boundary_states(update, gate, dv, T):
    x = inputs(17, update, gate, T=T, dv=dv, bf16=True)
    q, k, v, g, beta, S0 = _dev_inputs(x)[:6]
    nch = (T + 63) // 64
    states = torch.empty((1, 2, nch, dv, 128), dtype=torch.float32, device="cuda")
    gdn.device_status(clear=True)
    o1, S1 = gdn.chunk_fwd(q, k, v, g, beta, S0, update=update, gate=gate, states=states)
    o2, S2 = gdn.chunk_fwd(q, k, v, g, beta, S0, update=update, gate=gate, algo="tc")
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    # the same forward as the plain tensor-core call
    assert rel_err(np64(o1), np64(o2)) <= 1e-6 and rel_err(np64(S1), np64(S2)) <= 1e-6
    qn, kn, vn, gn, bn, S0n = x[:6]
    for c in range(nch):
        if c == 0:
            ref = S0n
        else:
            t = 64 * c
            sl = lambda a: None if a is None else np.ascontiguousarray(a[:, :, :t])
            _, ref = oracle.gdn_forward(update, gate, sl(qn), sl(kn), sl(vn), g=sl(gn), beta=sl(bn), S0=S0n)
        assert rel_err(np64(states[:, :, c]), ref) <= TOL_STATES, c


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dv,T", [(128, 150), (64, 200)])
def test_backward_from_saved_states(update, gate, dv, T):
    x = inputs(23, update, gate, T=T, dv=dv, bf16=True)
    q, k, v, g, beta, S0, dO, dST = _dev_inputs(x)
    states = torch.empty((1, 2, (T + 63) // 64, dv, 128), dtype=torch.float32, device="cuda")
    gdn.device_status(clear=True)
    gdn.chunk_fwd(q, k, v, g, beta, S0, update=update, gate=gate, states=states)
    got = gdn.chunk_bwd(q, k, v, g, beta, None, dO, dST, update=update, gate=gate, states=states)
    plain = gdn.chunk_bwd(q, k, v, g, beta, S0, dO, dST, update=update, gate=gate)
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    ref = oracle.gdn_backward_np(update, gate, *x)
    for name, a, b, c in zip(["dq", "dk", "dv", "dg", "dbeta", "dS0"], got, ref, plain):
        if b is None:
            assert a is None, name
            continue
        assert rel_err(np64(a), b) <= TOL_STATES, (name, rel_err(np64(a), b))
        assert rel_err(np64(a), np64(c)) <= TOL_STATES, name


def test_saved_states_reject_requests_the_tensor_core_forward_cannot_serve():
    x = inputs(29, "delta", "scalar", T=70, dv=128)
    q, k, v, g, beta, S0 = (dev(a) for a in x[:6])  # fp32 inputs
    states = torch.empty((1, 2, 2, 128, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(gdn.GDNError):
        gdn.chunk_fwd(q, k, v, g, beta, S0, update="delta", gate="scalar", states=states)


# ----------------------------------------------------------------------------
# Input prologue: the gradients with respect to the raw q, k, beta, g that the
# forward's maps took (oracle.gdn_backward_prologue_np, pinned by central
# differences through maps and recurrence).
PRO_CASES = [("delta", "scalar", oracle.PRO_QK_L2 | oracle.PRO_BETA_SIGMOID | oracle.PRO_G_NEG_SOFTPLUS),
             ("delta", "channel", oracle.PRO_QK_ELU1 | oracle.PRO_QK_L2 | oracle.PRO_G_NEG_SOFTPLUS),
             ("delta", "none", oracle.PRO_QK_ELU1 | oracle.PRO_QK_L2 | oracle.PRO_BETA_SIGMOID),
             ("additive", "none", oracle.PRO_QK_ELU1),
             ("decay", "scalar", oracle.PRO_QK_L2 | oracle.PRO_G_NEG_SOFTPLUS)]


def raw_inputs(seed, update, gate, T=130, dk=128, dv=128, bf16=False):
    r = np.random.default_rng(seed)
    q = r.standard_normal((1, 2, T, dk)) / (np.sqrt(dk) if update == "additive" else 1.0)
    k = r.standard_normal((1, 2, T, dk)) / (np.sqrt(dk) if update == "additive" else 1.0)
    v = r.standard_normal((1, 2, T, dv))
    rnd = (lambda x: round_to_bf16(np.asarray(x, np.float32)).astype(np.float64)) if bf16 else \
        (lambda x: np.asarray(x, np.float32).astype(np.float64))
    q, k, v = rnd(q), rnd(k), rnd(v)
    f32 = lambda x: None if x is None else np.asarray(x, np.float32).astype(np.float64)
    g = None
    if gate == "scalar":
        g = f32(r.standard_normal((1, 2, T)) - 3.0)
    elif gate == "channel":
        g = f32(r.standard_normal((1, 2, T, dk)) - 4.0)
    beta = f32(r.standard_normal((1, 2, T))) if update == "delta" else None
    S0 = f32(0.05 * r.standard_normal((1, 2, dv, dk)))
    dO = f32(r.standard_normal((1, 2, T, dv)))
    dST = f32(r.standard_normal((1, 2, dv, dk)))
    return q, k, v, g, beta, S0, dO, dST


@pytest.mark.parametrize("update,gate,flags", PRO_CASES)
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64)])
@pytest.mark.parametrize("bf16", [False, True])
def test_backward_with_input_prologue(update, gate, flags, dk, dv, bf16):
    x = raw_inputs(41, update, gate, dk=dk, dv=dv, bf16=bf16)
    q, k, v, g, beta, S0, dO, dST = x
    dt = torch.bfloat16 if bf16 else torch.float32
    gdn.device_status(clear=True)
    got = gdn.chunk_bwd(dev(q, dt), dev(k, dt), dev(v, dt), dev(g), dev(beta), dev(S0), dev(dO), dev(dST),
                        update=update, gate=gate, prologue=flags)
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    ref = oracle.gdn_backward_prologue_np(update, gate, flags, *x)
    for name, a, b in zip(["dq", "dk", "dv", "dg", "dbeta", "dS0"], got, ref):
        if b is None:
            assert a is None, name
            continue
        err = rel_err(np64(a), b)
        assert err <= TOL, (name, err)
