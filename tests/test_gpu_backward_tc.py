"""GPU parity of the chunkwise tensor-core backward (gdn_chunk_bwd_tc) against
the float64 oracle ``oracle.gdn_backward_np`` (pinned to finite differences of
the forward definition).

The call runs from saved chunk-entry states.  Two sources of states:
* the oracle's own states (float64 recurrence over each prefix, rounded to
  fp32), so only the backward's tf32 products separate it from the oracle;
* the tensor-core forward's states (gdn_chunk_fwd_states), the training path,
  at the bf16 bound of the forward parity tests."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import dev, np64, rel_err
from test_gpu_backward import inputs

pytestmark = pytest.mark.gpu

MODES = [("additive", "none"), ("decay", "scalar"), ("delta", "none"), ("delta", "scalar")]
NAMES = ["dq", "dk", "dv", "dg", "dbeta", "dS0"]
# tf32 products (10-bit significand, fp32 accumulation) on exact states
TOL_TC = 1e-2
# the tensor-core forward's states (fp16 operands) on top
TOL_STATES = 2e-2


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    gdn.device_status(clear=True)


def oracle_states(update, gate, q, k, v, g, beta, S0):
    """The state entering every chunk of 64 tokens, from the float64 recurrence."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    nch = (T + 63) // 64
    out = np.zeros((B, H, nch, dv, dk))
    for c in range(nch):
        if c == 0:
            out[:, :, 0] = 0.0 if S0 is None else S0
            continue
        t = 64 * c
        sl = lambda a: None if a is None else np.ascontiguousarray(a[:, :, :t])
        _, out[:, :, c] = oracle.gdn_forward(update, gate, sl(q), sl(k), sl(v), g=sl(g), beta=sl(beta), S0=S0)
    return out


def run_tc(update, gate, x, bf16, states=None, tol=TOL_TC):
    q, k, v, g, beta, S0, dO, dST = x
    dt = torch.bfloat16 if bf16 else torch.float32
    if states is None:
        states = dev(oracle_states(update, gate, q, k, v, g, beta, S0))
    gdn.device_status(clear=True)
    got = gdn.chunk_bwd(dev(q, dt), dev(k, dt), dev(v, dt), dev(g), dev(beta), None, dev(dO), dev(dST),
                        update=update, gate=gate, states=states, algo="tc")
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    ref = oracle.gdn_backward_np(update, gate, q, k, v, g, beta, S0, dO, dST)
    errs = {}
    for name, a, b in zip(NAMES, got, ref):
        if b is None:
            assert a is None, name
            continue
        errs[name] = rel_err(np64(a), b)
    assert all(e <= tol for e in errs.values()), errs
    return got


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("T", [1, 64, 150, 300])
def test_tc_backward_matches_oracle(update, gate, dv, T):
    # one to five chunks, ragged tails
    run_tc(update, gate, inputs(31, update, gate, T=T, dv=dv), bf16=False)


@pytest.mark.parametrize("update,gate", MODES)
def test_tc_backward_bf16_inputs(update, gate):
    run_tc(update, gate, inputs(32, update, gate, T=200, bf16=True), bf16=True)


@pytest.mark.parametrize("s0,grads", [(False, (True, False)), (True, (False, True)), (False, (False, False))])
def test_tc_backward_optional_inputs(s0, grads):
    run_tc("delta", "scalar", inputs(33, "delta", "scalar", T=130, s0=s0, grads=grads), bf16=False)


def test_tc_backward_many_heads():
    run_tc("delta", "scalar", inputs(34, "delta", "scalar", B=3, H=5, T=140, bf16=True), bf16=True)


def test_tc_backward_deep_decay():
    """About -2 nats per token: e^G of a chunk falls below the fp32 range; the
    gradient must stay finite and match.  Bound: the tensor-core one (2e-2) of
    the forward parity tests; this stress case measures 1.2e-2 on dk (every
    product's operands rounded to tf32; rounding q and k alone gives 2.5e-3 in a
    float64 model of the chunk algebra)."""
    x = list(inputs(35, "delta", "scalar", T=200))
    r = np.random.default_rng(35)
    x[3] = np.asarray(-2.0 + 0.3 * r.standard_normal(x[3].shape), np.float32).astype(np.float64)
    got = run_tc("delta", "scalar", tuple(x), bf16=False, tol=TOL_STATES)
    assert all(a is None or torch.isfinite(a).all() for a in got)


def test_tc_backward_repeated_key_in_chunk():
    """One unit key written 8 times in a chunk with beta = 1: the worst case of
    the triangular solve."""
    x = list(inputs(36, "delta", "none", T=96))
    x[1][:, :, 10:18] = x[1][:, :, 10:11]
    x[4][:, :, 10:18] = 1.0
    run_tc("delta", "none", tuple(x), bf16=False)


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dv,T", [(128, 150), (64, 200)])
def test_tc_backward_from_tensor_core_forward_states(update, gate, dv, T):
    """The training path: gdn_chunk_fwd_states, then gdn_chunk_bwd_tc; also
    against the token backward from the same states."""
    x = inputs(37, update, gate, T=T, dv=dv, bf16=True)
    q, k, v, g, beta, S0, dO, dST = x
    t = [dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), dev(g), dev(beta)]
    states = torch.empty((1, 2, (T + 63) // 64, dv, 128), dtype=torch.float32, device="cuda")
    gdn.chunk_fwd(*t, dev(S0), update=update, gate=gate, states=states)
    got = run_tc(update, gate, x, bf16=True, states=states, tol=TOL_STATES)
    tok = gdn.chunk_bwd(*t, None, dev(dO), dev(dST), update=update, gate=gate, states=states)
    torch.cuda.synchronize()
    for name, a, b in zip(NAMES, got, tok):
        if a is not None:
            assert rel_err(np64(a), np64(b)) <= TOL_TC, name


def test_tc_backward_is_deterministic():
    x = inputs(38, "delta", "scalar", T=200, bf16=True)
    q, k, v, g, beta, S0, dO, dST = x
    t = [dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), dev(g), dev(beta)]
    states = dev(oracle_states("delta", "scalar", q, k, v, g, beta, S0))
    a = gdn.chunk_bwd(*t, None, dev(dO), dev(dST), update="delta", gate="scalar", states=states, algo="tc")
    b = gdn.chunk_bwd(*t, None, dev(dO), dev(dST), update="delta", gate="scalar", states=states, algo="tc")
    torch.cuda.synchronize()
    assert all(torch.equal(u, w) for u, w in zip(a, b))


def test_tc_backward_rejects_unsupported_requests():
    x = inputs(39, "delta", "channel", T=70)
    q, k, v, g, beta = (dev(a) for a in x[:5])
    states = torch.zeros((1, 2, 2, 128, 128), device="cuda")
    with pytest.raises(gdn.GDNError):
        gdn.chunk_bwd(q, k, v, g, beta, None, None, None, update="delta", gate="channel", states=states, algo="tc")
    x = inputs(39, "delta", "scalar", T=70, dk=64, dv=64)
    q, k, v, g, beta = (dev(a) for a in x[:5])
    states = torch.zeros((1, 2, 2, 64, 64), device="cuda")
    with pytest.raises(gdn.GDNError):
        gdn.chunk_bwd(q, k, v, g, beta, None, None, None, update="delta", gate="scalar", states=states, algo="tc")


def test_tc_backward_full_size_sampled_heads():
    """The GDN workload (8 x 16 x 8192) at full size, in the launch configuration
    the benchmark times: gdn_chunk_fwd_states, then gdn_chunk_bwd_tc over all 128
    heads.  Sampled heads are compared whole against the oracle's gradients."""
    from synth import WORKLOADS, make_prefill_inputs

    w = WORKLOADS["gdn_prefill_bf16"]
    x = make_prefill_inputs(w)
    t = [dev(x["q"], torch.bfloat16), dev(x["k"], torch.bfloat16), dev(x["v"], torch.bfloat16), dev(x["g"]),
         dev(x["beta"])]
    S0 = dev(x["S0"])
    del x
    gen = torch.Generator(device="cuda").manual_seed(41)
    dO = torch.randn((w.B, w.H, w.T, w.dv), device="cuda", generator=gen)
    dST = torch.randn((w.B, w.H, w.dv, w.dk), device="cuda", generator=gen)
    states = torch.empty((w.B, w.H, (w.T + 63) // 64, w.dv, w.dk), device="cuda")
    gdn.device_status(clear=True)
    gdn.chunk_fwd(*t, S0, update=w.update, gate=w.gate, states=states)
    got = gdn.chunk_bwd(*t, None, dO, dST, update=w.update, gate=w.gate, states=states, algo="tc")
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    assert all(a is None or torch.isfinite(a).all() for a in got)
    heads = [(0, 0), (7, 15), (3, 9)]
    xs = make_prefill_inputs(w, heads=heads)
    for i, (b, h) in enumerate(heads):
        one = lambda a: None if a is None else np.asarray(a[i:i + 1], np.float64)
        ref = oracle.gdn_backward_np(w.update, w.gate, one(xs["q"]), one(xs["k"]), one(xs["v"]), one(xs["g"]),
                                     one(xs["beta"]), one(xs["S0"]), np64(dO[b, h])[None, None],
                                     np64(dST[b, h])[None, None])
        for name, a, r in zip(NAMES, got, ref):
            if r is None:
                continue
            err = rel_err(np64(a[b, h]), r[0, 0])
            assert err <= TOL_STATES, ((b, h), name, err)


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dv,T", [(128, 150), (64, 200)])
def test_one_call_tensor_core_backward(update, gate, dv, T):
    """gdn_chunk_bwd with GDN_ALGO_TC (no saved states): the tensor-core forward
    writes the states into the workspace (without o), then the chunkwise
    backward.  Equals the two-call training path bit for bit, and the oracle at
    the tensor-core bound."""
    x = inputs(47, update, gate, T=T, dv=dv, bf16=True)
    q, k, v, g, beta, S0, dO, dST = x
    t = [dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), dev(g), dev(beta)]
    gdn.device_status(clear=True)
    one = gdn.chunk_bwd(*t, dev(S0), dev(dO), dev(dST), update=update, gate=gate, algo="tc")
    states = torch.empty((1, 2, (T + 63) // 64, dv, 128), dtype=torch.float32, device="cuda")
    gdn.chunk_fwd(*t, dev(S0), update=update, gate=gate, states=states)
    two = gdn.chunk_bwd(*t, None, dev(dO), dev(dST), update=update, gate=gate, states=states, algo="tc")
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    ref = oracle.gdn_backward_np(update, gate, *x)
    for name, a, b, r in zip(NAMES, one, two, ref):
        if r is None:
            assert a is None, name
            continue
        assert torch.equal(a, b), name
        assert rel_err(np64(a), r) <= TOL_STATES, (name, rel_err(np64(a), r))
