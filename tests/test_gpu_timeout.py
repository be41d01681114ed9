"""The bounded waits' expiry path, forced on the GPU without a fault: the wait
bound is set to 1 ns (gdn_set_wait_limit_ns), so the first hand-off that is not
already complete runs out.  The call must record GDN_ERR_TIMEOUT and return
(its kernel lets the copies and MMAs it issued land before it frees its memory),
and the next call with the default bound must be correct."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, np64, rel_err
from synth import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu

TIMEOUT = -5


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    oracle.build()
    gdn.device_status(clear=True)
    yield
    gdn.set_wait_limit_ns(0)


def _prefill(w, x, algo):
    t = {n: dev(x[n], torch.bfloat16) for n in ("q", "k", "v")}
    return gdn.chunk_fwd(t["q"], t["k"], t["v"], dev(x["g"]), dev(x["beta"]), dev(x["S0"]), update=w.update,
                         gate=w.gate, algo=algo)


@pytest.mark.parametrize("name,update,gate,algo", [
    ("gdn_prefill_bf16", "delta", "scalar", "tc"),      # the pipelined tensor-core kernel
    ("kda_prefill_bf16", "delta", "channel", "tc"),     # its per-channel gate instantiation
    ("linear_attn_bf16", "additive", "none", "auto"),   # the linear-attention kernel
])
def test_prefill_wait_expiry_then_recovery(name, update, gate, algo):
    w = WORKLOADS[name].with_(B=1, H=3, T=700, s0_std=0.05, name="timeout_case")
    x = make_prefill_inputs(w)
    gdn.device_status(clear=True)
    gdn.set_wait_limit_ns(1)
    try:
        _prefill(w, x, algo)
        torch.cuda.synchronize()
        assert gdn.device_status(clear=True) == TIMEOUT
    finally:
        gdn.set_wait_limit_ns(0)
    o, ST = _prefill(w, x, algo)
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    ro, rS = oracle.gdn_forward(update, gate, x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(ST), rS) <= TOL["bf16"]


def test_multi_token_decode_wait_expiry_then_recovery():
    w = WORKLOADS["decode_gdn_bf16"].with_(B=4, H=8)
    r = np.random.default_rng(31)
    B, H, T, d = 4, 8, 4, 128
    q = r.standard_normal((B, H, T, d)).astype(np.float32)
    k = r.standard_normal((B, H, T, d)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, H, T, d)).astype(np.float32)
    g = -r.uniform(0.0, 0.05, (B, H, T)).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-r.standard_normal((B, H, T))))).astype(np.float32)
    S0 = (0.02 * r.standard_normal((B, H, d, d))).astype(np.float32)
    args = [dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), dev(g), dev(beta)]
    gdn.device_status(clear=True)
    S = dev(S0)
    gdn.set_wait_limit_ns(1)
    try:
        gdn.decode_step(*args, S, update=w.update, gate=w.gate)
        torch.cuda.synchronize()
        assert gdn.device_status(clear=True) == TIMEOUT
    finally:
        gdn.set_wait_limit_ns(0)
    S = dev(S0)
    o = gdn.decode_step(*args, S, update=w.update, gate=w.gate)
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    rnd = lambda a: np64(dev(a, torch.bfloat16))
    steps = [{"q": rnd(q[:, :, t:t + 1]), "k": rnd(k[:, :, t:t + 1]), "v": rnd(v[:, :, t:t + 1]),
              "g": g[:, :, t:t + 1].astype(np.float64), "beta": beta[:, :, t:t + 1].astype(np.float64)}
             for t in range(T)]
    ro, rS = oracle.decode_sequence("delta", "scalar", S0.astype(np.float64), steps)
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(S), rS) <= TOL["bf16"]
