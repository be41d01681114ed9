"""GPU parity of the input prologue (GDN_PRO_* maps applied in-kernel) against
the oracle run on the host-mapped inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, np64, rel_err
from synth import round_to_bf16

pytestmark = pytest.mark.gpu

L2, ELU1, SIG, SP = gdn.PRO_QK_L2, gdn.PRO_QK_ELU1, gdn.PRO_BETA_SIGMOID, gdn.PRO_G_NEG_SOFTPLUS


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    gdn.device_status(clear=True)


def raw_inputs(update, gate, dtype, B=2, H=2, T=150, dk=128, dv=128, seed=3, nh=None):
    """Raw projections: q, k ~ N(0,1) (unnormalised), v ~ N(0,1), beta and gate as
    logits (beta ~ N(0,1), g ~ N(-3,1) or N(-4,1) per channel)."""
    r = np.random.default_rng(seed)
    kshape = (B, H, T, dk) if nh is None else (B, H, T, nh, dk)
    vshape = (B, H, T, dv) if nh is None else (B, H, T, nh, dv)
    rd = (lambda a: round_to_bf16(a.astype(np.float32))) if dtype == "bf16" else (lambda a: a.astype(np.float32))
    x = {"q": rd(r.standard_normal((B, H, T, dk))), "k": rd(r.standard_normal(kshape)),
         "v": rd(r.standard_normal(vshape)), "beta": None, "g": None,
         "S0": (0.05 * r.standard_normal((B, H, dv, dk))).astype(np.float32)}
    if update == "delta":
        x["beta"] = r.standard_normal(kshape[:-1]).astype(np.float32)
    if gate == "scalar":
        x["g"] = (r.standard_normal((B, H, T)) - 3.0).astype(np.float32)
    elif gate == "channel":
        x["g"] = (r.standard_normal((B, H, T, dk)) - 4.0).astype(np.float32)
    return x


def to_dev(x, dtype):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return {k_: (None if v_ is None else dev(v_, dt if k_ in ("q", "k", "v") else torch.float32))
            for k_, v_ in x.items()}


CASES = [("delta", "scalar", L2 | SIG | SP), ("delta", "channel", L2 | SIG | SP), ("delta", "none", L2 | SIG),
         ("additive", "none", ELU1), ("decay", "scalar", ELU1 | L2 | SP), ("delta", "scalar", ELU1 | L2 | SIG | SP)]
# (the delta rule needs unit keys, so every delta case normalises them)


@pytest.mark.parametrize("update,gate,flags", CASES)
@pytest.mark.parametrize("dtype,algo", [("f32", "simt"), ("bf16", "simt"), ("bf16", "auto")])
def test_prefill_prologue(update, gate, flags, dtype, algo):
    x = raw_inputs(update, gate, dtype)
    if update == "additive" and not flags & (L2 | ELU1):
        pytest.skip("unmapped additive inputs")
    t = to_dev(x, dtype)
    o, ST = gdn.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], update=update, gate=gate,
                          algo=algo, prologue=flags)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    q, k, beta, g = oracle.prologue(flags, x["q"], x["k"], x["beta"], x["g"])
    ro, rS = oracle.gdn_forward(update, gate, q, k, x["v"], g=g, beta=beta, S0=x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    tol = TOL["f32"] if dtype == "f32" else TOL["bf16"]
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.parametrize("update,gate,flags", CASES)
@pytest.mark.parametrize("T", [1, 4])
def test_decode_prologue(update, gate, flags, T):
    x = raw_inputs(update, gate, "bf16", B=3, H=4, T=T)
    t = to_dev(x, "bf16")
    S = t["S0"].clone()
    o = gdn.decode_step(t["q"], t["k"], t["v"], t["g"], t["beta"], S, update=update, gate=gate, prologue=flags)
    torch.cuda.synchronize()
    q, k, beta, g = oracle.prologue(flags, x["q"], x["k"], x["beta"], x["g"])
    ro, rS = oracle.gdn_forward(update, gate, q, k, x["v"], g=g, beta=beta, S0=x["S0"])
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(S), rS) <= TOL["bf16"]


@pytest.mark.parametrize("gate,flags", [("scalar", L2 | SIG | SP), ("none", L2 | SIG)])
@pytest.mark.parametrize("nh,algo", [(2, "auto"), (3, "auto"), (2, "simt")])
def test_product_prologue(gate, flags, nh, algo):
    x = raw_inputs("delta", gate, "bf16", T=70, nh=nh)
    t = to_dev(x, "bf16")
    o, ST = gdn.product_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], gate=gate, algo=algo,
                            prologue=flags)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    q, k, beta, g = oracle.prologue(flags, x["q"], x["k"], x["beta"], x["g"])
    ro, rS = oracle.gdp_forward(gate, q, k, x["v"], g, beta, x["S0"])
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(ST), rS) <= TOL["bf16"]
