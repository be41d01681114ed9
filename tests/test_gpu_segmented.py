"""GPU parity of the segmented (sequence-parallel) prefill against the oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, np64, rel_err
from synth import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu

MODES = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
         ("delta", "none"), ("delta", "scalar"), ("delta", "channel")]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    gdn.device_status(clear=True)


def workload(update, gate, dtype, T, B=1, H=2, d=128, seed=13):
    if update == "additive":
        base = WORKLOADS["linear_attn_bf16"]
    else:
        base = WORKLOADS["kda_prefill_bf16"] if gate == "channel" else WORKLOADS["gdn_prefill_bf16"]
    gate_dist = base.gate_dist if gate != "none" else None
    if gate != "none" and gate_dist is None:
        gate_dist = ("uniform", -0.05, 0.0)
    return base.with_(B=B, H=H, T=T, dk=d, dv=d, update=update, gate=gate, gate_dist=gate_dist, dtype=dtype,
                      s0_std=0.05, seed=seed, name="seg_small")


def run(w, x, nseg, **kw):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t = {k_: (None if v_ is None else dev(v_, dt if k_ in ("q", "k", "v") else torch.float32)) for k_, v_ in x.items()}
    o, ST = gdn.chunk_fwd_segmented(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], update=w.update,
                                    gate=w.gate, nseg=nseg, **kw)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return o, ST


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,nseg", [(256, 2), (200, 4)])
def test_segmented_matches_oracle(update, gate, dtype, T, nseg):
    w = workload(update, gate, dtype, T)
    x = make_prefill_inputs(w)
    o, ST = run(w, x, nseg)
    ro, rS = oracle.gdn_forward(update, gate, x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (eo, es)


def test_segmented_many_segments_full_width():
    # 16 segments of 256 tokens on 4 heads: 64 segment-heads through the tensor-core kernel
    w = workload("delta", "scalar", "bf16", 4096, B=1, H=4)
    x = make_prefill_inputs(w)
    o, ST = run(w, x, 16)
    ro, rS = oracle.gdn_forward("delta", "scalar", x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(ST), rS) <= TOL["bf16"]


def test_segmented_with_prologue():
    r = np.random.default_rng(17)
    B, H, T, d = 1, 2, 192, 128
    from synth import round_to_bf16
    q = round_to_bf16(r.standard_normal((B, H, T, d)).astype(np.float32))
    k = round_to_bf16(r.standard_normal((B, H, T, d)).astype(np.float32))
    v = round_to_bf16(r.standard_normal((B, H, T, d)).astype(np.float32))
    bl = r.standard_normal((B, H, T)).astype(np.float32)
    gl = (r.standard_normal((B, H, T)) - 3.0).astype(np.float32)
    flags = gdn.PRO_QK_L2 | gdn.PRO_BETA_SIGMOID | gdn.PRO_G_NEG_SOFTPLUS
    o, ST = gdn.chunk_fwd_segmented(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16),
                                    dev(gl), dev(bl), None, update="delta", gate="scalar", nseg=3, prologue=flags)
    torch.cuda.synchronize()
    qq, kk, bb, gg = oracle.prologue(flags, q, k, bl, gl)
    ro, rS = oracle.gdn_forward("delta", "scalar", qq, kk, v, g=gg, beta=bb)
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(ST), rS) <= TOL["bf16"]


def test_segmented_rejects_uneven_split():
    w = workload("delta", "scalar", "bf16", 100)
    x = make_prefill_inputs(w)
    with pytest.raises(gdn.GDNError):
        run(w, x, 3)
