"""GPU parity of Gated DeltaProduct (gdn_product_fwd) against the oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, np64, rel_err
from synth import WORKLOADS, make_product_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    gdn.device_status(clear=True)


def workload(gate, dtype, T, d=64, B=2, H=2, s0=0.05, seed=21):
    base = WORKLOADS["kda_prefill_bf16"] if gate == "channel" else WORKLOADS["gdn_prefill_bf16"]
    gate_dist = base.gate_dist if gate != "none" else None
    return base.with_(B=B, H=H, T=T, dk=d, dv=d, gate=gate, gate_dist=gate_dist, dtype=dtype, s0_std=s0,
                      seed=seed, name="gdp_small")


def run(w, x, nh, algo="auto"):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t = {k_: (None if v_ is None else dev(v_, dt if k_ in ("q", "k", "v") else torch.float32)) for k_, v_ in x.items()}
    o, ST = gdn.product_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], gate=w.gate, algo=algo)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return o, ST


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("nh", [2, 3, 4])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_product_matches_oracle(gate, nh, dtype):
    # T = 50 real tokens: 100 to 200 virtual steps, ragged, with tokens that
    # straddle chunk boundaries when nh does not divide 64
    w = workload(gate, dtype, T=50)
    x = make_product_inputs(w, nh)
    o, ST = run(w, x, nh)
    ro, rS = oracle.gdp_forward(gate, x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (eo, es)


def test_product_full_width_bf16():
    w = workload("scalar", "bf16", T=100, d=128, B=1, H=3)
    x = make_product_inputs(w, 2)
    o, ST = run(w, x, 2)
    ro, rS = oracle.gdp_forward("scalar", x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(ST), rS) <= TOL["bf16"]


def test_product_one_substep_is_chunk_fwd():
    w = workload("scalar", "f32", T=90)
    x = make_product_inputs(w, 1)
    o, ST = run(w, x, 1)
    t = {k_: (None if v_ is None else dev(v_)) for k_, v_ in x.items()}
    o1, S1 = gdn.chunk_fwd(t["q"], t["k"][:, :, :, 0].contiguous(), t["v"][:, :, :, 0].contiguous(), t["g"],
                           t["beta"][:, :, :, 0].contiguous(), t["S0"], update="delta", gate="scalar")
    assert torch.equal(o, o1) and torch.equal(ST, S1)


def test_product_empty_sequence_copies_state():
    w = workload("scalar", "f32", T=0)
    S0 = dev(np.random.default_rng(5).standard_normal((2, 2, 64, 64)))
    q = torch.empty((2, 2, 0, 64), device="cuda")
    k = torch.empty((2, 2, 0, 3, 64), device="cuda")
    o, ST = gdn.product_fwd(q, k, k, torch.empty((2, 2, 0), device="cuda"), torch.empty((2, 2, 0, 3), device="cuda"),
                            S0, gate="scalar")
    torch.cuda.synchronize()
    assert o.shape == (2, 2, 0, 64) and torch.equal(ST, S0)


@pytest.mark.parametrize("nh", [2, 3, 5, 16])
@pytest.mark.parametrize("dv,T", [(128, 37), (64, 100)])
def test_product_tensor_core_channel_gate(nh, dv, T):
    # per-channel (KDA) gate: each token's gate row sits on its first substep and
    # the other rows of the chunk carry g = 0
    w = workload("channel", "bf16", T=T, d=128).with_(dv=dv)
    x = make_product_inputs(w, nh)
    o, ST = run(w, x, nh, algo="tc")
    ro, rS = oracle.gdp_forward("channel", x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)


@pytest.mark.parametrize("gate", ["none", "scalar"])
@pytest.mark.parametrize("nh", [2, 3, 4, 5, 7, 8, 16])
@pytest.mark.parametrize("dv,T", [(128, 37), (128, 200), (64, 100)])
def test_product_tensor_core_matches_oracle(gate, nh, dv, T):
    # a chunk holds 64 / nh whole tokens (with nh = 3, 5, 7 its last rows are identity
    # steps and tokens never straddle a chunk); T ragged in tokens
    w = workload(gate, "bf16", T=T, d=128).with_(dv=dv)
    x = make_product_inputs(w, nh)
    o, ST = run(w, x, nh, algo="tc")
    ro, rS = oracle.gdp_forward(gate, x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)


@pytest.mark.parametrize("nh", [3, 4])
def test_product_tensor_core_matches_simt(nh):
    w = workload("scalar", "bf16", T=300, d=128, B=1, H=4)
    x = make_product_inputs(w, nh)
    o_tc, S_tc = run(w, x, nh, algo="tc")
    o_s, S_s = run(w, x, nh, algo="simt")
    assert rel_err(np64(o_tc), np64(o_s)) <= TOL["bf16"] and rel_err(np64(S_tc), np64(S_s)) <= TOL["bf16"]
