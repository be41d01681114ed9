"""GPU parity of the linear-attention tensor-core kernel (additive update, no
gate; taken by gdn_chunk_fwd with GDN_ALGO_AUTO) against the float64 oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, np64, rel_err, run_prefill
from synth import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    oracle.build()
    gdn.device_status(clear=True)


def workload(T, B=1, H=2, dv=128, s0=0.05, seed=5):
    return WORKLOADS["linear_attn_bf16"].with_(B=B, H=H, T=T, dv=dv, s0_std=s0, seed=seed, name="la_small")


def check(w, x, out_dtype=torch.float32, algo="auto"):
    o, ST = run_prefill(w, x, algo=algo, out_dtype=out_dtype)
    ro, rS = oracle.gdn_forward("additive", "none", x["q"], x["k"], x["v"], S0=x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)
    return o, ST


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 128, 129, 200, 257])
@pytest.mark.parametrize("dv", [64, 128])
def test_la_matches_oracle(T, dv):
    # one to five chunks, ragged tails: the two stages, the two P / O buffers
    # and their phases all start and wrap here
    w = workload(T, dv=dv)
    check(w, make_prefill_inputs(w))


def test_la_wide_value_slice():
    """More heads than SMs: 320 CTAs of 64 value rows, in several waves."""
    w = workload(130, B=2, H=80)
    check(w, make_prefill_inputs(w))


def test_la_equals_masked_product():
    """With S0 = 0 the output is the causal masked (Q K^T) V product, here
    formed in float64 from the bf16-rounded inputs."""
    w = workload(300, s0=0.0)
    x = make_prefill_inputs(w)
    o, ST = check(w, x)
    q = np64(dev(x["q"], torch.bfloat16))
    k = np64(dev(x["k"], torch.bfloat16))
    v = np64(dev(x["v"], torch.bfloat16))
    A = np.tril(np.einsum("bhtd,bhsd->bhts", q, k))
    ref = np.einsum("bhts,bhsv->bhtv", A, v)
    assert rel_err(np64(o), ref) <= TOL["bf16"]
    assert rel_err(np64(ST), np.einsum("bhsv,bhsd->bhvd", v, k)) <= TOL["bf16"]


def test_la_agrees_with_general_tensor_core_kernel():
    w = workload(400, B=2, H=3)
    x = make_prefill_inputs(w)
    o1, S1 = check(w, x)
    o2, S2 = check(w, x, algo="tc")
    assert rel_err(np64(o1), np64(o2)) <= TOL["bf16"] and rel_err(np64(S1), np64(S2)) <= TOL["bf16"]


def test_la_bf16_output_is_rounded_fp32_output():
    w = workload(150)
    x = make_prefill_inputs(w)
    o32, S32 = run_prefill(w, x)
    o16, S16 = run_prefill(w, x, out_dtype=torch.bfloat16)
    assert torch.equal(o32.to(torch.bfloat16), o16) and torch.equal(S32, S16)


def test_la_without_initial_state_and_deterministic():
    w = workload(260, s0=0.0)
    x = make_prefill_inputs(w)
    t = {k_: dev(x[k_], torch.bfloat16) for k_ in ("q", "k", "v")}
    o1, S1 = gdn.chunk_fwd(t["q"], t["k"], t["v"], None, None, None, update="additive", gate="none")
    o2, S2 = gdn.chunk_fwd(t["q"], t["k"], t["v"], None, None, None, update="additive", gate="none")
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    ro, rS = oracle.gdn_forward("additive", "none", x["q"], x["k"], x["v"])
    assert rel_err(np64(o1), ro) <= TOL["bf16"] and rel_err(np64(S1), rS) <= TOL["bf16"]


def test_la_state_chains_across_calls():
    """Two calls over the halves of a sequence, the second starting from the
    first's final state, give the one-call result."""
    w = workload(256)
    x = make_prefill_inputs(w)
    t = {k_: dev(x[k_], torch.bfloat16) for k_ in ("q", "k", "v")}
    S0 = dev(x["S0"])
    o, S = gdn.chunk_fwd(t["q"], t["k"], t["v"], None, None, S0, update="additive", gate="none")
    h = 128
    oa, Sa = gdn.chunk_fwd(*(t[k_][:, :, :h].contiguous() for k_ in ("q", "k", "v")), None, None, S0,
                           update="additive", gate="none")
    ob, Sb = gdn.chunk_fwd(*(t[k_][:, :, h:].contiguous() for k_ in ("q", "k", "v")), None, None, Sa,
                           update="additive", gate="none")
    torch.cuda.synchronize()
    assert rel_err(np64(torch.cat([oa, ob], dim=2)), np64(o)) <= 1e-5
    assert rel_err(np64(Sb), np64(S)) <= 1e-5


def test_la_state_in_place():
    """S_T may be S0 itself: each CTA reads its rows of S0 before it writes them."""
    w = workload(200, B=2, H=3)
    x = make_prefill_inputs(w)
    t = {k_: dev(x[k_], torch.bfloat16) for k_ in ("q", "k", "v")}
    o1, S1 = gdn.chunk_fwd(t["q"], t["k"], t["v"], None, None, dev(x["S0"]), update="additive", gate="none")
    S = dev(x["S0"])
    o2, S2 = gdn.chunk_fwd(t["q"], t["k"], t["v"], None, None, S, update="additive", gate="none", S_T=S)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2) and S2.data_ptr() == S.data_ptr()
