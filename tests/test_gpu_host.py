"""gdn_chunk_fwd_host: the prefill on host buffers, streamed in head slices.

Each slice runs the same kernel as gdn_chunk_fwd on a subset of heads, so the
results equal the device call bit for bit; the slices cover ragged splits,
more slices than heads, pageable memory and T = 0.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, rel_err
from synth import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    gdn.device_status(clear=True)


def host(x, dt, pin):
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dt).contiguous()
    return t.pin_memory() if pin else t


def run_both(w, n_slices, pin=True, with_state=True):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    x = make_prefill_inputs(w)
    h = {k: host(v, dt if k in ("q", "k", "v") else torch.float32, pin) for k, v in x.items()}
    o_h, S_h = gdn.chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], h["S0"], update=w.update, gate=w.gate,
                                  n_slices=n_slices, return_state=with_state)
    torch.cuda.synchronize()
    d = {k: (None if v is None else v.cuda()) for k, v in h.items()}
    o_d, S_d = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], update=w.update, gate=w.gate,
                             return_state=with_state)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return x, (o_h, S_h), (o_d.cpu(), None if S_d is None else S_d.cpu())


def test_ragged_slices_equal_the_device_call_and_the_oracle():
    w = WORKLOADS["gdn_prefill_bf16"].with_(B=2, H=5, T=300, s0_std=0.05, name="host")
    x, (o_h, S_h), (o_d, S_d) = run_both(w, 4)  # 3 + 3 + 3 + 1 heads
    assert torch.equal(o_h, o_d) and torch.equal(S_h, S_d)
    ro, rS = oracle.gdn_forward("delta", "scalar", x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    assert rel_err(o_h.double().numpy(), ro) <= TOL["bf16"] and rel_err(S_h.double().numpy(), rS) <= TOL["bf16"]


@pytest.mark.parametrize("n_slices,pin", [(1, False), (16, True), (3, False)])
def test_slicing_and_memory_kinds(n_slices, pin):
    w = WORKLOADS["kda_prefill_bf16"].with_(B=1, H=4, T=200, s0_std=0.05, name="host_kda")
    _, (o_h, S_h), (o_d, S_d) = run_both(w, n_slices, pin=pin)
    assert torch.equal(o_h, o_d) and torch.equal(S_h, S_d)


def test_fp32_additive_without_states():
    w = WORKLOADS["linear_attn_bf16"].with_(B=1, H=3, T=130, dtype="f32", name="host_la")
    _, (o_h, S_h), (o_d, _) = run_both(w, 2, with_state=False)
    assert S_h is None and torch.equal(o_h, o_d)


def test_zero_tokens_copy_the_state():
    w = WORKLOADS["gdn_prefill_bf16"].with_(B=1, H=3, T=0, s0_std=0.05, name="host_empty")
    x, (o_h, S_h), _ = run_both(w, 2)
    assert o_h.numel() == 0 and np.array_equal(S_h.numpy(), x["S0"])
