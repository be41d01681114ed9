"""GPU parity of the tensor-core (tcgen05) prefill kernel against the oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, io_dtype, np64, rel_err, run_prefill
from synth import WORKLOADS, make_prefill_inputs, round_to_bf16

pytestmark = pytest.mark.gpu

MODES = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
         ("delta", "none"), ("delta", "scalar"), ("delta", "channel")]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    oracle.build()
    gdn.device_status(clear=True)


def workload(update, gate, T, B=2, H=2, dv=128, s0=0.05, seed=7):
    # the delta rule needs normalised keys (beta |k|^2 <= 1 keeps the transition
    # contractive); elu+1 features only feed the additive write
    if update == "additive":
        base = WORKLOADS["linear_attn_bf16"]
    else:
        base = WORKLOADS["kda_prefill_bf16"] if gate == "channel" else WORKLOADS["gdn_prefill_bf16"]
    gate_dist = base.gate_dist if gate != "none" else None
    if gate != "none" and gate_dist is None:
        gate_dist = ("uniform", -0.05, 0.0)
    return base.with_(B=B, H=H, T=T, dv=dv, update=update, gate=gate, gate_dist=gate_dist, s0_std=s0,
                      seed=seed, name="tc_small")


def check(w, x, algo="tc", tol=TOL["bf16"], out_dtype=torch.float32):
    o, ST = run_prefill(w, x, algo=algo, out_dtype=out_dtype)
    ro, rS = oracle.gdn_forward(w.update, w.gate, x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dv", [64, 128])
def test_tc_modes(update, gate, dv):
    w = workload(update, gate, T=200, dv=dv)
    check(w, make_prefill_inputs(w))


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 128, 130, 257])
def test_tc_ragged_lengths(T):
    w = workload("delta", "scalar", T=T, B=1, H=3)
    check(w, make_prefill_inputs(w))


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("T", [1, 65, 129])
def test_tc_short_and_ragged_all_modes(update, gate, dv, T):
    # one, two and three chunks: the pipeline's prologue, the chunk-parity buffers
    # (A', K>, beta, the decay factors, V without the delta rule) and the separate v
    # load all start from their first phases here
    w = workload(update, gate, T=T, B=1, H=2, dv=dv, seed=11)
    check(w, make_prefill_inputs(w))


@pytest.mark.parametrize("update,gate", [("delta", "scalar"), ("additive", "none"), ("delta", "none")])
def test_tc_wide_value_slice(update, gate):
    """Enough heads that each CTA takes all 128 value rows of its head."""
    w = workload(update, gate, T=130, B=1, H=80)
    check(w, make_prefill_inputs(w))


@pytest.mark.parametrize("update", ["delta", "decay"])
def test_tc_channel_gate_exact_path(update):
    """Per-channel decay far beyond the factored fp16 range inside a chunk:
    those chunks take the exact fp32 path and still match."""
    w = workload(update, "channel", T=150, B=1, H=2).with_(gate_dist=("uniform", -1.5, -0.2))
    check(w, make_prefill_inputs(w))


def test_tc_matches_simt_path():
    w = workload("delta", "channel", T=300)
    x = make_prefill_inputs(w)
    o1, S1 = run_prefill(w, x, algo="tc")
    o2, S2 = run_prefill(w, x, algo="simt")
    assert rel_err(np64(o1), np64(o2)) < TOL["bf16"] and rel_err(np64(S1), np64(S2)) < TOL["bf16"]


def test_tc_bf16_output_is_rounded_fp32_output():
    w = workload("delta", "scalar", T=130)
    x = make_prefill_inputs(w)
    o32, _ = run_prefill(w, x, algo="tc")
    o16, _ = run_prefill(w, x, algo="tc", out_dtype=torch.bfloat16)
    assert torch.equal(o32.to(torch.bfloat16), o16)


def test_tc_deterministic():
    w = workload("delta", "scalar", T=500)
    x = make_prefill_inputs(w)
    o1, S1 = run_prefill(w, x, algo="tc")
    o2, S2 = run_prefill(w, x, algo="tc")
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_tc_range_overflow_is_reported():
    """Values far beyond fp16 range make an operand overflow: the kernel
    finishes, and the device status word reports GDN_ERR_RANGE."""
    w = workload("additive", "none", T=70, B=1, H=1)
    x = make_prefill_inputs(w)
    x["v"] = (x["v"] * 1e6).astype(np.float32)
    dt = io_dtype(w)
    gdn.device_status(clear=True)
    gdn.chunk_fwd(dev(x["q"], dt), dev(x["k"], dt), dev(x["v"], dt), None, None, dev(x["S0"]),
                  update="additive", gate="none", algo="tc")
    assert gdn.device_status(clear=True) == -6
    assert gdn.device_status() == 0


def test_checked_prefill_recovers_from_range_overflow():
    """gdn_chunk_fwd_checked on values far beyond fp16 range: the tensor-core
    kernel reports GDN_ERR_RANGE, the call runs the request again on the fp32
    kernel and returns its results, at fp32 parity with the oracle."""
    w = workload("delta", "scalar", T=130, B=1, H=2)
    x = make_prefill_inputs(w)
    x["v"] = round_to_bf16((x["v"] * 1e6).astype(np.float32))  # the bf16 values both sides read
    dt = io_dtype(w)
    t = [dev(x["q"], dt), dev(x["k"], dt), dev(x["v"], dt), dev(x["g"]), dev(x["beta"]), dev(x["S0"])]
    gdn.device_status(clear=True)
    o, S, reran = gdn.chunk_fwd(*t, update="delta", gate="scalar", checked=True)
    assert reran and gdn.device_status() == 0
    ro, rS = oracle.gdn_forward("delta", "scalar", x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    assert rel_err(np64(o), ro) <= TOL["f32"] and rel_err(np64(S), rS) <= TOL["f32"]
    o2, S2 = run_prefill(w, x, algo="simt")
    assert torch.equal(o, o2) and torch.equal(S, S2)


def test_checked_prefill_without_overflow_is_the_plain_call():
    w = workload("delta", "scalar", T=200, B=1, H=2)
    x = make_prefill_inputs(w)
    dt = io_dtype(w)
    t = [dev(x["q"], dt), dev(x["k"], dt), dev(x["v"], dt), dev(x["g"]), dev(x["beta"]), dev(x["S0"])]
    gdn.device_status(clear=True)
    o, S, reran = gdn.chunk_fwd(*t, update="delta", gate="scalar", checked=True)
    o2, S2 = gdn.chunk_fwd(*t, update="delta", gate="scalar")
    torch.cuda.synchronize()
    assert not reran and gdn.device_status() == 0
    assert torch.equal(o, o2) and torch.equal(S, S2)


@pytest.mark.parametrize("update,gate", MODES)
def test_tensor_core_matches_simt_kernel(update, gate):
    """The tensor-core kernel (fp16 operands) and the fp32 SIMT kernel agree
    on every mode (same definition, different arithmetic and schedule)."""
    w = workload(update, gate, T=330, B=1, H=3)
    x = make_prefill_inputs(w)
    o1, S1 = run_prefill(w, x, algo="tc")
    o2, S2 = run_prefill(w, x, algo="simt")
    assert rel_err(np64(o1), np64(o2)) < 1e-2 and rel_err(np64(S1), np64(S2)) < 1e-2
