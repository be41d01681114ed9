"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle,
element by element on the same seeded inputs."""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, io_dtype, np64, rel_err, run_prefill
from synth import WORKLOADS, iter_decode_blocks, make_decode_inputs, make_decode_state, make_prefill_inputs

pytestmark = pytest.mark.gpu

MODES = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
         ("delta", "none"), ("delta", "scalar"), ("delta", "channel")]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    gdn.load()
    oracle.build()
    gdn.device_status(clear=True)


def small_workload(update, gate, dtype, T, dk=128, dv=128, B=2, H=2, s0=0.05, seed=5):
    base = WORKLOADS["kda_prefill_bf16"] if gate == "channel" else WORKLOADS["gdn_prefill_bf16"]
    if update == "additive":
        base = WORKLOADS["linear_attn_bf16"]
    return base.with_(B=B, H=H, T=T, dk=dk, dv=dv, update=update, gate=gate, dtype=dtype, s0_std=s0,
                      seed=seed, name="small")


def check_against_oracle(w, x, o, ST, tol):
    ro, rS = oracle.gdn_forward(w.update, w.gate, x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    eo, es = rel_err(np64(o), ro), rel_err(np64(ST), rS)
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


# ---------------------------------------------------------------------------
# Small cases: every mode, gate, head dim and dtype; several chunks + ragged tail
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_simt_small(update, gate, dtype, dk, dv):
    w = small_workload(update, gate, dtype, T=200, dk=dk, dv=dv)
    x = make_prefill_inputs(w)
    o, ST = run_prefill(w, x, algo="simt")
    check_against_oracle(w, x, o, ST, TOL[dtype])


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 129, 300])
def test_simt_ragged_lengths(T):
    w = small_workload("delta", "channel", "f32", T=T, B=1, H=3)
    x = make_prefill_inputs(w)
    o, ST = run_prefill(w, x, algo="simt")
    check_against_oracle(w, x, o, ST, TOL["f32"])


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def test_tiny_gdn_f32_full():
    """Tiny fp32 GDN workload, whole tensors."""
    w = WORKLOADS["tiny_gdn_f32"]
    x = make_prefill_inputs(w)
    o, ST = run_prefill(w, x)
    check_against_oracle(w, x, o, ST, TOL["f32"])


SAMPLED = [(0, 0), (1, 7), (-1, -1)]


@pytest.mark.parametrize("name", ["linear_attn_bf16", "gdn_prefill_bf16", "kda_prefill_bf16"])
def test_full_size_sampled_heads(name):
    """Full-size workload run in one launch (as the benchmark runs it);
    sampled heads compared whole against the oracle."""
    w = WORKLOADS[name]
    x = make_prefill_inputs(w)
    o, ST = run_prefill(w, x)
    heads = [(b % w.B, h % w.H) for b, h in SAMPLED]
    xs = make_prefill_inputs(w, heads=heads)
    ro, rS = oracle.gdn_forward(w.update, w.gate, xs["q"], xs["k"], xs["v"], g=xs["g"], beta=xs["beta"],
                                S0=xs["S0"])
    og = np.stack([np64(o[b, h]) for b, h in heads])
    Sg = np.stack([np64(ST[b, h]) for b, h in heads])
    eo, es = rel_err(og, ro[:, 0]), rel_err(Sg, rS[:, 0])
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)
    # whole-tensor properties that hold at any size
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()


def test_decode_full_size_1000_steps():
    """256 x 32 heads, 1000 consecutive in-place steps; sampled heads compared
    at every step and at the end against the oracle."""
    w = WORKLOADS["decode_gdn_bf16"]
    S = dev(make_decode_state(w))
    dt = io_dtype(w)
    heads = [(0, 0), (100, 17), (255, 31)]
    sel = lambda a: None if a is None else np.stack([a[b, h] for b, h in heads])
    outs, seq = [], []
    for _, blk in iter_decode_blocks(w):
        for s in blk:
            d = {k_: dev(v_, dt if k_ in ("q", "k", "v") else torch.float32) for k_, v_ in s.items()}
            o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, update=w.update, gate=w.gate)
            outs.append(torch.stack([o[b, h, 0] for b, h in heads]))
            seq.append({k_: sel(v_) for k_, v_ in s.items()})
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    og = np64(torch.stack(outs, dim=1))  # [heads, steps, dv]
    S0h = make_decode_state(w, heads=heads)
    ro, rS = oracle.decode_sequence(w.update, w.gate, S0h[:, 0], seq)
    eo = rel_err(og, ro)
    es = rel_err(np.stack([np64(S[b, h]) for b, h in heads]), rS)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)
    assert torch.isfinite(S).all()


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("dtype,dk", [("f32", 64), ("bf16", 128), ("f32", 128)])
def test_decode_small_all_modes(update, gate, dtype, dk):
    w = small_workload(update, gate, dtype, T=1, dk=dk, dv=dk, B=3, H=5).with_(steps=20, q_map="none")
    steps = make_decode_inputs(w, 20)
    S0 = np.random.default_rng(1).standard_normal((3, 5, dk, dk)).astype(np.float32) * 0.05
    S = dev(S0)
    dt = io_dtype(w)
    outs = []
    for s in steps:
        d = {k_: dev(v_, dt if k_ in ("q", "k", "v") else torch.float32) for k_, v_ in s.items()}
        outs.append(np64(gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, update=update,
                                         gate=gate))[:, :, 0])
    og = np.stack(outs, axis=2)
    ro, rS = oracle.decode_sequence(update, gate, S0, steps)
    assert rel_err(og, ro) <= TOL[dtype] and rel_err(np64(S), rS) <= TOL[dtype]


def _stack_steps(steps):
    """List of single-token step inputs -> one [B,H,T,...] input of T tokens."""
    out = {}
    for key in steps[0]:
        out[key] = None if steps[0][key] is None else np.concatenate([s[key] for s in steps], axis=2)
    return out


@pytest.mark.parametrize("update,gate", MODES)
@pytest.mark.parametrize("T", [2, 5, 16])
def test_decode_multi_token_all_modes(update, gate, T):
    # T tokens in one call: the state stays on chip between them
    w = small_workload(update, gate, "bf16", T=1, dk=128, dv=128, B=3, H=5).with_(steps=T, q_map="none")
    steps = make_decode_inputs(w, T)
    x = _stack_steps(steps)
    S0 = np.random.default_rng(2).standard_normal((3, 5, 128, 128)).astype(np.float32) * 0.05
    S = dev(S0)
    d = {k_: (None if v_ is None else dev(v_, torch.bfloat16 if k_ in ("q", "k", "v") else torch.float32))
         for k_, v_ in x.items()}
    o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, update=update, gate=gate)
    ro, rS = oracle.decode_sequence(update, gate, S0, steps)
    assert rel_err(np64(o), ro) <= TOL["bf16"] and rel_err(np64(S), rS) <= TOL["bf16"]


def _decode_multi_case(update, gate, dtype, T, dk, dv, B, H, seed=3, gfix=None):
    w = small_workload(update, gate, dtype, T=1, dk=dk, dv=dv, B=B, H=H, seed=seed).with_(steps=T, q_map="none")
    steps = make_decode_inputs(w, T)
    if gfix is not None:  # a fixed log-gate per token
        for s_ in steps:
            s_["g"] = np.full_like(s_["g"], gfix)
    x = _stack_steps(steps)
    S0 = np.random.default_rng(seed).standard_normal((B, H, dv, dk)).astype(np.float32) * 0.05
    S = dev(S0)
    io = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = {k_: (None if v_ is None else dev(v_, io if k_ in ("q", "k", "v") else torch.float32)) for k_, v_ in x.items()}
    o = gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, update=update, gate=gate)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rS = oracle.decode_sequence(update, gate, S0, steps)
    eo, es = rel_err(np64(o), ro), rel_err(np64(S), rS)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (eo, es)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("update,gate", [("delta", "scalar"), ("delta", "channel"), ("additive", "none")])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_multi_token_head_dims(dk, dv, update, gate, dtype):
    # the persistent kernel's other layouts: dk = 64 (two column blocks per lane), 4 tasks per head at dv = 64
    _decode_multi_case(update, gate, dtype, T=3, dk=dk, dv=dv, B=3, H=7)


def test_decode_multi_token_deep_scalar_decay():
    # g = -30 per token: the carried decay factor falls below 2^-64 after three tokens and is folded
    # into the rows (fp32 inputs, fp32 bound)
    _decode_multi_case("delta", "scalar", "f32", T=9, dk=128, dv=128, B=2, H=3, gfix=-30.0)


def test_decode_multi_token_many_tasks_per_warp():
    # more 16-row tasks (4096) than warps of the persistent grid: every warp walks several tasks and
    # its two state slots cycle through their mbarrier phases
    _decode_multi_case("delta", "scalar", "bf16", T=4, dk=128, dv=128, B=16, H=32, seed=9)


def test_decode_multi_token_equals_single_steps():
    w = small_workload("delta", "channel", "f32", T=1, dk=128, dv=128, B=2, H=3).with_(steps=8, q_map="none")
    steps = make_decode_inputs(w, 8)
    S0 = np.random.default_rng(4).standard_normal((2, 3, 128, 128)).astype(np.float32) * 0.05
    S1, S8 = dev(S0), dev(S0)
    singles = []
    for s in steps:
        d = {k_: (None if v_ is None else dev(v_)) for k_, v_ in s.items()}
        singles.append(gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S1, update="delta",
                                       gate="channel"))
    x = {k_: (None if v_ is None else dev(v_)) for k_, v_ in _stack_steps(steps).items()}
    o8 = gdn.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S8, update="delta", gate="channel")
    torch.cuda.synchronize()
    # the same per-token arithmetic in the same order
    assert rel_err(np64(o8), np64(torch.cat(singles, dim=2))) < 1e-6
    assert rel_err(np64(S8), np64(S1)) < 1e-6


def test_decode_token_count_limits():
    q = torch.zeros((1, 1, gdn.DECODE_MAX_T + 1, 64), device="cuda")
    S = torch.zeros((1, 1, 64, 64), device="cuda")
    with pytest.raises(ValueError):
        gdn.decode_step(q, q, q, None, None, S, update="additive", gate="none")


# ---------------------------------------------------------------------------
# Edge cases and consistency
# ---------------------------------------------------------------------------

def test_zero_length_copies_state():
    S0 = dev(np.random.default_rng(3).standard_normal((2, 2, 64, 64)))
    q = torch.empty((2, 2, 0, 64), device="cuda")
    v = torch.empty((2, 2, 0, 64), device="cuda")
    o, ST = gdn.chunk_fwd(q, q, v, torch.empty((2, 2, 0), device="cuda"), torch.empty((2, 2, 0), device="cuda"),
                          S0, update="delta", gate="scalar")
    torch.cuda.synchronize()
    assert torch.equal(ST, S0) and o.numel() == 0


@pytest.mark.parametrize("algo", ["simt", "auto"])
def test_state_in_place_and_null_state(algo):
    w = small_workload("delta", "scalar", "bf16", T=150)
    x = make_prefill_inputs(w)
    dt = io_dtype(w)
    args = [dev(x["q"], dt), dev(x["k"], dt), dev(x["v"], dt), dev(x["g"]), dev(x["beta"])]
    S = dev(x["S0"])
    o1, ST1 = gdn.chunk_fwd(*args, S.clone(), update="delta", gate="scalar", algo=algo)
    o2, ST2 = gdn.chunk_fwd(*args, S, update="delta", gate="scalar", S_T=S, algo=algo)   # S_T aliases S0
    o3, _ = gdn.chunk_fwd(*args, S0=None, update="delta", gate="scalar", return_state=False, algo=algo)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(ST1, S)
    x0 = dict(x, S0=None)
    ro, _ = oracle.gdn_forward("delta", "scalar", x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"])
    assert rel_err(np64(o3), ro) <= TOL["bf16"]


def test_split_sequence_equals_whole():
    w = small_workload("delta", "channel", "f32", T=300)
    x = make_prefill_inputs(w)
    o, ST = run_prefill(w, x, algo="simt")
    cut = 137
    xa = {k_: (None if v_ is None else (v_[:, :, :cut] if k_ != "S0" else v_)) for k_, v_ in x.items()}
    oa, Sa = run_prefill(w.with_(T=cut), xa, algo="simt")
    xb = {k_: (None if v_ is None else v_[:, :, cut:]) for k_, v_ in x.items() if k_ != "S0"}
    ob, Sb = run_prefill(w.with_(T=300 - cut), dict(xb, S0=None), algo="simt", S0_dev=Sa)
    assert rel_err(np64(torch.cat([oa, ob], dim=2)), np64(o)) < 1e-5
    assert rel_err(np64(Sb), np64(ST)) < 1e-5


def test_prefill_equals_decode_chain():
    w = small_workload("delta", "scalar", "f32", T=70, B=1, H=2, dk=64, dv=64)
    x = make_prefill_inputs(w)
    o, ST = run_prefill(w, x, algo="simt")
    S = dev(x["S0"])
    outs = []
    for t in range(70):
        sl = lambda a: dev(a[:, :, t:t + 1])
        outs.append(gdn.decode_step(sl(x["q"]), sl(x["k"]), sl(x["v"]), dev(x["g"][:, :, t:t + 1]),
                                    dev(x["beta"][:, :, t:t + 1]), S, update="delta", gate="scalar"))
    od = torch.cat(outs, dim=2)
    torch.cuda.synchronize()
    assert rel_err(np64(od), np64(o)) < 1e-5 and rel_err(np64(S), np64(ST)) < 1e-5


def test_bf16_output_is_rounded_fp32_output():
    w = small_workload("delta", "scalar", "bf16", T=130)
    x = make_prefill_inputs(w)
    o32, _ = run_prefill(w, x, algo="simt")
    o16, _ = run_prefill(w, x, algo="simt", out_dtype=torch.bfloat16)
    assert torch.equal(o32.to(torch.bfloat16), o16)


def test_nan_propagates_without_fault():
    w = small_workload("delta", "scalar", "f32", T=100, B=1, H=1)
    x = make_prefill_inputs(w)
    x["v"][0, 0, 10, 3] = np.nan
    o, ST = run_prefill(w, x, algo="simt")
    on = np64(o)
    assert np.isnan(on[0, 0, 10:]).any() and not np.isnan(on[0, 0, :10]).any()


def test_decode_steps_replayed_from_a_cuda_graph_equal_eager_steps():
    """The library's calls can be captured in a CUDA graph (no synchronisation,
    allocation or host read inside them): 12 single-token steps and 3 calls of
    4 tokens, replayed, give the eager results bit for bit."""
    w = small_workload("delta", "scalar", "bf16", T=1, dk=128, dv=128, B=2, H=4).with_(steps=12, q_map="none")
    steps = make_decode_inputs(w, 12)
    S0 = np.random.default_rng(6).standard_normal((2, 4, 128, 128)).astype(np.float32) * 0.05
    dsteps = [{k_: (None if v_ is None else dev(v_, torch.bfloat16 if k_ in ("q", "k", "v") else torch.float32))
               for k_, v_ in s_.items()} for s_ in steps]
    multi = [{k_: (None if v_ is None else dev(v_, torch.bfloat16 if k_ in ("q", "k", "v") else torch.float32))
              for k_, v_ in _stack_steps(steps[4 * c:4 * c + 4]).items()} for c in range(3)]
    o1 = torch.empty((2, 4, 1, 128), device="cuda")
    o4 = torch.empty((2, 4, 4, 128), device="cuda")

    def run(S, outs1, outs4):
        for i, d in enumerate(dsteps):
            gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, update="delta", gate="scalar", o=o1)
            outs1[i].copy_(o1)
        for c, d in enumerate(multi):
            gdn.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, update="delta", gate="scalar", o=o4)
            outs4[c].copy_(o4)

    S_e = dev(S0)
    e1 = [torch.empty_like(o1) for _ in dsteps]
    e4 = [torch.empty_like(o4) for _ in multi]
    run(S_e, e1, e4)
    S_g = dev(S0)
    g1 = [torch.empty_like(o1) for _ in dsteps]
    g4 = [torch.empty_like(o4) for _ in multi]
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        run(S_g, g1, g4)
    S_g.copy_(dev(S0))
    graph.replay()
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(S_g, S_e)
    assert all(torch.equal(a, b) for a, b in zip(g1, e1)) and all(torch.equal(a, b) for a, b in zip(g4, e4))
