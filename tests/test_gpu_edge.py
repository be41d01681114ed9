"""GPU parity on the method's own edge cases, through the tensor-core and the
SIMT prefill kernels, against the float64 oracle.

The cases are the invariants "Linear Attention, Visualized" fixes for the delta
rule and the gates:

* "DeltaNet: correcting memory collisions", "An intuitive example": with
  beta = 1 and orthonormal unit keys a read at a key returns the most recent
  value written there;
* beta = 0 with alpha = 1 leaves the state at S0, so o_t = S0 q_t;
* one key written 8 times in a row inside a chunk with beta = 1: the strictly
  lower block of (I + L) is all ones there, the hardest case for the
  triangular solve (its inverse alternates along the first sub-diagonal);
* "Mamba-2: input-dependent scalar decay", "Chunkwise form": a scalar gate of
  about -2 per token, 128 nats over a chunk, beyond the range in which the
  chunk's decay ratios b_l / b_m are formed from a product of two exponentials;
* "Kimi Delta Attention (KDA)": a per-channel gate with alpha = 1 on half the
  key channels and log alpha = -3 on the rest.

Inputs are built so that the bf16 values the kernels read are exactly the ones
the statements above are about (keys from a Hadamard matrix of order 64 scaled
by 1/8 are exactly orthonormal in bf16).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_97_b200 as gdn
import oracle
from gpu_util import TOL, dev, np64, rel_err
from synth import round_to_bf16

pytestmark = pytest.mark.gpu

ALGOS = [("tc", 64), ("tc", 128), ("simt", 64), ("simt", 128)]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.build()
    oracle.build()
    gdn.device_status(clear=True)


def hadamard_keys(dk, seed):
    """dk orthonormal rows, exact in bf16: Sylvester-Hadamard rows of order 64
    times 1/8 in one 64-channel half of the key, zeros in the other, rows
    permuted and signed at random."""
    h = np.array([[1.0]])
    while h.shape[0] < 64:
        h = np.block([[h, h], [h, -h]])
    rows = []
    for half in range(dk // 64):
        blk = np.zeros((64, dk))
        blk[:, 64 * half:64 * half + 64] = h / 8.0
        rows.append(blk)
    keys = np.concatenate(rows)
    r = np.random.default_rng(seed)
    keys = keys[r.permutation(dk)] * r.choice([-1.0, 1.0], size=(dk, 1))
    assert np.allclose(keys @ keys.T, np.eye(dk), atol=0)
    return keys


def bf16_vals(x):
    return round_to_bf16(np.asarray(x, np.float32)).astype(np.float64)


def run(algo, update, gate, q, k, v, g, beta, S0):
    """One prefill call on bf16 q, k, v; returns float64 (o, S_T) after checking
    the device status word."""
    gdn.device_status(clear=True)
    o, ST = gdn.chunk_fwd(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), dev(g),
                          dev(beta), dev(S0), update=update, gate=gate, algo=algo)
    torch.cuda.synchronize()
    assert gdn.device_status(clear=True) == 0
    return np64(o), np64(ST)


def parity(algo, update, gate, q, k, v, g, beta, S0):
    o, ST = run(algo, update, gate, q, k, v, g, beta, S0)
    ro, rS = oracle.gdn_forward(update, gate, q, k, v, g=g, beta=beta, S0=S0)
    eo, es = rel_err(o, ro), rel_err(ST, rS)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)
    return o, ST, ro, rS


@pytest.mark.parametrize("algo,dv", ALGOS)
def test_beta_one_orthonormal_keys_recall_latest_value(algo, dv):
    dk, T, BH = 128, 200, 2
    keys = hadamard_keys(dk, seed=5)
    r = np.random.default_rng(21)
    widx = r.integers(0, 24, (BH, T))
    ridx = r.integers(0, 24, (BH, T))
    k = keys[widx].reshape(1, BH, T, dk)
    q = keys[ridx].reshape(1, BH, T, dk)
    v = bf16_vals(r.standard_normal((1, BH, T, dv)))
    beta = np.ones((1, BH, T))
    o, _, _, _ = parity(algo, "delta", "none", q, k, v, None, beta, None)
    # the read-back itself: the latest value written at the read key (zero if none yet)
    expect = np.zeros_like(o)
    for h in range(BH):
        latest = {}
        for t in range(T):
            latest[widx[h, t]] = v[0, h, t]
            expect[0, h, t] = latest.get(ridx[h, t], 0.0)
    assert rel_err(o, expect) <= TOL["bf16"]


@pytest.mark.parametrize("algo,dv", ALGOS)
def test_beta_zero_keeps_the_initial_state(algo, dv):
    dk, T, BH = 128, 150, 2
    r = np.random.default_rng(22)
    q = bf16_vals(r.standard_normal((1, BH, T, dk)))
    k = r.standard_normal((1, BH, T, dk))
    k = bf16_vals(k / np.linalg.norm(k, axis=-1, keepdims=True))
    v = bf16_vals(r.standard_normal((1, BH, T, dv)))
    S0 = 0.05 * r.standard_normal((1, BH, dv, dk))
    o, ST, _, _ = parity(algo, "delta", "none", q, k, v, None, np.zeros((1, BH, T)), S0)
    assert rel_err(ST, S0) <= TOL["bf16"]
    assert rel_err(o, np.einsum("bhij,bhtj->bhti", S0, q)) <= TOL["bf16"]


@pytest.mark.parametrize("algo,dv", ALGOS)
@pytest.mark.parametrize("gate", ["none", "scalar"])
def test_one_key_repeated_inside_a_chunk(algo, dv, gate):
    dk, T, BH = 128, 140, 2
    r = np.random.default_rng(23)
    k = r.standard_normal((1, BH, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    for s in (10, 70, 131):  # 8 equal keys at tokens s..s+7 (the last run crosses no chunk edge)
        k[:, :, s:s + 8] = k[:, :, s:s + 1]
    k = bf16_vals(k)
    q = bf16_vals(r.standard_normal((1, BH, T, dk)))
    v = bf16_vals(r.standard_normal((1, BH, T, dv)))
    beta = np.full((1, BH, T), 0.6)
    for s in (10, 70, 131):
        beta[:, :, s:s + 8] = 1.0
    g = r.uniform(-0.05, 0.0, (1, BH, T)) if gate == "scalar" else None
    parity(algo, "delta", gate, q, k, v, g, beta, None)


@pytest.mark.parametrize("algo,dv", ALGOS)
@pytest.mark.parametrize("update", ["delta", "decay"])
def test_strong_scalar_decay_beyond_80_nats_per_chunk(algo, dv, update):
    dk, T, BH = 128, 190, 2
    r = np.random.default_rng(24)
    q = r.standard_normal((1, BH, T, dk))
    k = r.standard_normal((1, BH, T, dk))
    q = bf16_vals(q / np.linalg.norm(q, axis=-1, keepdims=True))
    k = bf16_vals(k / np.linalg.norm(k, axis=-1, keepdims=True))
    v = bf16_vals(r.standard_normal((1, BH, T, dv)))
    g = r.uniform(-2.2, -1.8, (1, BH, T))
    assert np.all(-g[..., :64].sum(-1) > 80.0)
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((1, BH, T)))) if update == "delta" else None
    S0 = 0.05 * r.standard_normal((1, BH, dv, dk))
    parity(algo, update, "scalar", q, k, v, g, beta, S0)


@pytest.mark.parametrize("algo,dv", ALGOS)
def test_channel_gate_half_open_half_strong(algo, dv):
    dk, T, BH = 128, 160, 2
    r = np.random.default_rng(25)
    q = r.standard_normal((1, BH, T, dk))
    k = r.standard_normal((1, BH, T, dk))
    q = bf16_vals(q / np.linalg.norm(q, axis=-1, keepdims=True))
    k = bf16_vals(k / np.linalg.norm(k, axis=-1, keepdims=True))
    v = bf16_vals(r.standard_normal((1, BH, T, dv)))
    g = np.zeros((1, BH, T, dk))
    strong = r.permutation(dk)[:dk // 2]
    g[..., strong] = -3.0
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((1, BH, T))))
    S0 = 0.05 * r.standard_normal((1, BH, dv, dk))
    parity(algo, "delta", "channel", q, k, v, g, beta, S0)
