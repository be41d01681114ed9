"""Seeded synthetic inputs for the gated delta-rule hot path.

This module is the ONLY code shared by the oracle side (``oracle/``) and the
CUDA side (``gated_delta_rule_97_b200``).  It draws random tensors with the
shapes and value distributions of the five workloads, applies the input feature
maps that those workloads prescribe (L2 normalisation, elu+1, sigmoid,
-softplus) and rounds q, k, v to the run dtype.  It contains none of the
recurrence's arithmetic.

Streams.  Every tensor of every (b, h) head comes from its own NumPy PCG64
stream keyed by ``(seed, tensor_id, b, h)``; decode inputs of step ``s`` come
from a stream keyed by ``(seed, tensor_id, 1_000_000 + s)``.  A head can
therefore be regenerated alone (full-size parity checks on sampled heads) and
the result does not depend on how many threads draw it.

bf16.  q, k and v of bf16 workloads are rounded from float32 with
round-to-nearest-even and handed to both sides as the exact bf16 values
(the oracle upcasts them to float64).
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# --------------------------------------------------------------------------
# bf16 helpers (pure bit manipulation; no recurrence arithmetic)
# --------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 with round-to-nearest-even; returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded[nan] = 0x7FC0
    return rounded


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits (uint16) to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 array holding the nearest bf16 values (RNE)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# --------------------------------------------------------------------------
# Workload descriptions
# --------------------------------------------------------------------------

UPDATES = ("additive", "decay", "delta")
GATES = ("none", "scalar", "channel")
DTYPES = ("f32", "bf16")


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, mode and input distribution of one synthetic workload."""

    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    update: str  # additive | decay | delta
    gate: str  # none | scalar | channel
    dtype: str  # f32 | bf16  (dtype of q, k, v, o; g, beta, S are fp32)
    q_map: str  # l2 | elu1 | none
    k_map: str  # l2 | elu1
    gate_dist: tuple | None  # ("uniform", lo, hi) | ("neg_softplus", mu, sigma)
    s0_std: float  # 0 -> S0 = 0 (passed as NULL)
    seed: int
    steps: int = 0  # >0: decode workload with this many consecutive steps
    chunk: int = 64

    @property
    def n_heads(self) -> int:
        return self.B * self.H

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads (shapes and distributions as specified for this path).
WORKLOADS = {
    "tiny_gdn_f32": Workload(
        "tiny_gdn_f32", B=1, H=2, T=256, dk=64, dv=64, update="delta", gate="scalar",
        dtype="f32", q_map="l2", k_map="l2", gate_dist=("uniform", -0.05, 0.0),
        s0_std=0.0, seed=0),
    "linear_attn_bf16": Workload(
        "linear_attn_bf16", B=4, H=16, T=4096, dk=128, dv=128, update="additive",
        gate="none", dtype="bf16", q_map="elu1", k_map="elu1", gate_dist=None,
        s0_std=0.0, seed=1),
    "gdn_prefill_bf16": Workload(
        "gdn_prefill_bf16", B=8, H=16, T=8192, dk=128, dv=128, update="delta",
        gate="scalar", dtype="bf16", q_map="l2", k_map="l2",
        gate_dist=("neg_softplus", -3.0, 1.0), s0_std=0.02, seed=2),
    "kda_prefill_bf16": Workload(
        "kda_prefill_bf16", B=2, H=32, T=32768, dk=128, dv=128, update="delta",
        gate="channel", dtype="bf16", q_map="l2", k_map="l2",
        gate_dist=("neg_softplus", -4.0, 1.0), s0_std=0.0, seed=3),
    "decode_gdn_bf16": Workload(
        "decode_gdn_bf16", B=256, H=32, T=1, dk=128, dv=128, update="delta",
        gate="scalar", dtype="bf16", q_map="none", k_map="l2",
        gate_dist=("uniform", -0.05, 0.0), s0_std=0.02, seed=4, steps=1000),
}

_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "beta": 4, "g": 5, "S0": 6}
_DECODE_STEP_BASE = 1_000_000


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _feature(x: np.ndarray, kind: str) -> np.ndarray:
    """Input feature maps named by the workloads (applied in float32)."""
    if kind == "none":
        return x
    if kind == "l2":
        n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
        return (x / np.maximum(n, 1e-30)).astype(np.float32)
    if kind == "elu1":
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0))).astype(np.float32)
    raise ValueError(kind)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _neg_softplus(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    sp = np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))
    return (-sp).astype(np.float32)


def _draw_gate(rng: np.random.Generator, shape, dist) -> np.ndarray:
    kind = dist[0]
    if kind == "uniform":
        return rng.uniform(dist[1], dist[2], size=shape).astype(np.float32)
    if kind == "neg_softplus":
        x = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(dist[2]) + np.float32(dist[1])
        return _neg_softplus(x)
    raise ValueError(kind)


def _round_io(x: np.ndarray, dtype: str) -> np.ndarray:
    return round_to_bf16(x) if dtype == "bf16" else x.astype(np.float32)


def _head_block(w: Workload, b: int, h: int, T: int, key_extra: tuple = ()) -> dict:
    """Inputs of one (b, h) head: q,k [T,dk], v [T,dv], beta [T], g [T] | [T,dk]."""
    key = (w.seed,) + key_extra
    out = {}
    r = _rng(*key, _TENSOR_IDS["q"], b, h)
    out["q"] = _round_io(_feature(r.standard_normal((T, w.dk), dtype=np.float32), w.q_map), w.dtype)
    r = _rng(*key, _TENSOR_IDS["k"], b, h)
    out["k"] = _round_io(_feature(r.standard_normal((T, w.dk), dtype=np.float32), w.k_map), w.dtype)
    r = _rng(*key, _TENSOR_IDS["v"], b, h)
    out["v"] = _round_io(r.standard_normal((T, w.dv), dtype=np.float32), w.dtype)
    if w.update == "delta":
        r = _rng(*key, _TENSOR_IDS["beta"], b, h)
        out["beta"] = _sigmoid(r.standard_normal(T, dtype=np.float32))
    if w.gate != "none":
        r = _rng(*key, _TENSOR_IDS["g"], b, h)
        shape = (T,) if w.gate == "scalar" else (T, w.dk)
        out["g"] = _draw_gate(r, shape, w.gate_dist)
    return out


def _threads() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    return max(1, min(16, n))


def make_prefill_inputs(w: Workload, heads=None) -> dict:
    """All prefill inputs of workload ``w`` as float32 numpy arrays.

    Layouts: q,k [B,H,T,dk]; v [B,H,T,dv]; beta [B,H,T]; g [B,H,T] (scalar) or
    [B,H,T,dk] (channel); S0 [B,H,dv,dk] or None.  q, k, v hold exact bf16 values
    when ``w.dtype == 'bf16'``.  With ``heads`` (a list of (b, h)), only those
    heads are drawn and arrays are shaped [len(heads),1,...] in that order.
    """
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        shape_bh = (w.B, w.H)
    else:
        heads = [tuple(x) for x in heads]
        shape_bh = (len(heads), 1)
    n = len(heads)
    T = w.T
    q = np.empty((n, T, w.dk), np.float32)
    k = np.empty((n, T, w.dk), np.float32)
    v = np.empty((n, T, w.dv), np.float32)
    beta = np.empty((n, T), np.float32) if w.update == "delta" else None
    g = None
    if w.gate == "scalar":
        g = np.empty((n, T), np.float32)
    elif w.gate == "channel":
        g = np.empty((n, T, w.dk), np.float32)
    S0 = np.empty((n, w.dv, w.dk), np.float32) if w.s0_std > 0 else None

    def fill(i):
        b, h = heads[i]
        blk = _head_block(w, b, h, T)
        q[i], k[i], v[i] = blk["q"], blk["k"], blk["v"]
        if beta is not None:
            beta[i] = blk["beta"]
        if g is not None:
            g[i] = blk["g"]
        if S0 is not None:
            r = _rng(w.seed, _TENSOR_IDS["S0"], b, h)
            S0[i] = r.standard_normal((w.dv, w.dk), dtype=np.float32) * np.float32(w.s0_std)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(n)))

    def rs(a):
        return None if a is None else a.reshape(shape_bh + a.shape[1:])

    return {"q": rs(q), "k": rs(k), "v": rs(v), "beta": rs(beta), "g": rs(g), "S0": rs(S0)}


def make_product_inputs(w: Workload, nh: int, heads=None) -> dict:
    """Inputs of a Gated DeltaProduct run with ``nh`` substeps per token.

    q [B,H,T,dk] and g ([B,H,T] or [B,H,T,dk]) per real token (the streams of
    ``make_prefill_inputs``); k [B,H,T,nh,dk], v [B,H,T,nh,dv] and beta
    [B,H,T,nh] per substep, drawn as one sequence of T*nh positions from streams
    keyed additionally by nh; S0 as in ``make_prefill_inputs``.
    """
    base = make_prefill_inputs(w, heads)
    wv = w.with_(T=w.T * nh, seed=w.seed + 7919 * nh)
    sub = make_prefill_inputs(wv, heads)
    lead = base["q"].shape[:2]
    out = {"q": base["q"], "g": base["g"], "S0": base["S0"]}
    out["k"] = sub["k"].reshape(lead + (w.T, nh, w.dk))
    out["v"] = sub["v"].reshape(lead + (w.T, nh, w.dv))
    out["beta"] = None if sub["beta"] is None else sub["beta"].reshape(lead + (w.T, nh))
    return out


def make_decode_state(w: Workload, heads=None) -> np.ndarray:
    """Initial decode state S [B,H,dv,dk] float32 (or [n,1,dv,dk] for ``heads``)."""
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        shape_bh = (w.B, w.H)
    else:
        shape_bh = (len(heads), 1)
    S = np.empty((len(heads), w.dv, w.dk), np.float32)

    def fill(i):
        b, h = heads[i]
        r = _rng(w.seed, _TENSOR_IDS["S0"], b, h)
        S[i] = r.standard_normal((w.dv, w.dk), dtype=np.float32) * np.float32(w.s0_std)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(len(heads))))
    return S.reshape(shape_bh + (w.dv, w.dk))


def make_decode_step_inputs(w: Workload, step: int) -> dict:
    """Inputs of decode step ``step`` for all heads: q,k [B,H,1,dk], v [B,H,1,dv],
    beta [B,H,1], g [B,H,1] or [B,H,1,dk]."""
    blk = _head_block(w.with_(T=w.B * w.H), 0, 0, w.B * w.H, key_extra=(_DECODE_STEP_BASE + step,))
    out = {}
    for name in ("q", "k", "v"):
        a = blk[name]
        out[name] = a.reshape(w.B, w.H, 1, a.shape[-1])
    out["beta"] = blk["beta"].reshape(w.B, w.H, 1) if "beta" in blk else None
    if "g" in blk:
        out["g"] = blk["g"].reshape((w.B, w.H, 1) + blk["g"].shape[1:])
    else:
        out["g"] = None
    return out


def make_decode_inputs(w: Workload, steps: int | None = None) -> list:
    """Per-step decode inputs for ``steps`` consecutive steps (default w.steps)."""
    steps = w.steps if steps is None else steps
    with ThreadPoolExecutor(_threads()) as ex:
        return list(ex.map(lambda s: make_decode_step_inputs(w, s), range(steps)))


def orthonormal_keys(d: int, n: int, seed: int) -> np.ndarray:
    """n rows of a random orthonormal basis of R^d (n <= d), float64 (QR of a Gaussian)."""
    r = _rng(seed, 99)
    a = r.standard_normal((d, d))
    qm, _ = np.linalg.qr(a)
    return qm[:, :n].T.copy()


def iter_decode_blocks(w: Workload, steps: int | None = None, block: int = 32):
    """Yields (first_step, [inputs of steps first_step .. first_step+block-1]),
    drawing one block at a time so host memory stays bounded."""
    steps = w.steps if steps is None else steps
    with ThreadPoolExecutor(_threads()) as ex:
        for s0 in range(0, steps, block):
            n = min(block, steps - s0)
            yield s0, list(ex.map(lambda s: make_decode_step_inputs(w, s), range(s0, s0 + n)))
