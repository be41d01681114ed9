"""Oracle for the causal gated delta-rule recurrence (float64, CPU).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product package
``gated_delta_rule_97_b200`` never does, and this package never imports it.

Two implementations of the same definition:

* ``gdn_forward`` -- the C recurrence in ``gdn_oracle.c`` (float64, OpenMP
  over heads), for every size the tests and the benchmark use;
* ``gdn_forward_np`` -- the same three steps written with NumPy, vectorised
  over heads, for small cases and to cross-check the compiled one;
* ``gdp_forward`` -- Gated DeltaProduct (n_h delta substeps per token), NumPy;
* ``prologue`` -- the optional input maps (feature map, L2 rows, sigmoid,
  -softplus) applied before the recurrence;
* ``segment_maps`` -- the affine map (H, Lambda) of a run of tokens, Lambda as
  the dense product of the per-token transition matrices;
* ``gdn_backward_np`` -- the gradients of the recurrence (reverse mode through
  the token loop, states recomputed from chunk-start checkpoints).

Definition (column convention, S in R^{dv x dk}, stored [B,H,dv,dk]):
``S_t = S_{t-1} Diag(alpha_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T``,
``o_t = S_t q_t``, alpha_t = exp(g_t).  Expanded: decay the columns of S by
alpha_t, then write (``v k^T`` in the additive/decay modes; ``u k^T`` with
``u = beta (v - S k)`` in the delta mode), then read ``o = S q``.
Sources ("Linear Attention, Visualized"): "Naive linear attention",
"Mamba-2: input-dependent scalar decay", "DeltaNet" / "Recurrent form",
"Gated DeltaNet (GDN)", "Gated Linear Attention (GLA)",
"Kimi Delta Attention (KDA)".

Pins (tests/test_oracle_pins.py) tie this definition to closed forms,
invariants and brute-force constructions that do not reuse it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

UPDATE_IDS = {"additive": 0, "decay": 1, "delta": 2}
GATE_IDS = {"none": 0, "scalar": 1, "channel": 2}

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_gdn_forward.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_long, ctypes.c_long,
                                           ctypes.c_long, ctypes.c_long, dp, dp, dp, dp, dp, dp, dp, dp]
        lib.oracle_gdn_forward.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the C oracle's OpenMP region uses."""
    return int(_load().oracle_num_threads())


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return ctypes.cast(None, ctypes.POINTER(ctypes.c_double))
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(update, gate, q, k, v, g, beta):
    if update not in UPDATE_IDS or gate not in GATE_IDS:
        raise ValueError("bad mode")
    if update == "delta" and beta is None:
        raise ValueError("delta mode needs beta")
    if (gate != "none") != (g is not None):
        raise ValueError("g must be given iff gate != 'none'")
    if q.shape[:-1] != k.shape[:-1] or q.shape[-1] != k.shape[-1] or v.shape[:-1] != q.shape[:-1]:
        raise ValueError("shape mismatch")
    # the gate is one value per token (scalar) or one per token and key channel;
    # beta one per token: a tensor laid out along another axis is an error here,
    # not a silently different recurrence
    if g is not None:
        want = q.shape[:-1] if gate == "scalar" else q.shape
        if np.shape(g) != tuple(want):
            raise ValueError("g has shape %s, expected %s" % (np.shape(g), tuple(want)))
    if beta is not None and np.shape(beta) != tuple(q.shape[:-1]):
        raise ValueError("beta has shape %s, expected %s" % (np.shape(beta), tuple(q.shape[:-1])))


def gdn_forward(update, gate, q, k, v, g=None, beta=None, S0=None):
    """Recurrence over T tokens for every head (C, float64).

    q, k: [..., T, dk]; v: [..., T, dv]; g: [..., T] (scalar) or [..., T, dk]
    (channel) or None; beta: [..., T] or None; S0: [..., dv, dk] or None.
    Returns (o [..., T, dv], S_T [..., dv, dk]) as float64.
    """
    _check(update, gate, q, k, v, g, beta)
    lead = q.shape[:-2]
    T, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    qd, kd, vd = _f64(q), _f64(k), _f64(v)
    gd, bd, sd = _f64(g), _f64(beta), _f64(S0)
    o = np.empty(lead + (T, dv), np.float64)
    ST = np.empty(lead + (dv, dk), np.float64)
    rc = _load().oracle_gdn_forward(UPDATE_IDS[update], GATE_IDS[gate], BH, T, dk, dv,
                                    _ptr(qd), _ptr(kd), _ptr(vd), _ptr(gd), _ptr(bd), _ptr(sd),
                                    _ptr(o), _ptr(ST))
    if rc != 0:
        raise RuntimeError("oracle_gdn_forward failed: %d" % rc)
    return o, ST


def gdn_forward_np(update, gate, q, k, v, g=None, beta=None, S0=None):
    """The same recurrence with NumPy (vectorised over heads; loops over t)."""
    _check(update, gate, q, k, v, g, beta)
    q, k, v = _f64(q), _f64(k), _f64(v)
    g, beta = _f64(g), _f64(beta)
    lead = q.shape[:-2]
    T, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    S = np.zeros(lead + (dv, dk)) if S0 is None else _f64(S0).copy()
    o = np.empty(lead + (T, dv))
    for t in range(T):
        if gate == "scalar":
            S = S * np.exp(g[..., t])[..., None, None]
        elif gate == "channel":
            S = S * np.exp(g[..., t, :])[..., None, :]
        kt = k[..., t, :]
        if update == "delta":
            pred = np.einsum("...ij,...j->...i", S, kt)
            u = beta[..., t][..., None] * (v[..., t, :] - pred)
        else:
            u = v[..., t, :]
        S = S + u[..., :, None] * kt[..., None, :]
        o[..., t, :] = np.einsum("...ij,...j->...i", S, q[..., t, :])
    return o, S


def gdp_forward(gate, q, k, v, g=None, beta=None, S0=None):
    """Gated DeltaProduct, token by token ("Linear Attention, Visualized",
    "Gated Delta Product (GDP)"): for each real token t the state decays once by
    a_t = exp(g_t), then takes n_h delta-rule substeps j = 1..n_h, each with its
    own key k_{t,j}, value v_{t,j} and write strength beta_{t,j}, and only then
    is read, o_t = S q_t.

    q [...,T,dk]; k [...,T,nh,dk]; v [...,T,nh,dv]; beta [...,T,nh];
    g [...,T] (scalar) or [...,T,dk] (channel) or None.  Returns (o, S_T).
    """
    q, k, v, g, beta = _f64(q), _f64(k), _f64(v), _f64(g), _f64(beta)
    lead = q.shape[:-2]
    T, dk = q.shape[-2], q.shape[-1]
    nh, dv = k.shape[-2], v.shape[-1]
    if (gate == "none") != (g is None) or beta is None:
        raise ValueError("gate / g mismatch or missing beta")
    S = np.zeros(lead + (dv, dk)) if S0 is None else _f64(S0).copy()
    o = np.empty(lead + (T, dv))
    for t in range(T):
        if gate == "scalar":
            S = S * np.exp(g[..., t])[..., None, None]
        elif gate == "channel":
            S = S * np.exp(g[..., t, :])[..., None, :]
        for j in range(nh):
            kj = k[..., t, j, :]
            pred = np.einsum("...ij,...j->...i", S, kj)
            u = beta[..., t, j][..., None] * (v[..., t, j, :] - pred)
            S = S + u[..., :, None] * kj[..., None, :]
        o[..., t, :] = np.einsum("...ij,...j->...i", S, q[..., t, :])
    return o, S


def segment_maps(update, gate, k, v, g=None, beta=None):
    """The affine map of a run of tokens ("Linear Attention, Visualized", "One
    chunk as an affine recurrence" and "Update the state"): for any incoming
    state, S_out = S_in Lam + H.

    H [..., dv, dk] is the recurrence from the zero state (``gdn_forward`` with
    S0 = 0).  Lam [..., dk, dk] is the ordered product of the tokens' transition
    matrices, formed densely one token at a time: M_t = Diag(alpha_t)
    (I - beta_t k_t k_t^T) for the delta write, Diag(alpha_t) for the decay
    write, I for the additive write (alpha_t = exp(g_t), a scalar or one per key
    channel).  Returns (H, Lam) as float64.
    """
    _check(update, gate, k, k, v, g, beta)
    k, g, beta = _f64(k), _f64(g), _f64(beta)
    lead = k.shape[:-2]
    T, dk = k.shape[-2], k.shape[-1]
    _, H = gdn_forward(update, gate, np.zeros_like(k), k, v, g=g, beta=beta)
    eye = np.eye(dk)
    Lam = np.broadcast_to(eye, lead + (dk, dk)).copy()
    for t in range(T):
        if gate == "scalar":
            D = np.exp(g[..., t])[..., None, None] * eye
        elif gate == "channel":
            D = np.exp(g[..., t, :])[..., None, :] * eye
        else:
            D = np.broadcast_to(eye, lead + (dk, dk))
        if update == "delta":
            kt = k[..., t, :]
            P = eye - beta[..., t][..., None, None] * (kt[..., :, None] * kt[..., None, :])
            M = D @ P
        else:
            M = D
        Lam = Lam @ M
    return H, Lam


PRO_QK_ELU1, PRO_QK_L2, PRO_BETA_SIGMOID, PRO_G_NEG_SOFTPLUS = 1, 2, 4, 8


def prologue(flags, q=None, k=None, beta=None, g=None):
    """The input maps of the prologue bits, in float64, applied before the
    recurrence: q, k <- elu(x) + 1 ("Linear attention: a running sum"); q, k rows
    <- x / |x|_2, a zero row kept zero (the DeltaNet forward's normalised q, k);
    beta <- sigmoid(beta); g <- -softplus(g) ("Optional: Constructing the decay
    gate").  Returns (q, k, beta, g)."""
    def feat(x):
        if x is None:
            return None
        x = _f64(x)
        if flags & PRO_QK_ELU1:
            x = np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
        if flags & PRO_QK_L2:
            n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
            x = np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)
        return x
    q, k = feat(q), feat(k)
    beta, g = _f64(beta), _f64(g)
    if beta is not None and flags & PRO_BETA_SIGMOID:
        beta = 1.0 / (1.0 + np.exp(-beta))
    if g is not None and flags & PRO_G_NEG_SOFTPLUS:
        g = -(np.maximum(g, 0.0) + np.log1p(np.exp(-np.abs(g))))
    return q, k, beta, g


def decode_sequence(update, gate, S0, steps):
    """Oracle for ``len(steps)`` consecutive decode steps on the same state.

    ``steps`` is a list of dicts with q,k [..., 1, d], v [..., 1, dv], beta
    [..., 1], g [..., 1] or [..., 1, dk].  Consecutive single-token steps are
    the recurrence over the stacked sequence, so this stacks them along T.
    Returns (o [..., n_steps, dv], S_final).
    """
    def cat(name):
        if steps[0].get(name) is None:
            return None
        return np.concatenate([np.asarray(s[name], dtype=np.float64) for s in steps],
                              axis=-2 if name in ("q", "k", "v") or (name == "g" and gate == "channel") else -1)

    return gdn_forward(update, gate, cat("q"), cat("k"), cat("v"), cat("g"), cat("beta"), S0)


def gdn_backward_np(update, gate, q, k, v, g=None, beta=None, S0=None, dO=None, dS_T=None, checkpoint=64):
    """Gradients of the recurrence (reverse mode through the token loop), float64.

    For the scalar loss L = sum(dO * o) + sum(dS_T * S_T) of ``gdn_forward``
    (dO [..., T, dv] and dS_T [..., dv, dk] are the upstream gradients; either
    may be None = 0), returns (dq, dk, dv, dg, dbeta, dS0) shaped like q, k, v,
    g, beta, S0 (dg / dbeta None when g / beta are None; dS0 always returned).

    Each token's step is differentiated as written in ``gdn_forward_np``:
    S' = S_{t-1} Diag(alpha_t); delta: r = v_t - S' k_t, u = beta_t r, else
    u = v_t; S_t = S' + u k_t^T; o_t = S_t q_t.  Going back from t = T-1 with
    dS = dL/dS_t: dq_t = S_t^T dO_t; dS += dO_t q_t^T; du = dS k_t;
    dk_t = dS^T u; dS' = dS; delta: dbeta_t = du . r, dv_t = beta_t du,
    dS' -= dv_t k_t^T, dk_t -= S'^T dv_t; else dv_t = du; the gate:
    dg_t = sum(dS' * S') (over the key channel j alone for a per-channel gate,
    since S'[:, j] = alpha_j S[:, j] and d alpha / d g = alpha); then
    dL/dS_{t-1} = dS' Diag(alpha_t).  The states S' are recomputed a chunk of
    ``checkpoint`` tokens at a time from the states saved at chunk starts
    ("Update the state": autograd keeps the chunk-boundary states)."""
    _check(update, gate, q, k, v, g, beta)
    q, k, v, g, beta = _f64(q), _f64(k), _f64(v), _f64(g), _f64(beta)
    lead = q.shape[:-2]
    T, dk_ = q.shape[-2], q.shape[-1]
    dv_ = v.shape[-1]
    S = np.zeros(lead + (dv_, dk_)) if S0 is None else _f64(S0).copy()
    dO = np.zeros(lead + (T, dv_)) if dO is None else _f64(dO)

    def alpha(t):
        if gate == "scalar":
            return np.exp(g[..., t])[..., None, None]
        if gate == "channel":
            return np.exp(g[..., t, :])[..., None, :]
        return None

    def step(S, t):
        """One token forward: returns (S', r or None, u, S_t)."""
        a = alpha(t)
        Sp = S * a if a is not None else S
        kt = k[..., t, :]
        if update == "delta":
            r = v[..., t, :] - np.einsum("...ij,...j->...i", Sp, kt)
            u = beta[..., t][..., None] * r
        else:
            r, u = None, v[..., t, :]
        return Sp, r, u, Sp + u[..., :, None] * kt[..., None, :]

    # forward: the state entering every chunk
    starts = []
    for t in range(T):
        if t % checkpoint == 0:
            starts.append(S.copy())
        S = step(S, t)[3]
    dS = np.zeros(lead + (dv_, dk_)) if dS_T is None else _f64(dS_T).copy()
    dq, dk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg = None if g is None else np.zeros_like(g)
    db = None if beta is None else np.zeros_like(beta)
    for c in range(len(starts) - 1, -1, -1):
        t0, t1 = c * checkpoint, min(T, (c + 1) * checkpoint)
        S = starts[c].copy()
        saved = []
        for t in range(t0, t1):
            Sp, r, u, S = step(S, t)
            saved.append((Sp, r, u, S))
        for t in range(t1 - 1, t0 - 1, -1):
            Sp, r, u, St = saved[t - t0]
            qt, kt, dOt = q[..., t, :], k[..., t, :], dO[..., t, :]
            dq[..., t, :] = np.einsum("...ij,...i->...j", St, dOt)
            dS = dS + dOt[..., :, None] * qt[..., None, :]
            du = np.einsum("...ij,...j->...i", dS, kt)
            dk[..., t, :] = np.einsum("...ij,...i->...j", dS, u)
            dSp = dS
            if update == "delta":
                db[..., t] = np.sum(du * r, axis=-1)
                dvt = beta[..., t][..., None] * du
                dvv[..., t, :] = dvt
                dSp = dSp - dvt[..., :, None] * kt[..., None, :]
                dk[..., t, :] -= np.einsum("...ij,...i->...j", Sp, dvt)
            else:
                dvv[..., t, :] = du
            a = alpha(t)
            if gate == "scalar":
                dg[..., t] = np.sum(dSp * Sp, axis=(-2, -1))
            elif gate == "channel":
                dg[..., t, :] = np.sum(dSp * Sp, axis=-2)
            dS = dSp * a if a is not None else dSp
    return dq, dk, dvv, dg, db, dS


def gdn_backward_prologue_np(update, gate, flags, q, k, v, g=None, beta=None, S0=None, dO=None, dS_T=None):
    """Gradients of the recurrence with the input prologue ``flags`` (the maps
    of ``prologue``) in front of it, with respect to the raw inputs, float64.

    The maps are applied, ``gdn_backward_np`` runs on the mapped inputs, and the
    chain rule takes each gradient back through its map:
      unit rows y = e / |e| (|e| > 0):  de = (dy - y (y . dy)) / |e|; zero row: 0
      elu(x) + 1:                       dx = de where x > 0, de e^x elsewhere
      beta = sigmoid(b):                db = dbeta sigmoid(b) (1 - sigmoid(b))
      g = -softplus(x):                 dx = -dg sigmoid(x)
    Returns (dq, dk, dv, dg, dbeta, dS0) shaped like the raw inputs."""
    qm, km, bm, gm = prologue(flags, q=q, k=k, beta=beta, g=g)
    dqm, dkm, dv, dgm, dbm, dS0 = gdn_backward_np(update, gate, qm, km, v, gm, bm, S0, dO, dS_T)

    def back_feat(x, dy):
        x = _f64(x)
        e = np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0))) if flags & PRO_QK_ELU1 else x
        de = dy
        if flags & PRO_QK_L2:
            n = np.sqrt(np.sum(e * e, axis=-1, keepdims=True))
            safe = np.where(n > 0, n, 1.0)
            y = e / safe
            de = np.where(n > 0, (dy - y * np.sum(y * dy, axis=-1, keepdims=True)) / safe, 0.0)
        if flags & PRO_QK_ELU1:
            de = np.where(x > 0, de, de * np.exp(np.minimum(x, 0.0)))
        return de

    dq, dk = back_feat(q, dqm), back_feat(k, dkm)
    dbeta, dg = dbm, dgm
    if dbm is not None and flags & PRO_BETA_SIGMOID:
        sb = 1.0 / (1.0 + np.exp(-_f64(beta)))
        dbeta = dbm * sb * (1.0 - sb)
    if dgm is not None and flags & PRO_G_NEG_SOFTPLUS:
        dg = -dgm / (1.0 + np.exp(-_f64(g)))
    return dq, dk, dv, dg, dbeta, dS0
