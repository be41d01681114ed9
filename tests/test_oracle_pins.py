"""Pins for the float64 oracle: closed forms, invariants and brute force.

Each check below comes from something the pages fix ("Linear Attention,
Visualized" unless stated) and is computed without the oracle's token loop, so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them (``test_planted_mistakes_are_caught`` shows
this for a list of such mistakes, planted in a copy of the NumPy oracle).
"""
import json
import os

import numpy as np
import pytest
from scipy.linalg import solve_triangular

import oracle
from synth import orthonormal_keys

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-11


def rel_err(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(np.sqrt(np.mean(b * b)), 1e-300)
    return float(np.max(np.abs(a - b)) / scale)


def rand_inputs(seed, BH=3, T=40, dk=8, dv=6, gate="none", delta=False, s0=False, gmin=-0.3):
    r = np.random.default_rng(seed)
    q = r.standard_normal((BH, T, dk))
    k = r.standard_normal((BH, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((BH, T, dv))
    g = None
    if gate == "scalar":
        g = r.uniform(gmin, 0.0, (BH, T))
    elif gate == "channel":
        g = r.uniform(gmin, 0.0, (BH, T, dk))
    beta = r.uniform(0.05, 1.0, (BH, T)) if delta else None
    S0 = 0.3 * r.standard_normal((BH, dv, dk)) if s0 else None
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------------------
# Independent constructions (no token loop over the state)
# ---------------------------------------------------------------------------

def decay_matrix_scalar(g):
    """Gamma[t, j] = prod_{s=j+1}^{t} a_s for j <= t, else 0 ("Mamba-2 ...",
    "Parallel form"), built by explicit products of a_s = exp(g_s)."""
    a = np.exp(g)
    T = len(a)
    G = np.zeros((T, T))
    for t in range(T):
        p = 1.0
        G[t, t] = 1.0
        for j in range(t - 1, -1, -1):
            p *= a[j + 1]
            G[t, j] = p
    return G


def decay_products_channel(g):
    """lam[t, j, :] = prod_{s=j+1}^{t} a_s (Hadamard) for j <= t ("Gated Linear
    Attention (GLA)", "Chunkwise form"), by explicit elementwise products."""
    a = np.exp(g)
    T, d = a.shape
    lam = np.zeros((T, T, d))
    for t in range(T):
        p = np.ones(d)
        lam[t, t] = p
        for j in range(t - 1, -1, -1):
            p = p * a[j + 1]
            lam[t, j] = p
    return lam


def brute_force_matrices(update, gate, q, k, v, g, beta, S0):
    """The defining product written with explicit d x d matrices per token:
    S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
    (delta), S_t = S_{t-1} Diag(alpha_t) + v_t k_t^T (additive / decay)."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else S0.copy()
    o = np.zeros((T, dv))
    for t in range(T):
        if gate == "none":
            D = np.eye(dk)
        elif gate == "scalar":
            D = np.exp(g[t]) * np.eye(dk)
        else:
            D = np.diag(np.exp(g[t]))
        kk = np.outer(k[t], k[t])
        if update == "delta":
            S = S @ D @ (np.eye(dk) - beta[t] * kk) + beta[t] * np.outer(v[t], k[t])
        else:
            S = S @ D + np.outer(v[t], k[t])
        o[t] = S @ q[t]
    return o, S


# ---------------------------------------------------------------------------
# Additive (naive linear attention)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("impl", ["c", "np"])
def test_additive_equals_causal_masked_product(oracle_mod, impl):
    """alpha=1, additive: O = (Q K^T (.) M) V ("Naive linear attention", the
    causal version) plus the S0 read Q S0^T."""
    q, k, v, _, _, S0 = rand_inputs(1, BH=2, T=37, dk=8, dv=5, s0=True)
    fwd = oracle.gdn_forward if impl == "c" else oracle.gdn_forward_np
    o, ST = fwd("additive", "none", q, k, v, S0=S0)
    for h in range(q.shape[0]):
        M = np.tril(np.ones((37, 37)))
        ref = (q[h] @ k[h].T * M) @ v[h] + q[h] @ S0[h].T
        assert rel_err(o[h], ref) < TOL
        assert rel_err(ST[h], S0[h] + v[h].T @ k[h]) < TOL


def test_additive_last_row_is_noncausal_reassociation(oracle_mod):
    """Last output row reads the whole summary K^T V (row convention), i.e.
    o_T = (V^T K) q_T here ("Naive linear attention", reassociation)."""
    q, k, v, _, _, _ = rand_inputs(2, BH=1, T=50, dk=7, dv=9)
    o, _ = oracle.gdn_forward("additive", "none", q, k, v)
    assert rel_err(o[0, -1], v[0].T @ k[0] @ q[0, -1]) < TOL


# ---------------------------------------------------------------------------
# Decay (RetNet / Mamba-2 scalar, GLA channel)
# ---------------------------------------------------------------------------

def test_scalar_decay_equals_gamma_masked_product(oracle_mod):
    """O = (Q K^T (.) Gamma) V with Gamma[t,j] = prod_{s=j+1}^t a_s, plus the
    decayed S0 read ("Mamba-2: input-dependent scalar decay", "Parallel form")."""
    q, k, v, g, _, S0 = rand_inputs(3, BH=2, T=41, dk=6, dv=4, gate="scalar", s0=True)
    o, ST = oracle.gdn_forward("decay", "scalar", q, k, v, g=g, S0=S0)
    for h in range(2):
        G = decay_matrix_scalar(g[h])
        lam0 = np.cumprod(np.exp(g[h]))  # decay of S0 up to and including t
        ref = (q[h] @ k[h].T * G) @ v[h] + lam0[:, None] * (q[h] @ S0[h].T)
        assert rel_err(o[h], ref) < TOL
        refS = lam0[-1] * S0[h] + (v[h] * G[-1][:, None]).T @ k[h]
        assert rel_err(ST[h], refS) < TOL


def test_constant_decay_is_retnet_power_law(oracle_mod):
    """Constant gamma gives Gamma[t, j] = gamma^(t-j) ("RetNet: scalar decay")."""
    q, k, v, _, _, _ = rand_inputs(4, BH=1, T=30, dk=5, dv=5)
    gamma = 0.9
    g = np.full((1, 30), np.log(gamma))
    o, _ = oracle.gdn_forward("decay", "scalar", q, k, v, g=g)
    t = np.arange(30)
    G = np.where(t[:, None] >= t[None, :], gamma ** (t[:, None] - t[None, :]).astype(float), 0.0)
    assert rel_err(o[0], (q[0] @ k[0].T * G) @ v[0]) < TOL


def test_channel_decay_equals_gla_brute_force(oracle_mod):
    """o_t = sum_{j<=t} v_j * ((q_t (.) lam[j+1:t]) . k_j) ("Gated Linear
    Attention (GLA)", "Chunkwise form", local writes) -- the gate acts on the
    key channels."""
    q, k, v, g, _, _ = rand_inputs(5, BH=2, T=23, dk=6, dv=3, gate="channel")
    o, ST = oracle.gdn_forward("decay", "channel", q, k, v, g=g)
    for h in range(2):
        lam = decay_products_channel(g[h])
        ref = np.zeros((23, 3))
        for t in range(23):
            for j in range(t + 1):
                ref[t] += v[h, j] * np.dot(q[h, t] * lam[t, j], k[h, j])
        assert rel_err(o[h], ref) < TOL
        refS = sum(np.outer(v[h, j], k[h, j] * lam[22, j]) for j in range(23))
        assert rel_err(ST[h], refS) < TOL


# ---------------------------------------------------------------------------
# Delta rule
# ---------------------------------------------------------------------------

def test_delta_recall_with_orthonormal_keys(oracle_mod):
    """beta=1, alpha=1, orthonormal unit keys: a read at a key returns the most
    recent value written there, exactly ("DeltaNet", "An intuitive example":
    with beta=1 the new value replaces the old prediction exactly)."""
    d, n_keys, T, dv = 16, 6, 60, 5
    keys = orthonormal_keys(d, n_keys, seed=7)
    r = np.random.default_rng(11)
    widx = r.integers(0, n_keys, T)
    ridx = r.integers(0, n_keys, T)
    k = keys[widx][None]
    q = keys[ridx][None]
    v = r.standard_normal((1, T, dv))
    beta = np.ones((1, T))
    o, _ = oracle.gdn_forward("delta", "none", q, k, v, beta=beta)
    latest = {}
    for t in range(T):
        latest[widx[t]] = v[0, t]
        expect = latest.get(ridx[t], np.zeros(dv))
        assert np.max(np.abs(o[0, t] - expect)) < 1e-12


def test_delta_beta_zero_keeps_state(oracle_mod):
    """beta=0, alpha=1: nothing is written, S_T = S0 and o_t = S0 q_t."""
    q, k, v, _, _, S0 = rand_inputs(6, BH=2, T=25, dk=8, dv=8, s0=True)
    o, ST = oracle.gdn_forward("delta", "none", q, k, v, beta=np.zeros((2, 25)), S0=S0)
    assert np.array_equal(ST, S0)
    for h in range(2):
        assert rel_err(o[h], q[h] @ S0[h].T) < TOL


def test_golden_alice_bob(oracle_mod):
    """The page's worked example, encoded in tests/golden/alice_bob.json."""
    with open(os.path.join(GOLDEN, "alice_bob.json")) as f:
        ex = json.load(f)
    K, V = ex["keys"], ex["values"]
    ks = np.array([K[w[0]] for w in ex["writes"]])[None]
    vs = np.array([V[w[1]] for w in ex["writes"]])[None]
    bs = np.array([w[2] for w in ex["writes"]])[None]
    _, S = oracle.gdn_forward("delta", "none", ks, ks, vs, beta=bs)
    for name, expect in ex["expected_reads_after_last_write"].items():
        assert np.allclose(S[0] @ np.array(K[name]), expect, atol=1e-14)
    bs2 = bs.copy()
    bs2[0, -1] = ex["partial_beta"]
    _, S2 = oracle.gdn_forward("delta", "none", ks, ks, vs, beta=bs2)
    assert np.allclose(S2[0] @ np.array(K["bob"]), ex["expected_bob_read_partial"], atol=1e-14)
    assert np.allclose(S2[0] @ np.array(K["alice"]), V["school"], atol=1e-14)


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
def test_delta_step_is_gradient_step(oracle_mod, gate):
    """Each delta step equals one gradient step of 1/2 ||S k - v||^2 with
    learning rate beta from the decayed state ("Optional: Test-time training
    (TTT) interpretation").  The gradient is taken by central differences."""
    q, k, v, g, beta, S0 = rand_inputs(8, BH=1, T=4, dk=4, dv=3, gate=gate, delta=True, s0=True)
    S_prev = S0[0]
    for t in range(4):
        _, S_t = oracle.gdn_forward("delta", gate, q[:, :t + 1], k[:, :t + 1], v[:, :t + 1],
                                    g=None if g is None else g[:, :t + 1], beta=beta[:, :t + 1], S0=S0)
        if gate == "none":
            Sd = S_prev.copy()
        elif gate == "scalar":
            Sd = S_prev * np.exp(g[0, t])
        else:
            Sd = S_prev * np.exp(g[0, t])[None, :]
        kt, vt = k[0, t], v[0, t]

        def loss(S):
            r = S @ kt - vt
            return 0.5 * float(r @ r)

        grad = np.zeros_like(Sd)
        eps = 1e-6
        for i in range(Sd.shape[0]):
            for j in range(Sd.shape[1]):
                E = np.zeros_like(Sd)
                E[i, j] = eps
                grad[i, j] = (loss(Sd + E) - loss(Sd - E)) / (2 * eps)
        expect = Sd - beta[0, t] * grad
        assert np.max(np.abs(S_t[0] - expect)) < 1e-8
        S_prev = S_t[0]


def _triangular_reference(gate, q, k, v, g, beta):
    """Full-sequence form with S0 = 0: (I + B L) U = B V with
    L[t,j] = k_t . (lam[j+1:t] (.) k_j) for j < t, then O = A U with
    A[t,j] = q_t . (lam[j+1:t] (.) k_j) for j <= t ("The triangular correction
    system", "Parallel output"; gated forms per the GDN and KDA tables)."""
    T, dk = k.shape
    if gate == "none":
        lam = np.ones((T, T, dk))
    elif gate == "scalar":
        lam = decay_matrix_scalar(g)[:, :, None] * np.ones((1, 1, dk))
    else:
        lam = decay_products_channel(g)
    L = np.zeros((T, T))
    A = np.zeros((T, T))
    for t in range(T):
        for j in range(t + 1):
            A[t, j] = np.dot(q[t], lam[t, j] * k[j])
            if j < t:
                L[t, j] = np.dot(k[t], lam[t, j] * k[j])
    Bm = np.diag(beta)
    U = solve_triangular(np.eye(T) + Bm @ L, Bm @ v, lower=True, unit_diagonal=True)
    O = A @ U
    S = sum(np.outer(U[j], lam[T - 1, j] * k[j]) for j in range(T))
    return O, S


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
def test_delta_equals_triangular_solve(oracle_mod, gate):
    q, k, v, g, beta, _ = rand_inputs(9, BH=2, T=48, dk=8, dv=5, gate=gate, delta=True)
    o, ST = oracle.gdn_forward("delta", gate, q, k, v, g=g, beta=beta)
    for h in range(2):
        O, S = _triangular_reference(gate, q[h], k[h], v[h], None if g is None else g[h], beta[h])
        assert rel_err(o[h], O) < 1e-10
        assert rel_err(ST[h], S) < 1e-10


@pytest.mark.parametrize("update,gate", [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
                                         ("delta", "none"), ("delta", "scalar"), ("delta", "channel")])
def test_brute_force_transition_matrices(oracle_mod, update, gate):
    """T <= 16: the defining product with explicit d x d matrices, S0 != 0."""
    q, k, v, g, beta, S0 = rand_inputs(10, BH=2, T=16, dk=6, dv=5, gate=gate,
                                       delta=(update == "delta"), s0=True, gmin=-1.0)
    o, ST = oracle.gdn_forward(update, gate, q, k, v, g=g, beta=beta, S0=S0)
    for h in range(2):
        ro, rS = brute_force_matrices(update, gate, q[h], k[h], v[h], None if g is None else g[h],
                                      None if beta is None else beta[h], S0[h])
        assert rel_err(o[h], ro) < TOL
        assert rel_err(ST[h], rS) < TOL


def test_kda_uniform_gate_reduces_to_gdn(oracle_mod):
    """If every channel of the gate is equal, KDA is GDN ("Kimi Delta
    Attention (KDA)": it reduces exactly to GDN)."""
    q, k, v, g, beta, S0 = rand_inputs(12, BH=2, T=70, dk=8, dv=8, gate="scalar", delta=True, s0=True)
    o1, S1 = oracle.gdn_forward("delta", "scalar", q, k, v, g=g, beta=beta, S0=S0)
    gc = np.repeat(g[..., None], 8, axis=-1)
    o2, S2 = oracle.gdn_forward("delta", "channel", q, k, v, g=gc, beta=beta, S0=S0)
    assert rel_err(o2, o1) < 1e-12 and rel_err(S2, S1) < 1e-12


@pytest.mark.parametrize("update,gate", [("additive", "none"), ("decay", "channel"), ("delta", "scalar"),
                                         ("delta", "channel")])
def test_c_and_numpy_oracles_agree(oracle_mod, update, gate):
    q, k, v, g, beta, S0 = rand_inputs(13, BH=3, T=90, dk=16, dv=12, gate=gate,
                                       delta=(update == "delta"), s0=True)
    a = oracle.gdn_forward(update, gate, q, k, v, g=g, beta=beta, S0=S0)
    b = oracle.gdn_forward_np(update, gate, q, k, v, g=g, beta=beta, S0=S0)
    assert rel_err(a[0], b[0]) < 1e-12 and rel_err(a[1], b[1]) < 1e-12


def test_split_sequence_composes(oracle_mod):
    """Running T1 tokens, then the rest from S_{T1}, equals one run (the state
    is the whole carry; "Update the state")."""
    q, k, v, g, beta, S0 = rand_inputs(14, BH=2, T=50, dk=8, dv=8, gate="channel", delta=True, s0=True)
    o, ST = oracle.gdn_forward("delta", "channel", q, k, v, g=g, beta=beta, S0=S0)
    oa, Sa = oracle.gdn_forward("delta", "channel", q[:, :19], k[:, :19], v[:, :19], g=g[:, :19],
                                beta=beta[:, :19], S0=S0)
    ob, Sb = oracle.gdn_forward("delta", "channel", q[:, 19:], k[:, 19:], v[:, 19:], g=g[:, 19:],
                                beta=beta[:, 19:], S0=Sa)
    assert rel_err(np.concatenate([oa, ob], axis=1), o) < 1e-13 and rel_err(Sb, ST) < 1e-13


SEG_MODES = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"), ("delta", "none"),
             ("delta", "scalar"), ("delta", "channel")]


@pytest.mark.parametrize("update,gate", SEG_MODES)
def test_segment_map_is_affine(oracle_mod, update, gate):
    """The run's final state from any S0 is S0 Lam + H ("One chunk as an affine
    recurrence"): the recurrence against the dense transition product."""
    q, k, v, g, beta, S0 = rand_inputs(21, BH=2, T=30, dk=8, dv=6, gate=gate, delta=update == "delta", s0=True)
    H, Lam = oracle.segment_maps(update, gate, k, v, g=g, beta=beta)
    _, ST = oracle.gdn_forward(update, gate, q, k, v, g=g, beta=beta, S0=S0)
    assert rel_err(S0 @ Lam + H, ST) < 1e-12
    _, H0 = oracle.gdn_forward(update, gate, q, k, v, g=g, beta=beta)
    assert rel_err(H, H0) < 1e-14


def test_segment_map_special_cases(oracle_mod):
    # additive write: the identity transition
    q, k, v, _, _, _ = rand_inputs(22, BH=2, T=12, dk=8, dv=6)
    assert np.array_equal(oracle.segment_maps("additive", "none", k, v)[1], np.broadcast_to(np.eye(8), (2, 8, 8)))
    # delta write with beta = 0 under a scalar gate: exp(sum g) I, and H = 0
    q, k, v, g, beta, _ = rand_inputs(23, BH=2, T=12, dk=8, dv=6, gate="scalar", delta=True)
    H, Lam = oracle.segment_maps("delta", "scalar", k, v, g=g, beta=np.zeros_like(beta))
    expect = np.exp(g.sum(-1))[:, None, None] * np.eye(8)
    assert rel_err(Lam, expect) < 1e-14 and np.all(H == 0)
    # beta = 1 on orthonormal keys, no gate: the projector onto their complement
    kk = orthonormal_keys(8, 5, seed=24)[None]
    H, Lam = oracle.segment_maps("delta", "none", kk, np.zeros((1, 5, 3)), beta=np.ones((1, 5)))
    assert rel_err(Lam[0], np.eye(8) - kk[0].T @ kk[0]) < 1e-14


def test_segment_maps_compose_along_the_sequence(oracle_mod):
    """Three consecutive runs composed through their maps give the one-run
    state; each run's incoming state is the composition of those before it."""
    q, k, v, g, beta, S0 = rand_inputs(25, BH=2, T=36, dk=8, dv=6, gate="channel", delta=True, s0=True)
    cuts = [0, 10, 23, 36]
    S = S0
    for a, b in zip(cuts[:-1], cuts[1:]):
        _, S_ref = oracle.gdn_forward("delta", "channel", q[:, :a], k[:, :a], v[:, :a], g=g[:, :a],
                                      beta=beta[:, :a], S0=S0) if a else (None, S0)
        assert rel_err(S, S_ref) < 1e-12
        H, Lam = oracle.segment_maps("delta", "channel", k[:, a:b], v[:, a:b], g=g[:, a:b], beta=beta[:, a:b])
        S = S @ Lam + H
    _, ST = oracle.gdn_forward("delta", "channel", q, k, v, g=g, beta=beta, S0=S0)
    assert rel_err(S, ST) < 1e-12


# ---------------------------------------------------------------------------
# Planted mistakes: each must break at least one pin
# ---------------------------------------------------------------------------

def _mutant(kind):
    """A copy of the NumPy oracle with one plausible mistake planted."""
    def fwd(update, gate, q, k, v, g=None, beta=None, S0=None):
        T, dk = q.shape[-2], q.shape[-1]
        dv = v.shape[-1]
        S = np.zeros(q.shape[:-2] + (dv, dk)) if S0 is None else S0.copy()
        o = np.empty(q.shape[:-1][:-1] + (T, dv))
        for t in range(T):
            def decay(S):
                if gate == "scalar":
                    return S * np.exp(g[..., t])[..., None, None]
                if gate == "channel":
                    if kind == "gate_on_value_axis":
                        return S * np.exp(g[..., t, :dv])[..., :, None]
                    return S * np.exp(g[..., t, :])[..., None, :]
                return S
            if kind != "decay_after_write":
                S = decay(S)
            kt = k[..., t, :]
            if kind == "read_before_write":
                o[..., t, :] = np.einsum("...ij,...j->...i", S, q[..., t, :])
            if update == "delta":
                Sp = S if kind != "predict_with_undecayed" else (S if gate == "none" else S / 1.0)
                pred = np.einsum("...ij,...j->...i", Sp, kt)
                b = beta[..., t][..., None]
                if kind == "beta_outside":
                    u = b * v[..., t, :] - pred
                elif kind == "sign_flip":
                    u = b * (v[..., t, :] + pred)
                else:
                    u = b * (v[..., t, :] - pred)
            else:
                u = v[..., t, :]
            if kind == "transposed_write":
                S = S + (kt[..., :, None] * u[..., None, :])[..., :dv, :dk]
            else:
                S = S + u[..., :, None] * kt[..., None, :]
            if kind == "decay_after_write":
                S = decay(S)
            if kind == "read_with_key":
                o[..., t, :] = np.einsum("...ij,...j->...i", S, kt)
            elif kind != "read_before_write":
                o[..., t, :] = np.einsum("...ij,...j->...i", S, q[..., t, :])
        return o, S
    return fwd


MUTANTS = ["decay_after_write", "read_before_write", "beta_outside", "sign_flip",
           "transposed_write", "read_with_key", "gate_on_value_axis"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistakes_are_caught(oracle_mod, kind):
    """Runs the brute-force and closed-form pins against a mutated oracle;
    at least one must fail."""
    fwd = _mutant(kind)
    failures = 0
    cases = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
             ("delta", "none"), ("delta", "scalar"), ("delta", "channel")]
    for update, gate in cases:
        q, k, v, g, beta, S0 = rand_inputs(21, BH=1, T=12, dk=6, dv=6, gate=gate,
                                           delta=(update == "delta"), s0=True, gmin=-1.0)
        o, ST = fwd(update, gate, q, k, v, g=g, beta=beta, S0=S0)
        ro, rS = brute_force_matrices(update, gate, q[0], k[0], v[0], None if g is None else g[0],
                                      None if beta is None else beta[0], S0[0])
        if rel_err(o[0], ro) > 1e-6 or rel_err(ST[0], rS) > 1e-6:
            failures += 1
    assert failures > 0, "planted mistake %s was not caught" % kind


# ---------------------------------------------------------------------------
# Gated DeltaProduct ("Gated Delta Product (GDP)", "GDP as GDN over a virtual
# sequence")
# ---------------------------------------------------------------------------

def gdp_inputs(seed, BH=3, T=12, nh=3, dk=8, dv=6, gate="scalar"):
    r = np.random.default_rng(seed)
    q = r.standard_normal((BH, T, dk))
    k = r.standard_normal((BH, T, nh, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((BH, T, nh, dv))
    beta = r.uniform(0.1, 1.0, (BH, T, nh))
    g = None
    if gate == "scalar":
        g = r.uniform(-0.3, 0.0, (BH, T))
    elif gate == "channel":
        g = r.uniform(-0.3, 0.0, (BH, T, dk))
    S0 = 0.3 * r.standard_normal((BH, dv, dk))
    return q, k, v, g, beta, S0


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
def test_gdp_with_one_substep_is_gdn(oracle_mod, gate):
    q, k, v, g, beta, S0 = gdp_inputs(31, nh=1, gate=gate)
    o, S = oracle.gdp_forward(gate, q, k, v, g, beta, S0)
    ro, rS = oracle.gdn_forward("delta", gate, q, k[:, :, 0], v[:, :, 0], g, beta[:, :, 0], S0)
    assert rel_err(o, ro) < TOL and rel_err(S, rS) < TOL


@pytest.mark.parametrize("gate", ["none", "scalar", "channel"])
@pytest.mark.parametrize("nh", [2, 3])
def test_gdp_is_gdn_over_the_virtual_sequence(oracle_mod, gate, nh):
    # the page's table: substep (t, j) is virtual step t*nh + j; the decay sits on
    # the first substep of a token, the query on the last, and every nh-th output
    # is kept
    q, k, v, g, beta, S0 = gdp_inputs(32, nh=nh, gate=gate)
    BH, T, dk = q.shape
    Tv = T * nh
    qv = np.zeros((BH, Tv, dk))
    qv[:, nh - 1::nh] = q
    gv = None
    if gate == "scalar":
        gv = np.zeros((BH, Tv))
        gv[:, 0::nh] = g
    elif gate == "channel":
        gv = np.zeros((BH, Tv, dk))
        gv[:, 0::nh] = g
    ov, Sv = oracle.gdn_forward("delta", gate, qv, k.reshape(BH, Tv, dk), v.reshape(BH, Tv, -1), gv,
                                beta.reshape(BH, Tv), S0)
    o, S = oracle.gdp_forward(gate, q, k, v, g, beta, S0)
    assert rel_err(o, ov[:, nh - 1::nh]) < TOL and rel_err(S, Sv) < TOL


def test_gdp_brute_force_products(oracle_mod):
    # per token: S <- S Diag(a_t) H_1 ... H_nh + (write terms), each substep the
    # explicit matrix map S -> S (I - beta k k^T) + beta v k^T
    q, k, v, g, beta, S0 = gdp_inputs(33, BH=1, T=5, nh=3, dk=4, dv=3, gate="channel")
    S = S0[0].copy()
    outs = []
    for t in range(5):
        S = S @ np.diag(np.exp(g[0, t]))
        for j in range(3):
            kk = k[0, t, j][:, None]
            S = S @ (np.eye(4) - beta[0, t, j] * kk @ kk.T) + beta[0, t, j] * v[0, t, j][:, None] @ kk.T
        outs.append(S @ q[0, t])
    o, Sf = oracle.gdp_forward("channel", q, k, v, g, beta, S0)
    assert rel_err(o[0], np.array(outs)) < TOL and rel_err(Sf[0], S) < TOL


def test_gdp_zero_write_strength_only_decays(oracle_mod):
    q, k, v, g, beta, S0 = gdp_inputs(34, gate="scalar")
    beta[:] = 0.0
    o, S = oracle.gdp_forward("scalar", q, k, v, g, beta, S0)
    G = np.cumsum(g, axis=1)
    expect = np.einsum("bij,btj->bti", S0, q) * np.exp(G)[..., None]
    assert rel_err(o, expect) < TOL and rel_err(S, S0 * np.exp(G[:, -1])[:, None, None]) < TOL


# ---------------------------------------------------------------------------
# Input prologue maps: values fixed by the definitions of elu, the 2-norm,
# the logistic function and softplus
# ---------------------------------------------------------------------------

def test_prologue_closed_forms():
    x = np.array([[-np.inf, -1.0, 0.0, 2.0]])
    q, _, _, _ = oracle.prologue(oracle.PRO_QK_ELU1, q=x)
    assert np.allclose(q, [[0.0, np.exp(-1.0), 1.0, 3.0]], rtol=0, atol=1e-15)
    b = np.array([0.0, np.log(3.0), -np.log(3.0)])
    _, _, beta, _ = oracle.prologue(oracle.PRO_BETA_SIGMOID, beta=b)
    assert np.allclose(beta, [0.5, 0.75, 0.25], rtol=0, atol=1e-15)
    gx = np.array([0.0, np.log(np.e - 1.0), -50.0, 50.0])
    _, _, _, g = oracle.prologue(oracle.PRO_G_NEG_SOFTPLUS, g=gx)
    assert np.allclose(g, [-np.log(2.0), -1.0, -np.exp(-50.0), -50.0 - np.exp(-50.0)], rtol=1e-14, atol=1e-300)


def test_prologue_l2_rows():
    r = np.random.default_rng(41)
    x = r.standard_normal((3, 7, 16)) * r.uniform(0.1, 10.0, (3, 7, 1))
    x[1, 2] = 0.0
    q, k, _, _ = oracle.prologue(oracle.PRO_QK_L2, q=x, k=3.0 * x)
    n = np.linalg.norm(q, axis=-1)
    mask = np.ones((3, 7), bool)
    mask[1, 2] = False
    assert np.allclose(n[mask], 1.0, atol=1e-14) and np.all(q[1, 2] == 0.0)
    assert np.allclose(q, k, atol=1e-15)  # scale-free
    # feature map first, then the norm
    q2, _, _, _ = oracle.prologue(oracle.PRO_QK_ELU1 | oracle.PRO_QK_L2, q=x)
    e = np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    assert np.allclose(q2, e / np.linalg.norm(e, axis=-1, keepdims=True), atol=1e-15)


# ---------------------------------------------------------------------------
# Decode: consecutive single-token steps are the recurrence over the stacked
# sequence ("Optional: Linear attention as an RNN": one state, one token at a
# time).  decode_sequence is the reference of every decode GPU test, so its
# stacking (per tensor, along the token axis) is pinned against explicit d x d
# products over the same tokens, gathered by hand one step and head at a time.
# ---------------------------------------------------------------------------

def _decode_steps(seed, gate, update, B=2, H=2, n=9, dk=6, dv=5):
    r = np.random.default_rng(seed)
    steps = []
    for _ in range(n):
        k = r.standard_normal((B, H, 1, dk))
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        s = {"q": r.standard_normal((B, H, 1, dk)), "k": k, "v": r.standard_normal((B, H, 1, dv)),
             "beta": r.uniform(0.05, 1.0, (B, H, 1)) if update == "delta" else None, "g": None}
        if gate == "scalar":
            s["g"] = r.uniform(-0.4, 0.0, (B, H, 1))
        elif gate == "channel":
            s["g"] = r.uniform(-0.4, 0.0, (B, H, 1, dk))
        steps.append(s)
    S0 = 0.3 * r.standard_normal((B, H, dv, dk))
    return steps, S0


@pytest.mark.parametrize("update,gate", [("delta", "scalar"), ("delta", "channel"), ("delta", "none"),
                                         ("decay", "scalar"), ("decay", "channel"), ("additive", "none")])
def test_decode_sequence_equals_explicit_products(oracle_mod, update, gate):
    steps, S0 = _decode_steps(61, gate, update)
    o, S = oracle.decode_sequence(update, gate, S0, steps)
    n = len(steps)
    B, H = S0.shape[:2]
    assert o.shape == (B, H, n, steps[0]["v"].shape[-1]) and S.shape == S0.shape
    for b in range(B):
        for h in range(H):
            # this head's tokens, taken from each step's dict in order
            q = np.stack([s["q"][b, h, 0] for s in steps])
            k = np.stack([s["k"][b, h, 0] for s in steps])
            v = np.stack([s["v"][b, h, 0] for s in steps])
            g = None if gate == "none" else np.stack([np.asarray(s["g"][b, h, 0]) for s in steps])
            beta = None if update != "delta" else np.array([s["beta"][b, h, 0] for s in steps])
            ro, rS = brute_force_matrices(update, gate, q, k, v, g, beta, S0[b, h])
            assert rel_err(o[b, h], ro) < TOL and rel_err(S[b, h], rS) < TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_decode_sequence_chains_one_step_calls(oracle_mod, gate):
    """n calls of one step each, the state handed on, equal one call of n steps."""
    steps, S0 = _decode_steps(62, gate, "delta")
    o, S = oracle.decode_sequence("delta", gate, S0, steps)
    Sc = S0
    for i, s in enumerate(steps):
        oi, Sc = oracle.decode_sequence("delta", gate, Sc, [s])
        assert rel_err(oi[..., 0, :], o[..., i, :]) < TOL
    assert rel_err(Sc, S) < TOL


def test_gate_and_beta_layouts_are_checked(oracle_mod):
    """A gate or write strength laid out along the wrong axis is rejected."""
    q, k, v, g, beta, _ = rand_inputs(63, BH=2, T=5, dk=4, dv=3, gate="channel", delta=True)
    with pytest.raises(ValueError):
        oracle.gdn_forward("delta", "channel", q, k, v, g=g[..., 0], beta=beta)
    with pytest.raises(ValueError):
        oracle.gdn_forward("delta", "scalar", q, k, v, g=g, beta=beta)
    with pytest.raises(ValueError):
        oracle.gdn_forward("delta", "channel", q, k, v, g=g, beta=beta[..., None])


# ---------------------------------------------------------------------------
# Backward: gdn_backward_np is pinned to central finite differences of the
# forward definition (every input element of tiny cases, all six modes) and to
# the closed-form gradients of causal linear attention.
# ---------------------------------------------------------------------------

BWD_MODES = [("additive", "none"), ("decay", "scalar"), ("decay", "channel"),
             ("delta", "none"), ("delta", "scalar"), ("delta", "channel")]


def _bwd_case(seed, update, gate, BH=2, T=7, dk=4, dv=3):
    q, k, v, g, beta, S0 = rand_inputs(seed, BH=BH, T=T, dk=dk, dv=dv, gate=gate, delta=update == "delta",
                                       s0=True, gmin=-0.6)
    r = np.random.default_rng(seed + 1000)
    dO = r.standard_normal((BH, T, dv))
    dST = r.standard_normal((BH, dv, dk))
    return q, k, v, g, beta, S0, dO, dST


@pytest.mark.parametrize("update,gate", BWD_MODES)
def test_backward_equals_finite_differences(oracle_mod, update, gate):
    q, k, v, g, beta, S0, dO, dST = _bwd_case(71, update, gate)
    got = oracle.gdn_backward_np(update, gate, q, k, v, g, beta, S0, dO, dST, checkpoint=3)
    inputs = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "S0": S0}
    names = ["q", "k", "v", "g", "beta", "S0"]

    def loss(x):
        o, ST = oracle.gdn_forward_np(update, gate, x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
        return float(np.sum(o * dO) + np.sum(ST * dST))

    h = 1e-6
    for name, grad in zip(names, got):
        if inputs[name] is None:
            assert grad is None
            continue
        fd = np.zeros_like(inputs[name])
        it = np.nditer(inputs[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = {n: (None if a is None else a.copy()) for n, a in inputs.items()}
            xm = {n: (None if a is None else a.copy()) for n, a in inputs.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            fd[idx] = (loss(xp) - loss(xm)) / (2 * h)
        assert rel_err(grad, fd) < 1e-6, (name, rel_err(grad, fd))


def test_backward_independent_of_checkpoint_spacing(oracle_mod):
    q, k, v, g, beta, S0, dO, dST = _bwd_case(72, "delta", "channel", T=11)
    ref = oracle.gdn_backward_np("delta", "channel", q, k, v, g, beta, S0, dO, dST, checkpoint=64)
    for c in (1, 4, 5):
        got = oracle.gdn_backward_np("delta", "channel", q, k, v, g, beta, S0, dO, dST, checkpoint=c)
        for a, b in zip(got, ref):
            assert np.array_equal(a, b)


def test_backward_additive_closed_forms(oracle_mod):
    """Causal linear attention o_t = sum_{s<=t} (q_t . k_s) v_s + S0 q_t and
    S_T = S0 + V^T K ("Naive linear attention", causal): with M the causal
    mask, dQ = (dO V^T (.) M) K + dO S0, dK = (dO V^T (.) M)^T Q + V dS_T,
    dV = (Q K^T (.) M)^T dO + K dS_T^T, dS0 = dO^T Q + dS_T."""
    q, k, v, _, _, S0, dO, dST = _bwd_case(73, "additive", "none", BH=2, T=29, dk=6, dv=5)
    dq, dk, dv, dg, db, dS0 = oracle.gdn_backward_np("additive", "none", q, k, v, None, None, S0, dO, dST,
                                                     checkpoint=8)
    assert dg is None and db is None
    M = np.tril(np.ones((29, 29)))
    for h in range(2):
        G = dO[h] @ v[h].T * M
        assert rel_err(dq[h], G @ k[h] + dO[h] @ S0[h]) < TOL
        assert rel_err(dk[h], G.T @ q[h] + v[h] @ dST[h]) < TOL
        assert rel_err(dv[h], (q[h] @ k[h].T * M).T @ dO[h] + k[h] @ dST[h].T) < TOL
        assert rel_err(dS0[h], dO[h].T @ q[h] + dST[h]) < TOL



@pytest.mark.parametrize("update,gate,flags", [
    ("delta", "scalar", oracle.PRO_QK_L2 | oracle.PRO_BETA_SIGMOID | oracle.PRO_G_NEG_SOFTPLUS),
    ("delta", "channel", oracle.PRO_QK_ELU1 | oracle.PRO_QK_L2 | oracle.PRO_G_NEG_SOFTPLUS),
    ("delta", "none", oracle.PRO_QK_ELU1 | oracle.PRO_BETA_SIGMOID),
    ("additive", "none", oracle.PRO_QK_ELU1),
    ("decay", "scalar", oracle.PRO_QK_L2 | oracle.PRO_G_NEG_SOFTPLUS),
])
def test_prologue_backward_equals_finite_differences(oracle_mod, update, gate, flags):
    """The gradients with respect to the raw inputs match central differences
    of the loss through the maps and the recurrence (raw gate and beta drawn as
    logits, some raw q / k entries negative so both branches of elu are hit)."""
    q, k, v, g, beta, S0, dO, dST = _bwd_case(91, update, gate)
    r = np.random.default_rng(92)
    q = q + 0.3 * r.standard_normal(q.shape)
    k = k + 0.3 * r.standard_normal(k.shape)
    if beta is not None:
        beta = r.standard_normal(beta.shape)
    if g is not None:
        g = r.standard_normal(g.shape) - 2.0
    got = oracle.gdn_backward_prologue_np(update, gate, flags, q, k, v, g, beta, S0, dO, dST)
    inputs = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "S0": S0}

    def loss(x):
        qm, km, bm, gm = oracle.prologue(flags, q=x["q"], k=x["k"], beta=x["beta"], g=x["g"])
        o, ST = oracle.gdn_forward_np(update, gate, qm, km, x["v"], gm, bm, x["S0"])
        return float(np.sum(o * dO) + np.sum(ST * dST))

    h = 1e-6
    for name, grad in zip(["q", "k", "v", "g", "beta", "S0"], got):
        if inputs[name] is None:
            assert grad is None
            continue
        fd = np.zeros_like(inputs[name])
        it = np.nditer(inputs[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = {n: (None if a is None else a.copy()) for n, a in inputs.items()}
            xm = {n: (None if a is None else a.copy()) for n, a in inputs.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            fd[idx] = (loss(xp) - loss(xm)) / (2 * h)
        assert rel_err(grad, fd) < 1e-6, (name, rel_err(grad, fd))


def test_prologue_backward_without_maps_is_the_plain_backward(oracle_mod):
    q, k, v, g, beta, S0, dO, dST = _bwd_case(93, "delta", "channel")
    a = oracle.gdn_backward_prologue_np("delta", "channel", 0, q, k, v, g, beta, S0, dO, dST)
    b = oracle.gdn_backward_np("delta", "channel", q, k, v, g, beta, S0, dO, dST)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
