"""Float64 NumPy model of the chunkwise algorithm the CUDA kernels implement.

Test infrastructure: it is checked against the oracle (token recurrence) for
several chunk sizes.  With ``emulate_bf16="bf16"`` or ``"fp16"`` it rounds to
that format at every point where a tensor-core kernel hands an operand to the
tensor cores (T diag(beta), K<, W, S, Z, Q<, A, K>), which predicts the size of
such a kernel's parity error before it runs.

Per chunk r (rows l, m are positions in the chunk; S is [dv, dk]):
  G_l    = sum_{s<=l} g_s                       (scalar or per key channel)
  Q<_l   = q_l (.) e^{G_l},  K<_l = k_l (.) e^{G_l},  K>_m = k_m (.) e^{G_C - G_m}
  A[l,m] = sum_i q_li k_mi e^{G_li - G_mi}      (m <= l)
  delta:   L[l,m] = sum_i k_li k_mi e^{G_li - G_mi} (m < l)
           T = (I + diag(beta) L)^{-1},  W = T diag(beta) K<,  U = T diag(beta) V
           Z = U - W S^T
  else:    Z = V
  O_r     = Q< S^T + A Z
  S      <- S Diag(e^{G_C}) + Z^T K>
("Linear Attention, Visualized": "Chunkwise algorithm", "Mamba-2 ...
Chunkwise form", "Optional: Use UT to share the triangular transform",
"Correct the incoming state", the GDN method table, "Gated Linear Attention
(GLA)" and the KDA table.)  A ragged last chunk is padded with identity tokens
(q = k = v = 0, beta = 0, g = 0).
"""
import numpy as np

from synth import round_to_bf16


def _bf(x, on):
    """Operand rounding: off (False), "bf16" (True or "bf16") or "fp16"."""
    if not on:
        return x
    if on == "fp16":
        return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)
    return round_to_bf16(np.asarray(x, np.float32)).astype(np.float64)


def chunk_forward(update, gate, q, k, v, g=None, beta=None, S0=None, C=64, emulate_bf16=False):
    """One head. q,k [T,dk]; v [T,dv]; g [T] or [T,dk]; beta [T]; S0 [dv,dk]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.asarray(S0, np.float64).copy()
    O = np.zeros((T, dv))
    eb = emulate_bf16
    for t0 in range(0, T, C):
        n = min(C, T - t0)
        qc = np.zeros((C, dk)); qc[:n] = q[t0:t0 + n]
        kc = np.zeros((C, dk)); kc[:n] = k[t0:t0 + n]
        vc = np.zeros((C, dv)); vc[:n] = v[t0:t0 + n]
        if gate == "none":
            G = np.zeros((C, dk))
        elif gate == "scalar":
            gc = np.zeros(C); gc[:n] = g[t0:t0 + n]
            G = np.repeat(np.cumsum(gc)[:, None], dk, axis=1)
        else:
            gc = np.zeros((C, dk)); gc[:n] = g[t0:t0 + n]
            G = np.cumsum(gc, axis=0)
        Ql = qc * np.exp(G)
        Kl = kc * np.exp(G)
        Kr = kc * np.exp(G[-1][None, :] - G)
        diff = G[:, None, :] - G[None, :, :]          # [l, m, i] = G_li - G_mi
        mask_incl = np.tril(np.ones((C, C)))
        E = np.exp(np.where(mask_incl[:, :, None] > 0, diff, -np.inf))
        A = np.einsum("li,mi,lmi->lm", qc, kc, E)
        if update == "delta":
            bc = np.zeros(C); bc[:n] = beta[t0:t0 + n]
            L = np.einsum("li,mi,lmi->lm", kc, kc, E) * np.tril(np.ones((C, C)), -1)
            Tm = np.linalg.inv(np.eye(C) + bc[:, None] * L)
            TB = _bf(Tm * bc[None, :], eb)
            W = _bf(TB @ _bf(Kl, eb), eb)
            U = TB @ vc
            Z = U - W @ _bf(S, eb).T
        else:
            Z = vc
        Zb = _bf(Z, eb)
        O[t0:t0 + n] = (_bf(Ql, eb) @ _bf(S, eb).T + _bf(A, eb) @ Zb)[:n]
        S = S * np.exp(G[-1])[None, :] + Zb.T @ _bf(Kr, eb)
    return O, S


def chunk_forward_heads(update, gate, q, k, v, g=None, beta=None, S0=None, C=64, emulate_bf16=False):
    """Batched over leading head dims [..., T, d]."""
    lead = q.shape[:-2]
    n = int(np.prod(lead)) if lead else 1
    T, dk = q.shape[-2:]
    dv = v.shape[-1]
    qf, kf, vf = q.reshape(n, T, dk), k.reshape(n, T, dk), v.reshape(n, T, dv)
    gf = None if g is None else g.reshape((n,) + g.shape[len(lead):])
    bf = None if beta is None else beta.reshape(n, T)
    sf = None if S0 is None else S0.reshape(n, dv, dk)
    O = np.empty((n, T, dv))
    S = np.empty((n, dv, dk))
    for i in range(n):
        O[i], S[i] = chunk_forward(update, gate, qf[i], kf[i], vf[i], None if gf is None else gf[i],
                                   None if bf is None else bf[i], None if sf is None else sf[i], C,
                                   emulate_bf16)
    return O.reshape(lead + (T, dv)), S.reshape(lead + (dv, dk))
