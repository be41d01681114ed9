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


def chunk_backward(update, gate, q, k, v, g=None, beta=None, S0=None, dO=None, dS_T=None, C=64):
    """Reverse mode through the chunk algebra above, float64, one head, the
    scalar or no gate: the passes the tensor-core backward runs.  Returns (dq,
    dk, dv, dg, dbeta, dS0) (dg / dbeta None without gate / delta rule).

    Per chunk, with S the state entering it and dSn the gradient of the state
    leaving it (Qb = diag(b) q, Kb = diag(b) k, Kc = diag(b_C / b) k, PG =
    strict-lower(k k^T) Gamma, Mv = diag(beta) v, Mk = diag(beta) Kb):
      dZ = A^T dO + Kc dSn^T;   dKc = Z dSn;   dA = dO Z^T;   dQb = dO S
      delta: dW = -dZ S;  dT = dZ Mv^T + dW Mk^T;  dL = strict-lower(-T^T dT T^T)
             dv = diag(beta) T^T dZ;  dKb = diag(beta) T^T dW
      else:  dv = dZ
      dS_r = b_C dSn + dO^T Qb - dZ^T W = b_C dSn - (dSn Kc^T) W + dO^T (Qb - A W)
    then dq, dk, dbeta through Qb, Kb, Kc, L = diag(beta) PG and A = lower(q k^T)
    Gamma, and the gate through every exponential: dG_l from b_l, b_C / b_l,
    Gamma and b_C S, with dg_s = sum_{l >= s} dG_l."""
    assert gate in ("none", "scalar")
    T, dk = q.shape
    dv_ = v.shape[1]
    delta, gated = update == "delta", gate == "scalar"
    n = max(1, -(-T // C))
    pad = lambda a, w: np.concatenate([a, np.zeros((n * C - T,) + a.shape[1:])]) if a is not None else np.zeros(w)
    qq, kk, vv = pad(q, None), pad(k, None), pad(v, None)
    gg = pad(g, None) if gated else np.zeros(n * C)
    bb = pad(beta, None) if delta else np.zeros(n * C)
    do = pad(dO, None) if dO is not None else np.zeros((n * C, dv_))
    S = np.zeros((dv_, dk)) if S0 is None else np.array(S0, np.float64)
    # forward over the chunks: the states entering them and the chunk tiles
    states, tiles = [], []
    for r in range(n):
        sl = slice(r * C, r * C + C)
        qc, kc, vc, bc = qq[sl], kk[sl], vv[sl], bb[sl]
        G = np.cumsum(gg[sl])
        b, ec, bC = np.exp(G), np.exp(G[-1] - G), np.exp(G[-1])
        Gam = np.tril(np.exp(G[:, None] - G[None, :]))
        A = np.tril(qc @ kc.T) * Gam
        tl = dict(G=G, b=b, ec=ec, bC=bC, Gam=Gam, A=A)
        if delta:
            tl["PG"] = np.tril(kc @ kc.T, -1) * Gam
            tl["T"] = np.linalg.inv(np.eye(C) + bc[:, None] * tl["PG"])
            tl["W"] = tl["T"] @ ((bc * b)[:, None] * kc)
            Z = tl["T"] @ (bc[:, None] * vc) - tl["W"] @ S.T
        else:
            Z = vc
        tl["Qt"] = b[:, None] * qc - (A @ tl["W"] if delta else 0.0)
        tl["Kc"] = ec[:, None] * kc
        states.append(S)
        tiles.append(tl)
        S = bC * S + Z.T @ tl["Kc"]
    # the state-gradient chain, chunks last to first
    dS = np.zeros((dv_, dk)) if dS_T is None else np.array(dS_T, np.float64)
    dSn = [None] * n
    for r in range(n - 1, -1, -1):
        tl, doc = tiles[r], do[r * C:(r + 1) * C]
        dSn[r] = dS
        nxt = tl["bC"] * dS + doc.T @ tl["Qt"]
        if delta:
            nxt = nxt - (dS @ tl["Kc"].T) @ tl["W"]
        dS = nxt
    out_q, out_k, out_v = np.zeros((n * C, dk)), np.zeros((n * C, dk)), np.zeros((n * C, dv_))
    out_g, out_b = np.zeros(n * C), np.zeros(n * C)
    # every chunk's local gradients
    for r in range(n):
        tl, sl = tiles[r], slice(r * C, r * C + C)
        qc, kc, vc, bc, doc = qq[sl], kk[sl], vv[sl], bb[sl], do[sl]
        Sr, dSr = states[r], dSn[r]
        b, ec, bC, Gam, A = tl["b"], tl["ec"], tl["bC"], tl["Gam"], tl["A"]
        Z = (tl["T"] @ (bc[:, None] * vc) - tl["W"] @ Sr.T) if delta else vc
        dZ = ec[:, None] * (kc @ dSr.T) + A.T @ doc
        dKc, dQb, dA = Z @ dSr, doc @ Sr, doc @ Z.T
        dG, db = np.zeros(C), np.zeros(C)
        H = np.tril(dA * A, -1)
        dkk = ec[:, None] * dKc
        if delta:
            Tm, PG = tl["T"], tl["PG"]
            dW = -dZ @ Sr
            tdz, kb = Tm.T @ dZ, Tm.T @ dW
            dvv = bc[:, None] * tdz
            dT = bc[None, :] * (dZ @ vc.T + b[None, :] * (dW @ kc.T))
            dL = np.tril(-Tm.T @ dT @ Tm.T, -1)
            E = dL * bc[:, None] * Gam
            s = np.sum(kb * kc, axis=1)
            db += np.sum(tdz * vc, axis=1) + b * s + np.sum(dL * PG, axis=1)
            dG += b * bc * s
            H = H + dL * bc[:, None] * PG
            dkk = dkk + (b * bc)[:, None] * kb + E @ kc + E.T @ kc
        else:
            dvv = dZ
        F = np.tril(dA) * Gam
        dkk = dkk + F.T @ qc
        dqq = b[:, None] * dQb + F @ kc
        cp = ec * np.sum(kc * dKc, axis=1)
        dG += b * np.sum(qc * dQb, axis=1) - cp + H.sum(1) - H.sum(0)
        dG[-1] += bC * np.sum(dSr * Sr) + cp.sum()
        out_q[sl], out_k[sl], out_v[sl] = dqq, dkk, dvv
        out_g[sl] = np.cumsum(dG[::-1])[::-1]
        out_b[sl] = db
    return (out_q[:T], out_k[:T], out_v[:T], out_g[:T] if gated else None, out_b[:T] if delta else None, dS)


def chunk_backward_channel(update, q, k, v, g, beta=None, S0=None, dO=None, dS_T=None, C=64):
    """The chunkwise backward for a per-channel gate (KDA / GLA), float64, one
    head: g [T, dk] (log alpha per key channel).  Returns (dq, dk, dv, dg,
    dbeta, dS0) (dbeta None without the delta rule).

    With G [C, dk] the in-chunk prefix, Qb = q (.) e^G, Kb = k (.) e^G,
    Ki = k (.) e^{-G}, Kc = k (.) e^{G_C - G}, every Gamma factor sits inside a
    product: A = lower-incl(Qb Ki^T), L = diag(beta) strict-lower(Kb Ki^T)
    ("Kimi Delta Attention (KDA)": the channel-wise decay table; "Gated Linear
    Attention (GLA)", Chunkwise form), and S' = S Diag(e^{G_C}) + Z^T Kc.  The
    reverse pass is the scalar one with the gate gradient per channel:
      dQb += tril(dA) Ki;  dKi = tril(dA)^T Qb + E^T Kb;  dKb += E Ki,
      E = diag(beta) dL (strict lower);  dbeta_l += sum_m dL[l,m] (Kb Ki^T)[l,m]
      dq = dQb e^G;  dk = dKb e^G + dKi e^{-G} + dKc e^{G_C - G}
      dG += dQb Qb + dKb Kb - dKi Ki - dKc Kc  (elementwise), and in row C - 1
      sum_l dKc_l Kc_l + e^{G_C} (.) sum_v dSn[v] (.) S[v]; dg = reverse prefix sums."""
    T, dk = q.shape
    dv_ = v.shape[1]
    delta = update == "delta"
    n = max(1, -(-T // C))
    pad = lambda a: np.concatenate([a, np.zeros((n * C - T,) + a.shape[1:])])
    qq, kk, vv, gg = pad(q), pad(k), pad(v), pad(g)
    bb = pad(beta) if delta else np.zeros(n * C)
    do = pad(dO) if dO is not None else np.zeros((n * C, dv_))
    S = np.zeros((dv_, dk)) if S0 is None else np.array(S0, np.float64)
    states, tiles = [], []
    for r in range(n):
        sl = slice(r * C, r * C + C)
        qc, kc, vc, bc = qq[sl], kk[sl], vv[sl], bb[sl]
        G = np.cumsum(gg[sl], axis=0)
        GC = G[-1]
        Qb, Kb, Ki, Kc = qc * np.exp(G), kc * np.exp(G), kc * np.exp(-G), kc * np.exp(GC - G)
        A = np.tril(Qb @ Ki.T)
        tl = dict(G=G, GC=GC, Qb=Qb, Kb=Kb, Ki=Ki, Kc=Kc, A=A)
        if delta:
            tl["P"] = np.tril(Kb @ Ki.T, -1)
            tl["T"] = np.linalg.inv(np.eye(C) + bc[:, None] * tl["P"])
            tl["W"] = tl["T"] @ (bc[:, None] * Kb)
            Z = tl["T"] @ (bc[:, None] * vc) - tl["W"] @ S.T
        else:
            Z = vc
        tl["Qt"] = Qb - (A @ tl["W"] if delta else 0.0)
        states.append(S)
        tiles.append(tl)
        S = S * np.exp(GC)[None, :] + Z.T @ Kc
    dS = np.zeros((dv_, dk)) if dS_T is None else np.array(dS_T, np.float64)
    dSn = [None] * n
    for r in range(n - 1, -1, -1):
        tl, doc = tiles[r], do[r * C:(r + 1) * C]
        dSn[r] = dS
        nxt = dS * np.exp(tl["GC"])[None, :] + doc.T @ tl["Qt"]
        if delta:
            nxt = nxt - (dS @ tl["Kc"].T) @ tl["W"]
        dS = nxt
    out_q, out_k, out_v = np.zeros((n * C, dk)), np.zeros((n * C, dk)), np.zeros((n * C, dv_))
    out_g, out_b = np.zeros((n * C, dk)), np.zeros(n * C)
    for r in range(n):
        tl, sl = tiles[r], slice(r * C, r * C + C)
        vc, bc, doc = vv[sl], bb[sl], do[sl]
        Sr, dSr = states[r], dSn[r]
        G, GC, Qb, Kb, Ki, Kc, A = (tl[x] for x in ("G", "GC", "Qb", "Kb", "Ki", "Kc", "A"))
        Z = (tl["T"] @ (bc[:, None] * vc) - tl["W"] @ Sr.T) if delta else vc
        dZ = Kc @ dSr.T + A.T @ doc
        dKc, dQb, dA = Z @ dSr, doc @ Sr, np.tril(doc @ Z.T)
        dKb, db = np.zeros_like(Kb), np.zeros(C)
        dQb = dQb + dA @ Ki
        dKi = dA.T @ Qb
        if delta:
            Tm = tl["T"]
            dW = -dZ @ Sr
            tdz = Tm.T @ dZ
            dvv = bc[:, None] * tdz
            dT = (dZ @ (bc[:, None] * vc).T) + (dW @ (bc[:, None] * Kb).T)
            dL = np.tril(-Tm.T @ dT @ Tm.T, -1)
            kbw = Tm.T @ dW
            dKb = dKb + bc[:, None] * kbw
            db += np.sum(tdz * vc, axis=1) + np.sum(kbw * Kb, axis=1) + np.sum(dL * tl["P"], axis=1)
            E = bc[:, None] * dL
            dKb = dKb + E @ Ki
            dKi = dKi + E.T @ Kb
        else:
            dvv = dZ
        eG, emG, ec = np.exp(G), np.exp(-G), np.exp(GC - G)
        out_q[sl] = dQb * eG
        out_k[sl] = dKb * eG + dKi * emG + dKc * ec
        out_v[sl] = dvv
        dG = dQb * Qb + dKb * Kb - dKi * Ki - dKc * Kc
        dG[-1] += np.sum(dKc * Kc, axis=0) + np.exp(GC) * np.sum(dSr * Sr, axis=0)
        out_g[sl] = np.cumsum(dG[::-1], axis=0)[::-1]
        out_b[sl] = db
    return (out_q[:T], out_k[:T], out_v[:T], out_g[:T], out_b[:T] if delta else None, dS)
