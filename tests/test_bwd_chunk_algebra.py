"""The chunk form of the gradient that the backward kernels implement (the
formulas at the head of csrc/kda_bwd.cu), written out in fp64 NumPy and
checked against the per-token backward oracle (oracle/backward.py) on random
inputs: ragged lengths, partial last chunks, an initial state and a
final-state gradient.  This pins the algebra itself on the CPU; the GPU tests
pin the kernels against the same oracle.
"""
import numpy as np
import pytest

from oracle import backward as B

C = 16


def _chunk_ops(q, k, v, g, beta, scale):
    """Per-chunk operands of the forward chunk form (rows past the end are zero)."""
    G = np.cumsum(g, axis=0)
    Kd, Ki, Qd = k * np.exp(G), k * np.exp(-G), scale * q * np.exp(G)
    Fb = np.exp(G[-1][None, :] - G)
    Kb = k * Fb
    A = np.tril(Kd @ Ki.T, -1)
    P = np.tril(Qd @ Ki.T)
    X = np.linalg.inv(np.eye(C) + beta[:, None] * A)
    T = X * beta[None, :]
    return dict(G=G, Kd=Kd, Ki=Ki, Qd=Qd, Kb=Kb, Fb=Fb, A=A, P=P, X=X, T=T, W=T @ Kd,
                U0=T @ v, gC=np.exp(G[-1]))


def chunk_backward(q, k, v, g, beta, gate, dy, s0, dsT, scale):
    L, dk = k.shape
    dv = v.shape[1]
    nc = (L + C - 1) // C
    chunks = []
    for c in range(nc):
        a, b = c * C, min(L, c * C + C)
        pad = lambda x: np.concatenate([x[a:b], np.zeros((C - (b - a),) + x.shape[1:])])
        xs = [pad(x) for x in (q, k, v, g, beta, gate, dy)]
        chunks.append((a, b, xs, _chunk_ops(xs[0], xs[1], xs[2], xs[3], xs[4], scale)))
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g),
                                            ("dbeta", beta), ("dgate", gate))}
    # forward chain: S entering each chunk, U; dgate = dy (.) O
    S, Ss, Us = s0.copy(), [], []
    for a, b, xs, o in chunks:
        U = o["U0"] - o["W"] @ S
        out["dgate"][a:b] = (xs[6] * (o["Qd"] @ S + o["P"] @ U))[: b - a]
        Ss.append(S)
        Us.append(U)
        S = o["gC"][:, None] * S + o["Kb"].T @ U
    # reverse chain: dS' leaving each chunk, dU
    dS, dSs, dUs = dsT.copy(), [None] * nc, [None] * nc
    for c in range(nc - 1, -1, -1):
        _, _, xs, o = chunks[c]
        dO = xs[5] * xs[6]
        dU = o["P"].T @ dO + o["Kb"] @ dS
        dSs[c], dUs[c] = dS, dU
        dS = o["Qd"].T @ dO + o["gC"][:, None] * dS - o["W"].T @ dU
    out["ds0"] = dS
    # per-chunk gradients
    for c, (a, b, xs, o) in enumerate(chunks):
        n = b - a
        S, dSp, U, dU = Ss[c], dSs[c], Us[c], dUs[c]
        dO = xs[5] * xs[6]
        dQd, dW, dKb = dO @ S.T, -dU @ S.T, U @ dSp.T
        dgC = np.sum(dSp * S, axis=1)
        dP = np.tril(dO @ U.T)
        dT = dU @ xs[2].T + dW @ o["Kd"].T
        M = o["X"].T @ dT * xs[4][None, :]
        dL = np.tril(-M @ o["X"].T, -1)
        dbeta = np.sum(o["X"] * dT, axis=0) + np.sum(dL * o["A"], axis=1)
        dA = xs[4][:, None] * dL
        dKd = o["T"].T @ dW + dA @ o["Ki"]
        dKi = dA.T @ o["Kd"] + dP.T @ o["Qd"]
        dQd = dQd + dP @ o["Ki"]
        dG = dKd * o["Kd"] - dKi * o["Ki"] + dQd * o["Qd"] - dKb * o["Kb"]
        dG[-1] += np.sum(dKb * o["Kb"], axis=0) + dgC * o["gC"]
        E = np.exp(o["G"])
        out["dq"][a:b] = (scale * dQd * E)[:n]
        out["dk"][a:b] = (dKd * E + dKi / E + dKb * o["Fb"])[:n]
        out["dv"][a:b] = (o["T"].T @ dU)[:n]
        out["dg"][a:b] = np.cumsum(dG[::-1], axis=0)[::-1][:n]
        out["dbeta"][a:b] = dbeta[:n]
    return out


@pytest.mark.parametrize("L,dk,dv,seed", [(1, 4, 3, 0), (16, 6, 5, 1), (37, 8, 6, 2), (50, 5, 7, 3),
                                          (64, 8, 8, 4)])
def test_chunk_form_gradient_equals_per_token_gradient(L, dk, dv, seed):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=1, keepdims=True)
    q, k = unit(rng.standard_normal((L, dk))), unit(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    g = np.maximum(-np.logaddexp(0.0, 2.0 * rng.standard_normal((L, dk))), np.log(0.0067))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    gate = 1.0 / (1.0 + np.exp(-rng.standard_normal((L, dv))))
    dy = rng.standard_normal((L, dv))
    s0, dsT = 0.1 * rng.standard_normal((dk, dv)), rng.standard_normal((dk, dv))
    ref = B.head_backward(q, k, v, g, beta, gate, dy, s0, dsT, 0.7)
    got = chunk_backward(q, k, v, g, beta, gate, dy, s0, dsT, 0.7)
    for name in ref:
        err = np.abs(got[name] - ref[name]).max() / max(1.0, np.abs(ref[name]).max())
        assert err < 1e-12, (name, err)
