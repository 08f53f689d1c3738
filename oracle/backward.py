"""Gradient of the KDA forward, fp64 NumPy.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The CUDA library shares no code with it.

The pages give the forward only: the per-token order "forget, corrective
write with an update strength, read, output gate" (Kimi K3 report explainer,
affta.cn, section "第一关：KDA 解决算得动").  Nothing on them states a gradient,
so this module derives it from that recurrence by the chain rule, one forward
step at a time, and nothing else:

  forward, token t (S = S_{t-1} on entry, alpha = exp(g_t)):
    S'  = Diag(alpha) S                 (forget)
    a   = S'^T k_t                       (read with the key)
    u   = beta_t (v_t - a)               (error, scaled by the update strength)
    S_t = S' + k_t u^T                   (corrective write)
    o   = S_t^T (scale q_t)              (read)
    y_t = gate_t (.) o                   (output gate; no gate: y_t = o)

  reverse, token t, with dS = dL/dS_t from the later tokens (dL/dS_L = the
  gradient of the final state) and the loss L = sum dy (.) y + sum dS_L (.) S_L:
    do      = gate_t (.) dy_t            dgate_t = dy_t (.) o
    dS     += scale q_t do^T             dq_t    = scale S_t do
    du      = dS^T k_t                   dk_t    = dS u
    dv_t    = beta_t du                  dbeta_t = du . (v_t - a)
    da      = -beta_t du
    dS'     = dS + k_t da^T              dk_t   += S' da
    dg_t    = rowsum(dS' (.) S')         (d alpha = rowsum(dS' (.) S); alpha = exp(g))
    dS      = Diag(alpha) dS'            (= dL/dS_{t-1})

The states S_{t-1} come from a forward pass that keeps all of them (fine at the
sizes the tests use).  Only the plain forward is covered: beta and gate as
given (no logits), no q/k normalisation, the delta-rule write.

Pinned (tests/test_oracle_bwd.py) by central finite differences of the same
loss on tiny inputs, by torch autograd through a separately written forward,
and by the reductions the derivation must respect (beta = 0 kills dk and dv).
"""
from __future__ import annotations

import numpy as np


def head_forward(q, k, v, g, beta, gate, s0, scale=1.0):
    """Per-token fp64 forward of one (sequence, head).  q, k, g [L, dk];
    v, gate [L, dv] (gate may be None); beta [L]; s0 [dk, dv] or None.
    Returns (y [L, dv], S_L [dk, dv], states [L, dk, dv] = S_{t-1} per t)."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    L, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if s0 is None else np.array(s0, dtype=np.float64)
    y = np.zeros((L, dv))
    states = np.zeros((L, dk, dv))
    for t in range(L):
        states[t] = S
        Sp = np.exp(g[t])[:, None] * S
        a = Sp.T @ k[t]
        u = beta[t] * (v[t] - a)
        S = Sp + np.outer(k[t], u)
        o = S.T @ (scale * q[t])
        y[t] = o if gate is None else np.asarray(gate[t], dtype=np.float64) * o
    return y, S, states


def head_backward(q, k, v, g, beta, gate, dy, s0=None, ds_final=None, scale=1.0):
    """Gradients of L = sum dy (.) y + sum ds_final (.) S_L for one (sequence,
    head).  Returns a dict of fp64 arrays: dq, dk, dg [L, dk]; dv, dgate
    [L, dv] (dgate None without a gate); dbeta [L]; ds0 [dk, dv]."""
    q, k, v, g, beta, dy = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta, dy))
    gate = None if gate is None else np.asarray(gate, dtype=np.float64)
    L, dk = q.shape
    dv = v.shape[1]
    _, _, states = head_forward(q, k, v, g, beta, gate, s0, scale)
    dS = np.zeros((dk, dv)) if ds_final is None else np.array(ds_final, dtype=np.float64)
    out = {x: np.zeros((L, dk)) for x in ("dq", "dk", "dg")}
    out["dv"] = np.zeros((L, dv))
    out["dgate"] = None if gate is None else np.zeros((L, dv))
    out["dbeta"] = np.zeros(L)
    for t in reversed(range(L)):
        alpha = np.exp(g[t])
        Sp = alpha[:, None] * states[t]
        a = Sp.T @ k[t]
        u = beta[t] * (v[t] - a)
        St = Sp + np.outer(k[t], u)
        o = St.T @ (scale * q[t])
        do = dy[t] if gate is None else gate[t] * dy[t]
        if gate is not None:
            out["dgate"][t] = dy[t] * o
        dS = dS + scale * np.outer(q[t], do)
        out["dq"][t] = scale * (St @ do)
        du = dS.T @ k[t]
        out["dv"][t] = beta[t] * du
        out["dbeta"][t] = du @ (v[t] - a)
        da = -beta[t] * du
        dSp = dS + np.outer(k[t], da)
        out["dk"][t] = dS @ u + Sp @ da
        out["dg"][t] = np.sum(dSp * Sp, axis=1)
        dS = alpha[:, None] * dSp
    out["ds0"] = dS
    return out


def varlen_backward(q, k, v, g, beta, gate, cu_seqlens, dy, *, initial_state=None,
                    d_final_state=None, scale=1.0):
    """Packed sequences: q, k, g [T, H, dk]; v, gate, dy [T, H, dv]; beta
    [T, H]; initial_state, d_final_state [N, H, dk, dv] or None.  Returns the
    gradients packed the same way (fp64); ds0 [N, H, dk, dv]."""
    q, k, v, g, beta, dy = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta, dy))
    gate = None if gate is None else np.asarray(gate, dtype=np.float64)
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu = [int(x) for x in cu_seqlens]
    N = len(cu) - 1
    res = {x: np.zeros((T, H, dk)) for x in ("dq", "dk", "dg")}
    res["dv"] = np.zeros((T, H, dv))
    res["dgate"] = None if gate is None else np.zeros((T, H, dv))
    res["dbeta"] = np.zeros((T, H))
    res["ds0"] = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        for h in range(H):
            r = head_backward(q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h], beta[a:b, h],
                              None if gate is None else gate[a:b, h], dy[a:b, h],
                              None if initial_state is None else initial_state[n, h],
                              None if d_final_state is None else d_final_state[n, h], scale)
            for x in ("dq", "dk", "dg", "dv"):
                res[x][a:b, h] = r[x]
            if gate is not None:
                res["dgate"][a:b, h] = r["dgate"]
            res["dbeta"][a:b, h] = r["dbeta"]
            res["ds0"][n, h] = r["ds0"]
    return res
