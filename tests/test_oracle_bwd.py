"""Pins of the backward oracle (oracle/backward.py), CPU only.

The gradient is not on the pages; the oracle derives it from the forward
recurrence by the chain rule.  These tests tie it to things other than its own
formulas: the C forward oracle (its forward must be the same layer), central
finite differences of the loss, torch autograd through a forward written here
with torch ops, and closed forms of reduced cases.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as B


def _rand_head(rng, L, dk, dv, gate=True):
    q = rng.standard_normal((L, dk)) / np.sqrt(dk)
    k = rng.standard_normal((L, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, dv))
    g = -rng.uniform(0.05, 1.0, (L, dk))
    beta = rng.uniform(0.2, 0.9, L)
    gt = rng.uniform(0.1, 0.9, (L, dv)) if gate else None
    return q, k, v, g, beta, gt


def test_forward_is_the_c_oracle():
    rng = np.random.default_rng(3)
    q, k, v, g, beta, gate = (None if x is None else x.astype(np.float32)
                              for x in _rand_head(rng, 37, 8, 6))
    s0 = rng.standard_normal((8, 6)).astype(np.float32)
    y, S, _ = B.head_forward(q, k, v, g, beta, gate, s0, scale=0.7)
    y_c, S_c = oracle.head(q, k, v, g, beta, gate, scale=0.7, initial_state=s0)
    np.testing.assert_allclose(y, y_c, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_c, rtol=1e-12, atol=1e-12)


def _loss(q, k, v, g, beta, gate, s0, dy, dsf, scale):
    y, S, _ = B.head_forward(q, k, v, g, beta, gate, s0, scale)
    return float(np.sum(dy * y) + np.sum(dsf * S))


@pytest.mark.parametrize("gate", [True, False])
def test_finite_differences(gate):
    """Every gradient entry against a central difference of the loss."""
    rng = np.random.default_rng(11)
    L, dk, dv, scale = 5, 3, 2, 0.8
    q, k, v, g, beta, gt = _rand_head(rng, L, dk, dv, gate)
    s0 = rng.standard_normal((dk, dv))
    dy = rng.standard_normal((L, dv))
    dsf = rng.standard_normal((dk, dv))
    grads = B.head_backward(q, k, v, g, beta, gt, dy, s0, dsf, scale)
    args = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "gate": gt, "s0": s0}
    names = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "beta": "dbeta", "gate": "dgate",
             "s0": "ds0"}
    eps = 1e-6
    for name, arr in args.items():
        if arr is None:
            assert grads[names[name]] is None
            continue
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            plus = {n: (a.copy() if a is not None else None) for n, a in args.items()}
            minus = {n: (a.copy() if a is not None else None) for n, a in args.items()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd[idx] = (_loss(**plus, dy=dy, dsf=dsf, scale=scale) -
                       _loss(**minus, dy=dy, dsf=dsf, scale=scale)) / (2 * eps)
        np.testing.assert_allclose(grads[names[name]], fd, rtol=1e-6, atol=1e-8,
                                   err_msg=f"d{name}")


def _torch_forward(q, k, v, g, beta, gate, s0, cu, scale):
    """The layer once more, with torch ops (autograd records it)."""
    ys, finals = [], []
    for n in range(len(cu) - 1):
        heads_y, heads_S = [], []
        for h in range(q.shape[1]):
            S = s0[n, h]
            rows = []
            for t in range(cu[n], cu[n + 1]):
                S = torch.exp(g[t, h]).unsqueeze(1) * S
                u = beta[t, h] * (v[t, h] - S.t() @ k[t, h])
                S = S + torch.outer(k[t, h], u)
                rows.append(gate[t, h] * (S.t() @ (scale * q[t, h])))
            heads_y.append(torch.stack(rows) if rows else q.new_zeros(0, v.shape[-1]))
            heads_S.append(S)
        ys.append(torch.stack(heads_y, 1))
        finals.append(torch.stack(heads_S))
    return torch.cat(ys, 0), torch.stack(finals)


def test_autograd_varlen():
    rng = np.random.default_rng(21)
    lengths, H, dk, dv, scale = (0, 7, 12), 2, 4, 3, 0.6
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    T, N = cu[-1], len(lengths)
    parts = [_rand_head(rng, T, dk, dv) for _ in range(H)]
    q, k, v, g, beta, gate = (np.stack([p[i] for p in parts], 1) for i in range(6))
    s0 = rng.standard_normal((N, H, dk, dv))
    dy = rng.standard_normal((T, H, dv))
    dsf = rng.standard_normal((N, H, dk, dv))
    ref = B.varlen_backward(q, k, v, g, beta, gate, cu, dy, initial_state=s0,
                            d_final_state=dsf, scale=scale)
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True)
          for x in (q, k, v, g, beta, gate, s0)]
    y, S = _torch_forward(*ts, cu, scale)
    loss = (y * torch.tensor(dy)).sum() + (S * torch.tensor(dsf)).sum()
    loss.backward()
    for t, name in zip(ts, ("dq", "dk", "dv", "dg", "dbeta", "dgate", "ds0")):
        np.testing.assert_allclose(ref[name], t.grad.numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=name)


def test_no_write_reductions():
    """beta = 0: nothing is written, so dk and dv vanish, and with dy = 0 the
    initial state's gradient is the final one decayed by exp(sum of g)."""
    rng = np.random.default_rng(31)
    L, dk, dv = 9, 5, 4
    q, k, v, g, _, gate = _rand_head(rng, L, dk, dv)
    beta = np.zeros(L)
    s0 = rng.standard_normal((dk, dv))
    dsf = rng.standard_normal((dk, dv))
    r = B.head_backward(q, k, v, g, beta, gate, rng.standard_normal((L, dv)), s0, dsf)
    assert not r["dk"].any() and not r["dv"].any()
    r0 = B.head_backward(q, k, v, g, beta, gate, np.zeros((L, dv)), s0, dsf)
    np.testing.assert_allclose(r0["ds0"], np.exp(g.sum(0))[:, None] * dsf, rtol=1e-13)
    assert not r0["dq"].any() and not r0["dgate"].any()
