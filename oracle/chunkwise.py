"""Chunk-parallel form of the KDA forward, fp64 NumPy.  TEST INFRASTRUCTURE ONLY.

A second CPU statement of the layer, independent of the per-token C oracle, in
the block-recurrent shape the pages describe: work inside a chunk is done with
whole-block matrix products, and only the state is carried from one chunk to
the next (prism.simon-ai.net, "从架构创新出发：K3的MoE与混合注意力设计",
section "计算范式演进：从递归低效到 GPU 友好的 Chunk Recurrent").  The decay
is applied as an absolute-position transform -- multiply the query/key side
by the cumulative decay and the other key side by its inverse, so that the
relative decay between two tokens of a chunk becomes a matrix product
(same page, section "数值稳定性与 Co-Design：BF16 约束下的衰减控制策略").

For a chunk of tokens r = 1..C (C may be anything; the result must not
depend on it -- same page, section "Linear Attention 的分层 Chunking 策略")
with incoming state S0:

    G_r  = g_1 + ... + g_r                       (per channel, inclusive)
    Qd   = (scale q) * exp(G)       Kd = k * exp(G)
    Ki   = k * exp(-G)              Kb = k * exp(G_C - G)
    A    = strictly-lower(Kd Ki^T)  (A[r,s] = sum_i k_r[i] k_s[i] exp(G_r[i]-G_s[i]), s<r)
    T    = (I + Diag(beta) A)^-1
    W    = T Diag(beta) Kd          U0 = T Diag(beta) V
    U    = U0 - W S0                (row r of U is the delta-rule update u_r)
    P    = lower(Qd Ki^T)           (diagonal included)
    O    = Qd S0 + P U              Y = gate * O
    S1   = Diag(exp(G_C)) S0 + Kb^T U

Why: unrolling S_r = Diag(a_r) S_{r-1} + k_r u_r^T inside the chunk gives
S_r = Diag(exp G_r) S0 + sum_{s<=r} Diag(exp(G_r - G_s)) k_s u_s^T.  Putting
that into u_r = beta_r (v_r - S_r'^T k_r), where S_r' is the state after the
forget of token r and before its write, gives
u_r + beta_r sum_{s<r} A[r,s] u_s = beta_r (v_r - S0^T Kd_r), i.e.
(I + Diag(beta) A) U = Diag(beta)(V - Kd S0); the read o_r = S_r^T (scale q_r)
gives O; S_C gives S1.
"""
from __future__ import annotations

import numpy as np


def chunk_step(q, k, v, g, beta, gate, S0, scale=1.0):
    """One chunk (rows are tokens).  Returns (Y [C, dv], S1 [dk, dv])."""
    q = np.asarray(q, np.float64) * scale
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    C = q.shape[0]
    G = np.cumsum(g, axis=0)
    Qd = q * np.exp(G)
    Kd = k * np.exp(G)
    Ki = k * np.exp(-G)
    Kb = k * np.exp(G[-1][None, :] - G)
    A = np.tril(Kd @ Ki.T, -1)
    T = np.linalg.inv(np.eye(C) + beta[:, None] * A)
    W = T @ (beta[:, None] * Kd)
    U0 = T @ (beta[:, None] * v)
    U = U0 - W @ S0
    P = np.tril(Qd @ Ki.T)
    O = Qd @ S0 + P @ U
    Y = O if gate is None else np.asarray(gate, np.float64) * O
    S1 = np.exp(G[-1])[:, None] * S0 + Kb.T @ U
    return Y, S1


def head(q, k, v, g, beta, gate=None, *, chunk=16, scale=1.0, initial_state=None):
    """One (sequence, head) in chunks of ``chunk`` tokens (last chunk partial).
    Returns (y [L, dv], S [dk, dv]) in fp64."""
    q = np.asarray(q)
    L, dk = q.shape
    dv = np.asarray(v).shape[-1]
    S = np.zeros((dk, dv)) if initial_state is None else np.array(initial_state, np.float64)
    y = np.zeros((L, dv))
    for t0 in range(0, L, chunk):
        t1 = min(L, t0 + chunk)
        gt = None if gate is None else np.asarray(gate)[t0:t1]
        y[t0:t1], S = chunk_step(q[t0:t1], np.asarray(k)[t0:t1], np.asarray(v)[t0:t1],
                                 np.asarray(g)[t0:t1], np.asarray(beta)[t0:t1], gt, S, scale)
    return y, S
