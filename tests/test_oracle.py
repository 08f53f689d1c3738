"""Pins for the CPU oracle (no GPU).

Each test checks the fp64 per-token oracle against something fixed outside
it: a hand-worked example, a closed form the layer reduces to, an invariant
the pages state, or brute force on tiny sizes.  Together they catch a dropped
term, a wrong sign, a wrong order of forget / write / read, or a transposed
state.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import chunkwise

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(20251202)


def rand_inputs(L, dk, dv, *, rng=RNG, unit_k=True, g_floor=math.log(0.0067)):
    q = rng.standard_normal((L, dk)).astype(np.float32)
    k = rng.standard_normal((L, dk)).astype(np.float32)
    if unit_k:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, dv)).astype(np.float32)
    beta = (1 / (1 + np.exp(-rng.standard_normal(L)))).astype(np.float32)
    g = np.maximum(-np.log1p(np.exp(2 * rng.standard_normal((L, dk)))), g_floor).astype(np.float32)
    gate = (1 / (1 + np.exp(-rng.standard_normal((L, dv))))).astype(np.float32)
    return q, k, v, g, beta, gate


def test_hand_worked_example():
    """Three tokens worked by hand (tests/golden/kda_hand_example.json)."""
    with open(os.path.join(GOLDEN, "kda_hand_example.json")) as f:
        ex = json.load(f)
    g = np.log(np.array(ex["alpha"], dtype=np.float64))
    y, S = oracle.head(np.array(ex["q"]), np.array(ex["k"]), np.array(ex["v"]), g,
                       np.array(ex["beta"]), np.array(ex["gate"]))
    # fp32 input rounding of 0.6/0.8 and ln(alpha) bounds the agreement at ~1e-7
    np.testing.assert_allclose(y, np.array(ex["y"]), atol=1e-6, rtol=0)
    np.testing.assert_allclose(S, np.array(ex["final_state"]), atol=1e-6, rtol=0)


def test_read_after_write_returns_value():
    """beta = 1 and a unit key: reading the state with the key right after the
    write returns the new value exactly (the delta rule writes the error)."""
    L, dk, dv = 40, 16, 8
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    # exactly unit-norm keys: four channels of +-1/2
    k = np.zeros((L, dk), np.float32)
    for t in range(L):
        idx = RNG.choice(dk, 4, replace=False)
        k[t, idx] = RNG.choice([-0.5, 0.5], 4)
    beta = np.ones(L, np.float32)
    s0 = RNG.standard_normal((dk, dv)) * 0.3
    y, _ = oracle.head(k, k, v, g, beta, None, initial_state=s0)  # q_t = k_t
    np.testing.assert_allclose(y, v, atol=1e-12, rtol=0)


def test_linear_attention_closed_form():
    """No decay, no erase, beta = 1, zero state: plain causal linear attention
    y_t = gate_t * sum_{s<=t} (q_t . k_s) v_s."""
    L, dk, dv = 37, 12, 7
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv, unit_k=False)
    g = np.zeros_like(g)
    beta = np.ones_like(beta)
    y, _ = oracle.head(q, k, v, g, beta, gate, erase=False)
    ref = (np.tril(q.astype(np.float64) @ k.T.astype(np.float64)) @ v.astype(np.float64)) * gate
    np.testing.assert_allclose(y, ref, atol=1e-11, rtol=0)


def test_beta_zero_decay_only():
    """beta = 0: no write, the initial state only decays per channel:
    o_t = S0^T (q_t * exp(G_t)), S_L = Diag(exp(G_L)) S0, G_t = sum_{r<=t} g_r."""
    L, dk, dv = 29, 10, 6
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    beta = np.zeros_like(beta)
    s0 = RNG.standard_normal((dk, dv))
    y, S = oracle.head(q, k, v, g, beta, None, initial_state=s0)
    G = np.cumsum(g.astype(np.float64), axis=0)
    ref = (q * np.exp(G)) @ s0
    np.testing.assert_allclose(y, ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(S, np.exp(G[-1])[:, None] * s0, atol=1e-12, rtol=0)


def test_additive_write_decay_sum():
    """No erase, beta = 1, zero state: the per-channel cumulative-product decay
    sum y_t = sum_{s<=t} (sum_i q_t[i] k_s[i] prod_{s<r<=t} alpha_r[i]) v_s."""
    L, dk, dv = 23, 9, 5
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    beta = np.ones_like(beta)
    y, _ = oracle.head(q, k, v, g, beta, None, erase=False)
    a = np.exp(g.astype(np.float64))
    q, k, v = (x.astype(np.float64) for x in (q, k, v))
    ref = np.zeros((L, dv))
    for t in range(L):
        for s in range(t + 1):
            decay = np.prod(a[s + 1:t + 1], axis=0) if t > s else np.ones(dk)
            ref[t] += np.sum(q[t] * k[s] * decay) * v[s]
    np.testing.assert_allclose(y, ref, atol=1e-12, rtol=0)


def test_scalar_recurrence_brute_force():
    """dk = dv = 1: s_t = (1 - beta_t k_t^2) alpha_t s_{t-1} + beta_t k_t v_t,
    y_t = gate_t scale q_t s_t."""
    L = 50
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((L, 1)).astype(np.float32) for _ in range(3))
    g = -rng.random((L, 1)).astype(np.float32)
    beta = rng.random(L).astype(np.float32)
    gate = rng.random((L, 1)).astype(np.float32)
    s0 = np.array([[0.7]])
    y, S = oracle.head(q, k, v, g, beta, gate, scale=0.5, initial_state=s0)
    s = 0.7
    for t in range(L):
        kt, vt, bt = float(k[t, 0]), float(v[t, 0]), float(beta[t])
        s = (1 - bt * kt * kt) * math.exp(float(g[t, 0])) * s + bt * kt * vt
        assert abs(y[t, 0] - float(gate[t, 0]) * 0.5 * float(q[t, 0]) * s) < 1e-12
    assert abs(S[0, 0] - s) < 1e-12


@pytest.mark.parametrize("cut", [1, 15, 16, 17, 64, 99])
def test_split_state_invariance(cut):
    """Running [0, cut) then [cut, L) from the handed-over state equals one run
    (the hand-off carries exactly the state -- KDA context parallelism)."""
    L, dk, dv = 130, 16, 12
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    s0 = RNG.standard_normal((dk, dv)) * 0.1
    y, S = oracle.head(q, k, v, g, beta, gate, initial_state=s0)
    y1, S1 = oracle.head(q[:cut], k[:cut], v[:cut], g[:cut], beta[:cut], gate[:cut],
                         initial_state=s0)
    y2, S2 = oracle.head(q[cut:], k[cut:], v[cut:], g[cut:], beta[cut:], gate[cut:],
                         initial_state=S1)
    np.testing.assert_allclose(np.concatenate([y1, y2]), y, atol=1e-13, rtol=0)
    np.testing.assert_allclose(S2, S, atol=1e-13, rtol=0)


def test_segment_summary_is_affine():
    """A segment's effect on the state is S_out = M S_in + S_zero, where M is
    what the segment does to an incoming state (push the identity through with
    v = 0) and S_zero what it makes from zero; fixed size, whatever its length."""
    L, dk, dv = 75, 8, 6
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    s_in = RNG.standard_normal((dk, dv))
    _, S_full = oracle.head(q, k, v, g, beta, gate, initial_state=s_in)
    _, S_zero = oracle.head(q, k, v, g, beta, gate)
    _, M = oracle.head(q, k, np.zeros((L, dk), np.float32), g, beta, None,
                       initial_state=np.eye(dk))
    np.testing.assert_allclose(M @ s_in + S_zero, S_full, atol=1e-12, rtol=0)
    # and M is the ordered product of the per-token maps (I - b k k^T) Diag(alpha)
    Mp = np.eye(dk)
    for t in range(L):
        kt = k[t].astype(np.float64)
        Mp = (np.eye(dk) - float(beta[t]) * np.outer(kt, kt)) @ np.diag(np.exp(g[t])) @ Mp
    np.testing.assert_allclose(M, Mp, atol=1e-12, rtol=0)


@pytest.mark.parametrize("chunk", [1, 2, 4, 16, 64])
def test_chunk_size_invariance(chunk):
    """The chunkwise form gives the per-token result for any chunk size
    (ragged last chunk, nonzero initial state)."""
    L, dk, dv = 150, 16, 12
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    s0 = RNG.standard_normal((dk, dv)) * 0.2
    y, S = oracle.head(q, k, v, g, beta, gate, scale=0.75, initial_state=s0)
    yc, Sc = chunkwise.head(q, k, v, g, beta, gate, chunk=chunk, scale=0.75, initial_state=s0)
    np.testing.assert_allclose(yc, y, atol=1e-10, rtol=0)
    np.testing.assert_allclose(Sc, S, atol=1e-10, rtol=0)


def test_decay_floor_keeps_chunk_ratios_finite():
    """At the floor every channel keeps >= 0.67% per step, so over a 16-token
    chunk exp(-G) <= 0.0067^-16 stays below the bf16/fp32 maximum, and a run
    pinned at the floor stays finite in the chunk form."""
    assert 16 * -math.log(0.0067) < math.log(3.3895e38)
    L, dk, dv = 64, 8, 8
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    g[:] = np.float32(math.log(0.0067))
    yc, Sc = chunkwise.head(q, k, v, g, beta, gate, chunk=16)
    y, S = oracle.head(q, k, v, g, beta, gate)
    assert np.isfinite(yc).all() and np.isfinite(Sc).all()
    np.testing.assert_allclose(yc, y, atol=1e-10, rtol=0)


def test_contraction_without_values():
    """v = 0, unit keys, beta in [0, 1]: each token maps S through
    (I - beta k k^T) Diag(alpha), a contraction, so ||S||_F never grows."""
    L, dk, dv = 60, 12, 10
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    s = RNG.standard_normal((dk, dv))
    norms = [np.linalg.norm(s)]
    for t in range(L):
        _, s = oracle.head(q[t:t + 1], k[t:t + 1], np.zeros((1, dv), np.float32), g[t:t + 1],
                           beta[t:t + 1], None, initial_state=s)
        norms.append(np.linalg.norm(s))
    assert all(b <= a * (1 + 1e-12) for a, b in zip(norms, norms[1:]))


def test_gate_and_scale_are_elementwise():
    L, dk, dv = 33, 8, 8
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv)
    y_none, S_none = oracle.head(q, k, v, g, beta, None)
    y_ones, _ = oracle.head(q, k, v, g, beta, np.ones_like(gate))
    y_gate, S_gate = oracle.head(q, k, v, g, beta, gate)
    y_half, _ = oracle.head(q, k, v, g, beta, gate, scale=0.5)
    assert np.array_equal(y_none, y_ones)
    np.testing.assert_allclose(y_gate, gate * y_none, atol=1e-14, rtol=0)
    np.testing.assert_allclose(y_half, 0.5 * y_gate, atol=1e-14, rtol=0)
    assert np.array_equal(S_none, S_gate)


def test_qk_l2norm_flag():
    L, dk, dv = 20, 8, 4
    q, k, v, g, beta, gate = rand_inputs(L, dk, dv, unit_k=False)
    y1, S1 = oracle.head(q, k, v, g, beta, gate, qk_l2norm=True)
    qn = q / np.sqrt((q.astype(np.float64) ** 2).sum(1, keepdims=True) + 1e-6)
    kn = k / np.sqrt((k.astype(np.float64) ** 2).sum(1, keepdims=True) + 1e-6)
    # normalised inputs rounded to fp32 on the way in: agreement at ~1e-7
    y2, S2 = oracle.head(qn, kn, v, g, beta, gate)
    np.testing.assert_allclose(y1, y2, atol=5e-6, rtol=0)
    np.testing.assert_allclose(S1, S2, atol=5e-6, rtol=0)


def test_varlen_packing_matches_separate_runs():
    """Chunks and states never cross a sequence boundary."""
    dk, dv, H = 8, 6, 3
    lens = [5, 0, 17, 1, 33]
    T = sum(lens)
    q = RNG.standard_normal((T, H, dk)).astype(np.float32)
    k = RNG.standard_normal((T, H, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = RNG.standard_normal((T, H, dv)).astype(np.float32)
    g = -RNG.random((T, H, dk)).astype(np.float32)
    beta = RNG.random((T, H)).astype(np.float32)
    gate = RNG.random((T, H, dv)).astype(np.float32)
    s0 = RNG.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    y, S, _ = oracle.varlen(q, k, v, g, beta, gate, cu, initial_state=s0)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        for h in range(H):
            yh, Sh = oracle.head(q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h], beta[a:b, h],
                                 gate[a:b, h], initial_state=s0[n, h])
            np.testing.assert_array_equal(y[a:b, h], yh)
            np.testing.assert_array_equal(S[n, h], Sh)
    # an empty sequence hands its initial state straight through
    np.testing.assert_array_equal(S[1], s0[1])


def test_step_layout_matches_varlen():
    """The decode-step layout runs the same recurrence as the packed layout."""
    steps, N, H, dk, dv = 7, 3, 2, 8, 4
    q = RNG.standard_normal((steps, N, H, dk)).astype(np.float32)
    k = RNG.standard_normal((steps, N, H, dk)).astype(np.float32)
    v = RNG.standard_normal((steps, N, H, dv)).astype(np.float32)
    g = -RNG.random((steps, N, H, dk)).astype(np.float32)
    beta = RNG.random((steps, N, H)).astype(np.float32)
    gate = RNG.random((steps, N, H, dv)).astype(np.float32)
    s0 = RNG.standard_normal((N, H, dk, dv))
    y, S, _ = oracle.steps(q, k, v, g, beta, gate, s0)
    for n in range(N):
        for h in range(H):
            yh, Sh = oracle.head(q[:, n, h], k[:, n, h], v[:, n, h], g[:, n, h],
                                 beta[:, n, h], gate[:, n, h], initial_state=s0[n, h])
            np.testing.assert_array_equal(y[:, n, h], yh)
            np.testing.assert_array_equal(S[n, h], Sh)


def test_mask_selects_heads():
    steps, N, H, dk, dv = 3, 2, 2, 4, 4
    q, k, v = (RNG.standard_normal((steps, N, H, d)).astype(np.float32) for d in (dk, dk, dv))
    g = -RNG.random((steps, N, H, dk)).astype(np.float32)
    beta = RNG.random((steps, N, H)).astype(np.float32)
    s0 = RNG.standard_normal((N, H, dk, dv))
    mask = np.array([[True, False], [False, True]])
    y, S, _ = oracle.steps(q, k, v, g, beta, None, s0, mask=mask)
    yf, Sf, _ = oracle.steps(q, k, v, g, beta, None, s0)
    np.testing.assert_array_equal(y[:, mask], yf[:, mask])
    np.testing.assert_array_equal(S[mask], Sf[mask])
    assert not y[:, ~mask].any()
