"""The extended entry points on the GPU, through the C ABI, against the fp64
oracle: in-kernel preprocessing (beta / gate given as logits, decay floor
clamp, q/k norms) and state snapshots every B tokens.

The oracle side applies the same preprocessing as a plain definition in fp64
(sigmoid, max with ln 0.0067) to the very inputs the GPU reads, then runs the
per-token recurrence.  A snapshot after m*B tokens of sequence n must equal the
oracle's final state over the first m*B tokens of that sequence.
"""
import math

import numpy as np
import pytest
import torch

from kda_linear_attention_fwd_b200 import kda, workloads as W
from tests.parity import assert_close, np32, round_to

import oracle

LN_FLOOR = math.log(0.0067)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, np.float64)))


def _logit_inputs(inp, dtype, seed):
    """Replace beta and gate by logits and push a fifth of g below the floor
    (all rounded to the input dtype)."""
    gen = torch.Generator().manual_seed(seed)
    dt = inp["q"].dtype
    T, H = inp["beta"].shape
    dv = inp["v"].shape[-1]
    out = dict(inp)
    out["beta"] = (1.5 * torch.randn(T, H, generator=gen)).to(dt).to(inp["q"].device)
    out["gate"] = torch.randn(T, H, dv, generator=gen).to(dt).to(inp["q"].device)
    g = inp["g"].cpu().float().clone()
    low = torch.rand(g.shape, generator=gen) < 0.2
    g[low] = -9.0
    out["g"] = g.to(dt).to(inp["q"].device)
    return out


def _preprocessed(inp):
    """fp64 beta, gate, g as the kernels see them after the flags."""
    beta = _sigmoid(np32(inp["beta"]))
    gate = _sigmoid(np32(inp["gate"]))
    g = np.maximum(np32(inp["g"]).astype(np.float64), LN_FLOOR)
    return beta, gate, g


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d,piece,sub", [("bf16", 128, None, None), ("bf16", 64, None, None),
                                              ("f32", 64, None, None), ("bf16", 128, 128, 4)])
def test_prefill_preprocessing_flags(cuda_lib, monkeypatch, dtype, d, piece, sub):
    """beta and gate as logits, g clamped at the floor, q/k normalised in the
    kernel (bf16 d=128: tcgen05 kernel; bf16 d=64: warp-MMA kernel; fp32: CUDA
    cores); the last case on a forced plan whose summary runs over sub-pieces."""
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
        monkeypatch.setenv("KDA_SUB_PIECES", str(sub))
    w = W.custom(dtype=dtype, H=2, dk=d, dv=d, lengths=(37, 300), init_state=True, seed=41)
    inp = _logit_inputs(W.pack_prefill(w, device="cuda"), dtype, seed=42)
    cu = inp["cu_seqlens"].tolist()
    y, S = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"],
                         inp["cu_seqlens"], initial_state=inp["initial_state"], qk_l2norm=True,
                         beta_logits=True, gate_logits=True, clamp_decay=True,
                         cu_seqlens_host=cu, scale=0.5)
    torch.cuda.synchronize()
    beta, gate, g = _preprocessed(inp)
    y_ref, S_ref, _ = oracle.varlen(np32(inp["q"]), np32(inp["k"]), np32(inp["v"]), g, beta,
                                    gate, cu, scale=0.5, qk_l2norm=True,
                                    initial_state=np32(inp["initial_state"]))
    assert_close(np32(y), round_to(y_ref, dtype), dtype, "y")
    assert_close(np32(S), S_ref, dtype, "final state")


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_decode_preprocessing_flags(cuda_lib, dtype, d):
    N, H, steps = 3, 2, 4
    gen = torch.Generator().manual_seed(51)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.nn.functional.normalize(torch.randn(steps, N, H, d, generator=gen), dim=-1).to(dt)
    k = torch.nn.functional.normalize(torch.randn(steps, N, H, d, generator=gen), dim=-1).to(dt)
    v = torch.randn(steps, N, H, d, generator=gen).to(dt)
    g = (-torch.nn.functional.softplus(2 * torch.randn(steps, N, H, d, generator=gen)))
    g[torch.rand(g.shape, generator=gen) < 0.2] = -9.0
    g = g.to(dt)
    beta = (1.5 * torch.randn(steps, N, H, generator=gen)).to(dt)
    gate = torch.randn(steps, N, H, d, generator=gen).to(dt)
    state0 = 0.02 * torch.randn(N, H, d, d, generator=gen)
    state = state0.cuda()
    ys = []
    for s in range(steps):
        ys.append(kda.decode_step(q[s].cuda(), k[s].cuda(), v[s].cuda(), g[s].cuda(),
                                  beta[s].cuda(), gate[s].cuda(), state, beta_logits=True,
                                  gate_logits=True, clamp_decay=True))
    torch.cuda.synchronize()
    y = torch.stack(ys).cpu().float().numpy()
    y_ref, S_ref, _ = oracle.steps(np32(q), np32(k), np32(v),
                                   np.maximum(np32(g).astype(np.float64), LN_FLOOR),
                                   _sigmoid(np32(beta)), _sigmoid(np32(gate)), np32(state0))
    assert_close(y, round_to(y_ref, dtype), dtype, "y")
    assert_close(np32(state), S_ref, dtype, "state")


def _snapshot_refs(inp, B):
    """Oracle state after every B tokens of each sequence (fp64), in the
    library's order."""
    cu = inp["cu_seqlens"].tolist()
    q, k, v, g, beta, gate = (np32(inp[x]) for x in ("q", "k", "v", "g", "beta", "gate"))
    s0 = np32(inp["initial_state"])
    refs = []
    for n in range(len(cu) - 1):
        a, L = cu[n], cu[n + 1] - cu[n]
        for m in range(1, (max(L, 1) - 1) // B + 1):
            e = a + m * B
            _, S, _ = oracle.varlen(q[a:e], k[a:e], v[a:e], g[a:e], beta[a:e], gate[a:e],
                                    [0, e - a], initial_state=None if s0 is None else s0[n:n + 1],
                                    want_y=False)
            refs.append(S[0])
    return np.stack(refs)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d,piece,sub", [("bf16", 128, None, None), ("bf16", 128, 256, None),
                                                ("bf16", 64, 256, None), ("f32", 64, 256, None),
                                                ("bf16", 128, 256, 2)])
def test_snapshots(cuda_lib, monkeypatch, dtype, d, piece, sub):
    """State snapshots every 64 tokens: single-piece and forced multi-piece
    plans (the snapshots of later pieces start from the scanned state), one of
    them with the summary over sub-pieces."""
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    if sub:
        monkeypatch.setenv("KDA_SUB_PIECES", str(sub))
    B = 64
    w = W.custom(dtype=dtype, H=2, dk=d, dv=d, lengths=(0, 5, 64, 300, 701), init_state=True,
                 seed=61)
    inp = W.pack_prefill(w, device="cuda")
    cu = inp["cu_seqlens"].tolist()
    y, S, snaps = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"],
                                inp["cu_seqlens"], initial_state=inp["initial_state"],
                                cu_seqlens_host=cu, snapshot_tokens=B)
    torch.cuda.synchronize()
    offs = kda.snapshot_offsets([cu[i + 1] - cu[i] for i in range(len(cu) - 1)], B)
    assert offs == [0, 0, 0, 0, 4, 14]
    ref = _snapshot_refs(inp, B)
    assert snaps.shape[0] == ref.shape[0] == offs[-1]
    assert_close(np32(snaps), ref, dtype, "snapshots")
    # the plain outputs are unchanged by asking for snapshots: the same call
    # without them, on the same 16-token kernels (the ones that take
    # snapshots), is bit-identical, and both match the oracle
    if dtype == "bf16" and d == 128:
        monkeypatch.setenv("KDA_PREFILL_IMPL", "tc5")
    y2, S2 = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"],
                           inp["cu_seqlens"], initial_state=inp["initial_state"],
                           cu_seqlens_host=cu)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(S, S2)
    monkeypatch.delenv("KDA_PREFILL_IMPL", raising=False)
    y_ref, S_ref, _ = oracle.varlen(*(np32(inp[x]) for x in ("q", "k", "v", "g", "beta", "gate")),
                                    cu, initial_state=np32(inp["initial_state"]))
    assert_close(np32(y), round_to(y_ref, dtype), dtype, "y with snapshots")
    assert_close(np32(S), S_ref, dtype, "final state with snapshots")
