"""Prefill parity: kda_chunk_fwd (through the C-ABI) vs the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from kda_linear_attention_fwd_b200 import kda
from kda_linear_attention_fwd_b200 import workloads as W
from parity import assert_close, np32, oracle_prefill, round_to

pytestmark = pytest.mark.gpu


def run(inp, *, scale=1.0, qk_l2norm=False, gate=True, alias=False, host_cu=True):
    s0 = inp.get("initial_state")
    kw = {}
    if alias:
        st = s0.clone() if s0 is not None else torch.zeros(
            inp["cu_seqlens"].numel() - 1, inp["q"].shape[1], inp["q"].shape[2],
            inp["v"].shape[2], device="cuda")
        kw = dict(initial_state=st, final_state=st)
    else:
        kw = dict(initial_state=s0)
    cu_host = inp["cu_seqlens"].tolist() if host_cu else None
    y, S = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                         inp["gate"] if gate else None, inp["cu_seqlens"], scale=scale,
                         qk_l2norm=qk_l2norm, cu_seqlens_host=cu_host, **kw)
    torch.cuda.synchronize()
    return np32(y), np32(S)


def compare(inp, y, S, yr, Sr, dtype, heads=None, what=""):
    cu = inp["cu_seqlens"].tolist()
    if heads is None:
        assert_close(y, round_to(yr, dtype), dtype, f"{what} y")
        assert_close(S, Sr, dtype, f"{what} final state")
        return
    ya, ye, sa, se = [], [], [], []
    for n, h in heads:
        ya.append(y[cu[n]:cu[n + 1], h])
        ye.append(round_to(yr[cu[n]:cu[n + 1], h], dtype))
        sa.append(S[n, h])
        se.append(Sr[n, h])
    assert_close(np.concatenate(ya), np.concatenate(ye), dtype, f"{what} y")
    assert_close(np.stack(sa), np.stack(se), dtype, f"{what} final state")


def test_tiny_fp32(cuda_lib):
    w = W.get("tiny_fp32")
    inp = W.pack_prefill(w, device="cuda")
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp)
    compare(inp, y, S, yr, Sr, "f32", what="tiny_fp32")


def test_prefill_bf16_all_heads(cuda_lib):
    w = W.get("prefill_bf16")
    inp = W.pack_prefill(w, device="cuda")
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp)
    compare(inp, y, S, yr, Sr, "bf16", what="prefill_bf16")


def test_varlen_bf16_sampled_heads(cuda_lib):
    w = W.get("varlen_bf16")
    heads = [(n, h) for n in range(w.num_seqs) for h in (0, 13, 31)]
    inp = W.pack_prefill(w, heads=heads, device="cuda")
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp, heads=heads)
    compare(inp, y, S, yr, Sr, "bf16", heads=heads, what="varlen_bf16")


def test_long_bf16_sampled_heads(cuda_lib):
    w = W.get("long_bf16")
    heads = [(0, 4), (0, 27)]
    inp = W.pack_prefill(w, heads=heads, device="cuda")
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp, heads=heads)
    compare(inp, y, S, yr, Sr, "bf16", heads=heads, what="long_bf16")


CASES = [
    # dtype, dk, dv, lengths, init, gate, l2norm, scale, forced piece length
    ("bf16", 64, 64, (1, 15, 16, 17, 100), True, True, False, 1.0, None),
    ("bf16", 128, 64, (300, 0, 33), True, False, False, 0.5, None),
    ("bf16", 64, 128, (513,), False, True, True, 1.0, None),
    ("f32", 128, 128, (40, 257), True, True, False, 1.0, None),
    ("bf16", 128, 128, (1000, 700, 5, 256), True, True, False, 1.0, 256),
    ("f32", 64, 64, (900, 31), True, True, False, 1.0, 256),
    ("f32", 128, 64, (2000, 1, 600), True, True, True, 0.8, 272),
    ("bf16", 64, 128, (4111,), True, True, False, 1.0, 512),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-{c[1]}x{c[2]}-{len(c[3])}seq-p{c[8]}"
                                             for c in CASES])
def test_custom_shapes(cuda_lib, monkeypatch, case):
    dtype, dk, dv, lengths, init, gate, l2, scale, piece = case
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    w = W.custom(dtype=dtype, H=3, dk=dk, dv=dv, lengths=lengths, init_state=init,
                 seed=100 + CASES.index(case))
    inp = W.pack_prefill(w, device="cuda")
    if l2:  # un-normalised q, k so that the in-kernel normalisation matters
        inp["q"] = (inp["q"].float() * 3.0).to(inp["q"].dtype)
        inp["k"] = (inp["k"].float() * 0.5).to(inp["k"].dtype)
    y, S = run(inp, scale=scale, qk_l2norm=l2, gate=gate)
    yr, Sr = oracle_prefill(inp, scale=scale, qk_l2norm=l2, gate=gate)
    compare(inp, y, S, yr, Sr, dtype, what=str(case))


@pytest.mark.parametrize("piece", [None, 256])
def test_final_state_may_alias_initial_state(cuda_lib, monkeypatch, piece):
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=(700, 300), init_state=True, seed=3)
    inp = W.pack_prefill(w, device="cuda")
    y1, S1 = run(inp)
    y2, S2 = run(inp, alias=True)
    assert np.array_equal(y1, y2)
    assert np.array_equal(S1, S2)


def test_without_host_offsets(cuda_lib, monkeypatch):
    """The same forced plan with and without the host copy of the offsets:
    identical results, both matching the oracle."""
    monkeypatch.setenv("KDA_PIECE_LEN", "256")
    w = W.custom(dtype="bf16", H=2, dk=64, dv=64, lengths=(600, 17), init_state=True, seed=11)
    inp = W.pack_prefill(w, device="cuda")
    y1, S1 = run(inp, host_cu=True)
    y2, S2 = run(inp, host_cu=False)
    assert np.array_equal(y1, y2) and np.array_equal(S1, S2)
    yr, Sr = oracle_prefill(inp)
    compare(inp, y2, S2, yr, Sr, "bf16", what="no host offsets")


def test_length_blind_plan_bf16_128_matches_oracle(cuda_lib):
    """bf16 dk = dv = 128 without the host copy of the offsets: the plan only
    knows the average length, so the longer sequences of the varlen workload
    are split into two pieces (summary, scan, output); one sampled head of
    every sequence against the oracle."""
    w = W.get("varlen_bf16")
    plan = kda.plan(w.total_tokens, w.num_seqs, w.H)
    assert max(w.lengths) > plan["piece_len"], plan  # some sequence has several pieces
    heads = [(n, 3 + 4 * n) for n in range(w.num_seqs)]
    inp = W.pack_prefill(w, heads=heads, device="cuda")
    y, S = run(inp, host_cu=False)
    yr, Sr = oracle_prefill(inp, heads=heads)
    compare(inp, y, S, yr, Sr, "bf16", heads=heads, what="length-blind plan")


SUB_CASES = [
    # lengths, forced piece length, sub-pieces per summarised piece
    ((3000, 700, 1, 1500), 512, 2),
    ((4111, 300, 0, 2049), 1024, 4),
    ((2600,), 768, 3),
]


@pytest.mark.parametrize("case", SUB_CASES, ids=[f"p{c[1]}-sub{c[2]}" for c in SUB_CASES])
def test_sub_pieces_match_oracle(cuda_lib, monkeypatch, case):
    """bf16, dk = dv = 128 with the summary pass over sub-pieces and the fold
    of their maps (forced plans: several pieces per sequence, partial last
    pieces, an empty and a one-token sequence, initial states): y and the
    final states against the oracle, identical with and without the host
    copy of the offsets."""
    lengths, piece, sub = case
    monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    monkeypatch.setenv("KDA_SUB_PIECES", str(sub))
    T, N, H = sum(lengths), len(lengths), 3
    assert kda.plan(T, N, H)["sub_pieces"] == sub
    w = W.custom(dtype="bf16", H=H, dk=128, dv=128, lengths=lengths, init_state=True,
                 seed=700 + SUB_CASES.index(case))
    inp = W.pack_prefill(w, device="cuda")
    y1, S1 = run(inp, host_cu=True)
    y2, S2 = run(inp, host_cu=False)
    assert np.array_equal(y1, y2) and np.array_equal(S1, S2)
    yr, Sr = oracle_prefill(inp)
    compare(inp, y1, S1, yr, Sr, "bf16", what=f"sub-pieces {case}")


def test_beta_zero_closed_form(cuda_lib):
    """beta = 0: o_t = S0^T (q_t exp(G_t)), S_L = Diag(exp G_L) S0 -- checked
    against the closed form itself, not the oracle."""
    w = W.custom(dtype="f32", H=2, dk=64, dv=64, lengths=(77, 160), init_state=True, seed=21)
    inp = W.pack_prefill(w, device="cuda")
    inp["beta"] = torch.zeros_like(inp["beta"])
    y, S = run(inp)
    cu = inp["cu_seqlens"].tolist()
    q, g, gate = np32(inp["q"]).astype(np.float64), np32(inp["g"]), np32(inp["gate"])
    s0 = np32(inp["initial_state"]).astype(np.float64)
    for n in range(2):
        for h in range(2):
            a, b = cu[n], cu[n + 1]
            G = np.cumsum(g[a:b, h].astype(np.float64), axis=0)
            ref = ((q[a:b, h] * np.exp(G)) @ s0[n, h]) * gate[a:b, h]
            assert np.abs(y[a:b, h] - ref).max() < 1e-4
            assert np.abs(S[n, h] - np.exp(G[-1])[:, None] * s0[n, h]).max() < 1e-5


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decay_at_the_floor_stays_finite(cuda_lib, monkeypatch, dtype):
    """Every channel at the minimum retention in every token: the largest
    decay ratios a 16-token chunk can hold.  Outputs stay finite and match."""
    monkeypatch.setenv("KDA_PIECE_LEN", "256")
    w = W.custom(dtype=dtype, H=2, dk=128, dv=128, lengths=(530,), init_state=True, seed=5)
    inp = W.pack_prefill(w, device="cuda")
    inp["g"] = torch.full_like(inp["g"], math.log(0.0067))
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp)
    compare(inp, y, S, yr, Sr, dtype, what="floor")


def test_device_error_word_stays_clear(cuda_lib, monkeypatch):
    """Bounded device waits record a failure in the workspace header (int32 at
    byte 8); a normal call leaves it zero."""
    monkeypatch.setenv("KDA_PIECE_LEN", "256")
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=(700, 33), init_state=True, seed=12)
    inp = W.pack_prefill(w, device="cuda")
    T, H = inp["q"].shape[:2]
    ws = torch.full((kda.workspace_size(T, 2, H, 128, 128),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"],
                  inp["cu_seqlens"], initial_state=inp["initial_state"], workspace=ws)
    torch.cuda.synchronize()
    header = ws[:16].view(torch.int32).cpu().tolist()
    assert header[2] == 0 and header[1] == 0 and header[0] > 2
