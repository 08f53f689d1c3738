"""Parity of the 32-token tcgen05 prefill kernels (KDA_PREFILL_IMPL=c32:
bf16, dk = dv = 128, plain calls) against the fp64 oracle, through the C-ABI.

These kernels carry the state across 32-token chunks of two 16-token decay
tiles and compute the Gram blocks and W on the tensor cores; the library runs
the 16-token kernels by default, so every case here selects them explicitly.
Tolerances: bf16 max-abs <= 2e-2 and rel-L2 <= 1e-2 (y and final states).
"""
import math

import numpy as np
import pytest
import torch

from kda_linear_attention_fwd_b200 import kda
from kda_linear_attention_fwd_b200 import workloads as W
from parity import np32, oracle_prefill
from test_prefill_gpu import compare, run

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def chunk32(monkeypatch):
    monkeypatch.setenv("KDA_PREFILL_IMPL", "c32")


def test_plan_uses_32_token_pieces(cuda_lib):
    assert kda.plan(131072, 1, 32)["piece_len"] % 32 == 0


def test_prefill_bf16_all_heads(cuda_lib):
    w = W.get("prefill_bf16")
    inp = W.pack_prefill(w, device="cuda")
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp)
    compare(inp, y, S, yr, Sr, "bf16", what="c32 prefill_bf16")


def test_long_bf16_sampled_heads(cuda_lib):
    w = W.get("long_bf16")
    heads = [(0, 7), (0, 30)]
    inp = W.pack_prefill(w, heads=heads, device="cuda")
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp, heads=heads)
    compare(inp, y, S, yr, Sr, "bf16", heads=heads, what="c32 long_bf16")


def test_varlen_bf16_sampled_heads_without_host_offsets(cuda_lib):
    w = W.get("varlen_bf16")
    heads = [(n, h) for n in range(w.num_seqs) for h in (2, 29)]
    inp = W.pack_prefill(w, heads=heads, device="cuda")
    y, S = run(inp, host_cu=False)
    yr, Sr = oracle_prefill(inp, heads=heads)
    compare(inp, y, S, yr, Sr, "bf16", heads=heads, what="c32 varlen_bf16")


CASES = [
    # lengths, initial state, gate, scale, forced piece length
    ((1, 15, 16, 17, 31, 32, 33, 100), True, True, 1.0, None),
    ((300, 0, 65), False, False, 0.5, None),
    ((1000, 700, 5, 256), True, True, 1.0, 256),
    ((4111, 63), True, True, 0.8, 512),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{len(c[0])}seq-p{c[4]}" for c in CASES])
def test_custom_shapes(cuda_lib, monkeypatch, case):
    lengths, init, gate, scale, piece = case
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    w = W.custom(dtype="bf16", H=3, dk=128, dv=128, lengths=lengths, init_state=init,
                 seed=300 + CASES.index(case))
    inp = W.pack_prefill(w, device="cuda")
    y, S = run(inp, scale=scale, gate=gate)
    yr, Sr = oracle_prefill(inp, scale=scale, gate=gate)
    compare(inp, y, S, yr, Sr, "bf16", what="c32 " + str(case))


def test_decay_at_the_floor_stays_finite(cuda_lib, monkeypatch):
    """Every channel at the minimum retention: the largest ratios a 16-token
    tile holds, and products across the two tiles of a chunk underflow."""
    monkeypatch.setenv("KDA_PIECE_LEN", "256")
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=(530,), init_state=True, seed=305)
    inp = W.pack_prefill(w, device="cuda")
    inp["g"] = torch.full_like(inp["g"], math.log(0.0067))
    y, S = run(inp)
    yr, Sr = oracle_prefill(inp)
    compare(inp, y, S, yr, Sr, "bf16", what="c32 floor")


@pytest.mark.parametrize("piece", [None, 256])
def test_final_state_may_alias_initial_state(cuda_lib, monkeypatch, piece):
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=(700, 300), init_state=True, seed=306)
    inp = W.pack_prefill(w, device="cuda")
    y1, S1 = run(inp)
    y2, S2 = run(inp, alias=True)
    assert np.array_equal(y1, y2) and np.array_equal(S1, S2)


def test_device_error_word_stays_clear(cuda_lib, monkeypatch):
    monkeypatch.setenv("KDA_PIECE_LEN", "256")
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=(700, 33), init_state=True, seed=307)
    inp = W.pack_prefill(w, device="cuda")
    T, H = inp["q"].shape[:2]
    ws = torch.full((kda.workspace_size(T, 2, H, 128, 128),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"],
                  inp["cu_seqlens"], initial_state=inp["initial_state"], workspace=ws)
    torch.cuda.synchronize()
    header = ws[:16].view(torch.int32).cpu().tolist()
    assert header[2] == 0 and header[1] == 0 and header[0] > 2


@pytest.mark.parametrize("piece", [None, 256])
def test_summary_maps_match_oracle(cuda_lib, monkeypatch, piece):
    """The summary pass of the 32-token kernels (zero-start state and
    transition of every sequence) through kda_chunk_fwd_summary."""
    import oracle
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=(0, 40, 700), seed=308)
    inp = W.pack_prefill(w, device="cuda")
    M, Z = kda.chunk_summary(inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                             cu_seqlens_host=inp["cu_seqlens"].tolist())
    torch.cuda.synchronize()
    q, k, v, g, beta = (np32(inp[x]) for x in ("q", "k", "v", "g", "beta"))
    cu = inp["cu_seqlens"].tolist()
    eye = np.broadcast_to(np.eye(128), (3, 2, 128, 128)).copy()
    _, M_ref, _ = oracle.varlen(q, k, np.zeros_like(k), g, beta, None, cu, initial_state=eye,
                                want_y=False)
    _, Z_ref, _ = oracle.varlen(q, k, v, g, beta, None, cu, want_y=False)
    from parity import assert_close
    assert_close(np32(M), M_ref, "bf16", "c32 transition")
    assert_close(np32(Z), Z_ref, "bf16", "c32 zero-start state")
