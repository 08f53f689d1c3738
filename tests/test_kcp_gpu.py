"""Context parallelism on one GPU, through the C ABI, against the fp64 oracle:
the affine map of each sequence (kda_chunk_fwd_summary), and a sequence split
into segments whose incoming states come from folding the earlier segments'
maps (kda_state_compose) before the plain prefill of each segment.

Oracle side (plain definitions): the transition of a token run is the final
state of the recurrence started from the identity with v = 0 (dv = dk); the
zero-start state is the final state started from zeros.
"""
import numpy as np
import pytest
import torch

from kda_linear_attention_fwd_b200 import kda, workloads as W
from tests.parity import assert_close, np32, round_to

import oracle


def _oracle_map(inp):
    q, k, v, g, beta = (np32(inp[x]) for x in ("q", "k", "v", "g", "beta"))
    cu = inp["cu_seqlens"].tolist()
    N, H, dk = len(cu) - 1, k.shape[1], k.shape[2]
    eye = np.broadcast_to(np.eye(dk), (N, H, dk, dk)).copy()
    _, M, _ = oracle.varlen(q, k, np.zeros_like(k), g, beta, None, cu, initial_state=eye,
                            want_y=False)
    _, Z, _ = oracle.varlen(q, k, v, g, beta, None, cu, want_y=False)
    return M, Z


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d,piece", [("bf16", 128, None), ("bf16", 128, 256),
                                            ("bf16", 64, 256), ("f32", 64, 256)])
def test_summary_matches_oracle(cuda_lib, monkeypatch, dtype, d, piece):
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", str(piece))
    w = W.custom(dtype=dtype, H=2, dk=d, dv=d, lengths=(0, 40, 700), seed=71)
    inp = W.pack_prefill(w, device="cuda")
    M, Z = kda.chunk_summary(inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                             cu_seqlens_host=inp["cu_seqlens"].tolist())
    torch.cuda.synchronize()
    M_ref, Z_ref = _oracle_map(inp)
    assert_close(np32(M), M_ref, dtype, "transition")
    assert_close(np32(Z), Z_ref, dtype, "zero-start state")
    # the empty sequence has the identity map
    assert torch.equal(M[0].cpu(), torch.eye(d).expand(2, d, d))
    assert not Z[0].any()


def _segment(inp, bounds, r):
    """Packed inputs of segment r: tokens [bounds[n][r], bounds[n][r+1]) of
    every sequence n (positions within the sequence)."""
    cu = inp["cu_seqlens"].tolist()
    idx, cu_r = [], [0]
    for n in range(len(cu) - 1):
        a, b = cu[n] + bounds[n][r], cu[n] + bounds[n][r + 1]
        idx.extend(range(a, b))
        cu_r.append(cu_r[-1] + (b - a))
    ix = torch.tensor(idx, dtype=torch.long, device=inp["q"].device)
    seg = {x: inp[x].index_select(0, ix) for x in ("q", "k", "v", "g", "beta", "gate")}
    seg["cu_seqlens"] = torch.tensor(cu_r, dtype=torch.int32, device=inp["q"].device)
    return seg, ix


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_segments_fold_to_the_whole_sequence(cuda_lib, dtype, d):
    """Three segments per sequence (one of them empty): the folded incoming
    states make the segment prefills equal the whole-sequence oracle."""
    lengths = (300, 517)
    bounds = [(0, 100, 100, 300), (0, 256, 400, 517)]
    w = W.custom(dtype=dtype, H=2, dk=d, dv=d, lengths=lengths, init_state=True, seed=73)
    inp = W.pack_prefill(w, device="cuda")
    R = 3
    segs = [_segment(inp, bounds, r) for r in range(R)]
    maps = [kda.chunk_summary(s["k"], s["v"], s["g"], s["beta"], s["cu_seqlens"],
                              cu_seqlens_host=s["cu_seqlens"].tolist()) for s, _ in segs]
    M_all = torch.stack([m for m, _ in maps])
    Z_all = torch.stack([z for _, z in maps])
    y = torch.empty_like(inp["v"])
    state = inp["initial_state"]
    for r, (s, ix) in enumerate(segs):
        s_in = inp["initial_state"] if r == 0 else kda.state_compose(M_all[:r], Z_all[:r],
                                                                     inp["initial_state"])
        y_r, state = kda.chunk_fwd(s["q"], s["k"], s["v"], s["g"], s["beta"], s["gate"],
                                   s["cu_seqlens"], initial_state=s_in,
                                   cu_seqlens_host=s["cu_seqlens"].tolist())
        y.index_copy_(0, ix, y_r)
    # composing all three maps onto the initial state gives the final state too
    s_all = kda.state_compose(M_all, Z_all, inp["initial_state"])
    torch.cuda.synchronize()
    y_ref, S_ref, _ = oracle.varlen(np32(inp["q"]), np32(inp["k"]), np32(inp["v"]),
                                    np32(inp["g"]), np32(inp["beta"]), np32(inp["gate"]),
                                    inp["cu_seqlens"].tolist(),
                                    initial_state=np32(inp["initial_state"]))
    assert_close(np32(y), round_to(y_ref, dtype), dtype, "y")
    assert_close(np32(state), S_ref, dtype, "final state (last segment)")
    assert_close(np32(s_all), S_ref, dtype, "final state (folded maps)")


@pytest.mark.gpu
def test_compose_in_place_and_zero_maps(cuda_lib):
    N, H, d = 2, 3, 64
    gen = torch.Generator().manual_seed(5)
    M = torch.randn(2, N, H, d, d, generator=gen).cuda() / d ** 0.5
    Z = torch.randn(2, N, H, d, d, generator=gen).cuda()
    s0 = torch.randn(N, H, d, d, generator=gen).cuda()
    ref = s0.double()
    for i in range(2):
        ref = M[i].double() @ ref + Z[i].double()
    s = s0.clone()
    kda.state_compose(M, Z, s, out=s)  # in place
    assert torch.allclose(s.double(), ref, atol=1e-4, rtol=1e-4)
    copy = kda.state_compose(M[:0], Z[:0], s0)  # no maps: a copy
    assert torch.equal(copy, s0)
