"""KDA context parallelism across ranks (gloo, world size 2, CPU): the
orchestration in kcp.py -- segment maps, one all-gather, the fold into each
rank's incoming state -- with an fp64 oracle backend in place of the CUDA
kernels.  The segments' outputs and the last rank's final state must equal
the oracle over the whole sequences.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleBackend:
    """The three steps of kcp.py with the fp64 oracle on CPU tensors."""

    @staticmethod
    def summary(k, v, g, beta, cu_seqlens, cu_seqlens_host, **flags):
        import oracle
        cu = cu_seqlens.tolist()
        N, H, dk = len(cu) - 1, k.shape[1], k.shape[2]
        eye = np.broadcast_to(np.eye(dk), (N, H, dk, dk)).copy()
        kk, gg, bb = (x.numpy() for x in (k, g, beta))
        _, M, _ = oracle.varlen(kk, kk, np.zeros_like(kk), gg, bb, None, cu, initial_state=eye,
                                want_y=False)
        _, Z, _ = oracle.varlen(kk, kk, v.numpy(), gg, bb, None, cu, want_y=False)
        return torch.from_numpy(M), torch.from_numpy(Z)

    @staticmethod
    def compose(M, Z, state_in):
        s = torch.zeros_like(Z[0]) if state_in is None else state_in.double()
        for i in range(M.shape[0]):
            s = M[i] @ s + Z[i]
        return s

    @staticmethod
    def prefill(q, k, v, g, beta, gate, cu_seqlens, cu_seqlens_host, initial_state, **kw):
        import oracle
        s0 = None if initial_state is None else initial_state.numpy()
        y, S, _ = oracle.varlen(q.numpy(), k.numpy(), v.numpy(), g.numpy(), beta.numpy(),
                                gate.numpy(), cu_seqlens.tolist(), initial_state=s0)
        return torch.from_numpy(y), torch.from_numpy(S)


def _inputs():
    sys.path.insert(0, ROOT)
    from kda_linear_attention_fwd_b200 import workloads as W
    w = W.custom(dtype="f32", H=2, dk=16, dv=16, lengths=(40, 70), init_state=True, seed=81)
    return W.pack_prefill(w, device="cpu")


BOUNDS = [(0, 17, 40), (0, 48, 70)]  # segment r of sequence n: [BOUNDS[n][r], BOUNDS[n][r+1])


def _segment(inp, r):
    cu = inp["cu_seqlens"].tolist()
    idx, cu_r = [], [0]
    for n in range(len(cu) - 1):
        a, b = cu[n] + BOUNDS[n][r], cu[n] + BOUNDS[n][r + 1]
        idx.extend(range(a, b))
        cu_r.append(cu_r[-1] + b - a)
    ix = torch.tensor(idx, dtype=torch.long)
    seg = {x: inp[x].index_select(0, ix) for x in ("q", "k", "v", "g", "beta", "gate")}
    seg["cu_seqlens"] = torch.tensor(cu_r, dtype=torch.int32)
    return seg, ix


def _rank_main(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    from kda_linear_attention_fwd_b200 import kcp
    inp = _inputs()
    seg, ix = _segment(inp, rank)
    y, S = kcp.kcp_chunk_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"], seg["gate"],
                             seg["cu_seqlens"], initial_state=inp["initial_state"].double(),
                             backend=OracleBackend)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ix.numpy(), y.numpy(), S.numpy()))


def test_kcp_two_ranks_match_the_whole_sequence():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(2))
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    sys.path.insert(0, ROOT)
    import oracle
    inp = _inputs()
    y_ref, S_ref, _ = oracle.varlen(*(inp[x].numpy() for x in ("q", "k", "v", "g", "beta", "gate")),
                                    inp["cu_seqlens"].tolist(),
                                    initial_state=inp["initial_state"].numpy())
    y = np.zeros_like(y_ref)
    for rank, ix, y_r, S_r in res:
        y[ix] = y_r
    np.testing.assert_allclose(y, y_ref, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(res[-1][3], S_ref, rtol=1e-9, atol=1e-9)


def test_incoming_state_rank0_is_the_initial_state():
    sys.path.insert(0, ROOT)
    from kda_linear_attention_fwd_b200 import kcp
    s0 = torch.randn(1, 1, 4, 4, dtype=torch.float64)
    M = torch.randn(3, 1, 1, 4, 4, dtype=torch.float64)
    Z = torch.randn(3, 1, 1, 4, 4, dtype=torch.float64)
    assert kcp.incoming_state(M, Z, 0, s0, OracleBackend) is s0
    s2 = kcp.incoming_state(M, Z, 2, s0, OracleBackend)
    ref = M[1] @ (M[0] @ s0 + Z[0]) + Z[1]
    assert torch.allclose(s2, ref)
