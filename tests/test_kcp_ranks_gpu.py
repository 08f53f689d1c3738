"""KDA context parallelism across ranks with the CUDA kernels: two processes
on cuda:0 joined by a gloo group run kcp.kcp_chunk_fwd with its default
backend (the C ABI): each computes the affine map of its segment of every
sequence, the maps are all-gathered, each rank folds the maps before its
own into its incoming state and runs the prefill of its segment.  The
segments' outputs and the last rank's final state must equal the fp64 oracle
over the whole sequences at the bf16 bar (affta.cn K3 explainer, section
"KDA 上下文并行，让上下文的交接变薄").

The ranks' kernels never wait on one another (the exchange is a host-side
gloo collective), so sharing one GPU is safe.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

# segment r of sequence n: tokens [BOUNDS[n][r], BOUNDS[n][r + 1]); the cuts
# are not chunk-aligned, and the second sequence's first segment is short
LENGTHS = (1700, 900, 40)
BOUNDS = [(0, 1000, 1700), (0, 333, 900), (0, 40, 40)]


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    sys.path.insert(0, ROOT)
    from kda_linear_attention_fwd_b200 import workloads as W
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=LENGTHS, init_state=True, seed=91)
    return W.pack_prefill(w, device="cpu")


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
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=timedelta(seconds=120))
    from kda_linear_attention_fwd_b200 import kcp
    inp = _inputs()
    seg, ix = _segment(inp, rank)
    dev = {x: t.cuda() for x, t in seg.items()}
    y, S = kcp.kcp_chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["gate"],
                             dev["cu_seqlens"], cu_seqlens_host=seg["cu_seqlens"].tolist(),
                             initial_state=inp["initial_state"].cuda())
    torch.cuda.synchronize()
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ix.numpy(), y.float().cpu().numpy(), S.float().cpu().numpy()))


def test_kcp_cuda_backend_two_ranks_match_the_whole_sequence(cuda_lib):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import assert_close, round_to
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=600) for _ in range(2)), key=lambda x: x[0])
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    import oracle
    inp = _inputs()
    f = lambda t: t.float().numpy()
    y_ref, S_ref, _ = oracle.varlen(*(f(inp[x]) for x in ("q", "k", "v", "g", "beta", "gate")),
                                    inp["cu_seqlens"].tolist(),
                                    initial_state=f(inp["initial_state"]))
    y = np.zeros_like(y_ref)
    for rank, ix, y_r, S_r in res:
        y[ix] = y_r
    assert_close(y, round_to(y_ref, "bf16"), "bf16", "kcp y")
    assert_close(res[-1][3], S_ref, "bf16", "kcp final state")
