"""KDA context parallelism over ranks: each rank holds one segment of every
sequence (rank r the r-th), in rank order along the sequence.

Per rank: the affine map of its segment (transition M, dk x dk, and the state
Z its tokens produce from zero, dk x dv, per sequence and head); one
all-gather of the packed [M | Z] of all ranks; the incoming state of rank r is
the initial state folded through the maps of ranks 0 .. r-1; then the plain
prefill of its segment from that state.  The exchange is fixed-size --
H * dk * (dk + dv) * 4 bytes per sequence, whatever the segment length --
which is the point of the scheme (affta.cn K3 explainer, section
"KDA 上下文并行，让上下文的交接变薄"; prism.simon-ai.net, section
"Linear Attention 的分层 Chunking 策略").

The kernels come from `backend` (default: the CUDA library through kda.py);
the collective is torch.distributed's all_gather on `group`.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import kda


class CudaBackend:
    """The three steps on the GPU through the C ABI."""

    @staticmethod
    def summary(k, v, g, beta, cu_seqlens, cu_seqlens_host, **flags):
        return kda.chunk_summary(k, v, g, beta, cu_seqlens, cu_seqlens_host=cu_seqlens_host,
                                 **flags)

    @staticmethod
    def compose(M, Z, state_in):
        return kda.state_compose(M, Z, state_in)

    @staticmethod
    def prefill(q, k, v, g, beta, gate, cu_seqlens, cu_seqlens_host, initial_state, **kw):
        return kda.chunk_fwd(q, k, v, g, beta, gate, cu_seqlens, cu_seqlens_host=cu_seqlens_host,
                             initial_state=initial_state, **kw)


def incoming_state(M_all, Z_all, rank, initial_state, backend=CudaBackend):
    """The state entering segment `rank`: initial_state folded through the maps
    of segments 0 .. rank-1 (M_all [R, N, H, dk, dk], Z_all [R, N, H, dk, dv])."""
    if rank == 0:
        return initial_state
    return backend.compose(M_all[:rank], Z_all[:rank], initial_state)


def kcp_chunk_fwd(q, k, v, g, beta, gate, cu_seqlens, *, cu_seqlens_host=None,
                  initial_state=None, group=None, backend=CudaBackend, scale=1.0,
                  qk_l2norm=False, beta_logits=False, gate_logits=False, clamp_decay=False):
    """Prefill of this rank's segments.  Shapes as kda.chunk_fwd, for the local
    tokens; initial_state [N, H, dk, dv] is the state before segment 0 (the
    same on every rank; None = zeros).  Returns (out, state after this rank's
    segments): on the last rank that state is the sequences' final state."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    flags = dict(qk_l2norm=qk_l2norm, beta_logits=beta_logits, clamp_decay=clamp_decay)
    M, Z = backend.summary(k, v, g, beta, cu_seqlens, cu_seqlens_host, **flags)
    dk = M.shape[-1]
    packed = torch.cat([M, Z], dim=-1).contiguous()  # [N, H, dk, dk + dv]
    # NCCL gathers the device tensors directly; a gloo group moves host copies
    via_host = packed.is_cuda and dist.get_backend(group) == "gloo"
    send = packed.cpu() if via_host else packed
    gathered = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(gathered, send, group=group)
    allp = torch.stack(gathered)                     # [R, N, H, dk, dk + dv]
    if via_host:
        allp = allp.to(packed.device)
    M_all, Z_all = allp[..., :dk].contiguous(), allp[..., dk:].contiguous()
    s_in = incoming_state(M_all, Z_all, rank, initial_state, backend)
    return backend.prefill(q, k, v, g, beta, gate, cu_seqlens, cu_seqlens_host, s_in, scale=scale,
                           gate_logits=gate_logits, **flags)
