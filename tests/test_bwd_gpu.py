"""The backward (kda_bwd) on the GPU, through the C ABI, against the fp64
backward oracle (oracle/backward.py) on identical inputs.

Tolerance: the kernels take the chunk form of the gradient to fp32 accuracy on
the dtype-rounded inputs (CUDA-core fp32, and tensor-core products whose
operands are split into two tf32 parts, leaving out terms below 2^-20
relative), and the gradients are fp32 outputs (no output rounding), so each
gradient gets the forward's fp32 bar scaled by its own magnitude:
max |err| <= 1e-4 * max(1, max |ref|).  A gradient entry sums O(dk + dv)
products per token and, through dS, contributions from the later tokens that
decay by exp(g) per step; fp32 rounding of those sums (relative error of
order 1e-6 per sum) stays well below this bar.
"""
import numpy as np
import pytest
import torch

from kda_linear_attention_fwd_b200 import kda, workloads as W
from oracle import backward as B
from tests.parity import np32

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dgate", "ds0")


def assert_grad_close(actual, expected, what):
    a = np.asarray(actual, dtype=np.float64)
    e = np.asarray(expected, dtype=np.float64)
    assert a.shape == e.shape, (what, a.shape, e.shape)
    assert np.isfinite(a).all(), f"{what}: non-finite values"
    if e.size == 0:
        return
    bar = 1e-4 * max(1.0, float(np.abs(e).max()))
    err = float(np.abs(a - e).max())
    assert err <= bar, f"{what}: max|err| {err:.3e} > {bar:.3e}"


def _grads_in(inp, dtype, seed, with_final=True):
    gen = torch.Generator().manual_seed(seed)
    T, H, dv = inp["v"].shape
    N = inp["cu_seqlens"].numel() - 1
    dk = inp["q"].shape[-1]
    dy = torch.randn(T, H, dv, generator=gen).to(inp["q"].dtype).to(inp["q"].device)
    dsf = torch.randn(N, H, dk, dv, generator=gen).to(inp["q"].device) if with_final else None
    return dy, dsf


def _oracle(inp, dy, dsf, scale, gate=True):
    return B.varlen_backward(np32(inp["q"]), np32(inp["k"]), np32(inp["v"]), np32(inp["g"]),
                             np32(inp["beta"]), np32(inp["gate"]) if gate else None,
                             inp["cu_seqlens"].tolist(), np32(dy),
                             initial_state=np32(inp["initial_state"]),
                             d_final_state=np32(dsf), scale=scale)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("bf16", 64, 128),
                                          ("f32", 64, 64), ("f32", 128, 64)])
def test_bwd_matches_oracle(cuda_lib, dtype, dk, dv):
    """Varlen with an empty, a one-partial-chunk and multi-chunk sequences
    (16-token chunks), initial state, final-state gradient and a gate."""
    w = W.custom(dtype=dtype, H=2, dk=dk, dv=dv, lengths=(0, 5, 64, 130, 300),
                 init_state=True, seed=91)
    inp = W.pack_prefill(w, device="cuda")
    dy, dsf = _grads_in(inp, dtype, seed=92)
    got = kda.bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"], dy,
                  inp["cu_seqlens"], scale=0.5, initial_state=inp["initial_state"],
                  d_final_state=dsf, cu_seqlens_host=inp["cu_seqlens"].tolist())
    torch.cuda.synchronize()
    ref = _oracle(inp, dy, dsf, 0.5)
    for name in NAMES:
        assert_grad_close(np32(got[name]), ref[name], name)


@pytest.mark.gpu
def test_bwd_without_gate_state_or_final_gradient(cuda_lib):
    w = W.custom(dtype="bf16", H=3, dk=128, dv=64, lengths=(200, 1, 77), seed=93)
    inp = W.pack_prefill(w, device="cuda")
    dy, _ = _grads_in(inp, "bf16", seed=94, with_final=False)
    got = kda.bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, dy,
                  inp["cu_seqlens"])
    torch.cuda.synchronize()
    assert got["dgate"] is None
    ref = _oracle(inp, dy, None, 1.0, gate=False)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "ds0"):
        assert_grad_close(np32(got[name]), ref[name], name)


@pytest.mark.gpu
def test_bwd_sampled_heads_full_size(cuda_lib):
    """The benchmark's backward workload (2 x 4096 tokens, H = 16, d = 128,
    bf16) in the launch the benchmark times; the oracle checks three sampled
    (sequence, head) pairs, which depend on nothing else."""
    w = W.get("prefill_bf16")
    inp = W.fast_prefill(w, seed=95, device="cuda")
    dy, dsf = _grads_in(inp, "bf16", seed=96)
    got = kda.bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"], dy,
                  inp["cu_seqlens"], d_final_state=dsf,
                  cu_seqlens_host=inp["cu_seqlens"].tolist())
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    for n, h in [(0, 0), (1, 7), (1, 15)]:
        a, b = cu[n], cu[n + 1]
        r = B.head_backward(*(np32(inp[x][a:b, h]) for x in ("q", "k", "v", "g", "beta", "gate")),
                            np32(dy[a:b, h]), None, np32(dsf[n, h]), 1.0)
        for name in NAMES:
            act = np32(got[name][n, h]) if name == "ds0" else np32(got[name][a:b, h])
            assert_grad_close(act, r[name], f"{name} (n={n}, h={h})")


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bwd_decay_at_the_floor(cuda_lib, dtype):
    """Every channel at the minimum retention in every token: the chunk form's
    decay factors exp(-G) reach about 6e34 inside a 16-token chunk, the widest
    range its fp32 products see; the gradients still match the oracle."""
    import math
    w = W.custom(dtype=dtype, H=2, dk=128, dv=128, lengths=(77, 130), init_state=True, seed=97)
    inp = W.pack_prefill(w, device="cuda")
    inp["g"] = torch.full_like(inp["g"], math.log(0.0067))
    dy, dsf = _grads_in(inp, dtype, seed=98)
    got = kda.bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["gate"], dy,
                  inp["cu_seqlens"], scale=0.5, initial_state=inp["initial_state"],
                  d_final_state=dsf, cu_seqlens_host=inp["cu_seqlens"].tolist())
    torch.cuda.synchronize()
    ref = _oracle(inp, dy, dsf, 0.5)
    for name in NAMES:
        assert_grad_close(np32(got[name]), ref[name], name)
