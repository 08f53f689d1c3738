"""Decode parity: kda_decode_step (through the C-ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from kda_linear_attention_fwd_b200 import kda
from kda_linear_attention_fwd_b200 import workloads as W
from parity import assert_close, np32, oracle_prefill, round_to

pytestmark = pytest.mark.gpu


def run_steps(d, steps, *, scale=1.0, qk_l2norm=False, gate=True, keep=None):
    """Run `steps` decode steps in place on a copy of d['state'].  keep: list
    of (n, h) whose outputs are kept (None = all).  Returns (y, state)."""
    state = d["state"].clone()
    ys = []
    for s in range(steps):
        y = kda.decode_step(d["q"][s], d["k"][s], d["v"][s], d["g"][s], d["beta"][s],
                            d["gate"][s] if gate else None, state, scale=scale,
                            qk_l2norm=qk_l2norm)
        if keep is None:
            ys.append(y.float().cpu())
        else:
            idx_n = torch.tensor([n for n, _ in keep], device=y.device)
            idx_h = torch.tensor([h for _, h in keep], device=y.device)
            ys.append(y[idx_n, idx_h].float().cpu())
    torch.cuda.synchronize()
    return torch.stack(ys).numpy(), np32(state)


def oracle_steps(d, steps, *, scale=1.0, qk_l2norm=False, gate=True, heads=None):
    sl = slice(0, steps)
    if heads is None:
        args = [np32(d[x][sl]) for x in ("q", "k", "v", "g", "beta")]
        gt = np32(d["gate"][sl]) if gate else None
        y, S, _ = oracle.steps(*args, gt, np32(d["state"]), scale=scale, qk_l2norm=qk_l2norm)
        return y, S
    n_idx = [n for n, _ in heads]
    h_idx = [h for _, h in heads]
    sub = {x: np32(d[x][sl][:, n_idx, h_idx])[:, :, None] for x in ("q", "k", "v", "g", "gate")}
    beta = np32(d["beta"][sl][:, n_idx, h_idx])[:, :, None]
    st = np32(d["state"][n_idx, h_idx])[:, None]
    y, S, _ = oracle.steps(sub["q"], sub["k"], sub["v"], sub["g"], beta,
                           sub["gate"] if gate else None, st, scale=scale, qk_l2norm=qk_l2norm)
    return y[:, :, 0], S[:, 0]


def test_decode_first_steps_all_heads(cuda_lib):
    w = W.get("decode_bf16")
    d = W.pack_decode(w, steps=10, device="cuda")
    y, S = run_steps(d, 10)
    yr, Sr = oracle_steps(d, 10)
    assert_close(y, round_to(yr, "bf16"), "bf16", "decode y, 10 steps x 8192 heads")
    assert_close(S, Sr, "bf16", "decode state after 10 steps")


def test_decode_1000_steps_sampled_heads(cuda_lib):
    w = W.get("decode_bf16")
    rng = np.random.default_rng(w.seed)
    flat = rng.choice(w.num_seqs * w.H, 64, replace=False)
    heads = sorted((int(i) // w.H, int(i) % w.H) for i in flat)
    d = W.pack_decode(w, heads=heads, device="cuda")
    y, S = run_steps(d, w.decode_steps, keep=heads)
    yr, Sr = oracle_steps(d, w.decode_steps, heads=heads)
    assert_close(y, round_to(yr, "bf16"), "bf16", "decode y, 1000 steps x 64 heads")
    S_sel = np.stack([S[n, h] for n, h in heads])
    assert_close(S_sel, Sr, "bf16", "decode state after 1000 steps")


DCASES = [("f32", 64, 64, False, True, 1.0), ("f32", 128, 64, True, False, 0.7),
          ("bf16", 64, 128, False, True, 1.0), ("f32", 128, 128, False, True, 1.0)]


@pytest.mark.parametrize("case", DCASES)
def test_decode_shapes(cuda_lib, case):
    dtype, dk, dv, l2, gate, scale = case
    w = W.Workload("dec", -1, dtype, 3, dk, dv, init_state=True, decode_steps=12,
                   num_seqs_decode=5, seed=300 + DCASES.index(case))
    d = W.pack_decode(w, device="cuda")
    if l2:
        d["q"] = d["q"] * 2.5
        d["k"] = d["k"] * 0.4
    y, S = run_steps(d, 12, scale=scale, qk_l2norm=l2, gate=gate)
    yr, Sr = oracle_steps(d, 12, scale=scale, qk_l2norm=l2, gate=gate)
    assert_close(y, round_to(yr, dtype), dtype, f"{case} y")
    assert_close(S, Sr, dtype, f"{case} state")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_steps_equal_prefill(cuda_lib, dtype):
    """L decode steps from S0 give the same outputs and state as one prefill
    over the same L tokens from S0."""
    N, H, dk, dv, L = 4, 2, 128, 128, 40
    w = W.Workload("dec", -1, dtype, H, dk, dv, init_state=True, decode_steps=L,
                   num_seqs_decode=N, seed=77)
    d = W.pack_decode(w, device="cuda")
    y_dec, S_dec = run_steps(d, L)
    # the same tokens, packed sequence-major: token t of sequence n is step t
    pk = {x: d[x].transpose(0, 1).reshape(N * L, *d[x].shape[2:]).contiguous()
          for x in ("q", "k", "v", "g", "beta", "gate")}
    cu = torch.arange(0, N * L + 1, L, dtype=torch.int32, device="cuda")
    y_pre, S_pre = kda.chunk_fwd(pk["q"], pk["k"], pk["v"], pk["g"], pk["beta"], pk["gate"], cu,
                                 initial_state=d["state"].clone())
    torch.cuda.synchronize()
    y_pre = np32(y_pre).reshape(N, L, H, dv).transpose(1, 0, 2, 3)
    assert_close(y_dec, y_pre, dtype, "decode vs prefill y")
    assert_close(S_dec, np32(S_pre), dtype, "decode vs prefill state")
    yr, Sr = oracle_steps(d, L)
    assert_close(y_pre, round_to(yr, dtype), dtype, "prefill vs oracle")
