"""Parity helpers shared by the GPU tests: tolerances and oracle drivers.

Tolerances (applied to outputs y and final states S, GPU vs fp64 oracle on
identical inputs):
  fp32 inputs           max |err| <= 1e-4
  bf16 inputs           max |err| <= 2e-2 and ||err||_2 / ||ref||_2 <= 1e-2
The oracle's y is rounded to the output dtype before comparison (the GPU
output is rounded to nearest-even in that dtype as well).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"f32": dict(max_abs=1e-4, rel_l2=None), "bf16": dict(max_abs=2e-2, rel_l2=1e-2)}


def errors(actual, expected):
    a = np.asarray(actual, dtype=np.float64)
    e = np.asarray(expected, dtype=np.float64)
    assert a.shape == e.shape, (a.shape, e.shape)
    assert np.isfinite(a).all(), "non-finite values in GPU result"
    d = a - e
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    den = float(np.linalg.norm(e))
    rel = float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def assert_close(actual, expected, dtype: str, what: str = ""):
    max_abs, rel = errors(actual, expected)
    t = TOL[dtype]
    assert max_abs <= t["max_abs"], f"{what}: max|err| {max_abs:.3e} > {t['max_abs']}"
    if t["rel_l2"] is not None:
        assert rel <= t["rel_l2"], f"{what}: rel-L2 {rel:.3e} > {t['rel_l2']}"
    return max_abs, rel


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16).to(torch.float32)
    return t.numpy().astype(np.float64)


def np32(t):
    return None if t is None else t.detach().to("cpu", torch.float32).numpy()


def oracle_prefill(inp: dict, *, scale=1.0, qk_l2norm=False, heads=None, gate=True):
    """fp64 oracle on the packed inputs (CPU copies).  heads: list of (n, h) or
    None for all.  Returns (y [T, H, dv], S [N, H, dk, dv]) in fp64."""
    cu = inp["cu_seqlens"].cpu().numpy()
    N = len(cu) - 1
    H = inp["q"].shape[1]
    mask = None
    if heads is not None:
        mask = np.zeros((N, H), bool)
        for n, h in heads:
            mask[n, h] = True
    s0 = np32(inp.get("initial_state"))
    y, S, _ = oracle.varlen(np32(inp["q"]), np32(inp["k"]), np32(inp["v"]), np32(inp["g"]),
                            np32(inp["beta"]), np32(inp["gate"]) if gate else None, cu,
                            scale=scale, qk_l2norm=qk_l2norm, initial_state=s0, mask=mask)
    return y, S
