"""Seeded synthetic inputs for the KDA forward workloads.

This module only draws random numbers and shapes them into the layer's
inputs; it holds none of the layer's arithmetic.  The CUDA tests, the oracle
tests and the benchmark all take their inputs from here, so both sides of a
parity check read the very same rounded values.

Workloads (sizes of the layer's prefill and decode use):

  tiny_fp32     1 x 256 tokens, H=2,  dk=dv=64,  fp32, zero initial state
  prefill_bf16  2 x 4096 tokens, H=16, dk=dv=128, bf16, zero initial state
  varlen_bf16   8 sequences, lengths uniform in [512, 8192] (seeded), H=32,
                dk=dv=128, bf16, initial states ~ N(0, 0.02^2) fp32
  long_bf16     1 x 131072 tokens, H=32, dk=dv=128, bf16; a fixed 25% of each
                head's key channels sit on the decay floor, the rest
                -softplus(N(0,1))
  decode_bf16   256 sequences x H=32, dk=dv=128, one bf16 token per sequence
                per step, 1000 steps, fp32 state ~ N(0, 0.02^2) updated in place

Value recipe (per token t and head h; drawn in fp32, then rounded once to the
workload dtype):
  q, k  ~ N(0, 1), then divided by their L2 norm over the head dimension
  v     ~ N(0, 1)
  beta  = sigmoid(N(0, 1))
  g     = log alpha = max(-softplus(2 N(0, 1)), ln 0.0067)   (decay floor: a
          channel keeps at least about 0.67% of its state per step)
  gate  = sigmoid(N(0, 1)), one value per output channel
Draw order per (sequence, head): q, k, v, beta, g, gate, [floor channels],
initial state.  Each (sequence, head) has its own generator seeded from the
workload seed, so any subset of heads can be regenerated alone.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import torch

LN_FLOOR = math.log(0.0067)
CHUNK = 16


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    dtype: str          # "f32" | "bf16"
    H: int
    dk: int
    dv: int
    lengths: tuple = field(default=())   # prefill: tokens per sequence
    init_state: bool = False
    g_mode: str = "standard"             # "standard" | "floor25"
    decode_steps: int = 0                # decode workloads: number of steps
    num_seqs_decode: int = 0
    seed: int = 0

    @property
    def is_decode(self) -> bool:
        return self.decode_steps > 0

    @property
    def num_seqs(self) -> int:
        return self.num_seqs_decode if self.is_decode else len(self.lengths)

    @property
    def total_tokens(self) -> int:
        return sum(self.lengths)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def cu_seqlens(self):
        cu = [0]
        for L in self.lengths:
            cu.append(cu[-1] + L)
        return cu


def _varlen_lengths(seed: int, n: int, lo: int, hi: int) -> tuple:
    gen = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen))


def _make(name: str) -> Workload:
    if name == "tiny_fp32":
        return Workload(name, 0, "f32", 2, 64, 64, lengths=(256,), seed=1000)
    if name == "prefill_bf16":
        return Workload(name, 1, "bf16", 16, 128, 128, lengths=(4096, 4096), seed=1001)
    if name == "varlen_bf16":
        return Workload(name, 2, "bf16", 32, 128, 128,
                        lengths=_varlen_lengths(1002, 8, 512, 8192), init_state=True,
                        seed=1002)
    if name == "long_bf16":
        return Workload(name, 3, "bf16", 32, 128, 128, lengths=(131072,), g_mode="floor25",
                        seed=1003)
    if name == "decode_bf16":
        return Workload(name, 4, "bf16", 32, 128, 128, init_state=True, decode_steps=1000,
                        num_seqs_decode=256, seed=1004)
    raise KeyError(name)


NAMES = ("tiny_fp32", "prefill_bf16", "varlen_bf16", "long_bf16", "decode_bf16")
WORKLOADS = {n: _make(n) for n in NAMES}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def custom(name="custom", *, dtype="bf16", H=2, dk=64, dv=64, lengths=(64,), init_state=False,
           g_mode="standard", seed=7) -> Workload:
    """A workload with the same value recipe at other sizes (tests)."""
    return Workload(name, -1, dtype, H, dk, dv, lengths=tuple(lengths), init_state=init_state,
                    g_mode=g_mode, seed=seed)


def _head_seed(seed: int, n: int, h: int) -> int:
    x = (seed * 0x9E3779B97F4A7C15 + (n + 1) * 0xBF58476D1CE4E5B9 + (h + 1) * 0x94D049BB133111EB)
    x &= (1 << 64) - 1
    x ^= x >> 31
    return x & ((1 << 63) - 1)


def _round(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(torch.bfloat16).to(torch.float32) if dtype == "bf16" else x


def _draw(gen, L, dk, dv, g_mode, with_init, dtype, device="cpu", heads=1):
    """Rows are [L // heads][heads] when heads > 1 (all heads of a packed
    tensor at once); with g_mode "floor25" every head then gets its own fixed
    subset of floor channels, as a per-head draw does."""
    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)

    q = randn(L, dk)
    q = q / q.norm(dim=-1, keepdim=True)
    k = randn(L, dk)
    k = k / k.norm(dim=-1, keepdim=True)
    v = randn(L, dv)
    beta = torch.sigmoid(randn(L))
    if g_mode == "floor25":
        g = -torch.nn.functional.softplus(randn(L, dk))
    else:
        g = torch.clamp_min(-torch.nn.functional.softplus(2.0 * randn(L, dk)), LN_FLOOR)
    gate = torch.sigmoid(randn(L, dv))
    if g_mode == "floor25":
        gh = g.view(L // heads, heads, dk)
        for h in range(heads):
            perm = torch.randperm(dk, generator=gen, device=device)[: dk // 4]
            gh[:, h, perm] = LN_FLOOR
    s0 = 0.02 * randn(dk, dv) if with_init else None
    out = dict(q=_round(q, dtype), k=_round(k, dtype), v=_round(v, dtype),
               beta=_round(beta, dtype), g=_round(g, dtype), gate=_round(gate, dtype))
    out["init"] = s0
    return out


def head_inputs(w: Workload, n: int, h: int, length: int | None = None) -> dict:
    """Inputs of one (sequence n, head h) as fp32 CPU tensors holding the
    dtype-rounded values: q, k, g [L, dk]; v, gate [L, dv]; beta [L]; init
    [dk, dv] fp32 or None.  For decode workloads L = number of steps."""
    L = length if length is not None else (w.decode_steps if w.is_decode else w.lengths[n])
    gen = torch.Generator().manual_seed(_head_seed(w.seed, n, h))
    return _draw(gen, L, w.dk, w.dv, w.g_mode, w.init_state, w.dtype)


def _select(w: Workload, heads):
    N, H = w.num_seqs, w.H
    if heads is None:
        return [(n, h) for n in range(N) for h in range(H)]
    return sorted({(int(n), int(h)) for n, h in heads})


def pack_prefill(w: Workload, heads=None, device="cpu", threads: int = 0) -> dict:
    """Packed [T, H, d] inputs in the workload dtype, on `device`.

    heads: iterable of (n, h) generated from their own seeds (None = all).
    The remaining heads, if any, are filled on `device` from a fast generator
    with the same distributions (their values do not match the per-head
    seeds, and no check reads them).
    Returns dict(q, k, v, g, beta, gate, cu_seqlens (int32), initial_state
    (fp32 [N, H, dk, dv] or None), exact (sorted list of (n, h)))."""
    assert not w.is_decode
    cu = w.cu_seqlens()
    T, H, dk, dv, N = cu[-1], w.H, w.dk, w.dv, w.num_seqs
    sel = _select(w, heads)
    dt = w.torch_dtype
    if len(sel) == N * H:
        out = dict(q=torch.empty(T, H, dk, dtype=dt), k=torch.empty(T, H, dk, dtype=dt),
                   g=torch.empty(T, H, dk, dtype=dt), v=torch.empty(T, H, dv, dtype=dt),
                   gate=torch.empty(T, H, dv, dtype=dt), beta=torch.empty(T, H, dtype=dt),
                   initial_state=torch.zeros(N, H, dk, dv) if w.init_state else None)
        fill_dev = "cpu"
    else:
        out = fast_prefill(w, seed=w.seed + 77, device=device)
        out.pop("cu_seqlens")
        fill_dev = device

    def one(nh):
        n, h = nh
        d = head_inputs(w, n, h)
        t0, t1 = cu[n], cu[n + 1]
        for key in ("q", "k", "g", "v", "gate", "beta"):
            out[key][t0:t1, h] = d[key].to(device=fill_dev, dtype=dt)
        if out["initial_state"] is not None:
            out["initial_state"][n, h] = d["init"].to(fill_dev)

    _run(one, sel, threads)
    out = {key: (val.to(device) if torch.is_tensor(val) else val) for key, val in out.items()}
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    out["exact"] = sel
    return out


def _run(fn, items, threads):
    nthreads = threads or min(32, max(1, torch.get_num_threads()))
    if len(items) > 1 and nthreads > 1:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(fn, items))
    else:
        for it in items:
            fn(it)


def fast_prefill(w: Workload, seed: int, device="cpu") -> dict:
    """All heads at once from one generator (same distributions, different
    values from the per-head streams).  Used to fill heads that no check
    reads and to build large timing inputs quickly on the device."""
    cu = w.cu_seqlens()
    T, H, dk, dv, N = cu[-1], w.H, w.dk, w.dv, w.num_seqs
    gen = torch.Generator(device=device).manual_seed(seed)
    d = _draw(gen, T * H, dk, dv, "standard" if w.g_mode != "floor25" else "floor25",
              False, w.dtype, device, heads=H)
    dt = w.torch_dtype
    out = dict(q=d["q"].view(T, H, dk).to(dt), k=d["k"].view(T, H, dk).to(dt),
               v=d["v"].view(T, H, dv).to(dt), g=d["g"].view(T, H, dk).to(dt),
               beta=d["beta"].view(T, H).to(dt), gate=d["gate"].view(T, H, dv).to(dt),
               cu_seqlens=torch.tensor(cu, dtype=torch.int32, device=device))
    if w.init_state:
        out["initial_state"] = 0.02 * torch.randn(N, H, dk, dv, generator=gen, device=device)
    else:
        out["initial_state"] = None
    return out


def pack_decode(w: Workload, steps: int | None = None, heads=None, device="cpu",
                threads: int = 0) -> dict:
    """Decode inputs on `device`: q, k, g [steps, N, H, dk]; v, gate
    [steps, N, H, dv]; beta [steps, N, H] (workload dtype) and the fp32 state
    [N, H, dk, dv].  heads: (n, h) drawn from their own seeds (None = all);
    the rest are filled on `device` from a fast generator."""
    assert w.is_decode
    S = steps if steps is not None else w.decode_steps
    N, H, dk, dv = w.num_seqs, w.H, w.dk, w.dv
    sel = _select(w, heads)
    dt = w.torch_dtype
    if len(sel) == N * H:
        out = dict(q=torch.empty(S, N, H, dk, dtype=dt), k=torch.empty(S, N, H, dk, dtype=dt),
                   g=torch.empty(S, N, H, dk, dtype=dt), v=torch.empty(S, N, H, dv, dtype=dt),
                   gate=torch.empty(S, N, H, dv, dtype=dt), beta=torch.empty(S, N, H, dtype=dt),
                   state=torch.empty(N, H, dk, dv))
        fill_dev = "cpu"
    else:
        out = fast_decode(w, S, seed=w.seed + 77, device=device)
        fill_dev = device

    def one(nh):
        n, h = nh
        d = head_inputs(w, n, h, length=S)
        for key in ("q", "k", "g", "v", "gate", "beta"):
            out[key][:, n, h] = d[key].to(device=fill_dev, dtype=dt)
        out["state"][n, h] = d["init"].to(fill_dev)

    _run(one, sel, threads)
    out = {key: val.to(device) for key, val in out.items()}
    out["exact"] = sel
    return out


def fast_decode(w: Workload, steps: int, seed: int, device="cpu") -> dict:
    """Decode inputs for all heads from one generator (see fast_prefill)."""
    N, H, dk, dv = w.num_seqs, w.H, w.dk, w.dv
    gen = torch.Generator(device=device).manual_seed(seed)
    d = _draw(gen, steps * N * H, dk, dv, "standard", False, w.dtype, device)
    dt = w.torch_dtype
    return dict(q=d["q"].view(steps, N, H, dk).to(dt), k=d["k"].view(steps, N, H, dk).to(dt),
                v=d["v"].view(steps, N, H, dv).to(dt), g=d["g"].view(steps, N, H, dk).to(dt),
                beta=d["beta"].view(steps, N, H).to(dt),
                gate=d["gate"].view(steps, N, H, dv).to(dt),
                state=0.02 * torch.randn(N, H, dk, dv, generator=gen, device=device))
