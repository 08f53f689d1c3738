"""kda_chunk_fwd_noalloc -- the prefill entry point that allocates nothing.

It exists for callers that cannot allocate device memory when they run the
layer (allocator callbacks, runtimes that hand out only fixed buffers, hosts
that forbid allocation after start-up): its scratch is a fixed array inside
the library.  These tests call it through the C-ABI twice in a row and check
each result against the fp64 oracle at the bf16 parity tolerance used
everywhere else, that device memory use does not change between the calls,
and that kda_chunk_fwd_noalloc_check reads the device error words back.
"""
import ctypes
import math

import pytest
import torch

from kda_linear_attention_fwd_b200 import kda
from kda_linear_attention_fwd_b200 import workloads as W
from parity import assert_close, np32, oracle_prefill, round_to

pytestmark = pytest.mark.gpu

SCRATCH = 32 << 20


def call_noalloc(lib, d, out, fin, stream):
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    N = d["cu_seqlens"].numel() - 1
    return lib.kda_chunk_fwd_noalloc(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["g"]),
                                     ptr(d["beta"]), ptr(d["gate"]), ptr(out),
                                     ptr(d["cu_seqlens"]), None, N, T, H, dk, dv,
                                     kda.KDA_DTYPE_BF16, 1.0, 0, ptr(d.get("initial_state")),
                                     ptr(fin), ctypes.c_void_p(stream.cuda_stream))


CASES = [
    # (heads, lengths, forced piece length, heads checked against the oracle)
    (4, (3000, 700, 1, 1500), "512", None),  # several pieces per sequence
    (4, (3000, 700, 1, 1500), None, None),   # the default plan fits the scratch
    (24, (6000, 6000), None, [(0, 5), (1, 17)]),  # default plan too big: pieces lengthened
]


@pytest.mark.parametrize("case", CASES, ids=["pieces512", "default", "lengthened"])
def test_noalloc_matches_oracle(cuda_lib, monkeypatch, case):
    H, lengths, piece, heads = case
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", piece)
    lib = kda.load()
    T, N = sum(lengths), len(lengths)
    if piece is None and heads is not None:
        # the plan kda_chunk_fwd would use needs more than the fixed scratch
        plan = kda.plan(T, N, H)
        assert plan["max_pieces"] * H * 3 * 128 * 128 * 4 > SCRATCH, plan
    w = W.custom(dtype="bf16", H=H, dk=128, dv=128, lengths=lengths, init_state=True, seed=404)
    d = W.pack_prefill(w, heads=heads, device="cuda")
    yr, Sr = oracle_prefill(d, heads=heads)
    cu = d["cu_seqlens"].tolist()
    sel = heads or [(n, h) for n in range(N) for h in range(H)]

    def check(out, fin, what):
        import numpy as np
        y, S = np32(out), np32(fin)
        ya = np.concatenate([y[cu[n]:cu[n + 1], h] for n, h in sel])
        ye = np.concatenate([round_to(yr[cu[n]:cu[n + 1], h], "bf16") for n, h in sel])
        assert_close(ya, ye, "bf16", f"noalloc y {what}")
        assert_close(np.stack([S[n, h] for n, h in sel]), np.stack([Sr[n, h] for n, h in sel]),
                     "bf16", f"noalloc final state {what}")

    stream = torch.cuda.current_stream()
    out = torch.empty(T, H, 128, dtype=torch.bfloat16, device="cuda")
    fin = torch.empty(N, H, 128, 128, device="cuda")
    # the one-time placement of the array when the library's device code is
    # first loaded (the start-up call the header asks for)
    assert lib.kda_chunk_fwd_noalloc_check(ctypes.c_void_p(stream.cuda_stream)) == 0
    free = []
    for call in range(2):  # two calls in a row share (and reuse) the scratch array
        out.fill_(float("nan"))
        fin.fill_(float("nan"))
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        rc = call_noalloc(lib, d, out, fin, stream)
        assert rc == 0, kda.status_string(rc)
        assert lib.kda_chunk_fwd_noalloc_check(ctypes.c_void_p(stream.cuda_stream)) == 0
        check(out, fin, f"call {call}")
    torch.cuda.synchronize()
    free.append(torch.cuda.mem_get_info()[0])
    assert free[0] == free[1] == free[2], free  # the calls allocate no device memory


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_lib):
    """A plan table larger than the fixed scratch is refused up front."""
    lib = kda.load()
    N = 4 << 20  # four million empty sequences: a plan table of ~80 MB
    cu = torch.zeros(N + 1, dtype=torch.int32, device="cuda")
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = lib.kda_chunk_fwd_noalloc(None, None, None, None, None, None, None, ptr(cu), None, N, 0,
                                   1, 64, 64, kda.KDA_DTYPE_BF16, 1.0, 0, None, None,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -4, kda.status_string(rc)  # KDA_ERR_WORKSPACE


def test_noalloc_check_reports_device_errors(cuda_lib):
    """The checked build flags g below the decay floor in the scratch's error
    word; kda_chunk_fwd_noalloc_check maps it to KDA_ERR_INVALID_ARG, and a
    following valid call clears it again."""
    lib = kda.load_checked()
    assert lib.kda_build_checks_g() == 1
    w = W.custom(dtype="bf16", H=2, dk=128, dv=128, lengths=(300, 40), init_state=True, seed=405)
    d = W.pack_prefill(w, device="cuda")
    out = torch.empty(340, 2, 128, dtype=torch.bfloat16, device="cuda")
    fin = torch.empty(2, 2, 128, 128, device="cuda")
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    bad = dict(d)
    bad["g"] = d["g"].clone()
    bad["g"][17, 1, 3] = 1.5 * math.log(0.0067)  # below the floor
    assert call_noalloc(lib, bad, out, fin, stream) == 0
    assert lib.kda_chunk_fwd_noalloc_check(sp) == -1  # KDA_ERR_INVALID_ARG
    assert call_noalloc(lib, d, out, fin, stream) == 0
    assert lib.kda_chunk_fwd_noalloc_check(sp) == 0
