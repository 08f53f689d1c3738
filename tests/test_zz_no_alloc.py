"""kda_chunk_fwd_noalloc -- the prefill entry point that allocates nothing.

It exists for callers that cannot allocate device memory when they run the
layer (allocator callbacks, runtimes that hand out only fixed buffers, hosts
that forbid allocation after start-up): its scratch is a fixed array inside
the library.  This test calls it through the C-ABI and checks that two calls
in a row give the same result as kda_chunk_fwd with a caller-supplied
workspace, within the bf16 parity tolerance used everywhere else.
"""
import ctypes

import pytest
import torch

from kda_linear_attention_fwd_b200 import kda
from kda_linear_attention_fwd_b200 import workloads as W
from parity import assert_close, np32

pytestmark = pytest.mark.gpu


def noalloc_fn(lib):
    f = lib.kda_chunk_fwd_noalloc
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    f.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_int,
                  ctypes.c_float, i32, P, P, P]
    f.restype = ctypes.c_int
    return f


def call_noalloc(f, d, out, fin, stream):
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    N = d["cu_seqlens"].numel() - 1
    return f(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["g"]), ptr(d["beta"]), ptr(d["gate"]),
             ptr(out), ptr(d["cu_seqlens"]), None, N, T, H, dk, dv, kda.KDA_DTYPE_BF16, 1.0, 0,
             ptr(d.get("initial_state")), ptr(fin), ctypes.c_void_p(stream.cuda_stream))


CASES = [
    # (heads, lengths, forced piece length)
    (4, (3000, 700, 1, 1500), "512"),   # several pieces per sequence
    (4, (3000, 700, 1, 1500), None),    # the default plan fits the scratch
    (16, (4096, 4096), None),           # default plan too big: pieces lengthened to fit
]


@pytest.mark.parametrize("case", CASES, ids=["pieces512", "default", "lengthened"])
def test_noalloc_matches_workspace_entry_point(cuda_lib, monkeypatch, case):
    H, lengths, piece = case
    if piece:
        monkeypatch.setenv("KDA_PIECE_LEN", piece)
    lib = kda.load()
    f = noalloc_fn(lib)
    w = W.custom(dtype="bf16", H=H, dk=128, dv=128, lengths=lengths, init_state=True,
                 seed=404)
    d = W.pack_prefill(w, device="cuda")
    y_ref, s_ref = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["gate"],
                                 d["cu_seqlens"], initial_state=d["initial_state"])
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    for _ in range(2):  # two calls in a row share (and reuse) the scratch array
        out = torch.full_like(y_ref, float("nan"))
        fin = torch.full_like(s_ref, float("nan"))
        rc = call_noalloc(f, d, out, fin, stream)
        assert rc == 0, kda.status_string(rc)
        torch.cuda.synchronize()
        assert_close(np32(out), np32(y_ref), "bf16", "noalloc y")
        assert_close(np32(fin), np32(s_ref), "bf16", "noalloc final state")


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_lib):
    """A plan table larger than the fixed scratch is refused up front."""
    lib = kda.load()
    f = noalloc_fn(lib)
    N = 4 << 20  # four million empty sequences: a plan table of ~80 MB
    cu = torch.zeros(N + 1, dtype=torch.int32, device="cuda")
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = f(None, None, None, None, None, None, None, ptr(cu), None, N, 0, 1, 64, 64,
           kda.KDA_DTYPE_BF16, 1.0, 0, None, None,
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -4, kda.status_string(rc)  # KDA_ERR_WORKSPACE
