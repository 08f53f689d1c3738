"""The checked build (libkda_b200_checked.so, -DKDA_CHECK_G) verifies the
log-decay precondition ln(0.0067) <= g <= 0 on the device and reports a
violation through the workspace error word, read by kda_chunk_fwd_check; the
release build does not check.  A value below the floor or a NaN is not a
fault: the kernels only compute with it (no index depends on g).
"""
import ctypes
import math

import pytest
import torch

from kda_linear_attention_fwd_b200 import build, kda, workloads as W

OK, INVALID = 0, -1


def _run(lib, inp, flags=0):
    T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    N = inp["cu_seqlens"].numel() - 1
    out = torch.empty(T, H, dv, dtype=inp["q"].dtype, device="cuda")
    ws = torch.empty(kda.workspace_size(T, N, H, dk, dv, inp["q"].dtype), dtype=torch.uint8,
                     device="cuda")
    P = ctypes.c_void_p
    p = lambda t: None if t is None else P(t.data_ptr())
    st = P(torch.cuda.current_stream().cuda_stream)
    rc = lib.kda_chunk_fwd_ex(p(inp["q"]), p(inp["k"]), p(inp["v"]), p(inp["g"]), p(inp["beta"]),
                              p(inp["gate"]), p(out), p(inp["cu_seqlens"]), None, N, T, H, dk, dv,
                              kda._dtype_code(inp["q"]), 1.0, flags, None, None, 0, None, None,
                              p(ws), ws.numel(), st)
    assert rc == OK
    return kda.chunk_fwd_check(ws, lib=lib)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_checked_build_flags_g_out_of_range(cuda_lib, dtype):
    build.build(checked=True)
    chk, rel = kda.load_checked(), kda.load()
    w = W.custom(dtype=dtype, H=2, dk=128, dv=128, lengths=(300, 40), seed=31)
    inp = W.pack_prefill(w, device="cuda")
    # in range (values at the floor included): both builds report OK
    inp["g"][5, 1, 7] = math.log(0.0067)
    assert _run(chk, inp) == OK and _run(rel, inp) == OK
    # below the floor: the checked build reports it, unless the clamp flag is set
    inp["g"][200, 0, 3] = -9.0
    assert _run(chk, inp) == INVALID
    assert _run(chk, inp, flags=kda.FLAG_CLAMP_DECAY) == OK
    assert _run(rel, inp) == OK
    # positive or NaN: rejected with or without the clamp
    inp["g"][200, 0, 3] = 0.5
    assert _run(chk, inp, flags=kda.FLAG_CLAMP_DECAY) == INVALID
    inp["g"][200, 0, 3] = float("nan")
    assert _run(chk, inp) == INVALID
    # a later clean call clears the word
    inp["g"][200, 0, 3] = -1.0
    assert _run(chk, inp) == OK
