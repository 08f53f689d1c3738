"""The C-ABI library builds, loads, exports what include/kda.h declares, and
rejects bad arguments on the host (no GPU needed: nothing here launches)."""
import ctypes
import os
import re

import pytest

from kda_linear_attention_fwd_b200 import build, kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, INVALID, UNSUPPORTED, ALIGN, WORKSPACE, CUDA, TIMEOUT = 0, -1, -2, -3, -4, -5, -6
BF16, F32 = 1, 0
A = 0x100000  # a 16-byte aligned fake device address; never dereferenced on the host


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kda.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_workspace_size",
              "kda_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(kda.EXPORTS) <= set(declared_functions())


def test_exports_are_c_symbols():
    out = os.popen(f"nm -D --defined-only {kda.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_status_strings(lib):
    for code, name in [(OK, "KDA_OK"), (INVALID, "KDA_ERR_INVALID_ARG"),
                       (UNSUPPORTED, "KDA_ERR_UNSUPPORTED"), (ALIGN, "KDA_ERR_ALIGNMENT"),
                       (WORKSPACE, "KDA_ERR_WORKSPACE"), (CUDA, "KDA_ERR_CUDA"),
                       (TIMEOUT, "KDA_ERR_TIMEOUT")]:
        assert kda.status_string(code) == name
    assert kda.status_string(12345) == "KDA_ERR_UNKNOWN"


def test_workspace_size(lib):
    f = lib.kda_chunk_fwd_workspace_size
    assert f(4096, 2, 16, 128, 128, BF16) > 0
    assert f(0, 1, 1, 64, 64, F32) > 0
    assert f(-1, 1, 1, 64, 64, F32) == 0
    assert f(16, 1, 1, 96, 64, F32) == 0
    assert f(16, 1, 0, 64, 64, F32) == 0
    assert f(16, 1, 1, 64, 64, 7) == 0
    # covers the plan: one transition and two states per (piece, head)
    for T, N, H, dk, dv in [(8192, 2, 32, 128, 128), (8192, 2, 16, 128, 128),
                            (131072, 1, 32, 128, 128), (48317, 8, 32, 128, 128),
                            (5000, 7, 3, 64, 128)]:
        plan = kda.plan(T, N, H)
        per_piece = H * (dk * dk + 2 * dk * dv) * 4
        assert plan["piece_len"] % 16 == 0 and plan["piece_len"] >= 256
        assert plan["max_pieces"] >= N + (T + plan["piece_len"] - 1) // plan["piece_len"] - 1
        assert f(T, N, H, dk, dv, BF16) >= plan["max_pieces"] * per_piece
    # a larger state needs more workspace for the same plan
    assert f(8192, 2, 16, 128, 128, BF16) > f(8192, 2, 16, 64, 64, BF16)


def call_fwd(lib, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, gate=None, out=A, cu=A, cu_host=None, N=1, T=16, H=1,
             dk=64, dv=64, dtype=BF16, scale=1.0, l2=0, s0=None, s1=None, ws=A, ws_bytes=1 << 40,
             stream=None)
    a.update(kw)
    cu_host = a["cu_host"]
    if cu_host is not None:
        arr = (ctypes.c_int32 * len(cu_host))(*cu_host)
        cu_host = ctypes.cast(arr, ctypes.c_void_p)
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["gate"], a["out"],
                             a["cu"], cu_host, a["N"], a["T"], a["H"], a["dk"], a["dv"],
                             a["dtype"], a["scale"], a["l2"], a["s0"], a["s1"], a["ws"],
                             a["ws_bytes"], a["stream"])


def test_chunk_fwd_validation(lib):
    assert call_fwd(lib, N=0, T=0) == OK
    assert call_fwd(lib, N=0, T=5) == INVALID
    assert call_fwd(lib, N=-1) == INVALID
    assert call_fwd(lib, H=0) == INVALID
    assert call_fwd(lib, T=-3) == INVALID
    assert call_fwd(lib, dk=96) == UNSUPPORTED
    assert call_fwd(lib, dv=32) == UNSUPPORTED
    assert call_fwd(lib, dtype=5) == UNSUPPORTED
    assert call_fwd(lib, l2=2) == INVALID
    assert call_fwd(lib, q=None) == INVALID
    assert call_fwd(lib, cu=None) == INVALID
    assert call_fwd(lib, out=None) == INVALID
    assert call_fwd(lib, q=A + 8) == ALIGN
    assert call_fwd(lib, gate=A + 4) == ALIGN
    assert call_fwd(lib, s1=A + 2) == ALIGN
    assert call_fwd(lib, beta=A + 1) == ALIGN
    assert call_fwd(lib, ws=A + 8) == ALIGN
    assert call_fwd(lib, ws=None) == WORKSPACE
    assert call_fwd(lib, ws_bytes=16) == WORKSPACE
    # host copy of cu_seqlens is checked when given
    assert call_fwd(lib, cu_host=[0, 15]) == INVALID
    assert call_fwd(lib, N=2, cu_host=[0, 10, 5]) == INVALID
    assert call_fwd(lib, cu_host=[1, 16]) == INVALID
    # final state may alias the initial state exactly, but not overlap partially
    assert call_fwd(lib, s0=A, s1=A + 256, ws_bytes=16) == INVALID
    assert call_fwd(lib, s0=A, s1=A, ws_bytes=16) == WORKSPACE  # aliasing accepted


def call_dec(lib, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, gate=None, out=A, state=A, N=4, H=2, dk=128, dv=128,
             dtype=BF16, scale=1.0, l2=0, stream=None)
    a.update(kw)
    return lib.kda_decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["gate"], a["out"],
                               a["state"], a["N"], a["H"], a["dk"], a["dv"], a["dtype"],
                               a["scale"], a["l2"], a["stream"])


def test_decode_validation(lib):
    assert call_dec(lib, N=0) == OK
    assert call_dec(lib, N=-1) == INVALID
    assert call_dec(lib, H=0) == INVALID
    assert call_dec(lib, dk=32) == UNSUPPORTED
    assert call_dec(lib, dtype=3) == UNSUPPORTED
    assert call_dec(lib, state=None) == INVALID
    assert call_dec(lib, beta=None) == INVALID
    assert call_dec(lib, state=A + 4) == ALIGN
    assert call_dec(lib, k=A + 2) == ALIGN
    assert call_dec(lib, beta=A + 1) == ALIGN
    assert call_dec(lib, l2=-1) == INVALID


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(16, 1, 64, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        kda.chunk_fwd(x, x, x, x, torch.zeros(16, 1, dtype=torch.bfloat16), None,
                      torch.tensor([0, 16], dtype=torch.int32))


def call_fwd_ex(lib, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, gate=None, out=A, cu=A, cu_host=None, N=1, T=16, H=1,
             dk=64, dv=64, dtype=BF16, scale=1.0, flags=0, s0=None, s1=None, snap_tokens=0,
             snaps=None, snap_offs=None, ws=A, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.kda_chunk_fwd_ex(a["q"], a["k"], a["v"], a["g"], a["beta"], a["gate"], a["out"],
                                a["cu"], a["cu_host"], a["N"], a["T"], a["H"], a["dk"], a["dv"],
                                a["dtype"], a["scale"], a["flags"], a["s0"], a["s1"],
                                a["snap_tokens"], a["snaps"], a["snap_offs"], a["ws"],
                                a["ws_bytes"], a["stream"])


def test_chunk_fwd_ex_validation(lib):
    assert call_fwd_ex(lib, N=0, T=0) == OK
    assert call_fwd_ex(lib, N=0, T=0, flags=15) == OK
    assert call_fwd_ex(lib, flags=16) == INVALID
    assert call_fwd_ex(lib, flags=-1) == INVALID
    assert call_fwd_ex(lib, snap_tokens=8, snaps=A, snap_offs=A) == INVALID
    assert call_fwd_ex(lib, snap_tokens=-16, snaps=A, snap_offs=A) == INVALID
    assert call_fwd_ex(lib, snap_tokens=64) == INVALID          # no buffers
    assert call_fwd_ex(lib, snap_tokens=64, snaps=A) == INVALID  # no offsets
    assert call_fwd_ex(lib, snap_tokens=64, snaps=A + 8, snap_offs=A) == ALIGN
    assert call_fwd_ex(lib, snap_tokens=64, snaps=A, snap_offs=A + 2) == ALIGN
    assert call_fwd_ex(lib, flags=15, ws=None) == WORKSPACE     # flags accepted, then workspace
    # the plain entry point still accepts only 0 / 1 for qk_l2norm
    assert call_fwd(lib, l2=2) == INVALID


def test_decode_ex_validation(lib):
    f = lib.kda_decode_step_ex
    args = [A, A, A, A, A, None, A, A, 4, 2, 128, 128, BF16, 1.0]
    assert f(*args[:8], 0, 2, 128, 128, BF16, 1.0, 15, None) == OK  # no sequences
    assert f(*args, 16, None) == INVALID
    assert f(*args[:2], A + 2, *args[3:], 3, None) == ALIGN


def test_snapshot_offsets_host_helper():
    assert kda.snapshot_offsets([0, 5, 64, 300, 701], 64) == [0, 0, 0, 0, 4, 14]
    assert kda.snapshot_offsets([65, 128, 129], 64) == [0, 1, 2, 4]


def test_summary_and_compose_validation(lib):
    s = lib.kda_chunk_fwd_summary
    base = [A, A, A, A, A, None, 1, 16, 1, 64, 64, BF16, 0, A, A, A, 1 << 40, None]
    assert s(*base[:6], 0, 0, *base[8:]) == OK                   # no sequences
    assert s(*base[:12], 16, *base[13:]) == INVALID               # unknown flag
    assert s(*base[:13], None, *base[14:]) == INVALID             # no transition buffer
    assert s(*base[:13], A + 4, *base[14:]) == ALIGN
    assert s(*base[:15], None, *base[16:]) == WORKSPACE
    assert s(*base[:9], 96, *base[10:]) == UNSUPPORTED
    c = lib.kda_state_compose
    assert c(A, A, 2, A, A, 0, 1, 64, 64, None) == OK               # no sequences
    assert c(A, A, -1, A, A, 1, 1, 64, 64, None) == INVALID
    assert c(A, A, 1, A, None, 1, 1, 64, 64, None) == INVALID       # no output
    assert c(None, A, 1, A, A, 1, 1, 64, 64, None) == INVALID       # maps missing
    assert c(A, A, 1, A, A + 8, 1, 1, 64, 64, None) == ALIGN
    assert c(A, A, 1, A, A + 256, 1, 1, 64, 64, None) == INVALID    # partial overlap
    assert c(A, A, 1, A, A, 1, 1, 32, 64, None) == UNSUPPORTED


def test_bwd_validation(lib):
    """kda_bwd rejects bad arguments before touching the device."""
    f = lib.kda_bwd
    ws = lib.kda_bwd_workspace_size(16, 1, 1, 64, 64)
    assert ws > 0 and lib.kda_bwd_workspace_size(16, 1, 1, 96, 64) == 0
    # q k v g beta gate dy cu cu_host N T H dk dv dtype scale s0 dsT
    # dq dk dv dg dbeta dgate ds0 ws ws_bytes stream
    base = [A, A, A, A, A, A, A, A, None, 1, 16, 1, 64, 64, BF16, 1.0, None, None,
            A, A, A, A, A, A, A, A, ws, None]
    assert f(*base[:9], 0, 0, *base[11:]) == OK                   # no sequences
    assert f(*base[:12], 96, *base[13:]) == UNSUPPORTED             # dk
    assert f(*base[:14], 7, *base[15:]) == UNSUPPORTED              # dtype
    assert f(*base[:5], None, *base[6:]) == INVALID                 # dgate without gate
    assert f(*base[:7], None, *base[8:]) == INVALID                 # no device offsets
    assert f(*base[:18], None, *base[19:]) == INVALID               # no dq
    assert f(*base[:4], A + 1, *base[5:]) == ALIGN                  # beta (bf16)
    assert f(*base[:20], A + 2, *base[21:]) == ALIGN                # dv (fp32)
    assert f(*base[:25], None, *base[26:]) == WORKSPACE
    assert f(*base[:26], ws - 1, *base[27:]) == WORKSPACE
    assert f(*base[:25], A + 16, *base[26:]) == ALIGN               # workspace alignment
    bad = (ctypes.c_int32 * 2)(0, 15)                                # does not end at T
    assert f(*base[:8], ctypes.cast(bad, ctypes.c_void_p), *base[9:]) == INVALID


def test_checked_build_exports_the_same_symbols(lib):
    build.build(checked=True)
    chk = kda.load_checked()
    for name in declared_functions():
        assert hasattr(chk, name), name
    assert lib.kda_build_checks_g() == 0 and chk.kda_build_checks_g() == 1


def test_chunk_fwd_check_validation(lib):
    assert lib.kda_chunk_fwd_check(None, 1 << 20, None) == INVALID
    assert lib.kda_chunk_fwd_check(A, 8, None) == INVALID  # smaller than the error words


def test_plan_choices_on_148_sms(lib, monkeypatch):
    """The piece plan's cost model on a 148-SM device (without a device the
    library assumes 148 SMs).  Default (16-token kernels): waves of the output
    pass at two CTAs per SM and of the paired summary pass at one -- over
    sub-pieces where they fill its waves better -- plus scan and fold steps.
    With the 32-token kernels (KDA_PREFILL_IMPL=c32): both passes one
    CTA per SM, pieces a multiple of 32 tokens."""
    import torch
    if torch.cuda.is_available() and torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("plan depends on the SM count")
    long = kda.plan(131072, 1, 32)  # 9 pieces per head: 288 output CTAs, one wave; summary over
    assert (long["piece_len"], long["sub_pieces"], long["launches"]) == (14592, 4, 6)  # 4 sub-pieces each
    assert kda.plan(8192, 2, 16)["piece_len"] == 464      # 9 pieces per sequence, no sub-pieces
    assert kda.plan(8192, 2, 16)["sub_pieces"] == 1
    assert kda.plan(256, 1, 2) == {"piece_len": 256, "max_pieces": 2, "launches": 2,
                                   "sub_pieces": 1}  # one piece
    monkeypatch.setenv("KDA_PREFILL_IMPL", "c32")
    assert kda.plan(131072, 1, 32)["piece_len"] == 14592  # 9 pieces per head: 288 CTAs, 2 waves
    assert kda.plan(8192, 2, 16)["piece_len"] == 1024     # 4 pieces per sequence
    # the workspace covers either plan
    f = lib.kda_chunk_fwd_workspace_size
    for T, N, H in [(131072, 1, 32), (8192, 2, 16), (48317, 8, 32)]:
        for impl in ("c32", "tc5"):
            monkeypatch.setenv("KDA_PREFILL_IMPL", impl)
            p = kda.plan(T, N, H)
            assert f(T, N, H, 128, 128, BF16) >= p["max_pieces"] * H * 3 * 128 * 128 * 4
