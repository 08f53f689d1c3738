"""ctypes binding of libkda_b200.so (see include/kda.h).

Argument marshalling only: PyTorch supplies device memory and the current
stream, every step of the layer runs in the library's CUDA kernels.  There is
no CPU fallback; if the library is missing or no CUDA device is present the
calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda_b200.so")
# the checked build (-DKDA_CHECK_G): the prefill also verifies the log-decay range
LIB_CHECKED_PATH = os.path.join(_HERE, "libkda_b200_checked.so")

KDA_DTYPE_F32 = 0
KDA_DTYPE_BF16 = 1

EXPORTS = ("kda_status_string", "kda_chunk_fwd_workspace_size", "kda_chunk_fwd_plan",
           "kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_ex", "kda_decode_step_ex",
           "kda_chunk_fwd_summary", "kda_state_compose", "kda_bwd_workspace_size", "kda_bwd",
           "kda_chunk_fwd_check", "kda_build_checks_g", "kda_chunk_fwd_noalloc",
           "kda_chunk_fwd_noalloc_check", "kda_chunk_fwd_sub_pieces")

# flags of the extended entry points (include/kda.h)
FLAG_QK_L2NORM, FLAG_BETA_LOGITS, FLAG_GATE_LOGITS, FLAG_CLAMP_DECAY = 1, 2, 4, 8

_lib = None
_lib_checked = None


class KdaError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


def load(path: str = LIB_PATH):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if path == LIB_PATH and _lib is not None:
        return _lib
    lib = _open(path)
    if path == LIB_PATH:
        _lib = lib
    return lib


def load_checked():
    """The checked build of the library (a separate handle)."""
    global _lib_checked
    if _lib_checked is None:
        _lib_checked = _open(LIB_CHECKED_PATH)
    return _lib_checked


def _open(path):
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} not found: build it first (python -m kda_linear_attention_fwd_b200.build)")
    lib = ctypes.CDLL(path)
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_chunk_fwd_workspace_size.argtypes = [i32, i32, i32, i32, i32, ctypes.c_int]
    lib.kda_chunk_fwd_workspace_size.restype = sz
    lib.kda_chunk_fwd_plan.argtypes = [i32, i32, i32, P, P, P]
    lib.kda_chunk_fwd_plan.restype = ctypes.c_int
    lib.kda_chunk_fwd_sub_pieces.argtypes = [i32, i32, i32]
    lib.kda_chunk_fwd_sub_pieces.restype = ctypes.c_int32
    lib.kda_chunk_fwd.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                  ctypes.c_int, f32, i32, P, P, P, sz, P]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_decode_step.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, ctypes.c_int,
                                    f32, i32, P]
    lib.kda_decode_step.restype = ctypes.c_int
    lib.kda_chunk_fwd_ex.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                     ctypes.c_int, f32, i32, P, P, i32, P, P, P, sz, P]
    lib.kda_chunk_fwd_ex.restype = ctypes.c_int
    lib.kda_decode_step_ex.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, ctypes.c_int,
                                       f32, i32, P]
    lib.kda_decode_step_ex.restype = ctypes.c_int
    lib.kda_chunk_fwd_summary.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_int,
                                          i32, P, P, P, sz, P]
    lib.kda_chunk_fwd_summary.restype = ctypes.c_int
    lib.kda_state_compose.argtypes = [P, P, i32, P, P, i32, i32, i32, i32, P]
    lib.kda_state_compose.restype = ctypes.c_int
    lib.kda_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.kda_bwd_workspace_size.restype = sz
    lib.kda_bwd.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, ctypes.c_int,
                            f32, P, P, P, P, P, P, P, P, P, P, sz, P]
    lib.kda_bwd.restype = ctypes.c_int
    lib.kda_chunk_fwd_check.argtypes = [P, sz, P]
    lib.kda_chunk_fwd_check.restype = ctypes.c_int
    lib.kda_build_checks_g.argtypes = []
    lib.kda_build_checks_g.restype = ctypes.c_int
    lib.kda_chunk_fwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                          ctypes.c_int, f32, i32, P, P, P]
    lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.kda_chunk_fwd_noalloc_check.argtypes = [P]
    lib.kda_chunk_fwd_noalloc_check.restype = ctypes.c_int
    return lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def _check(fn, status):
    if status != 0:
        raise KdaError(fn, status, status_string(status))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def workspace_size(total_tokens, num_seqs, H, dk, dv, dtype=torch.bfloat16) -> int:
    code = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_F32
    return int(load().kda_chunk_fwd_workspace_size(total_tokens, num_seqs, H, dk, dv, code))


def plan(total_tokens, num_seqs, H) -> dict:
    """Piece length, piece bound, launch count and sub-pieces of one
    kda_chunk_fwd call (bf16, dk = dv = 128)."""
    L, P, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    lib = load()
    _check("kda_chunk_fwd_plan", lib.kda_chunk_fwd_plan(
        total_tokens, num_seqs, H, ctypes.byref(L), ctypes.byref(P), ctypes.byref(n)))
    sub = int(lib.kda_chunk_fwd_sub_pieces(total_tokens, num_seqs, H))
    if sub < 1:
        _check("kda_chunk_fwd_sub_pieces", sub)
    return dict(piece_len=L.value, max_pieces=P.value, launches=n.value, sub_pieces=sub)


def _flags(qk_l2norm, beta_logits, gate_logits, clamp_decay):
    return ((FLAG_QK_L2NORM if qk_l2norm else 0) | (FLAG_BETA_LOGITS if beta_logits else 0) |
            (FLAG_GATE_LOGITS if gate_logits else 0) | (FLAG_CLAMP_DECAY if clamp_decay else 0))


def snapshot_offsets(lengths, snapshot_tokens):
    """Running sums of the per-sequence snapshot counts (L - 1) // B."""
    offs = [0]
    for L in lengths:
        offs.append(offs[-1] + (max(int(L), 1) - 1) // snapshot_tokens)
    return offs


def chunk_fwd(q, k, v, g, beta, gate, cu_seqlens, *, scale=1.0, qk_l2norm=False,
              initial_state=None, final_state=None, out=None, workspace=None,
              cu_seqlens_host=None, output_final_state=True, stream=None,
              beta_logits=False, gate_logits=False, clamp_decay=False, snapshot_tokens=0):
    """Prefill over packed sequences.  q, k, g [T, H, dk]; v, gate [T, H, dv];
    beta [T, H]; cu_seqlens int32 [N+1] (device).  Returns (out, final_state),
    plus the snapshots [count, H, dk, dv] fp32 when snapshot_tokens > 0 (the
    state after every snapshot_tokens tokens of each sequence, sequence-major;
    needs the offsets on the host: cu_seqlens_host, else one device read)."""
    lib = load()
    _require_cuda(q, k, v, g, beta, gate, cu_seqlens, initial_state, final_state, out, workspace)
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.shape[0] - 1
    code = _dtype_code(q)
    if out is None:
        out = torch.empty(T, H, dv, dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    need = int(lib.kda_chunk_fwd_workspace_size(T, N, H, dk, dv, code))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    host = None
    if cu_seqlens_host is not None:
        host_arr = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
        host = ctypes.cast(host_arr, ctypes.c_void_p)
    flags = _flags(qk_l2norm, beta_logits, gate_logits, clamp_decay)
    if flags & ~FLAG_QK_L2NORM == 0 and not snapshot_tokens:
        st = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate),
                               _ptr(out), _ptr(cu_seqlens), host, N, T, H, dk, dv, code,
                               float(scale), flags, _ptr(initial_state), _ptr(final_state),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream))
        _check("kda_chunk_fwd", st)
        return out, final_state
    snaps = offs_dev = None
    if snapshot_tokens:
        cu = list(cu_seqlens_host) if cu_seqlens_host is not None else cu_seqlens.tolist()
        offs = snapshot_offsets([cu[i + 1] - cu[i] for i in range(N)], snapshot_tokens)
        offs_dev = torch.tensor(offs, dtype=torch.int32, device=q.device)
        snaps = torch.empty(max(offs[-1], 1), H, dk, dv, dtype=torch.float32, device=q.device)
    st = lib.kda_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate),
                              _ptr(out), _ptr(cu_seqlens), host, N, T, H, dk, dv, code,
                              float(scale), flags, _ptr(initial_state), _ptr(final_state),
                              int(snapshot_tokens), _ptr(snaps), _ptr(offs_dev), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check("kda_chunk_fwd_ex", st)
    if snapshot_tokens:
        return out, final_state, snaps[:offs[-1]]
    return out, final_state


def decode_step(q, k, v, g, beta, gate, state, *, scale=1.0, qk_l2norm=False, out=None,
                stream=None, beta_logits=False, gate_logits=False, clamp_decay=False):
    """One token per sequence.  q, k, g [N, H, dk]; v, gate [N, H, dv]; beta
    [N, H]; state [N, H, dk, dv] fp32, updated in place.  Returns out."""
    lib = load()
    _require_cuda(q, k, v, g, beta, gate, state, out)
    N, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    st = lib.kda_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate),
                                _ptr(out), _ptr(state), N, H, dk, dv, _dtype_code(q),
                                float(scale), _flags(qk_l2norm, beta_logits, gate_logits,
                                                     clamp_decay), _stream(stream))
    _check("kda_decode_step_ex", st)
    return out


def chunk_summary(k, v, g, beta, cu_seqlens, *, qk_l2norm=False, beta_logits=False,
                  clamp_decay=False, cu_seqlens_host=None, workspace=None, stream=None):
    """The affine map S -> M S + Z of every sequence's tokens.  k, g [T, H, dk];
    v [T, H, dv]; beta [T, H].  Returns (M [N, H, dk, dk], Z [N, H, dk, dv]) fp32."""
    lib = load()
    _require_cuda(k, v, g, beta, cu_seqlens, workspace)
    T, H, dk = k.shape
    dv = v.shape[-1]
    N = cu_seqlens.shape[0] - 1
    code = _dtype_code(k)
    M = torch.empty(N, H, dk, dk, dtype=torch.float32, device=k.device)
    Z = torch.empty(N, H, dk, dv, dtype=torch.float32, device=k.device)
    need = int(lib.kda_chunk_fwd_workspace_size(T, N, H, dk, dv, code))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=k.device)
    host = None
    if cu_seqlens_host is not None:
        host_arr = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
        host = ctypes.cast(host_arr, ctypes.c_void_p)
    st = lib.kda_chunk_fwd_summary(_ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), host,
                                   N, T, H, dk, dv, code,
                                   _flags(qk_l2norm, beta_logits, False, clamp_decay),
                                   _ptr(M), _ptr(Z), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check("kda_chunk_fwd_summary", st)
    return M, Z


def state_compose(M, Z, state_in=None, *, out=None, stream=None):
    """Apply the maps (M [R, N, H, dk, dk], Z [R, N, H, dk, dv]) in order to
    state_in [N, H, dk, dv] (None = zeros).  Returns the state."""
    lib = load()
    _require_cuda(M, Z, state_in, out)
    R, N, H, dk, _ = M.shape
    dv = Z.shape[-1]
    M, Z = M.contiguous(), Z.contiguous()
    if out is None:
        out = torch.empty(N, H, dk, dv, dtype=torch.float32, device=M.device)
    st = lib.kda_state_compose(_ptr(M), _ptr(Z), R, _ptr(state_in), _ptr(out), N, H, dk, dv,
                               _stream(stream))
    _check("kda_state_compose", st)
    return out


def bwd_workspace_size(total_tokens, num_seqs, H, dk, dv) -> int:
    return int(load().kda_bwd_workspace_size(total_tokens, num_seqs, H, dk, dv))


def bwd(q, k, v, g, beta, gate, dy, cu_seqlens, *, scale=1.0, initial_state=None,
        d_final_state=None, cu_seqlens_host=None, workspace=None, stream=None):
    """Gradients of the plain forward (kda_bwd): returns a dict of fp32
    tensors dq, dk, dg [T, H, dk]; dv, dgate [T, H, dv] (dgate None without a
    gate); dbeta [T, H]; ds0 [N, H, dk, dv]."""
    lib = load()
    _require_cuda(q, k, v, g, beta, gate, dy, cu_seqlens, initial_state, d_final_state)
    q, k, v, g, beta, dy = (t.contiguous() for t in (q, k, v, g, beta, dy))
    gate = None if gate is None else gate.contiguous()
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dq": torch.empty(T, H, dk, **f32), "dk": torch.empty(T, H, dk, **f32),
           "dg": torch.empty(T, H, dk, **f32), "dv": torch.empty(T, H, dv, **f32),
           "dbeta": torch.empty(T, H, **f32),
           "dgate": None if gate is None else torch.empty(T, H, dv, **f32),
           "ds0": torch.empty(N, H, dk, dv, **f32)}
    need = bwd_workspace_size(T, N, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    cu_arr = None
    if cu_seqlens_host is not None:
        cu_arr = (ctypes.c_int32 * len(cu_seqlens_host))(*cu_seqlens_host)
    s0 = None if initial_state is None else initial_state.float().contiguous()
    dsf = None if d_final_state is None else d_final_state.float().contiguous()
    st = lib.kda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate), _ptr(dy),
                     _ptr(cu_seqlens), None if cu_arr is None else ctypes.cast(cu_arr, ctypes.c_void_p),
                     N, T, H, dk, dv, _dtype_code(q), float(scale), _ptr(s0), _ptr(dsf),
                     _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                     _ptr(out["dbeta"]), _ptr(out["dgate"]), _ptr(out["ds0"]), _ptr(workspace),
                     workspace.numel(), _stream(stream))
    _check("kda_bwd", st)
    return out


def chunk_fwd_check(workspace, stream=None, lib=None) -> int:
    """Status of the last prefill that used `workspace` (waits for the
    stream): 0 = KDA_OK, else a kda_status code (see include/kda.h)."""
    lib = lib or load()
    return int(lib.kda_chunk_fwd_check(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)))
