"""CPU oracle for the KDA (Kimi Delta Attention) forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library in
``kda_linear_attention_fwd_b200`` shares no code with it and never calls it.

Two independent CPU forms of the same layer:

* ``varlen`` / ``steps`` -- the plain per-token recurrence in fp64 (C, threaded
  over (sequence, head)); the definition itself.  See ``kda_oracle.c``.
* ``chunkwise`` -- the chunk-parallel form in fp64 NumPy, used to pin the
  per-token form (chunk-size invariance) and to state the chunk algebra.

Functions here take and return NumPy arrays; inputs are fp32 arrays holding
the exact values the GPU receives (bf16 values widen to fp32 exactly).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libkda_oracle.so`` (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        # -ffp-contract=off keeps every fp64 multiply and add separately rounded
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", tmp, _SRC,
             "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32 = ctypes.c_int
        d = ctypes.c_double
        lib.kda_oracle_varlen.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, d, i32,
                                          i32, P, P, P, i32]
        lib.kda_oracle_varlen.restype = i32
        lib.kda_oracle_steps.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, d, i32,
                                         i32, P, P, P, i32]
        lib.kda_oracle_steps.restype = i32
        _lib = lib
    return _lib


def _f32(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data


def varlen(q, k, v, g, beta, gate, cu_seqlens, *, scale=1.0, qk_l2norm=False,
           initial_state=None, erase=True, mask=None, threads=0, want_y=True):
    """Per-token fp64 recurrence over packed sequences.

    q, k, g: [T, H, dk]; v, gate: [T, H, dv] (gate may be None); beta: [T, H];
    cu_seqlens: [N+1] int; initial_state: [N, H, dk, dv] or None (zeros).
    mask: [N, H] bool selecting the (n, h) to compute (None = all).
    Returns (y [T, H, dv] fp64 or None, final_state [N, H, dk, dv] fp64, threads).
    Entries of y / final_state for unselected (n, h) are zero.
    """
    lib = _load()
    q, k, v, g, beta, gate = map(_f32, (q, k, v, g, beta, gate))
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    N = cu.shape[0] - 1
    if initial_state is None:
        state = np.zeros((N, H, dk, dv), dtype=np.float64)
    else:
        state = np.array(initial_state, dtype=np.float64, copy=True).reshape(N, H, dk, dv)
    y = np.zeros((T, H, dv), dtype=np.float64) if want_y else None
    m = None
    if mask is not None:
        m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8).reshape(N * H))
        state[~m.reshape(N, H).astype(bool)] = 0.0
    used = lib.kda_oracle_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate),
                                 _ptr(cu), N, H, dk, dv, float(scale), int(bool(qk_l2norm)),
                                 int(bool(erase)), _ptr(state), _ptr(y), _ptr(m), int(threads))
    if used < 0:
        raise MemoryError("oracle allocation failed")
    return y, state, used


def steps(q, k, v, g, beta, gate, state, *, scale=1.0, qk_l2norm=False, erase=True,
          mask=None, threads=0):
    """Run single-token steps: q, k, g [steps, N, H, dk]; v, gate [steps, N, H, dv];
    beta [steps, N, H]; state [N, H, dk, dv] (fp64 copy is advanced).
    Returns (y [steps, N, H, dv] fp64, state fp64, threads)."""
    lib = _load()
    q, k, v, g, beta, gate = map(_f32, (q, k, v, g, beta, gate))
    n_steps, N, H, dk = q.shape
    dv = v.shape[-1]
    st = np.array(state, dtype=np.float64, copy=True).reshape(N, H, dk, dv)
    y = np.zeros((n_steps, N, H, dv), dtype=np.float64)
    m = None
    if mask is not None:
        m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8).reshape(N * H))
    used = lib.kda_oracle_steps(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate),
                                n_steps, N, H, dk, dv, float(scale), int(bool(qk_l2norm)),
                                int(bool(erase)), _ptr(st), _ptr(y), _ptr(m), int(threads))
    if used < 0:
        raise MemoryError("oracle allocation failed")
    return y, st, used


def head(q, k, v, g, beta, gate=None, *, scale=1.0, qk_l2norm=False, initial_state=None,
         erase=True):
    """One (sequence, head): q, k, g [L, dk]; v, gate [L, dv]; beta [L].
    Returns (y [L, dv], S [dk, dv]) in fp64."""
    q = np.asarray(q)
    L, dk = q.shape
    dv = np.asarray(v).shape[-1]
    s0 = None if initial_state is None else np.asarray(initial_state).reshape(1, 1, dk, dv)
    y, S, _ = varlen(q.reshape(L, 1, dk), np.asarray(k).reshape(L, 1, dk),
                     np.asarray(v).reshape(L, 1, dv), np.asarray(g).reshape(L, 1, dk),
                     np.asarray(beta).reshape(L, 1),
                     None if gate is None else np.asarray(gate).reshape(L, 1, dv),
                     [0, L], scale=scale, qk_l2norm=qk_l2norm, initial_state=s0,
                     erase=erase, threads=1)
    return y.reshape(L, dv), S.reshape(dk, dv)
