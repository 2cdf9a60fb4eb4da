"""fp64 CPU oracle for Gated DeltaNet tail replay and suffix prefill.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The product path (``gated_deltanet_state_tail_b200``) never does,
and this package never imports the product path: the two share no code.

The arithmetic lives in ``gdn_oracle.c`` (plain token-by-token fp64 loops);
this module only builds it with gcc and marshals numpy arrays through ctypes.
See the header of ``gdn_oracle.c`` for what is computed and which passage of
the Tail-Replay pages each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")

F32, BF16 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into libgdn_oracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_replay_state.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_replay_state.restype = I
        lib.oracle_prefill.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P]
        lib.oracle_prefill.restype = I
        lib.oracle_recurrence_f64.argtypes = [ctypes.c_int64, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_recurrence_f64.restype = None
        lib.oracle_replay_window.argtypes = [I, P, P, P, I, P, P]
        lib.oracle_replay_window.restype = I
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _qkv(x):
    """Return (contiguous array, dtype code): float32 stays fp32, uint16 means bf16 bits."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle takes float32 or bf16 bits (uint16), got {x.dtype}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def recurrence(k, v, alpha, beta, q=None, S0=None):
    """Token-by-token gated delta rule for one head in fp64.

    k [n, dk], v [n, dv], alpha [n], beta [n], q [n, dk] or None, S0 [dk, dv] or None.
    Returns (S_final [dk, dv], o [n, dv] or None).
    """
    lib = _load()
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    n, dk = k.shape
    dv = v.shape[1]
    a = np.ascontiguousarray(alpha, dtype=np.float64)
    b = np.ascontiguousarray(beta, dtype=np.float64)
    qq = None if q is None else np.ascontiguousarray(q, dtype=np.float64)
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64, copy=True)
    o = None if q is None else np.zeros((n, dv))
    work = np.zeros(dv)
    lib.oracle_recurrence_f64(n, dk, dv, _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(qq),
                              _ptr(S), _ptr(o), _ptr(work))
    return S, o


def replay_window(seq_offsets, match_len, R, b):
    """(first row, length) of sequence b's replay window, or None if invalid."""
    lib = _load()
    so = np.ascontiguousarray(seq_offsets, dtype=np.int32)
    ml = np.ascontiguousarray(match_len, dtype=np.int32)
    rr = np.ascontiguousarray(R, dtype=np.int32)
    r0 = ctypes.c_int64()
    ln = ctypes.c_int64()
    rc = lib.oracle_replay_window(len(ml), _ptr(so), _ptr(ml), _ptr(rr), b,
                                  ctypes.byref(r0), ctypes.byref(ln))
    return None if rc else (r0.value, ln.value)


def replay_state(k, v, alpha, beta, seq_offsets, match_len, R):
    """Tail replay over a packed varlen batch; returns fp64 state [B, H, dk, dv].

    k [rows, H, dk], v [rows, H, dv] as float32 or bf16 bits (uint16);
    alpha, beta [rows, H] float32; seq_offsets [B+1], match_len [B], R [B] int32.
    """
    lib = _load()
    k, dt = _qkv(k)
    v, dt2 = _qkv(v)
    assert dt == dt2
    rows, H, dk = k.shape
    dv = v.shape[2]
    a = np.ascontiguousarray(alpha, dtype=np.float32)
    b = np.ascontiguousarray(beta, dtype=np.float32)
    so = np.ascontiguousarray(seq_offsets, dtype=np.int32)
    ml = np.ascontiguousarray(match_len, dtype=np.int32)
    rr = np.ascontiguousarray(R, dtype=np.int32)
    B = len(ml)
    out = np.zeros((B, H, dk, dv))
    rc = lib.oracle_replay_state(B, H, dk, dv, dt, _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                 _ptr(so), _ptr(ml), _ptr(rr), _ptr(out))
    if rc:
        raise ValueError(f"oracle_replay_state rejected its arguments (rc={rc})")
    return out


def prefill(q, k, v, alpha, beta, cu_seqlens, state_in=None, want_state=True):
    """Prefill over a packed varlen batch from state_in (None = zero state).

    Returns (o [rows, H, dv] fp64, state_out [B, H, dk, dv] fp64 or None).
    """
    lib = _load()
    q, dt = _qkv(q)
    k, dt1 = _qkv(k)
    v, dt2 = _qkv(v)
    assert dt == dt1 == dt2
    rows, H, dk = k.shape
    dv = v.shape[2]
    a = np.ascontiguousarray(alpha, dtype=np.float32)
    b = np.ascontiguousarray(beta, dtype=np.float32)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    B = len(cu) - 1
    si = None if state_in is None else np.ascontiguousarray(state_in, dtype=np.float64)
    o = np.zeros((rows, H, dv))
    so = np.zeros((B, H, dk, dv)) if want_state else None
    rc = lib.oracle_prefill(B, H, dk, dv, dt, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                            _ptr(cu), _ptr(si), _ptr(o), _ptr(so))
    if rc:
        raise ValueError(f"oracle_prefill rejected its arguments (rc={rc})")
    return o, so
