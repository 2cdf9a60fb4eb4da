"""Python binding of the Tail-Replay C ABI (``include/gdn_tail_replay.h``).

Argument marshalling only: every step of the replay and the prefill runs in
the CUDA kernels of ``libgdn_tail_replay.so``.  PyTorch provides device
memory and streams.  There is no CPU fallback: if the library is missing the
import fails, and every call checks the status the library returns.

The low-level names mirror the C entry points (``gdn_plan_create_replay``,
``gdn_tail_replay_state``, ``gdn_tail_replay_outputs``, ``gdn_chunk_prefill``,
``gdn_decode_step``, ...).  ``ReplayPlan`` and
``PrefillPlan`` wrap a plan's lifetime; ``tail_replay_state`` and
``chunk_prefill`` are the one-call conveniences on torch tensors.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# GDN_DEBUG_BOUNDS=1 in the environment selects the debug build, whose kernels
# check every global index against the plan and report GDN_ERR_BOUNDS.
DEBUG_BOUNDS = os.environ.get("GDN_DEBUG_BOUNDS", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libgdn_tail_replay_debug.so" if DEBUG_BOUNDS else "libgdn_tail_replay.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, \
    GDN_ERR_ALLOC, GDN_ERR_MISMATCH, GDN_ERR_BOUNDS = range(8)
GDN_F32, GDN_BF16 = 0, 1
GDN_KERNEL_AUTO, GDN_KERNEL_RECURRENT, GDN_KERNEL_CHUNKED_TC = 0, 1, 2
# the chunked kernel with the state-only replay pinned to its two-CTA-per-SM kernel (the
# default), its warp-specialised one or its cluster-pair one
GDN_KERNEL_CHUNKED_TC_TWO_CTA, GDN_KERNEL_CHUNKED_TC_WARP_SPEC, GDN_KERNEL_CHUNKED_TC_PAIR = 3, 4, 5

EXPORTED = (
    "gdn_plan_create_replay", "gdn_plan_create_prefill", "gdn_plan_destroy", "gdn_replay_windows",
    "gdn_plan_window",
    "gdn_plan_info", "gdn_plan_launches", "gdn_workspace_bytes", "gdn_tail_replay_state", "gdn_chunk_prefill",
    "gdn_workspace_status", "gdn_status_string", "gdn_version", "gdn_tail_replay_state_noalloc",
    "gdn_tail_replay_outputs", "gdn_decode_step", "gdn_plan_create_fused", "gdn_tail_replay_prefill",
    "gdn_selftest_bounded_wait", "gdn_debug_fail_plan_allocations", "gdn_selftest_index_check",
    "gdn_debug_bounds_enabled",
)


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {gdn_status_string(status)} (status {status})")
        self.status = status


class gdn_varlen_desc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("d_k", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("kernel", ctypes.c_int32),
        ("seq_offsets_host", ctypes.POINTER(ctypes.c_int32)),
        ("row_stride_elems", ctypes.c_int64),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m gated_deltanet_state_tail_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    pd = ctypes.POINTER(gdn_varlen_desc)
    sig = {
        "gdn_plan_create_replay": (I32, [pd, P, P, ctypes.POINTER(P)]),
        "gdn_plan_create_prefill": (I32, [pd, ctypes.POINTER(P)]),
        "gdn_plan_destroy": (None, [P]),
        "gdn_replay_windows": (I32, [I32, P, P, P, P, P]),
        "gdn_plan_window": (I32, [P, I32, ctypes.POINTER(I64), ctypes.POINTER(I32)]),
        "gdn_plan_info": (I32, [P, ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I32)]),
        "gdn_plan_launches": (I32, [P, ctypes.POINTER(I32)]),
        "gdn_workspace_bytes": (ctypes.c_size_t, [P]),
        "gdn_tail_replay_state": (I32, [P, P, P, P, P, P, P, P, P, P, P, P]),
        "gdn_chunk_prefill": (I32, [P, P, P, P, P, P, P, P, P, P, P, P]),
        "gdn_workspace_status": (I32, [P, P]),
        "gdn_status_string": (ctypes.c_char_p, [I32]),
        "gdn_version": (I32, []),
        "gdn_tail_replay_state_noalloc": (I32, [pd, P, P, P, P, P, P, P, P, ctypes.POINTER(ctypes.c_uint32)]),
        "gdn_tail_replay_outputs": (I32, [P, P, P, P, P, P, P, P, P, P, P, P, P]),
        "gdn_decode_step": (I32, [I32, I32, I32, I32, I32, P, P, P, P, P, P, P, P, P]),
        "gdn_plan_create_fused": (I32, [pd, P, P, P, ctypes.POINTER(P)]),
        "gdn_tail_replay_prefill": (I32, [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P]),
        "gdn_selftest_bounded_wait": (I32, [ctypes.c_uint64, P, P]),
        "gdn_debug_fail_plan_allocations": (None, [I32]),
        "gdn_selftest_index_check": (I32, [P, P]),
        "gdn_debug_bounds_enabled": (I32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib_handle = None


def library():
    """The loaded ctypes handle of libgdn_tail_replay.so (loaded on first use;
    raises ImportError if the library has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


class _LazyLib:
    def __getattr__(self, name):
        return getattr(library(), name)


_lib = _LazyLib()


def gdn_status_string(status: int) -> str:
    return _lib.gdn_status_string(int(status)).decode()


def gdn_version() -> int:
    return int(_lib.gdn_version())


def _check(status: int, what: str):
    if status != GDN_OK:
        raise GdnError(status, what)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(t):
    """Device (or host) address of a tensor / numpy array, or None."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dtype_code(dtype) -> int:
    import torch
    if dtype in (torch.float32, "f32"):
        return GDN_F32
    if dtype in (torch.bfloat16, "bf16"):
        return GDN_BF16
    raise ValueError(f"unsupported dtype {dtype}")


def _make_desc(batch, H, dk, dv, dtype, kernel, offsets: np.ndarray, row_stride=0):
    d = gdn_varlen_desc()
    d.batch, d.num_heads, d.d_k, d.d_v = int(batch), int(H), int(dk), int(dv)
    d.dtype = _dtype_code(dtype)
    d.kernel = int(kernel)
    d.seq_offsets_host = offsets.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    d.row_stride_elems = int(row_stride)
    return d


def row_stride_of(*tensors) -> int:
    """Row stride (elements) shared by [rows, H, d] views of q, k and v, or 0 when each
    is packed.  Heads must be contiguous inside a row (strides (., d, 1))."""
    ts = [t for t in tensors if t is not None]
    for t in ts:
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("q/k/v must be [rows, H, d] views with contiguous heads inside a row")
    if all(t.stride(0) == t.shape[1] * t.shape[2] for t in ts):
        return 0
    rs = {t.stride(0) for t in ts}
    if len(rs) != 1:
        raise ValueError("q, k and v must share one row stride (or all be packed)")
    return rs.pop()


def gdn_plan_create_replay(H, dk, dv, dtype, seq_offsets, match_len, R, kernel=GDN_KERNEL_AUTO, row_stride=0):
    """Create a replay plan; returns the raw handle (int).  Host int arrays."""
    off, ml, rr = _i32(seq_offsets), _i32(match_len), _i32(R)
    if len(off) != len(ml) + 1 or len(rr) != len(ml):
        raise ValueError("seq_offsets must have batch + 1 entries, match_len and R batch entries")
    d = _make_desc(len(ml), H, dk, dv, dtype, kernel, off, row_stride)
    h = ctypes.c_void_p()
    _check(_lib.gdn_plan_create_replay(ctypes.byref(d), ml.ctypes.data, rr.ctypes.data,
                                       ctypes.byref(h)), "gdn_plan_create_replay")
    return h.value


def gdn_plan_create_prefill(H, dk, dv, dtype, cu_seqlens, kernel=GDN_KERNEL_AUTO, row_stride=0):
    off = _i32(cu_seqlens)
    d = _make_desc(len(off) - 1, H, dk, dv, dtype, kernel, off, row_stride)
    h = ctypes.c_void_p()
    _check(_lib.gdn_plan_create_prefill(ctypes.byref(d), ctypes.byref(h)), "gdn_plan_create_prefill")
    return h.value


def gdn_plan_create_fused(H, dk, dv, dtype, seq_offsets, match_len, R, suffix_offsets,
                          kernel=GDN_KERNEL_AUTO, row_stride=0):
    """Create a fused replay + suffix plan; returns the raw handle (int).  Host int arrays."""
    off, ml, rr, so = _i32(seq_offsets), _i32(match_len), _i32(R), _i32(suffix_offsets)
    if len(off) != len(ml) + 1 or len(rr) != len(ml) or len(so) != len(ml) + 1:
        raise ValueError("seq_offsets and suffix_offsets need batch + 1 entries, match_len and R batch")
    d = _make_desc(len(ml), H, dk, dv, dtype, kernel, off, row_stride)
    h = ctypes.c_void_p()
    _check(_lib.gdn_plan_create_fused(ctypes.byref(d), ml.ctypes.data, rr.ctypes.data, so.ctypes.data,
                                      ctypes.byref(h)), "gdn_plan_create_fused")
    return h.value


def gdn_replay_windows(seq_offsets, match_len, R):
    """Host-side replay windows: (row0 int64 [B], len int32 [B])."""
    off, ml, rr = _i32(seq_offsets), _i32(match_len), _i32(R)
    if len(off) != len(ml) + 1 or len(rr) != len(ml):
        raise ValueError("seq_offsets must have batch + 1 entries, match_len and R batch entries")
    row0 = np.zeros(len(ml), np.int64)
    ln = np.zeros(len(ml), np.int32)
    _check(_lib.gdn_replay_windows(len(ml), off.ctypes.data, ml.ctypes.data, rr.ctypes.data,
                                   row0.ctypes.data, ln.ctypes.data), "gdn_replay_windows")
    return row0, ln


def gdn_plan_destroy(handle):
    _lib.gdn_plan_destroy(handle)


def gdn_plan_window(handle, b):
    r0, ln = ctypes.c_int64(), ctypes.c_int32()
    _check(_lib.gdn_plan_window(handle, int(b), ctypes.byref(r0), ctypes.byref(ln)), "gdn_plan_window")
    return r0.value, ln.value


def gdn_plan_info(handle):
    u, t, k = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
    _check(_lib.gdn_plan_info(handle, ctypes.byref(u), ctypes.byref(t), ctypes.byref(k)), "gdn_plan_info")
    return {"units": u.value, "total_tokens": t.value, "kernel": k.value}


def gdn_plan_launches(handle) -> int:
    n = ctypes.c_int32()
    _check(_lib.gdn_plan_launches(handle, ctypes.byref(n)), "gdn_plan_launches")
    return n.value


def gdn_workspace_bytes(handle) -> int:
    return int(_lib.gdn_workspace_bytes(handle))


def gdn_tail_replay_state(handle, q, k, v, alpha, beta, seq_offsets, match_len, R, state_out,
                          workspace, stream=None):
    """Launch the tail replay (tensors on the plan's device; any may be a raw int address)."""
    _check(_lib.gdn_tail_replay_state(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                      _ptr(seq_offsets), _ptr(match_len), _ptr(R), _ptr(state_out),
                                      _ptr(workspace), _stream_handle(stream)),
           "gdn_tail_replay_state")


def gdn_tail_replay_outputs(handle, q, k, v, alpha, beta, seq_offsets, match_len, R, o_out, state_out,
                            workspace, stream=None):
    """Tail replay that also writes o_t = S_t^T q_t for every window row (rows of o_out
    outside the windows are left untouched)."""
    _check(_lib.gdn_tail_replay_outputs(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                        _ptr(seq_offsets), _ptr(match_len), _ptr(R), _ptr(o_out),
                                        _ptr(state_out), _ptr(workspace), _stream_handle(stream)),
           "gdn_tail_replay_outputs")


def gdn_tail_replay_prefill(handle, k, v, alpha, beta, sq, sk, sv, salpha, sbeta, o_out, state_mid,
                            state_out, workspace, stream=None):
    """Fused rebuild of the states and prefill of the suffixes (one launch on the
    tensor-core kernel)."""
    _check(_lib.gdn_tail_replay_prefill(handle, _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(sq), _ptr(sk),
                                        _ptr(sv), _ptr(salpha), _ptr(sbeta), _ptr(o_out), _ptr(state_mid),
                                        _ptr(state_out), _ptr(workspace), _stream_handle(stream)),
           "gdn_tail_replay_prefill")


def gdn_decode_step(q, k, v, alpha, beta, state_in, state_out, o_out, stream=None):
    """One decode step on dense [B, H, d] tensors (state [B, H, dk, dv] fp32; state_out may be
    state_in for an in-place update)."""
    B, H, dk = k.shape
    dv = v.shape[2]
    _check(_lib.gdn_decode_step(int(B), int(H), int(dk), int(dv), _dtype_code(k.dtype), _ptr(q), _ptr(k),
                                _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state_in), _ptr(state_out),
                                _ptr(o_out), _stream_handle(stream)),
           "gdn_decode_step")


def gdn_chunk_prefill(handle, q, k, v, alpha, beta, cu_seqlens, state_in, o_out, state_out,
                      workspace, stream=None):
    _check(_lib.gdn_chunk_prefill(handle, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                  _ptr(cu_seqlens), _ptr(state_in), _ptr(o_out), _ptr(state_out),
                                  _ptr(workspace), _stream_handle(stream)),
           "gdn_chunk_prefill")


def gdn_tail_replay_state_noalloc(H, dk, dv, dtype, seq_offsets, match_len, R, k, v, alpha, beta,
                                  state_out, kernel=GDN_KERNEL_AUTO, stream=None, wait_status=True,
                                  row_stride=0):
    """Replay without any device allocation (schedule in the library's fixed
    device array).  Returns the device status word when wait_status is set."""
    off, ml, rr = _i32(seq_offsets), _i32(match_len), _i32(R)
    if len(off) != len(ml) + 1 or len(rr) != len(ml):
        raise ValueError("seq_offsets must have batch + 1 entries, match_len and R batch entries")
    d = _make_desc(len(ml), H, dk, dv, dtype, kernel, off, row_stride)
    st = ctypes.c_uint32(0xFFFFFFFF)
    _check(_lib.gdn_tail_replay_state_noalloc(ctypes.byref(d), ml.ctypes.data, rr.ctypes.data,
                                              _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                              _ptr(state_out), _stream_handle(stream),
                                              ctypes.byref(st) if wait_status else None),
           "gdn_tail_replay_state_noalloc")
    return st.value if wait_status else None


def gdn_selftest_bounded_wait(limit_ns, workspace, stream=None):
    """Launch the failure-path self-test: a device wait bounded by limit_ns that runs out."""
    _check(_lib.gdn_selftest_bounded_wait(int(limit_ns), _ptr(workspace), _stream_handle(stream)),
           "gdn_selftest_bounded_wait")


def gdn_selftest_index_check(workspace, stream=None):
    """Debug build only: run one failing index check (access skipped); the workspace
    status then reads GDN_ERR_BOUNDS."""
    _check(_lib.gdn_selftest_index_check(_ptr(workspace), _stream_handle(stream)), "gdn_selftest_index_check")


def gdn_debug_bounds_enabled() -> bool:
    return bool(_lib.gdn_debug_bounds_enabled())


def gdn_debug_fail_plan_allocations(count):
    """Make the next `count` plan creations fail with GDN_ERR_ALLOC (0 clears it)."""
    _lib.gdn_debug_fail_plan_allocations(int(count))


def gdn_workspace_status(workspace, stream=None) -> int:
    """Synchronise the stream and return the device-side status of the last call."""
    return int(_lib.gdn_workspace_status(_ptr(workspace), _stream_handle(stream)))


class _Plan:
    def __init__(self, handle, H, dk, dv, dtype, batch):
        import torch
        self.handle, self.H, self.dk, self.dv, self.dtype, self.batch = handle, H, dk, dv, dtype, batch
        self.info = gdn_plan_info(handle)
        self.launches = gdn_plan_launches(handle)   # kernel launches per call
        self.workspace = torch.zeros(gdn_workspace_bytes(handle), dtype=torch.uint8, device="cuda")

    def window(self, b):
        return gdn_plan_window(self.handle, b)

    def status(self, stream=None) -> int:
        return gdn_workspace_status(self.workspace, stream)

    def check(self, stream=None):
        _check(self.status(stream), "device status")

    def close(self):
        if self.handle:
            gdn_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ReplayPlan(_Plan):
    """Plan of a tail replay over a packed varlen cache (host int arrays)."""

    def __init__(self, H, dk, dv, dtype, seq_offsets, match_len, R, kernel=GDN_KERNEL_AUTO, row_stride=0):
        h = gdn_plan_create_replay(H, dk, dv, dtype, seq_offsets, match_len, R, kernel, row_stride)
        super().__init__(h, H, dk, dv, dtype, len(match_len))

    def run(self, k, v, alpha, beta, state_out, q=None, seq_offsets=None, match_len=None, R=None,
            stream=None, workspace=None):
        gdn_tail_replay_state(self.handle, q, k, v, alpha, beta, seq_offsets, match_len, R,
                              state_out, self.workspace if workspace is None else workspace, stream)

    def run_outputs(self, q, k, v, alpha, beta, o_out, state_out=None, seq_offsets=None, match_len=None,
                    R=None, stream=None, workspace=None):
        """Replay that also writes the window rows of o_out (see gdn_tail_replay_outputs)."""
        gdn_tail_replay_outputs(self.handle, q, k, v, alpha, beta, seq_offsets, match_len, R, o_out,
                                state_out, self.workspace if workspace is None else workspace, stream)


class PrefillPlan(_Plan):
    """Plan of a chunked prefill over whole packed sequences (host cu_seqlens)."""

    def __init__(self, H, dk, dv, dtype, cu_seqlens, kernel=GDN_KERNEL_AUTO, row_stride=0):
        h = gdn_plan_create_prefill(H, dk, dv, dtype, cu_seqlens, kernel, row_stride)
        super().__init__(h, H, dk, dv, dtype, len(cu_seqlens) - 1)

    def run(self, q, k, v, alpha, beta, o_out, state_in=None, state_out=None, cu_seqlens=None,
            stream=None, workspace=None):
        gdn_chunk_prefill(self.handle, q, k, v, alpha, beta, cu_seqlens, state_in, o_out, state_out,
                          self.workspace if workspace is None else workspace, stream)


class FusedPlan(_Plan):
    """Plan of a fused replay + suffix prefill (host int arrays)."""

    def __init__(self, H, dk, dv, dtype, seq_offsets, match_len, R, suffix_offsets, kernel=GDN_KERNEL_AUTO,
                 row_stride=0):
        h = gdn_plan_create_fused(H, dk, dv, dtype, seq_offsets, match_len, R, suffix_offsets, kernel,
                                  row_stride)
        super().__init__(h, H, dk, dv, dtype, len(match_len))

    def run(self, k, v, alpha, beta, sq, sk, sv, salpha, sbeta, o_out, state_out, state_mid=None, stream=None,
            workspace=None):
        gdn_tail_replay_prefill(self.handle, k, v, alpha, beta, sq, sk, sv, salpha, sbeta, o_out, state_mid,
                                state_out, self.workspace if workspace is None else workspace, stream)


def tail_replay_state(k, v, alpha, beta, seq_offsets, match_len, R, kernel=GDN_KERNEL_AUTO):
    """One-shot replay on torch CUDA tensors; returns state [B, H, dk, dv] fp32.  k and v
    may be row-strided views (e.g. slices of one fused projection buffer)."""
    import torch
    rows, H, dk = k.shape
    dv = v.shape[2]
    plan = ReplayPlan(H, dk, dv, k.dtype, seq_offsets, match_len, R, kernel, row_stride_of(k, v))
    out = torch.empty((plan.batch, H, dk, dv), dtype=torch.float32, device=k.device)
    plan.run(k, v, alpha, beta, out)
    plan.check()
    plan.close()
    return out


def chunk_prefill(q, k, v, alpha, beta, cu_seqlens, state_in=None, kernel=GDN_KERNEL_AUTO):
    """One-shot prefill on torch CUDA tensors; returns (o, state_out).  q, k and v may be
    row-strided views sharing one row stride; o is packed."""
    import torch
    rows, H, dk = k.shape
    dv = v.shape[2]
    plan = PrefillPlan(H, dk, dv, k.dtype, cu_seqlens, kernel, row_stride_of(q, k, v))
    o = torch.empty((rows, H, dv), dtype=k.dtype, device=k.device)
    st = torch.empty((plan.batch, H, dk, dv), dtype=torch.float32, device=k.device)
    plan.run(q, k, v, alpha, beta, o, state_in=state_in, state_out=st)
    plan.check()
    plan.close()
    return o, st


def decode_step(q, k, v, alpha, beta, state, o=None, in_place=True):
    """One decode step on torch CUDA tensors ([B, H, d], state [B, H, dk, dv] fp32).
    Updates `state` in place (or returns a new one) and returns (o, state)."""
    import torch
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    out = state if in_place else torch.empty_like(state)
    gdn_decode_step(q, k, v, alpha, beta, state, out, o)
    return o, out
