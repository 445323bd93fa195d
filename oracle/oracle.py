"""Python face of the fp64 CPU oracle for Lightning Attention.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check of the entry module
and the CPU-baseline leg of the benchmark may import this module; the product
package never does, and this module never imports the product package.

The arithmetic lives in ``lightning_oracle.c`` (plain fp64 loops, OpenMP over
independent (sequence, head) pairs).  This wrapper only builds that file with
gcc, checks shapes and marshals numpy arrays.  Inputs are bf16 bit patterns
(``numpy.uint16``), packed token-major ``[T, H, d]``; outputs are float64.

Forms (see the C file for the cited passages):
  recurrent(...)   S_t = S_{t-1} + k_t^T v_t,  o_t = q_t S_t
  quadratic(...)   o_t = sum_{s<=t} (q_t . k_s) v_s  (+ q_t S_in)
  blocked(...)     intra-block left product + inter-block right product
  segmented(...)   LASP+ recipe: local sums, gather, global prefix, blocked scan
  decode_step(...) one recurrent step on a persistent state
  *_decay(...)     the same forms with a per-head decay lambda_h (a reading:
                   S_t = lambda S_{t-1} + k_t^T v_t; see the C file)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lightning_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD_DIR, "liblaoracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (OpenMP, -O2, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def build_variant(source_text: str, so_path: str):
    """Compile ``source_text`` (a modified copy of the oracle, used by the tests
    that plant a mistake to show the pins catch it) and return its handle."""
    c_path = so_path[:-3] + ".c"
    with open(c_path, "w") as f:
        f.write(source_text)
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11", c_path,
                    "-o", so_path, "-lm"], check=True)
    return _bind(so_path)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _bind(path: str):
    """Load an oracle shared library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    i32p = ctypes.POINTER(ctypes.c_int32)
    f64p = ctypes.POINTER(ctypes.c_double)
    c_int = ctypes.c_int
    common = [u16p, u16p, u16p, i32p, c_int, c_int, c_int, i32p, c_int]
    for name in ("lao_recurrent", "lao_quadratic"):
        fn = getattr(lib, name)
        fn.argtypes = common + [f64p, f64p, f64p, c_int]
        fn.restype = c_int
    lib.lao_blocked.argtypes = common + [c_int, f64p, f64p, f64p, c_int]
    lib.lao_blocked.restype = c_int
    lib.lao_segmented.argtypes = common + [c_int, c_int, f64p, f64p, f64p, c_int]
    lib.lao_segmented.restype = c_int
    lib.lao_decode_step.argtypes = [u16p, u16p, u16p, c_int, c_int, c_int, f64p, f64p, c_int]
    lib.lao_decode_step.restype = c_int
    lib.lao_backward.argtypes = [u16p, u16p, u16p, u16p, i32p, c_int, c_int, c_int, i32p, c_int,
                                 f64p, f64p, f64p, f64p, f64p, f64p, c_int]
    lib.lao_backward.restype = c_int
    f64c = ctypes.POINTER(ctypes.c_double)
    for name in ("lao_recurrent_decay", "lao_quadratic_decay"):
        fn = getattr(lib, name)
        fn.argtypes = common + [f64c, f64p, f64p, f64p, c_int]
        fn.restype = c_int
    lib.lao_blocked_decay.argtypes = common + [c_int, f64c, f64p, f64p, f64p, c_int]
    lib.lao_blocked_decay.restype = c_int
    lib.lao_segmented_decay.argtypes = common + [c_int, c_int, f64c, f64p, f64p, f64p, c_int]
    lib.lao_segmented_decay.restype = c_int
    lib.lao_decode_step_decay.argtypes = [u16p, u16p, u16p, c_int, c_int, c_int, f64c, f64p, f64p, c_int]
    lib.lao_decode_step_decay.restype = c_int
    lib.lao_max_threads.argtypes = []
    lib.lao_max_threads.restype = c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def max_threads() -> int:
    """Threads the oracle's OpenMP loops use by default on this host."""
    return int(_load().lao_max_threads())


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype)) if a is not None else None


def _prep(q, k, v, cu_seqlens, heads, state_in):
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must be [T, H, d] bf16 bit arrays of one shape")
    T, H, d = q.shape
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    if cu.ndim != 1 or cu.size < 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must be int32 [nseq+1], 0, non-decreasing, ending at T")
    nseq = cu.size - 1
    hs = np.arange(H, dtype=np.int32) if heads is None else np.ascontiguousarray(heads, dtype=np.int32)
    nh = hs.size
    if state_in is not None:
        state_in = np.ascontiguousarray(state_in, dtype=np.float64)
        if state_in.shape != (nseq, nh, d, d):
            raise ValueError(f"state_in must be [nseq, nheads, d, d] = {(nseq, nh, d, d)}")
    return q, k, v, cu, nseq, T, H, d, hs, nh, state_in


def _run(name, q, k, v, cu_seqlens, heads, state_in, threads, extra=(), lib=None):
    q, k, v, cu, nseq, T, H, d, hs, nh, state_in = _prep(q, k, v, cu_seqlens, heads, state_in)
    out = np.zeros((T, nh, d), dtype=np.float64)
    state_out = np.zeros((nseq, nh, d, d), dtype=np.float64)
    fn = getattr(lib or _load(), name)
    rc = fn(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
            _ptr(cu, ctypes.c_int32), nseq, H, d, _ptr(hs, ctypes.c_int32), nh, *extra,
            _ptr(state_in, ctypes.c_double), _ptr(out, ctypes.c_double),
            _ptr(state_out, ctypes.c_double), int(threads or 0))
    if rc != 0:
        raise ValueError(f"{name} rejected its arguments")
    return out, state_out


def recurrent(q, k, v, cu_seqlens, heads=None, state_in=None, threads=None, lib=None):
    """Token-by-token recurrent form. Returns (out [T, nh, d], state [nseq, nh, d, d])."""
    return _run("lao_recurrent", q, k, v, cu_seqlens, heads, state_in, threads, lib=lib)


def quadratic(q, k, v, cu_seqlens, heads=None, state_in=None, threads=None, lib=None):
    """Masked left-product form O = (QK^T ⊙ M)V (+ Q S_in)."""
    return _run("lao_quadratic", q, k, v, cu_seqlens, heads, state_in, threads, lib=lib)


def blocked(q, k, v, cu_seqlens, block, heads=None, state_in=None, threads=None, lib=None):
    """Blocked form: intra-block left product, inter-block right product."""
    return _run("lao_blocked", q, k, v, cu_seqlens, heads, state_in, threads, (int(block),),
                lib=lib)


def segmented(q, k, v, cu_seqlens, seg_len, block, heads=None, state_in=None, threads=None,
              lib=None):
    """LASP+ recipe over segments of ``seg_len`` tokens, each scanned in blocks."""
    return _run("lao_segmented", q, k, v, cu_seqlens, heads, state_in, threads,
                (int(seg_len), int(block)), lib=lib)


def _decay_arr(decay, H):
    lam = np.ascontiguousarray(decay, dtype=np.float64)
    if lam.shape != (H,):
        raise ValueError(f"decay must hold one value per head, shape ({H},)")
    return lam


def _run_decay(name, q, k, v, cu_seqlens, decay, heads, state_in, threads, extra=(), lib=None):
    q, k, v, cu, nseq, T, H, d, hs, nh, state_in = _prep(q, k, v, cu_seqlens, heads, state_in)
    lam = _decay_arr(decay, H)
    out = np.zeros((T, nh, d), dtype=np.float64)
    state_out = np.zeros((nseq, nh, d, d), dtype=np.float64)
    fn = getattr(lib or _load(), name)
    rc = fn(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
            _ptr(cu, ctypes.c_int32), nseq, H, d, _ptr(hs, ctypes.c_int32), nh, *extra,
            _ptr(lam, ctypes.c_double), _ptr(state_in, ctypes.c_double), _ptr(out, ctypes.c_double),
            _ptr(state_out, ctypes.c_double), int(threads or 0))
    if rc != 0:
        raise ValueError(f"{name} rejected its arguments")
    return out, state_out


def recurrent_decay(q, k, v, cu_seqlens, decay, heads=None, state_in=None, threads=None, lib=None):
    """Decayed recurrent form S_t = lambda_h S_{t-1} + k_t^T v_t, o_t = q_t S_t;
    decay: one value per head (length H, indexed by head number)."""
    return _run_decay("lao_recurrent_decay", q, k, v, cu_seqlens, decay, heads, state_in, threads, lib=lib)


def quadratic_decay(q, k, v, cu_seqlens, decay, heads=None, state_in=None, threads=None, lib=None):
    """Decayed closed form o_t = sum_{s<=t} lambda^{t-s} (q_t . k_s) v_s + lambda^{t+1} q_t S_in."""
    return _run_decay("lao_quadratic_decay", q, k, v, cu_seqlens, decay, heads, state_in, threads, lib=lib)


def blocked_decay(q, k, v, cu_seqlens, block, decay, heads=None, state_in=None, threads=None, lib=None):
    """Decayed blocked form (intra-block decay mask, row-scaled inter term, decayed state update)."""
    return _run_decay("lao_blocked_decay", q, k, v, cu_seqlens, decay, heads, state_in, threads,
                      (int(block),), lib=lib)


def segmented_decay(q, k, v, cu_seqlens, seg_len, block, decay, heads=None, state_in=None, threads=None,
                    lib=None):
    """Decayed LASP+ recipe over segments of ``seg_len`` tokens."""
    return _run_decay("lao_segmented_decay", q, k, v, cu_seqlens, decay, heads, state_in, threads,
                      (int(seg_len), int(block)), lib=lib)


def decode_step_decay(q, k, v, state, decay, threads=None, lib=None):
    """One decayed decode step S <- lambda_h S + k^T v, o = q S (copies the state)."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must be [B, H, d] bf16 bit arrays of one shape")
    B, H, d = q.shape
    lam = _decay_arr(decay, H)
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    if st.shape != (B, H, d, d):
        raise ValueError("state must be [B, H, d, d]")
    out = np.zeros((B, H, d), dtype=np.float64)
    rc = (lib or _load()).lao_decode_step_decay(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                                                _ptr(v, ctypes.c_uint16), B, H, d, _ptr(lam, ctypes.c_double),
                                                _ptr(st, ctypes.c_double), _ptr(out, ctypes.c_double),
                                                int(threads or 0))
    if rc != 0:
        raise ValueError("lao_decode_step_decay rejected its arguments")
    return out, st


def decode_step(q, k, v, state, threads=None, lib=None):
    """One decode step. q, k, v: bf16 bits [B, H, d]; state: float64 [B, H, d, d]
    (a copy is updated and returned). Returns (out [B, H, d], new_state)."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must be [B, H, d] bf16 bit arrays of one shape")
    B, H, d = q.shape
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    if st.shape != (B, H, d, d):
        raise ValueError("state must be [B, H, d, d]")
    out = np.zeros((B, H, d), dtype=np.float64)
    rc = (lib or _load()).lao_decode_step(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                                 _ptr(v, ctypes.c_uint16), B, H, d,
                                 _ptr(st, ctypes.c_double), _ptr(out, ctypes.c_double),
                                 int(threads or 0))
    if rc != 0:
        raise ValueError("lao_decode_step rejected its arguments")
    return out, st


def backward(q, k, v, dout, cu_seqlens, heads=None, state_in=None, dstate_out=None, threads=None,
             lib=None):
    """Gradients of the forward definition for dL/dO = dout (bf16 bits, like
    q) and dL/dS_out = dstate_out (float64 [nseq, nh, d, d] or None).
    Returns (dq, dk, dv [T, nh, d], dstate_in [nseq, nh, d, d])."""
    q, k, v, cu, nseq, T, H, d, hs, nh, state_in = _prep(q, k, v, cu_seqlens, heads, state_in)
    g = np.ascontiguousarray(dout, dtype=np.uint16)
    if g.shape != q.shape:
        raise ValueError("dout must have the shape of q")
    if dstate_out is not None:
        dstate_out = np.ascontiguousarray(dstate_out, dtype=np.float64)
        if dstate_out.shape != (nseq, nh, d, d):
            raise ValueError(f"dstate_out must be [nseq, nheads, d, d] = {(nseq, nh, d, d)}")
    dq, dk, dv = (np.zeros((T, nh, d), dtype=np.float64) for _ in range(3))
    dsin = np.zeros((nseq, nh, d, d), dtype=np.float64)
    rc = (lib or _load()).lao_backward(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                                       _ptr(v, ctypes.c_uint16), _ptr(g, ctypes.c_uint16),
                                       _ptr(cu, ctypes.c_int32), nseq, H, d, _ptr(hs, ctypes.c_int32), nh,
                                       _ptr(state_in, ctypes.c_double), _ptr(dstate_out, ctypes.c_double),
                                       _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                                       _ptr(dv, ctypes.c_double), _ptr(dsin, ctypes.c_double),
                                       int(threads or 0))
    if rc != 0:
        raise ValueError("lao_backward rejected its arguments")
    return dq, dk, dv, dsin
