"""fp64 CPU oracle for the varlen attention forward — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  It shares no code with the CUDA
library in ``flash_attention_fwd_b200`` and never imports it.

Two independent implementations live here:

* ``varlen_attn_oracle.c`` (loaded through ctypes): the packed attention
  forward defined by the boostr 0.2.0 source page
  src/ops/cpu/attention/varlen_attention.rs (``varlen_attention_fwd``),
  written from the definition in double precision (visible keys gathered
  first, the LSE as a separate log-sum-exp, O as the exp(s - LSE)-weighted
  sum of values) and threaded over (sequence, head) work items.
* ``brute.py``: a dense NumPy restatement of the same definition that builds
  the full [Tq, Tk] score matrix with a block-diagonal (and causal) mask.
  Used only on tiny inputs to pin the C oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "varlen_attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_varlen.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODE = {"bf16": 0, "fp16": 1}


def build(force: bool = False) -> str:
    """Compile the C oracle into a shared object next to its source."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_varlen_attn_fwd.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32,
                                           i32, f64, P, P, i32]
    lib.oracle_varlen_attn_fwd.restype = i32
    lib.oracle_varlen_attn_rows.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32,
                                            i32, f64, P, P, i64, P, P, i32]
    lib.oracle_varlen_attn_rows.restype = i32
    lib.oracle_decode16.argtypes = [ctypes.c_uint16, i32]
    lib.oracle_decode16.restype = f64
    lib.oracle_varlen_attn_fwd_ext.argtypes = [P, P, P, i32, P, P, P, i32, i32, i32, i32,
                                               i32, i32, i32, P, f64, P, P, i32]
    lib.oracle_varlen_attn_fwd_ext.restype = i32
    lib.oracle_varlen_attn_rows_ext.argtypes = [P, P, P, i32, P, P, P, i32, i32, i32, i32,
                                                i32, i32, i32, P, f64, P, P, i64, P, P, i32]
    lib.oracle_varlen_attn_rows_ext.restype = i32
    lib.oracle_varlen_attn_bwd.argtypes = [P, P, P, P, P, P, i32, P, P, i32, i32, i32, i32,
                                           i32, f64, P, P, P, i32]
    lib.oracle_varlen_attn_bwd.restype = i32
    return lib


def load_variant(src_path: str, so_path: str):
    """Compile another copy of the oracle source (used by the tests that plant
    a mistake in the oracle to show that the pins catch it)."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", src_path, "-o", so_path, "-lm"]
    subprocess.run(cmd, check=True)
    return _bind(ctypes.CDLL(so_path))


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def default_threads() -> int:
    return os.cpu_count() or 1


def _bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a CPU bf16/fp16 tensor, C-contiguous."""
    t = t.detach().contiguous().cpu()
    return t.view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(x) -> np.ndarray:
    """Any float tensor or array, widened exactly to a C-contiguous float64 array."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def decode16(bits: int, dtype: str) -> float:
    return _load().oracle_decode16(bits, DTYPE_CODE[dtype])


def _seqused(seqused_k):
    if seqused_k is None:
        return None, ctypes.c_void_p(0)
    a = np.ascontiguousarray(np.asarray(seqused_k, dtype=np.int32))
    return a, _ptr(a)


def _sinks(sinks, H):
    if sinks is None:
        return None, ctypes.c_void_p(0)
    a = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(-1))
    if a.shape[0] != H:
        raise ValueError("sinks needs one value per query head")
    return a, _ptr(a)


def varlen_attn_fwd(q, k, v, cu_q, cu_k, H, Hkv, D, causal, scale, dtype, nthreads=None,
                    lib=None, window_left=-1, window_right=-1, seqused_k=None, sinks=None):
    """Full fp64 forward.  Returns (out [Tq,H,D] float64, lse [Tq,H] float64).
    window_left/right < 0 mean unbounded; seqused_k (length B) caps the keys
    of each sequence; sinks (length H) adds one logit per query head to the
    softmax normalisation."""
    lib = lib or _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    B = len(cq) - 1
    Tq = int(cq[-1]) if B >= 0 else 0
    out = np.zeros((Tq, H, D), dtype=np.float64)
    lse = np.zeros((Tq, H), dtype=np.float64)
    keep, su = _seqused(seqused_k)
    keep_s, sk = _sinks(sinks, H)
    if window_left < 0 and window_right < 0 and seqused_k is None and sinks is None:
        rc = lib.oracle_varlen_attn_fwd(_ptr(qb), _ptr(kb), _ptr(vb), DTYPE_CODE[dtype],
                                        _ptr(cq), _ptr(ck), B, H, Hkv, D, int(bool(causal)),
                                        float(scale), _ptr(out), _ptr(lse),
                                        nthreads or default_threads())
    else:
        rc = lib.oracle_varlen_attn_fwd_ext(_ptr(qb), _ptr(kb), _ptr(vb), DTYPE_CODE[dtype],
                                            _ptr(cq), _ptr(ck), su, B, H, Hkv, D,
                                            int(bool(causal)), int(window_left),
                                            int(window_right), sk, float(scale), _ptr(out),
                                            _ptr(lse), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_varlen_attn_fwd failed with code %d" % rc)
    return out, lse


def varlen_attn_rows(q, k, v, cu_q, cu_k, H, Hkv, D, causal, scale, dtype, rows,
                     nthreads=None, lib=None, window_left=-1, window_right=-1,
                     seqused_k=None, sinks=None):
    """fp64 forward of selected rows.  rows: int array [n, 2] of (token, head).
    Returns (out [n, D], lse [n])."""
    lib = lib or _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
    tok = np.ascontiguousarray(rows[:, 0])
    head = np.ascontiguousarray(rows[:, 1].astype(np.int32))
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    keep, su = _seqused(seqused_k)
    keep_s, sk = _sinks(sinks, H)
    rc = lib.oracle_varlen_attn_rows_ext(_ptr(qb), _ptr(kb), _ptr(vb), DTYPE_CODE[dtype],
                                         _ptr(cq), _ptr(ck), su, len(cq) - 1, H, Hkv, D,
                                         int(bool(causal)), int(window_left), int(window_right),
                                         sk, float(scale), _ptr(tok), _ptr(head), n, _ptr(out),
                                         _ptr(lse), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_varlen_attn_rows failed with code %d" % rc)
    return out, lse


def run_case(case, nthreads=None, lib=None, **mask):
    """Full oracle forward of a ``workloads.Case`` (mask: window_left,
    window_right, seqused_k, sinks)."""
    return varlen_attn_fwd(case.q, case.k, case.v, case.cu_q.numpy(), case.cu_k.numpy(),
                           case.H, case.Hkv, case.D, case.causal, case.scale, case.dtype,
                           nthreads, lib=lib, **mask)


def run_case_rows(case, rows, nthreads=None, **mask):
    return varlen_attn_rows(case.q, case.k, case.v, case.cu_q.numpy(), case.cu_k.numpy(),
                            case.H, case.Hkv, case.D, case.causal, case.scale, case.dtype,
                            rows, nthreads, **mask)


def varlen_attn_bwd(dout, q, k, v, out, lse, cu_q, cu_k, H, Hkv, D, causal, scale, dtype,
                    nthreads=None, lib=None):
    """fp64 gradient of the forward (the page's varlen_attention_bwd).  dout/q [Tq,H,D] and k/v [Tk,Hkv,D]
    are bf16/fp16 tensors; out [Tq,H,D] and lse [Tq,H] any float tensor or
    array (widened to double).  Returns (dq [Tq,H,D], dk [Tk,Hkv,D],
    dv [Tk,Hkv,D]) float64."""
    lib = lib or _load()
    db, qb, kb, vb = _bits(dout), _bits(q), _bits(k), _bits(v)
    ob = _f64(out)
    lse_d = _f64(lse)
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    B = len(cq) - 1
    Tq, Tk = int(cq[-1]), int(ck[-1])
    dq = np.zeros((Tq, H, D), dtype=np.float64)
    dk = np.zeros((Tk, Hkv, D), dtype=np.float64)
    dv = np.zeros((Tk, Hkv, D), dtype=np.float64)
    rc = lib.oracle_varlen_attn_bwd(_ptr(db), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(ob),
                                    _ptr(lse_d), DTYPE_CODE[dtype], _ptr(cq), _ptr(ck), B, H, Hkv,
                                    D, int(bool(causal)), float(scale), _ptr(dq), _ptr(dk),
                                    _ptr(dv), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("oracle_varlen_attn_bwd failed with code %d" % rc)
    return dq, dk, dv


def run_case_bwd(case, dout, out, lse, nthreads=None, lib=None):
    """Backward of a ``workloads.Case`` for the given dO, O and LSE."""
    return varlen_attn_bwd(dout, case.q, case.k, case.v, out, lse, case.cu_q.numpy(),
                           case.cu_k.numpy(), case.H, case.Hkv, case.D, case.causal, case.scale,
                           case.dtype, nthreads, lib=lib)
