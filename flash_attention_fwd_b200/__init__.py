"""B200-native (sm_100a) packed variable-length attention forward.

Python binding of the C ABI declared in ``include/varlen_attn.h``.  This
module only marshals arguments: every step of the attention forward runs in
the CUDA kernels of ``libvarlen_attn.so``.  There is no CPU or PyTorch
fallback; if the library cannot be loaded, calls raise.

The operation is the varlen attention forward of boostr 0.2.0,
src/ops/cpu/attention/varlen_attention.rs (``varlen_attention_fwd``), with
the out-variant calling convention of PyTorch pull request #176015
(``_flash_attention_forward_no_dropout_inplace``: output written into a
caller buffer, log-sum-exp returned).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvarlen_attn.so")

VARLEN_BF16 = 0
VARLEN_FP16 = 1
DTYPE_CODES = {torch.bfloat16: VARLEN_BF16, torch.float16: VARLEN_FP16}

VARLEN_OK = 0
STATUS_NAMES = {
    0: "VARLEN_OK", -1: "VARLEN_ERR_NULL", -2: "VARLEN_ERR_SHAPE", -3: "VARLEN_ERR_DTYPE",
    -4: "VARLEN_ERR_ALIGN", -5: "VARLEN_ERR_LAUNCH", -6: "VARLEN_ERR_DEVICE",
    -7: "VARLEN_ERR_ARCH", -8: "VARLEN_ERR_WORKSPACE",
}

# Every symbol include/varlen_attn.h declares.
EXPORTED_SYMBOLS = (
    "varlen_attn_fwd_v1",
    "varlen_attn_fwd_v2",
    "varlen_attn_fwd_v3",
    "varlen_attn_fwd_v4",
    "varlen_attn_fwd_num_splits",
    "varlen_attn_fwd_workspace_size",
    "varlen_attn_fwd",
    "varlen_attn_strerror",
    "varlen_attn_device_status",
    "varlen_attn_abi_version",
    "varlen_attn_bwd_workspace_size",
    "varlen_attn_bwd_v1",
    "varlen_attn_bwd_noalloc",
    "varlen_attn_plan_shards",
    "varlen_attn_set_wait_limit",
)

_lock = threading.Lock()
_lib = None


class VarlenAttnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("%s (%d): %s" % (STATUS_NAMES.get(code, "?"), code, msg))
        self.code = code


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
    fwd_args = [P, P, P, P, P, i32, i64, i64, i32, i32, i32, i32, i32, i32, f32, i32, P, P, P]
    for name in ("varlen_attn_fwd_v1", "varlen_attn_fwd"):
        fn = getattr(lib, name)
        fn.argtypes = fwd_args
        fn.restype = i32
    # v2: v1's arguments with window_left, window_right, seqused_k after scale
    lib.varlen_attn_fwd_v2.argtypes = fwd_args[:15] + [i32, i32, P] + fwd_args[15:]
    lib.varlen_attn_fwd_v2.restype = i32
    # v3: v2's arguments with page_table, page_table_stride, page_size, sinks after seqused_k
    lib.varlen_attn_fwd_v3.argtypes = (fwd_args[:15] + [i32, i32, P, P, i32, i32, P]
                                       + fwd_args[15:])
    lib.varlen_attn_fwd_v3.restype = i32
    # v4: v3's arguments with num_splits, workspace, workspace_bytes after sinks
    lib.varlen_attn_fwd_v4.argtypes = (fwd_args[:15] + [i32, i32, P, P, i32, i32, P, i32, P,
                                                        ctypes.c_size_t] + fwd_args[15:])
    lib.varlen_attn_fwd_v4.restype = i32
    lib.varlen_attn_fwd_num_splits.argtypes = [i32, i64, i64, i32, i32, i32, i32, i32, i32, i32,
                                               i32, i32, i32]
    lib.varlen_attn_fwd_num_splits.restype = i32
    lib.varlen_attn_fwd_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32, i32]
    lib.varlen_attn_fwd_workspace_size.restype = ctypes.c_size_t
    lib.varlen_attn_strerror.argtypes = [i32]
    lib.varlen_attn_strerror.restype = ctypes.c_char_p
    lib.varlen_attn_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), i32]
    lib.varlen_attn_device_status.restype = i32
    lib.varlen_attn_abi_version.argtypes = []
    lib.varlen_attn_abi_version.restype = i32
    lib.varlen_attn_bwd_workspace_size.argtypes = [i64, i32]
    lib.varlen_attn_bwd_workspace_size.restype = ctypes.c_size_t
    lib.varlen_attn_bwd_v1.argtypes = ([P] * 8 + [i32, i64, i64, i32, i32, i32, i32, i32, i32, f32,
                                                  i32, P, P, P, P, ctypes.c_size_t, P])
    lib.varlen_attn_bwd_v1.restype = i32
    lib.varlen_attn_bwd_noalloc.argtypes = lib.varlen_attn_bwd_v1.argtypes[:22] + [P]
    lib.varlen_attn_bwd_noalloc.restype = i32
    lib.varlen_attn_plan_shards.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, i32, P,
                                            P, P, P]
    lib.varlen_attn_plan_shards.restype = i32
    lib.varlen_attn_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    lib.varlen_attn_set_wait_limit.restype = i32
    return lib


def load_library(build_if_missing: bool = True):
    """Load (building first if it is missing or stale) the CUDA library.

    The environment variable VARLEN_ATTN_LIB may name another build of the
    same library (same ABI) to load instead."""
    global _lib
    with _lock:
        if _lib is None:
            path = os.environ.get("VARLEN_ATTN_LIB") or LIB_PATH
            if path == LIB_PATH and build_if_missing:
                from . import build as _build
                _build.build()
            if not os.path.exists(path):
                raise RuntimeError("CUDA extension %s is missing; run "
                                   "`python -m flash_attention_fwd_b200.build`" % path)
            _lib = _bind(ctypes.CDLL(path))
    return _lib


def strerror(code: int) -> str:
    return load_library().varlen_attn_strerror(int(code)).decode()


def device_status(clear: bool = True) -> int:
    """Device-side status word (bit 1 = a bounded pipeline wait timed out)."""
    val = ctypes.c_uint(0)
    rc = load_library().varlen_attn_device_status(ctypes.byref(val), int(clear))
    if rc != VARLEN_OK:
        raise VarlenAttnError(rc, strerror(rc))
    return int(val.value)


# Opt-in check after every varlen_attn_fwd / varlen_attn_bwd call: when this
# environment variable is set to anything but "" or "0", the call waits for
# its stream and raises VarlenAttnError(VARLEN_ERR_DEVICE) if the device
# status word is set (a bounded wait inside a kernel ran out, so that call's
# results may be incomplete).  Off by default: the check synchronises.
STATUS_CHECK_ENV = "VARLEN_ATTN_CHECK_STATUS"
VARLEN_ERR_DEVICE = -6


def status_check_enabled() -> bool:
    return os.environ.get(STATUS_CHECK_ENV, "") not in ("", "0")


def raise_on_status(word: int) -> None:
    """Raises VarlenAttnError(VARLEN_ERR_DEVICE) when `word` (a device status
    word) is non-zero."""
    if word:
        raise VarlenAttnError(VARLEN_ERR_DEVICE,
                              "device status word 0x%x: a bounded wait inside a kernel ran out; "
                              "the results of the calls since the last check may be incomplete"
                              % word)


def check_device_status(stream: Optional[torch.cuda.Stream] = None) -> None:
    """Waits for `stream` (default: the current stream), then reads and clears
    the device status word of the current device and raises
    VarlenAttnError(VARLEN_ERR_DEVICE) when it was set."""
    (stream or torch.cuda.current_stream()).synchronize()
    raise_on_status(device_status(clear=True))


def set_wait_limit(ns: int = 0) -> None:
    """Testing hook (varlen_attn_set_wait_limit): the kernels' pipeline-wait
    limit on the current device in ns; 0 restores the default (2 s)."""
    rc = load_library().varlen_attn_set_wait_limit(int(ns))
    if rc != VARLEN_OK:
        raise VarlenAttnError(rc, strerror(rc))


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr() if t is not None and t.numel() > 0 else 0)


def varlen_attn_fwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, cu_q_ptr: int, cu_k_ptr: int,
                        batch: int, total_q: int, total_k: int, max_seqlen_q: int,
                        max_seqlen_k: int, num_heads: int, num_kv_heads: int, head_dim: int,
                        causal: bool, scale: float, dtype_code: int, out_ptr: int,
                        lse_ptr: int, stream: int, window_left: int = -1,
                        window_right: int = -1, seqused_k_ptr: int = 0,
                        page_table_ptr: int = 0, page_table_stride: int = 0,
                        page_size: int = 0, sinks_ptr: int = 0, num_splits: int = 1,
                        workspace_ptr: int = 0, workspace_bytes: int = 0) -> int:
    """Direct call of the C entry point with integer addresses; returns the
    status code unchanged.  Calls varlen_attn_fwd (v1) unless a window bound,
    a seqused_k array, a page table, sinks, num_splits != 1 or a workspace are
    given; varlen_attn_fwd_v2 for a window / seqused_k, varlen_attn_fwd_v3 for
    a page table or sinks, varlen_attn_fwd_v4 for a key-range split or a
    workspace."""
    lib = load_library()
    V = ctypes.c_void_p
    head = (V(q_ptr), V(k_ptr), V(v_ptr), V(cu_q_ptr), V(cu_k_ptr), int(batch), int(total_q),
            int(total_k), int(max_seqlen_q), int(max_seqlen_k), int(num_heads),
            int(num_kv_heads), int(head_dim), int(bool(causal)), float(scale))
    tail = (int(dtype_code), V(out_ptr), V(lse_ptr), V(stream))
    if num_splits != 1 or workspace_ptr:
        return lib.varlen_attn_fwd_v4(*head, int(window_left), int(window_right),
                                      V(seqused_k_ptr), V(page_table_ptr),
                                      int(page_table_stride), int(page_size), V(sinks_ptr),
                                      int(num_splits), V(workspace_ptr), int(workspace_bytes),
                                      *tail)
    if page_table_ptr or sinks_ptr:
        return lib.varlen_attn_fwd_v3(*head, int(window_left), int(window_right),
                                      V(seqused_k_ptr), V(page_table_ptr),
                                      int(page_table_stride), int(page_size), V(sinks_ptr),
                                      *tail)
    if window_left < 0 and window_right < 0 and not seqused_k_ptr:
        return lib.varlen_attn_fwd(*head, *tail)
    return lib.varlen_attn_fwd_v2(*head, int(window_left), int(window_right),
                                  V(seqused_k_ptr), *tail)


def varlen_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    cu_seqlens_q: torch.Tensor, cu_seqlens_k: Optional[torch.Tensor],
                    max_seqlen_q: int, max_seqlen_k: int, causal: bool = False,
                    scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None,
                    window_size_left: int = -1, window_size_right: int = -1,
                    seqused_k: Optional[torch.Tensor] = None,
                    page_table: Optional[torch.Tensor] = None,
                    sinks: Optional[torch.Tensor] = None,
                    num_splits: Optional[int] = None,
                    workspace: Optional[torch.Tensor] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Packed attention forward on the GPU.

    q [Tq, H, D], k/v [Tk, Hkv, D] (bf16 or fp16, contiguous, on one CUDA
    device); cu_seqlens_q/k int32 [B+1] on the same device.  Writes ``out``
    ([Tq, H, D], q's dtype) and ``lse`` ([Tq, H], float32) — allocated here
    when not given — and returns them.  ``scale=None`` selects 1/sqrt(D).
    ``window_size_left/right`` (negative = unbounded) and ``seqused_k`` (int32
    [B] on the device, or None) restrict the visible keys as in the varlen
    forward schema of PyTorch pull request #176015: key ki is visible to query
    qi iff ki < min(Lk, seqused_k[b]), qi - left <= ki <= qi + right, and
    not (causal and qi < ki).

    With ``page_table`` (int32 [B, pages_per_seq] on the device) k and v are
    paged caches [num_pages, page_size, Hkv, D], key ki of sequence b is
    ``k[page_table[b, ki // page_size], ki % page_size]``, ``seqused_k`` is
    required and gives the key counts, and ``cu_seqlens_k`` is not used (it
    may be None).

    ``sinks`` (float32 [H] on the device) adds one logit per query head to
    the softmax normalisation (attention sinks): the row's weights become
    exp(s - m) / (sum exp(s - m) + exp(sinks[h] - m)).

    ``num_splits`` (non-causal calls without a window only): the key range of
    a row may be computed in up to that many pieces merged by their LSE
    (varlen_attn_fwd_v4), and decode-like calls (at most 32 query rows per
    KV head) in replicated rows, four copies over interleaved key subsets
    merged the same way; None lets the library choose, 1 turns both off.
    The pieces need a device workspace, allocated here unless ``workspace``
    (a uint8 CUDA tensor of at least ``fwd_workspace_size(...)`` bytes) is
    given.
    """
    if q.dtype not in DTYPE_CODES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share dtype bfloat16 or float16")
    paged = page_table is not None
    if q.dim() != 3 or k.dim() != (4 if paged else 3) or v.shape != k.shape:
        raise ValueError("expected q [Tq,H,D] and k, v [Tk,Hkv,D] "
                         "(paged: [num_pages,page_size,Hkv,D])")
    tensors = [("q", q), ("k", k), ("v", v), ("cu_seqlens_q", cu_seqlens_q)]
    if not paged or cu_seqlens_k is not None:
        tensors.append(("cu_seqlens_k", cu_seqlens_k))
    for name, t in tensors:
        if t is None or not t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    B = cu_seqlens_q.numel() - 1
    if cu_seqlens_q.dtype != torch.int32 or (cu_seqlens_k is not None
                                             and cu_seqlens_k.dtype != torch.int32):
        raise TypeError("cu_seqlens must be int32")
    if B < 0 or (cu_seqlens_k is not None and cu_seqlens_k.numel() != B + 1):
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B+1 >= 1 entries")
    total_q, H, D = q.shape
    page_size = stride = 0
    if paged:
        num_pages, page_size, Hkv, Dk = k.shape
        total_k = num_pages * page_size
        if (not page_table.is_cuda or not page_table.is_contiguous()
                or page_table.dtype != torch.int32 or page_table.dim() != 2
                or page_table.shape[0] != B):
            raise ValueError("page_table must be a contiguous int32 CUDA tensor [B, pages]")
        if seqused_k is None:
            raise ValueError("a page table needs seqused_k (the key count of each sequence)")
        stride = page_table.shape[1]
    else:
        total_k, Hkv, Dk = k.shape
    if Dk != D:
        raise ValueError("head dims of q and k differ")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((total_q, H), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor shaped and typed like q")
    if lse.shape != (total_q, H) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [Tq, H]")
    if seqused_k is not None:
        if (not seqused_k.is_cuda or not seqused_k.is_contiguous()
                or seqused_k.dtype != torch.int32 or seqused_k.numel() != B):
            raise ValueError("seqused_k must be a contiguous int32 CUDA tensor [B]")
    if sinks is not None:
        if (not sinks.is_cuda or not sinks.is_contiguous() or sinks.dtype != torch.float32
                or sinks.numel() != H):
            raise ValueError("sinks must be a contiguous float32 CUDA tensor [H]")
    if stream is None:
        stream = torch.cuda.current_stream(q.device)

    def addr(t):
        return t.data_ptr() if t is not None and t.numel() else 0

    splits, ws_bytes = 1, 0
    if not causal and window_size_left < 0 and window_size_right < 0 and num_splits != 1:
        splits = (fwd_num_splits(B, total_q, total_k, max_seqlen_q, max_seqlen_k, H, Hkv, D,
                                 paged=paged, device=q.device)
                  if num_splits is None else int(num_splits))
        ws_bytes = fwd_workspace_size(total_q, H, Hkv, D, max_seqlen_q, max_seqlen_k, splits)
        if ws_bytes == 0:
            splits = 1
        elif workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
        elif (not workspace.is_cuda or workspace.dtype != torch.uint8
              or not workspace.is_contiguous() or workspace.numel() < ws_bytes):
            raise ValueError("workspace must be a contiguous uint8 CUDA tensor of at least "
                             "%d bytes" % ws_bytes)
    with torch.cuda.device(q.device):
        rc = varlen_attn_fwd_raw(
            addr(q), addr(k), addr(v), addr(cu_seqlens_q), addr(cu_seqlens_k), B,
            total_q, total_k, int(max_seqlen_q), int(max_seqlen_k), H, Hkv, D, causal,
            0.0 if scale is None else float(scale), DTYPE_CODES[q.dtype], addr(out), addr(lse),
            stream.cuda_stream, int(window_size_left), int(window_size_right), addr(seqused_k),
            addr(page_table), stride, page_size, addr(sinks), splits,
            addr(workspace) if ws_bytes else 0, ws_bytes)
        if rc == VARLEN_OK and status_check_enabled():
            check_device_status(stream)
    if rc != VARLEN_OK:
        raise VarlenAttnError(rc, strerror(rc))
    return out, lse


_sms = {}


def fwd_num_splits(batch: int, total_q: int, total_k: int, max_seqlen_q: int, max_seqlen_k: int,
                   num_heads: int, num_kv_heads: int, head_dim: int, causal: bool = False,
                   window_size_left: int = -1, window_size_right: int = -1, paged: bool = False,
                   device=None, num_sms: Optional[int] = None) -> int:
    """Key-range piece count the library picks for these sizes
    (varlen_attn_fwd_num_splits); ``num_sms`` defaults to the device's."""
    if num_sms is None:
        dev = torch.device(device if device is not None else "cuda")
        idx = dev.index if dev.index is not None else torch.cuda.current_device()
        if idx not in _sms:
            _sms[idx] = torch.cuda.get_device_properties(idx).multi_processor_count
        num_sms = _sms[idx]
    rc = load_library().varlen_attn_fwd_num_splits(
        int(batch), int(total_q), int(total_k), int(max_seqlen_q), int(max_seqlen_k),
        int(num_heads), int(num_kv_heads), int(head_dim), int(bool(causal)),
        int(window_size_left), int(window_size_right), int(bool(paged)), int(num_sms))
    if rc < 0:
        raise VarlenAttnError(rc, strerror(rc))
    return int(rc)


def fwd_workspace_size(total_q: int, num_heads: int, num_kv_heads: int, head_dim: int,
                       max_seqlen_q: int, max_seqlen_k: int, num_splits: int) -> int:
    """Bytes of device workspace a non-causal, windowless forward with at most
    ``num_splits`` key-range pieces needs (0: none; see
    varlen_attn_fwd_workspace_size)."""
    return int(load_library().varlen_attn_fwd_workspace_size(
        int(total_q), int(num_heads), int(num_kv_heads), int(head_dim), int(max_seqlen_q),
        int(max_seqlen_k), int(num_splits)))


def bwd_workspace_size(total_q: int, num_heads: int) -> int:
    """Bytes of device workspace ``varlen_attn_bwd`` needs."""
    return int(load_library().varlen_attn_bwd_workspace_size(int(total_q), int(num_heads)))


def varlen_attn_bwd_raw(dout_ptr: int, q_ptr: int, k_ptr: int, v_ptr: int, out_ptr: int,
                        lse_ptr: int, cu_q_ptr: int, cu_k_ptr: int, batch: int, total_q: int,
                        total_k: int, max_seqlen_q: int, max_seqlen_k: int, num_heads: int,
                        num_kv_heads: int, head_dim: int, causal: bool, scale: float,
                        dtype_code: int, dq_ptr: int, dk_ptr: int, dv_ptr: int,
                        workspace_ptr: int, workspace_bytes: int, stream: int) -> int:
    """Direct call of varlen_attn_bwd_v1 with integer addresses; returns the
    status code unchanged."""
    lib = load_library()
    V = ctypes.c_void_p
    return lib.varlen_attn_bwd_v1(V(dout_ptr), V(q_ptr), V(k_ptr), V(v_ptr), V(out_ptr),
                                  V(lse_ptr), V(cu_q_ptr), V(cu_k_ptr), int(batch), int(total_q),
                                  int(total_k), int(max_seqlen_q), int(max_seqlen_k),
                                  int(num_heads), int(num_kv_heads), int(head_dim),
                                  int(bool(causal)), float(scale), int(dtype_code), V(dq_ptr),
                                  V(dk_ptr), V(dv_ptr), V(workspace_ptr), int(workspace_bytes),
                                  V(stream))


def varlen_attn_bwd(dout: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    out: torch.Tensor, lse: torch.Tensor, cu_seqlens_q: torch.Tensor,
                    cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int,
                    causal: bool = False, scale: Optional[float] = None,
                    dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                    dv: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients (dq, dk, dv) of the packed attention forward, given dO and
    the forward's out and lse.  Shapes and dtypes as in ``varlen_attn_fwd``
    (head dim 64, 128 or 256); outputs and the workspace (``bwd_workspace_size``
    bytes, uint8 on the device) are allocated here when not given."""
    if q.dtype not in DTYPE_CODES or any(t.dtype != q.dtype for t in (k, v, dout, out)):
        raise TypeError("dout, q, k, v, out must share dtype bfloat16 or float16")
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or dout.shape != q.shape \
            or out.shape != q.shape:
        raise ValueError("expected dout/q/out [Tq,H,D] and k, v [Tk,Hkv,D]")
    for name, t in (("dout", dout), ("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse),
                    ("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous CUDA tensor" % name)
    total_q, H, D = q.shape
    total_k, Hkv, _ = k.shape
    if lse.dtype != torch.float32 or lse.shape != (total_q, H):
        raise ValueError("lse must be float32 [Tq, H]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t.shape != ref.shape or t.dtype != ref.dtype or not t.is_contiguous():
            raise ValueError("%s must be contiguous and shaped / typed like its input" % name)
    need = bwd_workspace_size(total_q, H)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)

    def addr(t):
        return t.data_ptr() if t is not None and t.numel() else 0

    with torch.cuda.device(q.device):
        rc = varlen_attn_bwd_raw(
            addr(dout), addr(q), addr(k), addr(v), addr(out), addr(lse), addr(cu_seqlens_q),
            addr(cu_seqlens_k), cu_seqlens_q.numel() - 1, total_q, total_k, int(max_seqlen_q),
            int(max_seqlen_k), H, Hkv, D, causal, 0.0 if scale is None else float(scale),
            DTYPE_CODES[q.dtype], addr(dq), addr(dk), addr(dv), addr(workspace),
            workspace.numel() * workspace.element_size(), stream.cuda_stream)
        if rc == VARLEN_OK and status_check_enabled():
            check_device_status(stream)
    if rc != VARLEN_OK:
        raise VarlenAttnError(rc, strerror(rc))
    return dq, dk, dv


def varlen_attn_bwd_noalloc(dout: torch.Tensor, q: torch.Tensor, k: torch.Tensor,
                            v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
                            cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                            max_seqlen_q: int, max_seqlen_k: int, dq: torch.Tensor,
                            dk: torch.Tensor, dv: torch.Tensor, causal: bool = False,
                            scale: Optional[float] = None,
                            stream: Optional[torch.cuda.Stream] = None) -> int:
    """varlen_attn_bwd_noalloc: the backward into the given dq/dk/dv with the
    library's own fixed scratch (no workspace, nothing allocated).  Returns
    the status code (raises nothing); see the header for its limits."""
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    total_q, H, D = q.shape
    total_k, Hkv, _ = k.shape

    def addr(t):
        return t.data_ptr() if t is not None and t.numel() else 0

    V = ctypes.c_void_p
    with torch.cuda.device(q.device):
        return load_library().varlen_attn_bwd_noalloc(
            V(addr(dout)), V(addr(q)), V(addr(k)), V(addr(v)), V(addr(out)), V(addr(lse)),
            V(addr(cu_seqlens_q)), V(addr(cu_seqlens_k)), cu_seqlens_q.numel() - 1, total_q,
            total_k, int(max_seqlen_q), int(max_seqlen_k), H, Hkv, D, int(bool(causal)),
            0.0 if scale is None else float(scale), DTYPE_CODES[q.dtype], V(addr(dq)),
            V(addr(dk)), V(addr(dv)), V(stream.cuda_stream))


SHARD_AUTO, SHARD_KV_HEADS, SHARD_SEQUENCES = 0, 1, 2
SHARD_MODES = {"auto": SHARD_AUTO, "kv_heads": SHARD_KV_HEADS, "sequences": SHARD_SEQUENCES}


def plan_shards(cu_seqlens_q, cu_seqlens_k, num_heads: int, num_kv_heads: int, world: int,
                mode: str = "auto", causal: bool = False, window_size_left: int = -1,
                window_size_right: int = -1, seqused_k=None) -> dict:
    """Split of one packed batch over ``world`` GPUs with no exchange
    (varlen_attn_plan_shards, a host-only call).  cu_seqlens_q/k: host
    sequences of B+1 ints; ``mode`` "auto", "kv_heads" or "sequences".
    Returns {"mode", "seq_rank" (B ints, -1 = every rank), "kv_heads"
    (per rank (lo, hi)), "pairs" (per rank)}."""
    import numpy as np
    cq = np.ascontiguousarray(np.asarray(cu_seqlens_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_seqlens_k, dtype=np.int32))
    B = cq.shape[0] - 1
    if ck.shape[0] != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B+1 entries")
    used = None if seqused_k is None else np.ascontiguousarray(np.asarray(seqused_k,
                                                                          dtype=np.int32))
    seq_rank = np.zeros(max(B, 1), dtype=np.int32)
    lo = np.zeros(world, dtype=np.int32)
    hi = np.zeros(world, dtype=np.int32)
    pairs = np.zeros(world, dtype=np.int64)
    P = ctypes.c_void_p
    rc = load_library(build_if_missing=False).varlen_attn_plan_shards(
        P(cq.ctypes.data), P(ck.ctypes.data), P(used.ctypes.data if used is not None else 0),
        int(B), int(num_heads), int(num_kv_heads), int(bool(causal)), int(window_size_left),
        int(window_size_right), int(world), int(SHARD_MODES[mode]), P(seq_rank.ctypes.data),
        P(lo.ctypes.data), P(hi.ctypes.data), P(pairs.ctypes.data))
    if rc < 0:
        raise VarlenAttnError(rc, strerror(rc))
    return {"mode": {SHARD_KV_HEADS: "kv_heads", SHARD_SEQUENCES: "sequences"}[rc],
            "seq_rank": [int(x) for x in seq_rank[:B]],
            "kv_heads": [(int(a), int(b)) for a, b in zip(lo, hi)],
            "pairs": [int(x) for x in pairs]}
