"""Dense brute-force checker — TEST INFRASTRUCTURE ONLY, tiny inputs only.

An independent NumPy fp64 restatement of the varlen attention forward
definition (boostr 0.2.0, src/ops/cpu/attention/varlen_attention.rs,
``varlen_attention_fwd``): instead of looping per sequence it materialises,
per query head, the full [Tq, Tk] score matrix of the packed batch and masks
every pair that is not in the same sequence (block-diagonal) or that the
causal rule hides (sequence-local qi < ki).  Softmax is then an ordinary
dense row softmax.  It shares no code with the C oracle.
"""
from __future__ import annotations

import numpy as np


def segment_ids(cu: np.ndarray) -> np.ndarray:
    """Sequence id of every packed token and its index inside the sequence."""
    cu = np.asarray(cu, dtype=np.int64)
    T = int(cu[-1])
    seg = np.empty(T, dtype=np.int64)
    pos = np.empty(T, dtype=np.int64)
    for b in range(len(cu) - 1):
        seg[cu[b]:cu[b + 1]] = b
        pos[cu[b]:cu[b + 1]] = np.arange(cu[b + 1] - cu[b])
    return seg, pos


def dense_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_q, cu_k, causal: bool,
                  scale: float, window_left: int = -1, window_right: int = -1,
                  seqused_k=None, sinks=None):
    """q [Tq,H,D], k/v [Tk,Hkv,D] float64.  Returns (out [Tq,H,D], lse [Tq,H]).
    Optional sliding window (sequence-local: key ki visible to query qi only
    if qi - left <= ki <= qi + right, negative = unbounded) and per-sequence
    used-key counts; rows without a visible key give O = 0, LSE = -inf.
    With ``sinks`` (one logit per query head) the score matrix gets one more
    column holding sinks[h] for every row, and the value matrix a zero row:
    the dense softmax over [S | sink] then weights V."""
    Tq, H, D = q.shape
    Tk, Hkv, _ = k.shape
    G = H // Hkv
    sq, pq = segment_ids(cu_q)
    sk, pk = segment_ids(cu_k)
    visible = sq[:, None] == sk[None, :]
    if causal:
        visible &= ~(pq[:, None] < pk[None, :])
    if window_left >= 0:
        visible &= pk[None, :] >= pq[:, None] - window_left
    if window_right >= 0:
        visible &= pk[None, :] <= pq[:, None] + window_right
    if seqused_k is not None:
        used = np.asarray(seqused_k, dtype=np.int64)[sk]
        visible &= (pk < used)[None, :]
    out = np.zeros((Tq, H, D))
    lse = np.full((Tq, H), -np.inf)
    for h in range(H):
        kh = k[:, h // G, :]
        vh = v[:, h // G, :]
        s = (q[:, h, :] @ kh.T) * scale
        s = np.where(visible, s, -np.inf)
        if sinks is not None:
            s = np.concatenate([s, np.full((Tq, 1), float(sinks[h]))], axis=1)
            vh = np.concatenate([vh, np.zeros((1, D))], axis=0)
        m = s.max(axis=1, initial=-np.inf)
        has = np.isfinite(m)
        e = np.zeros_like(s)
        e[has] = np.exp(s[has] - m[has, None])
        denom = e.sum(axis=1)
        w = np.zeros_like(e)
        w[has] = e[has] / denom[has, None]
        out[:, h, :] = w @ vh
        lse[has, h] = m[has] + np.log(denom[has])
    return out, lse
