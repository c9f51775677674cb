"""The online-softmax recurrence, evaluated tile by tile in fp64.

Test infrastructure only (see ``oracle/__init__.py``).  This is the recurrence
that the Phase 08 page states in its Lab 01 "Talking Points" and that the
Concepts list calls online softmax and FlashAttention tiling: for each block of
B_c key columns, with t indexing the blocks,

    m_t = max(m_{t-1}, rowmax(S_t))
    l_t = exp(m_{t-1} - m_t) * l_{t-1} + rowsum(exp(S_t - m_t))
    O_t = diag(exp(m_{t-1} - m_t)) O_{t-1} + exp(S_t - m_t) V_t

where S_t holds the scaled scores of the block.  The page leaves two things
implicit, read here in the plainest way: the scores carry the 1/sqrt(d) (here
``scale``) factor, and the final output is O_T / l_T with L = m_T + ln l_T.
The pins in ``tests/test_oracle.py`` check that this equals the two-pass
definition in ``attn_oracle.c`` for tile sizes 1, 7 and N.
"""
from __future__ import annotations

import numpy as np


def online_attention(q, k, v, scale: float, block_cols: int, causal: bool = False):
    """One head: q [Nq,d], k/v [Nk,d] -> (O [Nq,d], L [Nq]) via the recurrence."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, d = q.shape
    nk = k.shape[0]
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    o = np.zeros((nq, d))
    rows = np.arange(nq)[:, None]
    for start in range(0, nk, block_cols):
        stop = min(start + block_cols, nk)
        s = scale * (q @ k[start:stop].T)
        if causal:
            cols = np.arange(start, stop)[None, :]
            s = np.where(cols <= rows, s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        # A row with nothing visible so far keeps m = -inf; guard the 0 * inf.
        alpha = np.where(np.isneginf(m_new), 0.0, np.exp(m - np.where(np.isneginf(m_new), 0.0, m_new)))
        p = np.where(np.isneginf(s), 0.0, np.exp(s - np.where(np.isneginf(m_new), 0.0, m_new)[:, None]))
        l = alpha * l + p.sum(axis=1)
        o = alpha[:, None] * o + p @ v[start:stop]
        m = m_new
    out = o / l[:, None]
    return out, m + np.log(l)
