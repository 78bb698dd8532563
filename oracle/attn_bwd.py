"""CPU oracle for the backward pass of the sparse GQA attention.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests,
``__graft_entry__.smoke()`` and the benchmark's CPU legs use it.  Plain numpy
in float64, one query row at a time; it shares nothing with the CUDA path.

Kwai Keye-VL-2.0 technical-report summary, section 1 (two-stage training):
after the dense warm-up of the indexer, the sparse-adaptation stage unfreezes
every parameter and trains the model on the next-token loss with the
attention truly sparse, i.e. each query attends only to the positions its
index row selects.  The loss gradient therefore flows through the sparse
attention below, with the index rows fixed (the selection is not
differentiable).  Forward, for query row t, query head h and its KV group
g = h // (Hq / Hkv), over the valid entries i of idx[t] (0 <= idx[t,i] < n;
an entry that repeats a key counts once per entry, as in the forward the
library computes):

    x[i]     = scale * Q[t,h] . K[s_i, g]
    P[i]     = exp(x[i]) / sum_j exp(x[j])
    O[t,h]   = sum_i P[i] V[s_i, g]

Backward, given dO = dLoss/dO (the chain rule through the softmax written
out; D is the usual softmax-backward row term):

    dP[i]    = dO[t,h] . V[s_i, g]
    D        = sum_i P[i] dP[i]          (= dO[t,h] . O[t,h])
    dS[i]    = P[i] (dP[i] - D)
    dQ[t,h]  = scale * sum_i dS[i] K[s_i, g]
    dK[s,g] += scale * dS[i] Q[t,h]       for every (t, h in g, i) with s_i = s
    dV[s,g] += P[i] dO[t,h]               for every (t, h in g, i) with s_i = s

A row with no valid entry has O = 0 and contributes nothing.
"""
from __future__ import annotations

from typing import Dict

import numpy as np


def decode_bf16(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (a bf16 is the upper half of a binary32)."""
    bits = np.asarray(a, np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def _rows(idx: np.ndarray, t: int, n: int) -> np.ndarray:
    r = np.asarray(idx[t], np.int64)
    return r[(r >= 0) & (r < n)]


def forward(Q, K, V, idx, scale: float) -> np.ndarray:
    """O [L][Hq][d] in float64 from float64 Q [L][Hq][d], K/V [n][Hkv][d]."""
    Q, K, V = (np.asarray(a, np.float64) for a in (Q, K, V))
    L, Hq, d = Q.shape
    n, Hkv, _ = K.shape
    G = Hq // Hkv
    O = np.zeros((L, Hq, d))
    for t in range(L):
        s = _rows(idx, t, n)
        if s.size == 0:
            continue
        for h in range(Hq):
            g = h // G
            x = scale * (K[s, g, :] @ Q[t, h])
            p = np.exp(x - x.max())
            p /= p.sum()
            O[t, h] = p @ V[s, g, :]
    return O


def backward(Q, K, V, idx, dO, scale: float, magnitudes: bool = False) -> Dict[str, np.ndarray]:
    """dQ [L][Hq][d], dK and dV [n][Hkv][d] (float64) of sum(dO * O).

    Rows of one KV group are handled together (they share the selected K and
    V rows); each head's softmax is its own row of the [G][m] arrays.

    With ``magnitudes``, also the sums of the absolute values of the terms
    behind each output element (what a rounding of the operands perturbs):
    mQ = scale * sum |dS| |K| (+ P E |K|), mK = scale * sum |dS| |Q| (+ P E |Q|),
    mV = sum P |dO|, where E = sum_c |dO_c| |O_c| bounds the row term D."""
    Q, K, V, dO = (np.asarray(a, np.float64) for a in (Q, K, V, dO))
    L, Hq, d = Q.shape
    n, Hkv, _ = K.shape
    G = Hq // Hkv
    dQ = np.zeros((L, Hq, d))
    dK = np.zeros((n, Hkv, d))
    dV = np.zeros((n, Hkv, d))
    if magnitudes:
        mQ, mK, mV = np.zeros_like(dQ), np.zeros_like(dK), np.zeros_like(dV)
    for t in range(L):
        s = _rows(idx, t, n)
        if s.size == 0:
            continue
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)          # the query heads of group g
            Ks, Vs = K[s, g, :], V[s, g, :]         # [m][d]
            x = scale * (Q[t, hs] @ Ks.T)           # [G][m]
            p = np.exp(x - x.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            dp = dO[t, hs] @ Vs.T                   # [G][m]
            D = (p * dp).sum(axis=1, keepdims=True)
            ds = p * (dp - D)
            dQ[t, hs] = scale * (ds @ Ks)
            np.add.at(dK[:, g, :], s, scale * (ds.T @ Q[t, hs]))
            np.add.at(dV[:, g, :], s, p.T @ dO[t, hs])
            if magnitudes:
                E = (np.abs(dO[t, hs]) * np.abs(p @ Vs)).sum(axis=1, keepdims=True)
                a = np.abs(ds) + p * E
                mQ[t, hs] = scale * (a @ np.abs(Ks))
                np.add.at(mK[:, g, :], s, scale * (a.T @ np.abs(Q[t, hs])))
                np.add.at(mV[:, g, :], s, p.T @ np.abs(dO[t, hs]))
    out = dict(dQ=dQ, dK=dK, dV=dV)
    if magnitudes:
        out.update(mQ=mQ, mK=mK, mV=mV)
    return out


def lse(Q, K, idx, scale: float) -> np.ndarray:
    """Natural log of each row's softmax normaliser, [L][Hq] (-inf for a row
    with no valid entry): log sum_i exp(scale * Q[t,h] . K[s_i, g])."""
    Q, K = np.asarray(Q, np.float64), np.asarray(K, np.float64)
    L, Hq, d = Q.shape
    n, Hkv, _ = K.shape
    G = Hq // Hkv
    out = np.full((L, Hq), -np.inf)
    for t in range(L):
        s = _rows(idx, t, n)
        if s.size == 0:
            continue
        for h in range(Hq):
            x = scale * (K[s, h // G, :] @ Q[t, h])
            m = x.max()
            out[t, h] = m + np.log(np.exp(x - m).sum())
    return out
