"""CPU oracle for the indexer's dense warm-up loss (KL to the full attention).

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests,
``__graft_entry__.smoke()`` and the benchmark's CPU legs use it.  Plain numpy
in float64, one query row at a time, following the definitions below; it
shares nothing with the CUDA path.

Kwai Keye-VL-2.0 technical-report summary, section 1 (two-stage training of
the sparse attention): in the dense warm-up stage the full attention is kept
and only the Lightning Indexer is trained, so that its judgement of which
positions matter approaches the full attention's distribution, the gap being
measured and minimised by a KL divergence.  The pages give no formula; the
reading taken here is the plainest one consistent with the rest of the
section:

* indexer logits, causal (s <= t):
      I[t,s] = sum_j w[t,j] * max(q_I[t,j] . k_I[s], 0)
  (the same scores the indexer ranks for the top-k);
* indexer distribution  P_I[t,:] = softmax_s(scale_I * I[t,s]),  s <= t
  (scale_I is a plain temperature; 1 reproduces the scores as they are);
* target  p[t,s] = (1 / Hq) * sum_h softmax_s(scale * Q[t,h] . K[s, h // (Hq/Hkv)])
  (every query head's full causal attention weights, averaged over heads,
  so that the row sums to one);
* loss per token  kl[t] = sum_s p[t,s] * (log p[t,s] - log P_I[t,s]),
  with 0 * log 0 = 0; the training objective is sum_t kl[t];
* gradients of sum_t kl[t] with respect to the indexer's inputs (the target
  is fixed: the full attention is not trained in this stage):
      G[t,s]    = dL/dI[t,s] = scale_I * (P_I[t,s] - p[t,s])
      dw[t,j]   = sum_s G[t,s] * max(S[t,j,s], 0)
      dq_I[t,j] = w[t,j] * sum_s G[t,s] * [S[t,j,s] > 0] * k_I[s]
      dk_I[s]   = sum_t sum_j G[t,s] * w[t,j] * [S[t,j,s] > 0] * q_I[t,j]
  where S[t,j,s] = q_I[t,j] . k_I[s] and the ReLU's derivative at 0 is 0.
"""
from __future__ import annotations

from typing import Dict

import numpy as np


def _e4m3_table() -> np.ndarray:
    from . import e4m3_value
    return np.array([e4m3_value(b) for b in range(256)], np.float64)


_E4M3 = None


def decode_e4m3(a: np.ndarray) -> np.ndarray:
    global _E4M3
    if _E4M3 is None:
        _E4M3 = _e4m3_table()
    return _E4M3[np.asarray(a, np.uint8)]


def decode_bf16(a: np.ndarray) -> np.ndarray:
    bits = np.asarray(a, np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def _softmax(x: np.ndarray) -> np.ndarray:
    m = x.max()
    e = np.exp(x - m)
    return e / e.sum()


def target_row(Qf: np.ndarray, Kf: np.ndarray, scale: float, t: int) -> np.ndarray:
    """p[t, 0..t]: the mean over query heads of each head's causal softmax."""
    Hq = Qf.shape[1]
    Hkv = Kf.shape[1]
    G = Hq // Hkv
    p = np.zeros(t + 1)
    for h in range(Hq):
        a = scale * (Kf[:t + 1, h // G, :] @ Qf[t, h, :])
        p += _softmax(a)
    return p / Hq


def kl_grads_f64(qf: np.ndarray, kf: np.ndarray, w: np.ndarray, Qf: np.ndarray, Kf: np.ndarray,
                 scale: float, scale_I: float, grads: bool = True) -> Dict[str, np.ndarray]:
    """The loss and its gradients on real-valued inputs.

    qf [L][H_I][d_I], kf [L][d_I], w [L][H_I], Qf [L][Hq][d], Kf [L][Hkv][d]
    (float64).  Returns kl [L], and with grads: G [L][L] (zero above the
    diagonal), dq_I [L][H_I][d_I], dk_I [L][d_I], dw [L][H_I]."""
    L, H, dI = qf.shape
    kl = np.zeros(L)
    out = {"kl": kl}
    if grads:
        Gm = np.zeros((L, L))
        dq = np.zeros_like(qf)
        dk = np.zeros_like(kf)
        dw = np.zeros_like(w, dtype=np.float64)
    for t in range(L):
        S = qf[t] @ kf[:t + 1].T                      # [H][t+1]
        I = w[t].astype(np.float64) @ np.maximum(S, 0.0)  # [t+1]
        z = scale_I * I
        m = z.max()
        lse = m + np.log(np.exp(z - m).sum())
        logq = z - lse
        p = target_row(Qf, Kf, scale, t)
        pos = p > 0
        kl[t] = float((p[pos] * (np.log(p[pos]) - logq[pos])).sum())
        if grads:
            g = scale_I * (np.exp(logq) - p)            # dL/dI[t, 0..t]
            Gm[t, :t + 1] = g
            dw[t] = np.maximum(S, 0.0) @ g
            dS = (S > 0) * g[None, :] * w[t][:, None]   # [H][t+1]
            dq[t] = dS @ kf[:t + 1]
            dk[:t + 1] += dS.T @ qf[t]
    if grads:
        out.update(G=Gm, dq_I=dq, dk_I=dk, dw=dw)
    return out


def indexer_kl(q_I, k_I, w, Q, K, scale: float, scale_I: float = 1.0,
               grads: bool = True) -> Dict[str, np.ndarray]:
    """The same on the encoded inputs of the hot path: q_I uint8 e4m3
    [L][H_I][d_I], k_I uint8 e4m3 [L][d_I], w float32 [L][H_I], Q bf16 bits
    (uint16) [L][Hq][d], K bf16 bits [L][Hkv][d]."""
    return kl_grads_f64(decode_e4m3(q_I), decode_e4m3(k_I), np.asarray(w, np.float64),
                        decode_bf16(Q), decode_bf16(K), scale, scale_I, grads)
