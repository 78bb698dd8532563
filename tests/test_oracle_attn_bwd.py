"""Pins of the sparse-attention backward oracle (oracle/attn_bwd.py) against
things other than itself: the C oracle's forward, central finite
differences of sum(dO * O), the dense causal attention's gradient from torch
autograd (when every visible key is selected), and closed forms.  Each check
takes the module under test, so that the mutation test runs the same checks
on copies with a planted mistake.

Source of the operation: Kwai Keye-VL-2.0 technical-report summary,
section 1 (sparse adaptation stage: all parameters trained on the
next-token loss through the truly sparse attention)."""
import importlib.util

import numpy as np
import pytest
import torch

import gen
import oracle
import oracle.attn_bwd as AB


def _case(L=7, Hq=4, Hkv=2, d=4, k=3, seed=0, holes=True):
    """Small float64 inputs (bf16-representable) and index rows with a hole
    (-1), an out-of-range entry, a repeated key and an empty row."""
    rng = np.random.default_rng(seed)
    bits = lambda *s: gen.encode_bf16(rng.normal(size=s))  # noqa: E731
    Qb, Kb, Vb, dOb = bits(L, Hq, d), bits(L, Hkv, d), bits(L, Hkv, d), bits(L, Hq, d)
    idx = np.full((L, k), -1, np.int32)
    for t in range(L):
        m = min(k, t + 1)
        idx[t, :m] = rng.choice(t + 1, m, replace=False)
    if holes and L >= 7:
        idx[3, 1] = -1          # a hole
        idx[4, 2] = L + 5       # out of range: skipped
        idx[5, 2] = idx[5, 0]   # a key listed twice counts twice
        idx[6, :] = -1          # an empty row
    return Qb, Kb, Vb, dOb, idx


def check_forward_matches_c_oracle(M):
    Qb, Kb, Vb, dOb, idx = _case(L=9, Hq=8, Hkv=2, d=8, k=4, seed=1)
    ref = oracle.sparse_attn(Qb, Kb, Vb, idx, 0.35)
    got = M.forward(M.decode_bf16(Qb), M.decode_bf16(Kb), M.decode_bf16(Vb), idx, 0.35)
    assert np.abs(got - ref).max() <= 1e-12


def check_finite_differences(M):
    Qb, Kb, Vb, dOb, idx = _case(seed=2)
    Q, K, V, dO = (M.decode_bf16(a) for a in (Qb, Kb, Vb, dOb))
    scale = 0.7
    g = M.backward(Q, K, V, idx, dO, scale)
    f = lambda Q_, K_, V_: float((dO * M.forward(Q_, K_, V_, idx, scale)).sum())  # noqa: E731
    eps = 1e-6
    for name, X, pos in (("dQ", Q, 0), ("dK", K, 1), ("dV", V, 2)):
        num = np.zeros_like(X)
        for i in np.ndindex(X.shape):
            args = [Q.copy(), K.copy(), V.copy()]
            args[pos][i] += eps
            fp = f(*args)
            args[pos][i] -= 2 * eps
            fm = f(*args)
            num[i] = (fp - fm) / (2 * eps)
        assert np.abs(num - g[name]).max() <= 1e-7 * (1 + np.abs(num).max()), name


def check_dense_equals_autograd(M):
    """With every visible key selected, the sparse attention is the dense
    causal attention: its gradient comes from torch autograd."""
    L, Hq, Hkv, d = 12, 6, 3, 5
    Qb, Kb, Vb, dOb, _ = _case(L=L, Hq=Hq, Hkv=Hkv, d=d, k=L, seed=3, holes=False)
    idx = np.full((L, L + 2), -1, np.int32)
    for t in range(L):
        idx[t, :t + 1] = np.arange(t, -1, -1)   # any order
    Q, K, V, dO = (M.decode_bf16(a) for a in (Qb, Kb, Vb, dOb))
    scale = 0.45
    g = M.backward(Q, K, V, idx, dO, scale)
    tQ, tK, tV = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    G = Hq // Hkv
    Ke, Ve = tK.repeat_interleave(G, dim=1), tV.repeat_interleave(G, dim=1)  # [L][Hq][d]
    s = torch.einsum("thc,shc->hts", tQ, Ke) * scale
    mask = torch.ones(L, L, dtype=torch.bool).triu(1)
    p = torch.softmax(s.masked_fill(mask, float("-inf")), dim=-1)
    O = torch.einsum("hts,shc->thc", p, Ve)
    (O * torch.tensor(dO)).sum().backward()
    for name, t in (("dQ", tQ), ("dK", tK), ("dV", tV)):
        assert np.abs(t.grad.numpy() - g[name]).max() <= 1e-12, name


def check_constant_values_give_no_query_key_gradient(M):
    """V constant over keys: O does not depend on Q or K, so dQ = dK = 0 and
    dV[s] = sum of P dO over the (t, h) that select s."""
    Qb, Kb, Vb, dOb, idx = _case(seed=4)
    Q, K, dO = (M.decode_bf16(a) for a in (Qb, Kb, dOb))
    V = np.broadcast_to(np.array([0.5, -1.0, 2.0, 0.25]), (Q.shape[0], 2, 4)).copy()
    g = M.backward(Q, K, V, idx, dO, 0.6)
    assert np.abs(g["dQ"]).max() <= 1e-12 and np.abs(g["dK"]).max() <= 1e-12
    assert np.abs(g["dV"]).max() > 0.1


def check_single_key_rows(M):
    """One key per row: P = 1 and dS = 0, so dQ = dK = 0 and dV[s, g] is the
    sum of dO[t, h] over the heads h of group g of the rows that pick s."""
    L, Hq, Hkv, d = 6, 4, 2, 3
    Qb, Kb, Vb, dOb, _ = _case(L=L, Hq=Hq, Hkv=Hkv, d=d, seed=5, holes=False)
    idx = np.array([[0], [0], [1], [0], [3], [1]], np.int32)
    Q, K, V, dO = (M.decode_bf16(a) for a in (Qb, Kb, Vb, dOb))
    g = M.backward(Q, K, V, idx, dO, 1.1)
    want = np.zeros((L, Hkv, d))
    for t in range(L):
        for h in range(Hq):
            want[idx[t, 0], h // (Hq // Hkv)] += dO[t, h]
    assert np.abs(g["dV"] - want).max() <= 1e-12
    assert np.abs(g["dQ"]).max() <= 1e-12 and np.abs(g["dK"]).max() <= 1e-12


def check_lse_matches_c_oracle_weights(M):
    """exp(scale Q.K - lse) reproduces the C oracle's softmax weights."""
    Qb, Kb, Vb, dOb, idx = _case(L=9, Hq=8, Hkv=2, d=8, k=4, seed=6)
    Q, K = M.decode_bf16(Qb), M.decode_bf16(Kb)
    lse = M.lse(Q, K, idx, 0.35)
    for t, h in ((5, 3), (8, 7), (2, 0)):
        p = oracle.attn_weights(Qb, Kb, idx, 0.35, t, h)
        s = idx[t]
        valid = (s >= 0) & (s < Q.shape[0])
        x = 0.35 * (K[s[valid], h // 4] @ Q[t, h])
        assert np.abs(np.exp(x - lse[t, h]) - p[valid]).max() <= 1e-12
    assert np.all(np.isneginf(lse[6]))


CHECKS = [check_forward_matches_c_oracle, check_finite_differences, check_dense_equals_autograd,
          check_constant_values_give_no_query_key_gradient, check_single_key_rows,
          check_lse_matches_c_oracle_weights]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_attn_bwd_oracle_pin(check):
    check(AB)


def test_magnitudes_bound_the_gradients():
    Qb, Kb, Vb, dOb, idx = _case(L=9, Hq=8, Hkv=2, d=8, k=4, seed=7)
    args = [AB.decode_bf16(a) for a in (Qb, Kb, Vb)]
    g = AB.backward(*args, idx, AB.decode_bf16(dOb), 0.35, magnitudes=True)
    for n, m in (("dQ", "mQ"), ("dK", "mK"), ("dV", "mV")):
        assert np.all(np.abs(g[n]) <= g[m] + 1e-12)


# ------------------------------------------------------------- planted mistakes

MUTATIONS = {
    "row term D dropped": ("ds = p * (dp - D)", "ds = p * dp"),
    "softmax-backward sign": ("ds = p * (dp - D)", "ds = p * (D - dp)"),
    "scale missing in dK": ("np.add.at(dK[:, g, :], s, scale * (ds.T @ Q[t, hs]))",
                            "np.add.at(dK[:, g, :], s, ds.T @ Q[t, hs])"),
    "scale missing in dQ": ("dQ[t, hs] = scale * (ds @ Ks)", "dQ[t, hs] = ds @ Ks"),
    "dV from dS": ("np.add.at(dV[:, g, :], s, p.T @ dO[t, hs])",
                   "np.add.at(dV[:, g, :], s, ds.T @ dO[t, hs])"),
    "gqa heads of the wrong group": ("hs = slice(g * G, (g + 1) * G)",
                                     "hs = slice(g, Hq, Hkv)"),
    "repeated keys counted once": ("np.add.at(dK[:, g, :], s, scale * (ds.T @ Q[t, hs]))",
                                   "dK[s, g, :] += scale * (ds.T @ Q[t, hs])"),
    "out-of-range entries kept": ("return r[(r >= 0) & (r < n)]", "return r[r >= 0] % n"),
    "softmax over heads": ("p /= p.sum(axis=1, keepdims=True)\n            dp",
                           "p /= p.sum(axis=0, keepdims=True)\n            dp"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(AB.__file__).read()
    assert old in src, f"mutation site not found: {name}"
    src = src.replace(old, new)
    spec = importlib.util.spec_from_loader("oracle.attn_bwd_mut", loader=None,
                                           origin=AB.__file__)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    exec(compile(src, AB.__file__, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_an_attn_bwd_pin(name):
    mod = _mutant(name)
    failed = []
    for check in CHECKS:
        try:
            check(mod)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake: {name}"
