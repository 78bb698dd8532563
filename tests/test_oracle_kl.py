"""Pins of the indexer warm-up KL oracle (oracle/kl.py) against things other
than itself: finite differences of the loss, the C oracle's separately
written indexer scores and attention weights, closed forms for a uniform
target and a uniform indexer, and an exactly matching indexer.

Definition followed: Kwai Keye-VL-2.0 technical-report summary, section 1
(dense warm-up: the indexer is trained towards the full attention's
distribution under a KL divergence); the formula reading is stated in
oracle/kl.py.  Each check takes the module under test, so that the mutation
test below can run the same checks on copies with a planted mistake."""
import importlib.util
import types

import numpy as np
import pytest
from scipy.special import logsumexp

import gen
import oracle
import oracle.kl as KL


def _rand_case(rng, L=7, H=3, dI=5, Hq=4, Hkv=2, d=6):
    return dict(qf=rng.normal(size=(L, H, dI)), kf=rng.normal(size=(L, dI)),
                w=rng.uniform(0.2, 1.5, size=(L, H)), Qf=rng.normal(size=(L, Hq, d)),
                Kf=rng.normal(size=(L, Hkv, d)))


def check_finite_differences(mod):
    """Every coordinate of dq_I, dk_I and dw against a central difference of
    sum_t kl[t] (continuous inputs: no score sits on the ReLU's kink)."""
    rng = np.random.default_rng(3)
    c = _rand_case(rng)
    scale, scale_I = 0.4, 0.7
    base = mod.kl_grads_f64(**c, scale=scale, scale_I=scale_I)

    def loss(**kw):
        a = dict(c)
        a.update(kw)
        return mod.kl_grads_f64(**a, scale=scale, scale_I=scale_I, grads=False)["kl"].sum()

    eps = 1e-6
    for name, gname in (("qf", "dq_I"), ("kf", "dk_I"), ("w", "dw")):
        x = c[name]
        num = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            num[i] = (loss(**{name: xp}) - loss(**{name: xm})) / (2 * eps)
        assert np.allclose(base[gname], num, rtol=1e-5, atol=1e-8), name


def check_uniform_target_closed_form(mod):
    """Q = 0 makes every head's softmax uniform over t + 1 keys, so
    kl[t] = -log(t+1) - mean_s(c*I[t,s]) + logsumexp_s(c*I[t,s]), with I
    from the C oracle's indexer scores."""
    cfg = gen.custom(L=40, H_I=4, d_I=64, k=8, Hq=8, Hkv=2, d=64, seed=31)
    q, kI, w = gen.prefill_qI(cfg), gen.prefill_kI(cfg), gen.prefill_w(cfg)
    Q = np.zeros((cfg.L, cfg.Hq, cfg.d), np.uint16)
    K = gen.prefill_K(cfg)
    c = 1.0 / 256
    got = mod.indexer_kl(q, kI, w, Q, K, cfg.scale, c, grads=False)["kl"]
    I = oracle.index_scores(q, kI, w)
    for t in range(cfg.L):
        z = c * I[t, :t + 1]
        ref = -np.log(t + 1) - z.mean() + logsumexp(z)
        assert abs(got[t] - ref) <= 1e-9 * max(1.0, abs(ref)), t


def check_uniform_indexer_against_c_attention(mod):
    """w = 0 makes the indexer uniform, so kl[t] = log(t+1) + sum_s p log p
    with p the head mean of the C oracle's attention weights over all causal
    keys."""
    cfg = gen.custom(L=24, H_I=4, d_I=64, k=8, Hq=8, Hkv=2, d=64, seed=32)
    inp = gen.prefill_inputs(cfg)
    w0 = np.zeros_like(inp["w"])
    got = mod.indexer_kl(inp["q_I"], inp["k_I"], w0, inp["Q"], inp["K"], cfg.scale, 1.0,
                         grads=False)["kl"]
    ar = np.arange(cfg.L)
    idx = np.where(ar[None, :] <= ar[:, None], ar[None, :], -1).astype(np.int32)  # causal rows
    for t in range(cfg.L):
        p = np.mean([oracle.attn_weights(inp["Q"], inp["K"], idx, cfg.scale, t, h)[:t + 1]
                     for h in range(cfg.Hq)], axis=0)
        ref = np.log(t + 1) + float((p[p > 0] * np.log(p[p > 0])).sum())
        assert abs(got[t] - ref) <= 1e-10 * max(1.0, abs(ref)), t


def check_exact_match_gives_zero(mod):
    """One query head, one indexer head with weight 1 and q_I = scale * Q,
    k_I = K, all entries positive: the indexer logits equal the attention
    logits, so the loss and all its gradients vanish."""
    rng = np.random.default_rng(4)
    L, d, scale = 9, 5, 0.3
    Qf = rng.uniform(0.1, 1.0, size=(L, 1, d))
    Kf = rng.uniform(0.1, 1.0, size=(L, 1, d))
    r = mod.kl_grads_f64(scale * Qf, Kf[:, 0, :], np.ones((L, 1)), Qf, Kf, scale, 1.0)
    assert np.abs(r["kl"]).max() < 1e-12
    for g in ("G", "dq_I", "dk_I", "dw"):
        assert np.abs(r[g]).max() < 1e-12, g


def check_invariants(mod):
    """kl >= 0, kl[0] = 0 (one key), each G row sums to 0 and G is 0 above
    the diagonal."""
    rng = np.random.default_rng(5)
    c = _rand_case(rng, L=12)
    r = mod.kl_grads_f64(**c, scale=0.5, scale_I=1.3)
    assert (r["kl"] >= -1e-15).all() and abs(r["kl"][0]) < 1e-15
    assert np.allclose(r["G"].sum(axis=1), 0.0, atol=1e-14)
    assert np.array_equal(np.triu(r["G"], 1), np.zeros_like(r["G"]))


CHECKS = [check_finite_differences, check_uniform_target_closed_form,
          check_uniform_indexer_against_c_attention, check_exact_match_gives_zero,
          check_invariants]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_kl_oracle_pin(check):
    check(KL)


# ------------------------------------------------------------- planted mistakes

MUTATIONS = {
    "relu dropped in dw": ("dw[t] = np.maximum(S, 0.0) @ g", "dw[t] = S @ g"),
    "gradient sign flipped": ("g = scale_I * (np.exp(logq) - p)", "g = scale_I * (p - np.exp(logq))"),
    "gqa group h % Hkv": ("Kf[:t + 1, h // G, :]", "Kf[:t + 1, h % Hkv, :]"),
    "head mean over Hkv": ("return p / Hq", "return p / Hkv"),
    "dk from the wrong side": ("dk[:t + 1] += dS.T @ qf[t]", "dk[:t + 1] += dS.T @ qf[t] * w[t][:, None]"),
    "query row off by one": ("@ Qf[t, h, :])", "@ Qf[max(t - 1, 0), h, :])"),
    "indexer weights of the wrong row": ("I = w[t].astype(np.float64)", "I = w[max(t - 1, 0)].astype(np.float64)"),
    "temperature dropped in G": ("g = scale_I * (np.exp(logq) - p)", "g = np.exp(logq) - p"),
    "reverse KL": ("(p[pos] * (np.log(p[pos]) - logq[pos]))", "(np.exp(logq) * (logq - np.log(np.maximum(p, 1e-300))))"),
    "mask weight on dq": ("dq[t] = dS @ kf[:t + 1]", "dq[t] = (S > 0) * g[None, :] @ kf[:t + 1]"),
}


def _mutant(name) -> types.ModuleType:
    old, new = MUTATIONS[name]
    src = open(KL.__file__).read()
    assert old in src, f"mutation site not found: {name}"
    spec = importlib.util.spec_from_loader("oracle.kl_mut", loader=None, origin=KL.__file__)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new, 1), KL.__file__, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_kl_pin(name):
    mod = _mutant(name)
    failed = []
    for check in CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, f"no pin caught: {name}"
