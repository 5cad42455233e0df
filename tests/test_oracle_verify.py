"""Pins of the oracle's speculative verification (CPU only).

What fixes the expected values, none of it the oracle itself:
  * hand-worked cases (tests/golden/verify_hand.json);
  * losslessness: exact enumeration over every drafted block at V=4, L=2,
    for the independent proposal and a K=2 latent mixture, must give an
    emitted sequence distributed as the target rows (to 1e-12);
  * the closed form E[accepted] = sum_i prod_{k<i} sum_v min(p_k, q_k);
  * Monte Carlo of the deterministic path (u and g supplied) with a chi^2
    test against the target rows;
  * identities: q == p accepts everything; a K=1 mixture with w = [1] is the
    independent verifier; a one-hot target is always emitted; the noise row
    used is the terminal position's.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax
from scipy.stats import chisquare

import oracle
from speculative_decoding_block_spec_b200 import synth

LN9 = float(np.float32(math.log(9.0)))


def _num(v):
    if isinstance(v, list):
        return [_num(t) for t in v]
    return LN9 if v == "ln9" else float(v)


def test_golden_hand_cases(golden_dir):
    with open(os.path.join(golden_dir, "verify_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        L, V, K = c["L"], c["V"], c["K"]
        target = np.array([_num(c["target"])], np.float32)
        draft = np.array([_num(c["draft"])], np.float32)
        if K == 1:
            draft = draft.reshape(1, L, V)
        w = None if K == 1 else np.array([c["mix_w"]], np.float32)
        r = oracle.verify(target, draft, np.array([c["tokens"]]), np.array([c["u"]], np.float32),
                          np.array([c["g"]], np.float32), c["T"], mix_w=w)
        assert r["flags"] == 0, c["name"]
        assert r["accept_len"][0] == c["accept_len"], c["name"]
        assert list(r["out_tokens"][0]) == c["out_tokens"], c["name"]


def _enumerate(target, draft, w, T):
    """Distribution of the emitted sequence, built from the oracle's accept
    ratios and terminal distributions for every drafted block and every
    rejection point. target [L+1, V], draft [K, L, V], w [K]."""
    K, L, V = draft.shape
    seqs = list(itertools.product(range(V), repeat=L))
    reqs = [(x, j) for x in seqs for j in range(L + 1)]
    B = len(reqs)
    ONE_MINUS = np.float32(1.0 - 2.0 ** -24)
    tokens = np.array([x for x, _ in reqs], np.int32)
    u = np.zeros((B, L), np.float32)
    for n, (_, j) in enumerate(reqs):
        if j < L:
            u[n, j] = ONE_MINUS
    r = oracle.verify(target, np.broadcast_to(draft, (B, K, L, V)).copy(), tokens, u,
                      np.zeros((B, L + 1, V), np.float32), T,
                      mix_w=np.broadcast_to(w, (B, K)).copy(), target_row_off=np.zeros(B, np.int32),
                      diag=True)
    assert r["flags"] == 0
    qz = softmax(draft.astype(np.float64) / T, axis=-1)          # [K, L, V]
    out = {}
    exp_len = 0.0
    for n, (x, j) in enumerate(reqs):
        q_x = sum(w[z] * np.prod([qz[z, i, x[i]] for i in range(L)]) for z in range(K))
        nall = reqs.index((x, L))
        a = np.minimum(1.0, r["rho"][nall])
        pj = np.prod(a[:j]) * ((1.0 - a[j]) if j < L else 1.0)
        if pj == 0.0:
            continue
        if j < L:
            assert a[j] < ONE_MINUS, "rejection at j cannot be forced with u < 1"
        assert r["terminal_row"][n] == j and r["accept_len"][n] == j
        dist = r["terminal_dist"][n]
        assert abs(dist.sum() - 1.0) < 1e-12
        exp_len += q_x * pj * j
        for t in range(V):
            s = tuple(x[:j]) + (t,)
            out[s] = out.get(s, 0.0) + q_x * pj * dist[t]
    return out, exp_len


def _check_lossless(out, target, T):
    p = softmax(target.astype(np.float64) / T, axis=-1)
    L1, V = p.shape
    assert abs(sum(out.values()) - 1.0) < 1e-12
    for k in range(L1):
        prefixes = {s[:k] for s in out if len(s) > k}
        for pre in prefixes:
            mass = np.zeros(V)
            for s, pr in out.items():
                if len(s) > k and s[:k] == pre:
                    mass[s[k]] += pr
            np.testing.assert_allclose(mass, p[k] * mass.sum(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("K", [1, 2])
@pytest.mark.parametrize("T", [1.0, 1.5])
def test_exact_enumeration_is_lossless(K, T):
    rng = np.random.default_rng(10 + K)
    L, V = 2, 4
    target = (rng.standard_normal((L + 1, V)) * 1.5).astype(np.float32)
    draft = (target[None, :L] + rng.standard_normal((K, L, V)) * 1.2).astype(np.float32)
    w = np.array([1.0] if K == 1 else [0.3, 0.7], np.float32)
    out, _ = _enumerate(target, draft, w, T)
    _check_lossless(out, target, T)


def test_enumeration_expected_length_closed_form():
    rng = np.random.default_rng(21)
    L, V, T = 3, 4, 1.0
    target = (rng.standard_normal((L + 1, V)) * 1.5).astype(np.float32)
    draft = (target[None, :L] + rng.standard_normal((1, L, V))).astype(np.float32)
    _, exp_len = _enumerate(target, draft, np.array([1.0], np.float32), T)
    p = softmax(target.astype(np.float64) / T, axis=-1)
    q = softmax(draft[0].astype(np.float64) / T, axis=-1)
    alpha = np.minimum(p[:L], q).sum(axis=1)
    closed = sum(np.prod(alpha[:i]) for i in range(1, L + 1))
    assert abs(exp_len - closed) < 1e-12


def _sample_categorical(rng, probs, n):
    c = np.cumsum(probs)
    return np.minimum(np.searchsorted(c, rng.random(n), side="right"), len(probs) - 1)


def test_monte_carlo_deterministic_path_chi2():
    """10^6 verify calls with drafted blocks from q_dep, u ~ U[0,1), g ~ Gumbel:
    the emitted tokens at every position follow the target rows."""
    rng = np.random.default_rng(31)
    N, L, V, K, T = 1_000_000, 2, 4, 2, 1.0
    target = (rng.standard_normal((L + 1, V)) * 1.5).astype(np.float32)
    branches = (target[None, :L] + rng.standard_normal((K, L, V)) * 1.5).astype(np.float32)
    w = np.array([0.35, 0.65], np.float32)
    qz = softmax(branches.astype(np.float64) / T, axis=-1)
    z = _sample_categorical(rng, w.astype(np.float64), N)
    tokens = np.empty((N, L), np.int32)
    for zz in range(K):
        idx = np.nonzero(z == zz)[0]
        for i in range(L):
            tokens[idx, i] = _sample_categorical(rng, qz[zz, i], len(idx))
    u = rng.random((N, L), dtype=np.float32)
    g = synth.gumbel(rng, (N, L + 1, V)).astype(np.float32)
    r = oracle.verify(target, np.broadcast_to(branches, (N, K, L, V)), tokens, u, g, T,
                      mix_w=np.broadcast_to(w, (N, K)), target_row_off=np.zeros(N, np.int32),
                      n_threads=oracle.n_cores())
    assert r["flags"] == 0
    p = softmax(target.astype(np.float64) / T, axis=-1)
    acc, out = r["accept_len"], r["out_tokens"]
    for k in range(L + 1):
        sel = acc >= k
        counts = np.bincount(out[sel, k], minlength=V)
        res = chisquare(counts, p[k] * sel.sum())
        assert res.pvalue > 1e-3, (k, counts, p[k] * sel.sum())
    # a mixture that matches the target branch structure beats chance acceptance
    assert acc.mean() > 0


def test_monte_carlo_expected_length_closed_form():
    """Independent drafts at V=1000, L=16: the mean accepted length over 2000
    blocks lies within 4 standard errors of the closed form."""
    rng = np.random.default_rng(41)
    N, L, V, T = 2000, 16, 1000, 1.0
    target = (rng.standard_normal((L + 1, V)) * 2).astype(np.float32)
    draft_rows = (target[:L] + rng.standard_normal((L, V)) * 0.6).astype(np.float32)
    q = softmax(draft_rows.astype(np.float64) / T, axis=-1)
    tokens = np.stack([_sample_categorical(rng, q[i], N) for i in range(L)], axis=1).astype(np.int32)
    u = rng.random((N, L), dtype=np.float32)
    g = synth.gumbel(rng, (N, L + 1, V)).astype(np.float32)
    r = oracle.verify(target, np.broadcast_to(draft_rows, (N, L, V)), tokens, u, g, T,
                      target_row_off=np.zeros(N, np.int32), n_threads=oracle.n_cores())
    assert r["flags"] == 0
    p = softmax(target.astype(np.float64) / T, axis=-1)
    alpha = np.minimum(p[:L], q).sum(axis=1)
    closed = sum(np.prod(alpha[:i]) for i in range(1, L + 1))
    a = r["accept_len"].astype(np.float64)
    assert abs(a.mean() - closed) < 4 * a.std() / math.sqrt(N) + 1e-12, (a.mean(), closed)


def test_identity_q_equals_p_accepts_all():
    x = synth.custom(B=4, L=6, V=300, K=1, dtype="bf16", n_peaks=3, peak=5.0, seed=5)
    draft = x.target[:, :6].copy()
    vl = np.array([6, 3, 0, 1], np.int32)
    r = oracle.verify(x.target, draft, x.tokens, x.u, x.g, 1.0, verify_len=vl, diag=True)
    assert r["flags"] == 0
    np.testing.assert_array_equal(r["accept_len"], vl)
    for b in range(4):
        assert np.all(r["rho"][b, :vl[b]] == 1.0)
        assert r["terminal_kind"][b] == 1 and r["terminal_row"][b] == vl[b]


def test_k1_mixture_equals_independent():
    for dtype in ("f32", "bf16"):
        x = synth.custom(B=3, L=5, V=257, K=1, dtype=dtype, seed=7)
        a = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.3, diag=True)
        b = oracle.verify(x.target, x.draft[:, None], x.tokens, x.u, x.g, 1.3,
                          mix_w=np.ones((3, 1), np.float32), diag=True)
        for k in a:
            np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_one_hot_target_is_emitted():
    rng = np.random.default_rng(8)
    B, L, V = 6, 3, 50
    target = rng.standard_normal((B, L + 1, V)).astype(np.float32)
    star = rng.integers(0, V, size=(B, L + 1))
    for b in range(B):
        for i in range(L + 1):
            target[b, i, star[b, i]] = 1000.0
    draft = rng.standard_normal((B, L, V)).astype(np.float32)
    tokens = (star[:, :L] + 1) % V
    u = rng.random((B, L), dtype=np.float32)
    g = synth.gumbel(rng, (B, L + 1, V)).astype(np.float32)
    r = oracle.verify(target, draft, tokens, u, g, 1.0)
    np.testing.assert_array_equal(r["accept_len"], 0)
    np.testing.assert_array_equal(r["out_tokens"][:, 0], star[:, 0])
    # q == p: every position accepted, the bonus is the one-hot token of row L
    r = oracle.verify(target, target[:, :L].copy(), star[:, :L], u, g, 1.0)
    np.testing.assert_array_equal(r["accept_len"], L)
    np.testing.assert_array_equal(r["out_tokens"][:, L], star[:, L])


def test_noise_row_is_the_terminal_position():
    rng = np.random.default_rng(9)
    L, V = 3, 40
    target = (rng.standard_normal((1, L + 1, V)) * 0.01).astype(np.float32)
    g = np.zeros((1, L + 1, V), np.float32)
    spikes = [5, 11, 17, 23]
    for i, v in enumerate(spikes):
        g[0, i, v] = 50.0
    tokens = np.array([[0, 1, 2]], np.int32)
    # q == p: all accepted, bonus uses row L
    r = oracle.verify(target, target[:, :L].copy(), tokens, np.full((1, L), 0.5, np.float32), g, 1.0)
    assert r["out_tokens"][0, L] == spikes[L]
    # draft row 1 overweights token 1: rho_1 < 1 and u_1 ~ 1 rejects at 1, residual uses g row 1
    draft = target[:, :L].copy()
    draft[0, 1, 1] += 5.0
    u = np.array([[0.5, 0.999, 0.5]], np.float32)
    r = oracle.verify(target, draft, tokens, u, g, 1.0)
    assert r["accept_len"][0] == 1
    assert list(r["out_tokens"][0]) == [0, spikes[1], -1, -1]


def test_zero_verify_length_is_a_bonus_draw():
    x = synth.custom(B=2, L=4, V=64, dtype="f32", seed=3)
    r = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, verify_len=np.array([0, 0]), diag=True)
    np.testing.assert_array_equal(r["accept_len"], 0)
    zb = x.target[:, 0].astype(np.float64) + x.g[:, 0]
    np.testing.assert_array_equal(r["out_tokens"][:, 0], zb.argmax(axis=1))
    assert np.all(r["out_tokens"][:, 1:] == -1)


def test_rejection_with_empty_residual_uses_the_bonus_rule_on_row_j():
    """After a rejection the residual max(0, p - q) is empty only through
    rounding: here target and draft rows are all zero except the drafted
    token (-200 in the target, -199 in the draft), so the test rejects
    (rho = exp(-1) < u = 0.99) while both normalisers are exactly V - 1 and
    p == q everywhere else. The reading taken: row j is then drawn by the
    bonus rule, argmax_v x_j(v) / T + g[b, j, v]."""
    B, L, V = 2, 3, 50
    rng = np.random.default_rng(8)
    target = np.zeros((B, L + 1, V), np.float32)
    tokens = rng.integers(0, V, (B, L)).astype(np.int32)
    for b in range(B):
        for i in range(L):
            target[b, i, tokens[b, i]] = -200.0
    draft = target[:, :L].copy()
    for b in range(B):
        for i in range(L):
            draft[b, i, tokens[b, i]] = -199.0
    u = np.full((B, L), 0.99, np.float32)
    g = synth.gumbel(rng, (B, L + 1, V)).astype(np.float32)
    r = oracle.verify(target, draft, tokens, u, g, 1.0, diag=True)
    np.testing.assert_array_equal(r["accept_len"], 0)
    np.testing.assert_allclose(r["rho"][:, 0], math.exp(-1.0), rtol=1e-12)
    expect = (target[:, 0].astype(np.float64) + g[:, 0].astype(np.float64)).argmax(axis=1)
    np.testing.assert_array_equal(r["out_tokens"][:, 0], expect)
    assert np.all(r["out_tokens"][:, 1:] == -1)


def test_device_style_error_flags():
    x = synth.custom(B=3, L=4, V=64, dtype="f32", seed=4)
    tok = x.tokens.copy()
    tok[1, 2] = 64
    r = oracle.verify(x.target, x.draft, tok, x.u, x.g, 1.0)
    assert r["flags"] & oracle.FLAG_TOKEN_RANGE
    assert r["accept_len"][1] == -1 and np.all(r["out_tokens"][1] == -1)
    assert r["accept_len"][0] >= 0 and r["accept_len"][2] >= 0
    r = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, verify_len=np.array([4, 5, 0]))
    assert r["flags"] & oracle.FLAG_VERIFY_LEN and r["accept_len"][1] == -1
    t = x.target.copy()
    t[2, 1, 7] = np.nan
    r = oracle.verify(t, x.draft, x.tokens, x.u, x.g, 1.0)
    assert r["flags"] & oracle.FLAG_NONFINITE and r["accept_len"][2] == -1


def test_workload_one_is_deterministic():
    x = synth.workload_inputs(1)
    a = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, x.w.T)
    b = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, x.w.T, n_threads=2)
    np.testing.assert_array_equal(a["out_tokens"], b["out_tokens"])
    assert a["flags"] == 0
