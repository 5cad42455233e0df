"""Pins of the oracle's top-p (nucleus) filtered verification (CPU only).

Target sampling runs at a temperature with top-p filtering ("DBLAST: Dependent
Block Drafting for Stochastic Speculative Decoding", Pith review, "What would
settle it": temperature 1.5, top-p 0.95), and target probabilities are taken
under the same sampling filter ("Assumptions"). The pages do not spell the
filter out; the reading taken is the usual nucleus: the smallest set of most
probable tokens (ties to the lower index) whose mass reaches top-p,
renormalised, every other token at probability 0, applied to the target rows
and to every draft category.

What fixes the expected values, none of it the oracle itself:
  * the nucleus equals the brute-force smallest subset of mass >= top-p over
    all subsets of a small vocabulary (with tied probabilities);
  * a vanishing top-p is greedy decoding: the draw is the argmax whatever the
    noise;
  * a drafted token outside the target's nucleus is always rejected;
  * losslessness: exact enumeration over every drafted block (drafted from
    the filtered proposal) must emit the filtered target rows.
"""
import itertools

import numpy as np
import pytest
from scipy.special import softmax

import oracle


def _brute_nucleus(p, top_p):
    """The filtered distribution of probability vector p: among the subsets of
    minimum size whose mass reaches top_p, the one that holds every token
    ranked above any of its members (rank: probability descending, then index
    ascending)."""
    V = len(p)
    order = sorted(range(V), key=lambda v: (-p[v], v))
    rank = {v: k for k, v in enumerate(order)}
    best = None
    for size in range(1, V + 1):
        for S in itertools.combinations(range(V), size):
            if sum(p[v] for v in S) < top_p:
                continue
            if max(rank[v] for v in S) != size - 1:  # not the top `size` tokens
                continue
            best = S
            break
        if best is not None:
            break
    # minimality over all subsets, not only top sets
    for size in range(1, len(best)):
        assert all(sum(p[v] for v in S) < top_p for S in itertools.combinations(range(V), size))
    q = np.zeros(V)
    idx = list(best)
    q[idx] = p[idx] / p[idx].sum()
    return q


def _well_separated(p, top_p, eps=1e-9):
    """True when no subset mass lies within eps of top_p (so that summation
    order cannot move the boundary)."""
    V = len(p)
    return all(abs(sum(p[list(S)]) - top_p) > eps for n in range(1, V + 1)
               for S in itertools.combinations(range(V), n))


@pytest.mark.parametrize("top_p", [0.3, 0.55, 0.8, 0.95, 0.999])
def test_nucleus_matches_brute_force(top_p):
    rng = np.random.default_rng(int(top_p * 1000))
    V, T = 7, 1.3
    rows = (rng.standard_normal((12, V)) * 1.5).astype(np.float32)
    rows[::3, 4] = rows[::3, 1]      # tied probabilities across the boundary
    rows[1::3, 6] = rows[1::3, 2]
    checked = 0
    for row in rows:
        p = softmax(row.astype(np.float64) / T)
        if not _well_separated(p, top_p):
            continue
        target = np.broadcast_to(row, (1, 2, V)).copy()  # bonus row 0 (verify_len 0)
        draft = target[:, :1].copy()
        r = oracle.verify(target, draft, np.zeros((1, 1), np.int32), np.zeros((1, 1), np.float32),
                          np.zeros((1, 2, V), np.float32), T, verify_len=np.zeros(1, np.int32), diag=True,
                          top_p=top_p)
        assert r["flags"] == 0 and r["terminal_kind"][0] == 1
        np.testing.assert_allclose(r["terminal_dist"][0], _brute_nucleus(p, top_p), rtol=1e-12, atol=1e-15)
        checked += 1
    assert checked >= 6


def test_top_p_one_changes_nothing():
    rng = np.random.default_rng(5)
    B, L, V, K = 4, 5, 40, 2
    target = rng.standard_normal((B, L + 1, V)).astype(np.float32)
    draft = (target[:, None, :L] + rng.standard_normal((B, K, L, V))).astype(np.float32)
    w = rng.random((B, K)).astype(np.float32)
    tokens = rng.integers(0, V, (B, L)).astype(np.int32)
    u = rng.random((B, L)).astype(np.float32)
    g = rng.gumbel(size=(B, L + 1, V)).astype(np.float32)
    a = oracle.verify(target, draft, tokens, u, g, 1.2, mix_w=w, diag=True)
    b = oracle.verify(target, draft, tokens, u, g, 1.2, mix_w=w, diag=True, top_p=1.0)
    for k in ("accept_len", "out_tokens", "rho", "terminal_dist"):
        np.testing.assert_array_equal(a[k], b[k])


def test_vanishing_top_p_is_greedy():
    rng = np.random.default_rng(6)
    B, V = 16, 30
    target = rng.standard_normal((B, 1, V)).astype(np.float32)
    g = rng.gumbel(size=(B, 1, V)).astype(np.float32) * 5.0  # noise that would usually move the draw
    r = oracle.verify(target, target[:, :0].copy(), np.zeros((B, 0), np.int32), np.zeros((B, 0), np.float32),
                      g, 0.8, top_p=1e-12)
    np.testing.assert_array_equal(r["out_tokens"][:, 0], target[:, 0].argmax(axis=1))


def test_drafted_token_outside_the_target_nucleus_is_rejected():
    V, T = 8, 1.0
    t0 = np.array([5.0, 4.0, 0.0, 0.0, 0.0, 0.0, 0.0, -1.0], np.float32)  # nucleus at 0.9: {0, 1}
    target = np.stack([t0, t0 * 0.5])[None]                             # [1, 2, V]
    d0 = np.array([0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 9.0], np.float32)  # the draft is sure of token 7
    draft = d0[None, None]
    tokens = np.array([[7]], np.int32)
    g = np.random.default_rng(7).gumbel(size=(1, 2, V)).astype(np.float32)
    p = softmax(t0.astype(np.float64) / T)
    assert _brute_nucleus(p, 0.9)[7] == 0.0 and p[:2].sum() >= 0.9
    for uu in (0.0, 0.5, 0.999):
        r = oracle.verify(target, draft, tokens, np.full((1, 1), uu, np.float32), g, T, diag=True, top_p=0.9)
        assert r["accept_len"][0] == 0 and r["rho"][0, 0] == 0.0
        assert r["out_tokens"][0, 0] in (0, 1)  # the residual lives inside the target's nucleus
    # outside both nuclei (the draft is sure of token 0 here): p = 0 still gives rho = 0
    draft0 = np.array([9.0, 0, 0, 0, 0, 0, 0, 0], np.float32)[None, None]
    r = oracle.verify(target, draft0, tokens, np.zeros((1, 1), np.float32), g, T, diag=True, top_p=0.9)
    assert r["flags"] == 0 and r["accept_len"][0] == 0 and r["rho"][0, 0] == 0.0
    assert r["out_tokens"][0, 0] == 1  # residual p' - q' > 0 only at token 1


def _enumerate_filtered(target, draft, w, T, top_p):
    """Every drafted block x (drafted from the filtered proposal) and every
    forced rejection point, through oracle.verify with u and g chosen to
    select each branch; returns the distribution of the emitted sequence."""
    L1, V = target.shape
    L = L1 - 1
    K = draft.shape[0]
    qf = np.array([[_brute_nucleus(softmax(draft[z, i].astype(np.float64) / T), top_p) for i in range(L)]
                   for z in range(K)])                                  # [K, L, V]
    seqs = [x for x in itertools.product(range(V), repeat=L)
            if sum(w[z] * np.prod([qf[z, i, x[i]] for i in range(L)]) for z in range(K)) > 0.0]
    reqs = [(x, j) for x in seqs for j in range(L + 1)]
    B = len(reqs)
    ONE_MINUS = np.float32(1.0 - 2.0 ** -24)
    tokens = np.array([x for x, _ in reqs], np.int32)
    u = np.zeros((B, L), np.float32)
    for n, (_, j) in enumerate(reqs):
        if j < L:
            u[n, j] = ONE_MINUS
    r = oracle.verify(target[None].repeat(B, 0), np.broadcast_to(draft, (B, K, L, V)).copy(), tokens, u,
                      np.zeros((B, L + 1, V), np.float32), T, mix_w=np.broadcast_to(w, (B, K)).copy(), diag=True,
                      top_p=top_p)
    assert r["flags"] == 0
    out = {}
    for n, (x, j) in enumerate(reqs):
        q_x = sum(w[z] * np.prod([qf[z, i, x[i]] for i in range(L)]) for z in range(K))
        nall = reqs.index((x, L))
        # positions after one whose token has filtered target probability 0
        # (rho = 0) are never tested (NaN): they are unreachable
        a = np.nan_to_num(np.minimum(1.0, r["rho"][nall]), nan=0.0)
        pj = np.prod(a[:j]) * ((1.0 - a[j]) if j < L else 1.0)
        if pj == 0.0:
            continue
        if j < L:
            assert a[j] < ONE_MINUS, "rejection at j cannot be forced with u < 1"
        assert r["terminal_row"][n] == j and r["accept_len"][n] == j
        dist = r["terminal_dist"][n]
        assert abs(dist.sum() - 1.0) < 1e-12
        for t in range(V):
            s = tuple(x[:j]) + (t,)
            out[s] = out.get(s, 0.0) + q_x * pj * dist[t]
    return out


@pytest.mark.parametrize("K", [1, 2])
@pytest.mark.parametrize("top_p", [0.6, 0.9])
def test_exact_enumeration_is_lossless_under_the_filter(K, top_p):
    rng = np.random.default_rng(30 + K + int(top_p * 10))
    L, V, T = 2, 5, 1.0
    for _ in range(50):  # draw rows whose nuclei are not decided by rounding
        target = (rng.standard_normal((L + 1, V)) * 1.5).astype(np.float32)
        draft = (target[None, :L] + rng.standard_normal((K, L, V)) * 1.2).astype(np.float32)
        rows = [softmax(target[i].astype(np.float64) / T) for i in range(L + 1)] + \
               [softmax(draft[z, i].astype(np.float64) / T) for z in range(K) for i in range(L)]
        if all(_well_separated(p, top_p) for p in rows):
            break
    w = np.array([1.0] if K == 1 else [0.3, 0.7], np.float32)  # sums to exactly 1 in fp32
    out = _enumerate_filtered(target, draft, w, T, top_p)
    pf = np.array([_brute_nucleus(softmax(target[k].astype(np.float64) / T), top_p) for k in range(L + 1)])
    assert abs(sum(out.values()) - 1.0) < 1e-12
    for k in range(L + 1):
        prefixes = {s[:k] for s in out if len(s) > k}
        for pre in prefixes:
            mass = np.zeros(V)
            for s, pr in out.items():
                if len(s) > k and s[:k] == pre:
                    mass[s[k]] += pr
            np.testing.assert_allclose(mass, pf[k] * mass.sum(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("top_p,expect", [(0.4, 0.1), (0.6, 0.1), (0.75, 0.05), (0.9, 0.1), (1.0, np.inf)])
def test_nucleus_margin_is_the_distance_to_the_cut(top_p, expect):
    """p = (0.5, 0.3, 0.2): the cumulative masses are 0.5, 0.8 and 1, and the
    margin is the distance from top_p to the masses just before and at the
    cut (e.g. 0.75 -> min(0.8 - 0.75, 0.75 - 0.5) = 0.05)."""
    row = np.log(np.array([0.5, 0.3, 0.2])).astype(np.float32)  # fp32 logits: p within ~1e-7 of these
    target = np.broadcast_to(row, (1, 2, 3)).copy()
    r = oracle.verify(target, target[:, :1].copy(), np.zeros((1, 1), np.int32), np.zeros((1, 1), np.float32),
                      np.zeros((1, 2, 3), np.float32), 1.0, verify_len=np.zeros(1, np.int32), diag=True,
                      top_p=top_p)
    m = r["nucleus_margin"][0]
    assert np.isinf(m) if np.isinf(expect) else abs(m - expect) < 1e-6


def test_nucleus_margin_takes_the_smallest_over_the_rows_used():
    """Target row 0 (0.5, 0.3, 0.2) has margin 0.05 at top_p 0.75; draft row 0
    (0.74, 0.16, 0.1) has min(0.9 - 0.75, 0.75 - 0.74) = 0.01, the request's."""
    t = np.log(np.array([[0.5, 0.3, 0.2], [0.5, 0.3, 0.2]])).astype(np.float32)[None]
    d = np.log(np.array([[0.74, 0.16, 0.1]])).astype(np.float32)[None]
    for uu in (0.0, 0.999):  # accepted (bonus row used) or rejected (residual on row 0)
        r = oracle.verify(t, d, np.zeros((1, 1), np.int32), np.full((1, 1), uu, np.float32),
                          np.zeros((1, 2, 3), np.float32), 1.0, diag=True, top_p=0.75)
        assert r["flags"] == 0 and abs(r["nucleus_margin"][0] - 0.01) < 1e-6


def test_rejects_bad_top_p():
    x = np.zeros((1, 2, 4), np.float32)
    for bad in (0.0, -0.5, 1.5, float("nan")):
        with pytest.raises(ValueError):
            oracle.verify(x, x[:, :1].copy(), np.zeros((1, 1), np.int32), np.zeros((1, 1), np.float32),
                          np.zeros((1, 2, 4), np.float32), 1.0, top_p=bad)
