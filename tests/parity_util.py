"""Helpers shared by the GPU parity tests: move seeded inputs to the device and
compare the CUDA path's decisions with the oracle's under the low-margin rule.

Rule: accepted lengths and tokens must match bit for bit. A decision whose
oracle margin is below 1e-6 (accept test: |u - min(1, rho)|; terminal draw:
the fp64 gap between the two best scores below 1e-6 * max(1, kappa), kappa =
p / (p - q) being the amplification of rounding in log(p - q); with top-p
filtering, a nucleus boundary whose cumulative mass lies within 1e-6 of
top-p, over the rows the request's outputs depend on) is logged in the
run-wide tally. If the GPU differs from the oracle on such a request,
the request is exempt from the comparison from that decision on (its earlier
outputs must still match) and counts as an exempted difference. Over the
whole test run the exempted differences must stay at or below 1e-5 of all
decisions (tests/conftest.py checks the tally when the session ends), so with
fewer than 100,000 decisions none is allowed.

Normalisers: a relative error e in sum_v exp(z_v) is an absolute error e in
its log, so `assert_lse_close` bounds |lse_gpu - lse_oracle| by 1e-5.
"""
import numpy as np
import torch

EPS = 1e-6
NORMALISER_RTOL = 1e-5

# Run-wide tally of verify decisions (see the module docstring).
TALLY = {"decisions": 0, "low_margin": [], "exempted": []}


def logits_to_torch(a, device="cuda"):
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_torch(x, device="cuda"):
    """synth.Inputs -> dict of device tensors."""
    d = dict(target=logits_to_torch(x.target, device), draft=logits_to_torch(x.draft, device),
             tokens=torch.from_numpy(x.tokens).to(device), u=torch.from_numpy(x.u).to(device),
             g=torch.from_numpy(x.g).to(device))
    if x.mix_w is not None:
        d["mix_w"] = torch.from_numpy(x.mix_w).to(device)
    if x.scores is not None:
        d["scores"] = torch.from_numpy(x.scores).to(device)
    return d


def assert_lse_close(got, ref):
    """Log-normalisers: 1e-5 relative on the normaliser itself."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    np.testing.assert_allclose(got, ref, rtol=0, atol=NORMALISER_RTOL)


def assert_softmax_close(got, ref):
    """(row_max, row_lse[, probs]) of the GPU against the oracle's: maxima and
    probabilities within 1e-5 relative, normalisers within 1e-5 relative."""
    np.testing.assert_allclose(got[0], ref[0], rtol=1e-5, atol=0)
    assert_lse_close(got[1], ref[1])
    if len(ref) > 2 and ref[2] is not None:
        np.testing.assert_allclose(got[2], ref[2], rtol=1e-5, atol=1e-37)


def check_verify(acc, out, ref, verify_len=None, log=None):
    """Compare GPU (acc [B], out [B, L+1]) with oracle.verify(diag=True) output.
    Returns (decisions, low-margin entries of this call)."""
    acc = np.asarray(acc)
    out = np.asarray(out)
    B, L1 = out.shape
    L = L1 - 1
    n_dec = 0
    low_here = []
    for b in range(B):
        ja = int(ref["accept_len"][b])
        ro = ref["out_tokens"][b]
        if ja < 0:
            assert acc[b] == -1 and np.all(out[b] == -1), (b, acc[b], out[b])
            continue
        ell = L if verify_len is None else int(verify_len[b])
        tested = ja + 1 if ja < ell else ja
        m = ref["accept_margin"][b]
        low = [i for i in range(tested) if m[i] < EPS]
        n_dec += tested + 1
        same = acc[b] == ja and np.array_equal(out[b], ro)
        nm = ref.get("nucleus_margin")
        if nm is not None and nm[b] < EPS:  # top-p: a nucleus boundary the outputs depend on is low-margin
            entry = (b, "nucleus", 0, float(nm[b]), bool(same))
            low_here.append(entry)
            if not same:
                TALLY["exempted"].append(entry)
            continue
        if low:
            i0 = low[0]
            entry = (b, "accept", i0, float(m[i0]), bool(same))
            low_here.append(entry)
            if not same:
                assert acc[b] >= i0, (b, acc[b], i0)
                assert np.array_equal(out[b, :i0], ro[:i0]), b
                TALLY["exempted"].append(entry)
            continue
        assert acc[b] == ja, ("accept_len", b, int(acc[b]), ja)
        assert np.array_equal(out[b, :ja], ro[:ja]), ("prefix", b)
        assert np.all(out[b, ja + 1:] == -1), ("padding", b)
        gap, kap = ref["argmax_gap"][b], ref["argmax_kappa"][b]
        if gap < EPS * max(1.0, kap):
            entry = (b, "argmax", ja, float(gap), bool(same))
            low_here.append(entry)
            if not same:
                TALLY["exempted"].append(entry)
            continue
        assert out[b, ja] == ro[ja], ("terminal token", b, int(out[b, ja]), int(ro[ja]), float(gap), float(kap))
    TALLY["decisions"] += n_dec
    TALLY["low_margin"].extend(low_here)
    if log is not None:
        log.extend(low_here)
    return n_dec, low_here


def exemption_budget_ok():
    """True when the run's exempted differences are at most 1e-5 of its decisions."""
    return len(TALLY["exempted"]) <= int(np.floor(1e-5 * TALLY["decisions"]))
