"""Helpers shared by the GPU parity tests: move seeded inputs to the device and
compare the CUDA path's decisions with the oracle's under the low-margin rule.

Rule: accepted lengths and tokens must match bit for bit, except a decision
whose oracle margin is below 1e-6 (accept test: |u - min(1, rho)|; terminal
draw: the fp64 gap between the two best scores below 1e-6 * max(1, kappa),
kappa = p / (p - q) being the amplification of rounding in log(p - q)). Such a
decision, and everything after it in its request, is exempt and logged; at
most max(1, 1e-5 * decisions) of them may occur in one comparison.
"""
import math

import numpy as np
import torch

EPS = 1e-6


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


def check_verify(acc, out, ref, verify_len=None, log=None):
    """Compare GPU (acc [B], out [B, L+1]) with oracle.verify(diag=True) output."""
    acc = np.asarray(acc)
    out = np.asarray(out)
    B, L1 = out.shape
    L = L1 - 1
    n_dec = 0
    exempt = []
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
        if low:
            i0 = low[0]
            exempt.append((b, "accept", i0, float(m[i0])))
            assert acc[b] >= i0, (b, acc[b], i0)
            assert np.array_equal(out[b, :i0], ro[:i0]), b
            continue
        assert acc[b] == ja, ("accept_len", b, int(acc[b]), ja)
        assert np.array_equal(out[b, :ja], ro[:ja]), ("prefix", b)
        assert np.all(out[b, ja + 1:] == -1), ("padding", b)
        gap, kap = ref["argmax_gap"][b], ref["argmax_kappa"][b]
        if gap < EPS * max(1.0, kap):
            exempt.append((b, "argmax", ja, float(gap)))
            continue
        assert out[b, ja] == ro[ja], ("terminal token", b, int(out[b, ja]), int(ro[ja]), float(gap), float(kap))
    if log is not None:
        log.extend(exempt)
    assert len(exempt) <= max(1, math.floor(1e-5 * n_dec)), exempt
    return n_dec, exempt
