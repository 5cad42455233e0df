"""spec_softmax_T_noalloc: the softmax statistics with the library's fixed
device scratch instead of a caller workspace, for callers that cannot
allocate device memory. Each call is compared, through the C ABI, with the
oracle and with spec_softmax_T (the workspace entry point) on the same
inputs, for two calls in a row that share the scratch. The file is named so
that pytest collects it last; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_block_spec_b200 as specv
from speculative_decoding_block_spec_b200.synth import f32_to_bf16_bits

from parity_util import assert_softmax_close, logits_to_torch

_F32, _BF16 = 0, 1


def _inputs(rows, V, dtype, seed):
    """Host logits (bf16 bits or fp32) and their device copy."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, V)).astype(np.float32) * 2
    x[:, -1] += 9.0  # a peak in the final chunk of every row
    xs = f32_to_bf16_bits(x) if dtype == "bf16" else x
    return xs, logits_to_torch(xs)


def _noalloc(logits, T, probs):
    """Call the entry point directly through ctypes (no Python-side allocation)."""
    rows, V = logits.shape
    rmax = torch.empty(rows, dtype=torch.float32, device=logits.device)
    rlse = torch.empty_like(rmax)
    p = torch.empty((rows, V), dtype=torch.float32, device=logits.device) if probs else None
    st = specv.lib().spec_softmax_T_noalloc(
        logits.data_ptr(), _BF16 if logits.dtype == torch.bfloat16 else _F32, rows, V, V, float(T),
        rmax.data_ptr(), rlse.data_ptr(), None if p is None else p.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, specv.lib().spec_status_string(st).decode()
    return rmax, rlse, p


def _with_workspace(logits, T, probs):
    rows, V = logits.shape
    rmax = torch.empty(rows, dtype=torch.float32, device=logits.device)
    rlse = torch.empty_like(rmax)
    p = torch.empty((rows, V), dtype=torch.float32, device=logits.device) if probs else None
    specv.spec_softmax_T(logits, T, rmax, rlse, p)
    return rmax, rlse, p


def _host(t):
    return [None if a is None else a.cpu().numpy() for a in t]


def _check(got, xs, logits, T, probs):
    """Against the oracle (1e-5 relative on maxima, normalisers and
    probabilities) and against the workspace entry point (same tolerance)."""
    got = _host(got)
    assert_softmax_close(got, oracle.softmax_T(xs, T, probs=probs))
    assert_softmax_close(got, _host(_with_workspace(logits, T, probs)))


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_workspace_path_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # call 1: bf16, 16-byte vector path, many rows; call 2: fp32, odd V (scalar path), with probabilities
    xa, a = _inputs(3000, 32000, "bf16", seed=1)
    xb, b = _inputs(517, 50257, "f32", seed=2)
    got_a = _noalloc(a, 0.8, probs=False)
    got_b = _noalloc(b, 1.3, probs=True)  # reuses the scratch call 1 just wrote
    torch.cuda.synchronize()
    _check(got_a, xa, a, 0.8, probs=False)
    _check(got_b, xb, b, 1.3, probs=True)


@pytest.mark.gpu
def test_noalloc_at_the_row_limit():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    xs, x = _inputs(specv.NOALLOC_MAX_ROWS, 2048, "bf16", seed=3)
    for _ in range(2):
        got = _noalloc(x, 1.0, probs=False)
        torch.cuda.synchronize()
        _check(got, xs, x, 1.0, probs=False)


def test_noalloc_rejects_rows_beyond_the_scratch_before_any_launch():
    """Run where no GPU is visible (tests/host_rejections.py)."""
    from host_rejections import run_without_gpu
    r = run_without_gpu("noalloc_rejects")
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), (r.stdout[-2000:], r.stderr[-4000:])
