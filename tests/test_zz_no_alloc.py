"""spec_softmax_T_noalloc: the softmax statistics with the library's fixed
device scratch instead of a caller workspace. It is compared, through the C
ABI, with spec_softmax_T on the same inputs, for two calls in a row that share
the scratch. The file is named so that pytest collects it last; it also passes
alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import speculative_decoding_block_spec_b200 as specv
from speculative_decoding_block_spec_b200.synth import f32_to_bf16_bits

from parity_util import logits_to_torch

_F32, _BF16 = 0, 1
_ERR_UNSUPPORTED = -2


def _inputs(rows, V, dtype, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, V)).astype(np.float32) * 2
    x[:, -1] += 9.0  # a peak in the final chunk of every row
    return logits_to_torch(f32_to_bf16_bits(x) if dtype == "bf16" else x)


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


def _close(got, ref):
    # the softmax parity tolerance: 1e-5 relative on maxima, normalisers and probabilities
    np.testing.assert_allclose(got[0].cpu().numpy(), ref[0].cpu().numpy(), rtol=1e-5, atol=0)
    np.testing.assert_allclose(got[1].cpu().numpy(), ref[1].cpu().numpy(), rtol=1e-5, atol=1e-6)
    if ref[2] is not None:
        np.testing.assert_allclose(got[2].cpu().numpy(), ref[2].cpu().numpy(), rtol=1e-5, atol=1e-37)


@pytest.mark.gpu
def test_noalloc_matches_workspace_path_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # call 1: bf16, 16-byte vector path, many rows; call 2: fp32, odd V (scalar path), with probabilities
    a = _inputs(3000, 32000, "bf16", seed=1)
    b = _inputs(517, 50257, "f32", seed=2)
    got_a = _noalloc(a, 0.8, probs=False)
    got_b = _noalloc(b, 1.3, probs=True)  # reuses the scratch call 1 just wrote
    torch.cuda.synchronize()
    _close(got_a, _with_workspace(a, 0.8, probs=False))
    _close(got_b, _with_workspace(b, 1.3, probs=True))


@pytest.mark.gpu
def test_noalloc_at_the_row_limit():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    x = _inputs(specv.NOALLOC_MAX_ROWS, 2048, "bf16", seed=3)
    for _ in range(2):
        got = _noalloc(x, 1.0, probs=False)
        _close(got, _with_workspace(x, 1.0, probs=False))


def test_noalloc_rejects_rows_beyond_the_scratch_before_any_launch():
    lib = specv.lib()
    fake = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    st = lib.spec_softmax_T_noalloc(fake, _F32, specv.NOALLOC_MAX_ROWS + 1, 1024, 1024, 1.0, fake, fake, None, None)
    assert st == _ERR_UNSUPPORTED
    assert "supported limits" in lib.spec_status_string(st).decode()
