"""The C-ABI library: loads without a GPU, exports every function declared in
include/specv.h, and rejects bad arguments on the host before any CUDA call."""
import os
import re
import subprocess

import pytest

import speculative_decoding_block_spec_b200 as specv
from speculative_decoding_block_spec_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return specv.lib()


def _declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_]\w*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert len(declared) >= 9, declared
    dyn = subprocess.run(["nm", "-D", "--defined-only", specv.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in dyn.splitlines() if line.strip()}
    for name in declared:
        assert name in exported, name
        assert hasattr(lib, name)
    assert set(specv.EXPORTS) == set(declared)


def test_status_strings(lib):
    for st in (0, -1, -2, -3, -4):
        assert lib.spec_status_string(st).decode().startswith("SPEC_")
    assert b"unknown" in lib.spec_status_string(7)


def test_workspace_sizes(lib):
    V = 151936
    assert lib.spec_verify_workspace_size(8, 16, 1, V) > 0
    assert lib.spec_verify_workspace_size(8, 16, 4, V) > lib.spec_verify_workspace_size(8, 16, 1, V)
    assert lib.spec_verify_workspace_size(0, 16, 1, V) == 0
    assert lib.spec_verify_workspace_size(8, 33, 1, V) == 0
    assert lib.spec_verify_workspace_size(8, 16, 9, V) == 0
    assert lib.spec_verify_workspace_size(8, 16, 1, 0) == 0
    assert lib.spec_verify_workspace_size(4097, 16, 1, V) == 0
    assert lib.spec_softmax_workspace_size(100) > lib.spec_softmax_workspace_size(0) > 0
    assert lib.spec_softmax_workspace_size(-1) == 0
    assert lib.spec_dvl_workspace_size(32) > 0 and lib.spec_dvl_workspace_size(0) == 0
    for B, L, K in [(1, 0, 1), (8, 16, 1), (64, 16, 4), (4096, 32, 8)]:
        assert lib.spec_verify_workspace_size(B, L, K, V) % 256 == 0


def _no_gpu(*checks):
    """Host-rejection checks run in a child process that sees no GPU, so a call
    that slipped past its argument checks could not launch on the placeholder
    addresses the checks pass (tests/host_rejections.py)."""
    from host_rejections import run_without_gpu
    r = run_without_gpu(*checks)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), (r.stdout[-2000:], r.stderr[-4000:])


def test_verify_rejects_before_launch(lib):
    _no_gpu("verify_rejects")


def test_softmax_and_dvl_reject_before_launch(lib):
    _no_gpu("softmax_and_dvl_reject")


def test_binding_fails_loudly_without_cuda_tensors(lib):
    import torch
    x = torch.zeros((2, 8), dtype=torch.float32)
    with pytest.raises((TypeError, RuntimeError)):
        specv.softmax_T(x, 1.0, workspace=object())
