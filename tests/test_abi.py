"""The C-ABI library: loads without a GPU, exports every function declared in
include/specv.h, and rejects bad arguments on the host before any CUDA call."""
import ctypes
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


P = 1 << 20  # a fake, aligned "device" address: never dereferenced, validation fails first


def test_verify_rejects_before_launch(lib):
    ws = lib.spec_verify_workspace_size(2, 4, 1, 64)
    args = [P, None, P, 1, P, None, P, P, 2, 4, 64, 1.0, P, P, P, ws, None]

    def call(**kw):
        a = list(args)
        names = ["target", "off", "draft", "dtype", "tokens", "vlen", "u", "g", "B", "L", "V", "T", "acc", "out",
                 "ws", "wsb", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return lib.spec_verify_block(*a)

    assert call(target=None) == -1
    assert call(tokens=None) == -1
    assert call(g=None) == -1
    assert call(dtype=3) == -1
    assert call(T=0.0) == -1
    assert call(T=-1.0) == -1
    assert call(T=float("nan")) == -1
    assert call(V=0) == -1
    assert call(B=0) == -1
    assert call(L=-1) == -1
    assert call(L=33) == -2
    assert call(B=5000) == -2
    assert call(ws=None) == -4
    assert call(wsb=ws - 1) == -4
    assert call(target=P + 1) == -1        # bf16 logits need 2-byte alignment
    assert call(u=P + 2) == -1
    # mixture: K limits and weights
    mws = lib.spec_verify_workspace_size(2, 4, 8, 64)
    assert lib.spec_verify_mixture(P, None, P, None, 4, 1, P, None, P, P, 2, 4, 64, 1.0, P, P, P, mws, None) == -1
    assert lib.spec_verify_mixture(P, None, P, P, 9, 1, P, None, P, P, 2, 4, 64, 1.0, P, P, P, mws, None) == -2
    assert lib.spec_verify_mixture(P, None, P, P, 0, 1, P, None, P, P, 2, 4, 64, 1.0, P, P, P, mws, None) == -1


def test_softmax_and_dvl_reject_before_launch(lib):
    ws = lib.spec_softmax_workspace_size(4)
    assert lib.spec_softmax_T(None, 1, 4, 64, 64, 1.0, P, P, None, P, ws, None) == -1
    assert lib.spec_softmax_T(P, 1, 4, 64, 32, 1.0, P, P, None, P, ws, None) == -1      # stride < V
    assert lib.spec_softmax_T(P, 1, 4, 64, 64, 0.0, P, P, None, P, ws, None) == -1
    assert lib.spec_softmax_T(P, 1, 4, 64, 64, 1.0, P, P, None, P, ws - 8, None) == -4
    dws = lib.spec_dvl_workspace_size(4)
    assert lib.dvl_allocate_pack(P, 4, 4, 3, P, P, P, None, None, 1, 64, P, dws, None) == -1   # budget < B
    assert lib.dvl_allocate_pack(None, 4, 4, 8, P, P, P, None, None, 1, 64, P, dws, None) == -1
    assert lib.dvl_allocate_pack(P, 4, 4, 8, P, P, P, P, None, 1, 64, P, dws, None) == -1      # pack needs both
    assert lib.dvl_allocate_pack(P, 4, 33, 8, P, P, P, None, None, 1, 64, P, dws, None) == -2
    assert lib.dvl_allocate_pack(P, 4, 4, 8, P, P, P, None, None, 1, 64, None, dws, None) == -4
    assert lib.spec_workspace_init(None, 16, None) == -1


def test_binding_fails_loudly_without_cuda_tensors(lib):
    import torch
    x = torch.zeros((2, 8), dtype=torch.float32)
    with pytest.raises((TypeError, RuntimeError)):
        specv.softmax_T(x, 1.0, workspace=object())
