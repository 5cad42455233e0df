"""Host-side argument rejection of the C ABI, run by tests/test_abi.py,
tests/test_zz_no_alloc.py and tests/test_c_header.py in a child process
that sees no GPU (CUDA_VISIBLE_DEVICES=""). Every call here must be rejected
on the host before any CUDA call; the pointers are placeholders that are
never dereferenced, and without a visible device a call that slipped past
its checks would fail on the host instead of launching on them.

    python tests/host_rejections.py <check>...
"""
import ctypes
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import speculative_decoding_block_spec_b200 as specv  # noqa: E402

P = 1 << 20  # an aligned placeholder address, never dereferenced


def verify_rejects(lib):
    ws = lib.spec_verify_workspace_size(2, 4, 1, 64)
    args = [P, None, P, 1, P, None, P, P, 2, 4, 64, 1.0, P, P, P, ws, None]
    names = ["target", "off", "draft", "dtype", "tokens", "vlen", "u", "g", "B", "L", "V", "T", "acc", "out",
             "ws", "wsb", "stream"]

    def call(**kw):
        a = list(args)
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


def softmax_and_dvl_reject(lib):
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


def noalloc_rejects(lib):
    fake = ctypes.c_void_p(P)
    st = lib.spec_softmax_T_noalloc(fake, 0, specv.NOALLOC_MAX_ROWS + 1, 1024, 1024, 1.0, fake, fake, None, None)
    assert st == -2, st
    assert "supported limits" in lib.spec_status_string(st).decode()
    assert lib.spec_softmax_T_noalloc(None, 0, 4, 1024, 1024, 1.0, fake, fake, None, None) == -1
    assert lib.spec_softmax_T_noalloc(fake, 0, 4, 1024, 1024, 0.0, fake, fake, None, None) == -1


CHECKS = {"verify_rejects": verify_rejects, "softmax_and_dvl_reject": softmax_and_dvl_reject,
          "noalloc_rejects": noalloc_rejects}


def run_without_gpu(*names):
    """Run the named checks in a child process with no visible GPU; returns its CompletedProcess."""
    import subprocess
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, os.path.abspath(__file__)] + list(names), env=env, capture_output=True,
                          text=True, timeout=300)


if __name__ == "__main__":
    if os.environ.get("CUDA_VISIBLE_DEVICES") != "":
        sys.exit("run with CUDA_VISIBLE_DEVICES= (no visible GPU)")
    lib = specv.lib()
    for name in sys.argv[1:]:
        CHECKS[name](lib)
    print("ok")
