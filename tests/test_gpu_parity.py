"""GPU <-> oracle parity through the C ABI (needs a B200).

Every input is seeded and synthetic (speculative_decoding_block_spec_b200.synth).
Decisions (accepted lengths, tokens, verify lengths, offsets, slot maps,
packed rows) must match bit for bit, under the low-margin rule of
tests/parity_util.py (run-wide exemption budget); softmax maxima, normalisers
and probabilities within 1e-5 relative (a normaliser through its log:
|lse_gpu - lse_oracle| <= 1e-5).
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_block_spec_b200 as specv
from speculative_decoding_block_spec_b200 import synth
from speculative_decoding_block_spec_b200.synth import f32_to_bf16_bits

from parity_util import assert_softmax_close, check_verify, logits_to_torch, to_torch

pytestmark = pytest.mark.gpu
NT = oracle.n_cores()


@pytest.fixture(scope="module", autouse=True)
def side_stream():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    specv.lib()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        yield s
    s.synchronize()


def _cpu(t):
    torch.cuda.current_stream().synchronize()
    return t.cpu().numpy()


# ----------------------------------------------------------------- softmax_T

@pytest.mark.parametrize("rows,V,dtype,T,probs", [
    (6, 64, "f32", 1.0, True),
    (9, 1001, "f32", 1.5, True),        # scalar path (V*4 not a multiple of 16)
    (5, 1001, "bf16", 0.7, True),       # scalar path
    (1, 8, "bf16", 1.0, True),
    (300, 4096, "bf16", 1.0, True),     # many rows per block
    (40, 151936, "bf16", 1.0, False),   # balanced one-block-per-SM kernel (5,133 units per SM)
    (40, 151936, "bf16", 1.3, True),    # the same kernel, with probabilities
    (12, 151936, "bf16", 1.5, True),
    (3, 151936, "f32", 1.0, True),
])
def test_softmax_parity(rows, V, dtype, T, probs):
    rng = np.random.default_rng(rows * 7 + V)
    x = rng.standard_normal((rows, V)).astype(np.float32) * 2
    x[:, -1] += 9.0                      # the peak sits in the final chunk
    x[0, 0] += 12.0
    xs = f32_to_bf16_bits(x) if dtype == "bf16" else x
    ref = oracle.softmax_T(xs, T, probs=probs)
    got = specv.softmax_T(logits_to_torch(xs), T, probs=probs)
    assert_softmax_close([_cpu(t) for t in got], ref)


@pytest.mark.parametrize("dtype,V,stride", [("bf16", 4000, 4096), ("bf16", 4000, 4003), ("f32", 1000, 1024)])
def test_softmax_padded_row_stride(dtype, V, stride):
    """Rows start every `stride` elements and only their first V are logits
    (row_stride > V in the C ABI); the padding holds values that would
    dominate every row if it were read. 4096 keeps the 16-byte path, 4003
    forces the scalar one."""
    rows, T = 37, 1.3
    rng = np.random.default_rng(stride + V)
    full = rng.standard_normal((rows, stride)).astype(np.float32) * 2
    full[:, V:] = 1.0e4
    xs = f32_to_bf16_bits(full) if dtype == "bf16" else full
    ref = oracle.softmax_T(np.ascontiguousarray(xs[:, :V]), T, probs=True)
    logits = logits_to_torch(xs)
    rmax = torch.empty(rows, dtype=torch.float32, device="cuda")
    rlse = torch.empty_like(rmax)
    probs = torch.empty((rows, V), dtype=torch.float32, device="cuda")
    ws = specv.Workspace(specv.softmax_workspace_size(rows))
    st = specv.lib().spec_softmax_T(logits.data_ptr(), 1 if dtype == "bf16" else 0, rows, V, stride, T,
                                    rmax.data_ptr(), rlse.data_ptr(), probs.data_ptr(), ws.ptr(), ws.nbytes,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert_softmax_close([_cpu(rmax), _cpu(rlse), _cpu(probs)], ref)


@pytest.mark.parametrize("K", [1, 3])
@pytest.mark.parametrize("T", [0.3, 3.0])
def test_extreme_temperatures(T, K):
    """Sharp (T = 0.3: logits / T reach about 30) and flat (T = 3) target and
    draft distributions, same T for both ("DBLAST", "Assumptions")."""
    x = synth.custom(B=6, L=12, V=65536, K=K, T=T, dtype="bf16", n_peaks=8, peak=6.0, draft_sigma=0.7,
                     seed=int(T * 10) + K, cid=480 + int(T * 10) + K)
    vl = np.random.default_rng(int(T * 10) + K).integers(0, 13, size=6).astype(np.int32)
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, T, mix_w=x.mix_w, verify_len=vl, n_threads=NT,
                        diag=True)
    d = to_torch(x)
    acc, out = _verify(d, x, T, verify_len=torch.from_numpy(vl).cuda())
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


# ------------------------------------------------------------ the workloads

def _verify(d, x, T, verify_len=None, target=None, row_off=None, path="fused"):
    """One verification through the C ABI. path 'fused' is the public one-call
    entry point (spec_verify_block / spec_verify_mixture, which launch both
    stages chained); 'split' makes the two stage calls itself,
    spec_verify_window_stats then spec_verify_accept."""
    tgt = d["target"] if target is None else target
    mix = d.get("mix_w") if x.w.K > 1 else None
    if path == "split":
        B, L = d["tokens"].shape
        ws = specv.Workspace(specv.verify_workspace_size(B, L, x.w.K, x.w.V))
        specv.spec_verify_window_stats(tgt, d["draft"], d["tokens"], T, ws, verify_len=verify_len,
                                       target_row_off=row_off)
        return specv.spec_verify_accept(tgt, d["draft"], d["tokens"], d["u"], d["g"], T, ws, mix_w=mix,
                                        verify_len=verify_len, target_row_off=row_off)
    if x.w.K == 1:
        return specv.spec_verify_block(tgt, d["draft"], d["tokens"], d["u"], d["g"], T, verify_len=verify_len,
                                       target_row_off=row_off)
    return specv.spec_verify_mixture(tgt, d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], T,
                                     verify_len=verify_len, target_row_off=row_off)


PATHS = ["fused", "split"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("cid", [1, 2, 3])
def test_dense_workloads(cid, path):
    x = synth.workload_inputs(cid)
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, x.w.T, mix_w=x.mix_w, n_threads=NT, diag=True)
    d = to_torch(x)
    acc, out = _verify(d, x, x.w.T, path=path)
    check_verify(_cpu(acc), _cpu(out), ref)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("cid", [4, 5])
def test_dvl_packed_workloads(cid, path):
    x = synth.workload_inputs(cid)
    w = x.w
    rd = oracle.dvl_allocate(x.scores, w.budget)
    packed_ref = oracle.pack(x.target, rd["verify_len"], rd["offsets"], w.budget)
    ref = oracle.verify(packed_ref, x.draft, x.tokens, x.u, x.g, w.T, mix_w=x.mix_w, n_threads=NT, diag=True,
                        verify_len=rd["verify_len"], target_row_off=rd["offsets"][:w.B])
    d = to_torch(x)
    packed = torch.zeros((w.budget, w.V), dtype=d["target"].dtype, device="cuda")
    vl, off, sm = specv.dvl_allocate_pack(d["scores"], w.budget, dense_target=d["target"], packed_target=packed)
    np.testing.assert_array_equal(_cpu(vl), rd["verify_len"])
    np.testing.assert_array_equal(_cpu(off), rd["offsets"])
    np.testing.assert_array_equal(_cpu(sm), rd["slot_map"])
    pk = _cpu(packed.view(torch.int16)).view(np.uint16)
    np.testing.assert_array_equal(pk[:rd["offsets"][-1]], packed_ref[:rd["offsets"][-1]])
    acc, out = _verify(d, x, w.T, verify_len=vl, target=packed, row_off=off[:w.B], path=path)
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=rd["verify_len"])


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("seed", range(6))
def test_seed_sweep_block_and_mixture(seed, path):
    K = 1 if seed % 2 == 0 else 3
    x = synth.custom(B=8, L=16, V=32768, K=K, T=1.0 + 0.25 * (seed % 3), dtype="bf16", n_peaks=8, peak=6.0,
                     draft_sigma=0.7, seed=seed, cid=200 + seed)
    vl = np.random.default_rng(seed).integers(0, 17, size=8).astype(np.int32)
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, x.w.T, mix_w=x.mix_w, verify_len=vl,
                        n_threads=NT, diag=True)
    d = to_torch(x)
    acc, out = _verify(d, x, x.w.T, verify_len=torch.from_numpy(vl).cuda(), path=path)
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("K,L,V,dtype", [(5, 16, 32768, "bf16"), (8, 32, 8192, "bf16"), (8, 7, 1001, "f32")])
def test_mixture_beyond_one_draft_batch_and_largest_shapes(K, L, V, dtype, path):
    """Latent-mixture drafts ("DBLAST", "What carries the argument", Eq. 5)
    with more categories than one batch of terminal draft loads (K > 4), up to
    the largest K = 8 and L = 32, on the vector and the scalar path."""
    x = synth.custom(B=6, L=L, V=V, K=K, T=1.1, dtype=dtype, n_peaks=4, peak=5.0, draft_sigma=0.6, seed=K + L,
                     cid=400 + K + L)
    vl = np.random.default_rng(K * L).integers(0, L + 1, size=6).astype(np.int32)
    vl[0] = L
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, x.w.T, mix_w=x.mix_w, verify_len=vl,
                        n_threads=NT, diag=True)
    assert np.any(ref["accept_len"] < vl)  # some request rejects: the residual over K draft rows is exercised
    d = to_torch(x)
    acc, out = _verify(d, x, x.w.T, verify_len=torch.from_numpy(vl).cuda(), path=path)
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


@pytest.mark.parametrize("K", [1, 2])
def test_largest_batch(K):
    """B = SPEC_MAX_B requests (one sampling block each) with ragged verify lengths."""
    B, L, V = 4096, 2, 256
    x = synth.custom(B=B, L=L, V=V, K=K, T=1.0, dtype="bf16", n_peaks=2, peak=3.0, draft_sigma=0.5, seed=50 + K,
                     cid=450 + K)
    vl = np.random.default_rng(50 + K).integers(0, L + 1, size=B).astype(np.int32)
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, mix_w=x.mix_w, verify_len=vl, n_threads=NT,
                        diag=True)
    d = to_torch(x)
    acc, out = _verify(d, x, 1.0, verify_len=torch.from_numpy(vl).cuda())
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


def test_largest_vocabulary_and_top_token_index():
    """V = SPEC_MAX_V = 2^20: the terminal keys carry the token in 20 bits, so
    the draws land on tokens V - 1 (bonus row) and V - 2 (residual)."""
    B, L, V = 2, 2, 1 << 20
    rng = np.random.default_rng(60)
    t = rng.standard_normal((B, L + 1, V)).astype(np.float32)
    dr = t[:, :L].copy()
    tokens = np.array([[3, 5], [7, 9]], np.int32)
    t[0, L, V - 1] = 60.0        # request 0 accepts both positions (draft == target): bonus row peaks at V - 1
    t[1, 0, V - 2] = 60.0        # request 1: target row 0 peaks at V - 2, which the draft lacks, so x_0 is
    dr[1, 0, tokens[1, 0]] = 40.0  # rejected (the draft is confident in it) and the residual is V - 2
    tt, dd = f32_to_bf16_bits(t), f32_to_bf16_bits(dr)
    u = np.full((B, L), 0.5, np.float32)
    g = synth.gumbel(rng, (B, L + 1, V)).astype(np.float32)
    ref = oracle.verify(tt, dd, tokens, u, g, 1.0, n_threads=NT, diag=True)
    np.testing.assert_array_equal(ref["accept_len"], [2, 0])
    assert ref["out_tokens"][0, 2] == V - 1 and ref["out_tokens"][1, 0] == V - 2
    acc, out = specv.spec_verify_block(logits_to_torch(tt), logits_to_torch(dd), torch.from_numpy(tokens).cuda(),
                                       torch.from_numpy(u).cuda(), torch.from_numpy(g).cuda(), 1.0)
    check_verify(_cpu(acc), _cpu(out), ref)


# -------------------------------------------------------------- identities

def test_k1_mixture_is_bit_identical_to_block():
    x = synth.custom(B=6, L=16, V=151936, K=1, dtype="bf16", n_peaks=32, peak=8.0, seed=11, cid=300)
    d = to_torch(x)
    a1, o1 = specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0)
    a2, o2 = specv.spec_verify_mixture(d["target"], d["draft"][:, None].contiguous(),
                                       torch.ones((6, 1), dtype=torch.float32, device="cuda"),
                                       d["tokens"], d["u"], d["g"], 1.0)
    assert torch.equal(a1, a2) and torch.equal(o1, o2)


def test_q_equals_p_accepts_everything():
    x = synth.custom(B=4, L=16, V=151936, K=1, dtype="bf16", n_peaks=32, peak=8.0, seed=12, cid=301)
    x.draft = x.target[:, :16].copy()
    vl = np.array([16, 5, 0, 1], np.int32)
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, verify_len=vl, n_threads=NT, diag=True)
    d = to_torch(x)
    acc, out = specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0,
                                       verify_len=torch.from_numpy(vl).cuda())
    np.testing.assert_array_equal(_cpu(acc), vl)
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


def test_rejection_with_empty_residual_draws_row_j_by_the_bonus_rule():
    """Speculative sampling with rejection correction ("DBLAST", Pith review,
    "Assumptions"): after a rejection the residual max(0, p - q) has positive
    mass in exact arithmetic. Here target and draft rows are all zero except
    at the drafted token, which sits at -200 in the target and -199 in the
    draft: the test rejects (rho = exp(-1)), but that token's share of either
    normaliser is below the precision of the sum, and every other term is
    exactly 1, so both normalisers are exactly V - 1 in any summation order,
    fp32 and fp64 alike, and no element has p > q. Both sides then draw row j
    by the bonus rule, which on the GPU is the request's last block scanning
    the row."""
    rng = np.random.default_rng(41)
    B, L, V = 3, 4, 151936
    tt = np.zeros((B, L + 1, V), np.uint16)  # bf16 zeros
    tokens = rng.integers(0, V, (B, L)).astype(np.int32)
    for b in range(B):
        for i in range(L):
            tt[b, i, tokens[b, i]] = 0xC348  # -200.0
    dd = tt[:, :L].copy()
    for b in range(B):
        for i in range(L):
            dd[b, i, tokens[b, i]] = 0xC347  # -199.0
    u = np.full((B, L), 0.99, np.float32)
    g = synth.gumbel(rng, (B, L + 1, V)).astype(np.float32)
    ref = oracle.verify(tt, dd, tokens, u, g, 1.0, n_threads=NT, diag=True)
    np.testing.assert_array_equal(ref["accept_len"], np.zeros(B, np.int32))
    ws = specv.Workspace(specv.verify_workspace_size(B, L, 1, V))
    acc, out = specv.spec_verify_block(logits_to_torch(tt), logits_to_torch(dd), torch.from_numpy(tokens).cuda(),
                                       torch.from_numpy(u).cuda(), torch.from_numpy(g).cuda(), 1.0, workspace=ws)
    np.testing.assert_array_equal(_cpu(acc), ref["accept_len"])
    np.testing.assert_array_equal(_cpu(out), ref["out_tokens"])
    assert ws.status() == 0


def test_one_hot_target_and_vocab_edge_tokens():
    rng = np.random.default_rng(13)
    B, L, V = 4, 6, 151936
    t = rng.standard_normal((B, L + 1, V)).astype(np.float32)
    star = np.array([[0, V - 1, 5, V - 2, 77, 1000, V - 1]] * B)
    for b in range(B):
        for i in range(L + 1):
            t[b, i, star[b, i]] = 1000.0
    dr = rng.standard_normal((B, L, V)).astype(np.float32)
    tokens = np.zeros((B, L), np.int32)
    tokens[1] = V - 1
    tokens[2, ::2] = V - 1
    u = rng.random((B, L), dtype=np.float32)
    g = synth.gumbel(rng, (B, L + 1, V)).astype(np.float32)
    for dtype in ("f32", "bf16"):
        tt = f32_to_bf16_bits(t) if dtype == "bf16" else t
        dd = f32_to_bf16_bits(dr) if dtype == "bf16" else dr
        ref = oracle.verify(tt, dd, tokens, u, g, 1.0, n_threads=NT, diag=True)
        acc, out = specv.spec_verify_block(logits_to_torch(tt), logits_to_torch(dd), torch.from_numpy(tokens).cuda(),
                                           torch.from_numpy(u).cuda(), torch.from_numpy(g).cuda(), 1.0)
        check_verify(_cpu(acc), _cpu(out), ref)
        # rows where the drafted token is not the one-hot token reject at 0 and emit the one-hot token
        o = _cpu(out)
        for b in range(B):
            if tokens[b, 0] != star[b, 0]:
                assert o[b, 0] == star[b, 0]


def test_exact_ties_go_to_lowest_index():
    B, L, V = 2, 2, 4096
    target = np.zeros((B, L + 1, V), np.float32)          # uniform target rows
    draft = np.zeros((B, L, V), np.float32)
    draft[0, 0, 100] = 6.0                                  # request 0 drafts an over-weighted token
    tokens = np.array([[100, 0], [3, 4]], np.int32)
    u = np.array([[0.999, 0.5], [0.5, 0.5]], np.float32)
    g = np.zeros((B, L + 1, V), np.float32)
    acc, out = specv.spec_verify_block(*(torch.from_numpy(a).cuda() for a in (target, draft, tokens, u, g)), 1.0)
    acc, out = _cpu(acc), _cpu(out)
    # request 0: rejected at 0; residual mass is equal on every token but 100 -> lowest index 0
    assert acc[0] == 0 and out[0, 0] == 0
    # request 1: q == p (uniform) -> all accepted; uniform bonus row, zero noise -> token 0
    assert acc[1] == 2 and list(out[1]) == [3, 4, 0]


# ----------------------------------------------------------- device errors

@pytest.mark.parametrize("path", PATHS)
def test_device_flags_and_isolation(path):
    x = synth.custom(B=4, L=8, V=4096, K=2, dtype="bf16", n_peaks=4, peak=5.0, seed=14, cid=302)
    x.tokens[1, 3] = 4096                        # out of range
    x.target[3, 2, 17] = 0x7FC0                  # NaN in a tested row of request 3
    vl = np.array([8, 8, 8, 8], np.int32)
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, mix_w=x.mix_w, verify_len=vl, diag=True)
    assert ref["flags"] & oracle.FLAG_TOKEN_RANGE and ref["flags"] & oracle.FLAG_NONFINITE
    d = to_torch(x)
    ws = specv.Workspace(specv.verify_workspace_size(4, 8, 2, 4096))
    if path == "split":
        vlt = torch.from_numpy(vl).cuda()
        specv.spec_verify_window_stats(d["target"], d["draft"], d["tokens"], 1.0, ws, verify_len=vlt)
        acc, out = specv.spec_verify_accept(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0, ws,
                                            mix_w=d["mix_w"], verify_len=vlt)
    else:
        acc, out = specv.spec_verify_mixture(d["target"], d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"],
                                             1.0, verify_len=torch.from_numpy(vl).cuda(), workspace=ws)
    st = ws.status()
    assert st & specv.DEV_TOKEN_RANGE and st & specv.DEV_NONFINITE
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)
    # an out-of-range verify length
    ws.init()
    bad = torch.tensor([8, 9, -1, 0], dtype=torch.int32, device="cuda")
    acc, out = specv.spec_verify_mixture(d["target"], d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], 1.0,
                                         verify_len=bad, workspace=ws)
    a = _cpu(acc)
    assert ws.status() & specv.DEV_VERIFY_LEN
    assert a[1] == -1 and a[2] == -1 and a[3] == 0


def test_workspace_reuse_is_self_resetting():
    """Many calls on one workspace, alternating the fused and the two-stage
    paths and changing shapes within its capacity: no re-initialisation."""
    x = synth.custom(B=5, L=16, V=65536, K=1, dtype="bf16", n_peaks=8, peak=6.0, seed=15, cid=303)
    d = to_torch(x)
    ws = specv.Workspace(specv.verify_workspace_size(5, 16, 2, 65536))
    first = specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0, workspace=ws)
    first = [t.clone() for t in first]
    for it in range(6):
        if it % 3 == 2:
            specv.spec_verify_window_stats(d["target"], d["draft"], d["tokens"], 1.0, ws)
            again = specv.spec_verify_accept(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0, ws)
        else:
            again = specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0,
                                            workspace=ws)
        assert torch.equal(first[0], again[0]) and torch.equal(first[1], again[1]), it
    vl = torch.tensor([3, 0, 16, 7, 1], dtype=torch.int32, device="cuda")
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, verify_len=vl.cpu().numpy(), diag=True)
    for _ in range(3):
        acc, out = specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0,
                                           verify_len=vl, workspace=ws)
        check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl.cpu().numpy())
    assert ws.status() == 0


def test_scalar_path_odd_vocab():
    for dtype, K in (("bf16", 1), ("f32", 2)):
        x = synth.custom(B=3, L=5, V=1001, K=K, dtype=dtype, n_peaks=3, peak=4.0, seed=16, cid=304)
        ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.3, mix_w=x.mix_w, diag=True)
        d = to_torch(x)
        if K == 1:
            acc, out = specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.3)
        else:
            acc, out = specv.spec_verify_mixture(d["target"], d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], 1.3)
        check_verify(_cpu(acc), _cpu(out), ref)


def test_zero_length_block():
    x = synth.custom(B=3, L=0, V=2048, K=1, dtype="bf16", seed=17, cid=305)
    ref = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, diag=True)
    d = to_torch(x)
    acc, out = specv.spec_verify_block(d["target"], d["draft"], d["tokens"], d["u"], d["g"], 1.0)
    check_verify(_cpu(acc), _cpu(out), ref)


# ---------------------------------------------------------------------- DVL

@pytest.mark.parametrize("B,L,budget", [(1, 4, 1), (3, 4, 7), (32, 16, 272), (64, 16, 544), (16, 32, 300),
                                        (7, 5, 100), (200, 16, 1700), (512, 32, 8000), (4096, 4, 9000),
                                        (9, 3, 9), (6, 4, 1000), (5, 0, 5), (4096, 1, 4097)])
def test_dvl_parity(B, L, budget):
    rng = np.random.default_rng(B * 1000 + L)
    s = rng.beta(6.0, 2.0, size=(B, L)).astype(np.float32)
    if B % 2:
        s[:, ::3] = 0.5                            # many equal products: tie-break by (b, i)
    ref = oracle.dvl_allocate(s, budget)
    vl, off, sm = specv.dvl_allocate_pack(torch.from_numpy(s).cuda(), budget)
    np.testing.assert_array_equal(_cpu(vl), ref["verify_len"])
    np.testing.assert_array_equal(_cpu(off), ref["offsets"])
    np.testing.assert_array_equal(_cpu(sm), ref["slot_map"])


@pytest.mark.parametrize("case", ["signed_zeros", "all_equal", "coarse_ties", "unsorted"])
def test_dvl_ties_zeros_and_unsorted_rows(case):
    """The order (P desc, b asc, i asc) decides every tie, -0 and +0 are
    equal products, and rows whose scores are not sorted still get the
    oracle's counts (the selection is then not a prefix of the row)."""
    rng = np.random.default_rng(7)
    B, L = 48, 12
    if case == "signed_zeros":
        s = rng.choice(np.float32([0.0, -0.0, 0.5, 1.0]), size=(B, L)).astype(np.float32)
        s = np.where(np.arange(L)[None, :] < 3, np.float32(1.0), s)
    elif case == "all_equal":
        s = np.full((B, L), 0.75, np.float32)
    elif case == "coarse_ties":
        s = -np.sort(-(np.round(rng.beta(6.0, 2.0, size=(B, L)) * 4) / 4), axis=1).astype(np.float32)
    else:
        s = rng.beta(6.0, 2.0, size=(B, L)).astype(np.float32)
    for budget in (B, B + 1, B * (L + 1) // 2, B * (L + 1) - 1, B * (L + 1) + 7):
        ref = oracle.dvl_allocate(s, budget)
        vl, off, sm = specv.dvl_allocate_pack(torch.from_numpy(s).cuda(), budget)
        np.testing.assert_array_equal(_cpu(vl), ref["verify_len"])
        np.testing.assert_array_equal(_cpu(off), ref["offsets"])
        np.testing.assert_array_equal(_cpu(sm), ref["slot_map"])


def test_dvl_misaligned_scores_take_the_staged_load():
    """Scores whose rows are not 16-byte aligned (a view 4 bytes into an
    allocation) are staged through shared memory instead of loaded as
    vectors; the allocation is the same."""
    rng = np.random.default_rng(11)
    B, L = 64, 16
    s = -np.sort(-rng.beta(6.0, 2.0, size=(B, L)), axis=1).astype(np.float32)
    flat = torch.zeros(B * L + 1, dtype=torch.float32, device="cuda")
    flat[1:] = torch.from_numpy(s.reshape(-1)).cuda()
    view = flat[1:].view(B, L)
    assert view.data_ptr() % 16 != 0
    for budget in (B, B * (L + 1) // 2, B * (L + 1)):
        ref = oracle.dvl_allocate(s, budget)
        vl, off, sm = specv.dvl_allocate_pack(view, budget)
        np.testing.assert_array_equal(_cpu(vl), ref["verify_len"])
        np.testing.assert_array_equal(_cpu(off), ref["offsets"])
        np.testing.assert_array_equal(_cpu(sm), ref["slot_map"])


def test_dvl_flags_bad_scores():
    s = torch.full((4, 4), 0.5, device="cuda")
    s[2, 1] = 1.5
    ws = specv.Workspace(specv.dvl_workspace_size(4))
    specv.dvl_allocate_pack(s, 8, workspace=ws)
    assert ws.status() & specv.DEV_SCORES
