"""GPU <-> oracle parity of top-p (nucleus) filtered verification, through the
C ABI (needs a B200).

Target sampling with temperature and top-p, target probabilities under the
same sampling filter ("DBLAST: Dependent Block Drafting for Stochastic
Speculative Decoding", Pith review, "What would settle it": T = 1.5, top-p
0.95; "Assumptions"): every target row and every draft category is filtered
to its nucleus. The oracle (oracle.verify(..., top_p=...)) decides; outputs
must match bit for bit under the low-margin rule of tests/parity_util.py,
which with top-p also exempts a request whose nucleus boundary lies within
1e-6 of top-p (the oracle's nucleus_margin diagnostic).

Drafted tokens: the seeded generator samples them from the unfiltered draft
rows, which a filtered drafter would not do; the tests here redraw them from
the filtered proposal (nucleus of the drafted category, Gumbel-max with the
test's own noise), and one test keeps the unfiltered tokens to exercise
tokens outside the nuclei (rejections, and requests without a posterior).
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_block_spec_b200 as specv
from speculative_decoding_block_spec_b200 import synth
from speculative_decoding_block_spec_b200.synth import bf16_bits_to_f32

from parity_util import check_verify, logits_to_torch, to_torch

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


def _values(a):
    return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a


def _nucleus_members(row, T, top_p):
    """Tokens of the nucleus of logit row `row` at temperature T (fp64): the
    shortest run, by probability descending then index ascending, whose mass
    reaches top_p."""
    z = row.astype(np.float64) / T
    p = np.exp(z - z.max())
    p /= p.sum()
    order = np.lexsort((np.arange(len(p)), -p))
    c = np.cumsum(p[order])
    n = int(np.searchsorted(c, top_p, side="left")) + 1
    return order[:min(n, len(p))]


def redraw_from_filtered(x, top_p, seed):
    """Draft tokens sampled from the filtered proposal: category z by
    Gumbel-max over log w (K > 1), then every position by Gumbel-max over the
    nucleus of branch z's row."""
    rng = np.random.default_rng(seed)
    w = x.w
    d = _values(x.draft)
    tokens = np.empty((w.B, w.L), np.int32)
    for b in range(w.B):
        zb = 0
        if w.K > 1:
            zb = int(np.argmax(np.log(x.mix_w[b].astype(np.float64)) + synth.gumbel(rng, w.K)))
        for i in range(w.L):
            row = d[b, i] if w.K == 1 else d[b, zb, i]
            mem = _nucleus_members(row, w.T, top_p)
            sc = row[mem].astype(np.float64) / w.T + synth.gumbel(rng, len(mem))
            tokens[b, i] = int(mem[np.argmax(sc)])
    x.tokens = tokens
    return x


def _verify(d, x, top_p, verify_len=None, workspace=None):
    vl = None if verify_len is None else torch.from_numpy(np.asarray(verify_len, np.int32)).cuda()
    if x.w.K == 1:
        return specv.spec_verify_block_top_p(d["target"], d["draft"], d["tokens"], d["u"], d["g"], x.w.T, top_p,
                                             verify_len=vl, workspace=workspace)
    return specv.spec_verify_mixture_top_p(d["target"], d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], x.w.T,
                                           top_p, verify_len=vl, workspace=workspace)


def _ref(x, top_p, verify_len=None):
    return oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, x.w.T, mix_w=x.mix_w, verify_len=verify_len,
                         n_threads=NT, diag=True, top_p=float(np.float32(top_p)))


def test_mixture_workload_at_t15_top_p_095():
    """The mixture workload (B=32, L=16, K=4, T=1.5) with top-p 0.95, drafts
    from the filtered proposal."""
    x = redraw_from_filtered(synth.make_inputs(synth.WORKLOADS[3]), 0.95, seed=3)
    ref = _ref(x, 0.95)
    assert (ref["flags"] & oracle.FLAG_NONFINITE) == 0
    acc, out = _verify(to_torch(x), x, 0.95)
    check_verify(_cpu(acc), _cpu(out), ref)


@pytest.mark.parametrize("top_p", [0.5, 0.9, 0.99])
def test_independent_drafts(top_p):
    """K = 1 (the block workload's recipe, B = 8, V = 151936) at several top-p."""
    x = redraw_from_filtered(synth.custom(B=8, L=16, V=151936, K=1, T=1.0, dtype="bf16", n_peaks=32, peak=8.0,
                                          draft_sigma=1.0, seed=int(top_p * 100), cid=600 + int(top_p * 100)),
                             top_p, seed=int(top_p * 1000))
    vl = np.random.default_rng(int(top_p * 7)).integers(0, 17, size=8).astype(np.int32)
    ref = _ref(x, top_p, vl)
    acc, out = _verify(to_torch(x), x, top_p, verify_len=vl)
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


@pytest.mark.parametrize("K", [2, 3])
def test_mixture_ragged_lengths(K):
    x = redraw_from_filtered(synth.custom(B=10, L=12, V=32768, K=K, T=1.3, dtype="bf16", n_peaks=8, peak=5.0,
                                          draft_sigma=0.8, seed=K, cid=620 + K), 0.9, seed=K)
    vl = np.random.default_rng(K).integers(0, 13, size=10).astype(np.int32)
    ref = _ref(x, 0.9, vl)
    acc, out = _verify(to_torch(x), x, 0.9, verify_len=vl)
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


def test_unfiltered_drafts_leave_the_nuclei():
    """Tokens drafted from the unfiltered rows: some fall outside the target's
    nucleus (rejected) or outside every draft category's (accepted, then the
    request has no posterior and fails with accept_len = -1 on both sides)."""
    x = synth.custom(B=24, L=16, V=16384, K=2, T=1.5, dtype="bf16", n_peaks=0, draft_sigma=1.5, seed=9, cid=640)
    ref = _ref(x, 0.6)
    acc, out = _verify(to_torch(x), x, 0.6)
    check_verify(_cpu(acc), _cpu(out), ref)
    assert np.any(ref["accept_len"] >= 0)


@pytest.mark.parametrize("K", [1, 2])
def test_tiny_vocabulary_ties_across_the_boundary(K):
    """V = 7 fp32 rows (the scalar path) with tied probabilities straddling the
    nucleus boundary, several top-p; the tie cut goes by token index."""
    rng = np.random.default_rng(70 + K)
    B, L, V, T = 40, 3, 7, 1.3
    base = (rng.standard_normal((B, L + 1, V)) * 1.5).astype(np.float32)
    base[::2, :, 4] = base[::2, :, 1]
    base[1::2, :, 6] = base[1::2, :, 2]
    draft = np.repeat(base[:, None, :L], K, axis=1) + (rng.standard_normal((B, K, L, V)) * 0.5).astype(np.float32)
    draft[::3, :, :, 3] = draft[::3, :, :, 5]
    w = synth.Workload(650 + K, "ties", B, L, V, K, T, "f32", 1.0, 0, 0.0, 0.5)
    x = synth.Inputs(w, base, draft[:, 0].copy() if K == 1 else draft, np.zeros((B, L), np.int32),
                     rng.random((B, L), dtype=np.float32), synth.gumbel(rng, (B, L + 1, V)).astype(np.float32),
                     mix_w=None if K == 1 else np.full((B, K), 1.0 / K, np.float32))
    for top_p in (0.3, 0.55, 0.8, 0.95):
        xx = redraw_from_filtered(x, top_p, seed=int(top_p * 100) + K)
        ref = _ref(xx, top_p)
        acc, out = _verify(to_torch(xx), xx, top_p)
        check_verify(_cpu(acc), _cpu(out), ref)


def test_top_p_one_is_the_unfiltered_call():
    x = synth.custom(B=6, L=8, V=4096, K=2, T=1.2, dtype="bf16", n_peaks=4, peak=5.0, seed=5, cid=660)
    d = to_torch(x)
    a1, o1 = specv.spec_verify_mixture(d["target"], d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], 1.2)
    a2, o2 = specv.spec_verify_mixture_top_p(d["target"], d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], 1.2,
                                             1.0)
    assert torch.equal(a1, a2) and torch.equal(o1, o2)


def test_zero_length_blocks_draw_from_the_filtered_bonus_row():
    x = synth.custom(B=5, L=4, V=8192, K=1, T=1.0, dtype="bf16", n_peaks=8, peak=6.0, seed=6, cid=661)
    vl = np.zeros(5, np.int32)
    ref = _ref(x, 0.7, vl)
    acc, out = _verify(to_torch(x), x, 0.7, verify_len=vl)
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=vl)


def test_workspace_reuse_and_status():
    """One top-p workspace, several calls with changing top-p: self-resetting."""
    x = redraw_from_filtered(synth.custom(B=6, L=10, V=20000, K=3, T=1.1, dtype="bf16", n_peaks=6, peak=5.0,
                                          seed=7, cid=662), 0.8, seed=7)
    d = to_torch(x)
    ws = specv.Workspace(specv.verify_top_p_workspace_size(6, 10, 3, 20000))
    for top_p in (0.8, 0.5, 0.8, 1.0, 0.8):
        ref = _ref(x, top_p)
        acc, out = _verify(d, x, top_p, workspace=ws)
        check_verify(_cpu(acc), _cpu(out), ref)
    assert ws.status() & ~specv.DEV_NONFINITE == 0


def test_dvl_packed_rows_with_top_p():
    """Top-p on DVL-packed target rows (verify lengths and row offsets read on
    the device): the bonus row of request b is packed row offsets[b] + l_b."""
    x = synth.custom(B=16, L=12, V=32768, K=3, T=1.5, dtype="bf16", n_peaks=8, peak=4.0, draft_sigma=1.0,
                     budget=16 * 13 // 2, seed=13, cid=670)
    x = redraw_from_filtered(x, 0.95, seed=13)
    w = x.w
    rd = oracle.dvl_allocate(x.scores, w.budget)
    packed_ref = oracle.pack(x.target, rd["verify_len"], rd["offsets"], w.budget)
    ref = oracle.verify(packed_ref, x.draft, x.tokens, x.u, x.g, w.T, mix_w=x.mix_w, verify_len=rd["verify_len"],
                        target_row_off=rd["offsets"][:w.B], n_threads=NT, diag=True, top_p=float(np.float32(0.95)))
    d = to_torch(x)
    packed = torch.zeros((w.budget, w.V), dtype=d["target"].dtype, device="cuda")
    vl, off, _ = specv.dvl_allocate_pack(d["scores"], w.budget, dense_target=d["target"], packed_target=packed)
    acc, out = specv.spec_verify_mixture_top_p(packed, d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], w.T,
                                               0.95, verify_len=vl, target_row_off=off[:w.B])
    check_verify(_cpu(acc), _cpu(out), ref, verify_len=rd["verify_len"])


def test_graph_replay_with_top_p_across_allocations():
    """One captured graph (DVL allocation, packing, filtered verification)
    replayed with new survival scores and uniforms in the same buffers."""
    B, L, V, K, T, top_p = 12, 10, 16384, 2, 1.3, 0.9
    budget = B * (L + 1) // 2
    x = redraw_from_filtered(synth.custom(B=B, L=L, V=V, K=K, T=T, dtype="bf16", n_peaks=6, peak=5.0,
                                          draft_sigma=0.8, budget=budget, seed=14, cid=671), top_p, seed=14)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        d = to_torch(x)
        packed = torch.zeros((budget, V), dtype=d["target"].dtype, device="cuda")
        dvl_ws = specv.Workspace(specv.dvl_workspace_size(B))
        ver_ws = specv.Workspace(specv.verify_top_p_workspace_size(B, L, K, V))
        dvl_out = (torch.empty(B, dtype=torch.int32, device="cuda"), torch.empty(B + 1, dtype=torch.int32, device="cuda"),
                   torch.empty(budget, dtype=torch.int32, device="cuda"))
        ver_out = (torch.empty(B, dtype=torch.int32, device="cuda"),
                   torch.empty((B, L + 1), dtype=torch.int32, device="cuda"))

        def step():
            vl, off, _ = specv.dvl_allocate_pack(d["scores"], budget, dense_target=d["target"], packed_target=packed,
                                                 workspace=dvl_ws, out=dvl_out)
            specv.spec_verify_mixture_top_p(packed, d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], T, top_p,
                                            verify_len=vl, target_row_off=off[:B], workspace=ver_ws, out=ver_out)

        step()
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            step()
        s.synchronize()
    rng = np.random.default_rng(77)
    seen = set()
    for trial in range(4):
        scores = -np.sort(-rng.beta(6.0 - trial, 2.0 + trial, size=(B, L)), axis=1).astype(np.float32)
        u = rng.random((B, L), dtype=np.float32)
        with torch.cuda.stream(s):
            d["scores"].copy_(torch.from_numpy(scores))
            d["u"].copy_(torch.from_numpy(u))
            graph.replay()
        s.synchronize()
        rd = oracle.dvl_allocate(scores, budget)
        np.testing.assert_array_equal(dvl_out[0].cpu().numpy(), rd["verify_len"])
        pk = oracle.pack(x.target, rd["verify_len"], rd["offsets"], budget)
        ref = oracle.verify(pk, x.draft, x.tokens, u, x.g, T, mix_w=x.mix_w, verify_len=rd["verify_len"],
                            target_row_off=rd["offsets"][:B], n_threads=NT, diag=True, top_p=float(np.float32(top_p)))
        check_verify(ver_out[0].cpu().numpy(), ver_out[1].cpu().numpy(), ref, verify_len=rd["verify_len"])
        seen.add(tuple(rd["verify_len"]))
    assert len(seen) > 1
    assert ver_ws.status() & ~specv.DEV_NONFINITE == 0


def _edge_rows_inputs(V, seed):
    """Requests whose rows take every branch of the windowed nucleus kernel
    (bf16 rows of 16-byte vectors, V >= 4096): constant rows (one tie value),
    signed zeros, half the vocabulary at -inf, rows far below zero, a handful
    of peaks a strided sample misses (the cut lies above the sampled window),
    a very wide spread, and rows holding +inf or a NaN (handed to the exact
    kernel, the request flagged)."""
    x = synth.custom(B=9, L=3, V=V, K=2, T=1.0, dtype="bf16", n_peaks=0, draft_sigma=1.0, seed=seed, cid=700)
    rng = np.random.default_rng(seed)
    t = bf16_bits_to_f32(x.target).copy()
    d = bf16_bits_to_f32(x.draft).copy()
    t[0] = 0.0
    d[0] = 1.0
    t[1] = 0.0
    t[1, :, ::3] = -0.0
    d[1, :, :, 1::2] = -0.0
    t[2, :, : V // 2] = -np.inf
    d[2, :, :, V // 2:] = -np.inf
    t[3] -= 50.0
    d[3] -= 80.0
    for i in range(t.shape[1]):  # four peaks between the sampled units
        t[4, i, rng.choice(V, 4, replace=False) | 1] = 30.0
    t[5] *= 8.0
    d[5] *= 6.0
    t[6, 1, 17] = np.inf
    d[7, 1, 2, 5] = np.nan
    t[8] = np.round(t[8] * 4) / 4  # few distinct values, many ties
    x.target = synth.f32_to_bf16_bits(t)
    x.draft = synth.f32_to_bf16_bits(d)
    return x


@pytest.mark.parametrize("top_p", [0.3, 0.9, 0.97])
def test_windowed_nucleus_edge_rows(top_p):
    x = _edge_rows_inputs(8192, seed=int(top_p * 100))
    ref = _ref(x, top_p)
    acc, out = _verify(to_torch(x), x, top_p)
    acc, out = _cpu(acc), _cpu(out)
    check_verify(acc, out, ref)
    assert acc[6] == -1 and acc[7] == -1  # the non-finite rows flag their requests
    assert (acc[[0, 1, 3, 4, 5, 8]] >= 0).all()


@pytest.mark.parametrize("dtype,V", [("f32", 32768), ("bf16", 20001)])
def test_exact_nucleus_kernel_rows(dtype, V):
    """Rows the windowed kernel does not take (fp32 rows; bf16 rows whose
    length is not a whole number of 16-byte vectors) go to the exact kernel
    alone: its fp32 radix descent and its scalar bf16 path, at sizes that span
    many digits and a ragged tail."""
    x = redraw_from_filtered(synth.custom(B=6, L=8, V=V, K=2, T=1.2, dtype=dtype, n_peaks=6, peak=5.0,
                                          draft_sigma=1.0, seed=V % 97, cid=710 + (dtype == "f32")), 0.9, seed=41)
    ref = _ref(x, 0.9)
    acc, out = _verify(to_torch(x), x, 0.9)
    check_verify(_cpu(acc), _cpu(out), ref)
