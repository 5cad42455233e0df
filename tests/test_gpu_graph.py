"""One captured CUDA graph serves every allocation (fixed-address workspaces,
'DScale: Scaling Block-Diffusion Speculative Decoding with Adaptive
Verification', Abstract): DVL allocation + packing + mixture verification are
captured once, then replayed with new survival scores and noise written into
the same input buffers; each replay must match the oracle."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_block_spec_b200 as specv
from speculative_decoding_block_spec_b200 import synth

from parity_util import check_verify, to_torch

pytestmark = pytest.mark.gpu


def test_graph_replay_across_changing_allocations():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, L, V, K = 16, 16, 32768, 2
    budget = B * (L + 1) // 2
    x = synth.custom(B=B, L=L, V=V, K=K, T=1.2, dtype="bf16", n_peaks=8, peak=5.0, draft_sigma=0.8,
                     budget=budget, seed=21, cid=500)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        d = to_torch(x)
        packed = torch.zeros((budget, V), dtype=d["target"].dtype, device="cuda")
        dvl_ws = specv.Workspace(specv.dvl_workspace_size(B))
        ver_ws = specv.Workspace(specv.verify_workspace_size(B, L, K, V))
        dvl_out = (torch.empty(B, dtype=torch.int32, device="cuda"),
                   torch.empty(B + 1, dtype=torch.int32, device="cuda"),
                   torch.empty(budget, dtype=torch.int32, device="cuda"))
        ver_out = (torch.empty(B, dtype=torch.int32, device="cuda"),
                   torch.empty((B, L + 1), dtype=torch.int32, device="cuda"))

        def step():
            vl, off, _ = specv.dvl_allocate_pack(d["scores"], budget, dense_target=d["target"],
                                                 packed_target=packed, workspace=dvl_ws, out=dvl_out)
            specv.spec_verify_mixture(packed, d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], 1.2,
                                      verify_len=vl, target_row_off=off[:B], workspace=ver_ws, out=ver_out)

        step()
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            step()
        s.synchronize()

    rng = np.random.default_rng(99)
    seen = set()
    for trial in range(5):
        scores = -np.sort(-rng.beta(6.0 - trial, 2.0 + trial, size=(B, L)), axis=1).astype(np.float32)
        u = rng.random((B, L), dtype=np.float32)
        with torch.cuda.stream(s):
            d["scores"].copy_(torch.from_numpy(scores))
            d["u"].copy_(torch.from_numpy(u))
            graph.replay()
        s.synchronize()
        rd = oracle.dvl_allocate(scores, budget)
        np.testing.assert_array_equal(dvl_out[0].cpu().numpy(), rd["verify_len"])
        np.testing.assert_array_equal(dvl_out[1].cpu().numpy(), rd["offsets"])
        pk = oracle.pack(x.target, rd["verify_len"], rd["offsets"], budget)
        ref = oracle.verify(pk, x.draft, x.tokens, u, x.g, 1.2, mix_w=x.mix_w, verify_len=rd["verify_len"],
                            target_row_off=rd["offsets"][:B], n_threads=oracle.n_cores(), diag=True)
        check_verify(ver_out[0].cpu().numpy(), ver_out[1].cpu().numpy(), ref, verify_len=rd["verify_len"])
        seen.add(tuple(rd["verify_len"]))
    assert len(seen) > 1  # the allocation really changed between replays
    assert ver_ws.status() == 0 and dvl_ws.status() == 0
