"""The multi-rank path on CPU (gloo, world size 2): request sharding and the
max-over-ranks timing reduction. Verification itself needs no exchange, so
the union of the ranks' results equals one verification of the whole batch
(checked with the oracle, the only CPU implementation)."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from speculative_decoding_block_spec_b200.dist import shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import oracle
    from speculative_decoding_block_spec_b200 import synth
    from speculative_decoding_block_spec_b200.dist import max_over_ranks, shard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x = synth.custom(B=7, L=6, V=256, K=2, dtype="bf16", n_peaks=3, peak=4.0, seed=3, cid=400)
    sl = shard(x.w.B, rank, world)
    r = oracle.verify(x.target[sl], x.draft[sl], x.tokens[sl], x.u[sl], x.g[sl], 1.0, mix_w=x.mix_w[sl])
    np.save(os.path.join(out_dir, "acc%d.npy" % rank), r["accept_len"])
    np.save(os.path.join(out_dir, "out%d.npy" % rank), r["out_tokens"])
    m = max_over_ranks(10.0 * (rank + 1))
    np.save(os.path.join(out_dir, "max%d.npy" % rank), np.array([m]))
    dist.barrier()
    dist.destroy_process_group()


def test_shard_covers_batch():
    for n in (1, 7, 8, 64):
        for world in (1, 2, 3, 8):
            sl = [shard(n, r, world) for r in range(world)]
            idx = [i for s in sl for i in range(n)[s]]
            assert idx == list(range(n))


def test_two_ranks_gloo(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    import oracle
    from speculative_decoding_block_spec_b200 import synth
    x = synth.custom(B=7, L=6, V=256, K=2, dtype="bf16", n_peaks=3, peak=4.0, seed=3, cid=400)
    whole = oracle.verify(x.target, x.draft, x.tokens, x.u, x.g, 1.0, mix_w=x.mix_w)
    acc = np.concatenate([np.load(tmp_path / ("acc%d.npy" % r)) for r in range(world)])
    out = np.concatenate([np.load(tmp_path / ("out%d.npy" % r)) for r in range(world)])
    np.testing.assert_array_equal(acc, whole["accept_len"])
    np.testing.assert_array_equal(out, whole["out_tokens"])
    for r in range(world):
        assert float(np.load(tmp_path / ("max%d.npy" % r))[0]) == 20.0
