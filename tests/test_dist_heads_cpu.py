"""The head-sharded mixer's host logic on world_size-2 gloo ranks, CPU only.

Each rank takes its heads' slice of the parameters (shard_weights), runs the
oracle's whole mixer on that slice (shard_config), and the ranks sum their
partial deltas with reduce_partial_delta.  Against the oracle on all heads:
* the sum is the whole mixer's delta (the output projection is a sum over
  heads; fp64 partial sums, so equal to rounding);
* each rank's selection is the whole run's selection of its heads, bit for
  bit (routing, posting lists and probes are per head);
* a wrong slice (a transposed Wo slice, the wrong codebook heads) would break
  the first or the second.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _cfg():
    from learned_product_hash_proj_b200 import synth
    return synth.Config(B=1, S=96, W=16, H=4, d=8, Bs=8, L=2, R=2, E=3, M=2, C=4, T=3, cap=2, dtype="f32")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch

    import oracle
    from learned_product_hash_proj_b200 import dist, synth
    r, _, w = dist.init("gloo", timeout_s=60)
    cfg = _cfg()
    inp = synth.make_inputs(cfg, 3)
    shard = dist.shard_weights(inp, cfg, r, w)
    part = oracle.forward(dist.shard_config(cfg, r, w), shard)
    delta = torch.from_numpy(np.ascontiguousarray(part["delta"], dtype=np.float64))
    dist.reduce_partial_delta(delta)
    dist.barrier()
    dist.finalize()
    q.put((r, delta.numpy(), np.asarray(part["sel"])))


def test_two_rank_head_sharded_mixer():
    import oracle
    from learned_product_hash_proj_b200 import dist, synth
    cfg = _cfg()
    full = oracle.forward(cfg, synth.make_inputs(cfg, 3))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=180) for _ in procs), key=lambda o: o[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = np.asarray(full["delta"], np.float64)
    for r, delta, sel in out:
        np.testing.assert_allclose(delta, ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))
        h0, h1 = dist.head_range(cfg.H, r, 2)
        np.testing.assert_array_equal(sel, np.asarray(full["sel"])[:, h0:h1])


def test_shard_slices_and_errors():
    from learned_product_hash_proj_b200 import dist, synth
    cfg = _cfg()
    inp = synth.make_inputs(cfg, 4)
    s1 = dist.shard_weights(inp, cfg, 1, 4)       # heads [1, 2)
    d = cfg.d
    np.testing.assert_array_equal(s1["Wq"], inp["Wq"][d:2 * d])
    np.testing.assert_array_equal(s1["Wo"], inp["Wo"][:, d:2 * d])
    np.testing.assert_array_equal(s1["codebooks"], inp["codebooks"][1:2])
    assert s1["Wo"].flags["C_CONTIGUOUS"] and s1["x"] is inp["x"]
    assert dist.shard_config(cfg, 3, 4).H == 1
    assert [dist.head_range(16, r, 8) for r in (0, 7)] == [(0, 2), (14, 16)]
    with pytest.raises(ValueError):
        dist.head_range(6, 0, 4)
    with pytest.raises(ValueError):
        dist.head_range(8, 4, 4)
    # no process group: the partial delta is the delta
    import torch
    t = torch.ones(3)
    assert dist.reduce_partial_delta(t) is t and float(t.sum()) == 3.0


def test_reduce_scatter_chunks_tile_the_rows():
    # the row chunks of the fused output-projection reduce-scatter cover the B*S rows once, in rank order
    from learned_product_hash_proj_b200 import dist as d
    from learned_product_hash_proj_b200 import synth
    cfg = synth.Config(B=2, S=96, W=16, H=4, d=8, Bs=8, L=1, R=2, E=3, M=2, C=4, T=3, cap=2, dtype="f32")
    for world in (1, 2, 3, 4):
        rows = d.stage_rows(cfg, world)
        got = np.concatenate([np.arange(cfg.B * cfg.S)[d.chunk_of(cfg, world, r)] for r in range(world)])
        np.testing.assert_array_equal(got, np.arange(cfg.B * cfg.S))
        assert rows * world == cfg.B * cfg.S
    with pytest.raises(ValueError):
        d.stage_rows(cfg, 5)
