"""GPU parity: the CUDA library through its C-ABI against the oracle.

Routing outputs must be bit-exact; attention and projections must be within
1e-5 max abs (fp32 storage) or 2e-2 x RMS (bf16 storage).  Small workloads are
compared element by element on every output; the full-size workloads (run in
the launch configuration the benchmark times) on sampled outputs the oracle
computes one by one, with the integer routing tables compared in full.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_parity import (Run, check_attention, check_fp64_rule, check_out_projection, check_projection, check_routing,
                        check_routing_slices, check_walk_queries, log_routing, sample_queries, sample_tokens,
                        to_np)
from learned_product_hash_proj_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_product_hash_proj_b200 import build
    build.build()


def small(**kw):
    base = dict(B=2, S=1056, W=128, H=3, d=64, Bs=32, L=2, R=2, E=5, M=2, C=8, T=4, cap=3, dtype="f32", x="normal")
    base.update(kw)
    return synth.Config(**base)


def full_check(run: Run):
    run.run_stages()
    check_projection(run)
    info = check_routing(run)
    info.update(check_fp64_rule(run))
    log_routing(run, info)
    check_attention(run)
    check_out_projection(run)
    delta_fwd = run.run_forward()
    # the whole-mixer entry point runs the same deterministic kernels
    assert torch.equal(delta_fwd, run.delta)
    return info


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_ragged_workload(dtype):
    # 33 blocks of 32, 2112 token rows: ragged against every kernel tile
    info = full_check(Run(small(dtype=dtype), seed=1))
    assert info["overflow"] > 0


@pytest.mark.parametrize("d", [64, 128])
def test_head_dims(d):
    full_check(Run(small(d=d, H=2, S=512, Bs=64, C=16, cap=4, dtype="bf16"), seed=2))


def test_pr1_reference_workload():
    full_check(Run(synth.config("pr1"), seed=0))


def test_recall_shape_reduced():
    full_check(Run(synth.config("recall", B=2, S=2048), seed=0))


def test_forced_blocks_match():
    run = Run(small(S=1024, dtype="bf16", cap=6), seed=3, forced_frac=0.5)
    full_check(run)
    assert run.stats["forced_ignored"] > 0


def test_local_only_budget():
    full_check(Run(small(R=0, E=0, S=512), seed=4))


def test_zero_input_ties():
    cfg = small(S=512, x="zeros", dtype="bf16")
    run = Run(cfg, seed=5)
    full_check(run)
    assert (run.route_ws["addr"] == 0).all()


def test_duplicate_codewords_ties():
    cfg = small(S=1024, C=8, M=2, dtype="f32")
    inp = synth.make_inputs(cfg, seed=6)
    inp["codebooks"][:, 0, 5] = inp["codebooks"][:, 0, 1]
    inp["codebooks"][:, 1, 2] = inp["codebooks"][:, 1, 7]
    full_check(Run(cfg, seed=6, inputs=inp))


def test_four_subspaces_probe():
    # M=4 exercises the staged exact top-T with middle stages
    full_check(Run(small(S=1024, M=4, C=4, T=8, E=8, R=4, cap=2, dtype="bf16"), seed=7))


def test_full_budget_is_dense_causal_attention():
    cfg = small(S=512, Bs=32, M=2, C=4, L=1, dtype="f32", H=2, B=1)
    nb = cfg.S // cfg.Bs
    cfg = cfg.with_(T=cfg.A, E=nb, R=nb, cap=nb)
    run = Run(cfg, seed=8)
    full_check(run)
    q, k, v = (t.float() for t in (run.Q, run.K, run.V))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    got = run.O.float().view(cfg.B, cfg.S, cfg.H, cfg.d).transpose(1, 2)
    assert (got - ref).abs().max().item() <= 1e-5


def test_empty_batch_is_a_no_op():
    from learned_product_hash_proj_b200 import mono
    for change in (dict(B=0), dict(S=0)):
        run = Run(small(**change), seed=0)
        d = run.dev
        mono.forward(run.plan, d["x"], d["Wq"], d["Wk"], d["Wv"], d["Wo"], d["codebooks"], run.delta, run.ws)
        torch.cuda.synchronize()
        assert mono.stats(run.plan, run.ws)["overflow_total"] == 0


# ---------------------------------------------------------------------------
# tensor-core attention path (bf16, Bs in {64, 128}): shapes, raggedness, budgets
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,Bs,L,R,S", [
    (64, 64, 2, 2, 832),      # 13 blocks: last query tile half full
    (128, 64, 2, 4, 1024),
    (64, 128, 2, 2, 1408),    # 11 blocks of 128
    (128, 128, 1, 3, 768),
    (64, 64, 3, 2, 960),      # widest local range: 256 keys
    (64, 64, 1, 2, 640),
])
def test_tensor_core_attention_shapes(d, Bs, L, R, S):
    cfg = small(d=d, Bs=Bs, L=L, R=R, E=max(5, R), S=S, H=2, C=8, cap=6, dtype="bf16")
    full_check(Run(cfg, seed=10 + d + Bs + L))


def test_tensor_core_attention_more_slices_than_one_launch_group():
    # 2 x 130 = 260 (b, h) slices: the attention runs as a launch pair over 256 slices, then one over 4
    full_check(Run(small(B=2, H=130, S=256, Bs=64, C=8, cap=3, dtype="bf16"), seed=23))


def test_tensor_core_attention_edge_cases():
    full_check(Run(small(S=640, Bs=64, R=0, E=0, dtype="bf16"), seed=20))           # local only
    full_check(Run(small(S=640, Bs=64, x="zeros", dtype="bf16"), seed=21))          # all ties
    run = Run(small(S=1024, Bs=64, dtype="bf16", cap=8), seed=22, forced_frac=0.5)  # forced blocks
    full_check(run)


@pytest.mark.parametrize("B,S,W,H,d", [(1, 832, 256, 2, 64), (2, 640, 384, 1, 128), (1, 1024, 128, 4, 64)])
def test_tensor_core_projections(B, S, W, H, d):
    # ragged token count (B*S not a multiple of the 128-row tile), several K and N
    cfg = small(B=B, S=S, W=W, H=H, d=d, Bs=64, C=8, cap=6, dtype="bf16")
    full_check(Run(cfg, seed=30 + W))


def test_simple_and_tensor_core_paths_agree():
    from learned_product_hash_proj_b200 import mono
    cfg = small(S=1024, Bs=64, C=16, cap=8, dtype="bf16")
    fast = Run(cfg, seed=23).run_stages()
    simple = Run(cfg, seed=23, flags=mono.MONO_FLAG_SIMPLE_KERNELS).run_stages()
    assert torch.equal(fast.sel, simple.sel)
    a, b = fast.O.float(), simple.O.float()
    rms = b.pow(2).mean().sqrt().item()
    assert ((a - b).abs() - 2.0 ** -7 * b.abs()).max().item() <= 2e-2 * rms


# ---------------------------------------------------------------------------
# full-size workloads: integer tables in full, sampled outputs
# ---------------------------------------------------------------------------
def sampled_check(name, n_rows=96, n_queries=1500, seed=0, slices=None, flags=0):
    """Full-size workload: integer tables in full; every query of `slices` ((b, h) pairs, default all) routed
    by both statements of the oracle (fp32 bit-exact, fp64 margin rule); sampled projection, attention and
    output rows; causality and order of every selection."""
    cfg = synth.config(name)
    run = Run(cfg, seed=seed, flags=flags).run_stages()
    rng = np.random.default_rng(123)
    rows = sample_tokens(cfg, n_rows, rng)
    qidx = sample_queries(cfg, n_queries, rng)
    check_projection(run, rows=rows)
    info = check_routing(run, qidx=qidx)
    if slices is None:
        slices = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
    info.update(check_routing_slices(run, slices))
    info["probe_walks"], info["walks_outside_slices_checked"] = check_walk_queries(run, slices)
    log_routing(run, info, f" ({len(slices)} of {cfg.B * cfg.H} slices, every query)")
    check_attention(run, qidx=qidx)
    check_out_projection(run, rows=rows)
    # properties that hold at any size, on every query
    sel = to_np(run.sel)
    t = np.arange(cfg.S)
    lim = (t // cfg.Bs - cfg.L)[None, None, :, None]
    valid = sel >= 0
    assert (sel[valid] <= np.broadcast_to(lim, sel.shape)[valid]).all()
    srt = np.sort(np.where(valid, sel, np.iinfo(np.int32).max), axis=-1)
    assert (np.where(valid, sel, np.iinfo(np.int32).max) == srt).all()
    return run, info


@pytest.mark.parametrize("name", ["scale4k", "scale8k", "scale16k", "scale32k"])
def test_scale_workloads(name):
    run, info = sampled_check(name)
    assert info["overflow"] == 0 or name == "scale4k"


def test_recall_full_size():
    sampled_check("recall", n_queries=800)


def test_long_context_full_size():
    sampled_check("long", n_rows=48, n_queries=600)


def test_skewed_batch_full_size():
    # the oracle sorts all 65536 addresses per query: four whole (b, h) slices, spread over the batch
    run, info = sampled_check("stress", n_rows=48, n_queries=400, slices=[(0, 0), (5, 3), (10, 9), (15, 15)])
    assert info["overflow"] > 0
    assert run.stats["overflow_total"] == info["overflow"]


# ---------------------------------------------------------------------------
# redirect-on-overflow (plan flag): lists, overflow, selections, attention
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,C", [("f32", 8), ("bf16", 4), ("bf16", 3)])
def test_redirect_on_overflow(dtype, C):
    from learned_product_hash_proj_b200 import mono
    # 33 blocks per (b, h) over C^2 addresses with cap 3: lists overflow; with C = 3 (27 slots) blocks drop too
    run = Run(small(dtype=dtype, C=C, T=4, cap=3), seed=40 + C, forced_frac=0.3, flags=mono.MONO_FLAG_REDIRECT)
    info = full_check(run)
    # some blocks sit in a list other than their own address's (the export is checked in full by full_check)
    ids, la, own = run.route_ws["post_ids"], run.route_ws["post_addr"], run.route_ws["addr"]
    listed = la < run.cfg.A
    assert (np.take_along_axis(own, ids, axis=-1)[listed] != la[listed]).any()
    assert (info["overflow"] > 0) == (C == 3)


def test_redirect_on_overflow_skewed_batch_full_size():
    from learned_product_hash_proj_b200 import mono
    # the batched skewed workload, whose drop-mode lists overflow: redirect keeps those blocks
    run, info = sampled_check("stress", n_rows=48, n_queries=400, slices=[(0, 0), (7, 11), (15, 15)],
                              flags=mono.MONO_FLAG_REDIRECT)
    assert info["overflow"] == 0


# ---------------------------------------------------------------------------
# the largest block count a plan accepts (8192 blocks): the posting kernels'
# shared memory then passes the default 48 KB (dense kernel: 64 KB of
# addresses and ranks).  Routing only, on seeded Q/K, against the oracle in full.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,C,T,redirect", [(2, 8, 4, False), (4, 16, 16, False), (4, 16, 16, True)])
def test_routing_at_the_largest_block_count(M, C, T, redirect):
    from gpu_parity import oracle_lists
    from learned_product_hash_proj_b200 import mono
    cfg = synth.Config(B=1, S=8192 * 32, W=64, H=1, d=64, Bs=32, L=2, R=2, E=5, M=M, C=C, T=T, cap=1,
                       dtype="bf16")
    rng = np.random.default_rng(40 + M)
    shape = (cfg.B, cfg.H, cfg.S, cfg.d)
    Qn = synth.round_bf16(rng.standard_normal(shape, dtype=np.float32))
    Kn = synth.round_bf16(rng.standard_normal(shape, dtype=np.float32) * 3.0)
    cb = synth.make_codebooks(cfg, 40 + M)
    plan = mono.Plan(cfg, flags=mono.MONO_FLAG_REDIRECT if redirect else 0)
    ws = plan.workspace()
    Q, K = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (Qn, Kn))
    sel = torch.empty((cfg.B, cfg.H, cfg.S, cfg.R), dtype=torch.int32, device="cuda")
    mono.route(plan, Q, K, torch.from_numpy(cb).cuda(), sel, ws)
    torch.cuda.synchronize()
    st = mono.stats(plan, ws)
    kbar, addr, _ = oracle.summary_assign(cfg, Kn, cb)
    np.testing.assert_array_equal(to_np(plan.region(ws, "addr")), addr, err_msg="addresses")
    laddr, ids, saddr, rank, ov = oracle_lists(cfg, addr, redirect)
    np.testing.assert_array_equal(to_np(plan.region(ws, "post_ids")), ids, err_msg="posting ids")
    np.testing.assert_array_equal(to_np(plan.region(ws, "post_addr")), saddr, err_msg="posting addresses")
    np.testing.assert_array_equal(to_np(plan.region(ws, "post_rank")), rank, err_msg="posting ranks")
    np.testing.assert_array_equal(to_np(plan.region(ws, "overflow")).astype(np.int64), ov, err_msg="overflow")
    assert st["overflow_total"] == int(ov.sum())
    assert (ov.sum() > 0) != redirect          # 8192 blocks fill 8192 of 65536 lists of one: nothing drops
    # every 7th query; the oracle sorts the whole grid per query, so the 65536-address grid gets 400
    qidx = np.arange(0, cfg.S, 7, dtype=np.int64) if cfg.A <= 4096 else \
        np.sort(rng.choice(cfg.S, 400, replace=False)).astype(np.int64)
    osel, *_ = oracle.route_queries(cfg, Qn, kbar, cb, laddr, qidx=qidx)
    np.testing.assert_array_equal(to_np(sel).reshape(-1, cfg.R)[qidx], osel, err_msg="sel")


@pytest.mark.parametrize("dtype,H", [("bf16", 2), ("bf16", 130), ("f32", 2)])
def test_attention_stages_one_at_a_time_equal_the_whole_call(dtype, H):
    # mono_attend_pairs, _remote and _local in turn give mono_attend's output bit for bit (with 2 x 130 slices,
    # more than one launch group of the remote and local kernels)
    from learned_product_hash_proj_b200 import mono
    run = Run(small(dtype=dtype, H=H, S=640 if H == 2 else 256, Bs=64, C=8, cap=4), seed=50).run_stages()
    O2 = torch.full_like(run.O, float("nan"))
    mono.attend_pairs(run.plan, run.sel, run.ws)
    mono.attend_remote(run.plan, run.Q, run.K, run.V, run.ws)
    mono.attend_local(run.plan, run.Q, run.K, run.V, run.sel, O2, run.ws)
    torch.cuda.synchronize()
    assert torch.equal(O2, run.O)
