"""The head-sharded mixer on one GPU: the shards of a 2- and a 4-way split run
one after another (no rank waits on another), and their partial deltas are
summed on the device the way the all-reduce of dist.head_sharded_forward sums
them.  Against the whole mixer and the oracle:
* each shard's selection equals the whole run's selection of its heads, bit for
  bit, and the oracle's;
* the summed delta is within the batch tolerances of the oracle's delta: fp32
  1e-5 absolute; bf16 2e-2 x RMS beyond the storage rounding, which here is
  that of each partial delta (up to 2^-8 of its magnitude, summed over the
  shards) instead of one rounding of delta;
* fp32: within 1e-5 of the whole mixer's delta (only the order of the sum over
  heads differs).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_parity import BF16_UNIT_ROUNDOFF, TOL_BF16_REL_RMS, assert_close, to_dev, to_np
from learned_product_hash_proj_b200 import dist, mono, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_product_hash_proj_b200 import build
    build.build()


def _cfg(dtype):
    return synth.Config(B=2, S=512, W=128, H=4, d=64, Bs=32, L=2, R=2, E=5, M=2, C=8, T=4, cap=3, dtype=dtype)


def _run(cfg, params):
    plan = mono.Plan(cfg)
    ws = plan.workspace()
    delta = torch.empty((cfg.B, cfg.S, cfg.W), dtype=plan.dtype, device="cuda")
    mono.forward(plan, params["x"], params["Wq"], params["Wk"], params["Wv"], params["Wo"], params["codebooks"],
                 delta, ws)
    torch.cuda.synchronize()
    return delta, to_np(plan.region(ws, "sel")).copy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("world", [2, 4])
def test_head_shards_sum_to_the_mixer(dtype, world):
    cfg = _cfg(dtype)
    inp = synth.make_inputs(cfg, 5)
    dev = {k: to_dev(v, dtype) for k, v in inp.items() if k != "codebooks"}
    dev["codebooks"] = torch.from_numpy(inp["codebooks"]).cuda().contiguous()
    whole, whole_sel = _run(cfg, dev)
    total = torch.zeros((cfg.B, cfg.S, cfg.W), dtype=torch.float32, device="cuda")
    abs_parts = torch.zeros_like(total)
    for r in range(world):
        part, sel = _run(dist.shard_config(cfg, r, world), dist.shard_weights(dev, cfg, r, world))
        h0, h1 = dist.head_range(cfg.H, r, world)
        np.testing.assert_array_equal(sel, whole_sel[:, h0:h1])
        total += part.float()
        abs_parts += part.float().abs()
    ref = oracle.forward(cfg, inp)
    np.testing.assert_array_equal(whole_sel, ref["sel"])
    got = to_np(total).astype(np.float64)
    if dtype == "f32":
        assert float(np.abs(got - to_np(whole).astype(np.float64)).max()) <= 1e-5
        assert_close(got, ref["delta"], dtype, f"delta summed over {world} head shards")
        return
    d = np.asarray(ref["delta"], np.float64)
    rms = float(np.sqrt(np.mean(d * d)))
    excess = float((np.abs(got - d) - BF16_UNIT_ROUNDOFF * to_np(abs_parts).astype(np.float64)).max())
    assert excess <= TOL_BF16_REL_RMS * rms, f"{world} shards: excess {excess:.3e} > 2e-2 x RMS {rms:.3e}"


# ---------------------------------------------------------------------------
# output projection fused with the reduce-scatter: each shard's GEMM stores its
# fp32 rows into the owners' staging buffers (here all on one GPU, the shards
# run one after another, nothing waits on another), then each owner sums its
# staged partials in rank order and rounds once.
# ---------------------------------------------------------------------------
def _fused_cfg():
    return synth.Config(B=2, S=512, W=256, H=8, d=64, Bs=64, L=2, R=2, E=5, M=2, C=8, T=4, cap=3, dtype="bf16")


@pytest.mark.parametrize("world", [2, 4])
def test_fused_scatter_reduce_is_one_rounding_of_the_fp32_sum(world):
    cfg = _fused_cfg()
    inp = synth.make_inputs(cfg, 6)
    dev = {k: to_dev(v, "bf16") for k, v in inp.items() if k != "codebooks"}
    dev["codebooks"] = torch.from_numpy(inp["codebooks"]).cuda().contiguous()
    rows = dist.stage_rows(cfg, world)
    stages = [torch.full((world, rows, cfg.W), float("nan"), dtype=torch.float32, device="cuda")
              for _ in range(world)]
    keep, Os = [], []
    for r in range(world):
        plan = mono.Plan(dist.shard_config(cfg, r, world))
        sh = dist.shard_weights(dev, cfg, r, world)
        ws = plan.workspace()
        Q, K, V, sel, O = (plan.region(ws, k) for k in ("Q", "K", "V", "sel", "O"))
        mono.project(plan, dev["x"], sh["Wq"], sh["Wk"], sh["Wv"], Q, K, V, ws)
        mono.route(plan, Q, K, sh["codebooks"], sel, ws)
        mono.attend(plan, Q, K, V, sel, O, ws)
        mono.out_project_scatter(plan, O, sh["Wo"], stages, r, ws)
        keep.append((plan, ws, sh))
        Os.append(O)
    delta = torch.empty((cfg.B, cfg.S, cfg.W), dtype=torch.bfloat16, device="cuda")
    flat = delta.view(-1, cfg.W)
    for c in range(world):
        mono.stage_reduce(keep[c][0], stages[c], world, flat[dist.chunk_of(cfg, world, c)])
    torch.cuda.synchronize()
    # every slot holds the fp32 product of its shard's rows (against fp64 on the same bf16 operands)
    for c in range(world):
        for r in range(world):
            Of = Os[r].view(-1, Os[r].shape[-1])[dist.chunk_of(cfg, world, c)].double()
            want = Of @ keep[r][2]["Wo"].double().T
            got = stages[c][r].double()
            assert torch.isfinite(got).all()
            assert (got - want).abs().max().item() <= 1e-4 * want.abs().max().item()
    # each chunk is the rank-order fp32 sum of its slots, rounded once
    for c in range(world):
        acc = stages[c][0].clone()
        for r in range(1, world):
            acc = acc + stages[c][r]
        assert torch.equal(flat[dist.chunk_of(cfg, world, c)], acc.to(torch.bfloat16))
    # and the whole delta is within the single-rounding tolerance of the oracle's output projection of the
    # shards' own O (heads concatenated in rank order), as the batch parity checks that stage
    O_full = torch.cat(Os, dim=-1)
    ref = oracle.out_project(cfg, to_np(O_full).astype(np.float64), inp["Wo"])
    assert_close(to_np(delta), ref, "bf16", f"fused reduce-scatter over {world} shards")


def test_fused_head_sharded_forward_on_one_rank():
    cfg = _fused_cfg()
    inp = synth.make_inputs(cfg, 7)
    dev = {k: to_dev(v, "bf16") for k, v in inp.items() if k != "codebooks"}
    dev["codebooks"] = torch.from_numpy(inp["codebooks"]).cuda().contiguous()
    plan = mono.Plan(cfg)
    ws = plan.workspace()
    stage, _ = dist.alloc_stage(cfg, 1, "cuda")
    delta = torch.empty((cfg.B, cfg.S, cfg.W), dtype=torch.bfloat16, device="cuda")
    dist.head_sharded_forward_fused(plan, dev["x"], dev, delta, ws, stage, [stage], 0, 1)
    torch.cuda.synchronize()
    ref = oracle.forward(cfg, inp)
    np.testing.assert_array_equal(to_np(plan.region(ws, "sel")), ref["sel"])
    assert_close(to_np(delta), ref["delta"], "bf16", "fused head-sharded forward, one rank")
