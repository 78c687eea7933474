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
