"""GPU parity of the backward pass for a fixed selection against the backward oracle.

* mono_attend_backward on the GPU's own stored Q/K/V and selection: the oracle
  (float64, autograd on the dense masked attention) gets the same values, so
  the only difference is fp32 arithmetic: max |err| <= 2e-4 x RMS(ref).
* mono_backward (projection, RoPE, attention, output projection) on the stored
  inputs, against the oracle that stores Q, K, V and O in the storage type
  between stages as the forward pass does (rounding with derivative 1):
  max |err| <= 1e-4 x RMS(ref) for fp32.  For bf16 the forward attention forms
  O with bf16 probabilities on the tensor cores, which is what the batch
  tolerance for O (2e-2 x RMS) covers, and dWo = ddelta^T O inherits it: the
  bf16 bound is that same 2e-2 x RMS.  The bf16 projection gradients run on
  the tensor cores with the fp32 gradients before the projections split into
  two bf16 terms (16 significant bits).  Rounding them to one bf16 term would
  alone cost up to 2.2e-2 x RMS in dx at these sizes (a float64 emulation of
  that rounding), which is why they are split.
"""
import numpy as np
import pytest
import torch

from gpu_parity import Run, to_np
from learned_product_hash_proj_b200 import mono, synth
from oracle import backward as bwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_product_hash_proj_b200 import build
    build.build()


def small(**kw):
    base = dict(B=2, S=256, W=128, H=2, d=64, Bs=32, L=2, R=2, E=5, M=2, C=8, T=4, cap=3, dtype="f32", x="normal")
    base.update(kw)
    return synth.Config(**base)


CASES = {
    "f32": dict(),
    "bf16": dict(dtype="bf16"),
    "d128_bf16": dict(d=128, Bs=64, C=16, cap=4, dtype="bf16"),
    "M4_L1_R4": dict(M=4, C=4, T=8, E=8, R=4, L=1, cap=2),
    "local_only": dict(R=0),
    "Bs96": dict(S=384, Bs=96, cap=2),
}


def close(got, ref, rel, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.abs(got - ref).max())
    import gpu_parity
    gpu_parity.PARITY_LOG.append(f"backward {what}: max |err| / RMS = {err / max(rms, 1e-300):.3e} (bound {rel})")
    assert err <= rel * rms + 1e-7, f"{what}: max |err| {err:.3e} > {rel} x RMS {rms:.3e}"


@pytest.mark.parametrize("name", list(CASES))
def test_attend_backward_matches_oracle(name):
    cfg = small(**CASES[name])
    run = Run(cfg, seed=6).run_stages()
    rng = np.random.default_rng(7)
    dO = torch.from_numpy(rng.standard_normal((cfg.B, cfg.S, cfg.H * cfg.d)).astype(np.float32)).cuda()
    dQ, dK, dV = (torch.empty((cfg.B, cfg.H, cfg.S, cfg.d), dtype=torch.float32, device="cuda") for _ in range(3))
    bws = mono.backward_workspace(run.plan)
    mono.attend_backward(run.plan, run.Q, run.K, run.V, run.sel, dO, dQ, dK, dV, bws)
    torch.cuda.synchronize()
    Q, K, V = (to_np(a).astype(np.float64) for a in (run.Q, run.K, run.V))
    gq, gk, gv = bwd.attention_gradients(cfg, Q, K, V, to_np(run.sel), to_np(dO).astype(np.float64))
    for nm, got, ref in (("dQ", dQ, gq), ("dK", dK, gk), ("dV", dV, gv)):
        close(to_np(got), ref, 2e-4, f"attention {nm}")


FULL_CASES = {
    "f32": dict(),
    "bf16": dict(dtype="bf16"),
    # widths off the 128-wide tensor-core tiles: ragged tiles in every gradient GEMM, split K in dWq/dWk/dWv
    "bf16_ragged": dict(dtype="bf16", S=320, W=192, H=3),
    # a longer sequence: 64 blocks of 64, selections reaching far back
    "bf16_S4096": dict(dtype="bf16", B=1, S=4096, Bs=64, C=16, cap=8),
}


@pytest.mark.parametrize("name", list(FULL_CASES))
def test_backward_matches_oracle(name):
    cfg = small(**FULL_CASES[name])
    dtype = cfg.dtype
    run = Run(cfg, seed=8).run_stages()
    plan, d = run.plan, run.dev
    rng = np.random.default_rng(9)
    dd = synth.round_bf16(rng.standard_normal((cfg.B, cfg.S, cfg.W))) if dtype == "bf16" else \
        rng.standard_normal((cfg.B, cfg.S, cfg.W)).astype(np.float32)
    ddelta = torch.from_numpy(np.asarray(dd, np.float32)).to(plan.dtype).cuda().contiguous()
    hd = cfg.H * cfg.d
    f32 = dict(dtype=torch.float32, device="cuda")
    dx = torch.empty((cfg.B, cfg.S, cfg.W), **f32)
    dWq, dWk, dWv = (torch.empty((hd, cfg.W), **f32) for _ in range(3))
    dWo = torch.empty((cfg.W, hd), **f32)
    ws, bws = plan.workspace(), mono.backward_workspace(plan)
    mono.backward(plan, d["x"], d["Wq"], d["Wk"], d["Wv"], d["Wo"], run.sel, ddelta, dx, dWq, dWk, dWv, dWo, ws, bws)
    torch.cuda.synchronize()
    stored = {k: to_np(d[k]).astype(np.float64) for k in ("x", "Wq", "Wk", "Wv", "Wo")}
    ref = bwd.gradients(cfg, stored["x"], stored["Wq"], stored["Wk"], stored["Wv"], stored["Wo"], to_np(run.sel),
                        to_np(ddelta).astype(np.float64), storage=dtype)
    rel = 1e-4 if dtype == "f32" else 2e-2
    for nm, got in (("x", dx), ("Wq", dWq), ("Wk", dWk), ("Wv", dWv), ("Wo", dWo)):
        close(to_np(got), ref[nm], rel, f"d{nm}")


@pytest.mark.parametrize("name", ["f32", "bf16_S4096"])
def test_backward_is_bit_reproducible(name):
    # Every sum of the backward runs in a fixed order (block lists sorted, the remote blocks' dQ parts summed in
    # slot order, split-K partial tiles summed in range order): two calls give the same bits.  bf16_S4096 takes
    # the tensor-core attention gradients, f32 the SIMT ones; both split K in the weight gradients.
    cfg = small(**FULL_CASES[name])
    run = Run(cfg, seed=8).run_stages()
    plan, d = run.plan, run.dev
    rng = np.random.default_rng(9)
    dd = rng.standard_normal((cfg.B, cfg.S, cfg.W)).astype(np.float32)
    if cfg.dtype == "bf16":
        dd = synth.round_bf16(dd)
    ddelta = torch.from_numpy(np.asarray(dd, np.float32)).to(plan.dtype).cuda().contiguous()
    hd = cfg.H * cfg.d
    f32 = dict(dtype=torch.float32, device="cuda")
    outs = []
    for _ in range(2):
        dx = torch.empty((cfg.B, cfg.S, cfg.W), **f32)
        dWq, dWk, dWv = (torch.empty((hd, cfg.W), **f32) for _ in range(3))
        dWo = torch.empty((cfg.W, hd), **f32)
        ws, bws = plan.workspace(), mono.backward_workspace(plan)
        mono.backward(plan, d["x"], d["Wq"], d["Wk"], d["Wv"], d["Wo"], run.sel, ddelta, dx, dWq, dWk, dWv, dWo, ws,
                      bws)
        torch.cuda.synchronize()
        outs.append((dx, dWq, dWk, dWv, dWo))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
