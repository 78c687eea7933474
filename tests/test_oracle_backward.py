"""Pins of the backward oracle (oracle/backward.py) against things other than itself.

* its forward equals the C oracle's fp64 stages (projection + RoPE, selected-set
  attention, output projection) on the same selection -- two independent
  statements of the forward pass; with activations stored in fp32 or bf16
  between stages it equals the C oracle's forward, which stores them the same way;
* its gradients equal central finite differences (torch.autograd.gradcheck, fp64);
* a closed form: with one-token blocks, one local block and no remote budget each
  query attends to itself only, so O = V and dV = dO, dQ = dK = 0.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bwd
from learned_product_hash_proj_b200 import synth


def tiny(**kw):
    base = dict(B=1, S=64, W=16, H=2, d=8, Bs=8, L=2, R=2, E=3, M=2, C=4, T=3, cap=2, dtype="f32", x="normal")
    base.update(kw)
    return synth.Config(**base)


def routed(cfg, seed=0):
    inp = synth.make_inputs(cfg, seed)
    fw = oracle.forward(cfg, inp)
    return inp, fw["sel"]


@pytest.mark.parametrize("R", [0, 2])
def test_dense_forward_matches_the_c_oracle(R):
    cfg = tiny(R=R, E=max(R, 1))
    inp, sel = routed(cfg, seed=1)
    Q, K, V = oracle.project(cfg, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"])
    O = oracle.heads_to_tokens(oracle.attend(cfg, Q, K, V, sel))
    ref = oracle.out_project(cfg, O, inp["Wo"])
    t = {k: torch.tensor(np.asarray(inp[k], np.float64)) for k in ("x", "Wq", "Wk", "Wv", "Wo")}
    got = bwd.forward(cfg, t["x"], t["Wq"], t["Wk"], t["Wv"], t["Wo"], sel).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_stored_forward_matches_the_c_oracle_forward(dtype):
    # the C oracle's forward stores Q, K, V and O in the storage type between stages
    cfg = tiny(dtype=dtype)
    inp, sel = routed(cfg, seed=2)
    ref = oracle.forward(cfg, inp)["delta"]
    t = {k: torch.tensor(np.asarray(inp[k], np.float64)) for k in ("x", "Wq", "Wk", "Wv", "Wo")}
    got = bwd.forward(cfg, t["x"], t["Wq"], t["Wk"], t["Wv"], t["Wo"], sel, storage=dtype).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-10)


def test_gradients_match_finite_differences():
    cfg = tiny(B=1, S=12, W=6, H=2, d=4, Bs=3, L=1, R=1, E=2, M=2, C=2, T=2, cap=2)
    rng = np.random.default_rng(3)
    sel = np.full((cfg.B, cfg.H, cfg.S, cfg.R), -1, np.int32)
    for t in range(cfg.S):
        lim = t // cfg.Bs - cfg.L
        if lim >= 0:
            sel[0, :, t, 0] = rng.integers(0, lim + 1, size=cfg.H)
    args = [torch.tensor(rng.standard_normal(shape), dtype=torch.float64, requires_grad=True)
            for shape in ((cfg.B, cfg.S, cfg.W), (cfg.H * cfg.d, cfg.W), (cfg.H * cfg.d, cfg.W),
                          (cfg.H * cfg.d, cfg.W), (cfg.W, cfg.H * cfg.d))]
    f = lambda x, wq, wk, wv, wo: bwd.forward(cfg, x, wq, wk, wv, wo, sel)
    assert torch.autograd.gradcheck(f, args, eps=1e-6, atol=1e-6, rtol=1e-5)


def test_attention_gradients_match_finite_differences():
    cfg = tiny(B=1, S=12, H=1, d=4, Bs=3, L=2, R=1)
    rng = np.random.default_rng(4)
    sel = np.full((1, 1, cfg.S, 1), -1, np.int32)
    for t in range(cfg.S):
        if t // cfg.Bs - cfg.L >= 0:
            sel[0, 0, t, 0] = 0
    Q, K, V = (rng.standard_normal((1, 1, cfg.S, cfg.d)) for _ in range(3))
    dO = rng.standard_normal((1, cfg.S, cfg.d))
    gq, gk, gv = bwd.attention_gradients(cfg, Q, K, V, sel, dO)
    # directional derivative of <O, dO> along a random direction, by central differences
    mask = bwd.selected_mask(cfg, sel)[0, 0].numpy()

    def loss(q, k, v):
        s = (q[0, 0] @ k[0, 0].T) / np.sqrt(cfg.d)
        s = np.where(mask, s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        return float(((p @ v[0, 0]) * dO[0]).sum())

    for g, which in ((gq, 0), (gk, 1), (gv, 2)):
        u = rng.standard_normal(Q.shape)
        h = 1e-6
        plus = [Q, K, V]
        minus = [Q, K, V]
        plus = [a + h * u if i == which else a for i, a in enumerate(plus)]
        minus = [a - h * u if i == which else a for i, a in enumerate(minus)]
        fd = (loss(*plus) - loss(*minus)) / (2 * h)
        assert abs(fd - float((g * u).sum())) <= 1e-6 * max(1.0, abs(fd))


def test_self_attention_only_closed_form():
    cfg = tiny(S=16, Bs=1, L=1, R=0, E=1, H=1, d=4)
    rng = np.random.default_rng(5)
    Q, K, V = (rng.standard_normal((1, 1, cfg.S, cfg.d)) for _ in range(3))
    dO = rng.standard_normal((1, cfg.S, cfg.d))
    sel = np.zeros((1, 1, cfg.S, 0), np.int32)
    gq, gk, gv = bwd.attention_gradients(cfg, Q, K, V, sel, dO)
    np.testing.assert_allclose(gv[0, 0], dO[0], atol=1e-14)
    np.testing.assert_allclose(gq, 0.0, atol=1e-14)
    np.testing.assert_allclose(gk, 0.0, atol=1e-14)
