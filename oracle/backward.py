"""Gradients of the mixer for a fixed selection -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use
anything under oracle/.  Plain PyTorch on the CPU in float64, written from the
definition of the forward pass, with the gradients taken by autograd:

* projection without bias, q = x Wq^T (nn.Linear layout), per head
  ("Monodratic Routes Sparse Attention with Learned Product Hashes", Key
  Points; the aitechinspire.com article, Snapshot: a stateless [batch,
  sequence, width] -> attention-delta mixer);
* RoPE on q and k, interleaved pairs (2i, 2i+1) rotated by t * theta^(-2i/d);
* exact causal softmax over the selected token set of each query: the tokens
  of the remote blocks in sel[b, h, t] that lie in [0, t/Bs - L] plus the
  local tokens [max(0, t/Bs - L + 1) * Bs, t] (aitechinspire.com article,
  Snapshot), scale 1/sqrt(d) -- written here as dense attention under that
  mask;
* delta = O Wo^T.
With storage="bf16" (or "f32") the activations are rounded to the storage type
between stages, as the library and the C oracle's forward store them (Q and K
after RoPE, V, O), and the rounding's derivative is taken as 1: the gradient
of the computation as performed on its stored values.
The routing (summaries, addresses, lists, probe, rerank) is piecewise
constant in its inputs and has no gradient: the selection is an input.
"""
from __future__ import annotations

import numpy as np
import torch


def _rope(x: torch.Tensor, theta: float) -> torch.Tensor:
    """x [B, H, S, d]: rotate the pairs (2i, 2i+1) of position t by t * theta^(-2i/d)."""
    B, H, S, d = x.shape
    i = torch.arange(d // 2, dtype=torch.float64)
    t = torch.arange(S, dtype=torch.float64)
    ang = t[:, None] * theta ** (-2.0 * i / d)[None, :]          # [S, d/2]
    c, s = torch.cos(ang), torch.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y0 = x0 * c - x1 * s
    y1 = x0 * s + x1 * c
    return torch.stack((y0, y1), dim=-1).reshape(B, H, S, d)


def selected_mask(cfg, sel: np.ndarray) -> torch.Tensor:
    """[B, H, S, S] bool: key s is in the selected token set of query t."""
    B, H, S, Bs, L = cfg.B, cfg.H, cfg.S, cfg.Bs, cfg.L
    t = np.arange(S)
    bq = t // Bs
    lo = np.maximum(0, bq - L + 1) * Bs
    s = np.arange(S)
    local = (s[None, :] >= lo[:, None]) & (s[None, :] <= t[:, None])        # [S, S]
    mask = np.broadcast_to(local, (B, H, S, S)).copy()
    blk = s // Bs
    lim = bq - L
    for r in range(sel.shape[-1]):
        j = sel[..., r]                                                        # [B, H, S]
        ok = (j >= 0) & (j <= lim[None, None, :])
        mask |= ok[..., None] & (blk[None, None, None, :] == j[..., None])
    return torch.from_numpy(mask)


def _stored(a: torch.Tensor, storage) -> torch.Tensor:
    """a rounded to the storage type (round to nearest even), with derivative 1."""
    if storage is None:
        return a
    r = a.to(torch.bfloat16 if storage == "bf16" else torch.float32).to(torch.float64)
    return a + (r - a).detach()


def forward(cfg, x, Wq, Wk, Wv, Wo, sel, storage=None):
    """delta [B, S, W] (float64 tensors in, float64 out), for a fixed selection sel [B, H, S, R]."""
    B, S, W, H, d = cfg.B, cfg.S, cfg.W, cfg.H, cfg.d
    theta = float(getattr(cfg, "theta", 10000.0))

    def heads(w):
        return (x @ w.T).reshape(B, S, H, d).permute(0, 2, 1, 3)             # [B, H, S, d]

    Q, K, V = (_stored(a, storage) for a in (_rope(heads(Wq), theta), _rope(heads(Wk), theta), heads(Wv)))
    scores = (Q @ K.transpose(-1, -2)) / np.sqrt(d)
    scores = scores.masked_fill(~selected_mask(cfg, sel), float("-inf"))
    P = torch.softmax(scores, dim=-1)
    O = _stored((P @ V).permute(0, 2, 1, 3).reshape(B, S, H * d), storage)
    return O @ Wo.T


def gradients(cfg, x, Wq, Wk, Wv, Wo, sel, ddelta, storage=None) -> dict:
    """d(<delta, ddelta>) with respect to x, Wq, Wk, Wv, Wo (numpy float64 in and out)."""
    ts = {k: torch.tensor(np.asarray(v, np.float64), requires_grad=True)
          for k, v in (("x", x), ("Wq", Wq), ("Wk", Wk), ("Wv", Wv), ("Wo", Wo))}
    delta = forward(cfg, ts["x"], ts["Wq"], ts["Wk"], ts["Wv"], ts["Wo"], np.asarray(sel), storage=storage)
    g = torch.autograd.grad(delta, list(ts.values()), grad_outputs=torch.tensor(np.asarray(ddelta, np.float64)))
    return {k: gi.numpy() for k, gi in zip(ts, g)}


def attention_gradients(cfg, Q, K, V, sel, dO) -> tuple:
    """dQ, dK, dV [B, H, S, d] of <O, dO> for the selected-set attention on given post-RoPE Q, K, V
    ([B, H, S, d]) and dO [B, S, H*d] (numpy float64 in and out)."""
    B, S, H, d = cfg.B, cfg.S, cfg.H, cfg.d
    q, k, v = (torch.tensor(np.asarray(a, np.float64), requires_grad=True) for a in (Q, K, V))
    scores = (q @ k.transpose(-1, -2)) / np.sqrt(d)
    scores = scores.masked_fill(~selected_mask(cfg, np.asarray(sel)), float("-inf"))
    O = (torch.softmax(scores, dim=-1) @ v).permute(0, 2, 1, 3).reshape(B, S, H * d)
    g = torch.autograd.grad(O, [q, k, v], grad_outputs=torch.tensor(np.asarray(dO, np.float64)))
    return tuple(gi.numpy() for gi in g)
