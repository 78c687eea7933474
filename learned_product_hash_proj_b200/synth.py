"""Seeded synthetic inputs for the Monodratic mixer.

This module only draws random numbers and shapes them into the workloads the
library is tested and measured on.  It holds none of the method's arithmetic
(no projection, rotation, routing or attention) so that the CUDA library and
the CPU oracle can both be fed from it without sharing any computation.

Workloads (shapes as in the scope of this library; the pages publish no
dataset, so every input is synthetic):

* ``pr1``     B=1 S=1024 W=256 H=4 d=64 fp32, Bs=32 L=2 R=2 E=5 M=2 C=8 T=4 cap=16
* ``recall``  B=8 S=4096 W=512 H=8 d=64 fp32, Bs=64 L=1 R=2 E=5 M=2 C=16 T=4 cap=32;
              token ids over a 512-row N(0,1) embedding table with 16 planted
              key->value pairs per sequence, the keys re-presented at the end
              (the associative-recall shape of "Monodratic Routes Sparse
              Attention with Learned Product Hashes", Key Points)
* ``scaleNk`` B=1 S=N*1024 (4K..32K) W=1024 H=16 d=64 bf16, Bs=64 L=2 R=2 E=5
              M=2 C=16 T=4 cap=64 (S=32768 is the headline point)
* ``long``    B=1 S=131072 W=2048 H=16 d=128 bf16, Bs=128 L=2 R=4 E=8 M=2 C=32
              T=8 cap=256; x = N(0,1) + per-channel AR(1) drift (rho=0.999)
* ``stress``  B=16 S=16384 W=2048 H=16 d=128 bf16, Bs=64 L=2 R=4 E=8 M=4 C=16
              T=16 cap=8; a batch of variable-length sequences: each token of
              the valid prefix drawn from a 32-component Gaussian mixture (sd
              0.1, centres N(0,1)), the rest of the row zero padding.  The
              valid length of each sequence is a uniform whole number of
              blocks in [nb/4, 3nb/4]; all-padding blocks share one address,
              so posting lists overflow.

Weights are N(0, 1/W); codewords N(0,1) scaled to unit L2 norm per
(head, subspace, code).  bf16 workloads round x and the weights to bf16 once
(round-to-nearest-even) and both sides consume those stored values.
"""
from __future__ import annotations

import copy
from dataclasses import dataclass, field, replace

import numpy as np

_BASE = dict(theta=10000.0)

CONFIGS: dict[str, dict] = {
    "pr1": dict(B=1, S=1024, W=256, H=4, d=64, Bs=32, L=2, R=2, E=5, M=2, C=8, T=4, cap=16,
                dtype="f32", x="normal", **_BASE),
    "recall": dict(B=8, S=4096, W=512, H=8, d=64, Bs=64, L=1, R=2, E=5, M=2, C=16, T=4, cap=32,
                   dtype="f32", x="recall", **_BASE),
    "long": dict(B=1, S=131072, W=2048, H=16, d=128, Bs=128, L=2, R=4, E=8, M=2, C=32, T=8,
                 cap=256, dtype="bf16", x="drift", **_BASE),
    "stress": dict(B=16, S=16384, W=2048, H=16, d=128, Bs=64, L=2, R=4, E=8, M=4, C=16, T=16,
                   cap=8, dtype="bf16", x="mixture", **_BASE),
}
for _k in (4, 8, 16, 32):
    CONFIGS[f"scale{_k}k"] = dict(B=1, S=_k * 1024, W=1024, H=16, d=64, Bs=64, L=2, R=2, E=5, M=2,
                                  C=16, T=4, cap=64, dtype="bf16", x="normal", **_BASE)

HEADLINE = "scale32k"
SHAPE_KEYS = ("B", "S", "W", "H", "d", "Bs", "L", "R", "E", "M", "C", "T", "cap")


@dataclass(frozen=True)
class Config:
    B: int
    S: int
    W: int
    H: int
    d: int
    Bs: int
    L: int
    R: int
    E: int
    M: int
    C: int
    T: int
    cap: int
    theta: float = 10000.0
    dtype: str = "bf16"          # storage type of x, weights, Q/K/V, O, delta
    x: str = "normal"            # input recipe
    name: str = field(default="custom", compare=False)

    @property
    def nb(self) -> int:
        return self.S // self.Bs

    @property
    def A(self) -> int:
        return self.C ** self.M

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


def config(name: str, **overrides) -> Config:
    """The named workload preset, optionally with fields overridden."""
    c = copy.deepcopy(CONFIGS[name])
    c.update(overrides)
    return Config(name=name, **c)


# --------------------------------------------------------------------------
# random streams: one independent PCG64 stream per (seed, tensor, index)
# --------------------------------------------------------------------------
_STREAM = {"x": 1, "Wq": 2, "Wk": 3, "Wv": 4, "Wo": 5, "cb": 6, "mix": 7, "recall": 8, "forced": 9}


def _rng(seed: int, what: str, *idx: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), _STREAM[what], *map(int, idx)])


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(a)
    out = r.astype(np.uint32).view(np.float32)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def _store(a: np.ndarray, cfg: Config) -> np.ndarray:
    return round_bf16(a) if cfg.dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def make_weights(cfg: Config, seed: int = 0) -> dict[str, np.ndarray]:
    """Wq, Wk, Wv [H*d, W] and Wo [W, H*d] (out_features x in_features), N(0, 1/W)."""
    hd = cfg.H * cfg.d
    sd = 1.0 / np.sqrt(cfg.W)
    out = {}
    for name, shape in (("Wq", (hd, cfg.W)), ("Wk", (hd, cfg.W)), ("Wv", (hd, cfg.W)), ("Wo", (cfg.W, hd))):
        w = _rng(seed, name).standard_normal(shape, dtype=np.float64) * sd
        out[name] = _store(w.astype(np.float32), cfg)
    return out


def make_codebooks(cfg: Config, seed: int = 0) -> np.ndarray:
    """Codewords [H, M, C, d/M] fp32: N(0,1), then unit L2 norm per (h, m, c)."""
    dm = cfg.d // cfg.M
    g = _rng(seed, "cb").standard_normal((cfg.H, cfg.M, cfg.C, dm), dtype=np.float64)
    g /= np.linalg.norm(g, axis=-1, keepdims=True)
    return g.astype(np.float32)


def make_x_batch(cfg: Config, seed: int, b: int) -> np.ndarray:
    """x[b] as a [S, W] float32 array (bf16-representable for bf16 workloads)."""
    S, W = cfg.S, cfg.W
    r = _rng(seed, "x", b)
    kind = cfg.x
    if kind == "normal":
        x = r.standard_normal((S, W), dtype=np.float32)
    elif kind == "zeros":
        x = np.zeros((S, W), dtype=np.float32)
    elif kind == "drift":
        from scipy.signal import lfilter
        rho = 0.999
        z = r.standard_normal((S, W), dtype=np.float32)
        e = r.standard_normal((S, W), dtype=np.float64)
        g0 = r.standard_normal(W)
        g = np.empty((S, W), dtype=np.float64)
        g[0] = g0
        if S > 1:
            g[1:] = lfilter([np.sqrt(1.0 - rho * rho)], [1.0, -rho], e[1:], axis=0, zi=(rho * g0)[None, :])[0]
        x = (z + g).astype(np.float32)
    elif kind == "mixture":
        centres = _rng(seed, "mix").standard_normal((32, W), dtype=np.float32)
        k = r.integers(0, 32, size=S)
        x = centres[k] + np.float32(0.1) * r.standard_normal((S, W), dtype=np.float32)
        x[valid_length(cfg, seed, b):] = 0.0
    elif kind == "recall":
        ids, _ = recall_tokens(cfg, seed, b)
        table = _rng(seed, "recall").standard_normal((512, W), dtype=np.float32)
        x = table[ids]
    else:
        raise ValueError(f"unknown input recipe {kind!r}")
    return _store(x, cfg)


def valid_length(cfg: Config, seed: int, b: int) -> int:
    """Number of non-padding tokens of sequence b in the batched skewed workload."""
    nb = cfg.S // cfg.Bs
    lo, hi = nb // 4, max(nb // 4, (3 * nb) // 4)
    return int(_rng(seed, "mix", 1, b).integers(lo, hi + 1)) * cfg.Bs


def recall_tokens(cfg: Config, seed: int, b: int, n_pairs: int = 16, vocab: int = 512):
    """Token ids [S] for the associative-recall shape and the planted pairs.

    Each of the n_pairs (key, value) id pairs is written at a seeded position
    p (key at p, value at p+1) inside blocks 0..nb-2, pairs never overlapping;
    the final n_pairs tokens of the sequence repeat the keys in shuffled order.
    Returns (ids, pairs) with pairs = [(key_pos, key_id, value_id, query_pos)].
    """
    S, Bs = cfg.S, cfg.Bs
    r = _rng(seed, "x", b)
    ids = r.integers(0, vocab, size=S)
    if S < 2 * n_pairs + Bs or S // Bs < 2:
        return ids, []
    limit = (S // Bs - 1) * Bs - 1            # key and value inside blocks 0..nb-2
    slots = r.choice(limit // 2, size=n_pairs, replace=False) * 2
    keys = r.choice(vocab, size=n_pairs, replace=False)
    vals = r.integers(0, vocab, size=n_pairs)
    order = r.permutation(n_pairs)
    pairs = []
    for i in range(n_pairs):
        ids[slots[i]] = keys[i]
        ids[slots[i] + 1] = vals[i]
    for qpos, i in enumerate(order):
        ids[S - n_pairs + qpos] = keys[i]
        pairs.append((int(slots[i]), int(keys[i]), int(vals[i]), S - n_pairs + qpos))
    return ids, pairs


def make_x(cfg: Config, seed: int = 0) -> np.ndarray:
    """x [B, S, W] float32."""
    out = np.empty((cfg.B, cfg.S, cfg.W), dtype=np.float32)
    for b in range(cfg.B):
        out[b] = make_x_batch(cfg, seed, b)
    return out


def make_forced(cfg: Config, seed: int = 0, frac: float = 0.5) -> np.ndarray:
    """A forced-block id per query-head [B, H, S] (int32, -1 = none).

    About `frac` of the queries get a uniformly drawn earlier block id (which
    may or may not be eligible); the rest get -1.
    """
    r = _rng(seed, "forced")
    t = np.arange(cfg.S)
    bq = t // cfg.Bs
    f = np.full((cfg.B, cfg.H, cfg.S), -1, dtype=np.int32)
    draw = r.random((cfg.B, cfg.H, cfg.S)) < frac
    ids = (r.random((cfg.B, cfg.H, cfg.S)) * (bq[None, None, :] + 1)).astype(np.int32)
    f[draw] = ids[draw]
    return f


def make_inputs(cfg: Config, seed: int = 0) -> dict[str, np.ndarray]:
    """Every input of the mixer as float32 numpy arrays (stored values)."""
    out = make_weights(cfg, seed)
    out["x"] = make_x(cfg, seed)
    out["codebooks"] = make_codebooks(cfg, seed)
    return out
