"""The benchmark's host-side arithmetic, CPU only: the algorithmic bytes behind
its roofline, counted from the tensor shapes, and the committed traffic record
it reports next to them.

The per-unit figures are recomputed here from first principles (what each stage
must read and write once) rather than from bench.py's own formula: a dropped or
doubled tensor there fails one of these.
"""
import importlib.util
import json
import os

import pytest

from learned_product_hash_proj_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_probe_bytes_per_query_head(bench):
    cfg = synth.config("scale32k")
    ab = bench.algorithmic_bytes(cfg)
    qh = cfg.B * cfg.H * cfg.S
    # per query-head: its bf16 Q row (d x 2 bytes) and its R sel ids (4 bytes each) ...
    own = cfg.d * 2 + cfg.R * 4
    # ... plus per-head tables read once: kbar rows (d fp32 per block), the sorted ids and their addresses,
    # and the head's codebooks (C x d fp32)
    tables = cfg.B * cfg.H * cfg.nb * (cfg.d * 4 + 8) + cfg.H * cfg.C * cfg.d * 4
    assert ab["queries"] == qh * own + tables
    assert 140.0 <= ab["queries"] / qh <= 140.5          # the 140 B per query-head quoted with the roofline


def test_route_attend_bytes_per_token(bench):
    cfg = synth.config("scale32k")
    ab = bench.algorithmic_bytes(cfg)
    B, H, S, d, R, nb = cfg.B, cfg.H, cfg.S, cfg.d, cfg.R, cfg.nb
    unique = 4 * B * H * S * d * 2                          # Q, K, V read, O written (bf16)
    tables = 2 * (B * H * nb * d * 4) + 2 * (B * H * nb * 4) + 2 * (B * H * nb * 5) + 2 * (B * H * S * R * 4)
    assert ab["route_attend"] == unique + tables
    assert ab["route_attend"] / (B * S) == 8580.5           # B per token of the window
    # the window's figure is below the sum of its stages' (each stage re-reads what the previous wrote)
    assert ab["route_attend"] < sum(ab[k] for k in ("summaries", "lists", "queries", "attend"))


def test_fp32_storage_doubles_the_activation_bytes(bench):
    b16 = bench.algorithmic_bytes(synth.config("scale4k"))
    f32 = bench.algorithmic_bytes(synth.config("scale4k", dtype="f32"))
    cfg = synth.config("scale4k")
    qkv = cfg.B * cfg.H * cfg.S * cfg.d * 2
    assert f32["attend"] - b16["attend"] == 4 * qkv            # Q, K, V and O at 4 instead of 2 bytes


def test_traffic_record_is_consistent(bench):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    half = t["scale16k"]["queries"]["bytes_per_launch"]
    full = t["scale32k"]["queries"]["bytes_per_launch"]
    assert full == 2 * half                                  # scaled by the number of queries
    assert bench.load_traffic("queries", synth.config("scale32k")) == float(full)
    assert bench.load_traffic("attend", synth.config("scale32k")) is None
    # DRAM traffic of the probe stays at or below its algorithmic bytes: no re-reads
    assert full <= bench.algorithmic_bytes(synth.config("scale32k"))["queries"]
