"""mono_route_static: routing for callers that cannot allocate device memory.

Some callers of this library never get to allocate device memory: a plugin
whose host framework owns every allocation, or a serving loop that forbids
cudaMalloc once it is running.  mono_route_static keeps the routing tables in
one fixed array that the library places in global memory, instead of in a
caller workspace.  These tests call it through the C-ABI and check that it
returns exactly what mono_route returns, on two calls in a row with different
inputs (the array keeps the previous call's contents, so the second call
checks that nothing stale leaks through), and that an oversize problem is
refused before anything is launched.  The statistics a static call leaves in
the array (overflow counts, selection counters, device error word) are read
back through mono_stats with no workspace and must equal mono_route's.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from learned_product_hash_proj_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mono():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_product_hash_proj_b200 import build
    build.build()
    from learned_product_hash_proj_b200 import mono as m
    lib = m.lib()
    lib.mono_route_static.argtypes = [ctypes.c_void_p] * 7
    lib.mono_route_static.restype = ctypes.c_int
    lib.mono_route_static_capacity.argtypes = []
    lib.mono_route_static_capacity.restype = ctypes.c_size_t
    return m


def _inputs(cfg, seed):
    rng = np.random.default_rng(seed)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = (cfg.B, cfg.H, cfg.S, cfg.d)
    Q = torch.from_numpy(rng.standard_normal(shape, dtype=np.float32)).to(dt).cuda()
    K = torch.from_numpy(rng.standard_normal(shape, dtype=np.float32) * 3.0).to(dt).cuda()
    cb = torch.from_numpy(synth.make_codebooks(cfg, seed)).cuda()
    return Q, K, cb


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("name", ["scale4k", "pr1"])
def test_matches_mono_route_on_two_calls_in_a_row(mono, name):
    cfg = synth.config(name)
    plan = mono.Plan(cfg)
    ws = plan.workspace()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (1, 2):
        Q, K, cb = _inputs(cfg, seed)
        forced = torch.from_numpy(synth.make_forced(cfg, seed, 0.3)).cuda() if seed == 2 else None
        ref = torch.empty((cfg.B, cfg.H, cfg.S, cfg.R), dtype=torch.int32, device="cuda")
        mono.route(plan, Q, K, cb, ref, ws, forced=forced)
        got = torch.full_like(ref, -7)
        rc = mono.lib().mono_route_static(plan.handle, _p(Q), _p(K), _p(cb),
                                          None if forced is None else _p(forced), _p(got), stream)
        assert rc == 0, mono.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"seed {seed}: {(got != ref).sum().item()} selections differ"


def test_stats_of_the_static_call_match_mono_stats(mono):
    # Routing statistics and the device error word of a static call stay in the fixed array; mono_stats reads
    # them back when it is given no workspace.  Every other block of K is zero, so those blocks share address 0
    # and the lists overflow: the overflow totals must agree with mono_route's, and so must the other counters.
    cfg = synth.Config(B=2, S=2048, W=128, H=3, d=64, Bs=32, L=2, R=2, E=5, M=2, C=8, T=4, cap=3, dtype="bf16")
    plan = mono.Plan(cfg)
    ws = plan.workspace()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    Q, K, cb = _inputs(cfg, 3)
    blk = (torch.arange(cfg.S, device="cuda") // cfg.Bs) % 2 == 0
    K = (K * blk.view(1, 1, cfg.S, 1).to(K.dtype)).contiguous()
    ref = torch.empty((cfg.B, cfg.H, cfg.S, cfg.R), dtype=torch.int32, device="cuda")
    mono.route(plan, Q, K, cb, ref, ws)
    want = mono.stats(plan, ws)
    assert want["overflow_total"] > 0
    got_sel = torch.full_like(ref, -7)
    for _ in range(2):
        rc = mono.lib().mono_route_static(plan.handle, _p(Q), _p(K), _p(cb), None, _p(got_sel), stream)
        assert rc == 0, mono.STATUS.get(rc, rc)
        st = mono.Stats()
        rc = mono.lib().mono_stats(plan.handle, None, stream, ctypes.byref(st))
        assert rc == 0, mono.STATUS.get(rc, rc)
        assert torch.equal(got_sel, ref)
        assert st.as_dict() == {k: want[k] for k in st.as_dict()}


def test_rejects_problems_beyond_the_fixed_array(mono):
    cap = mono.lib().mono_route_static_capacity()
    assert cap == 16 << 20
    cfg = synth.config("stress")                       # 16*16*256 blocks x (128*4 + 16) bytes > 16 MiB
    plan = mono.Plan(cfg)
    one = torch.zeros(16, dtype=torch.uint8, device="cuda")
    rc = mono.lib().mono_route_static(plan.handle, _p(one), _p(one), _p(one), None, _p(one), None)
    assert rc == 8                                     # MONO_ERR_SCRATCH, nothing launched
