"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, validates plans, lays out the workspace, and rejects bad arguments
before launching anything.  No test here calls a kernel."""
import ctypes
import os
import re

import pytest

from learned_product_hash_proj_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mono():
    from learned_product_hash_proj_b200 import build
    build.build()
    from learned_product_hash_proj_b200 import mono as m
    return m


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(mono_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_function(mono):
    names = declared_functions()
    assert "mono_forward" in names and "mono_plan" in names
    lib = mono.lib()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert mono.version() == 1


def test_binding_covers_the_header(mono):
    assert set(mono.EXPORTS) == set(declared_functions())


@pytest.mark.parametrize("name", sorted(synth.CONFIGS))
def test_every_workload_plans(mono, name):
    p = mono.Plan(synth.config(name))
    assert p.workspace_bytes > 0


@pytest.mark.parametrize("change,status", [
    (dict(S=1000), "MONO_ERR_INVALID"),            # S % Bs != 0
    (dict(R=6, E=5), "MONO_ERR_INVALID"),          # R > E
    (dict(T=300), "MONO_ERR_INVALID"),             # T > C^M = 256
    (dict(L=0), "MONO_ERR_INVALID"),
    (dict(cap=0), "MONO_ERR_INVALID"),
    (dict(d=63), "MONO_ERR_INVALID"),              # odd head dim
    (dict(M=3), "MONO_ERR_INVALID"),               # d % M != 0
    (dict(d=96, M=2), "MONO_ERR_UNSUPPORTED"),     # d not in {64, 128}
    (dict(W=1000), "MONO_ERR_UNSUPPORTED"),        # W % 64 != 0
    (dict(T=33, C=64), "MONO_ERR_UNSUPPORTED"),
])
def test_plan_rejects(mono, change, status):
    cfg = synth.config("scale4k", **change)
    with pytest.raises(mono.MonoError) as e:
        mono.Plan(cfg)
    assert mono.STATUS[e.value.status] == status


def test_workspace_regions_are_aligned_and_disjoint(mono):
    for name in ("pr1", "scale32k", "long", "stress"):
        p = mono.Plan(synth.config(name))
        spans = []
        for region in range(len(mono.REGIONS)):
            off, nbytes = ctypes.c_size_t(), ctypes.c_size_t()
            assert mono.lib().mono_workspace_region(p.handle, region, ctypes.byref(off), ctypes.byref(nbytes)) == 0
            assert off.value % 256 == 0
            assert off.value + nbytes.value <= p.workspace_bytes
            spans.append((off.value, off.value + nbytes.value))
        spans.sort()
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 <= b0


def test_entry_points_reject_bad_arguments_before_launching(mono):
    lib = mono.lib()
    p = mono.Plan(synth.config("pr1"))
    fake = ctypes.c_void_p(1 << 20)            # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 8)       # 16-byte misaligned
    N = None
    assert lib.mono_route(None, fake, fake, fake, N, fake, fake, N) == 3          # NULL plan
    assert lib.mono_route(p.handle, fake, fake, fake, N, fake, N, N) == 4         # no workspace
    assert lib.mono_route(p.handle, N, fake, fake, N, fake, fake, N) == 3         # NULL Q
    assert lib.mono_attend(p.handle, fake, odd, fake, fake, fake, fake, N) == 7   # misaligned K
    assert lib.mono_forward(p.handle, fake, fake, fake, fake, fake, fake, N, fake, odd, N) == 7  # workspace %256
    assert lib.mono_project(p.handle, fake, fake, N, fake, fake, fake, fake, fake, N) == 3
    assert lib.mono_out_project(p.handle, fake, N, fake, fake, N) == 3


def test_empty_inputs_launch_nothing(mono):
    lib = mono.lib()
    fake = ctypes.c_void_p(1 << 20)
    for change in (dict(B=0), dict(S=0)):
        p = mono.Plan(synth.config("pr1", **change))
        assert lib.mono_forward(p.handle, fake, fake, fake, fake, fake, fake, None, fake, fake, None) == 0
        st = mono.Stats()
        assert lib.mono_stats(p.handle, fake, None, ctypes.byref(st)) == 0
        assert st.overflow_total == 0 and st.remote_selected == 0


def test_status_strings(mono):
    for code in mono.STATUS:
        assert mono.lib().mono_strerror(code)


def test_decode_cache_layout_and_argument_checks(mono):
    lib = mono.lib()
    cfg = synth.config("pr1")
    p = mono.Plan(cfg)
    n = ctypes.c_size_t()
    assert lib.mono_decode_cache_bytes(p.handle, ctypes.byref(n)) == 0 and n.value > 0
    spans = []
    for r in range(len(mono.DEC_REGIONS)):
        off, nb = ctypes.c_size_t(), ctypes.c_size_t()
        assert lib.mono_decode_cache_region(p.handle, r, ctypes.byref(off), ctypes.byref(nb)) == 0
        assert off.value % 256 == 0 and off.value + nb.value <= n.value
        spans.append((off.value, off.value + nb.value))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    off, nb = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.mono_decode_cache_region(p.handle, len(mono.DEC_REGIONS), ctypes.byref(off), ctypes.byref(nb)) == 1
    fake = ctypes.c_void_p(1 << 20)            # never dereferenced: validation fails first
    odd = ctypes.c_void_p((1 << 20) + 16)      # not 256-byte aligned
    N = None
    assert lib.mono_decode_step(None, 0, fake, fake, fake, fake, fake, fake, N, fake, fake, N) == 3  # NULL plan
    assert lib.mono_decode_step(p.handle, 0, fake, fake, fake, fake, fake, fake, N, fake, N, N) == 4  # no cache
    assert lib.mono_decode_route(p.handle, 0, fake, N, odd, N) == 7                                  # cache %256
    assert lib.mono_decode_attend(p.handle, cfg.S, fake, N) == 1                                     # t >= S
    assert lib.mono_decode_project(p.handle, -1, fake, fake, fake, fake, fake, N) == 1               # t < 0
    assert lib.mono_decode_prefill(p.handle, cfg.S + 1, fake, fake, N) == 1                          # t0 > S
    # the decode path scores every address of a query: C^M <= 4096
    big = mono.Plan(synth.config("stress"))
    assert lib.mono_decode_cache_bytes(big.handle, ctypes.byref(n)) == 2


def test_backward_workspace_and_argument_checks(mono):
    lib = mono.lib()
    sizes = []
    for S in (1024, 2048):
        p = mono.Plan(synth.config("pr1", S=S))
        n = ctypes.c_size_t()
        assert lib.mono_backward_workspace_bytes(p.handle, ctypes.byref(n)) == 0
        assert n.value % 256 == 0
        sizes.append(n.value)
    assert sizes[1] > sizes[0] > 0
    assert lib.mono_backward_workspace_bytes(None, ctypes.byref(ctypes.c_size_t())) == 3
    p = mono.Plan(synth.config("pr1"))
    fake = ctypes.c_void_p(1 << 20)            # never dereferenced: validation fails first
    odd16 = ctypes.c_void_p((1 << 20) + 8)     # not 16-byte aligned
    odd256 = ctypes.c_void_p((1 << 20) + 16)   # not 256-byte aligned
    N = None
    f6 = [fake] * 6
    # mono_backward(plan, x, Wq, Wk, Wv, Wo, sel, ddelta, dx, dWq, dWk, dWv, dWo, ws, bws, stream)
    assert lib.mono_backward(None, *f6, fake, *[fake] * 5, fake, fake, N) == 3                 # NULL plan
    assert lib.mono_backward(p.handle, *f6, fake, *[fake] * 5, N, fake, N) == 4                # no workspace
    assert lib.mono_backward(p.handle, *f6, fake, *[fake] * 5, fake, N, N) == 4                # no bwd workspace
    assert lib.mono_backward(p.handle, *f6, fake, *[fake] * 5, fake, odd256, N) == 7           # bws %256
    assert lib.mono_backward(p.handle, *f6, fake, odd16, *[fake] * 4, fake, fake, N) == 7      # misaligned dx
    assert lib.mono_backward(p.handle, fake, fake, fake, fake, fake, N, fake, *[fake] * 5, fake, fake, N) == 3  # sel
    # mono_attend_backward(plan, Q, K, V, sel, dO, dQ, dK, dV, bws, stream)
    assert lib.mono_attend_backward(p.handle, *[fake] * 8, N, N) == 4                           # no bwd workspace
    assert lib.mono_attend_backward(p.handle, fake, fake, fake, fake, fake, N, fake, fake, fake, N) == 3  # NULL dQ
    assert lib.mono_attend_backward(p.handle, fake, odd16, *[fake] * 6, fake, N) == 7         # misaligned K
    # empty batch: nothing to do, nothing launched
    pe = mono.Plan(synth.config("pr1", B=0))
    assert lib.mono_backward(pe.handle, *f6, fake, *[fake] * 5, fake, fake, N) == 0


def test_binding_refuses_host_tensors(mono):
    # no CPU fallback anywhere in the product path: host tensors are an error, before the library is called
    import torch
    cfg = synth.config("pr1")
    p = mono.Plan(cfg)
    dt = p.dtype
    hd = cfg.H * cfg.d
    x = torch.zeros((cfg.B, cfg.S, cfg.W), dtype=dt)
    W = torch.zeros((hd, cfg.W), dtype=dt)
    Wo = torch.zeros((cfg.W, hd), dtype=dt)
    cb = torch.zeros((cfg.H, cfg.M, cfg.C, cfg.d // cfg.M), dtype=torch.float32)
    ws = torch.zeros(p.workspace_bytes, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mono.forward(p, x, W, W, W, Wo, cb, torch.zeros_like(x), ws)
    sel = torch.zeros((cfg.B, cfg.H, cfg.S, cfg.R), dtype=torch.int32)
    f32 = dict(dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mono.backward(p, x, W, W, W, Wo, sel, x, torch.zeros(x.shape, **f32), torch.zeros(W.shape, **f32),
                      torch.zeros(W.shape, **f32), torch.zeros(W.shape, **f32), torch.zeros(Wo.shape, **f32), ws,
                      torch.zeros(256, dtype=torch.uint8))
