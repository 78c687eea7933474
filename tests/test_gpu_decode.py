"""GPU parity of the decode entry points (one token per sequence against a cache).

Every stage of the mixer is causal, so decode step t must reproduce row t of
the batch pass on the same values:

* routing: per-step selections bit-exact against the batch kernels and the
  oracle; after the last step the cache's summaries, addresses, posting lists
  and overflow counts equal the batch tables (lists compared as the kept ids
  of each address in ascending order);
* attention: against the oracle fp64 on the same Q/K/V and selections;
* projection and output projection (full steps): against the oracle fp64 on
  x, and on the decode's own attention output.
Tolerances as for the batch pass (1e-5 max abs for fp32, 2e-2 x RMS on top of
bf16 storage rounding for bf16).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_parity import Run, assert_close, to_np
from learned_product_hash_proj_b200 import mono, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from learned_product_hash_proj_b200 import build
    build.build()


def small(**kw):
    base = dict(B=2, S=384, W=128, H=3, d=64, Bs=32, L=2, R=2, E=5, M=2, C=8, T=4, cap=3, dtype="f32", x="normal")
    base.update(kw)
    return synth.Config(**base)


CASES = {
    "f32": dict(),
    "bf16": dict(dtype="bf16"),
    "d128_bf16": dict(d=128, H=2, S=256, Bs=64, C=16, cap=4, dtype="bf16"),
    "M4_L1_R4": dict(M=4, C=4, T=8, E=8, R=4, L=1, cap=2),
    # the route's per-lane address lists at their two longest compile-time lengths (16 and 32)
    "T16": dict(T=16, E=8, R=4),
    "M4_C8_T32": dict(M=4, C=8, T=32, E=16, R=4, cap=2),
    "local_only": dict(R=0),
    "zero_ties": dict(x="zeros"),
}


def walk_lists(plan, cache):
    """Per (b, h): {address: kept block ids in list order} from the decode cache."""
    c = plan.cfg
    cnt, head, nxt = (to_np(mono.decode_region(plan, cache, k)) for k in ("count", "head", "next"))
    out = {}
    for b in range(c.B):
        for h in range(c.H):
            lists = {}
            for a in np.nonzero(cnt[b, h])[0]:
                ids, j = [], int(head[b, h, a])
                while j >= 0:
                    ids.append(j)
                    j = int(nxt[b, h, j])
                lists[int(a)] = ids
            out[(b, h)] = lists
    return out


def batch_lists(cfg, route_ws):
    """The same from the batch posting arrays: kept entries (rank < cap) grouped by address."""
    ids, saddr, rank = route_ws["post_ids"], route_ws["post_addr"], route_ws["post_rank"]
    out = {}
    for b in range(cfg.B):
        for h in range(cfg.H):
            lists = {}
            for k in range(ids.shape[-1]):
                if rank[b, h, k] < cfg.cap:
                    lists.setdefault(int(saddr[b, h, k]), []).append(int(ids[b, h, k]))
            out[(b, h)] = lists
    return out


def run_decode_on_batch_values(run: Run, t0: int = 0):
    """Decode steps t0..S-1 on the batch pass's own Q/K/V; returns per-step sel and o."""
    cfg, plan = run.cfg, run.plan
    cache = mono.decode_cache(plan)
    mono.decode_region(plan, cache, "K").copy_(run.K)
    mono.decode_region(plan, cache, "V").copy_(run.V)
    cb = run.dev["codebooks"]
    mono.decode_prefill(plan, t0, cb, cache)
    qreg, sreg, oreg = (mono.decode_region(plan, cache, k) for k in ("q", "sel", "o"))
    sels, outs = [], []
    for t in range(t0, cfg.S):
        qreg.copy_(run.Q[:, :, t, :])
        ft = None if run.forced_dev is None else run.forced_dev[:, :, t].contiguous()
        mono.decode_route(plan, t, cb, cache, forced_t=ft)
        mono.decode_attend(plan, t, cache)
        sels.append(sreg[..., :max(cfg.R, 0)].clone())
        outs.append(oreg.clone())
    torch.cuda.synchronize()
    sel = torch.stack(sels, dim=2) if sels else None          # [B, H, S - t0, R]
    o = torch.stack(outs, dim=1)                              # [B, S - t0, H*d]
    return cache, sel, o


def check_tables(run: Run, cache):
    plan = run.plan
    ws = run.route_ws
    kb = to_np(mono.decode_region(plan, cache, "kbar"))
    np.testing.assert_array_equal(kb.view(np.uint32), ws["kbar"].view(np.uint32), err_msg="kbar bits")
    np.testing.assert_array_equal(to_np(mono.decode_region(plan, cache, "addr")), ws["addr"], err_msg="addresses")
    np.testing.assert_array_equal(to_np(mono.decode_region(plan, cache, "overflow")), ws["overflow"],
                                  err_msg="overflow")
    assert walk_lists(plan, cache) == batch_lists(run.cfg, ws)


@pytest.mark.parametrize("name", list(CASES))
def test_decode_route_attend_matches_batch(name):
    cfg = small(**CASES[name])
    run = Run(cfg, seed=3, forced_frac=0.05 if name == "f32" else None).run_stages()
    cache, sel, o = run_decode_on_batch_values(run)
    check_tables(run, cache)
    if cfg.R > 0:
        np.testing.assert_array_equal(to_np(sel), to_np(run.sel), err_msg="decode sel vs batch sel")
        ref_sel = oracle.route_queries(cfg, to_np(run.Q), run.route_ws["kbar"], run.inp["codebooks"],
                                       run.route_ws["addr"], forced=run.forced)[0]
        np.testing.assert_array_equal(to_np(sel), ref_sel, err_msg="decode sel vs oracle")
    Qg, Kg, Vg = (to_np(a).astype(np.float64) for a in (run.Q, run.K, run.V))
    ref = oracle.attend(cfg, Qg, Kg, Vg, to_np(run.sel))          # [B, H, S, d]
    got = to_np(o).reshape(cfg.B, cfg.S, cfg.H, cfg.d).transpose(0, 2, 1, 3)
    assert_close(got, ref, cfg.dtype, "decode attention")


@pytest.mark.parametrize("t0", [64, 100])
def test_decode_prefill_then_steps(t0):
    cfg = small(dtype="bf16")
    run = Run(cfg, seed=4).run_stages()
    cache, sel, _ = run_decode_on_batch_values(run, t0=t0)
    check_tables(run, cache)
    np.testing.assert_array_equal(to_np(sel), to_np(run.sel)[:, :, t0:], err_msg="sel after prefill")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_full_steps(dtype):
    """mono_decode_step from an empty cache: projection, routing on its own Q/K, attention, output."""
    cfg = small(dtype=dtype, B=2, S=256)
    run = Run(cfg, seed=5)
    plan, d = run.plan, run.dev
    cache = mono.decode_cache(plan)
    mono.decode_prefill(plan, 0, d["codebooks"], cache)
    qreg, sreg, oreg = (mono.decode_region(plan, cache, k) for k in ("q", "sel", "o"))
    qs, sels, outs, deltas = [], [], [], []
    for t in range(cfg.S):
        x_t = d["x"][:, t, :].contiguous()
        delta_t = torch.empty((cfg.B, cfg.W), dtype=plan.dtype, device="cuda")
        mono.decode_step(plan, t, x_t, d["Wq"], d["Wk"], d["Wv"], d["Wo"], d["codebooks"], delta_t, cache)
        qs.append(qreg.clone())
        sels.append(sreg.clone())
        outs.append(oreg.clone())
        deltas.append(delta_t)
    torch.cuda.synchronize()
    Qd = torch.stack(qs, dim=2)                                    # [B, H, S, d]
    Kd, Vd = mono.decode_region(plan, cache, "K"), mono.decode_region(plan, cache, "V")
    inp = run.inp
    Qr, Kr, Vr = oracle.project(cfg, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"])
    for nm, got, ref in (("q", Qd, Qr), ("k", Kd, Kr), ("v", Vd, Vr)):
        assert_close(to_np(got), ref, dtype, f"decode projection {nm}")
    # routing on the decode's own keys and queries, bit-exact
    Kg, Qg = to_np(Kd), to_np(Qd)
    kbar, addr, _ = oracle.summary_assign(cfg, Kg, inp["codebooks"])
    np.testing.assert_array_equal(to_np(mono.decode_region(plan, cache, "kbar")).view(np.uint32),
                                  kbar.view(np.uint32), err_msg="kbar bits")
    ref_sel = oracle.route_queries(cfg, Qg, kbar, inp["codebooks"], addr)[0]
    np.testing.assert_array_equal(to_np(torch.stack(sels, dim=2)), ref_sel, err_msg="decode sel")
    # attention and output projection on the decode's own values
    ref_o = oracle.attend(cfg, Qg.astype(np.float64), Kg.astype(np.float64), to_np(Vd).astype(np.float64), ref_sel)
    O = torch.stack(outs, dim=1)                                   # [B, S, H*d]
    assert_close(to_np(O).reshape(cfg.B, cfg.S, cfg.H, cfg.d).transpose(0, 2, 1, 3), ref_o, dtype, "decode attention")
    ref_delta = oracle.out_project(cfg, to_np(O).astype(np.float64), inp["Wo"])
    assert_close(to_np(torch.stack(deltas, dim=1)), ref_delta, dtype, "decode output projection")


def test_decode_steps_in_a_cuda_graph_equal_eager_steps():
    # The step's kernels start early under programmatic dependent launch and wait for their predecessor; captured
    # into one CUDA graph and replayed, the steps give the same bits as eager calls: deltas, selections and the
    # cache's tables.
    cfg = small(dtype="bf16", B=2, S=192)
    run = Run(cfg, seed=6)
    plan, d = run.plan, run.dev
    xs = [d["x"][:, t, :].contiguous() for t in range(cfg.S)]

    def steps(graph):
        cache = mono.decode_cache(plan)
        mono.decode_prefill(plan, 0, d["codebooks"], cache)
        sreg = mono.decode_region(plan, cache, "sel")
        deltas = [torch.empty((cfg.B, cfg.W), dtype=plan.dtype, device="cuda") for _ in range(cfg.S)]
        sels = [torch.empty_like(sreg) for _ in range(cfg.S)]

        def body():
            for t in range(cfg.S):
                mono.decode_step(plan, t, xs[t], d["Wq"], d["Wk"], d["Wv"], d["Wo"], d["codebooks"], deltas[t],
                                 cache)
                sels[t].copy_(sreg)

        torch.cuda.synchronize()
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                body()
            g.replay()
        else:
            body()
        torch.cuda.synchronize()
        tables = [mono.decode_region(plan, cache, k).clone() for k in ("kbar", "addr", "count", "head", "next")]
        return deltas, sels, tables

    eager, captured = steps(False), steps(True)
    for a, b in zip(eager[0], captured[0]):
        assert torch.equal(a, b)
    for a, b in zip(eager[1], captured[1]):
        assert torch.equal(a, b)
    for a, b in zip(eager[2], captured[2]):
        assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                           b.view(torch.int32) if b.dtype == torch.float32 else b)
