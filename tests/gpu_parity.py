"""Stage-wise parity of the CUDA library against the oracle (helpers).

Every stage of the GPU pass is checked against the oracle on the GPU's own
stored inputs of that stage, so that rounding in one stage does not leak into
the next one's comparison:

* projection + RoPE : oracle fp64 on x, rounded once to the storage type
* summaries, addresses, posting lists, overflow : bit-exact (fp32 decisions in
  the order the specification fixes)
* selected blocks   : bit-exact
* attention         : oracle fp64 on the GPU's Q/K/V and sel
* output projection : oracle fp64 on the GPU's O

Tolerances: fp32 storage -> max abs error 1e-5; bf16 storage -> max abs error
2e-2 x RMS of the reference, on top of the bf16 storage rounding of each
output element (at most 2^-8 of its magnitude).

Routing is also measured against the oracle's fp64 statement of the same
decisions (check_fp64_rule): a GPU address or selection may differ from the
fp64 one only where a margin of a decision behind it is below 1e-4, and such
queries must stay below 0.1 % of all queries.
"""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np
import torch

import oracle
from learned_product_hash_proj_b200 import mono, synth

TOL_F32_ABS = 1e-5
TOL_BF16_REL_RMS = 2e-2


def to_dev(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return (t.to(torch.bfloat16) if dtype == "bf16" else t).to(device).contiguous()


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy() if t.dtype != torch.int32 else t.detach().cpu().numpy()


BF16_UNIT_ROUNDOFF = 2.0 ** -8   # storing a value in bf16 moves it by at most this fraction of itself


def assert_close(got, ref, dtype: str, what: str):
    """fp32: max |got - ref| <= 1e-5.  bf16: max (|got - ref| - 2^-8 |ref|) <= 2e-2 x RMS(ref).

    `ref` is the unrounded fp64 reference.  A bf16 output carries up to half an
    ulp (<= 2^-8 of its magnitude) of storage rounding that no kernel can avoid,
    so that term is allowed on top of the 2e-2 x RMS computation tolerance.
    """
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if dtype == "f32":
        err = np.abs(got - ref).max() if got.size else 0.0
        assert err <= TOL_F32_ABS, f"{what}: max abs err {err:.3e} > {TOL_F32_ABS}"
        return err
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    excess = (np.abs(got - ref) - BF16_UNIT_ROUNDOFF * np.abs(ref)).max() if got.size else 0.0
    assert excess <= TOL_BF16_REL_RMS * rms, \
        f"{what}: max (|err| - 2^-8|ref|) {excess:.3e} > 2e-2 x RMS {rms:.3e}"
    return excess / max(rms, 1e-300)


def sample_tokens(cfg, n: int, rng) -> np.ndarray:
    """Flat token rows b*S + t: edges plus a uniform sample."""
    total = cfg.B * cfg.S
    edge = [0, cfg.S - 1, total - 1, cfg.Bs, cfg.Bs * cfg.L, min(total - 1, cfg.Bs * (cfg.L + 1) - 1)]
    rows = np.unique(np.concatenate([np.array(edge), rng.integers(0, total, size=n)]))
    return rows[(rows >= 0) & (rows < total)].astype(np.int64)


def sample_queries(cfg, n: int, rng) -> np.ndarray:
    """Flat query-heads (b*H + h)*S + t, sorted (the oracle rebuilds lists per (b, h))."""
    total = cfg.B * cfg.H * cfg.S
    edge = [0, cfg.S - 1, total - 1, cfg.Bs * cfg.L, cfg.Bs * (cfg.L + 1) - 1]
    q = np.unique(np.concatenate([np.array(edge), rng.integers(0, total, size=n)]))
    return np.sort(q[(q >= 0) & (q < total)]).astype(np.int64)


def oracle_lists(cfg, addr, redirect: bool):
    """The oracle's posting lists for block addresses `addr`: (the address of the list holding each block, or
    -1 when dropped -- what the query routing reads), ids, list address, rank, overflow."""
    if redirect:
        return oracle.posting_redirect(cfg, addr)
    ids, saddr, rank, ov = oracle.posting(cfg, addr)
    return addr, ids, saddr, rank, ov


class Run:
    """Inputs of one workload on the device plus the GPU results of each stage."""

    def __init__(self, cfg, seed=0, flags=0, forced_frac=None, inputs=None):
        self.cfg = cfg
        self.redirect = bool(flags & mono.MONO_FLAG_REDIRECT)
        self.inp = inputs if inputs is not None else synth.make_inputs(cfg, seed)
        self.forced = None if forced_frac is None else synth.make_forced(cfg, seed, forced_frac)
        self.plan = mono.Plan(cfg, flags=flags)
        dt = cfg.dtype
        self.dev = {k: to_dev(v, dt) for k, v in self.inp.items() if k != "codebooks"}
        self.dev["codebooks"] = torch.from_numpy(self.inp["codebooks"]).cuda().contiguous()
        self.forced_dev = None if self.forced is None else torch.from_numpy(self.forced).cuda().contiguous()
        self.ws = self.plan.workspace()
        B, H, S, d, R, W = cfg.B, cfg.H, cfg.S, cfg.d, cfg.R, cfg.W
        tdt = self.plan.dtype
        self.Q = torch.empty((B, H, S, d), dtype=tdt, device="cuda")
        self.K = torch.empty_like(self.Q)
        self.V = torch.empty_like(self.Q)
        self.sel = torch.empty((B, H, S, R), dtype=torch.int32, device="cuda")
        self.O = torch.empty((B, S, H * d), dtype=tdt, device="cuda")
        self.delta = torch.empty((B, S, W), dtype=tdt, device="cuda")

    def run_stages(self):
        d = self.dev
        mono.project(self.plan, d["x"], d["Wq"], d["Wk"], d["Wv"], self.Q, self.K, self.V, self.ws)
        mono.route(self.plan, self.Q, self.K, d["codebooks"], self.sel, self.ws, forced=self.forced_dev)
        self.route_ws = {k: to_np(self.plan.region(self.ws, k)).copy()
                         for k in ("kbar", "addr", "post_ids", "post_addr", "post_rank", "overflow", "walk_log")}
        self.stats = mono.stats(self.plan, self.ws)
        mono.attend(self.plan, self.Q, self.K, self.V, self.sel, self.O, self.ws)
        mono.out_project(self.plan, self.O, d["Wo"], self.delta, self.ws)
        torch.cuda.synchronize()
        return self

    def run_forward(self) -> torch.Tensor:
        d = self.dev
        out = torch.empty_like(self.delta)
        ws = self.plan.workspace()
        mono.forward(self.plan, d["x"], d["Wq"], d["Wk"], d["Wv"], d["Wo"], d["codebooks"], out, ws,
                     forced=self.forced_dev)
        torch.cuda.synchronize()
        self.forward_stats = mono.stats(self.plan, ws)
        return out


def check_projection(run: Run, rows=None):
    cfg = run.cfg
    inp = run.inp
    Q, K, V = oracle.project(cfg, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], rows=rows)
    errs = []
    for name, ref, got in (("Q", Q, run.Q), ("K", K, run.K), ("V", V, run.V)):
        g = to_np(got)
        if rows is not None:
            b, t = rows // cfg.S, rows % cfg.S
            g = g[b, :, t, :]                      # [n, H, d]
        errs.append(assert_close(g, ref, cfg.dtype, f"projection {name}"))
    return max(errs)


def check_routing(run: Run, qidx=None):
    """Bit-exact summaries, addresses, posting lists, overflow and sel."""
    cfg = run.cfg
    Kg = to_np(run.K)
    Qg = to_np(run.Q)
    kbar, addr, amargin = oracle.summary_assign(cfg, Kg, run.inp["codebooks"])
    ws = run.route_ws
    np.testing.assert_array_equal(ws["kbar"].view(np.uint32), kbar.view(np.uint32), err_msg="kbar bits")
    np.testing.assert_array_equal(ws["addr"], addr, err_msg="addresses")
    laddr, ids, saddr, rank, ov = oracle_lists(cfg, addr, run.redirect)
    np.testing.assert_array_equal(ws["post_ids"], ids, err_msg="posting ids")
    np.testing.assert_array_equal(ws["post_addr"], saddr, err_msg="posting addresses")
    np.testing.assert_array_equal(ws["post_rank"], rank, err_msg="posting ranks")
    np.testing.assert_array_equal(ws["overflow"].astype(np.int64), ov, err_msg="overflow")
    assert run.stats["overflow_total"] == int(ov.sum())
    sel, ncand, pm, rm, ign = oracle.route_queries(cfg, Qg, kbar, run.inp["codebooks"], laddr, forced=run.forced,
                                                   qidx=qidx)
    gsel = to_np(run.sel).reshape(cfg.B * cfg.H * cfg.S, cfg.R)
    if qidx is None:
        np.testing.assert_array_equal(gsel.reshape(sel.shape), sel, err_msg="sel")
        n_valid = (sel >= 0).sum()
        assert run.stats["remote_selected"] == int(n_valid)
        assert run.stats["queries_lt_R"] == int(((sel >= 0).sum(axis=-1) < cfg.R).sum())
        if run.forced is not None:
            assert run.stats["forced_ignored"] == ign
    else:
        np.testing.assert_array_equal(gsel[qidx], sel, err_msg="sel (sampled queries)")
    small = int((rm < 1e-4).sum())
    n = cfg.B * cfg.H * cfg.S if qidx is None else len(qidx)
    return dict(overflow=int(ov.sum()), queries=n, small_margin=small)


def check_attention(run: Run, qidx=None):
    cfg = run.cfg
    Og = to_np(run.O)                                      # [B, S, H*d]
    Oh = Og.reshape(cfg.B, cfg.S, cfg.H, cfg.d).transpose(0, 2, 1, 3)   # [B, H, S, d]
    if qidx is None:
        Qg, Kg, Vg = (to_np(a).astype(np.float64) for a in (run.Q, run.K, run.V))
        ref = oracle.attend(cfg, Qg, Kg, Vg, to_np(run.sel))
        return assert_close(Oh, ref, cfg.dtype, "attention")
    # sampled: one (b, h) slice at a time keeps host memory small at full size
    one = cfg.with_(B=1, H=1)
    refs, gots = [], []
    bh_of = qidx // cfg.S
    for bh in np.unique(bh_of):
        b, h = divmod(int(bh), cfg.H)
        ts = (qidx[bh_of == bh] % cfg.S).astype(np.int64)
        sl = [to_np(a[b:b + 1, h:h + 1]).astype(np.float64) for a in (run.Q, run.K, run.V)]
        sel = to_np(run.sel[b:b + 1, h:h + 1])
        refs.append(oracle.attend(one, *sl, sel, qidx=ts))
        gots.append(Oh[b, h, ts])
    return assert_close(np.concatenate(gots), np.concatenate(refs), cfg.dtype, "attention (sampled)")


def check_out_projection(run: Run, rows=None):
    cfg = run.cfg
    Og = to_np(run.O).astype(np.float64)
    ref = oracle.out_project(cfg, Og, run.inp["Wo"], rows=rows)
    got = to_np(run.delta)
    got = got.reshape(-1, cfg.W)[rows] if rows is not None else got
    return assert_close(got, ref, cfg.dtype, "output projection")


# ---------------------------------------------------------------------------
# routing of whole (b, h) slices against both statements of the oracle, in
# threads (the oracle's C calls release the interpreter lock)
# ---------------------------------------------------------------------------
PARITY_LOG: list[str] = []  # per workload: queries checked and counts against the fp64 oracle (printed at the end)
FP64_MARGIN = 1e-4          # decisions closer than this may differ from the fp64 oracle ...
FP64_MAX_SHARE = 1e-3       # ... on fewer than 0.1 % of the queries


def _pool():
    return cf.ThreadPoolExecutor(max_workers=max(1, min(64, os.cpu_count() or 1)))


def oracle_route_slices(run, bhs, chunk: int = 2048):
    """For each (b, h) in bhs: the oracle's fp32 and fp64 routing of every query of the slice on the GPU's
    stored Q and K.  Returns {(b, h): dict(addr32, ov32, sel32, addr64, am64, sel64, pm64, rm64)}."""
    cfg = run.cfg
    one = cfg.with_(B=1, H=1)
    cb = run.inp["codebooks"]
    res, jobs = {}, []
    with _pool() as ex:
        for b, h in bhs:
            Q1 = np.ascontiguousarray(to_np(run.Q[b:b + 1, h:h + 1]), np.float32)
            K1 = np.ascontiguousarray(to_np(run.K[b:b + 1, h:h + 1]), np.float32)
            Q64, K64 = Q1.astype(np.float64), K1.astype(np.float64)
            cb1 = np.ascontiguousarray(cb[h:h + 1])
            f1 = None if run.forced is None else np.ascontiguousarray(run.forced[b:b + 1, h:h + 1])
            kbar32, addr32, _ = oracle.summary_assign(one, K1, cb1)
            kbar64, addr64, am64 = oracle.summary_assign64(one, K64, cb1)
            la32, _, _, _, ov32 = oracle_lists(one, addr32, run.redirect)
            la64 = oracle_lists(one, addr64, run.redirect)[0]
            r = dict(addr32=addr32[0, 0], ov32=int(ov32.sum()), addr64=addr64[0, 0], am64=am64[0, 0],
                     sel32=np.empty((cfg.S, cfg.R), np.int32), sel64=np.empty((cfg.S, cfg.R), np.int32),
                     pm64=np.empty(cfg.S), rm64=np.empty(cfg.S))
            res[(b, h)] = r
            for q0 in range(0, cfg.S, chunk):
                qidx = np.arange(q0, min(cfg.S, q0 + chunk), dtype=np.int64)
                jobs.append((r, qidx, 32, ex.submit(oracle.route_queries, one, Q1, kbar32, cb1, la32, f1, qidx)))
                jobs.append((r, qidx, 64, ex.submit(oracle.route_queries64, one, Q64, kbar64, cb1, la64, f1, qidx)))
        for r, qidx, mode, fut in jobs:
            sel, _, pm, rm, _ = fut.result()
            if mode == 32:
                r["sel32"][qidx] = sel
            else:
                r["sel64"][qidx] = sel
                r["pm64"][qidx] = pm
                r["rm64"][qidx] = rm
    return res


def check_routing_slices(run, bhs):
    """Every query of the given (b, h) slices: selections bit-exact against the fp32 oracle, and the fp64
    margin rule.  Returns the counts for the report."""
    cfg = run.cfg
    res = oracle_route_slices(run, bhs)
    gaddr = run.route_ws["addr"]
    gov = run.route_ws["overflow"]
    n_q = n_blocks = n_mis = n_flip = small_p = small_r = 0
    for (b, h), r in res.items():
        np.testing.assert_array_equal(gaddr[b, h], r["addr32"], err_msg=f"addresses of slice {(b, h)}")
        assert int(gov[b, h]) == r["ov32"], f"overflow of slice {(b, h)}"
        gsel = to_np(run.sel[b, h])
        bad = np.nonzero((gsel != r["sel32"]).any(-1))[0]
        assert bad.size == 0, f"slice {(b, h)}: {bad.size} queries differ from the fp32 oracle, first t={bad[:8]}"
        flips = gaddr[b, h] != r["addr64"]
        assert (r["am64"][flips] < FP64_MARGIN).all(), f"slice {(b, h)}: address flip at an fp64 margin >= 1e-4"
        mis = (gsel != r["sel64"]).any(-1)
        expl = (r["pm64"] < FP64_MARGIN) | (r["rm64"] < FP64_MARGIN) | bool(flips.any())
        unexplained = np.nonzero(mis & ~expl)[0]
        assert unexplained.size == 0, \
            f"slice {(b, h)}: selections differ from the fp64 oracle at margins >= 1e-4, t={unexplained[:8]}"
        n_q += cfg.S
        n_blocks += cfg.nb
        n_mis += int(mis.sum())
        n_flip += int(flips.sum())
        small_p += int((r["pm64"] < FP64_MARGIN).sum())
        small_r += int((r["rm64"] < FP64_MARGIN).sum())
    assert n_flip <= FP64_MAX_SHARE * n_blocks, f"{n_flip} of {n_blocks} addresses differ from the fp64 oracle"
    assert n_mis < FP64_MAX_SHARE * n_q, f"{n_mis} of {n_q} selections differ from the fp64 oracle"
    return dict(queries=n_q, fp32_mismatch=0, fp64_mismatch=n_mis, fp64_addr_flips=n_flip,
                small_probe_margin=small_p, small_rerank_margin=small_r)


def check_fp64_rule(run):
    """All (b, h) slices of a workload: see check_routing_slices."""
    cfg = run.cfg
    return check_routing_slices(run, [(b, h) for b in range(cfg.B) for h in range(cfg.H)])


def log_routing(run, info: dict, what: str = ""):
    cfg = run.cfg
    PARITY_LOG.append(f"{cfg.name}{what} B={cfg.B} S={cfg.S} H={cfg.H} A={cfg.A} {cfg.dtype}: " +
                       " ".join(f"{k}={v}" for k, v in info.items()))


def check_walk_queries(run, checked_slices):
    """The query-heads whose probe took the general walk (the kernel logs the first mono.WALK_LOG_CAP of them)
    and that lie outside `checked_slices`: their selections against the fp32 oracle, bit for bit.  Returns
    (walks counted, walks compared here)."""
    cfg = run.cfg
    n = int(run.stats["probe_walks"])
    logged = np.sort(run.route_ws["walk_log"][:min(n, mono.WALK_LOG_CAP)].astype(np.int64))
    assert ((logged >= 0) & (logged < cfg.B * cfg.H * cfg.S)).all()
    done = {b * cfg.H + h for b, h in checked_slices}
    rest = logged[[int(q // cfg.S) not in done for q in logged]]
    if rest.size:
        kbar, addr, _ = oracle.summary_assign(cfg, to_np(run.K), run.inp["codebooks"])
        laddr = oracle_lists(cfg, addr, run.redirect)[0]
        sel, *_ = oracle.route_queries(cfg, to_np(run.Q), kbar, run.inp["codebooks"], laddr, forced=run.forced,
                                       qidx=rest)
        gsel = to_np(run.sel).reshape(-1, cfg.R)[rest]
        np.testing.assert_array_equal(gsel, sel, err_msg="sel of general-walk queries")
    return n, int(rest.size)
