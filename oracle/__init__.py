"""The oracle: a plain, slow, single-threaded CPU statement of the Monodratic
mixer forward pass, used to check the CUDA library.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
benchmark's CPU-baseline leg may import this package.  The CUDA library never
imports, links or calls it, and it shares no code with the CUDA library: the
arithmetic lives in ``mono_oracle.c`` (plain C, fp64 values, fp32 routing
decisions in a fixed plain order); this file only marshals numpy arrays.

Stages (each cites its source in ``mono_oracle.c``):

* :func:`project`         Q/K/V = x W^T, RoPE on Q and K (fp64)
* :func:`summary_assign`  block-mean key summary and product address (fp32)
* :func:`posting`         bounded causal posting lists, overflow count
* :func:`posting_redirect` the same lists with redirect-on-overflow (next address
                          in mixed-radix order with room)
* :func:`route_queries`   probe, union, causal filter, E cap, rerank (fp32)
* :func:`summary_assign64`, :func:`route_queries64`
                          the same routing decisions in fp64 (with margins), the
                          precision-independent reference for the fp32 ones
* :func:`attend`          exact softmax over the selected token set (fp64)
* :func:`out_project`     delta = O Wo^T (fp64)
* :func:`forward`         all of the above with the stored-precision rounding
                          of the activations between stages
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mono_oracle.c")
_LIB = os.path.join(_HERE, "libmono_oracle.so")
_lock = threading.Lock()
_lib = None


class _Cfg(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int) for k in ("B", "S", "W", "H", "d", "Bs", "L", "R", "E", "M", "C", "T", "cap")] + [
        ("theta", ctypes.c_double)
    ]


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, no fast-math, no contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-shared", "-fPIC",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            L = ctypes.c_long
            lib.orc_project.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, L, P, P, P, P]
            lib.orc_summary_assign.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P]
            lib.orc_posting.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P]
            lib.orc_posting_redirect.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P, P]
            lib.orc_route_queries.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P, L, P, P, P, P, P, P]
            lib.orc_attend.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, L, P, P]
            lib.orc_summary_assign64.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P]
            lib.orc_route_queries64.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P, L, P, P, P, P, P, P]
            lib.orc_out_project.argtypes = [ctypes.POINTER(_Cfg), P, P, L, P, P]
            for f in ("orc_project", "orc_summary_assign", "orc_posting", "orc_route_queries", "orc_attend",
                      "orc_out_project", "orc_summary_assign64", "orc_route_queries64", "orc_posting_redirect"):
                getattr(lib, f).restype = ctypes.c_int
            _lib = lib
    return _lib


def _cfg(c) -> _Cfg:
    return _Cfg(*(int(getattr(c, k)) for k in ("B", "S", "W", "H", "d", "Bs", "L", "R", "E", "M", "C", "T", "cap")),
                float(c.theta))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return None if a is None else np.ascontiguousarray(a, dtype=dt)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def project(cfg, x, Wq, Wk, Wv, rows=None):
    """Q, K, V (fp64).  [B,H,S,d] each, or [len(rows),H,d] for flat token rows b*S+t."""
    lib = _load()
    x, Wq, Wk, Wv = (_c(a, np.float64) for a in (x, Wq, Wk, Wv))
    rows = _c(rows, np.int64)
    shape = (cfg.B, cfg.H, cfg.S, cfg.d) if rows is None else (len(rows), cfg.H, cfg.d)
    Q, K, V = (np.empty(shape, np.float64) for _ in range(3))
    rc = lib.orc_project(ctypes.byref(_cfg(cfg)), _p(x), _p(Wq), _p(Wk), _p(Wv),
                         0 if rows is None else len(rows), _p(rows), _p(Q), _p(K), _p(V))
    _check(rc, "project")
    return Q, K, V


def summary_assign(cfg, K, codebooks):
    """kbar [B,H,nb,d] fp32, addr [B,H,nb] int32, assign margin [B,H,nb] fp32."""
    lib = _load()
    K = _c(K, np.float32)
    cb = _c(codebooks, np.float32)
    nb = cfg.S // cfg.Bs
    kbar = np.empty((cfg.B, cfg.H, nb, cfg.d), np.float32)
    addr = np.empty((cfg.B, cfg.H, nb), np.int32)
    margin = np.empty((cfg.B, cfg.H, nb), np.float32)
    _check(lib.orc_summary_assign(ctypes.byref(_cfg(cfg)), _p(K), _p(cb), _p(kbar), _p(addr), _p(margin)),
           "summary_assign")
    return kbar, addr, margin


def posting(cfg, addr):
    """Canonical posting lists: ids sorted by (addr, j), their addr, rank within the address, overflow [B,H]."""
    lib = _load()
    addr = _c(addr, np.int32)
    nb = cfg.S // cfg.Bs
    ids = np.empty((cfg.B, cfg.H, nb), np.int32)
    saddr = np.empty((cfg.B, cfg.H, nb), np.int32)
    rank = np.empty((cfg.B, cfg.H, nb), np.int32)
    ov = np.empty((cfg.B, cfg.H), np.int64)
    _check(lib.orc_posting(ctypes.byref(_cfg(cfg)), _p(addr), _p(ids), _p(saddr), _p(rank), _p(ov)), "posting")
    return ids, saddr, rank, ov


def posting_redirect(cfg, addr):
    """Redirect-on-overflow lists: list address of each block [B,H,nb] (-1 = dropped), and the canonical
    export over list addresses (dropped blocks last under C^M): ids, their list address, rank, overflow [B,H]."""
    lib = _load()
    addr = _c(addr, np.int32)
    nb = cfg.S // cfg.Bs
    la = np.empty((cfg.B, cfg.H, nb), np.int32)
    ids = np.empty((cfg.B, cfg.H, nb), np.int32)
    saddr = np.empty((cfg.B, cfg.H, nb), np.int32)
    rank = np.empty((cfg.B, cfg.H, nb), np.int32)
    ov = np.empty((cfg.B, cfg.H), np.int64)
    _check(lib.orc_posting_redirect(ctypes.byref(_cfg(cfg)), _p(addr), _p(la), _p(ids), _p(saddr), _p(rank),
                                    _p(ov)), "posting_redirect")
    return la, ids, saddr, rank, ov


def route_queries(cfg, Q, kbar, codebooks, addr, forced=None, qidx=None):
    """sel [n,R] (or [B,H,S,R] for all queries), ncand, probe margin, rerank margin, forced_ignored."""
    lib = _load()
    Q = _c(Q, np.float32)
    kbar = _c(kbar, np.float32)
    cb = _c(codebooks, np.float32)
    addr = _c(addr, np.int32)
    forced = _c(forced, np.int32)
    qidx = _c(qidx, np.int64)
    n = cfg.B * cfg.H * cfg.S if qidx is None else len(qidx)
    sel = np.empty((n, max(cfg.R, 0)), np.int32)
    ncand = np.empty(n, np.int32)
    pm = np.empty(n, np.float32)
    rm = np.empty(n, np.float32)
    ign = np.zeros(1, np.int64)
    rc = lib.orc_route_queries(ctypes.byref(_cfg(cfg)), _p(Q), _p(kbar), _p(cb), _p(addr), _p(forced),
                               0 if qidx is None else len(qidx), _p(qidx), _p(sel), _p(ncand), _p(pm), _p(rm),
                               _p(ign))
    _check(rc, "route_queries")
    if qidx is None:
        sel = sel.reshape(cfg.B, cfg.H, cfg.S, cfg.R)
        ncand = ncand.reshape(cfg.B, cfg.H, cfg.S)
        pm = pm.reshape(cfg.B, cfg.H, cfg.S)
        rm = rm.reshape(cfg.B, cfg.H, cfg.S)
    return sel, ncand, pm, rm, int(ign[0])


def summary_assign64(cfg, K, codebooks):
    """fp64 routing: kbar [B,H,nb,d] fp64, addr [B,H,nb] int32, assign margin [B,H,nb] fp64."""
    lib = _load()
    K = _c(K, np.float64)
    cb = _c(codebooks, np.float64)
    nb = cfg.S // cfg.Bs
    kbar = np.empty((cfg.B, cfg.H, nb, cfg.d), np.float64)
    addr = np.empty((cfg.B, cfg.H, nb), np.int32)
    margin = np.empty((cfg.B, cfg.H, nb), np.float64)
    _check(lib.orc_summary_assign64(ctypes.byref(_cfg(cfg)), _p(K), _p(cb), _p(kbar), _p(addr), _p(margin)),
           "summary_assign64")
    return kbar, addr, margin


def route_queries64(cfg, Q, kbar, codebooks, addr, forced=None, qidx=None):
    """fp64 routing: sel, ncand, probe margin (smallest neighbour gap among grid ranks 1..T+1), rerank
    margin (smallest neighbour gap among rerank ranks 1..R+1), forced_ignored.  Shapes as route_queries."""
    lib = _load()
    Q = _c(Q, np.float64)
    kbar = _c(kbar, np.float64)
    cb = _c(codebooks, np.float64)
    addr = _c(addr, np.int32)
    forced = _c(forced, np.int32)
    qidx = _c(qidx, np.int64)
    n = cfg.B * cfg.H * cfg.S if qidx is None else len(qidx)
    sel = np.empty((n, max(cfg.R, 0)), np.int32)
    ncand = np.empty(n, np.int32)
    pm = np.empty(n, np.float64)
    rm = np.empty(n, np.float64)
    ign = np.zeros(1, np.int64)
    rc = lib.orc_route_queries64(ctypes.byref(_cfg(cfg)), _p(Q), _p(kbar), _p(cb), _p(addr), _p(forced),
                                 0 if qidx is None else len(qidx), _p(qidx), _p(sel), _p(ncand), _p(pm), _p(rm),
                                 _p(ign))
    _check(rc, "route_queries64")
    if qidx is None:
        sel = sel.reshape(cfg.B, cfg.H, cfg.S, cfg.R)
        ncand = ncand.reshape(cfg.B, cfg.H, cfg.S)
        pm = pm.reshape(cfg.B, cfg.H, cfg.S)
        rm = rm.reshape(cfg.B, cfg.H, cfg.S)
    return sel, ncand, pm, rm, int(ign[0])


def attend(cfg, Q, K, V, sel, qidx=None):
    """Selected-set attention, fp64: O [B,H,S,d] (all queries) or [n,d] for flat query-heads qidx."""
    lib = _load()
    Q, K, V = (_c(a, np.float64) for a in (Q, K, V))
    sel = _c(sel, np.int32)
    qidx = _c(qidx, np.int64)
    shape = (cfg.B, cfg.H, cfg.S, cfg.d) if qidx is None else (len(qidx), cfg.d)
    O = np.empty(shape, np.float64)
    _check(lib.orc_attend(ctypes.byref(_cfg(cfg)), _p(Q), _p(K), _p(V), _p(sel),
                          0 if qidx is None else len(qidx), _p(qidx), _p(O)), "attend")
    return O


def out_project(cfg, O, Wo, rows=None):
    """delta = O Wo^T (fp64); O [B,S,H*d]; returns [B,S,W] or [len(rows),W]."""
    lib = _load()
    O = _c(O, np.float64)
    Wo = _c(Wo, np.float64)
    rows = _c(rows, np.int64)
    shape = (cfg.B, cfg.S, cfg.W) if rows is None else (len(rows), cfg.W)
    out = np.empty(shape, np.float64)
    _check(lib.orc_out_project(ctypes.byref(_cfg(cfg)), _p(O), _p(Wo), 0 if rows is None else len(rows), _p(rows),
                               _p(out)), "out_project")
    return out


def round_storage(a, dtype: str) -> np.ndarray:
    """Round fp64 values once to the storage type ("bf16": nearest-even on 8 mantissa bits; "f32")."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    if dtype == "f32":
        return a.astype(np.float32)
    if dtype != "bf16":
        raise ValueError(dtype)
    u = a.view(np.uint64)
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    r = ((u + np.uint64((1 << 44) - 1) + lsb) >> np.uint64(45)) << np.uint64(45)
    return r.view(np.float64).astype(np.float32)


def heads_to_tokens(O):
    """[B,H,S,d] -> [B,S,H*d]."""
    B, H, S, d = O.shape
    return np.ascontiguousarray(np.transpose(O, (0, 2, 1, 3)).reshape(B, S, H * d))


def forward(cfg, inputs, forced=None):
    """The whole mixer on the oracle.  Activations are stored in cfg.dtype between
    stages (Q/K/V after RoPE, O before the output projection), as the library does.
    Returns a dict of every stage's result."""
    Q, K, V = project(cfg, inputs["x"], inputs["Wq"], inputs["Wk"], inputs["Wv"])
    Qs, Ks, Vs = (round_storage(a, cfg.dtype) for a in (Q, K, V))
    kbar, addr, amargin = summary_assign(cfg, Ks, inputs["codebooks"])
    ids, saddr, rank, ov = posting(cfg, addr)
    sel, ncand, pm, rm, ign = route_queries(cfg, Qs, kbar, inputs["codebooks"], addr, forced=forced)
    O = attend(cfg, Qs, Ks, Vs, sel)
    Ot = round_storage(heads_to_tokens(O), cfg.dtype)
    delta = out_project(cfg, Ot, inputs["Wo"])
    return dict(Q=Qs, K=Ks, V=Vs, kbar=kbar, addr=addr, assign_margin=amargin, ids=ids, saddr=saddr, rank=rank,
                overflow=ov, sel=sel, ncand=ncand, probe_margin=pm, rerank_margin=rm, forced_ignored=ign,
                O=Ot, delta=delta)
