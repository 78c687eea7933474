"""A second, independently written router for tiny inputs (pure Python).

It restates the routing rules of the Monodratic mixer ("aitechinspire.com
Monodratic article", Snapshot: source blocks go to bounded causal posting
lists after RoPE; each query probes product addresses, reranks the returned
candidates and keeps a fixed number of remote blocks) with exact binary32
arithmetic on rationals, enumerating everything, with none of the oracle's
code.  Integer outputs must agree with the oracle bit for bit.
"""
import itertools

import numpy as np

from fp32_exact import add32, div32, dot_chain32


def summaries(K_bh, Bs):
    """kbar per block: ascending-t binary32 sums divided by Bs."""
    S, d = K_bh.shape
    out = []
    for j in range(S // Bs):
        row = []
        for i in range(d):
            acc = np.float32(0.0)
            for t in range(j * Bs, (j + 1) * Bs):
                acc = add32(acc, K_bh[t, i])
            row.append(div32(acc, np.float32(Bs)))
        out.append(row)
    return out


def codes_of(vec, cw_h, M, C):
    """Per-subspace argmax code (first index wins a tie) of a summary vector."""
    dm = len(vec) // M
    codes = []
    for m in range(M):
        scores = [dot_chain32(vec[m * dm:(m + 1) * dm], cw_h[m][c]) for c in range(C)]
        best = max(range(C), key=lambda c: (scores[c], -c))
        codes.append(best)
    return codes


def address(codes, C):
    a = 0
    for c in codes:
        a = a * C + c
    return a


def route_bh(Q_bh, K_bh, cw_h, cfg, forced_bh=None):
    """Route every query of one (batch, head).  Returns (addr, lists, overflow, sel)."""
    S, d = Q_bh.shape
    Bs, M, C, T, R, E, L, cap = cfg.Bs, cfg.M, cfg.C, cfg.T, cfg.R, cfg.E, cfg.L, cfg.cap
    nb = S // Bs
    kb = summaries(K_bh, Bs)
    addr = [address(codes_of(kb[j], cw_h, M, C), C) for j in range(nb)]
    lists = {}
    overflow = 0
    for j, a in enumerate(addr):
        bucket = lists.setdefault(a, [])
        if len(bucket) < cap:
            bucket.append(j)
        else:
            overflow += 1
    dm = d // M
    sel = []
    for t in range(S):
        q = Q_bh[t]
        sub = [[dot_chain32(q[m * dm:(m + 1) * dm], cw_h[m][c]) for c in range(C)] for m in range(M)]
        scored = []
        for combo in itertools.product(range(C), repeat=M):
            g = sub[0][combo[0]]
            for m in range(1, M):
                g = add32(g, sub[m][combo[m]])
            scored.append((-float(g), address(combo, C)))
        scored.sort()
        probes = [a for _, a in scored[:T]]
        bq = t // Bs
        cands = []
        for a in probes:
            for j in lists.get(a, []):
                if j <= bq - L and len(cands) < E:
                    cands.append(j)
        ranked = sorted(cands, key=lambda j: (-float(dot_chain32(q, kb[j])), j))
        chosen = ranked[:R]
        if forced_bh is not None and R > 0:
            f = int(forced_bh[t])
            if 0 <= f <= bq - L and f not in chosen:
                if len(chosen) < R:
                    chosen.append(f)
                else:
                    chosen[-1] = f
        chosen = sorted(chosen)
        sel.append(chosen + [-1] * (R - len(chosen)))
    return addr, lists, overflow, sel
