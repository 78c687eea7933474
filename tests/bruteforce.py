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

from fp32_exact import add32, div32, dot_chain32, dot_tree32


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


def redirect_lists(addr, A, cap):
    """Redirect-on-overflow placement: block j goes to the first list with room among its own address and the
    next ones in mixed-radix order (a, a+1, ... mod A); dropped only when every list is full."""
    lists, overflow = {}, 0
    for j, a in enumerate(addr):
        for step in range(A):
            b = (a + step) % A
            if len(lists.get(b, [])) < cap:
                lists.setdefault(b, []).append(j)
                break
        else:
            overflow += 1
    return lists, overflow


def route_bh(Q_bh, K_bh, cw_h, cfg, forced_bh=None, redirect=False, rerank_margins=None, rerank_dot=dot_tree32):
    """Route every query of one (batch, head).  Returns (addr, lists, overflow, sel).  With a list given as
    rerank_margins, appends each query's fp32 rerank margin: score(R-th) - score((R+1)-th) when more than R
    candidates remain, else +inf (rerank_dot: the fp32 dot product the scores use)."""
    S, d = Q_bh.shape
    Bs, M, C, T, R, E, L, cap = cfg.Bs, cfg.M, cfg.C, cfg.T, cfg.R, cfg.E, cfg.L, cfg.cap
    nb = S // Bs
    kb = summaries(K_bh, Bs)
    addr = [address(codes_of(kb[j], cw_h, M, C), C) for j in range(nb)]
    if redirect:
        lists, overflow = redirect_lists(addr, C ** M, cap)
    else:
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
        score = {j: rerank_dot(q, kb[j]) for j in cands}
        ranked = sorted(cands, key=lambda j: (-float(score[j]), j))
        if rerank_margins is not None:
            rerank_margins.append(add32(score[ranked[R - 1]], -score[ranked[R]]) if 0 < R < len(ranked)
                                  else np.float32(np.inf))
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


# ---------------------------------------------------------------------------
# The same rules on exact rationals: every sum, mean and dot product is exact
# (fractions.Fraction on the stored binary32 values), so each decision is the
# one the real-valued scores make.  The fp64 routing of the oracle must agree
# with it wherever no margin is within fp64 rounding of zero.
# ---------------------------------------------------------------------------
from fractions import Fraction  # noqa: E402


def _fr(v):
    return Fraction(float(v))


def _dot_exact(a, b):
    return sum((x * y for x, y in zip(a, b)), Fraction(0))


def route_bh_exact(Q_bh, K_bh, cw_h, cfg, forced_bh=None):
    """Route every query of one (batch, head) exactly.  Returns (addr, overflow, sel, assign margins,
    probe margins, rerank margins) with the margins defined as in the oracle's fp64 routing: per block the
    smallest best-minus-second code score over the subspaces; per query the smallest gap between neighbours
    among grid ranks 1..T+1 and among rerank ranks 1..R+1."""
    S, d = Q_bh.shape
    Bs, M, C, T, R, E, L, cap = cfg.Bs, cfg.M, cfg.C, cfg.T, cfg.R, cfg.E, cfg.L, cfg.cap
    nb, dm = S // Bs, d // M
    K = [[_fr(v) for v in row] for row in K_bh]
    Q = [[_fr(v) for v in row] for row in Q_bh]
    cw = [[[_fr(v) for v in cw_h[m][c]] for c in range(C)] for m in range(M)]
    kb = [[sum((K[t][i] for t in range(j * Bs, (j + 1) * Bs)), Fraction(0)) / Bs for i in range(d)]
          for j in range(nb)]
    addr, amargin = [], []
    for j in range(nb):
        a, mg = 0, None
        for m in range(M):
            sc = [_dot_exact(kb[j][m * dm:(m + 1) * dm], cw[m][c]) for c in range(C)]
            order = sorted(range(C), key=lambda c: (-sc[c], c))
            a = a * C + order[0]
            if C > 1:
                gap = sc[order[0]] - sc[order[1]]
                mg = gap if mg is None else min(mg, gap)
        addr.append(a)
        amargin.append(mg)
    lists, overflow = {}, 0
    for j, a in enumerate(addr):
        bucket = lists.setdefault(a, [])
        if len(bucket) < cap:
            bucket.append(j)
        else:
            overflow += 1
    sel, pmargin, rmargin = [], [], []
    for t in range(S):
        q = Q[t]
        sub = [[_dot_exact(q[m * dm:(m + 1) * dm], cw[m][c]) for c in range(C)] for m in range(M)]
        scored = sorted(((-sum((sub[m][combo[m]] for m in range(M)), Fraction(0)), address(combo, C))
                         for combo in itertools.product(range(C), repeat=M)))
        top = scored[:T + 1]
        pmargin.append(min((top[k + 1][0] - top[k][0] for k in range(len(top) - 1)), default=None))
        bq = t // Bs
        cands = []
        for _, a in scored[:T]:
            for j in lists.get(a, []):
                if j <= bq - L and len(cands) < E:
                    cands.append(j)
        ranked = sorted(((-_dot_exact(q, kb[j]), j) for j in cands))
        rk = ranked[:R + 1] if R > 0 else []
        rmargin.append(min((rk[k + 1][0] - rk[k][0] for k in range(len(rk) - 1)), default=None))
        chosen = [j for _, j in ranked[:R]]
        if forced_bh is not None and R > 0:
            f = int(forced_bh[t])
            if 0 <= f <= bq - L and f not in chosen:
                if len(chosen) < R:
                    chosen.append(f)
                else:
                    chosen[-1] = f
        chosen = sorted(chosen)
        sel.append(chosen + [-1] * (R - len(chosen)))
    return addr, overflow, sel, amargin, pmargin, rmargin
