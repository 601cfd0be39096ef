"""Bridges between the synthetic inputs and the oracle / the CUDA library."""
from __future__ import annotations

import numpy as np

import oracle


def dims_of(inp):
    c = inp.cfg
    return dict(T=c["T"], d=c["d"], E=c["E"], k=c["k"], f=c["f"],
                f_shared=c.get("f_shared", 0) if inp.shared is not None else 0,
                routing=c["routing"])


def oracle_run(inp, tokens=None, forced_ids=None, expert_range=None, include_shared=True):
    """Run the fp64 oracle on MoEInputs (tensors may live on any device).

    forced_ids: optional int [T, k] experts to use instead of the oracle's own
    top-k (the oracle's forced-routing mode).  expert_range / include_shared:
    the partial output of the experts begin <= e < end (expert parallelism)."""
    fmts = {n: (m.fmt, m.bits, m.group) for n, m in
            (("w1", inp.w1), ("w3", inp.w3), ("w2", inp.w2))}
    mats = {"w1": inp.w1, "w3": inp.w3, "w2": inp.w2}
    cache = {}

    def fetch(name, e):
        key = (name, e)
        if key not in cache:
            cache[key] = mats[name].expert_numpy(e)
        return cache[key]

    shared_fetch = shared_fmts = None
    if inp.shared is not None:
        sm = dict(zip(("w1", "w3", "w2"), inp.shared))
        shared_fmts = {n: (m.fmt, m.bits, m.group) for n, m in sm.items()}
        shared_fetch = lambda name, e: sm[name].expert_numpy(e)  # noqa: E731
    np_ = lambda t: None if t is None else t.detach().float().cpu().numpy()  # noqa: E731
    return oracle.forward(
        dims_of(inp), inp.x.float().cpu().numpy(),
        router_w=np_(inp.router_w), router_b=np_(inp.router_b),
        token_ids=None if inp.token_ids is None else inp.token_ids.cpu().numpy(),
        tid2eid=None if inp.tid2eid is None else inp.tid2eid.cpu().numpy(),
        fetch=fetch, fmts=fmts, shared_fetch=shared_fetch, shared_fmts=shared_fmts,
        tokens=tokens, forced_ids=None if forced_ids is None else np.asarray(forced_ids, np.int64),
        expert_range=expert_range, include_shared=include_shared)


def bigint_words(codes, bits):
    """Pack codes into uint32 words via one Python big integer (test-side only)."""
    v = 0
    for i, c in enumerate(codes):
        v |= int(c) << (i * bits)
    nw = (len(codes) * bits + 31) // 32
    return np.array([(v >> (32 * w)) & 0xFFFFFFFF for w in range(nw)], dtype=np.uint32)


# ---------------------------------------------------------------- parallel oracle calls
def _expert_rows_job(job):
    """One expert's SwiGLU rows: the oracle's dequant + swiglu_ffn (worker side)."""
    fmts, n_in, packs, xs = job
    W = {n: oracle.dequant(*fmts[n], n_in[n], *packs[n]) for n in ("w1", "w3", "w2")}
    return oracle.swiglu_ffn(W["w1"], W["w3"], W["w2"], xs)


def oracle_pool(workers=None):
    """A process pool for oracle work.  It uses the spawn start method (a
    worker forked from a process that has already used CUDA would hang) and
    raises, rather than waits, if a worker dies."""
    import multiprocessing as mp
    import os
    from concurrent.futures import ProcessPoolExecutor
    n = workers or max(1, min(16, len(os.sched_getaffinity(0))))
    return ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"))


def oracle_expert_rows(inp, jobs, pool=None, shared=False):
    """y rows of several experts: jobs = [(e, xs [n, d] fp64)], computed with
    the oracle's dequant and swiglu_ffn, in a spawn pool when one is given."""
    src = dict(zip(("w1", "w3", "w2"), inp.shared)) if shared else {"w1": inp.w1, "w3": inp.w3, "w2": inp.w2}
    fmts = {n: (m.fmt, m.bits, m.group) for n, m in src.items()}
    d = inp.cfg["d"]
    n_in = {"w1": d, "w3": d, "w2": src["w1"].n_out}
    work = [(fmts, n_in, {n: m.expert_numpy(e) for n, m in src.items()}, np.asarray(xs, np.float64))
            for e, xs in jobs]
    if pool is None:
        return [_expert_rows_job(j) for j in work]
    return list(pool.map(_expert_rows_job, work))


def oracle_outputs(inp, tokens, ids, w, pool=None):
    """The layer's fp64 outputs for `tokens` under routing (ids, w) [T, k]:
    every (token, slot) through its expert (oracle dequant + swiglu_ffn),
    then the oracle's combine (+ the shared expert)."""
    x = inp.x.float().cpu().numpy().astype(np.float64)
    tok = np.asarray(tokens, np.int64)
    ids = np.asarray(ids, np.int64)
    k = ids.shape[1]
    need = {}
    for a, t in enumerate(tok):
        for j in range(k):
            need.setdefault(int(ids[t, j]), []).append((a, j))
    experts = sorted(need)
    ys = oracle_expert_rows(inp, [(e, x[[tok[a] for a, _ in need[e]]]) for e in experts], pool)
    y = np.zeros((len(tok), k, inp.cfg["d"]))
    for e, ye in zip(experts, ys):
        for r, (a, j) in enumerate(need[e]):
            y[a, j] = ye[r]
    y_sh = None
    if inp.shared is not None:
        y_sh = oracle_expert_rows(inp, [(0, x[tok])], pool, shared=True)[0]
    return oracle.combine(y, np.asarray(w, np.float64)[tok], y_sh)
