"""Bridges between the synthetic inputs and the oracle / the CUDA library."""
from __future__ import annotations

import numpy as np

import oracle


def dims_of(inp):
    c = inp.cfg
    return dict(T=c["T"], d=c["d"], E=c["E"], k=c["k"], f=c["f"],
                f_shared=c.get("f_shared", 0) if inp.shared is not None else 0,
                routing=c["routing"])


def oracle_run(inp, tokens=None):
    """Run the fp64 oracle on MoEInputs (tensors may live on any device)."""
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
        tokens=tokens)


def bigint_words(codes, bits):
    """Pack codes into uint32 words via one Python big integer (test-side only)."""
    v = 0
    for i, c in enumerate(codes):
        v |= int(c) << (i * bits)
    nw = (len(codes) * bits + 31) // 32
    return np.array([(v >> (32 * w)) & 0xFFFFFFFF for w in range(nw)], dtype=np.uint32)
