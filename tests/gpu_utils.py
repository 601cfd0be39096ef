"""Helpers for the GPU parity tests: run the CUDA library on MoEInputs and
compare with the oracle under the stated tolerances.

Near-tie tokens (k-th and (k+1)-th oracle keys closer than TIE_EPS) are not
excused from anything: their GPU ids must form a valid top-k within TIE_EPS,
their weights must match the oracle's forced-routing weights for those ids,
and their outputs are compared against the oracle run in forced-routing mode
with the GPU's own ids."""
from __future__ import annotations

import numpy as np
import torch

import bit_quantized_moe_route_b200 as moe
import oracle
from tests.helpers import oracle_run

TIE_EPS = 1e-4           # top-k near-tie gap (oracle keys): ids may differ from the oracle's there
MAX_ERR_OVER_RMS = 2e-2  # max|out-ref| <= 2e-2 * rms(ref)
MEAN_REL_ERR = 5e-3      # sum|out-ref| / sum|ref| <= 5e-3


def dims_for(inp, T=None):
    c = inp.cfg
    return moe.make_dims(T or c["T"], c["d"], c["f"], c["E"], c["k"], c["routing"] == "hash",
                         c.get("vocab", 0) if c["routing"] == "hash" else 0,
                         c["f_shared"] if inp.shared is not None else 0,
                         router_dtype=None if inp.router_w is None else inp.router_w.dtype)


def run_forward(inp, ws=None):
    """moe_forward on device inputs; returns (out bf16, ids, w, ws)."""
    c = inp.cfg
    dims = dims_for(inp)
    if ws is None:
        ws = moe.alloc_workspace(dims, inp.x.device)
    out = torch.empty(c["T"], c["d"], dtype=torch.bfloat16, device=inp.x.device)
    ids = torch.empty(c["T"], c["k"], dtype=torch.int32, device=inp.x.device)
    w = torch.empty(c["T"], c["k"], dtype=torch.float32, device=inp.x.device)
    moe.forward(dims, inp.x, inp.token_ids, inp.router_w, inp.router_b, inp.tid2eid, inp.w1, inp.w3, inp.w2,
                inp.shared, out, ws, topk_ids_out=ids, topk_w_out=w)
    torch.cuda.synchronize()
    return out, ids, w, ws


def _np(a, dtype):
    return (a.cpu().numpy() if isinstance(a, torch.Tensor) else np.asarray(a)).astype(dtype)


def check_routing(res, ids_gpu, w_gpu, hash_mode=False):
    """Bit-exact ids for every token whose k-th/(k+1)-th oracle key gap is at
    least TIE_EPS.  For the other (near-tie) tokens the GPU's ids must be a
    valid top-k within TIE_EPS: every selected key >= every unselected key -
    TIE_EPS, with k distinct ids.  Weights: the oracle's for the same ids
    (its forced-routing weights on near-tie tokens), to 2e-5.

    Returns the list of near-tie tokens."""
    ids_gpu = _np(ids_gpu, np.int64)
    w_gpu = _np(w_gpu, np.float64)
    T = ids_gpu.shape[0]
    gap = res["gap"][:T]
    tie = np.nonzero(gap < TIE_EPS)[0]
    ok = gap >= TIE_EPS
    assert np.array_equal(ids_gpu[ok], res["ids"][:T][ok]), np.nonzero((ids_gpu != res["ids"][:T]).any(1) & ok)
    w_ref = res["w"][:T].copy()
    if len(tie):
        keys = res["keys"][:T]
        L = res["logits"][:T]
        s = oracle.sqrtsoftplus(L)
        for t in tie:
            sel = ids_gpu[t]
            assert len(set(sel.tolist())) == len(sel), (t, sel)
            rest = np.setdiff1d(np.arange(keys.shape[1]), sel)
            if len(rest):
                assert keys[t, sel].min() >= keys[t, rest].max() - TIE_EPS, (t, sel)
            w_ref[t] = oracle.renormalize(s[t, sel][None, :])[0]
    np.testing.assert_allclose(w_gpu, w_ref, rtol=2e-5, atol=2e-6)
    assert np.allclose(w_gpu.sum(1), 1.0, atol=1e-5)
    return tie.tolist()


def reference_outputs(inp, res, ids_gpu, tokens=None):
    """The oracle's fp64 outputs for `tokens` (default: res's tokens) under
    the GPU's routing: res itself when the GPU chose the oracle's ids for
    every token, else the oracle in forced-routing mode with the GPU's ids."""
    ids_gpu = _np(ids_gpu, np.int64)
    T = ids_gpu.shape[0]
    tok = res["tokens"] if tokens is None else np.asarray(tokens, np.int64)
    if np.array_equal(ids_gpu, res["ids"][:T]):
        pos = {int(t): a for a, t in enumerate(res["tokens"])}
        return res["out"][[pos[int(t)] for t in tok]]
    forced = res["ids"].copy()
    forced[:T] = ids_gpu
    return oracle_run(inp, tokens=tok, forced_ids=forced)["out"]


def check_layer(inp, res, out_gpu, ids_gpu, w_gpu, label="", tokens=None):
    """Routing (check_routing) and every requested token's output (no token
    excused).  out_gpu: bf16 [T, d] on the device or fp64 rows [T, d].
    Returns (near-tie tokens, output statistics)."""
    hash_mode = inp.cfg["routing"] == "hash"
    ties = check_routing(res, ids_gpu, w_gpu, hash_mode=hash_mode)
    tok = res["tokens"] if tokens is None else np.asarray(tokens, np.int64)
    ref = reference_outputs(inp, res, ids_gpu, tok)
    got = bf16_to_np(out_gpu) if isinstance(out_gpu, torch.Tensor) else np.asarray(out_gpu, np.float64)
    stats = check_output(got[tok], ref, label)
    return ties, stats


def check_output(out_gpu, ref, label=""):
    stats = oracle.parity_stats(out_gpu, ref)
    assert stats["max_err_over_rms"] <= MAX_ERR_OVER_RMS, (label, stats)
    assert stats["mean_rel_err"] <= MEAN_REL_ERR, (label, stats)
    return stats


def bf16_to_np(t):
    return t.float().cpu().numpy().astype(np.float64)
