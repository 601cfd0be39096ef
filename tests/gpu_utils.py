"""Helpers for the GPU parity tests: run the CUDA library on MoEInputs and
compare with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import bit_quantized_moe_route_b200 as moe
import oracle

TIE_EPS = 1e-4           # top-k near-tie gap (oracle keys) excused from id equality
MAX_ERR_OVER_RMS = 2e-2  # max|out-ref| <= 2e-2 * rms(ref)
MEAN_REL_ERR = 5e-3      # sum|out-ref| / sum|ref| <= 5e-3


def dims_for(inp, T=None):
    c = inp.cfg
    return moe.make_dims(T or c["T"], c["d"], c["f"], c["E"], c["k"], c["routing"] == "hash",
                         c.get("vocab", 0) if c["routing"] == "hash" else 0,
                         c["f_shared"] if inp.shared is not None else 0)


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


def check_routing(res, ids_gpu, w_gpu, hash_mode=False):
    """Bit-exact ids except tokens whose k-th/(k+1)-th oracle key gap < TIE_EPS.

    Returns the list of near-tie tokens (excused from id equality and from the
    output comparison).
    """
    ids_gpu = ids_gpu.cpu().numpy().astype(np.int64)
    w_gpu = w_gpu.cpu().numpy().astype(np.float64)
    gap = res["gap"]
    tie = np.nonzero(gap < TIE_EPS)[0]
    ok = gap >= TIE_EPS
    assert np.array_equal(ids_gpu[ok], res["ids"][ok]), np.nonzero((ids_gpu != res["ids"]).any(1) & ok)
    np.testing.assert_allclose(w_gpu[ok], res["w"][ok], rtol=2e-5, atol=2e-6)
    assert np.allclose(w_gpu.sum(1), 1.0, atol=1e-5)
    return tie.tolist()


def check_output(out_gpu, ref, label=""):
    stats = oracle.parity_stats(out_gpu, ref)
    assert stats["max_err_over_rms"] <= MAX_ERR_OVER_RMS, (label, stats)
    assert stats["mean_rel_err"] <= MEAN_REL_ERR, (label, stats)
    return stats


def bf16_to_np(t):
    return t.float().cpu().numpy().astype(np.float64)
