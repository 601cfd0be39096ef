"""The GPU parity harness itself, on the CPU: near-tie tokens are checked,
not excused.  A planted near tie lets a stand-in for the GPU pick the other
(equally valid) expert; the harness must then accept its output against the
oracle's forced-routing run, and reject an output computed with the
oracle's own ids, a swap on a token that is not a near tie, and weights that
do not belong to the chosen ids."""
import numpy as np
import pytest
import torch

import oracle
from synthetic import CONFIGS, make_custom
from tests.gpu_utils import TIE_EPS, check_layer, check_routing
from tests.helpers import oracle_run


def _planted_tie():
    cfg = dict(CONFIGS["tiny"], T=5, seed=71, bias_std=0.02)
    inp = make_custom(cfg)
    res = oracle_run(inp)
    k = cfg["k"]
    t = 2
    order = np.argsort(-res["keys"][t], kind="stable")
    e_in, e_out = order[k - 1], order[k]
    b = inp.router_b.clone()
    # lift the (k+1)-th expert's key to 5e-5 below the k-th one (selection bias only)
    b[e_out] += float(res["keys"][t, e_in] - res["keys"][t, e_out]) - 5e-5
    inp.router_b = b
    res = oracle_run(inp)
    assert res["gap"][t] < TIE_EPS
    return inp, res, t


def _gpu_standin(inp, res, ids):
    """What a correct implementation would return for these ids: the oracle's
    forced-routing output rounded to bf16, and its weights in fp32."""
    f = oracle_run(inp, forced_ids=ids)
    out = torch.from_numpy(oracle.round_bf16(f["out"])).to(torch.bfloat16)
    return out, torch.from_numpy(ids.astype(np.int32)), torch.from_numpy(f["w"].astype(np.float32))


def test_near_tie_checked_under_forced_routing():
    inp, res, t = _planted_tie()
    k = inp.cfg["k"]
    ids = res["ids"].copy()
    order = np.argsort(-res["keys"][t], kind="stable")
    ids[t, k - 1] = order[k]          # the other side of the near tie
    out, ids_g, w_g = _gpu_standin(inp, res, ids)
    ties, stats = check_layer(inp, res, out, ids_g, w_g, "planted tie")
    assert t in ties and stats["max_err_over_rms"] < 1e-2


def test_near_tie_output_must_follow_its_own_ids():
    inp, res, t = _planted_tie()
    k = inp.cfg["k"]
    ids = res["ids"].copy()
    order = np.argsort(-res["keys"][t], kind="stable")
    ids[t, k - 1] = order[k]
    out_wrong, _, _ = _gpu_standin(inp, res, res["ids"])   # output of the oracle's ids
    _, ids_g, w_g = _gpu_standin(inp, res, ids)
    with pytest.raises(AssertionError):
        check_layer(inp, res, out_wrong, ids_g, w_g, "mismatched")


def test_swap_outside_a_near_tie_is_rejected():
    inp, res, t = _planted_tie()
    k = inp.cfg["k"]
    u = 0 if t != 0 else 1
    assert res["gap"][u] >= TIE_EPS
    ids = res["ids"].copy()
    order = np.argsort(-res["keys"][u], kind="stable")
    ids[u, k - 1] = order[k]
    out, ids_g, w_g = _gpu_standin(inp, res, ids)
    with pytest.raises(AssertionError):
        check_routing(res, ids_g, w_g)


def test_tie_weights_must_match_the_chosen_ids():
    inp, res, t = _planted_tie()
    k = inp.cfg["k"]
    ids = res["ids"].copy()
    order = np.argsort(-res["keys"][t], kind="stable")
    ids[t, k - 1] = order[k]
    _, ids_g, _ = _gpu_standin(inp, res, ids)
    w_bad = torch.from_numpy(res["w"].astype(np.float32))  # weights of the oracle's ids
    if np.allclose(res["w"][t], oracle_run(inp, forced_ids=ids)["w"][t], rtol=2e-5, atol=2e-6):
        pytest.skip("the two selections' weights coincide for this seed")
    with pytest.raises(AssertionError):
        check_routing(res, ids_g, w_bad)
