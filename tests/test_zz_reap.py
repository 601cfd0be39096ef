"""REAP-pruned layers: routing over the surviving experts only.

DeepSeek-V4-Flash MLX quantisation notes, "REAP-pruned builds": the lowest
saliency routed experts are dropped from the learned-router layers (the
builds keep 192, 161 or 128 of 256), the router renormalises over the
survivors, and the hash-routed layers keep all 256.  A pruned layer is
therefore an ordinary layer over the survivors' router rows and packs (the
loader gives each layer its own expert count); no separate entry point is
needed.

CPU: a brute-force top-k over the survivors of the full 256-expert router
(pruned experts masked out, weights renormalised over the picks) gives the
oracle's routing of the compacted layer, mapped back through the survivor
list.  GPU: the CUDA path against the oracle at those expert counts (161 is
odd, so the last routing block and warp lanes are partly empty), on both
expert-FFN implementations.  Collected last: the other suites run first."""
import numpy as np
import pytest
import torch

import oracle
from synthetic import make_custom

KEPT = {"REAP25": 192, "REAP37": 161, "REAP50": 128}


def _brute_survivor_routing(x, W, b, k, survivors):
    """Per token: sqrtsoftplus score of every survivor, key = score + bias,
    the k largest keys (lower original index first on ties), weights =
    scores of the picks over their sum."""
    T = x.shape[0]
    ids = np.zeros((T, k), np.int64)
    w = np.zeros((T, k))
    for t in range(T):
        cand = []
        for e in survivors:
            logit = float(np.dot(x[t], W[e]))
            s = np.sqrt(np.logaddexp(logit, 0.0))
            cand.append((-(s + b[e]), e, s))
        cand.sort()
        pick = cand[:k]
        tot = sum(p[2] for p in pick)
        ids[t] = [p[1] for p in pick]
        w[t] = [p[2] / tot for p in pick]
    return ids, w


@pytest.mark.parametrize("build", list(KEPT))
def test_survivor_routing_is_the_compacted_layer(build):
    rng = np.random.default_rng(17)
    E, k, d, T = 256, 8, 64, 24
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((E, d)) * 0.3
    b = rng.standard_normal(E) * 0.05
    survivors = np.sort(rng.choice(E, KEPT[build], replace=False))
    ids_c, w_c, gap, _ = oracle.route_learned(x, W[survivors], b[survivors], k)
    ids_b, w_b = _brute_survivor_routing(x, W, b, k, survivors)
    ok = gap >= 1e-9
    assert ok.sum() >= T - 1
    assert np.array_equal(survivors[ids_c][ok], ids_b[ok])
    np.testing.assert_allclose(w_c[ok], w_b[ok], rtol=1e-12)
    assert not np.isin(ids_b, np.setdiff1d(np.arange(E), survivors)).any()


REAP_BASE = dict(d=512, k=8, f=384, routing="learned", vocab=0, w13=("affine", 4, 64), w2=("affine", 4, 64),
                 shared=None, f_shared=0, weight_std=0.02, router_std=0.05, bias_std=0.01)
GPU_CASES = {
    "REAP25_T1": dict(REAP_BASE, E=192, T=1, shared=("affine", 8, 64), f_shared=256, seed=601),
    "REAP37_T12": dict(REAP_BASE, E=161, T=12, seed=602),
    "REAP37_T37": dict(REAP_BASE, E=161, T=37, w13=("affine", 2, 128), w2=("affine", 3, 128), seed=603),
    "REAP50_T300": dict(REAP_BASE, E=128, T=300, seed=604),
}


@pytest.mark.gpu
@pytest.mark.parametrize("path", ["gemv", "tc"])
@pytest.mark.parametrize("name", list(GPU_CASES))
def test_pruned_expert_counts_match_oracle(cuda_device, name, path):
    import bit_quantized_moe_route_b200 as moe
    from tests.gpu_utils import check_layer, run_forward
    from tests.helpers import oracle_run
    moe.load_library()
    prev = moe.set_ffn_path(moe.FFN_GEMV if path == "gemv" else moe.FFN_TENSOR_CORE)
    try:
        inp = make_custom(GPU_CASES[name], cuda_device)
        res = oracle_run(inp)
        out, ids, w, ws = run_forward(inp)
    finally:
        moe.set_ffn_path(prev)
    check_layer(inp, res, out, ids, w, f"{name}/{path}")
    assert moe.read_device_error(ws) == 0
    assert int(torch.as_tensor(ids).max()) < inp.cfg["E"]
