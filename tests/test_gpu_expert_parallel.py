"""moe_forward_partial (expert parallelism on one GPU): each expert slice's
fp32 partial against the oracle's partial for the same slice (under the
GPU's routing, so near-tie tokens are not excused), the slices of a
partition adding up to the whole layer, the routing outputs identical to
moe_forward's, and the argument checks."""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
from synthetic import make_custom
from tests.gpu_utils import check_output, check_routing, dims_for, run_forward
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

B = dict(T=5, d=1024, E=16, k=4, f=1024, routing="learned", vocab=0, w13=("affine", 4, 64), w2=("affine", 4, 64),
         shared=("affine", 8, 64), f_shared=1024, weight_std=0.02, router_std=0.05, bias_std=0.01, seed=900)

CASES = {
    "learned_shared_T5": dict(B, seed=901),
    "learned_T1": dict(B, T=1, shared=None, f_shared=0, seed=902),
    "hash_mxfp4_T12": dict(B, T=12, E=32, k=8, routing="hash", vocab=400, w13=("mxfp4", 4, 32),
                           w2=("mxfp4", 4, 32), shared=None, f_shared=0, seed=903),
}


def _partial(inp, rng, include_shared, ws):
    c = inp.cfg
    dims = dims_for(inp)
    out = torch.empty(c["T"], c["d"], dtype=torch.float32, device=inp.x.device)
    ids = torch.empty(c["T"], c["k"], dtype=torch.int32, device=inp.x.device)
    w = torch.empty(c["T"], c["k"], dtype=torch.float32, device=inp.x.device)
    moe.forward_partial(dims, rng[0], rng[1], include_shared, inp.x, inp.token_ids, inp.router_w, inp.router_b,
                        inp.tid2eid, inp.w1, inp.w3, inp.w2, inp.shared, out, ws, topk_ids_out=ids, topk_w_out=w)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), ids, w


@pytest.mark.parametrize("name", list(CASES))
def test_slices_match_the_oracle_and_add_up(cuda_device, name):
    moe.load_library()
    inp = make_custom(CASES[name], cuda_device)
    E = inp.cfg["E"]
    full_out, full_ids, full_w, ws = run_forward(inp)
    res = oracle_run(inp)
    check_routing(res, full_ids, full_w, hash_mode=inp.cfg["routing"] == "hash")
    forced = None if inp.cfg["routing"] == "hash" else full_ids.cpu().numpy().astype(np.int64)
    cuts = [(0, 5), (5, 11), (11, E)]
    total = 0.0
    for i, rng in enumerate(cuts):
        part, ids, w = _partial(inp, rng, i == 0, ws)
        assert torch.equal(ids, full_ids) and torch.equal(w, full_w)
        ref = oracle_run(inp, forced_ids=forced, expert_range=rng, include_shared=i == 0)["out"]
        owned = ((full_ids >= rng[0]) & (full_ids < rng[1])).cpu().numpy()
        if not owned.any() and (i > 0 or inp.shared is None):
            assert not part.any()  # nothing owned: exact zero
        else:
            check_output(part, ref, f"{name} slice {rng}")
        total = total + part
    ref_full = oracle_run(inp, forced_ids=forced)["out"]
    check_output(total, ref_full, f"{name} sum of slices")
    # the layer's bf16 output is the rounding of (a different summation order of) the same sum
    np.testing.assert_allclose(full_out.float().cpu().numpy(), total, rtol=1e-2, atol=1e-3)
    assert moe.read_device_error(ws) == 0


def test_partial_arguments(cuda_device):
    moe.load_library()
    inp = make_custom(CASES["learned_T1"], cuda_device)
    ws = moe.alloc_workspace(dims_for(inp), cuda_device)
    E = inp.cfg["E"]
    for bad in ((-1, 4), (5, 4), (0, E + 1)):
        with pytest.raises(moe.MoEError):
            _partial(inp, bad, False, ws)
    # T above the fused path's limit: unsupported
    big = make_custom(dict(CASES["learned_T1"], T=40, seed=904), cuda_device)
    wsb = moe.alloc_workspace(dims_for(big), cuda_device)
    with pytest.raises(moe.MoEError, match="fused"):
        _partial(big, (0, E), True, wsb)
