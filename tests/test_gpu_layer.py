"""The resident-layer wrapper (MoELayer) vs the fp64 oracle.

One layer object holds the packed experts and a workspace sized for its
largest batch; it is then called with batches of several sizes (below and
above the tensor-core switch point).  Every token's output depends only on
that token's row of x under learned routing, so the oracle's rows for the
full batch are the expected values for every prefix of it."""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
from synthetic import make_custom
from tests.gpu_utils import check_layer
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

CFG = dict(T=96, d=512, E=16, k=4, f=384, routing="learned", vocab=0, w13=("affine", 4, 64),
           w2=("affine", 4, 64), shared=("affine", 8, 64), f_shared=256, weight_std=0.02, router_std=0.05,
           bias_std=0.01, seed=501)


def test_layer_object_matches_oracle_over_batch_sizes(cuda_device):
    inp = make_custom(CFG, cuda_device)
    c = inp.cfg
    res = oracle_run(inp)
    layer = moe.MoELayer(d_model=c["d"], d_ff=c["f"], n_experts=c["E"], top_k=c["k"], max_tokens=c["T"],
                         w1=inp.w1, w3=inp.w3, w2=inp.w2, router_w=inp.router_w, router_b=inp.router_b,
                         shared=inp.shared, device=cuda_device)
    for T in (2, 37, c["T"]):
        ids = torch.empty(T, c["k"], dtype=torch.int32, device=cuda_device)
        w = torch.empty(T, c["k"], dtype=torch.float32, device=cuda_device)
        out = layer(inp.x[:T], topk_ids=ids, topk_w=w)
        torch.cuda.synchronize()
        check_layer(inp, res, out, ids, w, f"layer T={T}", tokens=np.arange(T))
        assert layer.device_error() == 0


def test_layer_object_rejects_oversized_batch(cuda_device):
    inp = make_custom(dict(CFG, T=8), cuda_device)
    c = inp.cfg
    layer = moe.MoELayer(d_model=c["d"], d_ff=c["f"], n_experts=c["E"], top_k=c["k"], max_tokens=4,
                         w1=inp.w1, w3=inp.w3, w2=inp.w2, router_w=inp.router_w, router_b=inp.router_b,
                         shared=inp.shared, device=cuda_device)
    with pytest.raises(ValueError):
        layer(inp.x)
