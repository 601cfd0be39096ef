"""The fused mHC Sinkhorn mixing kernel (moe_hc_sinkhorn_mix) against the
oracle's hc_sinkhorn / hc_mix: P to 2e-6 absolute (fp32 iterations against
fp64), outputs within the layer's output tolerance, for several hc_mult
values, ragged widths, widths that need two passes, zero iterations, eps,
large logits, and the full 4096 x 4 x 4096 residual stream (sampled tokens)."""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
import oracle
from synthetic import HC_CONFIGS, make_hc_inputs
from tests.gpu_utils import check_output

pytestmark = pytest.mark.gpu

CASES = {
    "decode_n4": dict(HC_CONFIGS["mhc_decode"]),
    "T37_n4_eps": dict(T=37, n=4, d=1024, iters=20, eps=1e-6, logit_std=1.0, seed=61),
    "n2_d64": dict(T=5, n=2, d=64, iters=20, eps=0.0, logit_std=1.0, seed=62),
    "n3_ragged_d40": dict(T=9, n=3, d=40, iters=7, eps=0.0, logit_std=1.0, seed=63),
    "n8_two_passes": dict(T=3, n=8, d=8200, iters=20, eps=0.0, logit_std=1.0, seed=64),
    "n1": dict(T=4, n=1, d=128, iters=5, eps=0.0, logit_std=1.0, seed=65),
    "zero_iters": dict(T=6, n=4, d=256, iters=0, eps=0.0, logit_std=1.0, seed=66),
    "large_logits": dict(T=6, n=4, d=256, iters=20, eps=0.0, logit_std=30.0, seed=67),
    "many_iters": dict(T=6, n=5, d=256, iters=200, eps=1e-4, logit_std=2.0, seed=68),
}


def _run(inp, device):
    c = inp.cfg
    out = torch.empty_like(inp.h)
    P = torch.empty(c["T"], c["n"], c["n"], dtype=torch.float32, device=device)
    moe.hc_sinkhorn_mix(inp.logits, inp.h, out, c["iters"], c["eps"], P_out=P)
    torch.cuda.synchronize()
    return out, P


def _check(inp, out, P, tokens, label):
    c = inp.cfg
    L = inp.logits[tokens].cpu().double().numpy()
    h = inp.h[tokens].cpu().double().numpy()
    P_ref = oracle.hc_sinkhorn(L, c["iters"], c["eps"])
    np.testing.assert_allclose(P[tokens].cpu().double().numpy(), P_ref, atol=2e-6, rtol=0)
    ref = oracle.hc_mix(P_ref, h)
    return check_output(out[tokens].cpu().double().numpy(), ref, label)


@pytest.mark.parametrize("name", list(CASES))
def test_hc_sinkhorn_mix_matches_oracle(cuda_device, name):
    moe.load_library()
    inp = make_hc_inputs(CASES[name], cuda_device)
    out, P = _run(inp, cuda_device)
    stats = _check(inp, out, P, np.arange(inp.cfg["T"]), name)
    print(f"\n{name}: {stats}")


def test_hc_full_residual_stream(cuda_device):
    moe.load_library()
    inp = make_hc_inputs(HC_CONFIGS["mhc"], cuda_device)
    out, P = _run(inp, cuda_device)
    tok = np.array([0, 1, 1000, 2047, 3333, 4095])
    stats = _check(inp, out, P, tok, "mhc full")
    # every token's matrix is doubly stochastic to fp32 accuracy
    Pc = P.cpu().double().numpy()
    assert np.abs(Pc.sum(-1) - 1).max() < 1e-5 and np.abs(Pc.sum(-2) - 1).max() < 1e-2
    print(f"\nmhc full: {stats}")


def test_hc_rejects_bad_arguments(cuda_device):
    moe.load_library()
    h = torch.zeros(2, 9, 64, dtype=torch.bfloat16, device=cuda_device)
    L = torch.zeros(2, 9, 9, dtype=torch.float32, device=cuda_device)
    with pytest.raises(moe.MoEError) as ei:
        moe.hc_sinkhorn_mix(L, h, torch.empty_like(h), 20)
    assert ei.value.status == 2
    h = torch.zeros(2, 4, 12, dtype=torch.bfloat16, device=cuda_device)
    L = torch.zeros(2, 4, 4, dtype=torch.float32, device=cuda_device)
    with pytest.raises(moe.MoEError) as ei:
        moe.hc_sinkhorn_mix(L, h, torch.empty_like(h), 20)
    assert ei.value.status == 1
