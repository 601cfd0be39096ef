"""The fused small-batch layer (one launch: routing, both FFN stages on the
integer tensor-core MMA, combine) against the oracle, with the path forced,
over every packed format and group size it takes, hash routing, experts
with more than 4 tokens (several token groups), the shared expert, bf16
router weights and a pruned expert count; plus run-to-run determinism, the
AUTO choice, the bounded-wait timeout and the error word on bad hash
data."""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
from synthetic import CONFIGS, make_custom
from tests.gpu_utils import check_layer, dims_for, run_forward
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

B = dict(T=5, d=1024, E=16, k=4, f=1024, routing="learned", vocab=0, w13=("affine", 4, 64), w2=("affine", 4, 64),
         shared=None, f_shared=0, weight_std=0.02, router_std=0.05, bias_std=0.01, seed=800)

VARIANTS = {
    "a4g64_T1": dict(B, T=1, seed=801),
    "a4g64_shared8_T1": dict(B, T=1, shared=("affine", 8, 64), f_shared=1024, seed=802),
    "a4g32_T5": dict(B, w13=("affine", 4, 32), w2=("affine", 4, 32), seed=803),
    "a4g128_T8": dict(B, T=8, w13=("affine", 4, 128), w2=("affine", 4, 128), seed=804),
    "a8g64_T3": dict(B, T=3, w13=("affine", 8, 64), w2=("affine", 8, 64), seed=805),
    "a8g32_T2": dict(B, T=2, w13=("affine", 8, 32), w2=("affine", 8, 32), seed=806),
    "a8_shared_g128_T2": dict(B, T=2, shared=("affine", 8, 64), f_shared=512, seed=807),
    "a2g128_a3g128_T8": dict(B, T=8, d=2048, w13=("affine", 2, 128), w2=("affine", 3, 128), seed=808),
    "a2g64_T4": dict(B, T=4, d=2048, f=2048, w13=("affine", 2, 64), w2=("affine", 2, 64), seed=809),
    "a3g64_T6": dict(B, T=6, w13=("affine", 3, 64), w2=("affine", 3, 64), seed=810),
    "mxfp4_hash_T32": dict(B, T=32, E=32, k=8, routing="hash", vocab=500, w13=("mxfp4", 4, 32),
                           w2=("mxfp4", 4, 32), seed=811),
    "mxfp4_learned_T9": dict(B, T=9, w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32), seed=812),
    "groups_over_8_tokens": dict(B, T=32, E=4, k=2, seed=813),
    "shared_narrower_T12": dict(B, T=12, shared=("affine", 8, 64), f_shared=512, seed=814),
    "tokens_4_per_group_T24": dict(B, T=24, E=8, k=2, seed=820),
    "shared_a4_T9": dict(B, T=9, shared=("affine", 4, 64), f_shared=1024, seed=815),
    "bf16_router_T7": dict(B, T=7, router_dtype="bf16", seed=816),
    "E161_k8_T20": dict(B, T=20, E=161, k=8, seed=817),
    "d2048_f1024_T32": dict(B, T=32, d=2048, f=1024, E=64, k=8, seed=818),
    "hash_shared_T16": dict(B, T=16, E=32, k=8, routing="hash", vocab=300, shared=("affine", 8, 64),
                            f_shared=1024, seed=819),
}


@pytest.fixture(scope="module")
def fused(cuda_device):
    moe.load_library()
    prev = moe.set_ffn_path(moe.FFN_DECODE_FUSED)
    yield cuda_device
    moe.set_ffn_path(prev)


@pytest.mark.parametrize("name", list(VARIANTS))
def test_fused_layer_matches_oracle(fused, name):
    inp = make_custom(VARIANTS[name], fused)
    res = oracle_run(inp)
    out, ids, w, ws = run_forward(inp)
    ties, stats = check_layer(inp, res, out, ids, w, name)
    assert moe.read_device_error(ws) == 0
    print(f"\n{name}: ties={len(ties)} {stats}")


def test_fused_layer_is_deterministic_and_reusable(fused):
    inp = make_custom(VARIANTS["a4g64_shared8_T1"], fused)
    out1, _, _, ws = run_forward(inp)
    outs = [run_forward(inp, ws=ws)[0] for _ in range(3)]
    for o in outs:
        assert torch.equal(o, out1)
    assert moe.read_device_error(ws) == 0


def test_auto_takes_the_fused_launch(cuda_device):
    moe.load_library()
    inp = make_custom(VARIANTS["a4g64_T1"], cuda_device)
    dims = dims_for(inp)
    ws = moe.alloc_workspace(dims, cuda_device)
    out = torch.empty(1, inp.cfg["d"], dtype=torch.bfloat16, device=cuda_device)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    keep = moe.set_timing_events(evs)
    moe.forward(dims, inp.x, None, inp.router_w, inp.router_b, None, inp.w1, inp.w3, inp.w2, None, out, ws)
    torch.cuda.synchronize()
    assert moe.timing_labels() == ["decode_fused"]
    del keep


def test_fused_rejects_shapes_it_does_not_take(fused):
    inp = make_custom(dict(CONFIGS["tiny"]), fused)     # d_model = 256 is not a multiple of the 4-bit stage
    with pytest.raises(moe.MoEError) as ei:
        run_forward(inp)
    assert ei.value.status == 2


def test_fused_bad_hash_data_sets_error_word(fused):
    inp = make_custom(VARIANTS["mxfp4_hash_T32"], fused)
    good = oracle_run(inp)
    tok = inp.token_ids.clone()
    tok[3] = 10_000
    bad = type(inp)(**{**inp.__dict__, "token_ids": tok})
    out, ids, w, ws = run_forward(bad)
    assert moe.read_device_error(ws) == 6
    assert torch.all(w[3] == 0)
    keep = [t for t in range(inp.cfg["T"]) if t != 3]
    from tests.gpu_utils import bf16_to_np, check_output
    check_output(bf16_to_np(out)[keep], good["out"][keep], "bad hash token")
    assert torch.all(out[3] == 0)


def test_bounded_wait_times_out_and_recovers(fused):
    """A wait that nothing completes (the test hook) gives up within its short
    limit: the call reports MOE_ERR_TIMEOUT through the error word, the
    context stays usable and the next call on the same workspace is right."""
    inp = make_custom(VARIANTS["a4g64_shared8_T1"], fused)
    lib = moe.load_library()
    prev = lib.moe_test_stall_fused_wait(1)
    try:
        _, _, _, ws = run_forward(inp)
        assert moe.read_device_error(ws) == 5
    finally:
        lib.moe_test_stall_fused_wait(prev)
    out, ids, w, _ = run_forward(inp, ws=ws)
    res = oracle_run(inp)
    check_layer(inp, res, out, ids, w, "after a timed-out call")
    assert moe.read_device_error(ws) == 0
