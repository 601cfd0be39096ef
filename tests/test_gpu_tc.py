"""Tensor-core expert FFN (tcgen05 grouped GEMM) vs the fp64 oracle.

The path is forced with moe.set_ffn_path so that small cases the oracle
finishes in seconds still exercise it: ragged tiles (1..128 tokens, several
tiles per expert, empty experts), several weight-row and k tiles, every
packed format, the shared expert, hash routing, and the fp16 range check."""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
from synthetic import CONFIGS, make_custom
from tests.gpu_utils import bf16_to_np, check_layer, check_output, check_routing, dims_for, run_forward
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

BASE = dict(T=300, d=512, E=8, k=2, f=384, routing="learned", vocab=0, w13=("affine", 4, 64),
            w2=("affine", 4, 64), shared=None, f_shared=0, weight_std=0.02, router_std=0.05,
            bias_std=0.01, seed=201)

TC_VARIANTS = {
    "tiny": dict(CONFIGS["tiny"]),                                   # 1-2 tokens per tile
    "a4g64_ragged": BASE,                                            # ~75 tokens per expert
    "multi_tile": dict(BASE, T=520, E=4, d=256, f=256, seed=202),    # ~260 per expert: 3 tiles each
    "a8g64": dict(BASE, w13=("affine", 8, 64), w2=("affine", 8, 64), seed=203),
    "a2g128_a3g128": dict(BASE, w13=("affine", 2, 128), w2=("affine", 3, 128), seed=204),
    "a3g64_a2g64": dict(BASE, w13=("affine", 3, 64), w2=("affine", 2, 64), seed=205),
    "mxfp4": dict(BASE, w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32), seed=206),
    "a4g32": dict(BASE, w13=("affine", 4, 32), w2=("affine", 4, 32), seed=207),
    "a4g128_a8g32": dict(BASE, w13=("affine", 4, 128), w2=("affine", 8, 32), seed=208),
    "shared8": dict(BASE, T=200, shared=("affine", 8, 64), f_shared=256, seed=209),
    "hash_mxfp4": dict(BASE, T=200, routing="hash", vocab=700, w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32),
                       seed=210),
    "skewed": dict(BASE, T=256, E=32, k=4, bias_std=2.0, seed=211),  # empty and heavy experts
    "T1": dict(BASE, T=1, seed=212),
    "wide": dict(BASE, T=160, d=1024, f=1024, seed=213),             # 16 k-tiles per stage
    # shapes whose scale rows are whole 16-byte TMA boxes take the TMA/TMEM
    # kernel in both stages (the ones above mix it with the per-thread-copy one)
    "tma_a8g64": dict(BASE, T=200, d=1024, f=1024, w13=("affine", 8, 64), w2=("affine", 8, 64), seed=230),
    "tma_a2g128": dict(BASE, T=200, d=1024, f=1024, w13=("affine", 2, 128), w2=("affine", 2, 128), seed=231),
    "tma_mxfp4": dict(BASE, T=200, d=1024, f=1024, w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32), seed=232),
    "tma_a4g32_partial_slot": dict(BASE, T=150, d=768, f=768, w13=("affine", 4, 32), w2=("affine", 4, 32),
                                   seed=233),                          # 12 k-tiles: slots of 8 + 4
    "tma_a4g128_a8g32": dict(BASE, T=200, d=1024, f=1024, w13=("affine", 4, 128), w2=("affine", 8, 32), seed=234),
    "tma_shared8": dict(BASE, T=200, d=1024, f=512, shared=("affine", 8, 64), f_shared=512, seed=235),
    "tma_big_experts": dict(BASE, T=600, E=4, d=512, f=512, seed=236),  # ~300 tokens per expert: 192 + rest
    "tma_a3g128": dict(BASE, T=200, d=1024, f=1024, w13=("affine", 3, 128), w2=("affine", 3, 128), seed=237),
    "tma_bf16_router": dict(BASE, T=300, d=1024, f=1024, router_dtype="bf16", seed=238),
}


@pytest.fixture(scope="module")
def device(cuda_device):
    moe.load_library()
    prev = moe.set_ffn_path(moe.FFN_TENSOR_CORE)
    yield cuda_device
    moe.set_ffn_path(prev)


@pytest.mark.parametrize("name", list(TC_VARIANTS))
def test_tc_forward_matches_oracle(device, name):
    inp = make_custom(TC_VARIANTS[name], device)
    res = oracle_run(inp)
    out, ids, w, ws = run_forward(inp)
    check_layer(inp, res, out, ids, w, name)
    assert moe.read_device_error(ws) == 0


@pytest.mark.parametrize("name", ["a4g64_ragged", "multi_tile", "mxfp4", "a2g128_a3g128"])
def test_tc_expert_ffn_on_oracle_permutation(device, name):
    """moe_expert_ffn alone, fed the oracle's permutation: y per sorted slot."""
    inp = make_custom(TC_VARIANTS[name], device)
    c = inp.cfg
    T, k, E, d = c["T"], c["k"], c["E"], c["d"]
    res = oracle_run(inp)
    dims = dims_for(inp)
    ws = moe.alloc_workspace(dims, device)
    offs = torch.from_numpy(res["expert_offsets"].astype(np.int32)).to(device)
    rows = torch.from_numpy(res["sorted_rows"].astype(np.int32)).to(device)
    y = torch.empty(T * k, d, dtype=torch.float32, device=device)
    moe.expert_ffn(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y, ws)
    torch.cuda.synchronize()
    y_ref = res["y_slots"].reshape(T * k, d)[res["sorted_rows"]]
    check_output(y.cpu().double().numpy(), y_ref, name + ":ffn")
    assert moe.read_device_error(ws) == 0


def test_tc_deterministic(device):
    inp = make_custom(TC_VARIANTS["multi_tile"], device)
    a = run_forward(inp)[0].clone()
    b = run_forward(inp)[0]
    assert torch.equal(a, b)


def test_tc_matches_gemv_path(device):
    """Both implementations of step 3 on one input stay within the tolerance of each other's oracle."""
    inp = make_custom(TC_VARIANTS["a4g64_ragged"], device)
    res = oracle_run(inp)
    out_tc = bf16_to_np(run_forward(inp)[0])
    moe.set_ffn_path(moe.FFN_GEMV)
    try:
        out_gemv = bf16_to_np(run_forward(inp)[0])
    finally:
        moe.set_ffn_path(moe.FFN_TENSOR_CORE)
    check_output(out_tc, res["out"], "tc")
    check_output(out_gemv, res["out"], "gemv")


def test_tc_flags_fp16_overflow(device):
    """An activation beyond the fp16 range is reported, not silently rounded."""
    inp = make_custom(TC_VARIANTS["tiny"], device)
    inp.x[1, 7] = 1.0e5
    out, ids, w, ws = run_forward(inp)
    assert moe.read_device_error(ws) == 6  # MOE_ERR_DEVICE_INPUT


def test_auto_picks_tc_from_four_tokens(device):
    """AUTO uses the tensor-core kernels from T = 4 up (timing labels show which ran)."""
    moe.set_ffn_path(moe.FFN_AUTO)
    try:
        for T, want in ((1, False), (3, False), (4, True), (512, True)):
            inp = make_custom(dict(BASE, T=T, seed=220), device)
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(16)]
            keep = moe.set_timing_events(evs)
            run_forward(inp)
            torch.cuda.synchronize()
            del keep
            assert ("tile_plan" in moe.timing_labels()) == want, (T, moe.timing_labels())
    finally:
        moe.set_ffn_path(moe.FFN_TENSOR_CORE)
