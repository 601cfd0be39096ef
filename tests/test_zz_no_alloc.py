"""The allocation-free expert FFN entry point (moe_expert_ffn_noalloc).

It serves callers that cannot allocate device memory; its scratch is a fixed
static device array.  This file is collected last so that a run stopping at
the first failure has already run every other test.  Each case compares the
new entry point with moe_expert_ffn (which uses a caller workspace) on the
same inputs, twice in a row, so the second call also checks that leftover
contents of the shared static array do not leak into results.  The
allocation-free entry point always runs the weight-streaming GEMV, so
moe_expert_ffn is run with that path selected for the bitwise comparison.
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
from synthetic import CONFIGS, make_custom
from tests.gpu_utils import check_output, dims_for
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": dict(CONFIGS["tiny"]),
    "small_mixed_bits": dict(T=37, d=512, E=16, k=4, f=384, routing="learned", vocab=0, w13=("affine", 2, 128),
                             w2=("affine", 3, 128), shared=None, f_shared=0, weight_std=0.02, router_std=0.05,
                             bias_std=0.01, seed=401),
    "hash_mxfp4": dict(CONFIGS["tiny"], routing="hash", vocab=300, T=24, w13=("mxfp4", 4, 32),
                       w2=("mxfp4", 4, 32), seed=402),
}


def _routing(inp, device):
    res = oracle_run(inp)
    E = inp.cfg["E"]
    offs = torch.from_numpy(res["expert_offsets"].astype(np.int32)).to(device)
    rows = torch.from_numpy(res["sorted_rows"].astype(np.int32)).to(device)
    return res, offs, rows


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_point(cuda_device, name):
    inp = make_custom(CASES[name], cuda_device)
    c = inp.cfg
    res, offs, rows = _routing(inp, cuda_device)
    dims = dims_for(inp)
    ws = moe.alloc_workspace(dims, cuda_device)
    n = c["T"] * c["k"]
    y_ws = torch.empty(n, c["d"], dtype=torch.float32, device=cuda_device)
    prev = moe.set_ffn_path(moe.FFN_GEMV)
    try:
        moe.expert_ffn(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y_ws, ws)
    finally:
        moe.set_ffn_path(prev)
    y_ref = res["y_slots"].reshape(n, c["d"])[res["sorted_rows"]]
    for call in range(2):
        y_na = torch.full((n, c["d"]), float("nan"), dtype=torch.float32, device=cuda_device)
        moe.expert_ffn_noalloc(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y_na)
        torch.cuda.synchronize()
        got = y_na.cpu().double().numpy()
        check_output(got, y_ws.cpu().double().numpy(), f"{name} call {call}")
        assert np.array_equal(got, y_ws.cpu().double().numpy()), f"{name} call {call}: differs from moe_expert_ffn"
        check_output(got, y_ref, f"{name} call {call} vs oracle")


def test_noalloc_rejects_oversized_problem(cuda_device):
    dims = moe.make_dims(4096, 4096, 2048, 256, 8)
    inp = make_custom(CASES["tiny"], cuda_device)
    offs = torch.zeros(257, dtype=torch.int32, device=cuda_device)
    rows = torch.zeros(4096 * 8, dtype=torch.int32, device=cuda_device)
    y = torch.empty(8, 256, dtype=torch.float32, device=cuda_device)
    with pytest.raises(moe.MoEError) as ei:
        moe.expert_ffn_noalloc(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y)
    assert ei.value.status == 2 and "scratch" in str(ei.value)


def test_noalloc_error_word_is_readable(cuda_device):
    """The static scratch's error word: clean after a correct call, set by a
    permutation that fails its check (no expert runs then), cleared by the
    read."""
    inp = make_custom(CASES["tiny"], cuda_device)
    c = inp.cfg
    res, offs, rows = _routing(inp, cuda_device)
    dims = dims_for(inp)
    n = c["T"] * c["k"]
    y = torch.empty(n, c["d"], dtype=torch.float32, device=cuda_device)
    moe.expert_ffn_noalloc(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y)
    assert moe.read_noalloc_error() == 0
    bad_rows = rows.clone()
    bad_rows[1] = n + 5
    y_bad = torch.full((n, c["d"]), 3.0, dtype=torch.float32, device=cuda_device)
    moe.expert_ffn_noalloc(dims, inp.x, offs, bad_rows, inp.w1, inp.w3, inp.w2, y_bad)
    assert moe.read_noalloc_error() == 6
    assert torch.all(y_bad == 3.0)
    assert moe.read_noalloc_error() == 0
    moe.expert_ffn_noalloc(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y_bad)
    assert moe.read_noalloc_error() == 0
    assert torch.equal(y_bad, y)
