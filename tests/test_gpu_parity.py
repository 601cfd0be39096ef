"""CUDA path vs the fp64 oracle on seeded inputs small enough for the oracle
to finish in seconds, spanning several row blocks and ragged token counts;
both the whole layer and each C-ABI step."""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
from synthetic import CONFIGS, make_custom, make_inputs
from tests.gpu_utils import bf16_to_np, check_layer, check_output, check_routing, dims_for, run_forward
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

SMALL = dict(T=37, d=512, E=16, k=4, f=384, routing="learned", vocab=0, w13=("affine", 4, 64),
             w2=("affine", 4, 64), shared=None, f_shared=0, weight_std=0.02, router_std=0.05,
             bias_std=0.01, seed=101)

VARIANTS = {
    "tiny": dict(CONFIGS["tiny"]),
    "small_a4g64": SMALL,
    "small_a4g128": dict(SMALL, w13=("affine", 4, 128), w2=("affine", 4, 128), seed=102),
    "small_a8g64": dict(SMALL, w13=("affine", 8, 64), w2=("affine", 8, 32), seed=103),
    "small_a2g128_a3g128": dict(SMALL, w13=("affine", 2, 128), w2=("affine", 3, 128), seed=104),
    "small_a3g64_a2g64": dict(SMALL, w13=("affine", 3, 64), w2=("affine", 2, 64), seed=105),
    "small_mxfp4": dict(SMALL, w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32), seed=106),
    "small_shared8": dict(SMALL, shared=("affine", 8, 64), f_shared=256, seed=107),
    "small_hash": dict(SMALL, routing="hash", vocab=1000, w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32), seed=108),
    "small_hash_affine": dict(SMALL, routing="hash", vocab=333, seed=109, T=64),
    "small_T1": dict(SMALL, T=1, seed=110),
    "wide_chunks": dict(SMALL, d=1024, f=1408, T=9, seed=111),       # 32 and 44 chunks per row
    "odd_chunks": dict(SMALL, d=96, f=160, T=13, w13=("affine", 4, 32), w2=("affine", 4, 32), seed=112),
    "many_tokens": dict(SMALL, T=300, E=8, k=2, d=256, f=128, seed=113),
    "k1_E1": dict(SMALL, T=5, E=1, k=1, seed=114),
    # widths of 1024+ inputs take the bulk-copy streaming GEMV
    "stream_a4g64_T37": dict(SMALL, d=1024, f=1024, seed=120),
    "stream_a4g64_T5": dict(SMALL, d=1024, f=1024, T=5, seed=121),
    "stream_T1_shared8": dict(SMALL, d=1024, f=1024, T=1, shared=("affine", 8, 64), f_shared=1024, seed=122),
    "stream_T2_a2g128_a3g128": dict(SMALL, d=1024, f=1024, T=2, w13=("affine", 2, 128), w2=("affine", 3, 128),
                                    seed=123),
    "stream_a8g64_T12": dict(SMALL, d=1024, f=2048, T=12, w13=("affine", 8, 64), w2=("affine", 8, 64), seed=124),
    "stream_hash_mxfp4": dict(SMALL, d=2048, f=1024, T=20, routing="hash", vocab=500, w13=("mxfp4", 4, 32),
                              w2=("mxfp4", 4, 32), seed=125),
    "stream_shared_wider": dict(SMALL, d=2048, f=1024, T=9, shared=("affine", 8, 128), f_shared=2048, seed=126),
    "stream_a4g32": dict(SMALL, d=1024, f=1024, T=3, w13=("affine", 4, 32), w2=("affine", 4, 32), seed=127),
    "stream_a2g64_a3g64": dict(SMALL, d=1024, f=1024, T=7, w13=("affine", 2, 64), w2=("affine", 3, 64), seed=128),
    "stream_many_per_expert": dict(SMALL, d=1024, f=1024, T=40, E=4, k=2, seed=129),
    "bf16_router": dict(SMALL, router_dtype="bf16", seed=130),
    "bf16_router_T1_d4096": dict(SMALL, T=1, d=4096, f=1024, E=64, k=8, router_dtype="bf16", seed=131),
    "bf16_router_hash": dict(SMALL, routing="hash", vocab=300, T=11, router_dtype="bf16", seed=132),
}


@pytest.fixture(scope="module")
def device(cuda_device):
    """These cases cover the weight-streaming GEMV path (the tensor-core path
    has its own file), so the module forces it."""
    moe.load_library()
    prev = moe.set_ffn_path(moe.FFN_GEMV)
    yield cuda_device
    moe.set_ffn_path(prev)


@pytest.mark.parametrize("name", list(VARIANTS))
def test_forward_matches_oracle(device, name):
    inp = make_custom(VARIANTS[name], device)
    res = oracle_run(inp)
    out, ids, w, ws = run_forward(inp)
    check_layer(inp, res, out, ids, w, name)
    assert moe.read_device_error(ws) == 0


@pytest.mark.parametrize("name", ["tiny", "small_a4g64", "small_a2g128_a3g128", "small_mxfp4", "many_tokens"])
def test_steps_match_oracle(device, name):
    """Each ABI step fed with the oracle's own upstream results."""
    inp = make_custom(VARIANTS[name], device)
    c = inp.cfg
    T, k, E, d = c["T"], c["k"], c["E"], c["d"]
    res = oracle_run(inp)
    dims = dims_for(inp)
    ws = moe.alloc_workspace(dims, device)
    # route
    ids = torch.empty(T, k, dtype=torch.int32, device=device)
    w = torch.empty(T, k, dtype=torch.float32, device=device)
    moe.route(dims, inp.x, inp.router_w, inp.router_b, inp.token_ids, inp.tid2eid, ids, w, ws)
    torch.cuda.synchronize()
    check_routing(res, ids, w)
    # permute the oracle's ids: bit-exact
    ids_o = torch.from_numpy(res["ids"].astype(np.int32)).to(device)
    offs = torch.empty(E + 1, dtype=torch.int32, device=device)
    rows = torch.empty(T * k, dtype=torch.int32, device=device)
    inv = torch.empty(T * k, dtype=torch.int32, device=device)
    moe.permute(dims, ids_o, offs, rows, inv, ws)
    torch.cuda.synchronize()
    assert np.array_equal(offs.cpu().numpy(), res["expert_offsets"])
    assert np.array_equal(rows.cpu().numpy(), res["sorted_rows"])
    assert np.array_equal(inv.cpu().numpy(), res["inv"])
    # expert FFN on the oracle's permutation
    y = torch.empty(T * k, d, dtype=torch.float32, device=device)
    moe.expert_ffn(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y, ws)
    torch.cuda.synchronize()
    y_ref = res["y_slots"].reshape(T * k, d)[res["sorted_rows"]]
    check_output(y.cpu().double().numpy(), y_ref, name + ":ffn")
    # combine the oracle's expert outputs (fp32) with the oracle weights
    y_o = torch.from_numpy(y_ref.astype(np.float32)).to(device)
    w_o = torch.from_numpy(res["w"].astype(np.float32)).to(device)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=device)
    moe.combine(dims, y_o, inv, w_o, None, out)
    torch.cuda.synchronize()
    ref = res["out"]
    got = bf16_to_np(out)
    # only fp32 rounding of y/w and one bf16 rounding separate the two
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2 ** -8 + 1e-6)


def test_permute_edge_cases(device):
    """All pairs on one expert; every expert once; empty experts in between."""
    for T, k, E, pattern in ((64, 1, 8, "one"), (16, 16, 16, "all"), (33, 3, 200, "sparse")):
        if pattern == "one":
            ids = np.full((T, k), 5)
        elif pattern == "all":
            ids = np.stack([np.roll(np.arange(E), t)[:k] for t in range(T)])
        else:
            rng = np.random.default_rng(1)
            ids = np.stack([rng.choice([3, 77, 199], size=k, replace=False) for _ in range(T)])
        dims = moe.make_dims(T, 256, 128, E, k)
        ws = moe.alloc_workspace(dims, device)
        ids_d = torch.from_numpy(ids.astype(np.int32)).to(device)
        offs = torch.empty(E + 1, dtype=torch.int32, device=device)
        rows = torch.empty(T * k, dtype=torch.int32, device=device)
        inv = torch.empty(T * k, dtype=torch.int32, device=device)
        moe.permute(dims, ids_d, offs, rows, inv, ws)
        torch.cuda.synchronize()
        import oracle
        o_off, o_rows, o_inv = oracle.permute(ids, E)
        assert np.array_equal(offs.cpu().numpy(), o_off)
        assert np.array_equal(rows.cpu().numpy(), o_rows)
        assert np.array_equal(inv.cpu().numpy(), o_inv)


def test_large_permutation_bit_exact(device):
    """T*k = 32768 pairs (prefill size), skewed expert loads."""
    rng = np.random.default_rng(5)
    T, k, E = 4096, 8, 256
    p = np.exp(rng.normal(0, 1.0, E))
    p /= p.sum()
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)])
    dims = moe.make_dims(T, 4096, 2048, E, k)
    ws = moe.alloc_workspace(dims, device)
    offs = torch.empty(E + 1, dtype=torch.int32, device=device)
    rows = torch.empty(T * k, dtype=torch.int32, device=device)
    inv = torch.empty(T * k, dtype=torch.int32, device=device)
    moe.permute(dims, torch.from_numpy(ids.astype(np.int32)).to(device), offs, rows, inv, ws)
    torch.cuda.synchronize()
    import oracle
    o_off, o_rows, o_inv = oracle.permute(ids, E)
    assert np.array_equal(offs.cpu().numpy(), o_off)
    assert np.array_equal(rows.cpu().numpy(), o_rows)
    assert np.array_equal(inv.cpu().numpy(), o_inv)


FUSED_HOST = dict(T=1, d=1024, E=16, k=4, f=1024, routing="learned", vocab=0, w13=("affine", 4, 64),
                  w2=("affine", 4, 64), shared=("affine", 8, 64), f_shared=1024, weight_std=0.02, router_std=0.05,
                  bias_std=0.01, seed=830)


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("layer", ["tiny", "fused"])
def test_forward_host_matches_device_path(device, layer, pinned):
    """Host buffers in and out: pinned (mapped) output is written directly by
    the layer's last kernel, pageable output is copied back; both equal the
    device-pointer call bit for bit."""
    inp = make_inputs("tiny", device) if layer == "tiny" else make_custom(FUSED_HOST, device)
    prev = moe.set_ffn_path(moe.FFN_DECODE_FUSED) if layer == "fused" else None  # this thread only
    try:
        out, _, _, ws = run_forward(inp)
        dims = dims_for(inp)
        x_h = inp.x.cpu().pin_memory()
        out_h = torch.full((inp.cfg["T"], inp.cfg["d"]), float("nan"), dtype=torch.bfloat16)
        if pinned:
            out_h = out_h.pin_memory()
        moe.forward_host(dims, x_h, None, inp.router_w, inp.router_b, None, inp.w1, inp.w3, inp.w2, inp.shared, out_h,
                         ws)
        torch.cuda.synchronize()
    finally:
        if prev is not None:
            moe.set_ffn_path(prev)
    assert moe.read_device_error(ws) == 0
    assert torch.equal(out_h, out.cpu())


def test_deterministic_repeat(device):
    inp = make_custom(VARIANTS["small_shared8"], device)
    a = run_forward(inp)[0]
    b = run_forward(inp)[0]
    assert torch.equal(a, b)
