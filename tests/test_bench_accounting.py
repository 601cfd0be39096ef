"""The roofline numerators bench.py reports (algorithmic bytes and flops per
kernel), checked on CPU against closed forms of the packed formats.

A packed matrix of n weights with b-bit codes and bf16 scale + bias per
group of g inputs holds n·(b/8 + 4/g) bytes; mxfp4 holds n·(1/2 + 1/32)
(one e8m0 byte per 32 codes).  The per-expert figures of the five layer
configurations follow from these; tensors are built on the meta device, so
nothing of the full-size packs is allocated."""
import os
import sys
import types

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synthetic.moe_inputs import QMat  # noqa: E402


def qmat(fmt, bits, group, E, n_out, n_in):
    q = torch.empty(E, n_out, n_in * bits // 32, dtype=torch.int32, device="meta")
    if fmt == "mxfp4":
        return QMat(fmt, 4, 32, n_out, n_in, q, torch.empty(E, n_out, n_in // 32, dtype=torch.uint8, device="meta"),
                    None)
    s = torch.empty(E, n_out, n_in // group, dtype=torch.bfloat16, device="meta")
    return QMat(fmt, bits, group, n_out, n_in, q, s, torch.empty_like(s))


def layer(T, d, E, k, f, w13, w2, shared=None, f_shared=0, routing="learned"):
    cfg = dict(T=T, d=d, E=E, k=k, f=f, routing=routing, f_shared=f_shared)
    sh = None
    if shared:
        sh = (qmat(*shared, 1, f_shared, d), qmat(*shared, 1, f_shared, d), qmat(*shared, 1, d, f_shared))
    return types.SimpleNamespace(cfg=cfg, w1=qmat(*w13, E, f, d), w3=qmat(*w13, E, f, d), w2=qmat(*w2, E, d, f),
                                 shared=sh)


def closed_form(n, fmt, bits, group):
    if fmt == "mxfp4":
        return n * (0.5 + 1 / 32)
    return n * (bits / 8 + 4 / group)


@pytest.mark.parametrize("w13,w2,want", [
    (("affine", 4, 64), ("affine", 4, 64), 14_155_776),
    (("mxfp4", 4, 32), ("mxfp4", 4, 32), 13_369_344),
    (("affine", 2, 128), ("affine", 3, 128), 8_126_464),
])
def test_per_expert_bytes(w13, w2, want):
    d, f = 4096, 2048
    inp = layer(1, d, 256, 8, f, w13, w2)
    per = (inp.w1.packed_bytes_per_expert() + inp.w3.packed_bytes_per_expert()
           + inp.w2.packed_bytes_per_expert())
    assert per == want
    assert per == closed_form(2 * d * f, *w13) + closed_form(d * f, *w2)


def test_decode_weight_bytes_count_distinct_experts_and_shared():
    d, f, k = 4096, 2048, 8
    inp = layer(1, d, 256, k, f, ("affine", 4, 64), ("affine", 4, 64), shared=("affine", 8, 64), f_shared=2048)
    ids = np.array([[3, 17, 17, 40, 41, 99, 200, 255]])  # 7 distinct experts (17 twice)
    work, flops, n_act, weight_bytes, kflops = bench.kernel_work(inp, ids)
    assert n_act == 7
    shared = 26_738_688
    assert shared == closed_form(3 * d * 2048, "affine", 8, 64)
    assert weight_bytes == 7 * 14_155_776 + shared
    # stage 1 reads W1 and W3 of each active expert and of the shared expert
    w13_routed = 7 * 2 * closed_form(d * f, "affine", 4, 64)
    w13_shared = 2 * closed_form(d * 2048, "affine", 8, 64)
    P = 1 * k + 1
    assert work["ffn_w13_swiglu"] == w13_routed + w13_shared + d * 2 + P * f * 4
    assert work["ffn_w2"] == 7 * closed_form(d * f, "affine", 4, 64) + closed_form(d * 2048, "affine", 8, 64) \
        + P * f * 4 + P * d * 4
    # the fp32 router matrix is read once
    assert work["router_logits"] == 256 * d * 4 + d * 2 + 256 * 4


def test_prefill_flops():
    T, d, E, k, f = 4096, 4096, 256, 8, 2048
    inp = layer(T, d, E, k, f, ("affine", 4, 64), ("affine", 4, 64))
    ids = np.arange(T * k).reshape(T, k) % E
    work, flops, n_act, weight_bytes, kflops = bench.kernel_work(inp, ids)
    assert flops == 2 * T * k * 3 * d * f
    assert abs(flops - 1.649e12) < 1e9
    assert kflops["ffn_w13_swiglu"] + kflops["ffn_w2"] == flops
    assert kflops["ffn_w13_swiglu"] == 2 * kflops["ffn_w2"]
    assert n_act == E and weight_bytes == E * 14_155_776


def test_whole_job_rate_is_tokens_over_slowest_time():
    assert bench.whole_job_rate(1, 1, 0.094) == pytest.approx(1 / 94e-6)
    assert bench.whole_job_rate(4096, 8, 2.5) == pytest.approx(8 * 4096 / 2.5e-3)


PEAK = (6539.5, 1624.7, 1376.7, "measured")


def test_roofline_decode_is_hbm_bound():
    work = {"ffn_w13_swiglu": 93_405_184, "ffn_w2": 46_882_816}
    r = bench.roofline_entry("ffn_w13_swiglu", 0.042, work, {}, False, PEAK, 93_613_824)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6539.5
    assert r["achieved"] == pytest.approx(93_405_184 / 42e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6539.5)
    assert r["frac_of_nominal"] == pytest.approx(r["achieved"] / 8000.0)
    assert r["traffic"] == 93_613_824 and "tensor_frac" not in r


def test_roofline_prefill_is_tensor_bound():
    flops = 2.0 * 4096 * 8 * 2 * 4096 * 2048
    r = bench.roofline_entry("ffn_w13_swiglu", 1.40, {"ffn_w13_swiglu": 3.0e9}, {"ffn_w13_swiglu": flops}, True,
                             PEAK, None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1624.7
    assert r["achieved"] == pytest.approx(flops / 1.40e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1624.7)
    assert r["frac_of_sustained_peak"] == pytest.approx(r["achieved"] / 1376.7)
    assert r["frac_of_nominal"] == pytest.approx(r["achieved"] / 2250.0)


def test_roofline_small_batch_tensor_path_stays_hbm_bound():
    # 32 tokens over ~160 experts: few flops per weight byte
    flops = 2.0 * 32 * 8 * 2 * 4096 * 2048
    r = bench.roofline_entry("ffn_w13_swiglu", 0.758, {"ffn_w13_swiglu": 1.49e9}, {"ffn_w13_swiglu": flops}, True,
                             PEAK, None)
    assert r["bound"] == "hbm"
    assert r["tensor_frac"] == pytest.approx(flops / 0.758e-3 / 1e12 / 1624.7)
    assert r["tensor_frac"] < r["frac"]


@pytest.mark.parametrize("name", ["tiny", "decode", "hash", "mixed", "prefill"])
def test_every_workload_accounts_and_describes(name):
    """kernel_work and workload_desc run for each layer configuration the
    benchmark knows, with a routing that touches min(E, T*k) experts."""
    from synthetic import CONFIGS
    c = dict(CONFIGS[name], name=name)
    inp = layer(c["T"], c["d"], c["E"], c["k"], c["f"], c["w13"], c["w2"], shared=c["shared"],
                f_shared=c["f_shared"], routing=c["routing"])
    ids = (np.arange(c["T"] * c["k"]) % c["E"]).reshape(c["T"], c["k"])
    work, flops, n_act, weight_bytes, kflops = bench.kernel_work(inp, ids)
    assert n_act == min(c["E"], c["T"] * c["k"])
    assert all(v > 0 for v in work.values() if v is not None)
    assert flops == 2 * c["T"] * c["k"] * 3 * c["d"] * c["f"] + 2 * c["T"] * 3 * c["d"] * c["f_shared"]
    assert ("route_hash" in work) == (c["routing"] == "hash")
    desc = bench.workload_desc(c)
    assert desc["workload"] == name and desc["T"] == c["T"] and desc["n_experts"] == c["E"]


def test_decode_layer_bytes_count_only_kernels_that_ran():
    """Decode on the GEMV path: the four launches read the routed experts,
    the shared expert once, the fp32 router, x, h and y -- about 144.2 MB
    with 8 distinct experts -- and nothing of the tensor-core path."""
    d, f, k, E = 4096, 2048, 8, 256
    inp = layer(1, d, E, k, f, ("affine", 4, 64), ("affine", 4, 64), shared=("affine", 8, 64), f_shared=2048)
    ids = np.array([[3, 17, 40, 41, 99, 120, 200, 255]])
    work, flops, n_act, weight_bytes, kflops = bench.kernel_work(inp, ids)
    labels = ["route_topk_permute", "ffn_w13_swiglu", "ffn_w2", "combine"]
    total = bench.layer_bytes(work, labels)
    assert weight_bytes == 8 * 14_155_776 + 26_738_688
    P = k + 1
    acts = (E * d * 4 + d * 2 + E * 4 + k * 8 + k * 12 + (E + 1) * 4     # routing + permutation
            + d * 2 + P * f * 4                                          # x in, h out
            + P * f * 4 + P * d * 4                                      # h in, y out
            + P * d * 4 + d * 2 + k * 8)                                 # combine
    assert total == weight_bytes + acts
    assert abs(total / 1e6 - 144.2) < 0.5
    assert "ffn_w13_swiglu_shared" not in work and "gather_f16" not in work


def test_tensor_core_path_counts_the_shared_expert_once():
    d, f, k, E, T = 1024, 512, 4, 16, 64
    inp = layer(T, d, E, k, f, ("affine", 4, 64), ("affine", 4, 64), shared=("affine", 8, 64), f_shared=512)
    ids = (np.arange(T * k) % E).reshape(T, k)
    work, flops, n_act, weight_bytes, kflops = bench.kernel_work(inp, ids, tensor_path=True)
    sh = sum(m.packed_bytes_per_expert() for m in inp.shared)
    routed = E * (inp.w1.packed_bytes_per_expert() * 2 + inp.w2.packed_bytes_per_expert())
    labels = ["router_logits", "topk", "permute", "gather_f16", "tile_plan", "ffn_w13_swiglu",
              "ffn_w13_swiglu_shared", "ffn_w2", "ffn_w2_shared", "combine"]
    weights_counted = (work["ffn_w13_swiglu"] - T * k * d * 2 - T * k * f * 2) + \
        (work["ffn_w2"] - T * k * f * 2 - T * k * d * 4) + \
        (work["ffn_w13_swiglu_shared"] - T * d * 2 - T * 512 * 2) + (work["ffn_w2_shared"] - T * 512 * 2 - T * d * 4)
    assert weights_counted == routed + sh == weight_bytes
    assert bench.layer_bytes(work, labels) > weight_bytes


def test_step_stats_median_is_the_reported_step():
    st = bench.step_stats([0.1, 0.5, 0.11, 0.12, 0.1])
    assert st["median"] == 0.11 and st["min"] == 0.1 and st["p90"] == 0.5
    assert st["mean"] == pytest.approx(0.186)


def test_roofline_tensor_bound_uses_the_burst_peak():
    flops = 2.0 * 4096 * 8 * 2 * 4096 * 2048
    r = bench.roofline_entry("ffn_w13_swiglu", 1.444, {"ffn_w13_swiglu": 3.0e9}, {"ffn_w13_swiglu": flops}, True,
                             PEAK, None)
    assert r["peak"] == 1624.7
    assert r["frac"] == pytest.approx(flops / 1.444e-3 / 1e12 / 1624.7)
    assert r["frac"] < 0.5 < r["frac_of_sustained_peak"]


def test_layer_copies_cycle_only_small_steps():
    l2 = 126 * 1024 * 1024
    # decode reads ~140 MB of weights per step: copies are cycled
    assert bench.layer_copies(0, 140_000_000, l2) == 4
    # a prefill step reads GBs: one copy, flushed between steps
    assert bench.layer_copies(0, 3_600_000_000, l2) == 1
    assert bench.layer_copies(0, 8 * l2, l2) == 1
    # an explicit request wins either way
    assert bench.layer_copies(1, 140_000_000, l2) == 1
    assert bench.layer_copies(6, 3_600_000_000, l2) == 6


def test_layer_copies_share_values_not_buffers():
    from synthetic import make_inputs
    inp = make_inputs("tiny", "cpu")
    cp = inp.clone()
    for a, b in zip(bench.layer_tensors(inp), bench.layer_tensors(cp)):
        assert torch.equal(a, b) and a.data_ptr() != b.data_ptr()
