"""The five layer configurations at full size, in the launch configuration the
benchmark times.

* Routing and permutation are compared for every token.
* Layer outputs are compared for every token of tiny, decode (1) and mixed
  (8), for 16 hash tokens and for sampled prefill tokens, under the GPU's own
  routing (the oracle's forced-routing mode, so near-tie tokens are checked
  too).
* At the prefill shape the tensor-core grouped GEMM is checked expert by
  expert: every y row of the three heaviest experts (several 192-token
  tiles and a partial one), the three lightest non-empty experts, and, with
  a constructed routing, experts of exactly 193 and 385 tokens (one token
  past a 192-token tile boundary).

The oracle's per-expert work runs in a spawn process pool."""
import gc

import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
import oracle
from synthetic import make_inputs
from tests.gpu_utils import bf16_to_np, check_output, check_routing, dims_for, run_forward
from tests.helpers import oracle_expert_rows, oracle_outputs, oracle_pool, oracle_run

pytestmark = pytest.mark.gpu

OUTPUT_TOKENS = {"tiny": None, "decode": None, "mixed": None, "hash": list(range(0, 32, 2)),
                 "prefill": [0, 1234, 2047, 4095]}
# the same layers with the router gate stored in bf16 (the released checkpoints' dtype)
BF16_ROUTER = {"decode": None, "prefill": [7, 4000]}


@pytest.fixture(scope="module")
def pool():
    with oracle_pool() as p:
        yield p


def _free(*objs):
    for o in objs:
        del o
    gc.collect()
    torch.cuda.empty_cache()


def _routing_weights(inp, res, ids):
    """The oracle's weights for the GPU's ids (forced routing; hash: table order)."""
    if inp.cfg["routing"] == "hash":
        return res["w"]
    x = inp.x.float().cpu().numpy()
    return oracle.route_forced(x, inp.router_w.float().cpu().numpy(), ids)[1]


@pytest.mark.parametrize("name,router", [(n, "fp32") for n in OUTPUT_TOKENS] + [(n, "bf16") for n in BF16_ROUTER])
def test_full_config(cuda_device, pool, name, router):
    inp = make_inputs(name, cuda_device, router_dtype=router)
    try:
        c = inp.cfg
        T, k, E = c["T"], c["k"], c["E"]
        out, ids, w, ws = run_forward(inp)
        res = oracle_run(inp, tokens=[])          # routing of every token, no outputs
        ties = check_routing(res, ids, w)
        # the permutation of the GPU's own ids must equal the oracle's
        # stable grouping of those same ids
        dims = dims_for(inp)
        offs = torch.empty(E + 1, dtype=torch.int32, device=cuda_device)
        rows = torch.empty(T * k, dtype=torch.int32, device=cuda_device)
        inv = torch.empty(T * k, dtype=torch.int32, device=cuda_device)
        moe.permute(dims, ids, offs, rows, inv, ws)
        torch.cuda.synchronize()
        ids_np = ids.cpu().numpy().astype(np.int64)
        o_off, o_rows, o_inv = oracle.permute(ids_np, E)
        assert np.array_equal(offs.cpu().numpy(), o_off)
        assert np.array_equal(rows.cpu().numpy(), o_rows)
        assert np.array_equal(inv.cpu().numpy(), o_inv)
        sample = (OUTPUT_TOKENS if router == "fp32" else BF16_ROUTER)[name]
        tok = np.arange(T) if sample is None else np.asarray(sample)
        ref = oracle_outputs(inp, tok, ids_np, _routing_weights(inp, res, ids_np), pool)
        stats = check_output(bf16_to_np(out)[tok], ref, name)
        assert moe.read_device_error(ws) == 0
        print(f"\n{name} ({router} router): tokens checked={len(tok)} near-ties={len(ties)} stats={stats}")
    finally:
        _free(inp)


def _expert_parity(inp, pool, offs, rows, y, experts, label):
    """Every y row of each listed expert against the oracle's rows."""
    k = inp.cfg["k"]
    x = inp.x.float().cpu().numpy().astype(np.float64)
    jobs = [(e, x[rows[offs[e]:offs[e + 1]] // k]) for e in experts]
    refs = oracle_expert_rows(inp, jobs, pool)
    for e, ref in zip(experts, refs):
        got = y[offs[e]:offs[e + 1]].astype(np.float64)
        stats = check_output(got, ref, f"{label} expert {e} ({len(ref)} tokens)")
        print(f"\n{label}: expert {e} tokens={len(ref)} max_err/rms={stats['max_err_over_rms']:.3e} "
              f"mean_rel={stats['mean_rel_err']:.3e}")


def _constructed_ids(T, E, k, counts, seed):
    """Routing ids [T, k] (distinct per token) in which expert e appears in
    exactly counts[e] tokens for each listed e; every other slot takes a
    random expert outside the list."""
    rng = np.random.default_rng(seed)
    special = list(counts)
    others = np.setdiff1d(np.arange(E), special)
    ids = np.stack([rng.choice(others, size=k, replace=False) for _ in range(T)])
    for j, (e, n) in enumerate(counts.items()):
        ids[rng.choice(T, size=n, replace=False), j] = e
    return ids


def test_prefill_tensor_core_whole_experts(cuda_device, pool):
    inp = make_inputs("prefill", cuda_device)
    try:
        c = inp.cfg
        T, k, E, d = c["T"], c["k"], c["E"], c["d"]
        dims = dims_for(inp)
        ws = moe.alloc_workspace(dims, cuda_device)
        res = oracle_run(inp, tokens=[])
        cases = [("oracle routing", res["ids"])]
        cases.append(("constructed 193/385", _constructed_ids(T, E, k, {17: 193, 201: 385, 3: 192, 99: 1}, 5)))
        y = torch.empty(T * k, d, dtype=torch.float32, device=cuda_device)
        for label, ids in cases:
            offs_np, rows_np, _ = oracle.permute(ids, E)
            offs = torch.from_numpy(offs_np.astype(np.int32)).to(cuda_device)
            rows = torch.from_numpy(rows_np.astype(np.int32)).to(cuda_device)
            moe.expert_ffn(dims, inp.x, offs, rows, inp.w1, inp.w3, inp.w2, y, ws)
            torch.cuda.synchronize()
            assert moe.read_device_error(ws) == 0
            counts = np.diff(offs_np)
            if label == "oracle routing":
                order = np.argsort(-counts, kind="stable")
                nonempty = [int(e) for e in order if counts[e] > 0]
                experts = nonempty[:3] + nonempty[-3:]
                assert counts[experts[0]] > 2 * 192, "the skewed routing should give a multi-tile expert"
            else:
                experts = [17, 201, 3, 99]
                assert [int(counts[e]) for e in experts] == [193, 385, 192, 1]
            _expert_parity(inp, pool, offs_np, rows_np, y.cpu().numpy(), experts, f"prefill/{label}")
    finally:
        _free(inp)
