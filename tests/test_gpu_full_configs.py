"""The five layer configurations at full size, in the launch configuration the
benchmark times: routing and permutation compared for every token, outputs
for sampled tokens the oracle computes one by one."""
import gc

import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
import oracle
from synthetic import make_inputs
from tests.gpu_utils import bf16_to_np, check_output, check_routing, dims_for, run_forward
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

SAMPLES = {"tiny": None, "decode": None, "hash": [0, 7, 19, 31], "mixed": [0, 3, 7], "prefill": [0, 1234, 4095]}


@pytest.mark.parametrize("name", list(SAMPLES))
def test_full_config(cuda_device, name):
    inp = make_inputs(name, cuda_device)
    try:
        out, ids, w, ws = run_forward(inp)
        res = oracle_run(inp, tokens=SAMPLES[name])
        ties = check_routing(res, ids, w)
        # the permutation of the GPU's own ids must equal the oracle's
        # stable grouping of those same ids
        dims = dims_for(inp)
        c = inp.cfg
        T, k, E = c["T"], c["k"], c["E"]
        offs = torch.empty(E + 1, dtype=torch.int32, device=cuda_device)
        rows = torch.empty(T * k, dtype=torch.int32, device=cuda_device)
        inv = torch.empty(T * k, dtype=torch.int32, device=cuda_device)
        moe.permute(dims, ids, offs, rows, inv, ws)
        torch.cuda.synchronize()
        o_off, o_rows, o_inv = oracle.permute(ids.cpu().numpy(), E)
        assert np.array_equal(offs.cpu().numpy(), o_off)
        assert np.array_equal(rows.cpu().numpy(), o_rows)
        assert np.array_equal(inv.cpu().numpy(), o_inv)
        tok = res["tokens"]
        keep = np.array([i for i, t in enumerate(tok) if t not in ties])
        got = bf16_to_np(out)[tok]
        stats = check_output(got[keep], res["out"][keep], name)
        assert moe.read_device_error(ws) == 0
        print(f"\n{name}: near-ties={len(ties)} stats={stats}")
    finally:
        del inp
        gc.collect()
        torch.cuda.empty_cache()
