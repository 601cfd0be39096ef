"""Error paths: synchronous host validation and the device error word.
Nothing here faults a GPU: bad data is reported through the error word."""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
from bit_quantized_moe_route_b200 import _lib
from synthetic import CONFIGS, make_custom, make_inputs
from tests.gpu_utils import bf16_to_np, check_output, dims_for, run_forward
from tests.helpers import oracle_run

pytestmark = pytest.mark.gpu

HASH_SMALL = dict(CONFIGS["tiny"], routing="hash", vocab=50, T=12, w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32),
                  seed=301)


def test_bad_token_id_sets_error_word(cuda_device):
    inp = make_custom(HASH_SMALL, cuda_device)
    good = oracle_run(inp)
    bad_tok = inp.token_ids.clone()
    bad_tok[3] = 50 + 7
    bad_tok[8] = -1
    inp_bad = type(inp)(**{**inp.__dict__, "token_ids": bad_tok})
    out, ids, w, ws = run_forward(inp_bad)
    assert moe.read_device_error(ws) == 6
    assert moe.read_device_error(ws) == 0          # read clears the word
    assert torch.all(w[3] == 0) and torch.all(w[8] == 0)
    keep = [t for t in range(12) if t not in (3, 8)]
    check_output(bf16_to_np(out)[keep], good["out"][keep])
    assert torch.all(out[3] == 0) and torch.all(out[8] == 0)


def test_bad_table_entry_sets_error_word(cuda_device):
    inp = make_custom(HASH_SMALL, cuda_device)
    table = inp.tid2eid.clone()
    tok5 = int(inp.token_ids[5])
    table[tok5, 1] = 999
    inp_bad = type(inp)(**{**inp.__dict__, "tid2eid": table})
    _, ids, w, ws = run_forward(inp_bad)
    assert moe.read_device_error(ws) == 6
    assert float(w[5, 1]) == 0.0 and int(ids[5, 1]) == 0
    assert abs(float(w[5].sum()) - 1.0) < 1e-5


def test_bad_ids_in_permute(cuda_device):
    dims = moe.make_dims(4, 256, 128, 8, 2)
    ws = moe.alloc_workspace(dims, cuda_device)
    ids = torch.tensor([[0, 1], [2, 9], [3, -2], [4, 5]], dtype=torch.int32, device=cuda_device)
    offs = torch.empty(9, dtype=torch.int32, device=cuda_device)
    rows = torch.empty(8, dtype=torch.int32, device=cuda_device)
    inv = torch.empty(8, dtype=torch.int32, device=cuda_device)
    moe.permute(dims, ids, offs, rows, inv, ws)
    assert moe.read_device_error(ws) == 6
    assert int(offs[-1]) == 8


def test_workspace_too_small(cuda_device):
    inp = make_inputs("tiny", cuda_device)
    dims = dims_for(inp)
    ws = torch.zeros(1024, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(moe.MoEError) as ei:
        run_forward(inp, ws=ws)
    assert ei.value.status == 3


def test_host_pointer_rejected(cuda_device):
    inp = make_inputs("tiny", cuda_device)
    dims = dims_for(inp)
    ws = moe.alloc_workspace(dims, cuda_device)
    lib = moe.load_library()
    x_host = inp.x.cpu()
    q1, q3, q2 = _lib.qmat(inp.w1), _lib.qmat(inp.w3), _lib.qmat(inp.w2)
    out = torch.empty(4, 256, dtype=torch.bfloat16, device=cuda_device)
    st = lib.moe_forward(ctypes.byref(dims), x_host.data_ptr(), None, inp.router_w.data_ptr(),
                         inp.router_b.data_ptr(), None, ctypes.byref(q1), ctypes.byref(q3), ctypes.byref(q2), None,
                         out.data_ptr(), None, None, ws.data_ptr(), ws.numel(), None)
    assert st == 1 and b"x" in lib.moe_last_error_detail()


def test_misaligned_and_unsupported(cuda_device):
    inp = make_inputs("tiny", cuda_device)
    dims = dims_for(inp)
    ws = moe.alloc_workspace(dims, cuda_device)
    lib = moe.load_library()
    q1, q3, q2 = _lib.qmat(inp.w1), _lib.qmat(inp.w3), _lib.qmat(inp.w2)
    out = torch.empty(4, 256, dtype=torch.bfloat16, device=cuda_device)
    xbuf = torch.zeros(4 * 256 + 8, dtype=torch.bfloat16, device=cuda_device)
    st = lib.moe_forward(ctypes.byref(dims), xbuf.data_ptr() + 2, None, inp.router_w.data_ptr(),
                         inp.router_b.data_ptr(), None, ctypes.byref(q1), ctypes.byref(q3), ctypes.byref(q2), None,
                         out.data_ptr(), None, None, ws.data_ptr(), ws.numel(), None)
    assert st == 1
    q5 = _lib.qmat(inp.w1)
    q5.bits = 5
    st = lib.moe_forward(ctypes.byref(dims), inp.x.data_ptr(), None, inp.router_w.data_ptr(),
                         inp.router_b.data_ptr(), None, ctypes.byref(q5), ctypes.byref(q3), ctypes.byref(q2), None,
                         out.data_ptr(), None, None, ws.data_ptr(), ws.numel(), None)
    assert st == 2
    qm = _lib.qmat(inp.w3)
    qm.fmt = 1
    qm.group = 32
    st = lib.moe_forward(ctypes.byref(dims), inp.x.data_ptr(), None, inp.router_w.data_ptr(),
                         inp.router_b.data_ptr(), None, ctypes.byref(q1), ctypes.byref(qm), ctypes.byref(q2), None,
                         out.data_ptr(), None, None, ws.data_ptr(), ws.numel(), None)
    assert st == 2 and b"share" in lib.moe_last_error_detail()


BAD_PERMUTATIONS = {
    "offsets_start_nonzero": lambda o, r: o.__setitem__(0, 1),
    "offsets_decrease": lambda o, r: (o.__setitem__(3, int(o[5]) + 1)),
    "offsets_end_past_pairs": lambda o, r: o.__setitem__(-1, int(o[-1]) + 64),
    "row_past_pairs": lambda o, r: r.__setitem__(5, len(r) + 1000),
    "row_negative": lambda o, r: r.__setitem__(0, -7),
}


@pytest.mark.parametrize("path", ["gemv", "tc"])
@pytest.mark.parametrize("bad", list(BAD_PERMUTATIONS))
def test_bad_permutation_in_expert_ffn(cuda_device, bad, path):
    """A caller permutation that fails its device-side check records
    MOE_ERR_DEVICE_INPUT, runs no expert (y keeps its contents) and touches
    nothing out of bounds; a correct call afterwards is clean."""
    inp = make_custom(dict(CONFIGS["tiny"], T=12, seed=303), cuda_device)
    c = inp.cfg
    res = oracle_run(inp)
    dims = dims_for(inp)
    ws = moe.alloc_workspace(dims, cuda_device)
    n = c["T"] * c["k"]
    offs = res["expert_offsets"].astype(np.int32).copy()
    rows = res["sorted_rows"].astype(np.int32).copy()
    BAD_PERMUTATIONS[bad](offs, rows)
    prev = moe.set_ffn_path(moe.FFN_GEMV if path == "gemv" else moe.FFN_TENSOR_CORE)
    try:
        y = torch.full((n, c["d"]), 7.0, dtype=torch.float32, device=cuda_device)
        moe.expert_ffn(dims, inp.x, torch.from_numpy(offs).to(cuda_device), torch.from_numpy(rows).to(cuda_device),
                       inp.w1, inp.w3, inp.w2, y, ws)
        assert moe.read_device_error(ws) == 6
        assert torch.all(y == 7.0)
        good_offs = torch.from_numpy(res["expert_offsets"].astype(np.int32)).to(cuda_device)
        good_rows = torch.from_numpy(res["sorted_rows"].astype(np.int32)).to(cuda_device)
        moe.expert_ffn(dims, inp.x, good_offs, good_rows, inp.w1, inp.w3, inp.w2, y, ws)
        assert moe.read_device_error(ws) == 0
    finally:
        moe.set_ffn_path(prev)
    y_ref = res["y_slots"].reshape(n, c["d"])[res["sorted_rows"]]
    check_output(y.cpu().double().numpy(), y_ref, f"{bad}/{path} follow-up")
