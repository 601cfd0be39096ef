"""moe_dequant_mxfp8 against the oracle's mxfp8 decode, bit for bit: random
e4m3 bytes (every finite code, subnormals included) with e8m0 scales over a
wide exponent range, rows of several lengths, scales taken from 128x128
checkpoint blocks through the oracle's block-to-group mapping, and the
argument checks."""
import numpy as np
import pytest
import torch

import bit_quantized_moe_route_b200 as moe
import oracle

pytestmark = pytest.mark.gpu


def _words(codes):
    return np.ascontiguousarray(codes.astype(np.uint8)).view(np.uint32)


def _check(codes, scales, dev):
    rows, n_in = codes.shape
    out = torch.empty(rows, n_in, dtype=torch.bfloat16, device=dev)
    moe.dequant_mxfp8(torch.from_numpy(codes.astype(np.uint8)).to(dev),
                      torch.from_numpy(scales.astype(np.uint8)).to(dev), out)
    torch.cuda.synchronize()
    ref = oracle.dequant_mxfp8(_words(codes), scales, n_in)
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16)
    assert torch.equal(ref_bf16.double(), torch.from_numpy(ref)), "reference not exact in bf16"
    got = out.cpu()
    same = (got.view(torch.int16) == ref_bf16.view(torch.int16))
    assert bool(same.all()), np.argwhere(~same.numpy())[:5]


@pytest.mark.parametrize("rows,n_in", [(1, 32), (3, 96), (37, 1024), (300, 4096)])
def test_dequant_matches_oracle(cuda_device, rows, n_in):
    moe.load_library()
    rng = np.random.default_rng(rows * 7 + n_in)
    codes = rng.integers(0, 256, size=(rows, n_in))
    codes[(codes & 0x7F) == 0x7F] = 0x38           # no NaN codes in weights
    scales = rng.integers(96, 160, size=(rows, n_in // 32))
    _check(codes, scales, cuda_device)


def test_every_code_and_extreme_scales(cuda_device):
    """Group g of a row holds bytes 32g .. 32g+31: small positive codes at
    scale 250, the largest finite codes at 127, subnormal negatives at 5 and
    normal negatives at 1 (bf16-subnormal results), all exact."""
    moe.load_library()
    codes = np.tile(np.arange(256), (4, 1))
    codes[(codes & 0x7F) == 0x7F] = 0x00
    scales = np.array([[250, 127, 200, 127, 5, 1, 127, 127]] * 4)
    _check(codes, scales, cuda_device)


def test_block128_checkpoint_scales(cuda_device):
    moe.load_library()
    rng = np.random.default_rng(9)
    n_out, n_in = 260, 512
    codes = rng.integers(0, 256, size=(n_out, n_in))
    codes[(codes & 0x7F) == 0x7F] = 0x38
    blocks = rng.integers(110, 140, size=((n_out + 127) // 128, n_in // 128))
    scales = oracle.block128_scales_to_group32(blocks, n_out, n_in)
    _check(codes, scales, cuda_device)


def test_arguments(cuda_device):
    from bit_quantized_moe_route_b200 import _lib
    lib = moe.load_library()
    c = torch.zeros(4, 64, dtype=torch.uint8, device=cuda_device)
    s = torch.zeros(4, 2, dtype=torch.uint8, device=cuda_device)
    o = torch.empty(4, 64, dtype=torch.bfloat16, device=cuda_device)
    moe.dequant_mxfp8(c, s, o)
    torch.cuda.synchronize()
    assert not o.float().any()
    assert lib.moe_dequant_mxfp8(c.data_ptr(), s.data_ptr(), 4, 48, o.data_ptr(), None) == 1
    assert lib.moe_dequant_mxfp8(c.data_ptr() + 8, s.data_ptr(), 4, 32, o.data_ptr(), None) == 1
    assert _lib.STATUS_NAMES[1]
