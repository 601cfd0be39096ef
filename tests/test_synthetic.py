"""Properties of the seeded input generators (CPU)."""
import numpy as np
import torch

from synthetic import CONFIGS, make_custom, make_inputs, pack_bits


def test_tiny_shapes_and_determinism():
    a = make_inputs("tiny")
    b = make_inputs("tiny")
    c = CONFIGS["tiny"]
    assert a.x.shape == (c["T"], c["d"]) and a.x.dtype == torch.bfloat16
    assert a.router_w.shape == (c["E"], c["d"]) and a.router_w.dtype == torch.float32
    assert a.w1.q.shape == (8, 128, 256 * 4 // 32) and a.w1.scales.shape == (8, 128, 4)
    assert a.w2.q.shape == (8, 256, 128 * 4 // 32) and a.w2.biases.dtype == torch.bfloat16
    for t1, t2 in ((a.x, b.x), (a.w1.q, b.w1.q), (a.w2.scales, b.w2.scales), (a.router_b, b.router_b)):
        assert torch.equal(t1, t2)


def test_hash_table_rows_distinct_and_e8m0_range():
    cfg = dict(CONFIGS["hash"])
    cfg.update(T=16, d=256, f=128, E=32, vocab=500, seed=5)
    inp = make_custom(cfg)
    t = inp.tid2eid.numpy()
    assert t.shape == (500, 8)
    assert all(len(set(r.tolist())) == 8 for r in t)
    assert t.min() >= 0 and t.max() < 32
    s = inp.w1.scales.numpy()
    assert s.dtype == np.uint8 and s.min() >= 117 and s.max() <= 123
    assert inp.token_ids.min() >= 0 and inp.token_ids.max() < 500
    assert inp.w1.biases is None and inp.w1.q.shape == (32, 128, 256 // 8)


def test_pack_bits_matches_bigint():
    from tests.helpers import bigint_words
    g = torch.Generator().manual_seed(1)
    for bits in (2, 3, 4, 8):
        q = torch.randint(0, 1 << bits, (3, 64), generator=g)
        w = pack_bits(q, bits).numpy().view(np.uint32)
        for r in range(3):
            assert np.array_equal(w[r], bigint_words(q[r].tolist(), bits))
