"""Checks that tie the oracle to what the pages and mathematics fix.

Each ``pin_*`` raises AssertionError on a mismatch.  They are run as plain
tests (test_oracle_pins.py) and, with deliberate mistakes planted in the
oracle, as mutation tests (test_oracle_mutations.py) to show each one bites.
None of them re-types the oracle's own formula: each compares against a
different formulation, a library routine, hand-derived fixtures, or brute
force.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from synthetic import make_custom, quantize_affine
from tests.helpers import bigint_words, dims_of, oracle_run

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- formats
def pin_e2m1_table():
    """e2m1 values from the bit fields (sign | 2-bit exponent, bias 1 | 1-bit mantissa)."""
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = (m * 0.5) if e == 0 else (2.0 ** (e - 1)) * (1.0 + m / 2.0)
        want = -mag if s else mag
        got = oracle.E2M1_VALUES[code]
        assert got == want and np.signbit(got) == bool(s), (code, got, want)


def pin_e8m0():
    """e8m0 byte b -> 2^(b-127), against torch's float8_e8m0fnu widening."""
    b = torch.arange(0, 255, dtype=torch.uint8)
    lib = b.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = oracle.e8m0_value(b.numpy())
    assert np.array_equal(got, lib), np.nonzero(got != lib)


def pin_unpack_golden():
    with open(os.path.join(GOLDEN, "affine_bitstream.txt")) as fh:
        n = 0
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits_s, codes_s, words_s = [p.strip() for p in line.split("|")]
            bits = int(bits_s)
            codes = [int(c) for c in codes_s.split(",")]
            words = np.array([int(w, 16) for w in words_s.split(",")], dtype=np.uint32)
            got = oracle.unpack_codes(words, bits, len(codes))
            assert got.tolist() == codes, (bits, got.tolist(), codes)
            n += 1
    assert n >= 8


def pin_unpack_bigint():
    rng = np.random.default_rng(11)
    for bits in (2, 3, 4, 8):
        for n in (32, 64, 96, 128):
            codes = rng.integers(0, 1 << bits, size=n)
            words = bigint_words(codes, bits)
            got = oracle.unpack_codes(words, bits, n)
            assert np.array_equal(got, codes), (bits, n)
    # several rows at once: rows are independent streams
    codes = rng.integers(0, 8, size=(5, 64))
    words = np.stack([bigint_words(r, 3) for r in codes])
    assert np.array_equal(oracle.unpack_codes(words, 3, 64), codes)


def pin_affine_dequant():
    """Dequantised packs reproduce the weights they were made from.

    The generator's min/max quantiser bounds the reconstruction error by half
    a quantisation step (plus bf16 rounding of scale and bias); a wrong group
    index, a transposed row or a dropped term breaks the bound by orders of
    magnitude.  Special codes: q = 0 gives the bias exactly, q = 2^b-1 gives
    scale*(2^b-1)+bias.
    """
    g = torch.Generator().manual_seed(5)
    for bits, group in ((2, 64), (2, 128), (3, 64), (3, 128), (4, 64), (4, 128), (8, 64), (8, 128)):
        w = torch.randn(24, 256, generator=g) * 0.02 + torch.randn(24, 1, generator=g) * 0.01
        q, s, b = quantize_affine(w, bits, group)
        s32, b32 = s.float().numpy(), b.float().numpy()
        W = oracle.dequant_affine(q.numpy().view(np.uint32), s32, b32, bits, group, 256)
        levels = (1 << bits) - 1
        tol = (np.repeat(s32, group, -1) * (0.5 + levels / 256.0)
               + np.repeat(np.abs(b32), group, -1) / 256.0 + 1e-12)
        err = np.abs(W - w.double().numpy())
        assert (err <= tol).all(), (bits, group, float((err / tol).max()))
    rows, n_in, group = 3, 128, 64
    for bits in (2, 3, 4, 8):
        nw = n_in * bits // 32
        s = np.array([[0.25, 0.5]] * rows)
        b = np.array([[-1.0, 2.0]] * rows)
        W0 = oracle.dequant_affine(np.zeros((rows, nw), np.uint32), s, b, bits, group, n_in)
        assert np.array_equal(W0, np.repeat(b, group, -1))
        W1 = oracle.dequant_affine(np.full((rows, nw), 0xFFFFFFFF, np.uint32), s, b, bits, group, n_in)
        assert np.array_equal(W1, np.repeat(s * ((1 << bits) - 1) + b, group, -1))


def pin_mxfp4_dequant():
    """mxfp4 rows decode code-by-code; every value is exact in bf16."""
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, size=(4, 64))
    scales = rng.integers(117, 124, size=(4, 2)).astype(np.uint8)
    words = np.stack([bigint_words(r, 4) for r in codes])
    W = oracle.dequant_mxfp4(words, scales, 64)
    for r in range(4):
        for i in range(64):
            c = int(codes[r, i])
            s, e, m = c >> 3, (c >> 1) & 3, c & 1
            mag = (m * 0.5) if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
            want = (-mag if s else mag) * math.ldexp(1.0, int(scales[r, i // 32]) - 127)
            assert W[r, i] == want, (r, i, W[r, i], want)
    # lossless in bf16 (model card conversion notes): bf16 round-trip is exact
    t = torch.from_numpy(W)
    assert torch.equal(t.to(torch.bfloat16).double(), t)
    # low nibble holds the even element: a byte 0x3F is codes (15, 3)
    W2 = oracle.dequant_mxfp4(np.array([[0x0000003F, 0, 0, 0]], np.uint32), np.array([[127]], np.uint8), 32)
    assert W2[0, 0] == -6.0 and W2[0, 1] == 1.5


def pin_e4m3_table():
    """e4m3 decode for all 256 bytes against torch's float8_e4m3fn widening,
    plus hand-derived values (1.0, the largest finite 448, the smallest
    subnormal 2^-9 and normal 2^-6, -1.0, -0.0, NaN)."""
    b = torch.arange(0, 256, dtype=torch.int32).to(torch.uint8)
    lib = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.E4M3_VALUES
    assert np.array_equal(np.isnan(got), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(got[ok], lib[ok]) and np.array_equal(np.signbit(got[ok]), np.signbit(lib[ok]))
    hand = {0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0xB8: -1.0, 0x3F: 1.875, 0x07: 7 * 2.0 ** -9}
    for code, want in hand.items():
        assert got[code] == want, (hex(code), got[code], want)
    assert got[0x80] == 0.0 and np.signbit(got[0x80])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert np.nanmax(got) == 448.0


def pin_mxfp8_dequant():
    """mxfp8 rows decode byte-by-byte (torch e4m3 widening times the e8m0
    power of two); byte i of a row is element i; every value is exact in bf16."""
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, size=(3, 96))
    codes[(codes & 0x7F) == 0x7F] = 0x38           # no NaN codes in weights
    scales = rng.integers(118, 132, size=(3, 3)).astype(np.uint8)
    words = np.stack([bigint_words(r, 8) for r in codes])
    # the review thread's count: group_size 32 at 8 bits is 8 uint32 words per scale
    assert words.shape[1] // scales.shape[1] == 8
    W = oracle.dequant_mxfp8(words, scales, 96)
    f8 = torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for r in range(3):
        for i in range(96):
            want = f8[r, i] * math.ldexp(1.0, int(scales[r, i // 32]) - 127)
            assert W[r, i] == want, (r, i, W[r, i], want)
    t = torch.from_numpy(W)
    assert torch.equal(t.to(torch.bfloat16).double(), t)
    # little-endian bytes: the word 0x003F00B8 holds elements (-1.0, 0, 1.875, 0)
    W2 = oracle.dequant_mxfp8(np.array([[0x003F00B8] + [0] * 7], np.uint32), np.array([[127]], np.uint8), 32)
    assert W2[0, :4].tolist() == [-1.0, 0.0, 1.875, 0.0]


def pin_block128_scales():
    """128x128 block scales spread to (row, 32-input group): element (o, i)
    takes block (o // 128, i // 128), checked element by element."""
    rng = np.random.default_rng(6)
    n_out, n_in = 300, 512
    bs = rng.integers(100, 140, size=((n_out + 127) // 128, n_in // 128)).astype(np.uint8)
    g = oracle.block128_scales_to_group32(bs, n_out, n_in)
    assert g.shape == (n_out, n_in // 32)
    for o in range(n_out):
        for i in range(0, n_in, 7):
            assert g[o, i // 32] == bs[o // 128, i // 128], (o, i)


# ---------------------------------------------------------------- routing
def pin_sqrtsoftplus():
    with open(os.path.join(GOLDEN, "sqrtsoftplus.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            x, v, rt = (float(p) for p in line.split("|"))
            got = float(oracle.sqrtsoftplus(np.array([x]))[0])
            assert math.isfinite(got)
            assert abs(got - v) <= rt * abs(v) + (0.0 if rt else 0.0), (x, got, v)
    from scipy.special import softplus
    x = np.linspace(-700, 700, 20001)
    lib = np.sqrt(softplus(x))
    got = oracle.sqrtsoftplus(x)
    assert np.all(np.isfinite(got))
    rel = np.abs(got - lib) / np.maximum(lib, 1e-300)
    assert rel.max() < 1e-12, rel.max()
    assert np.all(np.diff(got) > 0)                 # strictly increasing
    big = np.array([1e4, 1e6, 1e8])
    assert np.allclose(oracle.sqrtsoftplus(big), np.sqrt(big), rtol=1e-15)


def _rank_count_topk(keys, k):
    """Brute force: e is selected iff fewer than k experts beat it."""
    T, E = keys.shape
    ids = np.zeros((T, k), np.int64)
    for t in range(T):
        beats = []
        for e in range(E):
            n = sum(1 for j in range(E) if keys[t, j] > keys[t, e] or (keys[t, j] == keys[t, e] and j < e))
            beats.append(n)
        for e in range(E):
            if beats[e] < k:
                ids[t, beats[e]] = e
    return ids


def pin_topk_bruteforce():
    rng = np.random.default_rng(7)
    for E, k in ((8, 2), (16, 4), (12, 12), (9, 1)):
        keys = rng.normal(size=(20, E))
        keys[:5, : E // 2] = keys[:5, [0]]          # exact ties
        keys[5:8] = 0.25                            # all equal
        ids, gap = oracle.topk_select(keys, k)
        want = _rank_count_topk(keys, k)
        assert np.array_equal(ids, want), (E, k)
        for t in range(keys.shape[0]):
            srt = sorted(keys[t], reverse=True)
            g = srt[k - 1] - srt[k] if k < E else np.inf
            assert gap[t] == g
    # subset brute force on a small case: the chosen set has the largest key sum
    keys = rng.normal(size=(6, 8))
    ids, _ = oracle.topk_select(keys, 3)
    for t in range(6):
        best = max(itertools.combinations(range(8), 3), key=lambda c: sum(keys[t, list(c)]))
        assert set(ids[t].tolist()) == set(best)


def pin_route_learned():
    """With zero bias top-k of sqrtsoftplus equals top-k of the raw logits
    (monotone score); weights are positive and sum to one; the bias only moves
    the selection, never the weights."""
    rng = np.random.default_rng(9)
    x = rng.normal(size=(33, 64))
    wr = rng.normal(scale=0.2, size=(16, 64))
    ids, w, gap, L = oracle.route_learned(x, wr, np.zeros(16), 4)
    ids_raw, _ = oracle.topk_select(x @ wr.T, 4)
    assert np.array_equal(ids, ids_raw)
    assert np.allclose(L, x @ wr.T, rtol=1e-13, atol=1e-13)
    assert np.allclose(w.sum(1), 1.0, atol=1e-14) and (w > 0).all()
    from scipy.special import softplus
    s_lib = np.sqrt(softplus(x @ wr.T))
    assert np.allclose(w, np.take_along_axis(s_lib, ids, 1) / np.take_along_axis(s_lib, ids, 1).sum(1, keepdims=True), rtol=1e-12)
    # a huge bias on expert 3 forces it in; its weight still comes from the score
    b = np.zeros(16)
    b[3] = 1e3
    ids_b, w_b, _, _ = oracle.route_learned(x, wr, b, 4)
    assert (ids_b[:, 0] == 3).all()
    sel = np.take_along_axis(s_lib, ids_b, 1)
    assert np.allclose(w_b, sel / sel.sum(1, keepdims=True), rtol=1e-12)


def pin_route_hash():
    """ids are exactly the table rows of each token id, independent of the
    token's position or batch; permuting tokens permutes ids and weights."""
    rng = np.random.default_rng(13)
    vocab, E, k, d = 50, 16, 4, 32
    table = np.stack([rng.permutation(E)[:k] for _ in range(vocab)]).astype(np.int32)
    tok = rng.integers(0, vocab, size=12)
    x = rng.normal(size=(12, d))
    wr = rng.normal(scale=0.3, size=(E, d))
    ids, w = oracle.route_hash(x, wr, tok, table)
    assert np.array_equal(ids, table[tok])
    assert np.allclose(w.sum(1), 1.0, atol=1e-14)
    perm = rng.permutation(12)
    ids_p, w_p = oracle.route_hash(x[perm], wr, tok[perm], table)
    assert np.array_equal(ids_p, ids[perm]) and np.allclose(w_p, w[perm], rtol=0, atol=0)
    ids_u, w_u = oracle.route_hash(x, None, tok, table)
    assert np.array_equal(ids_u, ids) and np.all(w_u == 1.0 / k)
    # weights = renormalised scores of the table's experts, via a per-pair loop
    from scipy.special import softplus
    for t in range(12):
        s = np.array([math.sqrt(softplus(float(x[t] @ wr[e]))) for e in table[tok[t]]])
        assert np.allclose(w[t], s / s.sum(), rtol=1e-12)


def pin_permutation():
    rng = np.random.default_rng(17)
    for T, k, E in ((1, 8, 256), (37, 4, 16), (64, 2, 8), (5, 3, 40)):
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])
        offs, rows, inv = oracle.permute(ids, E)
        flat = ids.reshape(-1)
        assert offs[0] == 0 and offs[-1] == T * k and np.all(np.diff(offs) >= 0)
        assert sorted(rows.tolist()) == list(range(T * k))
        assert np.array_equal(inv[rows], np.arange(T * k))
        for e in range(E):
            seg = rows[offs[e]:offs[e + 1]]
            assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)
            assert len(seg) == int((flat == e).sum())
        # brute force: walk experts in order, scan flat indices in order
        want = [i for e in range(E) for i in range(T * k) if flat[i] == e]
        assert rows.tolist() == want


# ---------------------------------------------------------------- whole layer
def _dense_reference(inp, res):
    """Dense mixture: every token through every expert, masked by the gate.

    Uses torch fp64 linear/silu (library routines) on the oracle-dequantised
    weights, so it shares only the (separately pinned) decode with the oracle.
    """
    c = inp.cfg
    T, E, d, f = c["T"], c["E"], c["d"], c["f"]
    x = inp.x.double()
    G = torch.zeros(T, E, dtype=torch.float64)
    ids = torch.from_numpy(res["ids"])
    G.scatter_add_(1, ids, torch.from_numpy(res["w"]))
    out = torch.zeros(T, d, dtype=torch.float64)
    for e in range(E):
        W = {}
        for name, m, n_in in (("w1", inp.w1, d), ("w3", inp.w3, d), ("w2", inp.w2, f)):
            W[name] = torch.from_numpy(oracle.dequant(m.fmt, m.bits, m.group, n_in, *m.expert_numpy(e)))
        h = F.silu(F.linear(x, W["w1"])) * F.linear(x, W["w3"])
        out += G[:, e:e + 1] * F.linear(h, W["w2"])
    if inp.shared is not None:
        s1, s3, s2 = inp.shared
        fs = c["f_shared"]
        Ws = [torch.from_numpy(oracle.dequant(m.fmt, m.bits, m.group, n_in, *m.expert_numpy(0)))
              for m, n_in in ((s1, d), (s3, d), (s2, fs))]
        out += F.linear(F.silu(F.linear(x, Ws[0])) * F.linear(x, Ws[1]), Ws[2])
    return out.numpy()


def pin_dense_equivalence():
    for name, over in (("tiny", {}),
                       ("tiny", dict(w13=("affine", 3, 64), w2=("affine", 2, 64), seed=21)),
                       ("tiny", dict(w13=("mxfp4", 4, 32), w2=("mxfp4", 4, 32), seed=22)),
                       ("tiny", dict(shared=("affine", 8, 64), f_shared=64, seed=23)),
                       ("tiny", dict(routing="hash", vocab=97, seed=24, T=9))):
        from synthetic import CONFIGS
        cfg = dict(CONFIGS[name])
        cfg.update(over)
        inp = make_custom(cfg)
        res = oracle_run(inp)
        dense = _dense_reference(inp, res)
        rel = np.abs(res["out"] - dense).max() / np.abs(dense).max()
        assert rel < 1e-12, (over, rel)


def pin_single_expert_swiglu():
    """E=1, k=1: the layer is one plain SwiGLU FFN with routing weight 1."""
    cfg = dict(T=7, d=64, E=1, k=1, f=96, routing="learned", vocab=0,
               w13=("affine", 4, 32), w2=("affine", 4, 32), shared=None, f_shared=0,
               weight_std=0.05, bias_std=0.1, seed=31)
    inp = make_custom(cfg)
    res = oracle_run(inp)
    assert np.all(res["ids"] == 0) and np.all(res["w"] == 1.0)
    W = [torch.from_numpy(oracle.dequant("affine", 4, 32, n, *m.expert_numpy(0)))
         for m, n in ((inp.w1, 64), (inp.w3, 64), (inp.w2, 96))]
    xd = inp.x.double()
    want = F.linear(F.silu(F.linear(xd, W[0])) * F.linear(xd, W[1]), W[2]).numpy()
    assert np.allclose(res["out"], want, rtol=1e-12, atol=1e-14)


def pin_round_bf16():
    g = torch.Generator().manual_seed(3)
    a = torch.randn(100000, generator=g) * torch.exp(torch.randn(100000, generator=g) * 5)
    lib = a.to(torch.bfloat16).double().numpy()           # torch: fp32 -> bf16 RNE
    got = oracle.round_bf16(a.double().numpy())
    assert np.array_equal(got, lib)
    # exact halfway cases: 1 + 2^-8 (tie, even is 1), 1 + 3*2^-8 (tie, even is 1+2^-6)
    assert oracle.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert oracle.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


# ---------------------------------------------------------------- parity harness
def pin_parity_stats():
    """The output tolerance statistics on hand-computed vectors.

    ref = [3, -4, 0, 1], out = [3.5, -4, 0.25, 1]: |err| = [0.5, 0, 0.25, 0],
    max|err| = 0.5, rms(ref) = sqrt(26/4), sum|err| / sum|ref| = 0.75 / 8.
    A second case has a zero in ref where out is not zero (an elementwise
    relative error would be infinite there) and out's rms differing from ref's.
    """
    st = oracle.parity_stats(np.array([3.5, -4.0, 0.25, 1.0]), np.array([3.0, -4.0, 0.0, 1.0]))
    assert st["max_err"] == 0.5
    assert abs(st["rms_ref"] - math.sqrt(6.5)) < 1e-15
    assert abs(st["max_err_over_rms"] - 0.5 / math.sqrt(6.5)) < 1e-15
    assert abs(st["mean_rel_err"] - 0.09375) < 1e-15
    st = oracle.parity_stats(np.array([[0.0, 2.0], [10.0, 1.0]]), np.array([[1.0, 0.0], [2.0, 1.0]]))
    # |err| = [1, 2, 8, 0]; rms(ref) = sqrt(6/4); sum|ref| = 4
    assert st["max_err"] == 8.0
    assert abs(st["max_err_over_rms"] - 8.0 / math.sqrt(1.5)) < 1e-14
    assert abs(st["mean_rel_err"] - 11.0 / 4.0) < 1e-15
    # identical arrays: zero error; the statistics are symmetric in nothing else
    z = oracle.parity_stats(np.ones(5), np.ones(5))
    assert z["max_err"] == 0.0 and z["mean_rel_err"] == 0.0 and z["rms_ref"] == 1.0


def pin_forward_token_subset():
    """forward(tokens=S) gives, for each token of S, the row the all-tokens
    run gives (same routing, same slot outputs, same combine), up to fp64
    rounding order (BLAS blocks a matrix product differently per batch)."""
    from synthetic import CONFIGS
    for name, over, subset in (("tiny", {}, [3, 0, 2]),
                               ("tiny", dict(shared=("affine", 8, 64), f_shared=64, T=9, seed=41), [8, 1, 1, 4]),
                               ("tiny", dict(routing="hash", vocab=61, T=7, seed=42), [6, 2])):
        cfg = dict(CONFIGS[name])
        cfg.update(over)
        inp = make_custom(cfg)
        full = oracle_run(inp)
        part = oracle_run(inp, tokens=subset)
        assert list(part["tokens"]) == list(subset)
        for a, t in enumerate(subset):
            scale = np.abs(full["out"]).max()
            assert np.allclose(part["out"][a], full["out"][t], rtol=1e-12, atol=1e-13 * scale), (over, t)
            assert np.allclose(part["y_slots"][a], full["y_slots"][t], rtol=1e-12, atol=1e-13 * scale), (over, t)
        assert np.array_equal(part["ids"], full["ids"]) and np.array_equal(part["w"], full["w"])


def pin_forced_routing():
    """Forced routing: with the oracle's own ids it reproduces the free run;
    with other ids the output is the dense mixture gated by those ids with
    weights = renormalised sqrtsoftplus of their fp64 logits (scipy softplus),
    whatever the selection bias; slot order permutes weights and slot outputs
    only."""
    from scipy.special import softplus
    from synthetic import CONFIGS
    cfg = dict(CONFIGS["tiny"])
    cfg.update(T=6, seed=43, bias_std=0.3)
    inp = make_custom(cfg)
    free = oracle_run(inp)
    same = oracle_run(inp, forced_ids=free["ids"])
    assert np.array_equal(same["out"], free["out"]) and np.array_equal(same["w"], free["w"])
    rng = np.random.default_rng(44)
    T, E, k = cfg["T"], cfg["E"], cfg["k"]
    forced = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    res = oracle_run(inp, forced_ids=forced)
    assert np.array_equal(res["ids"], forced) and np.array_equal(res["free_ids"], free["ids"])
    assert np.array_equal(res["gap"], free["gap"])
    L = inp.x.double().numpy() @ inp.router_w.double().numpy().T
    s = np.sqrt(softplus(L))
    sel = np.take_along_axis(s, forced, 1)
    assert np.allclose(res["w"], sel / sel.sum(1, keepdims=True), rtol=1e-12)
    dense = _dense_reference(inp, {"ids": forced, "w": sel / sel.sum(1, keepdims=True)})
    assert np.abs(res["out"] - dense).max() / np.abs(dense).max() < 1e-12
    swapped = forced[:, ::-1].copy()
    res2 = oracle_run(inp, forced_ids=swapped)
    assert np.allclose(res2["w"], res["w"][:, ::-1], rtol=1e-15)
    assert np.allclose(res2["out"], res["out"], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- mHC Sinkhorn mixing
def pin_hc_sinkhorn_softmax():
    """Zero iterations: the row-wise softmax (scipy); rows sum to one after
    any number of iterations, columns approach one as they grow."""
    from scipy.special import softmax
    rng = np.random.default_rng(51)
    L = rng.normal(scale=2.0, size=(6, 4, 4))
    assert np.allclose(oracle.hc_sinkhorn(L, 0), softmax(L, axis=-1), rtol=1e-14, atol=1e-16)
    errs = []
    for it in (1, 3, 10, 40, 300):
        P = oracle.hc_sinkhorn(L, it)
        assert np.abs(P.sum(-1) - 1).max() < 1e-14
        errs.append(np.abs(P.sum(-2) - 1).max())
    assert errs[-1] < 1e-9 and errs == sorted(errs, reverse=True)


def pin_hc_sinkhorn_limits():
    """The Sinkhorn limit of a positive matrix A is the unique doubly
    stochastic D1 A D2.  For 2x2 it has the closed form [[p, 1-p], [1-p, p]],
    p = sqrt(ad) / (sqrt(ad) + sqrt(bc)); for 4x4 it is checked against an
    independent solve of u_i sum_j A_ij v_j = 1 = v_j sum_i A_ij u_i
    (scipy root finding on log u, log v).  The limit is invariant under
    positive diagonal scalings, i.e. adding r_i + c_j to the logits."""
    from scipy.optimize import root
    rng = np.random.default_rng(52)
    for _ in range(5):
        L = rng.normal(size=(1, 2, 2))
        A = np.exp(L[0])
        a, b, c, d = A[0, 0], A[0, 1], A[1, 0], A[1, 1]
        pp = math.sqrt(a * d) / (math.sqrt(a * d) + math.sqrt(b * c))
        want = np.array([[pp, 1 - pp], [1 - pp, pp]])
        assert np.abs(oracle.hc_sinkhorn(L, 200)[0] - want).max() < 1e-12
    for _ in range(3):
        L = rng.normal(size=(1, 4, 4))
        A = np.exp(L[0])

        def eqs(z):
            u, v = np.exp(z[:4]), np.exp(z[4:])
            return np.concatenate([u * (A @ v) - 1, v * (A.T @ u) - 1])

        sol = root(eqs, np.zeros(8), tol=1e-14)
        u, v = np.exp(sol.x[:4]), np.exp(sol.x[4:])
        want = u[:, None] * A * v[None, :]
        assert np.abs(oracle.hc_sinkhorn(L, 500)[0] - want).max() < 1e-10
        shifted = L + rng.normal(size=(1, 4, 1)) + rng.normal(size=(1, 1, 4))
        assert np.abs(oracle.hc_sinkhorn(shifted, 500)[0] - want).max() < 1e-10


def pin_hc_sinkhorn_fixed_point():
    """A doubly stochastic matrix (a mixture of permutation matrices) given
    as logits log(P) comes back unchanged after any number of iterations."""
    rng = np.random.default_rng(53)
    perms = [np.eye(4)[rng.permutation(4)] for _ in range(5)]
    wts = rng.dirichlet(np.ones(5))
    P0 = sum(w * m for w, m in zip(wts, perms)) * 0.9 + 0.1 / 4   # strictly positive, doubly stochastic
    for it in (0, 1, 20):
        assert np.abs(oracle.hc_sinkhorn(np.log(P0)[None], it)[0] - P0).max() < 1e-14


def pin_hc_mix():
    """The n -> n mix against torch.bmm in fp64; a permutation matrix moves
    the copies."""
    rng = np.random.default_rng(54)
    P = rng.random(size=(3, 4, 4))
    h = rng.normal(size=(3, 4, 16))
    want = torch.bmm(torch.from_numpy(P), torch.from_numpy(h)).numpy()
    assert np.allclose(oracle.hc_mix(P, h), want, rtol=1e-14, atol=1e-14)
    perm = np.eye(4)[[2, 0, 3, 1]][None]
    assert np.array_equal(oracle.hc_mix(perm, h[:1])[0], h[0][[2, 0, 3, 1]])


def pin_bf16_router_is_its_values():
    """A bf16-stored router gate routes exactly like an fp32 gate holding the
    same (widened) values: the logits are fp32-or-wider dot products of the
    stored values, so the oracle's routing depends on the values only --
    checked against torch's bf16 -> fp64 widening and F.linear."""
    from synthetic import CONFIGS
    cfg = dict(CONFIGS["tiny"], T=9, seed=45, router_dtype="bf16")
    inp = make_custom(cfg)
    assert inp.router_w.dtype == torch.bfloat16
    wide = inp.router_w.double()
    res = oracle_run(inp)
    want = F.linear(inp.x.double(), wide).numpy()
    assert np.allclose(res["logits"], want, rtol=1e-13, atol=1e-13)
    ids, w, _, _ = oracle.route_learned(inp.x.double().numpy(), wide.numpy(), inp.router_b.double().numpy(), cfg["k"])
    assert np.array_equal(ids, res["ids"]) and np.array_equal(w, res["w"])


def pin_expert_partition():
    """Expert parallelism: the partial of an expert range is the dense
    mixture gated by the routing weights of the owned experts only (library
    fp64 linear/silu on every expert), the shared expert added once; partials
    over a partition of [0, E) (shared in one part) add up to the full layer,
    and an empty range gives zero (or the shared expert alone)."""
    from synthetic import CONFIGS
    cfg = dict(CONFIGS["tiny"])
    cfg.update(T=5, seed=51, shared=("affine", 8, 64), f_shared=128)
    inp = make_custom(cfg)
    full = oracle_run(inp)
    E = cfg["E"]
    cuts = [(0, 3), (3, 5), (5, E)]  # (3, 5) owns no (token, slot) pair of this draw: its partial is 0
    parts = [oracle_run(inp, expert_range=r, include_shared=(i == 0)) for i, r in enumerate(cuts)]
    total = sum(p["out"] for p in parts)
    assert np.abs(total - full["out"]).max() / np.abs(full["out"]).max() < 1e-13
    for i, (r, p) in enumerate(zip(cuts, parts)):
        assert np.array_equal(p["ids"], full["ids"]) and np.array_equal(p["w"], full["w"])
        owned = (full["ids"] >= r[0]) & (full["ids"] < r[1])
        gated = {"ids": full["ids"], "w": np.where(owned, full["w"], 0.0)}
        dense = _dense_reference(inp, gated)
        if i > 0:  # the dense reference always adds the shared expert: take it out for the other parts
            dense = dense - oracle_run(inp, expert_range=(0, 0))["out"]
        assert np.abs(p["out"] - dense).max() / np.abs(full["out"]).max() < 1e-12
    assert not parts[1]["out"].any()
    none = oracle_run(inp, expert_range=(0, 0), include_shared=False)
    assert not none["out"].any()
    shared_only = oracle_run(inp, expert_range=(2, 2))
    assert np.allclose(shared_only["out"], full["y_shared"], rtol=0, atol=0)


ALL_PINS = [pin_e2m1_table, pin_e8m0, pin_unpack_golden, pin_unpack_bigint, pin_affine_dequant,
            pin_mxfp4_dequant, pin_sqrtsoftplus, pin_topk_bruteforce, pin_route_learned,
            pin_route_hash, pin_permutation, pin_dense_equivalence, pin_single_expert_swiglu,
            pin_round_bf16, pin_e4m3_table, pin_mxfp8_dequant, pin_block128_scales, pin_parity_stats,
            pin_forward_token_subset, pin_forced_routing, pin_hc_sinkhorn_softmax, pin_hc_sinkhorn_limits,
            pin_hc_sinkhorn_fixed_point, pin_hc_mix, pin_bf16_router_is_its_values, pin_expert_partition]
