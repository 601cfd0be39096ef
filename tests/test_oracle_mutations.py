"""Plant plausible mistakes in the oracle (on the CPU) and check a pin fails.

Each case monkeypatches one oracle function or table with a realistic bug --
a flipped sign, an off-by-one exponent bias, the wrong bit order, a dropped
term, a wrong tie-break -- and asserts that at least one pin raises.
"""
import numpy as np
import pytest

import oracle
import oracle.moe_oracle as om
from tests import pins


def _msb_first_unpack(words, bits, n):
    w = np.ascontiguousarray(np.asarray(words).astype("<u4"))
    stream = np.unpackbits(w.view(np.uint8), axis=-1, bitorder="big")
    stream = stream[..., : n * bits].reshape(*w.shape[:-1], n, bits).astype(np.int64)
    return (stream * (1 << np.arange(bits))).sum(-1)


def _no_bias_dequant(words, scales, biases, bits, group, n_in):
    q = om.unpack_codes(words, bits, n_in).astype(np.float64)
    return np.repeat(np.asarray(scales, np.float64), group, -1) * q


def _naive_sqrtsoftplus(L):
    with np.errstate(over="ignore"):
        return np.sqrt(np.log(1.0 + np.exp(np.asarray(L, np.float64))))


def _tie_high_topk(keys, k):
    keys = np.asarray(keys, np.float64)
    order = np.argsort(-keys[:, ::-1], axis=1, kind="stable")
    order = keys.shape[1] - 1 - order
    ids = order[:, :k]
    srt = np.take_along_axis(keys, order, 1)
    gap = srt[:, k - 1] - srt[:, k] if keys.shape[1] > k else np.full(keys.shape[0], np.inf)
    return ids, gap


def _bad_silu(a):
    return a / (1.0 + np.exp(a))


def _unweighted_combine(y, w, y_shared=None):
    out = np.asarray(y, np.float64).sum(1)
    return out if y_shared is None else out + y_shared


def _bad_e2m1():
    t = om.E2M1_VALUES.copy()
    t[8:] = -t[8:]          # sign bit ignored
    return t


def _bad_e4m3():
    t = om.E4M3_VALUES.copy()
    return t * 0.5          # exponent bias 8 instead of 7


def _block_scales_wrong_group(bs, n_out, n_in):
    # eight 32-input groups per block (the word count per scale) instead of four
    bs = np.asarray(bs)
    g = np.minimum(np.arange(n_in // 32) // 8, bs.shape[1] - 1)
    return bs[(np.arange(n_out) // 128)[:, None], g[None, :]]


def _round_trunc(a):
    m, e = np.frexp(np.asarray(a, np.float64))
    return np.ldexp(np.trunc(m * 256) / 256, e)


def _stats_rms_of_out(out, ref):
    st = _ORIG_STATS(out, ref)
    out = np.asarray(out, np.float64)
    rms = float(np.sqrt(np.mean(out * out)))
    st["rms_ref"] = rms
    st["max_err_over_rms"] = st["max_err"] / rms if rms > 0 else 0.0
    return st


def _stats_mean_err(out, ref):
    st = _ORIG_STATS(out, ref)
    err = np.abs(np.asarray(out, np.float64) - np.asarray(ref, np.float64))
    st["mean_rel_err"] = float(err.mean() / np.abs(np.asarray(ref, np.float64)).sum())
    return st


def _stats_elementwise_rel(out, ref):
    st = _ORIG_STATS(out, ref)
    out, ref = np.asarray(out, np.float64), np.asarray(ref, np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        st["mean_rel_err"] = float(np.mean(np.abs(out - ref) / np.abs(ref)))
    return st


def _forced_biased_weights(x, w_router, forced_ids):
    # weights from the biased keys would need the bias; a plausible slip is
    # to take the weights without renormalising them
    ids = np.asarray(forced_ids, np.int64)
    s = om.sqrtsoftplus(om.router_logits(x, w_router))
    return ids, np.take_along_axis(s, ids, axis=1), None


def _sk_rows_first(logits, iters, eps=0.0):
    L = np.asarray(logits, np.float64)
    P = np.exp(L - L.max(-1, keepdims=True))
    P = P / P.sum(-1, keepdims=True)
    for _ in range(iters):
        P = P / (P.sum(-1, keepdims=True) + eps)
        P = P / (P.sum(-2, keepdims=True) + eps)
    return P


def _sk_column_softmax(logits, iters, eps=0.0):
    L = np.asarray(logits, np.float64)
    P = np.exp(L - L.max(-2, keepdims=True))
    P = P / P.sum(-2, keepdims=True)
    for _ in range(iters):
        P = P / (P.sum(-2, keepdims=True) + eps)
        P = P / (P.sum(-1, keepdims=True) + eps)
    return P


def _sk_no_exp(logits, iters, eps=0.0):
    P = np.abs(np.asarray(logits, np.float64))
    P = P / P.sum(-1, keepdims=True)
    for _ in range(iters):
        P = P / (P.sum(-2, keepdims=True) + eps)
        P = P / (P.sum(-1, keepdims=True) + eps)
    return P


def _mix_transposed(P, h):
    return np.einsum("tji,tjd->tid", np.asarray(P, np.float64), np.asarray(h, np.float64))


_ORIG_STATS = om.parity_stats


MUTATIONS = [
    ("E2M1_VALUES", _bad_e2m1(), [pins.pin_e2m1_table, pins.pin_mxfp4_dequant]),
    ("e8m0_value", lambda e: np.ldexp(1.0, np.asarray(e, np.int64) - 128), [pins.pin_e8m0, pins.pin_mxfp4_dequant]),
    ("unpack_codes", _msb_first_unpack, [pins.pin_unpack_golden, pins.pin_unpack_bigint]),
    ("dequant_affine", _no_bias_dequant, [pins.pin_affine_dequant]),
    ("sqrtsoftplus", _naive_sqrtsoftplus, [pins.pin_sqrtsoftplus]),
    ("sqrtsoftplus", lambda L: np.maximum(L, 0) + np.log1p(np.exp(-np.abs(L))), [pins.pin_sqrtsoftplus, pins.pin_route_learned]),
    ("topk_select", _tie_high_topk, [pins.pin_topk_bruteforce]),
    ("silu", _bad_silu, [pins.pin_single_expert_swiglu, pins.pin_dense_equivalence]),
    ("combine", _unweighted_combine, [pins.pin_dense_equivalence]),
    ("round_bf16", _round_trunc, [pins.pin_round_bf16]),
    ("E4M3_VALUES", _bad_e4m3(), [pins.pin_e4m3_table, pins.pin_mxfp8_dequant]),
    ("block128_scales_to_group32", _block_scales_wrong_group, [pins.pin_block128_scales]),
    ("parity_stats", _stats_rms_of_out, [pins.pin_parity_stats]),
    ("parity_stats", _stats_mean_err, [pins.pin_parity_stats]),
    ("parity_stats", _stats_elementwise_rel, [pins.pin_parity_stats]),
    ("route_forced", _forced_biased_weights, [pins.pin_forced_routing]),
    ("hc_sinkhorn", _sk_rows_first, [pins.pin_hc_sinkhorn_softmax]),
    ("hc_sinkhorn", _sk_column_softmax, [pins.pin_hc_sinkhorn_softmax]),
    ("hc_sinkhorn", _sk_no_exp, [pins.pin_hc_sinkhorn_limits]),
    ("hc_mix", _mix_transposed, [pins.pin_hc_mix]),
]


@pytest.mark.parametrize("name,bad,catchers", MUTATIONS, ids=[f"{m[0]}-{i}" for i, m in enumerate(MUTATIONS)])
def test_planted_mistake_is_caught(monkeypatch, name, bad, catchers):
    monkeypatch.setattr(om, name, bad)
    monkeypatch.setattr(oracle, name, bad, raising=False)
    for pin in catchers:
        with pytest.raises(AssertionError):
            pin()
