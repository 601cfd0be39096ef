"""fp64 CPU oracle for the DeepSeek-V4-style routed MoE FFN over low-bit packs.

TEST INFRASTRUCTURE ONLY.  Only tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the library never does, and this
module imports nothing from the library.

Sources (web pages about running DeepSeek-V4-Flash with MLX), cited by title
and section:

[PR1192]  mlx-lm pull request "Add DeepSeek-v4 (Flash/Pro)" -- the
          "sqrtsoftplus numerical stability" note (softplus via
          logaddexp(x, 0)) and the cross-reference table row "MoE gate dtype"
          (router logits computed in fp32 in both the top-k and the hash
          router); the weight-key notes naming the pre-stacked experts
          w1/w2/w3 = gate/down/up projections of the switch MLP; the
          dequantise notes for mode="mxfp4" with group_size=32.
[CARD-4BIT]   model card "mlx-community / DeepSeek-V4-Flash-4bit",
          Architecture list ("Hash-routed MoE": deterministic tid2eid table
          in the first layers; "sqrtsoftplus scoring": sqrt(softplus(x))
          replaces softmax) and Conversion (affine 4-bit, group 64).
[CARD-MLX4]   model card "DeepSeek-V4-Flash-MLX-4bit", section
          "REAP-pruned builds" (the router renormalises over the experts it
          keeps; hash layers route through a fixed tid2eid table) and the
          table "What this port implements" (tid2eid keyed on token id,
          routing independent of context); FP4 e2m1 packed two per byte.
[PR1190]  mlx-lm pull request "Add DeepSeek-V4 model and safetensors/tokenizer
          fallback handling" -- description: E8M0 scales are unsigned
          exponents, 2^(b-127).
[PR1192-FP8]  the same pull request's review thread on re-quantising from the
          FP8 source: e4m3 weight bytes with e8m0 block scales decode through
          MLX's mxfp8 mode with group_size=32 (four weight bytes per uint32
          word, eight words per scale); the checkpoint's 128x128 block
          scales are repeated four times along the input axis and 128 times
          along the output axis to reach that grouping.
[CARD-MLX4-SRC]  model card "DeepSeek-V4-Flash-MLX-4bit", the note after
          "What this port implements": the source checkpoint stores most
          matmuls as FP8 e4m3 with e8m0 128x128 block scales.
[PR1192-SK]  the same pull request's review note "Sinkhorn normalization":
          the reference path is a softmax followed by a loop of sum-and-divide
          steps (about forty launches per call), which a fused kernel does in
          one register-resident pass.
[CARD-4BIT-MHC]  model card "mlx-community / DeepSeek-V4-Flash-4bit",
          Architecture ("mHC": hc_mult = 4 parallel copies of the hidden
          state recombined through a doubly-stochastic, Sinkhorn-normalised
          mixing matrix) and Performance (the fused Sinkhorn kernel).
[CARD-MIXED]  model card "DeepSeek-V4-Flash-0731-MLX-Serve-mixed-2-3-8bit",
          precision table (w1/w3 affine 2-bit g128, w2 affine 3-bit g128,
          shared experts 8-bit g64) and conversion notes (fp4 e2m1 with e8m0
          group scales decodes losslessly; expert packs use MLX's affine
          layout, w = scale*q + bias).

Readings taken where the pages are silent (each is also listed with the
design notes): the router bias is added to the scores for selection only and
the weights use the unbiased scores; ties in top-k go to the lower expert
index; routing weights are renormalised over the k selected experts with a
scaling factor of 1; the hash router's weights are the renormalised
sqrtsoftplus scores of the table's experts (uniform 1/k when no router weight
is given); affine codes are an LSB-first bitstream along the input dimension;
mxfp4 puts the even element in the low nibble and uses code bit 3 as the
sign; the shared expert is added with weight 1; per-expert token lists are in
ascending flat-index order t*k+j.
"""
from __future__ import annotations

from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "E2M1_VALUES", "E4M3_VALUES", "unpack_codes", "e8m0_value", "dequant_affine", "dequant_mxfp4",
    "dequant_mxfp8", "block128_scales_to_group32",
    "dequant", "router_logits", "sqrtsoftplus", "topk_select", "renormalize",
    "route_learned", "route_hash", "route_forced", "permute", "silu", "swiglu_ffn", "combine",
    "round_bf16", "forward", "parity_stats", "hc_sinkhorn", "hc_mix",
]

# --------------------------------------------------------------------------
# Weight decode  [CARD-MIXED conversion notes; CARD-MLX4; PR1190; PR1192]
# --------------------------------------------------------------------------
# e2m1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; exponent 0 is
# subnormal (0 or 0.5).  Code 8 is negative zero.
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
                        -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0], dtype=np.float64)



def _e4m3_table() -> np.ndarray:
    """e4m3 (the "fn" variant: no infinities): sign bit 7, exponent bits 6..3
    with bias 7, mantissa bits 2..0; exponent 0 is subnormal (m/8 * 2^-6);
    exponent 15 with mantissa 7 is NaN, so the largest finite value is 448."""
    out = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        exp = (code >> 3) & 0xF
        man = code & 0x7
        if exp == 0xF and man == 0x7:
            out[code] = np.nan
        elif exp == 0:
            out[code] = sign * (man / 8.0) * 2.0 ** -6
        else:
            out[code] = sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)
    return out


E4M3_VALUES = _e4m3_table()


def unpack_codes(words: np.ndarray, bits: int, n: int) -> np.ndarray:
    """Integer codes from an LSB-first little-endian bitstream.

    ``words``: uint32 ``[..., nw]`` (one row's stream in the last axis).
    Returns int64 ``[..., n]``; code ``i`` is bits ``[i*bits, (i+1)*bits)``.
    """
    w = np.ascontiguousarray(np.asarray(words).astype("<u4"))
    stream = np.unpackbits(w.view(np.uint8), axis=-1, bitorder="little")
    if stream.shape[-1] < n * bits:
        raise ValueError("bitstream shorter than n*bits")
    stream = stream[..., : n * bits].reshape(*w.shape[:-1], n, bits).astype(np.int64)
    place = (np.int64(1) << np.arange(bits, dtype=np.int64))
    return (stream * place).sum(axis=-1)


def e8m0_value(e: np.ndarray) -> np.ndarray:
    """E8M0 scale byte -> 2^(e-127)  [PR1190 description]."""
    return np.ldexp(1.0, np.asarray(e, dtype=np.int64) - 127)


def dequant_affine(words, scales, biases, bits: int, group: int, n_in: int) -> np.ndarray:
    """W[o, i] = scale[o, i//group] * q[o, i] + bias[o, i//group], in fp64."""
    q = unpack_codes(words, bits, n_in).astype(np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), group, axis=-1)
    b = np.repeat(np.asarray(biases, dtype=np.float64), group, axis=-1)
    return s * q + b


def dequant_mxfp4(words, scales_u8, n_in: int) -> np.ndarray:
    """W[o, i] = e2m1(code[o, i]) * 2^(e[o, i//32] - 127), in fp64."""
    c = unpack_codes(words, 4, n_in)
    return E2M1_VALUES[c] * np.repeat(e8m0_value(scales_u8), 32, axis=-1)


def dequant_mxfp8(words, scales_u8, n_in: int) -> np.ndarray:
    """W[o, i] = e4m3(byte i of row o) * 2^(e[o, i//32] - 127), in fp64
    [PR1192-FP8].  Bytes are the same LSB-first stream with 8-bit codes:
    byte i of a row is element i."""
    c = unpack_codes(words, 8, n_in)
    return E4M3_VALUES[c] * np.repeat(e8m0_value(scales_u8), 32, axis=-1)


def block128_scales_to_group32(block_scales, n_out: int, n_in: int) -> np.ndarray:
    """Per-(row, 32-input group) e8m0 bytes from 128x128 block scales
    [CARD-MLX4-SRC; PR1192-FP8]: row o, group g takes block (o // 128, g // 4)."""
    bs = np.asarray(block_scales)
    rows = np.arange(n_out) // 128
    groups = np.arange(n_in // 32) // 4
    return bs[rows[:, None], groups[None, :]]


def dequant(fmt: str, bits: int, group: int, n_in: int, words, scales, biases) -> np.ndarray:
    if fmt == "affine":
        return dequant_affine(words, scales, biases, bits, group, n_in)
    if fmt == "mxfp4":
        return dequant_mxfp4(words, scales, n_in)
    if fmt == "mxfp8":
        return dequant_mxfp8(words, scales, n_in)
    raise ValueError(fmt)


# --------------------------------------------------------------------------
# Routing  [PR1192 gate dtype + sqrtsoftplus note; CARD-4BIT Architecture;
#           CARD-MLX4 REAP section and port table]
# --------------------------------------------------------------------------
def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """L = x . W^T in fp64 (the pages demand at least fp32)."""
    return np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T


def sqrtsoftplus(logits: np.ndarray) -> np.ndarray:
    """sqrt(softplus(L)) with softplus(L) = logaddexp(L, 0) written stably."""
    L = np.asarray(logits, np.float64)
    return np.sqrt(np.maximum(L, 0.0) + np.log1p(np.exp(-np.abs(L))))


def topk_select(keys: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per row, the k largest keys; equal keys go to the lower expert index.

    Returns (ids [T, k] in descending key order, gap [T] = k-th minus
    (k+1)-th largest key, +inf when every expert is selected).
    """
    keys = np.asarray(keys, np.float64)
    order = np.argsort(-keys, axis=1, kind="stable")
    ids = order[:, :k]
    srt = np.take_along_axis(keys, order, axis=1)
    if keys.shape[1] > k:
        gap = srt[:, k - 1] - srt[:, k]
    else:
        gap = np.full(keys.shape[0], np.inf)
    return ids.astype(np.int64), gap


def renormalize(s_sel: np.ndarray) -> np.ndarray:
    """w = s / sum(s) over the selected experts (uniform if the sum is 0)."""
    s_sel = np.asarray(s_sel, np.float64)
    tot = s_sel.sum(axis=1, keepdims=True)
    k = s_sel.shape[1]
    with np.errstate(invalid="ignore", divide="ignore"):
        w = np.where(tot > 0, s_sel / np.where(tot > 0, tot, 1.0), 1.0 / k)
    return w


def route_learned(x, w_router, b_router, k: int):
    """Learned top-k routing.

    score = sqrtsoftplus(x.W^T); key = score + bias (selection only);
    ids = top-k(key); weights = renormalised unbiased scores of the ids.
    """
    L = router_logits(x, w_router)
    s = sqrtsoftplus(L)
    keys = s if b_router is None else s + np.asarray(b_router, np.float64)[None, :]
    ids, gap = topk_select(keys, k)
    w = renormalize(np.take_along_axis(s, ids, axis=1))
    return ids, w, gap, L


def route_hash(x, w_router, token_ids, tid2eid):
    """Hash routing: ids = tid2eid[token_id] in table column order.

    Weights: renormalised sqrtsoftplus of the router logits of those experts
    (both router kinds compute fp32 logits); uniform 1/k without a router.
    """
    ids = np.asarray(tid2eid)[np.asarray(token_ids, np.int64)].astype(np.int64)
    k = ids.shape[1]
    if w_router is None:
        return ids, np.full(ids.shape, 1.0 / k)
    xs = np.asarray(x, np.float64)
    wr = np.asarray(w_router, np.float64)
    L = np.einsum("td,tkd->tk", xs, wr[ids])
    return ids, renormalize(sqrtsoftplus(L))


# --------------------------------------------------------------------------
# Permutation: stable grouping of the T*k (token, slot) pairs by expert
# --------------------------------------------------------------------------
def permute(ids: np.ndarray, n_experts: int):
    """Returns (expert_offsets [E+1], sorted_rows [T*k], inv [T*k]).

    sorted_rows lists flat indices t*k+j grouped by expert, ascending within
    each expert; inv[sorted_rows[p]] = p.
    """
    flat = np.asarray(ids, np.int64).reshape(-1)
    rows, offsets = [], [0]
    for e in range(n_experts):
        r = np.nonzero(flat == e)[0]
        rows.append(r)
        offsets.append(offsets[-1] + len(r))
    sorted_rows = np.concatenate(rows) if rows else np.zeros(0, np.int64)
    inv = np.empty_like(sorted_rows)
    inv[sorted_rows] = np.arange(len(sorted_rows))
    return np.asarray(offsets, np.int64), sorted_rows.astype(np.int64), inv


# --------------------------------------------------------------------------
# Expert FFN (SwiGLU) and combine
# --------------------------------------------------------------------------
def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def swiglu_ffn(W1: np.ndarray, W3: np.ndarray, W2: np.ndarray, xs: np.ndarray) -> np.ndarray:
    """y = W2 . (silu(W1 . x) * (W3 . x)) for each row of xs ([n, d] -> [n, d])."""
    xs = np.asarray(xs, np.float64)
    g = xs @ W1.T
    u = xs @ W3.T
    return (silu(g) * u) @ W2.T


def combine(y_slots: np.ndarray, w: np.ndarray, y_shared: Optional[np.ndarray] = None) -> np.ndarray:
    """out[t] = sum_j w[t, j] * y[t, j] (+ shared expert output, weight 1)."""
    out = np.einsum("tk,tkd->td", np.asarray(w, np.float64), np.asarray(y_slots, np.float64))
    if y_shared is not None:
        out = out + y_shared
    return out


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (ties to even); returns fp64."""
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)                  # a = m * 2^e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits: scale the mantissa to [128, 256)
    r = np.rint(m * 256.0)              # np.rint rounds half to even
    out = np.ldexp(r / 256.0, e)
    return np.where(np.isfinite(a), out, a)


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------
ExpertFetch = Callable[[str, int], Tuple[np.ndarray, np.ndarray, Optional[np.ndarray]]]


def route_forced(x, w_router, forced_ids):
    """Forced routing: the experts are given (e.g. the ids another
    implementation selected for a token whose k-th and (k+1)-th keys nearly
    tie); the weights are computed for them exactly as in learned routing,
    w = s[ids] / sum(s[ids]) with the unbiased scores, in the given slot order.
    """
    ids = np.asarray(forced_ids, np.int64)
    L = router_logits(x, w_router)
    s = sqrtsoftplus(L)
    return ids, renormalize(np.take_along_axis(s, ids, axis=1)), L


def forward(dims: Dict, x: np.ndarray, *, router_w=None, router_b=None, token_ids=None,
            tid2eid=None, fetch: ExpertFetch, fmts: Dict[str, Tuple[str, int, int]],
            shared_fetch: Optional[ExpertFetch] = None, shared_fmts=None,
            tokens: Optional[Sequence[int]] = None,
            forced_ids: Optional[np.ndarray] = None,
            expert_range: Optional[Tuple[int, int]] = None,
            include_shared: bool = True) -> Dict[str, np.ndarray]:
    """Run the layer for all tokens' routing and the requested tokens' outputs.

    dims: T, d, E, k, f, f_shared, routing ("learned"|"hash").
    fetch(name, e) -> packs of expert e for name in {"w1","w3","w2"}.
    fmts[name] = (fmt, bits, group).  tokens: subset whose outputs are wanted
    (default: all).  Routing is computed for every token.
    forced_ids: int [T, k] -- learned routing only: use these experts instead
    of the top-k selection (weights as in route_forced); "gap" is then the
    free routing's gap, so near-tie tokens can still be recognised.
    expert_range: (begin, end) -- expert parallelism: routing over all E
    experts as usual, but only experts begin <= e < end are run and only their
    slots enter the combine; the shared expert is added when include_shared.
    The layer's output is the sum of such partials over a partition of
    [0, E) with the shared expert in exactly one of them, because the combine
    is a sum over (token, slot) terms.
    """
    T, d, E, k, f = dims["T"], dims["d"], dims["E"], dims["k"], dims["f"]
    xs = np.asarray(x, np.float64)
    res: Dict[str, np.ndarray] = {}
    if dims["routing"] == "hash":
        if forced_ids is not None:
            raise ValueError("forced routing applies to learned routing only")
        ids, w = route_hash(xs, router_w, token_ids, tid2eid)
        gap = np.full(T, np.inf)
    else:
        ids, w, gap, L = route_learned(xs, router_w, router_b, k)
        res["logits"] = L
        # the selection keys, so a caller can check that another selection
        # of a near-tie token is also a valid top-k
        res["keys"] = sqrtsoftplus(L) + (0.0 if router_b is None else np.asarray(router_b, np.float64)[None, :])
        if forced_ids is not None:
            res["free_ids"] = ids
            ids, w, _ = route_forced(xs, router_w, forced_ids)
    res["ids"], res["w"], res["gap"] = ids, w, gap
    offs, rows, inv = permute(ids, E)
    res["expert_offsets"], res["sorted_rows"], res["inv"] = offs, rows, inv

    tok = np.arange(T) if tokens is None else np.asarray(tokens, np.int64)
    y = np.zeros((len(tok), k, d))
    eb, ee = (0, E) if expert_range is None else (int(expert_range[0]), int(expert_range[1]))
    if not 0 <= eb <= ee <= E:
        raise ValueError(f"expert_range {expert_range} outside [0, {E}]")
    owned = (ids >= eb) & (ids < ee)
    need: Dict[int, list] = {}
    for a, t in enumerate(tok):
        for j in range(k):
            if owned[t, j]:
                need.setdefault(int(ids[t, j]), []).append((a, j))
    dims_of = {"w1": (f, d), "w3": (f, d), "w2": (d, f)}
    for e in sorted(need):
        W = {}
        for name in ("w1", "w3", "w2"):
            fm, bits, grp = fmts[name]
            W[name] = dequant(fm, bits, grp, dims_of[name][1], *fetch(name, e))
        xs_e = np.stack([xs[tok[a]] for a, _ in need[e]])
        ye = swiglu_ffn(W["w1"], W["w3"], W["w2"], xs_e)
        for r, (a, j) in enumerate(need[e]):
            y[a, j] = ye[r]
    y_sh = None
    if shared_fetch is not None and include_shared:
        fs = dims["f_shared"]
        dsh = {"w1": (fs, d), "w3": (fs, d), "w2": (d, fs)}
        Ws = {}
        for name in ("w1", "w3", "w2"):
            fm, bits, grp = shared_fmts[name]
            Ws[name] = dequant(fm, bits, grp, dsh[name][1], *shared_fetch(name, 0))
        y_sh = swiglu_ffn(Ws["w1"], Ws["w3"], Ws["w2"], xs[tok])
        res["y_shared"] = y_sh
    res["tokens"] = tok
    res["y_slots"] = y
    res["out"] = combine(y, np.where(owned, w, 0.0)[tok], y_sh)
    res["out_bf16"] = round_bf16(res["out"])
    return res


def parity_stats(out: np.ndarray, ref: np.ndarray) -> Dict[str, float]:
    """max|err| / rms(ref) and sum|err| / sum|ref| (the output tolerances)."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(out - ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return {
        "max_err": float(err.max()) if err.size else 0.0,
        "rms_ref": rms,
        "max_err_over_rms": float(err.max() / rms) if err.size and rms > 0 else 0.0,
        "mean_rel_err": float(err.sum() / np.abs(ref).sum()) if err.size and np.abs(ref).sum() > 0 else 0.0,
    }


# --------------------------------------------------------------------------
# mHC residual mixing  [PR1192-SK; CARD-4BIT-MHC]
# --------------------------------------------------------------------------
# Readings where the pages are silent: the mixing logits are per token,
# [T, n, n] with n = hc_mult; the softmax runs along each row (the last
# axis); one iteration is a column normalisation followed by a row
# normalisation (so rows sum to one on exit); eps is added to every divisor
# (0 by default); the n -> n mix is out[t, i] = sum_j P[t, i, j] * h[t, j].
def hc_sinkhorn(logits, iters: int, eps: float = 0.0) -> np.ndarray:
    """Sinkhorn-normalised mixing matrices P [T, n, n] in fp64: a row-wise
    softmax of the logits, then `iters` rounds of dividing every column by
    its sum and then every row by its sum."""
    L = np.asarray(logits, np.float64)
    P = np.exp(L - L.max(axis=-1, keepdims=True))
    P = P / P.sum(axis=-1, keepdims=True)
    for _ in range(iters):
        P = P / (P.sum(axis=-2, keepdims=True) + eps)
        P = P / (P.sum(axis=-1, keepdims=True) + eps)
    return P


def hc_mix(P, h) -> np.ndarray:
    """out[t, i, :] = sum_j P[t, i, j] * h[t, j, :] for the n parallel copies
    h [T, n, d] of the residual stream."""
    return np.einsum("tij,tjd->tid", np.asarray(P, np.float64), np.asarray(h, np.float64))
