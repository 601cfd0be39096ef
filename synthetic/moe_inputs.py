"""Seeded generators for the routed-MoE layer's inputs.

Workloads follow the five layer configurations this library is measured on
(tiny, decode, hash, mixed, prefill) plus ad-hoc shapes for parity tests.

Stored formats produced here (the layouts the C ABI consumes):

* affine (MLX-style "w = scale*q + bias"): per matrix ``[E, out, in]`` the
  integer codes are packed LSB-first into a little-endian bitstream along the
  input dimension, ``in*bits/32`` uint32 words per row; element ``i`` of a row
  lives at bits ``[i*bits, i*bits+bits)`` of that row's stream (for 3-bit codes
  32 values fill 3 words and codes straddle word boundaries).  ``scales`` and
  ``biases`` are bf16 ``[E, out, in/group]``.
* mxfp4: e2m1 codes, two per byte with the low nibble holding the even
  element (the same LSB-first stream with bits=4), ``in/8`` words per row, and
  one e8m0 exponent byte per 32 inputs, uint8 ``[E, out, in/32]``.

The quantiser used to *produce* affine packs is the min/max rule: per group
``scale = (max-min)/(2^b-1)`` and ``bias = min``, both rounded to bf16, then
``q = clamp(round_half_even((w-bias)/scale), 0, 2^b-1)`` (``q = 0`` when
``scale == 0``).  It only makes data: the layer never quantises.

Draw order for a configuration (one ``torch.Generator`` seeded with the
config's seed, on the device the tensors are built on):
x, router weight, router bias, [token ids, tid2eid], then per routed expert
``e = 0..E-1``: w1[e], w3[e], w2[e] (drawn in chunks of experts), then the
shared expert's w1, w3, w2.

Generation on a CUDA device uses torch's CUDA generator, so the same seed
gives different (but equally distributed, and deterministic) tensors on CPU
and on GPU; every comparison runs both sides on the same tensors.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import torch

# --------------------------------------------------------------------------
# Layer configurations.  fmt tuples are (format, bits, group).
# --------------------------------------------------------------------------
AFF4_G64 = ("affine", 4, 64)
AFF8_G64 = ("affine", 8, 64)
AFF2_G128 = ("affine", 2, 128)
AFF3_G128 = ("affine", 3, 128)
MXFP4 = ("mxfp4", 4, 32)

CONFIGS: Dict[str, dict] = {
    # T=4 tokens, d_model=256, 8 routed experts, top-2, d_ff=128, affine 4-bit
    # g64, weights ~N(0,0.02), router ~N(0,0.02), bias ~N(0,0.01), seed 0.
    "tiny": dict(T=4, d=256, E=8, k=2, f=128, routing="learned", vocab=0,
                 w13=AFF4_G64, w2=AFF4_G64, shared=None, f_shared=0,
                 weight_std=0.02, router_std=0.02, bias_std=0.01, seed=0),
    # Decode, learned routing, one always-on 8-bit shared expert.
    "decode": dict(T=1, d=4096, E=256, k=8, f=2048, routing="learned", vocab=0,
                   w13=AFF4_G64, w2=AFF4_G64, shared=AFF8_G64, f_shared=2048,
                   weight_std=0.02, router_std=0.02, bias_std=0.01, seed=1),
    # Hash-routed early layer: tid2eid [129280, 8] of distinct experts, mxfp4
    # experts with e8m0 exponents uniform in [117, 123].
    "hash": dict(T=32, d=4096, E=256, k=8, f=2048, routing="hash", vocab=129280,
                 w13=MXFP4, w2=MXFP4, shared=None, f_shared=0,
                 weight_std=0.02, router_std=0.02, bias_std=0.0, seed=2,
                 e8m0_lo=117, e8m0_hi=123),
    # Mixed low-bit decode: w1/w3 affine 2-bit g128, w2 affine 3-bit g128.
    "mixed": dict(T=8, d=4096, E=256, k=8, f=2048, routing="learned", vocab=0,
                  w13=AFF2_G128, w2=AFF3_G128, shared=None, f_shared=0,
                  weight_std=0.02, router_std=0.02, bias_std=0.01, seed=3),
    # Prefill: per-expert selection offset ~N(0,0.5) (realised as the router's
    # selection bias) makes per-expert token counts imbalanced.
    "prefill": dict(T=4096, d=4096, E=256, k=8, f=2048, routing="learned", vocab=0,
                    w13=AFF4_G64, w2=AFF4_G64, shared=None, f_shared=0,
                    weight_std=0.02, router_std=0.02, bias_std=0.5, seed=4),
}


@dataclasses.dataclass
class QMat:
    """One stacked expert matrix ``[E, out, in]`` in a packed format."""

    fmt: str            # "affine" | "mxfp4"
    bits: int
    group: int
    n_out: int
    n_in: int
    q: torch.Tensor                 # int32 bit patterns [E, out, in*bits/32]
    scales: torch.Tensor            # bf16 [E, out, in/group] | uint8 [E, out, in/32]
    biases: Optional[torch.Tensor]  # bf16 [E, out, in/group] | None

    @property
    def n_experts(self) -> int:
        return self.q.shape[0]

    def to(self, device) -> "QMat":
        return dataclasses.replace(
            self, q=self.q.to(device), scales=self.scales.to(device),
            biases=None if self.biases is None else self.biases.to(device))

    def clone(self) -> "QMat":
        """The same packs in fresh buffers (equal values, other addresses)."""
        return dataclasses.replace(
            self, q=self.q.clone(), scales=self.scales.clone(),
            biases=None if self.biases is None else self.biases.clone())

    def expert_numpy(self, e: int):
        """Host copies of expert ``e``'s packs: (uint32 words, scales, biases).

        Scales/biases come back as float32 (bf16 widens exactly) for affine and
        as uint8 exponents for mxfp4.
        """
        q = self.q[e].cpu().contiguous().view(torch.int32).numpy().view("<u4")
        if self.fmt == "affine":
            s = self.scales[e].float().cpu().numpy()
            b = self.biases[e].float().cpu().numpy()
            return q, s, b
        return q, self.scales[e].cpu().numpy(), None

    def packed_bytes_per_expert(self) -> int:
        n = self.q[0].numel() * 4 + self.scales[0].numel() * self.scales.element_size()
        if self.biases is not None:
            n += self.biases[0].numel() * self.biases.element_size()
        return n


@dataclasses.dataclass
class MoEInputs:
    cfg: dict
    x: torch.Tensor                       # bf16 [T, d]
    router_w: torch.Tensor                # fp32 [E, d]
    router_b: Optional[torch.Tensor]      # fp32 [E]
    token_ids: Optional[torch.Tensor]     # int32 [T]
    tid2eid: Optional[torch.Tensor]       # int32 [vocab, k]
    w1: QMat
    w3: QMat
    w2: QMat
    shared: Optional[Tuple[QMat, QMat, QMat]]

    def to(self, device) -> "MoEInputs":
        mv = lambda t: None if t is None else t.to(device)  # noqa: E731
        return dataclasses.replace(
            self, x=mv(self.x), router_w=mv(self.router_w), router_b=mv(self.router_b),
            token_ids=mv(self.token_ids), tid2eid=mv(self.tid2eid),
            w1=self.w1.to(device), w3=self.w3.to(device), w2=self.w2.to(device),
            shared=None if self.shared is None else tuple(m.to(device) for m in self.shared))

    def clone(self) -> "MoEInputs":
        """The same layer in fresh buffers on the same device: equal values
        (so equal routing and work), other addresses (so no cache line of one
        copy serves a read of another)."""
        cp = lambda t: None if t is None else t.clone()  # noqa: E731
        return dataclasses.replace(
            self, x=cp(self.x), router_w=cp(self.router_w), router_b=cp(self.router_b),
            token_ids=cp(self.token_ids), tid2eid=cp(self.tid2eid),
            w1=self.w1.clone(), w3=self.w3.clone(), w2=self.w2.clone(),
            shared=None if self.shared is None else tuple(m.clone() for m in self.shared))


# --------------------------------------------------------------------------
# Encoders (data production only)
# --------------------------------------------------------------------------
def pack_bits(q: torch.Tensor, bits: int) -> torch.Tensor:
    """Pack integer codes ``q[..., n]`` (0 <= q < 2^bits) into int32 words.

    LSB-first little-endian bitstream per row: code ``i`` occupies bits
    ``[i*bits, (i+1)*bits)`` of the row's stream; ``n*bits`` must be a multiple
    of 32 (32 codes always fill exactly ``bits`` words).
    """
    *lead, n = q.shape
    if n % 32:
        raise ValueError("row length must be a multiple of 32 codes")
    q = q.to(torch.int64).reshape(*lead, n // 32, 32)
    words = torch.zeros(*lead, n // 32, bits, dtype=torch.int64, device=q.device)
    for j in range(32):
        wi, sh = divmod(j * bits, 32)
        v = q[..., j]
        words[..., wi] |= (v << sh) & 0xFFFFFFFF
        if sh + bits > 32:
            words[..., wi + 1] |= v >> (32 - sh)
    words = words.reshape(*lead, n * bits // 32)
    words = torch.where(words >= 2 ** 31, words - 2 ** 32, words)
    return words.to(torch.int32)


def quantize_affine(w: torch.Tensor, bits: int, group: int):
    """Min/max per-group affine quantiser -> (int32 words, bf16 scales, bf16 biases)."""
    *lead, n = w.shape
    wg = w.float().reshape(*lead, n // group, group)
    lo = wg.amin(-1)
    hi = wg.amax(-1)
    levels = (1 << bits) - 1
    scale = ((hi - lo) / levels).to(torch.bfloat16)
    bias = lo.to(torch.bfloat16)
    s32 = scale.float().unsqueeze(-1)
    b32 = bias.float().unsqueeze(-1)
    pos = s32 > 0
    q = torch.round((wg - b32) / torch.where(pos, s32, torch.ones_like(s32)))
    q = torch.where(pos, q.clamp(0, levels), torch.zeros_like(q))
    q = q.to(torch.int64).reshape(*lead, n)
    return pack_bits(q, bits), scale, bias


def _gen_qmat(gen, device, fmt, n_exp, n_out, n_in, std, cfg, chunk=8) -> QMat:
    kind, bits, group = fmt
    if n_in % 32 or n_in % group:
        raise ValueError(f"in={n_in} must be a multiple of 32 and of group={group}")
    if kind == "affine":
        qs, ss, bs = [], [], []
        for e0 in range(0, n_exp, chunk):
            ne = min(chunk, n_exp - e0)
            w = torch.randn(ne, n_out, n_in, generator=gen, device=device) * std
            q, s, b = quantize_affine(w, bits, group)
            qs.append(q)
            ss.append(s)
            bs.append(b)
            del w
        return QMat("affine", bits, group, n_out, n_in, torch.cat(qs), torch.cat(ss), torch.cat(bs))
    if kind == "mxfp4":
        if group != 32 or bits != 4:
            raise ValueError("mxfp4 is 4-bit codes with 32-element scale groups")
        # codes uniform over the 16 e2m1 levels == uniform random 32-bit words
        q = torch.randint(-2 ** 31, 2 ** 31, (n_exp, n_out, n_in // 8), generator=gen,
                          device=device, dtype=torch.int64).to(torch.int32)
        lo, hi = cfg.get("e8m0_lo", 117), cfg.get("e8m0_hi", 123)
        s = torch.randint(lo, hi + 1, (n_exp, n_out, n_in // 32), generator=gen,
                          device=device, dtype=torch.int32).to(torch.uint8)
        return QMat("mxfp4", 4, 32, n_out, n_in, q, s, None)
    raise ValueError(f"unknown format {kind}")


def make_custom(cfg: dict, device="cpu") -> MoEInputs:
    """Build inputs for an arbitrary configuration dict (keys as in CONFIGS)."""
    T, d, E, k, f = cfg["T"], cfg["d"], cfg["E"], cfg["k"], cfg["f"]
    gen = torch.Generator(device=device)
    gen.manual_seed(int(cfg["seed"]))
    x = torch.randn(T, d, generator=gen, device=device).to(torch.bfloat16)
    router_w = torch.randn(E, d, generator=gen, device=device) * cfg.get("router_std", 0.02)
    if cfg.get("router_dtype", "fp32") == "bf16":
        router_w = router_w.to(torch.bfloat16)   # the gate stored in bf16 (RNE of the fp32 draw)
    bias_std = cfg.get("bias_std", 0.0)
    router_b = None
    if cfg["routing"] == "learned":
        router_b = torch.randn(E, generator=gen, device=device) * bias_std
    token_ids = tid2eid = None
    if cfg["routing"] == "hash":
        vocab = cfg["vocab"]
        token_ids = torch.randint(0, vocab, (T,), generator=gen, device=device,
                                  dtype=torch.int64).to(torch.int32)
        # each row: k distinct experts, uniformly without replacement
        keys = torch.rand(vocab, E, generator=gen, device=device)
        tid2eid = keys.topk(k, dim=1).indices.to(torch.int32).contiguous()
        del keys
    std = cfg.get("weight_std", 0.02)
    w1 = _gen_qmat(gen, device, cfg["w13"], E, f, d, std, cfg)
    w3 = _gen_qmat(gen, device, cfg["w13"], E, f, d, std, cfg)
    w2 = _gen_qmat(gen, device, cfg["w2"], E, d, f, std, cfg)
    shared = None
    if cfg.get("shared"):
        fs = cfg["f_shared"]
        shared = (_gen_qmat(gen, device, cfg["shared"], 1, fs, d, std, cfg),
                  _gen_qmat(gen, device, cfg["shared"], 1, fs, d, std, cfg),
                  _gen_qmat(gen, device, cfg["shared"], 1, d, fs, std, cfg))
    return MoEInputs(dict(cfg), x, router_w.contiguous(), router_b, token_ids, tid2eid,
                     w1, w3, w2, shared)


def make_inputs(name: str, device="cpu", **overrides) -> MoEInputs:
    """Inputs for one of the named layer configurations (optionally overridden)."""
    cfg = dict(CONFIGS[name])
    cfg["name"] = name
    cfg.update(overrides)
    return make_custom(cfg, device)


# --------------------------------------------------------------------------
# mHC residual mixing inputs (the block beside the MoE layer)
# --------------------------------------------------------------------------
HC_CONFIGS: Dict[str, dict] = {
    # the residual stream of a prefill batch: 4096 tokens, hc_mult = 4 copies
    # of a 4096-wide hidden state, 20 Sinkhorn iterations
    "mhc": dict(T=4096, n=4, d=4096, iters=20, eps=0.0, logit_std=1.0, seed=5),
    # one decode token
    "mhc_decode": dict(T=1, n=4, d=4096, iters=20, eps=0.0, logit_std=1.0, seed=6),
}


@dataclasses.dataclass
class HcInputs:
    cfg: dict
    logits: torch.Tensor   # fp32 [T, n, n]
    h: torch.Tensor        # bf16 [T, n, d]


def make_hc_inputs(cfg: dict, device="cpu") -> HcInputs:
    """Mixing logits ~ N(0, logit_std) and residual copies ~ N(0, 1) (bf16),
    drawn in that order from one generator seeded with cfg["seed"]."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(cfg["seed"]))
    T, n, d = cfg["T"], cfg["n"], cfg["d"]
    logits = torch.randn(T, n, n, generator=gen, device=device) * cfg.get("logit_std", 1.0)
    h = torch.randn(T, n, d, generator=gen, device=device).to(torch.bfloat16)
    return HcInputs(dict(cfg), logits.contiguous(), h.contiguous())


# --------------------------------------------------------------------------
# mxfp8 weight rows (e4m3 bytes with e8m0 group-32 scales)
# --------------------------------------------------------------------------
FP8_CONFIGS: Dict[str, dict] = {
    # a 16384 x 4096 weight matrix (64 Mi elements: 64 MiB of codes, 128 MiB
    # of bf16 out, more than L2) with e8m0 exponents uniform in [117, 123]
    # like the mxfp4 experts
    "mxfp8": dict(rows=16384, n_in=4096, e_lo=117, e_hi=123, seed=7),
}


@dataclasses.dataclass
class Fp8Inputs:
    cfg: dict
    codes: torch.Tensor    # uint8 [rows, n_in]
    scales: torch.Tensor   # uint8 [rows, n_in / 32]


def make_fp8_inputs(cfg: dict, device="cpu") -> Fp8Inputs:
    """e4m3 bytes uniform over the finite codes (the two NaN bytes 0x7F and
    0xFF become 0x38 = 1.0) and e8m0 bytes uniform in [e_lo, e_hi], drawn in
    that order from one generator seeded with cfg["seed"]."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(cfg["seed"]))
    rows, n_in = cfg["rows"], cfg["n_in"]
    codes = torch.randint(0, 256, (rows, n_in), generator=gen, device=device, dtype=torch.int32)
    codes = torch.where((codes & 0x7F) == 0x7F, torch.full_like(codes, 0x38), codes).to(torch.uint8)
    scales = torch.randint(cfg["e_lo"], cfg["e_hi"] + 1, (rows, n_in // 32), generator=gen, device=device,
                           dtype=torch.int32).to(torch.uint8)
    return Fp8Inputs(dict(cfg), codes.contiguous(), scales.contiguous())
