"""A resident MoE layer: device weights + workspace, one call per forward."""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import _lib


def expert_range(rank: int, world: int, n_experts: int) -> tuple:
    """Contiguous expert slice [begin, end) owned by `rank` of `world` in the
    expert-parallel split (routing replicated, each rank runs its experts and
    the partial outputs are all-reduced; the shared expert goes to rank 0).
    Slices differ in size by at most one expert."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    return rank * n_experts // world, (rank + 1) * n_experts // world


class MoELayer:
    """Holds the packed experts, router and workspace of one routed-MoE layer.

    w1/w3/w2 (and the optional shared triple) are objects with attributes
    fmt, bits, group, q, scales, biases whose tensors live on the device;
    router_w is fp32 or bf16 [E, d]; router_b fp32 [E] or None; tid2eid int32
    [vocab, k] selects hash routing.
    """

    def __init__(self, *, d_model: int, d_ff: int, n_experts: int, top_k: int, max_tokens: int,
                 w1, w3, w2, router_w: Optional[torch.Tensor], router_b: Optional[torch.Tensor] = None,
                 tid2eid: Optional[torch.Tensor] = None, shared: Optional[Sequence] = None,
                 device="cuda"):
        self.d_model, self.d_ff, self.n_experts, self.top_k = d_model, d_ff, n_experts, top_k
        self.w1, self.w3, self.w2 = w1, w3, w2
        self.router_w, self.router_b, self.tid2eid = router_w, router_b, tid2eid
        self.shared = shared
        self.d_ff_shared = shared[0].n_out if shared is not None else 0
        self.hash_mode = tid2eid is not None
        self.vocab = tid2eid.shape[0] if tid2eid is not None else 0
        self.device = torch.device(device)
        self.max_tokens = max_tokens
        self.ws = _lib.alloc_workspace(self.dims(max_tokens), self.device)

    def dims(self, T: int) -> _lib.Dims:
        return _lib.make_dims(T, self.d_model, self.d_ff, self.n_experts, self.top_k, self.hash_mode,
                              self.vocab, self.d_ff_shared,
                              router_dtype=None if self.router_w is None else self.router_w.dtype)

    def __call__(self, x: torch.Tensor, token_ids: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, topk_ids: Optional[torch.Tensor] = None,
                 topk_w: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds max_tokens={self.max_tokens}")
        if out is None:
            out = torch.empty(T, self.d_model, dtype=torch.bfloat16, device=self.device)
        _lib.forward(self.dims(T), x, token_ids, self.router_w, self.router_b, self.tid2eid, self.w1, self.w3,
                     self.w2, self.shared, out, self.ws, topk_ids_out=topk_ids, topk_w_out=topk_w, stream=stream)
        return out

    def forward_host(self, x_host: torch.Tensor, token_ids_host: Optional[torch.Tensor], out_host: torch.Tensor,
                     stream=None) -> torch.Tensor:
        _lib.forward_host(self.dims(x_host.shape[0]), x_host, token_ids_host, self.router_w, self.router_b,
                          self.tid2eid, self.w1, self.w3, self.w2, self.shared, out_host, self.ws, stream=stream)
        return out_host

    def device_error(self, stream=None) -> int:
        return _lib.read_device_error(self.ws, stream)
