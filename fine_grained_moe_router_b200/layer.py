"""MoELayer: one fine-grained MoE FFN layer with device-resident weights.

A thin convenience wrapper over the C ABI: it keeps the weights and a
workspace on the device and calls ``moe_layer_forward`` / ``moe_expert_stats``.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


class MoELayer:
    """Forward pass of one fine-grained MoE layer (router, dispatch, grouped
    expert FFN with an optional shared expert, combine) on one GPU.

    Weights (device tensors, nn.Linear [out, in] layout): w_router [E, H],
    w1 [E, D, H], w2 [E, H, D], optional shared expert ws1 [Ds, H] and
    ws2 [H, Ds], optional fp32 expert bias [E]. All weight tensors share one
    dtype (torch.float32 or torch.bfloat16)."""

    def __init__(self, w_router, w1, w2, top_k: int, ws1=None, ws2=None, bias=None,
                 capacity_factor=(5, 4)):
        self.E, self.H = w_router.shape
        self.D = w1.shape[1]
        self.Ds = 0 if ws1 is None else ws1.shape[0]
        self.K = int(top_k)
        self.dtype = w_router.dtype
        self.device = w_router.device
        self.cf = capacity_factor
        self.tensors = [t.contiguous() if t is not None else None
                        for t in (w_router, w1, w2, ws1, ws2, bias)]
        self.weights = B.make_weights(*self.tensors)
        self._ws: Optional[torch.Tensor] = None

    def desc(self, T: int) -> B.MoELayerDesc:
        return B.make_desc(T, self.H, self.E, self.K, self.D, self.Ds, B.dtype_code(self.dtype),
                           self.cf)

    def workspace(self, T: int) -> torch.Tensor:
        need = B.moe_workspace_size(self.desc(T))
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def routing_buffers(self, T: int) -> dict:
        dev, K, E = self.device, self.K, self.E
        i32 = torch.int32
        return {
            "topk_idx": torch.empty((T, K), dtype=i32, device=dev),
            "topk_w": torch.empty((T, K), dtype=torch.float32, device=dev),
            "counts": torch.empty(E, dtype=i32, device=dev),
            "offsets": torch.empty(E + 1, dtype=i32, device=dev),
            "perm": torch.empty(T * K, dtype=i32, device=dev),
            "inv": torch.empty(T * K, dtype=i32, device=dev),
            "logits": torch.empty((T, E), dtype=torch.float32, device=dev),
        }

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, routing: Optional[dict] = None,
                stream=None, gumbel_noise: Optional[torch.Tensor] = None) -> torch.Tensor:
        """y = MoE(x) for x [T, H]; fills `routing` (see routing_buffers) if given.
        gumbel_noise [T, E] fp32: noisy routing (Gumbel draws added to l + B)."""
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        r = B.make_routing(**routing) if routing is not None else None
        if gumbel_noise is None:
            B.moe_layer_forward(self.desc(T), self.weights, x, y, r, self.workspace(T), stream)
        else:
            B.moe_layer_forward_noisy(self.desc(T), self.weights, x, gumbel_noise, y, r,
                                      self.workspace(T), stream)
        return y

    __call__ = forward

    def stats(self, counts: torch.Tensor, T: int, straggler_mask: Optional[torch.Tensor] = None,
              stream=None) -> dict:
        return B.moe_expert_stats(self.desc(T), counts, straggler_mask, self.workspace(T), stream)

    def update_bias(self, counts: torch.Tensor, tokens: int, gamma: float, stream=None) -> None:
        """Dynamic bias update from expert counts accumulated over `tokens`
        tokens: B_e -= gamma for overloaded experts, += gamma for idle ones."""
        if self.tensors[5] is None:
            raise ValueError("the layer has no expert bias tensor to update")
        B.moe_bias_update(self.desc(tokens), counts, self.tensors[5], gamma, stream)
