"""A buffer-owning wrapper around moe_layer_forward.

``MoELayer`` keeps the descriptor, the weight pointers and a workspace sized
by the library, so a forward pass is one C-ABI call on the current stream.
Torch only provides the device memory and the stream.
"""
from __future__ import annotations

import torch

from . import ops
from .synthetic import LayerConfig, desc_dict


class MoELayer:
    def __init__(self, cfg: LayerConfig, weights: dict, device="cuda", S=None, with_outputs=True):
        self.cfg = cfg
        self.S = cfg.S if S is None else S
        self.device = torch.device(device)
        self.desc = ops.make_desc(**desc_dict(cfg, self.S))
        self.tensors = weights
        self.weights = ops.make_weights(weights)
        nbytes = ops.moe_workspace_size(self.desc)
        self.ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        ops.moe_workspace_init(self.ws)
        adt = torch.float32 if cfg.act_dtype == 0 else torch.bfloat16
        self.y = torch.empty((self.S, cfg.d), dtype=adt, device=self.device)
        self.topk_idx = self.topk_w = self.counts = None
        if with_outputs:
            self.topk_idx = torch.empty((self.S, cfg.K), dtype=torch.int32, device=self.device)
            self.topk_w = torch.empty((self.S, cfg.K), dtype=torch.float32, device=self.device)
            self.counts = torch.empty((cfg.E,), dtype=torch.int32, device=self.device)

    def forward(self, x: torch.Tensor, y: torch.Tensor = None, stream=None) -> torch.Tensor:
        out = self.y if y is None else y
        ops.moe_layer_forward(self.desc, self.weights, x, out, self.topk_idx, self.topk_w, self.counts, self.ws,
                              stream)
        return out

    def status(self):
        return ops.moe_get_status(self.ws)
