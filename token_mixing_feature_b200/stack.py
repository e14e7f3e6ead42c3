"""Device-resident RankMixer stack: one rm_handle plus the weights in HBM.

Plumbing only (PyTorch allocates device memory and supplies the stream); every
step of the forward pass runs in librankmixer through the C ABI.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import torch

from . import rankmixer as rm
from .synth import Workload

TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32}


def to_device(blk: Dict[str, torch.Tensor], device) -> Dict[str, torch.Tensor]:
    return {k: v.to(device).contiguous() for k, v in blk.items()}


class RankMixerStack:
    def __init__(self, wl: Workload, blocks: Sequence[Dict[str, torch.Tensor]], head: Optional[Dict] = None,
                 device="cuda", B_max: Optional[int] = None, ln_eps: float = 1e-5):
        self.wl = wl
        self.device = torch.device(device)
        self.dtype = TORCH_DTYPE[wl.dtype]
        self.B_max = B_max or wl.B
        with torch.cuda.device(self.device):
            self.h = rm.rm_create(self.B_max, wl.T, wl.D, wl.hidden, wl.L, wl.n_experts, wl.dtype,
                                  ln_eps, wl.act, wl.mix_addnorm)
        self.blocks: List[Dict[str, torch.Tensor]] = [to_device(b, self.device) for b in blocks]
        self.head = to_device(head, self.device) if head else None

    def close(self) -> None:
        self.h.close()

    def empty_act(self, B: int) -> torch.Tensor:
        return torch.empty(B, self.wl.T, self.wl.D, dtype=self.dtype, device=self.device)

    def forward(self, X0: torch.Tensor, pooled: Optional[torch.Tensor] = None,
                Xlast: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        B = X0.shape[0]
        if pooled is None:
            pooled = torch.empty(B, self.wl.D, dtype=torch.float32, device=self.device)
        rm.rm_stack_forward(self.h, self.blocks, X0, pooled, Xlast, B, stream)
        return pooled

    def forward_host(self, X0_host: torch.Tensor, pooled_host: torch.Tensor, stream=None) -> torch.Tensor:
        rm.rm_stack_forward_host(self.h, self.blocks, X0_host, pooled_host, X0_host.shape[0], stream)
        return pooled_host

    def forward_host_async(self, X0_host: torch.Tensor, pooled_host: torch.Tensor, stream=None) -> None:
        """Enqueue one host-buffer call (input copy overlaps the previous call's stack)."""
        rm.rm_stack_forward_host_async(self.h, self.blocks, X0_host, pooled_host, X0_host.shape[0], stream)

    def host_wait(self) -> None:
        rm.rm_host_wait(self.h)

    def block(self, l: int, X: torch.Tensor, Xout: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        Xout = self.empty_act(X.shape[0]) if Xout is None else Xout
        rm.rm_block_forward(self.h, self.blocks[l], X, Xout, X.shape[0], stream)
        return Xout

    def tokenize(self, groups: Sequence[torch.Tensor], X0: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        B = groups[0].shape[0]
        X0 = self.empty_act(B) if X0 is None else X0
        rm.rm_padsplit_tokenize(self.h, groups, X0, B, stream)
        return X0

    def head_forward(self, pooled: torch.Tensor, prob: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        B = pooled.shape[0]
        prob = torch.empty(B, dtype=torch.float32, device=self.device) if prob is None else prob
        rm.rm_head_forward(self.h, self.head["w"], self.head["b"], pooled, prob, B, stream)
        return prob
