"""Seeded synthetic inputs for the RankMixer stack workloads.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the model's arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from it without sharing any computation.

Every row along a tensor's first axis is drawn from its own CPU
``torch.Generator`` (mt19937) seeded with a fixed function of (seed, tensor
index, row).  A tensor's values therefore do not depend on the batch size, on
which other tensors were drawn, or on how many threads drew them, and the
rows of any subset of samples can be regenerated exactly for sampled parity
checks.

bf16 workloads draw in fp32 and round to bf16 (round-to-nearest-even) before
anyone uses the values; the oracle consumes those rounded values widened to
fp64.  Biases, LayerNorm parameters and router parameters stay fp32.

Weight layout (per token t, "out-major", the orientation of the product
``W1 s_t`` in the per-token FFN equation of the fun-rec chapter "Rankmixer:
硬件效率优化", section Per-Token FFN):
  dense:  W1 [T, kD, D], b1 [T, kD], W2 [T, D, kD], b2 [T, D]
  MoE:    W1 [T, Ne, kDe, D], b1 [T, Ne, kDe], W2 [T, Ne, D, kDe], b2 [T, Ne, D]
          Wr [T, Ne, D], br [T, Ne]
  LN:     ln1_g, ln1_b, ln2_g, ln2_b  [D] each (shared across tokens)
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import math
import os
from typing import Dict, List, Optional, Sequence

import torch

_THREADS = os.cpu_count() or 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic RankMixer stack."""

    name: str
    B: int
    T: int
    D: int
    hidden: int          # kD (dense) or kDe (per expert)
    L: int
    dtype: str = "bf16"  # "bf16" or "f32"
    n_experts: int = 0   # 0 = dense per-token FFN
    ln_params: str = "unit"     # "unit": gamma=1, beta=0; "perturbed": 1+N(0,.02), N(0,.02)
    x0_std: float = 1.0
    bias_std: float = 0.01
    group_widths: tuple = ()    # Pad-Split feature groups (empty = X0 drawn directly)
    group_std: float = 0.1
    head: bool = False          # D -> 1 linear head + sigmoid after pooling
    router_std: float = 0.02
    router_bias: float = -0.5
    act: str = "tanh"           # FFN activation: "tanh" / "erf" (GELU) or "relu"
    mix_addnorm: bool = True    # False: S = TokenMixing(X), no Add & Norm after mixing

    @property
    def dh(self) -> int:
        return self.D // self.T

    @property
    def padded_width(self) -> int:
        return self.T * self.D

    def with_batch(self, B: int) -> "Workload":
        return dataclasses.replace(self, B=B)


# The five synthetic stacks.  Sizes follow the RankMixer pages: the 100M and
# 1B shapes of the paper's Table 1 (batch 512), the Taobao Pad-Split serving
# stack (12 feature groups concatenated, padded to 5120 = 16 x 320), and a
# per-token sparse MoE with ReLU routing.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", B=64, T=8, D=64, hidden=256, L=2, dtype="f32"),
    "rm100m": Workload("rm100m", B=512, T=16, D=768, hidden=3072, L=2,
                       ln_params="perturbed"),
    "rm1b": Workload("rm1b", B=512, T=32, D=1536, hidden=6144, L=2),
    "padsplit": Workload("padsplit", B=4096, T=16, D=320, hidden=1280, L=4,
                         group_widths=(512, 480, 448, 448, 416, 416, 384, 384,
                                       352, 352, 320, 288),
                         head=True),
    "moe": Workload("moe", B=2048, T=16, D=768, hidden=768, L=2, n_experts=8),
    # the three-layer Mixer backbone timed in Appendix B of the MFU re-reading
    # article: batch 256, 8 tokens of width 256, FFN hidden 1024, ReLU, no MoE
    "appendix_b": Workload("appendix_b", B=256, T=8, D=256, hidden=1024, L=3, act="relu"),
}


def _row_seed(seed: int, index: int, row: int) -> int:
    return ((seed * 1_000_003 + index) * 1_000_000_007 + row) % (1 << 63)


def _normal(shape, std: float, mean: float, seed: int, index: int,
            rows: Optional[Sequence[int]] = None) -> torch.Tensor:
    """N(mean, std^2) fp32 tensor; row i of the first axis from its own stream.
    With ``rows`` given, only those rows are drawn (in that order)."""
    if len(shape) == 1:     # a vector is one row
        return _normal((1,) + tuple(shape), std, mean, seed, index)[0]
    rows = list(range(shape[0])) if rows is None else [int(r) for r in rows]
    out = torch.empty((len(rows),) + tuple(shape[1:]), dtype=torch.float32)

    def fill(lo: int, hi: int) -> None:
        g = torch.Generator(device="cpu")
        for k in range(lo, hi):
            g.manual_seed(_row_seed(seed, index, rows[k]))
            out[k].normal_(mean=mean, std=std, generator=g)

    n = len(rows)
    workers = max(1, min(_THREADS, n, (out.numel() >> 20) + 1))
    if workers == 1:
        fill(0, n)
    else:
        step = (n + workers - 1) // workers
        with cf.ThreadPoolExecutor(workers) as ex:
            list(ex.map(lambda lo: fill(lo, min(n, lo + step)), range(0, n, step)))
    return out


def _store(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def xavier_std(fan_in: int, fan_out: int) -> float:
    """Xavier/Glorot normal standard deviation sqrt(2 / (fan_in + fan_out))."""
    return math.sqrt(2.0 / (fan_in + fan_out))


# Tensor index plan: 0..31 inputs, 100 + 32*l + k for block l, 90 for the head.
_IDX_X0 = 0
_IDX_GROUP0 = 1


def make_x0(wl: Workload, seed: int = 0, samples: Optional[torch.Tensor] = None) -> torch.Tensor:
    """X0 [B, T, D] in the workload's storage dtype (no Pad-Split)."""
    x = _normal((wl.B, wl.T, wl.D), wl.x0_std, 0.0, seed, _IDX_X0, rows=samples)
    return _store(x, wl.dtype)


def make_groups(wl: Workload, seed: int = 0, samples: Optional[torch.Tensor] = None) -> List[torch.Tensor]:
    """Pad-Split feature-group embeddings, one [B, w_i] tensor per group."""
    out = []
    for i, w in enumerate(wl.group_widths):
        g = _normal((wl.B, w), wl.group_std, 0.0, seed, _IDX_GROUP0 + i, rows=samples)
        out.append(_store(g, wl.dtype))
    return out


def make_block(wl: Workload, l: int, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Weights of block l.  Matrices in storage dtype; vectors fp32."""
    T, D, Hd, Ne = wl.T, wl.D, wl.hidden, wl.n_experts
    base = 100 + 32 * l
    blk: Dict[str, torch.Tensor] = {}
    if Ne == 0:
        blk["W1"] = _store(_normal((T, Hd, D), xavier_std(D, Hd), 0.0, seed, base + 0), wl.dtype)
        blk["b1"] = _normal((T, Hd), wl.bias_std, 0.0, seed, base + 1)
        blk["W2"] = _store(_normal((T, D, Hd), xavier_std(Hd, D), 0.0, seed, base + 2), wl.dtype)
        blk["b2"] = _normal((T, D), wl.bias_std, 0.0, seed, base + 3)
    else:
        blk["W1"] = _store(_normal((T, Ne, Hd, D), xavier_std(D, Hd), 0.0, seed, base + 0), wl.dtype)
        blk["b1"] = _normal((T, Ne, Hd), wl.bias_std, 0.0, seed, base + 1)
        blk["W2"] = _store(_normal((T, Ne, D, Hd), xavier_std(Hd, D), 0.0, seed, base + 2), wl.dtype)
        blk["b2"] = _normal((T, Ne, D), wl.bias_std, 0.0, seed, base + 3)
        blk["Wr"] = _normal((T, Ne, D), wl.router_std, 0.0, seed, base + 8)
        blk["br"] = torch.full((T, Ne), wl.router_bias, dtype=torch.float32)
    if wl.ln_params == "perturbed":
        blk["ln1_g"] = _normal((D,), 0.02, 1.0, seed, base + 4)
        blk["ln1_b"] = _normal((D,), 0.02, 0.0, seed, base + 5)
        blk["ln2_g"] = _normal((D,), 0.02, 1.0, seed, base + 6)
        blk["ln2_b"] = _normal((D,), 0.02, 0.0, seed, base + 7)
    else:
        blk["ln1_g"] = torch.ones(D)
        blk["ln1_b"] = torch.zeros(D)
        blk["ln2_g"] = torch.ones(D)
        blk["ln2_b"] = torch.zeros(D)
    return blk


def make_head(wl: Workload, seed: int = 0) -> Dict[str, torch.Tensor]:
    """D -> 1 head: Xavier-normal weight [D] (storage dtype), bias 0 (fp32)."""
    w = _store(_normal((wl.D,), xavier_std(wl.D, 1), 0.0, seed, 90), wl.dtype)
    return {"w": w, "b": torch.zeros(1)}


def make_inputs(wl: Workload, seed: int = 0, samples: Optional[torch.Tensor] = None) -> Dict:
    """All inputs of a workload: X0 or groups, L blocks, optional head."""
    d: Dict = {"wl": wl, "seed": seed}
    if wl.group_widths:
        d["groups"] = make_groups(wl, seed, samples)
    else:
        d["X0"] = make_x0(wl, seed, samples)
    d["blocks"] = [make_block(wl, l, seed) for l in range(wl.L)]
    if wl.head:
        d["head"] = make_head(wl, seed)
    return d


def random_like_block(T: int, D: int, hidden: int, dtype: str = "f32", seed: int = 0,
                      n_experts: int = 0, ln_params: str = "perturbed",
                      router_std: float = 0.02, router_bias: float = -0.5) -> Dict[str, torch.Tensor]:
    """Block weights for arbitrary small shapes (test cases)."""
    wl = Workload("adhoc", B=1, T=T, D=D, hidden=hidden, L=1, dtype=dtype,
                  n_experts=n_experts, ln_params=ln_params,
                  router_std=router_std, router_bias=router_bias)
    return make_block(wl, 0, seed)


def random_activations(shape, dtype: str = "f32", seed: int = 0, std: float = 1.0,
                       index: int = 7) -> torch.Tensor:
    """Seeded N(0, std^2) activations of any shape (test cases)."""
    return _store(_normal(tuple(shape), std, 0.0, seed, index), dtype)
