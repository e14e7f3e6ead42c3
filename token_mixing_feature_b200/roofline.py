"""Algorithmic work and traffic of a RankMixer stack forward.

FLOPs count 2 per multiply-add and only matrix products, the convention that
reproduces the matrix-FLOP column of the Appendix B table of
"重新理解 RankMixer：扩参为什么有效，又为什么划算？" (three Mixer layers,
B=256, T=8, d=256, h=1024 -> 6.442451 GFLOPs).  Per-token FFN parameters are
2 T k D^2 per block, as the fun-rec chapter "Rankmixer: 硬件效率优化" states in
its Per-Token FFN section.

Algorithmic bytes are what the stack must move at least once: all weights,
one read and one write of the [B, T, D] activations per block, the Pad-Split
embeddings read, and the pooled output.  Implementation intermediates (the
FFN hidden tensor, pre-LayerNorm rows) are not counted.
"""
from __future__ import annotations

from typing import Optional, Sequence

from .synth import Workload

ELEM_BYTES = {"bf16": 2, "f32": 4}


def pffn_params(T: int, D: int, hidden: int) -> int:
    """Matrix parameters of one dense per-token FFN layer: 2 T kD D."""
    return 2 * T * hidden * D


def gemm_flops(M: int, N: int, K: int, groups: int = 1) -> int:
    return 2 * M * N * K * groups


def dense_block_flops(B: int, T: int, D: int, hidden: int) -> int:
    """Both FFN projections of one block: 2 * (2 B T D kD)."""
    return gemm_flops(B, hidden, D, T) + gemm_flops(B, D, hidden, T)


def moe_block_flops(active: int, B: int, T: int, D: int, hidden: int, n_experts: int) -> int:
    """Active (b, t, j) expert evaluations, each two projections, plus the router."""
    return active * 4 * D * hidden + 2 * B * T * D * n_experts


def stack_flops(wl: Workload, active_per_block: Optional[Sequence[int]] = None) -> int:
    if wl.n_experts == 0:
        f = wl.L * dense_block_flops(wl.B, wl.T, wl.D, wl.hidden)
    else:
        if active_per_block is None:
            raise ValueError("MoE FLOPs need the measured active-expert counts")
        f = sum(moe_block_flops(a, wl.B, wl.T, wl.D, wl.hidden, wl.n_experts)
                for a in active_per_block)
    if wl.head:
        f += 2 * wl.B * wl.D
    return f


def block_weight_bytes(wl: Workload, experts_touched: Optional[int] = None) -> int:
    es = ELEM_BYTES[wl.dtype]
    T, D, Hd, Ne = wl.T, wl.D, wl.hidden, wl.n_experts
    ln = 4 * D * 4
    if Ne == 0:
        return pffn_params(T, D, Hd) * es + (T * Hd + T * D) * 4 + ln
    touched = T * Ne if experts_touched is None else experts_touched
    per_expert = 2 * Hd * D * es + (Hd + D) * 4
    return touched * per_expert + T * Ne * (D + 1) * 4 + ln


def stack_bytes(wl: Workload, experts_touched_per_block: Optional[Sequence[int]] = None) -> int:
    es = ELEM_BYTES[wl.dtype]
    act = wl.B * wl.T * wl.D * es
    total = 0
    for l in range(wl.L):
        et = None if experts_touched_per_block is None else experts_touched_per_block[l]
        total += block_weight_bytes(wl, et) + 2 * act
    total += wl.B * wl.D * 4                       # pooled (fp32)
    if wl.group_widths:
        total += wl.B * sum(wl.group_widths) * es  # embeddings read by Pad-Split
    if wl.head:
        total += wl.D * es + wl.B * 4
    return total


def roofline_seconds(flops: float, nbytes: float, peak_flops: float, peak_bw: float) -> float:
    """Lower bound on time: the slower of compute at peak and traffic at bandwidth."""
    return max(flops / peak_flops, nbytes / peak_bw)


def stat_slices(wl: Workload) -> int:
    """LayerNorm partials per row that the FFN stage writes: one per 64
    columns from the dense bf16 second projection, else one per row."""
    return wl.D // 64 if (wl.dtype == "bf16" and wl.n_experts == 0 and wl.D % 64 == 0) else 1


def kernel_work(wl: Workload, kind: str, active_mean: Optional[float] = None):
    """Algorithmic work of one launch of a kernel kind of the stack:
    ("bytes", n) for memory-bound kernels (what the kernel must read and write
    at least once), ("flops", n) for the FFN contractions.  For MoE kinds,
    active_mean is the mean number of active (sample, token, expert) entries
    per block."""
    es = ELEM_BYTES[wl.dtype]
    B, T, D, Hd, L = wl.B, wl.T, wl.D, wl.hidden, wl.L
    act = B * T * D * es
    stats = B * T * stat_slices(wl) * 8              # (mean, M2) float pairs
    A = active_mean or 0.0
    if kind == "mix_ln":        # X in, S out; blocks after the first also read the previous LN2 statistics
        return "bytes", 2 * act + stats * (L - 1) / L
    if kind == "ln_pool":       # Y and its statistics in, pooled (fp32) out
        return "bytes", act + stats + B * D * 4
    if kind == "padsplit":      # feature groups in, tokens out
        return "bytes", B * sum(wl.group_widths) * es + act
    if kind == "head":
        return "bytes", B * D * 4 + D * es + B * 4
    if kind == "token_mix":
        return "bytes", 2 * act
    if kind == "layernorm":     # in a stack: row statistics of the FFN output (fp32 path), V in, (mean, M2) out
        return "bytes", act + B * T * 8
    if kind == "moe_route":     # S and the routers in, gates out
        return "bytes", act + T * wl.n_experts * (D + 1) * 4 + B * T * wl.n_experts * 4
    if kind == "moe_gather":    # active rows copied
        return "bytes", 2 * A * D * es
    if kind == "moe_combine":   # expert rows and the residual in, block output and its statistics out
        return "bytes", A * D * es + 2 * act + B * T * 8
    if kind in ("gemm1", "gemm2"):
        return "flops", (2.0 * A * D * Hd) if wl.n_experts else (2.0 * B * T * D * Hd)
    raise KeyError(kind)
