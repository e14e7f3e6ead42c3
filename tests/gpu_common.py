"""Shared helpers of the GPU parity tests (not a test module)."""
import numpy as np
import torch

# Tolerances.  bf16 storage with fp32 accumulation: every block output X_l and
# the pooled output within 1e-2 relative L2 AND 5e-2 max-abs of the fp64
# oracle; fp32 storage on CUDA cores: 1e-5 relative L2.  Token mixing,
# Pad-Split and router masks: bit-exact.  Outputs that no LayerNorm scales
# (the FFN / MoE output V alone) are not O(1): for those ("raw") the max-abs
# bound applies to the error divided by max(1, max |reference|).
BF16_REL_L2 = 1e-2
BF16_MAX_ABS = 5e-2
F32_REL_L2 = 1e-5


def dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda").contiguous()


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def max_abs(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.abs(got - ref).max()) if got.size else 0.0


def assert_close(got, ref, dtype: str, what: str = "", raw: bool = False) -> None:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    r = rel_l2(got, ref)
    if dtype == "f32":
        assert r <= F32_REL_L2, f"{what}: rel L2 {r:.3e} > {F32_REL_L2}"
    else:
        m = max_abs(got, ref)
        if raw:
            m /= max(1.0, float(np.abs(ref).max()))
        assert r <= BF16_REL_L2 and m <= BF16_MAX_ABS, f"{what}: rel L2 {r:.3e}, max abs {m:.3e}"


def sample_rows(B: int, n: int, seed: int = 1234) -> torch.Tensor:
    """n distinct sample indices (sorted), always including the first and last."""
    g = torch.Generator().manual_seed(seed)
    idx = torch.randperm(B, generator=g)[: max(0, n - 2)].tolist()
    return torch.tensor(sorted(set(idx) | {0, B - 1}), dtype=torch.long)
