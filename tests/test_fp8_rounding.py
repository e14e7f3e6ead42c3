"""The e4m3 rounding that the quantiser's GPU test compares against,
pinned on the CPU to an independent implementation of the format: PyTorch's
float8_e4m3fn conversion (round to nearest even, 3 mantissa bits, exponent
bias 7, subnormals below 2^-6), on every representable value, the midpoints
between neighbours (ties), and random values inside the saturation bound."""
import numpy as np
import torch

from test_gpu_fp8 import _e4m3_round


def _torch_e4m3(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _representable() -> np.ndarray:
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    v = v[np.isfinite(v)]
    return np.unique(v)


def test_representable_values_are_fixed_points():
    v = _representable()
    assert v.max() == 448.0 and v.min() == -448.0
    assert np.array_equal(_e4m3_round(v), v)


def test_midpoints_round_to_even():
    v = _representable()
    pos = v[v >= 0]
    mid = (pos[:-1] + pos[1:]) / 2
    got = _e4m3_round(np.concatenate([mid, -mid]))
    want = _torch_e4m3(np.concatenate([mid, -mid]))
    assert np.array_equal(got, want)


def test_random_values_match_the_format():
    g = np.random.default_rng(7)
    x = np.concatenate([g.uniform(-448, 448, 20000),
                        g.standard_normal(20000) * 2.0 ** g.integers(-12, 8, 20000)])
    x = np.clip(x, -448, 448)
    assert np.array_equal(_e4m3_round(x), _torch_e4m3(x))
