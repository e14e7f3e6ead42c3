"""rm_pffn_forward_static: the per-token FFN for callers that cannot allocate
device memory (no handle, so no cudaMalloc'd workspace; its scratch is a fixed
array inside the library).  Its output must match rm_pffn_forward's on the same
inputs, call after call, since every call reuses the same array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import pytest
import torch

from gpu_common import assert_close, dev, host64
from token_mixing_feature_b200 import synth

pytestmark = pytest.mark.gpu


def test_static_scratch_pffn_matches_handle_path():
    from token_mixing_feature_b200 import rankmixer as rm
    T, D, hidden, B = 8, 384, 1536, 130          # hidden activations: 3.2 MB of the 16 MB array
    blk = {k: dev(v) for k, v in synth.random_like_block(T, D, hidden, "bf16", seed=77).items()}
    S = dev(synth.random_activations((B, T, D), "bf16", seed=78))
    ref = torch.empty_like(S)
    with rm.rm_create(B, T, D, hidden, 1, 0, "bf16") as h:
        rm.rm_pffn_forward(h, blk, S, ref, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):                             # two calls in a row share the array
        V = torch.full_like(S, float("nan"))
        rm.rm_pffn_forward_static(blk, S, V, B, T, D, hidden, "bf16", "tanh", status)
        torch.cuda.synchronize()
        assert int(status.item()) == rm.RM_OK
        assert_close(host64(V), host64(ref), "bf16", "static-scratch pffn", raw=True)


def test_static_scratch_pffn_f32_matches_handle_path():
    """The fp32 form (CUDA-core kernels, hidden activations in the array)
    against rm_pffn_forward on an fp32 handle, two calls in a row."""
    from token_mixing_feature_b200 import rankmixer as rm
    T, D, hidden, B = 4, 64, 256, 37
    blk = {k: dev(v) for k, v in synth.random_like_block(T, D, hidden, "f32", seed=83).items()}
    S = dev(synth.random_activations((B, T, D), "f32", seed=84))
    ref = torch.empty_like(S)
    with rm.rm_create(B, T, D, hidden, 1, 0, "f32") as h:
        rm.rm_pffn_forward(h, blk, S, ref, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        V = torch.full_like(S, float("nan"))
        rm.rm_pffn_forward_static(blk, S, V, B, T, D, hidden, "f32", "tanh", status)
        torch.cuda.synchronize()
        assert int(status.item()) == rm.RM_OK
        assert_close(host64(V), host64(ref), "f32", "static-scratch pffn (fp32)")


def test_static_scratch_rejects_oversize():
    from token_mixing_feature_b200 import rankmixer as rm
    T, D, hidden = 8, 384, 1536
    B = rm.RM_STATIC_SCRATCH_BYTES // (T * hidden * 2) + 1     # one sample too many
    blk = {k: dev(v) for k, v in synth.random_like_block(T, D, hidden, "bf16", seed=79).items()}
    S = torch.zeros(B, T, D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RankMixerError) as e:
        rm.rm_pffn_forward_static(blk, S, torch.empty_like(S), B, T, D, hidden)
    assert e.value.status == rm.RM_ERR_INVALID_ARG
    # sizes whose product would wrap a 64-bit byte count are rejected before any launch
    with pytest.raises(rm.RankMixerError) as e:
        rm.rm_pffn_forward_static(blk, S, torch.empty_like(S), 2 ** 31 - 1, T, D, 2 ** 31 - 16)
    assert e.value.status == rm.RM_ERR_INVALID_ARG
