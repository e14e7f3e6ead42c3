"""The fused per-token FFN (both projections in one tcgen05 kernel, the hidden
activation kept on chip) against the fp64 oracle, through the C ABI.

RM_FFN_FUSED=1 selects the fused kernel (run_pffn uses the two grouped
GEMMs otherwise).
Shapes cover every supported width D <= 320 (one or two second-projection
MMAs per chunk, D = 64 where one epilogue half has no output slice), one and several
hidden chunks, ragged row tails (a partial tile, a CTA with no valid row,
B = 1), and more tiles than CTA pairs, so that pairs run the cross-tile
pipeline (the next tile's first hidden chunk before the previous tile's
output rows)."""
import dataclasses

import pytest
import torch

from gpu_common import assert_close, dev, host64
from token_mixing_feature_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rm():
    from token_mixing_feature_b200 import rankmixer
    return rankmixer


@pytest.fixture
def fused(monkeypatch):
    monkeypatch.setenv("RM_FFN_FUSED", "1")


def _pffn(rm, blk, S, B, T, D, hidden, act="tanh"):
    with rm.rm_create(B, T, D, hidden, 1, 0, "bf16", 1e-5, act) as h:
        V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_pffn_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    return V


@pytest.mark.parametrize("T,D,hidden,B,act", [
    (4, 64, 128, 200, "tanh"),      # D = 64: one 64-wide MMA; second CTA of the tile partly valid
    (4, 128, 256, 300, "relu"),     # two tiles per token, the second CTA of tile 2 has no rows
    (2, 192, 384, 513, "erf"),      # N = 192 second projection, one row in the last tile
    (4, 256, 1024, 256, "tanh"),    # exactly one tile per token, 8 hidden chunks
    (16, 320, 1280, 257, "tanh"),   # the Pad-Split width: two 160-wide MMAs per chunk
    (8, 256, 384, 130, "tanh"),     # one 256-wide second-projection MMA, 3 hidden chunks
    (2, 320, 128, 1, "tanh"),       # B = 1, a single hidden chunk
    (64, 64, 256, 2048, "tanh"),    # 512 tiles: every CTA pair runs several tiles
    (32, 320, 256, 1024, "relu"),   # 128 tiles over the pairs: some run two
])
def test_ffn_fused_parity(rm, O, fused, T, D, hidden, B, act):
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=D + hidden + T)
    S = synth.random_activations((B, T, D), "bf16", seed=B + 3)
    V = _pffn(rm, blk, S, B, T, D, hidden, act)
    ref = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"], gelu=act)
    assert_close(host64(V), ref, "bf16", f"fused pffn D={D} kD={hidden} B={B} {act}", raw=True)


@pytest.mark.parametrize("T,D,hidden,B", [(16, 320, 1280, 300), (8, 256, 512, 700), (4, 192, 768, 260)])
def test_ffn_fused_matches_two_gemm_path(rm, monkeypatch, T, D, hidden, B):
    """Same sums in the same K order as the two grouped GEMMs without their
    split-K tail (both round the hidden activation to bf16 before the second
    projection): the outputs are identical bit for bit."""
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=D * 3 + B)
    S = synth.random_activations((B, T, D), "bf16", seed=D + 1)
    monkeypatch.setenv("RM_GEMM_SPLIT", "0")
    monkeypatch.setenv("RM_FFN_FUSED", "1")
    Vf = _pffn(rm, blk, S, B, T, D, hidden)
    monkeypatch.setenv("RM_FFN_FUSED", "0")
    Vg = _pffn(rm, blk, S, B, T, D, hidden)
    diff = (Vf.float() - Vg.float()).abs().max().item()
    assert torch.equal(Vf, Vg), f"fused and two-GEMM outputs differ (max abs {diff:.3e})"


def test_ffn_fused_deterministic(rm, fused):
    T, D, hidden, B = 16, 320, 1280, 1100
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=5)
    S = synth.random_activations((B, T, D), "bf16", seed=6)
    runs = [_pffn(rm, blk, S, B, T, D, hidden) for _ in range(3)]
    for V in runs[1:]:
        assert torch.equal(V, runs[0])


@pytest.mark.parametrize("L,T,D,hidden,B", [(2, 16, 320, 1280, 300), (3, 8, 256, 1024, 130)])
def test_stack_with_fused_ffn(rm, O, fused, L, T, D, hidden, B):
    """The stack consumes the fused kernel's LayerNorm partials (next block's
    mixing, final LayerNorm + pooling) and its residual path."""
    wl = dataclasses.replace(synth.WORKLOADS["padsplit"], B=B, T=T, D=D, hidden=hidden, L=L,
                             group_widths=(), head=False, ln_params="perturbed")
    d = synth.make_inputs(wl)
    from token_mixing_feature_b200.stack import RankMixerStack
    st = RankMixerStack(wl, d["blocks"])
    pooled = st.forward(dev(d["X0"]))
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    ref = O.stack(d["X0"], d["blocks"])
    assert_close(host64(pooled), ref["pooled"], "bf16", f"pooled, fused FFN, L={L} D={D}")
    st.close()


def test_ffn_fused_padsplit_size(rm, O, monkeypatch):
    """The Pad-Split serving size (16 tokens x 16 tiles of 256 samples): the
    launch is the fused kernel when asked for, the two grouped GEMMs
    otherwise; sampled rows against the oracle."""
    T, D, hidden, B = 16, 320, 1280, 4096
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=1)
    S = synth.random_activations((B, T, D), "bf16", seed=2)
    rows = torch.tensor([0, 1, 255, 256, 2047, 4095])
    ref = O.pffn(S[rows], blk["W1"], blk["b1"], blk["W2"], blk["b2"])   # (the full batch is 21 GFLOP of fp64)
    for flag, kinds in (("1", {"ffn_fused"}), (None, {"gemm1", "gemm2"})):
        if flag is None:
            monkeypatch.delenv("RM_FFN_FUSED", raising=False)
        else:
            monkeypatch.setenv("RM_FFN_FUSED", flag)
        with rm.rm_create(B, T, D, hidden, 1, 0, "bf16") as h:
            w = {k: dev(v) for k, v in blk.items()}
            V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
            rm.rm_profile_begin(h, 8)
            rm.rm_pffn_forward(h, w, dev(S), V, B)
            prof = rm.rm_profile_end(h)
            assert rm.rm_sync_status(h) == rm.RM_OK
        assert set(prof) == kinds, prof
        assert_close(host64(V[rows.cuda()]), ref, "bf16", f"pffn {kinds}, Pad-Split size (sampled rows)", raw=True)


def test_ffn_fused_unsupported_width_uses_gemms(rm, O, fused):
    """D = 384 leaves no tensor-memory room for the hidden chunk: even when
    asked for, the library runs the two grouped GEMMs."""
    T, D, hidden, B = 8, 384, 512, 130
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=11)
    S = synth.random_activations((B, T, D), "bf16", seed=12)
    with rm.rm_create(B, T, D, hidden, 1, 0, "bf16") as h:
        V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_profile_begin(h, 8)
        rm.rm_pffn_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, B)
        prof = rm.rm_profile_end(h)
        assert rm.rm_sync_status(h) == rm.RM_OK
    assert set(prof) == {"gemm1", "gemm2"}, prof
    ref = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"])
    assert_close(host64(V), ref, "bf16", "pffn D=384", raw=True)
