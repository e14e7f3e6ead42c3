"""Per-kernel parity of the CUDA path against the fp64 oracle, through the C ABI,
on small and ragged shapes (several tiles plus a ragged tail)."""
import numpy as np
import pytest
import torch

from gpu_common import assert_close, dev, host64
from token_mixing_feature_b200 import synth

pytestmark = pytest.mark.gpu

TD = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module")
def rm():
    from token_mixing_feature_b200 import rankmixer
    return rankmixer


def _handle(rm, B, T, D, hidden, dtype, n_experts=0, L=1):
    return rm.rm_create(B, T, D, hidden, L, n_experts, dtype)


# ------------------------------------------------------------------ token mix
@pytest.mark.parametrize("dtype,T,dh,B", [
    ("bf16", 8, 8, 3), ("bf16", 16, 48, 5), ("bf16", 16, 20, 7), ("bf16", 32, 48, 2),
    ("bf16", 1, 64, 4), ("f32", 8, 8, 3), ("f32", 4, 6, 2), ("f32", 2, 4, 9),
    ("bf16", 16, 1, 3),     # dh = 1: every output element from a different token
    ("bf16", 64, 24, 2)])   # T = 64, the largest token count
def test_token_mix_bitexact(rm, O, dtype, T, dh, B):
    D = T * dh
    X = synth.random_activations((B, T, D), dtype, seed=T + dh)
    with _handle(rm, B, T, D, 64, dtype) as h:
        Xd = dev(X)
        Y = torch.empty_like(Xd)
        rm.rm_token_mix(h, Xd, Y, B)
        Z = torch.empty_like(Xd)
        rm.rm_token_mix(h, Y, Z, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    np.testing.assert_array_equal(host64(Y), O.token_mix(X))
    assert torch.equal(Z, Xd)          # mixing twice is the identity


# ------------------------------------------------------------------ LayerNorm
@pytest.mark.parametrize("dtype,D,rows", [("bf16", 768, 300), ("bf16", 320, 33), ("f32", 64, 129)])
def test_layernorm(rm, O, dtype, D, rows):
    A = synth.random_activations((rows, D), dtype, seed=1, std=2.0)
    R = synth.random_activations((rows, D), dtype, seed=2)
    g = synth.random_activations((D,), "f32", seed=3, std=0.1) + 1
    b = synth.random_activations((D,), "f32", seed=4, std=0.1)
    with _handle(rm, rows, 1, D, 64, dtype) as h:
        out = torch.empty(rows, D, dtype=TD[dtype], device="cuda")
        rm.rm_layernorm(h, dev(A), dev(R), dev(g), dev(b), out, rows)
        assert rm.rm_sync_status(h) == rm.RM_OK
    ref = O.layernorm(A.double() + R.double(), g, b)
    assert_close(host64(out), ref, dtype, "layernorm")


# ------------------------------------------------------------ per-token FFN
@pytest.mark.parametrize("T,D,hidden,B", [
    (4, 64, 128, 200),       # narrow N: one 128-wide tile, half masked
    (8, 384, 1536, 130),     # 6 K slices, ragged M tail
    (16, 320, 1280, 257),    # D = 320: 160-wide tiles, 20 K slices
    (2, 96, 256, 1),         # K = 96: partial second K slice, B = 1
])
def test_pffn_bf16_tensor_cores(rm, O, T, D, hidden, B):
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=T * 7 + 1)
    S = synth.random_activations((B, T, D), "bf16", seed=5)
    with _handle(rm, B, T, D, hidden, "bf16") as h:
        V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_pffn_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    ref = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"])
    assert_close(host64(V), ref, "bf16", "pffn", raw=True)


@pytest.mark.parametrize("T,D,hidden,B", [(8, 64, 256, 64), (3, 24, 40, 5), (1, 128, 64, 70)])
def test_pffn_f32_cuda_cores(rm, O, T, D, hidden, B):
    blk = synth.random_like_block(T, D, hidden, "f32", seed=T + 11)
    S = synth.random_activations((B, T, D), "f32", seed=6)
    with _handle(rm, B, T, D, hidden, "f32") as h:
        V = torch.empty(B, T, D, dtype=torch.float32, device="cuda")
        rm.rm_pffn_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    ref = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"])
    assert_close(host64(V), ref, "f32", "pffn f32")


def test_pffn_gelu_erf(rm, O):
    T, D, hidden, B = 4, 128, 256, 140
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=17)
    S = synth.random_activations((B, T, D), "bf16", seed=18)
    with rm.rm_create(B, T, D, hidden, 1, 0, "bf16", 1e-5, "erf") as h:
        V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_pffn_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    ref = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"], gelu="erf")
    assert_close(host64(V), ref, "bf16", "pffn erf", raw=True)


@pytest.mark.parametrize("T,D,hidden,B", [(4, 256, 2048, 256), (4, 320, 1536, 300)])
def test_pffn_split_k_tail(rm, O, monkeypatch, T, D, hidden, B):
    """Few output tiles over a long K: the second projection's last wave is
    split into K slices on otherwise idle SMs, summed in slice order by the
    slice that finishes last.  Parity with the oracle, bitwise repeatability
    (whichever slice finishes last), agreement with the unsplit kernel."""
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=D + hidden)
    S = synth.random_activations((B, T, D), "bf16", seed=21)
    with _handle(rm, B, T, D, hidden, "bf16") as h:
        w = {k: dev(v) for k, v in blk.items()}
        Sd = dev(S)
        runs = []
        for _ in range(3):
            V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
            rm.rm_pffn_forward(h, w, Sd, V, B)
            runs.append(V)
        monkeypatch.setenv("RM_GEMM_SPLIT", "0")
        V0 = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_pffn_forward(h, w, Sd, V0, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    for V in runs[1:]:
        assert torch.equal(V, runs[0])
    ref = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"])
    assert_close(host64(runs[0]), ref, "bf16", "pffn split-K", raw=True)
    assert_close(host64(V0), ref, "bf16", "pffn unsplit", raw=True)


@pytest.mark.parametrize("bn", ["256", "192", "128"])
def test_pffn_dense_tile_widths(rm, O, monkeypatch, bn):
    """Every dense tile width of the 2-SM kernel on N = 320 (ragged last
    tile), with the split-K tail (few tiles over K = 1536): 64-column chunks
    alternate between the epilogue halves, so 192-wide tiles give one half
    two chunks and the other one."""
    monkeypatch.setenv("RM_GEMM_BN", bn)
    T, D, hidden, B = 4, 320, 1536, 300
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=77)
    S = synth.random_activations((B, T, D), "bf16", seed=78)
    with _handle(rm, B, T, D, hidden, "bf16") as h:
        V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_pffn_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    ref = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"])
    assert_close(host64(V), ref, "bf16", f"pffn BN={bn}", raw=True)


# --------------------------------------------------------------------- block
@pytest.mark.parametrize("dtype,T,D,hidden,B", [
    ("bf16", 16, 768, 3072, 96), ("bf16", 16, 320, 1280, 130), ("bf16", 8, 128, 512, 3),
    ("bf16", 8, 96, 256, 33),     # dh = 12: mixed term in 8-byte pieces
    ("bf16", 8, 80, 256, 17),     # dh = 10: mixed term element by element
    ("f32", 8, 64, 256, 64), ("f32", 4, 32, 64, 7),
    ("f32", 4, 24, 64, 5)])       # dh = 6: 8-byte pieces of fp32
def test_block_forward(rm, O, dtype, T, D, hidden, B):
    blk = synth.random_like_block(T, D, hidden, dtype, seed=D + T)
    X = synth.random_activations((B, T, D), dtype, seed=9)
    with _handle(rm, B, T, D, hidden, dtype) as h:
        Xout = torch.empty(B, T, D, dtype=TD[dtype], device="cuda")
        rm.rm_block_forward(h, {k: dev(v) for k, v in blk.items()}, dev(X), Xout, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    assert_close(host64(Xout), O.block(X, blk), dtype, "block")


# ----------------------------------------------------------------- Pad-Split
def test_padsplit_bitexact(rm, O):
    wl = synth.WORKLOADS["padsplit"].with_batch(37)
    groups = synth.make_groups(wl)
    with _handle(rm, wl.B, wl.T, wl.D, wl.hidden, "bf16") as h:
        X0 = torch.empty(wl.B, wl.T, wl.D, dtype=torch.bfloat16, device="cuda")
        rm.rm_padsplit_tokenize(h, [dev(g) for g in groups], X0, wl.B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    ref = O.padsplit(groups, wl.padded_width).reshape(wl.B, wl.T, wl.D)
    np.testing.assert_array_equal(host64(X0), ref)


def test_head(rm, O):
    B, D = 77, 320
    pooled = synth.random_activations((B, D), "f32", seed=21, std=0.3)
    w = synth.random_activations((D,), "bf16", seed=22, std=0.08)
    bias = torch.tensor([0.125])
    with _handle(rm, B, 16, D, 64, "bf16") as h:
        prob = torch.empty(B, dtype=torch.float32, device="cuda")
        rm.rm_head_forward(h, dev(w), dev(bias), dev(pooled), prob, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    np.testing.assert_allclose(host64(prob), O.head(pooled, w, 0.125), rtol=0, atol=1e-6)


# ----------------------------------------------------------------- sparse MoE
def _moe_case(B, T, D, hidden, Ne, seed, router_std=0.1, router_bias=-0.05):
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=seed, n_experts=Ne,
                                  router_std=router_std, router_bias=router_bias)
    S = synth.random_activations((B, T, D), "bf16", seed=seed + 1)
    return blk, S


@pytest.mark.parametrize("B,T,D,hidden,Ne", [(300, 4, 64, 128, 8), (129, 2, 256, 256, 3), (1, 4, 64, 64, 2),
                                             (40, 2, 1280, 64, 32)])   # 32 experts, router rows at 160 KB
def test_moe_router_masks_and_output(rm, O, B, T, D, hidden, Ne):
    blk, S = _moe_case(B, T, D, hidden, Ne, seed=B + Ne)
    with _handle(rm, B, T, D, hidden, "bf16", n_experts=Ne) as h:
        V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        G = torch.empty(B, T, Ne, dtype=torch.float32, device="cuda")
        rm.rm_moe_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, G, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    Vref, logits = O.moe(S, blk)
    g = host64(G)
    decided = np.abs(logits) >= 1e-3      # the kernel decides in fp32, the oracle in fp64
    np.testing.assert_array_equal((g > 0)[decided], (logits > 0)[decided])
    np.testing.assert_allclose(g, np.maximum(logits, 0), rtol=0, atol=1e-4)
    assert_close(host64(V), Vref, "bf16", "moe", raw=True)


def test_moe_all_gates_closed(rm, O):
    B, T, D, hidden, Ne = 64, 4, 64, 64, 4
    blk, S = _moe_case(B, T, D, hidden, Ne, seed=3, router_bias=-10.0)
    with _handle(rm, B, T, D, hidden, "bf16", n_experts=Ne) as h:
        V = torch.full((B, T, D), 7.0, dtype=torch.bfloat16, device="cuda")
        rm.rm_moe_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, None, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    assert torch.count_nonzero(V).item() == 0


def test_moe_single_open_expert_is_pffn(rm, O):
    B, T, D, hidden = 150, 4, 128, 256
    blk, S = _moe_case(B, T, D, hidden, 1, seed=5)
    blk["Wr"].zero_()
    blk["br"].fill_(1.0)
    with _handle(rm, B, T, D, hidden, "bf16", n_experts=1) as h:
        V = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_moe_forward(h, {k: dev(v) for k, v in blk.items()}, dev(S), V, None, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    ref = O.pffn(S, blk["W1"][:, 0], blk["b1"][:, 0], blk["W2"][:, 0], blk["b2"][:, 0])
    assert_close(host64(V), ref, "bf16", "moe single expert", raw=True)


def test_moe_block(rm, O):
    B, T, D, hidden, Ne = 200, 4, 128, 128, 8
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=31, n_experts=Ne, router_std=0.05,
                                  router_bias=-0.02)
    X = synth.random_activations((B, T, D), "bf16", seed=32)
    with _handle(rm, B, T, D, hidden, "bf16", n_experts=Ne) as h:
        Xout = torch.empty(B, T, D, dtype=torch.bfloat16, device="cuda")
        rm.rm_block_forward(h, {k: dev(v) for k, v in blk.items()}, dev(X), Xout, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    assert_close(host64(Xout), O.block(X, blk), "bf16", "moe block")


def test_moe_pair_tiles_match(rm, O, tmp_path):
    """Expert GEMMs on CTA pairs with 256-row tiles (tuning override
    RM_MOE_PAIR=1, read once per process: a child process) give the MoE block
    within the bf16 bounds of the oracle; a group's odd CTA past the group's
    end computes nothing it stores."""
    import os
    import subprocess
    import sys
    B, T, D, hidden, Ne = 300, 4, 128, 128, 8
    blk = synth.random_like_block(T, D, hidden, "bf16", seed=33, n_experts=Ne, router_std=0.1,
                                  router_bias=-0.05)
    X = synth.random_activations((B, T, D), "bf16", seed=34)
    torch.save({"blk": blk, "X": X}, tmp_path / "in.pt")
    script = tmp_path / "run.py"
    script.write_text(
        "import sys, torch\n"
        "sys.path.insert(0, %r)\n"
        "from token_mixing_feature_b200 import rankmixer as rm\n"
        "d = torch.load(sys.argv[1])\n"
        "blk = {k: v.cuda().contiguous() for k, v in d['blk'].items()}\n"
        "X = d['X'].cuda()\n"
        "with rm.rm_create(%d, %d, %d, %d, 1, %d, 'bf16') as h:\n"
        "    out = torch.empty_like(X)\n"
        "    rm.rm_block_forward(h, blk, X, out, %d)\n"
        "    assert rm.rm_sync_status(h) == rm.RM_OK\n"
        "torch.save(out.cpu(), sys.argv[2])\n" % (os.getcwd(), B, T, D, hidden, Ne, B))
    env = dict(os.environ, RM_MOE_PAIR="1")
    subprocess.run([sys.executable, str(script), str(tmp_path / "in.pt"), str(tmp_path / "out.pt")], check=True,
                   env=env, timeout=600)
    got = torch.load(tmp_path / "out.pt")
    assert_close(host64(got), O.block(X, blk), "bf16", "moe block, pair tiles")


# ------------------------------------------------------ robustness / checks
def test_deterministic(rm):
    T, D, hidden, B = 16, 256, 1024, 200
    blk = {k: dev(v) for k, v in synth.random_like_block(T, D, hidden, "bf16", seed=41).items()}
    X = dev(synth.random_activations((B, T, D), "bf16", seed=42))
    with _handle(rm, B, T, D, hidden, "bf16") as h:
        a = torch.empty_like(X)
        b = torch.empty_like(X)
        rm.rm_block_forward(h, blk, X, a, B)
        rm.rm_block_forward(h, blk, X, b, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    assert torch.equal(a, b)


def test_bounded_wait_times_out_and_context_survives(rm):
    with _handle(rm, 4, 4, 64, 64, "bf16") as h:
        rm.rm_set_wait_budget(h, 20_000_000)    # 20 ms
        rm.rm_selftest_wait_timeout(h)
        assert rm.rm_sync_status(h) == rm.RM_ERR_DEVICE_TIMEOUT
        assert rm.rm_last_error_site(h) == 9
        assert rm.rm_sync_status(h) == rm.RM_OK       # cleared
        X = dev(synth.random_activations((4, 4, 64), "bf16", seed=1))
        Y = torch.empty_like(X)
        rm.rm_token_mix(h, X, Y, 4)
        assert rm.rm_sync_status(h) == rm.RM_OK


def test_argument_errors(rm):
    with _handle(rm, 8, 4, 64, 64, "bf16") as h:
        X = torch.zeros(16, 4, 64, dtype=torch.bfloat16, device="cuda")
        Y = torch.zeros_like(X)
        with pytest.raises(rm.RankMixerError) as e:
            rm.rm_token_mix(h, X, Y, 9)                     # B > B_max
        assert e.value.status == rm.RM_ERR_INVALID_ARG
        for B in (0, -1):                                   # empty / negative batch
            with pytest.raises(rm.RankMixerError) as e:
                rm.rm_token_mix(h, X, Y, B)
            assert e.value.status == rm.RM_ERR_INVALID_ARG
        with pytest.raises(rm.RankMixerError):
            rm.rm_token_mix(h, X.data_ptr() + 2, Y, 4)      # misaligned
        with pytest.raises(rm.RankMixerError) as e:
            rm.rm_moe_forward(h, {}, X, Y, None, 4)          # dense handle
        assert e.value.status == rm.RM_ERR_UNSUPPORTED
        assert rm.rm_sync_status(h) == rm.RM_OK


# ------------------------------------------------ variants on the pages
@pytest.mark.parametrize("dtype,act,addnorm,T,D,hidden,B", [
    ("bf16", "relu", True, 8, 256, 1024, 130),      # the Appendix B Mixer's ReLU
    ("bf16", "tanh", False, 16, 320, 1280, 70),     # no Add & Norm after mixing (dh = 20)
    ("bf16", "relu", False, 8, 128, 512, 3),
    ("f32", "relu", False, 8, 64, 256, 64),
    ("f32", "erf", True, 4, 32, 64, 9)])
def test_block_variants(rm, O, dtype, act, addnorm, T, D, hidden, B):
    blk = synth.random_like_block(T, D, hidden, dtype, seed=D + 3 * T)
    X = synth.random_activations((B, T, D), dtype, seed=19)
    with rm.rm_create(B, T, D, hidden, 1, 0, dtype, 1e-5, act, addnorm) as h:
        Xout = torch.empty(B, T, D, dtype=TD[dtype], device="cuda")
        rm.rm_block_forward(h, {k: dev(v) for k, v in blk.items()}, dev(X), Xout, B)
        assert rm.rm_sync_status(h) == rm.RM_OK
    assert_close(host64(Xout), O.block(X, blk, gelu=act, mix_addnorm=addnorm), dtype, f"block {act} {addnorm}")


def test_stack_without_mix_addnorm(rm, O):
    import dataclasses
    wl = dataclasses.replace(synth.WORKLOADS["rm100m"], B=96, mix_addnorm=False)
    d = synth.make_inputs(wl)
    from token_mixing_feature_b200.stack import RankMixerStack
    st = RankMixerStack(wl, d["blocks"])
    pooled = st.forward(dev(d["X0"]))
    assert rm.rm_sync_status(st.h) == rm.RM_OK
    ref = O.stack(d["X0"], d["blocks"], mix_addnorm=False)
    assert_close(host64(pooled), ref["pooled"], "bf16", "pooled, no Add & Norm")
    st.close()
