"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks an oracle function against a worked example, a closed form,
an invariant of the definitions, or a library routine (torch fp64) that
computes the same thing by a different route.  Together they are chosen so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from token_mixing_feature_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
EPS = 1e-5


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.float64)


# ---------------------------------------------------------------- token mixing
def test_mix_hand_examples(O):
    """Worked examples of SplitHead/Concat with H = T (fun-rec chapter, Token Mixing机制)."""
    with open(os.path.join(GOLDEN, "token_mix_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        X = np.array(c["X"], dtype=np.float64)[None]
        Y = O.token_mix(X)
        assert Y.shape == (1, c["T"], c["D"])
        np.testing.assert_array_equal(Y[0], np.array(c["Y"], dtype=np.float64))


@pytest.mark.parametrize("T,dh", [(1, 8), (2, 4), (4, 3), (8, 8), (16, 20), (32, 48)])
def test_mix_involution_and_permutation(O, T, dh):
    X = synth.random_activations((3, T, T * dh), seed=T * 100 + dh).double().numpy()
    Y = O.token_mix(X)
    np.testing.assert_array_equal(O.token_mix(Y), X)              # TM o TM = id
    np.testing.assert_array_equal(np.sort(Y.ravel()), np.sort(X.ravel()))  # pure permutation
    if T == 1:
        np.testing.assert_array_equal(Y, X)


@pytest.mark.parametrize("T,dh", [(2, 4), (8, 8), (16, 20)])
def test_mix_matches_library_permute(O, T, dh):
    """The chunk transpose equals torch's view/transpose of [B, T, H, dh] -> [B, H, T, dh]."""
    B = 5
    X = synth.random_activations((B, T, T * dh), seed=3).double()
    ref = X.view(B, T, T, dh).transpose(1, 2).reshape(B, T, T * dh)
    np.testing.assert_array_equal(O.token_mix(X), ref.numpy())


def test_mix_rejects_indivisible(O):
    with pytest.raises(ValueError):
        O.token_mix(np.zeros((1, 3, 8)))


# ---------------------------------------------------------------- LayerNorm
def test_layernorm_moments(O):
    """gamma=1, beta=0: each row has mean 0 and variance sigma^2/(sigma^2+eps)."""
    Z = synth.random_activations((64, 96), seed=11, std=0.05).double().numpy() + 0.3
    out = O.layernorm(Z, np.ones(96), np.zeros(96), eps=EPS)
    var_in = Z.var(axis=1)
    assert np.abs(out.mean(axis=1)).max() < 1e-12
    np.testing.assert_allclose(out.var(axis=1), var_in / (var_in + EPS), rtol=1e-12)


def test_layernorm_matches_library(O):
    Z = synth.random_activations((40, 48), seed=12, std=3.0).double()
    g = synth.random_activations((48,), seed=13, std=0.5) + 1.0
    b = synth.random_activations((48,), seed=14, std=0.5)
    ref = F.layer_norm(Z, (48,), g.double(), b.double(), eps=EPS)
    np.testing.assert_allclose(O.layernorm(Z, g, b, EPS), ref.numpy(), rtol=0, atol=1e-12)


def test_layernorm_zero_row_and_scale_invariance(O):
    g = np.linspace(0.5, 1.5, 32).astype(np.float32)
    b = np.linspace(-1, 1, 32).astype(np.float32)
    out = O.layernorm(np.zeros((1, 32)), g, b, EPS)
    np.testing.assert_array_equal(out[0], b.astype(np.float64))   # zero row -> beta
    Z = synth.random_activations((4, 32), seed=15).double().numpy()
    np.testing.assert_allclose(O.layernorm(7.5 * Z, g, b, 0.0), O.layernorm(Z, g, b, 0.0),
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------------- GELU
def test_gelu_forms(O):
    u = np.linspace(-8, 8, 1001)
    ref_tanh = F.gelu(_t(u), approximate="tanh").numpy()
    ref_erf = np.array([0.5 * x * (1 + math.erf(x / math.sqrt(2))) for x in u])
    np.testing.assert_allclose(O.gelu(u, "tanh"), ref_tanh, rtol=0, atol=1e-14)
    np.testing.assert_allclose(O.gelu(u, "erf"), ref_erf, rtol=0, atol=1e-14)
    # the two forms agree to the published accuracy of the tanh approximation
    assert np.abs(O.gelu(u, "tanh") - ref_erf).max() < 1e-3
    assert O.gelu(np.array([0.0]))[0] == 0.0


# ---------------------------------------------------------------- per-token FFN
def _torch_ffn(S, W1, b1, W2, b2):
    return F.linear(F.gelu(F.linear(S, W1, b1), approximate="tanh"), W2, b2)


def test_pffn_tied_weights_is_shared_ffn(O):
    """All T weight sets equal -> a shared FFN applied to every token."""
    B, T, D, Hd = 6, 4, 16, 40
    blk = synth.random_like_block(1, D, Hd, seed=21)
    W1, b1, W2, b2 = (blk[k].repeat(T, *([1] * (blk[k].dim() - 1))) for k in ("W1", "b1", "W2", "b2"))
    S = synth.random_activations((B, T, D), seed=22).double()
    V = O.pffn(S, W1, b1, W2, b2)
    ref = _torch_ffn(S, blk["W1"][0].double(), blk["b1"][0].double(), blk["W2"][0].double(),
                     blk["b2"][0].double())
    np.testing.assert_allclose(V, ref.numpy(), rtol=0, atol=1e-12)


def test_pffn_grouped_matches_einsum(O):
    """Per-token weights: the grouped [T,B,D]@[T,D,kD] form via einsum."""
    B, T, D, Hd = 5, 6, 12, 20
    blk = synth.random_like_block(T, D, Hd, seed=23)
    S = synth.random_activations((B, T, D), seed=24).double()
    W1, b1, W2, b2 = (blk[k].double() for k in ("W1", "b1", "W2", "b2"))
    u = torch.einsum("btd,thd->bth", S, W1) + b1
    ref = torch.einsum("bth,tdh->btd", F.gelu(u, approximate="tanh"), W2) + b2
    np.testing.assert_allclose(O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"]), ref.numpy(),
                               rtol=0, atol=1e-12)


def test_pffn_token_isolation(O):
    """Changing token 2's weights changes token 2's output only."""
    B, T, D, Hd = 3, 4, 8, 16
    blk = synth.random_like_block(T, D, Hd, seed=25)
    S = synth.random_activations((B, T, D), seed=26)
    V0 = O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"])
    W1 = blk["W1"].clone()
    W1[2] *= -1.7
    V1 = O.pffn(S, W1, blk["b1"], blk["W2"], blk["b2"])
    changed = np.abs(V1 - V0).max(axis=(0, 2))
    assert changed[2] > 1e-3 and np.all(changed[[0, 1, 3]] == 0)


# ---------------------------------------------------------------- block / stack
def _torch_block(X, blk):
    B, T, D = X.shape
    dh = D // T
    mixed = X.view(B, T, T, dh).transpose(1, 2).reshape(B, T, D)
    S = F.layer_norm(mixed + X, (D,), blk["ln1_g"].double(), blk["ln1_b"].double(), eps=EPS)
    W1, b1, W2, b2 = (blk[k].double() for k in ("W1", "b1", "W2", "b2"))
    u = torch.einsum("btd,thd->bth", S, W1) + b1
    V = torch.einsum("bth,tdh->btd", F.gelu(u, approximate="tanh"), W2) + b2
    return F.layer_norm(V + S, (D,), blk["ln2_g"].double(), blk["ln2_b"].double(), eps=EPS)


@pytest.mark.parametrize("T,dh,Hd", [(2, 4, 24), (4, 6, 32), (8, 8, 64)])
def test_block_matches_torch_composition(O, T, dh, Hd):
    D = T * dh
    blk = synth.random_like_block(T, D, Hd, seed=31 + T)
    X = synth.random_activations((7, T, D), seed=32 + T).double()
    np.testing.assert_allclose(O.block(X, blk, EPS), _torch_block(X, blk).numpy(), rtol=0, atol=1e-12)


def test_block_single_token_is_plain_mlp(O):
    """T = 1: mixing is the identity, so X' = LN(MLP(LN(2X)) + LN(2X))."""
    D, Hd = 24, 48
    blk = synth.random_like_block(1, D, Hd, seed=41)
    X = synth.random_activations((9, 1, D), seed=42).double()
    S = F.layer_norm(2 * X, (D,), blk["ln1_g"].double(), blk["ln1_b"].double(), eps=EPS)
    V = _torch_ffn(S, blk["W1"][0].double(), blk["b1"][0].double(), blk["W2"][0].double(),
                   blk["b2"][0].double())
    ref = F.layer_norm(V + S, (D,), blk["ln2_g"].double(), blk["ln2_b"].double(), eps=EPS)
    np.testing.assert_allclose(O.block(X, blk, EPS), ref.numpy(), rtol=0, atol=1e-12)


def test_stack_composes_blocks_and_pools_last(O):
    wl = synth.WORKLOADS["tiny_f32"].with_batch(6)
    d = synth.make_inputs(wl)
    r = O.stack(d["X0"], d["blocks"], EPS, want_all=True)
    x = d["X0"].double()
    for l, blk in enumerate(d["blocks"]):
        x = _torch_block(x, blk)
        np.testing.assert_allclose(r["Xall"][l], x.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(r["Xlast"], r["Xall"][-1])
    np.testing.assert_allclose(r["pooled"], x.mean(dim=1).numpy(), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- sparse MoE
def _moe_block(T, D, Hd, Ne, seed, **kw):
    return synth.random_like_block(T, D, Hd, seed=seed, n_experts=Ne, **kw)


def test_moe_single_always_on_expert_is_pffn(O):
    """N_e = 1, router weights 0, bias 1 -> gate 1 -> the dense per-token FFN."""
    B, T, D, Hd = 4, 4, 16, 24
    blk = _moe_block(T, D, Hd, 1, 51)
    blk["Wr"].zero_()
    blk["br"].fill_(1.0)
    S = synth.random_activations((B, T, D), seed=52)
    V, logits = O.moe(S, blk)
    np.testing.assert_array_equal(logits, np.ones((B, T, 1)))
    ref = O.pffn(S, blk["W1"][:, 0], blk["b1"][:, 0], blk["W2"][:, 0], blk["b2"][:, 0])
    np.testing.assert_allclose(V, ref, rtol=0, atol=1e-13)


def test_moe_all_gates_closed(O):
    """Bias -10 closes every gate: V = 0 and the block output is LN2(S)."""
    B, T, D, Hd, Ne = 3, 4, 16, 16, 4
    blk = _moe_block(T, D, Hd, Ne, 53, router_bias=-10.0)
    S = synth.random_activations((B, T, D), seed=54)
    V, _ = O.moe(S, blk)
    assert np.all(V == 0)
    X = synth.random_activations((B, T, D), seed=55).double()
    dh = D // T
    mixed = X.view(B, T, T, dh).transpose(1, 2).reshape(B, T, D)
    Sx = F.layer_norm(mixed + X, (D,), blk["ln1_g"].double(), blk["ln1_b"].double(), eps=EPS)
    ref = F.layer_norm(Sx, (D,), blk["ln2_g"].double(), blk["ln2_b"].double(), eps=EPS)
    np.testing.assert_allclose(O.block(X, blk, EPS), ref.numpy(), rtol=0, atol=1e-12)


def test_moe_skipping_equals_dense_evaluation(O):
    """Evaluating every expert and weighting by ReLU(logit) equals the skipping form."""
    B, T, D, Hd, Ne = 16, 4, 16, 24, 6
    blk = _moe_block(T, D, Hd, Ne, 56, router_std=0.3, router_bias=-0.2)
    S = synth.random_activations((B, T, D), seed=57).double()
    V, logits = O.moe(S, blk)
    ref_logits = torch.einsum("btd,tjd->btj", S, blk["Wr"].double()) + blk["br"].double()
    np.testing.assert_allclose(logits, ref_logits.numpy(), rtol=0, atol=1e-13)
    gates = torch.relu(ref_logits)
    assert 0 < float((gates > 0).double().mean()) < 1         # some skipped, some active
    ref = torch.zeros(B, T, D, dtype=torch.float64)
    for j in range(Ne):   # expert j of every token, evaluated densely with library ops
        W1, b1, W2, b2 = (blk[k][:, j].double() for k in ("W1", "b1", "W2", "b2"))
        u = torch.einsum("btd,thd->bth", S, W1) + b1
        e = torch.einsum("bth,tdh->btd", F.gelu(u, approximate="tanh"), W2) + b2
        ref += gates[:, :, j:j + 1] * e
    np.testing.assert_allclose(V, ref.numpy(), rtol=0, atol=1e-12)


def test_router_logits_alone(O):
    """The router-only entry equals the logits the MoE forward reports, and a
    router that reads one input column per expert returns that column plus the
    bias (a hand-checkable case of the linear router h_t)."""
    B, T, D, Hd, Ne = 6, 3, 16, 8, 5
    blk = _moe_block(T, D, Hd, Ne, 60, router_std=0.4, router_bias=-0.1)
    S = synth.random_activations((B, T, D), seed=61)
    _, logits = O.moe(S, blk)
    np.testing.assert_array_equal(O.router(S, blk["Wr"], blk["br"]), logits)
    Wr = torch.zeros(T, Ne, D)
    for t in range(T):
        for j in range(Ne):
            Wr[t, j, (3 * t + j) % D] = 1.0          # expert j of token t reads column 3t + j
    br = torch.arange(T * Ne, dtype=torch.float32).reshape(T, Ne) * 0.25
    got = O.router(S, Wr, br)
    Sd = S.double().numpy()
    for t in range(T):
        for j in range(Ne):
            np.testing.assert_array_equal(got[:, t, j], Sd[:, t, (3 * t + j) % D] + float(br[t, j]))


def test_moe_gate_scales_second_bias(O):
    """W2 = 0: every active expert returns its b2, scaled by its gate."""
    B, T, D, Hd, Ne = 5, 2, 8, 8, 3
    blk = _moe_block(T, D, Hd, Ne, 58, router_std=0.5, router_bias=0.1)
    blk["W2"].zero_()
    S = synth.random_activations((B, T, D), seed=59)
    V, logits = O.moe(S, blk)
    ref = np.einsum("btj,tjd->btd", np.maximum(logits, 0), blk["b2"].double().numpy())
    np.testing.assert_allclose(V, ref, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- Pad-Split / head
def test_padsplit_matches_concat_and_pad(O):
    wl = synth.WORKLOADS["padsplit"].with_batch(3)
    groups = synth.make_groups(wl)
    X0 = O.padsplit(groups, wl.padded_width)
    ref = F.pad(torch.cat([g.double() for g in groups], dim=1), (0, wl.padded_width - 4800))
    np.testing.assert_array_equal(X0, ref.numpy())
    tokens = X0.reshape(3, wl.T, wl.D)
    assert np.all(tokens[:, 15] == 0)          # columns 4800..5119: padding token
    assert np.all(tokens[:, 14] != 0)


def test_head_sigmoid(O):
    P = synth.random_activations((10, 32), seed=61).double()
    w = synth.random_activations((32,), seed=62)
    ref = torch.sigmoid(P @ w.double() + 0.25)
    np.testing.assert_allclose(O.head(P, w, 0.25), ref.numpy(), rtol=0, atol=1e-15)


# ------------------------------------------------ variants on the pages
def test_relu_activation_matches_library(O):
    """ReLU per-token FFN (the Appendix B Mixer's activation)."""
    B, T, D, Hd = 4, 4, 16, 32
    blk = synth.random_like_block(T, D, Hd, seed=71)
    S = synth.random_activations((B, T, D), seed=72).double()
    W1, b1, W2, b2 = (blk[k].double() for k in ("W1", "b1", "W2", "b2"))
    ref = torch.einsum("bth,tdh->btd", torch.relu(torch.einsum("btd,thd->bth", S, W1) + b1), W2) + b2
    np.testing.assert_allclose(O.pffn(S, blk["W1"], blk["b1"], blk["W2"], blk["b2"], gelu="relu"),
                               ref.numpy(), rtol=0, atol=1e-12)
    u = np.linspace(-3, 3, 13)
    np.testing.assert_array_equal(O.gelu(u, "relu"), np.maximum(u, 0))


def test_block_without_mix_addnorm(O):
    """S = TokenMixing(X) (no residual, no LayerNorm after the mix)."""
    B, T, dh, Hd = 5, 4, 6, 40
    D = T * dh
    blk = synth.random_like_block(T, D, Hd, seed=73)
    X = synth.random_activations((B, T, D), seed=74).double()
    S = X.view(B, T, T, dh).transpose(1, 2).reshape(B, T, D)
    W1, b1, W2, b2 = (blk[k].double() for k in ("W1", "b1", "W2", "b2"))
    V = torch.einsum("bth,tdh->btd", F.gelu(torch.einsum("btd,thd->bth", S, W1) + b1, approximate="tanh"), W2) + b2
    ref = F.layer_norm(V + S, (D,), blk["ln2_g"].double(), blk["ln2_b"].double(), eps=EPS)
    np.testing.assert_allclose(O.block(X, blk, EPS, mix_addnorm=False), ref.numpy(), rtol=0, atol=1e-12)
    # the variant differs from the equation on the pages
    assert np.abs(O.block(X, blk, EPS) - ref.numpy()).max() > 1e-3
