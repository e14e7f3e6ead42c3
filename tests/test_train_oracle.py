"""Pins of the training-step oracle (oracle/train_oracle.py) against what the
mathematics fixes, not against itself:

  - its forward equals the C oracle's stack forward (an independent
    restatement of the block equations, pinned in test_oracle_pins.py);
  - every gradient equals a central finite difference of the loss, and every
    entry equals torch autograd (float64, CPU) of a forward written here
    with torch ops;
  - LayerNorm input gradients sum to zero over a row (LayerNorm ignores a
    shift of its input row) and, with eps = 0, are orthogonal to the
    normalised input (it then also ignores a scaling);
  - the token mixing is its own adjoint (a permutation that is its own
    inverse), which is what carries the gradient back through it;
  - degenerate cases: W2 = 0 cuts every first-projection gradient to zero;
    the head-bias gradient is mean(sigmoid(logit) - y);
  - sparse MoE (ReLU routing, L_reg, DTSI's second router): its forward
    equals the C oracle's block, every gradient a finite difference, and
    h_infer's bias gradient is lambda times its count of positive logits.
"""
import numpy as np
import pytest

from oracle import train_oracle as TO
from token_mixing_feature_b200 import synth


def _stack(T, D, hidden, L, seed=0):
    blocks = []
    for l in range(L):
        blk = synth.random_like_block(T, D, hidden, "f32", seed=seed + 17 * l)
        # larger LayerNorm perturbations than the default, so their gradients are not near-degenerate
        rng = np.random.default_rng(seed + l)
        blk = {k: v.double().numpy() for k, v in blk.items()}
        for k in ("ln1_g", "ln2_g"):
            blk[k] = 1.0 + 0.3 * rng.standard_normal(D)
        for k in ("ln1_b", "ln2_b"):
            blk[k] = 0.3 * rng.standard_normal(D)
        blocks.append(blk)
    return blocks


def _inputs(B, T, D, seed=3):
    rng = np.random.default_rng(seed)
    X0 = rng.standard_normal((B, T, D))
    w = 0.5 * rng.standard_normal(D)
    c = np.array([0.1])
    y = (rng.random(B) < 0.4).astype(np.float64)
    return X0, w, c, y


def test_forward_matches_c_oracle(O):
    T, D, hidden, L, B = 4, 16, 24, 2, 5
    # the C oracle reads parameters and X0 as float: both get the same float values
    blocks = [{k: v.astype(np.float32).astype(np.float64) for k, v in b.items()} for b in _stack(T, D, hidden, L)]
    X0, w, c, _ = _inputs(B, T, D)
    fw = TO.forward(X0, blocks, w, c)
    ref = O.stack(X0.astype(np.float32), blocks, want_all=True)
    fw32 = TO.forward(X0.astype(np.float32), blocks, w, c)
    np.testing.assert_allclose(fw32["pooled"], ref["pooled"], rtol=0, atol=1e-12)
    for l in range(L):
        np.testing.assert_allclose(fw32["Xall"][l], ref["Xall"][l], rtol=0, atol=1e-12)
    assert fw["pooled"].shape == (B, D)


def _fd_check(fun_loss, params, grads, name, n_probe=6, h=1e-5, seed=0):
    rng = np.random.default_rng(seed)
    flat = params.reshape(-1)
    gflat = grads.reshape(-1)
    scale = max(1e-12, float(np.abs(gflat).max()))
    for i in rng.choice(flat.size, size=min(n_probe, flat.size), replace=False):
        old = flat[i]
        flat[i] = old + h
        lp = fun_loss()
        flat[i] = old - h
        lm = fun_loss()
        flat[i] = old
        fd = (lp - lm) / (2 * h)
        assert abs(fd - gflat[i]) <= 1e-6 * scale + 1e-9, f"{name}[{i}]: fd {fd:.10e} vs grad {gflat[i]:.10e}"


@pytest.mark.parametrize("act,addnorm", [("tanh", True), ("erf", True), ("relu", True), ("tanh", False)])
def test_gradients_match_finite_differences(act, addnorm):
    T, D, hidden, L, B = 4, 8, 12, 2, 3
    blocks = _stack(T, D, hidden, L, seed=11)
    X0, w, c, y = _inputs(B, T, D, seed=5)

    def loss():
        return TO.loss_only(X0, blocks, w, c, y, gelu_mode=act, mix_addnorm=addnorm)

    st = TO.train_step(X0, blocks, w, c, y, gelu_mode=act, mix_addnorm=addnorm)
    assert abs(st["loss"] - loss()) < 1e-14
    _fd_check(loss, X0, st["dX0"], "X0")
    _fd_check(loss, w, st["dhead_w"], "head_w")
    _fd_check(loss, c, np.array([st["dhead_b"]]), "head_b")
    for l in range(L):
        keys = ("W1", "b1", "W2", "b2", "ln2_g", "ln2_b") + (("ln1_g", "ln1_b") if addnorm else ())
        for k in keys:
            _fd_check(loss, blocks[l][k], st["blocks"][l][k], f"block{l}.{k}", seed=l)


def test_layernorm_input_gradient_is_orthogonal_to_shift_and_scale():
    """A LayerNorm row is unchanged when a constant is added to its input, so
    the input gradient sums to zero; with eps = 0 it is also unchanged when the
    input is scaled, so the gradient is orthogonal to the normalised input
    (with eps > 0 that holds only up to eps / var)."""
    rng = np.random.default_rng(7)
    Z = rng.standard_normal((6, 5, 24)) * 3.0 + 1.5
    g = 1.0 + 0.5 * rng.standard_normal(24)
    b = rng.standard_normal(24)
    dout = rng.standard_normal(Z.shape)
    for eps in (1e-5, 0.0):
        _, xhat, rstd = TO.layernorm_fwd(Z, g, b, eps)
        dZ, _, _ = TO.layernorm_bwd(dout, xhat, rstd, g)
        np.testing.assert_allclose(dZ.sum(axis=-1), 0.0, atol=1e-12)
        if eps == 0.0:
            np.testing.assert_allclose((dZ * xhat).sum(axis=-1), 0.0, atol=1e-11)


def test_token_mix_is_its_own_adjoint():
    rng = np.random.default_rng(9)
    for T, D in ((4, 16), (8, 40), (1, 8)):
        x = rng.standard_normal((3, T, D))
        yv = rng.standard_normal((3, T, D))
        assert abs(np.sum(TO.token_mix(x) * yv) - np.sum(x * TO.token_mix(yv))) < 1e-10
        np.testing.assert_array_equal(TO.token_mix(TO.token_mix(x)), x)


def test_zero_second_projection_cuts_first_projection_gradients():
    T, D, hidden, L, B = 4, 8, 12, 1, 4
    blocks = _stack(T, D, hidden, L, seed=21)
    blocks[0]["W2"][:] = 0.0
    X0, w, c, y = _inputs(B, T, D, seed=8)
    st = TO.train_step(X0, blocks, w, c, y)
    assert np.all(st["blocks"][0]["W1"] == 0.0) and np.all(st["blocks"][0]["b1"] == 0.0)
    assert np.abs(st["blocks"][0]["W2"]).max() > 0.0


def test_head_bias_gradient_closed_form():
    T, D, hidden, L, B = 4, 8, 12, 2, 7
    blocks = _stack(T, D, hidden, L, seed=31)
    X0, w, c, y = _inputs(B, T, D, seed=4)
    st = TO.train_step(X0, blocks, w, c, y)
    p = 1.0 / (1.0 + np.exp(-st["logit"]))
    assert abs(st["dhead_b"] - float(np.mean(p - y))) < 1e-15


def _moe_stack(T, D, hidden, Ne, L, seed=0, dtsi=False):
    blocks = []
    for l in range(L):
        blk = synth.random_like_block(T, D, hidden, "f32", seed=seed + 13 * l, n_experts=Ne,
                                      router_std=0.4, router_bias=0.0)
        rng = np.random.default_rng(seed + 100 + l)
        blk = {k: v.double().numpy() for k, v in blk.items()}
        for k in ("ln1_g", "ln2_g"):
            blk[k] = 1.0 + 0.3 * rng.standard_normal(D)
        for k in ("ln1_b", "ln2_b"):
            blk[k] = 0.3 * rng.standard_normal(D)
        if dtsi:
            blk["Wr_infer"] = 0.4 * rng.standard_normal((T, Ne, D))
            blk["br_infer"] = 0.1 * rng.standard_normal((T, Ne))
        blocks.append({k: v.astype(np.float32).astype(np.float64) for k, v in blk.items()})
    return blocks


def test_moe_forward_matches_c_oracle(O):
    T, D, hidden, Ne, B = 4, 16, 12, 3, 5
    blocks = _moe_stack(T, D, hidden, Ne, 1, seed=2)
    X0, w, c, _ = _inputs(B, T, D)
    X0 = X0.astype(np.float32).astype(np.float64)
    fw = TO.forward(X0, blocks, w, c)
    ref = O.block(X0, blocks[0])
    np.testing.assert_allclose(fw["Xall"][0], ref, rtol=0, atol=1e-12)
    G = fw["caches"][0]["G"]
    assert 0 < np.count_nonzero(G) < G.size     # some experts open, some closed


@pytest.mark.parametrize("dtsi", [False, True])
def test_moe_gradients_match_finite_differences(dtsi):
    T, D, hidden, Ne, L, B = 4, 8, 6, 3, 2, 3
    lam = 0.05
    blocks = _moe_stack(T, D, hidden, Ne, L, seed=5, dtsi=dtsi)
    X0, w, c, y = _inputs(B, T, D, seed=6)

    def loss():
        return TO.loss_only(X0, blocks, w, c, y, reg_lambda=lam)

    st = TO.train_step(X0, blocks, w, c, y, reg_lambda=lam)
    assert abs(st["loss"] - loss()) < 1e-14 and st["l_reg"] > 0.0
    _fd_check(loss, X0, st["dX0"], "X0")
    for l in range(L):
        keys = ["W1", "b1", "W2", "b2", "Wr", "br", "ln1_g", "ln1_b", "ln2_g", "ln2_b"]
        if dtsi:
            keys += ["Wr_infer", "br_infer"]
        for k in keys:
            _fd_check(loss, blocks[l][k], st["blocks"][l][k], f"block{l}.{k}", seed=l)


def test_dtsi_inference_router_gradient_is_the_regulariser_count():
    """Under DTSI the task loss does not depend on h_infer, so its bias
    gradient is lambda times the number of the batch's positive h_infer
    logits for that (token, expert), and zero without the regulariser."""
    T, D, hidden, Ne, B = 4, 8, 6, 3, 9
    blocks = _moe_stack(T, D, hidden, Ne, 1, seed=8, dtsi=True)
    X0, w, c, y = _inputs(B, T, D, seed=9)
    for lam in (0.0, 0.25):
        st = TO.train_step(X0, blocks, w, c, y, reg_lambda=lam)
        R_inf = TO.forward(X0, blocks, w, c)["caches"][0]["R_inf"]
        np.testing.assert_array_equal(st["blocks"][0]["br_infer"], lam * (R_inf > 0).sum(axis=0))
        if lam == 0.0:
            assert not np.any(st["blocks"][0]["Wr_infer"])


def _torch_loss(X0, blocks, w, c, y, act, addnorm, lam, eps=1e-5):
    """The stack's loss written with torch ops in float64, for autograd."""
    import torch
    import torch.nn.functional as F

    def mix(X):
        B, T, D = X.shape
        return X.reshape(B, T, T, D // T).transpose(1, 2).reshape(B, T, D)

    def ln(Z, g, b):
        mu = Z.mean(-1, keepdim=True)
        var = ((Z - mu) ** 2).mean(-1, keepdim=True)
        return (Z - mu) / torch.sqrt(var + eps) * g + b

    def act_fn(u):
        if act == "tanh":
            return F.gelu(u, approximate="tanh")
        if act == "erf":
            return F.gelu(u)
        return torch.relu(u)

    X = X0
    l_reg = X0.new_zeros(())
    for p in blocks:
        S = ln(mix(X) + X, p["ln1_g"], p["ln1_b"]) if addnorm else mix(X)
        if "Wr" in p:
            G = torch.relu(torch.einsum("btd,tjd->btj", S, p["Wr"]) + p["br"])
            E = torch.einsum("btjk,tjdk->btjd", act_fn(torch.einsum("btd,tjkd->btjk", S, p["W1"]) + p["b1"]),
                             p["W2"]) + p["b2"]
            V = torch.einsum("btj,btjd->btd", G, E)
            if "Wr_infer" in p:
                l_reg = l_reg + torch.relu(torch.einsum("btd,tjd->btj", S, p["Wr_infer"]) + p["br_infer"]).sum()
            else:
                l_reg = l_reg + G.sum()
        else:
            H = act_fn(torch.einsum("btd,tkd->btk", S, p["W1"]) + p["b1"])
            V = torch.einsum("btk,tdk->btd", H, p["W2"]) + p["b2"]
        X = ln(V + S, p["ln2_g"], p["ln2_b"])
    logit = X.mean(1) @ w + c[0]
    return F.binary_cross_entropy_with_logits(logit, y) + lam * l_reg


@pytest.mark.parametrize("kind,act,addnorm", [("dense", "tanh", True), ("dense", "erf", False),
                                              ("dense", "relu", True), ("moe", "tanh", True),
                                              ("dtsi", "tanh", True)])
def test_gradients_match_autograd(kind, act, addnorm):
    """Every entry of every gradient against torch autograd (float64, CPU) of
    a forward written separately with torch ops."""
    import torch
    T, D, hidden, L, B = 4, 8, 6, 2, 5
    lam = 0.05 if kind != "dense" else 0.0
    if kind == "dense":
        blocks = _stack(T, D, hidden, L, seed=41)
    else:
        blocks = _moe_stack(T, D, hidden, 3, L, seed=43, dtsi=kind == "dtsi")
    X0, w, c, y = _inputs(B, T, D, seed=44)
    st = TO.train_step(X0, blocks, w, c, y, gelu_mode=act, mix_addnorm=addnorm, reg_lambda=lam)
    tt = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)   # noqa: E731
    tb = [{k: tt(v) for k, v in b.items()} for b in blocks]
    tX, tw, tc = tt(X0), tt(w), tt(c)
    loss = _torch_loss(tX, tb, tw, tc, torch.tensor(y, dtype=torch.float64), act, addnorm, lam)
    loss.backward()
    assert abs(loss.item() - st["loss"]) < 1e-12
    np.testing.assert_allclose(st["dX0"], tX.grad.numpy(), rtol=1e-9, atol=1e-13)
    np.testing.assert_allclose(st["dhead_w"], tw.grad.numpy(), rtol=1e-9, atol=1e-13)
    assert abs(st["dhead_b"] - tc.grad.item()) < 1e-12
    for l in range(L):
        for k, v in tb[l].items():
            if not addnorm and k in ("ln1_g", "ln1_b"):
                continue   # unused without the Add & Norm (the oracle reports zeros)
            np.testing.assert_allclose(st["blocks"][l][k], v.grad.numpy(), rtol=1e-9, atol=1e-13,
                                       err_msg=f"block{l}.{k}")
