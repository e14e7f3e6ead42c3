"""Training step of dense bf16 stacks through the C ABI (rm_train_step),
against the fp64 training-step oracle (oracle/train_oracle.py): the loss, the
gradient of every block parameter, of the head and of the stack input.

Tolerance.  The forward keeps S, the FFN activation input and output and the
pre-LN rows in bf16, and the backward stores dY, dU, dS, dZ and dX in bf16:
about a dozen roundings of relative size 2^-9 lie on the path of each
gradient, each contributing about 2^-9 / sqrt(3) ~ 1.1e-3 relative L2, which
compound to roughly 4e-3 over a two-block stack.  The bound is 2e-2 relative
L2 per gradient tensor (five times that estimate, the same margin the forward
parity uses over its measured error), and the loss within 1e-2 relative.

ReLU is the exception: its derivative [U > 0] is a decision, and the kernel
takes it on its own U (bf16 storage of an fp32 sum over bf16 S) while the
oracle takes it on the fp64 U.  Where the two straddle zero the whole
entry of dU differs, so the relative L2 error of dU is about the square root
of the fraction of such entries: with |U - U_oracle| ~ 2e-3 and U ~ N(0, 0.8^2)
about 0.2 % of the entries flip, i.e. ~4e-2.  Every gradient downstream of
dU (dW1, db1, LN1's parameters, and everything of the earlier blocks and dX0)
is held to 1e-1 in the ReLU case; dW2, db2 and LN2's parameters of the last
block, which the mask does not reach, keep the 2e-2 bound.
"""
import numpy as np
import pytest
import torch

from gpu_common import dev, host64, rel_l2
from token_mixing_feature_b200 import synth

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 2e-2
KEYS = ("W1", "b1", "W2", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")


@pytest.fixture(scope="module")
def rm():
    from token_mixing_feature_b200 import rankmixer
    return rankmixer


def _case(B, T, D, hidden, L, act, seed):
    wl = synth.Workload("train", B=B, T=T, D=D, hidden=hidden, L=L, ln_params="perturbed", act=act)
    d = synth.make_inputs(wl, seed=seed)
    head = synth.make_head(wl, seed)
    head["b"] = torch.tensor([0.1])
    g = torch.Generator().manual_seed(seed + 17)
    labels = (torch.rand(B, generator=g) < 0.5).float()
    return wl, d, head, labels


def _run_gpu(rm, wl, d, head, labels):
    B, T, D, Hd, L = wl.B, wl.T, wl.D, wl.hidden, wl.L
    blocks = [{k: dev(v) for k, v in blk.items()} for blk in d["blocks"]]
    grads = [{"W1": torch.zeros(T, Hd, D, device="cuda"), "b1": torch.zeros(T, Hd, device="cuda"),
              "W2": torch.zeros(T, D, Hd, device="cuda"), "b2": torch.zeros(T, D, device="cuda"),
              **{k: torch.zeros(D, device="cuda") for k in ("ln1_g", "ln1_b", "ln2_g", "ln2_b")}}
             for _ in range(L)]
    out = {"dX0": torch.zeros(B, T, D, dtype=torch.bfloat16, device="cuda"),
           "dhead_w": torch.zeros(D, device="cuda"), "dhead_b": torch.zeros(1, device="cuda"),
           "loss": torch.zeros(1, device="cuda"), "pooled": torch.zeros(B, D, device="cuda")}
    with rm.rm_train_create(B, T, D, Hd, L, act=wl.act) as tr:
        rm.rm_train_step(tr, blocks, dev(d["X0"]), dev(head["w"]), dev(head["b"]), dev(labels), grads,
                         out["dX0"], out["dhead_w"], out["dhead_b"], out["loss"], out["pooled"], B)
        assert rm.rm_train_sync_status(tr) == rm.RM_OK
    return grads, out


def _check(got, ref, what, tol=GRAD_REL_L2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    r = rel_l2(got, ref)
    assert r <= tol, f"{what}: rel L2 {r:.3e} > {tol}"
    return r


@pytest.mark.parametrize("B,T,D,hidden,L,act", [
    (64, 4, 128, 256, 2, "tanh"),
    (96, 8, 256, 512, 2, "relu"),
    (40, 2, 64, 128, 1, "erf"),       # ragged M tiles (40 rows), K = B = 40 (a partial 64-row slab)
    (72, 16, 768, 3072, 1, "tanh"),   # the 100M-scale widths: several 256-column tiles, split-K tail
])
def test_train_step_matches_oracle(rm, B, T, D, hidden, L, act):
    from oracle import train_oracle as TO
    wl, d, head, labels = _case(B, T, D, hidden, L, act, seed=B + T)
    grads, out = _run_gpu(rm, wl, d, head, labels)
    ref = TO.train_step(d["X0"], d["blocks"], head["w"], head["b"], labels, gelu_mode=act)
    assert abs(float(out["loss"].item()) - ref["loss"]) <= 1e-2 * abs(ref["loss"])
    _check(host64(out["pooled"]), ref["pooled"], "pooled")
    _check(host64(out["dhead_w"]), ref["dhead_w"], "dhead_w")
    assert abs(float(out["dhead_b"].item()) - ref["dhead_b"]) <= 2e-2 * max(abs(ref["dhead_b"]), 1e-3)
    masked = 1e-1 if act == "relu" else GRAD_REL_L2     # gradients the ReLU mask reaches
    for l in range(L):
        for k in KEYS:
            untouched = l == L - 1 and k in ("W2", "b2", "ln2_g", "ln2_b")
            _check(host64(grads[l][k]), ref["blocks"][l][k], f"block {l} d{k}",
                   GRAD_REL_L2 if untouched else masked)
    _check(host64(out["dX0"]), ref["dX0"], "dX0", masked)


def test_train_step_is_deterministic(rm):
    wl, d, head, labels = _case(64, 4, 128, 256, 2, "tanh", seed=5)
    g1, o1 = _run_gpu(rm, wl, d, head, labels)
    g2, o2 = _run_gpu(rm, wl, d, head, labels)
    for l in range(wl.L):
        for k in KEYS:
            assert torch.equal(g1[l][k], g2[l][k]), (l, k)
    assert torch.equal(o1["dX0"], o2["dX0"])


def test_train_rejects_unsupported(rm):
    with pytest.raises(rm.RankMixerError) as e:
        rm.rm_train_create(64, 4, 96, 256, 1)          # D not a multiple of 64
    assert e.value.status == rm.RM_ERR_UNSUPPORTED
    with pytest.raises(rm.RankMixerError) as e:
        rm.rm_train_create(64, 16, 64, 256, 1)         # heads of width 4 (not whole 16-byte pieces)
    assert e.value.status == rm.RM_ERR_UNSUPPORTED
    wl, d, head, labels = _case(48, 4, 128, 256, 1, "tanh", seed=9)
    with rm.rm_train_create(48, 4, 128, 256, 1) as tr:
        grads = [{k: torch.zeros(1024, device="cuda") for k in KEYS}]
        z = torch.zeros(64, device="cuda")
        with pytest.raises(rm.RankMixerError) as e:     # batch not a multiple of 8
            rm.rm_train_step(tr, [{k: dev(v) for k, v in d["blocks"][0].items()}], dev(d["X0"]), dev(head["w"]),
                             dev(head["b"]), dev(labels), grads, None, z, z, z, None, 41)
        assert e.value.status == rm.RM_ERR_INVALID_ARG


# ------------------------------------------------------------- sparse MoE
# Gradients of the sparse-MoE step (fun-rec "Rankmixer: 硬件效率优化",
# section Sparse MoE扩展: ReLU routing, L = L_task + lambda L_reg, DTSI-MoE)
# against the oracle's train_step.  The router's mask [R > 0] is a decision
# like the ReLU activation's: where the kernel's fp32 logit from the bf16 S
# and the oracle's fp64 logit straddle zero, dR of that entry (dG, not small:
# the expert output e_j is not small) is present on one side only.  Block
# l's S deviates more from the oracle the later the block (it carries the
# earlier blocks' roundings), so with logits ~N(-0.05, 1.1^2) about 0.5 % of
# block 1's entries sit inside the band and the gradients the flips reach
# move by a few percent in relative L2 (measured up to 6 %).  So:
#   * routers with a fixed sign (|R| > 1, no entry near zero): every
#     gradient within GRAD_REL_L2 (2e-2), two blocks, with DTSI and L_reg;
#   * random routers: the last block's expert weights and biases (with ReLU
#     experts, W2 and b2 only: the activation's mask reaches W1 and b1), its
#     LN2 parameters and the head within 2e-2; everything a mask reaches
#     (router gradients, every gradient of earlier blocks, LN1 parameters,
#     dX0) within MASK_REL_L2 = 1e-1.
MASK_REL_L2 = 1e-1
MOE_KEYS = KEYS + ("Wr", "br")


def _moe_case(B, T, D, hidden, L, act, Ne, seed, dtsi, fixed_sign, rstd=0.1, rbias=-0.05):
    wl = synth.Workload("train_moe", B=B, T=T, D=D, hidden=hidden, L=L, ln_params="perturbed", act=act,
                        n_experts=Ne, router_std=rstd, router_bias=rbias)
    d = synth.make_inputs(wl, seed=seed)
    g = torch.Generator().manual_seed(seed + 31)
    sign = torch.tensor([2.0 if j % 2 == 0 else -2.0 for j in range(Ne)])
    for blk in d["blocks"]:
        if fixed_sign:   # |R| > 1 everywhere: experts 0, 2, ... always open, 1, 3, ... always closed
            blk["Wr"] = (torch.randn(T, Ne, D, generator=g) * 0.02).float()
            blk["br"] = sign.repeat(T, 1).float()
        if dtsi:
            blk["Wr_infer"] = (torch.randn(T, Ne, D, generator=g) * (0.02 if fixed_sign else rstd)).float()
            blk["br_infer"] = (sign.flip(0).repeat(T, 1) if fixed_sign
                               else torch.full((T, Ne), rbias)).float()
    head = synth.make_head(wl, seed)
    head["b"] = torch.tensor([0.1])
    labels = (torch.rand(B, generator=torch.Generator().manual_seed(seed + 17)) < 0.5).float()
    return wl, d, head, labels


def _run_gpu_moe(rm, wl, d, head, labels, lam):
    B, T, D, Hd, L, Ne = wl.B, wl.T, wl.D, wl.hidden, wl.L, wl.n_experts
    blocks = [{k: dev(v) for k, v in blk.items()} for blk in d["blocks"]]
    shapes = {"W1": (T, Ne, Hd, D), "b1": (T, Ne, Hd), "W2": (T, Ne, D, Hd), "b2": (T, Ne, D), "Wr": (T, Ne, D),
              "br": (T, Ne), "ln1_g": (D,), "ln1_b": (D,), "ln2_g": (D,), "ln2_b": (D,)}
    if "Wr_infer" in d["blocks"][0]:
        shapes.update({"Wr_infer": (T, Ne, D), "br_infer": (T, Ne)})
    # NaN-filled: every entry must be written
    grads = [{k: torch.full(sh, float("nan"), device="cuda") for k, sh in shapes.items()} for _ in range(L)]
    out = {"dX0": torch.zeros(B, T, D, dtype=torch.bfloat16, device="cuda"),
           "dhead_w": torch.zeros(D, device="cuda"), "dhead_b": torch.zeros(1, device="cuda"),
           "loss": torch.zeros(1, device="cuda"), "pooled": torch.zeros(B, D, device="cuda")}
    with rm.rm_train_create(B, T, D, Hd, L, act=wl.act, n_experts=Ne) as tr:
        rm.rm_train_set_reg(tr, lam)
        rm.rm_train_step(tr, blocks, dev(d["X0"]), dev(head["w"]), dev(head["b"]), dev(labels), grads,
                         out["dX0"], out["dhead_w"], out["dhead_b"], out["loss"], out["pooled"], B)
        assert rm.rm_train_sync_status(tr) == rm.RM_OK
    return grads, out


def _check_moe(grads, out, ref, L, tight, act):
    assert abs(float(out["loss"].item()) - ref["loss"]) <= 1e-2 * abs(ref["loss"])
    _check(host64(out["pooled"]), ref["pooled"], "pooled")
    _check(host64(out["dhead_w"]), ref["dhead_w"], "dhead_w")
    # the last block's expert weights and biases and LN2 parameters; with ReLU
    # experts the activation's own mask reaches W1 and b1 as in the dense case
    last = ("W2", "b2", "ln2_g", "ln2_b") + (() if act == "relu" else ("W1", "b1"))
    for l in range(L):
        for k, v in grads[l].items():
            unreached = l == L - 1 and k in last
            _check(host64(v), ref["blocks"][l][k], f"block {l} d{k}",
                   GRAD_REL_L2 if (tight or unreached) else MASK_REL_L2)
    _check(host64(out["dX0"]), ref["dX0"], "dX0", GRAD_REL_L2 if tight else MASK_REL_L2)


@pytest.mark.parametrize("B,T,D,hidden,L,act,Ne,dtsi,lam", [
    (64, 4, 128, 128, 2, "tanh", 4, True, 0.05),    # two blocks, DTSI, L_reg; half the experts never open
    (40, 2, 64, 128, 2, "erf", 2, False, 0.01),     # ragged batch (40), L_reg on the routing gates
])
def test_moe_train_step_fixed_sign_routers(rm, B, T, D, hidden, L, act, Ne, dtsi, lam):
    """No logit near zero: every gradient of a two-block sparse-MoE step within 2e-2."""
    from oracle import train_oracle as TO
    wl, d, head, labels = _moe_case(B, T, D, hidden, L, act, Ne, seed=B + Ne, dtsi=dtsi, fixed_sign=True)
    grads, out = _run_gpu_moe(rm, wl, d, head, labels, lam)
    ref = TO.train_step(d["X0"], d["blocks"], head["w"], head["b"], labels, gelu_mode=act, reg_lambda=lam)
    _check_moe(grads, out, ref, L, tight=True, act=act)


@pytest.mark.parametrize("B,T,D,hidden,L,act,Ne,dtsi,lam,rstd,rbias", [
    (64, 4, 128, 128, 2, "tanh", 4, False, 0.01, 0.1, -0.05),
    (40, 2, 64, 128, 1, "erf", 8, True, 0.05, 0.1, -0.05),
    (48, 8, 256, 64, 1, "tanh", 2, False, 0.0, 0.02, -0.5),     # the moe workload's router constants
    (96, 4, 128, 64, 2, "relu", 3, True, 0.02, 0.1, -0.05),     # ReLU experts: a second mask
])
def test_moe_train_step_matches_oracle(rm, B, T, D, hidden, L, act, Ne, dtsi, lam, rstd, rbias):
    from oracle import train_oracle as TO
    wl, d, head, labels = _moe_case(B, T, D, hidden, L, act, Ne, seed=B + T + Ne, dtsi=dtsi, fixed_sign=False,
                                    rstd=rstd, rbias=rbias)
    grads, out = _run_gpu_moe(rm, wl, d, head, labels, lam)
    ref = TO.train_step(d["X0"], d["blocks"], head["w"], head["b"], labels, gelu_mode=act, reg_lambda=lam)
    _check_moe(grads, out, ref, L, tight=False, act=act)


def test_moe_train_step_is_deterministic(rm):
    wl, d, head, labels = _moe_case(64, 4, 128, 128, 2, "tanh", 4, seed=11, dtsi=True, fixed_sign=False)
    g1, o1 = _run_gpu_moe(rm, wl, d, head, labels, 0.01)
    g2, o2 = _run_gpu_moe(rm, wl, d, head, labels, 0.01)
    for l in range(wl.L):
        for k in g1[l]:
            assert torch.equal(g1[l][k], g2[l][k]), (l, k)
    assert torch.equal(o1["dX0"], o2["dX0"]) and torch.equal(o1["loss"], o2["loss"])


def test_moe_train_rejects_unsupported(rm):
    with pytest.raises(rm.RankMixerError) as e:
        rm.rm_train_create(64, 4, 128, 128, 1, n_experts=33)
    assert e.value.status == rm.RM_ERR_UNSUPPORTED
    wl, d, head, labels = _moe_case(48, 4, 128, 128, 1, "tanh", 2, seed=9, dtsi=False, fixed_sign=False)
    with rm.rm_train_create(48, 4, 128, 128, 1, n_experts=2) as tr:
        with pytest.raises(rm.RankMixerError) as e:
            rm.rm_train_set_reg(tr, -1.0)
        assert e.value.status == rm.RM_ERR_INVALID_ARG
        g = {k: torch.zeros(1 << 16, device="cuda") for k in KEYS}   # no router gradient outputs
        z = torch.zeros(128, device="cuda")
        with pytest.raises(rm.RankMixerError) as e:
            rm.rm_train_step(tr, [{k: dev(v) for k, v in d["blocks"][0].items()}], dev(d["X0"]), dev(head["w"]),
                             dev(head["b"]), dev(labels), [g], None, z, z, z, None, 48)
        assert e.value.status == rm.RM_ERR_INVALID_ARG
