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
