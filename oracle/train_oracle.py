"""fp64 CPU oracle of one training step of a RankMixer stack (dense or
sparse-MoE per-token FFN): forward, loss, and the gradient of the loss with
respect to every parameter and to the stack input.

TEST INFRASTRUCTURE.  Only the test suite may import this module.  It shares
no code with the CUDA library and never imports it.  Its forward restates the
block equations independently of the C oracle (rankmixer_oracle.c), and the
tests check that the two agree.

What it computes (the pages on RankMixer; primary source the fun-rec chapter
"Rankmixer: 硬件效率优化"):

  block l (section RankMixer整体架构):
      Z1 = TokenMixing(X) + X,      S  = LN1(Z1)
      U  = W1_t s_t + b1_t,  Hh = GELU(U),  V = W2_t Hh + b2_t   (section Per-Token FFN)
      Z2 = V + S,                   X' = LN2(Z2)
  pooling:   pooled_b = (1/T) sum_t X_L[b, t]
  head:      logit_b = w . pooled_b + c,  p_b = sigmoid(logit_b)
  loss:      L = (1/B) sum_b BCE(p_b, y_b) = (1/B) sum_b [softplus(logit_b) - y_b logit_b]
             + lambda L_reg
  sparse MoE in place of the PFFN (section Sparse MoE扩展, ReLU Routing and
  DTSI-MoE):
      G_{t,j} = ReLU(h_t(s_t))_j,  v_t = sum_j G_{t,j} e_{t,j}(s_t),  h_t linear
      L_reg   = sum over the batch's tokens and experts of the regularised gates:
                those of the routing router itself, or, with a second router
                h_infer (DTSI), G^infer = ReLU(h_infer(s_t)), which the forward
                computes beside the routing gates but does not use.

Readings where the pages leave a step open:
  - The task loss.  The pages name L_task without defining it (section Sparse
    MoE扩展 writes L = L_task + lambda L_reg).  The plainest reading for a
    ranking model with the sigmoid head of the Pad-Split serving stack is the
    mean binary cross-entropy against 0/1 labels, computed from the logit.
  - Token mixing with H = T is a permutation of the D T entries of a sample
    that is its own inverse (applying it twice is the identity), so its
    transpose, which carries the gradient back, is the mixing itself.
  - LayerNorm, GELU forms and weight layouts as in rankmixer_oracle.c: LN over
    D with the population variance and eps inside the square root, one
    (gamma, beta) per LN instance shared by all tokens; W1_t stored [kD][D],
    W2_t [D][kD]; MoE experts W1 [T][Ne][kD][D], W2 [T][Ne][D][kD], routers
    Wr [T][Ne][D], br [T][Ne] (h_infer: Wr_infer, br_infer, same shapes).
  - L_reg's gradient is the plain derivative of the written loss: it reaches
    the regularised router's parameters and, through the router's input,
    the tokens s_t.  Under DTSI as written, h_infer receives no other
    gradient (the task loss does not depend on it).

Each derivative below is the chain rule applied to these definitions, in
the order the forward computed them; the only library routines are array
products (numpy einsum / matmul) in float64.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)
GELU_C = 0.044715


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):      # torch tensors (bf16 widened exactly through float32)
        a = a.detach().to("cpu").float().numpy()
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------- pieces
def token_mix(X: np.ndarray) -> np.ndarray:
    """X [B, T, D] -> Y with Y[b, h, t*dh + j] = X[b, t, h*dh + j], dh = D / T."""
    B, T, D = X.shape
    dh = D // T
    # X[b, t, h, j] -> Y[b, h, t, j]
    return X.reshape(B, T, T, dh).transpose(0, 2, 1, 3).reshape(B, T, D)


def gelu(u: np.ndarray, mode: str) -> np.ndarray:
    if mode == "tanh":
        return 0.5 * u * (1.0 + np.tanh(SQRT_2_OVER_PI * (u + GELU_C * u ** 3)))
    if mode == "erf":
        from scipy.special import erf
        return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))
    if mode == "relu":
        return np.maximum(u, 0.0)
    raise ValueError(mode)


def gelu_grad(u: np.ndarray, mode: str) -> np.ndarray:
    """d GELU(u) / du."""
    if mode == "tanh":
        a = SQRT_2_OVER_PI * (u + GELU_C * u ** 3)
        th = np.tanh(a)
        return 0.5 * (1.0 + th) + 0.5 * u * (1.0 - th * th) * SQRT_2_OVER_PI * (1.0 + 3.0 * GELU_C * u * u)
    if mode == "erf":
        from scipy.special import erf
        return 0.5 * (1.0 + erf(u / math.sqrt(2.0))) + u * np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)
    if mode == "relu":
        return (u > 0.0).astype(np.float64)
    raise ValueError(mode)


def layernorm_fwd(Z: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float):
    """Row LayerNorm over the last axis; returns (out, xhat, rstd)."""
    mu = Z.mean(axis=-1, keepdims=True)
    var = ((Z - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (Z - mu) * rstd
    return xhat * g + b, xhat, rstd


def layernorm_bwd(dout: np.ndarray, xhat: np.ndarray, rstd: np.ndarray, g: np.ndarray):
    """Gradients of out = g * xhat + b, xhat = (z - mean) / sqrt(var + eps):
    returns (dZ, dg, db), dg and db summed over every row."""
    D = xhat.shape[-1]
    dxhat = dout * g
    dZ = rstd / D * (D * dxhat - dxhat.sum(axis=-1, keepdims=True)
                     - xhat * (dxhat * xhat).sum(axis=-1, keepdims=True))
    dg = (dout * xhat).reshape(-1, D).sum(axis=0)
    db = dout.reshape(-1, D).sum(axis=0)
    return dZ, dg, db


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 0.5 * (1.0 + np.tanh(0.5 * x))


# --------------------------------------------------------------- the step
PARAM_KEYS = ("W1", "b1", "W2", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b", "Wr", "br", "Wr_infer", "br_infer")


def _block_params(blk: Dict) -> Dict[str, np.ndarray]:
    return {k: _f64(blk[k]) for k in PARAM_KEYS if k in blk}


def _moe_forward(S: np.ndarray, p: Dict[str, np.ndarray], gelu_mode: str, c: Dict) -> np.ndarray:
    """v_t = sum_j ReLU(h_t(s_t))_j e_{t,j}(s_t) for every token; fills the cache."""
    c["R"] = np.einsum("btd,tjd->btj", S, p["Wr"]) + p["br"][None]
    c["G"] = np.maximum(c["R"], 0.0)
    c["U"] = np.einsum("btd,tjkd->btjk", S, p["W1"]) + p["b1"][None]
    c["Hh"] = gelu(c["U"], gelu_mode)
    c["E"] = np.einsum("btjk,tjdk->btjd", c["Hh"], p["W2"]) + p["b2"][None]
    if "Wr_infer" in p:
        c["R_inf"] = np.einsum("btd,tjd->btj", S, p["Wr_infer"]) + p["br_infer"][None]
    return np.einsum("btj,btjd->btd", c["G"], c["E"])


def _reg_gates(c: Dict) -> np.ndarray:
    """The gates L_reg sums: h_infer's under DTSI, else the routing gates."""
    return np.maximum(c["R_inf"], 0.0) if "R_inf" in c else c["G"]


def forward(X0, blocks: Sequence[Dict], head_w, head_b, eps: float = 1e-5, gelu_mode: str = "tanh",
            mix_addnorm: bool = True):
    """Forward pass with everything the backward needs.  Returns a dict with
    'pooled' [B, D], 'logit' [B], 'Xall' (X_1 .. X_L) and the per-block caches."""
    X = _f64(X0)
    caches = []
    Xall = []
    for blk in blocks:
        p = _block_params(blk)
        M = token_mix(X)
        if mix_addnorm:
            S, xh1, rs1 = layernorm_fwd(M + X, p["ln1_g"], p["ln1_b"], eps)
        else:
            S, xh1, rs1 = M, None, None
        c = {"p": p, "S": S, "xh1": xh1, "rs1": rs1}
        if "Wr" in p:
            V = _moe_forward(S, p, gelu_mode, c)
        else:
            c["U"] = np.einsum("btd,tkd->btk", S, p["W1"]) + p["b1"][None]
            c["Hh"] = gelu(c["U"], gelu_mode)
            V = np.einsum("btk,tdk->btd", c["Hh"], p["W2"]) + p["b2"][None]
        Xn, c["xh2"], c["rs2"] = layernorm_fwd(V + S, p["ln2_g"], p["ln2_b"], eps)
        caches.append(c)
        X = Xn
        Xall.append(X)
    pooled = X.mean(axis=1)
    logit = pooled @ _f64(head_w) + float(_f64(head_b).reshape(-1)[0])
    return {"pooled": pooled, "logit": logit, "Xall": Xall, "caches": caches}


def loss_from_logit(logit: np.ndarray, y: np.ndarray) -> float:
    """Mean binary cross-entropy of sigmoid(logit) against labels y."""
    return float(np.mean(_softplus(logit) - y * logit))


def train_step(X0, blocks: Sequence[Dict], head_w, head_b, labels, eps: float = 1e-5,
               gelu_mode: str = "tanh", mix_addnorm: bool = True, reg_lambda: float = 0.0):
    """Loss and gradients of one training step.

    Returns {'loss', 'pooled', 'logit', 'dX0' [B, T, D], 'dhead_w' [D],
    'dhead_b' (float), 'l_reg', 'blocks': [per block the gradients of every
    parameter the block has, same keys and shapes]}."""
    y = _f64(labels).reshape(-1)
    fw = forward(X0, blocks, head_w, head_b, eps, gelu_mode, mix_addnorm)
    pooled, logit = fw["pooled"], fw["logit"]
    B = pooled.shape[0]
    T = fw["caches"][0]["S"].shape[1]
    l_reg = sum(float(_reg_gates(c).sum()) for c in fw["caches"] if "G" in c)
    loss = loss_from_logit(logit, y) + reg_lambda * l_reg

    # head and pooling
    dlogit = (_sigmoid(logit) - y) / B                       # d mean(softplus(l) - y l) / dl
    dhead_w = pooled.T @ dlogit
    dhead_b = float(dlogit.sum())
    dpooled = dlogit[:, None] * _f64(head_w)[None, :]
    dX = np.repeat(dpooled[:, None, :] / T, T, axis=1)      # pooled = mean over t

    grads: List[Dict[str, np.ndarray]] = [None] * len(blocks)
    for l in range(len(blocks) - 1, -1, -1):
        c = fw["caches"][l]
        p = c["p"]
        g = {}
        # X' = LN2(V + S)
        dZ2, g["ln2_g"], g["ln2_b"] = layernorm_bwd(dX, c["xh2"], c["rs2"], p["ln2_g"])
        dV = dZ2
        dS = dZ2.copy()                                      # residual branch
        if "Wr" in p:
            dS += _moe_backward(dV, c, p, g, gelu_mode, reg_lambda)
        else:
            # V = W2_t Hh + b2_t
            g["W2"] = np.einsum("btd,btk->tdk", dV, c["Hh"])
            g["b2"] = dV.sum(axis=0)
            dHh = np.einsum("btd,tdk->btk", dV, p["W2"])
            # Hh = GELU(U), U = W1_t S + b1_t
            dU = dHh * gelu_grad(c["U"], gelu_mode)
            g["W1"] = np.einsum("btk,btd->tkd", dU, c["S"])
            g["b1"] = dU.sum(axis=0)
            dS += np.einsum("btk,tkd->btd", dU, p["W1"])
        # S = LN1(TokenMixing(X) + X)   (or S = TokenMixing(X))
        if mix_addnorm:
            dZ1, g["ln1_g"], g["ln1_b"] = layernorm_bwd(dS, c["xh1"], c["rs1"], p["ln1_g"])
            dX = dZ1 + token_mix(dZ1)                          # the mixing's transpose is itself
        else:
            g["ln1_g"] = np.zeros_like(p["ln1_g"])
            g["ln1_b"] = np.zeros_like(p["ln1_b"])
            dX = token_mix(dS)
        grads[l] = g
    return {"loss": loss, "l_reg": l_reg, "pooled": pooled, "logit": logit, "dX0": dX, "dhead_w": dhead_w,
            "dhead_b": dhead_b, "blocks": grads}


def _moe_backward(dV: np.ndarray, c: Dict, p: Dict[str, np.ndarray], g: Dict, gelu_mode: str,
                  reg_lambda: float) -> np.ndarray:
    """Gradients of the MoE FFN (into g) given dL/dV; returns dL/dS from the
    experts and the routers."""
    S = c["S"]
    # v = sum_j G_j e_j
    dG = np.einsum("btd,btjd->btj", dV, c["E"])
    dE = c["G"][..., None] * dV[:, :, None, :]
    # e_j = W2_{t,j} GELU(U_j) + b2_{t,j},  U_j = W1_{t,j} s + b1_{t,j}
    g["W2"] = np.einsum("btjd,btjk->tjdk", dE, c["Hh"])
    g["b2"] = dE.sum(axis=0)
    dU = np.einsum("btjd,tjdk->btjk", dE, p["W2"]) * gelu_grad(c["U"], gelu_mode)
    g["W1"] = np.einsum("btjk,btd->tjkd", dU, S)
    g["b1"] = dU.sum(axis=0)
    dS = np.einsum("btjk,tjkd->btd", dU, p["W1"])
    # G = ReLU(R), R = Wr s + br; L_reg on these gates unless a second router carries it
    active = (c["R"] > 0.0).astype(np.float64)
    dR = dG * active
    if "R_inf" not in c:
        dR = dR + reg_lambda * active
    g["Wr"] = np.einsum("btj,btd->tjd", dR, S)
    g["br"] = dR.sum(axis=0)
    dS += np.einsum("btj,tjd->btd", dR, p["Wr"])
    if "R_inf" in c:
        dR_inf = reg_lambda * (c["R_inf"] > 0.0).astype(np.float64)
        g["Wr_infer"] = np.einsum("btj,btd->tjd", dR_inf, S)
        g["br_infer"] = dR_inf.sum(axis=0)
        dS += np.einsum("btj,tjd->btd", dR_inf, p["Wr_infer"])
    return dS


def loss_only(X0, blocks: Sequence[Dict], head_w, head_b, labels, eps: float = 1e-5,
              gelu_mode: str = "tanh", mix_addnorm: bool = True, reg_lambda: float = 0.0) -> float:
    fw = forward(X0, blocks, head_w, head_b, eps, gelu_mode, mix_addnorm)
    l_reg = sum(float(_reg_gates(c).sum()) for c in fw["caches"] if "G" in c)
    return loss_from_logit(fw["logit"], _f64(labels).reshape(-1)) + reg_lambda * l_reg
