"""fp64 CPU oracle of one training step of a dense RankMixer stack: forward,
loss, and the gradient of the loss with respect to every parameter and to
the stack input.

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
    W2_t [D][kD].

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
def _block_params(blk: Dict) -> Dict[str, np.ndarray]:
    return {k: _f64(blk[k]) for k in ("W1", "b1", "W2", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b")}


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
        U = np.einsum("btd,tkd->btk", S, p["W1"]) + p["b1"][None]
        Hh = gelu(U, gelu_mode)
        V = np.einsum("btk,tdk->btd", Hh, p["W2"]) + p["b2"][None]
        Xn, xh2, rs2 = layernorm_fwd(V + S, p["ln2_g"], p["ln2_b"], eps)
        caches.append({"p": p, "S": S, "U": U, "Hh": Hh, "xh1": xh1, "rs1": rs1, "xh2": xh2, "rs2": rs2})
        X = Xn
        Xall.append(X)
    pooled = X.mean(axis=1)
    logit = pooled @ _f64(head_w) + float(_f64(head_b).reshape(-1)[0])
    return {"pooled": pooled, "logit": logit, "Xall": Xall, "caches": caches}


def loss_from_logit(logit: np.ndarray, y: np.ndarray) -> float:
    """Mean binary cross-entropy of sigmoid(logit) against labels y."""
    return float(np.mean(_softplus(logit) - y * logit))


def train_step(X0, blocks: Sequence[Dict], head_w, head_b, labels, eps: float = 1e-5,
               gelu_mode: str = "tanh", mix_addnorm: bool = True):
    """Loss and gradients of one training step.

    Returns {'loss', 'pooled', 'logit', 'dX0' [B, T, D], 'dhead_w' [D],
    'dhead_b' (float), 'blocks': [per block {'W1', 'b1', 'W2', 'b2', 'ln1_g',
    'ln1_b', 'ln2_g', 'ln2_b'} gradients, same shapes as the parameters]}."""
    y = _f64(labels).reshape(-1)
    fw = forward(X0, blocks, head_w, head_b, eps, gelu_mode, mix_addnorm)
    pooled, logit = fw["pooled"], fw["logit"]
    B = pooled.shape[0]
    T = fw["caches"][0]["S"].shape[1]
    loss = loss_from_logit(logit, y)

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
    return {"loss": loss, "pooled": pooled, "logit": logit, "dX0": dX, "dhead_w": dhead_w,
            "dhead_b": dhead_b, "blocks": grads}


def loss_only(X0, blocks: Sequence[Dict], head_w, head_b, labels, eps: float = 1e-5,
              gelu_mode: str = "tanh", mix_addnorm: bool = True) -> float:
    fw = forward(X0, blocks, head_w, head_b, eps, gelu_mode, mix_addnorm)
    return loss_from_logit(fw["logit"], _f64(labels).reshape(-1))
