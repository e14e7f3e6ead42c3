"""Python front end of the fp64 CPU oracle for the RankMixer stack forward.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its binding) never imports it, and it never imports them.

The arithmetic lives in ``rankmixer_oracle.c`` (plain fp64 loops, OpenMP over
samples).  This module compiles it with gcc on first use, converts inputs to
contiguous float64/float32 numpy arrays and returns float64 results.
Definitions and readings are stated in the C file's header.
"""
from __future__ import annotations

import ctypes
import os
import pathlib
import subprocess
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = pathlib.Path(__file__).resolve().parent
_SRC = _HERE / "rankmixer_oracle.c"
_LIB_PATH = _HERE / "_build" / "liboracle.so"
_lib = None

GELU_MODES = {"tanh": 0, "erf": 1, "relu": 2}   # FFN activation: GELU forms or ReLU
MAX_EXPERTS = 64


class _BlockParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("W1", "b1", "W2", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b", "Wr", "br")]


def build(force: bool = False) -> pathlib.Path:
    """Compile the oracle into oracle/_build/liboracle.so (gcc, -O2, OpenMP)."""
    _LIB_PATH.parent.mkdir(exist_ok=True)
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-fopenmp", "-fPIC",
                               "-shared", "-o", str(tmp), str(_SRC), "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB_PATH))
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_gelu.restype = ctypes.c_double
        lib.orc_gelu.argtypes = [ctypes.c_double, ctypes.c_int]
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().orc_num_threads()


def set_threads(n: int) -> None:
    _load().orc_set_threads(ctypes.c_int(n))


def _np(x, dtype) -> np.ndarray:
    if hasattr(x, "detach"):          # torch tensor (any dtype, incl. bf16)
        x = x.detach().to("cpu")
        x = x.double().numpy() if dtype == np.float64 else x.float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _params(blk: Dict) -> (_BlockParams, List[np.ndarray]):
    keep = []
    vals = {}
    for n, _ in _BlockParams._fields_:
        if n in blk and blk[n] is not None:
            a = _np(blk[n], np.float32)
            keep.append(a)
            vals[n] = a.ctypes.data
        else:
            vals[n] = None
    return _BlockParams(**vals), keep


def gelu(u, mode: str = "tanh") -> np.ndarray:
    u = _np(u, np.float64)
    out = np.empty_like(u)
    _load().orc_gelu_array(ctypes.c_long(u.size), _p(u), ctypes.c_int(GELU_MODES[mode]), _p(out))
    return out


def token_mix(X) -> np.ndarray:
    """[B, T, D] -> [B, T, D]: output token h = concat_t chunk h of token t."""
    X = _np(X, np.float64)
    B, T, D = X.shape
    if D % T:
        raise ValueError("token mixing with H = T needs D divisible by T")
    Y = np.empty_like(X)
    _load().orc_token_mix(ctypes.c_long(B), ctypes.c_int(T), ctypes.c_int(D), _p(X), _p(Y))
    return Y


def layernorm(Z, gamma, beta, eps: float = 1e-5) -> np.ndarray:
    """Row-wise LayerNorm over the last axis."""
    Z = _np(Z, np.float64)
    D = Z.shape[-1]
    g, b = _np(gamma, np.float32), _np(beta, np.float32)
    out = np.empty_like(Z)
    _load().orc_layernorm(ctypes.c_long(Z.size // D), ctypes.c_int(D), _p(Z), _p(g), _p(b),
                          ctypes.c_double(eps), _p(out))
    return out


def pffn(S, W1, b1, W2, b2, gelu: str = "tanh") -> np.ndarray:
    """V[b, t] = W2_t GELU(W1_t S[b, t] + b1_t) + b2_t."""
    S = _np(S, np.float64)
    B, T, D = S.shape
    W1, b1, W2, b2 = (_np(a, np.float32) for a in (W1, b1, W2, b2))
    Hd = W1.shape[1]
    assert W1.shape == (T, Hd, D) and W2.shape == (T, D, Hd)
    V = np.empty_like(S)
    _load().orc_pffn(ctypes.c_long(B), ctypes.c_int(T), ctypes.c_int(D), ctypes.c_int(Hd), _p(S),
                     _p(W1), _p(b1), _p(W2), _p(b2), ctypes.c_int(GELU_MODES[gelu]), _p(V))
    return V


def moe(S, blk: Dict, gelu: str = "tanh"):
    """Sparse-MoE per-token FFN.  Returns (V [B,T,D], logits [B,T,Ne])."""
    S = _np(S, np.float64)
    B, T, D = S.shape
    T2, Ne, Hd, D2 = tuple(blk["W1"].shape)
    assert (T2, D2) == (T, D) and Ne <= MAX_EXPERTS
    prm, keep = _params(blk)
    V = np.empty_like(S)
    logits = np.empty((B, T, Ne), dtype=np.float64)
    _load().orc_moe(ctypes.c_long(B), ctypes.c_int(T), ctypes.c_int(D), ctypes.c_int(Hd),
                    ctypes.c_int(Ne), _p(S), ctypes.byref(prm), ctypes.c_int(GELU_MODES[gelu]),
                    _p(V), _p(logits))
    del keep
    return V, logits


def router(S, Wr, br) -> np.ndarray:
    """Router logits h_t(s) = Wr_t s + br_t of every token row, [B, T, Ne]
    (before the ReLU; an expert is active iff its logit is > 0)."""
    S = _np(S, np.float64)
    B, T, D = S.shape
    Wr, br = _np(Wr, np.float32), _np(br, np.float32)
    Ne = Wr.shape[1]
    assert Wr.shape == (T, Ne, D) and br.shape == (T, Ne)
    logits = np.empty((B, T, Ne), dtype=np.float64)
    _load().orc_router(ctypes.c_long(B), ctypes.c_int(T), ctypes.c_int(D), ctypes.c_int(Ne), _p(S), _p(Wr),
                       _p(br), _p(logits))
    return logits


def _dims(blk: Dict, T: int, D: int):
    W1 = blk["W1"]
    if len(W1.shape) == 3:
        return int(W1.shape[1]), 0
    return int(W1.shape[2]), int(W1.shape[1])


def block(X, blk: Dict, eps: float = 1e-5, gelu: str = "tanh", want_logits: bool = False,
          mix_addnorm: bool = True):
    """X' = LN2(PFFN(S) + S), S = LN1(TokenMixing(X) + X) (or S = TokenMixing(X)
    without the Add & Norm when mix_addnorm is False)."""
    X = _np(X, np.float64)
    B, T, D = X.shape
    Hd, Ne = _dims(blk, T, D)
    prm, keep = _params(blk)
    Y = np.empty_like(X)
    logits = np.empty((B, T, max(Ne, 1)), dtype=np.float64) if (Ne and want_logits) else None
    _load().orc_block(ctypes.c_long(B), ctypes.c_int(T), ctypes.c_int(D), ctypes.c_int(Hd),
                      ctypes.c_int(Ne), _p(X), ctypes.byref(prm), ctypes.c_double(eps),
                      ctypes.c_int(GELU_MODES[gelu]), ctypes.c_int(1 if mix_addnorm else 0), _p(Y), _p(logits))
    del keep
    return (Y, logits) if want_logits else Y


def stack(X0, blocks: Sequence[Dict], eps: float = 1e-5, gelu: str = "tanh",
          want_all: bool = False, want_last: bool = True, mix_addnorm: bool = True) -> Dict[str, np.ndarray]:
    """L blocks then mean pooling over tokens.  Returns pooled [B, D], and
    optionally Xlast [B, T, D] and Xall [L, B, T, D]."""
    X0 = _np(X0, np.float32)
    B, T, D = X0.shape
    L = len(blocks)
    Hd, Ne = _dims(blocks[0], T, D)
    arr = (_BlockParams * L)()
    keep = []
    for l, blk in enumerate(blocks):
        arr[l], k = _params(blk)
        keep += k
    pooled = np.empty((B, D), dtype=np.float64)
    Xlast = np.empty((B, T, D), dtype=np.float64) if want_last else None
    Xall = np.empty((L, B, T, D), dtype=np.float64) if want_all else None
    _load().orc_stack(ctypes.c_long(B), ctypes.c_int(T), ctypes.c_int(D), ctypes.c_int(Hd),
                      ctypes.c_int(Ne), ctypes.c_int(L), _p(X0), arr, ctypes.c_double(eps),
                      ctypes.c_int(GELU_MODES[gelu]), ctypes.c_int(1 if mix_addnorm else 0), _p(pooled), _p(Xlast),
                      _p(Xall))
    del keep
    out = {"pooled": pooled}
    if want_last:
        out["Xlast"] = Xlast
    if want_all:
        out["Xall"] = Xall
    return out


def padsplit(groups: Sequence, padded: int) -> np.ndarray:
    """Concatenate [B, w_i] groups and zero-pad to [B, padded]."""
    gs = [_np(g, np.float32) for g in groups]
    B = gs[0].shape[0]
    widths = np.array([g.shape[1] for g in gs], dtype=np.int32)
    if widths.sum() > padded:
        raise ValueError("groups wider than the padded width")
    ptrs = (ctypes.c_void_p * len(gs))(*[g.ctypes.data for g in gs])
    X0 = np.empty((B, padded), dtype=np.float64)
    _load().orc_padsplit(ctypes.c_long(B), ctypes.c_int(len(gs)), _p(widths), ptrs,
                         ctypes.c_int(padded), _p(X0))
    return X0


def head(pooled, w, bias: float) -> np.ndarray:
    """prob[b] = sigmoid(pooled[b] . w + bias)."""
    P = _np(pooled, np.float64)
    w = _np(w, np.float32)
    prob = np.empty(P.shape[0], dtype=np.float64)
    _load().orc_head(ctypes.c_long(P.shape[0]), ctypes.c_int(P.shape[1]), _p(P), _p(w),
                     ctypes.c_double(float(bias)), _p(prob))
    return prob
