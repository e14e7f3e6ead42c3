"""ctypes binding of librankmixer.so (declared in include/rankmixer.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
library.  Functions keep the C names; tensors are passed as device pointers
(``tensor.data_ptr()``), streams default to torch's current stream.  If the
library is not built, importing this module raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import pathlib
from typing import Dict, List, Optional, Sequence

_LIB_PATH = pathlib.Path(__file__).resolve().with_name("librankmixer.so")

RM_OK, RM_ERR_INVALID_ARG, RM_ERR_UNSUPPORTED, RM_ERR_CUDA, RM_ERR_OOM, \
    RM_ERR_DEVICE_TIMEOUT, RM_ERR_DEVICE_BOUNDS = range(7)
RM_F32, RM_BF16 = 0, 1
RM_ACT_GELU_TANH, RM_ACT_GELU_ERF, RM_ACT_RELU = 0, 1, 2
DTYPES = {"f32": RM_F32, "bf16": RM_BF16}
ACTS = {"tanh": RM_ACT_GELU_TANH, "erf": RM_ACT_GELU_ERF, "relu": RM_ACT_RELU}

EXPORTED = (
    "rm_create", "rm_destroy", "rm_workspace_bytes", "rm_token_mix", "rm_layernorm",
    "rm_pffn_forward", "rm_moe_forward", "rm_block_forward", "rm_stack_forward",
    "rm_stack_forward_host", "rm_padsplit_tokenize", "rm_head_forward", "rm_sync_status",
    "rm_last_error_site", "rm_set_wait_budget", "rm_selftest_wait_timeout", "rm_status_string",
    "rm_profile_begin", "rm_profile_end", "rm_kernel_name", "rm_pffn_forward_static",
    "rm_stack_forward_host_async", "rm_host_wait",
    "rm_train_create", "rm_train_destroy", "rm_train_workspace_bytes", "rm_train_step", "rm_train_sync_status",
    "rm_train_set_reg", "rm_tokshard_pack", "rm_tokshard_mix_ln", "rm_tokshard_pool",
    "rm_quantize_fp8", "rm_stack_forward_fp8",
)
RM_STATIC_SCRATCH_BYTES = 16 << 20
RM_K_COUNT = 11


class rm_config(ctypes.Structure):
    _fields_ = [("B_max", ctypes.c_int), ("T", ctypes.c_int), ("D", ctypes.c_int),
                ("hidden", ctypes.c_int), ("L", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("dtype", ctypes.c_int), ("ln_eps", ctypes.c_float), ("act", ctypes.c_int),
                ("mix_addnorm", ctypes.c_int)]


class rm_block_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("W1", "b1", "W2", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b", "Wr", "br", "Wr_infer", "br_infer")]


class rm_fp8_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W1q", "W2q", "W1s", "W2s")]


class rm_block_grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W1", "b1", "W2", "b2", "ln1_g", "ln1_b", "ln2_g", "ln2_b",
                                                "Wr", "br", "Wr_infer", "br_infer")]


class RankMixerError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not _LIB_PATH.exists():
        raise RuntimeError(f"{_LIB_PATH.name} is not built; run `python -m token_mixing_feature_b200.build`")
    lib = ctypes.CDLL(str(_LIB_PATH))
    vp, ci, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    sig = {
        "rm_create": (st, [ctypes.POINTER(rm_config), ctypes.POINTER(vp)]),
        "rm_destroy": (st, [vp]),
        "rm_workspace_bytes": (ctypes.c_size_t, [vp]),
        "rm_token_mix": (st, [vp, vp, vp, ci, vp]),
        "rm_layernorm": (st, [vp, vp, vp, vp, vp, vp, ci, vp]),
        "rm_pffn_forward": (st, [vp, ctypes.POINTER(rm_block_weights), vp, vp, ci, vp]),
        "rm_moe_forward": (st, [vp, ctypes.POINTER(rm_block_weights), vp, vp, vp, ci, vp]),
        "rm_block_forward": (st, [vp, ctypes.POINTER(rm_block_weights), vp, vp, ci, vp]),
        "rm_stack_forward": (st, [vp, ctypes.POINTER(rm_block_weights), vp, vp, vp, ci, vp]),
        "rm_stack_forward_host": (st, [vp, ctypes.POINTER(rm_block_weights), vp, vp, ci, vp]),
        "rm_stack_forward_host_async": (st, [vp, ctypes.POINTER(rm_block_weights), vp, vp, ci, vp]),
        "rm_host_wait": (st, [vp]),
        "rm_padsplit_tokenize": (st, [vp, ctypes.POINTER(vp), ctypes.POINTER(ci), ci, vp, ci, vp]),
        "rm_head_forward": (st, [vp, vp, vp, vp, vp, ci, vp]),
        "rm_sync_status": (st, [vp, vp]),
        "rm_last_error_site": (ci, [vp]),
        "rm_set_wait_budget": (st, [vp, ctypes.c_ulonglong]),
        "rm_selftest_wait_timeout": (st, [vp, vp]),
        "rm_status_string": (ctypes.c_char_p, [st]),
        "rm_profile_begin": (st, [vp, ci]),
        "rm_profile_end": (st, [vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ci), ci]),
        "rm_kernel_name": (ctypes.c_char_p, [ci]),
        "rm_pffn_forward_static": (st, [ctypes.POINTER(rm_block_weights), vp, vp, ci, ci, ci, ci, ci, ci,
                                        vp, vp]),
        "rm_train_create": (st, [ctypes.POINTER(rm_config), ctypes.POINTER(vp)]),
        "rm_train_destroy": (st, [vp]),
        "rm_train_workspace_bytes": (ctypes.c_size_t, [vp]),
        "rm_train_step": (st, [vp, ctypes.POINTER(rm_block_weights), vp, vp, vp, vp, ctypes.POINTER(rm_block_grads),
                               vp, vp, vp, vp, vp, ci, vp]),
        "rm_train_sync_status": (st, [vp, vp]),
        "rm_train_set_reg": (st, [vp, ctypes.c_float]),
        "rm_tokshard_pack": (st, [vp, vp, vp, vp, vp, vp, vp, ci, ci, vp]),
        "rm_tokshard_mix_ln": (st, [vp, vp, vp, vp, vp, vp, ci, ci, vp]),
        "rm_tokshard_pool": (st, [vp, vp, vp, vp, vp, vp, ci, vp]),
        "rm_quantize_fp8": (st, [vp, vp, vp, ctypes.c_longlong, ci, vp]),
        "rm_stack_forward_fp8": (st, [vp, ctypes.POINTER(rm_block_weights), ctypes.POINTER(rm_fp8_weights), vp, vp,
                                      ci, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = _load()


def library_path() -> str:
    return str(_LIB_PATH)


def status_string(s: int) -> str:
    return _lib.rm_status_string(s).decode()


def _check(s: int, what: str) -> None:
    if s != RM_OK:
        raise RankMixerError(s, what)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def block_weights(blk: Dict) -> rm_block_weights:
    """rm_block_weights from a dict of device tensors (missing keys -> NULL)."""
    return rm_block_weights(**{n: _ptr(blk.get(n)) for n, _ in rm_block_weights._fields_})


class Handle:
    """Owns one rm_handle.  Call close() (or use as a context manager)."""

    def __init__(self, ptr: int, cfg: rm_config):
        self.ptr = ptr
        self.cfg = cfg

    def close(self) -> None:
        if self.ptr:
            p, self.ptr = self.ptr, None
            _check(_lib.rm_destroy(p), "rm_destroy")

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rm_create(B_max: int, T: int, D: int, hidden: int, L: int = 1, n_experts: int = 0,
              dtype: str = "bf16", ln_eps: float = 1e-5, act: str = "tanh", mix_addnorm: bool = True) -> Handle:
    """act: "tanh" / "erf" (GELU forms) or "relu"."""
    cfg = rm_config(B_max, T, D, hidden, L, n_experts, DTYPES[dtype], ln_eps, ACTS[act], 1 if mix_addnorm else 0)
    out = ctypes.c_void_p()
    _check(_lib.rm_create(ctypes.byref(cfg), ctypes.byref(out)), "rm_create")
    return Handle(out.value, cfg)


def rm_destroy(h: Handle) -> None:
    h.close()


def rm_workspace_bytes(h: Handle) -> int:
    return _lib.rm_workspace_bytes(h.ptr)


def rm_token_mix(h: Handle, X, Y, B: int, stream=None) -> None:
    _check(_lib.rm_token_mix(h.ptr, _ptr(X), _ptr(Y), B, _stream(stream)), "rm_token_mix")


def rm_layernorm(h: Handle, A, R, gamma, beta, out, rows: int, stream=None) -> None:
    _check(_lib.rm_layernorm(h.ptr, _ptr(A), _ptr(R), _ptr(gamma), _ptr(beta), _ptr(out), rows,
                             _stream(stream)), "rm_layernorm")


def rm_pffn_forward(h: Handle, w: Dict, S, V, B: int, stream=None) -> None:
    bw = block_weights(w)
    _check(_lib.rm_pffn_forward(h.ptr, ctypes.byref(bw), _ptr(S), _ptr(V), B, _stream(stream)),
           "rm_pffn_forward")


def rm_moe_forward(h: Handle, w: Dict, S, V, gates, B: int, stream=None) -> None:
    bw = block_weights(w)
    _check(_lib.rm_moe_forward(h.ptr, ctypes.byref(bw), _ptr(S), _ptr(V), _ptr(gates), B,
                               _stream(stream)), "rm_moe_forward")


def rm_block_forward(h: Handle, w: Dict, X, Xout, B: int, stream=None) -> None:
    bw = block_weights(w)
    _check(_lib.rm_block_forward(h.ptr, ctypes.byref(bw), _ptr(X), _ptr(Xout), B, _stream(stream)),
           "rm_block_forward")


def _block_array(blocks: Sequence[Dict]):
    arr = (rm_block_weights * len(blocks))()
    for i, b in enumerate(blocks):
        arr[i] = block_weights(b)
    return arr


def rm_stack_forward(h: Handle, blocks: Sequence[Dict], X0, pooled, Xlast, B: int, stream=None) -> None:
    arr = _block_array(blocks)
    _check(_lib.rm_stack_forward(h.ptr, arr, _ptr(X0), _ptr(pooled), _ptr(Xlast), B, _stream(stream)),
           "rm_stack_forward")


def rm_stack_forward_host(h: Handle, blocks: Sequence[Dict], X0_host, pooled_host, B: int,
                          stream=None) -> None:
    """X0_host / pooled_host: CPU tensors (pinned for full copy speed)."""
    arr = _block_array(blocks)
    _check(_lib.rm_stack_forward_host(h.ptr, arr, _ptr(X0_host), _ptr(pooled_host), B,
                                      _stream(stream)), "rm_stack_forward_host")


def rm_stack_forward_host_async(h: Handle, blocks: Sequence[Dict], X0_host, pooled_host, B: int,
                                stream=None) -> None:
    """Enqueue one host-buffer stack call; results valid after rm_host_wait."""
    arr = _block_array(blocks)
    _check(_lib.rm_stack_forward_host_async(h.ptr, arr, _ptr(X0_host), _ptr(pooled_host), B,
                                            _stream(stream)), "rm_stack_forward_host_async")


def rm_host_wait(h: Handle) -> None:
    _check(_lib.rm_host_wait(h.ptr), "rm_host_wait")


def rm_padsplit_tokenize(h: Handle, groups: Sequence, X0, B: int, stream=None) -> None:
    ptrs = (ctypes.c_void_p * len(groups))(*[_ptr(g) for g in groups])
    widths = (ctypes.c_int * len(groups))(*[int(g.shape[1]) for g in groups])
    _check(_lib.rm_padsplit_tokenize(h.ptr, ptrs, widths, len(groups), _ptr(X0), B, _stream(stream)),
           "rm_padsplit_tokenize")


def rm_head_forward(h: Handle, w, bias, pooled, prob, B: int, stream=None) -> None:
    _check(_lib.rm_head_forward(h.ptr, _ptr(w), _ptr(bias), _ptr(pooled), _ptr(prob), B,
                                _stream(stream)), "rm_head_forward")


def rm_sync_status(h: Handle, stream=None) -> int:
    """Synchronise and return (and clear) the device error status."""
    return _lib.rm_sync_status(h.ptr, _stream(stream))


def rm_last_error_site(h: Handle) -> int:
    return _lib.rm_last_error_site(h.ptr)


def rm_set_wait_budget(h: Handle, ns: int) -> None:
    _check(_lib.rm_set_wait_budget(h.ptr, ns), "rm_set_wait_budget")


def rm_selftest_wait_timeout(h: Handle, stream=None) -> None:
    _check(_lib.rm_selftest_wait_timeout(h.ptr, _stream(stream)), "rm_selftest_wait_timeout")


def rm_status_string(s: int) -> str:
    return status_string(s)


def rm_profile_begin(h: Handle, max_launches: int) -> None:
    _check(_lib.rm_profile_begin(h.ptr, max_launches), "rm_profile_begin")


def rm_profile_end(h: Handle) -> Dict[str, tuple]:
    """{kernel name: (summed ms, launches)} of the recorded launches."""
    ms = (ctypes.c_float * RM_K_COUNT)()
    n = (ctypes.c_int * RM_K_COUNT)()
    _check(_lib.rm_profile_end(h.ptr, ms, n, RM_K_COUNT), "rm_profile_end")
    return {rm_kernel_name(k): (float(ms[k]), int(n[k])) for k in range(RM_K_COUNT) if n[k]}


def rm_kernel_name(kind: int) -> str:
    return _lib.rm_kernel_name(kind).decode()


def rm_pffn_forward_static(w: Dict, S, V, B: int, T: int, D: int, hidden: int, dtype: str = "bf16",
                           act: str = "tanh", device_status=None, stream=None) -> None:
    """V = PFFN(S) with no handle and no device allocation: the hidden
    activations use a fixed array inside the library (RM_STATIC_SCRATCH_BYTES),
    shared by all calls; overlapping calls race on it."""
    bw = block_weights(w)
    _check(_lib.rm_pffn_forward_static(ctypes.byref(bw), _ptr(S), _ptr(V), B, T, D, hidden, DTYPES[dtype],
                                       ACTS[act], _ptr(device_status), _stream(stream)),
           "rm_pffn_forward_static")


# ------------------------------------------------------------- training step
class Trainer:
    """Owns one rm_trainer.  Call close() (or use as a context manager)."""

    def __init__(self, ptr: int, cfg: rm_config):
        self.ptr = ptr
        self.cfg = cfg

    def close(self) -> None:
        if self.ptr:
            p, self.ptr = self.ptr, None
            _check(_lib.rm_train_destroy(p), "rm_train_destroy")

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rm_train_create(B_max: int, T: int, D: int, hidden: int, L: int, ln_eps: float = 1e-5,
                    act: str = "tanh", n_experts: int = 0) -> Trainer:
    cfg = rm_config(B_max, T, D, hidden, L, n_experts, RM_BF16, ln_eps, ACTS[act], 1)
    out = ctypes.c_void_p()
    _check(_lib.rm_train_create(ctypes.byref(cfg), ctypes.byref(out)), "rm_train_create")
    return Trainer(out.value, cfg)


def rm_train_destroy(t: Trainer) -> None:
    t.close()


def rm_train_set_reg(t: Trainer, reg_lambda: float) -> None:
    _check(_lib.rm_train_set_reg(t.ptr, float(reg_lambda)), "rm_train_set_reg")


def rm_train_workspace_bytes(t: Trainer) -> int:
    return _lib.rm_train_workspace_bytes(t.ptr)


def block_grads(g: Dict) -> rm_block_grads:
    return rm_block_grads(**{n: _ptr(g.get(n)) for n, _ in rm_block_grads._fields_})


def rm_train_step(t: Trainer, blocks: Sequence[Dict], X0, head_w, head_b, labels, grads: Sequence[Dict], dX0,
                  dhead_w, dhead_b, loss, pooled, B: int, stream=None) -> None:
    """grads: one dict of float device tensors per block (keys of rm_block_grads)."""
    arr = _block_array(blocks)
    garr = (rm_block_grads * len(grads))()
    for i, g in enumerate(grads):
        garr[i] = block_grads(g)
    _check(_lib.rm_train_step(t.ptr, arr, _ptr(X0), _ptr(head_w), _ptr(head_b), _ptr(labels), garr, _ptr(dX0),
                              _ptr(dhead_w), _ptr(dhead_b), _ptr(loss), _ptr(pooled), B, _stream(stream)),
           "rm_train_step")


def rm_train_sync_status(t: Trainer, stream=None) -> int:
    return _lib.rm_train_sync_status(t.ptr, _stream(stream))


# ------------------------------------------------------- token-sharded forward
def rm_tokshard_pack(h: Handle, Za, Zb, ln_g, ln_b, Xh, send, B: int, world: int, stream=None) -> None:
    _check(_lib.rm_tokshard_pack(h.ptr, _ptr(Za), _ptr(Zb), _ptr(ln_g), _ptr(ln_b), _ptr(Xh), _ptr(send), B, world,
                                 _stream(stream)), "rm_tokshard_pack")


def rm_tokshard_mix_ln(h: Handle, recv, Xh, ln1_g, ln1_b, S, B: int, world: int, stream=None) -> None:
    _check(_lib.rm_tokshard_mix_ln(h.ptr, _ptr(recv), _ptr(Xh), _ptr(ln1_g), _ptr(ln1_b), _ptr(S), B, world,
                                   _stream(stream)), "rm_tokshard_mix_ln")


def rm_tokshard_pool(h: Handle, V, S, ln2_g, ln2_b, pooled_part, B: int, stream=None) -> None:
    _check(_lib.rm_tokshard_pool(h.ptr, _ptr(V), _ptr(S), _ptr(ln2_g), _ptr(ln2_b), _ptr(pooled_part), B,
                                 _stream(stream)), "rm_tokshard_pool")


# ------------------------------------------------- stack with e4m3 FFN weights
def rm_quantize_fp8(src, dst, scale, rows: int, K: int, stream=None) -> None:
    _check(_lib.rm_quantize_fp8(_ptr(src), _ptr(dst), _ptr(scale), rows, K, _stream(stream)), "rm_quantize_fp8")


def rm_stack_forward_fp8(h: Handle, blocks: Sequence[Dict], qblocks: Sequence[Dict], X0, pooled, B: int,
                         stream=None) -> None:
    """qblocks: per block {"W1q", "W2q", "W1s", "W2s"} device tensors."""
    arr = _block_array(blocks)
    qarr = (rm_fp8_weights * len(qblocks))()
    for i, q in enumerate(qblocks):
        qarr[i] = rm_fp8_weights(**{n: _ptr(q[n]) for n, _ in rm_fp8_weights._fields_})
    _check(_lib.rm_stack_forward_fp8(h.ptr, arr, qarr, _ptr(X0), _ptr(pooled), B, _stream(stream)),
           "rm_stack_forward_fp8")
