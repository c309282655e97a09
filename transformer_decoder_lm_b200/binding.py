"""ctypes binding of libgpt2.so (include/gpt2.h), argument marshalling only.

Every function here has the name of the C entry point it calls and takes
torch tensors (device memory owned by the caller) or plain integers; it
converts them to pointers and sizes, calls the library, and raises
``GPT2Error`` on a non-zero return code. All computation happens in the CUDA
kernels of libgpt2.so: there is no fallback of any kind, and importing this
module fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgpt2.so")

GPT2_BF16, GPT2_FP32 = 0, 1
GPT2_EPI_BIAS, GPT2_EPI_BIAS_GELU, GPT2_EPI_BIAS_RESID, GPT2_EPI_BIAS_GELU_TANH = 0, 1, 2, 3
GPT2_FLAG_GELU_TANH = 1
ERRORS = {
    0: "GPT2_OK", 1: "GPT2_ERR_INVALID_ARG", 2: "GPT2_ERR_UNSUPPORTED", 3: "GPT2_ERR_CUDA",
    4: "GPT2_ERR_WORKSPACE", 5: "GPT2_ERR_BAD_TOKEN", 6: "GPT2_ERR_DEVICE_TIMEOUT", 7: "GPT2_ERR_NO_TARGETS",
    8: "GPT2_ERR_SCRATCH_LIMIT",
}
GPT2_NOALLOC_SCRATCH_BYTES = 32 << 20
ERR_CODE = {v: k for k, v in ERRORS.items()}

LAYER_KEYS = (
    "ln1_g", "ln1_b", "attn_w", "attn_b", "attn_proj_w", "attn_proj_b",
    "ln2_g", "ln2_b", "fc_w", "fc_b", "mlp_proj_w", "mlp_proj_b",
)


class GPT2Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {ERRORS.get(code, code)} ({code})")


class gpt2_config_t(ctypes.Structure):
    _fields_ = [("n_layer", ctypes.c_int), ("n_head", ctypes.c_int), ("n_embd", ctypes.c_int),
                ("vocab", ctypes.c_int), ("n_ctx", ctypes.c_int), ("dtype", ctypes.c_int),
                ("flags", ctypes.c_uint)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class gpt2_weights_t(ctypes.Structure):
    _fields_ = [("wte", ctypes.c_void_p), ("wpe", ctypes.c_void_p)] + \
               [(k, _PP) for k in LAYER_KEYS] + \
               [("lnf_g", ctypes.c_void_p), ("lnf_b", ctypes.c_void_p)]


class gpt2_grads_t(ctypes.Structure):
    _fields_ = [("wte", ctypes.c_void_p), ("wpe", ctypes.c_void_p)] + \
               [(k, _PP) for k in LAYER_KEYS] + \
               [("lnf_g", ctypes.c_void_p), ("lnf_b", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libgpt2.so is not built ({LIB_PATH}); run python transformer_decoder_lm_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "gpt2_workspace_bytes": (sz, [ctypes.POINTER(gpt2_config_t), i, i]),
        "gpt2_create": (i, [ctypes.POINTER(gpt2_config_t), ctypes.POINTER(gpt2_weights_t), vp, sz, i, i,
                            ctypes.POINTER(vp)]),
        "gpt2_forward": (i, [vp, vp, i, i, vp, vp]),
        "gpt2_loss": (i, [vp, vp, vp, i, i, vp, vp]),
        "gpt2_forward_loss": (i, [vp, vp, vp, i, i, vp, vp, vp, vp]),
        "gpt2_status": (i, [vp, vp]),
        "gpt2_kv_cache_bytes": (sz, [ctypes.POINTER(gpt2_config_t), i]),
        "gpt2_prefill": (i, [vp, vp, sz, vp, i, i, vp, vp]),
        "gpt2_decode_step": (i, [vp, vp, sz, vp, i, i, vp, vp]),
        "gpt2_error_string": (ctypes.c_char_p, [i]),
        "gpt2_destroy": (None, [vp]),
        "gpt2_launch_count": (ctypes.c_uint64, [vp]),
        "gpt2_set_timing_events": (i, [vp, i, vp, vp]),
        "gpt2_op_embed": (i, [i, vp, vp, vp, i, i, i, i, vp, vp, vp]),
        "gpt2_op_layernorm": (i, [i, vp, vp, vp, i, i, vp, vp]),
        "gpt2_op_linear": (i, [i, i, vp, vp, vp, i, i, i, vp, vp, vp]),
        "gpt2_op_attention": (i, [i, vp, i, i, i, i, vp, vp, vp]),
        "gpt2_fill_sinusoidal_wpe": (i, [i, vp, i, i, vp]),
        "gpt2_op_embed_layernorm": (i, [vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp, vp]),
        "gpt2_op_lmhead_ce_workspace_bytes": (sz, [i, i, i]),
        "gpt2_op_lmhead_ce": (i, [i, vp, vp, vp, i, i, i, vp, vp, vp, vp, sz, vp, vp]),
        "gpt2_op_lmhead_ce_noalloc": (i, [i, vp, vp, vp, i, i, i, vp, vp, vp, vp, vp]),
        # include/gpt2_train.h
        "gpt2_train_workspace_bytes": (sz, [ctypes.POINTER(gpt2_config_t), i, i]),
        "gpt2_forward_backward": (i, [vp, vp, vp, i, i, vp, ctypes.POINTER(gpt2_grads_t), vp, sz, vp]),
        "gpt2_op_linear_dgrad": (i, [vp, vp, i, i, i, vp, i, vp, vp]),
        "gpt2_op_linear_wgrad": (i, [vp, vp, i, i, i, vp, vp, vp]),
        "gpt2_op_linear_dgrad_gelu": (i, [vp, vp, vp, i, i, i, i, vp, vp, vp]),
        "gpt2_op_layernorm_backward_workspace_bytes": (sz, [i, i]),
        "gpt2_op_layernorm_backward": (i, [vp, vp, vp, vp, i, i, vp, vp, vp, vp, sz, vp]),
        "gpt2_op_attention_train": (i, [vp, i, i, i, i, vp, vp, vp, vp]),
        "gpt2_op_attention_backward_workspace_bytes": (sz, [i, i, i, i]),
        "gpt2_op_attention_backward": (i, [vp, vp, vp, vp, i, i, i, i, vp, vp, sz, vp, vp]),
        "gpt2_op_lmhead_ce_backward_workspace_bytes": (sz, [i, i]),
        "gpt2_op_lmhead_ce_backward": (i, [vp, vp, vp, i, i, i, vp, vp, vp, vp, sz, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib, sig


lib, SIGNATURES = _load()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise GPT2Error(rc, where)


def make_config(n_layer: int, n_head: int, n_embd: int, vocab: int, n_ctx: int, dtype: int,
                flags: int = 0) -> gpt2_config_t:
    return gpt2_config_t(n_layer, n_head, n_embd, vocab, n_ctx, dtype, flags)


def gpt2_workspace_bytes(cfg: gpt2_config_t, max_B: int, max_T: int) -> int:
    return int(lib.gpt2_workspace_bytes(ctypes.byref(cfg), max_B, max_T))


class _Weights:
    """Keeps the ctypes pointer arrays alive as long as the handle."""

    def __init__(self, w: Dict[str, object]):
        n = len(w["layers"])
        self.arrays = {k: (ctypes.c_void_p * n)(*[_ptr(lw[k]) for lw in w["layers"]]) for k in LAYER_KEYS}
        self.struct = gpt2_weights_t(
            _ptr(w["wte"]), _ptr(w["wpe"]),
            *[ctypes.cast(self.arrays[k], _PP) for k in LAYER_KEYS],
            _ptr(w["lnf_g"]), _ptr(w["lnf_b"]))


def gpt2_create(cfg: gpt2_config_t, weights: Dict[str, object], workspace, max_B: int, max_T: int):
    """weights: {'wte','wpe','lnf_g','lnf_b': tensor, 'layers': [ {LAYER_KEYS: tensor} ]}
    (device tensors of cfg.dtype). Returns (handle, keepalive)."""
    keep = _Weights(weights)
    h = ctypes.c_void_p()
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.gpt2_create(ctypes.byref(cfg), ctypes.byref(keep.struct), _ptr(workspace), nbytes, max_B, max_T,
                           ctypes.byref(h)), "gpt2_create")
    return h, keep


def gpt2_forward(h, ids, B: int, T: int, logits=None, stream=None) -> None:
    _check(lib.gpt2_forward(h, _ptr(ids), B, T, _ptr(logits), _stream(stream)), "gpt2_forward")


def gpt2_loss(h, ids, targets, B: int, T: int, loss_out, stream=None) -> None:
    _check(lib.gpt2_loss(h, _ptr(ids), _ptr(targets), B, T, _ptr(loss_out), _stream(stream)), "gpt2_loss")


def gpt2_forward_loss(h, ids, targets, B: int, T: int, logits, loss_out, token_loss=None, stream=None) -> None:
    _check(lib.gpt2_forward_loss(h, _ptr(ids), _ptr(targets), B, T, _ptr(logits), _ptr(loss_out), _ptr(token_loss),
                                 _stream(stream)), "gpt2_forward_loss")


def gpt2_kv_cache_bytes(cfg: gpt2_config_t, max_B: int) -> int:
    return int(lib.gpt2_kv_cache_bytes(ctypes.byref(cfg), max_B))


def _nbytes(t) -> int:
    return 0 if t is None else int(t.numel() * t.element_size())


def gpt2_prefill(h, kv_cache, ids, B: int, T: int, logits=None, stream=None) -> None:
    _check(lib.gpt2_prefill(h, _ptr(kv_cache), _nbytes(kv_cache), _ptr(ids), B, T, _ptr(logits), _stream(stream)),
           "gpt2_prefill")


def gpt2_decode_step(h, kv_cache, ids_new, B: int, pos: int, logits, stream=None) -> None:
    _check(lib.gpt2_decode_step(h, _ptr(kv_cache), _nbytes(kv_cache), _ptr(ids_new), B, pos, _ptr(logits),
                                _stream(stream)), "gpt2_decode_step")


def gpt2_status(h, stream=None) -> int:
    return int(lib.gpt2_status(h, _stream(stream)))


def gpt2_error_string(code: int) -> str:
    return lib.gpt2_error_string(code).decode()


def gpt2_destroy(h) -> None:
    lib.gpt2_destroy(h)


def gpt2_launch_count(h) -> int:
    return int(lib.gpt2_launch_count(h))


GPT2_TIMED_LMHEAD = 0


def gpt2_set_timing_events(h, which: int, ev_begin=None, ev_end=None) -> None:
    """ev_begin / ev_end: torch.cuda.Event (created with enable_timing=True) or None."""
    b = ev_begin.cuda_event if ev_begin is not None else None
    e = ev_end.cuda_event if ev_end is not None else None
    _check(lib.gpt2_set_timing_events(h, which, b, e), "gpt2_set_timing_events")


def gpt2_op_embed(dtype, ids, wte, wpe, M, T, C, V, x, status=None, stream=None):
    _check(lib.gpt2_op_embed(dtype, _ptr(ids), _ptr(wte), _ptr(wpe), M, T, C, V, _ptr(x), _ptr(status),
                             _stream(stream)), "gpt2_op_embed")


def gpt2_op_layernorm(dtype, x, g, b, M, C, out, stream=None):
    _check(lib.gpt2_op_layernorm(dtype, _ptr(x), _ptr(g), _ptr(b), M, C, _ptr(out), _stream(stream)),
           "gpt2_op_layernorm")


def gpt2_op_linear(dtype, epilogue, A, W, bias, M, N, K, out, status=None, stream=None):
    _check(lib.gpt2_op_linear(dtype, epilogue, _ptr(A), _ptr(W), _ptr(bias), M, N, K, _ptr(out), _ptr(status),
                              _stream(stream)), "gpt2_op_linear")


def gpt2_op_embed_layernorm(ids, wte, wpe, M, T, C, V, g, b, x, h, status=None, stream=None):
    _check(lib.gpt2_op_embed_layernorm(_ptr(ids), _ptr(wte), _ptr(wpe), M, T, C, V, _ptr(g), _ptr(b), _ptr(x), _ptr(h),
                                       _ptr(status), _stream(stream)), "gpt2_op_embed_layernorm")


def gpt2_fill_sinusoidal_wpe(dtype, wpe, n_ctx, C, stream=None):
    _check(lib.gpt2_fill_sinusoidal_wpe(dtype, _ptr(wpe), n_ctx, C, _stream(stream)), "gpt2_fill_sinusoidal_wpe")


def gpt2_op_attention(dtype, qkv, B, T, H, C, y, status=None, stream=None):
    _check(lib.gpt2_op_attention(dtype, _ptr(qkv), B, T, H, C, _ptr(y), _ptr(status), _stream(stream)),
           "gpt2_op_attention")


def gpt2_op_lmhead_ce_workspace_bytes(dtype, M, V) -> int:
    return int(lib.gpt2_op_lmhead_ce_workspace_bytes(dtype, M, V))


def gpt2_op_lmhead_ce(dtype, hf, wte, targets, M, C, V, logits, token_loss, loss_out, workspace, status=None,
                      stream=None):
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib.gpt2_op_lmhead_ce(dtype, _ptr(hf), _ptr(wte), _ptr(targets), M, C, V, _ptr(logits), _ptr(token_loss),
                                 _ptr(loss_out), _ptr(workspace), nbytes, _ptr(status), _stream(stream)),
           "gpt2_op_lmhead_ce")


def gpt2_op_lmhead_ce_noalloc(dtype, hf, wte, targets, M, C, V, logits, token_loss, loss_out, status=None,
                              stream=None):
    """gpt2_op_lmhead_ce without a workspace: for callers that cannot allocate
    device memory; its scratch is a fixed array inside libgpt2.so (see
    include/gpt2.h for the size limit and the ordering rule)."""
    _check(lib.gpt2_op_lmhead_ce_noalloc(dtype, _ptr(hf), _ptr(wte), _ptr(targets), M, C, V, _ptr(logits),
                                         _ptr(token_loss), _ptr(loss_out), _ptr(status), _stream(stream)),
           "gpt2_op_lmhead_ce_noalloc")


# ---- include/gpt2_train.h ---------------------------------------------------

def gpt2_train_workspace_bytes(cfg: gpt2_config_t, max_B: int, max_T: int) -> int:
    return int(lib.gpt2_train_workspace_bytes(ctypes.byref(cfg), max_B, max_T))


class _Grads:
    """Keeps the ctypes pointer arrays of a gradient dict alive (layout of the
    weights dict: 'wte', 'wpe', 'lnf_g', 'lnf_b', 'layers': [{LAYER_KEYS}])."""

    def __init__(self, g: Dict[str, object]):
        n = len(g["layers"])
        self.arrays = {k: (ctypes.c_void_p * n)(*[_ptr(lg[k]) for lg in g["layers"]]) for k in LAYER_KEYS}
        self.struct = gpt2_grads_t(
            _ptr(g["wte"]), _ptr(g["wpe"]),
            *[ctypes.cast(self.arrays[k], _PP) for k in LAYER_KEYS],
            _ptr(g["lnf_g"]), _ptr(g["lnf_b"]))


def gpt2_forward_backward(h, ids, targets, B: int, T: int, loss_out, grads: Dict[str, object], train_ws,
                          stream=None) -> None:
    keep = _Grads(grads)
    _check(lib.gpt2_forward_backward(h, _ptr(ids), _ptr(targets), B, T, _ptr(loss_out), ctypes.byref(keep.struct),
                                     _ptr(train_ws), _nbytes(train_ws), _stream(stream)), "gpt2_forward_backward")


def gpt2_op_linear_dgrad(dy, W, M, N, K, dx, out_f32=True, status=None, stream=None):
    _check(lib.gpt2_op_linear_dgrad(_ptr(dy), _ptr(W), M, N, K, _ptr(dx), int(bool(out_f32)), _ptr(status),
                                    _stream(stream)), "gpt2_op_linear_dgrad")


def gpt2_op_linear_wgrad(dy, x, M, N, K, dW, status=None, stream=None):
    _check(lib.gpt2_op_linear_wgrad(_ptr(dy), _ptr(x), M, N, K, _ptr(dW), _ptr(status), _stream(stream)),
           "gpt2_op_linear_wgrad")


def gpt2_op_linear_dgrad_gelu(dy, W, u, M, N, K, tanh_form, du, status=None, stream=None):
    _check(lib.gpt2_op_linear_dgrad_gelu(_ptr(dy), _ptr(W), _ptr(u), M, N, K, int(tanh_form), _ptr(du), _ptr(status),
                                         _stream(stream)), "gpt2_op_linear_dgrad_gelu")


def gpt2_op_layernorm_backward_workspace_bytes(M, C) -> int:
    return int(lib.gpt2_op_layernorm_backward_workspace_bytes(M, C))


def gpt2_op_layernorm_backward(x, gamma, dh, dx_in, M, C, dx_out, dgamma, dbeta, workspace, stream=None):
    _check(lib.gpt2_op_layernorm_backward(_ptr(x), _ptr(gamma), _ptr(dh), _ptr(dx_in), M, C, _ptr(dx_out),
                                          _ptr(dgamma), _ptr(dbeta), _ptr(workspace), _nbytes(workspace),
                                          _stream(stream)), "gpt2_op_layernorm_backward")


def gpt2_op_attention_train(qkv, B, T, H, C, y, lse2, status=None, stream=None):
    _check(lib.gpt2_op_attention_train(_ptr(qkv), B, T, H, C, _ptr(y), _ptr(lse2), _ptr(status), _stream(stream)),
           "gpt2_op_attention_train")


def gpt2_op_attention_backward_workspace_bytes(B, T, H, C) -> int:
    return int(lib.gpt2_op_attention_backward_workspace_bytes(B, T, H, C))


def gpt2_op_attention_backward(qkv, y, dy, lse2, B, T, H, C, dqkv, workspace, status=None, stream=None):
    _check(lib.gpt2_op_attention_backward(_ptr(qkv), _ptr(y), _ptr(dy), _ptr(lse2), B, T, H, C, _ptr(dqkv),
                                          _ptr(workspace), _nbytes(workspace), _ptr(status), _stream(stream)),
           "gpt2_op_attention_backward")


def gpt2_op_lmhead_ce_backward_workspace_bytes(M, V) -> int:
    return int(lib.gpt2_op_lmhead_ce_backward_workspace_bytes(M, V))


def gpt2_op_lmhead_ce_backward(hf, wte, targets, M, C, V, loss_out, dhf, dwte, workspace, status=None, stream=None):
    _check(lib.gpt2_op_lmhead_ce_backward(_ptr(hf), _ptr(wte), _ptr(targets), M, C, V, _ptr(loss_out), _ptr(dhf),
                                          _ptr(dwte), _ptr(workspace), _nbytes(workspace), _ptr(status),
                                          _stream(stream)), "gpt2_op_lmhead_ce_backward")
