"""GPT2Model: owns device weights, the workspace and a libgpt2 handle.

PyTorch provides the device memory and the streams; every step of the
forward pass runs in libgpt2.so through the C ABI (binding.py).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import binding as B


def upload_weights(w: Dict[str, object], dtype: str, device="cuda") -> Dict[str, object]:
    """Copy a weight dict of float32 numpy arrays (synthetic.make_weights layout)
    to the device as bf16 or fp32 tensors (each its own 256-byte-aligned
    allocation)."""
    td = torch.bfloat16 if dtype == "bf16" else torch.float32

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=td)

    return {
        "wte": up(w["wte"]), "wpe": up(w["wpe"]),
        "layers": [{k: up(lw[k]) for k in B.LAYER_KEYS} for lw in w["layers"]],
        "lnf_g": up(w["lnf_g"]), "lnf_b": up(w["lnf_b"]),
    }


class GPT2Model:
    """A GPT-2 forward pass bound to device weights.

    n_layer, n_head, n_embd, vocab, n_ctx: the model shape. dtype: "bf16" or
    "fp32". weights: device tensors (upload_weights) or float32 numpy arrays.
    max_B, max_T: the largest batch the workspace is sized for.
    """

    def __init__(self, n_layer, n_head, n_embd, vocab, n_ctx, dtype, weights, max_B, max_T, device="cuda",
                 flags=0):
        self.dtype = dtype
        self.cfg = B.make_config(n_layer, n_head, n_embd, vocab, n_ctx,
                                 B.GPT2_BF16 if dtype == "bf16" else B.GPT2_FP32, flags)
        if isinstance(weights["wte"], np.ndarray):
            weights = upload_weights(weights, dtype, device)
        self.weights = weights
        self.vocab = vocab
        nbytes = B.gpt2_workspace_bytes(self.cfg, max_B, max_T)
        if nbytes == 0:
            raise B.GPT2Error(B.ERR_CODE["GPT2_ERR_INVALID_ARG"], "gpt2_workspace_bytes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.max_B = max_B
        self.max_T = max_T
        self.handle, self._keep = B.gpt2_create(self.cfg, weights, self.workspace, max_B, max_T)

    @classmethod
    def from_workload(cls, wl, weights, max_B=None, max_T=None, dtype=None, device="cuda", flags=0):
        return cls(wl.n_layer, wl.n_head, wl.n_embd, wl.vocab, wl.n_ctx, dtype or wl.dtype, weights,
                   max_B or wl.batch, max_T or wl.seq, device, flags)

    def forward(self, ids: torch.Tensor, logits: Optional[torch.Tensor] = None, want_logits=True, stream=None):
        Bsz, T = ids.shape
        if logits is None and want_logits:
            logits = torch.empty(Bsz, T, self.vocab, dtype=torch.float32, device=ids.device)
        B.gpt2_forward(self.handle, ids, Bsz, T, logits, stream)
        return logits

    def loss(self, ids: torch.Tensor, targets: torch.Tensor, loss_out: Optional[torch.Tensor] = None, stream=None):
        Bsz, T = ids.shape
        if loss_out is None:
            loss_out = torch.empty(1, dtype=torch.float32, device=ids.device)
        B.gpt2_loss(self.handle, ids, targets, Bsz, T, loss_out, stream)
        return loss_out

    def forward_loss(self, ids, targets, logits=None, want_logits=True, token_loss=None, loss_out=None, stream=None):
        Bsz, T = ids.shape
        if logits is None and want_logits:
            logits = torch.empty(Bsz, T, self.vocab, dtype=torch.float32, device=ids.device)
        if loss_out is None:
            loss_out = torch.empty(1, dtype=torch.float32, device=ids.device)
        B.gpt2_forward_loss(self.handle, ids, targets, Bsz, T, logits, loss_out, token_loss, stream)
        return logits, loss_out

    def new_kv_cache(self) -> torch.Tensor:
        """A key/value cache for incremental decoding (gpt2_kv_cache_bytes bytes)."""
        n = B.gpt2_kv_cache_bytes(self.cfg, self.max_B)
        return torch.empty(n, dtype=torch.uint8, device=self.workspace.device)

    def prefill(self, ids: torch.Tensor, kv_cache: torch.Tensor, want_logits=True, stream=None):
        """The forward over ids [B, T], storing every layer's keys and values in kv_cache."""
        Bsz, T = ids.shape
        logits = torch.empty(Bsz, T, self.vocab, dtype=torch.float32, device=ids.device) if want_logits else None
        B.gpt2_prefill(self.handle, kv_cache, ids, Bsz, T, logits, stream)
        return logits

    def decode_step(self, ids_new: torch.Tensor, pos: int, kv_cache: torch.Tensor, logits=None, stream=None):
        """Logits [B, vocab] of one new token per sequence at position pos."""
        Bsz = ids_new.shape[0]
        if logits is None:
            logits = torch.empty(Bsz, self.vocab, dtype=torch.float32, device=ids_new.device)
        B.gpt2_decode_step(self.handle, kv_cache, ids_new, Bsz, pos, logits, stream)
        return logits

    def new_train_workspace(self) -> torch.Tensor:
        """The training workspace of gpt2_forward_backward for this handle's max_B x max_T."""
        n = B.gpt2_train_workspace_bytes(self.cfg, self.max_B, self.max_T)
        if n == 0:
            raise B.GPT2Error(B.ERR_CODE["GPT2_ERR_UNSUPPORTED"], "gpt2_train_workspace_bytes")
        return torch.empty(n, dtype=torch.uint8, device=self.workspace.device)

    def new_grads(self) -> Dict[str, object]:
        """fp32 gradient buffers shaped like the weights."""
        def like(t):
            return torch.empty(t.shape, dtype=torch.float32, device=t.device)
        w = self.weights
        return {"wte": like(w["wte"]), "wpe": like(w["wpe"]), "lnf_g": like(w["lnf_g"]), "lnf_b": like(w["lnf_b"]),
                "layers": [{k: like(lw[k]) for k in B.LAYER_KEYS} for lw in w["layers"]]}

    def forward_backward(self, ids, targets, grads, train_ws, loss_out=None, stream=None):
        """Loss and the gradient of every weight (gpt2_forward_backward)."""
        Bsz, T = ids.shape
        if loss_out is None:
            loss_out = torch.empty(1, dtype=torch.float32, device=ids.device)
        B.gpt2_forward_backward(self.handle, ids, targets, Bsz, T, loss_out, grads, train_ws, stream)
        return loss_out

    def status(self, stream=None) -> int:
        return B.gpt2_status(self.handle, stream)

    def close(self):
        if getattr(self, "handle", None) is not None:
            B.gpt2_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
