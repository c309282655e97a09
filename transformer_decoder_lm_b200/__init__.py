"""GPT-2 decoder forward and backward passes on one B200 (sm_100a).

The product is the C-ABI library libgpt2.so (include/gpt2.h,
include/gpt2_train.h) built from
csrc/; ``binding`` is its ctypes binding (same names as the C entry points)
and ``model.GPT2Model`` a small owner of device weights, workspace and
handle. Importing this package fails if libgpt2.so has not been built.
"""
from . import binding  # noqa: F401  (raises ImportError when libgpt2.so is missing)
from .binding import (  # noqa: F401
    GPT2_BF16, GPT2_FP32, GPT2_EPI_BIAS, GPT2_EPI_BIAS_GELU, GPT2_EPI_BIAS_RESID, GPT2Error,
    GPT2_EPI_BIAS_GELU_TANH, GPT2_FLAG_GELU_TANH, gpt2_fill_sinusoidal_wpe,
    gpt2_kv_cache_bytes, gpt2_prefill, gpt2_decode_step,
    gpt2_workspace_bytes, gpt2_create, gpt2_forward, gpt2_loss, gpt2_forward_loss, gpt2_status,
    gpt2_error_string, gpt2_destroy, gpt2_launch_count, gpt2_set_timing_events, GPT2_TIMED_LMHEAD,
    gpt2_op_embed, gpt2_op_layernorm, gpt2_op_linear, gpt2_op_embed_layernorm,
    gpt2_op_attention, gpt2_op_lmhead_ce_workspace_bytes, gpt2_op_lmhead_ce, make_config,
    gpt2_op_lmhead_ce_noalloc, GPT2_NOALLOC_SCRATCH_BYTES,
    gpt2_train_workspace_bytes, gpt2_forward_backward, gpt2_op_linear_dgrad, gpt2_op_linear_wgrad,
    gpt2_op_linear_dgrad_gelu, gpt2_op_layernorm_backward_workspace_bytes, gpt2_op_layernorm_backward,
    gpt2_op_attention_train, gpt2_op_attention_backward_workspace_bytes, gpt2_op_attention_backward,
    gpt2_op_lmhead_ce_backward_workspace_bytes, gpt2_op_lmhead_ce_backward,
)
from .model import GPT2Model, upload_weights  # noqa: F401
