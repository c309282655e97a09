/* gpt2_train.h - C ABI of the GPT-2 backward pass on B200 (sm_100a).
 *
 * The gradient of the training loss - the mean next-token cross-entropy of
 * gpt2_loss - with respect to every weight of the model: the loss.backward()
 * of the training loop in "Hand-writing GPT-2 from scratch: the Transformer
 * decoder core modules in PyTorch", section 4.3, written out as kernels. The
 * lm_head is tied to the token embedding (same page, section 2.2), so the
 * gradient of wte is the sum of the head's term (dlogits^T . ln_f output)
 * and the embedding's term (the residual gradient of each position added
 * into the row of its token id).
 *
 * Conventions are those of gpt2.h: device pointers, caller-owned buffers,
 * asynchronous on `stream`, GPT2_ERR_* return codes (host-side checks before
 * any launch; device-side conditions through gpt2_status). Only bf16 models
 * with d_head 64 and more than 16 positions per call are supported (the
 * tensor-core path); anything else returns GPT2_ERR_UNSUPPORTED.
 *
 * Precision: bf16 operands with fp32 accumulation in every product, as in
 * the forward pass; the residual-stream gradient, the LayerNorm gradients and
 * every weight gradient are fp32. Column sums (bias, gamma, beta gradients)
 * add in a fixed order; the attention's dq and the token-embedding rows of
 * repeated ids are summed with fp32 atomics, so their last bits can differ
 * from run to run.
 */
#ifndef GPT2_B200_TRAIN_H
#define GPT2_B200_TRAIN_H

#include "gpt2.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Gradient buffers, fp32, one per weight with the weight's shape
 * (gpt2_weights_t): wte [vocab, C], wpe [n_ctx, C], per layer (host arrays of
 * n_layer device pointers) ln1_g/ln1_b [C], attn_w [3C, C], attn_b [3C],
 * attn_proj_w [C, C], attn_proj_b [C], ln2_g/ln2_b [C], fc_w [4C, C],
 * fc_b [4C], mlp_proj_w [C, 4C], mlp_proj_b [C]; lnf_g/lnf_b [C]. Every
 * element is overwritten (not accumulated) by gpt2_forward_backward; rows of
 * wpe at or past T get 0. 16-byte aligned. */
typedef struct {
  float *wte, *wpe;
  float **ln1_g, **ln1_b, **attn_w, **attn_b, **attn_proj_w, **attn_proj_b,
        **ln2_g, **ln2_b, **fc_w, **fc_b, **mlp_proj_w, **mlp_proj_b;
  float *lnf_g, *lnf_b;
} gpt2_grads_t;

/* Bytes of the training workspace for up to max_B x max_T tokens: the
 * activations the backward pass differentiates at (per layer: the inputs of
 * both LayerNorms, their outputs, qkv, the attention output and its row
 * log-sum-exp, the c_fc pre-activation and GELU output; the ln_f input and
 * output), the logits gradient [M, vocab rounded up to 64] bf16 and the
 * backward's scratch. 0 for a bad or unsupported config. */
size_t gpt2_train_workspace_bytes(const gpt2_config_t* cfg, int max_B, int max_T);

/* One training step's forward and backward: the loss of gpt2_loss over ids,
 * targets [B, T] (negative target = not scored) into loss_out (fp32 [1]),
 * then every weight's gradient into `grads`. train_ws: device, 256-byte
 * aligned, at least gpt2_train_workspace_bytes(cfg, B_max, T_max) for the
 * B_max, T_max it was sized for (B <= the handle's max_B, T <= its max_T);
 * GPT2_ERR_WORKSPACE if smaller. The handle's own workspace is used too, so
 * calls on one handle must not overlap. */
int gpt2_forward_backward(gpt2_handle_t h, const int32_t* ids, const int32_t* targets, int B, int T,
                          float* loss_out, const gpt2_grads_t* grads, void* train_ws, size_t train_ws_bytes,
                          void* stream);

/* ---- single steps of the backward pass (each checked on its own) --------- */

/* Linear layer y = x W^T (W [N, K] bf16, the nn.Linear [out, in] layout of
 * section 3.4 of the first page), backward:
 *   dgrad: dx [M, K] = dy [M, N] . W          (out fp32 if out_f32, else bf16)
 *   wgrad: dW [N, K] = dy^T [N, M] . x [M, K] (fp32)
 * bf16 dy and x, M > 0, N and K multiples of 8. */
int gpt2_op_linear_dgrad(const void* dy, const void* W, int M, int N, int K, void* dx, int out_f32,
                         int* status, void* stream);
int gpt2_op_linear_wgrad(const void* dy, const void* x, int M, int N, int K, float* dW, int* status,
                         void* stream);

/* MLP activation backward fused into the dgrad of c_proj ("GPT-2 architecture
 * analysis and implementation guide", section 2.2: F.gelu; the tanh form of
 * the first page's section 3.4 when tanh_form is 1):
 *   du [M, K] (bf16) = (dy [M, N] . W [N, K]) * gelu'(u [M, K] bf16). */
int gpt2_op_linear_dgrad_gelu(const void* dy, const void* W, const void* u, int M, int N, int K, int tanh_form,
                              void* du, int* status, void* stream);

/* LayerNorm backward ("Reproducing GPT-2 124M", section 2.1: biased variance,
 * eps 1e-5 inside the square root): x fp32 [M, C] (the LayerNorm input),
 * gamma bf16 [C], dh fp32 [M, C] (the output's gradient), dx_in fp32 [M, C]
 * or NULL (a gradient to add, the residual path) -> dx_out fp32 [M, C],
 * dgamma, dbeta fp32 [C]. Scratch: gpt2_op_layernorm_backward_workspace_bytes. */
size_t gpt2_op_layernorm_backward_workspace_bytes(int M, int C);
int gpt2_op_layernorm_backward(const float* x, const void* gamma, const float* dh, const float* dx_in, int M, int C,
                               float* dx_out, float* dgamma, float* dbeta, void* workspace, size_t ws_bytes,
                               void* stream);

/* Causal attention forward that also returns each query row's log-sum-exp:
 * as gpt2_op_attention (bf16, D = 64), plus lse2 fp32 [B, H, T] = log2 of the
 * sum over visible keys of 2^(q.k log2(e) / sqrt(D)). */
int gpt2_op_attention_train(const void* qkv, int B, int T, int H, int C, void* y, float* lse2, int* status,
                            void* stream);

/* Causal attention backward ("Reproducing GPT-2 124M", sections 2.1-2.2, the
 * attention it differentiates): qkv, y bf16 and lse2 from
 * gpt2_op_attention_train, dy bf16 [B*T, C] -> dqkv bf16 [B*T, 3C] (dq | dk |
 * dv in the column layout of qkv). Scratch:
 * gpt2_op_attention_backward_workspace_bytes. status (int32 on the device,
 * may be NULL): GPT2_ERR_DEVICE_TIMEOUT is or-ed in if a wait inside the
 * kernel runs out (the kernel then returns early; dqkv is not valid). */
size_t gpt2_op_attention_backward_workspace_bytes(int B, int T, int H, int C);
int gpt2_op_attention_backward(const void* qkv, const void* y, const void* dy, const float* lse2, int B, int T, int H,
                               int C, void* dqkv, void* workspace, size_t ws_bytes, int* status, void* stream);

/* Tied lm_head + cross-entropy backward on a final hidden state hf bf16 [M, C]
 * and wte bf16 [V, C] (targets int32 [M], negative = not scored): the mean
 * loss into loss_out, dhf fp32 [M, C] = dz . wte and dwte fp32 [V, C] =
 * dz^T . hf with dz = (softmax(z) - onehot(target)) / n_scored on scored rows
 * ("Hand-writing GPT-2 from scratch: the Transformer decoder core modules in
 * PyTorch", section 4.1 step 5). Scratch:
 * gpt2_op_lmhead_ce_backward_workspace_bytes. */
size_t gpt2_op_lmhead_ce_backward_workspace_bytes(int M, int V);
int gpt2_op_lmhead_ce_backward(const void* hf, const void* wte, const int32_t* targets, int M, int C, int V,
                               float* loss_out, float* dhf, float* dwte, void* workspace, size_t ws_bytes,
                               int* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_TRAIN_H */
