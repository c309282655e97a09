/*
 * gpt2.h - C ABI of the GPT-2 decoder forward pass on one B200 (sm_100a).
 *
 * The forward pass computed here is the one described by
 *   "Hand-writing GPT-2 from scratch: the Transformer decoder core modules in
 *    PyTorch" (blog.csdn.net), sections 2.2 (embedding, block stack, ln_f,
 *    tied lm_head), 3.2-3.4 (Pre-LN block, causal mask, MLP) and 4.1
 *    (GPT2Model.forward with the shifted cross-entropy), and
 *   "Reproducing GPT-2 124M" (nzsm.cn), sections 2.1-2.4 (LayerNorm with the
 *    biased variance and eps 1e-5, c_attn split into q/k/v, scores scaled by
 *    1/sqrt(d_head), -inf above the diagonal before the softmax, weight tying).
 *
 *   x      = wte[ids] + wpe[0..T-1]
 *   for each layer:  x += c_proj(attn(ln_1(x)));  x += mlp_proj(gelu(c_fc(ln_2(x))))
 *   logits = ln_f(x) . wte^T
 *   loss   = mean over scored positions of  logsumexp(logits[t]) - logits[t, target[t]]
 *
 * GELU is the exact erf form (F.gelu; "GPT-2 architecture analysis and
 * implementation guide", section 2.2). Every Linear has a bias; the lm_head
 * has none and reads the wte buffer itself.
 *
 * Conventions
 *  - All tensors are caller-owned DEVICE pointers unless stated otherwise.
 *    The library never allocates device memory, never copies or frees the
 *    caller's buffers, and keeps only the pointers given to gpt2_create.
 *  - Row-major layouts. Linear weights use the nn.Linear [out, in] layout.
 *  - Parameters have the storage type cfg.dtype (bf16 or fp32). In bf16 mode
 *    activations are stored in bf16 at GEMM/attention inputs, the residual
 *    stream, LayerNorm statistics, softmax and logits are fp32, and all
 *    products accumulate in fp32. In fp32 mode everything is fp32.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). All work is stream-ordered and asynchronous; calls on one
 *    handle are not thread-safe.
 *  - Return value: 0 on success, else a GPT2_ERR_* code. Host-side argument
 *    errors are detected before any launch and leave the device untouched.
 *    Device-side conditions (a token id outside [0, vocab), a bounded wait
 *    that timed out) are recorded in a status word and reported by
 *    gpt2_status, like CUDA's own asynchronous errors.
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { GPT2_BF16 = 0, GPT2_FP32 = 1 } gpt2_dtype_t;

enum {
  GPT2_OK = 0,
  GPT2_ERR_INVALID_ARG = 1,     /* null pointer, non-positive size, size above the create-time maximum */
  GPT2_ERR_UNSUPPORTED = 2,     /* n_embd % n_head != 0, d_head not 32 or 64, T > n_ctx, dims not multiples of 8 */
  GPT2_ERR_CUDA = 3,            /* a CUDA runtime call or launch failed */
  GPT2_ERR_WORKSPACE = 4,       /* workspace too small or misaligned (256 B) */
  GPT2_ERR_BAD_TOKEN = 5,       /* device: an id was outside [0, vocab); it was clamped to 0 */
  GPT2_ERR_DEVICE_TIMEOUT = 6,  /* device: a bounded wait inside a kernel gave up */
  GPT2_ERR_NO_TARGETS = 7,      /* device: no position had a target >= 0; the loss was written as NaN */
  GPT2_ERR_SCRATCH_LIMIT = 8    /* the request needs more scratch than the allocation-free entry point holds */
};

/* Model shape. n_ctx is the size of the learned position table wpe
 * ("GPT-2 architecture analysis and implementation guide", section 1.2).
 * flags: 0 or GPT2_FLAG_GELU_TANH; other bits must be 0. */
typedef struct {
  int n_layer, n_head, n_embd, vocab, n_ctx;
  int dtype;          /* gpt2_dtype_t */
  unsigned flags;
} gpt2_config_t;

/* The MLP's activation is the tanh approximation
 *   gelu_tanh(x) = 0.5 x (1 + tanh(sqrt(2 / pi) (x + 0.044715 x^3))),
 * the form the pages attribute to the original GPT-2 ("Hand-writing GPT-2
 * from scratch: the Transformer decoder core modules in PyTorch", section
 * 3.4; "Reproducing GPT-2 124M", section 2.4), instead of the default exact
 * erf form (F.gelu, "GPT-2 architecture analysis and implementation guide",
 * section 2.2). */
#define GPT2_FLAG_GELU_TANH 1u

/* Weight pointers. wte [vocab, C] is also the lm_head weight (weight tying,
 * "Hand-writing GPT-2 from scratch ...", section 2.2 item 4). wpe [n_ctx, C].
 * The per-layer members are HOST arrays of n_layer DEVICE pointers:
 *   ln1_g, ln1_b, ln2_g, ln2_b  [C]
 *   attn_w [3C, C], attn_b [3C]         (c_attn; output columns q | k | v)
 *   attn_proj_w [C, C], attn_proj_b [C] (attention c_proj)
 *   fc_w [4C, C], fc_b [4C]             (mlp c_fc)
 *   mlp_proj_w [C, 4C], mlp_proj_b [C]  (mlp c_proj)
 * lnf_g, lnf_b [C]. Every device pointer must be 16-byte aligned.
 * gpt2_create copies the host arrays; the device buffers must outlive the
 * handle. */
typedef struct {
  const void* wte;
  const void* wpe;
  const void* const* ln1_g;
  const void* const* ln1_b;
  const void* const* attn_w;
  const void* const* attn_b;
  const void* const* attn_proj_w;
  const void* const* attn_proj_b;
  const void* const* ln2_g;
  const void* const* ln2_b;
  const void* const* fc_w;
  const void* const* fc_b;
  const void* const* mlp_proj_w;
  const void* const* mlp_proj_b;
  const void* lnf_g;
  const void* lnf_b;
} gpt2_weights_t;

typedef struct gpt2_model* gpt2_handle_t;

/* Bytes of device workspace a model needs for batches up to max_B x max_T
 * tokens (activations, the residual stream, cross-entropy partials and the
 * status word). Returns 0 if the arguments are invalid. */
size_t gpt2_workspace_bytes(const gpt2_config_t* cfg, int max_B, int max_T);

/* Validate cfg and the weight pointers, carve `workspace` (device,
 * 256-byte aligned, >= gpt2_workspace_bytes bytes, caller-owned) and return
 * a handle in *out. Selects the current CUDA device as the model's device. */
int gpt2_create(const gpt2_config_t* cfg, const gpt2_weights_t* w, void* workspace,
                size_t ws_bytes, int max_B, int max_T, gpt2_handle_t* out);

/* Forward pass of ids int32 [B, T] (B <= max_B, T <= min(max_T, n_ctx)).
 * logits_or_null: fp32 [B, T, vocab] (unpadded). With NULL only the trunk
 * and ln_f run; the final hidden state stays in the workspace. */
int gpt2_forward(gpt2_handle_t h, const int32_t* ids, int B, int T,
                 float* logits_or_null, void* stream);

/* Forward pass plus the next-token cross-entropy, without writing logits
 * (the lm_head and the log-sum-exp run fused; "Hand-writing GPT-2 from
 * scratch ...", section 4.1 step 5). targets int32 [B, T] is position-aligned:
 * targets[b,t] is the token that position t is scored against (ids[b,t+1]
 * for the shifted loss); any negative target is ignored. loss_out: one fp32,
 * the mean over positions with a target >= 0 (NaN and GPT2_ERR_NO_TARGETS in
 * the status word if there is none). */
int gpt2_loss(gpt2_handle_t h, const int32_t* ids, const int32_t* targets, int B, int T,
              float* loss_out, void* stream);

/* Both outputs in one pass: logits_or_null as in gpt2_forward, loss_out as
 * in gpt2_loss, and token_loss_or_null fp32 [B, T] with the loss of every
 * scored position (0 where the target is negative). */
int gpt2_forward_loss(gpt2_handle_t h, const int32_t* ids, const int32_t* targets, int B, int T,
                      float* logits_or_null, float* loss_out, float* token_loss_or_null,
                      void* stream);

/* Synchronise `stream`, return the first device-side error recorded since
 * the last call (GPT2_OK if none) and clear it. */
int gpt2_status(gpt2_handle_t h, void* stream);

/* Static description of an error code. */
const char* gpt2_error_string(int code);

/* Release the handle (host memory only; the workspace stays the caller's). */
void gpt2_destroy(gpt2_handle_t h);

/* Number of kernels this handle has launched so far (all calls). */
uint64_t gpt2_launch_count(gpt2_handle_t h);

/* Measurement hook: in every later gpt2_forward* / gpt2_loss call on h,
 * record ev_begin (a cudaEvent_t) on the call's stream just before the
 * launch of kernel `which` and ev_end just after it. which:
 * GPT2_TIMED_LMHEAD = the tied lm_head GEMM with the fused log-sum-exp.
 * NULL events switch the hook off. Returns GPT2_ERR_INVALID_ARG for an
 * unknown `which`. */
enum { GPT2_TIMED_LMHEAD = 0 };
int gpt2_set_timing_events(gpt2_handle_t h, int which, void* ev_begin, void* ev_end);

/* ------------------------------------------------------------------------
 * Single-step entry points. Each runs one step of the forward pass on its
 * own, with the same kernels gpt2_forward uses, so that every step can be
 * compared with the oracle separately. dtype is gpt2_dtype_t. `status` is
 * an int32 device word the kernels OR error bits into (may be NULL for
 * steps that cannot fail on the device).
 * ------------------------------------------------------------------------ */

/* x fp32 [M, C] = wte[ids[m]] + wpe[m % T] (wte/wpe of `dtype`). Ids outside
 * [0, V) read row 0 and set GPT2_ERR_BAD_TOKEN in *status. */
int gpt2_op_embed(int dtype, const int32_t* ids, const void* wte, const void* wpe,
                  int M, int T, int C, int V, float* x, int* status, void* stream);

/* out [M, C] (`dtype`) = LayerNorm(x fp32 [M, C]; g, b of `dtype`), biased
 * variance, eps 1e-5. C must be a multiple of 8 and <= 2048. */
int gpt2_op_layernorm(int dtype, const float* x, const void* g, const void* b,
                      int M, int C, void* out, void* stream);

/* Linear layer y = A W^T + bias with A [M, K], W [N, K], bias [N], all of
 * `dtype`, and one of four epilogues:
 *   GPT2_EPI_BIAS             out [M, N] (`dtype`) = y
 *   GPT2_EPI_BIAS_GELU        out [M, N] (`dtype`) = gelu_erf(y)
 *   GPT2_EPI_BIAS_RESID       out fp32 [M, N] += y    (residual add in place)
 *   GPT2_EPI_BIAS_GELU_TANH   out [M, N] (`dtype`) = gelu_tanh(y) (see GPT2_FLAG_GELU_TANH)
 * K and N must be multiples of 8 (bf16: K a multiple of 64). */
enum { GPT2_EPI_BIAS = 0, GPT2_EPI_BIAS_GELU = 1, GPT2_EPI_BIAS_RESID = 2, GPT2_EPI_BIAS_GELU_TANH = 3 };
int gpt2_op_linear(int dtype, int epilogue, const void* A, const void* W, const void* bias,
                   int M, int N, int K, void* out, int* status, void* stream);

/* The bf16 forward pass (M > 16) computes the embedding sum and the first
 * block's ln_1 in one kernel ("Hand-writing GPT-2 from scratch: the
 * Transformer decoder core modules in PyTorch", section 4.1 step 1 then the
 * Pre-LN block of section 3.2): x fp32 [M, C] = wte[ids] + wpe[m % T] as
 * gpt2_op_embed writes it, and h bf16 [M, C] = LayerNorm(x; g, b). bf16
 * tables and g, b; C a multiple of 64 and <= 2048. Ids outside [0, V) read
 * row 0 and set GPT2_ERR_BAD_TOKEN in *status. */
int gpt2_op_embed_layernorm(const int32_t* ids, const void* wte, const void* wpe, int M, int T, int C, int V,
                            const void* g, const void* b, float* x, void* h, int* status, void* stream);

/* ---- incremental decoding with a key/value cache ---------------------------
 * The pages' generate loops feed the sequence back one new token at a time
 * and keep every layer's keys and values of the earlier positions
 * ("Hand-writing GPT-2 from scratch: the Transformer decoder core modules in
 * PyTorch", section 6.3, past_key_values; "GPT-2 model development in
 * practice: from principles to deployment", section 4.1). With the cache, a
 * new position costs one row through every Linear and one query against the
 * cached keys, and its logits equal row `pos` of the full forward over
 * positions 0..pos.
 *
 * Cache layout, `dtype` elements: [n_layer][max_B][n_ctx][2C], position t of
 * sequence b of layer l holding k (C values, heads concatenated) then v (C
 * values). max_B is the one given to gpt2_create; the caller allocates the
 * cache (gpt2_kv_cache_bytes with that max_B, 0 for a bad config) and owns
 * it. Both calls below take the cache's size in bytes and return
 * GPT2_ERR_WORKSPACE, before any launch, when it is smaller than the layout
 * of the handle needs (a cache sized for a smaller max_B than the handle's). */
size_t gpt2_kv_cache_bytes(const gpt2_config_t* cfg, int max_B);

/* The forward pass of gpt2_forward over ids [B, T] that also stores every
 * layer's k and v of positions 0..T-1 of each sequence in the cache of
 * kv_bytes bytes. logits_or_null as in gpt2_forward. */
int gpt2_prefill(gpt2_handle_t h, void* kv_cache, size_t kv_bytes, const int32_t* ids, int B, int T,
                 float* logits_or_null, void* stream);

/* One new token per sequence at position pos (0 <= pos < n_ctx): ids_new
 * int32 [B]; the cache (kv_bytes bytes) must hold positions 0..pos-1 of these
 * B sequences (from gpt2_prefill or earlier steps). Stores the new position's
 * k and v in the cache and writes logits fp32 [B, vocab] of the new position.
 * GPT2_ERR_UNSUPPORTED if pos >= n_ctx; GPT2_ERR_INVALID_ARG if B > max_B. */
int gpt2_decode_step(gpt2_handle_t h, void* kv_cache, size_t kv_bytes, const int32_t* ids_new, int B, int pos,
                     float* logits, void* stream);

/* Fixed sinusoidal position table ("Hand-writing GPT-2 from scratch: the
 * Transformer decoder core modules in PyTorch", section 3.1, a variant the
 * other pages do not use: they learn wpe): for pos in [0, n_ctx) and i in
 * [0, C/2),
 *   wpe[pos, 2i]     = sin(pos / 10000^(2i / C))
 *   wpe[pos, 2i + 1] = cos(pos / 10000^(2i / C)),
 * evaluated in double precision and rounded once to `dtype`. wpe is a device
 * array [n_ctx, C] of `dtype`, C even; it can then be passed as the model's
 * wpe. Returns GPT2_OK or an error code; asynchronous on `stream`. */
int gpt2_fill_sinusoidal_wpe(int dtype, void* wpe, int n_ctx, int C, void* stream);

/* Causal multi-head self-attention. qkv [B*T, 3C] (`dtype`, columns q | k | v,
 * head h at columns h*D..h*D+D-1 of each) -> y [B*T, C] (`dtype`), heads
 * concatenated. D = C / H must be 32 or 64. The bf16, D = 64 kernel schedules
 * its work through a pair of counters that the library keeps per device, so
 * calls of this entry point on one device must not overlap on the GPU (the
 * model's own forward passes use counters in their workspace instead). */
int gpt2_op_attention(int dtype, const void* qkv, int B, int T, int H, int C, void* y,
                      int* status, void* stream);

/* Tied lm_head plus fused cross-entropy on a final hidden state.
 * hf [M, C] and wte [V, C] of `dtype`; targets int32 [M] (negative =
 * ignored). Writes logits fp32 [M, V] if logits_or_null, the per-position
 * losses to token_loss_or_null fp32 [M], and the mean to loss_out (fp32, may
 * be NULL). Scratch: `workspace` (device, 256-byte aligned) of at least
 * gpt2_op_lmhead_ce_workspace_bytes(dtype, M, V) bytes, caller-owned. */
size_t gpt2_op_lmhead_ce_workspace_bytes(int dtype, int M, int V);
int gpt2_op_lmhead_ce(int dtype, const void* hf, const void* wte, const int32_t* targets,
                      int M, int C, int V, float* logits_or_null, float* token_loss_or_null,
                      float* loss_out, void* workspace, size_t ws_bytes, int* status,
                      void* stream);

/* Allocation-free variant of gpt2_op_lmhead_ce. There is no counterpart in
 * the pages: this exists for callers that cannot call cudaMalloc, such as a
 * plugin inside a host application that owns every device allocation, or a
 * latency-critical path on which cudaMalloc's implicit device
 * synchronisation is not acceptable. Same arguments and results as
 * gpt2_op_lmhead_ce, minus the workspace: the scratch is a fixed device
 * array of GPT2_NOALLOC_SCRATCH_BYTES inside this library, held on every GPU
 * that loads the library until the process exits. A call needs
 * gpt2_op_lmhead_ce_workspace_bytes(dtype, M, V) of it (about
 * 8 * (ceil(V / 64) + 4) bytes per row; V = 50257 allows up to 5309 rows); larger
 * requests return GPT2_ERR_SCRATCH_LIMIT before any launch. The first call
 * on each device performs a one-time set-up there (it looks up the array's
 * device address, reads the SM count and sets kernel attributes), so make
 * that first call before any stream capture. All calls share the one array
 * and it keeps the last call's contents (no part of it needs to start at
 * zero): calls whose kernels overlap on the GPU race on it, so order them on
 * one stream. Never allocates device memory. */
#define GPT2_NOALLOC_SCRATCH_BYTES (32u << 20)
int gpt2_op_lmhead_ce_noalloc(int dtype, const void* hf, const void* wte, const int32_t* targets,
                              int M, int C, int V, float* logits_or_null,
                              float* token_loss_or_null, float* loss_out, int* status,
                              void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_H */
