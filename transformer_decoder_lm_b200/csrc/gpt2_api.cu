// gpt2_api.cu - the C ABI (include/gpt2.h): argument checks, workspace
// planning and the per-call schedule of the forward pass.
//
// Schedule of one forward ("Hand-writing GPT-2 from scratch: the Transformer
// decoder core modules in PyTorch", section 4.1, GPT2Model.forward; section
// 3.2, the Pre-LN block):
//   embed -> [ ln_1 -> c_attn(+b) -> attention -> c_proj(+b, += x)
//              -> ln_2 -> c_fc(+b, gelu) -> c_proj(+b, += x) ] x n_layer
//   -> ln_f -> lm_head (tied wte, fused log-sum-exp partials, optional logits)
//   -> cross-entropy finish.
// bf16 mode runs the GEMMs on tcgen05 (gemm_tc.cu) and attention on the
// tensor cores (attention.cu); fp32 mode runs the same schedule on fp32 SIMT
// kernels. All launches go to the caller's stream; nothing synchronises.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "gpt2.h"
#include "decode.h"
#include "kernels.h"
#include "model.h"

using namespace g2;

namespace {

Plan plan_workspace(const gpt2_config_t& c, int max_B, int max_T) {
  const long M = (long)max_B * max_T;
  const size_t es = c.dtype == GPT2_BF16 ? 2 : 4;
  const size_t C = (size_t)c.n_embd;
  const size_t n_tiles = lmhead_groups_max(c.vocab);
  Plan p;
  size_t o = 0;
  p.x = o;      o += align256(M * C * 4);
  p.h = o;      o += align256(M * C * es);
  p.qkv = o;    o += align256(M * 3 * C * es);
  p.y = o;      o += align256(M * C * es);
  p.f = o;      o += align256(M * 4 * C * es);
  p.part = o;   o += align256(n_tiles * M * sizeof(float2));
  p.tgt = o;    o += align256(M * 4);
  p.tok = o;    o += align256(M * 4);
  // attention split scratch: a flag block (zeroed at create) then the partials
  p.attn_pairs = 0;
  if (c.dtype == GPT2_BF16 && c.n_embd / c.n_head == 64)
    p.attn_pairs = (int)(attention_scratch_bytes(max_B, max_T, c.n_head) / (ATTN_PART_FLOATS * 4 + ATTN_PAIR_FLAGS * 4));
  p.attn_flags = o; o += align256((size_t)p.attn_pairs * ATTN_PAIR_FLAGS * 4);
  p.attn = o;   o += align256((size_t)p.attn_pairs * ATTN_PART_FLOATS * 4);
  p.status = o; o += 256;
  p.total = o;
  return p;
}

int check_config(const gpt2_config_t* c) {
  if (!c) return GPT2_ERR_INVALID_ARG;
  if (c->n_layer < 1 || c->n_head < 1 || c->n_embd < 1 || c->vocab < 1 || c->n_ctx < 1) return GPT2_ERR_INVALID_ARG;
  if (c->dtype != GPT2_BF16 && c->dtype != GPT2_FP32) return GPT2_ERR_INVALID_ARG;
  if (c->flags & ~GPT2_FLAG_GELU_TANH) return GPT2_ERR_INVALID_ARG;
  if (c->n_embd % c->n_head) return GPT2_ERR_UNSUPPORTED;
  const int D = c->n_embd / c->n_head;
  if (D != 32 && D != 64) return GPT2_ERR_UNSUPPORTED;
  if (c->n_embd > 2048 || (c->n_embd % 8)) return GPT2_ERR_UNSUPPORTED;
  if (c->dtype == GPT2_BF16 && (c->n_embd % 64)) return GPT2_ERR_UNSUPPORTED;
  return GPT2_OK;
}

struct DeviceInfo {
  int num_sms = 0;
  bool attrs = false;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

int device_setup(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPT2_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.attrs) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return GPT2_ERR_CUDA;
    if (gemm_tc_set_attributes() != cudaSuccess) return GPT2_ERR_CUDA;
    d.num_sms = n;
    d.attrs = true;
  }
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = d.num_sms;
  return GPT2_OK;
}


}  // namespace


namespace {

// One Linear layer of the schedule.
// extra: the few-row GEMV's cache-append fields, or NULL.
int run_linear(gpt2_model* m, int epi, const void* A, const CUtensorMap* tmA, const void* W, const CUtensorMap* wmaps,
               const CUtensorMap* tmC, const void* bias, int M, int N, int K, void* out, long long ldo, cudaStream_t s,
               const GemmArgs* extra = nullptr) {
  GemmArgs a = extra ? *extra : GemmArgs{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.bias = bias;
  a.out = out;
  a.ldo = ldo;
  a.status = m->status;
  a.gelu_tanh = (m->cfg.flags & GPT2_FLAG_GELU_TANH) ? 1 : 0;
  a.b_const = 1;   // the Linear weights
  cudaError_t e;
  if (m->bf16 && M <= GEMV_MAX_M) {   // a few rows (decoding): one warp per output column
    e = gemv_bf16_launch(epi, A, W, a, s);
  } else if (m->bf16) {
    const GemmPick p = gemm_tc_pick(M, N, m->num_sms, epi);
    e = gemm_tc_launch(epi, p.bn, *tmA, wmaps[box_index(gemm_tc_b_box_rows(p))], *tmC, a, m->num_sms, s, LAYOUT_KK,
                       nullptr, p.pair);
  } else {
    e = gemm_simt_launch(epi, static_cast<const float*>(A), static_cast<const float*>(W), a, s);
  }
  return e == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
}

// Bytes of one layer's slice of a key/value cache: [max_B][n_ctx][2C].
size_t kv_layer_bytes(const gpt2_model* m) {
  const size_t es = m->bf16 ? 2 : 4;
  return (size_t)m->max_B * m->cfg.n_ctx * 2 * m->cfg.n_embd * es;
}

int run_forward(gpt2_model* m, const int32_t* ids, const int32_t* targets, int B, int T, float* logits,
                float* loss_out, float* tok_out, cudaStream_t s, void* kv_cache = nullptr) {
  if (!m || !ids || B < 1 || T < 1) return GPT2_ERR_INVALID_ARG;
  if (B > m->max_B || T > m->max_T) return GPT2_ERR_INVALID_ARG;
  if (T > m->cfg.n_ctx) return GPT2_ERR_UNSUPPORTED;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return GPT2_ERR_CUDA;
  if (cur != m->device && cudaSetDevice(m->device) != cudaSuccess) return GPT2_ERR_CUDA;

  const gpt2_config_t& c = m->cfg;
  const int M = B * T, C = c.n_embd, H = c.n_head, V = c.vocab;
  CUtensorMap tm_h, tm_y, tm_f, out_qkv, out_f, out_x;
  if (m->bf16) {
    if (!make_tmap_bf16(&tm_h, m->h, M, C, C, 128) || !make_tmap_bf16(&tm_y, m->y, M, C, C, 128) ||
        !make_tmap_bf16(&tm_f, m->f, M, 4 * C, 4 * C, 128) ||
        !make_tmap_out_bf16(&out_qkv, m->qkv, M, 3 * C, 3 * C) || !make_tmap_out_bf16(&out_f, m->f, M, 4 * C, 4 * C) ||
        !make_tmap_out_f32(&out_x, m->x, M, C, C))
      return GPT2_ERR_CUDA;
  }
  int rc = GPT2_OK;
#define G2_CK(expr)                                  \
  do {                                               \
    if ((expr) != cudaSuccess) return GPT2_ERR_CUDA; \
  } while (0)
#define G2_RC(expr)                  \
  do {                               \
    rc = (expr);                     \
    if (rc != GPT2_OK) return rc;    \
  } while (0)

  // bf16 on the tensor cores: the first block's ln_1 rides on the embedding
  // kernel; every other LayerNorm is a launch of its own
  const bool fused_ln = m->bf16 && M > GEMV_MAX_M;
  if (fused_ln) {
    const LayerPtrs& L0 = m->layers[0];
    G2_CK(embed_ln_launch(ids, m->wte, m->wpe, m->x, L0.ln1_g, L0.ln1_b, m->h, M, T, C, V, m->status, s));
  } else {
    G2_CK(embed_launch(m->bf16, ids, m->wte, m->wpe, m->x, M, T, C, V, m->status, s));
  }
  m->launches += 1;
  for (int l = 0; l < c.n_layer; ++l) {
    const LayerPtrs& L = m->layers[l];
    const WeightMaps* W = m->bf16 ? &m->maps[l] : nullptr;
    if (l > 0 || !fused_ln) {
      G2_CK(layernorm_launch(m->bf16, m->x, L.ln1_g, L.ln1_b, m->h, M, C, s));
      m->launches += 1;
    }
    G2_RC(run_linear(m, EPI_BIAS, m->h, &tm_h, L.attn_w, W ? W->attn : nullptr, &out_qkv, L.attn_b, M, 3 * C, C, m->qkv, 3 * C, s));
    if (kv_cache) {   // k and v of positions 0..T-1 of every sequence into this layer's cache
      const size_t es = m->bf16 ? 2 : 4;
      uint8_t* cl = static_cast<uint8_t*>(kv_cache) + (size_t)l * kv_layer_bytes(m);
      for (int b = 0; b < B; ++b)
        G2_CK(cudaMemcpy2DAsync(cl + (size_t)b * c.n_ctx * 2 * C * es, 2 * C * es,
                                static_cast<uint8_t*>(m->qkv) + ((size_t)b * T * 3 * C + C) * es, 3 * C * es,
                                2 * C * es, T, cudaMemcpyDeviceToDevice, s));
    }
    G2_CK(attention_launch(m->bf16, m->qkv, m->y, B, T, H, C, &m->attn, m->status, s));
    G2_RC(run_linear(m, EPI_RESID, m->y, &tm_y, L.attn_proj_w, W ? W->proj : nullptr, &out_x, L.attn_proj_b, M, C, C, m->x, C, s));
    G2_CK(layernorm_launch(m->bf16, m->x, L.ln2_g, L.ln2_b, m->h, M, C, s));
    G2_RC(run_linear(m, EPI_GELU, m->h, &tm_h, L.fc_w, W ? W->fc : nullptr, &out_f, L.fc_b, M, 4 * C, C, m->f, 4 * C, s));
    G2_RC(run_linear(m, EPI_RESID, m->f, &tm_f, L.mlp_proj_w, W ? W->mproj : nullptr, &out_x, L.mlp_proj_b, M, C, 4 * C, m->x, C, s));
    m->launches += 6;
  }
  G2_CK(layernorm_launch(m->bf16, m->x, m->lnf_g, m->lnf_b, m->h, M, C, s));
  m->launches += 1;

  if (logits || targets) {
    GemmArgs a{};
    a.M = M;
    a.N = V;
    a.K = C;
    a.bias = nullptr;
    a.out = logits;
    a.ldo = V;
    a.targets = targets;
    a.part = m->part;
    a.tgt_logit = m->tgt;
    a.status = m->status;
    a.b_const = 1;   // wte
    int n_tiles;
    if (m->ev_lm_begin) G2_CK(cudaEventRecord(m->ev_lm_begin, s));
    if (m->bf16) {
      const GemmPick p = lmhead_pick(M, V, m->num_sms);
      n_tiles = gemm_tc_n_tiles(V, p.bn);
      G2_CK(gemm_tc_launch(EPI_LMHEAD, p.bn, tm_h, m->wte_map[box_index(gemm_tc_b_box_rows(p))], tm_h, a,
                           m->num_sms, s, LAYOUT_KK, nullptr, p.pair));
    } else {
      n_tiles = (V + SIMT_BN - 1) / SIMT_BN;
      G2_CK(gemm_simt_launch(EPI_LMHEAD, static_cast<const float*>(m->h), static_cast<const float*>(m->wte), a, s));
    }
    if (m->ev_lm_end) G2_CK(cudaEventRecord(m->ev_lm_end, s));
    m->launches += 1;
    if (targets) {
      G2_CK(ce_finish_launch(m->part, n_tiles, m->tgt, targets, M, V, tok_out ? tok_out : m->tok, loss_out,
                             m->status, s));
      m->launches += loss_out ? 2 : 1;
    }
  }
#undef G2_CK
#undef G2_RC
  return rc;
}

// One new token per sequence at position pos, against the key/value cache
// (gpt2_decode_step): every row-wise step of run_forward on B rows, the new
// k and v stored at `pos`, attention of the one query over positions 0..pos.
int run_decode(gpt2_model* m, void* kv_cache, const int32_t* ids, int B, int pos, float* logits, cudaStream_t s) {
  if (!m || !kv_cache || !ids || !logits || B < 1 || B > m->max_B || pos < 0) return GPT2_ERR_INVALID_ARG;
  if (pos >= m->cfg.n_ctx) return GPT2_ERR_UNSUPPORTED;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return GPT2_ERR_CUDA;
  if (cur != m->device && cudaSetDevice(m->device) != cudaSuccess) return GPT2_ERR_CUDA;
  const gpt2_config_t& c = m->cfg;
  const int M = B, C = c.n_embd, H = c.n_head, V = c.vocab;
  const size_t es = m->bf16 ? 2 : 4;
  CUtensorMap tm_h, tm_y, tm_f, out_qkv, out_f, out_x;
  if (m->bf16) {
    if (!make_tmap_bf16(&tm_h, m->h, M, C, C, 128) || !make_tmap_bf16(&tm_y, m->y, M, C, C, 128) ||
        !make_tmap_bf16(&tm_f, m->f, M, 4 * C, 4 * C, 128) ||
        !make_tmap_out_bf16(&out_qkv, m->qkv, M, 3 * C, 3 * C) || !make_tmap_out_bf16(&out_f, m->f, M, 4 * C, 4 * C) ||
        !make_tmap_out_f32(&out_x, m->x, M, C, C))
      return GPT2_ERR_CUDA;
  }
  int rc = GPT2_OK;
#define G2_CK(expr)                                  \
  do {                                               \
    if ((expr) != cudaSuccess) return GPT2_ERR_CUDA; \
  } while (0)
#define G2_RC(expr)                  \
  do {                               \
    rc = (expr);                     \
    if (rc != GPT2_OK) return rc;    \
  } while (0)
  // bf16 with a few rows: the GEMV path, whose c_attn also appends to the cache
  const bool gemv = m->bf16 && M <= GEMV_MAX_M;
  // x = wte[id] + wpe[pos]: the embedding of one position per row
  const void* wpe_pos = static_cast<const uint8_t*>(m->wpe) + (size_t)pos * C * es;
  G2_CK(embed_launch(m->bf16, ids, m->wte, wpe_pos, m->x, M, 1, C, V, m->status, s));
  for (int l = 0; l < c.n_layer; ++l) {
    const LayerPtrs& L = m->layers[l];
    const WeightMaps* W = m->bf16 ? &m->maps[l] : nullptr;
    uint8_t* cl = static_cast<uint8_t*>(kv_cache) + (size_t)l * kv_layer_bytes(m);
    G2_CK(layernorm_launch(m->bf16, m->x, L.ln1_g, L.ln1_b, m->h, M, C, s));
    if (gemv) {
      // the c_attn GEMV's k and v columns also go to position pos of each
      // sequence in the cache
      GemmArgs e{};
      e.kv = cl + (size_t)pos * 2 * C * es;
      e.ld_kv = (long long)c.n_ctx * 2 * C;
      e.kv_col0 = C;
      G2_RC(run_linear(m, EPI_BIAS, m->h, &tm_h, L.attn_w, W ? W->attn : nullptr, &out_qkv, L.attn_b, M, 3 * C, C,
                       m->qkv, 3 * C, s, &e));
    } else {
      G2_RC(run_linear(m, EPI_BIAS, m->h, &tm_h, L.attn_w, W ? W->attn : nullptr, &out_qkv, L.attn_b, M, 3 * C, C,
                       m->qkv, 3 * C, s));
      // the new k and v at position pos of each sequence
      G2_CK(cudaMemcpy2DAsync(cl + (size_t)pos * 2 * C * es, (size_t)c.n_ctx * 2 * C * es,
                              static_cast<uint8_t*>(m->qkv) + (size_t)C * es, 3 * C * es, 2 * C * es, B,
                              cudaMemcpyDeviceToDevice, s));
    }
    // the lm_head partials buffer is free until the end of the step: split-key scratch
    G2_CK(attention_decode_launch(m->bf16, m->qkv, cl, m->y, B, H, C, c.n_ctx, pos + 1,
                                  reinterpret_cast<float*>(m->part), (m->plan.tgt - m->plan.part) / sizeof(float), s));
    G2_RC(run_linear(m, EPI_RESID, m->y, &tm_y, L.attn_proj_w, W ? W->proj : nullptr, &out_x, L.attn_proj_b, M, C, C,
                     m->x, C, s));
    G2_CK(layernorm_launch(m->bf16, m->x, L.ln2_g, L.ln2_b, m->h, M, C, s));
    G2_RC(run_linear(m, EPI_GELU, m->h, &tm_h, L.fc_w, W ? W->fc : nullptr, &out_f, L.fc_b, M, 4 * C, C, m->f, 4 * C,
                     s));
    G2_RC(run_linear(m, EPI_RESID, m->f, &tm_f, L.mlp_proj_w, W ? W->mproj : nullptr, &out_x, L.mlp_proj_b, M, C,
                     4 * C, m->x, C, s));
    m->launches += 7;
  }
  G2_CK(layernorm_launch(m->bf16, m->x, m->lnf_g, m->lnf_b, m->h, M, C, s));
  GemmArgs a{};
  a.M = M;
  a.N = V;
  a.K = C;
  a.out = logits;
  a.ldo = V;
  a.part = m->part;
  a.tgt_logit = m->tgt;
  a.status = m->status;
  if (m->bf16) {
    const GemmPick p = lmhead_pick(M, V, m->num_sms);
    G2_CK(gemm_tc_launch(EPI_LMHEAD, p.bn, tm_h, m->wte_map[box_index(gemm_tc_b_box_rows(p))], tm_h, a, m->num_sms,
                         s, LAYOUT_KK, nullptr, p.pair));
  } else {
    G2_CK(gemm_simt_launch(EPI_LMHEAD, static_cast<const float*>(m->h), static_cast<const float*>(m->wte), a, s));
  }
  m->launches += 3;
#undef G2_CK
#undef G2_RC
  return rc;
}

}  // namespace

// =============================================================== public ABI

size_t g2::lmhead_ce_scratch_bytes(int M, int V) {
  return align256(lmhead_groups_max(V) * (size_t)M * sizeof(float2)) + 2 * align256((size_t)M * 4);
}

cudaError_t g2::lmhead_ce_launch(bool bf16, const void* hf, const void* wte, const int32_t* targets, int M, int C,
                                 int V, float* logits, float* token_loss, float* loss_out, void* scratch, int sms,
                                 int* status, cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  const size_t part_bytes = align256(lmhead_groups_max(V) * (size_t)M * sizeof(float2));
  float2* part = reinterpret_cast<float2*>(ws);
  float* tgt = reinterpret_cast<float*>(ws + part_bytes);
  float* tok = reinterpret_cast<float*>(ws + part_bytes + align256((size_t)M * 4));
  GemmArgs a{};
  a.M = M;
  a.N = V;
  a.K = C;
  a.out = logits;
  a.ldo = V;
  a.targets = targets;
  a.part = part;
  a.tgt_logit = tgt;
  a.status = status;
  int n_groups;
  cudaError_t e;
  if (bf16) {
    const GemmPick p = lmhead_pick(M, V, sms);
    n_groups = gemm_tc_n_tiles(V, p.bn);
    CUtensorMap ta, tb;
    if (!make_tmap_bf16(&ta, hf, M, C, C, 128) || !make_tmap_bf16(&tb, wte, V, C, C, gemm_tc_b_box_rows(p)))
      return cudaErrorInvalidValue;
    e = gemm_tc_launch(EPI_LMHEAD, p.bn, ta, tb, ta, a, sms, s, LAYOUT_KK, nullptr, p.pair);
  } else {
    n_groups = (V + SIMT_BN - 1) / SIMT_BN;
    e = gemm_simt_launch(EPI_LMHEAD, static_cast<const float*>(hf), static_cast<const float*>(wte), a, s);
  }
  if (e != cudaSuccess) return e;
  return ce_finish_launch(part, n_groups, tgt, targets, M, V, token_loss ? token_loss : tok, loss_out, status, s);
}

extern "C" {

size_t gpt2_workspace_bytes(const gpt2_config_t* cfg, int max_B, int max_T) {
  if (check_config(cfg) != GPT2_OK || max_B < 1 || max_T < 1) return 0;
  return plan_workspace(*cfg, max_B, max_T < cfg->n_ctx ? max_T : cfg->n_ctx).total;
}

int gpt2_create(const gpt2_config_t* cfg, const gpt2_weights_t* w, void* workspace, size_t ws_bytes, int max_B,
                int max_T, gpt2_handle_t* out) {
  if (!out) return GPT2_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_config(cfg);
  if (rc != GPT2_OK) return rc;
  if (!w || !workspace || max_B < 1 || max_T < 1) return GPT2_ERR_INVALID_ARG;
  if (max_T > cfg->n_ctx) max_T = cfg->n_ctx;
  const long maxM = (long)max_B * max_T;
  const Plan p = plan_workspace(*cfg, max_B, max_T);
  if (ws_bytes < p.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return GPT2_ERR_WORKSPACE;
  const int L = cfg->n_layer;
  const void* const* arrays[12] = {w->ln1_g, w->ln1_b, w->attn_w,  w->attn_b, w->attn_proj_w, w->attn_proj_b,
                                   w->ln2_g, w->ln2_b, w->fc_w,    w->fc_b,   w->mlp_proj_w,  w->mlp_proj_b};
  for (const void* const* a : arrays) {
    if (!a) return GPT2_ERR_INVALID_ARG;
    for (int l = 0; l < L; ++l)
      if (!aligned16(a[l])) return GPT2_ERR_INVALID_ARG;
  }
  if (!aligned16(w->wte) || !aligned16(w->wpe) || !aligned16(w->lnf_g) || !aligned16(w->lnf_b))
    return GPT2_ERR_INVALID_ARG;

  int dev = 0, sms = 0;
  rc = device_setup(&dev, &sms);
  if (rc != GPT2_OK) return rc;

  gpt2_model* m = new (std::nothrow) gpt2_model();
  if (!m) return GPT2_ERR_INVALID_ARG;
  m->cfg = *cfg;
  m->bf16 = cfg->dtype == GPT2_BF16;
  m->device = dev;
  m->num_sms = sms;
  m->max_B = max_B;
  m->max_T = max_T;
  m->max_M = maxM;
  m->wte = w->wte;
  m->wpe = w->wpe;
  m->lnf_g = w->lnf_g;
  m->lnf_b = w->lnf_b;
  m->layers.resize(L);
  for (int l = 0; l < L; ++l) {
    LayerPtrs& q = m->layers[l];
    q.ln1_g = w->ln1_g[l];
    q.ln1_b = w->ln1_b[l];
    q.attn_w = w->attn_w[l];
    q.attn_b = w->attn_b[l];
    q.attn_proj_w = w->attn_proj_w[l];
    q.attn_proj_b = w->attn_proj_b[l];
    q.ln2_g = w->ln2_g[l];
    q.ln2_b = w->ln2_b[l];
    q.fc_w = w->fc_w[l];
    q.fc_b = w->fc_b[l];
    q.mlp_proj_w = w->mlp_proj_w[l];
    q.mlp_proj_b = w->mlp_proj_b[l];
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  m->ws = ws;
  m->plan = p;
  m->x = reinterpret_cast<float*>(ws + p.x);
  m->h = ws + p.h;
  m->qkv = ws + p.qkv;
  m->y = ws + p.y;
  m->f = ws + p.f;
  m->part = reinterpret_cast<float2*>(ws + p.part);
  m->tgt = reinterpret_cast<float*>(ws + p.tgt);
  m->tok = reinterpret_cast<float*>(ws + p.tok);
  m->status = reinterpret_cast<int*>(ws + p.status);
  m->attn.sched = reinterpret_cast<unsigned*>(ws + p.status + 64);
  m->attn.flags = reinterpret_cast<int*>(ws + p.attn_flags);
  m->attn.part = reinterpret_cast<float*>(ws + p.attn);
  m->attn.cap_pairs = p.attn_pairs;

  if (m->bf16) {
    const int C = cfg->n_embd;
    m->maps.resize(L);
    bool ok = true;
    for (int i = 0; i < NUM_BOX && ok; ++i) {
      const uint32_t bn = BOX_ROWS[i];
      ok = ok && make_tmap_bf16(&m->wte_map[i], m->wte, cfg->vocab, C, C, bn);
      for (int l = 0; l < L && ok; ++l) {
        ok = ok && make_tmap_bf16(&m->maps[l].attn[i], m->layers[l].attn_w, 3 * C, C, C, bn);
        ok = ok && make_tmap_bf16(&m->maps[l].proj[i], m->layers[l].attn_proj_w, C, C, C, bn);
        ok = ok && make_tmap_bf16(&m->maps[l].fc[i], m->layers[l].fc_w, 4 * C, C, C, bn);
        ok = ok && make_tmap_bf16(&m->maps[l].mproj[i], m->layers[l].mlp_proj_w, C, 4 * C, 4 * C, bn);
      }
    }
    if (!ok) {
      delete m;
      return GPT2_ERR_CUDA;
    }
  }
  if (cudaMemset(m->status, 0, 256) != cudaSuccess ||
      (p.attn_pairs && cudaMemset(m->attn.flags, 0, (size_t)p.attn_pairs * ATTN_PAIR_FLAGS * 4) != cudaSuccess) ||
      cudaDeviceSynchronize() != cudaSuccess) {
    delete m;
    return GPT2_ERR_CUDA;
  }
  *out = m;
  return GPT2_OK;
}

int gpt2_forward(gpt2_handle_t h, const int32_t* ids, int B, int T, float* logits_or_null, void* stream) {
  return run_forward(h, ids, nullptr, B, T, logits_or_null, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

int gpt2_loss(gpt2_handle_t h, const int32_t* ids, const int32_t* targets, int B, int T, float* loss_out,
              void* stream) {
  if (!targets || !loss_out) return GPT2_ERR_INVALID_ARG;
  return run_forward(h, ids, targets, B, T, nullptr, loss_out, nullptr, static_cast<cudaStream_t>(stream));
}

int gpt2_forward_loss(gpt2_handle_t h, const int32_t* ids, const int32_t* targets, int B, int T,
                      float* logits_or_null, float* loss_out, float* token_loss_or_null, void* stream) {
  if (!targets || !loss_out) return GPT2_ERR_INVALID_ARG;
  return run_forward(h, ids, targets, B, T, logits_or_null, loss_out, token_loss_or_null,
                     static_cast<cudaStream_t>(stream));
}

size_t gpt2_kv_cache_bytes(const gpt2_config_t* cfg, int max_B) {
  if (check_config(cfg) != GPT2_OK || max_B < 1) return 0;
  const size_t es = cfg->dtype == GPT2_BF16 ? 2 : 4;
  return (size_t)cfg->n_layer * max_B * cfg->n_ctx * 2 * cfg->n_embd * es;
}

int gpt2_prefill(gpt2_handle_t h, void* kv_cache, size_t kv_bytes, const int32_t* ids, int B, int T,
                 float* logits_or_null, void* stream) {
  if (!h || !kv_cache || !aligned16(kv_cache)) return GPT2_ERR_INVALID_ARG;
  if (kv_bytes < (size_t)h->cfg.n_layer * kv_layer_bytes(h)) return GPT2_ERR_WORKSPACE;
  return run_forward(h, ids, nullptr, B, T, logits_or_null, nullptr, nullptr, static_cast<cudaStream_t>(stream),
                     kv_cache);
}

int gpt2_decode_step(gpt2_handle_t h, void* kv_cache, size_t kv_bytes, const int32_t* ids_new, int B, int pos,
                     float* logits, void* stream) {
  if (!h || !kv_cache || !aligned16(kv_cache)) return GPT2_ERR_INVALID_ARG;
  if (kv_bytes < (size_t)h->cfg.n_layer * kv_layer_bytes(h)) return GPT2_ERR_WORKSPACE;
  return run_decode(h, kv_cache, ids_new, B, pos, logits, static_cast<cudaStream_t>(stream));
}

int gpt2_status(gpt2_handle_t h, void* stream) {
  if (!h) return GPT2_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPT2_ERR_CUDA;
  int bits = 0;
  if (cudaMemcpy(&bits, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  if (bits && cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) return GPT2_ERR_CUDA;
  if (bits & DEV_TIMEOUT) return GPT2_ERR_DEVICE_TIMEOUT;
  if (bits & DEV_BAD_TOKEN) return GPT2_ERR_BAD_TOKEN;
  if (bits & DEV_NO_TARGETS) return GPT2_ERR_NO_TARGETS;
  return GPT2_OK;
}

const char* gpt2_error_string(int code) {
  switch (code) {
    case GPT2_OK: return "ok";
    case GPT2_ERR_INVALID_ARG: return "invalid argument";
    case GPT2_ERR_UNSUPPORTED: return "unsupported shape";
    case GPT2_ERR_CUDA: return "CUDA runtime error";
    case GPT2_ERR_WORKSPACE: return "workspace too small or misaligned";
    case GPT2_ERR_BAD_TOKEN: return "token id or target outside [0, vocab)";
    case GPT2_ERR_DEVICE_TIMEOUT: return "a bounded device wait timed out";
    case GPT2_ERR_NO_TARGETS: return "no position had a target";
    case GPT2_ERR_SCRATCH_LIMIT: return "request needs more than the fixed scratch of the allocation-free entry point";
  }
  return "unknown error";
}

void gpt2_destroy(gpt2_handle_t h) { delete h; }

uint64_t gpt2_launch_count(gpt2_handle_t h) { return h ? h->launches : 0; }

int gpt2_set_timing_events(gpt2_handle_t h, int which, void* ev_begin, void* ev_end) {
  if (!h || which != GPT2_TIMED_LMHEAD) return GPT2_ERR_INVALID_ARG;
  h->ev_lm_begin = static_cast<cudaEvent_t>(ev_begin);
  h->ev_lm_end = static_cast<cudaEvent_t>(ev_end);
  return GPT2_OK;
}

// ------------------------------------------------------ single-step entries

int gpt2_op_embed(int dtype, const int32_t* ids, const void* wte, const void* wpe, int M, int T, int C, int V,
                  float* x, int* status, void* stream) {
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || !ids || !aligned16(wte) || !aligned16(wpe) || !aligned16(x) ||
      M < 0 || T < 1 || C < 8 || (C % 8) || V < 1)
    return GPT2_ERR_INVALID_ARG;
  return embed_launch(dtype == GPT2_BF16, ids, wte, wpe, x, M, T, C, V, status, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

int gpt2_op_layernorm(int dtype, const float* x, const void* g, const void* b, int M, int C, void* out,
                      void* stream) {
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || !aligned16(x) || !aligned16(g) || !aligned16(b) ||
      !aligned16(out) || M < 0 || C < 8 || (C % 8) || C > 2048)
    return GPT2_ERR_INVALID_ARG;
  return layernorm_launch(dtype == GPT2_BF16, x, g, b, out, M, C, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

int gpt2_op_linear(int dtype, int epilogue, const void* A, const void* W, const void* bias, int M, int N, int K,
                   void* out, int* status, void* stream) {
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || epilogue < 0 || epilogue > 3 || !aligned16(A) || !aligned16(W) ||
      !aligned16(bias) || !aligned16(out) || M < 0 || N < 8 || K < 8 || (N % 8) || (K % 8))
    return GPT2_ERR_INVALID_ARG;
  if (M == 0) return GPT2_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.bias = bias;
  a.out = out;
  a.ldo = N;
  a.status = status;
  if (epilogue == GPT2_EPI_BIAS_GELU_TANH) {   // the GELU epilogue with the tanh form
    epilogue = EPI_GELU;
    a.gelu_tanh = 1;
  }
  if (dtype == GPT2_FP32)
    return gemm_simt_launch(epilogue, static_cast<const float*>(A), static_cast<const float*>(W), a, s) == cudaSuccess
               ? GPT2_OK
               : GPT2_ERR_CUDA;
  if (K % 64) return GPT2_ERR_UNSUPPORTED;
  if (M <= GEMV_MAX_M)
    return gemv_bf16_launch(epilogue, A, W, a, s) == cudaSuccess ? GPT2_OK : GPT2_ERR_CUDA;
  int sms = 0;
  int rc = device_setup(nullptr, &sms);
  if (rc != GPT2_OK) return rc;
  const GemmPick p = gemm_tc_pick(M, N, sms, epilogue);
  CUtensorMap ta, tb, tc;
  if (!make_tmap_bf16(&ta, A, M, K, K, 128) || !make_tmap_bf16(&tb, W, N, K, K, gemm_tc_b_box_rows(p)))
    return GPT2_ERR_CUDA;
  const bool ok_c = epilogue == GPT2_EPI_BIAS_RESID ? make_tmap_out_f32(&tc, out, M, N, N)
                                                     : make_tmap_out_bf16(&tc, out, M, N, N);
  if (!ok_c) return GPT2_ERR_CUDA;
  return gemm_tc_launch(epilogue, p.bn, ta, tb, tc, a, sms, s, LAYOUT_KK, nullptr, p.pair) == cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

int gpt2_op_embed_layernorm(const int32_t* ids, const void* wte, const void* wpe, int M, int T, int C, int V,
                            const void* g, const void* b, float* x, void* h, int* status, void* stream) {
  if (!ids || !aligned16(wte) || !aligned16(wpe) || !aligned16(g) || !aligned16(b) || !aligned16(x) || !aligned16(h) ||
      M < 0 || T < 1 || C < 64 || (C % 64) || C > 2048 || V < 1)
    return GPT2_ERR_INVALID_ARG;
  return embed_ln_launch(ids, wte, wpe, x, g, b, h, M, T, C, V, status, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

int gpt2_fill_sinusoidal_wpe(int dtype, void* wpe, int n_ctx, int C, void* stream) {
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || !wpe || n_ctx < 1 || C < 2 || (C % 2)) return GPT2_ERR_INVALID_ARG;
  return sinusoidal_wpe_launch(dtype == GPT2_BF16, wpe, n_ctx, C, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

int gpt2_op_attention(int dtype, const void* qkv, int B, int T, int H, int C, void* y, int* status, void* stream) {
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || !aligned16(qkv) || !aligned16(y) || B < 0 || T < 0 || H < 1 ||
      C < 8 || (C % 8) || (C % H))
    return GPT2_ERR_INVALID_ARG;
  const int D = C / H;
  if (D != 32 && D != 64) return GPT2_ERR_UNSUPPORTED;
  return attention_launch(dtype == GPT2_BF16, qkv, y, B, T, H, C, nullptr, status, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

size_t gpt2_op_lmhead_ce_workspace_bytes(int dtype, int M, int V) {
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || M < 1 || V < 1) return 0;
  return lmhead_ce_scratch_bytes(M, V);
}

int gpt2_op_lmhead_ce(int dtype, const void* hf, const void* wte, const int32_t* targets, int M, int C, int V,
                      float* logits_or_null, float* token_loss_or_null, float* loss_out, void* workspace,
                      size_t ws_bytes, int* status, void* stream) {
  if ((dtype != GPT2_BF16 && dtype != GPT2_FP32) || !aligned16(hf) || !aligned16(wte) || !targets || M < 1 || C < 8 ||
      (C % 8) || V < 1 || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return GPT2_ERR_INVALID_ARG;
  if (ws_bytes < gpt2_op_lmhead_ce_workspace_bytes(dtype, M, V)) return GPT2_ERR_WORKSPACE;
  int sms = 0;
  if (dtype == GPT2_BF16) {
    if (C % 64) return GPT2_ERR_UNSUPPORTED;
    const int rc = device_setup(nullptr, &sms);
    if (rc != GPT2_OK) return rc;
  }
  return lmhead_ce_launch(dtype == GPT2_BF16, hf, wte, targets, M, C, V, logits_or_null, token_loss_or_null, loss_out,
                          workspace, sms, status, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

}  // extern "C"
