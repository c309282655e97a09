// train.cu - the C ABI of the backward pass (include/gpt2_train.h): the
// training workspace plan, the forward pass that keeps its activations, the
// per-call schedule of the backward pass, and the single-step entry points.
//
// Schedule ("Hand-writing GPT-2 from scratch: the Transformer decoder core
// modules in PyTorch", section 4.3: loss.backward() after the forward of
// section 4.1), M = B T tokens:
//   forward: embed -> [ ln_1 (keeps x_in) -> c_attn -> attention (keeps the
//            row log-sum-exp) -> c_proj += x -> ln_2 (keeps x_mid) -> c_fc
//            (keeps u and gelu(u)) -> c_proj += x ] x L -> ln_f (keeps x_L)
//            -> lm_head log-sum-exp partials -> loss (keeps the row lse and
//            the scored count)
//   backward:
//     dz     = (softmax(z) - onehot) / n           lm_head GEMM, EPI_DLOGITS
//     dhf    = dz . wte                            dgrad (B MN-major)
//     dwte   = dz^T . hf                           wgrad (A, B MN-major)
//     dx     = ln_f'(dhf)                          layernorm_bwd
//     per layer, last first:
//       du  = (dx . W_mp) * gelu'(u)               dgrad, EPI_DGELU
//       dW_mp = dx^T f, db_mp = sum dx             wgrad, col_sum
//       dh2 = du . W_fc, dW_fc = du^T h2, db_fc    dgrad, wgrad, col_sum
//       dx += ln_2'(dh2)                           layernorm_bwd
//       dy  = dx . W_p, dW_p = dx^T y, db_p        dgrad, wgrad, col_sum
//       dqkv = attention'(dy)                      attention_bwd
//       dh1 = dqkv . W_a, dW_a = dqkv^T h1, db_a   dgrad, wgrad, col_sum
//       dx += ln_1'(dh1)                           layernorm_bwd
//     dwte[ids] += dx, dwpe = sum_b dx             embed_bwd
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "backward.h"
#include "common.cuh"
#include "decode.h"
#include "gpt2.h"
#include "gpt2_train.h"
#include "kernels.h"
#include "model.h"

using namespace g2;

namespace {

inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Byte offsets of the training workspace.
struct TrainPlan {
  size_t per_layer;                                        // bytes of one layer's saved activations
  size_t x_in, h1, qkv, y, lse, x_mid, h2, u, f;           // offsets inside a layer block
  size_t layers, x_fin, hf, lse_ce, n_scored, dz, dh, dx, dxb, du, dy, dqkv, dq, dv, part, total;
};

TrainPlan plan_train(const gpt2_config_t& c, int max_B, int max_T) {
  const size_t M = (size_t)max_B * max_T, C = c.n_embd, H = c.n_head;
  const size_t Vp = (size_t)round_up(c.vocab, 64);
  TrainPlan p;
  size_t o = 0;
  p.x_in = o;  o += align256(M * C * 4);
  p.h1 = o;    o += align256(M * C * 2);
  p.qkv = o;   o += align256(M * 3 * C * 2);
  p.y = o;     o += align256(M * C * 2);
  p.lse = o;   o += align256(M * H * 4);
  p.x_mid = o; o += align256(M * C * 4);
  p.h2 = o;    o += align256(M * C * 2);
  p.u = o;     o += align256(M * 4 * C * 2);
  p.f = o;     o += align256(M * 4 * C * 2);
  p.per_layer = o;
  o = 0;
  p.layers = o;   o += p.per_layer * c.n_layer;
  p.x_fin = o;    o += align256(M * C * 4);
  p.hf = o;       o += align256(M * C * 2);
  p.lse_ce = o;   o += align256(M * 4);
  p.n_scored = o; o += 256;
  p.dz = o;       o += align256(M * Vp * 2);
  p.dh = o;       o += align256(M * C * 4);
  p.dx = o;       o += align256(M * C * 4);
  p.dxb = o;      o += align256(M * C * 2);
  p.du = o;       o += align256(M * 4 * C * 2);
  p.dy = o;       o += align256(M * C * 2);
  p.dqkv = o;     o += align256(M * 3 * C * 2);
  p.dq = o;       o += align256(M * C * 4);
  p.dv = o;       o += align256(M * H * 4);
  p.part = o;     o += align256(layernorm_bwd_part_floats((int)M, (int)C, 4 * (int)C) * 4);
  p.total = o;
  return p;
}

bool train_supported(const gpt2_config_t* c) {
  return c && c->dtype == GPT2_BF16 && c->n_head > 0 && c->n_embd % c->n_head == 0 && c->n_embd / c->n_head == 64 &&
         c->n_embd % 64 == 0 && c->n_embd <= 2048;
}

// One tcgen05 GEMM. A and B are given with their storage: a_mn / b_mn =
// MN-major ([K, M] / [K, N] row-major), else K-major ([M, K] / [N, K]).
struct Gemm {
  int sms;
  int* status;
  cudaStream_t s;

  // b_rows: rows of an MN-major B in memory when fewer than K (the rest of
  // the K range reads as zero), e.g. wte's V rows against a K of V rounded up.
  int run(int epi, const void* A, bool a_mn, long long lda, const void* B, bool b_mn, long long ldb, void* out,
          long long ldo, bool out_f32, int M, int N, int K, const GemmArgs& extra = GemmArgs{},
          const void* out_d = nullptr, int b_rows = -1) const {
    const int layout = (a_mn ? LAYOUT_A_MN : 0) | (b_mn ? LAYOUT_B_MN : 0);
    GemmPick p = gemm_tc_pick(M, N, sms, epi == EPI_DLOGITS ? EPI_LMHEAD : epi, layout);
    // A weight gradient over many tokens (fp32 out, both operands MN-major)
    // may run as two K halves added into a zeroed output when twice its tiles
    // fit on the SMs: among the widths that allow that, the one with the
    // least estimated time (waves x K per item x the width's cost per
    // k-block, as in gemm_tc_pick), if it beats the pick without halves.
    const bool wgrad = epi == EPI_F32 && a_mn && b_mn && out_f32 && K >= 1024;
    bool halves = false;
    if (wgrad) {
      const int mt = (M + 127) / 128;
      auto cost = [&](int w, int split) {
        const long t = (long)mt * ((N + w - 1) / w) * split;
        const double unit = w == 256 ? 256.0 : (w == 192 ? 192.0 : (w == 128 ? 200.0 : 150.0));
        return (double)((t + sms - 1) / sms) * ((double)K / split) * unit;
      };
      double best = cost(p.bn, 1);
      for (int w : {256, 192, 128, 64}) {
        if (2L * mt * ((N + w - 1) / w) > sms) continue;
        if (cost(w, 2) < best) {
          best = cost(w, 2);
          p.bn = w;
          halves = true;
        }
      }
    }
    const int bn = p.bn;
    CUtensorMap ta, tb, tc, td;
    const bool ok_a = a_mn ? make_tmap_bf16(&ta, A, K, M, lda, 64) : make_tmap_bf16(&ta, A, M, K, lda, 128);
    const bool ok_b = b_mn ? make_tmap_bf16(&tb, B, b_rows > 0 ? std::min(b_rows, K) : K, N, ldb, 64)
                           : make_tmap_bf16(&tb, B, N, K, ldb, gemm_tc_b_box_rows(p));
    const bool ok_c = out_f32 ? make_tmap_out_f32(&tc, out, M, N, ldo) : make_tmap_out_bf16(&tc, out, M, N, ldo);
    const bool ok_d = out_d == nullptr || make_tmap_out_bf16(&td, out_d, M, N, ldo);
    if (!ok_a || !ok_b || !ok_c || !ok_d) return GPT2_ERR_CUDA;
    GemmArgs a = extra;
    a.M = M;
    a.N = N;
    a.K = K;
    a.out = out;
    a.ldo = ldo;
    a.status = status;
    // the K range in two halves, both added into the zeroed output (0 + a + b:
    // the same bits in either order)
    if (halves) {
      a.k_split = 2;
      if (cudaMemset2DAsync(out, (size_t)ldo * 4, 0, (size_t)N * 4, M, s) != cudaSuccess) return GPT2_ERR_CUDA;
    }
    return gemm_tc_launch(epi, bn, ta, tb, tc, a, sms, s, layout, out_d ? &td : nullptr, p.pair) == cudaSuccess
               ? GPT2_OK
               : GPT2_ERR_CUDA;
  }
};

int sms_of_current_device() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

// gemm_tc kernels need their shared-memory attribute once per device.
int gemm_setup(int* sms) {
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPT2_ERR_CUDA;
  if (!done[dev]) {
    if (gemm_tc_set_attributes() != cudaSuccess) return GPT2_ERR_CUDA;
    done[dev] = true;
  }
  *sms = sms_of_current_device();
  return *sms > 0 ? GPT2_OK : GPT2_ERR_CUDA;
}

#define G2_CK(expr)                                  \
  do {                                               \
    if ((expr) != cudaSuccess) return GPT2_ERR_CUDA; \
  } while (0)
#define G2_RC(expr)                 \
  do {                              \
    const int rc_ = (expr);         \
    if (rc_ != GPT2_OK) return rc_; \
  } while (0)

int run_train(gpt2_model* m, const int32_t* ids, const int32_t* targets, int B, int T, float* loss_out,
              const gpt2_grads_t* gr, uint8_t* ws, cudaStream_t s) {
  const gpt2_config_t& c = m->cfg;
  const int M = B * T, C = c.n_embd, H = c.n_head, V = c.vocab, L = c.n_layer;
  const int Vp = round_up(V, 64);
  const TrainPlan p = plan_train(c, m->max_B, m->max_T);
  auto layer = [&](int l, size_t off) { return ws + p.layers + (size_t)l * p.per_layer + off; };
  float* x_fin = reinterpret_cast<float*>(ws + p.x_fin);
  void* hf = ws + p.hf;
  float* lse_ce = reinterpret_cast<float*>(ws + p.lse_ce);
  int* n_scored = reinterpret_cast<int*>(ws + p.n_scored);
  void* dz = ws + p.dz;
  float* dh = reinterpret_cast<float*>(ws + p.dh);
  float* dx = reinterpret_cast<float*>(ws + p.dx);
  void* dxb = ws + p.dxb;
  void* du = ws + p.du;
  void* dy = ws + p.dy;
  void* dqkv = ws + p.dqkv;
  float* dq = reinterpret_cast<float*>(ws + p.dq);
  float* dvec = reinterpret_cast<float*>(ws + p.dv);
  float* part = reinterpret_cast<float*>(ws + p.part);
  const Gemm gm{m->num_sms, m->status, s};
  const int gelu_tanh = (c.flags & GPT2_FLAG_GELU_TANH) ? 1 : 0;

  // ------------------------------------------------------------ forward
  G2_CK(embed_launch(true, ids, m->wte, m->wpe, m->x, M, T, C, V, m->status, s));
  for (int l = 0; l < L; ++l) {
    const LayerPtrs& w = m->layers[l];
    float* x_in = reinterpret_cast<float*>(layer(l, p.x_in));
    float* x_mid = reinterpret_cast<float*>(layer(l, p.x_mid));
    void *h1 = layer(l, p.h1), *qkv = layer(l, p.qkv), *y = layer(l, p.y), *h2 = layer(l, p.h2);
    void *u = layer(l, p.u), *f = layer(l, p.f);
    float* lse = reinterpret_cast<float*>(layer(l, p.lse));
    G2_CK(layernorm_launch(true, m->x, w.ln1_g, w.ln1_b, h1, M, C, s, x_in));
    GemmArgs ab{};
    ab.bias = w.attn_b;
    G2_RC(gm.run(EPI_BIAS, h1, false, C, w.attn_w, false, C, qkv, 3 * C, false, M, 3 * C, C, ab));
    G2_CK(attention_tc_launch(qkv, y, B, T, H, C, &m->attn, m->status, s, lse));
    GemmArgs ap{};
    ap.bias = w.attn_proj_b;
    G2_RC(gm.run(EPI_RESID, y, false, C, w.attn_proj_w, false, C, m->x, C, true, M, C, C, ap));
    G2_CK(layernorm_launch(true, m->x, w.ln2_g, w.ln2_b, h2, M, C, s, x_mid));
    GemmArgs af{};
    af.bias = w.fc_b;
    af.gelu_tanh = gelu_tanh;
    G2_RC(gm.run(EPI_GELU_SAVE, h2, false, C, w.fc_w, false, C, f, 4 * C, false, M, 4 * C, C, af, u));
    GemmArgs am{};
    am.bias = w.mlp_proj_b;
    G2_RC(gm.run(EPI_RESID, f, false, 4 * C, w.mlp_proj_w, false, 4 * C, m->x, C, true, M, C, 4 * C, am));
  }
  G2_CK(layernorm_launch(true, m->x, m->lnf_g, m->lnf_b, hf, M, C, s, x_fin));
  {
    GemmArgs a{};
    a.targets = targets;
    a.part = m->part;
    a.tgt_logit = m->tgt;
    const GemmPick p = lmhead_pick(M, V, m->num_sms);
    CUtensorMap ta;
    if (!make_tmap_bf16(&ta, hf, M, C, C, 128)) return GPT2_ERR_CUDA;
    a.M = M;
    a.N = V;
    a.K = C;
    a.status = m->status;
    G2_CK(gemm_tc_launch(EPI_LMHEAD, p.bn, ta, m->wte_map[box_index(gemm_tc_b_box_rows(p))], ta, a, m->num_sms, s,
                         LAYOUT_KK, nullptr, p.pair));
    G2_CK(ce_finish_launch(m->part, gemm_tc_n_tiles(V, p.bn), m->tgt, targets, M, V, m->tok, loss_out, m->status, s,
                           lse_ce, n_scored));
  }

  // ----------------------------------------------------------- backward
  {
    GemmArgs a{};
    a.targets = targets;
    a.row_lse = lse_ce;
    a.n_scored = n_scored;
    // dz [M, Vp]: columns V..Vp-1 come out 0 (the epilogue zeroes columns >= V)
    G2_RC(gm.run(EPI_DLOGITS, hf, false, C, m->wte, false, C, dz, Vp, false, M, V, C, a));
    // the TMA store clips at column V of the map: clear the padding columns once
    if (Vp > V) G2_CK(cudaMemset2DAsync(static_cast<uint8_t*>(dz) + (size_t)V * 2, (size_t)Vp * 2, 0,
                                        (size_t)(Vp - V) * 2, M, s));
  }
  G2_RC(gm.run(EPI_F32, dz, false, Vp, m->wte, true, C, dh, C, true, M, C, Vp, GemmArgs{}, nullptr, V));   // dhf = dz . wte
  G2_RC(gm.run(EPI_F32, dz, true, Vp, hf, true, C, gr->wte, C, true, V, C, M));            // dwte = dz^T . hf
  // LayerNorm gradients; each also sums its dx over the rows (the bias
  // gradient of the residual projection above it) and the bias gradient of
  // the Linear layer whose output gradient is given as z
  auto ln_bwd = [&](const float* x, const void* g, const float* dx_in, const void* z, int nz, float* dgamma,
                    float* dbeta, float* dsum, float* dzsum) {
    LnBwdArgs a{};
    a.x = x;
    a.gamma = static_cast<const bf16*>(g);
    a.dh = dh;
    a.dx_in = dx_in;
    a.dx_out = dx;
    a.dx_bf16 = static_cast<bf16*>(dxb);
    a.z = static_cast<const bf16*>(z);
    a.nz = nz;
    a.part = part;
    a.M = M;
    a.C = C;
    return layernorm_bwd_launch(a, dgamma, dbeta, dsum, dzsum, s);
  };
  G2_CK(ln_bwd(x_fin, m->lnf_g, nullptr, nullptr, 0, gr->lnf_g, gr->lnf_b, gr->mlp_proj_b[L - 1], nullptr));
  for (int l = L - 1; l >= 0; --l) {
    const LayerPtrs& w = m->layers[l];
    const float* x_in = reinterpret_cast<const float*>(layer(l, p.x_in));
    const float* x_mid = reinterpret_cast<const float*>(layer(l, p.x_mid));
    const void *h1 = layer(l, p.h1), *qkv = layer(l, p.qkv), *y = layer(l, p.y), *h2 = layer(l, p.h2);
    const void *u = layer(l, p.u), *f = layer(l, p.f);
    const float* lse = reinterpret_cast<const float*>(layer(l, p.lse));
    // MLP: x_out = x_mid + c_proj(gelu(c_fc(ln_2(x_mid))))
    GemmArgs ag{};
    ag.aux = u;
    ag.ld_aux = 4 * C;
    ag.gelu_tanh = gelu_tanh;
    G2_RC(gm.run(EPI_DGELU, dxb, false, C, w.mlp_proj_w, true, 4 * C, du, 4 * C, false, M, 4 * C, C, ag));
    G2_RC(gm.run(EPI_F32, dxb, true, C, f, true, 4 * C, gr->mlp_proj_w[l], 4 * C, true, C, 4 * C, M));
    G2_RC(gm.run(EPI_F32, du, false, 4 * C, w.fc_w, true, C, dh, C, true, M, C, 4 * C));
    G2_RC(gm.run(EPI_F32, du, true, 4 * C, h2, true, C, gr->fc_w[l], C, true, 4 * C, C, M));
    G2_CK(ln_bwd(x_mid, w.ln2_g, dx, du, 4 * C, gr->ln2_g[l], gr->ln2_b[l], gr->attn_proj_b[l], gr->fc_b[l]));
    // attention: x_mid = x_in + c_proj(attn(c_attn(ln_1(x_in))))
    G2_RC(gm.run(EPI_BIAS, dxb, false, C, w.attn_proj_w, true, C, dy, C, false, M, C, C));
    G2_RC(gm.run(EPI_F32, dxb, true, C, y, true, C, gr->attn_proj_w[l], C, true, C, C, M));
    G2_CK(attention_bwd_launch(qkv, y, dy, lse, dvec, dq, dqkv, B, T, H, C, m->status, s));
    G2_RC(gm.run(EPI_F32, dqkv, false, 3 * C, w.attn_w, true, C, dh, C, true, M, C, 3 * C));
    G2_RC(gm.run(EPI_F32, dqkv, true, 3 * C, h1, true, C, gr->attn_w[l], C, true, 3 * C, C, M));
    G2_CK(ln_bwd(x_in, w.ln1_g, dx, dqkv, 3 * C, gr->ln1_g[l], gr->ln1_b[l], l > 0 ? gr->mlp_proj_b[l - 1] : nullptr,
                 gr->attn_b[l]));
  }
  G2_CK(embed_bwd_launch(ids, dx, gr->wte, gr->wpe, B, T, c.n_ctx, C, V, s));
  return GPT2_OK;
}

}  // namespace

extern "C" {

size_t gpt2_train_workspace_bytes(const gpt2_config_t* cfg, int max_B, int max_T) {
  if (!train_supported(cfg) || max_B < 1 || max_T < 1) return 0;
  return plan_train(*cfg, max_B, std::min(max_T, cfg->n_ctx)).total;
}

int gpt2_forward_backward(gpt2_handle_t h, const int32_t* ids, const int32_t* targets, int B, int T,
                          float* loss_out, const gpt2_grads_t* grads, void* train_ws, size_t train_ws_bytes,
                          void* stream) {
  if (!h || !ids || !targets || !loss_out || !grads || !train_ws || B < 1 || T < 1) return GPT2_ERR_INVALID_ARG;
  if (!train_supported(&h->cfg) || (long)B * T <= GEMV_MAX_M) return GPT2_ERR_UNSUPPORTED;
  if (B > h->max_B || T > h->max_T) return GPT2_ERR_INVALID_ARG;
  if (T > h->cfg.n_ctx) return GPT2_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(train_ws) & 255) || train_ws_bytes < plan_train(h->cfg, h->max_B, h->max_T).total)
    return GPT2_ERR_WORKSPACE;
  const gpt2_grads_t& g = *grads;
  const int L = h->cfg.n_layer;
  float** arrays[12] = {g.ln1_g, g.ln1_b, g.attn_w, g.attn_b, g.attn_proj_w, g.attn_proj_b,
                        g.ln2_g, g.ln2_b, g.fc_w,   g.fc_b,   g.mlp_proj_w,  g.mlp_proj_b};
  for (float** a : arrays) {
    if (!a) return GPT2_ERR_INVALID_ARG;
    for (int l = 0; l < L; ++l)
      if (!aligned16(a[l])) return GPT2_ERR_INVALID_ARG;
  }
  if (!aligned16(g.wte) || !aligned16(g.wpe) || !aligned16(g.lnf_g) || !aligned16(g.lnf_b))
    return GPT2_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return GPT2_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return GPT2_ERR_CUDA;
  return run_train(h, ids, targets, B, T, loss_out, grads, static_cast<uint8_t*>(train_ws),
                   static_cast<cudaStream_t>(stream));
}

int gpt2_op_linear_dgrad(const void* dy, const void* W, int M, int N, int K, void* dx, int out_f32, int* status,
                         void* stream) {
  if (!aligned16(dy) || !aligned16(W) || !aligned16(dx) || M < 1 || N < 8 || K < 8 || (N % 8) || (K % 8))
    return GPT2_ERR_INVALID_ARG;
  int sms = 0;
  G2_RC(gemm_setup(&sms));
  const Gemm gm{sms, status, static_cast<cudaStream_t>(stream)};
  return gm.run(out_f32 ? EPI_F32 : EPI_BIAS, dy, false, N, W, true, K, dx, K, out_f32 != 0, M, K, N);
}

int gpt2_op_linear_wgrad(const void* dy, const void* x, int M, int N, int K, float* dW, int* status, void* stream) {
  if (!aligned16(dy) || !aligned16(x) || !aligned16(dW) || M < 1 || N < 8 || K < 8 || (N % 8) || (K % 8))
    return GPT2_ERR_INVALID_ARG;
  int sms = 0;
  G2_RC(gemm_setup(&sms));
  const Gemm gm{sms, status, static_cast<cudaStream_t>(stream)};
  return gm.run(EPI_F32, dy, true, N, x, true, K, dW, K, true, N, K, M);
}

int gpt2_op_linear_dgrad_gelu(const void* dy, const void* W, const void* u, int M, int N, int K, int tanh_form,
                              void* du, int* status, void* stream) {
  if (!aligned16(dy) || !aligned16(W) || !aligned16(u) || !aligned16(du) || M < 1 || N < 8 || K < 8 || (N % 8) ||
      (K % 8))
    return GPT2_ERR_INVALID_ARG;
  int sms = 0;
  G2_RC(gemm_setup(&sms));
  const Gemm gm{sms, status, static_cast<cudaStream_t>(stream)};
  GemmArgs a{};
  a.aux = u;
  a.ld_aux = K;
  a.gelu_tanh = tanh_form ? 1 : 0;
  return gm.run(EPI_DGELU, dy, false, N, W, true, K, du, K, false, M, K, N, a);
}

size_t gpt2_op_layernorm_backward_workspace_bytes(int M, int C) {
  if (M < 1 || C < 4) return 0;
  return layernorm_bwd_part_floats(M, C, 0) * 4;
}

int gpt2_op_layernorm_backward(const float* x, const void* gamma, const float* dh, const float* dx_in, int M, int C,
                               float* dx_out, float* dgamma, float* dbeta, void* workspace, size_t ws_bytes,
                               void* stream) {
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(dh) || (dx_in && !aligned16(dx_in)) || !aligned16(dx_out) ||
      !dgamma || !dbeta || !aligned16(workspace) || M < 1 || C < 8 || (C % 8) || C > 2048)
    return GPT2_ERR_INVALID_ARG;
  if (ws_bytes < gpt2_op_layernorm_backward_workspace_bytes(M, C)) return GPT2_ERR_WORKSPACE;
  LnBwdArgs a{};
  a.x = x;
  a.gamma = static_cast<const bf16*>(gamma);
  a.dh = dh;
  a.dx_in = dx_in;
  a.dx_out = dx_out;
  a.part = static_cast<float*>(workspace);
  a.M = M;
  a.C = C;
  return layernorm_bwd_launch(a, dgamma, dbeta, nullptr, nullptr, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

int gpt2_op_attention_train(const void* qkv, int B, int T, int H, int C, void* y, float* lse2, int* status,
                            void* stream) {
  if (!aligned16(qkv) || !aligned16(y) || !lse2 || B < 1 || T < 1 || H < 1 || C % H || (C % 64))
    return GPT2_ERR_INVALID_ARG;
  if (C / H != 64) return GPT2_ERR_UNSUPPORTED;
  return attention_tc_launch(qkv, y, B, T, H, C, nullptr, status, static_cast<cudaStream_t>(stream), lse2) ==
                 cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

size_t gpt2_op_attention_backward_workspace_bytes(int B, int T, int H, int C) {
  if (B < 1 || T < 1 || H < 1 || C < 1) return 0;
  return align256((size_t)B * H * T * 4) + align256((size_t)B * T * C * 4);
}

int gpt2_op_attention_backward(const void* qkv, const void* y, const void* dy, const float* lse2, int B, int T, int H,
                               int C, void* dqkv, void* workspace, size_t ws_bytes, int* status, void* stream) {
  if (!aligned16(qkv) || !aligned16(y) || !aligned16(dy) || !lse2 || !aligned16(dqkv) || !workspace || B < 1 ||
      T < 1 || H < 1 || C % H || (C % 64) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return GPT2_ERR_INVALID_ARG;
  if (C / H != 64) return GPT2_ERR_UNSUPPORTED;
  if (ws_bytes < gpt2_op_attention_backward_workspace_bytes(B, T, H, C)) return GPT2_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* Dv = reinterpret_cast<float*>(w);
  float* dq = reinterpret_cast<float*>(w + align256((size_t)B * H * T * 4));
  return attention_bwd_launch(qkv, y, dy, lse2, Dv, dq, dqkv, B, T, H, C, status, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GPT2_OK
             : GPT2_ERR_CUDA;
}

size_t gpt2_op_lmhead_ce_backward_workspace_bytes(int M, int V) {
  if (M < 1 || V < 1) return 0;
  const size_t Vp = (size_t)round_up(V, 64);
  return align256(lmhead_groups_max(V) * (size_t)M * sizeof(float2)) + 3 * align256((size_t)M * 4) + 256 +
         align256((size_t)M * Vp * 2);
}

int gpt2_op_lmhead_ce_backward(const void* hf, const void* wte, const int32_t* targets, int M, int C, int V,
                               float* loss_out, float* dhf, float* dwte, void* workspace, size_t ws_bytes, int* status,
                               void* stream) {
  if (!aligned16(hf) || !aligned16(wte) || !targets || !loss_out || !aligned16(dhf) || !aligned16(dwte) ||
      !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || M < 1 || C < 64 || (C % 64) || V < 8 || (V % 8))
    return GPT2_ERR_INVALID_ARG;
  if (ws_bytes < gpt2_op_lmhead_ce_backward_workspace_bytes(M, V)) return GPT2_ERR_WORKSPACE;
  int sms = 0;
  G2_RC(gemm_setup(&sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int Vp = round_up(V, 64);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float2* part = reinterpret_cast<float2*>(w);
  w += align256(lmhead_groups_max(V) * (size_t)M * sizeof(float2));
  float* tgt = reinterpret_cast<float*>(w);
  w += align256((size_t)M * 4);
  float* tok = reinterpret_cast<float*>(w);
  w += align256((size_t)M * 4);
  float* lse = reinterpret_cast<float*>(w);
  w += align256((size_t)M * 4);
  int* n_scored = reinterpret_cast<int*>(w);
  w += 256;
  void* dz = w;
  GemmArgs a{};
  a.M = M;
  a.N = V;
  a.K = C;
  a.targets = targets;
  a.part = part;
  a.tgt_logit = tgt;
  a.status = status;
  const GemmPick p = lmhead_pick(M, V, sms);
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, hf, M, C, C, 128) || !make_tmap_bf16(&tb, wte, V, C, C, gemm_tc_b_box_rows(p)))
    return GPT2_ERR_CUDA;
  G2_CK(gemm_tc_launch(EPI_LMHEAD, p.bn, ta, tb, ta, a, sms, s, LAYOUT_KK, nullptr, p.pair));
  G2_CK(ce_finish_launch(part, gemm_tc_n_tiles(V, p.bn), tgt, targets, M, V, tok, loss_out, status, s, lse, n_scored));
  const Gemm gm{sms, status, s};
  GemmArgs d{};
  d.targets = targets;
  d.row_lse = lse;
  d.n_scored = n_scored;
  G2_RC(gm.run(EPI_DLOGITS, hf, false, C, wte, false, C, dz, Vp, false, M, V, C, d));
  if (Vp > V) G2_CK(cudaMemset2DAsync(static_cast<uint8_t*>(dz) + (size_t)V * 2, (size_t)Vp * 2, 0,
                                      (size_t)(Vp - V) * 2, M, s));
  G2_RC(gm.run(EPI_F32, dz, false, Vp, wte, true, C, dhf, C, true, M, C, Vp, GemmArgs{}, nullptr, V));
  return gm.run(EPI_F32, dz, true, Vp, hf, true, C, dwte, C, true, V, C, M);
}

}  // extern "C"
