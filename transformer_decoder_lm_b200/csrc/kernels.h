// kernels.h - host-side launchers of the forward-pass kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace g2 {

// Launch `kern` on `s` with programmatic stream serialisation (see pdl_wait /
// pdl_trigger in common.cuh).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Epilogues of the Linear layers (values match the public GPT2_EPI_*),
// plus the fused lm_head / cross-entropy epilogue.
// EPI_LMHEAD_LOGITS is the lm_head kernel that also writes the logits;
// gemm_tc_launch picks it for EPI_LMHEAD when GemmArgs::out is set.
// The training pass adds: EPI_GELU_SAVE (EPI_GELU that also stores the
// pre-activation through tmD), EPI_F32 (fp32 result, TMA store), EPI_DGELU
// (result times the GELU derivative at a saved pre-activation, bf16) and
// EPI_DLOGITS (the cross-entropy gradient of the logits, bf16).
enum EpiKind : int {
  EPI_BIAS = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_LMHEAD = 3, EPI_LMHEAD_LOGITS = 4,
  EPI_F32 = 5, EPI_DGELU = 6, EPI_DLOGITS = 7, EPI_GELU_SAVE = 8
};

// Operand layouts of the tcgen05 GEMM C = A . B^T (bit set: the operand is
// stored MN-major, its M or N index contiguous, as the transposed operands of
// the backward pass are: dX = dY W reads W [N_out, K_in] as B MN-major; dW =
// dY^T X reads dY [tokens, out] as A MN-major and X [tokens, in] as B MN-major).
enum GemmLayout : int { LAYOUT_KK = 0, LAYOUT_A_MN = 1, LAYOUT_B_MN = 2, LAYOUT_MN_MN = 3 };

struct GemmArgs {
  int M, N, K;             // K need not be a multiple of 64: the tail reads as zero
  const void* bias;        // [N] of the operand dtype, or NULL (no bias; NULL for the lm_head)
  void* out;               // EPI_BIAS/GELU/DGELU/DLOGITS: [M, ldo] bf16; EPI_RESID: fp32 [M, ldo] (+=);
                           // EPI_F32: fp32 [M, ldo]; EPI_LMHEAD: fp32 logits [M, ldo] or NULL
  long long ldo;
  const int* targets;      // EPI_LMHEAD, EPI_DLOGITS: [M]
  float2* part;            // EPI_LMHEAD: per (column group, row) (max, sum exp(z - max)), [n_groups, M]
  float* tgt_logit;        // EPI_LMHEAD: [M] logit of the target column
  int* status;
  int gelu_tanh;           // EPI_GELU(_SAVE), EPI_DGELU: 1 = tanh approximation, 0 = exact erf form
  const void* aux;         // EPI_DGELU: saved pre-activation u, bf16 [M, ld_aux]
  long long ld_aux;
  const float* row_lse;    // EPI_DLOGITS: natural-log log-sum-exp of each row [M]
  const int* n_scored;     // EPI_DLOGITS: number of rows with a target (device int)
  int k_split;             // EPI_F32: 2 = the K range in two work items reduce-added into a zeroed output
  int b_const;             // B is written by no kernel of this stream (the forward's weights): its
                           // first stages may be requested before the previous kernel completes
  // few-row GEMV only (decoding):
  void* kv;                // EPI_BIAS: when not NULL, columns n >= kv_col0 are also written as bf16 to
  long long ld_kv;         // kv[row * ld_kv + n - kv_col0] (the new key and value into the cache)
  int kv_col0;
};

// ---- tensor maps (host) -------------------------------------------------
// GEMM operand: a 2-D bf16 row-major tensor [rows, cols] (row pitch `ld`
// elements) read in boxes of box_rows x 64 columns with 128-byte swizzling.
bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                    uint32_t box_rows);
// GEMM outputs written by the epilogue in 32 x 32 boxes: bf16 (64-byte
// swizzle, TMA store) and fp32 (128-byte swizzle, TMA reduce-add).
bool make_tmap_out_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint64_t ld);
bool make_tmap_out_f32(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint64_t ld);
// A 3-D bf16 tensor [d2][d1][d0] (row strides s1, s2 in elements) read or
// written in boxes of box1 rows x box0 (= 64) columns, 128-byte swizzle.
bool make_tmap_3d_bf16(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                       uint64_t s2, uint32_t box0, uint32_t box1);
// The same for fp32 (box0 = 32 columns = 128 bytes).
bool make_tmap_3d_f32(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                      uint64_t s2, uint32_t box0, uint32_t box1);
// Column groups of lm_head partials for N columns (two per tile of width bn).
int gemm_tc_n_tiles(int N, int bn);
// The lm_head runs with tiles of at least this width (lmhead_pick).
constexpr int LMHEAD_MIN_BN = 128;
// lm_head partials per row: one per 64-column group of a tcgen05 tile (tiles
// of BN columns cover V padded up to a multiple of BN) or per 64-column SIMT
// tile; at most ceil(V / 64) + 3 either way.
inline size_t lmhead_groups_max(int V) { return (size_t)((V + 63) / 64) + 3; }
// The tied lm_head with the fused cross-entropy on caller-provided scratch of
// lmhead_ce_scratch_bytes(M, V) bytes, 256-byte aligned (partials
// [groups][M] float2, target logits [M], per-position losses [M]): the launch
// sequence of gpt2_op_lmhead_ce and gpt2_op_lmhead_ce_noalloc, arguments
// already checked. bf16: the tcgen05 path (sms = the device's SM count), else
// the fp32 SIMT path.
size_t lmhead_ce_scratch_bytes(int M, int V);
cudaError_t lmhead_ce_launch(bool bf16, const void* hf, const void* wte, const int32_t* targets, int M, int C, int V,
                             float* logits, float* token_loss, float* loss_out, void* scratch, int sms, int* status,
                             cudaStream_t s);

// ---- tcgen05 GEMM (bf16) -------------------------------------------------
// C = A[M,K] . B[N,K]^T with the epilogue `epi`. N % 8 == 0.
// K-major operands: tmA box 128 x 64 over A [M, K], tmB box BN x 64 over
// B [N, K] (make_tmap_bf16), BN from gemm_tc_pick_bn. MN-major operands
// (layout bits): the operand is stored [K, M] or [K, N] and read in boxes of
// 64 x 64 (make_tmap_bf16 with box_rows 64). tmC: the output map
// (make_tmap_out_*; unused by EPI_LMHEAD); tmD: EPI_GELU_SAVE's
// pre-activation output (bf16, like tmC).
// pair = 1: CTA pairs (clusters of two) compute 256 x BN tiles with one
// M = 256 tcgen05.mma; each CTA loads half of B, so tmB's box is BN / 2 rows
// (K-major operands, BN >= 128, not EPI_F32 / EPI_DGELU: gemm_tc_pair_ok).
struct GemmPick {
  int bn;     // tile width
  int pair;   // 1: CTA pairs
};
GemmPick gemm_tc_pick(int M, int N, int num_sms, int epi, int layout = LAYOUT_KK);
int gemm_tc_pick_bn(int M, int N, int num_sms, int epi);   // gemm_tc_pick(...).bn
bool gemm_tc_pair_ok(int epi, int layout, int bn);
// Rows of tmB's box for a pick: BN, or BN / 2 for a pair.
inline int gemm_tc_b_box_rows(const GemmPick& p) { return p.pair ? p.bn / 2 : p.bn; }
// The lm_head's pick: gemm_tc_pick with tiles of at least LMHEAD_MIN_BN.
inline GemmPick lmhead_pick(int M, int V, int num_sms) {
  GemmPick p = gemm_tc_pick(M, V, num_sms, EPI_LMHEAD);
  if (p.bn < LMHEAD_MIN_BN) p.bn = LMHEAD_MIN_BN;
  return p;
}
cudaError_t gemm_tc_launch(int epi, int bn, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                           const GemmArgs& a, int num_sms, cudaStream_t s, int layout = LAYOUT_KK,
                           const CUtensorMap* tmD = nullptr, int pair = 0);
cudaError_t gemm_tc_set_attributes();

// ---- SIMT fp32 GEMM (fp32 mode) ------------------------------------------
constexpr int SIMT_BN = 64;
cudaError_t gemm_simt_launch(int epi, const float* A, const float* W, const GemmArgs& a, cudaStream_t s);

// ---- embedding / LayerNorm -------------------------------------------------
cudaError_t embed_launch(bool bf16, const int* ids, const void* wte, const void* wpe, float* x, int M, int T,
                         int C, int V, int* status, cudaStream_t s);
// The embedding sum and the first block's ln_1 in one pass (bf16): x as
// embed_launch writes it, and h = LayerNorm(x; g, b) bf16 [M, C].
cudaError_t embed_ln_launch(const int* ids, const void* wte, const void* wpe, float* x, const void* g,
                            const void* b, void* h, int M, int T, int C, int V, int* status, cudaStream_t s);
cudaError_t layernorm_launch(bool bf16, const float* x, const void* g, const void* b, void* out, int M, int C,
                             cudaStream_t s, float* x_save = nullptr);

// ---- sinusoidal position table (bf16 or fp32 [n_ctx, C]) -------------------
cudaError_t sinusoidal_wpe_launch(bool bf16, void* wpe, int n_ctx, int C, cudaStream_t s);

// ---- attention ---------------------------------------------------------------
// tcgen05 flash attention (bf16, d_head 64); attention_launch dispatches to it.
// Scratch of the persistent kernel:
//   sched      two zeroed uint32 counters it schedules its work with (left
//              zeroed again when it ends);
//   flags      cap_pairs * ATTN_PAIR_FLAGS zeroed int32 words (left zeroed again);
//   part       cap_pairs * ATTN_PART_FLOATS floats, no initial contents.
// The longest query tiles are split in two key ranges; the half that
// finishes first leaves its unnormalised partial output in `part` for the
// other to merge.
// cap_pairs bounds how many (sequence, head, query tile) triples may split
// (0: none). A NULL sched uses the library's own per-device scratch, shared by
// every launch that passes NULL (those launches must not overlap).
constexpr int ATTN_PART_FLOATS = 128 * 64 + 2 * 128;
constexpr int ATTN_PAIR_FLAGS = 8;   // int32 flag words per split pair (ready + arrival count per 32-row quarter)
struct AttnScratch {
  unsigned* sched = nullptr;
  int* flags = nullptr;
  float* part = nullptr;
  int cap_pairs = 0;
};
// bytes of flags + partials that never limit the split of a (B, T, H) problem
size_t attention_scratch_bytes(int B, int T, int H);
// lse_out (training forward; if not NULL): per (b, h, query) the log2 of
// the softmax normaliser of the scores scaled by log2(e)/sqrt(d_head), [B, H, T];
// no query tile is split then.
cudaError_t attention_tc_launch(const void* qkv, void* y, int B, int T, int H, int C, const AttnScratch* scratch,
                                int* status, cudaStream_t s, float* lse_out = nullptr);
cudaError_t attention_launch(bool bf16, const void* qkv, void* y, int B, int T, int H, int C,
                             const AttnScratch* scratch, int* status, cudaStream_t s);

// ---- cross-entropy finalisation -------------------------------------------
// token_loss[m] = logsumexp over column tiles - tgt_logit[m] (0 where the
// target is negative); loss_out (if not NULL) = mean over scored rows.
// lse_out (if not NULL) receives each row's log-sum-exp, n_scored_out (if
// not NULL, with loss_out) the number of scored rows.
cudaError_t ce_finish_launch(const float2* part, int n_tiles, const float* tgt_logit, const int* targets, int M,
                             int V, float* token_loss, float* loss_out, int* status, cudaStream_t s,
                             float* lse_out = nullptr, int* n_scored_out = nullptr);

}  // namespace g2
