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
enum EpiKind : int { EPI_BIAS = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_LMHEAD = 3, EPI_LMHEAD_LOGITS = 4 };

struct GemmArgs {
  int M, N, K;
  const void* bias;        // [N] of the operand dtype (NULL for the lm_head)
  void* out;               // EPI_BIAS/GELU: [M, ldo] operand dtype; EPI_RESID: fp32 [M, ldo] (+=);
                           // EPI_LMHEAD: fp32 logits [M, ldo] or NULL
  long long ldo;
  const int* targets;      // EPI_LMHEAD: [M]
  float2* part;            // EPI_LMHEAD: per (column group, row) (max, sum exp(z - max)), [n_groups, M]
  float* tgt_logit;        // EPI_LMHEAD: [M] logit of the target column
  int* status;
  int gelu_tanh;           // EPI_GELU: 1 = tanh approximation, 0 = exact erf form
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
// Column groups of lm_head partials for N columns (two per tile of width bn).
int gemm_tc_n_tiles(int N, int bn);
// The lm_head runs with tiles of at least this width.
constexpr int LMHEAD_MIN_BN = 128;
// lm_head partials per row: one per 64-column group of a tcgen05 tile (tiles
// of BN columns cover V padded up to a multiple of BN) or per 64-column SIMT
// tile; at most ceil(V / 64) + 3 either way.
inline size_t lmhead_groups_max(int V) { return (size_t)((V + 63) / 64) + 3; }

// ---- tcgen05 GEMM (bf16) -------------------------------------------------
// C = A[M,K] . B[N,K]^T with the epilogue `epi`. K % 64 == 0, N % 8 == 0.
// tmA: box 128 x 64 over A; tmB: box BN x 64 over B, BN from gemm_tc_pick_bn;
// tmC: the output map (make_tmap_out_*; unused by EPI_LMHEAD).
int gemm_tc_pick_bn(int M, int N, int num_sms, int epi);
cudaError_t gemm_tc_launch(int epi, int bn, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                           const GemmArgs& a, int num_sms, cudaStream_t s);
cudaError_t gemm_tc_set_attributes();

// ---- SIMT fp32 GEMM (fp32 mode) ------------------------------------------
constexpr int SIMT_BN = 64;
cudaError_t gemm_simt_launch(int epi, const float* A, const float* W, const GemmArgs& a, cudaStream_t s);

// ---- embedding / LayerNorm -------------------------------------------------
cudaError_t embed_launch(bool bf16, const int* ids, const void* wte, const void* wpe, float* x, int M, int T,
                         int C, int V, int* status, cudaStream_t s);
cudaError_t layernorm_launch(bool bf16, const float* x, const void* g, const void* b, void* out, int M, int C,
                             cudaStream_t s);

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
cudaError_t attention_tc_launch(const void* qkv, void* y, int B, int T, int H, int C, const AttnScratch* scratch,
                                int* status, cudaStream_t s);
cudaError_t attention_launch(bool bf16, const void* qkv, void* y, int B, int T, int H, int C,
                             const AttnScratch* scratch, int* status, cudaStream_t s);

// ---- cross-entropy finalisation -------------------------------------------
// token_loss[m] = logsumexp over column tiles - tgt_logit[m] (0 where the
// target is negative); loss_out (if not NULL) = mean over scored rows.
cudaError_t ce_finish_launch(const float2* part, int n_tiles, const float* tgt_logit, const int* targets, int M,
                             int V, float* token_loss, float* loss_out, int* status, cudaStream_t s);

}  // namespace g2
