// decode.h - kernels of the few-row paths: the one-query attention of the
// key/value-cache decoding step and the Linear layers for a handful of rows.
#pragma once

#include "kernels.h"

namespace g2 {

// ---- Linear layers for a few rows (bf16, M <= GEMV_MAX_M) -------------------
// The epilogues EPI_BIAS / EPI_GELU / EPI_RESID of GemmArgs, one warp per
// output column; A [M, K] and W [N, K] 16-byte aligned, K a multiple of 8.
constexpr int GEMV_MAX_M = 16;
cudaError_t gemv_bf16_launch(int epi, const void* A, const void* W, const GemmArgs& a, cudaStream_t s);

// One query per (sequence, head) against `len` cached positions: y [B, C] =
// softmax(q k^T / sqrt(D)) v with q from qkv [B, 3C] and k, v from one
// layer's cache [max_B][n_ctx][2C] (k then v per position). D = C / H must
// divide 128.
// part: fp32 scratch of part_floats floats for the split-over-keys bf16
// kernels (B * H * ceil(len / 256) * (D + 2) needed; otherwise, or when NULL,
// one block per (sequence, head) takes all keys).
cudaError_t attention_decode_launch(bool bf16, const void* qkv, const void* cache, void* y, int B, int H, int C,
                                    int n_ctx, int len, float* part, size_t part_floats, cudaStream_t s);

}  // namespace g2
