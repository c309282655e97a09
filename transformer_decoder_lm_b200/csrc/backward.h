// backward.h - launchers of the backward-pass kernels (internal; backward.cu).
#pragma once

#include <cuda_runtime.h>

namespace g2 {

// LayerNorm gradient over rows of x [M, C] fp32 (the saved LayerNorm input),
// gamma bf16 [C], dh fp32 [M, C] (gradient of the LayerNorm output):
//   dx_out = dx_in + rstd (g dh - mean(g dh) - xh mean(g dh xh))
// (dx_in may be NULL, dx_out may equal dx_in; dx_bf16, if not NULL, receives a
// bf16 copy of dx_out), dgamma = sum_rows dh xh, dbeta = sum_rows dh (fp32 [C]).
// part: layernorm_bwd_blocks(M) * 2 * C floats of scratch.
int layernorm_bwd_blocks(int M);
cudaError_t layernorm_bwd_launch(const float* x, const void* gamma, const float* dh, const float* dx_in,
                                 float* dx_out, void* dx_bf16, float* part, float* dgamma, float* dbeta, int M, int C,
                                 cudaStream_t s);

// out[c] = sum over the M rows of a [M, N] matrix (bf16 or fp32, row pitch ld
// elements, N % 8 == 0), added in a fixed order. part: col_sum_blocks(M) * N floats.
int col_sum_blocks(int M);
cudaError_t col_sum_launch(const void* a, bool a_bf16, long long ld, int M, int N, float* part, float* out,
                           cudaStream_t s);

// Attention gradient (bf16, d_head 64): qkv [B, T, 3C] and y [B, T, C] of the
// forward, dy [B, T, C], lse2 [B, H, T] (per query row: log2 of the softmax
// normaliser of the scores scaled by log2(e)/sqrt(d_head), as the forward
// kernel wrote it) -> dqkv bf16 [B, T, 3C]. Scratch: Dv fp32 [B, H, T],
// dq_acc fp32 [B, T, C] (zeroed here).
cudaError_t attention_bwd_launch(const void* qkv, const void* y, const void* dy, const float* lse2, float* Dv,
                                 float* dq_acc, void* dqkv, int B, int T, int H, int C, cudaStream_t s);

// Embedding gradient: dwte[ids[m]] += dx[m] (dwte already holds the lm_head
// term), dwpe[t] = sum_b dx[b, t] for t < T and 0 up to n_ctx.
cudaError_t embed_bwd_launch(const int* ids, const float* dx, float* dwte, float* dwpe, int B, int T, int n_ctx,
                             int C, int V, cudaStream_t s);

}  // namespace g2
