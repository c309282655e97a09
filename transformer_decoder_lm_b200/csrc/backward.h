// backward.h - launchers of the backward-pass kernels (internal; backward.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace g2 {

// LayerNorm gradient over rows of x [M, C] fp32 (the saved LayerNorm input),
// gamma bf16 [C], dh fp32 [M, C] (gradient of the LayerNorm output):
//   dx_out = dx_in + rstd (g dh - mean(g dh) - xh mean(g dh xh))
// (dx_in may be NULL, dx_out may equal dx_in; dx_bf16, if not NULL, receives a
// bf16 copy of dx_out), dgamma = sum_rows dh xh, dbeta = sum_rows dh (fp32
// [C]); in the same pass dsum = sum_rows dx_out [C] and dz = sum_rows z [nz]
// of a bf16 matrix z [M, nz] (nz % 8 == 0), each when its pointer is not
// NULL. All sums add in a fixed order. part: layernorm_bwd_part_floats floats.
struct LnBwdArgs {
  const float* x;
  const __nv_bfloat16* gamma;
  const float* dh;
  const float* dx_in;
  float* dx_out;
  __nv_bfloat16* dx_bf16;
  const __nv_bfloat16* z;
  int nz;
  float* part;
  int M, C;
};
int layernorm_bwd_blocks(int M);
size_t layernorm_bwd_part_floats(int M, int C, int nz);
cudaError_t layernorm_bwd_launch(const LnBwdArgs& a, float* dgamma, float* dbeta, float* dsum, float* dz,
                                 cudaStream_t s);

// Attention gradient (bf16, d_head 64): qkv [B, T, 3C] and y [B, T, C] of the
// forward, dy [B, T, C], lse2 [B, H, T] (per query row: log2 of the softmax
// normaliser of the scores scaled by log2(e)/sqrt(d_head), as the forward
// kernel wrote it) -> dqkv bf16 [B, T, 3C]. Scratch: Dv fp32 [B, H, T],
// dq_acc fp32 [B, T, C] (zeroed here). A wait that runs out records
// DEV_TIMEOUT in *status (when not NULL).
cudaError_t attention_bwd_launch(const void* qkv, const void* y, const void* dy, const float* lse2, float* Dv,
                                 float* dq_acc, void* dqkv, int B, int T, int H, int C, int* status, cudaStream_t s);
// The tcgen05 kernel of it (attention_bwd_tc.cu): dK, dV into dqkv, dQ
// (unscaled) added into dq_acc, given Dv.
cudaError_t attention_bwd_tc_launch(const void* qkv, const void* dy, const float* lse2, const float* Dv, float* dq_acc,
                                    void* dqkv, int B, int T, int H, int C, int* status, cudaStream_t s);

// Embedding gradient: dwte[ids[m]] += dx[m] (dwte already holds the lm_head
// term), dwpe[t] = sum_b dx[b, t] for t < T and 0 up to n_ctx.
cudaError_t embed_bwd_launch(const int* ids, const float* dx, float* dwte, float* dwpe, int B, int T, int n_ctx,
                             int C, int V, cudaStream_t s);

}  // namespace g2
