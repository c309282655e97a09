// gemm_simt.cu - fp32 SIMT GEMM for the all-fp32 mode.
//
// Same contract as the tcgen05 GEMM (C = A . W^T, nn.Linear [out, in]
// weights, bias / GELU(erf) / residual / lm_head log-sum-exp epilogues), in
// plain fp32 FFMA. This path exists for exactness, not speed: tf32 tensor
// cores would not hold the fp32 mode's 1e-4 relative error bound.
// 64x64 output tiles, 16-wide k-slabs staged in shared memory, 4x4 outputs
// per thread.
#include "common.cuh"
#include "kernels.h"

namespace g2 {

constexpr int SB_M = 64, SB_N = SIMT_BN, SB_K = 16;

template <int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const float* __restrict__ A, const float* __restrict__ W,
                                                        const GemmArgs args) {
  __shared__ float As[SB_K][SB_M + 4];
  __shared__ float Bs[SB_K][SB_N + 4];
  __shared__ float Cs[EPI == EPI_LMHEAD ? SB_M : 1][SB_N + 1];
  const int M = args.M, N = args.N, K = args.K;
  const int m0 = blockIdx.y * SB_M, n0 = blockIdx.x * SB_N;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};

  const int lr = tid >> 2, lk = (tid & 3) * 4;   // loader: row lr, k offset lk..lk+3
  for (int k0 = 0; k0 < K; k0 += SB_K) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = k0 + lk + e;
      const int am = m0 + lr, bn = n0 + lr;
      As[lk + e][lr] = (am < M && k < K) ? A[(size_t)am * K + k] : 0.f;
      Bs[lk + e][lr] = (bn < N && k < K) ? W[(size_t)bn * K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SB_K; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  const float* bias = static_cast<const float*>(args.bias);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      float v = acc[i][j];
      if (EPI == EPI_LMHEAD) {
        Cs[ty * 4 + i][tx * 4 + j] = v;
        if (args.out != nullptr && m < M && n < N) static_cast<float*>(args.out)[(size_t)m * args.ldo + n] = v;
        continue;
      }
      if (m >= M || n >= N) continue;
      v += bias[n];
      float* o = static_cast<float*>(args.out) + (size_t)m * args.ldo + n;
      if (EPI == EPI_BIAS) *o = v;
      if (EPI == EPI_GELU)
        *o = args.gelu_tanh ? 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)))
                            : 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
      if (EPI == EPI_RESID) *o += v;
    }
  }
  if (EPI == EPI_LMHEAD) {
    __syncthreads();
    if (tid < SB_M) {
      const int m = m0 + tid;
      if (m < M) {
        const int tgt = args.targets != nullptr ? args.targets[m] : -1;
        const int nvalid = min(SB_N, N - n0);
        float mx = -INFINITY;
        for (int c = 0; c < nvalid; ++c) mx = fmaxf(mx, Cs[tid][c]);
        float s = 0.f;
        for (int c = 0; c < nvalid; ++c) s += expf(Cs[tid][c] - mx);
        args.part[(size_t)blockIdx.x * M + m] = make_float2(mx, s);
        if (tgt >= n0 && tgt < n0 + nvalid) args.tgt_logit[m] = Cs[tid][tgt - n0];
      }
    }
  }
}

cudaError_t gemm_simt_launch(int epi, const float* A, const float* W, const GemmArgs& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0) return cudaSuccess;
  dim3 grid((a.N + SB_N - 1) / SB_N, (a.M + SB_M - 1) / SB_M);
  switch (epi) {
    case EPI_BIAS: gemm_simt_kernel<EPI_BIAS><<<grid, 256, 0, s>>>(A, W, a); break;
    case EPI_GELU: gemm_simt_kernel<EPI_GELU><<<grid, 256, 0, s>>>(A, W, a); break;
    case EPI_RESID: gemm_simt_kernel<EPI_RESID><<<grid, 256, 0, s>>>(A, W, a); break;
    case EPI_LMHEAD: gemm_simt_kernel<EPI_LMHEAD><<<grid, 256, 0, s>>>(A, W, a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace g2
