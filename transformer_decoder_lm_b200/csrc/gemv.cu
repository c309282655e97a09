// gemv.cu - Linear layers for a few rows (M <= GEMV_MAX_M), bf16.
//
// y = A W^T + bias with the Linear epilogues of gemm_tc.cu (bias, GELU in the
// exact erf or the tanh form, residual add into fp32 x), for the decoding
// step and other calls with a handful of rows, where a 128-row tensor-core
// tile would be almost all padding and would leave most SMs idle. The work is
// bound by reading W once: one warp per output column n streams W's row n
// with 16-byte loads (lane-strided over K) against the M rows of A (from L1 /
// L2), keeps M running sums, reduces them with a fixed butterfly (the same
// bits on every run) and lane m writes row m.
#include <math.h>

#include "common.cuh"
#include "decode.h"
#include "kernels.h"

namespace g2 {

namespace {
constexpr int GEMV_WARPS = 8;

template <int EPI>
__global__ void __launch_bounds__(32 * GEMV_WARPS) gemv_bf16_kernel(const bf16* __restrict__ A,
                                                                    const bf16* __restrict__ W,
                                                                    const bf16* __restrict__ bias, void* out, int M,
                                                                    int N, int K, long long ldo, int gelu_tanh) {
  const int n = blockIdx.x * GEMV_WARPS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (n < N) {
    float acc[GEMV_MAX_M];
#pragma unroll
    for (int m = 0; m < GEMV_MAX_M; ++m) acc[m] = 0.f;
    const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)n * K);
    const int KU = K / 8;
#pragma unroll 2
    for (int u = lane; u < KU; u += 32) {
      const uint4 w = __ldg(wr + u);
      const bf16* wb = reinterpret_cast<const bf16*>(&w);
      float wf[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) wf[k] = __bfloat162float(wb[k]);
#pragma unroll
      for (int m = 0; m < GEMV_MAX_M; ++m) {
        if (m < M) {
          const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + (size_t)m * K) + u);
          const bf16* ab = reinterpret_cast<const bf16*>(&a);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[m] = fmaf(__bfloat162float(ab[k]), wf[k], acc[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < GEMV_MAX_M; ++m)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
    // every lane now holds all M sums; lane m writes row m
    float v = 0.f;
#pragma unroll
    for (int m = 0; m < GEMV_MAX_M; ++m)
      if (lane == m) v = acc[m];
    if (lane < M) {
      v += __bfloat162float(bias[n]);
      if (EPI == EPI_RESID) {
        float* x = static_cast<float*>(out) + (size_t)lane * ldo + n;
        *x += v;
      } else {
        if (EPI == EPI_GELU)
          v = gelu_tanh ? 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)))
                        : 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
        static_cast<bf16*>(out)[(size_t)lane * ldo + n] = __float2bfloat16_rn(v);
      }
    }
  }
}
}  // namespace

cudaError_t gemv_bf16_launch(int epi, const void* A, const void* W, const GemmArgs& a, cudaStream_t s) {
  if (a.M < 1 || a.M > GEMV_MAX_M || (a.K % 8)) return cudaErrorInvalidValue;
  const dim3 grid((a.N + GEMV_WARPS - 1) / GEMV_WARPS), block(32 * GEMV_WARPS);
  const bf16 *Ap = static_cast<const bf16*>(A), *Wp = static_cast<const bf16*>(W);
  const bf16* bp = static_cast<const bf16*>(a.bias);
  switch (epi) {
    case EPI_BIAS:
      return launch_pdl(gemv_bf16_kernel<EPI_BIAS>, grid, block, 0, s, Ap, Wp, bp, a.out, a.M, a.N, a.K, a.ldo,
                        a.gelu_tanh);
    case EPI_GELU:
      return launch_pdl(gemv_bf16_kernel<EPI_GELU>, grid, block, 0, s, Ap, Wp, bp, a.out, a.M, a.N, a.K, a.ldo,
                        a.gelu_tanh);
    case EPI_RESID:
      return launch_pdl(gemv_bf16_kernel<EPI_RESID>, grid, block, 0, s, Ap, Wp, bp, a.out, a.M, a.N, a.K, a.ldo,
                        a.gelu_tanh);
  }
  return cudaErrorInvalidValue;
}

}  // namespace g2
