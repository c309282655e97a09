// gemv.cu - Linear layers for a few rows (M <= GEMV_MAX_M), bf16.
//
// y = A W^T + bias with the Linear epilogues of gemm_tc.cu (bias, GELU in the
// exact erf or the tanh form, residual add into fp32 x), optionally with the
// new key / value columns also written into the key/value cache (the
// decoding step's c_attn), for the decoding
// step and other calls with a handful of rows, where a 128-row tensor-core
// tile would be almost all padding and would leave most SMs idle. The work is
// bound by reading W once. Each block copies the M rows of A into shared
// memory once; each warp takes an output column (COLS of them in general)
// and streams its row of W with 16-byte loads (lane-strided over K), up to
// LPC loads per lane issued before the first multiply, against the M rows of
// A read back from shared memory; the MT running sums per column are reduced with a fixed
// butterfly (the same bits on every run) and lane m writes row m.
#include <math.h>

#include "common.cuh"
#include "decode.h"
#include "kernels.h"

namespace g2 {

namespace {
constexpr int GEMV_WARPS = 8;

// MT >= M rows of sums per column; COLS columns per warp; LPC 16-byte W loads
// per lane and column held in registers at once (K / 8 / 32 rounded up, the
// column's whole row for K <= 32 * 8 * LPC, else it streams in LPC-sized steps)
template <int EPI, int MT, int COLS, int LPC>
__global__ void __launch_bounds__(32 * GEMV_WARPS) gemv_bf16_kernel(const bf16* __restrict__ A,
                                                                    const bf16* __restrict__ W,
                                                                    const bf16* __restrict__ bias, void* out, int M,
                                                                    int N, int K, long long ldo, int gelu_tanh,
                                                                    int w_const, bf16* __restrict__ kv,
                                                                    long long ld_kv, int kv_col0) {
  extern __shared__ uint4 gemv_a[];   // [M][K / 8]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KU = K / 8;
  const int n0 = (blockIdx.x * GEMV_WARPS + warp) * COLS;
  // w_const: W is written by no kernel of the stream (the model's weights),
  // so its first loads go out before the wait for the previous kernel
  uint4 w[COLS][LPC];
  auto load_w = [&](int u0) {
#pragma unroll
    for (int c = 0; c < COLS; ++c)
#pragma unroll
      for (int j = 0; j < LPC; ++j) {
        const int u = u0 + lane + 32 * j;
        w[c][j] = (n0 + c < N && u < KU) ? __ldg(reinterpret_cast<const uint4*>(W + (size_t)(n0 + c) * K) + u)
                                         : make_uint4(0, 0, 0, 0);
      }
  };
  if (w_const) load_w(0);
  pdl_wait();
  pdl_trigger();
  if (!w_const) load_w(0);
  {
    const uint4* src = reinterpret_cast<const uint4*>(A);
    for (int i = threadIdx.x; i < M * KU; i += blockDim.x) gemv_a[i] = __ldg(src + i);
  }
  __syncthreads();
  if (n0 >= N) return;
  float acc[COLS][MT];
#pragma unroll
  for (int c = 0; c < COLS; ++c)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[c][m] = 0.f;
  for (int u0 = 0; u0 < KU; u0 += 32 * LPC) {
    if (u0 > 0) load_w(u0);
#pragma unroll
    for (int j = 0; j < LPC; ++j) {
      const int u = u0 + lane + 32 * j;
      if (u < KU) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < M) {
            const uint4 a = gemv_a[m * KU + u];
            const bf16* ab = reinterpret_cast<const bf16*>(&a);
            float af[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) af[k] = __bfloat162float(ab[k]);
#pragma unroll
            for (int c = 0; c < COLS; ++c) {
              const bf16* wb = reinterpret_cast<const bf16*>(&w[c][j]);
#pragma unroll
              for (int k = 0; k < 8; ++k) acc[c][m] = fmaf(af[k], __bfloat162float(wb[k]), acc[c][m]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < COLS; ++c) {
    const int n = n0 + c;
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[c][m] += __shfl_xor_sync(0xffffffffu, acc[c][m], o);
    // every lane now holds all MT sums; lane m writes row m
    float v = 0.f;
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (lane == m) v = acc[c][m];
    if (n < N && lane < M) {
      v += __bfloat162float(bias[n]);
      if (EPI == EPI_RESID) {
        float* x = static_cast<float*>(out) + (size_t)lane * ldo + n;
        *x += v;
      } else {
        if (EPI == EPI_GELU)
          v = gelu_tanh ? 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)))
                        : 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
        static_cast<bf16*>(out)[(size_t)lane * ldo + n] = __float2bfloat16_rn(v);
        if (EPI == EPI_BIAS && kv != nullptr && n >= kv_col0)
          kv[(size_t)lane * ld_kv + (n - kv_col0)] = __float2bfloat16_rn(v);
      }
    }
  }
}

template <int EPI, int MT, int COLS, int LPC>
cudaError_t gemv_one(const bf16* A, const bf16* W, const GemmArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)a.M * a.K * 2;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {   // the largest need: GEMV_MAX_M rows of K = 6400
    const cudaError_t e = cudaFuncSetAttribute(gemv_bf16_kernel<EPI, MT, COLS, LPC>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const dim3 grid((a.N + GEMV_WARPS * COLS - 1) / (GEMV_WARPS * COLS)), block(32 * GEMV_WARPS);
  return launch_pdl(gemv_bf16_kernel<EPI, MT, COLS, LPC>, grid, block, smem, s, A, W,
                    static_cast<const bf16*>(a.bias), a.out, a.M, a.N, a.K, a.ldo, a.gelu_tanh, a.b_const,
                    static_cast<bf16*>(a.kv), a.ld_kv, a.kv_col0);
}

// rows held: 4, 8 or 16; one column per warp (the GPT-2 Linear layers have
// at most a few thousand columns: one warp each spreads W over every SM),
// the whole row in registers for K <= 1024 (LPC 4), else 12 loads at a time
template <int EPI>
cudaError_t gemv_epi(const bf16* A, const bf16* W, const GemmArgs& a, cudaStream_t s) {
  const bool narrow = a.K <= 1024;
  if (a.M <= 4) return narrow ? gemv_one<EPI, 4, 1, 4>(A, W, a, s) : gemv_one<EPI, 4, 1, 12>(A, W, a, s);
  if (a.M <= 8) return narrow ? gemv_one<EPI, 8, 1, 4>(A, W, a, s) : gemv_one<EPI, 8, 1, 12>(A, W, a, s);
  return narrow ? gemv_one<EPI, 16, 1, 4>(A, W, a, s) : gemv_one<EPI, 16, 1, 12>(A, W, a, s);
}
}  // namespace

cudaError_t gemv_bf16_launch(int epi, const void* A, const void* W, const GemmArgs& a, cudaStream_t s) {
  if (a.M < 1 || a.M > GEMV_MAX_M || (a.K % 8) || (size_t)a.M * a.K * 2 > 227 * 1024) return cudaErrorInvalidValue;
  const bf16 *Ap = static_cast<const bf16*>(A), *Wp = static_cast<const bf16*>(W);
  switch (epi) {
    case EPI_BIAS: return gemv_epi<EPI_BIAS>(Ap, Wp, a, s);
    case EPI_GELU: return gemv_epi<EPI_GELU>(Ap, Wp, a, s);
    case EPI_RESID: return gemv_epi<EPI_RESID>(Ap, Wp, a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace g2
