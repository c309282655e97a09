// ce.cu - finish the fused cross-entropy from per-tile log-sum-exp partials.
//
// loss_t = logsumexp_v(z[t, v]) - z[t, target_t]; loss = mean over positions
// with a target ("Hand-writing GPT-2 from scratch: the Transformer decoder
// core modules in PyTorch", section 4.1 step 5: CrossEntropyLoss with its
// mean reduction over the shifted targets).
//
// The lm_head epilogue left, per row and column group, (m_i, s_i) with
// s_i = sum over the group of exp(z - m_i). Here one warp per row merges them:
// M = max m_i, S = sum s_i exp(m_i - M), lse = M + log S. A single block then
// forms the mean in double precision in a fixed order (deterministic).
#include "common.cuh"
#include "kernels.h"

namespace g2 {

__global__ void __launch_bounds__(256) ce_rows_kernel(const float2* __restrict__ part, int n_tiles,
                                                      const float* __restrict__ tgt_logit,
                                                      const int* __restrict__ targets, int M, int V,
                                                      float* __restrict__ token_loss, int* status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (row >= M) return;
  float m = -INFINITY, s = 0.f;
  for (int i = lane; i < n_tiles; i += 32) {
    const float2 p = part[(size_t)i * M + row];
    if (p.x == -INFINITY) continue;   // a column group with no valid column
    const float mn = fmaxf(m, p.x);
    s = s * expf(m - mn) + p.y * expf(p.x - mn);
    m = mn;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(m, m2);
    const float a = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float a2 = (m2 == -INFINITY) ? 0.f : expf(m2 - mn);
    s = s * a + s2 * a2;
    m = mn;
  }
  if (lane == 0) {
    const int tg = targets[row];
    float l = 0.f;
    if (tg >= V) {
      record_error(status, DEV_BAD_TOKEN);
    } else if (tg >= 0) {
      l = (m + logf(s)) - tgt_logit[row];
    }
    token_loss[row] = l;
  }
}

__global__ void __launch_bounds__(1024) ce_mean_kernel(const float* __restrict__ token_loss,
                                                       const int* __restrict__ targets, int M, int V,
                                                       float* __restrict__ loss_out, int* status) {
  __shared__ double ssum[32];
  __shared__ int scnt[32];
  pdl_wait();
  pdl_trigger();
  double acc = 0.0;
  int cnt = 0;
  for (int r = threadIdx.x; r < M; r += blockDim.x) {
    const int tg = targets[r];
    if (tg >= 0 && tg < V) {
      acc += (double)token_loss[r];
      ++cnt;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    acc += __shfl_xor_sync(0xffffffffu, acc, off);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    ssum[w] = acc;
    scnt[w] = cnt;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    acc = lane < nw ? ssum[lane] : 0.0;
    cnt = lane < nw ? scnt[lane] : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      acc += __shfl_xor_sync(0xffffffffu, acc, off);
      cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    }
    if (lane == 0) {
      if (cnt == 0) {
        record_error(status, DEV_NO_TARGETS);
        *loss_out = __int_as_float(0x7fc00000);
      } else {
        *loss_out = (float)(acc / cnt);
      }
    }
  }
}

cudaError_t ce_finish_launch(const float2* part, int n_tiles, const float* tgt_logit, const int* targets, int M,
                             int V, float* token_loss, float* loss_out, int* status, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  cudaError_t e = launch_pdl(ce_rows_kernel, dim3((M + 7) / 8), dim3(256), 0, s, part, n_tiles, tgt_logit, targets, M,
                             V, token_loss, status);
  if (e == cudaSuccess && loss_out)
    e = launch_pdl(ce_mean_kernel, dim3(1), dim3(1024), 0, s, token_loss, targets, M, V, loss_out, status);
  return e;
}

}  // namespace g2
