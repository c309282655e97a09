// ce.cu - finish the fused cross-entropy from per-tile log-sum-exp partials.
//
// loss_t = logsumexp_v(z[t, v]) - z[t, target_t]; loss = mean over positions
// with a target ("Hand-writing GPT-2 from scratch: the Transformer decoder
// core modules in PyTorch", section 4.1 step 5: CrossEntropyLoss with its
// mean reduction over the shifted targets).
//
// The lm_head epilogue left, per row and column group, (m_i, s_i) with
// s_i = sum over the group of exp(z - m_i). ce_rows_kernel merges them per
// row: M = max m_i, S = sum s_i exp(m_i - M), lse = M + log S. A single block
// then forms the mean in double precision in a fixed order (deterministic).
#include "common.cuh"
#include "kernels.h"

namespace g2 {

// One block per 32 rows: lane = row, so every load of a partial is a
// coalesced 256-byte read of one column group for 32 consecutive rows. The 32
// warps take the column groups round-robin, each warp with 8 independent
// running (max, sum) pairs (groups 32 a + warp for a = j mod 8) whose loads
// are all issued before any merge, so a warp has 8 reads in flight and the
// ~25 groups of a 50257-column vocabulary take about three memory round
// trips; the pairs are merged in a fixed order, per warp and then across
// warps through shared memory (deterministic). Rescaling uses
// exp(d) = 2^(d log2 e) on the SFU.
constexpr int CE_WARPS = 32;
constexpr int CE_LOADS = 8;

__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  if (m2 == -INFINITY) return;   // a column group with no valid column
  const float mn = fmaxf(m, m2);
  s = s * ex2_approx((m - mn) * 1.4426950408889634f) + s2 * ex2_approx((m2 - mn) * 1.4426950408889634f);
  m = mn;
}

__global__ void __launch_bounds__(32 * CE_WARPS) ce_rows_kernel(const float2* __restrict__ part, int n_tiles,
                                                               const float* __restrict__ tgt_logit,
                                                               const int* __restrict__ targets, int M, int V,
                                                               float* __restrict__ token_loss, int* status,
                                                               float* __restrict__ lse_out) {
  __shared__ float sm_m[CE_WARPS][32], sm_s[CE_WARPS][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 32 + lane;
  pdl_wait();
  pdl_trigger();
  float m[CE_LOADS], s[CE_LOADS];
#pragma unroll
  for (int a = 0; a < CE_LOADS; ++a) {
    m[a] = -INFINITY;
    s[a] = 0.f;
  }
  if (row < M) {
    for (int i = warp; i < n_tiles; i += CE_LOADS * CE_WARPS) {
      float2 p[CE_LOADS];
#pragma unroll
      for (int a = 0; a < CE_LOADS; ++a) {
        const int g = i + a * CE_WARPS;
        p[a] = g < n_tiles ? part[(size_t)g * M + row] : make_float2(-INFINITY, 0.f);
      }
#pragma unroll
      for (int a = 0; a < CE_LOADS; ++a) lse_merge(m[a], s[a], p[a].x, p[a].y);
    }
  }
#pragma unroll
  for (int w = 1; w < CE_LOADS; w *= 2)
#pragma unroll
    for (int a = 0; a < CE_LOADS; a += 2 * w) lse_merge(m[a], s[a], m[a + w], s[a + w]);
  sm_m[warp][lane] = m[0];
  sm_s[warp][lane] = s[0];
  __syncthreads();
  if (warp == 0 && row < M) {
    float mm = -INFINITY, ss = 0.f;
#pragma unroll
    for (int w = 0; w < CE_WARPS; ++w) lse_merge(mm, ss, sm_m[w][lane], sm_s[w][lane]);
    const int tg = targets[row];
    float l = 0.f;
    if (lse_out) lse_out[row] = mm + logf(ss);
    if (tg >= V) {
      record_error(status, DEV_BAD_TOKEN);
    } else if (tg >= 0) {
      l = (mm + logf(ss)) - tgt_logit[row];
    }
    token_loss[row] = l;
  }
}

__global__ void __launch_bounds__(1024) ce_mean_kernel(const float* __restrict__ token_loss,
                                                       const int* __restrict__ targets, int M, int V,
                                                       float* __restrict__ loss_out, int* status,
                                                       int* __restrict__ n_scored_out) {
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
      if (n_scored_out) *n_scored_out = cnt;
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
                             int V, float* token_loss, float* loss_out, int* status, cudaStream_t s, float* lse_out,
                             int* n_scored_out) {
  if (M <= 0) return cudaSuccess;
  cudaError_t e = launch_pdl(ce_rows_kernel, dim3((M + 31) / 32), dim3(32 * CE_WARPS), 0, s, part, n_tiles, tgt_logit, targets,
                             M, V, token_loss, status, lse_out);
  if (e == cudaSuccess && loss_out)
    e = launch_pdl(ce_mean_kernel, dim3(1), dim3(1024), 0, s, token_loss, targets, M, V, loss_out, status,
                   n_scored_out);
  return e;
}

}  // namespace g2
