// backward.cu - the row-wise and attention kernels of the backward pass.
//
// The gradient of the mean shifted cross-entropy with respect to every weight
// ("Hand-writing GPT-2 from scratch: the Transformer decoder core modules in
// PyTorch", section 4.3: loss.backward() in the training loop; section 2.2:
// the tied lm_head makes wte's gradient the sum of the head's and the token
// embedding's terms). The dense products (every dgrad and wgrad, the logits
// gradient) run on the tcgen05 GEMM (gemm_tc.cu) with MN-major operands; this
// file holds the rest:
//
//   layernorm_bwd   dx = dx_in + r (g dh - mean(g dh) - xh mean(g dh xh)),
//                   per-block column partials of dh xh and dh (dgamma, dbeta),
//                   of dx (a residual projection's bias gradient) and of a
//                   second [M, nz] matrix (a bias gradient of a Linear layer)
//   lnb_reduce      sum of the partials over blocks, in a fixed order
//   attn_bwd_dvec   Dv[b, h, i] = sum_d dO[i, d] O[i, d]
//   dq_finish       dq (scaled, bf16) into the q columns of dqkv
// (the attention gradient itself is attention_bwd_tc.cu)
//   embed_bwd       dwte[id] += dx (fp32 atomics), dwpe[t] = sum_b dx[b, t]
//
// Every column reduction adds in a fixed order, so those gradients repeat
// bit for bit; the two atomic sums (dQ over key tiles, wte rows over repeated
// tokens) do not.
#include <math.h>

#include "backward.h"
#include "common.cuh"
#include "kernels.h"

namespace g2 {

namespace {

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float4 ld_bf16x4(const bf16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}

constexpr int LNB_WARPS = 8, LNB_ROWS_PER_WARP = 2;   // 16 rows per block, two blocks per SM
constexpr int LNB_ROWS_PER_BLOCK = LNB_WARPS * LNB_ROWS_PER_WARP;
template <int MAXV>
__global__ void __launch_bounds__(32 * LNB_WARPS, MAXV <= 6 ? 2 : 1) layernorm_bwd_kernel(const LnBwdArgs a) {
  extern __shared__ float lnb_smem[];   // [3][LNB_WARPS][C]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = a.C, M = a.M;
  float* sg = lnb_smem + (size_t)warp * C;
  float* sbt = lnb_smem + (size_t)(LNB_WARPS + warp) * C;
  float* ssum = lnb_smem + (size_t)(2 * LNB_WARPS + warp) * C;
  const size_t pw = (size_t)3 * C + a.nz;
  float* prow = a.part + (size_t)blockIdx.x * pw;
  pdl_wait();
  pdl_trigger();
  for (int c = lane * 4; c < C; c += 128) {
    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(sg + c) = z4;
    *reinterpret_cast<float4*>(sbt + c) = z4;
    *reinterpret_cast<float4*>(ssum + c) = z4;
  }
  __syncwarp();
  const int r_blk = blockIdx.x * LNB_ROWS_PER_BLOCK;
  const int r_end = min(M, r_blk + LNB_ROWS_PER_BLOCK);
  for (int rr = 0; rr < LNB_ROWS_PER_WARP; ++rr) {
    const int row = r_blk + warp * LNB_ROWS_PER_WARP + rr;
    if (row >= M) continue;
    const float* xr = a.x + (size_t)row * C;
    const float* gr = a.dh + (size_t)row * C;
    const float* dir = a.dx_in ? a.dx_in + (size_t)row * C : nullptr;
    float4 xv[MAXV], gv[MAXV], gm[MAXV], dv[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int c = (lane + 32 * i) * 4;
      if (c < C) {
        xv[i] = *reinterpret_cast<const float4*>(xr + c);
        gv[i] = *reinterpret_cast<const float4*>(gr + c);
        gm[i] = ld_bf16x4(a.gamma + c);
        dv[i] = dir ? *reinterpret_cast<const float4*>(dir + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i)
      if ((lane + 32 * i) * 4 < C) s += (xv[i].x + xv[i].y) + (xv[i].z + xv[i].w);
    const float mean = warp_sum_f(s) / (float)C;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i)
      if ((lane + 32 * i) * 4 < C) {
        const float a0 = xv[i].x - mean, b0 = xv[i].y - mean, c0 = xv[i].z - mean, d0 = xv[i].w - mean;
        q += (a0 * a0 + b0 * b0) + (c0 * c0 + d0 * d0);
      }
    const float rstd = rsqrtf(warp_sum_f(q) / (float)C + 1e-5f);
    // xh = (x - mean) rstd; gx = dh gamma; means of gx and gx xh
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int c = (lane + 32 * i) * 4;
      if (c < C) {
        xv[i] = make_float4((xv[i].x - mean) * rstd, (xv[i].y - mean) * rstd, (xv[i].z - mean) * rstd,
                            (xv[i].w - mean) * rstd);
        gm[i] = make_float4(gv[i].x * gm[i].x, gv[i].y * gm[i].y, gv[i].z * gm[i].z, gv[i].w * gm[i].w);
        s1 += (gm[i].x + gm[i].y) + (gm[i].z + gm[i].w);
        s2 += (gm[i].x * xv[i].x + gm[i].y * xv[i].y) + (gm[i].z * xv[i].z + gm[i].w * xv[i].w);
      }
    }
    const float m1 = warp_sum_f(s1) / (float)C, m2 = warp_sum_f(s2) / (float)C;
    float* dor = a.dx_out + (size_t)row * C;
    bf16* dbr = a.dx_bf16 ? a.dx_bf16 + (size_t)row * C : nullptr;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int c = (lane + 32 * i) * 4;
      if (c < C) {
        float4 d;
        d.x = dv[i].x + rstd * (gm[i].x - m1 - xv[i].x * m2);
        d.y = dv[i].y + rstd * (gm[i].y - m1 - xv[i].y * m2);
        d.z = dv[i].z + rstd * (gm[i].z - m1 - xv[i].z * m2);
        d.w = dv[i].w + rstd * (gm[i].w - m1 - xv[i].w * m2);
        *reinterpret_cast<float4*>(dor + c) = d;
        if (dbr) {
          uint2 u;
          u.x = pack_bf16x2(d.x, d.y);
          u.y = pack_bf16x2(d.z, d.w);
          *reinterpret_cast<uint2*>(dbr + c) = u;
        }
        // this warp's column partials: dh xh, dh, dx_out
        float4 pg = *reinterpret_cast<float4*>(sg + c);
        float4 pb = *reinterpret_cast<float4*>(sbt + c);
        float4 ps = *reinterpret_cast<float4*>(ssum + c);
        pg = make_float4(pg.x + gv[i].x * xv[i].x, pg.y + gv[i].y * xv[i].y, pg.z + gv[i].z * xv[i].z,
                         pg.w + gv[i].w * xv[i].w);
        pb = make_float4(pb.x + gv[i].x, pb.y + gv[i].y, pb.z + gv[i].z, pb.w + gv[i].w);
        ps = make_float4(ps.x + d.x, ps.y + d.y, ps.z + d.z, ps.w + d.w);
        *reinterpret_cast<float4*>(sg + c) = pg;
        *reinterpret_cast<float4*>(sbt + c) = pb;
        *reinterpret_cast<float4*>(ssum + c) = ps;
      }
    }
  }
  // z: thread t sums the 8-column groups t, t + 256, ... over the block's
  // rows, 8 row loads in flight at a time, rows added in order
  const int ngz = a.z ? a.nz / 8 : 0;
  for (int gz = threadIdx.x; gz < ngz; gz += 32 * LNB_WARPS) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int rb = r_blk; rb < r_end; rb += 8) {
      const bf16* zp = a.z + (size_t)rb * a.nz + 8 * gz;
      uint4 u[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (rb + k < r_end) u[k] = __ldg(reinterpret_cast<const uint4*>(zp + (size_t)k * a.nz));
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (rb + k < r_end) {
          const uint32_t w4[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[2 * j] += __uint_as_float(w4[j] << 16);
            acc[2 * j + 1] += __uint_as_float(w4[j] & 0xffff0000u);
          }
        }
    }
    float* pz = prow + 3 * (size_t)C + 8 * gz;
    *reinterpret_cast<float4*>(pz) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(pz + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  __syncthreads();
  // the block's partial row: warp slices added in warp order
  for (int j = threadIdx.x * 4; j < 3 * C; j += blockDim.x * 4) {
    const int part = j / C, c = j - part * C;
    const float* src = lnb_smem + (size_t)part * LNB_WARPS * C + c;
    float4 t = *reinterpret_cast<const float4*>(src);
#pragma unroll
    for (int w = 1; w < LNB_WARPS; ++w) {
      const float4 v = *reinterpret_cast<const float4*>(src + (size_t)w * C);
      t = make_float4(t.x + v.x, t.y + v.y, t.z + v.z, t.w + v.w);
    }
    *reinterpret_cast<float4*>(prow + j) = t;
  }
}

// Sums of the partial rows over the blocks: column j of [P, pw] partials,
// rows p = ty, ty + 16, ... in order by each of the 16 thread rows, then the
// 16 in order; column j goes to dgamma (j < C), dbeta (< 2C), dsum (< 3C) or dz.
constexpr int LNR_SLICES = 16;
__global__ void __launch_bounds__(32 * LNR_SLICES) lnb_reduce_kernel(const float* __restrict__ part, int P, int pw,
                                                                     int C, float* __restrict__ dgamma,
                                                                     float* __restrict__ dbeta,
                                                                     float* __restrict__ dsum, float* __restrict__ dz) {
  __shared__ float red[LNR_SLICES][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int j = blockIdx.x * 32 + tx;
  pdl_wait();
  pdl_trigger();
  float s = 0.f;
  if (j < pw) {
    const float* p = part + j;
#pragma unroll 8
    for (int r = ty; r < P; r += LNR_SLICES) s += p[(size_t)r * pw];
  }
  red[ty][tx] = s;
  __syncthreads();
  if (ty == 0 && j < pw) {
    float t = red[0][tx];
#pragma unroll
    for (int k = 1; k < LNR_SLICES; ++k) t += red[k][tx];
    if (j < C) dgamma[j] = t;
    else if (j < 2 * C) dbeta[j - C] = t;
    else if (j < 3 * C) {
      if (dsum) dsum[j - 2 * C] = t;
    } else if (dz) {
      dz[j - 3 * C] = t;
    }
  }
}

// Dv[(b H + h) T + i] = sum over the head's 64 columns of dO * O: one warp per
// row (b, i); each lane's 8 columns lie in one head, 8 lanes per head.
__global__ void __launch_bounds__(256) attn_bwd_dvec_kernel(const bf16* __restrict__ dO, const bf16* __restrict__ O,
                                                            float* __restrict__ Dv, int B, int T, int H, int C) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (row < B * T) {
    const int b = row / T, i = row % T;
    for (int c0 = lane * 8; c0 < C; c0 += 256) {
      const uint4 u = *reinterpret_cast<const uint4*>(dO + (size_t)row * C + c0);
      const uint4 v = *reinterpret_cast<const uint4*>(O + (size_t)row * C + c0);
      const uint32_t uw[4] = {u.x, u.y, u.z, u.w}, vw[4] = {v.x, v.y, v.z, v.w};
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        s += __uint_as_float(uw[j] << 16) * __uint_as_float(vw[j] << 16) +
             __uint_as_float(uw[j] & 0xffff0000u) * __uint_as_float(vw[j] & 0xffff0000u);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if ((lane & 7) == 0) Dv[((size_t)b * H + c0 / 64) * T + i] = s;
    }
  }
}

// dqkv[:, 0:C] = bf16(dq_acc * scale); 8 columns per thread.
__global__ void __launch_bounds__(256) dq_finish_kernel(const float* __restrict__ dq_acc, bf16* __restrict__ dqkv,
                                                        int M, int C, float scale) {
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  pdl_wait();
  pdl_trigger();
  if (i < (long long)M * C) {
    const long long row = i / C, col = i % C;
    const float4 a = *reinterpret_cast<const float4*>(dq_acc + i);
    const float4 c = *reinterpret_cast<const float4*>(dq_acc + i + 4);
    uint4 u;
    u.x = pack_bf16x2(a.x * scale, a.y * scale);
    u.y = pack_bf16x2(a.z * scale, a.w * scale);
    u.z = pack_bf16x2(c.x * scale, c.y * scale);
    u.w = pack_bf16x2(c.z * scale, c.w * scale);
    *reinterpret_cast<uint4*>(dqkv + row * 3 * C + col) = u;
  }
}

// dwte[ids[m]] += dx[m]: one warp per row, fp32 atomics (ids checked by the forward).
__global__ void __launch_bounds__(256) embed_bwd_wte_kernel(const int* __restrict__ ids, const float* __restrict__ dx,
                                                            float* __restrict__ dwte, int M, int C, int V) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (row < M) {
    const int id = ids[row];
    if (id >= 0 && id < V)
      for (int c = lane; c < C; c += 32) atomicAdd(dwte + (size_t)id * C + c, dx[(size_t)row * C + c]);
  }
}

// dwpe[t, c] = sum over b of dx[b, t, c] for t < T, 0 for T <= t < n_ctx.
__global__ void __launch_bounds__(256) embed_bwd_wpe_kernel(const float* __restrict__ dx, float* __restrict__ dwpe,
                                                            int B, int T, int n_ctx, int C) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (i < (long long)n_ctx * C) {
    const int t = (int)(i / C), c = (int)(i % C);
    float s = 0.f;
    if (t < T)
      for (int b = 0; b < B; ++b) s += dx[((size_t)b * T + t) * C + c];
    dwpe[i] = s;
  }
}

}  // namespace

int layernorm_bwd_blocks(int M) { return (M + LNB_ROWS_PER_BLOCK - 1) / LNB_ROWS_PER_BLOCK; }

size_t layernorm_bwd_part_floats(int M, int C, int nz) {
  return (size_t)layernorm_bwd_blocks(M) * ((size_t)3 * C + (size_t)nz);
}

cudaError_t layernorm_bwd_launch(const LnBwdArgs& a, float* dgamma, float* dbeta, float* dsum, float* dz,
                                 cudaStream_t s) {
  if (a.M <= 0) return cudaSuccess;
  if (a.C > 2048 || (a.C & 3) || a.nz < 0 || (a.z && (a.nz % 8)) || (!a.z && a.nz)) return cudaErrorInvalidValue;
  const int blocks = layernorm_bwd_blocks(a.M);
  const size_t smem = (size_t)3 * LNB_WARPS * a.C * sizeof(float);
  // the largest shared-memory need (C = 2048) once per device, outside any stream capture
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaError_t e = cudaSuccess;
  if (!attr_done[dev]) {
    const int most = 3 * LNB_WARPS * 2048 * (int)sizeof(float);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<6>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<13>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
#define G2_LNB(MV) e = launch_pdl(layernorm_bwd_kernel<MV>, dim3(blocks), dim3(32 * LNB_WARPS), smem, s, a);
  if (a.C <= 512) {
    G2_LNB(4)
  } else if (a.C <= 768) {
    G2_LNB(6)
  } else if (a.C <= 1024) {
    G2_LNB(8)
  } else if (a.C <= 1664) {
    G2_LNB(13)
  } else {
    G2_LNB(16)
  }
#undef G2_LNB
  if (e != cudaSuccess) return e;
  const int pw = 3 * a.C + a.nz;
  return launch_pdl(lnb_reduce_kernel, dim3((pw + 31) / 32), dim3(32 * LNR_SLICES), 0, s, (const float*)a.part, blocks,
                    pw, a.C,
                    dgamma, dbeta, dsum, dz);
}

cudaError_t attention_bwd_launch(const void* qkv, const void* y, const void* dy, const float* lse2, float* Dv,
                                 float* dq_acc, void* dqkv, int B, int T, int H, int C, int* status, cudaStream_t s) {
  constexpr int D = 64;   // d_head
  if (B <= 0 || T <= 0) return cudaSuccess;
  if (C / H != D || C % H || C % 8) return cudaErrorInvalidValue;
  const bf16* o = static_cast<const bf16*>(y);
  const bf16* d = static_cast<const bf16*>(dy);
  bf16* out = static_cast<bf16*>(dqkv);
  const int M = B * T;
  cudaError_t e = cudaMemsetAsync(dq_acc, 0, (size_t)M * C * sizeof(float), s);
  if (e == cudaSuccess) e = launch_pdl(attn_bwd_dvec_kernel, dim3((M + 7) / 8), dim3(256), 0, s, d, o, Dv, B, T, H, C);
  const float scale = (float)(1.0 / sqrt((double)D));
  if (e == cudaSuccess) e = attention_bwd_tc_launch(qkv, dy, lse2, Dv, dq_acc, dqkv, B, T, H, C, status, s);
  if (e == cudaSuccess)
    e = launch_pdl(dq_finish_kernel, dim3((unsigned)(((long long)M * C / 8 + 255) / 256)), dim3(256), 0, s,
                   (const float*)dq_acc, out, M, C, scale);
  return e;
}

cudaError_t embed_bwd_launch(const int* ids, const float* dx, float* dwte, float* dwpe, int B, int T, int n_ctx,
                             int C, int V, cudaStream_t s) {
  const int M = B * T;
  if (M <= 0) return cudaSuccess;
  cudaError_t e = launch_pdl(embed_bwd_wte_kernel, dim3((M + 7) / 8), dim3(256), 0, s, ids, dx, dwte, M, C, V);
  if (e == cudaSuccess)
    e = launch_pdl(embed_bwd_wpe_kernel, dim3((unsigned)(((long long)n_ctx * C + 255) / 256)), dim3(256), 0, s, dx,
                   dwpe, B, T, n_ctx, C);
  return e;
}

}  // namespace g2
