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
//                   per-block column partials of dh xh and dh (dgamma, dbeta)
//   col_partials    per-block column sums of a [M, N] matrix (bias gradients)
//   col_reduce      sum of the partials over blocks, in a fixed order
//   attn_bwd_dvec   Dv[b, h, i] = sum_d dO[i, d] O[i, d]
//   attn_bwd        per (sequence, head, 64-key tile): P^T, dP^T, dS^T
//                   recomputed over the query tiles at and after the key tile,
//                   dV += P^T dO, dK += dS^T Q, dQ += dS K (fp32 atomics)
//   dq_finish       dq (scaled, bf16) into the q columns of dqkv
//   embed_bwd       dwte[id] += dx (fp32 atomics), dwpe[t] = sum_b dx[b, t]
//
// Every column reduction adds in a fixed order, so those gradients repeat
// bit for bit; the two atomic sums (dQ over key tiles, wte rows over repeated
// tokens) do not.
//
// The attention kernel runs on mma.sync (m16n8k16 bf16, fp32 accumulation),
// the register-fragment form of the tensor cores, with the S^T accumulator
// reused as the A operand of dV and dK (no trip through shared memory) and
// dS^T transposed through shared memory for dQ.
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

constexpr int LNB_WARPS = 4, LNB_ROWS_PER_WARP = 8;
constexpr int LNB_ROWS_PER_BLOCK = LNB_WARPS * LNB_ROWS_PER_WARP;

// One warp per row, LNB_ROWS_PER_WARP rows per warp in a fixed order; the
// row (x, dh) stays in registers. Column partials: each warp accumulates its
// rows into its own shared-memory slice (lanes own distinct columns), then
// the block adds the slices in warp order and writes one partial row.
template <int MAXV>
__global__ void __launch_bounds__(32 * LNB_WARPS) layernorm_bwd_kernel(
    const float* __restrict__ x, const bf16* __restrict__ gamma, const float* __restrict__ dh,
    const float* __restrict__ dx_in, float* __restrict__ dx_out, bf16* __restrict__ dx_bf16,
    float* __restrict__ part_g, float* __restrict__ part_b, int M, int C) {
  extern __shared__ float lnb_smem[];   // [2][LNB_WARPS][C]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* sg = lnb_smem + (size_t)warp * C;
  float* sbt = lnb_smem + (size_t)(LNB_WARPS + warp) * C;
  pdl_wait();
  pdl_trigger();
  for (int c = lane; c < C; c += 32) {
    sg[c] = 0.f;
    sbt[c] = 0.f;
  }
  __syncwarp();
  for (int rr = 0; rr < LNB_ROWS_PER_WARP; ++rr) {
    const int row = blockIdx.x * LNB_ROWS_PER_BLOCK + warp * LNB_ROWS_PER_WARP + rr;
    if (row >= M) break;
    const float* xr = x + (size_t)row * C;
    const float* gr = dh + (size_t)row * C;
    float4 xv[MAXV], gv[MAXV], gm[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int c = (lane + 32 * i) * 4;
      if (c < C) {
        xv[i] = *reinterpret_cast<const float4*>(xr + c);
        gv[i] = *reinterpret_cast<const float4*>(gr + c);
        gm[i] = ld_bf16x4(gamma + c);
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
        const float a = xv[i].x - mean, b = xv[i].y - mean, c2 = xv[i].z - mean, d = xv[i].w - mean;
        q += (a * a + b * b) + (c2 * c2 + d * d);
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
        const float4 gx = make_float4(gv[i].x * gm[i].x, gv[i].y * gm[i].y, gv[i].z * gm[i].z, gv[i].w * gm[i].w);
        s1 += (gx.x + gx.y) + (gx.z + gx.w);
        s2 += (gx.x * xv[i].x + gx.y * xv[i].y) + (gx.z * xv[i].z + gx.w * xv[i].w);
        // column partials of dgamma (dh xh) and dbeta (dh)
        float* pg = sg + c;
        float* pb = sbt + c;
        pg[0] += gv[i].x * xv[i].x;
        pg[1] += gv[i].y * xv[i].y;
        pg[2] += gv[i].z * xv[i].z;
        pg[3] += gv[i].w * xv[i].w;
        pb[0] += gv[i].x;
        pb[1] += gv[i].y;
        pb[2] += gv[i].z;
        pb[3] += gv[i].w;
      }
    }
    const float m1 = warp_sum_f(s1) / (float)C, m2 = warp_sum_f(s2) / (float)C;
    float* dor = dx_out + (size_t)row * C;
    const float* dir = dx_in ? dx_in + (size_t)row * C : nullptr;
    bf16* dbr = dx_bf16 ? dx_bf16 + (size_t)row * C : nullptr;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int c = (lane + 32 * i) * 4;
      if (c < C) {
        float4 d;
        d.x = rstd * (gv[i].x * gm[i].x - m1 - xv[i].x * m2);
        d.y = rstd * (gv[i].y * gm[i].y - m1 - xv[i].y * m2);
        d.z = rstd * (gv[i].z * gm[i].z - m1 - xv[i].z * m2);
        d.w = rstd * (gv[i].w * gm[i].w - m1 - xv[i].w * m2);
        if (dir) {
          const float4 o = *reinterpret_cast<const float4*>(dir + c);
          d = make_float4(d.x + o.x, d.y + o.y, d.z + o.z, d.w + o.w);
        }
        *reinterpret_cast<float4*>(dor + c) = d;
        if (dbr) {
          uint2 u;
          u.x = pack_bf16x2(d.x, d.y);
          u.y = pack_bf16x2(d.z, d.w);
          *reinterpret_cast<uint2*>(dbr + c) = u;
        }
      }
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int w = 0; w < LNB_WARPS; ++w) {
      a += lnb_smem[(size_t)w * C + c];
      b += lnb_smem[(size_t)(LNB_WARPS + w) * C + c];
    }
    part_g[(size_t)blockIdx.x * C + c] = a;
    part_b[(size_t)blockIdx.x * C + c] = b;
  }
}

constexpr int COL_ROWS = 128;

// Column sums of rows [blockIdx.y * COL_ROWS, +COL_ROWS) of a [M, N] matrix
// (bf16 or fp32, row pitch ld); thread = 8 consecutive columns, rows in order.
template <typename T>
__global__ void __launch_bounds__(256) col_partials_kernel(const T* __restrict__ a, long long ld, int M, int N,
                                                           float* __restrict__ part) {
  const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  pdl_wait();
  pdl_trigger();
  if (c0 < N) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int r0 = blockIdx.y * COL_ROWS, r1 = min(M, r0 + COL_ROWS);
    for (int r = r0; r < r1; ++r) {
      const T* p = a + (size_t)r * ld + c0;
      if constexpr (sizeof(T) == 2) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * j] += __uint_as_float(w[j] << 16);
          acc[2 * j + 1] += __uint_as_float(w[j] & 0xffff0000u);
        }
      } else {
        const float4 u = *reinterpret_cast<const float4*>(p);
        const float4 v = *reinterpret_cast<const float4*>(p + 4);
        acc[0] += u.x;
        acc[1] += u.y;
        acc[2] += u.z;
        acc[3] += u.w;
        acc[4] += v.x;
        acc[5] += v.y;
        acc[6] += v.z;
        acc[7] += v.w;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) part[(size_t)blockIdx.y * N + c0 + j] = acc[j];
  }
}

// out[c] = sum over p of part[p, c], p in order.
__global__ void __launch_bounds__(256) col_reduce_kernel(const float* __restrict__ part, int P, int N,
                                                         float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (c < N) {
    float s = 0.f;
    for (int p = 0; p < P; ++p) s += part[(size_t)p * N + c];
    out[c] = s;
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

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// two bf16 from two rows of a row-major shared array (lo = first)
__device__ __forceinline__ uint32_t pair_rows(const bf16* lo, const bf16* hi) {
  return (uint32_t)(*reinterpret_cast<const uint16_t*>(lo)) | ((uint32_t)(*reinterpret_cast<const uint16_t*>(hi)) << 16);
}

constexpr int AB_T = 64, AB_D = 64, AB_LDS = AB_D + 8;

// Grid (T / 64 key tiles, H, B), 4 warps; warp w owns keys k0 + 16 w .. +15.
// Longest key tiles (most query tiles after them) first.
__global__ void __launch_bounds__(128) attn_bwd_kernel(const bf16* __restrict__ qkv, const bf16* __restrict__ dO,
                                                       const float* __restrict__ lse2, const float* __restrict__ Dv,
                                                       bf16* __restrict__ dqkv, float* __restrict__ dq_acc, int T,
                                                       int H, int C, float scale_log2, float scale) {
  __shared__ __align__(16) bf16 Ks[AB_T][AB_LDS];
  __shared__ __align__(16) bf16 Vs[AB_T][AB_LDS];
  __shared__ __align__(16) bf16 Qs[AB_T][AB_LDS];
  __shared__ __align__(16) bf16 dOs[AB_T][AB_LDS];
  __shared__ __align__(16) bf16 dSs[AB_T][AB_LDS];   // dS^T: [key][query]
  __shared__ float lse_s[AB_T], dv_s[AB_T];
  const int kt = blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int k0 = kt * AB_T;
  const int QT = (T + AB_T - 1) / AB_T;
  const size_t ld = 3 * (size_t)C;
  const bf16* base = qkv + (size_t)b * T * ld;
  const bf16* dob = dO + (size_t)b * T * C + h * AB_D;
  const float* lb = lse2 + ((size_t)b * H + h) * T;
  const float* db = Dv + ((size_t)b * H + h) * T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  constexpr int CH = AB_D / 8;
  pdl_wait();
  pdl_trigger();

  for (int i = tid; i < AB_T * CH; i += 128) {
    const int r = i / CH, c = (i % CH) * 8;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (k0 + r < T) {
      const bf16* src = base + (size_t)(k0 + r) * ld + h * AB_D + c;
      kv = *reinterpret_cast<const uint4*>(src + C);
      vv = *reinterpret_cast<const uint4*>(src + 2 * C);
    }
    *reinterpret_cast<uint4*>(&Ks[r][c]) = kv;
    *reinterpret_cast<uint4*>(&Vs[r][c]) = vv;
  }
  __syncthreads();
  const int wr = warp * 16;
  uint32_t kf[AB_D / 16][4], vf[AB_D / 16][4];
#pragma unroll
  for (int ks = 0; ks < AB_D / 16; ++ks) {
    kf[ks][0] = *reinterpret_cast<const uint32_t*>(&Ks[wr + g][ks * 16 + 2 * t]);
    kf[ks][1] = *reinterpret_cast<const uint32_t*>(&Ks[wr + g + 8][ks * 16 + 2 * t]);
    kf[ks][2] = *reinterpret_cast<const uint32_t*>(&Ks[wr + g][ks * 16 + 2 * t + 8]);
    kf[ks][3] = *reinterpret_cast<const uint32_t*>(&Ks[wr + g + 8][ks * 16 + 2 * t + 8]);
    vf[ks][0] = *reinterpret_cast<const uint32_t*>(&Vs[wr + g][ks * 16 + 2 * t]);
    vf[ks][1] = *reinterpret_cast<const uint32_t*>(&Vs[wr + g + 8][ks * 16 + 2 * t]);
    vf[ks][2] = *reinterpret_cast<const uint32_t*>(&Vs[wr + g][ks * 16 + 2 * t + 8]);
    vf[ks][3] = *reinterpret_cast<const uint32_t*>(&Vs[wr + g + 8][ks * 16 + 2 * t + 8]);
  }
  float dk[AB_D / 8][4], dv[AB_D / 8][4];
#pragma unroll
  for (int i = 0; i < AB_D / 8; ++i) dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  const int key0 = k0 + wr + g, key1 = key0 + 8;

  for (int qt = kt; qt < QT; ++qt) {
    const int q0 = qt * AB_T;
    __syncthreads();   // the previous tile's Q, dO, dS are no longer read
    for (int i = tid; i < AB_T * CH; i += 128) {
      const int r = i / CH, c = (i % CH) * 8;
      uint4 qv = make_uint4(0, 0, 0, 0), ov = make_uint4(0, 0, 0, 0);
      if (q0 + r < T) {
        qv = *reinterpret_cast<const uint4*>(base + (size_t)(q0 + r) * ld + h * AB_D + c);
        ov = *reinterpret_cast<const uint4*>(dob + (size_t)(q0 + r) * C + c);
      }
      *reinterpret_cast<uint4*>(&Qs[r][c]) = qv;
      *reinterpret_cast<uint4*>(&dOs[r][c]) = ov;
    }
    if (tid < AB_T) {
      const bool ok = q0 + tid < T;
      lse_s[tid] = ok ? lb[q0 + tid] : 0.f;
      dv_s[tid] = ok ? db[q0 + tid] : 0.f;
    }
    __syncthreads();

    // S^T = K Q^T and dP^T = V dO^T: 16 keys x 64 queries per warp
    float st[AB_T / 8][4], dpt[AB_T / 8][4];
#pragma unroll
    for (int nt = 0; nt < AB_T / 8; ++nt) {
      st[nt][0] = st[nt][1] = st[nt][2] = st[nt][3] = 0.f;
      dpt[nt][0] = dpt[nt][1] = dpt[nt][2] = dpt[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < AB_D / 16; ++ks) {
        const uint32_t q_b0 = *reinterpret_cast<const uint32_t*>(&Qs[nt * 8 + g][ks * 16 + 2 * t]);
        const uint32_t q_b1 = *reinterpret_cast<const uint32_t*>(&Qs[nt * 8 + g][ks * 16 + 2 * t + 8]);
        mma16816(st[nt], kf[ks], q_b0, q_b1);
        const uint32_t o_b0 = *reinterpret_cast<const uint32_t*>(&dOs[nt * 8 + g][ks * 16 + 2 * t]);
        const uint32_t o_b1 = *reinterpret_cast<const uint32_t*>(&dOs[nt * 8 + g][ks * 16 + 2 * t + 8]);
        mma16816(dpt[nt], vf[ks], o_b0, o_b1);
      }
    }
    // P^T = 2^(s scale_log2 - lse2) where key <= query < T, else 0;
    // dS^T = P^T (dP^T - Dv); both kept in the accumulator registers
#pragma unroll
    for (int nt = 0; nt < AB_T / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = nt * 8 + 2 * t + (e & 1);
        const int q = q0 + ql;
        const int key = e < 2 ? key0 : key1;
        const float p = (key <= q && q < T) ? ex2_approx(fmaf(st[nt][e], scale_log2, -lse_s[ql])) : 0.f;
        st[nt][e] = p;
        dpt[nt][e] = p * (dpt[nt][e] - dv_s[ql]);
      }
    }
    // dV += P^T dO and dK += dS^T Q: A from the accumulators, B = dO or Q
    // rows (k = query) read column-wise
#pragma unroll
    for (int kk = 0; kk < AB_T / 16; ++kk) {
      uint32_t pa[4], sa[4];
      pa[0] = pack_bf16x2(st[2 * kk][0], st[2 * kk][1]);
      pa[1] = pack_bf16x2(st[2 * kk][2], st[2 * kk][3]);
      pa[2] = pack_bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3]);
      sa[0] = pack_bf16x2(dpt[2 * kk][0], dpt[2 * kk][1]);
      sa[1] = pack_bf16x2(dpt[2 * kk][2], dpt[2 * kk][3]);
      sa[2] = pack_bf16x2(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]);
      sa[3] = pack_bf16x2(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3]);
      const int qr = kk * 16 + 2 * t;
#pragma unroll
      for (int dn = 0; dn < AB_D / 8; ++dn) {
        const int dc = dn * 8 + g;
        mma16816(dv[dn], pa, pair_rows(&dOs[qr][dc], &dOs[qr + 1][dc]), pair_rows(&dOs[qr + 8][dc], &dOs[qr + 9][dc]));
        mma16816(dk[dn], sa, pair_rows(&Qs[qr][dc], &Qs[qr + 1][dc]), pair_rows(&Qs[qr + 8][dc], &Qs[qr + 9][dc]));
      }
      // dS^T rows of this warp into shared memory for dQ
      *reinterpret_cast<uint32_t*>(&dSs[wr + g][kk * 16 + 2 * t]) = sa[0];
      *reinterpret_cast<uint32_t*>(&dSs[wr + g + 8][kk * 16 + 2 * t]) = sa[1];
      *reinterpret_cast<uint32_t*>(&dSs[wr + g][kk * 16 + 2 * t + 8]) = sa[2];
      *reinterpret_cast<uint32_t*>(&dSs[wr + g + 8][kk * 16 + 2 * t + 8]) = sa[3];
    }
    __syncthreads();
    // dQ rows wr..wr+15 of this query tile += dS K over the tile's 64 keys
    float dq[AB_D / 8][4];
#pragma unroll
    for (int i = 0; i < AB_D / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < AB_T / 16; ++kk) {
      const int kr = kk * 16 + 2 * t;   // key rows of dS^T
      uint32_t a[4];
      a[0] = pair_rows(&dSs[kr][wr + g], &dSs[kr + 1][wr + g]);
      a[1] = pair_rows(&dSs[kr][wr + g + 8], &dSs[kr + 1][wr + g + 8]);
      a[2] = pair_rows(&dSs[kr + 8][wr + g], &dSs[kr + 9][wr + g]);
      a[3] = pair_rows(&dSs[kr + 8][wr + g + 8], &dSs[kr + 9][wr + g + 8]);
#pragma unroll
      for (int dn = 0; dn < AB_D / 8; ++dn) {
        const int dc = dn * 8 + g;
        mma16816(dq[dn], a, pair_rows(&Ks[kr][dc], &Ks[kr + 1][dc]), pair_rows(&Ks[kr + 8][dc], &Ks[kr + 9][dc]));
      }
    }
    const int qa = q0 + wr + g, qb = qa + 8;
#pragma unroll
    for (int dn = 0; dn < AB_D / 8; ++dn) {
      const int col = h * AB_D + dn * 8 + 2 * t;
      if (qa < T) {
        float* p = dq_acc + ((size_t)b * T + qa) * C + col;
        atomicAdd(p, dq[dn][0]);
        atomicAdd(p + 1, dq[dn][1]);
      }
      if (qb < T) {
        float* p = dq_acc + ((size_t)b * T + qb) * C + col;
        atomicAdd(p, dq[dn][2]);
        atomicAdd(p + 1, dq[dn][3]);
      }
    }
  }
  // dK (scaled) and dV of this warp's 16 keys into dqkv
  bf16* ob = dqkv + (size_t)b * T * ld + h * AB_D;
#pragma unroll
  for (int dn = 0; dn < AB_D / 8; ++dn) {
    const int col = dn * 8 + 2 * t;
    if (key0 < T) {
      *reinterpret_cast<uint32_t*>(ob + (size_t)key0 * ld + C + col) = pack_bf16x2(dk[dn][0] * scale, dk[dn][1] * scale);
      *reinterpret_cast<uint32_t*>(ob + (size_t)key0 * ld + 2 * C + col) = pack_bf16x2(dv[dn][0], dv[dn][1]);
    }
    if (key1 < T) {
      *reinterpret_cast<uint32_t*>(ob + (size_t)key1 * ld + C + col) = pack_bf16x2(dk[dn][2] * scale, dk[dn][3] * scale);
      *reinterpret_cast<uint32_t*>(ob + (size_t)key1 * ld + 2 * C + col) = pack_bf16x2(dv[dn][2], dv[dn][3]);
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
int col_sum_blocks(int M) { return (M + COL_ROWS - 1) / COL_ROWS; }

cudaError_t layernorm_bwd_launch(const float* x, const void* gamma, const float* dh, const float* dx_in,
                                 float* dx_out, void* dx_bf16, float* part, float* dgamma, float* dbeta, int M, int C,
                                 cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (C > 2048 || (C & 3)) return cudaErrorInvalidValue;
  const int blocks = layernorm_bwd_blocks(M);
  const size_t smem = (size_t)2 * LNB_WARPS * C * sizeof(float);
  float* pg = part;
  float* pb = part + (size_t)blocks * C;
  const bf16* gm = static_cast<const bf16*>(gamma);
  bf16* dbf = static_cast<bf16*>(dx_bf16);
  // the largest shared-memory need (C = 2048) once per device, outside any stream capture
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaError_t e = cudaSuccess;
  if (!attr_done[dev]) {
    const int most = 2 * LNB_WARPS * 2048 * (int)sizeof(float);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<13>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(layernorm_bwd_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
#define G2_LNB(MV)                                                                                                   \
  e = launch_pdl(layernorm_bwd_kernel<MV>, dim3(blocks), dim3(32 * LNB_WARPS), smem, s, x, gm, dh, dx_in, dx_out,   \
                 dbf, pg, pb, M, C);
  if (C <= 512) {
    G2_LNB(4)
  } else if (C <= 1024) {
    G2_LNB(8)
  } else if (C <= 1664) {
    G2_LNB(13)
  } else {
    G2_LNB(16)
  }
#undef G2_LNB
  if (e != cudaSuccess) return e;
  e = launch_pdl(col_reduce_kernel, dim3((C + 255) / 256), dim3(256), 0, s, (const float*)pg, blocks, C, dgamma);
  if (e == cudaSuccess)
    e = launch_pdl(col_reduce_kernel, dim3((C + 255) / 256), dim3(256), 0, s, (const float*)pb, blocks, C, dbeta);
  return e;
}

cudaError_t col_sum_launch(const void* a, bool a_bf16, long long ld, int M, int N, float* part, float* out,
                           cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (N % 8) return cudaErrorInvalidValue;
  const int P = col_sum_blocks(M);
  const dim3 grid((N / 8 + 255) / 256, P);
  cudaError_t e = a_bf16 ? launch_pdl(col_partials_kernel<bf16>, grid, dim3(256), 0, s, static_cast<const bf16*>(a),
                                      ld, M, N, part)
                         : launch_pdl(col_partials_kernel<float>, grid, dim3(256), 0, s, static_cast<const float*>(a),
                                      ld, M, N, part);
  if (e == cudaSuccess)
    e = launch_pdl(col_reduce_kernel, dim3((N + 255) / 256), dim3(256), 0, s, (const float*)part, P, N, out);
  return e;
}

cudaError_t attention_bwd_launch(const void* qkv, const void* y, const void* dy, const float* lse2, float* Dv,
                                 float* dq_acc, void* dqkv, int B, int T, int H, int C, cudaStream_t s) {
  if (B <= 0 || T <= 0) return cudaSuccess;
  if (C / H != AB_D || C % 8) return cudaErrorInvalidValue;
  const bf16* q = static_cast<const bf16*>(qkv);
  const bf16* o = static_cast<const bf16*>(y);
  const bf16* d = static_cast<const bf16*>(dy);
  bf16* out = static_cast<bf16*>(dqkv);
  const int M = B * T;
  cudaError_t e = cudaMemsetAsync(dq_acc, 0, (size_t)M * C * sizeof(float), s);
  if (e == cudaSuccess) e = launch_pdl(attn_bwd_dvec_kernel, dim3((M + 7) / 8), dim3(256), 0, s, d, o, Dv, B, T, H, C);
  const float scale = (float)(1.0 / sqrt((double)AB_D));
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)AB_D));
  if (e == cudaSuccess)
    e = launch_pdl(attn_bwd_kernel, dim3((T + AB_T - 1) / AB_T, H, B), dim3(128), 0, s, q, d, lse2, (const float*)Dv,
                   out, dq_acc, T, H, C, scale_log2, scale);
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
