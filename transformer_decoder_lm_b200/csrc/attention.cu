// attention.cu - causal multi-head self-attention (flash-style, online softmax).
//
// Per sequence b and head h: y_h = softmax(q_h k_h^T / sqrt(D) with -inf where
// key j > query i) v_h, heads concatenated ("Reproducing GPT-2 124M",
// sections 2.1-2.2: split of the c_attn output into q, k, v by n_embd, the
// head view, the 1/sqrt(d_head) scale and the masked_fill before softmax;
// "Hand-writing GPT-2 from scratch: the Transformer decoder core modules in
// PyTorch", section 3.3: key j visible iff j <= i).
//
// q, k and v are read in place from the c_attn output [B*T, 3C] (head h of
// q at columns h*D, of k at C + h*D, of v at 2C + h*D), so the split and the
// [B,T,H,D] -> [B,H,T,D] transpose cost no pass over memory, and y is
// written straight into the merged [B*T, C] layout c_proj reads.
//
// bf16 path: 64 queries per CTA (16 per warp), 64-key tiles; S = Q K^T and
// O += P V on the tensor cores with fp32 accumulation, softmax state (row
// max, row sum) in fp32 registers, exp2 with the scale folded into log2(e).
// Key tiles wholly above the diagonal are never visited; the diagonal tile
// applies the mask per element. No score matrix is ever stored.
//
// fp32 path: one warp per query row, keys split over lanes, exact expf;
// partial (max, sum, o) merged across lanes at the end.
#include <math.h>

#include "common.cuh"
#include "decode.h"
#include "kernels.h"

namespace g2 {

__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_u16(const bf16* lo, const bf16* hi) {
  return (uint32_t)(*reinterpret_cast<const uint16_t*>(lo)) |
         ((uint32_t)(*reinterpret_cast<const uint16_t*>(hi)) << 16);
}

template <int D>
__global__ void __launch_bounds__(128) attn_fwd_bf16_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ y,
                                                            int T, int H, int C, float scale_log2) {
  constexpr int BQ = 64, BKV = 64, LDS = D + 8;
  __shared__ __align__(16) bf16 Qs[BQ][LDS];
  __shared__ __align__(16) bf16 Ks[BKV][LDS];
  __shared__ __align__(16) bf16 Vs[BKV][LDS];

  const int qb = gridDim.x - 1 - blockIdx.x;   // longest (most key tiles) first
  const int h = blockIdx.y, b = blockIdx.z;
  const int q0 = qb * BQ;
  const size_t ld = 3 * (size_t)C;
  const bf16* base = qkv + (size_t)b * T * ld;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  constexpr int CH = D / 8;   // 16-byte chunks per row

  for (int i = tid; i < BQ * CH; i += 128) {
    const int r = i / CH, c = (i % CH) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (q0 + r < T) v = *reinterpret_cast<const uint4*>(base + (size_t)(q0 + r) * ld + h * D + c);
    *reinterpret_cast<uint4*>(&Qs[r][c]) = v;
  }
  __syncthreads();
  const int wr = warp * 16;
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qf[ks][0] = *reinterpret_cast<const uint32_t*>(&Qs[wr + g][ks * 16 + 2 * t]);
    qf[ks][1] = *reinterpret_cast<const uint32_t*>(&Qs[wr + g + 8][ks * 16 + 2 * t]);
    qf[ks][2] = *reinterpret_cast<const uint32_t*>(&Qs[wr + g][ks * 16 + 2 * t + 8]);
    qf[ks][3] = *reinterpret_cast<const uint32_t*>(&Qs[wr + g + 8][ks * 16 + 2 * t + 8]);
  }

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int row0 = q0 + wr + g, row1 = row0 + 8;
  const int q_last = min(q0 + BQ, T) - 1;
  const int n_kv = q_last / BKV + 1;

  for (int kt = 0; kt < n_kv; ++kt) {
    const int k0 = kt * BKV;
    __syncthreads();
    for (int i = tid; i < BKV * CH; i += 128) {
      const int r = i / CH, c = (i % CH) * 8;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (k0 + r < T) {
        const bf16* src = base + (size_t)(k0 + r) * ld + h * D + c;
        kv = *reinterpret_cast<const uint4*>(src + C);
        vv = *reinterpret_cast<const uint4*>(src + 2 * C);
      }
      *reinterpret_cast<uint4*>(&Ks[r][c]) = kv;
      *reinterpret_cast<uint4*>(&Vs[r][c]) = vv;
    }
    __syncthreads();

    float s[BKV / 8][4];
#pragma unroll
    for (int nt = 0; nt < BKV / 8; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&Ks[nt * 8 + g][ks * 16 + 2 * t]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&Ks[nt * 8 + g][ks * 16 + 2 * t + 8]);
        mma_16816_bf16(s[nt], qf[ks], b0, b1);
      }
    }
    // scale (into log2 units) and causal mask
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < BKV / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + nt * 8 + 2 * t + (e & 1);
        const int row = (e < 2) ? row0 : row1;
        float v = s[nt][e] * scale_log2;
        if (key > row || key >= T) v = -INFINITY;
        s[nt][e] = v;
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(mrow[0], mx0), mn1 = fmaxf(mrow[1], mx1);
    const float al0 = exp2f(mrow[0] - mn0), al1 = exp2f(mrow[1] - mn1);
    float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < BKV / 8; ++nt) {
      s[nt][0] = exp2f(s[nt][0] - mn0);
      s[nt][1] = exp2f(s[nt][1] - mn0);
      s[nt][2] = exp2f(s[nt][2] - mn1);
      s[nt][3] = exp2f(s[nt][3] - mn1);
      sum0 += s[nt][0] + s[nt][1];
      sum1 += s[nt][2] + s[nt][3];
    }
    lrow[0] = lrow[0] * al0 + sum0;
    lrow[1] = lrow[1] * al1 + sum1;
    mrow[0] = mn0;
    mrow[1] = mn1;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o[i][0] *= al0;
      o[i][1] *= al0;
      o[i][2] *= al1;
      o[i][3] *= al1;
    }
    // O += P V (P re-used from the S accumulator layout as the A operand)
#pragma unroll
    for (int kk = 0; kk < BKV / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) {
        const int kr = kk * 16 + 2 * t, dc = dn * 8 + g;
        const uint32_t b0 = pack_u16(&Vs[kr][dc], &Vs[kr + 1][dc]);
        const uint32_t b1 = pack_u16(&Vs[kr + 8][dc], &Vs[kr + 9][dc]);
        mma_16816_bf16(o[dn], pa, b0, b1);
      }
    }
  }

  float l0 = lrow[0], l1 = lrow[1];
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  bf16* yb = y + (size_t)b * T * C + h * D;
#pragma unroll
  for (int dn = 0; dn < D / 8; ++dn) {
    const int col = dn * 8 + 2 * t;
    if (row0 < T)
      *reinterpret_cast<uint32_t*>(yb + (size_t)row0 * C + col) = pack_bf16x2(o[dn][0] * inv0, o[dn][1] * inv0);
    if (row1 < T)
      *reinterpret_cast<uint32_t*>(yb + (size_t)row1 * C + col) = pack_bf16x2(o[dn][2] * inv1, o[dn][3] * inv1);
  }
}

template <int D>
__global__ void __launch_bounds__(128) attn_fwd_f32_kernel(const float* __restrict__ qkv, float* __restrict__ y,
                                                           int B, int T, int H, int C, float scale) {
  __shared__ float qs[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long gw = (long)blockIdx.x * 4 + warp;
  const bool active = gw < (long)B * H * T;
  int i = 0, h = 0, b = 0;
  if (active) {
    i = (int)(gw % T);
    h = (int)((gw / T) % H);
    b = (int)(gw / ((long)T * H));
  }
  const size_t ld = 3 * (size_t)C;
  const float* base = qkv + (size_t)b * T * ld;
  if (active)
    for (int d = lane; d < D; d += 32) qs[warp][d] = base[(size_t)i * ld + h * D + d];
  __syncwarp();
  if (!active) return;
  float m = -INFINITY, l = 0.f, o[D];
#pragma unroll
  for (int d = 0; d < D; ++d) o[d] = 0.f;
  for (int j = lane; j <= i; j += 32) {
    const float* k = base + (size_t)j * ld + C + h * D;
    const float* v = k + C;
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) s = fmaf(qs[warp][d], k[d], s);
    s *= scale;
    const float mn = fmaxf(m, s);
    const float a = expf(m - mn), p = expf(s - mn);
    l = l * a + p;
#pragma unroll
    for (int d = 0; d < D; ++d) o[d] = o[d] * a + p * v[d];
    m = mn;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
    const float mn = fmaxf(m, m2);
    const float a = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float a2 = (m2 == -INFINITY) ? 0.f : expf(m2 - mn);
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const float o2 = __shfl_xor_sync(0xffffffffu, o[d], off);
      o[d] = o[d] * a + o2 * a2;
    }
    l = l * a + l2 * a2;
    m = mn;
  }
  float* yr = y + ((size_t)b * T + i) * C + h * D;
  const float inv = 1.f / l;
#pragma unroll
  for (int d = 0; d < D; ++d)
    if ((d & 31) == lane) yr[d] = o[d] * inv;
}

cudaError_t attention_launch(bool bf16_, const void* qkv, void* y, int B, int T, int H, int C,
                             const AttnScratch* scratch, int* status, cudaStream_t s) {
  (void)status;
  if (B <= 0 || T <= 0) return cudaSuccess;
  const int D = C / H;
  if (bf16_) {
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    if (D == 64) return attention_tc_launch(qkv, y, B, T, H, C, scratch, status, s);
    // d_head 32 (bf16): the mma.sync kernel; no workload of the forward pass
    // at the GPT-2 sizes uses it (all have d_head 64)
    dim3 grid((T + 63) / 64, H, B);
    if (D == 32)
      attn_fwd_bf16_kernel<32><<<grid, 128, 0, s>>>(static_cast<const bf16*>(qkv), static_cast<bf16*>(y), T, H, C,
                                                    scale_log2);
    else
      return cudaErrorInvalidValue;
  } else {
    const float scale = (float)(1.0 / sqrt((double)D));
    const long rows = (long)B * H * T;
    const int grid = (int)((rows + 3) / 4);
    if (D == 64)
      attn_fwd_f32_kernel<64><<<grid, 128, 0, s>>>(static_cast<const float*>(qkv), static_cast<float*>(y), B, T, H, C,
                                                   scale);
    else if (D == 32)
      attn_fwd_f32_kernel<32><<<grid, 128, 0, s>>>(static_cast<const float*>(qkv), static_cast<float*>(y), B, T, H, C,
                                                   scale);
    else
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- decode
// One new query per (sequence b, head h) against the cached keys and values
// of positions 0..len-1 (the new one included): the scores go to shared
// memory, then max, exp and sum, then every thread (d = tid % D) sums
// p_j v_j[d] over one residue class of j; the classes are added in a fixed
// order (deterministic). Memory-bound: each cached row is read once.
template <typename T>
__device__ __forceinline__ float dec_to_f(T v);
template <>
__device__ __forceinline__ float dec_to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float dec_to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T>
__global__ void __launch_bounds__(128) attn_decode_kernel(const T* __restrict__ qkv, const T* __restrict__ cache,
                                                          T* __restrict__ y, int C, int n_ctx, int len, float scale) {
  extern __shared__ float dsm[];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int D = C / gridDim.x;
  float* q = dsm;              // [D]
  float* p = dsm + D;          // [len]
  float* red = p + len;        // [128]
  const T* qrow = qkv + (size_t)b * 3 * C + h * D;
  for (int d = tid; d < D; d += 128) q[d] = dec_to_f(qrow[d]);
  __syncthreads();
  const T* kb = cache + (size_t)b * n_ctx * 2 * C + h * D;   // row t at kb + t * 2C
  const T* vb = kb + C;
  float mx = -INFINITY;
  for (int j = tid; j < len; j += 128) {
    const T* kr = kb + (size_t)j * 2 * C;
    float sc = 0.f;
    for (int d = 0; d < D; ++d) sc = fmaf(q[d], dec_to_f(kr[d]), sc);
    sc *= scale;
    p[j] = sc;
    mx = fmaxf(mx, sc);
  }
  red[tid] = mx;
  __syncthreads();
  for (int o = 64; o > 0; o >>= 1) {
    if (tid < o) red[tid] = fmaxf(red[tid], red[tid + o]);
    __syncthreads();
  }
  mx = red[0];
  __syncthreads();
  float sum = 0.f;
  for (int j = tid; j < len; j += 128) {
    const float e = expf(p[j] - mx);
    p[j] = e;
    sum += e;
  }
  red[tid] = sum;
  __syncthreads();
  for (int o = 64; o > 0; o >>= 1) {
    if (tid < o) red[tid] += red[tid + o];
    __syncthreads();
  }
  sum = red[0];
  __syncthreads();
  const int G = 128 / D, d = tid % D, g = tid / D;
  float acc = 0.f;
  for (int j = g; j < len; j += G) acc = fmaf(p[j], dec_to_f(vb[(size_t)j * 2 * C + d]), acc);
  red[tid] = acc;
  __syncthreads();
  if (g == 0) {
    for (int k = 1; k < G; ++k) acc += red[k * D + d];
    const float out = acc / sum;
    if constexpr (sizeof(T) == 2)
      y[(size_t)b * C + h * D + d] = __float2bfloat16_rn(out);
    else
      y[(size_t)b * C + h * D + d] = out;
  }
}

// bf16 decode, split over the keys: block (h, b, split) takes up to 128
// cached positions, one per thread for the scores (each key row read with
// 16-byte loads), then (D/8 column groups) x (256 / (D/8) key classes) for
// p v with 16-byte loads; it leaves (max, sum, unnormalised o[D]) in `part`.
// attn_decode_combine_kernel merges the splits in a fixed order. Both are
// launched with programmatic dependent launch.
constexpr int DEC_KEYS = 128;

template <int D>
__global__ void __launch_bounds__(DEC_KEYS) attn_decode_part_kernel(const bf16* __restrict__ qkv,
                                                                    const bf16* __restrict__ cache,
                                                                    float* __restrict__ part, int C, int n_ctx,
                                                                    int len, float scale) {
  constexpr int DG = D / 8, KG = DEC_KEYS / DG;
  __shared__ float qs[D];
  __shared__ float ps[DEC_KEYS];
  __shared__ float red[DEC_KEYS / 32];
  __shared__ float accs[KG][D];
  const int h = blockIdx.x, b = blockIdx.y, sp = blockIdx.z, H = gridDim.x, S = gridDim.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j0 = sp * DEC_KEYS, n = min(len - j0, DEC_KEYS);   // n >= 1
  const bf16* base = cache + (size_t)b * n_ctx * 2 * C + h * D;   // key row t at base + t * 2C, value at + C
  pdl_wait();
  pdl_trigger();
  // this thread's key row in flight before the query's round trip
  uint4 kr[DG];
  if (tid < n) {
#pragma unroll
    for (int u = 0; u < DG; ++u) kr[u] = reinterpret_cast<const uint4*>(base + (size_t)(j0 + tid) * 2 * C)[u];
  }
  if (tid < D) qs[tid] = __bfloat162float(qkv[(size_t)b * 3 * C + h * D + tid]);
  __syncthreads();
  float sc = -INFINITY;
  if (tid < n) {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < DG; ++u) {
      const uint4 w = kr[u];
      const bf16* e = reinterpret_cast<const bf16*>(&w);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc = fmaf(qs[u * 8 + k], __bfloat162float(e[k]), acc);
    }
    sc = acc * scale;
  }
  float mx = sc;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < DEC_KEYS / 32; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  const float e = tid < n ? expf(sc - mx) : 0.f;
  ps[tid] = e;
  float sum = e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  sum = 0.f;
#pragma unroll
  for (int w = 0; w < DEC_KEYS / 32; ++w) sum += red[w];
  const int dg = tid % DG, kg = tid / DG;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int jj = kg; jj < n; jj += KG) {
    const uint4 w = *reinterpret_cast<const uint4*>(base + (size_t)(j0 + jj) * 2 * C + C + dg * 8);
    const bf16* v = reinterpret_cast<const bf16*>(&w);
    const float pj = ps[jj];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = fmaf(pj, __bfloat162float(v[k]), acc[k]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) accs[kg][dg * 8 + k] = acc[k];
  __syncthreads();
  float* pp = part + ((size_t)(b * H + h) * S + sp) * (D + 2);
  if (tid < D) {
    float o = 0.f;
    for (int k = 0; k < KG; ++k) o += accs[k][tid];
    pp[2 + tid] = o;
  }
  if (tid == 0) {
    pp[0] = mx;
    pp[1] = sum;
  }
}

template <int D>
__global__ void __launch_bounds__(D) attn_decode_combine_kernel(const float* __restrict__ part, bf16* __restrict__ y,
                                                                int C, int S) {
  const int h = blockIdx.x, b = blockIdx.y, H = gridDim.x, d = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const float* pp = part + (size_t)(b * H + h) * S * (D + 2);
  float m = -INFINITY;
  for (int s = 0; s < S; ++s) m = fmaxf(m, pp[s * (D + 2)]);
  float l = 0.f, o = 0.f;
  for (int s = 0; s < S; ++s) {
    const float f = expf(pp[s * (D + 2)] - m);
    l = fmaf(pp[s * (D + 2) + 1], f, l);
    o = fmaf(pp[s * (D + 2) + 2 + d], f, o);
  }
  y[(size_t)b * C + h * D + d] = __float2bfloat16_rn(o / l);
}

template <int D>
cudaError_t decode_split_launch(const void* qkv, const void* cache, void* y, float* part, int B, int H, int C,
                                int n_ctx, int len, float scale, cudaStream_t s) {
  const int S = (len + DEC_KEYS - 1) / DEC_KEYS;
  cudaError_t e = launch_pdl(attn_decode_part_kernel<D>, dim3(H, B, S), dim3(DEC_KEYS), 0, s,
                             static_cast<const bf16*>(qkv), static_cast<const bf16*>(cache), part, C, n_ctx, len,
                             scale);
  if (e == cudaSuccess)
    e = launch_pdl(attn_decode_combine_kernel<D>, dim3(H, B), dim3(D), 0, s, (const float*)part, static_cast<bf16*>(y),
                   C, S);
  return e;
}

cudaError_t attention_decode_launch(bool bf16_, const void* qkv, const void* cache, void* y, int B, int H, int C,
                                    int n_ctx, int len, float* part, size_t part_floats, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  const int D = C / H;
  if (D < 1 || D > 128 || 128 % D || len < 1 || len > n_ctx) return cudaErrorInvalidValue;
  const float scale = (float)(1.0 / sqrt((double)D));
  const int S = (len + DEC_KEYS - 1) / DEC_KEYS;
  const bool split_ok = part != nullptr && (size_t)B * H * S * (D + 2) <= part_floats;
  if (bf16_ && split_ok && (D == 64 || D == 32)) {
    if (D == 64) return decode_split_launch<64>(qkv, cache, y, part, B, H, C, n_ctx, len, scale, s);
    return decode_split_launch<32>(qkv, cache, y, part, B, H, C, n_ctx, len, scale, s);
  }
  const size_t smem = (size_t)(D + len + 128) * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  dim3 grid(H, B);
  if (bf16_)
    attn_decode_kernel<bf16><<<grid, 128, smem, s>>>(static_cast<const bf16*>(qkv), static_cast<const bf16*>(cache),
                                                     static_cast<bf16*>(y), C, n_ctx, len, scale);
  else
    attn_decode_kernel<float><<<grid, 128, smem, s>>>(static_cast<const float*>(qkv),
                                                      static_cast<const float*>(cache), static_cast<float*>(y), C,
                                                      n_ctx, len, scale);
  return cudaGetLastError();
}

}  // namespace g2
