// embed_ln.cu - embedding sum and LayerNorm kernels (HBM-bound, SIMT).
//
// embed:      x[m, :] = wte[ids[m], :] + wpe[m % T, :]        fp32 residual stream
//             ("Hand-writing GPT-2 from scratch: the Transformer decoder core
//              modules in PyTorch", section 4.1 forward step 1).
// layernorm:  out[m, :] = (x - mean) * rsqrt(var_biased + 1e-5) * g + b
//             ("Reproducing GPT-2 124M", section 2.1, hand-written LayerNorm with
//              unbiased=False; eps 1e-5 per the first page, sections 3.2/4.2).
//
// Both kernels give each row to one warp and move 16-byte (fp32) or 8-byte
// (bf16) vectors; the row stays in registers between the two passes of the
// LayerNorm statistics (mean, then the centred second moment), so x is read
// from HBM exactly once.
#include "common.cuh"
#include "kernels.h"

namespace g2 {

template <typename T>
struct Vec4;
template <>
struct Vec4<float> {
  typedef float4 raw_t;   // four elements as stored
  static __device__ __forceinline__ raw_t load_raw(const float* p) { return *reinterpret_cast<const float4*>(p); }
  static __device__ __forceinline__ float4 to_f4(raw_t r) { return r; }
  static __device__ __forceinline__ float4 load(const float* p) { return *reinterpret_cast<const float4*>(p); }
  static __device__ __forceinline__ void store(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
};
template <>
struct Vec4<bf16> {
  typedef uint2 raw_t;
  static __device__ __forceinline__ raw_t load_raw(const bf16* p) { return *reinterpret_cast<const uint2*>(p); }
  static __device__ __forceinline__ float4 to_f4(raw_t u) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
  }
  static __device__ __forceinline__ float4 load(const bf16* p) { return to_f4(load_raw(p)); }
  static __device__ __forceinline__ void store(bf16* p, float4 v) {
    uint2 u;
    u.x = pack_bf16x2(v.x, v.y);
    u.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(p) = u;
  }
};

template <typename T>
__global__ void __launch_bounds__(256) embed_kernel(const int* __restrict__ ids, const T* __restrict__ wte,
                                                    const T* __restrict__ wpe, float* __restrict__ x, int M,
                                                    int Tlen, int C, int V, int* status) {
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (row >= M) return;
  int id = ids[row];
  if (id < 0 || id >= V) {
    if (lane == 0) record_error(status, DEV_BAD_TOKEN);
    id = 0;
  }
  const int t = row % Tlen;
  const T* te = wte + (size_t)id * C;
  const T* pe = wpe + (size_t)t * C;
  float* xr = x + (size_t)row * C;
  for (int c = lane * 4; c < C; c += 128) {
    const float4 a = Vec4<T>::load(te + c);
    const float4 b = Vec4<T>::load(pe + c);
    Vec4<float>::store(xr + c, make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w));
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The embedding sum of embed_kernel and the first block's ln_1 on the row it
// just formed (bf16, C <= 128 MAXV): x = wte[id] + wpe[t] (fp32, written),
// h = LayerNorm(x; g, b) with layernorm_kernel's arithmetic.
template <int MAXV>
__global__ void __launch_bounds__(256) embed_ln_kernel(const int* __restrict__ ids, const bf16* __restrict__ wte,
                                                       const bf16* __restrict__ wpe, float* __restrict__ x,
                                                       const bf16* __restrict__ g, const bf16* __restrict__ b,
                                                       bf16* __restrict__ h, int M, int Tlen, int C, int V,
                                                       int* status) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (row >= M) return;
  int id = ids[row];
  if (id < 0 || id >= V) {
    if (lane == 0) record_error(status, DEV_BAD_TOKEN);
    id = 0;
  }
  const bf16* te = wte + (size_t)id * C;
  const bf16* pe = wpe + (size_t)(row % Tlen) * C;
  float* xr = x + (size_t)row * C;
  float4 v[MAXV];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = (lane + 32 * i) * 4;
    if (c < C) {
      const float4 a = Vec4<bf16>::load(te + c), p = Vec4<bf16>::load(pe + c);
      v[i] = make_float4(a.x + p.x, a.y + p.y, a.z + p.z, a.w + p.w);
      Vec4<float>::store(xr + c, v[i]);
      s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
  }
  const float mean = warp_sum(s) / (float)C;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = (lane + 32 * i) * 4;
    if (c < C) {
      const float a = v[i].x - mean, bb = v[i].y - mean, cc = v[i].z - mean, d = v[i].w - mean;
      q += (a * a + bb * bb) + (cc * cc + d * d);
    }
  }
  const float rstd = rsqrtf(warp_sum(q) / (float)C + 1e-5f);
  bf16* orow = h + (size_t)row * C;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = (lane + 32 * i) * 4;
    if (c < C) {
      const float4 ga = Vec4<bf16>::load(g + c), be = Vec4<bf16>::load(b + c);
      float4 o;
      o.x = (v[i].x - mean) * rstd * ga.x + be.x;
      o.y = (v[i].y - mean) * rstd * ga.y + be.y;
      o.z = (v[i].z - mean) * rstd * ga.z + be.z;
      o.w = (v[i].w - mean) * rstd * ga.w + be.w;
      Vec4<bf16>::store(orow + c, o);
    }
  }
}

// C <= 32 lanes * 4 * MAXV = 2048.
// x_save (training forward): if not NULL, also receives a copy of x, the
// LayerNorm input the backward pass differentiates at.
template <typename T, int MAXV>
__global__ void __launch_bounds__(128) layernorm_kernel(const float* __restrict__ x, const T* __restrict__ g,
                                                        const T* __restrict__ b, T* __restrict__ out, int M,
                                                        int C, float* __restrict__ x_save) {
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (row >= M) return;
  const float* xr = x + (size_t)row * C;
  // x, gamma and beta are all requested before any of them is used, so a row
  // costs one memory round trip.
  float4 v[MAXV];
  typename Vec4<T>::raw_t gg[MAXV], bt[MAXV];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = (lane + 32 * i) * 4;
    if (c < C) {
      v[i] = Vec4<float>::load(xr + c);
      gg[i] = Vec4<T>::load_raw(g + c);
      bt[i] = Vec4<T>::load_raw(b + c);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = (lane + 32 * i) * 4;
    if (c < C) s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
  if (x_save != nullptr) {
    float* xs = x_save + (size_t)row * C;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int c = (lane + 32 * i) * 4;
      if (c < C) Vec4<float>::store(xs + c, v[i]);
    }
  }
  const float mean = warp_sum(s) / (float)C;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = (lane + 32 * i) * 4;
    if (c < C) {
      const float a = v[i].x - mean, bb = v[i].y - mean, cc = v[i].z - mean, d = v[i].w - mean;
      q += (a * a + bb * bb) + (cc * cc + d * d);
    }
  }
  const float var = warp_sum(q) / (float)C;
  const float rstd = rsqrtf(var + 1e-5f);
  T* orow = out + (size_t)row * C;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = (lane + 32 * i) * 4;
    if (c < C) {
      const float4 ga = Vec4<T>::to_f4(gg[i]), be = Vec4<T>::to_f4(bt[i]);
      float4 o;
      o.x = (v[i].x - mean) * rstd * ga.x + be.x;
      o.y = (v[i].y - mean) * rstd * ga.y + be.y;
      o.z = (v[i].z - mean) * rstd * ga.z + be.z;
      o.w = (v[i].w - mean) * rstd * ga.w + be.w;
      Vec4<T>::store(orow + c, o);
    }
  }
}

cudaError_t embed_launch(bool bf16_, const int* ids, const void* wte, const void* wpe, float* x, int M, int T,
                         int C, int V, int* status, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  const int threads = 256, rows_per_block = threads / 32;
  const int grid = (M + rows_per_block - 1) / rows_per_block;
  if (bf16_)
    return launch_pdl(embed_kernel<bf16>, grid, threads, 0, s, ids, static_cast<const bf16*>(wte),
                      static_cast<const bf16*>(wpe), x, M, T, C, V, status);
  else
    embed_kernel<float><<<grid, threads, 0, s>>>(ids, static_cast<const float*>(wte),
                                                  static_cast<const float*>(wpe), x, M, T, C, V, status);
  return cudaGetLastError();
}

cudaError_t embed_ln_launch(const int* ids, const void* wte, const void* wpe, float* x, const void* g,
                            const void* b, void* h, int M, int T, int C, int V, int* status, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (C > 2048 || (C & 3)) return cudaErrorInvalidValue;
  const int threads = 256, grid = (M + 7) / 8;
  const bf16 *te = static_cast<const bf16*>(wte), *pe = static_cast<const bf16*>(wpe);
  const bf16 *gp = static_cast<const bf16*>(g), *bp = static_cast<const bf16*>(b);
  bf16* hp = static_cast<bf16*>(h);
  if (C <= 768) return launch_pdl(embed_ln_kernel<6>, grid, threads, 0, s, ids, te, pe, x, gp, bp, hp, M, T, C, V, status);
  if (C <= 1024) return launch_pdl(embed_ln_kernel<8>, grid, threads, 0, s, ids, te, pe, x, gp, bp, hp, M, T, C, V, status);
  if (C <= 1280) return launch_pdl(embed_ln_kernel<10>, grid, threads, 0, s, ids, te, pe, x, gp, bp, hp, M, T, C, V, status);
  if (C <= 1664) return launch_pdl(embed_ln_kernel<13>, grid, threads, 0, s, ids, te, pe, x, gp, bp, hp, M, T, C, V, status);
  return launch_pdl(embed_ln_kernel<16>, grid, threads, 0, s, ids, te, pe, x, gp, bp, hp, M, T, C, V, status);
}

cudaError_t layernorm_launch(bool bf16_, const float* x, const void* g, const void* b, void* out, int M, int C,
                             cudaStream_t s, float* x_save) {
  if (M <= 0) return cudaSuccess;
  if (C > 2048 || (C & 3)) return cudaErrorInvalidValue;
  const int threads = 128, rows_per_block = threads / 32;
  const int grid = (M + rows_per_block - 1) / rows_per_block;
  if (bf16_) {
    // registers per lane grow with C: pick the smallest row capacity that fits
    const bf16 *gp = static_cast<const bf16*>(g), *bp = static_cast<const bf16*>(b);
    bf16* op = static_cast<bf16*>(out);
    if (C <= 768) return launch_pdl(layernorm_kernel<bf16, 6>, grid, threads, 0, s, x, gp, bp, op, M, C, x_save);
    if (C <= 1024) return launch_pdl(layernorm_kernel<bf16, 8>, grid, threads, 0, s, x, gp, bp, op, M, C, x_save);
    if (C <= 1280) return launch_pdl(layernorm_kernel<bf16, 10>, grid, threads, 0, s, x, gp, bp, op, M, C, x_save);
    if (C <= 1664) return launch_pdl(layernorm_kernel<bf16, 13>, grid, threads, 0, s, x, gp, bp, op, M, C, x_save);
    return launch_pdl(layernorm_kernel<bf16, 16>, grid, threads, 0, s, x, gp, bp, op, M, C, x_save);
  } else {
    if (C <= 1024)
      layernorm_kernel<float, 8><<<grid, threads, 0, s>>>(x, static_cast<const float*>(g),
                                                          static_cast<const float*>(b), static_cast<float*>(out), M, C, x_save);
    else
      layernorm_kernel<float, 16><<<grid, threads, 0, s>>>(x, static_cast<const float*>(g),
                                                           static_cast<const float*>(b), static_cast<float*>(out), M,
                                                           C, x_save);
  }
  return cudaGetLastError();
}

// Fixed sinusoidal position table ("Hand-writing GPT-2 from scratch: the
// Transformer decoder core modules in PyTorch", section 3.1): element
// (pos, j) of [n_ctx, C] is sin (j even) or cos (j odd) of
// pos / 10000^(2 (j / 2) / C), computed in double and rounded once.
template <typename T>
__global__ void sinusoidal_wpe_kernel(T* __restrict__ wpe, int n_ctx, int C) {
  const long long n = (long long)n_ctx * C;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int pos = (int)(idx / C), j = (int)(idx % C), i = j >> 1;
    const double angle = (double)pos / pow(10000.0, (2.0 * i) / C);
    const double v = (j & 1) ? cos(angle) : sin(angle);
    if constexpr (sizeof(T) == 2)
      wpe[idx] = __double2bfloat16(v);
    else
      wpe[idx] = (float)v;
  }
}

cudaError_t sinusoidal_wpe_launch(bool bf16_, void* wpe, int n_ctx, int C, cudaStream_t s) {
  const long long n = (long long)n_ctx * C;
  const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  if (bf16_)
    sinusoidal_wpe_kernel<bf16><<<grid, 256, 0, s>>>(static_cast<bf16*>(wpe), n_ctx, C);
  else
    sinusoidal_wpe_kernel<float><<<grid, 256, 0, s>>>(static_cast<float*>(wpe), n_ctx, C);
  return cudaGetLastError();
}

}  // namespace g2
