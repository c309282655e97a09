// attention_bwd_tc.cu - causal attention backward on tcgen05 / TMEM / TMA (sm_100a, d_head 64).
//
// The gradient of y = softmax(q k^T / sqrt(D), causal) v ("Reproducing GPT-2
// 124M", sections 2.1-2.2: the attention it differentiates; "Hand-writing
// GPT-2 from scratch: the Transformer decoder core modules in PyTorch",
// section 4.3: loss.backward()). With the forward's row log-sum-exp L (log2
// units of s log2(e)/sqrt(D)) and Dv = rowsum(dO * O):
//   P  = 2^(s log2(e)/sqrt(D) - L)      (recomputed, s = q.k)
//   dV = P^T dO,   dP = dO V^T,   dS = P * (dP - Dv),
//   dK = dS^T Q / sqrt(D),   dQ = dS K / sqrt(D).
//
// One CTA per (sequence b, head h, 128-key tile kt), walking the query tiles
// qt >= kt (the causal mask keeps the others at zero). 10 warps:
//   warp 4     TMA: the K and V tiles once, then Q and dO of each query tile
//              into a 2-deep ring (3-D maps over the c_attn output and dO;
//              rows past T read as zero).
//   warp 5     tcgen05.mma, per query tile: S^T = K Q^T and dP^T = V dO^T
//              (M = 128 keys, N = 128 queries) into TMEM; then, once P^T and
//              dS^T are in shared memory, dV += P^T dO and dK += dS^T Q
//              (N = 64, accumulated in TMEM over the query tiles) and
//              dQ = dS K (M = 128 queries; dS read as the MN-major view of
//              the same dS^T tile). S of the next tile is issued before the
//              gradient products of this one, so the softmax warps work while
//              those run.
//   warps 0-3  one thread per key row: P^T and dS^T from the S^T and dP^T
//              rows in TMEM (32 queries at a time), written as bf16 into
//              128-byte-swizzled tiles that serve as the K-major A operand of
//              dV / dK and the MN-major A operand of dQ; at the end dK (scaled)
//              and dV out of TMEM through shared memory and 3-D TMA stores
//              into dqkv (rows past T clipped).
//   warps 6-9  dQ of each query tile out of TMEM (one TMEM lane quadrant
//              each) and added into the fp32 dq accumulator by TMA
//              reduce-add (the key tiles of a sequence and head add into the
//              same rows; the order of those additions is not fixed).
// Every wait is bounded (common.cuh): on a timeout the CTA records
// GPT2_ERR_DEVICE_TIMEOUT, drains its copies and MMAs, frees TMEM and exits.
#include <math.h>

#include "backward.h"
#include "common.cuh"
#include "kernels.h"

namespace g2 {

namespace {
constexpr int AB_BK = 128, AB_BQ = 128, AB_DH = 64;
constexpr int AB_THREADS = 320;
constexpr int AW_PROD = 4, AW_MMA = 5, AW_DQ0 = 6;
constexpr int AB_TILE = 128 * 64 * 2;                   // one 128 x 64 bf16 box, 16 KB
constexpr int AB_OFF_K = 0;
constexpr int AB_OFF_V = AB_OFF_K + AB_TILE;
constexpr int AB_OFF_Q = AB_OFF_V + AB_TILE;            // [2] stages
constexpr int AB_OFF_DO = AB_OFF_Q + 2 * AB_TILE;       // [2] stages
constexpr int AB_OFF_P = AB_OFF_DO + 2 * AB_TILE;       // P^T: 2 blocks of 64 queries x 128 key rows (128 B each)
constexpr int AB_OFF_DS = AB_OFF_P + 2 * AB_TILE;       // dS^T, the same layout
constexpr int AB_OFF_STG = AB_OFF_DS + 2 * AB_TILE;     // dQ staging: 4 warps x 2 x (32 rows x 128 B)
constexpr int AB_OFF_LSE = AB_OFF_STG + 4 * 8192;       // per softmax warp: L[128], Dv[128] of the query tile
constexpr int AB_OFF_BAR = AB_OFF_LSE + 4 * 256 * 4;
constexpr int AB_NBARS = 12;
constexpr int AB_SMEM = AB_OFF_BAR + AB_NBARS * 8 + 16 + 1024;   // + TMEM holder, abort flag, 1 KB alignment slack
constexpr uint32_t AB_TMEM_COLS = 512;
constexpr uint32_t TM_ST = 0, TM_DPT = 128, TM_DV = 256, TM_DK = 320, TM_DQ = 384;
static_assert(AB_SMEM <= 232448, "shared memory budget");

// 16-byte unit u of row r of a 128-byte-swizzled tile (8-row groups of 1 KB)
__device__ __forceinline__ uint32_t sw128(uint32_t base, int r, int u) {
  return base + (uint32_t)r * 128u + ((uint32_t)(u ^ (r & 7)) << 4);
}

__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* tm, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
}  // namespace

// Grid: B * H * ceil(T / 128) CTAs, key tile slowest, so the CTAs with the
// most query tiles (kt = 0) start first.
__global__ void __launch_bounds__(AB_THREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dqkv, const __grid_constant__ CUtensorMap tm_dq,
                       const float* __restrict__ lse2, const float* __restrict__ Dv, int B, int T, int H, int C,
                       float scale_log2, float scale, int* status) {
  extern __shared__ uint8_t ab_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ab_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AB_OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;    // [2]
  uint64_t* qd_empty = bars + 3;   // [2]
  uint64_t* s_full = bars + 5;     // S^T, dP^T of a query tile in TMEM
  uint64_t* soft_done = bars + 6;  // 4 softmax warps: S^T, dP^T read; P^T, dS^T in shared memory
  uint64_t* pds_free = bars + 7;   // the gradient products of a tile have read P^T, dS^T
  uint64_t* dq_full = bars + 8;
  uint64_t* dq_empty = bars + 9;   // 4 dQ warps
  uint64_t* acc_done = bars + 10;  // every MMA has completed: dK, dV final
  uint64_t* drain = bars + 11;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + AB_NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = B * H;
  const int kt = (int)blockIdx.x / BH, bh = (int)blockIdx.x - kt * BH;
  const int b = bh / H, h = bh - b * H;
  const int QT = (T + AB_BQ - 1) / AB_BQ;
  const int k0 = kt * AB_BK;
  const int n = QT - kt;   // query tiles kt .. QT - 1

  if (threadIdx.x == 0) {
    for (int k = 0; k < AB_NBARS; ++k) mbar_init(&bars[k], (k == 6 || k == 9) ? 4u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == AW_PROD && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dqkv);
    tma_prefetch_desc(&tm_dq);
  }
  if (warp == AW_MMA) {
    tmem_alloc(tmem_holder, AB_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_wait();   // qkv, dO, the row log-sum-exps, Dv and the zeroed dq accumulator come from earlier work
  if (threadIdx.x == 0) pdl_trigger();

  if (warp == AW_PROD) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      uint32_t issued = 0, parity = 0;
      mbar_arrive_expect_tx(kv_full, 2 * AB_TILE);
      tma_load_3d(smem + AB_OFF_K, &tm_qkv, kv_full, C + h * AB_DH, k0, b);
      tma_load_3d(smem + AB_OFF_V, &tm_qkv, kv_full, 2 * C + h * AB_DH, k0, b);
      for (int i = 0; i < n; ++i) {
        const int st = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (i >= 2 && !mbar_wait(&qd_empty[st], (use & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const int q0 = (kt + i) * AB_BQ;
        mbar_arrive_expect_tx(&qd_full[st], 2 * AB_TILE);
        tma_load_3d(smem + AB_OFF_Q + st * AB_TILE, &tm_qkv, &qd_full[st], h * AB_DH, q0, b);
        tma_load_3d(smem + AB_OFF_DO + st * AB_TILE, &tm_do, &qd_full[st], h * AB_DH, q0, b);
        issued |= 1u << st;
        parity = (parity & ~(1u << st)) | ((use & 1u) << st);
      }
      if (!ok) {
        record_error(status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
      // every issued copy lands before the CTA can exit (bounded)
      volatile int no_abort = 0;
      mbar_wait(kv_full, 0, &no_abort);
      for (int st = 0; st < 2; ++st)
        if (issued & (1u << st)) mbar_wait(&qd_full[st], (parity >> st) & 1u, &no_abort);
    }
  } else if (warp == AW_MMA) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16_f32(AB_BK, AB_BQ);                       // S^T, dP^T
      constexpr uint32_t ID_G = idesc_bf16_f32_bmn(AB_BK, AB_DH);                    // dV, dK
      constexpr uint32_t ID_Q = idesc_bf16_f32_major(AB_BQ, AB_DH, true, true);      // dQ
      const uint32_t tS = tmem + TM_ST, tDP = tmem + TM_DPT, tDV = tmem + TM_DV, tDK = tmem + TM_DK,
                     tDQ = tmem + TM_DQ;
      const uint32_t sK = smem_u32(smem + AB_OFF_K), sV = smem_u32(smem + AB_OFF_V);
      const uint32_t sP = smem_u32(smem + AB_OFF_P), sDS = smem_u32(smem + AB_OFF_DS);
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      for (int i = 0; ok && i <= n; ++i) {
        if (i < n) {
          // S^T and dP^T of query tile i once its Q, dO have landed and the
          // softmax warps are done with tile i - 1
          const int st = i & 1;
          if (!mbar_wait(&qd_full[st], (uint32_t)(i >> 1) & 1u, abort_flag) ||
              (i > 0 && !mbar_wait(soft_done, (uint32_t)(i - 1) & 1u, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sQ = smem_u32(smem + AB_OFF_Q + st * AB_TILE), sO = smem_u32(smem + AB_OFF_DO + st * AB_TILE);
#pragma unroll
          for (int k = 0; k < AB_DH / 16; ++k)
            mma_bf16_ss(tS, sdesc_kmajor_sw128(sK) + 2 * k, sdesc_kmajor_sw128(sQ) + 2 * k, ID_S, k > 0);
#pragma unroll
          for (int k = 0; k < AB_DH / 16; ++k)
            mma_bf16_ss(tDP, sdesc_kmajor_sw128(sV) + 2 * k, sdesc_kmajor_sw128(sO) + 2 * k, ID_S, k > 0);
          mma_commit(s_full);
        } else {
          if (!mbar_wait(soft_done, (uint32_t)(n - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (i > 0) {
          // the gradient products of query tile j = i - 1 (P^T, dS^T written)
          const int j = i - 1, sj = j & 1;
          if (j > 0 && !mbar_wait(dq_empty, (uint32_t)(j - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sQ = smem_u32(smem + AB_OFF_Q + sj * AB_TILE), sO = smem_u32(smem + AB_OFF_DO + sj * AB_TILE);
#pragma unroll
          for (int kk = 0; kk < AB_BQ / 16; ++kk) {
            // 16 queries per step: the K-major P^T / dS^T blocks of 64 queries
            // (+32 B per step inside a block), dO / Q rows MN-major (+2048 B)
            const uint32_t blk = (uint32_t)(kk >> 2) * 16384u;
            const uint32_t adv = 2u * (uint32_t)(kk & 3);
            mma_bf16_ss(tDV, sdesc_kmajor_sw128(sP + blk) + adv, sdesc_mnmajor_sw128(sO + kk * 2048), ID_G,
                        (j | kk) != 0);
            mma_bf16_ss(tDK, sdesc_kmajor_sw128(sDS + blk) + adv, sdesc_mnmajor_sw128(sQ + kk * 2048), ID_G,
                        (j | kk) != 0);
          }
#pragma unroll
          for (int kk = 0; kk < AB_BK / 16; ++kk)   // 16 keys per step: dS as MN-major (query blocks 16 KB apart), K MN-major
            mma_bf16_ss(tDQ, sdesc_mn_sw128(sDS + kk * 2048, 16384), sdesc_mnmajor_sw128(sK + kk * 2048), ID_Q, kk != 0);
          mma_commit(pds_free);
          mma_commit(dq_full);
          mma_commit(&qd_empty[sj]);
        }
      }
      if (!ok) {
        record_error(status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
      mma_commit(acc_done);
      mma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else if (warp < 4) {
    // ------------------------------------------------- P^T, dS^T; dK, dV out
    const int r = warp * 32 + lane;   // key row of the tile
    const int kg = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + TM_ST + lane_off, tDP = tmem + TM_DPT + lane_off;
    const uint32_t sP = smem_u32(smem + AB_OFF_P), sDS = smem_u32(smem + AB_OFF_DS);
    // this warp's copy of the query tile's -L and Dv (read as pair broadcasts)
    float* nl_w = reinterpret_cast<float*>(smem + AB_OFF_LSE) + warp * 256;
    float* dv_w = nl_w + 128;
    const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
    const float* lrow = lse2 + (size_t)bh * T;
    const float* drow = Dv + (size_t)bh * T;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int q0 = (kt + i) * AB_BQ;
      __syncwarp();   // every lane is done with the previous tile's copy
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int jq = lane + 32 * m, q = q0 + jq;
        // queries past T: -L = -inf gives P = 0 (their Q, dO rows read as zero)
        nl_w[jq] = q < T ? -lrow[q] : -INFINITY;
        dv_w[jq] = q < T ? drow[q] : 0.f;
      }
      __syncwarp();
      if (!mbar_wait(s_full, (uint32_t)i & 1u, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = i == 0;   // the only tile with keys after some of its queries
      // P, dS of queries 32c .. 32c + 31 as bf16 pairs
      auto chunk = [&](int c, uint32_t (&pk)[16], uint32_t (&dk)[16]) {
        uint32_t sv[32], dpv[32];
        tmem_ld_32x32b_x32(tS + c * 32, sv);
        tmem_ld_32x32b_x32(tDP + c * 32, dpv);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // queries jq, jq + 1 in packed fp32 pairs: P = 2^(s c - L), dS = P (dP - Dv)
          const int jq = c * 32 + 2 * e;
          const float2 nl = *reinterpret_cast<const float2*>(nl_w + jq);
          const float2 dv = *reinterpret_cast<const float2*>(dv_w + jq);
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sc2,
                                     f2_pack(nl.x, nl.y));
          float x0, x1;
          f2_unpack(x2, x0, x1);
          float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          if (diag) {
            p0 = kg <= q0 + jq ? p0 : 0.f;
            p1 = kg <= q0 + jq + 1 ? p1 : 0.f;
          }
          const uint64_t p2 = f2_pack(p0, p1);
          const uint64_t d2 = f2_mul(p2, f2_sub(f2_pack(__uint_as_float(dpv[2 * e]), __uint_as_float(dpv[2 * e + 1])),
                                                f2_pack(dv.x, dv.y)));
          float d0, d1;
          f2_unpack(d2, d0, d1);
          pk[e] = pack_bf16x2(p0, p1);
          dk[e] = pack_bf16x2(d0, d1);
        }
      };
#pragma unroll 1
      for (int cb = 0; cb < 2; ++cb) {   // the two 64-query blocks of the tile
        uint32_t pk0[16], dk0[16], pk1[16], dk1[16];
        chunk(2 * cb, pk0, dk0);
        chunk(2 * cb + 1, pk1, dk1);
        // the first block's exponentials run before the wait for the previous
        // tile's gradient products to release P^T, dS^T
        if (cb == 0 && i > 0 && !mbar_wait(pds_free, (uint32_t)(i - 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        // row r of 64-query block cb: 16-byte units 0-3 (first chunk), 4-7
        const uint32_t blk = (uint32_t)cb * 16384u;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          st_shared_v4(sw128(sP + blk, r, v), pk0[4 * v], pk0[4 * v + 1], pk0[4 * v + 2], pk0[4 * v + 3]);
          st_shared_v4(sw128(sDS + blk, r, v), dk0[4 * v], dk0[4 * v + 1], dk0[4 * v + 2], dk0[4 * v + 3]);
          st_shared_v4(sw128(sP + blk, r, 4 + v), pk1[4 * v], pk1[4 * v + 1], pk1[4 * v + 2], pk1[4 * v + 3]);
          st_shared_v4(sw128(sDS + blk, r, 4 + v), dk1[4 * v], dk1[4 * v + 1], dk1[4 * v + 2], dk1[4 * v + 3]);
        }
      }
      if (!ok) break;
      tc_fence_before();
      fence_proxy_async_smem();   // the tensor core reads P^T, dS^T next
      __syncwarp();
      if (lane == 0) mbar_arrive(soft_done);
    }
    if (ok && !mbar_wait(acc_done, 0, abort_flag)) ok = false;
    if (ok) {
      // dK / sqrt(D) and dV of this warp's 32 keys: 32 rows x 128 B each,
      // staged in the (now unused) P^T tile, 3-D TMA stores into dqkv
      tc_fence_after();
      uint8_t* stg = smem + AB_OFF_P + warp * 8192;
      const uint32_t sb = smem_u32(stg);
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        const uint32_t tacc = tmem + (m == 0 ? TM_DK : TM_DV) + lane_off;
        const float f = m == 0 ? scale : 1.f;
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(tacc + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[c * 16 + e] = pack_bf16x2(__uint_as_float(o[2 * e]) * f, __uint_as_float(o[2 * e + 1]) * f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          st_shared_v4(sw128(sb + m * 4096, lane, u), pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && k0 + warp * 32 < T) {
        tma_store_3d(&tm_dqkv, stg, C + h * AB_DH, k0 + warp * 32, b);
        tma_store_3d(&tm_dqkv, stg + 4096, 2 * C + h * AB_DH, k0 + warp * 32, b);
        bulk_commit();
      }
    }
    if (!ok && lane == 0) {
      record_error(status, DEV_TIMEOUT);
      *abort_flag = 1;
    }
    if (lane == 0) bulk_wait_all();
  } else {
    // ------------------------------------------------ dQ into the accumulator
    const int quad = warp & 3;   // TMEM lane quadrant = query rows 32 quad ..
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* stg = smem + AB_OFF_STG + (warp - AW_DQ0) * 8192;
    const uint32_t sb = smem_u32(stg);
    bool ok = true, pending = false;
    for (int j = 0; j < n; ++j) {
      if (!mbar_wait(dq_full, (uint32_t)j & 1u, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld_32x32b_x32(tmem + TM_DQ + lane_off, v0);
      tmem_ld_32x32b_x32(tmem + TM_DQ + lane_off + 32, v1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_empty);
      if (pending) {   // the previous reduce-adds have read the staging
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        st_shared_v4(sw128(sb, lane, u), v0[4 * u], v0[4 * u + 1], v0[4 * u + 2], v0[4 * u + 3]);
        st_shared_v4(sw128(sb + 4096, lane, u), v1[4 * u], v1[4 * u + 1], v1[4 * u + 2], v1[4 * u + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int q0 = (kt + j) * AB_BQ + quad * 32;
      if (lane == 0 && q0 < T) {
        tma_reduce_add_3d(&tm_dq, stg, h * AB_DH, q0, b);
        tma_reduce_add_3d(&tm_dq, stg + 4096, h * AB_DH + 32, q0, b);
        bulk_commit();
      }
      pending = true;
    }
    if (!ok && lane == 0) {
      record_error(status, DEV_TIMEOUT);
      *abort_flag = 1;
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == AW_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, AB_TMEM_COLS);
  }
}

cudaError_t attention_bwd_tc_launch(const void* qkv, const void* dy, const float* lse2, const float* Dv, float* dq_acc,
                                    void* dqkv, int B, int T, int H, int C, int* status, cudaStream_t s) {
  if (B <= 0 || T <= 0) return cudaSuccess;
  if (C / H != AB_DH || C % H || C % 64) return cudaErrorInvalidValue;
  CUtensorMap tq, tdo, tdqkv, tdq;
  if (!make_tmap_3d_bf16(&tq, qkv, 3 * (uint64_t)C, T, B, 3 * (uint64_t)C, (uint64_t)T * 3 * C, 64, 128) ||
      !make_tmap_3d_bf16(&tdo, dy, C, T, B, C, (uint64_t)T * C, 64, 128) ||
      !make_tmap_3d_bf16(&tdqkv, dqkv, 3 * (uint64_t)C, T, B, 3 * (uint64_t)C, (uint64_t)T * 3 * C, 64, 32) ||
      !make_tmap_3d_f32(&tdq, dq_acc, C, T, B, C, (uint64_t)T * C, 32, 32))
    return cudaErrorInvalidValue;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AB_SMEM);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int KT = (T + AB_BK - 1) / AB_BK;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)AB_DH));
  const float scale = (float)(1.0 / sqrt((double)AB_DH));
  return launch_pdl(attn_bwd_tc_kernel, dim3((unsigned)(KT * B * H)), dim3(AB_THREADS), AB_SMEM, s, tq, tdo, tdqkv, tdq,
                    lse2, Dv, B, T, H, C, scale_log2, scale, status);
}

}  // namespace g2
