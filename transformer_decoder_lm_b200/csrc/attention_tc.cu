// attention_tc.cu - causal flash attention on tcgen05 / TMEM / TMA (sm_100a, d_head 64).
//
// Per sequence b, head h and 128-query tile: y = softmax(q k^T / sqrt(D),
// -inf where key j > query i) v ("Reproducing GPT-2 124M", sections 2.1-2.2;
// "Hand-writing GPT-2 from scratch: the Transformer decoder core modules in
// PyTorch", section 3.3: key j is visible iff j <= i), online over 128-key
// tiles so the T x T score matrix never exists.
//
// Persistent CTAs, 6 warps, two per SM, each taking (b, h, query tile) items:
//   warp 0     TMA: the 128x64 Q box once, then K and V boxes of 128 keys x 64
//              into a 2-deep ring, all read in place from the c_attn output
//              through a 3-D map [B, T, 3C] (rows past T read as zero).
//   warp 1     tcgen05.mma: S = Q K^T (M=128, N=128, K=64) into TMEM, then
//              O += P V (M=128, N=64, K=128; P from TMEM, V used MN-major
//              straight from the TMA box) into a TMEM accumulator. S of tile j+1 is issued while
//              the softmax warps work on tile j.
//   warps 2-5  one thread per query row: read the S row from TMEM, scale by
//              log2(e)/sqrt(D), mask the diagonal tile, keep the running max m
//              and sum l in registers, write P = exp2(s - m) as bf16 pairs
//              into TMEM, where the PV product reads it as its A operand. The max
//              used for P is raised only when the row max grows by more than
//              2^8; then the O row in TMEM is rescaled first (tcgen05.ld / st).
//              At the end O / l goes out through smem and a 3-D TMA store
//              (rows past T are not written).
// Key tiles above the diagonal are never loaded or multiplied; the fully
// masked 32-key chunks of a diagonal tile skip their exponentials. Items are
// taken longest first from a device counter.
//
// Every wait is bounded (common.cuh); on a timeout the CTA records
// GPT2_ERR_DEVICE_TIMEOUT, drains its copies and MMAs, frees TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace g2 {

namespace {
constexpr int AT_BQ = 128, AT_BK = 128, AT_D = 64;
constexpr int AT_THREADS = 192;
constexpr int TILE_BYTES = 128 * 64 * 2;                 // one 128 x 64 bf16 box
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;                // 2 stages
constexpr int OFF_V = OFF_K + 2 * TILE_BYTES;            // 2 stages
constexpr int OFF_P = OFF_V + 2 * TILE_BYTES;            // output staging, 4 x (32 rows x 128 B)
constexpr int OFF_BAR = OFF_P + TILE_BYTES;
constexpr int NUM_BARS = 16;
constexpr int AT_SMEM = OFF_BAR + NUM_BARS * 8 + 16;   // + TMEM holder, abort flag, item slots
constexpr uint32_t TMEM_COLS = 256;   // S: cols [0,128) fp32, O: [128,192) fp32, P: [192,256) bf16 pairs
constexpr uint32_t TM_S = 0, TM_O = 128, TM_P = 192;
constexpr float RESCALE_THRESHOLD = 8.0f;                // log2 units
}  // namespace

// Persistent: gridDim.x CTAs (two per SM) take work items - one (sequence,
// head, 128-query tile) each - from a device counter, most expensive first
// (query tile qt costs qt + 1 key tiles). Work is never handed to the
// hardware block scheduler, which would only start the short tail items once
// whole SMs drain. sched[0] is the next item, sched[1] counts finished CTAs;
// the last CTA to finish sets both back to 0 for the next launch.
__global__ void __launch_bounds__(AT_THREADS, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_y, int B,
                       int T, int H, int C, float scale_log2, unsigned* sched, int* status) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;     // [2]
  uint64_t* kv_empty = bars + 4;    // [2]
  uint64_t* s_full = bars + 6;
  uint64_t* s_free = bars + 7;      // 4 softmax warps
  uint64_t* p_full = bars + 8;      // 4 softmax warps
  uint64_t* pv_done = bars + 9;
  uint64_t* drain = bars + 10;
  uint64_t* item_full = bars + 11;  // [2]
  uint64_t* item_empty = bars + 13; // [2]: the MMA warp and the 4 softmax warps
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* item_slot = reinterpret_cast<volatile int*>(tmem_holder + 2);   // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int QT = (T + AT_BQ - 1) / AT_BQ;
  const int BH = B * H;
  const int total = BH * QT;

  if ((smem_u32(smem) & 1023u) != 0) {   // the swizzled TMA boxes need 1 KB alignment
    if (threadIdx.x == 0) record_error(status, DEV_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int k = 0; k < NUM_BARS; ++k) {
      uint32_t count = 1;
      if (k == 7 || k == 8) count = 4;
      if (k == 13 || k == 14) count = 5;
      mbar_init(&bars[k], count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_wait();   // qkv (and the schedule counter's reset) come from earlier kernels

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      uint32_t g = 0;                      // key tiles issued so far, over all items
      uint32_t issued = 0, issued_parity = 0, q_issued = 0, q_parity = 0;
      for (int it = 0; ok; ++it) {
        const int slot = it & 1;
        if (!mbar_wait(&item_empty[slot], ((it >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const unsigned rank = atomicAdd(&sched[0], 1u);
        const int item = rank < (unsigned)total ? (int)rank : -1;
        item_slot[slot] = item;
        mbar_arrive(&item_full[slot]);
        if (item < 0) break;
        const int qt = QT - 1 - item / BH, bh = item % BH;
        const int b = bh / H, h = bh % H;
        if (it > 0 && !mbar_wait(q_empty, (it - 1) & 1, abort_flag)) {   // S of the last item no longer reads Q
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(q_full, TILE_BYTES);
        tma_load_3d(smem + OFF_Q, &tm_qkv, q_full, h * AT_D, qt * AT_BQ, b);
        q_issued = 1;
        q_parity = it & 1;
        for (int j = 0; j <= qt; ++j, ++g) {
          const int st = g & 1;
          const uint32_t ph = (g >> 1) & 1;
          if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[st], 2 * TILE_BYTES);
          tma_load_3d(smem + OFF_K + st * TILE_BYTES, &tm_qkv, &kv_full[st], C + h * AT_D, j * AT_BK, b);
          tma_load_3d(smem + OFF_V + st * TILE_BYTES, &tm_qkv, &kv_full[st], 2 * C + h * AT_D, j * AT_BK, b);
          issued |= 1u << st;
          issued_parity = (issued_parity & ~(1u << st)) | (ph << st);
        }
      }
      if (!ok) {
        record_error(status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
      // every issued copy lands before the CTA can exit (bounded)
      volatile int no_abort = 0;
      if (q_issued) mbar_wait(q_full, q_parity, &no_abort);
      for (int st = 0; st < 2; ++st)
        if (issued & (1u << st)) mbar_wait(&kv_full[st], (issued_parity >> st) & 1u, &no_abort);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(AT_BQ, AT_BK);
      constexpr uint32_t IDESC_O = idesc_bf16_f32_bmn(AT_BQ, AT_D);
      const uint32_t tS = tmem_base + TM_S, tO = tmem_base + TM_O, tP = tmem_base + TM_P;
      const uint64_t qdesc = sdesc_kmajor_sw128(smem_u32(smem + OFF_Q));
      bool ok = true;
      uint32_t g = 0;                      // key tiles consumed so far, over all items
      for (int it = 0; ok; ++it) {
        const int slot = it & 1;
        if (!mbar_wait(&item_full[slot], (it >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int item = item_slot[slot];
        mbar_arrive(&item_empty[slot]);
        if (item < 0) break;
        const int n_kv = QT - item / BH;   // qt + 1
        // S of the item's first tile: its K has landed and the softmax warps
        // have read the previous S
        if (!mbar_wait(q_full, it & 1, abort_flag) || !mbar_wait(&kv_full[g & 1], (g >> 1) & 1, abort_flag) ||
            (g > 0 && !mbar_wait(s_free, (g - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          const uint64_t kdesc = sdesc_kmajor_sw128(smem_u32(smem + OFF_K + (g & 1) * TILE_BYTES));
#pragma unroll
          for (int k = 0; k < AT_D / 16; ++k) mma_bf16_ss(tS, qdesc + 2 * k, kdesc + 2 * k, IDESC_S, k > 0);
          mma_commit(s_full);
        }
        if (n_kv == 1) mma_commit(q_empty);
        for (int j = 0; j < n_kv; ++j) {
          const uint32_t gj = g + j;
          if (j + 1 < n_kv) {   // S of the next tile, overlapping the softmax of this one
            const uint32_t gn = gj + 1;
            if (!mbar_wait(&kv_full[gn & 1], (gn >> 1) & 1, abort_flag) || !mbar_wait(s_free, gj & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kdesc = sdesc_kmajor_sw128(smem_u32(smem + OFF_K + (gn & 1) * TILE_BYTES));
#pragma unroll
            for (int k = 0; k < AT_D / 16; ++k) mma_bf16_ss(tS, qdesc + 2 * k, kdesc + 2 * k, IDESC_S, k > 0);
            mma_commit(s_full);
            if (j + 2 == n_kv) mma_commit(q_empty);   // the item's last S has been issued
          }
          if (!mbar_wait(p_full, gj & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(smem + OFF_V + (gj & 1) * TILE_BYTES);
#pragma unroll
          for (int k = 0; k < AT_BK / 16; ++k) {
            // P from TMEM: keys 16k..16k+15 are 8 packed columns; V: MN-major, 16 key rows = 2048 B
            const uint64_t vdesc = sdesc_mnmajor_sw128(v_addr + k * 2048);
            mma_bf16_ts(tO, tP + 8 * k, vdesc, IDESC_O, (j | k) != 0);
          }
          mma_commit(&kv_empty[gj & 1]);
          mma_commit(pv_done);
        }
        g += n_kv;
      }
      if (!ok) {
        record_error(status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
      mma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    // ----------------------------------------------------- softmax / output
    const int qd = warp & 3;                     // TMEM lane quadrant
    const int r = qd * 32 + lane;                // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t tS = tmem_base + TM_S + lane_off, tO = tmem_base + TM_O + lane_off;
    const uint32_t tP = tmem_base + TM_P + lane_off;
    bool ok = true;
    uint32_t g = 0;                              // key tiles processed so far, over all items
    for (int it = 0; ok; ++it) {
      const int slot = it & 1;
      if (!mbar_wait(&item_full[slot], (it >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      const int item = item_slot[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[slot]);
      if (item < 0) break;
      const int qt = QT - 1 - item / BH, bh = item % BH;
      const int b = bh / H, h = bh % H;
      const int q0 = qt * AT_BQ;
      const int i = q0 + r;                      // query position in the sequence
      const int n_kv = qt + 1;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n_kv; ++j) {
        const uint32_t gj = g + j;
        if (!mbar_wait(s_full, gj & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the whole S row: four TMEM loads, one wait, then release S to the MMA warp
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tS + c * 32, sr[c]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);

        const int key0 = j * AT_BK;
        const bool diag = (j == qt);
        if (diag) {   // diagonal tile: keys after the query (or past T) get -inf
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (key0 + c * 32 + e > i || key0 + c * 32 + e >= T) sr[c][e] = __float_as_uint(-INFINITY);
        }
        float pm[8];   // 8 independent partial maxima keep the dependency chains short
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) pm[e & 7] = fmaxf(pm[e & 7], __uint_as_float(sr[c][e]));
        const float tmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        const float m_new = fmaxf(m, tmax * scale_log2);   // scale_log2 > 0
        const bool raise = m_new > m + RESCALE_THRESHOLD;
        float alpha = 1.f;
        if (raise) {
          alpha = ex2_approx(m - m_new);   // 0 on the first tile (m = -inf)
          m = m_new;
        }
        l *= alpha;
        uint32_t pk[4][16];
        float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (diag && c > qd) {   // keys of this chunk all lie after every row of this warp
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[c][e] = 0u;
            continue;
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = fmaf(__uint_as_float(sr[c][2 * e]), scale_log2, -m);
            const float x1 = fmaf(__uint_as_float(sr[c][2 * e + 1]), scale_log2, -m);
            const float p0 = ex2_approx(x0);
            const float p1 = ((e & 3) == 3) ? ex2_poly(x1) : ex2_approx(x1);   // 1 in 8 on the FMA pipe
            ls[(2 * e) & 7] += p0;
            ls[(2 * e + 1) & 7] += p1;
            pk[c][e] = pack_bf16x2(p0, p1);
          }
        }
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));

        if (gj > 0) {   // PV of the previous tile done: the P buffer is free (and O stable)
          if (!mbar_wait(pv_done, (gj - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              uint32_t o[32];
              tmem_ld_32x32b_x32(tO + c * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st_32x32b_x32(tO + c * 32, o);
            }
            tmem_st_wait();
          }
        }
        // P row r into TMEM: 128 keys as 64 columns of bf16 pairs, the A operand of O += P V
        {
          uint32_t lo[32], hi[32];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            lo[e] = pk[0][e];
            lo[16 + e] = pk[1][e];
            hi[e] = pk[2][e];
            hi[16 + e] = pk[3][e];
          }
          tmem_st_32x32b_x32(tP, lo);
          tmem_st_32x32b_x32(tP + 32, hi);
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      if (!mbar_wait(pv_done, (g + n_kv - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = 1.f / l;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tO + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[c * 16 + e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
      }
      // stage 32 rows x 128 B (128-byte swizzle) in this warp's 4 KB, then a 3-D TMA store (rows past T clipped);
      // the store has finished reading the staging before the next item reuses it
      uint8_t* stg = smem + OFF_P + qd * 4096;
      const uint32_t sb = smem_u32(stg);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_shared_v4(sb + lane * 128 + ((u ^ (lane & 7)) << 4), pk[4 * u], pk[4 * u + 1], pk[4 * u + 2],
                     pk[4 * u + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && q0 + qd * 32 < T) {
        tma_store_3d(&tm_y, stg, h * AT_D, q0 + qd * 32, b);
        bulk_commit();
        bulk_wait_all();
      }
      __syncwarp();
      g += n_kv;
    }
    if (!ok && lane == 0) {
      record_error(status, DEV_TIMEOUT);
      *abort_flag = 1;
    }
  }

  __syncthreads();
  if (threadIdx.x == 0) {
    // the last CTA to finish resets the schedule for the next launch
    __threadfence();
    if (atomicAdd(&sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&sched[0], 0u);
      atomicExch(&sched[1], 0u);
      __threadfence();
    }
    pdl_trigger();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

namespace {
__device__ unsigned g_attn_sched[2];   // schedule counters of gpt2_op_attention's launches (zero at load)
}

cudaError_t attention_tc_launch(const void* qkv, void* y, int B, int T, int H, int C, unsigned* sched, int* status,
                                cudaStream_t s) {
  if (B <= 0 || T <= 0) return cudaSuccess;
  if (C / H != AT_D) return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  static int sms[64] = {};
  static unsigned* own_sched[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&own_sched[dev]), g_attn_sched);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (sched == nullptr) sched = own_sched[dev];
  CUtensorMap tq, ty;
  // qkv as [B][T][3C], boxes of 64 columns x 128 rows; y as [B][T][C], boxes of 64 x 32.
  if (!make_tmap_3d_bf16(&tq, qkv, 3 * (uint64_t)C, T, B, 3 * (uint64_t)C, (uint64_t)T * 3 * C, 64, 128) ||
      !make_tmap_3d_bf16(&ty, y, C, T, B, C, (uint64_t)T * C, 64, 32))
    return cudaErrorInvalidValue;
  const int QT = (T + AT_BQ - 1) / AT_BQ;
  const int items = B * H * QT;
  const int grid = items < 2 * sms[dev] ? items : 2 * sms[dev];
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)AT_D));
  return launch_pdl(attn_fwd_tc_kernel, dim3(grid), dim3(AT_THREADS), AT_SMEM, s, tq, ty, B, T, H, C, scale_log2,
                    sched, status);
}

}  // namespace g2
