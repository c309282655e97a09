// attention_tc.cu - causal flash attention on tcgen05 / TMEM / TMA (sm_100a, d_head 64).
//
// Per sequence b, head h and 128-query tile: y = softmax(q k^T / sqrt(D),
// -inf where key j > query i) v ("Reproducing GPT-2 124M", sections 2.1-2.2;
// "Hand-writing GPT-2 from scratch: the Transformer decoder core modules in
// PyTorch", section 3.3: key j is visible iff j <= i), online over 128-key
// tiles so the T x T score matrix never exists.
//
// Persistent CTAs, 8 warps, two per SM, each taking (b, h, query tile) items:
//   warp 4     TMA: the 128x64 Q box, then K and V boxes of 128 keys x 64
//              into a 2-deep ring, all read in place from the c_attn output
//              through a 3-D map [B, T, 3C] (rows past T read as zero).
//   warp 5     tcgen05.mma: S = Q K^T (M=128, N=128, K=64) into TMEM, then
//              O += P V (M=128, N=64, K=128; P from TMEM, V used MN-major
//              straight from the TMA box) into a TMEM accumulator. S of tile j+1 is issued while
//              the softmax warps work on tile j.
//   warps 0-3  one thread per query row: read the S row from TMEM, scale by
//              log2(e)/sqrt(D), mask the diagonal tile, keep the running max m
//              and sum l in registers, write P = exp2(s - m) as bf16 pairs
//              into TMEM, where the PV product reads it as its A operand
//              (scaling, sums and maxima in packed fp32 pairs and
//              three-input maxima, sm_100 forms; exponentials on the SFU).
//              The max
//              used for P is raised only when the row max grows by more than
//              2^8; then the O row in TMEM is rescaled first (tcgen05.ld / st).
//              At the end O / l goes out through smem and a 3-D TMA store
//              (rows past T are not written).
//   warps 6-7  idle; with warps 4-5 they hand registers to warps 0-3
//              (setmaxnreg), whose whole S row, P row and exponential
//              pipelines live in registers.
// Key tiles above the diagonal are never loaded or multiplied; the fully
// masked 32-key chunks of a diagonal tile skip their exponentials. Items are
// taken longest first from a device counter.
//
// A query tile's cost grows with its index (tile qt reads qt + 1 key tiles), so
// the last tiles of long sequences can set the kernel's length when there are
// few items per CTA. Those longer than twice the average share of a CTA are split into two items over the key
// ranges [0, a) and [a, qt + 1), a = ceil((qt + 1) / 2). Per 32-row quarter,
// the half that finishes first leaves its unnormalised O rows with their
// running max m and sum l in a scratch buffer and raises a ready flag; the
// other merges: with M = max(m1, m2),
//   y = (O1 2^(m1 - M) + O2 2^(m2 - M)) / (l1 2^(m1 - M) + l2 2^(m2 - M)),
// the same result as one pass over all keys (the softmax's normaliser is a
// sum over keys, so it can be taken over the two ranges apart and combined).
// Which half merges is decided by an atomic arrival count, so a half only ever
// waits (bounded) for a partner that has already arrived and is writing.
//
// Every wait is bounded (common.cuh); on a timeout the CTA records
// GPT2_ERR_DEVICE_TIMEOUT, drains its copies and MMAs, frees TMEM and exits.
#include <math.h>

#include <utility>

#include "common.cuh"
#include "kernels.h"

namespace g2 {

namespace {
constexpr int AT_BQ = 128, AT_BK = 128, AT_D = 64;
constexpr int AT_THREADS = 256;
constexpr int WARP_PRODUCER = 4, WARP_MMA = 5;
// registers per thread after the split: 128 softmax threads + 128 others must
// fit in what the launch gives 256 threads (checked on the host against the
// kernel's register count before any launch)
constexpr int REG_SOFTMAX = 192, REG_OTHER = 48;
constexpr int TILE_BYTES = 128 * 64 * 2;                 // one 128 x 64 bf16 box
// Q slots: 2 would let the next item's Q land early, but then only one CTA
// fits on an SM, which costs more than the exposed Q load
constexpr int Q_SLOTS = 1;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_SLOTS * TILE_BYTES;      // 2 stages
constexpr int OFF_V = OFF_K + 2 * TILE_BYTES;            // 2 stages
constexpr int OFF_P = OFF_V + 2 * TILE_BYTES;            // output staging, 4 x (32 rows x 128 B)
constexpr int OFF_BAR = OFF_P + TILE_BYTES;
constexpr int NUM_BARS = 18;
constexpr int AT_SMEM = OFF_BAR + NUM_BARS * 8 + 16;   // + TMEM holder, abort flag, item slots
constexpr uint32_t TMEM_COLS = 256;   // S: cols [0,128) fp32, O: [128,192) fp32, P: [192,256) bf16 pairs
constexpr uint32_t TM_S = 0, TM_O = 128, TM_P = 192;
constexpr float RESCALE_THRESHOLD = 8.0f;                // log2 units
constexpr int AT_MAX_CLS = 64;
enum : uint32_t { ROLE_WHOLE = 0, ROLE_FIRST = 1, ROLE_SECOND = 2 };
constexpr int PART_M = 128 * 64, PART_L = PART_M + 128;  // partial: O as [16][128 rows][4], then m[128], l[128]
static_assert(PART_L + 128 == ATTN_PART_FLOATS, "partial layout");
}  // namespace

// Work classes, longest first: item = class * (B * H) + (b * H + h).
// n_cls == 0: class c is query tile QT - 1 - c, whole. Otherwise cls[c] packs
// qt | kv0 << 8 | kv1 << 16 | role << 24 | split << 26: the query tile, the
// key tiles [kv0, kv1) it covers, whether it is a whole item or the first or
// second half of a split one, and which split query tile (its scratch pair is
// split * (B * H) + b * H + h).
struct AttnPlan {
  int n_cls;
  uint32_t cls[AT_MAX_CLS];
};

namespace {
struct Item {
  int qt, bh, kv0, kv1, role, pair;
};

template <bool kSplit>
__device__ __forceinline__ Item decode_item(const AttnPlan& plan, int item, int BH, int QT) {
  Item w;
  const int c = item / BH;
  w.bh = item - c * BH;
  if (!kSplit) {
    w.qt = QT - 1 - c;
    w.kv0 = 0;
    w.kv1 = w.qt + 1;
    w.role = ROLE_WHOLE;
    w.pair = 0;
  } else {
    const uint32_t e = plan.cls[c];
    w.qt = (int)(e & 255u);
    w.kv0 = (int)((e >> 8) & 255u);
    w.kv1 = (int)((e >> 16) & 255u);
    w.role = (int)((e >> 24) & 3u);
    w.pair = (int)(e >> 26) * BH + w.bh;
  }
  return w;
}

// Bounded wait for a flag another CTA raises with a release store.
__device__ __forceinline__ bool wait_flag(const int* f, volatile int* abort_flag) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
  if (v != 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(128);
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (v != 0) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > G2_WAIT_LIMIT_NS) return false;
  }
}
}  // namespace

// Persistent: gridDim.x CTAs (two per SM) take work items - one (sequence,
// head, 128-query tile) each - CTA k item k first, then from a device counter,
// most expensive first
// (query tile qt costs qt + 1 key tiles). Work is never handed to the
// hardware block scheduler, which would only start the short tail items once
// whole SMs drain. sched[0] counts the items handed out past the grid, sched[1] counts finished CTAs;
// the last CTA to finish sets both back to 0 for the next launch.
// kSplit: the plan splits some query tiles (the merge code is compiled in).
template <bool kSplit>
__global__ void __launch_bounds__(AT_THREADS, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_y, int B,
                       int T, int H, int C, float scale_log2, const __grid_constant__ AttnPlan plan,
                       unsigned* sched, int* flags, float* part, int n_flags, int* status, float* lse_out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;      // [2]
  uint64_t* q_empty = bars + 2;     // [2]
  uint64_t* kv_full = bars + 4;     // [2]
  uint64_t* kv_empty = bars + 6;    // [2]
  uint64_t* s_full = bars + 8;
  uint64_t* s_free = bars + 9;      // 4 softmax warps
  uint64_t* p_full = bars + 10;     // 4 softmax warps
  uint64_t* pv_done = bars + 11;
  uint64_t* drain = bars + 12;
  uint64_t* item_full = bars + 13;  // [2]
  uint64_t* item_empty = bars + 15; // [2]: the MMA warp and the 4 softmax warps
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* item_slot = reinterpret_cast<volatile int*>(tmem_holder + 2);   // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int QT = (T + AT_BQ - 1) / AT_BQ;
  const int BH = B * H;
  const int total = BH * (plan.n_cls ? plan.n_cls : QT);

  if ((smem_u32(smem) & 1023u) != 0) {   // the swizzled TMA boxes need 1 KB alignment
    if (threadIdx.x == 0) record_error(status, DEV_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int k = 0; k < NUM_BARS; ++k) {
      uint32_t count = 1;
      if (k == 9 || k == 10) count = 4;
      if (k == 15 || k == 16) count = 5;
      mbar_init(&bars[k], count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_PRODUCER && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_y);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_wait();   // qkv (and the schedule counter's reset) come from earlier kernels
  if (threadIdx.x == 0) pdl_trigger();   // the next kernel may start its set-up as SMs free up

  // warpgroup 1 (warps 4-7) gives registers up, warpgroup 0 (softmax) takes them
  if (warp >= 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_OTHER));
  if (warp == WARP_PRODUCER) {
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
        // the first item of every CTA is its own index (the grid never exceeds
        // the item count); later ones come from the counter, past the grid
        const unsigned rank = it == 0 ? blockIdx.x : gridDim.x + atomicAdd(&sched[0], 1u);
        const int item = rank < (unsigned)total ? (int)rank : -1;
        item_slot[slot] = item;
        mbar_arrive(&item_full[slot]);
        if (item < 0) break;
        const Item w = decode_item<kSplit>(plan, item, BH, QT);
        const int b = w.bh / H, h = w.bh % H;
        const int qs = it % Q_SLOTS;   // the item Q_SLOTS back has finished its S products with this slot
        if (!mbar_wait(&q_empty[qs], ((it / Q_SLOTS) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[qs], TILE_BYTES);
        tma_load_3d(smem + OFF_Q + qs * TILE_BYTES, &tm_qkv, &q_full[qs], h * AT_D, w.qt * AT_BQ, b);
        q_issued |= 1u << qs;
        q_parity = (q_parity & ~(1u << qs)) | (((uint32_t)(it / Q_SLOTS) & 1u) << qs);
        for (int j = w.kv0; j < w.kv1; ++j, ++g) {
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
      for (int qs = 0; qs < Q_SLOTS; ++qs)
        if (q_issued & (1u << qs)) mbar_wait(&q_full[qs], (q_parity >> qs) & 1u, &no_abort);
      for (int st = 0; st < 2; ++st)
        if (issued & (1u << st)) mbar_wait(&kv_full[st], (issued_parity >> st) & 1u, &no_abort);
    }
  } else if (warp == WARP_MMA) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(AT_BQ, AT_BK);
      constexpr uint32_t IDESC_O = idesc_bf16_f32_bmn(AT_BQ, AT_D);
      const uint32_t tS = tmem_base + TM_S, tO = tmem_base + TM_O, tP = tmem_base + TM_P;
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
        const Item w = decode_item<kSplit>(plan, item, BH, QT);
        const int n_kv = w.kv1 - w.kv0;
        // S of the item's first tile: its K has landed and the softmax warps
        // have read the previous S
        const int qs = it % Q_SLOTS;
        const uint64_t qdesc = sdesc_kmajor_sw128(smem_u32(smem + OFF_Q + qs * TILE_BYTES));
        if (!mbar_wait(&q_full[qs], (it / Q_SLOTS) & 1, abort_flag) || !mbar_wait(&kv_full[g & 1], (g >> 1) & 1, abort_flag) ||
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
        if (n_kv == 1) mma_commit(&q_empty[qs]);
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
            if (j + 2 == n_kv) mma_commit(&q_empty[qs]);   // the item's last S has been issued
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
  }
  } else {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_SOFTMAX));
  {
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
      const Item w = decode_item<kSplit>(plan, item, BH, QT);
      const int b = w.bh / H, h = w.bh % H;
      const int q0 = w.qt * AT_BQ;
      const int i = q0 + r;                      // query position in the sequence
      const int n_kv = w.kv1 - w.kv0;
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < n_kv; ++jj) {
        const uint32_t gj = g + jj;
        const int j = w.kv0 + jj;                // key tile
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
        const bool diag = (j == w.qt);
        if (diag) {   // diagonal tile: keys after the query (or past T) get -inf
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (key0 + c * 32 + e > i || key0 + c * 32 + e >= T) sr[c][e] = __float_as_uint(-INFINITY);
        }
        float pm[8];   // 8 independent partial maxima, two new values per three-input max
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pm[e & 7] = fmax3(pm[e & 7], __uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1]));
        const float tmax = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        const float m_new = fmaxf(m, tmax * scale_log2);   // scale_log2 > 0
        const bool raise = m_new > m + RESCALE_THRESHOLD;
        float alpha = 1.f;
        if (raise) {
          alpha = ex2_approx(m - m_new);   // 0 on the first tile (m = -inf)
          m = m_new;
        }
        l *= alpha;
        // x = s log2(e)/sqrt(D) - m, p = 2^x: pairs of columns in packed fp32,
        // exponentials on the SFU
        const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m, -m);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (diag && c > qd) {   // keys of this chunk all lie after every row of this warp
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[c][e] = 0u;
            continue;
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])), sc2, nm2);
            float x0, x1;
            f2_unpack(x, x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            ls2[e & 3] = f2_add(ls2[e & 3], f2_pack(p0, p1));
            pk[c][e] = pack_bf16x2(p0, p1);
          }
        }
        {
          const uint64_t s2 = f2_add(f2_add(ls2[0], ls2[1]), f2_add(ls2[2], ls2[3]));
          float s0, s1;
          f2_unpack(s2, s0, s1);
          l += s0 + s1;
        }

        if (gj > 0) {   // PV of the previous tile done: the P buffer is free (and O stable)
          if (!mbar_wait(pv_done, (gj - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (jj > 0 && __any_sync(0xffffffffu, raise)) {
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
      bool merge = false;
      if (kSplit && w.role != ROLE_WHOLE) {
        // Of the two halves of a split query tile, the first to get here (per
        // 32-row quarter) leaves its partial rows and raises the quarter's
        // ready flag; the second merges. The second waits only on a partner
        // that has already arrived, so no CTA ever waits on one not running.
        int order = 0;
        if (lane == 0) order = atomicAdd(flags + n_flags / 2 + w.pair * 4 + qd, 1);
        order = __shfl_sync(0xffffffffu, order, 0);
        merge = order != 0;
      }
      if (kSplit && w.role != ROLE_WHOLE && !merge) {
        // unnormalised O row, m and l to the scratch pair; then this quarter's flag
        float* pb = part + (size_t)w.pair * ATTN_PART_FLOATS;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(tO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 8; ++u)
            __stcg(reinterpret_cast<float4*>(pb) + (c * 8 + u) * 128 + r,
                   make_float4(__uint_as_float(o[4 * u]), __uint_as_float(o[4 * u + 1]), __uint_as_float(o[4 * u + 2]),
                               __uint_as_float(o[4 * u + 3])));
        }
        __stcg(pb + PART_M + r, m);
        __stcg(pb + PART_L + r, l);
        __threadfence();
        __syncwarp();
        if (lane == 0) asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flags + w.pair * 4 + qd), "r"(1) : "memory");
        g += n_kv;
        continue;
      }
      float fa = 0.f, fb = 1.f / l;
      float lse2 = m + __log2f(l);   // log2 of the softmax normaliser, in the units of scale_log2 * s
      bool own_first = false;
      const float* pb = part + (size_t)w.pair * ATTN_PART_FLOATS;
      if (kSplit && merge) {   // merge with the other half's partial rows
        bool got = true;
        if (lane == 0) got = wait_flag(flags + w.pair * 4 + qd, abort_flag);
        got = __shfl_sync(0xffffffffu, got, 0);
        __syncwarp();
        if (!got) {
          ok = false;
          break;
        }
        // the same arithmetic whichever half merges: (1) is always the key
        // range [0, a), (2) the range holding the diagonal
        const float mo = __ldcg(pb + PART_M + r), lo = __ldcg(pb + PART_L + r);
        own_first = w.role == ROLE_FIRST;
        const float m1 = own_first ? m : mo, l1 = own_first ? l : lo;
        const float m2 = own_first ? mo : m, l2 = own_first ? lo : l;
        const float mx = fmaxf(m1, m2);
        const float a1 = ex2_approx(m1 - mx), a2 = ex2_approx(m2 - mx);
        const float inv = 1.f / (l1 * a1 + l2 * a2);
        fa = a1 * inv;   // factor of range (1)
        fb = a2 * inv;   // factor of range (2)
        lse2 = mx + __log2f(l1 * a1 + l2 * a2);
      }
      if (lse_out != nullptr && i < T) lse_out[((size_t)b * H + h) * T + i] = lse2;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tO + c * 32, o);
        tmem_ld_wait();
        float v[32];
        if (kSplit && merge) {   // y = O1 fa + O2 fb, rounded the same way whichever half holds O1
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float4 q = __ldcg(reinterpret_cast<const float4*>(pb) + (c * 8 + u) * 128 + r);
            const float qo[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float own = __uint_as_float(o[4 * u + k]);
              const float o1 = own_first ? own : qo[k], o2 = own_first ? qo[k] : own;
              v[4 * u + k] = fmaf(o1, fa, o2 * fb);
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * fb;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[c * 16 + e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
      }
      // stage 32 rows x 128 B (128-byte swizzle) in this warp's 4 KB, then a 3-D TMA store (rows past T clipped);
      // the previous item's store has finished reading the staging before it is overwritten
      uint8_t* stg = smem + OFF_P + qd * 4096;
      const uint32_t sb = smem_u32(stg);
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_shared_v4(sb + lane * 128 + ((u ^ (lane & 7)) << 4), pk[4 * u], pk[4 * u + 1], pk[4 * u + 2],
                     pk[4 * u + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && q0 + qd * 32 < T) {
        tma_store_3d(&tm_y, stg, h * AT_D, q0 + qd * 32, b);
        bulk_commit();
      }
      __syncwarp();
      g += n_kv;
    }
    if (!ok && lane == 0) {
      record_error(status, DEV_TIMEOUT);
      *abort_flag = 1;
    }
    if (lane == 0) bulk_wait_all();   // the last output store has landed
  }

  }
  __syncthreads();
  // the last CTA to finish (every second half has merged by then) clears the
  // split flags and resets the schedule for the next launch
  if (kSplit) {
    volatile int* last = item_slot;   // free now
    if (threadIdx.x == 0) {
      __threadfence();
      *last = atomicAdd(&sched[1], 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (*last) {
      __threadfence();
      for (int k = threadIdx.x; k < n_flags; k += blockDim.x) flags[k] = 0;
      __syncthreads();
      if (threadIdx.x == 0) {
        atomicExch(&sched[0], 0u);
        atomicExch(&sched[1], 0u);
      }
      __threadfence();
    }
  } else if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&sched[0], 0u);
      atomicExch(&sched[1], 0u);
      __threadfence();
    }
  }
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

namespace {
// scratch of gpt2_op_attention's launches (zero at load): counters, split flags, partials
constexpr int OWN_PAIRS = 248;   // about 8 MB of partials
__device__ unsigned g_attn_sched[2];
__device__ int g_attn_flags[OWN_PAIRS * ATTN_PAIR_FLAGS];
__device__ __align__(256) float g_attn_part[OWN_PAIRS * ATTN_PART_FLOATS];

// Split the query tiles whose key count exceeds twice the average work of a
// CTA slot, longest first, while the scratch holds them; order the classes by
// cost, the first half of a split tile before its second half.
AttnPlan make_plan(int BH, int QT, int slots, int cap_pairs, int* n_split) {
  AttnPlan p;
  p.n_cls = 0;
  *n_split = 0;
  if (QT > AT_MAX_CLS / 2 || slots < 1) return p;
  const long tiles = (long)BH * QT * (QT + 1) / 2;
  // more than twice a slot's average share: splitting costs a second Q load
  // and the merge, and only pays where a few long items set the kernel's length
  long target = 2 * ((tiles + slots - 1) / slots);
  if (target < 2) target = 2;
  int split_of[AT_MAX_CLS / 2];
  int S = 0;
  for (int qt = QT - 1; qt >= 0; --qt) {
    split_of[qt] = -1;
    if (qt + 1 > target && (long)(S + 1) * BH <= cap_pairs) split_of[qt] = S++;
  }
  if (S == 0) return p;
  struct Cls {
    int cost, second;
    uint32_t v;
  } e[AT_MAX_CLS];
  int n = 0;
  auto pack = [](int qt, int kv0, int kv1, uint32_t role, int split) {
    return (uint32_t)qt | (uint32_t)kv0 << 8 | (uint32_t)kv1 << 16 | role << 24 | (uint32_t)split << 26;
  };
  for (int qt = QT - 1; qt >= 0; --qt) {
    const int nk = qt + 1;
    if (split_of[qt] >= 0) {
      const int a = (nk + 1) / 2;
      e[n++] = {a, 0, pack(qt, 0, a, ROLE_FIRST, split_of[qt])};
      e[n++] = {nk - a, 1, pack(qt, a, nk, ROLE_SECOND, split_of[qt])};
    } else {
      e[n++] = {nk, 0, pack(qt, 0, nk, ROLE_WHOLE, 0)};
    }
  }
  for (int x = 1; x < n; ++x)   // stable insertion sort: cost descending, first halves and whole items first
    for (int y = x; y > 0; --y) {
      const Cls &u = e[y - 1], &t = e[y];
      if (t.cost > u.cost || (t.cost == u.cost && t.second < u.second)) std::swap(e[y - 1], e[y]);
      else break;
    }
  p.n_cls = n;
  for (int k = 0; k < n; ++k) p.cls[k] = e[k].v;
  *n_split = S;
  return p;
}
}  // namespace

size_t attention_scratch_bytes(int B, int T, int H) {
  const size_t QT = ((size_t)T + AT_BQ - 1) / AT_BQ;
  return QT * (size_t)B * H * (ATTN_PART_FLOATS * 4 + ATTN_PAIR_FLAGS * 4);
}

cudaError_t attention_tc_launch(const void* qkv, void* y, int B, int T, int H, int C, const AttnScratch* scratch,
                                int* status, cudaStream_t s, float* lse_out) {
  if (B <= 0 || T <= 0) return cudaSuccess;
  if (C / H != AT_D) return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  static int slots[64] = {};   // CTAs the device runs at once (two per SM)
  static AttnScratch own[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const auto kfalse = attn_fwd_tc_kernel<false>;
  const auto ktrue = attn_fwd_tc_kernel<true>;
  if (!attr_set[dev]) {
    cudaError_t e = cudaSuccess;
    for (auto k : {kfalse, ktrue}) {
      if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
      // two CTAs share an SM only with the largest shared-memory carveout
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    }
    int sms = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) slots[dev] = 2 * sms;   // __launch_bounds__(AT_THREADS, 2)
    if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&own[dev].sched), g_attn_sched);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&own[dev].flags), g_attn_flags);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&own[dev].part), g_attn_part);
    // the register split must fit in what the launch allocates, or the
    // softmax warps' setmaxnreg.inc would never be granted
    cudaFuncAttributes fa[2];
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa[0], kfalse);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa[1], ktrue);
    if (e != cudaSuccess) return e;
    for (const cudaFuncAttributes& f : fa)
      if (f.numRegs * AT_THREADS < 128 * (REG_SOFTMAX + REG_OTHER)) return cudaErrorInvalidConfiguration;
    own[dev].cap_pairs = OWN_PAIRS;
    attr_set[dev] = true;
  }
  const AttnScratch& sc = (scratch && scratch->sched) ? *scratch : own[dev];
  if (sc.sched == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tq, ty;
  // qkv as [B][T][3C], boxes of 64 columns x 128 rows; y as [B][T][C], boxes of 64 x 32.
  if (!make_tmap_3d_bf16(&tq, qkv, 3 * (uint64_t)C, T, B, 3 * (uint64_t)C, (uint64_t)T * 3 * C, 64, 128) ||
      !make_tmap_3d_bf16(&ty, y, C, T, B, C, (uint64_t)T * C, 64, 32))
    return cudaErrorInvalidValue;
  const int QT = (T + AT_BQ - 1) / AT_BQ;
  const int BH = B * H;
  int n_split = 0;
  const AttnPlan plan =
      make_plan(BH, QT, slots[dev], (sc.flags && sc.part && lse_out == nullptr) ? sc.cap_pairs : 0, &n_split);
  const int items = BH * (plan.n_cls ? plan.n_cls : QT);
  const int grid = items < slots[dev] ? items : slots[dev];
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)AT_D));
  if (n_split)
    return launch_pdl(ktrue, dim3(grid), dim3(AT_THREADS), AT_SMEM, s, tq, ty, B, T, H, C, scale_log2,
                      plan, sc.sched, sc.flags, sc.part, n_split * BH * ATTN_PAIR_FLAGS, status, lse_out);
  return launch_pdl(kfalse, dim3(grid), dim3(AT_THREADS), AT_SMEM, s, tq, ty, B, T, H, C, scale_log2,
                    plan, sc.sched, sc.flags, sc.part, 0, status, lse_out);
}

}  // namespace g2
