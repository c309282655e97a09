// gemm_tc.cu - tcgen05 / TMEM / TMA GEMM with fused epilogues (sm_100a).
//
// Computes C = A . B^T for the four Linear layers of a GPT-2 block and the
// tied lm_head ("Hand-writing GPT-2 from scratch: the Transformer decoder
// core modules in PyTorch", sections 2.2 and 3.4; "Reproducing GPT-2 124M",
// section 2.1: c_attn, c_proj, c_fc, c_proj and lm_head = wte^T), in bf16
// with fp32 accumulation, A [M, K] and B [N, K] both K-major (the
// nn.Linear [out, in] layout is already the K-major B operand).
//
// Design (one persistent CTA per SM, 2 + BN/16 warps):
//   warp 0      TMA producer: 128x64 A box and BNx64 B box per stage, 128-byte
//               swizzle, 4-deep ring of shared-memory stages.
//   warp 1      allocates 2*BN TMEM columns and issues tcgen05.mma
//               (M=128, N=BN, K=16, four per 64-wide k-block) into one of two
//               TMEM accumulators; tcgen05.commit frees smem stages and hands
//               finished accumulators to the epilogue.
//   warps 2..   epilogue, one warp per TMEM lane quadrant (32 rows) and
//               64-column group (BN/16 warps), 32 columns per tcgen05.ld:
//                 EPI_BIAS / EPI_GELU  +bias (+GELU erf), bf16, staged in
//                                      64B-swizzled smem, TMA store;
//                 EPI_RESID            +bias, fp32, staged in 128B-swizzled
//                                      smem, TMA reduce-add into the fp32
//                                      residual stream (x += y without the SM
//                                      ever reading x);
//                 EPI_LMHEAD           online max / sum-exp per row over the
//                                      valid columns, the target logit, and
//                                      optionally the fp32 logits through an
//                                      smem transposition (coalesced rows).
// The double-buffered accumulator lets the epilogue of tile i overlap the
// main loop of tile i+1. Tiles are walked M-fastest so that concurrently
// running CTAs share B tiles in L2 (the 77 MB wte is streamed ~once).
//
// The lm_head epilogue never needs the logits in HBM: per row and 64-column group
// it emits (max, sum exp(z - max)) and, where the target column lies, the
// target logit; ce.cu finishes the log-sum-exp. Columns at or past N (the
// vocabulary padded up to the tile width by TMA zero fill) are excluded from
// the sums and from the logits.
//
// Every wait is bounded (common.cuh): on a timeout the kernel records
// GPT2_ERR_DEVICE_TIMEOUT, lets its in-flight copies and MMAs land, frees its
// TMEM and returns.
#include <cudaTypedefs.h>
#include <stdlib.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace g2 {

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
constexpr int TC_STAGES = 4;
constexpr int TC_SMEM_MAX = 232448;   // dynamic shared memory per block (227 KB)
template <int BN, int EPI, int CG = 1>
struct TcLayout {
  // Each epilogue warp owns 32 rows (one TMEM lane quadrant) x COLS_PER_WARP
  // columns: 64 (BN / 16 warps), or half the tile (8 warps; BN = 128, 256) for the lm_head
  // without logits, whose epilogue has slack and whose warps would only
  // compete with the MMA issuer.
  static constexpr int COLS_PER_WARP = (EPI == EPI_LMHEAD && BN % 128 == 0) ? BN / 2 : 64;
  static constexpr int EPI_WARPS = 4 * (BN / COLS_PER_WARP);
  static constexpr int THREADS = 32 * (2 + EPI_WARPS);
  // per epilogue warp: one 32 x 32 chunk (bf16: 2 KB, fp32 residual: 4 KB),
  // or 8 logits rows x 64 fp32 (2 KB)
  static constexpr bool F32_OUT = EPI == EPI_RESID || EPI == EPI_F32;
  static constexpr int STAGE_BUF_BYTES = F32_OUT ? 4096 : 2048;
  static constexpr int EPI_BYTES = EPI_WARPS * STAGE_BUF_BYTES;
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  // CTA pair (CG = 2): each CTA stages half of the tile's BN rows of B
  static constexpr int B_ROWS = BN / CG;
  static constexpr int B_BYTES = B_ROWS * TC_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // a single CTA keeps a 4-deep ring (3-deep for fp32 output at BN = 256,
  // whose 4 KB staging per warp takes the fourth stage's room); a pair's
  // smaller stages buy up to 6
  static constexpr int STAGES_FIT = (TC_SMEM_MAX - 1024 - 256 - EPI_BYTES) / STAGE_BYTES;
  static constexpr int STAGES =
      CG == 1 ? (F32_OUT && BN == 256 ? 3 : TC_STAGES) : (STAGES_FIT < 6 ? STAGES_FIT : 6);
  static constexpr int EPI_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFFSET = EPI_OFFSET + EPI_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 5;   // full, empty, tmem_full[2], tmem_empty[2], drain
  static constexpr int SMEM_BYTES = BAR_OFFSET + NUM_BARS * 8 + 16 + 1024;   // + holders, 1 KB alignment slack
  static constexpr uint32_t TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
  static constexpr int CHUNKS = COLS_PER_WARP / 32;
  static constexpr int GROUPS = BN / 64;   // lm_head: 64-column log-sum-exp groups per tile
  static_assert(SMEM_BYTES <= TC_SMEM_MAX, "shared memory budget");
  static_assert(STAGES >= 2 && STAGE_BYTES % 1024 == 0, "ring of 1 KB-aligned stages");
  static_assert(BN % COLS_PER_WARP == 0 && COLS_PER_WARP % 64 == 0, "whole 64-column groups per warp");
};

// The 32 bias values of one 32-column chunk as bf16 pairs (lo = even
// column), zero past N or without a bias.
__device__ __forceinline__ void load_bias32_raw(const bf16* bias, int col0, int N, uint32_t (&b)[16]) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int col = col0 + g * 8;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (bias != nullptr && col < N) w = __ldg(reinterpret_cast<const uint4*>(bias + col));
    b[4 * g] = w.x;
    b[4 * g + 1] = w.y;
    b[4 * g + 2] = w.z;
    b[4 * g + 3] = w.w;
  }
}

// Derivative of the GELU at the pre-activation u, on a pair in packed fp32.
// Exact form: d/du [u Phi(u)] = Phi(u) + u phi(u), with Phi from the same
// Abramowitz-Stegun 7.1.28 erf as the forward (r ~= erfc(|u|/sqrt2): Phi is
// 1 - r/2 for u >= 0, r/2 below) and phi(u) = 2^(-u^2 log2(e) / 2) / sqrt(2 pi)
// on the SFU. Tanh form: d/du [u (1 + t) / 2], t = tanh(v), v = k (u + c u^3):
// (1 + t) / 2 + u (1 - t^2) k (1 + 3 c u^2) / 2, with (1 + t) / 2 = 1 / (1 +
// e^(-2v)) from the SFU exponential and reciprocal.
__device__ __forceinline__ uint64_t gelu_grad_x2(uint64_t u, int tanh_form) {
  float u0, u1;
  f2_unpack(u, u0, u1);
  if (tanh_form) {
    const float k = 0.7978845608028654f, c = 0.044715f;
    const uint64_t sq = f2_mul(u, u);
    const uint64_t v = f2_mul(f2_fma(f2_mul(sq, f2_pack(c, c)), u, u), f2_pack(k, k));
    float v0, v1;
    f2_unpack(v, v0, v1);
    // s = (1 + t) / 2 = 1 / (1 + 2^(-2 v log2 e)); 1 - t^2 = 4 s (1 - s)
    const float s0 = rcp_approx(1.f + ex2_approx(-2.8853900817779268f * v0));
    const float s1 = rcp_approx(1.f + ex2_approx(-2.8853900817779268f * v1));
    const uint64_t s2 = f2_pack(s0, s1);
    const uint64_t one_m_t2 = f2_mul(f2_mul(s2, f2_sub(f2_pack(1.f, 1.f), s2)), f2_pack(4.f, 4.f));
    // u k (1 + 3 c u^2) / 2
    const uint64_t w = f2_mul(f2_mul(u, f2_pack(0.5f * k, 0.5f * k)), f2_fma(sq, f2_pack(3.f * c, 3.f * c), f2_pack(1.f, 1.f)));
    return f2_fma(w, one_m_t2, s2);
  }
  const uint64_t z = f2_mul(f2_pack(fabsf(u0), fabsf(u1)), f2_pack(0.70710678118654752f, 0.70710678118654752f));
  uint64_t p = f2_fma(z, f2_pack(4.30638e-5f, 4.30638e-5f), f2_pack(2.765672e-4f, 2.765672e-4f));
  p = f2_fma(z, p, f2_pack(1.520143e-4f, 1.520143e-4f));
  p = f2_fma(z, p, f2_pack(9.2705272e-3f, 9.2705272e-3f));
  p = f2_fma(z, p, f2_pack(4.22820123e-2f, 4.22820123e-2f));
  p = f2_fma(z, p, f2_pack(7.05230784e-2f, 7.05230784e-2f));
  p = f2_fma(z, p, f2_pack(1.0f, 1.0f));
  p = f2_mul(p, p);
  p = f2_mul(p, p);
  p = f2_mul(p, p);
  p = f2_mul(p, p);   // ^16
  float p0, p1;
  f2_unpack(p, p0, p1);
  const float hr0 = 0.5f * rcp_approx(p0), hr1 = 0.5f * rcp_approx(p1);   // erfc(|u|/sqrt2) / 2
  const float Phi0 = u0 >= 0.f ? 1.f - hr0 : hr0, Phi1 = u1 >= 0.f ? 1.f - hr1 : hr1;
  // u phi(u) = u 2^(-u^2 log2(e) / 2) / sqrt(2 pi)
  const uint64_t e2 = f2_mul(f2_mul(u, u), f2_pack(-0.72134752044448170f, -0.72134752044448170f));
  float e0, e1;
  f2_unpack(e2, e0, e1);
  const uint64_t uphi = f2_mul(f2_mul(u, f2_pack(0.3989422804014327f, 0.3989422804014327f)),
                               f2_pack(ex2_approx(e0), ex2_approx(e1)));
  return f2_add(uphi, f2_pack(Phi0, Phi1));
}

// CG = 2: a CTA pair (cluster of two) computes 256 x BN tiles with one
// tcgen05.mma of M = 256 issued by the leader (cluster rank 0). Each CTA
// stages its 128 rows of A and half (BN / 2 rows) of B, so per SM the TMA
// writes and the tensor core's shared-memory reads per FLOP drop by a
// third at BN = 256; each CTA's epilogue drains its own 128 accumulator rows.
template <int BN, int EPI, int LAYOUT, int CG>
__global__ void __launch_bounds__(TcLayout<BN, EPI, CG>::THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                   const GemmArgs args) {
  using L = TcLayout<BN, EPI, CG>;
  constexpr bool kLM = EPI == EPI_LMHEAD || EPI == EPI_LMHEAD_LOGITS;
  constexpr bool kAmn = (LAYOUT & LAYOUT_A_MN) != 0, kBmn = (LAYOUT & LAYOUT_B_MN) != 0;
  constexpr bool kGelu = EPI == EPI_GELU || EPI == EPI_GELU_SAVE;
  constexpr bool kPair = CG == 2;
  static_assert(!kPair || (!kAmn && !kBmn), "CTA pairs read K-major operands");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFFSET);
  uint64_t* empty = full + L::STAGES;
  uint64_t* tfull = empty + L::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = args.M, N = args.N;
  // rank in the pair (the leader issues the MMAs) and the work walker: one
  // per CTA, or one per pair
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int walker = kPair ? (int)cluster_id_x() : (int)blockIdx.x;
  const int n_walkers = kPair ? (int)cluster_count_x() : (int)gridDim.x;
  const int m_tiles = (M + TC_BM * CG - 1) / (TC_BM * CG);
  const int n_tiles = (N + BN - 1) / BN;
  // EPI_F32 with k_split = 2: each output tile is two work items, the K range
  // halved, both reduce-added into a zeroed output (0 + a + b: the same bits
  // in either order)
  const int ks = (EPI == EPI_F32 && args.k_split == 2) ? 2 : 1;
  const int mn_tiles = m_tiles * n_tiles;
  const int num_tiles = mn_tiles * ks;
  const int nk_all = (args.K + TC_BK - 1) / TC_BK;   // a K tail past args.K reads as zero (TMA fill)
  const int nk = (nk_all + ks - 1) / ks;             // k-blocks per work item (the last may have fewer)

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], L::EPI_WARPS * CG);   // a pair: both CTAs' epilogue warps free the leader's MMA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (!kLM) tma_prefetch_desc(&tmC);
    if (EPI == EPI_GELU_SAVE) tma_prefetch_desc(&tmD);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(tmem_holder, L::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, L::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();   // the peer's barriers are initialised before any load or arrive targets them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // The operands and the residual stream come from the previous kernel:
  // every thread that touches them waits for it (the producer after it has
  // requested the first stages of a B operand that no kernel writes, the
  // weights of the forward pass).
  if (warp != 0) pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;   // per stage: a load was issued / its barrier phase parity
      bool ok = true;
      // a pair counts both CTAs' bytes on the leader's full barrier
      const uint32_t full_leader = kPair ? mapa_shared(smem_u32(full), 0) : 0u;
      auto load_2d = [&](void* dst, const CUtensorMap* tm, int s, int c0, int c1) {
        if (kPair)
          tma_load_2d_pair(dst, tm, full_leader + 8u * s, c0, c1);
        else
          tma_load_2d(dst, tm, &full[s], c0, c1);
      };
      auto expect = [&](int s) {
        if (leader) mbar_arrive_expect_tx(&full[s], CG * L::STAGE_BYTES);
      };
      auto load_b = [&](uint8_t* sa, int s, int n0, int kb) {
        if (kBmn) {
#pragma unroll
          for (int b = 0; b < BN / 64; ++b) load_2d(sa + L::A_BYTES + b * 8192, &tmB, s, n0 + b * 64, kb * TC_BK);
        } else {
          load_2d(sa + L::A_BYTES, &tmB, s, kb * TC_BK, n0);
        }
      };
      // B of the first tile's first stages ahead of the wait (fresh stages need no empty wait)
      const int npre = (args.b_const && ks == 1 && walker < num_tiles) ? min(nk, L::STAGES) : 0;
      for (int kb = 0; kb < npre; ++kb) {
        expect(kb);
        load_b(smem + kb * L::STAGE_BYTES, kb, (walker / m_tiles) * BN + (int)rank * L::B_ROWS, kb);
      }
      pdl_wait();
      pdl_trigger();   // the next kernel may start its set-up as SMs free up
      bool first = true;
      for (int tile = walker; tile < num_tiles && ok; tile += n_walkers, first = false) {
        const int mn = tile % mn_tiles, kq = tile / mn_tiles;
        const int m0 = ((mn % m_tiles) * CG + (int)rank) * TC_BM;
        const int n0 = (mn / m_tiles) * BN + (int)rank * L::B_ROWS;
        const int kb0 = kq * nk, kb1 = min(nk_all, kb0 + nk);
        for (int kb = kb0; kb < kb1; ++kb) {
          const bool pre = first && kb - kb0 < npre;   // stage already holds B and expects its bytes
          if (!pre && !mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * L::STAGE_BYTES;
          if (!pre) expect(stage);
          // K-major: one box of rows x 64 K; MN-major: 64-wide MN boxes of 64 K rows, 8 KB apart
          if (kAmn) {
#pragma unroll
            for (int b = 0; b < TC_BM / 64; ++b) load_2d(sa + b * 8192, &tmA, stage, m0 + b * 64, kb * TC_BK);
          } else {
            load_2d(sa, &tmA, stage, kb * TC_BK, m0);
          }
          if (!pre) load_b(sa, stage, n0, kb);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        record_error(args.status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
      // Let every issued copy land before the CTA can exit (bounded). A
      // pair's copies all complete on the leader's barriers: the leader
      // waits for both CTAs', and the closing cluster barrier keeps the
      // peer resident until then.
      volatile int no_abort = 0;
      if (leader)
        for (int s = 0; s < L::STAGES; ++s)
          if (issued & (1u << s)) mbar_wait(&full[s], (issued_parity >> s) & 1u, &no_abort);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && leader) {
      constexpr uint32_t IDESC = idesc_bf16_f32_major(TC_BM * CG, BN, kAmn, kBmn);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = walker; tile < num_tiles && ok; tile += n_walkers, ++it) {
        const int kq = tile / mn_tiles;
        const int n_kb = min(nk_all, kq * nk + nk) - kq * nk;
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * L::STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            // K step of 16: +32 B inside a K-major 128-byte row, +16 rows (2048 B) of an MN-major box
            const uint64_t adesc = kAmn ? sdesc_mn_sw128(sa + k * 2048, 8192) : sdesc_kmajor_sw128(sa) + 2 * k;
            const uint64_t bdesc =
                kBmn ? sdesc_mn_sw128(sa + L::A_BYTES + k * 2048, 8192) : sdesc_kmajor_sw128(sa + L::A_BYTES) + 2 * k;
            if (kPair)
              mma_bf16_ss_pair(d_tmem, adesc, bdesc, IDESC, (kb | k) != 0);
            else
              mma_bf16_ss(d_tmem, adesc, bdesc, IDESC, (kb | k) != 0);
          }
          if (kPair)
            mma_commit_pair_both(&empty[stage]);   // frees the stage in both CTAs
          else
            mma_commit(&empty[stage]);
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (kPair)
          mma_commit_pair_both(&tfull[acc]);
        else
          mma_commit(&tfull[acc]);
      }
      if (!ok) {
        record_error(args.status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
      // Every MMA issued above has completed once `drain` flips.
      if (kPair)
        mma_commit_pair(drain);
      else
        mma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quadrant = rows q*32 .. q*32+31
    const int cg = (warp - 2) >> 2;          // which 64-column group of the tile
    uint8_t* sbuf = smem + L::EPI_OFFSET + (warp - 2) * L::STAGE_BUF_BYTES;
    const uint32_t sb = smem_u32(sbuf);
    constexpr float LOG2E = 1.4426950408889634f;
    bool store_pending = false;
    // the accumulator buffers are handed back to the (leader's) MMA warp
    const uint32_t tempty_leader = kPair ? mapa_shared(smem_u32(tempty), 0) : 0u;
    auto release_acc = [&](int acc) {
      if (kPair)
        mbar_arrive_cluster(tempty_leader + 8u * acc);
      else
        mbar_arrive(&tempty[acc]);
    };
    int it = 0;
    for (int tile = walker; tile < num_tiles; tile += n_walkers, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int mn = tile % mn_tiles;
      const int m_blk = mn % m_tiles, n_blk = mn / m_tiles;
      const int m0 = (m_blk * CG + (int)rank) * TC_BM, n0 = n_blk * BN;
      const int row0 = m0 + q * 32;          // first row of this warp
      const int row = row0 + lane;
      const bool row_ok = row < M;
      const int cbase = n0 + cg * L::COLS_PER_WARP;
      const int nvalid = min(L::COLS_PER_WARP, N - cbase);   // may be <= 0 (warp-uniform)
      int tgt = -1;
      if (kLM) tgt = (row_ok && args.targets != nullptr) ? args.targets[row] : -1;

      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
        if (lane == 0) {
          record_error(args.status, DEV_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + cg * L::COLS_PER_WARP;
      // lm_head: pull this warp's whole slice of the accumulator into registers
      // with a single wait and give the TMEM buffer back before any arithmetic.
      uint32_t r[kLM ? L::CHUNKS : 1][32];
      if (kLM) {
#pragma unroll
        for (int c = 0; c < L::CHUNKS; ++c)
          if (c * 32 < nvalid) tmem_ld_32x32b_x32(t_row + c * 32, r[c]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(acc);
      }

      if (kLM) {
        // log-sum-exp partials of this row, one per 64-column group (the
        // same arithmetic whichever warp layout runs, so the losses do not
        // depend on whether logits are written): 8 independent partial
        // maxima / sums keep the dependency chains short; columns at or past
        // N count as -inf (exp2 gives 0)
#pragma unroll
        for (int c = 0; c < L::CHUNKS; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j >= nvalid) r[c][j] = __float_as_uint(-INFINITY);
#pragma unroll
        for (int gi = 0; gi < L::CHUNKS / 2; ++gi) {
          float pm[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) pm[j] = -INFINITY;
#pragma unroll
          for (int c = 2 * gi; c < 2 * gi + 2; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j) pm[j & 7] = fmaxf(pm[j & 7], __uint_as_float(r[c][j]));
          const float mx =
              fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
          const float nm2 = mx * LOG2E;
          float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 2 * gi; c < 2 * gi + 2; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j) ps[j & 7] += ex2_approx(fmaf(__uint_as_float(r[c][j]), LOG2E, -nm2));
          const float s0 = ps[0] + ps[1], s1 = ps[2] + ps[3], s2 = ps[4] + ps[5], s3 = ps[6] + ps[7];
          // rows of `part` are the 64-column groups of the vocabulary
          if (row_ok)
            args.part[(size_t)(n_blk * L::GROUPS + cg * (L::CHUNKS / 2) + gi) * M + row] =
                gi * 64 < nvalid ? make_float2(mx, (s0 + s1) + (s2 + s3)) : make_float2(-INFINITY, 0.f);
        }
        const int tj = tgt - cbase;
        float tgt_val = 0.f;
#pragma unroll
        for (int c = 0; c < L::CHUNKS; ++c) {
          const bool mine = tj >= c * 32 && tj < c * 32 + 32;
          if (__any_sync(0xffffffffu, mine)) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (mine && tj == c * 32 + j) tgt_val = __uint_as_float(r[c][j]);
          }
        }
        if (row_ok && tj >= 0 && tj < nvalid) args.tgt_logit[row] = tgt_val;
        if (EPI == EPI_LMHEAD_LOGITS) {
          // fp32 logits. The row pitch V is odd, so rows are only 4-byte
          // aligned and neither vector nor TMA stores apply; short unaligned
          // row pieces leave partial 32-byte sectors that write slowly. So
          // each row's 64 columns leave as one contiguous 256-byte run:
          // 8 rows at a time are transposed through this warp's 2 KB of
          // shared memory (row rr at rr * 256, 16-byte unit u stored at
          // unit u ^ rr, conflict-free both ways) and written by all 32 lanes
          // as two back-to-back 128-byte stores per row.
          float* lg = static_cast<float*>(args.out);
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {
            if ((lane >> 3) == g) {
              const int rr = lane & 7;
#pragma unroll
              for (int u = 0; u < 8 * L::CHUNKS; ++u)
                st_shared_v4(sb + rr * 256 + ((u ^ rr) << 4), r[u >> 3][4 * (u & 7)], r[u >> 3][4 * (u & 7) + 1],
                             r[u >> 3][4 * (u & 7) + 2], r[u >> 3][4 * (u & 7) + 3]);
            }
            __syncwarp();
#pragma unroll 2
            for (int rr = 0; rr < 8; ++rr) {
              const int grow = row0 + g * 8 + rr;
              float* dst = lg + (size_t)grow * args.ldo + cbase;
#pragma unroll
              for (int k = 0; k < L::CHUNKS; ++k) {
                const int e = 32 * k + lane;
                const float val = ld_shared_f32(sb + rr * 256 + (((8 * k + (lane >> 2)) ^ rr) << 4) + ((lane & 3) << 2));
                if (grow < M && e < nvalid) __stcs(dst + e, val);   // streaming: evict first from L2
              }
            }
            __syncwarp();
          }
        }
      } else {
        // bias / GELU / residual / backward epilogues: both 32-column chunks
        // of this warp's slice come out of TMEM with one wait and the
        // accumulator goes straight back to the MMA warp; then per chunk:
        // bias, activation, swizzled staging, TMA store or reduce-add.
        const int nch = (row0 < M && nvalid > 0) ? min(L::CHUNKS, (nvalid + 31) / 32) : 0;   // warp-uniform
        uint32_t v[L::CHUNKS][32];
#pragma unroll
        for (int c = 0; c < L::CHUNKS; ++c)
          if (c < nch) tmem_ld_32x32b_x32(t_row + c * 32, v[c]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(acc);
        const bf16* bias_p = static_cast<const bf16*>(args.bias);
        // EPI_DLOGITS: this row's target, log-sum-exp (log2 units) and 1 / scored rows
        int d_tgt = -1;
        float d_lse2 = 0.f, d_inv = 0.f;
        if (EPI == EPI_DLOGITS) {
          if (row_ok) {
            d_tgt = args.targets[row];
            d_lse2 = args.row_lse[row] * LOG2E;
          }
          const int ns = *args.n_scored;
          d_inv = ns > 0 ? 1.f / (float)ns : 0.f;
        }
        // stage 32 rows of one chunk in this warp's buffer and send it to `map`
        auto stage_and_send = [&](const uint32_t* pk, const CUtensorMap* map, int col0) {
          if (store_pending) {       // the previous TMA store must have read the staging buffer
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          }
          if (L::F32_OUT) {
            // 32 rows x 128 B, 128-byte swizzle: unit j of row r at unit j ^ (r & 7)
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_v4(sb + lane * 128 + ((j ^ (lane & 7)) << 4), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2],
                           pk[4 * j + 3]);
          } else {
            // 32 rows x 64 B, 64-byte swizzle: unit j of row r at unit j ^ ((r >> 1) & 3)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(sb + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2],
                           pk[4 * j + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (EPI == EPI_RESID || ks == 2)
              tma_reduce_add_2d(map, sbuf, col0, row0);
            else
              tma_store_2d(map, sbuf, col0, row0);
            bulk_commit();
          }
          store_pending = true;
        };
#pragma unroll
        for (int c = 0; c < L::CHUNKS; ++c) {
          if (c >= nch) break;
          const int col0 = cbase + c * 32;
          uint32_t* pk = v[c];   // results overwrite the accumulator values in place
          if (L::F32_OUT) {
            uint32_t bc[16];   // bias as bf16 pairs
            load_bias32_raw(bias_p, col0, N, bc);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              pk[2 * j] = __float_as_uint(__uint_as_float(v[c][2 * j]) + __uint_as_float(bc[j] << 16));
              pk[2 * j + 1] = __float_as_uint(__uint_as_float(v[c][2 * j + 1]) + __uint_as_float(bc[j] & 0xffff0000u));
            }
          } else if (EPI == EPI_DGELU) {
            // dU = dF * gelu'(u) with u the saved pre-activation (bf16 pairs)
            uint32_t ur[16];
            const bf16* up = static_cast<const bf16*>(args.aux) + (size_t)row * args.ld_aux + col0;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint4 w = make_uint4(0, 0, 0, 0);
              if (row_ok && col0 + g * 8 < N) w = __ldg(reinterpret_cast<const uint4*>(up + g * 8));
              ur[4 * g] = w.x;
              ur[4 * g + 1] = w.y;
              ur[4 * g + 2] = w.z;
              ur[4 * g + 3] = w.w;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint64_t u2 = f2_pack(__uint_as_float(ur[j] << 16), __uint_as_float(ur[j] & 0xffff0000u));
              const uint64_t d2 = f2_mul(f2_pack(__uint_as_float(v[c][2 * j]), __uint_as_float(v[c][2 * j + 1])),
                                         gelu_grad_x2(u2, args.gelu_tanh));
              float d0, d1;
              f2_unpack(d2, d0, d1);
              pk[j] = pack_bf16x2(d0, d1);
            }
          } else if (EPI == EPI_DLOGITS) {
            // dz = (softmax(z) - onehot(target)) / n_scored on scored rows and
            // valid columns, 0 elsewhere (padding columns included)
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float d[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int col = col0 + 2 * j + e;
                const float p = ex2_approx(fmaf(__uint_as_float(v[c][2 * j + e]), LOG2E, -d_lse2));
                d[e] = (d_tgt >= 0 && col < N) ? (p - (col == d_tgt ? 1.f : 0.f)) * d_inv : 0.f;
              }
              pk[j] = pack_bf16x2(d[0], d[1]);
            }
          } else {
            uint32_t bc[16];   // bias as bf16 pairs
            load_bias32_raw(bias_p, col0, N, bc);
            uint32_t zp[EPI == EPI_GELU_SAVE ? 16 : 1];   // EPI_GELU_SAVE: the pre-activation as bf16 pairs
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float b0 = __uint_as_float(bc[j] << 16), b1 = __uint_as_float(bc[j] & 0xffff0000u);
              const float x0 = __uint_as_float(v[c][2 * j]), x1 = __uint_as_float(v[c][2 * j + 1]);
              if (kGelu) {
                const uint64_t z2 = f2_add(f2_pack(x0, x1), f2_pack(b0, b1));
                const uint64_t y2 = args.gelu_tanh ? gelu_tanh_x2(z2) : gelu_erf_x2(z2);
                float a, b;
                f2_unpack(y2, a, b);
                pk[j] = pack_bf16x2(a, b);
                if (EPI == EPI_GELU_SAVE) {
                  f2_unpack(z2, a, b);
                  zp[EPI == EPI_GELU_SAVE ? j : 0] = pack_bf16x2(a, b);
                }
              } else {
                pk[j] = pack_bf16x2(x0 + b0, x1 + b1);
              }
            }
            if (EPI == EPI_GELU_SAVE) stage_and_send(zp, &tmD, col0);
          }
          stage_and_send(pk, &tmC, col0);
        }
      }
    }
    if (!kLM && lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncthreads();
  // A pair: the leader's MMAs (which read the peer's shared memory and write
  // its TMEM) have drained, and the peer's arrivals on the leader's
  // barriers have landed, before either CTA frees TMEM or exits.
  if (kPair) cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    if (kPair)
      tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool load_encode() {
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

bool encode_2d(CUtensorMap* tm, CUtensorMapDataType dt, int esize, const void* base, uint64_t rows, uint64_t cols,
               uint64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  if (!load_encode()) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((ld * esize) & 15) || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * (uint64_t)esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


// The fp32 epilogues' 4 KB staging per warp leaves room for a 3-deep ring at
// BN = 256 on a single CTA: instantiated for the weight gradient (both
// operands MN-major, the widest tiles whose K halves fill the SMs; the
// residual epilogue keeps BN <= 192). The backward layouts are instantiated
// only with the epilogues the backward pass uses; CTA pairs with K-major
// operands, 128 to 256 columns and the forward (and logits-gradient)
// epilogues.
template <int BN, int EPI, int LAYOUT, int CG>
constexpr bool tc_supported() {
  if (CG == 2)
    return LAYOUT == LAYOUT_KK && BN >= 128 && EPI != EPI_F32 && EPI != EPI_DGELU;
  if (EPI == EPI_RESID && BN == 256) return false;
  if (EPI == EPI_F32 && BN == 256 && LAYOUT != LAYOUT_MN_MN) return false;
  if (LAYOUT == LAYOUT_B_MN) return EPI == EPI_BIAS || EPI == EPI_F32 || EPI == EPI_DGELU;
  if (LAYOUT == LAYOUT_MN_MN) return EPI == EPI_F32;
  if (LAYOUT == LAYOUT_A_MN) return false;
  return EPI != EPI_DGELU && EPI != EPI_F32;
}

// Clusters of two that fit on the device at once (queried once per kernel).
template <typename Kern>
int pair_slots(Kern kern, int threads, int smem, int num_sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms / 2));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms / 2;
  }
  return std::min(n, num_sms / 2);
}

template <int BN, int EPI, int LAYOUT, int CG>
cudaError_t launch_one(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tC, const CUtensorMap& tD,
                       const GemmArgs& a, int num_sms, cudaStream_t s) {
  if constexpr (!tc_supported<BN, EPI, LAYOUT, CG>()) {
    return cudaErrorInvalidValue;
  } else {
    using L = TcLayout<BN, EPI, CG>;
    auto kern = gemm_tc_kernel<BN, EPI, LAYOUT, CG>;
    const int ks = (EPI == EPI_F32 && a.k_split == 2) ? 2 : 1;
    const int tiles = ((a.M + TC_BM * CG - 1) / (TC_BM * CG)) * ((a.N + BN - 1) / BN) * ks;
    if (CG == 1) {
      const int grid = std::min(tiles, num_sms);
      if (grid <= 0) return cudaSuccess;
      return launch_pdl(kern, dim3(grid), dim3(L::THREADS), L::SMEM_BYTES, s, tA, tB, tC, tD, a);
    }
    static const int slots = pair_slots(kern, L::THREADS, L::SMEM_BYTES, num_sms);
    const int pairs = std::min(tiles, slots);
    if (pairs <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(L::THREADS);
    cfg.dynamicSmemBytes = L::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tA, tB, tC, tD, a);
  }
}

template <int BN, int EPI, int LAYOUT, int CG>
cudaError_t set_attr_one() {
  if constexpr (!tc_supported<BN, EPI, LAYOUT, CG>()) return cudaSuccess;
  else return cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI, LAYOUT, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TcLayout<BN, EPI, CG>::SMEM_BYTES);
}

template <int BN, int LAYOUT, int CG>
cudaError_t launch_bn(int epi, const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tC,
                      const CUtensorMap& tD, const GemmArgs& a, int num_sms, cudaStream_t s) {
  switch (epi) {
    case EPI_BIAS: return launch_one<BN, EPI_BIAS, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
    case EPI_GELU: return launch_one<BN, EPI_GELU, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
    case EPI_RESID: return launch_one<BN, EPI_RESID, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
    case EPI_LMHEAD:
      return a.out != nullptr ? launch_one<BN, EPI_LMHEAD_LOGITS, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s)
                              : launch_one<BN, EPI_LMHEAD, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
    case EPI_F32: return launch_one<BN, EPI_F32, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
    case EPI_DGELU: return launch_one<BN, EPI_DGELU, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
    case EPI_DLOGITS: return launch_one<BN, EPI_DLOGITS, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
    case EPI_GELU_SAVE: return launch_one<BN, EPI_GELU_SAVE, LAYOUT, CG>(tA, tB, tC, tD, a, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

template <int BN>
cudaError_t launch_layout(int layout, int pair, int epi, const CUtensorMap& tA, const CUtensorMap& tB,
                          const CUtensorMap& tC, const CUtensorMap& tD, const GemmArgs& a, int num_sms,
                          cudaStream_t s) {
  if (pair) return layout == LAYOUT_KK ? launch_bn<BN, LAYOUT_KK, 2>(epi, tA, tB, tC, tD, a, num_sms, s)
                                       : cudaErrorInvalidValue;
  switch (layout) {
    case LAYOUT_KK: return launch_bn<BN, LAYOUT_KK, 1>(epi, tA, tB, tC, tD, a, num_sms, s);
    case LAYOUT_B_MN: return launch_bn<BN, LAYOUT_B_MN, 1>(epi, tA, tB, tC, tD, a, num_sms, s);
    case LAYOUT_MN_MN: return launch_bn<BN, LAYOUT_MN_MN, 1>(epi, tA, tB, tC, tD, a, num_sms, s);
  }
  return cudaErrorInvalidValue;
}
}  // namespace

bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                    uint32_t box_rows) {
  return encode_2d(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, ld, 64, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_tmap_out_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint64_t ld) {
  return encode_2d(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

bool make_tmap_out_f32(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint64_t ld) {
  return encode_2d(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, rows, cols, ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
}

namespace {
bool encode_3d(CUtensorMap* tm, CUtensorMapDataType dt, int esize, const void* base, uint64_t d0, uint64_t d1,
               uint64_t d2, uint64_t s1, uint64_t s2, uint32_t box0, uint32_t box1) {
  if (!load_encode()) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((s1 * esize) & 15) || ((s2 * esize) & 15) || !d0 || !d1 || !d2)
    return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1 * (uint64_t)esize, s2 * (uint64_t)esize};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(tm, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

bool make_tmap_3d_bf16(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                       uint64_t s2, uint32_t box0, uint32_t box1) {
  return encode_3d(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, d0, d1, d2, s1, s2, box0, box1);
}

bool make_tmap_3d_f32(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                      uint64_t s2, uint32_t box0, uint32_t box1) {
  return encode_3d(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, d0, d1, d2, s1, s2, box0, box1);
}

int gemm_tc_n_tiles(int N, int bn) { return (bn / 64) * ((N + bn - 1) / bn); }   // TcLayout::GROUPS per tile

bool gemm_tc_pair_ok(int epi, int layout, int bn) {
  return layout == LAYOUT_KK && bn >= 128 && epi != EPI_F32 && epi != EPI_DGELU;
}

GemmPick gemm_tc_pick(int M, int N, int num_sms, int epi, int layout) {
  // CTA pairs (K-major operands, at least two 128-row blocks, the forward
  // and logits-gradient epilogues) only on request, G2_GEMM_PAIR=1: on the
  // B200 they measured no faster on the GPT-2 shapes (the single-CTA main
  // loop is not bound by shared-memory bandwidth; the block's GEMMs are
  // bound by pipeline fill, the exposed last epilogue and whole waves of
  // tiles, and the pair's two epilogues gate each other's accumulator).
  bool pair = false;
  if (const char* e = getenv("G2_GEMM_PAIR"))
    pair = atoi(e) != 0 && layout == LAYOUT_KK && M > TC_BM && epi != EPI_F32 && epi != EPI_DGELU && num_sms >= 2;
  // The fp32 epilogues run with tiles of at most 192 columns on one CTA.
  const int max_bn = (!pair && (epi == EPI_RESID || epi == EPI_F32)) ? 192 : 256;
  const int min_bn = pair ? 128 : 64;
  // G2_GEMM_BN=64|128|192|256 pins the tile width (tests use it to cover
  // every instantiation); otherwise the width is chosen by the cost model below.
  if (const char* e = getenv("G2_GEMM_BN")) {
    const int v = atoi(e);
    if (v == 64 || v == 128 || v == 192 || v == 256) return GemmPick{std::max(std::min(v, max_bn), min_bn), pair};
  }
  // Estimated cost = waves x per-tile cost. Narrower tiles re-read A from
  // shared memory more often per FLOP (the 128-row MMA at N=128 runs at
  // about 60% of the N=256 rate), so their per-column cost is higher; N=192
  // still keeps the MMA's shared-memory reads under the per-SM bandwidth.
  // A narrower width must win by more than 2% to be taken. A pair's tile is
  // 256 rows and a wave is one tile per pair of SMs.
  const int cand[4] = {256, 192, 128, 64};
  const double unit[4] = {256.0, 192.0, 200.0, 150.0};
  const int bm = pair ? 2 * TC_BM : TC_BM;
  const int slots = pair ? num_sms / 2 : num_sms;
  const int mt = (M + bm - 1) / bm;
  int best = max_bn;
  double best_cost = 1e30;
  for (int i = 0; i < 4; ++i) {
    if (cand[i] > max_bn || cand[i] < min_bn) continue;
    const long tiles = (long)mt * ((N + cand[i] - 1) / cand[i]);
    const long waves = (tiles + slots - 1) / slots;
    const double cost = waves * unit[i];
    if (cost < best_cost * 0.98) {
      best_cost = cost;
      best = cand[i];
    }
  }
  return GemmPick{best, pair};
}

int gemm_tc_pick_bn(int M, int N, int num_sms, int epi) { return gemm_tc_pick(M, N, num_sms, epi).bn; }

cudaError_t gemm_tc_launch(int epi, int bn, const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tC,
                           const GemmArgs& a, int num_sms, cudaStream_t s, int layout, const CUtensorMap* tD,
                           int pair) {
  if (epi == EPI_GELU_SAVE && tD == nullptr) return cudaErrorInvalidValue;
  if (pair && !gemm_tc_pair_ok(epi, layout, bn)) return cudaErrorInvalidValue;
  const CUtensorMap& d = tD ? *tD : tC;
  switch (bn) {
    case 256: return launch_layout<256>(layout, pair, epi, tA, tB, tC, d, a, num_sms, s);
    case 192: return launch_layout<192>(layout, pair, epi, tA, tB, tC, d, a, num_sms, s);
    case 128: return launch_layout<128>(layout, pair, epi, tA, tB, tC, d, a, num_sms, s);
    case 64: return launch_layout<64>(layout, pair, epi, tA, tB, tC, d, a, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

namespace {
template <int BN, int LAYOUT, int CG>
cudaError_t set_attr_layout() {
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_BIAS, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_GELU, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_RESID, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_LMHEAD, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_LMHEAD_LOGITS, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_F32, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_DGELU, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_DLOGITS, LAYOUT, CG>();
  if (e == cudaSuccess) e = set_attr_one<BN, EPI_GELU_SAVE, LAYOUT, CG>();
  return e;
}
template <int BN>
cudaError_t set_attr_bn() {
  cudaError_t e = set_attr_layout<BN, LAYOUT_KK, 1>();
  if (e == cudaSuccess) e = set_attr_layout<BN, LAYOUT_B_MN, 1>();
  if (e == cudaSuccess) e = set_attr_layout<BN, LAYOUT_MN_MN, 1>();
  if (e == cudaSuccess) e = set_attr_layout<BN, LAYOUT_KK, 2>();
  return e;
}
}  // namespace

cudaError_t gemm_tc_set_attributes() {
  cudaError_t e = set_attr_bn<256>();
  if (e == cudaSuccess) e = set_attr_bn<192>();
  if (e == cudaSuccess) e = set_attr_bn<128>();
  if (e == cudaSuccess) e = set_attr_bn<64>();
  return e;
}

}  // namespace g2
