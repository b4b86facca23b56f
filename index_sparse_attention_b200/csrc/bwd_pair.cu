// bwd_pair.cu -- sparse attention backward main kernel for head dims (256, 256) on a
// pair of CTAs (a 2-CTA thread-block cluster) per key tile.
//
// Operation: as in bwd.cu (MagiAttention PR #334, Summary and sections 1 and 3):
// recompute P = exp(scale S - LSE), dV += P^T dO, dP = dO V^T, dS = P (dP - Delta),
// dQ += dS K, dK += dS^T Q, over the transposed (key -> query) tile lists of
// MagiAttention PR #331 ("CSR Tile Mapping").
//
// Why a pair.  With 256-wide heads the fp32 dK and dV accumulators of a 128-key tile
// need 512 TMEM columns, everything the SM has, so each CTA can hold only a 128-wide
// head-dim half of them.  Two CTAs that each recompute S^T and dP^T for their half
// would do those contractions twice and would leave room for only one Q/dO stage.
// Here the two CTAs of a cluster split the work instead of duplicating it:
//   rank 0: S^T = K Q^T (all of K resident), P^T = exp2(S^T scale log2e - LSE log2e)
//           with the element mask, P^T -> own TMEM and (bf16, distributed shared
//           memory) rank 1's exchange tile; dV[:, 0:128] += P^T dO, dK[:, 0:128] +=
//           dS^T Q, dQ^T[0:128] = K^T dS^T with dS^T received from rank 1.
//   rank 1: dP^T = V dO^T (all of V resident), dS^T = P^T (dP^T - Delta) with P^T from
//           rank 0, dS^T -> own TMEM, own shared memory and rank 0's exchange tile;
//           dV[:, 128:256] += P^T dO, dK[:, 128:256] += dS^T Q,
//           dQ^T[128:256] = K^T dS^T.
// Each rank does the same tensor-core work per step, keeps two Q/dO stages, and the
// exchange tiles are double-buffered, so the next step's S^T / dP^T overlap the
// current step's elementwise work on both ranks.
//
// Per 64-query step the exchanges are single 16 KB bulk copies (cp.async.bulk,
// shared::cta -> shared::cluster, no multicast) of a whole exchange tile, completing as
// transaction bytes on the receiving CTA's barrier XF[b].  The receiver arms XF[b] itself
// (one local arrival expecting the 16 KB) for step it+2 once it has consumed step it, so
// a sender issues nothing but the copy:
//   rank 0 stages P^T(it) in its own tile b and copies it into rank 1's tile b;
//   rank 1 overwrites its tile b with dS^T(it) (after dV has read P^T there) and copies
//   it into rank 0's tile b (rank 0's copy of P^T has landed by then).
// A copy signals only its receiver, so the receiver tells the sender when a tile may be
// reused, with a relaxed remote arrival (it carries no data: the readers have finished):
//   XS[b] on rank 1: dS^T(it) has landed in rank 0 (rank 1's dQ drain may stage in tile b);
//   XE[b] on rank 0: rank 1's tile b is free (its dQ drain used it as staging last).
// A release at cluster scope is avoided throughout: it would stall the signalling thread
// on all of its earlier memory operations.
// No TMA multicast and no multicast commit are used.  Every wait is bounded.
#include "sa_device.cuh"
#include "sa_kernels.h"

#include <cstdio>
#include <cstdlib>

namespace sa {
namespace pairbwd {

constexpr int BM = 64;                      // queries per step
constexpr int kKPanel = 128 * 128;          // [128 rows x 64 cols] bf16 (16 KB)
constexpr int kQPanel = BM * 128;           // [64 rows x 64 cols] bf16 (8 KB)
constexpr int kTile = 128 * BM * 2;         // [128 keys][64 q] bf16 exchange tile (16 KB)
constexpr int kOffA = 0;                    // rank 0: K (4 panels); rank 1: V (4 panels)
constexpr int kOffB = 64 * 1024;            // rank 1: K panels 2,3; rank 0: dQ staging + words
constexpr int kOffBM = kOffB + 16 * 1024;   // rank 0: presence words [2][64][4] (index mode)
constexpr int kOffStage = 96 * 1024;        // two stages of 48 KB
constexpr int kStageBytes = 48 * 1024;      // rank 0: Q p0-3, dO p0-1; rank 1: dO p0-3, Q p2-3
constexpr int kOffX = kOffStage + 2 * kStageBytes;   // two exchange tiles
constexpr int kOffL = kOffX + 2 * kTile;              // per stage lse2[64] / delta[64]
constexpr int kOffBar = kOffL + 2 * BM * 4;
constexpr int kSmem = kOffBar + 256 + 1024;
constexpr int kThreads = 448;
static_assert(kSmem <= 227 * 1024, "shared memory budget");
// TMEM columns
constexpr uint32_t kColBuf = 0;   // + 64 * b: S^T (rank 0) / dP^T (rank 1); packed bf16 in low cols
constexpr uint32_t kColDQ = 128;  // dQ^T (head-dim row x 64 queries)
constexpr uint32_t kColDV = 192;
constexpr uint32_t kColDK = 320;
constexpr uint32_t kTmemCols = 512;

enum : int {
  kBKV = 0, kBQF = 1, kBQE = 3, kBLF = 5, kBSF = 7, kBEW = 9, kBXF = 11, kBXE = 13, kBPV = 15,
  kBDQF = 17, kBDQE = 19, kBFin = 21, kBDrain = 22, kBXS = 23, kNumBars = 25
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(448, 1)
    sparse_bwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_dq, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + 8 * kNumBars + 4);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int nt = static_cast<int>(blockIdx.x) >> 1;
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = a.HQ / a.HK;
  const int64_t bg = static_cast<int64_t>(b) * a.HK + g;
  const int64_t trow = bg * a.Tn + nt;
  const int n_full = __ldg(a.tcnt + 2 * trow);
  const int n_mt = n_full + __ldg(a.tcnt + 2 * trow + 1);
  const int32_t* tlist = a.tidx + trow * a.Tm;
  const int n_iter = G * n_mt * 2;
  const int c0 = 128 * static_cast<int>(rank);  // this rank's head-dim half

  if (threadIdx.x == 0) {
    mbar_init(BAR(kBKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(kBQF + s), 1);
      mbar_init(BAR(kBQE + s), 1);
      mbar_init(BAR(kBLF + s), 32);
      mbar_init(BAR(kBSF + s), 1);
      mbar_init(BAR(kBEW + s), 256);
      mbar_init(BAR(kBXF + s), 1);
      mbar_init(BAR(kBXE + s), 1);
      mbar_init(BAR(kBXS + s), 1);
      mbar_init(BAR(kBPV + s), 1);
      mbar_init(BAR(kBDQF + s), 1);
      mbar_init(BAR(kBDQE + s), 128);
    }
    mbar_init(BAR(kBFin), 1);
    mbar_init(BAR(kBDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  // the exchange tiles of steps 0 and 1 may arrive from the peer at any time
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2 && s < n_iter; ++s) mbar_arrive_expect_tx(BAR(kBXF + s), kTile);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrive or copy
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, *tmem_slot, 0);

  auto decode = [&](int it, int& h, int& m0, bool& partial) {
    const int per_head = 2 * n_mt;
    const int hh = it / per_head;
    const int rest = it - hh * per_head;
    const int k = rest >> 1;
    h = g * G + hh;
    m0 = __ldg(tlist + k) * 128 + (rest & 1) * BM;
    partial = k >= n_full;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (n_iter > 0) {
      if (elect_one()) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_do);
        prefetch_tensormap(&tm_dq);
        if (rank == 0) {
          mbar_arrive_expect_tx(BAR(kBKV), 4 * kKPanel);
          for (int c = 0; c < 4; ++c)
            tma_load_4d(sbase + kOffA + c * kKPanel, &tm_k, BAR(kBKV), c * 64, nt * 128, g, b);
        } else {
          mbar_arrive_expect_tx(BAR(kBKV), 6 * kKPanel);
          for (int c = 0; c < 4; ++c)
            tma_load_4d(sbase + kOffA + c * kKPanel, &tm_v, BAR(kBKV), c * 64, nt * 128, g, b);
          for (int c = 2; c < 4; ++c)
            tma_load_4d(sbase + kOffB + (c - 2) * kKPanel, &tm_k, BAR(kBKV), c * 64, nt * 128, g, b);
        }
      }
      __syncwarp();
      float* lbuf = reinterpret_cast<float*>(smem + kOffL);
      uint32_t* bmbuf = reinterpret_cast<uint32_t*>(smem + kOffBM);
      for (int it = 0; it < n_iter; ++it) {
        int h, m0;
        bool partial;
        decode(it, h, m0, partial);
        m0 = __shfl_sync(0xFFFFFFFFu, m0, 0);
        const int st = it & 1, u = it >> 1;
        if (!warp_wait(BAR(kBQE + st), (u & 1) ^ 1, abort_flag, a.status)) break;
        const uint32_t qs = sbase + kOffStage + st * kStageBytes;
        if (elect_one()) {
          mbar_arrive_expect_tx(BAR(kBQF + st), kStageBytes);
          if (rank == 0) {
            for (int c = 0; c < 4; ++c)
              tma_load_4d(qs + c * kQPanel, &tm_q, BAR(kBQF + st), c * 64, m0, h, b);
            for (int c = 0; c < 2; ++c)
              tma_load_4d(qs + 32 * 1024 + c * kQPanel, &tm_do, BAR(kBQF + st), c * 64, m0, h, b);
          } else {
            for (int c = 0; c < 4; ++c)
              tma_load_4d(qs + c * kQPanel, &tm_do, BAR(kBQF + st), c * 64, m0, h, b);
            for (int c = 2; c < 4; ++c)
              tma_load_4d(qs + 32 * 1024 + (c - 2) * kQPanel, &tm_q, BAR(kBQF + st), c * 64, m0, h,
                          b);
          }
        }
        __syncwarp();
        // rank 0: LSE in log2 units (+inf past Sq); rank 1: Delta (0 past Sq)
        float* ls = lbuf + st * BM;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int q = lane + 32 * k;
          const int64_t i = m0 + q;
          float v = rank == 0 ? INFINITY : 0.f;
          if (i < a.Sq) {
            const int64_t li = (static_cast<int64_t>(b) * a.HQ + h) * a.Sq + i;
            v = rank == 0 ? __ldg(a.lse + li) * 1.4426950408889634f : __ldg(a.delta + li);
          }
          ls[q] = v;
        }
        if (rank == 0 && partial && a.mode == SA_MODE_INDEX) {
          uint32_t* bw = bmbuf + st * BM * 4;
          for (int e = lane; e < BM * 4; e += 32) {
            const int q = e >> 2, w = nt * 4 + (e & 3);
            const int64_t i = m0 + q;
            bw[e] = (i < a.Sq && w < a.W) ? __ldg(a.bitmap + (bg * a.Sq + i) * a.W + w) : 0u;
          }
        }
        mbar_arrive(BAR(kBLF + st));
      }
      if (lane == 0 && *abort_flag) {
        mbar_wait_limited(BAR(kBKV), 0);
        for (int it = max(0, n_iter - 2); it < n_iter; ++it)
          mbar_wait_limited(BAR(kBQF + (it & 1)), (it >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (n_iter > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, BM, 0, 0);     // S^T / dP^T
      constexpr uint32_t idesc_dq = idesc_bf16(128, BM, 1, 1);    // dQ^T = K^T dS^T
      constexpr uint32_t idesc_tsn = idesc_bf16(128, 128, 0, 1);  // A in TMEM, B MN-major
      constexpr uint32_t idesc_ssn = idesc_bf16(128, 128, 0, 1);  // A K-major smem, B MN-major
      const uint64_t ad = sw128_desc(sbase + kOffA, 16, 1024);    // K (rank 0) / V (rank 1)
      // dQ^T A operand: this rank's 128 head-dim rows of K (MN-major)
      const uint64_t kwd = sw128_desc(sbase + (rank == 0 ? kOffA : kOffB), kKPanel, 1024);
      bool ok = warp_wait(BAR(kBKV), 0, abort_flag, a.status);
      // S^T (rank 0) or dP^T (rank 1) of step j into TMEM buffer j & 1
      auto issue_first = [&](int j) -> bool {
        const int st = j & 1;
        if (!warp_wait(BAR(kBQF + st), (j >> 1) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint64_t bd = sw128_desc(sbase + kOffStage + st * kStageBytes, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            const uint32_t off_a = (kk >> 2) * kKPanel + (kk & 3) * 32;
            const uint32_t off_b = (kk >> 2) * kQPanel + (kk & 3) * 32;
            umma_ss(tmem + kColBuf + 64 * st, ad + (off_a >> 4), bd + (off_b >> 4), idesc_s,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(BAR(kBSF + st));
        }
        __syncwarp();
        return true;
      };
      if (ok) ok = issue_first(0);
      for (int it = 0; ok && it < n_iter; ++it) {
        const int bi = it & 1, st = it & 1, ph = (it >> 1) & 1;
        const uint32_t qs = sbase + kOffStage + st * kStageBytes;
        const uint32_t xt = sbase + kOffX + bi * kTile;
        // this rank's half of the second operand: rank 0 dO panels 0,1 / Q panels 0,1;
        // rank 1 dO panels 2,3 / Q panels 2,3
        const uint64_t do_half = sw128_desc(qs + (rank == 0 ? 32 * 1024 : 2 * kQPanel), kQPanel, 1024);
        const uint64_t q_half = sw128_desc(qs + (rank == 0 ? 0 : 32 * 1024), kQPanel, 1024);
        const uint64_t xk = sw128_desc(xt, 16, 1024);        // exchange tile, K-major A
        const uint64_t xmn = sw128_desc(xt, kKPanel, 1024);  // exchange tile, MN-major B
        if (rank == 0) {
          // the next S^T overlaps this step's elementwise work
          if (it + 1 < n_iter && !issue_first(it + 1)) break;
          // dV += P^T dO (P^T packed in TMEM by the elementwise warps)
          if (!warp_wait(BAR(kBEW + bi), ph, abort_flag, a.status)) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ts(tmem + kColDV, tmem + kColBuf + 64 * bi + (kk >> 1) * 32 + (kk & 1) * 8,
                      do_half + ((kk * 2048) >> 4), idesc_tsn, (it > 0 || kk > 0) ? 1u : 0u);
          }
          __syncwarp();
          // dK += dS^T Q with dS^T copied in by rank 1 (exchange tile, K-major A)
          if (!warp_wait(BAR(kBXF + bi), ph, abort_flag, a.status)) break;
          if (elect_one()) {
            mbar_arrive_remote_relaxed(mapa_shared(BAR(kBXS + bi), peer));
            if (it + 2 < n_iter) mbar_arrive_expect_tx(BAR(kBXF + bi), kTile);
          }
          __syncwarp();
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ss(tmem + kColDK, xk + ((kk * 32) >> 4), q_half + ((kk * 2048) >> 4), idesc_ssn,
                      (it > 0 || kk > 0) ? 1u : 0u);
            umma_commit(BAR(kBQE + st));
          }
          __syncwarp();
        } else {
          // dV += P^T dO with P^T copied in by rank 0 (exchange tile, K-major A), first,
          // so that the elementwise warps may overwrite the tile with dS^T soon
          if (!warp_wait(BAR(kBXF + bi), ph, abort_flag, a.status)) break;
          tc_fence_after();
          if (elect_one()) {
            // every reader of this phase has passed its wait (the elementwise warps read
            // the tile before step it+2 can be sent): arm the barrier for step it+2
            if (it + 2 < n_iter) mbar_arrive_expect_tx(BAR(kBXF + bi), kTile);
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ss(tmem + kColDV, xk + ((kk * 32) >> 4), do_half + ((kk * 2048) >> 4), idesc_ssn,
                      (it > 0 || kk > 0) ? 1u : 0u);
            umma_commit(BAR(kBPV + bi));
          }
          __syncwarp();
          // the next dP^T overlaps this step's elementwise work
          if (it + 1 < n_iter && !issue_first(it + 1)) break;
          // dK += dS^T Q (dS^T packed in TMEM by the elementwise warps)
          if (!warp_wait(BAR(kBEW + bi), ph, abort_flag, a.status)) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ts(tmem + kColDK, tmem + kColBuf + 64 * bi + (kk >> 1) * 32 + (kk & 1) * 8,
                      q_half + ((kk * 2048) >> 4), idesc_tsn, (it > 0 || kk > 0) ? 1u : 0u);
            umma_commit(BAR(kBQE + st));
          }
          __syncwarp();
        }
        // dQ^T = K^T dS^T for this rank's head-dim half, once the last one was drained
        if (it >= 1 &&
            !warp_wait(BAR(kBDQE + ((it - 1) & 1)), ((it - 1) >> 1) & 1, abort_flag, a.status))
          break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            umma_ss(tmem + kColDQ, kwd + ((kk * 2048) >> 4), xmn + ((kk * 2048) >> 4), idesc_dq,
                    kk > 0 ? 1u : 0u);
          umma_commit(BAR(kBDQF + bi));
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(BAR(kBFin));
      __syncwarp();
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------------ elementwise
    const int quarter = warp & 3;
    const int hc = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;  // key row = TMEM lane
    const int64_t j = static_cast<int64_t>(nt) * 128 + r;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float* lbuf = reinterpret_cast<const float*>(smem + kOffL);
    const uint32_t* bmbuf = reinterpret_cast<const uint32_t*>(smem + kOffBM);
    const bool key_ok = j < a.Sk;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      int h, m0;
      bool partial;
      decode(it, h, m0, partial);
      const int bi = it & 1, st = it & 1, ph = (it >> 1) & 1;
      bool w_ok = mbar_wait(BAR(kBLF + st), ph, abort_flag, a.status);
      w_ok = w_ok && mbar_wait(BAR(kBSF + bi), ph, abort_flag, a.status);
      if (rank == 1) {
        w_ok = w_ok && mbar_wait(BAR(kBXF + bi), ph, abort_flag, a.status);  // P^T(it) arrived
      } else if (it >= 2) {
        // own tile b: dK and dQ^T of step it-2 have read dS^T
        w_ok = w_ok && mbar_wait(BAR(kBDQF + bi), ((it - 2) >> 1) & 1, abort_flag, a.status);
      }
      if (!__all_sync(0xFFFFFFFFu, w_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* ls = lbuf + st * BM + 32 * hc;
      const uint32_t cbuf = kColBuf + 64 * bi + 32 * hc;
      uint32_t s_u[32];
      tmem_ld32(tl + cbuf, s_u);
      const uint32_t row_off = kOffX + bi * kTile + r * 128;  // row r of exchange tile b
      uint32_t pk[16];
      if (rank == 0) {
        uint32_t cm = 0xFFFFFFFFu;
        if (partial) {
          const int64_t q0 = m0 + 32 * hc;
          cm = key_ok ? 0xFFFFFFFFu : 0u;
          if (a.causal) {
            const int64_t lo = j - q0;
            cm &= lo <= 0 ? 0xFFFFFFFFu : (lo >= 32 ? 0u : (0xFFFFFFFFu << lo));
          }
          if (a.mode == SA_MODE_BLOCK && a.bs == 64 && key_ok) {
            const int64_t mb = m0 / 64;
            const bool m = mb < a.Mb &&
                           __ldg(a.mask + (bg * a.Mb + mb) * static_cast<int64_t>(a.Nb) + j / 64) != 0;
            if (!m) cm = 0u;
          } else if (a.mode == SA_MODE_INDEX) {
            const uint32_t* bw = bmbuf + st * BM * 4 + (32 * hc) * 4 + (r >> 5);
            uint32_t bits = 0u;
#pragma unroll 8
            for (int q = 0; q < 32; ++q) bits |= ((bw[q * 4] >> lane) & 1u) << q;
            cm &= bits;
          }
        }
        tmem_wait_ld();
        const float4* ls4 = reinterpret_cast<const float4*>(ls);
        const float sc = a.scale_log2;
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 l = ls4[e4];
          const float lv[4] = {l.x, l.y, l.z, l.w};
          float pv[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int q = 4 * e4 + t;
            pv[t] = ((cm >> q) & 1u) ? ex2(fmaf(__uint_as_float(s_u[q]), sc, -lv[t])) : 0.f;
          }
          pk[2 * e4] = pack_bf16x2(pv[0], pv[1]);
          pk[2 * e4 + 1] = pack_bf16x2(pv[2], pv[3]);
        }
        tmem_st16(tl + cbuf, pk);
        // P^T row (this half's 32 queries) into the own exchange tile, 128-byte swizzled:
        // 16-byte chunk c of row r lives at chunk c ^ (r % 8)
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = hc * 4 + c4;
          *reinterpret_cast<uint4*>(smem + row_off + ((c ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(kBEW + bi));
        // one thread copies the whole tile into rank 1 once every row is in and rank 1's
        // tile b is free (its dQ drain of step it-2 is done with it)
        if (threadIdx.x == 64 && mbar_wait(BAR(kBEW + bi), ph, abort_flag, a.status) &&
            (it < 2 || mbar_wait(BAR(kBXE + bi), ((it - 2) >> 1) & 1, abort_flag, a.status))) {
          bulk_copy_to_cluster(mapa_shared(sbase + kOffX + bi * kTile, peer),
                               sbase + kOffX + bi * kTile, kTile, mapa_shared(BAR(kBXF + bi), peer));
        }
      } else {
        // P^T row from the own exchange tile (written by rank 0)
        uint32_t pw[16];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = hc * 4 + c4;
          const uint4 v = *reinterpret_cast<const uint4*>(smem + row_off + ((c ^ (r & 7)) << 4));
          pw[4 * c4] = v.x;
          pw[4 * c4 + 1] = v.y;
          pw[4 * c4 + 2] = v.z;
          pw[4 * c4 + 3] = v.w;
        }
        tmem_wait_ld();
        const float4* dl4 = reinterpret_cast<const float4*>(ls);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 d = dl4[e4];
          const float dv4[4] = {d.x, d.y, d.z, d.w};
          float dsv[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int q = 4 * e4 + t;
            const __nv_bfloat162 p2 = *reinterpret_cast<const __nv_bfloat162*>(&pw[q >> 1]);
            const float p = (q & 1) ? __high2float(p2) : __low2float(p2);
            dsv[t] = p * (__uint_as_float(s_u[q]) - dv4[t]);
          }
          pk[2 * e4] = pack_bf16x2(dsv[0], dsv[1]);
          pk[2 * e4 + 1] = pack_bf16x2(dsv[2], dsv[3]);
        }
        tmem_st16(tl + cbuf, pk);
        // dV of this step must have read P^T before dS^T replaces it in the tile
        const bool pv_ok = mbar_wait(BAR(kBPV + bi), ph, abort_flag, a.status);
        if (!__all_sync(0xFFFFFFFFu, pv_ok)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = hc * 4 + c4;
          *reinterpret_cast<uint4*>(smem + row_off + ((c ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(kBEW + bi));
        // one thread copies the whole dS^T tile into rank 0 once every row is in
        if (threadIdx.x == 64 && mbar_wait(BAR(kBEW + bi), ph, abort_flag, a.status)) {
          bulk_copy_to_cluster(mapa_shared(sbase + kOffX + bi * kTile, peer),
                               sbase + kOffX + bi * kTile, kTile, mapa_shared(BAR(kBXF + bi), peer));
        }
      }
    }
    // ----------------------------------------------------------- dK / dV epilogue
    bool have = n_iter > 0 && ok;
    if (have) {
      const bool w_ok = mbar_wait(BAR(kBFin), 0, abort_flag, a.status);
      have = __all_sync(0xFFFFFFFFu, w_ok);
      tc_fence_after();
    }
    __nv_bfloat16* dkrow = reinterpret_cast<__nv_bfloat16*>(a.dk) +
                           ((static_cast<int64_t>(b) * a.Sk + j) * a.HK + g) * 256;
    __nv_bfloat16* dvrow = reinterpret_cast<__nv_bfloat16*>(a.dv) +
                           ((static_cast<int64_t>(b) * a.Sk + j) * a.HK + g) * 256;
    for (int pass = 0; pass < 2; ++pass) {
      const uint32_t col = pass == 0 ? kColDK : kColDV;
      const float sc = pass == 0 ? a.scale : 1.f;
      __nv_bfloat16* out = pass == 0 ? dkrow : dvrow;
      for (int c = 32 * hc; c < 128; c += 64) {
        uint32_t v[32];
        if (have) {
          tmem_ld32(tl + col + c, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        if (key_ok) {
          uint32_t pq[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pq[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
          uint4* dst = reinterpret_cast<uint4*>(out + c0 + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pq[4 * e], pq[4 * e + 1], pq[4 * e + 2], pq[4 * e + 3]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ dQ drain
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // head-dim row of this rank's half
    const int dtid = threadIdx.x - 320;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int p = r >> 6;
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      int h, m0;
      bool partial;
      decode(it, h, m0, partial);
      const int bi = it & 1;
      // the four drain warps leave together (they share named barrier 1 below)
      const bool w_ok = mbar_wait(BAR(kBDQF + bi), (it >> 1) & 1, abort_flag, a.status);
      if (!named_bar_and(1, 128, w_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t q_u[BM];
      tmem_ld32(tl + kColDQ, q_u);
      tmem_ld32(tl + kColDQ + 32, q_u + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(BAR(kBDQE + bi));
      if (rank == 1) {
        // the outgoing copy of dS^T must have read the exchange tile before staging
        const bool x_ok = mbar_wait(BAR(kBXS + bi), (it >> 1) & 1, abort_flag, a.status);
        if (!named_bar_and(1, 128, x_ok)) {
          ok = false;
          break;
        }
      }
      // staging: rank 0 has a buffer of its own, rank 1 reuses the exchange tile
      const int soff = rank == 0 ? kOffB : kOffX + bi * kTile;
      float* stage = reinterpret_cast<float*>(smem + soff);
      const uint32_t stage_s = sbase + soff;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (half == 1 || rank == 0) {
          if (dtid == 0) bulk_wait_group_read0();
          named_bar_sync(1, 128);
        }
#pragma unroll
        for (int q = 0; q < 32; ++q)
          stage[(p * 32 + q) * 64 + (r & 63)] = __uint_as_float(q_u[32 * half + q]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (dtid == 0) {
          tma_reduce_add_4d(&tm_dq, stage_s, c0, m0 + 32 * half, h, b);
          tma_reduce_add_4d(&tm_dq, stage_s + 32 * 64 * 4, c0 + 64, m0 + 32 * half, h, b);
          bulk_commit_group();
        }
      }
      if (rank == 1) {
        // the exchange tile is free once the reduce has read it: rank 0 may refill it
        if (dtid == 0) bulk_wait_group_read0();
        named_bar_sync(1, 128);
        if (dtid == 0) mbar_arrive_remote_relaxed(mapa_shared(BAR(kBXE + bi), peer));
      }
    }
    if (dtid == 0) bulk_wait_group0();
  }

  if (warp == 1 && *abort_flag) {
    if (elect_one()) {
      umma_commit(BAR(kBDrain));
      mbar_wait_limited(BAR(kBDrain), 0);
      // the peer may have a 16 KB copy into this CTA in flight: give it time to land
      for (int k = 0; k < 100; ++k) __nanosleep(1000);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still write to it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pairbwd

int launch_bwd_pair(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    const int rc = cuda_error(cudaFuncSetAttribute(pairbwd::sparse_bwd_pair_kernel,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   pairbwd::kSmem),
                              "pair backward smem attribute");
    if (rc) return rc;
    attr_set = true;
  }
  dim3 grid(a.Tn * 2, a.HK, a.B);
  record_event(3, st);
  pairbwd::sparse_bwd_pair_kernel<<<grid, pairbwd::kThreads, pairbwd::kSmem, st>>>(
      m.q, m.k, m.v, m.dout, m.dq_acc, a);
  record_event(4, st);
  return check_launch("pair backward kernel launch");
}

}  // namespace sa
