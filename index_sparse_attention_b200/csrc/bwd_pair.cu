// bwd_pair.cu -- sparse attention backward main kernel for head dims (256, 256) on a
// pair of CTAs (a 2-CTA thread-block cluster) per key tile.
//
// Operation: as in bwd.cu (MagiAttention PR #334, Summary and sections 1 and 3):
// recompute P = exp(scale S - LSE), dV += P^T dO, dP = dO V^T, dS = P (dP - Delta),
// dQ += dS K, dK += dS^T Q, over the transposed (key -> query) tile lists of
// MagiAttention PR #331 ("CSR Tile Mapping").
//
// Why a pair.  With 256-wide heads the fp32 dK and dV accumulators of a 128-key tile
// need 512 TMEM columns, everything one SM has.  Two CTAs that each recompute S^T and
// dP^T for a head-dim half would do those contractions twice and have room for only
// one Q/dO stage.  Here the two CTAs of a cluster split the work by role:
//   rank 0 holds K in TMEM (and K[:, 0:128] in shared memory) and stages of Q:
//           S^T = K Q^T (K as the TMEM operand), P^T = exp2(S^T scale log2e - LSE log2e)
//           with the element mask (bf16, into an exchange tile), dK += dS^T Q (all 256
//           columns), dQ^T[0:128] = K[:, 0:128]^T dS^T;
//   rank 1 holds V in TMEM, K[:, 128:256] and stages of dO: dP^T = V dO^T (V as the
//           TMEM operand), dS^T = P^T (dP^T - Delta) (bf16, into an exchange tile),
//           dV += P^T dO (all 256 columns), dQ^T[128:256] = K[:, 128:256]^T dS^T into
//           the TMEM buffer the elementwise warps have just read dP^T from.
// Each rank issues about the same tensor-core work per 64-query step, and a stage
// holds only Q or only dO.  Both contractions over the full head dim read their
// stationary operand from TMEM: with 256-wide heads a shared-memory operand would cost
// 64 KB of shared-memory reads per step, the resource that bounds this kernel (the
// tensor core reads at most 128 B/clk of operands from it, and the TMA loads, the
// exchanges and the dQ staging share the same bandwidth).  Rank 0 keeps four Q stages
// (its stages are held from the load to dK, across both exchanges), rank 1 three.
//
// Exchanges.  Per step, P^T (rank 0 -> 1) and dS^T (rank 1 -> 0) cross as bulk copies
// (cp.async.bulk shared::cta -> shared::cluster, no multicast) of 4 KB each, one per
// 32-row quarter of the 16 KB tile, issued as soon as that quarter's two warps have
// written it (barriers QH).  They complete their bytes on the receiver's barrier XF; the
// receiver arms XF itself (one local arrival expecting 16 KB) for the step that will use
// the tile next, so a sender issues nothing but the copies.
//   rank 0 has four tiles, step it using tile it % 4: it stages P^T, then receives
//           dS^T, then stages the dQ drain (XT: free again after the drain);
//   rank 1 receives P^T into three tiles (it % 3), each free once dV and the
//           elementwise warps have read it (PR), and writes dS^T into two tiles of its
//           own (it % 2), each free once dQ^T has read it and its copy has landed in
//           rank 0 (DF); it stages its dQ drain in a buffer of its own.
// A copy signals only its receiver, so the receivers report back with relaxed remote
// arrivals, which order no data (the readers have finished when they are sent):
//   XE[b] on rank 0: rank 1's P^T tile b is free again (sent by rank 1's MMA warp);
//   DF[b] on rank 1: its dS^T copy from tile b has landed in rank 0 (sent by rank 0's
//         MMA warp; DF also counts the commit of the dQ^T that reads the tile).
// A release at cluster scope is never used on the step path: it stalls the signalling
// thread on all of its earlier memory operations (about a microsecond on B200).
//
// Issue order.  The MMA warp of each rank does not follow a fixed order: it polls the
// barriers of its MMA streams and issues whichever is ready (rank 0: dK/dQ^T of the
// oldest step, else the next S^T; rank 1: dV, else dQ^T, else the next dP^T), and keeps
// S^T / dP^T at most a step or two ahead, because the tensor pipe runs in order and a
// queued batch would delay the contractions the exchange chain waits for.
//
// dK (rank 0) and dV (rank 1) leave through the idle stages: the elementwise warps write
// the bf16 rows there in the 128-byte-swizzled layout of the output map's box, and one
// thread issues four TMA tensor stores.
//
// No TMA multicast and no multicast commit are used.  Every wait is bounded.
#include "det_order.cuh"
#include "sa_device.cuh"
#include "sa_kernels.h"

#include <cstdio>

namespace sa {
namespace pairbwd {

constexpr int BM = 64;                      // queries per step
constexpr int kStages0 = 4;                 // Q stages (rank 0)
constexpr int kStages1 = 3;                 // dO stages (rank 1)
constexpr int kMaxStages = 4;
constexpr int kNX = 4;                      // exchange tiles per rank
constexpr int kKPanel = 128 * 128;          // [128 rows x 64 cols] bf16 (16 KB)
constexpr int kQPanel = BM * 128;           // [64 rows x 64 cols] bf16 (8 KB)
constexpr int kStageBytes = 4 * kQPanel;    // one 64 x 256 tile (32 KB)
constexpr int kTile = 128 * BM * 2;         // exchange tile [128 keys][64 q] bf16 (16 KB)
// rank 0: K columns 0..127 | 4 Q stages | 4 exchange tiles | lse2 per stage.  K columns
// 128..255 pass through exchange tiles 0 and 1 on their way into TMEM.
constexpr int kOffK0 = 0;
constexpr int kOffStage0 = 32 * 1024;
constexpr int kOffX0 = kOffStage0 + kStages0 * kStageBytes;
constexpr int kOffL0 = kOffX0 + kNX * kTile;
// rank 1: K columns 128..255 | 3 dO stages | 2 P^T tiles | 3 dS^T tiles | dQ staging |
// delta per stage.  V passes through stages 1 and 2 on its way into TMEM.
constexpr int kOffK1 = 0;
constexpr int kOffStage1 = 32 * 1024;
constexpr int kOffV1 = kOffStage1 + kStageBytes;
// rank 1: incoming P^T tiles (free once dV and the elementwise warps have read them) and
// outgoing dS^T tiles (free once dQ^T has read them and their copy has landed in rank 0)
constexpr int kNPI = 3;
constexpr int kNDO = 2;
constexpr int kOffPI1 = kOffStage1 + kStages1 * kStageBytes;
constexpr int kOffDO1 = kOffPI1 + kNPI * kTile;
constexpr int kOffDQ1 = kOffDO1 + kNDO * kTile;
constexpr int kOffL1 = kOffDQ1 + kTile;
// barriers at the same offset on both ranks (a rank addresses the peer's barriers
// through its own offsets)
constexpr int kOffBar = kOffL0 + 1024;
constexpr int kSmem = kOffBar + 512 + 1024;
constexpr int kThreads = 448;
static_assert(kOffL0 + kStages0 * BM * 4 <= kOffBar, "rank 0 shared-memory layout");
static_assert(kOffL1 + kStages1 * BM * 4 <= kOffBar, "rank 1 shared-memory layout");
static_assert(kSmem <= 227 * 1024, "shared memory budget");
// TMEM columns.  Rank 0: K as the A operand (bf16, two per column), one S^T buffer (the
// elementwise warps release it as soon as they have loaded it), dK, dQ^T.  Rank 1: dP^T
// buffers (each then holds the step's dQ^T half), dV, V as the A operand.
constexpr uint32_t kColK0 = 0;
constexpr uint32_t kColS0 = 128;
constexpr uint32_t kColAcc0 = 192;
constexpr uint32_t kColDQ0 = 448;
constexpr uint32_t kColP1 = 0;     // + 64 * (step % 2)
constexpr uint32_t kColAcc1 = 128;
constexpr uint32_t kColV1 = 384;
constexpr uint32_t kTmemCols = 512;
// how many steps S^T (rank 0) / dP^T (rank 1) may run ahead of the oldest dK / dV
constexpr int kLookS0 = 3;
constexpr int kLookS1 = 1;

enum : int {
  kBKV = 0,    // K / V (and rank 1's K half) loaded
  kBVT = 1,    // K (rank 0) / V (rank 1) copied into TMEM (256 threads)
  kBQF = 2,    // [4] stage loaded
  kBQE = 6,    // [4] stage free (commit after dK on rank 0, after dV on rank 1)
  kBLF = 10,   // [4] per-stage LSE / Delta written (32 producer lanes)
  kBSF = 14,   // [4] S^T / dP^T of step complete (commit), indexed by step % stages
  kBEW = 18,   // [4] elementwise work of the step done (256 threads)
  kBXF = 22,   // [4] rank 0: dS^T arrived in its tile; rank 1 [3]: P^T arrived
  kBXT = 26,   // [4] rank 0: own tile free after its dQ drain
  kBXE = 30,   // [3] rank 0: rank 1's P^T tile free (remote)
  kBDF = 33,   // [2] rank 1: dS^T tile free (dQ^T commit + remote arrival report)
  kBPR = 35,   // [3] rank 1: P^T tile read (256 elementwise threads + the dV commit)
  kBDQF = 38,  // [2] dQ^T complete (commit); rank 0 uses slot 0 only
  kBDQE = 40,  // [2] dQ^T drained from TMEM (128 threads)
  kBSR = 42,   // rank 0: the elementwise warps have loaded S^T (256 threads)
  kBFin = 43, kBDrain = 44,
  kBQH = 45,   // [2][4] exchange rows 32q..32q+31 of a step written (the 64 threads of
               // quarter q), by step parity: a warp reaches step it+2 only after every
               // elementwise thread has passed step it (S^T / dP^T of it+2 wait for that)
  kNumBars = 53
};
static_assert(8 * kNumBars + 8 + sizeof(WaitCtl) <= 512, "barrier area");

// DET: deterministic mode (det_order.cuh), a separate instance so that the default
// kernel carries none of its code.
template <bool DET>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(448, 1)
    sparse_bwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_dq,
                           const __grid_constant__ CUtensorMap tm_dk,
                           const __grid_constant__ CUtensorMap tm_dv, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * kNumBars);
  volatile WaitCtl* abort_flag =
      reinterpret_cast<volatile WaitCtl*>(smem + kOffBar + 8 * kNumBars + 8);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  // One cluster per (key tile, head).  Default: key tiles of one head run together
  // (they share that head's Q / dO in L2).  Deterministic mode: key tiles from the last
  // one down (det_order.cuh) with the heads interleaved, so that the key tiles that wait
  // for one another's dQ turns are spread out in time.
  const int cl = static_cast<int>(blockIdx.x) >> 1;
  const int ord = DET ? cl / a.HK : cl;
  const int nt = DET ? a.Tn - 1 - ord : ord;
  const int g = DET ? cl - ord * a.HK : static_cast<int>(blockIdx.y), b = blockIdx.z;
  const int G = a.HQ / a.HK;
  const int64_t bg = static_cast<int64_t>(b) * a.HK + g;
  const int64_t trow = bg * a.Tn + nt;
  const int n_full = __ldg(a.tcnt + 2 * trow);
  const int n_mt = n_full + __ldg(a.tcnt + 2 * trow + 1);
  const int32_t* tlist = a.tidx + trow * a.Tm;
  const int n_iter = G * n_mt * 2;  // (query head, query tile, 64-row half)
  const uint32_t off_stage = rank == 0 ? kOffStage0 : kOffStage1;
  const uint32_t off_l = rank == 0 ? kOffL0 : kOffL1;
  const uint32_t col_acc = rank == 0 ? kColAcc0 : kColAcc1;
  const int ns = rank == 0 ? kStages0 : kStages1;  // Q / dO stages of this rank
  int issued = 0;  // stage loads issued (the abort path drains the last ones)

  if (threadIdx.x == 0) {
    mbar_init(BAR(kBKV), 1);
    mbar_init(BAR(kBVT), 256);
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(BAR(kBQF + s), 1);
      mbar_init(BAR(kBQE + s), 1);
      mbar_init(BAR(kBLF + s), 32);
      mbar_init(BAR(kBSF + s), 1);
      mbar_init(BAR(kBEW + s), 256);
    }
    for (int s = 0; s < kNX; ++s) {
      mbar_init(BAR(kBXF + s), 1);
      mbar_init(BAR(kBXT + s), 1);
    }
    for (int s = 0; s < kNPI; ++s) {
      mbar_init(BAR(kBXE + s), 1);
      mbar_init(BAR(kBPR + s), 257);
    }
    for (int s = 0; s < kNDO; ++s) mbar_init(BAR(kBDF + s), 2);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(kBDQF + s), 1);
      mbar_init(BAR(kBDQE + s), 128);
    }
    mbar_init(BAR(kBSR), 256);
    for (int q = 0; q < 8; ++q) mbar_init(BAR(kBQH + q), 64);
    mbar_init(BAR(kBFin), 1);
    mbar_init(BAR(kBDrain), 1);
    abort_flag->abort = 0;
    abort_flag->peer_abort = 0;
    // the first exchange tiles may arrive from the peer at any time
    for (int s = 0; s < (rank == 0 ? kNX : kNPI) && s < n_iter; ++s)
      mbar_arrive_expect_tx(BAR(kBXF + s), kTile);
    fence_mbar_init();
    // K / V do not depend on the tile list: start their loads before the TMEM
    // allocation and the cluster handshake
    if (n_iter > 0) {
      if (rank == 0) {
        // K columns 0..127 stay in shared memory (the dQ^T operand); 128..255 land in
        // exchange tiles 0 and 1 until the elementwise warps have copied K into TMEM
        mbar_arrive_expect_tx(BAR(kBKV), 4 * kKPanel);
        for (int c = 0; c < 4; ++c)
          tma_load_4d(sbase + (c < 2 ? kOffK0 + c * kKPanel : kOffX0 + (c - 2) * kKPanel), &tm_k,
                      BAR(kBKV), c * 64, nt * 128, g, b);
      } else {
        mbar_arrive_expect_tx(BAR(kBKV), 6 * kKPanel);
        for (int c = 0; c < 4; ++c)
          tma_load_4d(sbase + kOffV1 + c * kKPanel, &tm_v, BAR(kBKV), c * 64, nt * 128, g, b);
        for (int c = 2; c < 4; ++c)
          tma_load_4d(sbase + kOffK1 + (c - 2) * kKPanel, &tm_k, BAR(kBKV), c * 64, nt * 128, g, b);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
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
    if constexpr (DET) {  // ascending query tiles (det_order.cuh)
      int tile;
      merged_tile(tlist, n_full, n_mt - n_full, k, tile, partial);
      m0 = tile * 128 + (rest & 1) * BM;
    } else {
      m0 = __ldg(tlist + k) * 128 + (rest & 1) * BM;
      partial = k >= n_full;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (n_iter > 0) {
      if (elect_one()) {
        prefetch_tensormap(rank == 0 ? &tm_q : &tm_do);
        prefetch_tensormap(&tm_dq);
      }
      __syncwarp();
      float* lbuf = reinterpret_cast<float*>(smem + off_l);
      const CUtensorMap* tm_stage = rank == 0 ? &tm_q : &tm_do;
      // rank 0: LSE in log2 units (+inf past Sq); rank 1: Delta (0 past Sq).  The values
      // of step it+1 are loaded while step it's stage is being waited for and loaded, so
      // that their latency stays off the issue path of the stage loads.
      auto load_rows = [&](int it_, float (&v)[2]) {
        int h_, m0_;
        bool partial_;
        decode(it_, h_, m0_, partial_);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int64_t i = m0_ + lane + 32 * k;
          v[k] = rank == 0 ? INFINITY : 0.f;
          if (i < a.Sq) {
            const int64_t li = (static_cast<int64_t>(b) * a.HQ + h_) * a.Sq + i;
            v[k] = rank == 0 ? __ldg(a.lse + li) * 1.4426950408889634f : __ldg(a.delta + li);
          }
        }
      };
      float rows[2];
      load_rows(0, rows);
      for (int it = 0; it < n_iter; ++it) {
        int h, m0;
        bool partial;
        decode(it, h, m0, partial);
        m0 = __shfl_sync(0xFFFFFFFFu, m0, 0);  // warp-uniform TMA coordinate
        const int s = it % ns, u = it / ns;
        if (!warp_wait(BAR(kBQE + s), (u & 1) ^ 1, abort_flag, a.status, a.wait_limit_ns)) break;
        // rank 1: V occupies stages 1 and 2 until it has been copied into TMEM
        if (rank == 1 && (it == 1 || it == 2) && !warp_wait(BAR(kBVT), 0, abort_flag, a.status, a.wait_limit_ns))
          break;
        const uint32_t qs = sbase + off_stage + s * kStageBytes;
        if (elect_one()) {
          mbar_arrive_expect_tx(BAR(kBQF + s), kStageBytes);
          for (int c = 0; c < 4; ++c) tma_load_4d(qs + c * kQPanel, tm_stage, BAR(kBQF + s), c * 64, m0, h, b);
        }
        __syncwarp();
        issued = it + 1;
        // rank 1 frees a stage when dV is done, which can precede the elementwise warps'
        // read of the step's Delta: wait for them before overwriting it
        if (rank == 1 && it >= ns &&
            !warp_wait(BAR(kBEW + s), ((it - ns) / ns) & 1, abort_flag, a.status, a.wait_limit_ns))
          break;
        float* ls = lbuf + s * BM;
        ls[lane] = rows[0];
        ls[lane + 32] = rows[1];
        mbar_arrive(BAR(kBLF + s));
        if (it + 1 < n_iter) load_rows(it + 1, rows);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (converged, warp-uniform decisions from lane 0);
    // one elected lane issues each batch of tcgen05 instructions.
    if (n_iter > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, BM, 0, 0);     // S^T / dP^T
      constexpr uint32_t idesc_acc = idesc_bf16(128, 256, 0, 1);  // dK / dV (tile K-major, stage MN-major)
      constexpr uint32_t idesc_dq = idesc_bf16(128, BM, 1, 1);    // dQ^T (both MN-major)
      // dQ^T A operand: this rank's 128 head-dim rows of K (MN-major)
      const uint64_t kwd = sw128_desc(sbase + (rank == 0 ? kOffK0 : kOffK1), kKPanel, 1024);
      auto ready = [&](int k, int parity) {
        return __shfl_sync(0xFFFFFFFFu, mbar_test(BAR(k), parity) ? 1 : 0, 0) != 0;
      };
      bool ok = warp_wait(BAR(kBKV), 0, abort_flag, a.status, a.wait_limit_ns);
      ok = ok && warp_wait(BAR(kBVT), 0, abort_flag, a.status, a.wait_limit_ns);
      int js = 0;  // next S^T (rank 0) / dP^T (rank 1)
      int jv = 0;  // rank 1: next dV
      int jk = 0;  // next dQ^T
      int jd = 0;  // rank 0: next dK (issued ahead of its dQ^T)
      int jx = 0;  // rank 0: next step whose dS^T arrival is reported back to rank 1
      int jp = 0;  // rank 1: next step whose P^T tile is handed back to rank 0
      uint64_t t_last = globaltimer_ns();
      while (ok && jk < n_iter) {
        bool prog = false;
        // rank 0: report each dS^T arrival at once and arm the barrier for the step that
        // uses the tile next
        if (rank == 0 && jx < js && ready(kBXF + jx % kNX, (jx / kNX) & 1)) {
          if (elect_one()) {
            mbar_arrive_remote_relaxed(mapa_shared(BAR(kBDF + jx % kNDO), peer));
            if (jx + kNX < n_iter) mbar_arrive_expect_tx(BAR(kBXF + jx % kNX), kTile);
          }
          __syncwarp();
          ++jx;
          prog = true;
        }
        // rank 1: hand a consumed P^T tile back to rank 0 (arm its barrier for the step
        // after next first)
        if (rank == 1 && jp < jv && ready(kBPR + jp % kNPI, (jp / kNPI) & 1)) {
          if (jp + kNPI < n_iter && elect_one()) {
            mbar_arrive_expect_tx(BAR(kBXF + jp % kNPI), kTile);
            mbar_arrive_remote_relaxed(mapa_shared(BAR(kBXE + jp % kNPI), peer));
          }
          __syncwarp();
          ++jp;
          prog = true;
        }
        // rank 1: dV += P^T dO as soon as P^T of the oldest step has arrived
        if (rank == 1 && jv < js && ready(kBXF + jv % kNPI, (jv / kNPI) & 1)) {
          tc_fence_after();
          const uint64_t xk = sw128_desc(sbase + kOffPI1 + (jv % kNPI) * kTile, 16, 1024);
          const uint64_t bmn = sw128_desc(sbase + off_stage + (jv % ns) * kStageBytes, kQPanel, 1024);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ss(tmem + col_acc, xk + ((kk * 32) >> 4), bmn + ((kk * 2048) >> 4), idesc_acc,
                      (jv > 0 || kk > 0) ? 1u : 0u);
            umma_commit(BAR(kBPR + jv % kNPI));  // P^T read by dV
            umma_commit(BAR(kBQE + jv % ns));    // dO stage free (dP^T read it earlier)
          }
          __syncwarp();
          ++jv;
          prog = true;
        }
        // rank 0: dK += dS^T Q as soon as dS^T has arrived (it frees the Q stage); it does
        // not wait for the single dQ^T buffer to be drained
        if (rank == 0 && jd < jx) {
          tc_fence_after();
          const uint32_t xt = sbase + kOffX0 + (jd % kNX) * kTile;
          const uint64_t xk = sw128_desc(xt, 16, 1024);  // exchange tile, K-major A
          const uint64_t bmn = sw128_desc(sbase + off_stage + (jd % ns) * kStageBytes, kQPanel, 1024);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              umma_ss(tmem + col_acc, xk + ((kk * 32) >> 4), bmn + ((kk * 2048) >> 4), idesc_acc,
                      (jd > 0 || kk > 0) ? 1u : 0u);
            umma_commit(BAR(kBQE + jd % ns));  // Q stage free
          }
          __syncwarp();
          ++jd;
          prog = true;
        }
        // dQ^T: rank 0 once its dK is issued (the tensor pipe runs in order, so that dK has
        // read the tile before the drain stages into it) and the last dQ^T has been
        // drained; rank 1 once its elementwise warps have written dS^T
        if (rank == 0 ? (jk < jd && (jk == 0 || ready(kBDQE, (jk - 1) & 1)))
                      : (jk < jv && ready(kBEW + jk % ns, (jk / ns) & 1))) {
          tc_fence_after();
          // rank 0: the dS^T that arrived in its tile; rank 1: its own dS^T tile
          const uint32_t xt = rank == 0 ? sbase + kOffX0 + (jk % kNX) * kTile
                                        : sbase + kOffDO1 + (jk % kNDO) * kTile;
          const uint64_t xmn = sw128_desc(xt, kKPanel, 1024);  // exchange tile, MN-major B
          const uint32_t dq_col = rank == 0 ? kColDQ0 : kColP1 + 64 * (jk & 1);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              umma_ss(tmem + dq_col, kwd + ((kk * 2048) >> 4), xmn + ((kk * 2048) >> 4), idesc_dq,
                      kk > 0 ? 1u : 0u);
            umma_commit(BAR(kBDQF + (rank == 0 ? 0 : (jk & 1))));
            if (rank == 1) umma_commit(BAR(kBDF + jk % kNDO));  // dS^T tile read by dQ^T
          }
          __syncwarp();
          ++jk;
          prog = true;
        }
        // S^T (rank 0) / dP^T (rank 1) of the next step: stage loaded, TMEM buffer free
        // (rank 0: loaded by the elementwise warps; rank 1: its dQ^T drained), not too far
        // ahead of the dK / dV stream
        if (js < n_iter && js <= (rank == 0 ? jd + kLookS0 : jv + kLookS1) &&
            ready(kBQF + js % ns, (js / ns) & 1) &&
            (rank == 0 ? (js == 0 || ready(kBSR, (js - 1) & 1))
                       : (js < 2 || ready(kBDQE + (js & 1), ((js - 2) >> 1) & 1)))) {
          tc_fence_after();
          const int s = js % ns;
          const uint64_t bd = sw128_desc(sbase + off_stage + s * kStageBytes, 16, 1024);
          // A = K (rank 0) / V (rank 1) from TMEM: 16 head-dim columns (8 TMEM columns)
          // per k-step
          const uint32_t d_col = rank == 0 ? kColS0 : kColP1 + 64 * (js & 1);
          const uint32_t a_col = rank == 0 ? kColK0 : kColV1;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
              const uint32_t off_b = (kk >> 2) * kQPanel + (kk & 3) * 32;
              umma_ts(tmem + d_col, tmem + a_col + kk * 8, bd + (off_b >> 4), idesc_s,
                      kk > 0 ? 1u : 0u);
            }
            umma_commit(BAR(kBSF + s));
          }
          __syncwarp();
          ++js;
          prog = true;
        }
        if (prog) {
          t_last = globaltimer_ns();
        } else {
          if (__shfl_sync(0xFFFFFFFFu, abort_flag->abort, 0) != 0) break;
          if (globaltimer_ns() - t_last > a.wait_limit_ns) {
            if (lane == 0) wait_timed_out(abort_flag, a.status);
            __syncwarp();
            break;
          }
          __nanosleep(32);
        }
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
    const float* lbuf = reinterpret_cast<const float*>(smem + off_l);
    const bool key_ok = j < a.Sk;
    bool ok = true;
    if (n_iter > 0) {
      // K (rank 0) / V (rank 1) row r into TMEM (row r in lane r, head dims 2e, 2e+1 in
      // column e): this half of the warps copies head dims [128 hc, 128 hc + 128) from
      // the swizzled panels
      const bool v_ok = __all_sync(0xFFFFFFFFu, mbar_wait(BAR(kBKV), 0, abort_flag, a.status, a.wait_limit_ns));
      if (v_ok) {
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
          const int p = 2 * hc + pl;
          const uint32_t panel = rank == 1 ? kOffV1 + p * kKPanel
                                           : (p < 2 ? kOffK0 + p * kKPanel : kOffX0 + (p - 2) * kKPanel);
          const uint8_t* prow = smem + panel + r * 128;
          uint32_t w[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 v = *reinterpret_cast<const uint4*>(prow + ((k ^ (r & 7)) << 4));
            w[4 * k] = v.x;
            w[4 * k + 1] = v.y;
            w[4 * k + 2] = v.z;
            w[4 * k + 3] = v.w;
          }
          tmem_st32(tl + (rank == 1 ? kColV1 : kColK0) + p * 32, w);
        }
        tmem_wait_st();
      }
      ok = v_ok;
      // rank 1: the producer reloads these stages with TMA next; rank 0: the exchange
      // tiles are written by bulk copies later
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(BAR(kBVT));
    }
    for (int it = 0; ok && it < n_iter; ++it) {
      int h, m0;
      bool partial;
      decode(it, h, m0, partial);
      const int s = it % ns, ph = (it / ns) & 1;
      const int xb = it % kNX, phx = (it / kNX) & 1;
      bool w_ok = mbar_wait(BAR(kBLF + s), ph, abort_flag, a.status, a.wait_limit_ns);
      w_ok = w_ok && mbar_wait(BAR(kBSF + s), ph, abort_flag, a.status, a.wait_limit_ns);
      if (rank == 0) {
        // own tile xb: the dQ drain of step it-4 is done with it
        if (it >= kNX)
          w_ok = w_ok && mbar_wait(BAR(kBXT + xb), phx ^ 1, abort_flag, a.status, a.wait_limit_ns);
      } else {
        w_ok = w_ok && mbar_wait(BAR(kBXF + it % kNPI), (it / kNPI) & 1, abort_flag,
                                 a.status, a.wait_limit_ns);  // P^T arrived
      }
      if (!__all_sync(0xFFFFFFFFu, w_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* ls = lbuf + s * BM + 32 * hc;
      // row r of the tile written (rank 0: own tile xb; rank 1: dS^T tile it % 3)
      const uint32_t row_off = (rank == 0 ? kOffX0 + xb * kTile : kOffDO1 + (it % kNDO) * kTile) +
                               r * 128;
      uint32_t s_u[32];
      tmem_ld32(tl + (rank == 0 ? kColS0 : kColP1 + 64 * (it & 1)) + 32 * hc, s_u);
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
            // lane L loads the presence word of query q0 + L over this warp's 32 key rows
            // (one word: key rows 32 quarter .. +31); a bit transpose across the warp
            // leaves in lane L the word of key row r over the 32 queries (the branch is
            // warp-uniform)
            const int w = nt * 4 + (r >> 5);
            const int64_t i = q0 + lane;
            const uint32_t word =
                (i < a.Sq && w < a.W) ? __ldg(a.bitmap + (bg * a.Sq + i) * a.W + w) : 0u;
            cm &= warp_transpose32(word, lane);
          }
        }
        tmem_wait_ld();
        // S^T is in registers: the buffer may take the next step's S^T
        tc_fence_before();
        mbar_arrive(BAR(kBSR));
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
        // P^T row (this half's 32 queries), 128-byte swizzled: 16-byte chunk c of row r
        // lives at chunk c ^ (r % 8)
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = hc * 4 + c4;
          *reinterpret_cast<uint4*>(smem + row_off + ((c ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(kBQH + (it & 1) * 4 + quarter));
        mbar_arrive(BAR(kBEW + s));
        // each quarter's 32 rows (4 KB) go to rank 1's P^T tile as soon as its two warps
        // have written them and that tile is free (rank 1 is done with step it-3 there):
        // four copies in flight instead of one
        if (hc == 0 && lane == 0 &&
            mbar_wait(BAR(kBQH + (it & 1) * 4 + quarter), (it >> 1) & 1, abort_flag, a.status, a.wait_limit_ns) &&
            (it < kNPI ||
             mbar_wait(BAR(kBXE + it % kNPI), ((it / kNPI) & 1) ^ 1, abort_flag, a.status, a.wait_limit_ns))) {
          bulk_copy_to_cluster(
              mapa_shared(sbase + kOffPI1 + (it % kNPI) * kTile + quarter * (kTile / 4), peer),
              sbase + kOffX0 + xb * kTile + quarter * (kTile / 4), kTile / 4,
              mapa_shared(BAR(kBXF + it % kNPI), peer));
        }
      } else {
        // P^T row (copied in by rank 0); once read, the tile may go back to rank 0
        const uint32_t pi_off = kOffPI1 + (it % kNPI) * kTile + r * 128;
        uint32_t pw[16];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = hc * 4 + c4;
          const uint4 v = *reinterpret_cast<const uint4*>(smem + pi_off + ((c ^ (r & 7)) << 4));
          pw[4 * c4] = v.x;
          pw[4 * c4 + 1] = v.y;
          pw[4 * c4 + 2] = v.z;
          pw[4 * c4 + 3] = v.w;
        }
        tmem_wait_ld();
        mbar_arrive(BAR(kBPR + it % kNPI));
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
        // dS^T tile it % 3: dQ^T of step it-3 has read it and its copy has landed in rank 0
        const bool df_ok =
            it < kNDO || mbar_wait(BAR(kBDF + it % kNDO), ((it / kNDO) & 1) ^ 1, abort_flag, a.status, a.wait_limit_ns);
        if (!__all_sync(0xFFFFFFFFu, df_ok)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = hc * 4 + c4;
          *reinterpret_cast<uint4*>(smem + row_off + ((c ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(kBQH + (it & 1) * 4 + quarter));
        mbar_arrive(BAR(kBEW + s));
        // each quarter's 32 rows of dS^T go to rank 0's tile xb as soon as they are in
        // (that tile held P^T of this step, which rank 1 has already received)
        if (hc == 0 && lane == 0 &&
            mbar_wait(BAR(kBQH + (it & 1) * 4 + quarter), (it >> 1) & 1, abort_flag, a.status, a.wait_limit_ns)) {
          bulk_copy_to_cluster(mapa_shared(sbase + kOffX0 + xb * kTile + quarter * (kTile / 4), peer),
                               sbase + kOffDO1 + (it % kNDO) * kTile + quarter * (kTile / 4),
                               kTile / 4, mapa_shared(BAR(kBXF + xb), peer));
        }
      }
    }
    // ----------------------------------------------------------- dK / dV epilogue
    bool have = n_iter > 0 && ok;
    if (have) {
      const bool w_ok = mbar_wait(BAR(kBFin), 0, abort_flag, a.status, a.wait_limit_ns);
      have = __all_sync(0xFFFFFFFFu, w_ok);
      tc_fence_after();
    }
    // rank 0 stores dK (times softmax_scale), rank 1 stores dV: the rows go to the idle
    // stages as four [128 keys][64 dims] 128-byte-swizzled panels (the output map's box)
    // and leave by four TMA stores, which drop rows past Sk
    const float sc = rank == 0 ? a.scale : 1.f;
    const uint32_t ep = off_stage;
    for (int c = 32 * hc; c < 256; c += 64) {
      uint32_t v[32];
      if (have) {
        tmem_ld32(tl + col_acc + c, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      uint32_t pq[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pq[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
      // columns [c, c+32) = 16-byte chunks (c % 64) / 8 .. +3 of row r in panel c / 64
      uint8_t* prow = smem + ep + (c >> 6) * kKPanel + r * 128;
      const int ch0 = (c & 63) >> 3;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<uint4*>(prow + (((ch0 + e) ^ (r & 7)) << 4)) =
            make_uint4(pq[4 * e], pq[4 * e + 1], pq[4 * e + 2], pq[4 * e + 3]);
    }
    fence_proxy_async_smem();
    named_bar_sync(2, 256);
    if (threadIdx.x == 64) {
      const CUtensorMap* om = rank == 0 ? &tm_dk : &tm_dv;
#pragma unroll
      for (int p = 0; p < 4; ++p) tma_store_4d(om, sbase + ep + p * kKPanel, p * 64, nt * 128, g, b);
      bulk_commit_group();
      bulk_wait_group_read0();  // the stages are read before the CTA may leave
    }
  } else {
    // ------------------------------------------------------------------ dQ drain
    // thread = head-dim row r of this rank's half; the 64 query columns are staged as
    // fp32 (rank 0: in the step's exchange tile, free once dQ^T has read it; rank 1: in
    // its staging buffer), 32 queries at a time, as [64-column panel][32 q][64 d] tiles
    // that bulk reduce-adds push into dQ_acc
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int dtid = threadIdx.x - 320;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int p = r >> 6;
    const int c0 = 128 * static_cast<int>(rank);
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      int h, m0;
      bool partial;
      decode(it, h, m0, partial);
      const int xb = it % kNX;
      const int qb = rank == 0 ? 0 : (it & 1);
      // the four drain warps leave together (they share named barrier 1 below)
      const bool w_ok = mbar_wait(BAR(kBDQF + qb), rank == 0 ? (it & 1) : ((it >> 1) & 1),
                                  abort_flag, a.status, a.wait_limit_ns);
      if (!named_bar_and(1, 128, w_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t q_u[BM];
      const uint32_t dq_col = rank == 0 ? kColDQ0 : kColP1 + 64 * (it & 1);
      tmem_ld32(tl + dq_col, q_u);
      tmem_ld32(tl + dq_col + 32, q_u + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(BAR(kBDQE + qb));
      const uint32_t soff = rank == 0 ? kOffX0 + xb * kTile : kOffDQ1;
      float* stage = reinterpret_cast<float*>(smem + soff);
      const uint32_t stage_s = sbase + soff;
      // deterministic mode: this CTA's turn on the query tile (its dQ column half) starts
      // at the first add of its first 64-row half and ends after the last add of its
      // second half
      const int mt = m0 >> 7, qhalf = (m0 >> 6) & 1;
      bool turn_ok = true;
      if (DET && qhalf == 0 && dtid == 0)
        turn_ok = det_wait_turn(det_slot(a, b, h, mt, static_cast<int>(rank)),
                                key_tile_rank(a, bg, mt, nt), abort_flag, a.status, a.wait_limit_ns);
      if (DET && !named_bar_and(1, 128, turn_ok)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        // the previous reduce (this step's first half; on rank 1 also the last step's
        // second half, which used the same staging buffer) must have read the buffer
        if (half == 1 || rank == 1) {
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
      if (DET && qhalf == 1 && dtid == 0) det_pass_turn(det_slot(a, b, h, mt, static_cast<int>(rank)));
      // rank 0: the tile is free once the reduces have read it
      if (rank == 0 && dtid == 0) {
        bulk_wait_group_read0();
        mbar_arrive(BAR(kBXT + xb));
      }
    }
    if (dtid == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  // This CTA's abort flag no longer changes: hand it to the peer (a store into the peer's
  // shared memory while both CTAs are certainly resident), then meet.
  if (threadIdx.x == 0)
    st_shared_cluster_u32(
        mapa_shared(smem_u32(const_cast<int*>(&abort_flag->peer_abort)), peer),
        static_cast<uint32_t>(abort_flag->abort));
  cluster_sync_all();  // past this point neither CTA issues a copy or an arrival to the other
  // Abort path, taken by both CTAs when either aborted (each reads both flags from its
  // own shared memory; neither changes any more).  A stage is reloaded only after the
  // MMAs that read its previous contents have completed, so at most the last `ns` stage
  // loads (and the K/V load) can still be in flight: wait for them and for every MMA this
  // CTA issued (time-limited waits).  Copies between the two CTAs issued before the barrier above may still be
  // landing, and nothing here can wait for them (they complete on the receiver's
  // barriers, whose phases an abort leaves unknown): both CTAs stay resident for 50 us,
  // against about a microsecond per copy, and meet once more before either leaves.
  const bool any_abort = abort_flag->abort != 0 || abort_flag->peer_abort != 0;
  if (any_abort) {
    if (warp == 0 && lane == 0 && n_iter > 0) {
      mbar_wait_limited(BAR(kBKV), 0);
      for (int it = max(0, issued - ns); it < issued; ++it)
        mbar_wait_limited(BAR(kBQF + it % ns), (it / ns) & 1);
    }
    if (warp == 1 && n_iter > 0) {
      tc_fence_after();
      if (elect_one()) {
        umma_commit(BAR(kBDrain));
        mbar_wait_limited(BAR(kBDrain), 0);
      }
      __syncwarp();
    }
    if (threadIdx.x == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 50000) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pairbwd

template <bool DET>
static int launch_bwd_pair_t(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  static PerDeviceOnce attr;
  const int rc = once_per_device(attr, [] {
    return cuda_error(cudaFuncSetAttribute(pairbwd::sparse_bwd_pair_kernel<DET>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           pairbwd::kSmem),
                      "pair backward smem attribute");
  });
  if (rc) return rc;
  const dim3 grid = DET ? dim3(a.Tn * 2 * a.HK, 1, a.B) : dim3(a.Tn * 2, a.HK, a.B);
  record_event(3, st);
  pairbwd::sparse_bwd_pair_kernel<DET><<<grid, pairbwd::kThreads, pairbwd::kSmem, st>>>(
      m.q, m.k, m.v, m.dout, m.dq_acc, m.dk, m.dv, a);
  record_event(4, st);
  return check_launch("pair backward kernel launch");
}

int launch_bwd_pair(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  return a.det ? launch_bwd_pair_t<true>(a, m, st) : launch_bwd_pair_t<false>(a, m, st);
}

}  // namespace sa
