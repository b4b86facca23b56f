// fwd.cu -- sparse attention forward on sm_100a: O and LSE.
//
// Operation: softmax attention over the allowed key set of each query (IndexSparse /
// BlockSparse attention, MagiAttention PR #334, Summary and section 2), computed as
// the online softmax over key tiles that the nvfp4-megamoe-kernel commit log spells
// out in its multi-row softmax notes: running max and running sum per row,
// un-normalised P = exp(s - max), accumulate P V, final O = acc / sum.
//
// B200 design: three forms of one kernel template, chosen per call (see
// sparse_attn_set_forward_form).
//
// One head per CTA (one CTA per 128-query tile of one (batch, query head)):
//   warp 0     TMA producer: Q once, then the K tiles of the ACTIVE key tiles only
//              (the forward list), 128-byte swizzled, double-buffered when shared
//              memory allows;
//   warp 6/10  TMA producer of the V tiles, so that a K load (which S waits for)
//              never queues behind a V load that waits for the previous P V;
//   warp 1     allocates 512 TMEM columns and issues the tcgen05 MMAs (one elected
//              lane per batch): S = Q K^T into one of two TMEM S buffers (so the next S is
//              computed while the softmax works on the current one), and
//              O += P V with P read from TMEM (A operand in tensor memory);
//   softmax    warps 2-5 in block and dense modes (a thread holds one query row, thread
//              = TMEM lane, all 128 columns); warps 2-9 in index mode, two per TMEM lane
//              quarter, each with half of every row (they exchange row maxima per tile
//              and row sums at the end through shared memory; one warp per SM
//              sub-partition was issue bound by the bitmap masks).  A thread tcgen05.ld's
//              its S columns, applies the element mask on partial tiles (range, causal,
//              64-block mask or index bitmap; index-mode inputs fetched a tile ahead),
//              updates the running max lazily (O is rescaled in TMEM only when the max
//              grows by more than 2^8), exponentiates with ex2 and writes bf16 P back over
//              the S buffer.  At the end it normalises O into the idle Q buffer (the output
//              map's swizzled box layout, sent by TMA tensor stores) and writes LSE (fp32,
//              natural log).
//   With Dqk <= 192 the softmax warps first copy Q into TMEM and S reads it from there,
//   so that only K comes from shared memory.
//   TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+Dv), Q [256+Dv, 256+Dv+Dqk/2).
//
// Two heads per CTA (QS2; GQA with an even group, Dqk <= 192, Dv <= 128): the query heads
// of one GQA group walk the same tile list, so heads 2j and 2j+1 of one query tile share a
// CTA, each with its own S buffer, O accumulator (TMEM: S_A, S_B, O_A, O_B), softmax
// warpgroup (warps 2-5 and 6-9, full rows) and barriers.  Warp 0 loads Q of both heads, K,
// and V one tile behind K.  Per key tile the MMA warp issues P V of head A, then head A's
// next S into the same buffer, then the same for head B, so that one head's softmax
// overlaps the other head's MMAs.  This form rescales O after writing P (ten warps cap
// registers at 168, and O columns must not be live beside the 128 S values).
//
// Two query tiles per CTA (QS2 == 2; Dqk, Dv <= 128, any group size): the same structure
// for query tiles 2u and 2u + 1 of one head, which share K and V but have lists of their
// own.  At the start warp 0 merges the two lists into their union in shared memory (the
// tiles full for both first), each entry flagged per tile as absent, partial or full;
// the CTA walks the union, and a tile's softmax masks out every key of a union entry
// that its own list lacks.  Where the lists agree (dense) or differ by the diagonal tile
// (causal) this adds no MMAs; where they share few tiles it costs up to twice the MMAs.
// Measured no faster than one head per CTA (see launch_fwd_dims), it is chosen
// explicitly only.
//
// CTA pair (CG2; GQA with an even group, Dv >= 128): two heads of one group (heads 2j and
// 2j+1, same query tile) run on a 2-CTA cluster whose MMAs are pair MMAs (tcgen05
// cta_group::2, M = 256: each CTA's 128 query rows).  The pair shares every K and V tile:
// each CTA loads and holds half of it (keys [64 r, 64 r + 64) of K, head-dim columns
// [Dv/2 r, Dv/2 r + Dv/2) of V, r = cluster rank), which halves the per-CTA copy volume and
// shared-memory operand reads of B.  The even CTA (the leader) issues every MMA; its
// commits arrive on the barriers of both CTAs; both CTAs' loads complete on the leader's
// full barriers; the odd CTA's softmax warps report P (and Q in TMEM) to the leader with
// one remote arrival per warp.  Softmax, masks, epilogue and LSE are per CTA, as in the
// one-head form.
// Every mbarrier wait is bounded; a timeout sets SA_ERR_TIMEOUT in the status word and
// the CTA leaves after releasing its tensor memory.
#include "sa_device.cuh"
#include "sa_kernels.h"
#include "sa_pair2.cuh"

namespace sa {

// Key tiles the two-query-tile form's union can hold (Sk up to 256K).
constexpr int kUnionMaxTiles = 2048;

// QS2: 0 one query tile of one head per CTA; 1 two heads of one GQA group (one query
// tile); 2 two consecutive query tiles of one head.  Both QS2 forms hold two units (A, B),
// each with its own Q tile, S buffer, O accumulator and softmax warpgroup.
template <int DQK, int DV, bool PAIRED, bool CG2, int QS2>
struct FwdCfg {
  static constexpr int kPanel = 128 * 128;  // one 64-column x 128-row swizzled panel
  static constexpr int kHeads = QS2 ? 2 : 1;  // Q tiles (units) per CTA
  // K rows and V columns one CTA holds per tile (a pair splits both in halves)
  static constexpr int kKRows = CG2 ? 64 : 128;
  static constexpr int kKPanel = kKRows * 128;  // one 64-column panel of K
  static constexpr int kVCols = CG2 ? DV / 2 : DV;
  static constexpr int kQBytes = 128 * DQK * 2;
  static constexpr int kKBytes = kKRows * DQK * 2;
  static constexpr int kVBytes = 128 * kVCols * 2;
  static constexpr int kKStages = QS2 ? 2 : CG2 ? (DQK == 256 ? 2 : 3) : (DQK == 256 ? 1 : 2);
  static constexpr int kVStages =
      QS2 ? (DQK == 192 ? 1 : 2) : CG2 ? (DV == 256 ? 2 : 3) : (DV == 256 ? 1 : 2);
  static constexpr int kQOff = 0;  // kHeads Q tiles
  static constexpr int kKOff = kQOff + kHeads * kQBytes;
  static constexpr int kVOff = kKOff + kKStages * kKBytes;
  static constexpr int kBarOff = kVOff + kVStages * kVBytes;
  // softmax exchange of the paired warps: row max [2 tile parities][2 column halves][128
  // rows] and row sum [2 halves][128 rows], fp32
  static constexpr int kXOff = kBarOff + 256;
  // two query tiles (QS2 == 2): the union of the two tiles' lists, built in shared memory
  // at the start: kUnionMax int32 entries, a byte per key tile, two int32 counts
  static constexpr int kUnionMax = kUnionMaxTiles;
  static constexpr int kUOff = kXOff + (PAIRED ? 3 * 1024 : 0);
  static constexpr int kUBytes = QS2 == 2 ? 5 * kUnionMax + 8 : 0;
  static constexpr int kSmem = kUOff + kUBytes + 1024;  // + alignment slack
  // softmax warps per TMEM lane quarter (PAIRED: two, each with half of every row)
  static constexpr int kHalves = PAIRED ? 2 : 1;
  static constexpr int kThreads = QS2 ? 320 : PAIRED ? 352 : 224;
  static constexpr int kVWarp = QS2 ? -1 : PAIRED ? 10 : 6;  // V producer (QS2: warp 0)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kOCol = 256;
  // Dqk <= 192: Q is held in TMEM after O (bf16 pairs) and S = Q K^T reads it from there,
  // so that only K is read from shared memory (an operand pair from shared memory costs
  // 8 KB per 64-cycle k-step, the whole port, before the TMA writes of K and V)
  static constexpr bool kQT = !QS2 && DQK <= 192;
  static constexpr uint32_t kColQ = kOCol + DV;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert(kOCol + DV <= kTmemCols, "tensor memory budget");
  static_assert(!kQT || kColQ + DQK / 2 <= kTmemCols, "tensor memory budget (Q)");
  static_assert(!CG2 || DV >= 128, "a CTA pair splits V into 64-column panels");
  static_assert(!QS2 || (!PAIRED && !CG2 && DQK <= 192), "two units per CTA: full rows, one CTA");
  static_assert(kOCol + kHeads * DV <= kTmemCols, "tensor memory budget (two heads)");
  static_assert(kKStages <= 4 && kVStages <= 4, "barrier slots");
};

// barrier slots (up to four K and four V stages; kBOD2 / kBOFin2: the second head's)
enum : int { kBQ = 0, kBKF = 1, kBKE = 5, kBVF = 9, kBVE = 13, kBSF = 17, kBPF = 19, kBOD = 21,
             kBDrain = 22, kBOFin = 23, kBQT = 24, kBOD2 = 25, kBOFin2 = 26, kNumBars = 27 };

// tm_kh: K in 64-row boxes (the half tile a CTA of a pair loads); unused by the
// single-CTA form.
template <int DQK, int DV, bool PAIRED, bool CG2, int QS2, bool PREFETCH>
__global__ void __launch_bounds__(QS2 ? 320 : PAIRED ? 352 : 224, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_kh,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const AttnArgs a) {
  using C = FwdCfg<DQK, DV, PAIRED, CG2, QS2>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * kNumBars);
  volatile WaitCtl* abort_flag =
      reinterpret_cast<volatile WaitCtl*>(smem + C::kBarOff + 8 * kNumBars + 8);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // pair: the two CTAs of a cluster are blockIdx.x = 2c, 2c + 1 (rank 0 leads)
  const uint32_t rank = CG2 ? cluster_ctarank() : 0u;
  const int xt = CG2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  // longest lists first under causal; two query tiles (kTiles): CTA xt holds tiles mt and
  // mt + 1 (the second one absent past the last tile)
  constexpr bool kTiles = QS2 == 2;
  const int mt = kTiles ? 2 * ((a.Tm + 1) / 2 - 1 - xt) : a.Tm - 1 - xt;
  // (two heads: h is the first of the CTA's two heads, h + 1 the second)
  const int h = (CG2 || QS2 == 1) ? 2 * static_cast<int>(blockIdx.y) + static_cast<int>(rank)
                                  : static_cast<int>(blockIdx.y);
  const int b = blockIdx.z;
  // the leader's barriers as seen from this CTA (remote arrivals and pair loads)
  const uint32_t lbar0 = CG2 ? mapa_shared(bar0, 0) : bar0;
  auto LBAR = [&](int k) { return lbar0 + 8u * static_cast<uint32_t>(k); };
  const int g = h / (a.HQ / a.HK);
  const int64_t bg = static_cast<int64_t>(b) * a.HK + g;
  const int64_t lrow = bg * a.Tm + mt;
  const int32_t* list = a.idx + lrow * a.Tn;
  // Two query tiles walk the union of their lists (uni), whose entries carry the key
  // tile (bits 0-27) and, per unit u, whether the tile is absent from (0), partial in (1)
  // or full in (2) that unit's own list (bits 28 + 2u, 29 + 2u); the entries full for both
  // come first.  n_iter is provisional until the union is built (it is > 0 exactly when
  // the union is not empty).
  const bool has_b = kTiles && mt + 1 < a.Tm;
  int32_t* uni = reinterpret_cast<int32_t*>(smem + C::kUOff);
  int n_full = __ldg(a.cnt + 2 * lrow);
  int n_iter = n_full + __ldg(a.cnt + 2 * lrow + 1);
  if (kTiles && has_b) n_iter += __ldg(a.cnt + 2 * lrow + 2) + __ldg(a.cnt + 2 * lrow + 3);
  auto entry_at = [&](int t) -> int { return kTiles ? uni[t] : __ldg(list + t); };
  auto tile_of = [](int e) -> int { return kTiles ? (e & 0x0FFFFFFF) : e; };
  // loads issued by the two producers (the abort path drains the last ones in flight)
  int issued_k = 0, issued_v = 0;

  // P / Q-in-TMEM ready: one arrival per softmax thread; in a pair, one per softmax
  // warp of either CTA on the leader's barrier
  constexpr uint32_t kReadyCount = CG2 ? 2 * 4 * C::kHalves : 128 * C::kHalves;
  if (threadIdx.x == 0) {
    mbar_init(BAR(kBQ), 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(BAR(kBKF + s), 1);
      mbar_init(BAR(kBKE + s), 1);
      mbar_init(BAR(kBVF + s), 1);
      mbar_init(BAR(kBVE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(kBSF + s), 1);
      mbar_init(BAR(kBPF + s), kReadyCount);
    }
    mbar_init(BAR(kBOD), 1);
    mbar_init(BAR(kBDrain), 1);
    mbar_init(BAR(kBOFin), 1);
    mbar_init(BAR(kBQT), kReadyCount);
    mbar_init(BAR(kBOD2), 1);
    mbar_init(BAR(kBOFin2), 1);
    abort_flag->abort = 0;
    abort_flag->peer_abort = 0;
    fence_mbar_init();
    if (kTiles && n_iter > 0) {
      // two query tiles: their Q loads start now, while warp 0 builds the union below
      // (past the last query tile, B's box lies beyond Sq and is zero-filled)
      fence_proxy_async_smem();
      prefetch_tensormap(&tm_q);
      mbar_arrive_expect_tx(BAR(kBQ), 2 * C::kQBytes);
      for (int u = 0; u < 2; ++u)
        for (int c = 0; c < DQK / 64; ++c)
          tma_load_4d(sbase + C::kQOff + u * C::kQBytes + c * C::kPanel, &tm_q, BAR(kBQ), c * 64,
                      (mt + u) * 128, h, b);
    }
  }
  if (kTiles && warp == 0) {
    // The union of the two query tiles' lists (each: full entries, then partial ones;
    // every key tile at most once).  cls[t] collects per key tile t: bit 2u + 1 full in
    // unit u's list, bit 2u partial in it.  Without a second tile, B takes A's flags.
    uint8_t* cls = smem + C::kUOff + 4 * C::kUnionMax;
    int32_t* cnts = reinterpret_cast<int32_t*>(cls + C::kUnionMax);
    const int tn = a.Tn;
    for (int t = lane; t < tn; t += 32) cls[t] = 0;
    __syncwarp();
    for (int u = 0; u < (has_b ? 2 : 1); ++u) {
      const int64_t lr = lrow + u;
      const int nf = __ldg(a.cnt + 2 * lr), nl = nf + __ldg(a.cnt + 2 * lr + 1);
      for (int e = lane; e < nl; e += 32) {
        const int t = __ldg(a.idx + lr * a.Tn + e);
        if (t >= 0 && t < tn) cls[t] |= static_cast<uint8_t>((e < nf ? 2 : 1) << (2 * u));
      }
      __syncwarp();
    }
    int n = 0, nfull = 0;
    for (int pass = 0; pass < 2; ++pass) {  // full for both, then the rest
      for (int t0 = 0; t0 < tn; t0 += 32) {
        const int t = t0 + lane;
        const uint32_t c = t < tn ? cls[t] : 0u;
        const uint32_t fa = c & 3u, fb = has_b ? (c >> 2) & 3u : fa;
        const bool both_full = fa == 2u && fb == 2u;
        const bool take = c != 0u && (pass == 0) == both_full;
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, take);
        if (take)
          uni[n + __popc(bal & ((1u << lane) - 1u))] =
              static_cast<int32_t>(static_cast<uint32_t>(t) | (fa << 28) | (fb << 30));
        n += __popc(bal);
      }
      if (pass == 0) nfull = n;
    }
    if (lane == 0) {
      cnts[0] = nfull;
      cnts[1] = n;
    }
  }
  if (warp == 1) {
    if constexpr (CG2) {
      tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CG2) cluster_sync_all();  // both CTAs' barriers exist before any remote use
  tc_fence_after();
  // broadcast from lane 0 so that the compiler can treat it as warp-uniform
  const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, *tmem_slot, 0);
  // (the Q loads above were issued on the provisional count)
  const bool q_issued = kTiles && n_iter > 0;
  if constexpr (kTiles) {
    const int32_t* cnts = reinterpret_cast<const int32_t*>(smem + C::kUOff + 5 * C::kUnionMax);
    n_full = cnts[0];
    n_iter = cnts[1];
  }

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // converged warp; one elected lane issues the copies
    if (n_iter > 0) {
      if (elect_one()) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        if (CG2 && !C::kQT) {
          // the leader's S MMAs read Q from both CTAs' shared memory: both Q loads
          // complete on the leader's barrier
          if (rank == 0) mbar_arrive_expect_tx(BAR(kBQ), 2 * C::kQBytes);
          for (int c = 0; c < DQK / 64; ++c)
            tma_load_4d_pair(sbase + C::kQOff + c * C::kPanel, &tm_q, LBAR(kBQ), c * 64, mt * 128,
                             h, b);
        } else if (!kTiles) {  // (two query tiles: loaded before the union was built)
          // (two heads: the tiles of heads h and h + 1, one after the other)
          mbar_arrive_expect_tx(BAR(kBQ), C::kHeads * C::kQBytes);
          for (int hd = 0; hd < C::kHeads; ++hd)
            for (int c = 0; c < DQK / 64; ++c)
              tma_load_4d(sbase + C::kQOff + hd * C::kQBytes + c * C::kPanel, &tm_q, BAR(kBQ),
                          c * 64, mt * 128, h + hd, b);
        }
      }
      __syncwarp();
      // key tile of list entry t (read by every lane, the same address)
      auto tile_at = [&](int t) -> int {
        if constexpr (kTiles) return tile_of(uni[t]);
        return __shfl_sync(0xFFFFFFFFu, __ldg(list + t), 0);
      };
      auto load_v = [&](int t) -> bool {  // V tile t (QS2)
        const int nt = tile_at(t);
        const int vs = t % C::kVStages, vu = t / C::kVStages;
        if (!warp_wait(BAR(kBVE + vs), (vu & 1) ^ 1, abort_flag, a.status, a.wait_limit_ns))
          return false;
        if (elect_one()) {
          mbar_arrive_expect_tx(BAR(kBVF + vs), C::kVBytes);
          for (int c = 0; c < DV / 64; ++c)
            tma_load_4d(sbase + C::kVOff + vs * C::kVBytes + c * C::kPanel, &tm_v, BAR(kBVF + vs),
                        c * 64, nt * 128, g, b);
        }
        __syncwarp();
        issued_v = t + 1;
        return true;
      };
      // K tiles: each one as soon as S of the tile that last used its buffer is done (V
      // tiles have a producer warp of their own, so a K load never waits behind P V)
      for (int it = 0; it < n_iter; ++it) {
        const int nt = tile_at(it);
        const int ks = it % C::kKStages, ku = it / C::kKStages;
        if (!warp_wait(BAR(kBKE + ks), (ku & 1) ^ 1, abort_flag, a.status, a.wait_limit_ns)) break;
        if (elect_one()) {
          if constexpr (CG2) {  // keys [64 rank, +64) of the tile, on the leader's barrier
            if (rank == 0) mbar_arrive_expect_tx(BAR(kBKF + ks), 2 * C::kKBytes);
            for (int c = 0; c < DQK / 64; ++c)
              tma_load_4d_pair(sbase + C::kKOff + ks * C::kKBytes + c * C::kKPanel, &tm_kh,
                               LBAR(kBKF + ks), c * 64, nt * 128 + 64 * static_cast<int>(rank), g, b);
          } else {
            mbar_arrive_expect_tx(BAR(kBKF + ks), C::kKBytes);
            for (int c = 0; c < DQK / 64; ++c)
              tma_load_4d(sbase + C::kKOff + ks * C::kKBytes + c * C::kPanel, &tm_k,
                          BAR(kBKF + ks), c * 64, nt * 128, g, b);
          }
        }
        __syncwarp();
        issued_k = it + 1;
        // QS2: V tiles from this warp too, one tile behind K (V(it-1) after K(it)): a K
        // stage frees when S of the second head is done, a V stage only when its P V is,
        // later in the tensor pipe's order, so K never waits behind a V stage
        if (QS2 && it > 0 && !load_v(it - 1)) break;
      }
      if (QS2 && issued_k == n_iter) load_v(n_iter - 1);
      // pair: the leader's commits arrive on this CTA's barriers too; wait for the ones
      // that free the last stages so that none is in flight when the CTA leaves
      if (CG2 && issued_k == n_iter)
        for (int it = n_iter; it < n_iter + C::kKStages; ++it)
          if (!warp_wait(BAR(kBKE + it % C::kKStages), ((it / C::kKStages) & 1) ^ 1, abort_flag,
                         a.status, a.wait_limit_ns))
            break;
    }
  } else if (warp == C::kVWarp) {
    // ------------------------------------------------------------------ V producer
    if (n_iter > 0) {
      for (int it = 0; it < n_iter; ++it) {
        const int nt = __shfl_sync(0xFFFFFFFFu, __ldg(list + it), 0);
        const int vs = it % C::kVStages, vu = it / C::kVStages;
        if (!warp_wait(BAR(kBVE + vs), (vu & 1) ^ 1, abort_flag, a.status, a.wait_limit_ns)) break;
        if (elect_one()) {
          if constexpr (CG2) {  // head-dim columns [Dv/2 rank, +Dv/2), on the leader's barrier
            if (rank == 0) mbar_arrive_expect_tx(BAR(kBVF + vs), 2 * C::kVBytes);
            for (int c = 0; c < C::kVCols / 64; ++c)
              tma_load_4d_pair(sbase + C::kVOff + vs * C::kVBytes + c * C::kPanel, &tm_v,
                               LBAR(kBVF + vs), static_cast<int>(rank) * C::kVCols + c * 64,
                               nt * 128, g, b);
          } else {
            mbar_arrive_expect_tx(BAR(kBVF + vs), C::kVBytes);
            for (int c = 0; c < DV / 64; ++c)
              tma_load_4d(sbase + C::kVOff + vs * C::kVBytes + c * C::kPanel, &tm_v,
                          BAR(kBVF + vs), c * 64, nt * 128, g, b);
          }
        }
        __syncwarp();
        issued_v = it + 1;
      }
      if (CG2 && issued_v == n_iter)
        for (int it = n_iter; it < n_iter + C::kVStages; ++it)
          if (!warp_wait(BAR(kBVE + it % C::kVStages), ((it / C::kVStages) & 1) ^ 1, abort_flag,
                         a.status, a.wait_limit_ns))
            break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (converged, warp-uniform operands); one elected
    // lane issues each batch of tcgen05 instructions.  In a pair only the leader issues
    // (M = 256: both CTAs' rows), and every commit arrives on both CTAs' barriers.
    if constexpr (QS2) {
      if (n_iter > 0) {
        // Two heads (A = h, B = h + 1): S_A(j), S_B(j) into each head's 128-column buffer,
        // P V into O_A, O_B.  Per key tile j: P V of head A once its P is ready, then
        // S_A(j+1) into the same buffer (the pipe runs in order, so P is read before it is
        // overwritten), then the same for head B.  While one head's softmax works on its S,
        // the tensor pipe runs the other head's MMAs.
        constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16(128, DV, 0, 1);
        bool ok = warp_wait(BAR(kBQ), 0, abort_flag, a.status, a.wait_limit_ns);
        auto issue_s2 = [&](int it, int hd) -> bool {
          const int ks = it % C::kKStages, ku = it / C::kKStages;
          if (hd == 0 && !warp_wait(BAR(kBKF + ks), ku & 1, abort_flag, a.status, a.wait_limit_ns))
            return false;
          tc_fence_after();
          const uint64_t kdesc = sw128_desc(sbase + C::kKOff + ks * C::kKBytes, 16, 1024);
          const uint64_t qd = sw128_desc(sbase + C::kQOff + hd * C::kQBytes, 16, 1024);
          const uint32_t d = tmem + static_cast<uint32_t>(hd * 128);
          if (elect_one()) {
  #pragma unroll
            for (int kk = 0; kk < DQK / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * C::kPanel + (kk & 3) * 32) >> 4;
              umma_ss(d, qd + off, kdesc + off, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(BAR(kBSF + hd));
            if (hd == 1) umma_commit(BAR(kBKE + ks));  // both heads have read the K tile
          }
          __syncwarp();
          return true;
        };
        auto issue_pv2 = [&](int it, int hd) -> bool {
          const int vs = it % C::kVStages, vu = it / C::kVStages;
          if (!warp_wait(BAR(kBPF + hd), it & 1, abort_flag, a.status, a.wait_limit_ns)) return false;
          if (hd == 0 && !warp_wait(BAR(kBVF + vs), vu & 1, abort_flag, a.status, a.wait_limit_ns))
            return false;
          tc_fence_after();
          const uint64_t vdesc = sw128_desc(sbase + C::kVOff + vs * C::kVBytes, C::kPanel, 1024);
          const uint32_t pa = tmem + static_cast<uint32_t>(hd * 128);
          if (elect_one()) {
  #pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              umma_ts(tmem + C::kOCol + hd * DV, pa + kk * 8, vdesc + ((kk * 2048) >> 4), idesc_pv,
                      (it > 0 || kk > 0) ? 1u : 0u);
            umma_commit(BAR(hd ? kBOD2 : kBOD));
            if (hd == 1) umma_commit(BAR(kBVE + vs));  // both heads have read the V tile
            if (it == n_iter - 1) umma_commit(BAR(hd ? kBOFin2 : kBOFin));
          }
          __syncwarp();
          return true;
        };
        if (ok) ok = issue_s2(0, 0) && issue_s2(0, 1);
        for (int it = 0; ok && it < n_iter; ++it)
          for (int hd = 0; ok && hd < 2; ++hd)
            ok = issue_pv2(it, hd) && (it + 1 >= n_iter || issue_s2(it + 1, hd));
      }
    } else {
      if (n_iter > 0 && rank == 0) {
        constexpr int kM = CG2 ? 256 : 128;
        constexpr uint32_t idesc_qk = idesc_bf16(kM, 128, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16(kM, DV, 0, 1);
        const uint64_t qdesc = sw128_desc(sbase + C::kQOff, 16, 1024);
        auto commit = [&](int bar) {
          if constexpr (CG2) umma_commit_pair(BAR(bar), 3);
          else umma_commit(BAR(bar));
        };
        // Q in TMEM (kQT): the softmax warps have copied it there
        bool ok = warp_wait(BAR(C::kQT ? kBQT : kBQ), 0, abort_flag, a.status, a.wait_limit_ns);
        auto issue_s = [&](int it) -> bool {
          const int ks = it % C::kKStages, ku = it / C::kKStages;
          if (!warp_wait(BAR(kBKF + ks), ku & 1, abort_flag, a.status, a.wait_limit_ns)) return false;
          tc_fence_after();
          const uint64_t kdesc = sw128_desc(sbase + C::kKOff + ks * C::kKBytes, 16, 1024);
          const uint32_t d = tmem + static_cast<uint32_t>((it & 1) * 128);
          if (elect_one()) {
  #pragma unroll
            for (int kk = 0; kk < DQK / 16; ++kk) {
              const uint32_t qoff = ((kk >> 2) * C::kPanel + (kk & 3) * 32) >> 4;
              const uint32_t koff = ((kk >> 2) * C::kKPanel + (kk & 3) * 32) >> 4;
              if constexpr (C::kQT) {  // A = Q from TMEM: 16 head dims = 8 columns per k-step
                if constexpr (CG2)
                  umma_ts_pair(d, tmem + C::kColQ + kk * 8, kdesc + koff, idesc_qk, kk > 0 ? 1u : 0u);
                else
                  umma_ts(d, tmem + C::kColQ + kk * 8, kdesc + koff, idesc_qk, kk > 0 ? 1u : 0u);
              } else {
                if constexpr (CG2)
                  umma_ss_pair(d, qdesc + qoff, kdesc + koff, idesc_qk, kk > 0 ? 1u : 0u);
                else
                  umma_ss(d, qdesc + qoff, kdesc + koff, idesc_qk, kk > 0 ? 1u : 0u);
              }
            }
            commit(kBSF + (it & 1));
            commit(kBKE + ks);
          }
          __syncwarp();
          return true;
        };
        if (ok) ok = issue_s(0);
        for (int it = 0; ok && it < n_iter; ++it) {
          if (it + 1 < n_iter && !issue_s(it + 1)) break;
          const int vs = it % C::kVStages, vu = it / C::kVStages;
          if (!warp_wait(BAR(kBPF + (it & 1)), (it >> 1) & 1, abort_flag, a.status, a.wait_limit_ns)) break;
          if (!warp_wait(BAR(kBVF + vs), vu & 1, abort_flag, a.status, a.wait_limit_ns)) break;
          tc_fence_after();
          const uint64_t vdesc = sw128_desc(sbase + C::kVOff + vs * C::kVBytes, C::kPanel, 1024);
          const uint32_t pa = tmem + static_cast<uint32_t>((it & 1) * 128);
          if (elect_one()) {
  #pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk) {
              if constexpr (CG2)
                umma_ts_pair(tmem + C::kOCol, pa + kk * 8, vdesc + ((kk * 2048) >> 4), idesc_pv,
                             (it > 0 || kk > 0) ? 1u : 0u);
              else
                umma_ts(tmem + C::kOCol, pa + kk * 8, vdesc + ((kk * 2048) >> 4), idesc_pv,
                        (it > 0 || kk > 0) ? 1u : 0u);
            }
            // (pair: no O-done arrival after the last P V, which nobody waits for: every
            // arrival on the other CTA's barriers is observed before it leaves)
            if (!CG2 || it < n_iter - 1) commit(kBOD);
            commit(kBVE + vs);
            if (it == n_iter - 1) commit(kBOFin);  // the final O is complete
          }
          __syncwarp();
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax
    // kHalves warps per TMEM lane quarter.  A thread holds one query row (thread = TMEM
    // lane) and 128 / kHalves of its columns.  PAIRED (index mode, whose partial-tile
    // masks make one warp per SM sub-partition issue bound): warp pair p (warps 2+p and
    // 6+p) splits every row's columns in halves (hc) and exchanges its row maxima per
    // tile (shared memory, double-buffered by tile parity, behind the pair's named
    // barrier) and its row sums at the end.  Every wait result is AND-ed over the pair
    // before either warp acts on it, so the two warps always take the same branch and
    // never leave one another waiting at the pair's barrier.
    constexpr int kH = C::kHalves;
    constexpr int kCols = 128 / kH;                  // S columns per thread
    constexpr int kOCols = DV / kH;                  // O columns rescaled / stored per thread
    const int quarter = warp & 3;
    const int hc = kH == 2 ? (warp - 2) >> 2 : 0;   // column part of this warp
    // QS2: warps 2-5 hold unit A, warps 6-9 unit B (head h + 1 of the same query tile, or
    // query tile mt + 1 of the same head), each with its own S buffer, O accumulator and
    // barriers
    const int hd = QS2 ? (warp - 2) >> 2 : 0;
    const int hh = QS2 == 1 ? h + hd : h;            // this warp's query head
    const int mtu = kTiles ? mt + hd : mt;           // and query tile
    const uint32_t ocol = C::kOCol + static_cast<uint32_t>(hd * DV);
    const int bar_od = hd ? kBOD2 : kBOD, bar_ofin = hd ? kBOFin2 : kBOFin;
    const int pair_bar = 1 + ((warp - 2) & 3);       // named barrier of a pair (64 threads)
    auto pair_all = [&](bool v) {                    // v: already uniform over the warp
      if constexpr (kH == 2) return named_bar_and(pair_bar, 64, v);
      return v;
    };
    const int r = quarter * 32 + lane;
    const int64_t i = static_cast<int64_t>(mtu) * 128 + r;
    const bool row_ok = i < a.Sq;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + C::kXOff);          // [2][2][128]
    float* xsum = reinterpret_cast<float*>(smem + C::kXOff + 2048);   // [2][128]
    float m_run = -INFINITY, l_run = 0.f;            // l_run: this thread's part of the sum
    bool ok = true;
    // Tell the MMA issuer that this warp's TMEM stores are done (the caller has waited
    // for them and fenced): per thread on this CTA's barrier, or in a pair per warp on
    // the leader's (a relaxed remote arrival: the stores have completed before it)
    auto ready = [&](int bar) {
      if constexpr (CG2) {
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(BAR(bar));
          else mbar_arrive_remote_relaxed(LBAR(bar));
        }
      } else {
        mbar_arrive(BAR(bar));
      }
    };
    if (C::kQT && n_iter > 0) {
      // Q row r into TMEM (row r in lane r, head dims 2e, 2e+1 in column e); the warps
      // of a quarter share the 64-column panels
      ok = pair_all(__all_sync(0xFFFFFFFFu, mbar_wait(BAR(kBQ), 0, abort_flag, a.status, a.wait_limit_ns)));
      if (ok) {
        for (int pnl = hc; pnl < DQK / 64; pnl += kH) {
          const uint8_t* prow = smem + C::kQOff + pnl * C::kPanel + r * 128;
          uint32_t w[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 v = *reinterpret_cast<const uint4*>(prow + ((k ^ (r & 7)) << 4));
            w[4 * k] = v.x;
            w[4 * k + 1] = v.y;
            w[4 * k + 2] = v.z;
            w[4 * k + 3] = v.w;
          }
          tmem_st32(tl + C::kColQ + pnl * 32, w);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      ready(kBQT);
    }
    // Partial-tile mask inputs come from global memory (the tile list, the 64-block mask
    // bytes, the row's presence words).  In index mode every tile is partial, and they
    // are fetched ahead, before the wait for S, so that their latency overlaps the work
    // of earlier tiles: the list entry two tiles ahead, the presence words one tile ahead
    // (with the list entry fetched the iteration before): index forward 3.29 -> 3.16 ms.
    // Block and dense modes mask only the diagonal tile (or a ragged edge); there the
    // loads stay inline, because the prefetch's per-tile instructions cost the issue-bound
    // softmax warp more than it saves (+3 to +4% measured).
    constexpr bool kPrefetch = PREFETCH;  // the index-mode instances
    constexpr int kWords = kCols / 32;
    auto fetch_nt = [&](int t) {  // a list entry (two query tiles: with its flags)
      return (kPrefetch && t < n_iter && t >= n_full) ? entry_at(t) : 0;
    };
    // the mask inputs of key tile nt for this thread's row and columns
    auto load_mask = [&](int nt, uint32_t (&wd)[kWords], bool& m0, bool& m1) {
      if (!row_ok) return;
      if (a.mode == SA_MODE_BLOCK && a.bs == 64) {
        const uint8_t* mrow = a.mask + (bg * a.Mb + i / 64) * a.Nb;
        const int c0 = nt * 2;
        m0 = __ldg(mrow + c0) != 0;
        m1 = (c0 + 1 < a.Nb) ? (__ldg(mrow + c0 + 1) != 0) : false;
      } else if (a.mode == SA_MODE_INDEX) {
        const uint32_t* brow = a.bitmap + (bg * a.Sq + i) * a.W;
        const int w0 = nt * 4 + kWords * hc;
#pragma unroll
        for (int k = 0; k < kWords; ++k) wd[k] = (w0 + k < a.W) ? __ldg(brow + w0 + k) : 0u;
      }
    };
    // prefetch form: tile t's inputs, or "allow all" for a full tile
    auto fetch_mask = [&](int t, int nt, uint32_t (&wd)[kWords], bool& m0, bool& m1) {
      m0 = m1 = true;
#pragma unroll
      for (int k = 0; k < kWords; ++k) wd[k] = ~0u;
      if (kPrefetch && t < n_iter && t >= n_full) load_mask(tile_of(nt), wd, m0, m1);
    };
    int nt_cur = fetch_nt(0), nt_nxt = fetch_nt(1);
    uint32_t wd_cur[kWords];
    bool m0_cur, m1_cur;
    fetch_mask(0, nt_cur, wd_cur, m0_cur, m1_cur);
    for (int it = 0; ok && it < n_iter; ++it) {
      // S / P buffer of this tile and the parity of its S-ready phase (QS2: the head's
      // single buffer, one phase per tile)
      const int sb = QS2 ? hd : (it & 1);
      const uint32_t s_par = QS2 ? (it & 1) : ((it >> 1) & 1);
      const int nt_nn = fetch_nt(it + 2);
      uint32_t wd_nxt[kWords];
      bool m0_nxt, m1_nxt;
      fetch_mask(it + 1, nt_nxt, wd_nxt, m0_nxt, m1_nxt);
      const bool w_ok = __all_sync(
          0xFFFFFFFFu, mbar_wait(BAR(kBSF + sb), s_par, abort_flag, a.status, a.wait_limit_ns));
      if (!pair_all(w_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t u[kCols];
#pragma unroll
      for (int j = 0; j < kCols / 32; ++j) tmem_ld32(tl + sb * 128 + kCols * hc + 32 * j, u + 32 * j);
      tmem_wait_ld();
      float x[kCols];
#pragma unroll
      for (int c = 0; c < kCols; ++c) x[c] = __uint_as_float(u[c]);
      if (it >= n_full) {
        // partial tile: element mask (tile columns kCols hc + c)
        const int ent = kPrefetch ? nt_cur : entry_at(it);
        const int nt = tile_of(ent);
        const int64_t n0 = static_cast<int64_t>(nt) * 128;
        int64_t lim = a.Sk;
        if (a.causal) lim = min64(lim, i + 1);
        const int lim_c = static_cast<int>(max64(0, min64(128, lim - n0))) - kCols * hc;
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          if (c >= lim_c) x[c] = -INFINITY;
        if (!kPrefetch) load_mask(nt, wd_cur, m0_cur, m1_cur);
        if (row_ok && a.mode == SA_MODE_BLOCK && a.bs == 64) {
#pragma unroll
          for (int c = 0; c < kCols; ++c)
            if (!(((kCols * hc + c) < 64) ? m0_cur : m1_cur)) x[c] = -INFINITY;
        } else if (row_ok && a.mode == SA_MODE_INDEX) {
#pragma unroll
          for (int c = 0; c < kCols; ++c)
            if (!((wd_cur[c >> 5] >> (c & 31)) & 1u)) x[c] = -INFINITY;
        }
        // two query tiles: a tile of the union that this unit's own list lacks
        if (kTiles && ((static_cast<uint32_t>(ent) >> (28 + 2 * hd)) & 3u) == 0u) {
#pragma unroll
          for (int c = 0; c < kCols; ++c) x[c] = -INFINITY;
        }
      }
      nt_cur = nt_nxt;
      nt_nxt = nt_nn;
#pragma unroll
      for (int k = 0; k < kWords; ++k) wd_cur[k] = wd_nxt[k];
      m0_cur = m0_nxt;
      m1_cur = m1_nxt;
      // row max over eight independent chains (a single chain of dependent fmaxf is
      // latency bound), then the pair's
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = x[k];
#pragma unroll
      for (int c = 8; c < kCols; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], x[c]);
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      if constexpr (kH == 2) {
        float* xm = xmax + sb * 256;
        xm[hc * 128 + r] = mx;
        // both halves have loaded their S columns past this barrier, so P may now be
        // written over them
        named_bar_sync(pair_bar, 64);
        mx = fmaxf(xm[r], xm[128 + r]);
      }
      const float m_tile = mx * a.scale_log2;
      // Lazy rescale: only when this row's max grows by more than 2^8; the decision is
      // taken per warp (the warps of a pair hold the same rows and decide alike) so that
      // the warp-collective TMEM accesses stay converged.
      const bool need = m_tile > m_run + 8.0f;
      const bool any_need = __any_sync(0xFFFFFFFFu, need);
      const float alpha = need ? ex2(m_run - m_tile) : 1.f;  // 0 when m_run = -inf
      // O holds P V up to tile it-1: rescale this thread's O columns in TMEM once that MMA
      // is done (false: a wait gave up)
      auto rescale_o = [&]() -> bool {
        const bool o_ok = __all_sync(
            0xFFFFFFFFu, mbar_wait(BAR(bar_od), (it - 1) & 1, abort_flag, a.status, a.wait_limit_ns));
        if (!pair_all(o_ok)) return false;
        tc_fence_after();
#pragma unroll 1
        for (int c = hc * kOCols; c < (hc + 1) * kOCols; c += 32) {
          uint32_t ov[32];
          tmem_ld32(tl + ocol + c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(tl + ocol + c, ov);
        }
        return true;
      };
      // QS2 rescales after P is written (still before P V of this tile, which waits for
      // the P-ready arrival below): the 32 O columns then never share registers with the
      // 128 S values, and the wait for P V of tile it-1 overlaps the exponentials
      constexpr bool kLateRescale = QS2;
      if (any_need) {
        if (!kLateRescale && it > 0) {
          if (!rescale_o()) {
            ok = false;
            break;
          }
          tmem_wait_st();
        }
        if (need) {
          l_run *= alpha;
          m_run = m_tile;
        }
      }
      const float m_eff = (m_run == -INFINITY) ? 0.f : m_run;
      const float sc = a.scale_log2;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
#pragma unroll
      for (int c0 = 0; c0 < kCols; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(fmaf(x[c0 + 2 * e], sc, -m_eff));
          const float p1 = ex2(fmaf(x[c0 + 2 * e + 1], sc, -m_eff));
          ps[e & 3] += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        // bf16 P of tile columns [kCols hc + c0, +32) over the S buffer
        tmem_st16(tl + sb * 128 + (kCols / 2) * hc + c0 / 2, pk);
      }
      l_run += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      if (kLateRescale && any_need && it > 0 && !rescale_o()) {
        ok = false;
        break;
      }
      tmem_wait_st();
      tc_fence_before();
      ready(kBPF + sb);
    }
    // ---------------------------------------------------------------- epilogue
    if (n_iter > 0 && ok) {
      const bool w_ok = __all_sync(
          0xFFFFFFFFu, mbar_wait(BAR(bar_ofin), 0, abort_flag, a.status, a.wait_limit_ns));
      ok = pair_all(w_ok);
      tc_fence_after();
    }
    const bool have_o = n_iter > 0 && ok;  // the same on both warps of a pair
    float l_row = l_run;
    if constexpr (kH == 2) {  // the row sum is the sum of the two halves'
      xsum[hc * 128 + r] = l_run;
      named_bar_sync(pair_bar, 64);
      l_row = xsum[r] + xsum[128 + r];
    }
    const float inv = (l_row > 0.f) ? 1.f / l_row : 0.f;
    // O rows go to the Q buffer (idle once the last P V is done: every S MMA came
    // before it) as [128 rows][64 cols] 128-byte-swizzled panels, the output map's box,
    // and leave by TMA stores, which drop rows past Sq; each thread writes its columns
#pragma unroll 1
    for (int c = hc * kOCols; c < (hc + 1) * kOCols; c += 32) {
      uint32_t ov[32];
      if (have_o) {
        tmem_ld32(tl + ocol + c, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
      // columns [c, c+32) = 16-byte chunks (c % 64) / 8 .. +3 of row r in panel c / 64
      uint8_t* prow = smem + C::kQOff + hd * C::kQBytes + (c >> 6) * C::kPanel + r * 128;
      const int ch0 = (c & 63) >> 3;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<uint4*>(prow + (((ch0 + e) ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
    }
    fence_proxy_async_smem();
    named_bar_sync(5 + hd, 128 * kH);  // every softmax warp (of this head)
    // (no store for a second query tile past the last one)
    if (threadIdx.x == 64 + 128 * hd && static_cast<int64_t>(mtu) * 128 < a.Sq) {
#pragma unroll
      for (int p = 0; p < DV / 64; ++p)
        tma_store_4d(&tm_o, sbase + C::kQOff + hd * C::kQBytes + p * C::kPanel, p * 64, mtu * 128,
                     hh, b);
      bulk_commit_group();
      bulk_wait_group_read0();  // the Q buffer is read before the CTA may leave
    }
    if (row_ok && hc == 0) {
      const float m_eff = (m_run == -INFINITY) ? 0.f : m_run;
      a.lse[(static_cast<int64_t>(b) * a.HQ + hh) * a.Sq + i] =
          (l_row > 0.f) ? (m_eff + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  bool any_abort = abort_flag->abort != 0;
  if constexpr (CG2) {
    // This CTA's abort flag no longer changes: hand it to the peer (a store into the
    // peer's shared memory while both CTAs are certainly resident), then meet.  Past the
    // meeting neither CTA issues an MMA, a copy or an arrival to the other, and neither
    // touches the pair's tensor memory: in the normal path every commit, remote arrival
    // and load of the pair has been observed by a wait of its receiver.
    if (threadIdx.x == 0)
      st_shared_cluster_u32(
          mapa_shared(smem_u32(const_cast<int*>(&abort_flag->peer_abort)), rank ^ 1u),
          static_cast<uint32_t>(abort_flag->abort));
    cluster_sync_all();
    any_abort = abort_flag->abort != 0 || abort_flag->peer_abort != 0;
  }
  // Abort path.  Past the barrier above no warp issues another copy or MMA, and the
  // abort flags no longer change (the branch is uniform).  A K or V buffer is reloaded
  // only after the MMA that read its previous tile has completed, so at most the last
  // kKStages K loads and kVStages V loads can still be in flight: wait for them, and for
  // every MMA this CTA issued, before shared memory and TMEM are released
  // (time-limited waits).  A pair's loads complete on the leader's barriers, whose
  // phases an abort leaves unknown: there both CTAs wait for the leader's MMAs, stay
  // resident for 50 us (against a few microseconds per load) and meet once more.
  if (any_abort) {
    if (n_iter > 0 && lane == 0) {
      if constexpr (CG2) {
        if (warp == 0 && (C::kQT || rank == 0)) mbar_wait_limited(BAR(kBQ), 0);
      } else if (warp == 0) {
        mbar_wait_limited(BAR(kBQ), 0);
        for (int it = max(0, issued_k - C::kKStages); it < issued_k; ++it)
          mbar_wait_limited(BAR(kBKF + it % C::kKStages), (it / C::kKStages) & 1);
        if constexpr (QS2)  // this warp loads V too
          for (int it = max(0, issued_v - C::kVStages); it < issued_v; ++it)
            mbar_wait_limited(BAR(kBVF + it % C::kVStages), (it / C::kVStages) & 1);
      } else if (warp == C::kVWarp) {
        for (int it = max(0, issued_v - C::kVStages); it < issued_v; ++it)
          mbar_wait_limited(BAR(kBVF + it % C::kVStages), (it / C::kVStages) & 1);
      }
    }
    if (warp == 1 && n_iter > 0 && rank == 0) {
      tc_fence_after();
      if (elect_one()) {
        if constexpr (CG2) umma_commit_pair(BAR(kBDrain), 1);  // this CTA's barrier only
        else umma_commit(BAR(kBDrain));
        mbar_wait_limited(BAR(kBDrain), 0);
      }
      __syncwarp();
    }
    if (CG2 && threadIdx.x == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 50000) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (CG2) cluster_sync_all();
  }
  // two query tiles whose lists held no valid key tile: nothing waited for their Q loads
  if (q_issued && n_iter == 0 && threadIdx.x == 0) mbar_wait_limited(BAR(kBQ), 0);
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG2) tmem_dealloc_pair(tmem, C::kTmemCols);
    else tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int DQK, int DV, bool PAIRED, bool CG2, int QS2, bool PREFETCH>
static int launch_fwd_t(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  using C = FwdCfg<DQK, DV, PAIRED, CG2, QS2>;
  auto kern = sparse_fwd_kernel<DQK, DV, PAIRED, CG2, QS2, PREFETCH>;
  static PerDeviceOnce attr;
  const int rc = once_per_device(attr, [&] {
    return cuda_error(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           C::kSmem),
                      "forward smem attribute");
  });
  if (rc) return rc;
  record_event(0, st);
  if constexpr (CG2) {
    // one 2-CTA cluster per (query tile, pair of query heads of one GQA group)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * a.Tm, a.HQ / 2, a.B);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, m.q, m.k, m.kh, m.v, m.o, a);
    record_event(1, st);
    return cuda_error(e, "forward (CTA pair) kernel launch");
  } else {
    // two heads: one CTA per pair of heads; two query tiles: per pair of query tiles
    dim3 grid(QS2 == 2 ? (a.Tm + 1) / 2 : a.Tm, QS2 == 1 ? a.HQ / 2 : a.HQ, a.B);
    kern<<<grid, C::kThreads, C::kSmem, st>>>(m.q, m.k, m.kh, m.v, m.o, a);
    record_event(1, st);
    return check_launch("forward kernel launch");
  }
}

// Forms (see sparse_attn_set_forward_form):
//   one head per CTA: index mode pairs the softmax warps (its partial-tile bitmap masks
//     make one softmax warp per SM sub-partition issue bound) and fetches the masks ahead;
//     block and dense modes keep one warp per quarter (measured faster);
//   CTA pair (GQA, even group, Dv >= 128): two heads on a 2-CTA cluster sharing each K/V
//     tile through cta_group::2 MMAs; the default at head dims 256, where one CTA's
//     forward waits on its single K and V stages;
//   two heads per CTA (GQA, even group, Dqk <= 192, Dv <= 128): S and O of both heads in
//     TMEM, one softmax warpgroup per head, so that one head's softmax overlaps the
//     other head's MMAs; the default there (forward 0.420 -> 0.368 ms on the D=128 GQA
//     workload, 3.143 -> 2.786 ms on the 192/128 index workload);
//   two query tiles per CTA (Dqk, Dv <= 128, at most 2048 key tiles): the same
//     structure for query tiles 2u and 2u + 1 of one head, walking the union of their
//     lists; chosen explicitly only.  On dense D=128 lists it measured no faster than
//     one head per CTA even with many waves (S=16384: causal 1.984 -> 2.085 ms, full
//     3.776 -> 3.75-3.84), and slower where halving the CTA count leaves a partial last
//     wave (S=4096: full 0.2705 -> 0.293, causal 0.180 -> 0.197): with two S and two O
//     buffers TMEM has no room for Q, so its S MMAs read both operands from shared
//     memory, the port the one-head form keeps half free.  On lists that share few
//     tiles the union costs up to twice the tensor work (random 25% block mask at
//     S=8192: 0.418 -> 0.727 ms).
template <int DQK, int DV>
static int launch_fwd_dims(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  constexpr bool kPairable = DV >= 128;
  constexpr bool kTwoHeadsOk = DV <= 128 && DQK <= 192;
  constexpr bool kTwoTilesOk = DV <= 128 && DQK <= 128;
  const bool even = (a.HQ / a.HK) % 2 == 0;
  const bool index = a.mode == SA_MODE_INDEX;
  const bool tiles_fit = a.Tn <= kUnionMaxTiles;
  int form = g_fwd_form.load(std::memory_order_relaxed);
  if (form == SA_FWD_FORM_AUTO)
    form = !even ? SA_FWD_FORM_ONE_HEAD
           : kPairable && !kTwoHeadsOk ? SA_FWD_FORM_CTA_PAIR
                                       : SA_FWD_FORM_TWO_HEADS;
  if (form == SA_FWD_FORM_CTA_PAIR && !(kPairable && even)) form = SA_FWD_FORM_ONE_HEAD;
  if (form == SA_FWD_FORM_TWO_HEADS && !(kTwoHeadsOk && even)) form = SA_FWD_FORM_ONE_HEAD;
  if (form == SA_FWD_FORM_TWO_TILES && !(kTwoTilesOk && tiles_fit)) form = SA_FWD_FORM_ONE_HEAD;
  if (form == SA_FWD_FORM_CTA_PAIR) {
    if constexpr (kPairable)
      return index ? launch_fwd_t<DQK, DV, true, true, 0, true>(a, m, st)
                   : launch_fwd_t<DQK, DV, false, true, 0, false>(a, m, st);
  }
  if (form == SA_FWD_FORM_TWO_HEADS) {
    if constexpr (kTwoHeadsOk)
      return index ? launch_fwd_t<DQK, DV, false, false, 1, true>(a, m, st)
                   : launch_fwd_t<DQK, DV, false, false, 1, false>(a, m, st);
  }
  if (form == SA_FWD_FORM_TWO_TILES) {
    if constexpr (kTwoTilesOk)
      return index ? launch_fwd_t<DQK, DV, false, false, 2, true>(a, m, st)
                   : launch_fwd_t<DQK, DV, false, false, 2, false>(a, m, st);
  }
  return index ? launch_fwd_t<DQK, DV, true, false, 0, true>(a, m, st)
               : launch_fwd_t<DQK, DV, false, false, 0, false>(a, m, st);
}

int launch_fwd(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  if (a.Dqk == 64 && a.Dv == 64) return launch_fwd_dims<64, 64>(a, m, st);
  if (a.Dqk == 128 && a.Dv == 128) return launch_fwd_dims<128, 128>(a, m, st);
  if (a.Dqk == 192 && a.Dv == 128) return launch_fwd_dims<192, 128>(a, m, st);
  if (a.Dqk == 256 && a.Dv == 256) return launch_fwd_dims<256, 256>(a, m, st);
  return SA_ERR_UNSUPPORTED;
}

}  // namespace sa
