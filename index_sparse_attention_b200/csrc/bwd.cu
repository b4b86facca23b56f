// bwd.cu -- sparse attention backward on sm_100a: dQ, dK, dV.
//
// Operation (MagiAttention PR #334, Summary and section 1): recompute P from the
// saved LSE, then dV += P^T dO, dP = dO V^T, dS = P * (dP - Delta), dQ += dS K,
// dK += dS^T Q, with Delta = rowsum(dO * O) from a preprocess kernel and a
// postprocess that multiplies the fp32 dQ accumulator by softmax_scale and casts
// (section 3: fp32 accumulation, then dtype conversion and softmax_scale scaling).
//
// B200 design.  The pages' two loop orders put either dQ or dK/dV in tensor memory.
// Here the key tile is stationary (the transposed, key-to-query lists of MagiAttention
// PR #331 "CSR Tile Mapping"): one CTA owns 128 keys of one (batch, KV head) and walks
// every query tile that attends to them, for every query head of the GQA group, so
// dK and dV accumulate in TMEM across the whole group and are stored once, with no
// atomics.  Query tiles are consumed in 64-row halves so that K, V, a double-buffered
// Q/dO half-tile and the dS^T staging tile fit in shared memory for every head dim.
// For each 64-query half:
//   S^T  = K Q^T      (M=128 keys, N=64)            -> TMEM  [SS]
//   dP^T = V dO^T     (M=128 keys, N=64)            -> TMEM  [SS]
//   elementwise warps: P^T = exp2(S^T*scale*log2e - LSE*log2e), dS^T = P^T (dP^T - Delta),
//     element mask on partial tiles; bf16 P^T and dS^T written back into TMEM (A
//     operands of the next two MMAs) and dS^T into shared memory (operand of dQ^T)
//   dV  += P^T dO     (M=128 keys, N=Dv chunk)      TMEM A operand   [TS]
//   dK  += dS^T Q     (M=128 keys, N=Dqk chunk)     TMEM A operand   [TS]
//   dQ^T = K^T dS^T   (M=128 head-dim window, N=64) both MN-major    [SS]
//   a drain warpgroup reads dQ^T from TMEM, stages it as fp32 tiles in the consumed
//   dS^T buffer and adds them into the dQ accumulator with TMA bulk tensor
//   reduce-adds.
// Element masks of partial tiles: causal and range by arithmetic, 64-wide blocks from
// the block mask, index mode from the presence bitmap (one word per lane and a warp
// bit transpose give each key row its 32-query word).  dK (scaled by softmax_scale)
// and dV leave through the idle stages by TMA tensor stores.
// Head dims (192,128) also run on one CTA per key tile, with a single S^T and a single
// dP^T buffer: dK (192 columns), dV (128) and V (64, the TMEM operand of dP^T) leave 128
// of the 512 TMEM columns.  The next step's S^T / dP^T then follow this step's dQ^T,
// which comes in two 128-row windows: head dims 0-127 into the consumed S^T buffer (the
// drain warps read it on its own commit), 64-191 into the consumed dP^T buffer (the
// elementwise warps of lane quarters 2 and 3 read its rows 64-127, head dims 128-191,
// and reduce-add them).  Measured on the index workload against a head-dim split over
// two CTAs that both recompute S^T and dP^T: backward main 13.11 -> 11.78 ms.  The
// deterministic mode keeps that split (its dQ turns assume one reduce issuer per CTA).
// Head dims 256/256 run on a 2-CTA cluster that splits the work by role (bwd_pair.cu).
// Every mbarrier wait is bounded (see sa_device.cuh).
#include "det_order.cuh"
#include "sa_device.cuh"
#include "sa_kernels.h"

#include <cstdio>
#include <cstdlib>

namespace sa {

// Backward form at head dims (192,128) (SA_BWD_FORM_*, set by sparse_attn_set_backward_form).
extern std::atomic<int> g_bwd_form;

// ------------------------------------------------------------------------------------
// preprocess: Delta = rowsum(dO * O) (fp32) and a zeroed dQ accumulator
// ------------------------------------------------------------------------------------
__global__ void bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                               const __nv_bfloat16* __restrict__ dout, float* __restrict__ delta,
                               float* __restrict__ dq_acc, int64_t rows, int64_t Sq, int HQ,
                               int Dv, int Dqk, int32_t* __restrict__ sem, int64_t nsem) {
  const int64_t gid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (sem && gid < nsem) sem[gid] = 0;  // deterministic mode's dQ turn counters
  const int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  // row = (b * Sq + i) * HQ + h  (the order of o / dout)
  const uint4* po = reinterpret_cast<const uint4*>(o + row * Dv);
  const uint4* pd = reinterpret_cast<const uint4*>(dout + row * Dv);
  float acc = 0.f;
  for (int c = lane; c < Dv / 8; c += 32) {
    const uint4 a = __ldg(po + c), d = __ldg(pd + c);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&d);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(a2[e]), y = __bfloat1622float2(d2[e]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  const int64_t bi = row / HQ;
  const int h = static_cast<int>(row % HQ);
  const int64_t b = bi / Sq, i = bi % Sq;
  if (lane == 0) delta[(b * HQ + h) * Sq + i] = acc;
  float4* z = reinterpret_cast<float4*>(dq_acc + row * Dqk);
  for (int c = lane; c < Dqk / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------------------------
// postprocess: dQ = bf16(softmax_scale * dQ_acc)
// ------------------------------------------------------------------------------------
__global__ void bwd_post_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq,
                                int64_t n4, float scale) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n4;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(dq_acc) + e);
    uint2 out;
    out.x = pack_bf16x2(v.x * scale, v.y * scale);
    out.y = pack_bf16x2(v.z * scale, v.w * scale);
    reinterpret_cast<uint2*>(dq)[e] = out;
  }
}

// ------------------------------------------------------------------------------------
// main kernel
// ------------------------------------------------------------------------------------
// DQK, DV: the head dims the kernel is built for (64-wide inputs run through the
// 128 instance with zero-filled loads); NSPLIT: CTAs sharing one key tile, each owning
// one head-dim chunk of dK / dV / dQ.
template <int DQK, int DV, int NSPLIT>
struct BwdCfg {
  static constexpr int kBM = 64;                     // queries per inner step
  static constexpr int kKPanel = 128 * 128;          // [128 rows x 64 cols] bf16 panel
  static constexpr int kQPanel = kBM * 128;          // [64 rows x 64 cols] bf16 panel
  static constexpr int kKBytes = 128 * DQK * 2;
  static constexpr int kVBytes = 128 * DV * 2;
  static constexpr int kQBytes = kBM * DQK * 2;
  static constexpr int kOBytes = kBM * DV * 2;
  // (192,128): V is held in TMEM (columns kColV, bf16 pairs) and dP^T = V dO^T reads it
  // from there, which leaves shared memory for a third Q/dO stage (the kernel is bound by
  // how long a stage is held: load latency plus one step).  V first lands in the last
  // stage's region and is copied into TMEM by the elementwise warps.
  static constexpr bool kVT = DQK == 192;
  static constexpr int kStages = 3;
  static constexpr int kDSBytes = 128 * kBM * 2;     // dS^T [128 keys][64 q] bf16 (16 KB)
  static constexpr int kKOff = 0;
  static constexpr int kQOff = kKOff + kKBytes + (kVT ? 0 : kVBytes);  // per stage: Q then dO
  static constexpr int kVOff = kVT ? kQOff + (kStages - 1) * (kQBytes + kOBytes) : kKOff + kKBytes;
  static constexpr int kStageBytes = kQBytes + kOBytes;
  // S^T / dP^T buffers in TMEM (and dS^T buffers in shared memory): two, so that the next
  // step's S^T and dP^T overlap this step's elementwise work, or one where TMEM must hold
  // dK and dV over the whole head dim beside V: (192,128) on one CTA per key tile takes
  // 64 + 64 + 192 + 128 + 64 = 512 columns.  Its dQ^T (192 rows) then comes in two
  // 128-row windows, head dims 0-127 into the consumed S^T buffer and 64-191 into the
  // consumed dP^T buffer; the elementwise warps of lane quarters 2 and 3 drain the second
  // window's rows 64-127 (head dims 128-191), the drain warps the first window.
  static constexpr bool kWhole = DQK == 192 && NSPLIT == 1;
  static constexpr int kNB = kWhole ? 1 : 2;
  static constexpr int kDSOff = kQOff + kStages * kStageBytes;     // kNB dS^T buffers
  // fp32 dQ staging tile [2 panels][32 q][64 d]
  static constexpr int kDQOff = kDSOff + kNB * kDSBytes;
  // (kWhole) fp32 staging of the second window's head dims 128-191: [2 query halves][32 q][64 d]
  static constexpr int kDQ2Off = kDQOff + 128 * 32 * 4;
  static constexpr int kLOff = kDQ2Off + (kWhole ? 64 * 64 * 4 : 0);  // per stage: lse2[64], delta[64]
  static constexpr int kBMOff = kLOff + kStages * 2 * kBM * 4;     // per stage: bitmap words [64][4]
  static constexpr int kBarOff = kBMOff + kStages * kBM * 4 * 4;
  static constexpr int kSmem = kBarOff + 256 + 1024;
  static constexpr int kThreads = 448;
  // head-dim chunks of this CTA: dK [kc0, kc0 + kcn), dV [vc0, vc0 + vcn)
  static constexpr int kDKMax = NSPLIT == 1 ? DQK : (DQK == 192 ? 128 : DQK / 2);
  static constexpr int kDVMax = DV / NSPLIT;
  // TMEM columns: S^T / P^T (/ dQ^T window 0) x kNB, dP^T / dS^T / dQ^T x kNB, dK, dV
  static constexpr uint32_t kColS = 0;                // + 64 * buffer
  static constexpr uint32_t kColDP = 64 * kNB;        // + 64 * buffer
  static constexpr uint32_t kColDK = 128 * kNB;
  static constexpr uint32_t kColDV = kColDK + kDKMax;
  static constexpr uint32_t kColV = kColDV + kDVMax;  // V (kVT), DV / 2 columns
  static constexpr uint32_t kTmemCols = 512;
  static_assert(DQK + DV < 512, "head dims 256/256 run in the 2-CTA kernel");
  static_assert(kColDV + kDVMax <= kTmemCols, "tensor memory budget");
  static_assert(!kVT || kColV + DV / 2 <= kTmemCols, "tensor memory budget (V)");
  static_assert(!kVT || kVBytes <= kQBytes + kOBytes, "V lands in one stage's region");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

enum : int {
  kBKV = 0, kBQF = 1, kBQE = 4, kBLF = 7, kBSF = 10, kBPF = 12, kBDQF = 14, kBDQE = 16,
  kBFin = 18, kBDrainB = 19,
  kBVT = 20,   // V copied into TMEM (256 elementwise threads; (192,128) only)
  kBDQE2 = 21, // (kWhole) dQ^T window 1 read from the dP^T buffer (128 elementwise threads)
  kBDQF2 = 22, // (kWhole) dQ^T window 1 complete (commit; with window 0 and dV / dK before it)
  kNumBarsB = 23
};

// Warp roles: 0 producer, 1 MMA, 2-9 elementwise (one key row and 32 of the 64 query
// columns per thread: warps 2-5 columns 0-31, warps 6-9 columns 32-63), 10-13 dQ drain
// (one head-dim row of the dQ^T window per thread).
// Bf16 P^T / dS^T of query columns [32h, 32h+32) are packed into TMEM columns
// [32h, 32h+16) of the S^T / dP^T buffer, inside the range that half itself read.
// DET: deterministic mode (det_order.cuh), a separate instance so that the default
// kernel carries none of its code.
template <int DQK, int DV, int NSPLIT, bool DET>
__global__ void __launch_bounds__(448, 1)
    sparse_bwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dq,
                      const __grid_constant__ CUtensorMap tm_dk,
                      const __grid_constant__ CUtensorMap tm_dv, const AttnArgs a) {
  using C = BwdCfg<DQK, DV, NSPLIT>;
  constexpr int BM = C::kBM;
  constexpr int NB = C::kNB;
  // (the deterministic mode's dQ turns assume one issuer of reduce-adds per CTA)
  static_assert(!(DET && C::kWhole), "deterministic mode keeps the head-dim split");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * kNumBarsB);
  volatile WaitCtl* abort_flag =
      reinterpret_cast<volatile WaitCtl*>(smem + C::kBarOff + 8 * kNumBarsB + 8);
  auto BAR = [&](int k) { return bar0 + 8u * static_cast<uint32_t>(k); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Default: key tiles of one head run together (they share that head's Q / dO in L2).
  // Deterministic mode: key tiles from the last one down (det_order.cuh) with the heads
  // interleaved, so that the key tiles that wait for one another's dQ turns are spread
  // out in time (measured: 8.3 -> 5.8 ms at S=32768, D=256).
  const int split = static_cast<int>(blockIdx.x) % NSPLIT;
  const int lin = static_cast<int>(blockIdx.x) / NSPLIT;
  const int ord = DET ? lin / a.HK : lin;
  // deterministic mode launches the key tiles from the last one down (det_order.cuh)
  const int nt = DET ? a.Tn - 1 - ord : ord;
  const int g = DET ? lin - ord * a.HK : static_cast<int>(blockIdx.y), b = blockIdx.z;
  const int G = a.HQ / a.HK;
  const int64_t bg = static_cast<int64_t>(b) * a.HK + g;
  const int64_t trow = bg * a.Tn + nt;
  const int n_full = __ldg(a.tcnt + 2 * trow);
  const int n_mt = n_full + __ldg(a.tcnt + 2 * trow + 1);
  const int32_t* tlist = a.tidx + trow * a.Tm;
  const int n_iter = G * n_mt * 2;  // (query head, query tile, 64-row half)
  int issued = 0;  // Q/dO stage loads issued (the abort path drains the last ones)

  // head-dim chunks owned by this CTA
  int kc0, kcn, vc0, vcn, qw0;  // qw0: first head-dim row of the 128-wide dQ^T window
  if (NSPLIT == 1) {
    kc0 = 0; kcn = DQK; vc0 = 0; vcn = DV; qw0 = 0;
  } else {  // (192, 128): dK 128 + 64 columns, dV 64 + 64
    static_assert(NSPLIT == 1 || DQK == 192, "head-dim split is built for (192, 128)");
    kc0 = split == 0 ? 0 : 128; kcn = split == 0 ? 128 : 64;
    vc0 = split * 64; vcn = 64;
    qw0 = split == 0 ? 0 : 64;
  }
  const int dqk_real = a.Dqk, dv_real = a.Dv;  // 64 when run through the 128 instance

  if (threadIdx.x == 0) {
    mbar_init(BAR(kBKV), 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(BAR(kBQF + s), 1);
      mbar_init(BAR(kBQE + s), 1);
      mbar_init(BAR(kBLF + s), 32);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(kBSF + s), 1);
      mbar_init(BAR(kBPF + s), 256);
      mbar_init(BAR(kBDQF + s), 1);
      mbar_init(BAR(kBDQE + s), 128);
    }
    mbar_init(BAR(kBFin), 1);
    mbar_init(BAR(kBDrainB), 1);
    mbar_init(BAR(kBVT), 256);
    mbar_init(BAR(kBDQE2), 128);
    mbar_init(BAR(kBDQF2), 1);
    abort_flag->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // broadcast from lane 0 so that the compiler can treat it as warp-uniform
  const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, *tmem_slot, 0);

  // iteration -> (query head, query tile, half)
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
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_do);
        prefetch_tensormap(&tm_dq);
        mbar_arrive_expect_tx(BAR(kBKV), C::kKBytes + C::kVBytes);
        for (int c = 0; c < DQK / 64; ++c)
          tma_load_4d(sbase + C::kKOff + c * C::kKPanel, &tm_k, BAR(kBKV), c * 64, nt * 128, g, b);
        for (int c = 0; c < DV / 64; ++c)
          tma_load_4d(sbase + C::kVOff + c * C::kKPanel, &tm_v, BAR(kBKV), c * 64, nt * 128, g, b);
      }
      float* lbuf = reinterpret_cast<float*>(smem + C::kLOff);
      uint32_t* bmbuf = reinterpret_cast<uint32_t*>(smem + C::kBMOff);
      for (int it = 0; it < n_iter; ++it) {
        int h, m0;
        bool partial;
        decode(it, h, m0, partial);
        m0 = __shfl_sync(0xFFFFFFFFu, m0, 0);  // warp-uniform TMA coordinate
        const int st = it % C::kStages, u = it / C::kStages;
        const uint32_t qs = sbase + C::kQOff + st * C::kStageBytes;
        if (!warp_wait(BAR(kBQE + st), (u & 1) ^ 1, abort_flag, a.status, a.wait_limit_ns)) break;
        // (192,128): V occupies the last stage until it has been copied into TMEM
        if (C::kVT && it == C::kStages - 1 && !warp_wait(BAR(kBVT), 0, abort_flag, a.status, a.wait_limit_ns))
          break;
        if (elect_one()) {
          mbar_arrive_expect_tx(BAR(kBQF + st), C::kQBytes + C::kOBytes);
          for (int c = 0; c < DQK / 64; ++c)
            tma_load_4d(qs + c * C::kQPanel, &tm_q, BAR(kBQF + st), c * 64, m0, h, b);
          for (int c = 0; c < DV / 64; ++c)
            tma_load_4d(qs + C::kQBytes + c * C::kQPanel, &tm_do, BAR(kBQF + st), c * 64, m0, h, b);
        }
        __syncwarp();
        issued = it + 1;
        // LSE (in log2 units) and Delta of the 64 queries; +inf / 0 past Sq
        float* ls = lbuf + st * 2 * BM;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int q = lane + 32 * k;
          const int64_t i = m0 + q;
          float l2 = INFINITY, dl = 0.f;
          if (i < a.Sq) {
            const int64_t li = (static_cast<int64_t>(b) * a.HQ + h) * a.Sq + i;
            l2 = __ldg(a.lse + li) * 1.4426950408889634f;
            dl = __ldg(a.delta + li);
          }
          ls[q] = l2;
          ls[BM + q] = dl;
        }
        if (partial && a.mode == SA_MODE_INDEX) {
          // presence words of this key tile for the 64 queries: [q][4]
          uint32_t* bw = bmbuf + st * BM * 4;
          for (int e = lane; e < BM * 4; e += 32) {
            const int q = e >> 2, w = nt * 4 + (e & 3);
            const int64_t i = m0 + q;
            bw[e] = (i < a.Sq && w < a.W) ? __ldg(a.bitmap + (bg * a.Sq + i) * a.W + w) : 0u;
          }
        }
        mbar_arrive(BAR(kBLF + st));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (converged, warp-uniform operands); one elected
    // lane issues each batch of tcgen05 instructions.
    if (n_iter > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, BM, 0, 0);      // S^T, dP^T
      constexpr uint32_t idesc_dq = idesc_bf16(128, BM, 1, 1);     // dQ^T = K^T dS^T
      const uint32_t idesc_dv = idesc_bf16(128, vcn, 0, 1);        // dV += P^T dO
      const uint32_t idesc_dk = idesc_bf16(128, kcn, 0, 1);        // dK += dS^T Q
      const uint32_t kbase = sbase + C::kKOff, vbase = sbase + C::kVOff;
      // descriptors of panel bases; a k-step adds its byte offset / 16 to the
      // start-address field (no carry: shared addresses stay below 2^18)
      const uint64_t kd = sw128_desc(kbase, 16, 1024), vd = sw128_desc(vbase, 16, 1024);
      const uint64_t kwd = sw128_desc(kbase + (qw0 / 64) * C::kKPanel, C::kKPanel, 1024);
      // (kWhole) dQ^T window 1: head dims 64-191 (K panels 1 and 2)
      const uint64_t kwd1 = sw128_desc(kbase + C::kKPanel, C::kKPanel, 1024);
      bool ok = warp_wait(BAR(kBKV), 0, abort_flag, a.status, a.wait_limit_ns);
      if (C::kVT) ok = ok && warp_wait(BAR(kBVT), 0, abort_flag, a.status, a.wait_limit_ns);
      // S^T(j) and dP^T(j) into TMEM buffer j % NB
      auto issue_sdp = [&](int j) -> bool {
        const int st = j % C::kStages, u = j / C::kStages, bj = NB == 2 ? (j & 1) : 0;
        if (!warp_wait(BAR(kBQF + st), u & 1, abort_flag, a.status, a.wait_limit_ns)) return false;
        // the dQ^T of step j-NB lives in this buffer until it has been drained (kWhole:
        // window 0 in the S^T buffer)
        if (j >= NB && !warp_wait(BAR(kBDQE + bj), ((j - NB) / NB) & 1, abort_flag, a.status, a.wait_limit_ns))
          return false;
        tc_fence_after();
        const uint32_t qs = sbase + C::kQOff + st * C::kStageBytes;
        const uint64_t qd = sw128_desc(qs, 16, 1024), od = sw128_desc(qs + C::kQBytes, 16, 1024);
        // one lane issues both MMA batches and the commit (a commit tracks the MMAs of
        // the thread that executes it)
        const bool leader = elect_one();
        if (leader) {
          for (int p = 0; p < DQK / 64; ++p) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint32_t ka = p * C::kKPanel + k4 * 32, qb = p * C::kQPanel + k4 * 32;
              umma_ss(tmem + C::kColS + 64 * bj, kd + (ka >> 4), qd + (qb >> 4), idesc_s,
                      (p > 0 || k4 > 0) ? 1u : 0u);
            }
          }
        }
        __syncwarp();
        // (kWhole) window 1 of dQ^T(j-1) lives in the dP^T buffer until the elementwise
        // warps of lane quarters 2 and 3 have read it
        if (C::kWhole && j >= 1) {
          if (!warp_wait(BAR(kBDQE2), (j - 1) & 1, abort_flag, a.status, a.wait_limit_ns)) return false;
          tc_fence_after();
        }
        if (leader) {
          for (int p = 0; p < DV / 64; ++p) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint32_t va = p * C::kKPanel + k4 * 32, ob = p * C::kQPanel + k4 * 32;
              if constexpr (C::kVT)  // A = V from TMEM: 16 head dims = 8 columns per k-step
                umma_ts(tmem + C::kColDP + 64 * bj, tmem + C::kColV + (p * 4 + k4) * 8,
                        od + (ob >> 4), idesc_s, (p > 0 || k4 > 0) ? 1u : 0u);
              else
                umma_ss(tmem + C::kColDP + 64 * bj, vd + (va >> 4), od + (ob >> 4), idesc_s,
                        (p > 0 || k4 > 0) ? 1u : 0u);
            }
          }
          umma_commit(BAR(kBSF + bj));
        }
        __syncwarp();
        return true;
      };
      if (ok) ok = issue_sdp(0);
      for (int it = 0; ok && it < n_iter; ++it) {
        const int st = it % C::kStages, bi = NB == 2 ? (it & 1) : 0;
        // the next S^T / dP^T overlap this step's elementwise work (two buffers; with one
        // they follow this step's dQ^T, once it has been drained)
        if (NB == 2 && it + 1 < n_iter && !issue_sdp(it + 1)) break;
        if (!warp_wait(BAR(kBPF + bi), (it / NB) & 1, abort_flag, a.status, a.wait_limit_ns)) break;
        tc_fence_after();
        const uint32_t qs = sbase + C::kQOff + st * C::kStageBytes;
        const uint64_t qmn = sw128_desc(qs + (kc0 / 64) * C::kQPanel, C::kQPanel, 1024);
        const uint64_t omn = sw128_desc(qs + C::kQBytes + (vc0 / 64) * C::kQPanel, C::kQPanel, 1024);
        const uint64_t dsd = sw128_desc(sbase + C::kDSOff + bi * C::kDSBytes, C::kKPanel, 1024);
        if (elect_one()) {
          // dV += P^T dO  and  dK += dS^T Q (K = 64 queries: four k-steps of 16)
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            umma_ts(tmem + C::kColDV, tmem + C::kColS + 64 * bi + (kk >> 1) * 32 + (kk & 1) * 8,
                    omn + ((kk * 2048) >> 4), idesc_dv, (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            umma_ts(tmem + C::kColDK, tmem + C::kColDP + 64 * bi + (kk >> 1) * 32 + (kk & 1) * 8,
                    qmn + ((kk * 2048) >> 4), idesc_dk, (it > 0 || kk > 0) ? 1u : 0u);
          umma_commit(BAR(kBQE + st));
          // dQ^T = K^T dS^T over the 128 keys, into the dP^T buffer dK has just consumed
          // (kWhole: window 0 into the S^T buffer dV has consumed, window 1 into dP^T's)
          const uint32_t dq0 = (C::kWhole ? C::kColS : C::kColDP) + 64 * bi;
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            umma_ss(tmem + dq0, kwd + ((kk * 2048) >> 4), dsd + ((kk * 2048) >> 4), idesc_dq,
                    kk > 0 ? 1u : 0u);
          // (kWhole: window 0 completes on its own barrier, so that the drain reads it, and
          // the next S^T can be queued, while window 1 is computed)
          umma_commit(BAR(kBDQF + bi));
          if constexpr (C::kWhole) {
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              umma_ss(tmem + C::kColDP, kwd1 + ((kk * 2048) >> 4), dsd + ((kk * 2048) >> 4),
                      idesc_dq, kk > 0 ? 1u : 0u);
            umma_commit(BAR(kBDQF2));
          }
        }
        __syncwarp();
        if (NB == 1 && it + 1 < n_iter && !issue_sdp(it + 1)) break;
      }
      if (elect_one()) umma_commit(BAR(kBFin));
      __syncwarp();
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------------ elementwise
    const int quarter = warp & 3;
    const int hc = (warp - 2) >> 2;              // which 32 of the 64 query columns
    const int r = quarter * 32 + lane;           // key row of the tile = TMEM lane
    // (kWhole) warps 2, 3 / 6, 7 (lane quarters 2 and 3, query halves 0 / 1) also drain
    // dQ^T window 1, whose useful rows 64-127 are their TMEM lanes
    const bool w1_helper = C::kWhole && quarter >= 2;
    const int64_t j = static_cast<int64_t>(nt) * 128 + r;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float* lbuf = reinterpret_cast<const float*>(smem + C::kLOff);
    const uint32_t* bmbuf = reinterpret_cast<const uint32_t*>(smem + C::kBMOff);
    const bool key_ok = j < a.Sk;
    bool ok = true;
    if (C::kVT && n_iter > 0) {
      // V row r into TMEM (row r in lane r, head dims 2e, 2e+1 in column e): this half of
      // the warps copies the 64-column panel hc from the swizzled smem tile
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(BAR(kBKV), 0, abort_flag, a.status, a.wait_limit_ns));
      if (ok) {
        const uint8_t* prow = smem + C::kVOff + hc * C::kKPanel + r * 128;
        uint32_t w[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(prow + ((k ^ (r & 7)) << 4));
          w[4 * k] = v.x;
          w[4 * k + 1] = v.y;
          w[4 * k + 2] = v.z;
          w[4 * k + 3] = v.w;
        }
        tmem_st32(tl + C::kColV + hc * 32, w);
        tmem_wait_st();
      }
      // the stage region V occupied is reloaded by TMA next
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(BAR(kBVT));
      // a helper pair enters the step loop together or not at all (its warps' waits above
      // can end differently when a wait runs out, and the loop meets at named barriers)
      if (w1_helper) ok = named_bar_and(3 + hc, 64, ok);
    }
    for (int it = 0; ok && it < n_iter; ++it) {
      int h, m0;
      bool partial;
      decode(it, h, m0, partial);
      const int st = it % C::kStages, u = it / C::kStages, bi = NB == 2 ? (it & 1) : 0;
      bool w_ok = mbar_wait(BAR(kBLF + st), u & 1, abort_flag, a.status, a.wait_limit_ns);
      w_ok = w_ok && mbar_wait(BAR(kBSF + bi), (it / NB) & 1, abort_flag, a.status, a.wait_limit_ns);
      // the dS^T buffer is free once dQ^T of step it-NB has read it (kWhole: both windows)
      if (it >= NB)
        w_ok = w_ok && mbar_wait(BAR(C::kWhole ? kBDQF2 : kBDQF + bi), ((it - NB) / NB) & 1,
                                 abort_flag, a.status, a.wait_limit_ns);
      w_ok = __all_sync(0xFFFFFFFFu, w_ok);
      // (the two warps of a dQ^T-window-1 helper pair leave together: they share a named
      // barrier below)
      if (w1_helper) w_ok = named_bar_and(3 + hc, 64, w_ok);
      if (!w_ok) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* ls = lbuf + st * 2 * BM + 32 * hc;
      uint8_t* dsrow = smem + C::kDSOff + bi * C::kDSBytes + r * 128;
      const uint32_t cs = C::kColS + 64 * bi + 32 * hc, cd = C::kColDP + 64 * bi + 32 * hc;
      uint32_t s_u[32], p_u[32];
      tmem_ld32(tl + cs, s_u);
      tmem_ld32(tl + cd, p_u);
      // allowed-query mask of this key row over this half's 32 queries (partial tiles)
      uint32_t cm = 0xFFFFFFFFu;
      if (partial) {
        const int64_t q0 = m0 + 32 * hc;
        cm = key_ok ? 0xFFFFFFFFu : 0u;
        if (a.causal) {  // i >= j
          const int64_t lo = j - q0;
          cm &= lo <= 0 ? 0xFFFFFFFFu : (lo >= 32 ? 0u : (0xFFFFFFFFu << lo));
        }
        if (a.mode == SA_MODE_BLOCK && a.bs == 64 && key_ok) {
          const int64_t mb = m0 / 64;
          const bool m = mb < a.Mb &&
                         __ldg(a.mask + (bg * a.Mb + mb) * static_cast<int64_t>(a.Nb) + j / 64) != 0;
          if (!m) cm = 0u;
        } else if (a.mode == SA_MODE_INDEX) {
          // lane L loads the presence word of query q0 + L over this warp's 32 key rows;
          // a bit transpose across the warp leaves in lane L the word of key row r over
          // the 32 queries (the branch is warp-uniform)
          cm &= warp_transpose32(bmbuf[st * BM * 4 + (32 * hc + lane) * 4 + (r >> 5)], lane);
        }
      }
      tmem_wait_ld();
      uint32_t pk[16], dk[16];
      const float4* ls4 = reinterpret_cast<const float4*>(ls);         // lse2[q] (log2 units)
      const float4* dl4 = reinterpret_cast<const float4*>(ls + BM);    // Delta[q]
      const float sc = a.scale_log2;
      if (!partial) {
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 l = ls4[e4], d = dl4[e4];
          const float lv[4] = {l.x, l.y, l.z, l.w}, dv4[4] = {d.x, d.y, d.z, d.w};
          float pv[4], dsv[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int q = 4 * e4 + t;
            pv[t] = ex2(fmaf(__uint_as_float(s_u[q]), sc, -lv[t]));
            dsv[t] = pv[t] * (__uint_as_float(p_u[q]) - dv4[t]);
          }
          pk[2 * e4] = pack_bf16x2(pv[0], pv[1]);
          pk[2 * e4 + 1] = pack_bf16x2(pv[2], pv[3]);
          dk[2 * e4] = pack_bf16x2(dsv[0], dsv[1]);
          dk[2 * e4 + 1] = pack_bf16x2(dsv[2], dsv[3]);
        }
      } else {
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 l = ls4[e4], d = dl4[e4];
          const float lv[4] = {l.x, l.y, l.z, l.w}, dv4[4] = {d.x, d.y, d.z, d.w};
          float pv[4], dsv[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int q = 4 * e4 + t;
            pv[t] = ((cm >> q) & 1u) ? ex2(fmaf(__uint_as_float(s_u[q]), sc, -lv[t])) : 0.f;
            dsv[t] = pv[t] * (__uint_as_float(p_u[q]) - dv4[t]);
          }
          pk[2 * e4] = pack_bf16x2(pv[0], pv[1]);
          pk[2 * e4 + 1] = pack_bf16x2(pv[2], pv[3]);
          dk[2 * e4] = pack_bf16x2(dsv[0], dsv[1]);
          dk[2 * e4 + 1] = pack_bf16x2(dsv[2], dsv[3]);
        }
      }
      tmem_st16(tl + cs, pk);
      tmem_st16(tl + cd, dk);
      // dS^T row into shared memory, 128-byte swizzled: 16-byte chunk c of row r
      // lives at chunk c ^ (r % 8)
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const int c = hc * 4 + c4;
        *reinterpret_cast<uint4*>(dsrow + ((c ^ (r & 7)) << 4)) =
            make_uint4(dk[4 * c4], dk[4 * c4 + 1], dk[4 * c4 + 2], dk[4 * c4 + 3]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(BAR(kBPF + bi));
      if (w1_helper) {
        // dQ^T window 1 (head dims 64-191 in the dP^T buffer): this thread's row r - 64 of
        // head dims 128-191 over this pair's 32 queries, read as soon as dQ^T is complete
        // (S^T / dP^T of the next step wait for that), then staged as a [32 q][64 d] fp32
        // tile and reduce-added into dQ_acc by one thread of the pair
        bool d_ok = mbar_wait(BAR(kBDQF2), it & 1, abort_flag, a.status, a.wait_limit_ns);
        if (!named_bar_and(3 + hc, 64, __all_sync(0xFFFFFFFFu, d_ok))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t w1[32];
        tmem_ld32(tl + C::kColDP + 32 * hc, w1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(BAR(kBDQE2));
        const bool issuer = threadIdx.x == 64 + 128 * hc;  // warp 2 / 6, lane 0
        float* st2 = reinterpret_cast<float*>(smem + C::kDQ2Off + hc * 32 * 64 * 4);
        if (issuer) bulk_wait_group_read0();  // the previous reduce has read the tile
        named_bar_sync(3 + hc, 64);
#pragma unroll
        for (int q = 0; q < 32; ++q) st2[q * 64 + (r - 64)] = __uint_as_float(w1[q]);
        fence_proxy_async_smem();
        named_bar_sync(3 + hc, 64);
        if (issuer) {
          tma_reduce_add_4d(&tm_dq, sbase + C::kDQ2Off + hc * 32 * 64 * 4, 128, m0 + 32 * hc, h, b);
          bulk_commit_group();
        }
      }
    }
    if (w1_helper && threadIdx.x == 64 + 128 * hc) bulk_wait_group0();  // every reduce landed
    // ----------------------------------------------------------- dK / dV epilogue
    bool have = n_iter > 0 && ok;
    if (have) {
      const bool w_ok = mbar_wait(BAR(kBFin), 0, abort_flag, a.status, a.wait_limit_ns);
      have = __all_sync(0xFFFFFFFFu, w_ok);
      tc_fence_after();
    }
    // The rows go to the idle stages as [128 keys][64 dims] 128-byte-swizzled panels
    // (dK's, then dV's; the output maps' box) and leave by TMA stores, which drop rows
    // past Sk; panels past the real head dim are not stored.  The two halves of the
    // elementwise warps fill alternating 32-column chunks.
    for (int pass = 0; pass < 2; ++pass) {
      const int n = pass == 0 ? kcn : vcn;
      const uint32_t col = pass == 0 ? C::kColDK : C::kColDV;
      const float sc = pass == 0 ? a.scale : 1.f;
      const uint32_t pbase = C::kQOff + (pass == 0 ? 0 : (kcn / 64) * C::kKPanel);
      for (int c = 32 * hc; c < n; c += 64) {
        uint32_t v[32];
        if (have) {
          tmem_ld32(tl + col + c, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * sc, __uint_as_float(v[2 * e + 1]) * sc);
        // columns [c, c+32) = 16-byte chunks (c % 64) / 8 .. +3 of row r in panel c / 64
        uint8_t* prow = smem + pbase + (c >> 6) * C::kKPanel + r * 128;
        const int ch0 = (c & 63) >> 3;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(prow + (((ch0 + e) ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(2, 256);
    if (threadIdx.x == 64) {
      for (int pp = 0; pp < kcn / 64; ++pp)
        if (kc0 + 64 * pp < dqk_real)
          tma_store_4d(&tm_dk, sbase + C::kQOff + pp * C::kKPanel, kc0 + 64 * pp, nt * 128, g, b);
      for (int pp = 0; pp < vcn / 64; ++pp)
        if (vc0 + 64 * pp < dv_real)
          tma_store_4d(&tm_dv, sbase + C::kQOff + (kcn / 64 + pp) * C::kKPanel, vc0 + 64 * pp,
                       nt * 128, g, b);
      bulk_commit_group();
      bulk_wait_group_read0();  // the stages are read before the CTA may leave
    }
  } else {
    // ------------------------------------------------------------------ dQ drain
    // thread = head-dim row r of the 128-wide dQ^T window; the 64 query columns are
    // staged as fp32 in the step's (now free) dS^T buffer, 32 queries at a time, as
    // [64-column panel][32 q][64 d] tiles that bulk reduce-adds push into dQ_acc.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int dtid = threadIdx.x - 320;  // 0..127 within the drain warpgroup
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int p = r >> 6;  // panel of this row within the window
    // a panel is reduced when it lies in this CTA's dQ range and inside Dqk
    auto panel_owned = [&](int pp) {
      const int d0 = qw0 + 64 * pp;
      return d0 >= kc0 && d0 + 64 <= kc0 + kcn && d0 < dqk_real;
    };
    const bool own0 = panel_owned(0), own1 = panel_owned(1);
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      int h, m0;
      bool partial;
      decode(it, h, m0, partial);
      const int bi = NB == 2 ? (it & 1) : 0;
      // the four drain warps leave together (they share named barrier 1 below)
      const bool w_ok = mbar_wait(BAR(kBDQF + bi), (it / NB) & 1, abort_flag, a.status, a.wait_limit_ns);
      if (!named_bar_and(1, 128, w_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t q_u[BM];
      // dQ^T window 0 (kWhole: in the S^T buffer)
      const uint32_t dq0 = (C::kWhole ? C::kColS : C::kColDP) + 64 * bi;
      tmem_ld32(tl + dq0, q_u);
      tmem_ld32(tl + dq0 + 32, q_u + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(BAR(kBDQE + bi));
      float* stage = reinterpret_cast<float*>(smem + C::kDQOff);
      const uint32_t stage_s = sbase + C::kDQOff;
      // deterministic mode: this CTA's turn on the query tile starts at the first add of
      // its first 64-row half and ends after the last add of its second half
      const int mt = m0 >> 7, qhalf = (m0 >> 6) & 1;
      bool turn_ok = true;
      if (DET && qhalf == 0 && dtid == 0)
        turn_ok = det_wait_turn(det_slot(a, b, h, mt, split), key_tile_rank(a, bg, mt, nt), abort_flag,
                                a.status, a.wait_limit_ns);
      if (DET && !named_bar_and(1, 128, turn_ok)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        // the previous reduce (this step's first half, or the last step's second half)
        // must have read the staging tile
        if (dtid == 0) bulk_wait_group_read0();
        named_bar_sync(1, 128);
#pragma unroll
        for (int q = 0; q < 32; ++q) stage[(p * 32 + q) * 64 + (r & 63)] = __uint_as_float(q_u[32 * half + q]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (dtid == 0) {
          if (own0) tma_reduce_add_4d(&tm_dq, stage_s, qw0, m0 + 32 * half, h, b);
          if (own1) tma_reduce_add_4d(&tm_dq, stage_s + 32 * 64 * 4, qw0 + 64, m0 + 32 * half, h, b);
          bulk_commit_group();
        }
      }
      if (DET && qhalf == 1 && dtid == 0) det_pass_turn(det_slot(a, b, h, mt, split));
    }
    if (dtid == 0) bulk_wait_group0();  // every reduce has landed before the CTA ends
  }

  tc_fence_before();
  __syncthreads();
  // Abort path.  Past the barrier above no warp issues another copy or MMA, and the
  // abort flag no longer changes (the branch is uniform).  A stage is reloaded only after
  // the MMAs that read its previous contents have completed, so at most the last
  // kStages stage loads (and the K/V load) can still be in flight: wait for them, and
  // for every MMA this CTA issued, before shared memory and TMEM are released
  // (time-limited waits).  The dQ reduce-adds and the dK/dV stores were waited for by
  // the threads that issued them.
  if (abort_flag->abort) {
    if (warp == 0 && lane == 0 && n_iter > 0) {
      mbar_wait_limited(BAR(kBKV), 0);
      for (int it = max(0, issued - C::kStages); it < issued; ++it)
        mbar_wait_limited(BAR(kBQF + it % C::kStages), (it / C::kStages) & 1);
    }
    if (warp == 1 && n_iter > 0) {
      tc_fence_after();
      if (elect_one()) {
        umma_commit(BAR(kBDrainB));
        mbar_wait_limited(BAR(kBDrainB), 0);
      }
      __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int DQK, int DV, int NSPLIT, bool DET>
static int launch_bwd_main_t(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  using C = BwdCfg<DQK, DV, NSPLIT>;
  static PerDeviceOnce attr;
  const int rc = once_per_device(attr, [] {
    const int r = cuda_error(cudaFuncSetAttribute(sparse_bwd_kernel<DQK, DV, NSPLIT, DET>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  C::kSmem),
                             "backward smem attribute");
    if (r == SA_OK && std::getenv("SA_DEBUG")) {
      cudaFuncAttributes fa;
      const cudaError_t qe = cudaFuncGetAttributes(&fa, sparse_bwd_kernel<DQK, DV, NSPLIT, DET>);
      int occ = -1;
      const cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
          &occ, sparse_bwd_kernel<DQK, DV, NSPLIT, DET>, C::kThreads, C::kSmem);
      std::fprintf(stderr, "sparse_attn: attribute query %s, occupancy query %s -> %d\n",
                   cudaGetErrorName(qe), cudaGetErrorName(oe), occ);
      if (qe == cudaSuccess)
        std::fprintf(stderr,
                     "sparse_attn: backward kernel regs %d, max threads %d, static smem %zu, "
                     "local %zu, max dyn smem %d, launch %d threads x %d B smem\n",
                     fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes, fa.localSizeBytes,
                     fa.maxDynamicSharedSizeBytes, C::kThreads, C::kSmem);
    }
    return r;
  });
  if (rc) return rc;
  const dim3 grid = DET ? dim3(a.Tn * NSPLIT * a.HK, 1, a.B) : dim3(a.Tn * NSPLIT, a.HK, a.B);
  record_event(3, st);
  sparse_bwd_kernel<DQK, DV, NSPLIT, DET><<<grid, C::kThreads, C::kSmem, st>>>(
      m.q, m.k, m.v, m.dout, m.dq_acc, m.dk, m.dv, a);
  record_event(4, st);
  return check_launch("backward main kernel launch");
}

template <int DQK, int DV, int NSPLIT>
static int launch_bwd_main(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  return a.det ? launch_bwd_main_t<DQK, DV, NSPLIT, true>(a, m, st)
               : launch_bwd_main_t<DQK, DV, NSPLIT, false>(a, m, st);
}

int launch_bwd(const AttnArgs& a, const TensorMaps& m, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.Sq * a.HQ;
  {
    const int warps = 8;
    const int64_t blocks = (rows + warps - 1) / warps;
    record_event(2, st);
    const int64_t nsem = a.det ? static_cast<int64_t>(a.B) * a.HQ * a.Tm * 2 : 0;
    bwd_pre_kernel<<<static_cast<unsigned>(blocks), warps * 32, 0, st>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.delta,
        a.dq_acc, rows, a.Sq, a.HQ, a.Dv, a.Dqk, a.det ? a.sem : nullptr, nsem);
    if (check_launch("backward preprocess launch")) return SA_ERR_CUDA;
  }
  int rc;
  if (a.Dqk == 64 && a.Dv == 64)
    rc = launch_bwd_main<128, 128, 1>(a, m, st);
  else if (a.Dqk == 128 && a.Dv == 128)
    rc = launch_bwd_main<128, 128, 1>(a, m, st);
  else if (a.Dqk == 192 && a.Dv == 128) {
    // One CTA per key tile (single-buffered S^T / dP^T, no recompute) once its grid fills
    // the SMs at least twice over; below that the head-dim split over two CTAs, which
    // keeps twice as many SMs busy (measured at total_q = 4096, 128 key-tile CTAs on 148
    // SMs: 1.51 ms against 1.22; at 16384, 512 CTAs: 11.8 against 13.1 ms).  The
    // deterministic mode always splits.
    int form = g_bwd_form.load(std::memory_order_relaxed);
    if (form == SA_BWD_FORM_AUTO) {
      int dev = 0, sms = 148;
      if (cudaGetDevice(&dev) == cudaSuccess)
        (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      const int64_t ctas = static_cast<int64_t>(a.Tn) * a.HK * a.B;
      form = ctas >= 2 * static_cast<int64_t>(sms) ? SA_BWD_FORM_WHOLE : SA_BWD_FORM_SPLIT;
    }
    rc = (a.det || form == SA_BWD_FORM_SPLIT) ? launch_bwd_main<192, 128, 2>(a, m, st)
                                              : launch_bwd_main_t<192, 128, 1, false>(a, m, st);
  }
  else if (a.Dqk == 256 && a.Dv == 256)
    rc = launch_bwd_pair(a, m, st);
  else
    return SA_ERR_UNSUPPORTED;
  if (rc) return rc;
  const int64_t n4 = rows * a.Dqk / 4;
  bwd_post_kernel<<<static_cast<unsigned>(min64((n4 + 255) / 256, 148 * 16)), 256, 0, st>>>(
      a.dq_acc, static_cast<__nv_bfloat16*>(a.dq), n4, a.scale);
  record_event(5, st);
  return check_launch("backward postprocess launch");
}

}  // namespace sa
