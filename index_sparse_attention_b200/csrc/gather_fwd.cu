// gather_fwd.cu -- token-gather forward for index mode: O and LSE with every query's
// selected K/V rows gathered one by one, instead of streaming whole 128-key tiles.
//
// The pages name this family as the alternative to block coarsening: the sparse MLA
// backends that consume top-k indices (xtuner PR #2096, Background) attend to exactly
// the selected keys.  The block path (fwd.cu) reaches the same result through the
// presence bitmap on partial tiles, at the cost of computing the whole tile.  This
// kernel is the measured comparison: same inputs (the converter's bitmap), same O and
// LSE (the oracle's), no tile-level redundancy.
//
// Design.  One warp per (batch, query token i, KV head g), the G <= 8 query heads of the
// group together (they share every gathered row):
//   keys     the warp reads the token's presence-bitmap row 32 words at a time and
//            enumerates the set bits below the causal / range limit in ascending order
//            (set semantics for repeated indices come with the bitmap);
//   gather   16 keys per chunk: their K and V rows (Dqk and Dv bf16) are copied into
//            shared memory with cp.async (16-byte pieces, zero-filled past the last key
//            of the row), double-buffered across chunks;
//   S        S = Q K^T with mma.sync m16n8k16 (bf16 in, fp32 out): M = the group's
//            query heads padded to 16 (rows >= G are zero), N = 8 keys, K = 16 head dims.
//            tcgen05's smallest M is 64; a gathered row is shared by G = 8 heads only;
//   softmax  online, in registers, per head: running max and sum over the chunks;
//   O        O += P V with mma.sync (P from the S accumulators, packed to bf16; V from
//            shared memory through ldmatrix.trans), fp32 accumulators in registers.
// Shared-memory rows are padded by 16 bytes so that the eight rows an ldmatrix matrix
// reads fall in distinct bank groups.  Supported: Dv <= 128 (O of 16 x Dv in registers),
// HQ / HK <= 8, index mode (the bitmap).
#include <cuda_bf16.h>

#include "sa_device.cuh"
#include "sa_kernels.h"

namespace sa {
namespace gather {

constexpr int kWarps = 8;
constexpr int kChunk = 16;  // keys per chunk

template <int DQK, int DV>
struct Cfg {
  static constexpr int kKStride = DQK * 2 + 16;  // bytes per staged K row (padded)
  static constexpr int kVStride = DV * 2 + 16;
  static constexpr int kVOff = kChunk * kKStride;
  static constexpr int kStage = kVOff + kChunk * kVStride;
  static constexpr int kWarpBytes = 2 * kStage;
  static constexpr int kSmem = kWarps * kWarpBytes;
  static constexpr int kKSeg = DQK / 8;  // 16-byte pieces per K row
  static constexpr int kVSeg = DV / 8;
  static constexpr int kSegs = kChunk * (kKSeg + kVSeg);
  static_assert(kSegs % 32 == 0, "every lane issues the same number of copies");
  static_assert(DV <= 128 && DQK % 16 == 0 && DV % 16 == 0, "supported head dims");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Four 8 x 8 bf16 matrices; lane l gives the address of row l % 8 of matrix l / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16 x 8, fp32) += A (16 x 16, bf16, row-major fragments) * B (16 x 8, bf16).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Position of the n-th (0-based) set bit of x; n < popc(x).
__device__ __forceinline__ int nth_set_bit(uint32_t x, int n) {
  int pos = 0, c = __popc(x & 0xFFFFu);
  if (n >= c) { n -= c; x >>= 16; pos += 16; }
  c = __popc(x & 0xFFu);
  if (n >= c) { n -= c; x >>= 8; pos += 8; }
  c = __popc(x & 0xFu);
  if (n >= c) { n -= c; x >>= 4; pos += 4; }
  c = __popc(x & 0x3u);
  if (n >= c) { n -= c; x >>= 2; pos += 2; }
  if (n >= static_cast<int>(x & 1u)) pos += 1;
  return pos;
}

template <int DQK, int DV>
__global__ void __launch_bounds__(kWarps * 32, 1)
    gather_fwd_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const AttnArgs a) {
  using C = Cfg<DQK, DV>;
  extern __shared__ __align__(16) uint8_t smem_g[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t wbase = smem_u32(smem_g) + warp * C::kWarpBytes;
  const int G = a.HQ / a.HK;
  const int row = lane >> 2;      // query head of the group this lane's fragments hold
  const int quad = lane & 3;
  const float sl2 = a.scale_log2;
  const int64_t items = static_cast<int64_t>(a.B) * a.Sq * a.HK;

  for (int64_t item = static_cast<int64_t>(blockIdx.x) * kWarps + warp; item < items;
       item += static_cast<int64_t>(gridDim.x) * kWarps) {
    const int g = static_cast<int>(item % a.HK);
    const int64_t bi = item / a.HK;  // b * Sq + i
    const int64_t i = bi % a.Sq;
    const int b = static_cast<int>(bi / a.Sq);
    const int64_t bg = static_cast<int64_t>(b) * a.HK + g;
    const uint32_t* brow = a.bitmap + (bg * a.Sq + i) * a.W;
    const int64_t lim = a.causal ? min64(a.Sk, i + 1) : a.Sk;  // keys j < lim

    // Q of the group's heads as A fragments (rows >= G are zero)
    uint32_t qa0[DQK / 16], qa2[DQK / 16];
    {
      const bool hv = row < G;
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(
          q + ((bi * a.HQ) + static_cast<int64_t>(g) * G + (hv ? row : 0)) * DQK);
#pragma unroll
      for (int kt = 0; kt < DQK / 16; ++kt) {
        qa0[kt] = hv ? __ldg(qr + kt * 8 + quad) : 0u;
        qa2[kt] = hv ? __ldg(qr + kt * 8 + 4 + quad) : 0u;
      }
    }

    // key enumeration over 32-word blocks of the bitmap row
    int64_t blk = 0;        // next block to read
    int64_t cur_base = 0;   // first word of the current block
    uint32_t word = 0u;     // this lane's word of the current block (bits >= lim cleared)
    int incl = 0, total = 0, pos = 0;
    const int64_t nblk = (lim + 1023) / 1024;
    auto load_block = [&]() -> bool {
      while (blk < nblk) {
        const int64_t w = blk * 32 + lane;
        uint32_t x = (w < a.W) ? __ldg(brow + w) : 0u;
        const int64_t j0 = w * 32;
        if (j0 + 32 > lim) x = (j0 >= lim) ? 0u : (x & ((1u << (lim - j0)) - 1u));
        int pre = __popc(x);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xFFFFFFFFu, pre, o);
          if (lane >= o) pre += y;
        }
        cur_base = blk * 32;
        ++blk;
        word = x;
        incl = pre;
        total = __shfl_sync(0xFFFFFFFFu, pre, 31);
        pos = 0;
        if (total > 0) return true;
      }
      return false;
    };
    // the next chunk: lane t < 16 receives the key of slot t, -1 past the row's keys;
    // returns the number of valid slots (warp-uniform)
    auto next_chunk = [&](int& key) -> int {
      key = -1;
      if (pos >= total && !load_block()) return 0;
      const int p = pos + lane;
      int lo = 0;  // owner: the first lane whose inclusive prefix exceeds p
#pragma unroll
      for (int step = 16; step >= 1; step >>= 1) {
        const int cand = __shfl_sync(0xFFFFFFFFu, incl, lo + step - 1);
        if (cand <= p) lo += step;
      }
      lo = min(lo, 31);
      const uint32_t ow = __shfl_sync(0xFFFFFFFFu, word, lo);
      const int excl = __shfl_sync(0xFFFFFFFFu, incl, lo) - __popc(ow);
      const int nval = min(kChunk, total - pos);
      if (lane < nval) key = static_cast<int>((cur_base + lo) * 32 + nth_set_bit(ow, p - excl));
      pos += kChunk;
      return nval;
    };
    auto issue = [&](int stage, int key) {
      const uint32_t sb = wbase + stage * C::kStage;
#pragma unroll
      for (int e0 = 0; e0 < C::kSegs; e0 += 32) {
        const int e = e0 + lane;
        const bool isk = e < kChunk * C::kKSeg;
        const int ee = isk ? e : e - kChunk * C::kKSeg;
        const int t = isk ? ee / C::kKSeg : ee / C::kVSeg;
        const int sg = isk ? ee % C::kKSeg : ee % C::kVSeg;
        const int kt = __shfl_sync(0xFFFFFFFFu, key, t);
        const bool valid = kt >= 0;
        const int64_t r = ((static_cast<int64_t>(b) * a.Sk + (valid ? kt : 0)) * a.HK + g);
        const __nv_bfloat16* src = isk ? k + r * DQK + sg * 8 : v + r * DV + sg * 8;
        const uint32_t dst =
            sb + (isk ? t * C::kKStride + sg * 16 : C::kVOff + t * C::kVStride + sg * 16);
        cp_async16(dst, src, valid);
      }
      cp_async_commit();
    };

    float oacc[DV / 8][4];
#pragma unroll
    for (int n = 0; n < DV / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) oacc[n][e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    int key_cur;
    int nv_cur = next_chunk(key_cur);
    if (nv_cur > 0) issue(0, key_cur);
    int stage = 0;
    while (nv_cur > 0) {
      int key_nxt;
      const int nv_nxt = next_chunk(key_nxt);
      if (nv_nxt > 0) {
        issue(stage ^ 1, key_nxt);
        cp_async_wait<1>();  // the current chunk has landed
      } else {
        cp_async_wait<0>();
      }
      __syncwarp();
      const uint32_t sb = wbase + stage * C::kStage;

      // S (rows = heads, columns = the chunk's 16 keys in two n-tiles of 8)
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int m = lane >> 3;  // matrix: (key half, head-dim half)
        const uint32_t kaddr = sb + ((m >> 1) * 8 + (lane & 7)) * C::kKStride + (m & 1) * 16;
#pragma unroll
        for (int kt = 0; kt < DQK / 16; ++kt) {
          uint32_t b00, b01, b10, b11;
          ldsm_x4(kaddr + kt * 32, b00, b01, b10, b11);
          mma16816(s[0], qa0[kt], 0u, qa2[kt], 0u, b00, b01);
          mma16816(s[1], qa0[kt], 0u, qa2[kt], 0u, b10, b11);
        }
      }
      // online softmax of row `row` over this chunk's keys (slots quad*2, +1, +8, +9)
      const bool v00 = quad * 2 < nv_cur, v01 = quad * 2 + 1 < nv_cur;
      const bool v10 = 8 + quad * 2 < nv_cur, v11 = 9 + quad * 2 < nv_cur;
      float mx = fmaxf(fmaxf(v00 ? s[0][0] : -INFINITY, v01 ? s[0][1] : -INFINITY),
                       fmaxf(v10 ? s[1][0] : -INFINITY, v11 ? s[1][1] : -INFINITY));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      const float m_new = fmaxf(m_run, mx * sl2);
      const float m_eff = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m_run - m_eff);  // 0 while m_run = -inf
      const float p00 = v00 ? ex2(fmaf(s[0][0], sl2, -m_eff)) : 0.f;
      const float p01 = v01 ? ex2(fmaf(s[0][1], sl2, -m_eff)) : 0.f;
      const float p10 = v10 ? ex2(fmaf(s[1][0], sl2, -m_eff)) : 0.f;
      const float p11 = v11 ? ex2(fmaf(s[1][1], sl2, -m_eff)) : 0.f;
      float rs = (p00 + p01) + (p10 + p11);
      rs += __shfl_xor_sync(0xFFFFFFFFu, rs, 1);
      rs += __shfl_xor_sync(0xFFFFFFFFu, rs, 2);
      l_run = l_run * alpha + rs;
      m_run = m_new;
#pragma unroll
      for (int n = 0; n < DV / 8; ++n) {
        oacc[n][0] *= alpha;
        oacc[n][1] *= alpha;
      }
      // O += P V: P as A fragments (rows >= 8 are padding), V through ldmatrix.trans
      const uint32_t pa0 = pack_bf16x2(p00, p01), pa2 = pack_bf16x2(p10, p11);
      {
        const int m = lane >> 3;  // matrix: (key half, head-dim half)
        const uint32_t vaddr =
            sb + C::kVOff + ((m & 1) * 8 + (lane & 7)) * C::kVStride + (m >> 1) * 16;
#pragma unroll
        for (int dn = 0; dn < DV / 16; ++dn) {
          uint32_t b0a, b1a, b0b, b1b;
          ldsm_x4_t(vaddr + dn * 32, b0a, b1a, b0b, b1b);
          mma16816(oacc[2 * dn], pa0, 0u, pa2, 0u, b0a, b1a);
          mma16816(oacc[2 * dn + 1], pa0, 0u, pa2, 0u, b0b, b1b);
        }
      }
      __syncwarp();  // the stage is rewritten two chunks from now
      key_cur = key_nxt;
      nv_cur = nv_nxt;
      stage ^= 1;
    }

    // epilogue: O / l (bf16) and LSE (natural log) for the group's real heads
    if (row < G) {
      const int64_t h = static_cast<int64_t>(g) * G + row;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint32_t* orow = reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(a.o) +
                                                   (bi * a.HQ + h) * DV);
#pragma unroll
      for (int n = 0; n < DV / 8; ++n) orow[n * 4 + quad] = pack_bf16x2(oacc[n][0] * inv, oacc[n][1] * inv);
      if (quad == 0) {
        const float m_eff = (m_run == -INFINITY) ? 0.f : m_run;
        a.lse[(static_cast<int64_t>(b) * a.HQ + h) * a.Sq + i] =
            l_run > 0.f ? (m_eff + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      }
    }
    __syncwarp();
  }
}

template <int DQK, int DV>
static int launch_t(const AttnArgs& a, const void* q, const void* k, const void* v,
                    cudaStream_t st) {
  using C = Cfg<DQK, DV>;
  static PerDeviceOnce attr;
  const int rc = once_per_device(attr, [] {
    return cuda_error(cudaFuncSetAttribute(gather_fwd_kernel<DQK, DV>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem),
                      "gather forward smem attribute");
  });
  if (rc) return rc;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t items = static_cast<int64_t>(a.B) * a.Sq * a.HK;
  const int64_t need = (items + kWarps - 1) / kWarps;
  const unsigned grid = static_cast<unsigned>(min64(need, static_cast<int64_t>(sms)));
  record_event(0, st);
  gather_fwd_kernel<DQK, DV><<<grid, kWarps * 32, C::kSmem, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), a);
  record_event(1, st);
  return check_launch("gather forward kernel launch");
}

}  // namespace gather

int launch_fwd_gather(const AttnArgs& a, const void* q, const void* k, const void* v,
                      cudaStream_t st) {
  if (a.mode != SA_MODE_INDEX || !a.bitmap) return SA_ERR_UNSUPPORTED;
  if (a.HQ / a.HK > 8) return SA_ERR_UNSUPPORTED;
  if (a.Dqk == 64 && a.Dv == 64) return gather::launch_t<64, 64>(a, q, k, v, st);
  if (a.Dqk == 128 && a.Dv == 128) return gather::launch_t<128, 128>(a, q, k, v, st);
  if (a.Dqk == 192 && a.Dv == 128) return gather::launch_t<192, 128>(a, q, k, v, st);
  return SA_ERR_UNSUPPORTED;
}

}  // namespace sa
