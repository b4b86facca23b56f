// converter.cu -- token-level top-k indices or block masks -> per-tile lists.
//
// MagiAttention PR #334, section 2: index_attn_indices_to_block_sparse turns indices
// (total_q, NHK, topk) into block-level lists through a presence matrix built with a
// scatter, and prepare_block_sparse_bwd_loopk normalises them per M-block.
// MagiAttention PR #331, "CSR Tile Mapping": the transposed key-to-query lists used by
// the backward.
//
// B200 design: the presence matrix is a packed bitmap built one (row, KV head) per CTA
// in shared memory (no global atomics, one coalesced store per row); classification
// reads the bitmap once, coalesced; the lists are compacted with warp ballots.  The
// class array is written into the forward-list buffer and compacted in place, so the
// conversion needs no workspace.  All of it is integer work bound by HBM bandwidth.
#include "sa_device.cuh"
#include "sa_kernels.h"

namespace sa {

constexpr int kAbsent = 0, kPartial = 1, kFull = 2;

// One CTA of kScatterThreads per (b, i, g): the W-word presence row of query i under KV
// head g.  Every thread's index loads are issued before any of their bits is set (16-byte
// loads when the rows allow), so a row costs one memory latency, not one per index.
constexpr int kScatterThreads = 128;
constexpr int kScatterUnroll = 4;

__device__ __forceinline__ void set_presence_bit(uint32_t* words, int32_t j, int64_t Sk,
                                                 int32_t* status) {
  if (j == -1) return;
  if (j < -1 || j >= Sk) {
    report_status(status, kStatusIndex);
    return;
  }
  atomicOr(&words[j >> 5], 1u << (j & 31));
}

__global__ void __launch_bounds__(kScatterThreads)
    scatter_bits_kernel(const int32_t* __restrict__ idx, uint32_t* __restrict__ bitmap,
                        int64_t Sq, int64_t Sk, int HK, int topk, int W, int vec,
                        int32_t* status) {
  extern __shared__ uint32_t words[];
  const int64_t row = blockIdx.x;  // ((b * Sq) + i) * HK + g, the order of idx
  const int g = static_cast<int>(row % HK);
  const int64_t bi = row / HK;  // b * Sq + i
  const int64_t b = bi / Sq, i = bi % Sq;
  for (int w = threadIdx.x; w < W; w += kScatterThreads) words[w] = 0u;
  __syncthreads();
  const int32_t* src = idx + row * topk;
  if (vec) {  // topk % 4 == 0 and a 16-byte aligned base: rows of int4
    const int4* s4 = reinterpret_cast<const int4*>(src);
    const int n4 = topk >> 2;
    for (int base = 0; base < n4; base += kScatterUnroll * kScatterThreads) {
      int4 v[kScatterUnroll];
#pragma unroll
      for (int u = 0; u < kScatterUnroll; ++u) {
        const int e = base + u * kScatterThreads + threadIdx.x;
        v[u] = e < n4 ? __ldg(s4 + e) : make_int4(-1, -1, -1, -1);
      }
#pragma unroll
      for (int u = 0; u < kScatterUnroll; ++u) {
        set_presence_bit(words, v[u].x, Sk, status);
        set_presence_bit(words, v[u].y, Sk, status);
        set_presence_bit(words, v[u].z, Sk, status);
        set_presence_bit(words, v[u].w, Sk, status);
      }
    }
  } else {
    for (int base = 0; base < topk; base += kScatterUnroll * kScatterThreads) {
      int32_t v[kScatterUnroll];
#pragma unroll
      for (int u = 0; u < kScatterUnroll; ++u) {
        const int t = base + u * kScatterThreads + threadIdx.x;
        v[u] = t < topk ? __ldg(src + t) : -1;
      }
#pragma unroll
      for (int u = 0; u < kScatterUnroll; ++u) set_presence_bit(words, v[u], Sk, status);
    }
  }
  __syncthreads();
  uint32_t* dst = bitmap + (((b * HK + g) * Sq) + i) * static_cast<int64_t>(W);
  for (int w = threadIdx.x; w < W; w += kScatterThreads) dst[w] = words[w];
}

// Bits of the 32 keys [j0, j0 + 32) of query i that are allowed: set in the presence
// word, below Sk and, when causal, at most i.  `in_range` receives the bits below Sk.
__device__ __forceinline__ uint32_t allowed_bits(uint32_t bits, int64_t i, int64_t j0, int64_t Sk,
                                                 int causal, uint32_t& in_range) {
  const int64_t n_in = min64(32, Sk - j0);
  in_range = n_in >= 32 ? 0xFFFFFFFFu : (n_in <= 0 ? 0u : ((1u << n_in) - 1u));
  const int64_t n_c = causal ? min64(32, max64(0, i + 1 - j0)) : 32;
  const uint32_t causal_ok = n_c >= 32 ? 0xFFFFFFFFu : ((1u << n_c) - 1u);
  return bits & in_range & causal_ok;
}

// One CTA per (b, g, mt): classify every key tile of the query tile from the bitmap.  A
// key tile is 4 words of a row: with W % 4 == 0 each thread reads one (row, key tile)
// as a 16-byte load.
__global__ void classify_index_kernel(const uint32_t* __restrict__ bitmap, int32_t* __restrict__ cls,
                                      int64_t Sq, int64_t Sk, int HK, int Tm, int Tn, int W,
                                      int causal, int vec) {
  extern __shared__ int32_t flags[];  // any[Tn], all[Tn]
  int32_t* any_f = flags;
  int32_t* all_f = flags + Tn;
  const int mt = blockIdx.x % Tm;
  const int64_t bg = blockIdx.x / Tm;
  for (int t = threadIdx.x; t < Tn; t += blockDim.x) {
    any_f[t] = 0;
    all_f[t] = 1;
  }
  __syncthreads();
  const int64_t i0 = static_cast<int64_t>(mt) * kTile;
  const int rows = static_cast<int>(min64(kTile, Sq - i0));
  constexpr int kWordsPerTile = kTile / 32;
  if (vec) {
    // one (row, key tile) per element; rows are W words apart (W % 4 == 0 and a 16-byte
    // aligned bitmap keep every load aligned)
    for (int e = threadIdx.x; e < rows * Tn; e += blockDim.x) {
      const int r = e / Tn, nt = e - (e / Tn) * Tn;
      const int64_t i = i0 + r;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(bitmap + (bg * Sq + i) * W) + nt);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      bool any = false, all = true;
#pragma unroll
      for (int k = 0; k < kWordsPerTile; ++k) {
        uint32_t in_range;
        const uint32_t allowed = allowed_bits(
            wv[k], i, static_cast<int64_t>(nt) * kTile + 32 * k, Sk, causal, in_range);
        any |= allowed != 0u;
        all &= allowed == in_range;
      }
      if (any) any_f[nt] = 1;
      if (!all) all_f[nt] = 0;
    }
  } else {
    for (int e = threadIdx.x; e < rows * W; e += blockDim.x) {
      const int r = e / W, w = e % W;
      const int64_t i = i0 + r;
      const uint32_t bits = __ldg(bitmap + (bg * Sq + i) * W + w);
      // FULL needs every in-range bit allowed
      uint32_t in_range;
      const uint32_t allowed = allowed_bits(bits, i, 32 * static_cast<int64_t>(w), Sk, causal,
                                            in_range);
      const int nt = w / kWordsPerTile;
      if (allowed) any_f[nt] = 1;
      if (allowed != in_range) all_f[nt] = 0;
    }
  }
  __syncthreads();
  for (int nt = threadIdx.x; nt < Tn; nt += blockDim.x) {
    const bool full = all_f[nt] && static_cast<int64_t>(nt + 1) * kTile <= Sk;
    cls[(bg * Tm + mt) * static_cast<int64_t>(Tn) + nt] =
        any_f[nt] ? (full ? kFull : kPartial) : kAbsent;
  }
}

// One thread per (b, g, mt, nt): classify a tile of block or dense mode analytically
// from its bs x bs sub-blocks (bs divides the tile edge).
__global__ void classify_block_kernel(const uint8_t* __restrict__ mask, int32_t* __restrict__ cls,
                                      int64_t Sq, int64_t Sk, int64_t n_tiles, int Tm, int Tn,
                                      int bs, int Mb, int Nb, int causal) {
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (t >= n_tiles) return;
  const int nt = static_cast<int>(t % Tn);
  const int mt = static_cast<int>((t / Tn) % Tm);
  const int64_t bg = t / (static_cast<int64_t>(Tn) * Tm);
  bool any = false, all = true;
  for (int64_t r0 = static_cast<int64_t>(mt) * kTile; r0 < static_cast<int64_t>(mt + 1) * kTile;
       r0 += bs) {
    if (r0 >= Sq) break;
    const int64_t r1 = min64(r0 + bs, Sq);
    for (int64_t c0 = static_cast<int64_t>(nt) * kTile; c0 < static_cast<int64_t>(nt + 1) * kTile;
         c0 += bs) {
      if (c0 >= Sk) break;
      const int64_t c1 = min64(c0 + bs, Sk);
      const bool m = mask == nullptr ||
                     __ldg(mask + (bg * Mb + r0 / bs) * static_cast<int64_t>(Nb) + c0 / bs) != 0;
      const bool some = m && (!causal || c0 <= r1 - 1);
      const bool every = m && (!causal || c1 - 1 <= r0);
      any |= some;
      all &= every;
    }
  }
  if (static_cast<int64_t>(nt + 1) * kTile > Sk) all = false;
  cls[t] = any ? (all ? kFull : kPartial) : kAbsent;
}

// Ascending compaction of `n` classes read through `get` into out[0..n): FULL entries
// first, then PARTIAL, then -1.  One warp; returns (n_full, n_partial) in lane 0.
template <class Get>
__device__ __forceinline__ void warp_compact(Get get, int n, int32_t* out, int32_t* counts) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  int n_full = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const int want = pass == 0 ? kFull : kPartial;
    for (int c0 = 0; c0 < n; c0 += 32) {
      const int e = c0 + lane;
      const bool hit = e < n && get(e) == want;
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, hit);
      if (hit) out[base + __popc(m & ((1u << lane) - 1u))] = e;
      base += __popc(m);
    }
    if (pass == 0) n_full = base;
  }
  for (int e = base + lane; e < n; e += 32) out[e] = -1;
  if (lane == 0) {
    counts[0] = n_full;
    counts[1] = base - n_full;
  }
}

// One warp per (b, g, nt): the transposed list over query tiles, from the class array.
__global__ void transpose_lists_kernel(const int32_t* __restrict__ cls, int32_t* __restrict__ tidx,
                                       int32_t* __restrict__ tcnt, int Tm, int Tn) {
  const int nt = blockIdx.x % Tn;
  const int64_t bg = blockIdx.x / Tn;
  const int32_t* col = cls + bg * Tm * static_cast<int64_t>(Tn) + nt;
  warp_compact([&](int mt) { return __ldg(col + static_cast<int64_t>(mt) * Tn); }, Tm,
               tidx + (bg * Tn + nt) * static_cast<int64_t>(Tm), tcnt + (bg * Tn + nt) * 2);
}

// One warp per (b, g, mt): the forward list, compacted in place over the class row.
__global__ void compact_lists_kernel(int32_t* __restrict__ idx, int32_t* __restrict__ cnt, int Tn) {
  extern __shared__ int8_t row_cls[];
  const int64_t r = blockIdx.x;
  int32_t* row = idx + r * Tn;
  for (int e = threadIdx.x; e < Tn; e += 32) row_cls[e] = static_cast<int8_t>(row[e]);
  __syncwarp();
  warp_compact([&](int e) { return static_cast<int>(row_cls[e]); }, Tn, row, cnt + r * 2);
}

}  // namespace sa

using namespace sa;

static int launch_lists(sa_block_sparse* s, int Tm, int Tn, cudaStream_t st) {
  const int64_t BG = static_cast<int64_t>(s->B) * s->HK;
  transpose_lists_kernel<<<static_cast<unsigned>(BG * Tn), 32, 0, st>>>(s->idx, s->tidx, s->tcnt,
                                                                        Tm, Tn);
  compact_lists_kernel<<<static_cast<unsigned>(BG * Tm), 32, Tn, st>>>(s->idx, s->cnt, Tn);
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

static int check_lists(const sa_block_sparse* s) {
  if (!s || s->B <= 0 || s->HK <= 0 || s->Sq <= 0 || s->Sk <= 0) return SA_ERR_INVALID;
  if (!s->cnt || !s->idx || !s->tcnt || !s->tidx) return SA_ERR_INVALID;
  const int64_t Tm = (s->Sq + kTile - 1) / kTile, Tn = (s->Sk + kTile - 1) / kTile;
  if (Tm > (1 << 20) || Tn > 8192) return SA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->B) * s->HK * Tm * Tn > (int64_t(1) << 31)) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

extern "C" int index_to_block_sparse(const int32_t* idx, int32_t topk, sa_block_sparse* out,
                                     int32_t* dev_status, sa_stream_t stream) {
  int rc = check_lists(out);
  if (rc) return rc;
  if (!idx || topk <= 0 || !out->bitmap) return SA_ERR_INVALID;
  const int64_t W = (out->Sk + 31) / 32;
  if (W * 4 > 96 * 1024) return SA_ERR_UNSUPPORTED;  // one presence row in shared memory
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = check_stream_device(st);
  if (rc) return rc;
  out->mode = SA_MODE_INDEX;
  const int Tm = static_cast<int>((out->Sq + kTile - 1) / kTile);
  const int Tn = static_cast<int>((out->Sk + kTile - 1) / kTile);
  const int64_t rows = static_cast<int64_t>(out->B) * out->Sq * out->HK;
  if (rows > 0x7FFFFFFF) return SA_ERR_UNSUPPORTED;
  const size_t smem_bits = static_cast<size_t>(W) * 4;
  if (smem_bits > 48 * 1024 &&
      cudaFuncSetAttribute(scatter_bits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem_bits)) != cudaSuccess)
    return SA_ERR_CUDA;
  const int vec = (topk % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
  scatter_bits_kernel<<<static_cast<unsigned>(rows), kScatterThreads, smem_bits, st>>>(
      idx, out->bitmap, out->Sq, out->Sk, out->HK, topk, static_cast<int>(W), vec, dev_status);
  const int64_t BG = static_cast<int64_t>(out->B) * out->HK;
  classify_index_kernel<<<static_cast<unsigned>(BG * Tm), 256, 2 * Tn * sizeof(int32_t), st>>>(
      out->bitmap, out->idx, out->Sq, out->Sk, out->HK, Tm, Tn, static_cast<int>(W), out->causal,
      static_cast<int>(W % 4 == 0 && reinterpret_cast<uintptr_t>(out->bitmap) % 16 == 0));
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  return launch_lists(out, Tm, Tn, st);
}

extern "C" int block_mask_to_block_sparse(sa_block_sparse* out, sa_stream_t stream) {
  int rc = check_lists(out);
  if (rc) return rc;
  if (out->mode == SA_MODE_BLOCK) {
    if (!out->mask) return SA_ERR_INVALID;
    if (out->bs != 64 && out->bs != 128) return SA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(out->Mb) * out->bs < out->Sq ||
        static_cast<int64_t>(out->Nb) * out->bs < out->Sk)
      return SA_ERR_INVALID;
  } else if (out->mode == SA_MODE_DENSE) {
    out->bs = kTile;
    out->Mb = out->Nb = 0;
  } else {
    return SA_ERR_INVALID;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rc = check_stream_device(st);
  if (rc) return rc;
  const int Tm = static_cast<int>((out->Sq + kTile - 1) / kTile);
  const int Tn = static_cast<int>((out->Sk + kTile - 1) / kTile);
  const int64_t n_tiles = static_cast<int64_t>(out->B) * out->HK * Tm * Tn;
  classify_block_kernel<<<static_cast<unsigned>((n_tiles + 255) / 256), 256, 0, st>>>(
      out->mode == SA_MODE_BLOCK ? out->mask : nullptr, out->idx, out->Sq, out->Sk, n_tiles, Tm,
      Tn, out->bs, out->Mb, out->Nb, out->causal);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  return launch_lists(out, Tm, Tn, st);
}
