// topk.cu -- top-k selection over fp32 scores with per-row valid ranges: the producer of
// the int32 index tensor that index-sparse attention consumes.
//
// Operation (xtuner PR #2096, "[Feature] Add optional TileLang Top-K selector", Main
// Changes 1): for each row r of a score matrix, select the k largest scores among the
// columns of its valid range [start_r, end_r), ordered by score (largest first, like
// torch.topk with sorted=True), and return their column indices as int32, with -1 in
// the slots past the number of valid columns.  Selection uses fp32 radix keys.  Ties
// (which torch.topk leaves unordered) go to the smaller column index; -0 equals +0;
// every NaN ranks above +inf.
//
// B200 design: one CTA of 512 threads per row, everything in shared memory.
//  1. Radix select of the k-th largest key in three digit passes (11, 11 and 10 bits):
//     each pass histograms the keys that match the digits fixed so far (shared-memory
//     atomics), and a block-wide scan from the top bin finds the bin holding the k-th
//     key.  Every pass streams the row from global memory (L2 after the first pass)
//     with 16-byte loads, two in flight per thread, so no candidate buffer can
//     overflow and a pass costs about two memory latencies for an 8K-column row.
//  2. Gather: keys above the k-th key are appended in any order.  When every key equal
//     to the k-th is needed (the count the last pass found equals the number still
//     missing, the usual case), those are appended in any order too: the sort puts them
//     in column order.  Otherwise the equal keys are compacted in column order (warp
//     ballots and a prefix over the warps) and only the first `need` of them are kept,
//     so ties resolve to the smaller column.
//  3. Sort of the k winners (as 64-bit (key, ~column) words, descending) and the write
//     of the indices (and optionally the scores).  For 2048 or 4096 words each thread
//     holds E = 4 or 8 consecutive words: every warp sorts its 32 E words with a bitonic
//     network in registers and shuffles, and four merge-path rounds through shared
//     memory (four barriers) merge the 16 warp runs.  The cross-warp bitonic stages this
//     replaces took 10 or 15 barriers, and the sort was 59% of the selector's time
//     (1.80 ms at k = 2048 against 0.74 ms at k = 64).  Other sizes use a plain
//     shared-memory bitonic sort.
// Rows with no more valid columns than k skip step 1 and 2.
#include "sa_device.cuh"
#include "sa_kernels.h"

namespace sa {
namespace topk {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

// Order-preserving map of an fp32 score to an unsigned key (larger score, larger key),
// after mapping -0 to +0 and every NaN to one positive quiet NaN (above +inf).
__device__ __forceinline__ uint32_t score_key(float v) {
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) u = 0x7FC00000u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
// sort word: key in the high half, the complemented column in the low half, so that a
// descending sort orders by score and then by ascending column; 0 (no real key is 0)
// marks an empty slot and sorts last
__device__ __forceinline__ uint64_t word(uint32_t key, int64_t col) {
  return (static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(col));
}

// Calls f(i, key) for every element i < n of the row (any order across threads):
// scalar loads up to the first 16-byte boundary, then float4 loads two per thread per
// iteration, then the scalar tail.
template <class F>
__device__ __forceinline__ void for_each_key(const float* __restrict__ xr, int64_t n, F&& f) {
  const int tid = threadIdx.x;
  int64_t head = static_cast<int64_t>(((16u - (reinterpret_cast<uintptr_t>(xr) & 15u)) & 15u) >> 2);
  if (head > n) head = n;
  if (tid < head) f(static_cast<int64_t>(tid), score_key(__ldg(xr + tid)));
  const float4* x4 = reinterpret_cast<const float4*>(xr + head);
  const int64_t n4 = (n - head) >> 2;
  for (int64_t q = tid; q < n4; q += 2 * kThreads) {
    const float4 a = __ldg(x4 + q);
    const bool has_b = q + kThreads < n4;
    const float4 b = has_b ? __ldg(x4 + q + kThreads) : make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t i = head + 4 * q;
    f(i, score_key(a.x));
    f(i + 1, score_key(a.y));
    f(i + 2, score_key(a.z));
    f(i + 3, score_key(a.w));
    if (has_b) {
      const int64_t ib = i + 4 * kThreads;
      f(ib, score_key(b.x));
      f(ib + 1, score_key(b.y));
      f(ib + 2, score_key(b.z));
      f(ib + 3, score_key(b.w));
    }
  }
  for (int64_t i = head + 4 * n4 + tid; i < n; i += kThreads) f(i, score_key(__ldg(xr + i)));
}

// Descending sort of w[0, 512 * E) (see step 3 above), using tmp[0, 512 * E) as scratch;
// ends with the words back in w and a barrier.
//  1. Each warp sorts its 32 * E words descending with a bitonic network whose
//     compare-exchanges stay in registers (partner in the same thread) or use shuffles
//     (partner in the same warp): no block barrier.
//  2. Merge rounds: runs of L = 32 E, 64 E, ... words are merged pairwise (descending,
//     the first run first among equal words) until one run remains.  Every thread
//     writes E consecutive words of the merged pair: a binary search over the first run
//     finds how many of its words precede the thread's first output (merge path), then
//     E steps merge sequentially.  512 * E / (32 * E) = 16 runs take four rounds, which
//     end in w.
template <int E>
__device__ __forceinline__ void sort_desc_blocked(uint64_t* w, uint64_t* tmp) {
  constexpr int kp = kThreads * E;
  constexpr int kRun = 32 * E;
  const int tid = threadIdx.x, lane = tid & 31;
  uint64_t r[E];
#pragma unroll
  for (int u = 0; u < E; ++u) r[u] = w[tid * E + u];
  for (int size = 2; size <= kRun; size <<= 1) {
    int stride = size >> 1;
    // partners in other lanes of this warp: shuffles
    for (; stride >= E; stride >>= 1) {
      const int lm = stride / E;
      const bool lower = (lane & lm) == 0;
#pragma unroll
      for (int u = 0; u < E; ++u) {
        const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, r[u], lm);
        // the last size sorts every warp's run descending (the merges need that)
        const bool desc = size == kRun || ((tid * E + u) & size) == 0;
        const bool keep_max = lower == desc;
        const uint64_t hi = r[u] > o ? r[u] : o, lo = r[u] > o ? o : r[u];
        r[u] = keep_max ? hi : lo;
      }
    }
    // partners in this thread: registers (strides unrolled at compile time so that the
    // words stay in registers)
#pragma unroll
    for (int sh = 2; sh >= 0; --sh) {
      constexpr int kMaxSh = E == 8 ? 2 : 1;
      if (sh > kMaxSh || (1 << sh) > stride) continue;
      const int st = 1 << sh;
#pragma unroll
      for (int u = 0; u < E; ++u) {
        if (u & st) continue;
        const uint64_t a = r[u], b = r[u + st];
        const bool desc = size == kRun || ((tid * E + u) & size) == 0;
        if (desc ? (a < b) : (a > b)) {
          r[u] = b;
          r[u + st] = a;
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < E; ++u) w[tid * E + u] = r[u];
  __syncthreads();
  uint64_t* src = w;
  uint64_t* dst = tmp;
  for (int L = kRun; L < kp; L <<= 1) {
    const int out0 = tid * E;                 // first output position of this thread
    const int base = out0 & ~(2 * L - 1);     // the pair of runs it falls in
    const int d = out0 - base;                // outputs of the pair before it
    const uint64_t* A = src + base;
    const uint64_t* B = A + L;
    // smallest i such that taking i words of A and d - i of B leaves nothing of A that
    // must come earlier: i == L, or j == 0, or A[i] < B[j - 1]
    int lo = d > L ? d - L : 0, hi = d < L ? d : L;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      const int j = d - mid;
      if (mid < L && j > 0 && A[mid] >= B[j - 1]) lo = mid + 1;
      else hi = mid;
    }
    int i = lo, j = d - lo;
#pragma unroll
    for (int u = 0; u < E; ++u) {
      const bool take_a = j >= L || (i < L && A[i] >= B[j]);
      dst[out0 + u] = take_a ? A[i] : B[j];
      i += take_a ? 1 : 0;
      j += take_a ? 0 : 1;
    }
    __syncthreads();
    uint64_t* t = src;
    src = dst;
    dst = t;
  }
  static_assert(kp / kRun == 16, "four merge rounds end in w");
}

__global__ void __launch_bounds__(kThreads, 4)
    topk_kernel(const float* __restrict__ x, int64_t ld, int64_t cols,
                const int32_t* __restrict__ starts, const int32_t* __restrict__ ends, int k,
                int kp, int32_t* __restrict__ out_idx, float* __restrict__ out_val,
                int32_t* status) {
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t found[3];  // bin holding the k-th key, keys above it, keys in it
  __shared__ uint32_t n_gt;
  extern __shared__ uint64_t sel[];  // kp sort words, then kp words of merge scratch

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = blockIdx.x;
  int64_t st = starts ? static_cast<int64_t>(__ldg(starts + row)) : 0;
  int64_t en = ends ? static_cast<int64_t>(__ldg(ends + row)) : cols;
  if (st < 0 || en > cols || st > en) {
    if (tid == 0) report_status(status, kStatusIndex);
    st = en = 0;
  }
  const int64_t n = en - st;
  const float* xr = x + row * ld + st;
  for (int i = tid; i < kp; i += kThreads) sel[i] = 0ull;
  __syncthreads();

  if (n <= k) {
    for (int64_t i = tid; i < n; i += kThreads) sel[i] = word(score_key(__ldg(xr + i)), st + i);
  } else {
    // ---- radix select of the k-th largest key
    uint32_t prefix = 0u, pmask = 0u;
    uint32_t need = static_cast<uint32_t>(k), n_eq = 0u;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nb = pass < 2 ? 2048 : 1024;
      for (int bq = tid; bq < nb; bq += kThreads) hist[bq] = 0u;
      __syncthreads();
      for_each_key(xr, n, [&](int64_t, uint32_t key) {
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
      });
      __syncthreads();
      // bins in descending order: thread t owns ranks [4t, 4t+4) (rank r = bin nb-1-r)
      const int per = nb / kThreads;  // 4 or 2
      uint32_t c[4], s = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[e] = e < per ? hist[nb - 1 - (tid * per + e)] : 0u;
        s += c[e];
      }
      // exclusive prefix of s over threads (in rank order)
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) wsum[warp] = incl;
      __syncthreads();
      uint32_t above = incl - s;
      for (int w = 0; w < warp; ++w) above += wsum[w];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (e < per && above < need && above + c[e] >= need) {
          found[0] = static_cast<uint32_t>(nb - 1 - (tid * per + e));
          found[1] = above;
          found[2] = c[e];
        }
        above += c[e];
      }
      __syncthreads();
      prefix |= found[0] << shift;
      pmask |= static_cast<uint32_t>(nb - 1) << shift;
      need -= found[1];
      n_eq = found[2];  // after the last pass: the number of keys equal to the k-th
      __syncthreads();  // found[] and wsum[] are rewritten by the next pass
    }
    // ---- gather: keys above the threshold in any order, equal keys in column order
    const uint32_t thr = prefix;
    const uint32_t base_eq = static_cast<uint32_t>(k) - need;
    if (tid == 0) n_gt = 0u;
    __syncthreads();
    if (n_eq == need) {
      // every key >= the k-th is selected: append in any order
      for_each_key(xr, n, [&](int64_t i, uint32_t key) {
        if (key >= thr) sel[atomicAdd(&n_gt, 1u)] = word(key, st + i);
      });
    } else {
    uint32_t eq_seen = 0u;  // equal keys in the chunks before this one (uniform)
    for (int64_t c0 = 0; c0 < n; c0 += kThreads) {
      const int64_t i = c0 + tid;
      const uint32_t key = i < n ? score_key(__ldg(xr + i)) : 0u;
      if (key > thr) sel[atomicAdd(&n_gt, 1u)] = word(key, st + i);
      const bool eq = i < n && key == thr;
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, eq);
      if (lane == 0) wsum[warp] = __popc(bal);
      __syncthreads();
      uint32_t off = 0u, tot = 0u;
      for (int w = 0; w < kWarps; ++w) {
        const uint32_t v = wsum[w];
        off += w < warp ? v : 0u;
        tot += v;
      }
      if (eq) {
        const uint32_t r = eq_seen + off + __popc(bal & ((1u << lane) - 1u));
        if (r < need) sel[base_eq + r] = word(thr, st + i);
      }
      eq_seen += tot;
      __syncthreads();  // wsum[] is rewritten by the next chunk
    }
    }
  }
  __syncthreads();

  // ---- bitonic sort of sel[0, ks), descending (ks: kp, or the power of two that
  // holds a short row's n entries; the slots past them are empty and stay last)
  int ks = kp;
  if (n < k) {
    ks = 2;
    while (ks < n) ks <<= 1;
  }
  if (ks == 4 * kThreads) {
    sort_desc_blocked<4>(sel, sel + kp);
  } else if (ks == 8 * kThreads) {
    sort_desc_blocked<8>(sel, sel + kp);
  } else {
    for (int size = 2; size <= ks; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int t = tid; t < (ks >> 1); t += kThreads) {
          const int i = 2 * t - (t & (stride - 1));
          const int j = i + stride;
          const uint64_t a = sel[i], b = sel[j];
          const bool desc = (i & size) == 0;
          if (desc ? (a < b) : (a > b)) {
            sel[i] = b;
            sel[j] = a;
          }
        }
        __syncthreads();
      }
    }
  }

  const int64_t valid = n < k ? n : k;
  for (int i = tid; i < k; i += kThreads) {
    const uint64_t wv = sel[i];
    const bool ok = i < valid;
    out_idx[row * k + i] = ok ? static_cast<int32_t>(~static_cast<uint32_t>(wv)) : -1;
    if (out_val) out_val[row * k + i] = ok ? key_score(static_cast<uint32_t>(wv >> 32)) : -INFINITY;
  }
}

}  // namespace topk
}  // namespace sa

using namespace sa;

extern "C" int topk_select(const float* scores, int64_t rows, int64_t cols, int64_t ld,
                           const int32_t* starts, const int32_t* ends, int32_t k,
                           int32_t* out_idx, float* out_val, int32_t* dev_status,
                           sa_stream_t stream) {
  if (rows < 0 || cols < 0 || ld < cols || k < 1 || k > SA_TOPK_MAX_K) return SA_ERR_INVALID;
  if (cols > 0x7FFFFFFFll || rows > 0x7FFFFFFFll) return SA_ERR_INVALID;
  if (rows == 0) return SA_OK;
  if (!scores || !out_idx) return SA_ERR_INVALID;
  int kp = 2;
  while (kp < k) kp <<= 1;
  const size_t smem = 2 * static_cast<size_t>(kp) * sizeof(uint64_t);  // words + merge scratch
  const int drc = check_stream_device(reinterpret_cast<cudaStream_t>(stream));
  if (drc) return drc;
  static PerDeviceOnce attr;
  const int rc = once_per_device(attr, [] {
    return cuda_error(cudaFuncSetAttribute(topk::topk_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           2 * SA_TOPK_MAX_K * static_cast<int>(sizeof(uint64_t))),
                      "top-k smem attribute");
  });
  if (rc) return rc;
  topk::topk_kernel<<<static_cast<unsigned>(rows), topk::kThreads, smem,
                      reinterpret_cast<cudaStream_t>(stream)>>>(scores, ld, cols, starts, ends, k, kp,
                                                               out_idx, out_val, dev_status);
  return check_launch("top-k kernel launch");
}
