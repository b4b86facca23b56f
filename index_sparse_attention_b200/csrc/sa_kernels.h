// sa_kernels.h -- host-side launch interface shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "sparse_attn.h"

namespace sa {

// Everything a forward or backward launch needs besides the TMA tensor maps.
struct AttnArgs {
  void* o;               // bf16 [B][Sq][HQ][Dv]
  float* lse;            // fp32 [B][HQ][Sq]
  const void* dout;      // bf16 [B][Sq][HQ][Dv]
  void* dq;              // bf16 [B][Sq][HQ][Dqk]
  void* dk;              // bf16 [B][Sk][HK][Dqk]
  void* dv;              // bf16 [B][Sk][HK][Dv]
  float* delta;          // fp32 [B][HQ][Sq]   (backward workspace)
  float* dq_acc;         // fp32 [B][Sq][HQ][Dqk] (backward workspace)
  const int32_t* cnt;    // forward lists
  const int32_t* idx;
  const int32_t* tcnt;   // backward (transposed) lists
  const int32_t* tidx;
  const uint8_t* mask;   // block mode, bs = 64 partial tiles
  const uint32_t* bitmap;  // index mode
  int64_t Sq, Sk;
  int B, HQ, HK, Dqk, Dv;
  int Tm, Tn, W;
  int mode, causal, bs, Mb, Nb;
  float scale;       // softmax_scale
  float scale_log2;  // softmax_scale * log2(e)
  int32_t* status;
  // deterministic backward: dQ contributions to each (b, query head, query tile, dQ
  // column part) are added in ascending key-tile order, sequenced by sem
  // [B][HQ][Tm][2] (backward workspace, zeroed by the preprocess)
  int det;
  int32_t* sem;
  // limit of every bounded wait of the launch (ns); kWaitLimitNs unless a test shortened
  // it through sparse_attn_set_wait_limit_ns
  uint64_t wait_limit_ns;
};

// Wait limit for the next launches (0: the default); see sparse_attn_set_wait_limit_ns.
extern std::atomic<uint64_t> g_wait_limit_ns;
// Forward form (SA_FWD_FORM_*); see sparse_attn_set_forward_form.
extern std::atomic<int> g_fwd_form;

struct TensorMaps {
  CUtensorMap q, k, v, dout, dq_acc, dk, dv, o;
  CUtensorMap kh;  // forward: K in 64-row boxes (the half tile of a CTA pair)
};

// Caller-owned events recorded around the launches (see sparse_attn_set_timing_events);
// nullptr when instrumentation is off.
extern cudaEvent_t* g_timing_events;
inline void record_event(int k, cudaStream_t st) {
  if (g_timing_events) cudaEventRecord(g_timing_events[k], st);
}

// Turns a CUDA error into SA_ERR_CUDA; with SA_DEBUG set in the environment it also
// prints which call failed and why.
int cuda_error(cudaError_t e, const char* what);
inline int check_launch(const char* what) { return cuda_error(cudaGetLastError(), what); }

// Runs `set` (a cudaFuncSetAttribute call and the like) once per device: a flag bit per
// device index (< 64), set only when `set` returns SA_OK, so a failure is retried on
// the next call; thread-safe.  Device = the current device.
struct PerDeviceOnce {
  std::atomic<uint64_t> done{0};
  std::mutex m;
};
template <class F>
inline int once_per_device(PerDeviceOnce& o, F&& set) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SA_ERR_CUDA;
  const uint64_t bit = 1ull << dev;
  if (o.done.load(std::memory_order_acquire) & bit) return SA_OK;
  std::lock_guard<std::mutex> lock(o.m);
  if (o.done.load(std::memory_order_relaxed) & bit) return SA_OK;
  const int rc = set();
  if (rc == SA_OK) o.done.fetch_or(bit, std::memory_order_release);
  return rc;
}

// Every kernel is launched on the current device.  A stream created on another device
// is refused with SA_ERR_DEVICE before anything is enqueued (the legacy and per-thread
// default streams always belong to the current device).
inline int check_stream_device(cudaStream_t st) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return SA_ERR_CUDA;
  if (st == nullptr || st == cudaStreamLegacy || st == cudaStreamPerThread) return SA_OK;
  int sd = -1;
  if (cudaStreamGetDevice(st, &sd) != cudaSuccess) return SA_ERR_CUDA;
  return sd == cur ? SA_OK : SA_ERR_DEVICE;
}

int launch_fwd(const AttnArgs& a, const TensorMaps& m, cudaStream_t st);
int launch_bwd(const AttnArgs& a, const TensorMaps& m, cudaStream_t st);
int launch_bwd_pair(const AttnArgs& a, const TensorMaps& m, cudaStream_t st);

}  // namespace sa
