// bwd_noalloc.cu -- sparse_attn_bwd_noalloc: the backward without a caller workspace.
//
// Some callers cannot call cudaMalloc (or hand this library a workspace): code that
// runs inside a host framework which owns every device allocation and passes only
// input and output tensors (a plugin or a serving backend), or latency-critical loops
// where cudaMalloc's implicit device synchronisation is not acceptable.  For them this
// entry point runs exactly the same kernels as sparse_attn_bwd, with the backward's
// scratch (fp32 Delta and the fp32 dQ accumulator) taken from a fixed, file-scope
// device array instead of a caller-provided buffer.
//
// Properties a caller must know:
//  - The array has SA_NOALLOC_SCRATCH_BYTES bytes; every GPU that loads this library
//    holds it until the process exits.  Problems whose scratch
//    (sparse_attn_bwd_workspace_size) exceeds it are rejected with
//    SA_ERR_SCRATCH_LIMIT before anything is enqueued.
//  - The first call on each device looks up the array's device address with
//    cudaGetSymbolAddress (with that device current; a failed lookup is retried by the
//    next call).  Make that first call before any stream capture.
//  - The array used is the current device's, so `stream` must belong to the current
//    device (checked: SA_ERR_DEVICE otherwise).
//  - Every call on a device shares the one array, and each call overwrites it (the
//    preprocess kernel writes Delta and zeroes the dQ accumulator before use).  Calls
//    whose work overlaps on the GPU (different streams without ordering, or several
//    host threads) race on it: serialise them.
//  - Nothing here allocates: no cudaMalloc, cudaFree or allocating library routine.
#include <mutex>

#include "sa_device.cuh"
#include "sa_kernels.h"

namespace {

constexpr int kMaxDevices = 64;

// In host code this name is only a host-side stand-in for the device array: its
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_bwd_scratch[SA_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices];  // guarded by g_scratch_mutex; null until a lookup succeeds

// Device address of the scratch array on the current device `device`.  The address is
// stored only once a lookup has succeeded, so a lookup that failed (made during a
// stream capture, say) is retried by the next call.
cudaError_t scratch_address(int device, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[device]) {
    void* p = nullptr;
    const cudaError_t rc = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (rc != cudaSuccess) return rc;
    g_scratch_ptr[device] = p;
  }
  *out = g_scratch_ptr[device];
  return cudaSuccess;
}

}  // namespace

extern "C" int sparse_attn_bwd_noalloc(const sparse_attn_params* p, sa_stream_t stream) {
  if (!p) return SA_ERR_INVALID;
  const size_t need = sparse_attn_bwd_workspace_size(p);
  if (need == 0) return SA_ERR_INVALID;
  if (need > static_cast<size_t>(SA_NOALLOC_SCRATCH_BYTES)) return SA_ERR_SCRATCH_LIMIT;
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices)
    return SA_ERR_CUDA;
  // the scratch used is the current device's: the stream must belong to that device
  const int drc = sa::check_stream_device(reinterpret_cast<cudaStream_t>(stream));
  if (drc) return drc;
  void* scratch = nullptr;
  if (scratch_address(device, &scratch) != cudaSuccess || scratch == nullptr) return SA_ERR_CUDA;
  return sparse_attn_bwd(p, scratch, static_cast<size_t>(SA_NOALLOC_SCRATCH_BYTES), stream);
}
