// api.cu -- the C ABI of libsparse_attn.so: argument checks, TMA tensor maps and the
// launches of the forward and backward kernels.  No device memory is allocated here.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "sa_device.cuh"
#include "sa_kernels.h"

using namespace sa;

namespace sa {
int cuda_error(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SA_OK;
  if (std::getenv("SA_DEBUG"))
    std::fprintf(stderr, "sparse_attn: %s: %s (%s)\n", what, cudaGetErrorName(e),
                 cudaGetErrorString(e));
  return SA_ERR_CUDA;
}
cudaEvent_t* g_timing_events = nullptr;
static cudaEvent_t g_events_copy[6];
std::atomic<uint64_t> g_wait_limit_ns{0};
std::atomic<int> g_fwd_form{SA_FWD_FORM_AUTO};
std::atomic<int> g_bwd_form{SA_BWD_FORM_AUTO};  // read by launch_bwd (bwd.cu)
}  // namespace sa

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D map over a [B][S][H][D] bf16 tensor with 64 x box_rows (D x S) boxes, 128-byte
// swizzle.  Out-of-range rows (and columns) read as zeros.
bool make_map(CUtensorMap* m, const void* base, int D, int64_t S, int H, int B, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(H) * D * 2, static_cast<cuuint64_t>(D) * 2,
                           static_cast<cuuint64_t>(S) * H * D * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D map over the fp32 dQ accumulator [B][Sq][HQ][D] with 64 x 32 (D x S) boxes, no
// swizzle: the target of the backward's bulk reduce-adds.
bool make_map_f32(CUtensorMap* m, const void* base, int D, int64_t S, int H, int B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(H) * D * 4, static_cast<cuuint64_t>(D) * 4,
                           static_cast<cuuint64_t>(S) * H * D * 4};
  cuuint32_t box[4] = {64, 32, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dims_supported(int dqk, int dv) {
  return (dqk == 64 && dv == 64) || (dqk == 128 && dv == 128) || (dqk == 192 && dv == 128) ||
         (dqk == 256 && dv == 256);
}

int fill_args(const sparse_attn_params* p, AttnArgs* a, bool backward) {
  if (!p || !p->sparse) return SA_ERR_INVALID;
  const sa_block_sparse* s = p->sparse;
  if (!p->q || !p->k || !p->v || !p->o || !p->lse) return SA_ERR_INVALID;
  if (backward && (!p->dout || !p->dq || !p->dk || !p->dv)) return SA_ERR_INVALID;
  if (p->B <= 0 || p->HQ <= 0 || p->HK <= 0 || p->Sq <= 0 || p->Sk <= 0) return SA_ERR_INVALID;
  if (p->HQ % p->HK != 0) return SA_ERR_INVALID;
  if (!dims_supported(p->Dqk, p->Dv)) return SA_ERR_UNSUPPORTED;
  if (s->B != p->B || s->HK != p->HK || s->Sq != p->Sq || s->Sk != p->Sk) return SA_ERR_INVALID;
  if (!s->cnt || !s->idx || !s->tcnt || !s->tidx) return SA_ERR_INVALID;
  if (s->mode == SA_MODE_INDEX && !s->bitmap) return SA_ERR_INVALID;
  if (s->mode == SA_MODE_BLOCK && (!s->mask || (s->bs != 64 && s->bs != 128)))
    return SA_ERR_INVALID;
  if (s->mode != SA_MODE_DENSE && s->mode != SA_MODE_BLOCK && s->mode != SA_MODE_INDEX)
    return SA_ERR_INVALID;
  if (!(p->softmax_scale > 0.f)) return SA_ERR_INVALID;
  const int64_t Tm = (p->Sq + kTile - 1) / kTile, Tn = (p->Sk + kTile - 1) / kTile;
  if (Tm > 65535 * 32 || Tn > 8192 || p->HQ > 65535 || p->B > 65535) return SA_ERR_UNSUPPORTED;
  if (p->Sq > 0x7FFFFFFF || p->Sk > 0x7FFFFFFF) return SA_ERR_UNSUPPORTED;
  const void* ptrs[] = {p->q, p->k, p->v, p->o};
  for (const void* q : ptrs)
    if (!aligned16(q)) return SA_ERR_ALIGN;
  if (backward) {
    const void* bp[] = {p->dout, p->dq, p->dk, p->dv};
    for (const void* q : bp)
      if (!aligned16(q)) return SA_ERR_ALIGN;
  }
  *a = AttnArgs{};
  a->o = p->o;
  a->lse = p->lse;
  a->dout = p->dout;
  a->dq = p->dq;
  a->dk = p->dk;
  a->dv = p->dv;
  a->cnt = s->cnt;
  a->idx = s->idx;
  a->tcnt = s->tcnt;
  a->tidx = s->tidx;
  a->mask = s->mode == SA_MODE_BLOCK ? s->mask : nullptr;
  a->bitmap = s->mode == SA_MODE_INDEX ? s->bitmap : nullptr;
  a->Sq = p->Sq;
  a->Sk = p->Sk;
  a->B = p->B;
  a->HQ = p->HQ;
  a->HK = p->HK;
  a->Dqk = p->Dqk;
  a->Dv = p->Dv;
  a->Tm = static_cast<int>(Tm);
  a->Tn = static_cast<int>(Tn);
  a->W = static_cast<int>((p->Sk + 31) / 32);
  a->mode = s->mode;
  a->causal = s->causal ? 1 : 0;
  a->bs = s->mode == SA_MODE_BLOCK ? s->bs : kTile;
  a->Mb = s->Mb;
  a->Nb = s->Nb;
  a->scale = p->softmax_scale;
  a->scale_log2 = p->softmax_scale * 1.4426950408889634f;
  a->status = p->dev_status;
  const uint64_t lim = g_wait_limit_ns.load(std::memory_order_relaxed);
  a->wait_limit_ns = lim ? lim : kWaitLimitNs;
  return SA_OK;
}

// Forward: Q in 128-row boxes, K also in 64-row boxes (CTA pairs load half tiles).
// Backward: Q and dO in 64-row boxes (the backward consumes query tiles in 64-row
// halves).  K and V: 128-row boxes.
int fill_maps(const sparse_attn_params* p, TensorMaps* m, bool backward) {
  const int qrows = backward ? 64 : 128;
  if (!make_map(&m->q, p->q, p->Dqk, p->Sq, p->HQ, p->B, qrows)) return SA_ERR_CUDA;
  if (!make_map(&m->k, p->k, p->Dqk, p->Sk, p->HK, p->B, 128)) return SA_ERR_CUDA;
  if (!make_map(&m->v, p->v, p->Dv, p->Sk, p->HK, p->B, 128)) return SA_ERR_CUDA;
  // O output of the forward (written by TMA stores in 128-row boxes)
  if (!backward && !make_map(&m->o, p->o, p->Dv, p->Sq, p->HQ, p->B, 128)) return SA_ERR_CUDA;
  // K half tiles of the forward's CTA pairs (64-row boxes)
  if (!backward && !make_map(&m->kh, p->k, p->Dqk, p->Sk, p->HK, p->B, 64)) return SA_ERR_CUDA;
  if (backward && !make_map(&m->dout, p->dout, p->Dv, p->Sq, p->HQ, p->B, qrows))
    return SA_ERR_CUDA;
  // dK / dV outputs (written by TMA stores in 128-row boxes)
  if (backward && !make_map(&m->dk, p->dk, p->Dqk, p->Sk, p->HK, p->B, 128)) return SA_ERR_CUDA;
  if (backward && !make_map(&m->dv, p->dv, p->Dv, p->Sk, p->HK, p->B, 128)) return SA_ERR_CUDA;
  return SA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

extern "C" const char* sparse_attn_error_string(int code) {
  switch (code) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID: return "invalid argument (null pointer, bad size or inconsistent shape)";
    case SA_ERR_UNSUPPORTED: return "unsupported head dims, block size, mode or extent";
    case SA_ERR_INDEX: return "index outside [-1, Sk)";
    case SA_ERR_ALIGN: return "a tensor base pointer is not 16-byte aligned";
    case SA_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case SA_ERR_WORKSPACE: return "workspace missing or too small";
    case SA_ERR_SCRATCH_LIMIT:
      return "problem needs more backward scratch than the fixed SA_NOALLOC_SCRATCH_BYTES array";
    case SA_ERR_DEVICE:
      return "the stream belongs to a device other than the current device";
    default: return "unknown error code";
  }
}

extern "C" int sparse_attn_set_timing_events(void* const* events) {
  if (!events) {
    g_timing_events = nullptr;
    return SA_OK;
  }
  for (int k = 0; k < 6; ++k) g_events_copy[k] = static_cast<cudaEvent_t>(events[k]);
  g_timing_events = g_events_copy;
  return SA_OK;
}

extern "C" int sparse_attn_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns, std::memory_order_relaxed);
  return SA_OK;
}

extern "C" int sparse_attn_set_forward_form(int form) {
  if (form < SA_FWD_FORM_AUTO || form > SA_FWD_FORM_TWO_TILES) return SA_ERR_INVALID;
  g_fwd_form.store(form, std::memory_order_relaxed);
  return SA_OK;
}

extern "C" int sparse_attn_set_backward_form(int form) {
  if (form < SA_BWD_FORM_AUTO || form > SA_BWD_FORM_WHOLE) return SA_ERR_INVALID;
  g_bwd_form.store(form, std::memory_order_relaxed);
  return SA_OK;
}

namespace sa {
// token-gather forward (gather_fwd.cu)
int launch_fwd_gather(const AttnArgs& a, const void* q, const void* k, const void* v,
                      cudaStream_t st);
}  // namespace sa

extern "C" int sparse_attn_fwd_gather(const sparse_attn_params* p, sa_stream_t stream) {
  AttnArgs a;
  int rc = fill_args(p, &a, false);
  if (rc) return rc;
  rc = check_stream_device(reinterpret_cast<cudaStream_t>(stream));
  if (rc) return rc;
  return launch_fwd_gather(a, p->q, p->k, p->v, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int sparse_attn_fwd(const sparse_attn_params* p, sa_stream_t stream) {
  AttnArgs a;
  int rc = fill_args(p, &a, false);
  if (rc) return rc;
  rc = check_stream_device(reinterpret_cast<cudaStream_t>(stream));
  if (rc) return rc;
  TensorMaps m;
  rc = fill_maps(p, &m, false);
  if (rc) return rc;
  return launch_fwd(a, m, reinterpret_cast<cudaStream_t>(stream));
}

// workspace layout: Delta fp32 [B][HQ][Sq] | dQ accumulator fp32 [B][Sq][HQ][Dqk] |
// deterministic mode's turn counters int32 [B][HQ][Tm][2]
extern "C" size_t sparse_attn_bwd_workspace_size(const sparse_attn_params* p) {
  if (!p || p->B <= 0 || p->HQ <= 0 || p->Sq <= 0 || p->Dqk <= 0) return 0;
  const size_t delta = sizeof(float) * static_cast<size_t>(p->B) * p->HQ * p->Sq;
  const size_t dq = sizeof(float) * static_cast<size_t>(p->B) * p->Sq * p->HQ * p->Dqk;
  const size_t sem = sizeof(int32_t) * 2 * static_cast<size_t>(p->B) * p->HQ *
                     static_cast<size_t>((p->Sq + kTile - 1) / kTile);
  return round256(delta) + round256(dq) + round256(sem);
}

static int run_bwd(const sparse_attn_params* p, void* workspace, size_t workspace_bytes,
                   sa_stream_t stream, int det) {
  AttnArgs a;
  int rc = fill_args(p, &a, true);
  if (rc) return rc;
  const size_t need = sparse_attn_bwd_workspace_size(p);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SA_ERR_WORKSPACE;
  rc = check_stream_device(reinterpret_cast<cudaStream_t>(stream));
  if (rc) return rc;
  const size_t delta_b = round256(sizeof(float) * static_cast<size_t>(p->B) * p->HQ * p->Sq);
  const size_t dq_b = round256(sizeof(float) * static_cast<size_t>(p->B) * p->Sq * p->HQ * p->Dqk);
  a.delta = static_cast<float*>(workspace);
  a.dq_acc = reinterpret_cast<float*>(static_cast<char*>(workspace) + delta_b);
  a.det = det;
  a.sem = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + delta_b + dq_b);
  TensorMaps m;
  rc = fill_maps(p, &m, true);
  if (rc) return rc;
  if (!make_map_f32(&m.dq_acc, a.dq_acc, p->Dqk, p->Sq, p->HQ, p->B)) return SA_ERR_CUDA;
  return launch_bwd(a, m, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int sparse_attn_bwd(const sparse_attn_params* p, void* workspace,
                               size_t workspace_bytes, sa_stream_t stream) {
  return run_bwd(p, workspace, workspace_bytes, stream, 0);
}

extern "C" int sparse_attn_bwd_deterministic(const sparse_attn_params* p, void* workspace,
                                             size_t workspace_bytes, sa_stream_t stream) {
  return run_bwd(p, workspace, workspace_bytes, stream, 1);
}
