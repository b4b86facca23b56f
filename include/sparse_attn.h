/*
 * sparse_attn.h -- C ABI of libsparse_attn.so: block-sparse and index-sparse softmax
 * attention on one NVIDIA B200 (sm_100a), forward (O, LSE) and backward (dQ, dK, dV),
 * and the conversion of token-level top-k indices or block masks into the per-tile
 * lists the kernels walk.
 *
 * Sources of the operation (web pages; no formulas are printed there):
 *  - MagiAttention PR #334, "[WIP]: feat(cutedsl-sm100): BWD LoopK with
 *    warp-specialized pipeline + IndexSparse/BlockSparse support": Summary (sparse
 *    attention forward/backward, dQ accumulation), section 1 (backward pipeline, fp32
 *    dK/dV accumulation, postprocess with softmax_scale), section 2
 *    (index_attn_indices_to_block_sparse: indices (total_q, NHK, topk) -> block lists
 *    via a presence matrix; per-M-block N-block lists).
 *  - MagiAttention PR #331, "feat: support 192/128 and 256/256 ffa_fa4 in magi":
 *    Summary (head dims (192,128) and (256,256)), "CSR Tile Mapping" (transposed
 *    key-to-query block lists for the backward).
 *  - xtuner PR #2096, "[Feature] Add optional TileLang Top-K selector", Main Changes 1:
 *    int32 top-k indices with -1 for invalid positions (the input of index mode).
 *  - nvfp4-megamoe-kernel commit log, multi-row softmax notes: online softmax over
 *    key tiles with a running max and sum, un-normalised P, final O = acc / sum.
 *
 * Definition implemented (textbook attention on an allowed key set A_i):
 *   s_ij = scale * q_i . k_j ;  LSE_i = ln sum_{j in A_i} exp(s_ij) ;
 *   O_i = sum_j exp(s_ij - LSE_i) v_j ;  dP_ij = dO_i . v_j ;  Delta_i = dO_i . O_i ;
 *   dS_ij = P_ij (dP_ij - Delta_i) ; dq_i = scale sum_j dS_ij k_j ;
 *   dk_j = scale sum_{h in group} sum_i dS_ij q_i ; dv_j = sum_{h in group} sum_i P_ij dO_i.
 *   Query head h uses KV head h / (HQ / HK).  A row with an empty set gets O = 0,
 *   LSE = -inf and zero gradients.
 * A_i: block mode -- mask[b][g][i/bs][j/bs] != 0 (bs = 64 or 128); dense mode -- all
 * keys; index mode -- the set of row i's indices (duplicates collapse, -1 skipped);
 * with causal != 0 additionally j <= i.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library never
 *    allocates or frees device memory.  Host pointers are only the parameter structs.
 *  - Layouts (row-major, last dimension contiguous, no padding):
 *      q [B][Sq][HQ][Dqk], k [B][Sk][HK][Dqk], v [B][Sk][HK][Dv],
 *      o, dO [B][Sq][HQ][Dv], dq [B][Sq][HQ][Dqk], dk [B][Sk][HK][Dqk],
 *      dv [B][Sk][HK][Dv]: bf16.  lse [B][HQ][Sq]: fp32 (natural log).
 *    Base pointers must be 16-byte aligned.
 *  - Supported (Dqk, Dv): (64,64), (128,128), (192,128), (256,256).  HQ % HK == 0.
 *  - Work is enqueued on `stream` and runs asynchronously; the call returns once it
 *    is enqueued.  Errors found on the host are returned before anything is enqueued.
 *  - Kernels run on the CURRENT device (cudaSetDevice); every pointer must be memory of
 *    that device and `stream` must belong to it (a stream created on another device is
 *    refused with SA_ERR_DEVICE).  Per-device set-up (kernel attributes, the no-alloc
 *    scratch address) is done on first use on each device, thread-safely.
 *  - Return value: SA_OK (0) or a negative SA_ERR_* code.  Errors found on the GPU
 *    (an index outside [-1, Sk), a pipeline wait that timed out) are OR-ed into the
 *    optional device int32 `dev_status` as the flags SA_STATUS_INDEX (value 1) and
 *    SA_STATUS_TIMEOUT (value 2); read it after synchronising.  No C++ exception crosses this boundary.
 */
#ifndef SPARSE_ATTN_H_
#define SPARSE_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sa_stream_t; /* the same handle as cudaStream_t */

#define SA_OK 0
#define SA_ERR_INVALID (-1)     /* null pointer, bad size or inconsistent shape */
#define SA_ERR_UNSUPPORTED (-2) /* head dims, block size or mode not supported */
#define SA_ERR_INDEX (-3)       /* reserved: index errors are reported on the device */
#define SA_ERR_ALIGN (-4)       /* a base pointer is not 16-byte aligned */
#define SA_ERR_CUDA (-5)        /* a CUDA call or kernel launch failed */
#define SA_ERR_WORKSPACE (-7)   /* workspace missing or too small */
#define SA_ERR_SCRATCH_LIMIT (-8) /* sparse_attn_bwd_noalloc: problem exceeds its fixed scratch */
#define SA_ERR_DEVICE (-9)      /* the stream belongs to a device other than the current one */

/* Flags OR-ed into the optional device status word (dev_status). */
#define SA_STATUS_INDEX 1   /* an index outside [-1, Sk), or a top-k row range outside [0, cols) */
#define SA_STATUS_TIMEOUT 2 /* a bounded pipeline wait ran out */

#define SA_MODE_DENSE 0
#define SA_MODE_BLOCK 1
#define SA_MODE_INDEX 2

#define SA_TILE 128 /* every list entry stands for a 128 x 128 (query x key) tile */

/*
 * Tile lists and the element data the kernels need inside partial tiles.  Filled by
 * block_mask_to_block_sparse() or index_to_block_sparse(); read by the attention
 * calls.  With Tm = ceil(Sq/128), Tn = ceil(Sk/128), W = ceil(Sk/32), the caller
 * allocates (device memory):
 *   cnt  int32 [B][HK][Tm][2]   (n_full, n_partial) per query tile
 *   idx  int32 [B][HK][Tm][Tn]  full key tiles ascending, then partial ascending, -1 fill
 *   tcnt int32 [B][HK][Tn][2]   the same per key tile over query tiles (backward)
 *   tidx int32 [B][HK][Tn][Tm]
 *   bitmap uint32 [B][HK][Sq][W] (index mode only): bit j%32 of word j/32 of row i is
 *          set iff j is one of row i's indices (the presence matrix).
 * A tile is FULL when every (i, j) in it with i < Sq, j < Sk is allowed and the tile
 * lies inside [0, Sk); PARTIAL when some (i, j) is allowed otherwise; absent when none
 * is.  `mask` (block mode) is the caller's mask, kept for partial tiles of bs = 64.
 */
typedef struct sa_block_sparse {
  int32_t mode;   /* SA_MODE_* */
  int32_t causal; /* non-zero: j <= i is also required */
  int32_t B, HK;
  int64_t Sq, Sk;
  int32_t bs, Mb, Nb;   /* block mode: granularity and mask extents (Mb*bs >= Sq, Nb*bs >= Sk) */
  const uint8_t *mask;  /* block mode: [B][HK][Mb][Nb]; NULL in dense mode */
  uint32_t *bitmap;     /* index mode */
  int32_t *cnt, *idx, *tcnt, *tidx;
} sa_block_sparse;

/*
 * index_to_block_sparse -- MagiAttention PR #334, section 2
 * (index_attn_indices_to_block_sparse and the per-M-block normalisation) and
 * MagiAttention PR #331, "CSR Tile Mapping" (the transposed lists).
 *   idx   device int32 [B][Sq][HK][topk]: key positions in [0, Sk) or -1 (padding).
 *   out   host struct: B, HK, Sq, Sk, causal and the device buffers bitmap, cnt, idx,
 *         tcnt, tidx must be set by the caller; mode is set to SA_MODE_INDEX.
 * Fills the bitmap and all four lists.  Values < -1 or >= Sk are skipped and set
 * SA_STATUS_INDEX in *dev_status (when dev_status is not NULL).
 */
int index_to_block_sparse(const int32_t *idx, int32_t topk, sa_block_sparse *out,
                          int32_t *dev_status, sa_stream_t stream);

/*
 * block_mask_to_block_sparse -- the block-mask counterpart (BlockSparse attention of
 * MagiAttention PR #334; block-sparsity computation of sgl-flash-attn PR #28).
 *   out   host struct with mode = SA_MODE_BLOCK (mask = device uint8
 *         [B][HK][Mb][Nb], bs in {64, 128}) or SA_MODE_DENSE (mask unused), plus B, HK,
 *         Sq, Sk, causal and the device list buffers.  bitmap is unused.
 */
int block_mask_to_block_sparse(sa_block_sparse *out, sa_stream_t stream);

typedef struct sparse_attn_params {
  const void *q, *k, *v; /* bf16 inputs */
  void *o;               /* bf16 [B][Sq][HQ][Dv]: forward output, backward input */
  float *lse;            /* fp32 [B][HQ][Sq]: forward output, backward input */
  const void *dout;      /* bf16 [B][Sq][HQ][Dv]: backward input */
  void *dq, *dk, *dv;    /* bf16 backward outputs */
  int32_t B, HQ, HK, Dqk, Dv;
  int64_t Sq, Sk;
  float softmax_scale;
  const sa_block_sparse *sparse; /* host pointer; lists built for the same B, HK, Sq, Sk */
  int32_t *dev_status;           /* optional device int32 */
} sparse_attn_params;
/* Sizes: B, HQ, HK, Sq and Sk are at least 1 here and in sa_block_sparse; a problem with
 * a zero extent has nothing to compute and is refused with SA_ERR_INVALID before any
 * launch (callers skip the call). */

/*
 * sparse_attn_fwd -- forward: O and LSE.  Streams only the listed key tiles of each
 * 128-query tile through shared memory, computes S = Q K^T and O += P V on the
 * tensor cores with fp32 accumulation in tensor memory, and runs the online softmax
 * (running max and sum, un-normalised P, O / sum at the end; nvfp4-megamoe-kernel
 * multi-row softmax notes).  Reads q, k, v; writes o, lse.
 */
int sparse_attn_fwd(const sparse_attn_params *p, sa_stream_t stream);

/*
 * sparse_attn_fwd_gather -- the same O and LSE in index mode, computed by gathering each
 * query's selected K/V rows instead of streaming whole key tiles (the token-level
 * alternative the sparse MLA backends of xtuner PR #2096, Background, stand for).  One
 * warp per (batch, query, KV head) enumerates the query's keys from the presence bitmap
 * of `sparse` (so repeated indices count once and the causal limit applies), gathers
 * their rows 16 at a time and runs S = Q K^T and O += P V for the group's query heads on
 * the tensor cores (mma.sync, the heads as M).  A comparison path: the benchmark times it
 * against sparse_attn_fwd.  Needs sparse->mode == SA_MODE_INDEX, HQ / HK <= 8 and
 * (Dqk, Dv) in {(64,64), (128,128), (192,128)} (SA_ERR_UNSUPPORTED otherwise).  Reads
 * q, k, v and the bitmap; writes o, lse.
 */
int sparse_attn_fwd_gather(const sparse_attn_params *p, sa_stream_t stream);

/* Bytes of device workspace sparse_attn_bwd needs for these shapes (fp32 Delta, the
 * fp32 dQ accumulator and the deterministic mode's int32 turn counters, each rounded
 * up to 256 B). */
size_t sparse_attn_bwd_workspace_size(const sparse_attn_params *p);

/*
 * sparse_attn_bwd -- backward: dq, dk, dv from q, k, v, o, lse, dout.
 * Preprocess Delta = rowsum(dO * O); main kernel over key tiles (walking the
 * transposed lists) recomputing P = exp(scale S - LSE), accumulating dV += P^T dO and
 * dK += dS^T Q in tensor memory (dK scaled by softmax_scale as it is stored) and
 * adding dQ += dS K into an fp32 accumulator; the postprocess scales dQ by
 * softmax_scale and casts it to bf16 (MagiAttention PR #334, section 1 and section 3).
 * At head dims (192,128) a key tile takes one CTA or two (sparse_attn_set_backward_form).
 * `workspace` is device memory of at least sparse_attn_bwd_workspace_size() bytes, owned
 * by the caller; its contents need not be initialised.
 */
int sparse_attn_bwd(const sparse_attn_params *p, void *workspace, size_t workspace_bytes,
                    sa_stream_t stream);

/*
 * sparse_attn_bwd_deterministic -- the same backward with a bitwise reproducible dQ
 * (the deterministic backward of sgl-flash-attn PR #28; fixed-order reduction).  dK and
 * dV are accumulated in a fixed order in every mode; dQ, which many key-tile CTAs add
 * into, is here accumulated in descending key-tile order for every (batch, query head,
 * query tile): a CTA waits for its turn on a counter in the workspace (same size as for
 * sparse_attn_bwd).  Same arguments, outputs and errors as sparse_attn_bwd; results
 * equal those of sparse_attn_bwd up to the rounding order of dQ, and two calls on the
 * same inputs give identical bits.  Slower where several key tiles reach the same
 * query tile at the same time.
 */
int sparse_attn_bwd_deterministic(const sparse_attn_params *p, void *workspace,
                                  size_t workspace_bytes, sa_stream_t stream);

/* Size of the fixed device scratch array used by sparse_attn_bwd_noalloc: 16 MiB. */
#define SA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * sparse_attn_bwd_noalloc -- the backward for callers that cannot allocate device
 * memory.  The pages have no counterpart to this entry point.
 * Some callers cannot call cudaMalloc or pass a workspace: code inside a host framework
 * that owns every device allocation and hands over only inputs and outputs (a plugin
 * or serving backend), or latency-critical loops where cudaMalloc's implicit device
 * synchronisation is not acceptable.  This call runs the same kernels as
 * sparse_attn_bwd (same arguments, same outputs) but takes the backward's scratch
 * (fp32 Delta and dQ accumulator) from a file-scope device array of
 * SA_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library holds until exit.
 *  - Returns SA_ERR_SCRATCH_LIMIT, before enqueuing anything, when
 *    sparse_attn_bwd_workspace_size(p) exceeds SA_NOALLOC_SCRATCH_BYTES.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current; a failed lookup is retried by the
 *    next call); make it before any stream capture.
 *  - The array used is the current device's: `stream` must belong to the current
 *    device (SA_ERR_DEVICE otherwise).
 *  - All calls on a device share the array and overwrite it; calls whose GPU work
 *    overlaps (unordered streams, several host threads) race: serialise them.
 *  - Allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 */
int sparse_attn_bwd_noalloc(const sparse_attn_params *p, sa_stream_t stream);

/*
 * sparse_attn_set_timing_events -- optional instrumentation (no counterpart on the
 * pages; it serves the benchmark's per-kernel timing).  `events` points to six
 * cudaEvent_t handles created by the caller, or is NULL to switch recording off.
 * While set, sparse_attn_fwd records events[0] before and events[1] after its kernel,
 * and sparse_attn_bwd records events[2] before the preprocess, events[3] before the
 * main kernel, events[4] after it and events[5] after the postprocess, each on the
 * call's stream.  Process-wide setting, not synchronised: set it while no other
 * thread calls into the library.  Returns SA_OK.
 */
int sparse_attn_set_timing_events(void *const *events);

/*
 * sparse_attn_set_wait_limit_ns -- test instrumentation (no counterpart on the pages).
 * Every pipeline wait inside the attention kernels is bounded: a wait that has not
 * completed after the limit gives up, sets SA_STATUS_TIMEOUT in *dev_status, and its CTA drains the
 * copies and tensor-core operations it has in flight and leaves (the outputs of that
 * call are then undefined, the CUDA context stays usable).  The default limit is 2 s.
 * This call sets the limit, in nanoseconds, for the calls enqueued after it (0 restores
 * the default).  A limit below 1000 ns means that a wait gives up at its first test if
 * the phase it waits for has not completed: ordinary waits (a TMA load just issued, the
 * first MMA) then run out, which is how the tests exercise the timeout path.
 * Process-wide; returns SA_OK.
 */
int sparse_attn_set_wait_limit_ns(uint64_t ns);

/* Forms of sparse_attn_set_forward_form. */
#define SA_FWD_FORM_AUTO 0
#define SA_FWD_FORM_ONE_HEAD 1
#define SA_FWD_FORM_CTA_PAIR 2
#define SA_FWD_FORM_TWO_HEADS 3
#define SA_FWD_FORM_TWO_TILES 4

/*
 * sparse_attn_set_forward_form -- selects how the forward maps query heads (and query
 * tiles) to CTAs.  The pages pick the number of query tiles per CTA ("q_stage",
 * sgl-flash-attn PR #28, "determine q_stage via seqlen_q for sm100"), have 256-row tiles on SM100 (MagiAttention PR #331,
 * "CSR Tile Mapping") and a switch that turns the 2-CTA mode off (MagiAttention PR #334,
 * section 3, disable_2cta); the forms here are this library's own.  The query heads of
 * one GQA group walk the same tile list, so with an even group size two of them (same
 * query tile) can share every K and V tile:
 *   SA_FWD_FORM_ONE_HEAD   one CTA per (query tile, query head);
 *   SA_FWD_FORM_CTA_PAIR   two heads on a 2-CTA cluster whose tensor-core MMAs span both
 *                          CTAs (tcgen05 cta_group::2, M = 256); each CTA holds half of
 *                          every K and V tile (needs Dv >= 128);
 *   SA_FWD_FORM_TWO_HEADS  two heads in one CTA, each with its own S and O in tensor
 *                          memory and its own softmax warps, so that one head's softmax
 *                          overlaps the other head's MMAs (needs Dqk <= 192, Dv <= 128);
 *   SA_FWD_FORM_TWO_TILES  two consecutive query tiles of one head in one CTA, arranged
 *                          as the two heads above; the CTA walks the union of the two
 *                          tiles' lists, and a key tile that one tile's list lacks is
 *                          masked out for that tile's rows (needs Dqk, Dv <= 128 and at
 *                          most 2048 key tiles).  Worth it where the two lists nearly
 *                          agree (dense and causal masks); on lists that share few tiles
 *                          the union costs up to twice the tensor work;
 *   SA_FWD_FORM_AUTO       the library's choice (measured): two heads per CTA where that
 *                          applies, CTA pairs at head dims 256, one head per CTA for MHA
 *                          and odd group sizes (two query tiles per CTA measured no
 *                          faster on dense lists, and slower where halving the CTA count
 *                          leaves a partial last wave).
 * A form that does not apply to a call falls back to one head per CTA.  All forms compute
 * the same O and LSE up to fp32 rounding.  Applies to the forward calls enqueued after it;
 * process-wide.  Returns SA_OK, or SA_ERR_INVALID for another value (the setting is then
 * unchanged).
 */
int sparse_attn_set_forward_form(int form);

/* Forms of sparse_attn_set_backward_form. */
#define SA_BWD_FORM_AUTO 0
#define SA_BWD_FORM_SPLIT 1
#define SA_BWD_FORM_WHOLE 2

/*
 * sparse_attn_set_backward_form -- selects how the backward main kernel covers a 128-key
 * tile at head dims (192,128), where the fp32 dK and dV of the whole head dim (320 TMEM
 * columns) leave too little tensor memory for double-buffered S^T / dP^T tiles
 * (MagiAttention PR #331 builds 192/128 with 2-CTA tiles; the forms here are this
 * library's own):
 *   SA_BWD_FORM_SPLIT  two CTAs per key tile, each owning part of the head dim of dK, dV
 *                      and dQ and each recomputing S^T and dP^T (double-buffered);
 *   SA_BWD_FORM_WHOLE  one CTA per key tile with single S^T / dP^T buffers: no
 *                      recompute, but each step's MMAs wait for the previous step;
 *   SA_BWD_FORM_AUTO   WHOLE when the grid of key tiles (B * HK * ceil(Sk/128)) is at
 *                      least twice the SM count, else SPLIT (measured: WHOLE is ~10%
 *                      faster once the SMs are filled, slower while half of them idle).
 * The deterministic backward always splits.  Other head dims ignore the setting.  All
 * forms compute the same gradients up to fp32 rounding.  Applies to the backward calls
 * enqueued after it; process-wide.  Returns SA_OK, or SA_ERR_INVALID for another value
 * (the setting is then unchanged).
 */
int sparse_attn_set_backward_form(int form);


/* Largest k that topk_select supports. */
#define SA_TOPK_MAX_K 4096

/*
 * topk_select -- xtuner PR #2096, "[Feature] Add optional TileLang Top-K selector", Main
 * Changes 1: the Top-K stage that turns fp32 indexer scores into the int32 key indices
 * (-1 for invalid positions) of index mode.
 *   scores  device fp32 [rows][ld]; row r's candidates are the columns j of its valid
 *           range [starts[r], ends[r]) (the whole row [0, cols) when starts / ends are
 *           NULL).  Requires 0 <= starts[r] <= ends[r] <= cols, cols <= ld.
 *   starts, ends  optional device int32 [rows].
 *   k       1 <= k <= SA_TOPK_MAX_K.
 *   out_idx device int32 [rows][k]: the columns of the k largest scores of the range,
 *           largest first (the order of torch.topk with sorted=True); ties go to the
 *           smaller column, -0 equals +0, NaN ranks above +inf; when the range holds
 *           n < k columns, slots n..k-1 are -1.
 *   out_val optional device fp32 [rows][k]: the selected scores (-inf in -1 slots).
 * A row whose range is invalid yields k times -1 and sets SA_STATUS_INDEX in *dev_status.  Needs
 * no workspace.  Returns SA_ERR_INVALID for a bad size, k or null pointer.
 */
int topk_select(const float *scores, int64_t rows, int64_t cols, int64_t ld,
                const int32_t *starts, const int32_t *ends, int32_t k, int32_t *out_idx,
                float *out_val, int32_t *dev_status, sa_stream_t stream);

/* Static description of an SA_* code. */
const char *sparse_attn_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H_ */
