/*
 * cbv.h - blockwise causal varlen attention on B200 (sm_100a): the C ABI of libcbv.so.
 *
 * What the library computes (sources are named by page title and section):
 *   - NeMo AutoModel API, eagle.zigzag_ring_attention: zig-zag context parallelism
 *     (module docstring), get_half_index / get_half_lse, _block_forward /
 *     _block_backward, update_out_and_lse, zigzag_ring_flash_attn_varlen_forward /
 *     _backward (the merged-lse backward);
 *   - NeMo AutoModel API, eagle.ring_attention: the contiguous ring (module
 *     docstring, ring_flash_attn_forward: step <= rank, causal only at step 0),
 *     _update_out_and_lse (sigmoid-form merge), _fa_forward's (out, lse) contract;
 *   - NKI library API, attention_kv_parallel_segmented_cte: KV-parallel segmented
 *     prefill over a paged KV cache, contiguous or round-robin shards, sliding window;
 *   - qsa_fa_fallback.py (SM121 recipe): one-query-per-sequence GQA varlen decode.
 *
 * Conventions shared by every call:
 *   - Tensors are plain pointers.  "device" pointers are CUDA global memory of the
 *     current device; "host" pointers are ordinary CPU memory read during the call
 *     and not retained.  The caller owns all memory; the library allocates nothing
 *     and keeps no state between calls (apart from the per-thread count of its kernel
 *     launches, cbv_launch_count).  Scratch memory comes from a caller-owned
 *     device `workspace` whose size the matching *_workspace_size() call reports
 *     (cbv_zigzag_ring_fwd_noalloc, at the end, is the one call with built-in scratch).
 *   - bf16 means IEEE bfloat16 (torch.bfloat16); token-major layouts are
 *     [tokens, heads, head_dim], contiguous.  lse is float32 [heads, tokens],
 *     natural log.  head_dim is 64 or 128.
 *   - Masks use positions.  In the ring and prefill calls a token's position is its
 *     global row in natural packed order (prefill: global_q_offset + i for q).  A key
 *     is visible when it is in the query's document and, if causal, kpos <= qpos;
 *     with window = W > 0 also qpos - kpos < W (W keys including the query itself;
 *     the NKI sliding_window integer, 0 = disabled).
 *   - A query with no visible key gets out = 0 and lse = -inf.
 *   - scale <= 0 selects head_dim^-0.5.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) unless stated otherwise, and returns CBV_OK (0) or a negative
 *     cbv_status; cbv_last_error_message() then describes the failure.  Argument
 *     errors are detected on the host before anything is launched.
 *   - No call copies host memory to the device with a copy engine.  The tile schedules
 *     built on the host travel inside kernel launch parameters, so a call neither waits
 *     for its stream nor queues behind the caller's own transfers.  A fixed-shape sequence
 *     of calls can be captured in a CUDA graph and replayed on new tensor contents.
 *   - Kernels never wait without a bound: a stalled pipeline records a code in the
 *     workspace status word and exits; cbv_read_status() returns CBV_ERR_TIMEOUT.
 *   - Argument structs start with struct_size and abi_version so that fields are
 *     never bound by position (the lesson of ring_attention's
 *     require_flash_attn_version); a mismatch returns CBV_ERR_VERSION.
 */
#ifndef CBV_H
#define CBV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CBV_ABI_VERSION 1

typedef enum cbv_status {
  CBV_OK = 0,
  CBV_ERR_BAD_ARG = -1,
  CBV_ERR_BAD_SHAPE = -2,
  CBV_ERR_BAD_DTYPE = -3,
  CBV_ERR_MISALIGNED = -4,
  CBV_ERR_UNSUPPORTED_HEAD_DIM = -5,
  CBV_ERR_NOT_DIVISIBLE_2CP = -6,
  CBV_ERR_NOT_CAUSAL = -7,
  CBV_ERR_GQA_MISMATCH = -8,
  CBV_ERR_BAD_CU_SEQLENS = -9,
  CBV_ERR_Q_LEN_NOT_ONE = -10,
  CBV_ERR_WORKSPACE_TOO_SMALL = -11,
  CBV_ERR_TIMEOUT = -12,
  CBV_ERR_CUDA = -13,
  CBV_ERR_VERSION = -14
} cbv_status;

typedef enum cbv_layout { CBV_LAYOUT_ZIGZAG = 0, CBV_LAYOUT_CONTIGUOUS = 1 } cbv_layout;
typedef enum cbv_kv_mode { CBV_KV_CONTIGUOUS = 0, CBV_KV_ROUND_ROBIN = 1 } cbv_kv_mode;
typedef enum cbv_dtype { CBV_DTYPE_BF16 = 0, CBV_DTYPE_F32 = 1 } cbv_dtype;
typedef enum cbv_schedule {
  /* one launch: each q tile visits every ring step's k/v block in ring order and
     merges the block results on chip (log-sum-exp identity on the accumulator) */
  CBV_SCHEDULE_FUSED = 0,
  /* one launch per ring step; each launch merges its block into an fp32 running
     (out, lse) pair in the workspace inside the kernel epilogue */
  CBV_SCHEDULE_STEPWISE = 1
} cbv_schedule;

/* Text of the last error on this thread ("" if none).  Valid until the next call. */
const char* cbv_last_error_message(void);
int cbv_abi_version(void);

/* Reads the device status word at the start of `workspace` (synchronises `stream`).
   *status_out receives the raw kernel code (0 = ok).  Returns CBV_ERR_TIMEOUT if a
   kernel gave up a wait, CBV_OK otherwise. */
int cbv_read_status(const void* workspace, int* status_out, void* stream);

/* Number of kernels the library has launched from the calling thread since it was loaded
 * (every call's schedule upload, helpers and attention kernels included).  A diagnostic: the
 * difference across a stretch of calls is exactly what those calls enqueued. */
size_t cbv_launch_count(void);

/* Measurement hook, per calling thread.  While set, every launch of an attention kernel (the
 * forward kernel of the ring, block, cached and paged forwards, the backward kernel, the decode
 * kernel) records `start_event` on the call's stream right before the launch and `stop_event`
 * right after it, so cudaEventElapsedTime gives that kernel's device time without the call's
 * helper kernels.  In a call that launches several attention kernels (the stepwise schedule)
 * the events bracket the last one.  The records are stream operations between launches and add
 * to the time of the steps they sit in, so a throughput measurement should time steps without
 * the hook and use it in a separate pass.  The events are caller-owned cudaEvent_t handles;
 * NULL, NULL clears the hook.  Returns CBV_OK; a failed record makes the call that launched
 * return CBV_ERR_CUDA. */
int cbv_set_kernel_events(void* start_event, void* stop_event);

/* How the library was built: CBV_BUILD_DEBUG is set in the bounds-checking build (libcbv_debug.so,
 * compiled with CBV_DEBUG), whose kernels check every row and page index they copy or store
 * against its tensor and report a violation as a status code 0x201-0x204 (read with
 * cbv_read_status) instead of touching memory outside the tensor.  The varlen decode checks its
 * device-side offsets in every build (status 0x205, the sequence is skipped). */
#define CBV_BUILD_DEBUG 1
int cbv_build_flags(void);

/* ========================================================================= planner (host only)
 * Integer, exact; all arrays are host memory.  cu_seqlens is GLOBAL, int32 [num_docs+1],
 * natural packed order.  NeMo AutoModel zigzag_ring_attention: module docstring
 * (2*cp chunks, rank r owns chunks r and 2cp-1-r), get_half_index, get_half_lse,
 * _block_forward (halved cu_seqlens).  Errors: CBV_ERR_BAD_CU_SEQLENS (not starting
 * at 0 or decreasing), CBV_ERR_NOT_DIVISIBLE_2CP, CBV_ERR_BAD_ARG. */

/* out[d] = cu_global[d] / cp, int32 [num_docs+1]: every virtual rank's local cu_seqlens. */
int cbv_local_cu_seqlens(const int32_t* cu_global, int32_t num_docs, int32_t cp, int32_t layout, int32_t* out);
/* out[d] = cu_global[d] / (2 cp): cu_seqlens of the front or back halves (zig-zag only). */
int cbv_half_cu_seqlens(const int32_t* cu_global, int32_t num_docs, int32_t cp, int32_t* out);
/* Ascending local positions of the front (front != 0) or back half of every local
   document, int32 [cu_local[num_docs] / 2]; *count_out receives the length. */
int cbv_get_half_index(const int32_t* cu_local, int32_t num_docs, int32_t front, int32_t* idx_out,
                       int64_t* count_out);
/* Front or back half of a host float32 lse [num_heads, seqlen] (seqlen = cu_local[num_docs]),
   per local document: out [num_heads, seqlen / 2]. */
int cbv_get_half_lse(const float* lse, int32_t num_heads, const int32_t* cu_local, int32_t num_docs, int32_t front,
                     float* out);
/* Global rows of virtual rank `rank`'s tokens in local order, int32 [S / cp]. */
int cbv_rank_tokens(const int32_t* cu_global, int32_t num_docs, int32_t cp, int32_t rank, int32_t layout,
                    int32_t* out);
/* Visible causal (q, k) pairs per virtual rank (the work each rank does), int64 [cp]. */
int cbv_rank_pair_counts(const int32_t* cu_global, int32_t num_docs, int32_t cp, int32_t layout, int32_t window,
                         int64_t* counts_out);
/* Ring step schedule: the rank whose k/v reach `rank` at `step` (src = (rank-step) mod cp)
   and the block kind: 0 diag (local q x local k, causal), 1 front-k (all local q x src's
   front halves), 2 back-q (local back halves x all of src's k), 3 full (contiguous,
   step <= rank), 4 skip (contiguous, step > rank). */
int cbv_ring_step(int32_t rank, int32_t step, int32_t cp, int32_t layout, int32_t* src_out, int32_t* kind_out);

/* The per-step block descriptors of the whole ring: one cbv_ring_block per (rank, step) that
 * runs a block (rank-major, steps in order; the contiguous layout's skipped steps are left out),
 * each the flash call of zigzag_ring_attention._block_forward / _block_backward (contiguous:
 * ring_attention.ring_flash_attn_forward):
 *   - step 0 (kind 0): every local q row against every local k row, causal, both sides with
 *     the local cu_seqlens (G / cp);
 *   - src < rank (kind 1): every local q row (local cu) against src's FRONT halves, whose
 *     cu_seqlens are the halved ones (G / (2 cp)), not causal;
 *   - src > rank (kind 2): the local BACK halves (halved cu; get_half_index / get_half_lse with
 *     front = 0 select them) against every local k row of src (local cu), not causal;
 *   - contiguous, 0 < step <= rank (kind 3): every local row against src's, not causal.
 * The rows of a side are runs of consecutive GLOBAL rows (natural packed order), document by
 * document in local order (a document's front chunk before its back chunk); a run's `local0`
 * is the index of its first row in its rank's local sequence (rank for q, src for k), and
 * `pos0` the position of its first row: positions are global rows, so pos0 == row0.  Empty
 * documents contribute no run.
 * Sizes: call with blocks == NULL or runs == NULL to get the counts only.  With arrays,
 * max_blocks / max_runs are their capacities; too small -> CBV_ERR_BAD_ARG (counts still set).
 * Errors: as the other planner calls.  (The sliding window does not change the blocks: the
 * flash call masks by position.) */
typedef struct cbv_row_run {
  int32_t doc;
  int32_t row0;   /* first global row */
  int32_t rows;
  int32_t pos0;   /* position of row0 (== row0) */
  int32_t local0; /* index of row0 in the rank's local sequence */
} cbv_row_run;
typedef struct cbv_ring_block {
  int32_t rank, step, src;
  int32_t kind;    /* as cbv_ring_step */
  int32_t causal;  /* 1 only for the step-0 block */
  int32_t q_half;  /* 0: every local q row, cu_seqlens_q = G / cp; 2: back halves, cu_seqlens_q = G / (2 cp) */
  int32_t k_half;  /* 0: every local k row of src, cu_seqlens_k = G / cp; 1: front halves, cu_seqlens_k = G / (2 cp) */
  int32_t q_run0, q_nruns;  /* this block's q rows: runs[q_run0 .. q_run0 + q_nruns) */
  int32_t k_run0, k_nruns;  /* its k rows (of src) */
} cbv_ring_block;
int cbv_plan_zigzag(const int32_t* cu_global, int32_t num_docs, int32_t cp, int32_t layout, cbv_ring_block* blocks,
                    int32_t max_blocks, int32_t* num_blocks_out, cbv_row_run* runs, int32_t max_runs,
                    int32_t* num_runs_out);

/* ========================================================================= block forward
 * One flash varlen block (zigzag_ring_attention._block_forward; ring_attention._fa_forward:
 * returns (out[B,S,H,D], lse[B,H,S])).  Documents pair q rows [cu_q[d], cu_q[d+1]) with k
 * rows [cu_k[d], cu_k[d+1]).  Positions: qpos = q_pos_base[d] + (i - cu_q[d]),
 * kpos = k_pos_base[d] + (j - cu_k[d]); NULL bases mean k_pos_base = 0 and
 * q_pos_base = L_k - L_q (bottom-right alignment).
 * merge = 0: writes out (bf16 or f32, out_dtype) and lse.
 * merge = 1: out must be f32; (out, lse) hold a running pair that is merged in place with
 *            this block by the online-softmax identity (update_out_and_lse) in the kernel
 *            epilogue.  Rows of the running pair outside this block are untouched. */
typedef struct cbv_block_fwd_args {
  uint32_t struct_size; /* sizeof(cbv_block_fwd_args) */
  uint32_t abi_version; /* CBV_ABI_VERSION */
  const void* q;        /* device bf16 [total_q, num_heads, head_dim] */
  const void* k;        /* device bf16 [total_k, num_kv_heads, head_dim] */
  const void* v;        /* device bf16 [total_k, num_kv_heads, head_dim] */
  int64_t total_q, total_k;
  int32_t num_heads, num_kv_heads, head_dim;
  int32_t num_docs;
  const int32_t* cu_seqlens_q; /* host int32 [num_docs+1] */
  const int32_t* cu_seqlens_k; /* host int32 [num_docs+1] */
  const int32_t* q_pos_base;   /* host int32 [num_docs] or NULL */
  const int32_t* k_pos_base;   /* host int32 [num_docs] or NULL */
  int32_t max_seqlen;          /* 0 or >= every document length (checked) */
  float scale;
  int32_t causal;
  int32_t window;
  int32_t merge;
  int32_t out_dtype;           /* cbv_dtype of out when merge = 0 */
  void* out;                   /* device [total_q, num_heads, head_dim] */
  float* lse;                  /* device f32 [num_heads, total_q] */
  void* workspace;             /* device, >= cbv_block_fwd_workspace_size() bytes, 256-byte aligned */
  size_t workspace_bytes;
} cbv_block_fwd_args;
size_t cbv_block_fwd_workspace_size(const cbv_block_fwd_args* a);
int cbv_attn_block_fwd(const cbv_block_fwd_args* a, void* stream);

/* ========================================================================= merge
 * In place: (out, lse) <- update_out_and_lse(out, lse, block_out, block_lse)
 * (zigzag_ring_attention.update_out_and_lse; ring_attention._update_out_and_lse).
 * out: device f32 [seqlen, num_heads, head_dim]; lse, block_lse: device f32 [num_heads, seqlen];
 * block_out: device [seqlen, num_heads, head_dim] of block_out_dtype (bf16 or f32);
 * weight_out: device f32 [num_heads, seqlen] or NULL, receives sigmoid(block_lse - lse)
 * computed with the running lse before the merge.  A side at -inf is the identity. */
int cbv_attn_merge(float* out, float* lse, const void* block_out, int32_t block_out_dtype, const float* block_lse,
                   float* weight_out, int64_t seqlen, int32_t num_heads, int32_t head_dim, void* stream);

/* ========================================================================= ring forward / backward
 * Causal varlen attention of the whole packed batch computed the ring way
 * (zigzag_ring_flash_attn_varlen_forward / _backward; ring_flash_attn_forward /
 * _backward for layout = CBV_LAYOUT_CONTIGUOUS): the batch is split over cp VIRTUAL
 * ranks on this GPU (zig-zag: rank r owns chunks r and 2cp-1-r of every document;
 * contiguous: the r-th of cp pieces of every document); at step s rank r attends to the
 * k/v of src = (r-s) mod cp with the block schedule of cbv_ring_step, and the block
 * results are merged with the log-sum-exp identity.  There is no communication: the
 * virtual ranks are address ranges in HBM.  q, k, v, out, dout, dq, dk, dv are in natural
 * packed order; lse is [num_heads, total].
 * Backward: every block is fed the MERGED out and lse (the merged-lse identity), dk/dv of
 * a key tile accumulate across all blocks that see it, dq accumulates in fp32.
 * Deterministic backward (the `deterministic` argument of zigzag_ring_flash_attn_varlen_backward
 * and ring_attention._fa_backward): dk and dv are always written once per key tile, but dq sums partials from every key
 * tile that sees a row, and fp32 reduce-adds land in whatever order the tiles finish.  With
 * deterministic = 1 every partial is rounded to 64-bit fixed point in units of 2^-32 and added as
 * an integer, so dq is bit-identical from run to run (the workspace holds 8 instead of 4 bytes per
 * dq element, and each partial's rounding adds at most 2^-33 absolute error).
 * Errors: causal = 0 -> CBV_ERR_NOT_CAUSAL (zig-zag is meaningless otherwise); a document
 * length not divisible by 2cp (zig-zag) or cp (contiguous) -> CBV_ERR_NOT_DIVISIBLE_2CP. */
typedef struct cbv_ring_args {
  uint32_t struct_size; /* sizeof(cbv_ring_args) */
  uint32_t abi_version; /* CBV_ABI_VERSION */
  const void* q;        /* device bf16 [total, num_heads, head_dim] */
  const void* k;        /* device bf16 [total, num_kv_heads, head_dim] */
  const void* v;
  int64_t total;
  int32_t num_heads, num_kv_heads, head_dim;
  int32_t num_docs;
  const int32_t* cu_seqlens; /* host int32 [num_docs+1], GLOBAL */
  int32_t max_seqlen;        /* 0 or >= every document length */
  int32_t cp;                /* virtual ranks, >= 1 */
  int32_t layout;            /* cbv_layout */
  float scale;
  int32_t causal;            /* must be 1 */
  int32_t window;
  int32_t schedule;          /* cbv_schedule (forward only) */
  int32_t deterministic;     /* backward only: 1 = bit-reproducible dq (see above), 0 = fastest */
  void* out;                 /* device bf16 [total, num_heads, head_dim]: forward output, backward input */
  float* lse;                /* device f32 [num_heads, total]: forward output, backward input (merged) */
  const void* dout;          /* backward: device bf16 [total, num_heads, head_dim] */
  void* dq;                  /* backward: device bf16 outputs */
  void* dk;
  void* dv;
  void* workspace;
  size_t workspace_bytes;
} cbv_ring_args;
size_t cbv_zigzag_ring_fwd_workspace_size(const cbv_ring_args* a);
int cbv_zigzag_ring_fwd(const cbv_ring_args* a, void* stream);
size_t cbv_zigzag_ring_bwd_workspace_size(const cbv_ring_args* a);
int cbv_zigzag_ring_bwd(const cbv_ring_args* a, void* stream);

/* ========================================================================= one ring step on real ranks
 * The ring over cp REAL ranks (one process per GPU), as the zig-zag page runs it: RingComm
 * rotates K/V one rank along per step, and each rank runs one flash block per step against the
 * K/V it holds (zigzag_ring_flash_attn_varlen_forward; ring_attention.ring_flash_attn_forward for
 * CBV_LAYOUT_CONTIGUOUS).  These calls are that block on a rank's LOCAL buffers; the exchange is
 * the caller's (the Python package's ring driver sends over torch.distributed).  At `step`, rank
 * `rank` holds the k/v of src = (rank - step) mod cp and runs the block of cbv_ring_step /
 * cbv_plan_zigzag against them.  Local buffers hold a rank's tokens in local order (for every
 * document its front chunk, then its back chunk: the rows of cbv_rank_tokens); masks use global
 * positions computed from cu_seqlens, so results equal the single-GPU ring's.
 * Forward: step 0 writes the rank's running (out_acc, lse_acc); later steps merge into them with
 * the online-softmax identity in the kernel epilogue; with `out` set, the running out is also
 * rounded into that bf16 tensor (pass it at the last step).
 * Backward (zigzag_ring_flash_attn_varlen_backward, the merged-lse identity): the block's
 * gradients, fed the MERGED out_merged / lse_merged of this rank's rows, are ADDED into dq_acc
 * (this rank's rows) and into dk_acc / dv_acc, the fp32 accumulators of src's k/v rows that
 * travel around the ring with k/v and arrive back at their owner after cp hops.
 * Errors: those of cbv_ring_args, plus rank / step outside [0, cp) -> CBV_ERR_BAD_ARG and
 * cu_seqlens[num_docs] != n_local * cp -> CBV_ERR_BAD_CU_SEQLENS. */
typedef struct cbv_ring_step_args {
  uint32_t struct_size;       /* sizeof(cbv_ring_step_args) */
  uint32_t abi_version;       /* CBV_ABI_VERSION */
  int32_t rank, step;
  const void* q;              /* device bf16 [n_local, num_heads, head_dim]: this rank's local q */
  const void* k;              /* device bf16 [n_local, num_kv_heads, head_dim]: src's local k (held at this step) */
  const void* v;
  int64_t n_local;            /* total / cp */
  int32_t num_heads, num_kv_heads, head_dim;
  int32_t num_docs;
  const int32_t* cu_seqlens;  /* host int32 [num_docs+1], GLOBAL */
  int32_t cp;                 /* ranks in the ring, >= 1 */
  int32_t layout;             /* cbv_layout */
  float scale;
  int32_t window;
  float* out_acc;             /* forward: device f32 [n_local, num_heads, head_dim], running out */
  float* lse_acc;             /* forward: device f32 [num_heads, n_local], running lse */
  void* out;                  /* forward: NULL, or device bf16 [n_local, num_heads, head_dim] */
  const void* dout;           /* backward: device bf16 [n_local, num_heads, head_dim] */
  const void* out_merged;     /* backward: device bf16, this rank's merged forward output */
  const float* lse_merged;    /* backward: device f32 [num_heads, n_local], this rank's merged lse */
  float* dq_acc;              /* backward: device f32 [n_local, num_heads, head_dim], += */
  float* dk_acc;              /* backward: device f32 [n_local, num_kv_heads, head_dim] of src's rows, += */
  float* dv_acc;
  void* workspace;
  size_t workspace_bytes;
} cbv_ring_step_args;
size_t cbv_ring_step_fwd_workspace_size(const cbv_ring_step_args* a);
int cbv_ring_step_fwd(const cbv_ring_step_args* a, void* stream);
size_t cbv_ring_step_bwd_workspace_size(const cbv_ring_step_args* a);
int cbv_ring_step_bwd(const cbv_ring_step_args* a, void* stream);

/* ========================================================================= EAGLE-3 cached ring
 * NeMo AutoModel ring_attention, _CachedZigZagRingAttention / cached_zigzag_ring_attention
 * (layout = CBV_LAYOUT_ZIGZAG) and _CachedRingAttention / cached_ring_attention
 * (CBV_LAYOUT_CONTIGUOUS): attention of the packed batch over a KV cache of num_blocks
 * blocks, each [total, num_kv_heads, head_dim] (the pages' list of [B, T, H, D] tensors, or the
 * block axis of [B, num_blocks, T, H, D], with B = 1).  Block 0 is the sequence itself and is
 * attended causally (sliding window optional) the ring way, exactly as cbv_zigzag_ring_fwd;
 * every block i >= 1 adds one key per query token t, the cache entry at the same position
 * (the per-position diagonal): score scale <q_t, cache_k[i][t]>, value cache_v[i][t].  All keys
 * of a row form ONE softmax: the diagonals are merged into block 0's result with the
 * log-sum-exp identity of update_out_and_lse (ring_attention._merge_diag).  The backward is fed
 * the merged out and lse: block 0 by the ring backward, the diagonals in closed form
 * (p_i = exp(s_i - lse), dS_i = p_i (<dO_t, v_i[t]> - <dO_t, out_t>); dv_i[t] and dk_i[t] sum
 * p_i dO_t and scale dS_i q_t over the kv head's q heads; dq_t += scale dS_i k_i[t]).
 * The blocks are passed as host arrays of num_blocks device pointers, so separate tensors and
 * slices of one stacked tensor serve alike; every pointer must be 16-byte aligned.
 * 1 <= num_blocks <= 8 (else CBV_ERR_BAD_ARG); causal only, fused schedule; the other rules,
 * errors and layouts are those of cbv_ring_args.  Every dcache block is written (not added). */
typedef struct cbv_cached_ring_args {
  uint32_t struct_size;        /* sizeof(cbv_cached_ring_args) */
  uint32_t abi_version;        /* CBV_ABI_VERSION */
  const void* q;               /* device bf16 [total, num_heads, head_dim] */
  const void* const* cache_k;  /* host array [num_blocks] of device bf16 [total, num_kv_heads, head_dim] */
  const void* const* cache_v;
  int32_t num_blocks;
  int64_t total;
  int32_t num_heads, num_kv_heads, head_dim;
  int32_t num_docs;
  const int32_t* cu_seqlens;   /* host int32 [num_docs+1], GLOBAL */
  int32_t max_seqlen;          /* 0 or >= every document length */
  int32_t cp;                  /* virtual ranks, >= 1 */
  int32_t layout;              /* cbv_layout */
  float scale;
  int32_t window;
  int32_t deterministic;       /* backward only: as cbv_ring_args.deterministic */
  void* out;                   /* device bf16 [total, num_heads, head_dim]: forward output, backward input */
  float* lse;                  /* device f32 [num_heads, total]: forward output, backward input (merged) */
  const void* dout;            /* backward: device bf16 [total, num_heads, head_dim] */
  void* dq;                    /* backward: device bf16 [total, num_heads, head_dim] */
  void* const* dcache_k;       /* backward: host array [num_blocks] of device bf16 outputs, shaped as cache_k */
  void* const* dcache_v;
  void* workspace;
  size_t workspace_bytes;
} cbv_cached_ring_args;
size_t cbv_cached_ring_fwd_workspace_size(const cbv_cached_ring_args* a);
int cbv_cached_ring_fwd(const cbv_cached_ring_args* a, void* stream);
size_t cbv_cached_ring_bwd_workspace_size(const cbv_cached_ring_args* a);
int cbv_cached_ring_bwd(const cbv_cached_ring_args* a, void* stream);

/* ========================================================================= cache diagonals alone
 * The per-position diagonals of the EAGLE-3 cache (blocks 1..num_blocks-1, as in
 * cbv_cached_ring_fwd / _bwd) applied to a block-0 result computed elsewhere: by Ulysses
 * (ulysses_attention._CachedUlyssesAttention: block 0 over the all-to-all-gathered sequence, the
 * diagonals merged shard-locally, comm-free) or by any caller.  Rows are independent, so the
 * tokens may be any slice of a sequence.  With num_blocks == 1 both calls only round.
 * cbv_cached_diag_merge: out0 is block 0's NORMALISED fp32 output [total, H, D] and lse holds
 *   block 0's lse [H, total] on entry; the merged lse replaces it and the merged output is
 *   rounded into out (bf16).
 * cbv_cached_diag_grad: fed the MERGED out / lse, writes dq = dq0 (block 0's fp32 dq) + the
 *   diagonal terms (bf16) and the gradients of blocks 1..num_blocks-1 into dcache_k / dcache_v
 *   (entries 0 are not touched). */
typedef struct cbv_diag_args {
  uint32_t struct_size;        /* sizeof(cbv_diag_args) */
  uint32_t abi_version;        /* CBV_ABI_VERSION */
  const void* q;               /* device bf16 [total, num_heads, head_dim] */
  const void* const* cache_k;  /* host array [num_blocks] of device bf16 [total, num_kv_heads, head_dim]; [0] unused */
  const void* const* cache_v;
  int32_t num_blocks;          /* 1..8 */
  int64_t total;
  int32_t num_heads, num_kv_heads, head_dim;
  float scale;
  const float* out0;           /* merge: device f32 [total, num_heads, head_dim], block 0 normalised */
  float* lse;                  /* merge: device f32 [num_heads, total], block 0's lse in, merged lse out */
  void* out;                   /* merge: device bf16 [total, num_heads, head_dim] */
  const void* dout;            /* grad: device bf16 [total, num_heads, head_dim] */
  const void* out_merged;      /* grad: device bf16, merged output */
  const float* lse_merged;     /* grad: device f32 [num_heads, total] */
  const float* dq0;            /* grad: device f32 [total, num_heads, head_dim], block 0's dq */
  void* dq;                    /* grad: device bf16 [total, num_heads, head_dim] */
  void* const* dcache_k;       /* grad: host array [num_blocks] of device bf16 outputs; [0] unused */
  void* const* dcache_v;
} cbv_diag_args;
int cbv_cached_diag_merge(const cbv_diag_args* a, void* stream);
int cbv_cached_diag_grad(const cbv_diag_args* a, void* stream);

/* ========================================================================= layout helpers
 * cbv_convert_f32_bf16: dst[i] = bf16_rne(src[i] * mul), n elements (n a multiple of 4, both
 *   16-byte aligned): the finalise of an fp32 accumulator.
 * cbv_swap_leading_axes: dst [b][a][row] = src [a][b][row] for an array of a * b rows of
 *   row_bytes bytes (a multiple of 4): the reordering on either side of an all-to-all that turns
 *   sequence shards into head shards and back (ulysses_attention._gather_seq_scatter_heads,
 *   _scatter_seq_gather_heads, _gather_lse, _scatter_lse).  src and dst must not overlap. */
int cbv_convert_f32_bf16(const float* src, void* dst, int64_t n, float mul, void* stream);
int cbv_swap_leading_axes(const void* src, void* dst, int64_t a, int64_t b, int64_t row_bytes, void* stream);

/* ========================================================================= block backward
 * One block's backward fed the MERGED softmax statistics (zigzag_ring_attention._block_backward;
 * ulysses_attention._block0_backward): with P = exp(scale q k^T - lse) over the block's visible
 * pairs, dV += P^T dO, dS = P (dO V^T - Delta), Delta = rowsum(dO * out), dQ += scale dS K,
 * dK += scale dS^T Q.  dq_acc, dk_acc, dv_acc are device f32 accumulators that are ADDED
 * to (token-major, like q and k).  Documents and positions as in cbv_attn_block_fwd. */
typedef struct cbv_block_bwd_args {
  uint32_t struct_size;
  uint32_t abi_version;
  const void* dout;    /* device bf16 [total_q, num_heads, head_dim] */
  const void* q;       /* device bf16 [total_q, num_heads, head_dim] */
  const void* k;       /* device bf16 [total_k, num_kv_heads, head_dim] */
  const void* v;
  const void* out;     /* device bf16 [total_q, num_heads, head_dim], the MERGED output */
  const float* lse;    /* device f32 [num_heads, total_q], the MERGED lse */
  int64_t total_q, total_k;
  int32_t num_heads, num_kv_heads, head_dim;
  int32_t num_docs;
  const int32_t* cu_seqlens_q;  /* host */
  const int32_t* cu_seqlens_k;  /* host */
  const int32_t* q_pos_base;    /* host or NULL */
  const int32_t* k_pos_base;    /* host or NULL */
  float scale;
  int32_t causal;
  int32_t window;
  int32_t deterministic;  /* 1: the block's dq is summed in 64-bit fixed point, then added to dq_acc
                             once: bit-reproducible (as cbv_ring_args.deterministic) */
  float* dq_acc;       /* device f32 [total_q, num_heads, head_dim], += */
  float* dk_acc;       /* device f32 [total_k, num_kv_heads, head_dim], += */
  float* dv_acc;
  void* workspace;
  size_t workspace_bytes;
} cbv_block_bwd_args;
size_t cbv_block_bwd_workspace_size(const cbv_block_bwd_args* a);
int cbv_attn_block_bwd(const cbv_block_bwd_args* a, void* stream);

/* ========================================================================= paged KV-parallel prefill
 * NKI attention_kv_parallel_segmented_cte: q token i (position global_q_offset + i) attends
 * causally (plus optional sliding window) to the whole context, which is spread over
 * `shards` KV shards of a paged cache.  Shard r reads its local tokens through row r of
 * block_tables; local token t sits at global position r * n_local + t (CBV_KV_CONTIGUOUS,
 * n_local = blocks_per_shard * block_size) or ((t / bs) * shards + r) * bs + t % bs
 * (CBV_KV_ROUND_ROBIN: shard r holds global blocks r, r + shards, ...).  Every shard's KV
 * is walked in segments of seg_size tokens and the partial results are merged by online
 * softmax: across segments and shards on chip in one launch (shard_out == NULL), or per
 * shard into shard_out / shard_lse for a later cbv_attn_merge (shard_out != NULL).
 * GQA: q head h reads kv head h / (num_heads / num_kv_heads).
 * Requirements: block_size is a power of two in [8, 128] (a page is whole 8-row atoms of the
 * 128-byte-swizzled tiles the tensor cores read, and a 128-key tile is whole pages); seg_size > 0,
 * rounded up to a multiple of 128 (whole key tiles): a performance parameter only, since the
 * segments are merged by the online-softmax identity and the result does not depend on it. */
typedef struct cbv_kvp_args {
  uint32_t struct_size;
  uint32_t abi_version;
  const void* q;              /* device bf16, element (h, i, d) at q[h*q_stride_head + i*q_stride_token + d] */
  int64_t q_stride_head, q_stride_token;  /* elements; [HQ, S, D] contiguous: S*D and D */
  int32_t q_len, num_heads, num_kv_heads, head_dim;
  const void* k_cache;        /* device bf16 [num_blocks, num_kv_heads, block_size, head_dim] */
  const void* v_cache;
  int32_t num_blocks, block_size;
  const int32_t* block_tables; /* device int32 [shards, blocks_per_shard] of page ids */
  int32_t shards, blocks_per_shard;
  int32_t kv_mode;            /* cbv_kv_mode */
  int32_t seg_size;
  float scale;
  int32_t global_q_offset;
  int32_t sliding_window;     /* 0 = disabled */
  int32_t tp_out;             /* 0: out is [num_heads, q_len, head_dim]; 1: transposed, [num_heads, head_dim, q_len] */
  void* out;                  /* device bf16 merged result, laid out as tp_out says */
  float* lse;                 /* device f32 [num_heads, q_len] or NULL */
  float* shard_out;           /* NULL, or device f32 [shards, num_heads, q_len, head_dim] per-shard partials */
  float* shard_lse;           /* with shard_out: device f32 [shards, num_heads, q_len] */
  void* workspace;
  size_t workspace_bytes;
  /* This call's block tables are shards shard_base .. shard_base + shards - 1 of total_shards
   * (0: total_shards = shards, shard_base = 0).  Key positions follow the global shard index, so a
   * process that holds only its own shards' pages computes their partials, which merge with the
   * other processes' ones by the log-sum-exp identity (the KV-parallel prefill over real ranks).
   * Requires 0 <= shard_base and shard_base + shards <= total_shards. */
  int32_t shard_base;
  int32_t total_shards;
} cbv_kvp_args;
/* Workspace bytes for a call with these arguments on the current device.  The size depends on
 * the device's SM count: when the last wave of the prefill's tasks would fill at most half the
 * SMs, those tasks run as two halves each, and the halves' fp32 partial results (8 bytes per
 * element of out, 8 per lse entry) live in the workspace.  Query it on the device that runs
 * the call; a smaller workspace makes the call return CBV_ERR_WORKSPACE_TOO_SMALL. */
size_t cbv_kvp_workspace_size(const cbv_kvp_args* a);
int cbv_kvp_segmented_prefill(const cbv_kvp_args* a, void* stream);

/* ========================================================================= varlen decode
 * qsa_fa_fallback.py, triton_varlen_attn_func: sequence s has exactly one query row
 * cu_seqlens_q[s] and keys [cu_seqlens_k[s], cu_seqlens_k[s+1]); q head h reads kv head
 * h / (num_heads / num_kv_heads); no mask; an empty key range writes zeros.  The offsets
 * are DEVICE arrays read by the kernel, so their contents may change between CUDA-graph
 * replays.  validate != 0 copies cu_seqlens_q to the host (synchronising the stream) and
 * returns CBV_ERR_Q_LEN_NOT_ONE unless every sequence has one query row; pass 0 while
 * capturing a graph.  The output row of sequence s is cu_seqlens_q[s].
 * Requirements: num_heads / num_kv_heads <= 16. */
typedef struct cbv_decode_args {
  uint32_t struct_size;
  uint32_t abi_version;
  const void* q;              /* device bf16 [total_q, num_heads, head_dim] */
  const void* k;              /* device bf16 [total_k, num_kv_heads, head_dim] */
  const void* v;
  void* out;                  /* device bf16 [total_q, num_heads, head_dim] */
  const int32_t* cu_seqlens_q; /* device int32 [num_seqs+1] */
  const int32_t* cu_seqlens_k; /* device int32 [num_seqs+1] */
  int32_t num_seqs;
  int64_t total_q, total_k;
  int32_t num_heads, num_kv_heads, head_dim;
  float scale;
  int32_t validate;
  void* workspace;            /* device, >= cbv_decode_workspace_size() bytes (status word) */
  size_t workspace_bytes;
} cbv_decode_args;
size_t cbv_decode_workspace_size(const cbv_decode_args* a);
int cbv_varlen_decode(const cbv_decode_args* a, void* stream);

/* ========================================================================= diagnostics
 * Tests of the failure path, which must fault or hang nothing.  The pages have no counterpart.
 * cbv_debug_ring_fwd_stalled runs the fused ring forward of cbv_zigzag_ring_fwd with its copy
 * producer told to issue no loads at all and every wait limited to wait_limit_ns (1e5..1e9 ns)
 * instead of the usual 2 s.  Every consumer's wait then runs out before any copy or
 * tensor-core operation is in flight: the first one to give up records its code in the status
 * word at the start of a->workspace, the others see it and leave, and the kernel ends normally
 * (out and lse are left unwritten).  cbv_read_status() then returns CBV_ERR_TIMEOUT with the
 * raw code, and the stream and context remain usable.  Arguments as cbv_zigzag_ring_fwd (fused
 * schedule only); a limit outside the range -> CBV_ERR_BAD_ARG. */
int cbv_debug_ring_fwd_stalled(const cbv_ring_args* a, uint64_t wait_limit_ns, void* stream);

/* ========================================================================= ring forward without allocation
 * The pages have no counterpart for this call; it serves callers that cannot allocate.
 * cbv_zigzag_ring_fwd takes its scratch (status word and tile schedule) from a workspace the
 * caller allocates.  Callers that cannot call cudaMalloc where they run attention (an
 * allocation-free serving loop with a memory budget fixed at start-up, a runtime that owns all
 * device memory through its own allocator, a plain C host with no device allocator) can use
 * this variant instead: it computes exactly what cbv_zigzag_ring_fwd computes with the fused
 * schedule (a->schedule is ignored: the fused schedule always runs), but its scratch is a fixed
 * array of cbv_noalloc_scratch_bytes() bytes (1 MiB) compiled into the library, which every GPU
 * that loads the library holds until the process exits.  a->workspace and a->workspace_bytes
 * are ignored; inputs and outputs are still the caller's.  It calls no cudaMalloc, cudaFree or
 * allocating library routine.
 * - Every call looks up the array's device address (cudaGetSymbolAddress) in the current
 *   device's context; the first call on a device also loads the library's module into that
 *   context, so make that first call before any stream capture.
 * - Every call, from any thread or stream, shares the one array, and each call overwrites what
 *   the last one left there: calls that overlap on the GPU race.  Serialise them (one stream,
 *   or events between streams).
 * - A problem whose tile schedule would exceed the array returns CBV_ERR_WORKSPACE_TOO_SMALL
 *   with a message; nothing is launched.
 * - Argument errors are those of cbv_zigzag_ring_fwd. */
size_t cbv_noalloc_scratch_bytes(void);
int cbv_zigzag_ring_fwd_noalloc(const cbv_ring_args* a, void* stream);
/* The status word the last cbv_zigzag_ring_fwd_noalloc call on the current device left in the
   static array (synchronises `stream`, which should be the stream that call used).
   *status_out receives the raw kernel code (0 = ok); returns CBV_ERR_TIMEOUT if a kernel gave
   up a wait, CBV_OK otherwise. */
int cbv_noalloc_read_status(int* status_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CBV_H */
