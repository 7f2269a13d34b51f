// Kernel parameter blocks and launchers shared by the C ABI and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "plan.h"

namespace cbv {

// Every kernel launch of the library ends with `return launched();`: it counts the launch for
// the calling thread (cbv_launch_count) and returns the launch's error code.
int launched();
size_t launch_count();
// Measurement hook (cbv_set_kernel_events): when set for the calling thread, the attention kernels
// (forward, backward, decode) record the start event on their stream right before their launch and
// the stop event right after it.  Both return the record's error code (0 when no hook is set).
void set_kernel_events(cudaEvent_t start, cudaEvent_t stop);
int kernel_event_start(cudaStream_t stream);
int kernel_event_stop(cudaStream_t stream);

// Output modes of the forward kernel's epilogue.
enum OutMode : int32_t {
  kOutBf16 = 0,   // write normalised out (bf16) and lse
  kOutF32 = 1,    // write normalised out (fp32) and lse
  kOutMerge = 2,  // merge into a running fp32 (out, lse) pair in place (online-softmax identity)
};

struct FwdParams {
  CUtensorMap tm_q;  // (D, H, T) bf16, box (64, 1, 128), 128B swizzle
  CUtensorMap tm_k;  // ring: (D, Hkv, T) box (64, 1, 128); paged: (D, bs, Hkv, pages) box (64, bs, 1, 1)
  CUtensorMap tm_v;
  const TileTask* tasks;
  const Seg* segs;
  int32_t num_tasks;
  int32_t num_heads;
  int32_t heads_per_kv;
  float scale_log2;  // softmax scale * log2(e)
  int32_t window;
  void* out;
  int64_t out_stride_t, out_stride_h;  // elements
  int64_t out_stride_d;  // bf16 out only: 0 or 1 = head dims contiguous; > 1 = transposed ([H, D, S]) output
  float* lse;
  int64_t lse_stride_h, lse_stride_t;  // elements
  int32_t out_mode;
  int64_t out_shard_stride, lse_shard_stride;  // per-shard outputs (task.aux = shard >= 0)
  // with split_halves, the tasks from split_from on run as two halves each: CTA split_from + 2j
  // takes segments [0, split1) of task split_from + j and CTA split_from + 2j + 1 the rest.  A
  // half writes its normalised partial (out, lse) in fp32 to slot 0 or 1 of half_out
  // [2][H][S][D] and half_lse [2][H][S] (half_rows = H * S, half_q_len = S).
  int32_t split_halves, split_from;
  float* half_out;
  float* half_lse;
  int64_t half_rows, half_q_len;
  // paged KV
  const int32_t* block_tables;  // [shards, blocks_per_shard]
  int32_t blocks_per_shard, block_size, shards, kv_mode, n_local;
  int32_t shard_base, total_shards;  // the call's shard s is shard shard_base + s of total_shards (positions)
  int* status;  // device status word (0 = ok)
  // diagnostics: every wait gives up after wait_limit_ns (0 = the default limit); with
  // withhold_loads the producer issues no copy at all, so every wait runs out (the test of the
  // timeout path: no copy or tensor-core operation is ever in flight when the kernel gives up)
  uint64_t wait_limit_ns;
  int32_t withhold_loads;
  // extents the CBV_DEBUG build checks coordinates against: rows of q / out, rows of k / v (paged:
  // pages of the cache)
  int64_t q_rows, kv_rows;
};

struct BwdParams {
  CUtensorMap tm_q;     // (D, H, T) bf16, box (64, 1, 64)
  CUtensorMap tm_do;    // (D, H, T) bf16, box (64, 1, 64)
  CUtensorMap tm_k;     // (D, Hkv, T) bf16, box (64, 1, 128)
  CUtensorMap tm_v;
  CUtensorMap tm_k8;    // the same, box (64, 1, 8): tiles of two key ranges load in 8-row pieces
  CUtensorMap tm_v8;
  CUtensorMap tm_dq;    // (D, H, T) fp32, box (D/4, 1, 16), no swizzle (reduce-add target)
  const TileTask* tasks;
  const Seg* segs;
  int32_t num_tasks;
  int32_t num_heads, heads_per_kv, num_kv_heads;
  float scale, scale_log2;
  int32_t window;
  CUtensorMap tm_rows;  // (2 Tpad, H) fp32: {merged lse * log2(e), rowsum(dO * O)} per q row, box (132, 1)
  // dk/dv outputs: bf16 (write) or fp32 (accumulate)
  void* dk;
  void* dv;
  int64_t dkv_stride_t, dkv_stride_h;
  int32_t dkv_accumulate;  // 0: write bf16; 1: add into fp32
  // non-null: dq accumulates here as 64-bit fixed point in units of 2^-32, added by integer
  // reduces, so the sum does not depend on the order the key tiles' partials arrive in
  // (deterministic mode); null: fp32 reduce-adds through tm_dq.  Layout: see fixed_index().
  unsigned long long* dq_fixed;
  int64_t dq_fixed_tpad;
  int64_t q_rows, kv_rows;  // extents the CBV_DEBUG build checks rows against
  // > 0: each CTA prefetches into L2 the key and value tile of task blockIdx.x + prefetch_ahead
  // (the SM count: roughly the task that starts on an SM when this wave's CTAs finish)
  int32_t prefetch_ahead;
  int* status;
};

// Forward with two 128-row q tiles per task (task.rows <= 256); paged selects the page-table K/V loads.
int launch_fwd_pingpong(const FwdParams& p, int head_dim, bool paged, int grid, cudaStream_t stream);
int launch_bwd(const BwdParams& p, int head_dim, int grid, cudaStream_t stream);

// Per (token, head): Delta = rowsum(dout * out) and lse * log2(e), written [H, t_pad]
// (t_pad = total rounded up to a multiple of 4).  Optionally zeroes a dq accumulator: an fp32
// [T, H, D] one in the same pass (dq_f32_zero), or any other (dq_other_zero, other_bytes) by memset.
int launch_bwd_preprocess(const void* dout, const void* out, const float* lse, int64_t total, int64_t t_pad,
                          int32_t heads, int32_t head_dim, float* rows, float* dq_f32_zero, void* dq_other_zero,
                          size_t other_bytes, cudaStream_t stream);
// Host -> device copy of a small host buffer without a copy engine: the bytes travel inside the
// launch parameters of one kernel per 30 KB.  A cudaMemcpyAsync from pageable host memory
// would block the calling thread until the stream had drained and queue behind any large
// transfer on the copy engine; this neither blocks nor queues.  dst 16-byte aligned.
int launch_inline_copy(void* dst, const void* src, size_t bytes, cudaStream_t stream);
// A schedule image (groups at 0, tiles at off_tiles, then segments) written to image_dst and
// expanded into `tasks`: one launch when the image fits one payload, else copy + expansion.  The
// single launch also clears *status (when non-null) and sets *status_cleared; otherwise the caller
// must clear it.
int launch_schedule(void* image_dst, const void* image, size_t bytes, size_t off_tiles, int ngroups, TileTask* tasks,
                    int ntasks, int* status, cudaStream_t stream, bool* status_cleared);
// The task list from its compact form (plan.h: PlanGroup): task i of group g is tile
// first_tile + (i - first_task) % ntiles with head (i - first_task) / ntiles.
int launch_expand_tasks(const PlanGroup* groups, int ngroups, const TileTask* tiles, TileTask* tasks, int ntasks,
                        cudaStream_t stream);
// dst [B][A][row] = src [A][B][row] (row_bytes a multiple of 4; 16-byte moves when aligned).
int launch_swap01(const void* src, void* dst, int64_t A, int64_t B, int64_t row_bytes, cudaStream_t stream);
// fp32 [T, H, D] -> bf16, times `mul`.
int launch_convert_bf16(const float* src, void* dst, int64_t n, float mul, cudaStream_t stream);
// The two halves of each of `ntasks` split prefill tasks (q tiles of up to 256 rows), whose
// partial (out, lse) sit in slots 0 and 1 of part [2][H][S][D] and part_lse [2][H][S], merged into
// the bf16 out (element (h, t, d) at h * out_stride_h + t * out_stride_t + d * out_stride_d) and,
// when lse is not null, lse [H][S].
int launch_merge_halves(const TileTask* tasks, int ntasks, const float* part, const float* part_lse, int heads,
                        int64_t q_len, int head_dim, void* out, int64_t out_stride_h, int64_t out_stride_t,
                        int64_t out_stride_d, float* lse, cudaStream_t stream);
// fp32 [H, S, D] -> bf16 [H, D, S] (the prefill's transposed output).
int launch_convert_bf16_transposed(const float* src, void* dst, int H, int64_t S, int D, cudaStream_t stream);
// The fixed-point dq accumulator of the deterministic backward is [H][4][t_pad][D/4]: each of the
// four dQ readout warps owns a quarter of the head dims, and its slice of consecutive q rows is
// contiguous, so one bulk reduce adds it.  t_pad = fixed_tpad(T) leaves room for a full 64-row
// q tile starting at any row < T.
__host__ __device__ inline int64_t fixed_tpad(int64_t T) { return (T + 64 + 7) / 8 * 8; }
__host__ __device__ inline int64_t fixed_index(int64_t t, int h, int d, int64_t tpad, int D) {
  const int dw = D / 4;
  return ((int64_t)(h * 4 + d / dw) * tpad + t) * dw + d % dw;
}
// Fixed-point dq (units of 2^-32, the layout above) -> bf16 [T, H, D], or added into fp32 [T, H, D].
int launch_fixed_to_bf16(const unsigned long long* src, void* dst, int64_t T, int H, int D, cudaStream_t stream);
int launch_fixed_add_f32(const unsigned long long* src, float* dst, int64_t T, int H, int D, cudaStream_t stream);

// EAGLE-3 cached attention diagonals (cached.cu).  Each cache block is [T, Hkv, D] bf16 at its
// own address; lse is [H, T] fp32.  diag_merge: o32 holds block 0's normalised fp32 output;
// writes out (bf16) and the merged lse in place.  diag_grad: with the merged out / lse, writes
// dq = dq_acc + diagonal terms (bf16) and the gradients of blocks 1..nb-1.
constexpr int kCacheMaxBlocks = 8;
struct CacheBlocks {
  const void* k[kCacheMaxBlocks];
  const void* v[kCacheMaxBlocks];
  void* dk[kCacheMaxBlocks];
  void* dv[kCacheMaxBlocks];
};
int launch_diag_merge(const void* q, const CacheBlocks& cb, int nb, int64_t T, int H, int Hkv, int D, float scale,
                      const float* o32, float* lse, void* out, cudaStream_t stream);
// Block 0's dq comes as fp32 (dq_acc) or, in deterministic mode, as 64-bit fixed point (dq_fixed).
int launch_diag_grad(const void* q, const CacheBlocks& cb, int nb, int64_t T, int H, int Hkv, int D, float scale,
                     const void* dout, const void* out, const float* lse, const float* dq_acc,
                     const unsigned long long* dq_fixed, void* dq, cudaStream_t stream);
// Standalone merge of (block_out, block_lse) into a running fp32 (out, lse).
int launch_merge(float* out, float* lse, const void* block_out, int32_t block_out_is_f32, const float* block_lse,
                 float* weight_out, int64_t seqlen, int32_t heads, int32_t head_dim, cudaStream_t stream);
// One-query varlen GQA decode.
struct DecodeParams {
  CUtensorMap tm_k;  // (D, Hkv, Tk) bf16, box (64, 1, 32), 128B swizzle
  CUtensorMap tm_v;
  const void* q;      // [Tq, HQ, D]
  void* out;          // [Tq, HQ, D]
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t num_seqs, hq, hkv, head_dim;
  int64_t total_q, total_k;  // every sequence's offsets are checked against these
  int32_t heads_per_cta;  // kv heads per CTA: 4, 2 or 1, dividing hkv (the TMA box never leaves the tensor)
  float scale_log2;
  int* status;
};
int launch_decode(const DecodeParams& p, cudaStream_t stream);

}  // namespace cbv
