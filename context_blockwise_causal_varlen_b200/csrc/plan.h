// Host planner: zig-zag / contiguous layouts over virtual ranks, and the tile
// schedules the kernels consume.
//
// The layout rules follow the NeMo AutoModel zig-zag ring page (module
// docstring, get_half_index, get_half_lse, _block_forward): each document is
// cut into 2*cp equal chunks and virtual rank r owns chunk r and chunk
// 2*cp-1-r; its local cu_seqlens are the global ones divided by cp and the
// half-blocks use the global ones divided by 2*cp.  The contiguous layout (the
// ring_attention page) gives rank r the r-th of cp equal pieces of every
// document.  All positions are global rows in natural packed order, so masks
// (causal, sliding window) mean the same thing in every block.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

namespace cbv {

// A stationary tile: one CTA owns it (q tile in the forward, k tile in the backward).
struct TileTask {
  int32_t row0;  // first row of the tile in its tensor
  int32_t rows;  // valid rows (<= tile height)
  int32_t pos0;  // position of row0 (positions of the tile are pos0 + i)
  int32_t seg0;  // first streamed segment of this tile
  int32_t nseg;  // number of streamed segments
  int32_t aux;   // paged prefill: shard of the single-shard variant (-1 = all shards)
  int32_t head;  // head (q head in the forward, kv head in the backward); one task per tile and head
  int32_t work;  // estimated visible pairs / 256 (scheduling weight)
  // backward: a second key range in the same tile (split1 > 0).  Tile rows [0, split1)
  // hold rows row0.. (valid: the first `rows`), tile rows [split1, 128) hold rows row1..
  // (valid: the first rows1, positions pos1..).  split1 is a multiple of 8.
  // paged prefill forward: split1 is the segment where the task is cut when it runs as two
  // halves of about equal visible work.
  int32_t row1, pos1, rows1, split1;
};

// A streamed range: rows [row0, row0 + rows) attended by (or attending) the tile.
struct Seg {
  int32_t row0;   // first row (paged prefill: first shard-local token)
  int32_t rows;
  int32_t pos0;   // position of row0 (paged prefill: unused)
  int32_t flags;  // kSegCausal | kSegBlockStart | (shard << kSegShardShift)
};

constexpr int32_t kSegCausal = 1;        // apply kpos <= qpos inside this segment
constexpr int32_t kSegBlockStart = 2;    // first segment of a new ring block / shard
constexpr int32_t kSegShardShift = 8;

enum Layout : int32_t { kZigZag = 0, kContiguous = 1 };
enum KvMode : int32_t { kKvContiguous = 0, kKvRoundRobin = 1 };

// ---------------------------------------------------------------- layout primitives (exported bit-exact)
// All return an empty string on success, else an error message.
std::string check_cu_seqlens(const int32_t* cu, int32_t num_docs);
std::string check_divisible(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout);
void local_cu_seqlens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t* out);
void half_cu_seqlens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t* out);
int64_t get_half_index(const int32_t* cu_local, int32_t num_docs, bool front, int32_t* out);
int64_t rank_tokens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t rank, Layout layout, int32_t* out);
void rank_pair_counts(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window, int64_t* out);

// One block of the ring: which rank's k/v arrive at step s and which chunks meet.
enum BlockKind : int32_t { kDiag = 0, kFrontK = 1, kBackQ = 2, kFull = 3, kSkip = 4 };
void ring_step(int32_t rank, int32_t step, int32_t cp, Layout layout, int32_t* src, int32_t* kind);

// The blocks of the ring as the pages run them: rank r's flash call at step s, with its q
// rows (all local rows, or the back halves), the k rows of src (all of src's local rows, or
// its front halves), the cu_seqlens each side uses (local G/cp or halved G/(2cp)) and the
// causal flag.  Rows are listed as runs of consecutive global rows, document by document in
// local order (front chunk before back chunk).
struct RowRun {
  int32_t doc, row0, rows, pos0, local0;
};
struct RingBlock {
  int32_t rank, step, src, kind, causal, q_half, k_half;
  int32_t q_run0, q_nruns, k_run0, k_nruns;
};
void ring_blocks(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, std::vector<RingBlock>* blocks,
                 std::vector<RowRun>* runs);

// A pair of chunks of one document that meet in a block: q chunk x against k chunk y.
struct ChunkPair {
  int32_t doc, rank, step, q_chunk, k_chunk, causal;
};
// Every chunk pair of every block, rank-major, step order inside a rank.
std::vector<ChunkPair> ring_chunk_pairs(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout,
                                        int32_t window, int32_t only_step /* -1 = all */);

// ---------------------------------------------------------------- tile schedules
// Tasks come in groups (e.g. one per document): inside a group, head by head, the group's tiles
// in order.  Task i of a group is tile first_tile + i % ntiles for head i / ntiles, so the
// tiles and this table describe the task list compactly (the device expands it).
struct PlanGroup {
  int32_t first_task, first_tile, ntiles, pad;
};

struct Plan {
  std::vector<TileTask> tasks;  // expanded: one per tile and head, in launch order
  std::vector<Seg> segs;
  std::vector<TileTask> tiles;  // compact form of `tasks`: the tiles of every group, in order
  std::vector<PlanGroup> groups;
};

// Forward over the ring: one task per 128-row q tile (inside one chunk, i.e. one virtual
// rank's rows) per head; segments = the k chunks of every block the tile's chunk meets, in
// ring-step order (only_step >= 0: that step only).  With `coalesce`, chunks that sit next
// to each other in memory are visited as one run, in position order: the same (q, k) pairs,
// merged on chip in a different order, with fewer ragged k tiles.
Plan plan_ring_fwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window, int32_t heads,
                   int32_t only_step, int32_t tile_m, bool coalesce);
// Backward over the ring: one task per 128-row k tile per kv head, segments = the q chunks
// that meet the tile's chunk (all blocks), coalesced into runs of adjacent rows.
Plan plan_ring_bwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window, int32_t kv_heads,
                   int32_t tile_n);
// One ring step of one rank on LOCAL buffers, for the ring over real ranks: q rows are rows of
// `rank`'s local sequence, k rows rows of the local sequence of the step's source rank, and
// positions stay global, so the masks mean what they mean in the single-GPU ring.
// Forward: one task per 128-row q tile of every chunk of `rank` that the block touches (per head),
// segments = the source chunks it meets.  Backward: one task per 128-row k tile of every source
// chunk the block touches (per kv head), segments = the q chunks of `rank` that meet it.
Plan plan_ring_step_fwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window,
                        int32_t heads, int32_t rank, int32_t step, int32_t tile_m);
Plan plan_ring_step_bwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window,
                        int32_t kv_heads, int32_t rank, int32_t step, int32_t tile_n);

// One varlen block with explicit per-document positions.
Plan plan_block_fwd(const int32_t* cu_q, const int32_t* cu_k, const int32_t* qbase, const int32_t* kbase,
                    int32_t num_docs, bool causal, int32_t window, int32_t heads, int32_t tile_m);
Plan plan_block_bwd(const int32_t* cu_q, const int32_t* cu_k, const int32_t* qbase, const int32_t* kbase,
                    int32_t num_docs, bool causal, int32_t window, int32_t kv_heads, int32_t tile_n);
// Paged KV-parallel prefill: one task per 128-row q tile per q head; segments = seg_size
// pieces of every shard's local KV (or of one shard when per_shard is set, one task per shard).
// The call's shards are shards shard_base .. shard_base + shards - 1 of total_shards (positions
// follow the global index).
Plan plan_kvp(int32_t q_len, int32_t heads, int32_t shards, int32_t n_local, int32_t seg_size, KvMode mode,
              int32_t block_size, int32_t global_q_offset, int32_t window, bool per_shard, int32_t tile_m,
              int32_t shard_base = 0, int32_t total_shards = 0);

// Global position of shard-local token t (paged prefill).
inline int64_t kvp_position(int32_t shard, int64_t t, int32_t n_local, int32_t block_size, int32_t shards, KvMode mode) {
  if (mode == kKvRoundRobin) return ((t / block_size) * shards + shard) * (int64_t)block_size + t % block_size;
  return (int64_t)shard * n_local + t;
}

}  // namespace cbv
