// Block forward on tcgen05: flash-style attention of up to 256 q rows (two 128-row
// tiles, "ping-pong") against a list of k/v segments, returning (out, lse) or merging
// into a running pair.
//
// This is the per-block kernel of the NeMo AutoModel zig-zag ring page
// (_block_forward: one flash varlen forward block) and, in its paged instantiation,
// of the KV-parallel segmented prefill (NKI attention_kv_parallel_segmented_cte:
// per-shard segment loop over a paged cache with online softmax).  Consecutive
// segments belonging to different ring blocks (or shards) are combined by the
// online-softmax log-sum-exp identity (update_out_and_lse) applied in place to the
// TMEM accumulator; with out_mode = kOutMerge the epilogue applies the same identity
// to a running (out, lse) pair in HBM, so no separate merge pass is needed.
//
// The two q tiles A and B of a CTA belong to the same head and stream the same k/v
// tiles, so the tensor core never waits for one softmax: while warpgroup A turns
// S_A into P_A, the tensor core computes S_B or PV_B, and the other way round.
// A task of a single q tile (a chunk's ragged last tile) splits its k tiles instead:
// both halves hold the same q rows, A takes the even k tiles and B the odd ones, and
// the epilogue merges the two partial softmax states with the log-sum-exp identity,
// so the tensor core still alternates between two independent chains.
// P never leaves TMEM: the softmax writes P (bf16, two per 32-bit column) over the
// S columns it has just read, and PV takes its A operand from TMEM.
//
// Warps: 0 TMA producer, 1 UMMA issuer (+ TMEM owner), 2-5 softmax / epilogue of
// tile A, 6-9 softmax / epilogue of tile B.  TMEM columns: S_A (and P_A) [0,128),
// S_B (and P_B) [128,256), O_A [256, 256+D), O_B [256+D, 256+2D).
#include "kernels.h"
#include "ptx.cuh"

namespace cbv {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 320;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: keep a stale max while it is within 2^8

// Scores outside the columns [lo, hi] of this thread's row set to -inf, 32 columns at a time: a
// chunk that every row of the warp sees whole is skipped, the others are tested column by column.
// On a window's edge tile most chunks are whole for all 32 rows of a warp.  (A separate branch
// that cleared the chunks no row sees pushed the kernel's scores into local memory.)  The warp
// must be converged.
template <int N>
__device__ __forceinline__ void mask_outside(uint32_t (&s)[N], int32_t lo, int32_t hi) {
#pragma unroll
  for (int c0 = 0; c0 < N; c0 += 32) {
    if (!__all_sync(0xffffffffu, lo <= c0 && hi >= c0 + 31)) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (c0 + e < lo || c0 + e > hi) s[c0 + e] = __float_as_uint(-INFINITY);
    }
  }
}

struct KTile {
  int32_t k_row;   // first row (non-paged: tensor row; paged: shard-local token)
  int32_t kpos0;   // position of column 0 (paged: position of the tile's first token)
  int32_t kmax;    // largest position in the tile
  int32_t nvalid;  // valid columns
  int32_t causal;
  int32_t shard;
};

struct KIter {
  int32_t si = 0, j = 0, jn = 0;
  Seg seg;
};

// global position of shard-local token t of the call's shard `shard` of a paged KV cache (its global
// index is shard_base + shard of total_shards; block_size is a power of two: the call accepts only
// divisors of 128)
__device__ __forceinline__ int32_t kvp_position(const FwdParams& p, int32_t shard, int32_t t) {
  if (p.kv_mode == kKvRoundRobin) {
    const int lbs = __ffs(p.block_size) - 1;
    return ((((t >> lbs) * p.total_shards + p.shard_base + shard)) << lbs) + (t & (p.block_size - 1));
  }
  return (p.shard_base + shard) * p.n_local + t;
}

// k tiles that at least one row of q positions [qp0, qp1] can see.  Every role runs
// its own copy and sees the same sequence.
template <bool PAGED>
__device__ __forceinline__ bool next_ktile(const FwdParams& p, const TileTask& t, int32_t qp0, int32_t qp1,
                                           KIter& it, KTile& r) {
  const int32_t W = p.window;
  while (true) {
    if (it.j >= it.jn) {
      if (it.si >= t.nseg) return false;
      it.seg = p.segs[t.seg0 + it.si];
      it.si++;
      if (!PAGED) {
        const bool cz = (it.seg.flags & kSegCausal) || W > 0;
        int32_t cmax = it.seg.rows - 1, cmin = 0;
        if (cz) cmax = min(cmax, qp1 - it.seg.pos0);
        if (W > 0) cmin = max(0, qp0 - W + 1 - it.seg.pos0);
        if (cmax < cmin) {
          it.j = it.jn = 0;
          continue;
        }
        it.j = cmin / BN;
        it.jn = cmax / BN + 1;
      } else {
        it.j = 0;
        it.jn = (it.seg.rows + BN - 1) / BN;
      }
    }
    const int32_t c0 = it.j++ * BN;
    r.nvalid = min(BN, it.seg.rows - c0);
    r.k_row = it.seg.row0 + c0;
    r.causal = it.seg.flags & kSegCausal;
    if (!PAGED) {
      r.shard = 0;
      r.kpos0 = it.seg.pos0 + c0;
      r.kmax = r.kpos0 + r.nvalid - 1;
    } else {
      r.shard = it.seg.flags >> kSegShardShift;
      r.kpos0 = kvp_position(p, r.shard, r.k_row);
      r.kmax = kvp_position(p, r.shard, r.k_row + r.nvalid - 1);
      if (r.kpos0 > qp1) continue;
      if (W > 0 && r.kmax < qp0 - W + 1) continue;
    }
    return true;
  }
}

template <int D>
struct PPSmem {
  static constexpr uint32_t kTile = BM * D * 2;  // a 128 x D bf16 tile
  static constexpr uint32_t kQ = 0;              // Q_A, Q_B
  static constexpr uint32_t kK = kQ + 2 * kTile; // 2 stages
  static constexpr uint32_t kV = kK + 2 * kTile; // 2 stages
  static constexpr uint32_t kBars = kV + 2 * kTile;
  static constexpr uint32_t kStats = kBars + 256;       // split tasks: half B's {m, l, rounded l} per row
  static constexpr uint32_t kEnd = kStats + BM * 16;
  static constexpr uint32_t kDynamic = (kEnd + 1024) < 120 * 1024 ? 120 * 1024 : (kEnd + 1024);
  static_assert(kDynamic <= 232448, "shared memory budget");
};

enum PBar {
  pQFull = 0,
  pKFull = 1,    // +stage
  pVFull = 3,    // +stage
  pKEmpty = 5,   // +stage
  pVEmpty = 7,   // +stage
  pSFull = 9,    // +tile
  pPFull = 11,   // +tile
  pPVDone = 13,  // +tile
  pODone = 15,
  pPHalf = 16,   // +tile: the first 64 columns of P are in TMEM (pPFull: all 128)
  pNum = 18
};

template <int D, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1) fwd_pp_kernel(const __grid_constant__ FwdParams p) {
  using L = PPSmem<D>;
  constexpr int QH = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align_smem_1024(smem_raw);
  uint8_t* sQ = sm + L::kQ;
  uint8_t* sK = sm + L::kK;
  uint8_t* sV = sm + L::kV;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + pNum);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;
  int tix = (int)blockIdx.x, half = -1;
  if (p.split_halves && tix >= p.split_from) {
    half = (tix - p.split_from) & 1;
    tix = p.split_from + ((tix - p.split_from) >> 1);
  }
  TileTask t = p.tasks[tix];
  if (half >= 0) {
    // one half of a split task: its share of the segments, written to output slot 0 or 1
    const int cut = min(max(t.split1, 0), t.nseg);
    if (half == 0) {
      t.nseg = cut;
    } else {
      t.seg0 += cut;
      t.nseg -= cut;
    }
    t.aux = half;
  }
  const int head = t.head;
  const int kvh = head / p.heads_per_kv;
  const bool has_b = t.rows > BM;
  const int32_t qp0 = t.pos0, qp1 = t.pos0 + t.rows - 1;  // union of the two tiles

  if (threadIdx.x == 0) {
    mbar_init(&bar[pQFull], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[pKFull + s], 1);
      mbar_init(&bar[pVFull + s], 1);
      mbar_init(&bar[pKEmpty + s], 1);
      mbar_init(&bar[pVEmpty + s], 1);
      mbar_init(&bar[pSFull + s], 1);
      mbar_init(&bar[pPFull + s], 4);
      mbar_init(&bar[pPHalf + s], 4);
      mbar_init(&bar[pPVDone + s], 1);
    }
    mbar_init(&bar[pODone], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && !p.withhold_loads) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(&bar[pQFull], (has_b ? 2 : 1) * L::kTile);
      for (int x = 0; x < (has_b ? 2 : 1); ++x) {
        int32_t qr = t.row0 + x * BM;
        CBV_CHECK_RANGE(qr, 0, p.q_rows, p.status, kDevBoundsQ);
        for (int h = 0; h < QH; ++h) tma_load_3d(sQ + x * L::kTile + h * 16384, &p.tm_q, &bar[pQFull], h * 64, head, qr);
      }
      KIter it;
      KTile r;
      int i = 0;
      while (next_ktile<PAGED>(p, t, qp0, qp1, it, r)) {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        bool ok = true;
        for (int kv = 0; kv < 2 && ok; ++kv) {
          uint64_t* empty = &bar[(kv == 0 ? pKEmpty : pVEmpty) + st];
          uint64_t* full = &bar[(kv == 0 ? pKFull : pVFull) + st];
          const CUtensorMap* map = kv == 0 ? &p.tm_k : &p.tm_v;
          uint8_t* dst = (kv == 0 ? sK : sV) + st * L::kTile;
          if (!mbar_wait(empty, ph ^ 1, p.status, kDevTimeoutTmaEmpty, lim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full, L::kTile);
          if (!PAGED) {
            int32_t kr = r.k_row;
            CBV_CHECK_RANGE(kr, 0, p.kv_rows, p.status, kDevBoundsKV);
            for (int h = 0; h < QH; ++h) tma_load_3d(dst + h * 16384, map, full, h * 64, kvh, kr);
          } else {
            // one box per page of block_size tokens, found through the shard's block table
            const int bs = p.block_size, lbs = __ffs(bs) - 1;
            int32_t shard = r.shard;
            CBV_CHECK_RANGE(shard, 0, p.shards, p.status, kDevBoundsPage);
            for (int pg = 0; pg < (BN >> lbs); ++pg) {
              const int blk = min((r.k_row >> lbs) + pg, p.blocks_per_shard - 1);  // k_row: a multiple of 128
              int32_t page = __ldg(&p.block_tables[(int64_t)shard * p.blocks_per_shard + blk]);
              CBV_CHECK_RANGE(page, 0, p.kv_rows, p.status, kDevBoundsPage);
              for (int h = 0; h < QH; ++h) tma_load_4d(dst + h * 16384 + pg * bs * 128, map, full, h * 64, 0, kvh, page);
            }
          }
        }
        if (!ok) break;
        ++i;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer (whole warp, one lane issues)
    {
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(BM, D, false, true);
      const uint64_t dQ0 = sdesc_sw128(smem_u32(sQ), 16, 1024);      // tile x at + x * kTile
      const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);      // stage s at + s * kTile
      const uint64_t dV0 = sdesc_sw128(smem_u32(sV), 16384, 1024);
      int n = 0;
      {
        KIter c;
        KTile r;
        while (next_ktile<PAGED>(p, t, qp0, qp1, c, r)) ++n;
      }
      const int ntile = has_b ? 2 : 1;
      bool ok = mbar_wait_warp(&bar[pQFull], 0, p.status, kDevTimeoutMma, lim);
      tc_fence_after();
      // S_x of k tile i (K stage i & 1); a split task's two halves both read q tile 0
      auto issue_s = [&](int x, int i) {
        const uint64_t dq = sdesc_add(dQ0, (has_b ? x : 0) * L::kTile), dk = sdesc_add(dK0, (i & 1) * L::kTile);
        const uint32_t ts = tmem + x * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_bf16_ss(ts, sdesc_add(dq, off), sdesc_add(dk, off), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar[pSFull + x]);
      };
      // PV_x of k tile i (V stage i & 1); `first` starts O_x afresh.  The first 64 keys' half runs
      // as soon as the softmax has stored that half of P (parity ph of pPHalf), the rest once all
      // of P is in (the caller has waited for pPFull); returns false if the half's wait gave up.
      auto issue_pv_half = [&](int x, int i, bool first, int half_i) {
        const uint64_t dv = sdesc_add(dV0, (i & 1) * L::kTile);
        const uint32_t tp = tmem + x * 128, to = tmem + 256 + x * D;
#pragma unroll
        for (int k4 = 0; k4 < BN / 32; ++k4) {
          const int kk = half_i * (BN / 32) + k4;
          umma_bf16_ts(to, tp + kk * 8, sdesc_add(dv, kk * 2048), idesc_o, (!first || kk > 0) ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int x, int i, bool first) {
        issue_pv_half(x, i, first, 1);
        umma_commit(&bar[pPVDone + x]);
      };
      if (!has_b) {
        // split task: k tile i belongs to half x = i & 1 and always sits in stage i & 1
        for (int i = 0; ok && i < min(n, 2); ++i) {
          ok = mbar_wait_warp(&bar[pKFull + i], 0, p.status, kDevTimeoutMma, lim);
          tc_fence_after();
          if (ok) {
            issue_s(i, i);
            umma_commit(&bar[pKEmpty + i]);
          }
        }
        for (int i = 0; ok && i < n; ++i) {
          const int x = i & 1;
          const uint32_t ph = (i >> 1) & 1;  // half x's own tile count, and stage x's load count
          if (!mbar_wait_warp(&bar[pVFull + x], ph, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
          if (!mbar_wait_warp(&bar[pPHalf + x], ph, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
          tc_fence_after();
          issue_pv_half(x, i, i < 2, 0);
          if (!mbar_wait_warp(&bar[pPFull + x], ph, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
          tc_fence_after();
          issue_pv(x, i, i < 2);
          umma_commit(&bar[pVEmpty + x]);
          if (i + 2 < n) {
            if (!mbar_wait_warp(&bar[pKFull + x], ph ^ 1, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
            // P_x lives in the columns S_x of tile i + 2 will overwrite
            if (!mbar_wait_warp(&bar[pPVDone + x], ph, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
            tc_fence_after();
            issue_s(x, i + 2);
            umma_commit(&bar[pKEmpty + x]);
          }
        }
      } else if (ok && n > 0) {
        ok = mbar_wait_warp(&bar[pKFull], 0, p.status, kDevTimeoutMma, lim);
        tc_fence_after();
        if (ok) {
          for (int x = 0; x < ntile; ++x) issue_s(x, 0);
          umma_commit(&bar[pKEmpty]);
        }
      }
      for (int i = 0; ok && has_b && i < n; ++i) {
        const int st = i & 1;
        if (!mbar_wait_warp(&bar[pVFull + st], (i >> 1) & 1, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
        for (int x = 0; x < ntile && ok; ++x) {
          if (!mbar_wait_warp(&bar[pPHalf + x], i & 1, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
          tc_fence_after();
          issue_pv_half(x, i, i == 0, 0);
          if (!mbar_wait_warp(&bar[pPFull + x], i & 1, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
          tc_fence_after();
          issue_pv(x, i, i == 0);
          if (i + 1 < n) {
            const int st1 = (i + 1) & 1;
            if (!mbar_wait_warp(&bar[pKFull + st1], ((i + 1) >> 1) & 1, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
            // P_x(i) lives in the columns S_x(i+1) will overwrite: let PV_x(i) finish reading it first
            if (!mbar_wait_warp(&bar[pPVDone + x], i & 1, p.status, kDevTimeoutMma, lim)) { ok = false; break; }
            tc_fence_after();
            issue_s(x, i + 1);
            if (x == ntile - 1) umma_commit(&bar[pKEmpty + st1]);
          }
        }
        if (ok) umma_commit(&bar[pVEmpty + st]);
      }
      if (n > 0) umma_commit(&bar[pODone]);
      else if (lane == 0) mbar_arrive(&bar[pODone]);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue (warps 2..9)
    const int x = (warp - 2) >> 2;  // tile: 0 = A, 1 = B (a split task: the two halves of one tile)
    const bool split = !has_b;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + x * 128 + lane_base;
    const uint32_t tO = tmem + 256 + x * D + lane_base;
    const int trow = (split ? 0 : x * BM) + row;  // row within the pair
    const int32_t qpos = t.pos0 + trow;
    const int32_t xq0 = t.pos0 + (split ? 0 : x * BM), xq1 = min(t.pos0 + t.rows - 1, xq0 + BM - 1);
    const float sl2 = p.scale_log2;
    const int32_t W = p.window;
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    int i = 0;  // k tiles this tile (half) has processed
    {
      KIter it;
      KTile r;
      int kidx = 0;
      while (next_ktile<PAGED>(p, t, qp0, qp1, it, r)) {
        if (split && ((kidx++ & 1) != x)) continue;  // the other half's k tile
        if (!mbar_wait_warp(&bar[pSFull + x], i & 1, p.status, kDevTimeoutSoftmax, lim)) { ok = false; break; }
        tc_fence_after();
        uint32_t s[BN];
#pragma unroll
        for (int c = 0; c < BN; c += 32) tmem_ld32(tS + c, s + c);
        tmem_ld_wait();
        const bool cz = r.causal || W > 0;
        const bool need_mask = !((r.nvalid == BN) && (!cz || r.kmax <= xq0) && (W <= 0 || xq1 - r.kpos0 < W));
        if (need_mask && (!PAGED || p.kv_mode == kKvContiguous)) {
          // positions are linear in the column: this row sees the columns [lo, hi]
          int32_t hi = r.nvalid - 1, lo = 0;
          if (cz) hi = min(hi, qpos - r.kpos0);
          if (W > 0) lo = max(lo, qpos - W + 1 - r.kpos0);
          mask_outside(s, lo, hi);
        } else if (need_mask) {
          // round-robin pages: column c sits at kpos0 + delta(c), delta(c) = (c / bs) * shards * bs
          // + c % bs, which grows with c, so the columns a row sees are again one range [lo, hi]:
          // invert delta at the row's two bounds (two divisions per row instead of a position per
          // score)
          const int lbs = __ffs(p.block_size) - 1;
          const int32_t bs = p.block_size, page_stride = p.total_shards << lbs;
          int32_t hi = r.nvalid - 1, lo = 0;
          if (cz) {
            const int32_t x = qpos - r.kpos0;  // largest visible delta
            if (x < 0) {
              hi = -1;
            } else {
              const int32_t pg = x / page_stride, off = x - pg * page_stride;
              hi = min(hi, off >= bs ? ((pg + 1) << lbs) - 1 : (pg << lbs) + off);
            }
          }
          if (W > 0) {
            const int32_t x = qpos - W + 1 - r.kpos0;  // smallest visible delta
            if (x > 0) {
              const int32_t pg = x / page_stride, off = x - pg * page_stride;
              lo = max(lo, off >= bs ? (pg + 1) << lbs : (pg << lbs) + off);
            }
          }
          mask_outside(s, lo, hi);
        }
        // row maximum of the raw scores (the scale is positive, so it commutes)
        // eight independent chains (the max is exact in any order), so the reduction sits on the
        // softmax's critical path for about 11 dependent steps instead of 64
        float mq[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) mq[j] = max3f(-INFINITY, __uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1]));
#pragma unroll
        for (int c = 16; c < BN; c += 16)
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mq[j] = max3f(mq[j], __uint_as_float(s[c + 2 * j]), __uint_as_float(s[c + 2 * j + 1]));
        const float mraw = max3f(max3f(mq[0], mq[1], mq[2]), max3f(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7]));
        const float mx = mraw * sl2;  // log2 units
        float m_use = m, alpha = 1.f;
        bool rescale_o = false;
        if (mx > m + kRescaleThreshold) {
          m_use = mx;
          alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - mx);
          rescale_o = (m != -INFINITY);
        }
        const float msub = (m_use == -INFINITY) ? 0.f : m_use;
        float rowsum = 0.f, rowsum_r = 0.f;
        uint32_t pk[BN / 2];
        // P in two halves of 64 keys: the first goes to TMEM (and its PV starts) while the second
        // is being formed
#pragma unroll
        for (int c = 0; c < BN / 2; c += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[c]), sl2, -msub));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[c + 1]), sl2, -msub));
          const uint32_t pb = pack_bf16x2(p0, p1);
          rowsum += p0 + p1;
          rowsum_r = add_bf16x2_f32(rowsum_r, pb);
          pk[c / 2] = pb;
        }
        // PV of the previous k tile must be done: O is rescaled and P overwrites its input
        if (i > 0 && !mbar_wait_warp(&bar[pPVDone + x], (i - 1) & 1, p.status, kDevTimeoutSoftmax, lim)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale_o)) {
          // 16 columns at a time: half of the scores are still held in registers here
#pragma unroll 1
          for (int c = 0; c < D; c += 16) {
            uint32_t o[16];
            tmem_ld16(tO + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(tO + c, o);
          }
        }
        tmem_st32(tS, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[pPHalf + x]);
#pragma unroll
        for (int c = BN / 2; c < BN; c += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[c]), sl2, -msub));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[c + 1]), sl2, -msub));
          const uint32_t pb = pack_bf16x2(p0, p1);
          rowsum += p0 + p1;
          rowsum_r = add_bf16x2_f32(rowsum_r, pb);
          pk[c / 2] = pb;
        }
        l = l * alpha + rowsum;
        lr = lr * alpha + rowsum_r;
        m = m_use;
        tmem_st32(tS + 32, pk + 32);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[pPFull + x]);
        ++i;
      }
    }
    // ---------------------------------------------------------------- epilogue
    // where this CTA writes: the call's output, or for one half of a split task its fp32 slot
    const bool hx = half >= 0;
    const int o_mode = hx ? (int)kOutF32 : p.out_mode;
    void* const o_base = hx ? static_cast<void*>(p.half_out) : p.out;
    const int64_t o_t = hx ? (int64_t)D : p.out_stride_t, o_h = hx ? p.half_q_len * D : p.out_stride_h;
    const int64_t o_d = hx ? 1 : p.out_stride_d, o_sh = hx ? p.half_rows * D : p.out_shard_stride;
    float* const l_base = hx ? p.half_lse : p.lse;
    const int64_t l_h = hx ? p.half_q_len : p.lse_stride_h, l_t = hx ? 1 : p.lse_stride_t;
    const int64_t l_sh = hx ? p.half_rows : p.lse_shard_stride;
    // split task: half B hands its softmax state to half A, which merges the two
    // (every softmax warp reaches the barrier once, whatever happened before)
    float wa_o = 1.f, wb_o = 0.f;  // weights of O_A and O_B in the merged accumulator
    if (split) {
      float4* stats = reinterpret_cast<float4*>(sm + L::kStats);
      if (x == 1) stats[row] = make_float4(m, l, lr, 0.f);
      named_bar_sync(1, 256);
      if (x == 0) {
        const float4 b = stats[row];
        const float mm = fmaxf(m, b.x);
        wa_o = (m == -INFINITY) ? 0.f : ex2_approx(m - mm);
        wb_o = (b.x == -INFINITY) ? 0.f : ex2_approx(b.x - mm);
        l = l * wa_o + b.y * wb_o;
        lr = lr * wa_o + b.z * wb_o;
        m = mm;
      }
    }
    if (ok && (x == 0 || has_b) && mbar_wait_warp(&bar[pODone], 0, p.status, kDevTimeoutEpilogue, lim)) {
      tc_fence_after();
      const bool has = (l > 0.f) && (m != -INFINITY);
      const float inv_l = (has && lr > 0.f) ? 1.f / lr : 0.f;
      const float lse_b = has ? (m + __log2f(l)) * kLn2 : -INFINITY;
      bool valid = trow < t.rows;
      const int64_t orow = (int64_t)(t.row0 + trow);
#ifdef CBV_DEBUG
      if (valid && (orow < 0 || orow >= p.q_rows)) {
        atomicCAS(p.status, 0, kDevBoundsOut);
        valid = false;
      }
#endif
      const int64_t shard_off = t.aux >= 0 ? (int64_t)t.aux : 0;  // per-shard outputs
      float* lse_ptr = l_base + shard_off * l_sh + (int64_t)head * l_h + orow * l_t;
      float wa = 0.f, wb = 1.f, lse_new = lse_b;
      if (o_mode == kOutMerge && valid) {
        const float lse_a = *lse_ptr;
        const float mm = fmaxf(lse_a, lse_b);
        if (mm == -INFINITY) {
          wa = 1.f;
          wb = 0.f;
          lse_new = -INFINITY;
        } else {
          lse_new = mm + __logf(__expf(lse_a - mm) + __expf(lse_b - mm));
          wa = __expf(lse_a - lse_new);
          wb = __expf(lse_b - lse_new);
        }
      }
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + c, o);
        tmem_ld_wait();
        if (split) {
          uint32_t ob[32];
          tmem_ld32(tO + D + c, ob);  // O_B, the same rows
          tmem_ld_wait();
          // a half without k tiles (weight 0) never wrote its accumulator: select, do not multiply
#pragma unroll
          for (int e = 0; e < 32; ++e)
            o[e] = __float_as_uint((wa_o != 0.f ? __uint_as_float(o[e]) * wa_o : 0.f) +
                                   (wb_o != 0.f ? __uint_as_float(ob[e]) * wb_o : 0.f));
        }
        if (!valid) continue;
        if (!has) {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (o_mode == kOutBf16 && o_d > 1) {
          // transposed output: lanes hold consecutive rows, so each store covers 32 adjacent rows
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(o_base) + shard_off * o_sh +
                               orow * o_t + (int64_t)head * o_h + (int64_t)c * o_d;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            dst[(int64_t)e * o_d] = __float2bfloat16_rn(__uint_as_float(o[e]) * inv_l);
        } else if (o_mode == kOutBf16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(o_base) + shard_off * o_sh + orow * o_t +
                               (int64_t)head * o_h + c;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
            *reinterpret_cast<uint4*>(dst + e) = v;
          }
        } else {
          float* dst = reinterpret_cast<float*>(o_base) + shard_off * o_sh + orow * o_t +
                     (int64_t)head * o_h + c;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 v;
            v.x = __uint_as_float(o[e + 0]) * inv_l;
            v.y = __uint_as_float(o[e + 1]) * inv_l;
            v.z = __uint_as_float(o[e + 2]) * inv_l;
            v.w = __uint_as_float(o[e + 3]) * inv_l;
            if (o_mode == kOutMerge) {
              const float4 a = *reinterpret_cast<const float4*>(dst + e);
              v.x = a.x * wa + v.x * wb;
              v.y = a.y * wa + v.y * wb;
              v.z = a.z * wa + v.z * wb;
              v.w = a.w * wa + v.w * wb;
            }
            *reinterpret_cast<float4*>(dst + e) = v;
          }
        }
      }
      if (valid) *lse_ptr = lse_new;
    }

  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, bool PAGED>
int launch_pp_t(const FwdParams& p, int grid, cudaStream_t stream) {
  auto kern = fwd_pp_kernel<D, PAGED>;
  const uint32_t smem = PPSmem<D>::kDynamic;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  if (const int ev = kernel_event_start(stream)) return ev;
  kern<<<grid, kThreads, smem, stream>>>(p);
  const int rc = launched();
  if (rc) return rc;
  return kernel_event_stop(stream);
}

}  // namespace

int launch_fwd_pingpong(const FwdParams& p, int head_dim, bool paged, int grid, cudaStream_t stream) {
  if (grid <= 0) return 0;
  if (head_dim == 128) return paged ? launch_pp_t<128, true>(p, grid, stream) : launch_pp_t<128, false>(p, grid, stream);
  if (head_dim == 64) return paged ? launch_pp_t<64, true>(p, grid, stream) : launch_pp_t<64, false>(p, grid, stream);
  return (int)cudaErrorInvalidValue;
}

}  // namespace cbv
